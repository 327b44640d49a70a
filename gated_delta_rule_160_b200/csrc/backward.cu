// backward.cu -- gradients of the recurrence (gdn2_chunk_bwd): a first, sequential form.
//
// For each token, with e = b (.) k, x = w (.) v, S' = Diag(alpha) S_prev, r = S'^T k,
// S = S' - e r^T + k x^T, o = S^T q, and the adjoint dS of S (from later tokens and dS_T):
//   dS  += q dO^T                                   (o's contribution)
//   dx   = dS^T k,  dr = -dS^T e                    (column sums over key channels)
//   de   = -dS r,   dk = dS x + Diag(alpha) S_prev dr + de (.) b,   db = de (.) k
//   dS'  = dS + k dr^T
//   dalpha = rowsum(dS' (.) S_prev),  dlog_alpha = dalpha (.) alpha
//   dq   = Diag(alpha) S_prev dO - e (r . dO) + k (x . dO)     (= S dO)
//   dw   = dx (.) v,  dv = dx (.) w,  and the adjoint of S_prev is Diag(alpha) dS'.
// One CTA per (sequence, value head). It runs the recurrence forward once, storing the
// state at the start of every 64-token chunk; then, chunk by chunk from the last, it
// recomputes the chunk's states from that checkpoint into a per-CTA scratch area and walks
// the chunk's tokens backwards. S_prev and dS live in shared memory with rows padded to
// DV + 1 floats, so that row sums (thread = row) and column sums (thread = column) are both
// free of bank conflicts. A query/key head's dq, dk sum over the value heads that read it:
// with groups of several value heads they are accumulated with atomics into outputs the
// host zeroed first.
#include "internal.cuh"

namespace gdn2 {
namespace {

constexpr int kBT = 256;     // threads per CTA
constexpr int kCk = 64;      // tokens per checkpoint interval

struct BwdParams {
    Params f;                // the forward's arguments
    const float* dO;         // [T, h_v, dv]
    const float* dS_T;       // nullable [N, h_v, dk, dv]
    float *dq, *dk, *dv, *dla, *db, *dw, *dS0;  // dS0 nullable
    float* ckpt;             // [sum of chunks, h_v, dk, dv]
    float* scratch;          // [N * h_v, kCk, dk, dv]
    int atomic_qk;           // dq, dk accumulate (groups of value heads)
};

template <int DK, int DV>
struct Smem {
    float S[DK][DV + 1];     // S_prev (or the running state in the forward passes)
    float dS[DK][DV + 1];    // adjoint of the state after the current token
    float k[DK], q[DK], al[DK], e[DK], b[DK];
    float x[DV], v[DV], w[DV], dO[DV], r[DV], dx[DV], dr[DV];
    float cpart[kBT / DV][3][DV];  // column-sum partials (r, dx, dr)
    float rpart[kBT / DK][5][DK];  // row-sum partials (de, dk, dalpha, S_prev dO, unused)
    float dots[2];                 // r . dO, x . dO
};

template <typename T>
__device__ __forceinline__ float ld(const void* base, size_t i) {
    return to_f32(static_cast<const T*>(base)[i]);
}

template <int DK, int DV, typename T>
__device__ void load_token(const Params& p, Smem<DK, DV>& sm, size_t tok, int g, int h, const float* dO) {
    const size_t tq = tok * p.h_qk + g, tv = tok * p.h_v + h;
    for (int c = threadIdx.x; c < DK; c += kBT) {
        const float kv = ld<T>(p.k, tq * DK + c), bv = ld<T>(p.b, tv * DK + c);
        sm.k[c] = kv;
        sm.q[c] = ld<T>(p.q, tq * DK + c);
        sm.al[c] = expf(p.log_alpha[tv * DK + c]);
        sm.b[c] = bv;
        sm.e[c] = bv * kv;
    }
    for (int m = threadIdx.x; m < DV; m += kBT) {
        const float vv = ld<T>(p.v, tv * DV + m), wv = ld<T>(p.w, tv * DV + m);
        sm.v[m] = vv;
        sm.w[m] = wv;
        sm.x[m] = wv * vv;
        if (dO) sm.dO[m] = dO[tv * DV + m];
    }
}

// One forward token on sm.S (state in, state out); token vectors already loaded.
template <int DK, int DV>
__device__ void forward_token(Smem<DK, DV>& sm) {
    constexpr int CP = kBT / DV;  // column parts
    const int m = threadIdx.x % DV, part = threadIdx.x / DV;
    float acc = 0.f;
    for (int c = part; c < DK; c += CP) acc = fmaf(sm.al[c] * sm.k[c], sm.S[c][m], acc);
    sm.cpart[part][0][m] = acc;
    __syncthreads();
    if (threadIdx.x < DV) {
        float r = 0.f;
#pragma unroll
        for (int j = 0; j < CP; ++j) r += sm.cpart[j][0][threadIdx.x];
        sm.r[threadIdx.x] = r;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < DK * DV; idx += kBT) {
        const int c = idx / DV, mm = idx % DV;
        sm.S[c][mm] = fmaf(sm.k[c], sm.x[mm], fmaf(-sm.e[c], sm.r[mm], sm.al[c] * sm.S[c][mm]));
    }
    __syncthreads();
}

// State copies between global memory ([DK][DV], contiguous) and the padded shared array:
// 16-byte global accesses, every load of a thread issued before its first store.
template <int DK, int DV>
__device__ void store_state(const Smem<DK, DV>& sm, float* dst) {
    constexpr int N4 = DK * DV / 4 / kBT;
#pragma unroll
    for (int j = 0; j < N4; ++j) {
        const int i4 = threadIdx.x + j * kBT, c = (4 * i4) / DV, m = (4 * i4) % DV;
        reinterpret_cast<float4*>(dst)[i4] = make_float4(sm.S[c][m], sm.S[c][m + 1], sm.S[c][m + 2], sm.S[c][m + 3]);
    }
}
template <int DK, int DV>
__device__ void load_state(Smem<DK, DV>& sm, const float* src) {
    constexpr int N4 = DK * DV / 4 / kBT;
    float4 r[N4];
#pragma unroll
    for (int j = 0; j < N4; ++j)
        r[j] = src ? reinterpret_cast<const float4*>(src)[threadIdx.x + j * kBT] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < N4; ++j) {
        const int i4 = threadIdx.x + j * kBT, c = (4 * i4) / DV, m = (4 * i4) % DV;
        sm.S[c][m] = r[j].x;
        sm.S[c][m + 1] = r[j].y;
        sm.S[c][m + 2] = r[j].z;
        sm.S[c][m + 3] = r[j].w;
    }
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(kBT, 1) chunk_bwd_kernel(const __grid_constant__ BwdParams bp) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    Smem<DK, DV>& sm = *reinterpret_cast<Smem<DK, DV>*>(smem_raw);
    const Params& p = bp.f;
    const int item = blockIdx.x;
    const int n = item / p.h_v, h = item % p.h_v, g = h / (p.h_v / p.h_qk);
    int t0, t1;
    seq_bounds(p, n, t0, t1);
    const int nck = (t1 - t0 + kCk - 1) / kCk;
    // this sequence's first checkpoint: the chunks of the sequences before it
    int base = 0;
    if (p.cu_seqlens) {
        for (int j = 0; j < n; ++j) {
            int a0, a1;
            seq_bounds(p, j, a0, a1);
            base += (a1 - a0 + kCk - 1) / kCk;
        }
    } else {
        base = n * ((p.T_fixed + kCk - 1) / kCk);
    }
    const size_t SZ = (size_t)DK * DV;
    float* ck = bp.ckpt + (size_t)base * p.h_v * SZ;
    auto ckpt_of = [&](int c) { return ck + ((size_t)c * p.h_v + h) * SZ; };
    float* scr = bp.scratch + (size_t)item * kCk * SZ;
    const size_t soff = ((size_t)n * p.h_v + h) * SZ;

    // ---- forward: checkpoints at the start of every chunk
    load_state(sm, p.S0 ? p.S0 + soff : nullptr);
    __syncthreads();
    for (int c = 0; c < nck; ++c) {
        store_state(sm, ckpt_of(c));
        const int te = min(t0 + (c + 1) * kCk, t1);
        for (int t = t0 + c * kCk; t < te; ++t) {
            load_token<DK, DV, T>(p, sm, (size_t)t, g, h, nullptr);
            __syncthreads();
            forward_token(sm);
        }
    }

    // ---- backward
    for (int idx = threadIdx.x; idx < DK * DV; idx += kBT)
        sm.dS[idx / DV][idx % DV] = bp.dS_T ? bp.dS_T[soff + idx] : 0.f;
    for (int c = nck - 1; c >= 0; --c) {
        const int ts = t0 + c * kCk, te = min(ts + kCk, t1);
        // the chunk's states: scr[i] = the state after token ts + i (i < te - ts - 1)
        __syncthreads();
        load_state(sm, ckpt_of(c));
        __syncthreads();
        for (int t = ts; t + 1 < te; ++t) {
            load_token<DK, DV, T>(p, sm, (size_t)t, g, h, nullptr);
            __syncthreads();
            forward_token(sm);
            store_state(sm, scr + (size_t)(t - ts) * SZ);
        }
        for (int t = te - 1; t >= ts; --t) {
            __syncthreads();
            load_state(sm, t == ts ? ckpt_of(c) : scr + (size_t)(t - ts - 1) * SZ);  // S_prev
            load_token<DK, DV, T>(p, sm, (size_t)t, g, h, bp.dO);
            __syncthreads();
            // pass A: dS += q dO^T; column sums r = S'^T k, dx = dS^T k, dr = -dS^T e
            {
                constexpr int CP = kBT / DV;
                const int m = threadIdx.x % DV, part = threadIdx.x / DV;
                const float dom = sm.dO[m];
                float ar = 0.f, adx = 0.f, adr = 0.f;
                for (int cc = part; cc < DK; cc += CP) {
                    const float d = fmaf(sm.q[cc], dom, sm.dS[cc][m]);
                    sm.dS[cc][m] = d;
                    ar = fmaf(sm.al[cc] * sm.k[cc], sm.S[cc][m], ar);
                    adx = fmaf(sm.k[cc], d, adx);
                    adr = fmaf(-sm.e[cc], d, adr);
                }
                sm.cpart[part][0][m] = ar;
                sm.cpart[part][1][m] = adx;
                sm.cpart[part][2][m] = adr;
                __syncthreads();
                if (threadIdx.x < DV) {
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f;
#pragma unroll
                    for (int j = 0; j < CP; ++j) {
                        a0 += sm.cpart[j][0][threadIdx.x];
                        a1 += sm.cpart[j][1][threadIdx.x];
                        a2 += sm.cpart[j][2][threadIdx.x];
                    }
                    sm.r[threadIdx.x] = a0;
                    sm.dx[threadIdx.x] = a1;
                    sm.dr[threadIdx.x] = a2;
                }
                __syncthreads();
            }
            // r . dO and x . dO (warps 0 and 1)
            if (threadIdx.x < 64) {
                const int wi = threadIdx.x / 32, l = threadIdx.x % 32;
                float s = 0.f;
                for (int m = l; m < DV; m += 32) s = fmaf(wi == 0 ? sm.r[m] : sm.x[m], sm.dO[m], s);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                if (l == 0) sm.dots[wi] = s;
            }
            // pass B: row sums; dS <- Diag(alpha) (dS + k dr^T)
            {
                constexpr int RP = kBT / DK;
                const int cc = threadIdx.x % DK, part = threadIdx.x / DK;
                const float kc = sm.k[cc], alc = sm.al[cc];
                float ade = 0.f, adk = 0.f, ada = 0.f, asd = 0.f;
                for (int m = part; m < DV; m += RP) {
                    const float d = sm.dS[cc][m], sp = sm.S[cc][m], drm = sm.dr[m];
                    const float dsp = fmaf(kc, drm, d);
                    ade = fmaf(-d, sm.r[m], ade);
                    adk = fmaf(d, sm.x[m], fmaf(alc * sp, drm, adk));
                    ada = fmaf(dsp, sp, ada);
                    asd = fmaf(sp, sm.dO[m], asd);
                    sm.dS[cc][m] = alc * dsp;
                }
                sm.rpart[part][0][cc] = ade;
                sm.rpart[part][1][cc] = adk;
                sm.rpart[part][2][cc] = ada;
                sm.rpart[part][3][cc] = asd;
                __syncthreads();
                if (threadIdx.x < DK) {
                    float de = 0.f, dk = 0.f, da = 0.f, sd = 0.f;
#pragma unroll
                    for (int j = 0; j < RP; ++j) {
                        de += sm.rpart[j][0][cc];
                        dk += sm.rpart[j][1][cc];
                        da += sm.rpart[j][2][cc];
                        sd += sm.rpart[j][3][cc];
                    }
                    const size_t tq = (size_t)t * p.h_qk + g, tv = (size_t)t * p.h_v + h;
                    dk += de * sm.b[cc];
                    const float dq = alc * sd - sm.e[cc] * sm.dots[0] + kc * sm.dots[1];
                    if (bp.atomic_qk) {
                        atomicAdd(bp.dq + tq * DK + cc, dq);
                        atomicAdd(bp.dk + tq * DK + cc, dk);
                    } else {
                        bp.dq[tq * DK + cc] = dq;
                        bp.dk[tq * DK + cc] = dk;
                    }
                    bp.db[tv * DK + cc] = de * kc;
                    bp.dla[tv * DK + cc] = da * alc;
                }
                if (threadIdx.x < DV) {
                    const int m = threadIdx.x;
                    const size_t tv = (size_t)t * p.h_v + h;
                    bp.dw[tv * DV + m] = sm.dx[m] * sm.v[m];
                    bp.dv[tv * DV + m] = sm.dx[m] * sm.w[m];
                }
            }
        }
    }
    __syncthreads();
    if (bp.dS0)
        for (int idx = threadIdx.x; idx < DK * DV; idx += kBT) bp.dS0[soff + idx] = sm.dS[idx / DV][idx % DV];
}

template <int DK, int DV, typename T>
cudaError_t launch_bwd_t(const BwdParams& bp, cudaStream_t s) {
    const size_t smem = sizeof(Smem<DK, DV>);
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<DK, DV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    chunk_bwd_kernel<DK, DV, T><<<bp.f.n_seq * bp.f.h_v, kBT, smem, s>>>(bp);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_d(const BwdParams& bp, cudaStream_t s) {
    if (bp.f.dk == 128) return bp.f.dv == 128 ? launch_bwd_t<128, 128, T>(bp, s) : launch_bwd_t<128, 64, T>(bp, s);
    return bp.f.dv == 128 ? launch_bwd_t<64, 128, T>(bp, s) : launch_bwd_t<64, 64, T>(bp, s);
}

}  // namespace

size_t bwd_workspace_bytes(const gdn2_shape* sh) {
    const size_t SZ = (size_t)sh->dk * sh->dv * sizeof(float);
    const size_t chunks = (size_t)(sh->T_total + kCk - 1) / kCk + (size_t)sh->n_seq;  // >= sum of per-sequence chunks
    return chunks * sh->h_v * SZ + (size_t)sh->n_seq * sh->h_v * kCk * SZ;
}

cudaError_t launch_bwd(const Params& p, gdn2_dtype dt, const float* dO, const float* dS_T, float* dq, float* dk,
                       float* dv, float* dla, float* db, float* dw, float* dS0, void* workspace, cudaStream_t s) {
    BwdParams bp{};
    bp.f = p;
    bp.dO = dO; bp.dS_T = dS_T;
    bp.dq = dq; bp.dk = dk; bp.dv = dv; bp.dla = dla; bp.db = db; bp.dw = dw; bp.dS0 = dS0;
    const size_t SZ = (size_t)p.dk * p.dv;
    const size_t chunks = (size_t)(p.T_total + kCk - 1) / kCk + (size_t)p.n_seq;
    bp.ckpt = static_cast<float*>(workspace);
    bp.scratch = bp.ckpt + chunks * p.h_v * SZ;
    bp.atomic_qk = p.h_v != p.h_qk;
    if (bp.atomic_qk) {
        const size_t qk_bytes = (size_t)p.T_total * p.h_qk * p.dk * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dq, 0, qk_bytes, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, qk_bytes, s);
        if (e != cudaSuccess) return e;
    }
    return dt == GDN2_F32 ? launch_bwd_d<float>(bp, s) : launch_bwd_d<__nv_bfloat16>(bp, s);
}

}  // namespace gdn2
