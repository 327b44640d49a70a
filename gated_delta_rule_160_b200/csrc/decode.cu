// decode.cu -- decode steps: n_tok (usually 1) new tokens per sequence, state updated in
// place (in a slot of a state pool for serving), optionally every intermediate state.
//
// The step is bound by HBM: the fp32 state [dk, dv] of every (sequence, value head) is
// read once and written once; everything else is a few hundred bytes. One CTA of 256
// threads owns one (sequence, head). Thread (row group rg, column group cg) holds four
// consecutive value columns (a float4) of DK/RG key rows, rows rg, rg+RG, ...; a warp
// therefore covers whole rows and every state load and store is a coalesced 16-byte
// access. All state loads are issued before anything else so the CTA keeps 64 KB in
// flight.
//
// With the token's decay alpha, key k, query q, erase gate b and x = w (.) v:
//   r = (Diag(alpha) S)^T k,  p = (Diag(alpha) S)^T q       (one pass over S)
//   S <- Diag(alpha) S - (b (.) k) r^T + k x^T              (second half of the same pass)
//   o  = p - (q . (b (.) k)) r + (q . k) x                  == S_new^T q
// which reads S once; the two column sums over the key axis are combined across row
// groups through shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace {

// Device status word of this file's kernels (kStatus* bits), read and cleared by
// gdn2_device_status.
__device__ unsigned int g_status_dec = 0;

constexpr int kThreads = 256;

// Activations of the fused pre-processing (kPro): raw q, k L2-normalised per token;
// alpha = exp(-softplus(a)) = 1 / (1 + e^a); sigmoid b, w. The norms need the whole token,
// so q and k are normalised after staging, together with the per-token dot products.

// ---------------------------------------------------------------- one token per sequence
template <int DK, int DV, typename T, typename TO, bool kPro>
__global__ void __launch_bounds__(kThreads) decode_kernel(Params p) {
    constexpr int TPR = DV / 4;          // threads per state row
    constexpr int RG = kThreads / TPR;   // row groups
    constexpr int RPT = DK / RG;         // rows per thread
    __shared__ float sa[DK], sk[DK], sq[DK], se[DK], sx[DV];
    __shared__ float4 red[2][RG][TPR];  // [r | p]
    __shared__ float dots[2];
    __shared__ float rnorm[2];  // 1 / |q|, 1 / |k| (fused pre-processing)

    const int item = blockIdx.x;  // n * h_v + h
    const int n = item / p.h_v;
    const int h = item % p.h_v;
    const int g = h / (p.h_v / p.h_qk);
    const int slot = p.slots ? p.slots[n] : n;
    if (slot < 0 || slot >= p.n_slots) return;  // an inactive sequence: nothing to do
    const int cg = threadIdx.x % TPR;
    const int rg = threadIdx.x / TPR;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    float* S = p.S_T + ((size_t)slot * p.h_v + h) * DK * DV;

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(rg + RG * i) * DV) + cg);

    // the token's decay, key, query, erase and write vectors
    const size_t tq = (size_t)n * p.h_qk + g, tv = (size_t)n * p.h_v + h;
    for (int c = threadIdx.x; c < DK; c += kThreads) {
        const float kv = to_f32(static_cast<const T*>(p.k)[tq * DK + c]);
        const float bv = to_f32(static_cast<const T*>(p.b)[tv * DK + c]);
        sk[c] = kv;
        sq[c] = to_f32(static_cast<const T*>(p.q)[tq * DK + c]);
        if (kPro) {
            sa[c] = sigmoid_f(-to_f32(static_cast<const T*>(p.a_raw)[tv * DK + c]));
            se[c] = sigmoid_f(bv) * kv;
        } else {
            sa[c] = expf(p.log_alpha[tv * DK + c]);
            se[c] = bv * kv;
        }
    }
    for (int c = threadIdx.x; c < DV; c += kThreads) {
        float wv = to_f32(static_cast<const T*>(p.w)[tv * DV + c]);
        if (kPro) wv = sigmoid_f(wv);
        sx[c] = wv * to_f32(static_cast<const T*>(p.v)[tv * DV + c]);
    }
    __syncthreads();
    // q . (b (.) k) and q . k (and |q|, |k| with the fused pre-processing): warp 0
    if (warp == 0) {
        float d1 = 0.f, d2 = 0.f, nq = 0.f, nk = 0.f;
        for (int c = lane; c < DK; c += 32) {
            d1 += sq[c] * se[c];
            d2 += sq[c] * sk[c];
            if (kPro) {
                nq += sq[c] * sq[c];
                nk += sk[c] * sk[c];
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            d1 += __shfl_xor_sync(0xffffffffu, d1, off);
            d2 += __shfl_xor_sync(0xffffffffu, d2, off);
            if (kPro) {
                nq += __shfl_xor_sync(0xffffffffu, nq, off);
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
            }
        }
        if (lane == 0) {
            float s2 = 1.f;
            if (kPro) {
                rnorm[0] = 1.f / fmaxf(sqrtf(nq), kL2NormEps);
                rnorm[1] = 1.f / fmaxf(sqrtf(nk), kL2NormEps);
                s2 = rnorm[0] * rnorm[1];
            }
            dots[0] = d1 * s2;
            dots[1] = d2 * s2;
        }
    }
    if (kPro) {  // normalise the staged q, k (and b (.) k)
        __syncthreads();
        for (int c = threadIdx.x; c < DK; c += kThreads) {
            sq[c] *= rnorm[0];
            sk[c] *= rnorm[1];
            se[c] *= rnorm[1];
        }
        __syncthreads();
    }

    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rw = rg + RG * i;
        const float a = sa[rw], kv = sk[rw], qv = sq[rw];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        r.x = fmaf(kv, s[i].x, r.x); r.y = fmaf(kv, s[i].y, r.y);
        r.z = fmaf(kv, s[i].z, r.z); r.w = fmaf(kv, s[i].w, r.w);
        pq.x = fmaf(qv, s[i].x, pq.x); pq.y = fmaf(qv, s[i].y, pq.y);
        pq.z = fmaf(qv, s[i].z, pq.z); pq.w = fmaf(qv, s[i].w, pq.w);
    }
    red[0][rg][cg] = r;
    red[1][rg][cg] = pq;
    __syncthreads();
    r = make_float4(0.f, 0.f, 0.f, 0.f);
    pq = r;
#pragma unroll
    for (int j = 0; j < RG; ++j) {
        const float4 a = red[0][j][cg], b = red[1][j][cg];
        r.x += a.x; r.y += a.y; r.z += a.z; r.w += a.w;
        pq.x += b.x; pq.y += b.y; pq.z += b.z; pq.w += b.w;
    }
    const float4 x = *reinterpret_cast<const float4*>(&sx[4 * cg]);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int rw = rg + RG * i;
        const float e = -se[rw], kv = sk[rw];
        s[i].x = fmaf(kv, x.x, fmaf(e, r.x, s[i].x));
        s[i].y = fmaf(kv, x.y, fmaf(e, r.y, s[i].y));
        s[i].z = fmaf(kv, x.z, fmaf(e, r.z, s[i].z));
        s[i].w = fmaf(kv, x.w, fmaf(e, r.w, s[i].w));
        __stcs(reinterpret_cast<float4*>(S + (size_t)rw * DV) + cg, s[i]);
    }
    if (rg == 0) {
        const float qe = dots[0], qk = dots[1];
        TO* o = static_cast<TO*>(p.o) + tv * DV + 4 * cg;
        o[0] = from_f32<TO>(pq.x - qe * r.x + qk * x.x);
        o[1] = from_f32<TO>(pq.y - qe * r.y + qk * x.y);
        o[2] = from_f32<TO>(pq.z - qe * r.z + qk * x.z);
        o[3] = from_f32<TO>(pq.w - qe * r.w + qk * x.w);
    }
}

// ---------------------------------------------------------------- several tokens per sequence
// Thread layout: warp w owns value columns 16w .. 16w+15 over all key rows; lane l holds the
// float4 of columns 16w + 4(l % 4) .. +3 for the RPT = dk / 8 key rows rq, rq + 8, rq + 16,
// ... (rq = l / 4). A column sum over the key axis is then a sum within the thread and over
// the eight lanes that share the column quad (three shuffles), so the token loop has no CTA
// barrier. The per-row vectors (alpha, k, q, b (.) k) are staged with row 8(4j + e) + rq at
// float index 4 (8j + rq) + e, so the eight row groups of a warp read eight consecutive
// float4s (no bank conflicts) and a thread's RPT rows come in RPT / 4 float4 loads.
// The next item's state arrives by TMA while the current item is processed: one thread
// issues dv / 32 box loads of [32 columns x dk rows] with the 128-byte swizzle (16-byte
// chunk c of row r at chunk c ^ (r % 8)), so the eight rows a warp reads at once fall in
// distinct banks. (Per-thread 16-byte copies issued 4096 copy instructions per item, and
// their issue stalled behind the previous item's stores.)
// Shared memory, dynamic (n_tok tokens; the base rounded up to 1024 bytes for the swizzle):
// the next item's state [dv / 32][dk][32] fp32, swizzled; the next item's raw token rows
// [n_tok][k, q, b, log_alpha or a, v, w]; then the current item's fp32 vectors alpha, k, q,
// b (.) k [n_tok][DK] and x [n_tok][DV].
template <int DK, int DV, typename T, bool kPro>
struct MultiCfg {
    static constexpr int NT = 2 * DV, RPT = DK / 8, ES = sizeof(T);
    static constexpr int RK = 0, RQ = DK * ES, RB = 2 * DK * ES, RA = 3 * DK * ES;
    static constexpr int RV = RA + (kPro ? DK * ES : DK * 4), RW = RV + DV * ES, RREC = RW + DV * ES;
    static constexpr int CK = DK * ES / 16, CA = (RV - RA) / 16, CV = DV * ES / 16;
    static constexpr int CPT = 3 * CK + CA + 2 * CV;  // 16-byte pieces per token
    static constexpr int SBUF = RPT * NT * 16;
    static size_t smem(int n_tok) { return 1024 + SBUF + (size_t)n_tok * RREC + (size_t)n_tok * (4 * DK + DV) * 4; }
};

template <int DK, int DV, typename T, typename TO, bool kPro>
__global__ void __launch_bounds__(MultiCfg<DK, DV, T, kPro>::NT, 2)
    decode_multi_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap smap) {
    using C = MultiCfg<DK, DV, T, kPro>;
    constexpr int NT = C::NT, RPT = C::RPT;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ float dots[GDN2_DECODE_MAX_TOKENS][2];
    __shared__ float rnorm[GDN2_DECODE_MAX_TOKENS][2];
    __shared__ __align__(8) uint64_t state_bar;  // the state's TMA loads landed
    const int n_tok = p.n_tok;
    uint8_t* dsm_a = dsm + ((1024u - (tc::smem_u32(dsm) & 1023u)) & 1023u);
    const uint32_t sbuf_a = tc::smem_u32(dsm_a);
    const uint32_t bar = tc::smem_u32(&state_bar);
    uint8_t* raw = dsm_a + C::SBUF;
    float* sa = reinterpret_cast<float*>(raw + (size_t)n_tok * C::RREC);
    float* sk = sa + n_tok * DK;
    float* sq = sk + n_tok * DK;
    float* se = sq + n_tok * DK;
    float* sx = se + n_tok * DK;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int rq = lane >> 2;                          // key rows rq, rq + 8, ..., rq + 8 (RPT - 1)
    const int col = 16 * warp + 4 * (lane & 3);        // first of its four value columns
    // this thread's float4 of row 8i + rq in the swizzled state buffer: box col / 32, chunk
    // (col % 32) / 4 xor (row % 8) = ... xor rq
    const uint32_t sofs = (uint32_t)(col >> 5) * (DK * 128) + (uint32_t)rq * 128 + ((((col & 31) >> 2) ^ rq) << 4);
    const int n_items = p.n_seq * p.h_v;
    auto slot_of = [&](int it) { const int nn = it / p.h_v; return p.slots ? p.slots[nn] : nn; };
    // the next active item from it on (its slot in *slot); a negative or out-of-range slot
    // marks an inactive sequence
    auto next_active = [&](int it, int* slot) {
        for (; it < n_items; it += gridDim.x) {
            const int sl = slot_of(it);
            if (sl >= 0 && sl < p.n_slots) {
                *slot = sl;
                break;
            }
        }
        return it;
    };
    auto state_of = [&](int it, int sl) { return p.S_T + ((size_t)sl * p.h_v + it % p.h_v) * DK * DV; };
    // queue item it's state (TMA, one thread; not when `withhold`, the testing hook) and raw
    // token rows (16-byte copies)
    auto issue = [&](int it, int sl, bool withhold) {
        const int nn = it / p.h_v, hh = it % p.h_v, gg = hh / (p.h_v / p.h_qk);
        if (tid == 0 && !withhold) {
            const int row0 = (sl * p.h_v + hh) * DK;
            tc::mbar_expect_tx(bar, DK * DV * 4);
#pragma unroll
            for (int b = 0; b < DV / 32; ++b) tc::tma_load_2d(sbuf_a + b * DK * 128, &smap, 32 * b, row0, bar);
        }
        for (int u = tid; u < n_tok * C::CPT; u += NT) {
            const int t = u / C::CPT, r = u - t * C::CPT;
            const size_t row = (size_t)nn * n_tok + t, rqk = row * p.h_qk + gg, rv = row * p.h_v + hh;
            const char* src;
            if (r < 3 * C::CK) {
                const int seg = r / C::CK, off = r - seg * C::CK;
                const void* base = seg == 0 ? p.k : (seg == 1 ? p.q : p.b);
                src = static_cast<const char*>(base) + (seg < 2 ? rqk : rv) * (DK * C::ES) + off * 16;
            } else if (r < 3 * C::CK + C::CA) {
                const int off = r - 3 * C::CK;
                src = kPro ? static_cast<const char*>(p.a_raw) + rv * (DK * C::ES) + off * 16
                           : reinterpret_cast<const char*>(p.log_alpha + rv * DK) + off * 16;
            } else {
                const int r2 = r - 3 * C::CK - C::CA, seg = r2 / C::CV, off = r2 - seg * C::CV;
                src = static_cast<const char*>(seg == 0 ? p.v : p.w) + rv * (DV * C::ES) + off * 16;
            }
            cp_async16(raw + t * C::RREC + r * 16, src);
        }
    };

    if (tid == 0) {
        tc::mbar_init(bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    int slot = 0, nslot = 0;
    int it = next_active(blockIdx.x, &slot);
    if (it < n_items) issue(it, slot, p.test_withhold_loads != 0);
    cp_async_commit();
    uint32_t lphase = 0;  // parity of the state load being waited for
    bool fault = false;
    while (it < n_items) {
        const int nx = next_active(it + gridDim.x, &nslot);  // its slot lookup overlaps the wait below
        cp_async_wait_all();
        // bounded: a load that never lands ends the kernel with a status bit, not a hang
        if (!tc::mbar_wait(bar, lphase, p.wait_ns)) fault = true;
        lphase ^= 1u;
        if (__syncthreads_or(fault)) {  // this item's rows are in; the previous item's readers are done
            fault = true;
            break;
        }
        float4 s[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            s[i] = *reinterpret_cast<const float4*>(dsm_a + sofs + (uint32_t)i * (8 * 128));
        for (int idx = tid; idx < n_tok * DK; idx += NT) {
            const int t = idx / DK, c = idx - t * DK;
            const uint8_t* rec = raw + t * C::RREC;
            const float kv = to_f32(reinterpret_cast<const T*>(rec + C::RK)[c]);
            const float bv = to_f32(reinterpret_cast<const T*>(rec + C::RB)[c]);
            const int i = c >> 3;  // staged position of row c = 8 (4j + e) + rq: 4 (8j + rq) + e
            const int ps = t * DK + 4 * (8 * (i >> 2) + (c & 7)) + (i & 3);
            sk[ps] = kv;
            sq[ps] = to_f32(reinterpret_cast<const T*>(rec + C::RQ)[c]);
            if (kPro) {
                sa[ps] = sigmoid_f(-to_f32(reinterpret_cast<const T*>(rec + C::RA)[c]));
                se[ps] = sigmoid_f(bv) * kv;
            } else {
                sa[ps] = expf(reinterpret_cast<const float*>(rec + C::RA)[c]);
                se[ps] = bv * kv;
            }
        }
        for (int idx = tid; idx < n_tok * DV; idx += NT) {
            const int t = idx / DV, c = idx - t * DV;
            const uint8_t* rec = raw + t * C::RREC;
            float wv = to_f32(reinterpret_cast<const T*>(rec + C::RW)[c]);
            if (kPro) wv = sigmoid_f(wv);
            sx[idx] = wv * to_f32(reinterpret_cast<const T*>(rec + C::RV)[c]);
        }
        __syncthreads();  // the raw rows are consumed, and so is each thread's state buffer
        if (nx < n_items) issue(nx, nslot, false);
        cp_async_commit();

        const int n = it / p.h_v, h = it % p.h_v;
        // With the fused pre-processing, |q| and |k| are needed before the token loop, so the
        // per-token dot products q . (b (.) k), q . k and the norms are taken here (warp t takes
        // token t); otherwise the token loop forms the dot products itself, from the rows each
        // thread reads anyway, and this phase and its barrier are skipped.
        for (int t = warp; kPro && t < n_tok; t += NT / 32) {
            const float *qt = sq + t * DK, *et = se + t * DK, *kt = sk + t * DK;
            float d1 = 0.f, d2 = 0.f, nq = 0.f, nk = 0.f;
            for (int c = lane; c < DK; c += 32) {
                d1 += qt[c] * et[c];
                d2 += qt[c] * kt[c];
                if (kPro) {
                    nq += qt[c] * qt[c];
                    nk += kt[c] * kt[c];
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                d1 += __shfl_xor_sync(0xffffffffu, d1, off);
                d2 += __shfl_xor_sync(0xffffffffu, d2, off);
                if (kPro) {
                    nq += __shfl_xor_sync(0xffffffffu, nq, off);
                    nk += __shfl_xor_sync(0xffffffffu, nk, off);
                }
            }
            if (lane == 0) {
                float s2 = 1.f;
                if (kPro) {
                    rnorm[t][0] = 1.f / fmaxf(sqrtf(nq), kL2NormEps);
                    rnorm[t][1] = 1.f / fmaxf(sqrtf(nk), kL2NormEps);
                    s2 = rnorm[t][0] * rnorm[t][1];
                }
                dots[t][0] = d1 * s2;
                dots[t][1] = d2 * s2;
            }
        }
        if (kPro) __syncthreads();
        if (kPro) {  // normalise the staged q, k (and b (.) k)
            for (int idx = tid; idx < n_tok * DK; idx += NT) {
                const int t = idx / DK;
                sq[idx] *= rnorm[t][0];
                sk[idx] *= rnorm[t][1];
                se[idx] *= rnorm[t][1];
            }
            __syncthreads();
        }

        // the state stays in registers from token to token; no barrier in this loop
        for (int t = 0; t < n_tok; ++t) {
            const size_t row = (size_t)n * n_tok + t;  // token t of sequence n
            const float4 *at = reinterpret_cast<const float4*>(sa + t * DK) + rq;
            const float4 *kt = reinterpret_cast<const float4*>(sk + t * DK) + rq;
            const float4 *qt = reinterpret_cast<const float4*>(sq + t * DK) + rq;
            const float4 *et = reinterpret_cast<const float4*>(se + t * DK) + rq;
            // the state as column pairs (x, y) and (z, w): packed two-wide arithmetic
            float2 r0 = make_float2(0.f, 0.f), r1 = r0, p0 = r0, p1 = r0;
            float2 dq = make_float2(0.f, 0.f);  // this thread's rows of q . (b (.) k), q . k
#pragma unroll
            for (int j = 0; j < RPT / 4; ++j) {
                const float4 a4 = at[8 * j], k4 = kt[8 * j], q4 = qt[8 * j];
                const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kvv[4] = {k4.x, k4.y, k4.z, k4.w};
                const float qvv[4] = {q4.x, q4.y, q4.z, q4.w};
                if (!kPro) {
                    const float4 e4 = et[8 * j];
                    dq = ffma2(make_float2(q4.x, q4.x), make_float2(e4.x, k4.x), dq);
                    dq = ffma2(make_float2(q4.y, q4.y), make_float2(e4.y, k4.y), dq);
                    dq = ffma2(make_float2(q4.z, q4.z), make_float2(e4.z, k4.z), dq);
                    dq = ffma2(make_float2(q4.w, q4.w), make_float2(e4.w, k4.w), dq);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float4& si = s[4 * j + e];
                    const float2 a = dup2(av[e]), kv = dup2(kvv[e]), qv = dup2(qvv[e]);
                    const float2 s0 = fmul2(make_float2(si.x, si.y), a), s1 = fmul2(make_float2(si.z, si.w), a);
                    r0 = ffma2(kv, s0, r0); r1 = ffma2(kv, s1, r1);
                    p0 = ffma2(qv, s0, p0); p1 = ffma2(qv, s1, p1);
                    si = make_float4(s0.x, s0.y, s1.x, s1.y);
                }
            }
            // sums over the eight lanes of this column quad (the other row groups)
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                if (!kPro)
                    dq = fadd2(dq, make_float2(__shfl_xor_sync(0xffffffffu, dq.x, off),
                                               __shfl_xor_sync(0xffffffffu, dq.y, off)));
                r0 = fadd2(r0, make_float2(__shfl_xor_sync(0xffffffffu, r0.x, off), __shfl_xor_sync(0xffffffffu, r0.y, off)));
                r1 = fadd2(r1, make_float2(__shfl_xor_sync(0xffffffffu, r1.x, off), __shfl_xor_sync(0xffffffffu, r1.y, off)));
                p0 = fadd2(p0, make_float2(__shfl_xor_sync(0xffffffffu, p0.x, off), __shfl_xor_sync(0xffffffffu, p0.y, off)));
                p1 = fadd2(p1, make_float2(__shfl_xor_sync(0xffffffffu, p1.x, off), __shfl_xor_sync(0xffffffffu, p1.y, off)));
            }
            const float4 r = make_float4(r0.x, r0.y, r1.x, r1.y), pq = make_float4(p0.x, p0.y, p1.x, p1.y);
            const float4 x = *reinterpret_cast<const float4*>(sx + t * DV + col);
            const float2 x0 = make_float2(x.x, x.y), x1 = make_float2(x.z, x.w);
#pragma unroll
            for (int j = 0; j < RPT / 4; ++j) {
                const float4 e4 = et[8 * j], k4 = kt[8 * j];
                const float ev[4] = {e4.x, e4.y, e4.z, e4.w}, kvv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float4& si = s[4 * j + e];
                    const float2 ne = dup2(-ev[e]), kv = dup2(kvv[e]);
                    const float2 s0 = ffma2(kv, x0, ffma2(ne, r0, make_float2(si.x, si.y)));
                    const float2 s1 = ffma2(kv, x1, ffma2(ne, r1, make_float2(si.z, si.w)));
                    si = make_float4(s0.x, s0.y, s1.x, s1.y);
                    if (p.S_steps)  // the parameter re-read here keeps no pointer live in the loop
                        __stcs(reinterpret_cast<float4*>(p.S_steps + (row * p.h_v + h) * DK * DV +
                                                         (size_t)(8 * (4 * j + e) + rq) * DV + col), si);
                }
            }
            if (rq == 0) {
                const float qe = kPro ? dots[t][0] : dq.x, qk = kPro ? dots[t][1] : dq.y;
                TO* o = static_cast<TO*>(p.o) + (row * p.h_v + h) * DV + col;
                o[0] = from_f32<TO>(pq.x - qe * r.x + qk * x.x);
                o[1] = from_f32<TO>(pq.y - qe * r.y + qk * x.y);
                o[2] = from_f32<TO>(pq.z - qe * r.z + qk * x.z);
                o[3] = from_f32<TO>(pq.w - qe * r.w + qk * x.w);
            }
        }
        float* S = state_of(it, slot);
#pragma unroll
        for (int i = 0; i < RPT; ++i) __stcs(reinterpret_cast<float4*>(S + (size_t)(8 * i + rq) * DV + col), s[i]);
        it = nx;
        slot = nslot;
    }
    if (fault) {
        if (tid == 0) atomicOr(&g_status_dec, kStatusWaitTimeout);
        // give a load still in flight a last bounded chance to land before the CTA exits
        if (tid == 0) tc::mbar_wait(bar, lphase ^ 1u, p.wait_ns);
    }
}

template <int DK, int DV, typename T, typename TO, bool kPro>
cudaError_t launch_dec_p(const Params& p, cudaStream_t st) {
    if (p.n_tok == 1 && !p.S_steps) {
        decode_kernel<DK, DV, T, TO, kPro><<<p.n_seq * p.h_v, kThreads, 0, st>>>(p);
        return cudaGetLastError();
    }
    using C = MultiCfg<DK, DV, T, kPro>;
    auto kern = decode_multi_kernel<DK, DV, T, TO, kPro>;
    const size_t smem = C::smem(p.n_tok);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int dev = 0, sms = 0, per_sm = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::NT, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // the state pool as a 2-d fp32 tensor [n_slots * h_v * dk rows][dv], in boxes of 32
    // columns x dk rows with the 128-byte swizzle
    const auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encoder());
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap smap;
    cuuint64_t dims[2] = {(cuuint64_t)DV, (cuuint64_t)p.n_slots * (cuuint64_t)p.h_v * DK};
    cuuint64_t strides[1] = {(cuuint64_t)DV * 4};
    cuuint32_t box[2] = {32u, (cuuint32_t)DK};
    cuuint32_t estr[2] = {1u, 1u};
    if (encode(&smap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.S_T, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int items = p.n_seq * p.h_v;
    const int grid = items < sms * per_sm ? items : sms * per_sm;  // persistent CTAs
    kern<<<grid, C::NT, smem, st>>>(p, smap);
    return cudaGetLastError();
}

template <int DK, int DV, typename T, typename TO>
cudaError_t launch_dec(const Params& p, cudaStream_t st) {
    return p.prologue ? launch_dec_p<DK, DV, T, TO, true>(p, st) : launch_dec_p<DK, DV, T, TO, false>(p, st);
}

template <typename T, typename TO>
cudaError_t launch_dec_t(const Params& p, cudaStream_t s) {
    if (p.dk == 128) return p.dv == 128 ? launch_dec<128, 128, T, TO>(p, s) : launch_dec<128, 64, T, TO>(p, s);
    return p.dv == 128 ? launch_dec<64, 128, T, TO>(p, s) : launch_dec<64, 64, T, TO>(p, s);
}

}  // namespace

cudaError_t read_clear_status_decode(unsigned int* out, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_status_dec, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    static const unsigned int zero = 0;
    return cudaMemcpyToSymbolAsync(g_status_dec, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
}

cudaError_t launch_decode(const Params& p, gdn2_dtype dt, gdn2_dtype odt, cudaStream_t s) {
    if (dt == GDN2_F32)
        return odt == GDN2_F32 ? launch_dec_t<float, float>(p, s) : launch_dec_t<float, __nv_bfloat16>(p, s);
    return odt == GDN2_F32 ? launch_dec_t<__nv_bfloat16, float>(p, s)
                           : launch_dec_t<__nv_bfloat16, __nv_bfloat16>(p, s);
}

}  // namespace gdn2
