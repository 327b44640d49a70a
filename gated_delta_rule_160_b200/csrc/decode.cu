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
#include "internal.cuh"

namespace gdn2 {
namespace {

constexpr int kThreads = 256;

// kMulti: several tokens, or every intermediate state, so the state is kept in registers
// across tokens and stored at the end; otherwise each state row is stored as soon as it is
// updated, which keeps fewer registers live (two CTAs per SM for dk = dv = 128). All the
// tokens' inputs are staged in shared memory before the first one is applied, so HBM latency
// is paid once per step, not once per token.
// kPro: fused pre-processing (raw q, k L2-normalised per token; log_alpha = -softplus of
// the decay pre-activation; sigmoid b, w), applied while the token inputs are staged.
template <int DK, int DV, typename T, typename TO, bool kMulti, bool kPro>
__global__ void __launch_bounds__(kThreads) decode_kernel(Params p) {
    constexpr int TPR = DV / 4;          // threads per state row
    constexpr int RG = kThreads / TPR;   // row groups
    constexpr int RPT = DK / RG;         // rows per thread
    constexpr int NTM = kMulti ? GDN2_DECODE_MAX_TOKENS : 1;
    __shared__ float sa[NTM][DK], sk[NTM][DK], sq[NTM][DK], se[NTM][DK], sx[NTM][DV];
    __shared__ float4 red[2][2][RG][TPR];  // [token parity][r | p]
    __shared__ float dots[NTM][2];
    __shared__ float rnorm[NTM][2];  // 1 / |q|, 1 / |k| (fused pre-processing)

    const int item = blockIdx.x;  // n * h_v + h
    const int n = item / p.h_v;
    const int h = item % p.h_v;
    const int g = h / (p.h_v / p.h_qk);
    const int slot = p.slots ? p.slots[n] : n;
    if (slot < 0 || slot >= p.n_slots) return;  // an inactive sequence: nothing to do
    const int cg = threadIdx.x % TPR;
    const int rg = threadIdx.x / TPR;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int n_tok = kMulti ? p.n_tok : 1;
    float* S = p.S_T + ((size_t)slot * p.h_v + h) * DK * DV;

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(rg + RG * i) * DV) + cg);

    // every token's decay, key, query, erase and write vectors
    for (int idx = threadIdx.x; idx < n_tok * DK; idx += kThreads) {
        const int t = idx / DK, c = idx % DK;
        const size_t row = (size_t)n * n_tok + t;
        const size_t tq = row * p.h_qk + g, tv = row * p.h_v + h;
        const float kv = to_f32(static_cast<const T*>(p.k)[tq * DK + c]);
        const float bv = to_f32(static_cast<const T*>(p.b)[tv * DK + c]);
        sk[t][c] = kv;
        sq[t][c] = to_f32(static_cast<const T*>(p.q)[tq * DK + c]);
        if (kPro) {  // alpha = exp(-softplus(a)) = 1 / (1 + e^a)
            sa[t][c] = sigmoid_f(-to_f32(static_cast<const T*>(p.a_raw)[tv * DK + c]));
            se[t][c] = sigmoid_f(bv) * kv;
        } else {
            sa[t][c] = expf(p.log_alpha[tv * DK + c]);
            se[t][c] = bv * kv;
        }
    }
    for (int idx = threadIdx.x; idx < n_tok * DV; idx += kThreads) {
        const int t = idx / DV, c = idx % DV;
        const size_t tv = ((size_t)n * n_tok + t) * p.h_v + h;
        float wv = to_f32(static_cast<const T*>(p.w)[tv * DV + c]);
        if (kPro) wv = sigmoid_f(wv);
        sx[t][c] = wv * to_f32(static_cast<const T*>(p.v)[tv * DV + c]);
    }
    __syncthreads();
    // q . (b (.) k) and q . k of every token (and |q|, |k| with the fused pre-processing):
    // warp t takes token t
    for (int t = warp; t < n_tok; t += kThreads / 32) {
        float d1 = 0.f, d2 = 0.f, nq = 0.f, nk = 0.f;
        for (int c = lane; c < DK; c += 32) {
            d1 += sq[t][c] * se[t][c];
            d2 += sq[t][c] * sk[t][c];
            if (kPro) {
                nq += sq[t][c] * sq[t][c];
                nk += sk[t][c] * sk[t][c];
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
    if (kPro) {  // normalise the staged q, k (and b (.) k)
        __syncthreads();
        for (int idx = threadIdx.x; idx < n_tok * DK; idx += kThreads) {
            const int t = idx / DK, c = idx % DK;
            sq[t][c] *= rnorm[t][0];
            sk[t][c] *= rnorm[t][1];
            se[t][c] *= rnorm[t][1];
        }
        __syncthreads();
    }

    // the state stays in registers from token to token
    for (int t = 0; t < n_tok; ++t) {
        const size_t row = (size_t)n * n_tok + t;  // token t of sequence n
        const size_t tv = row * p.h_v + h;
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int rw = rg + RG * i;
            const float a = sa[t][rw], kv = sk[t][rw], qv = sq[t][rw];
            s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
            r.x = fmaf(kv, s[i].x, r.x); r.y = fmaf(kv, s[i].y, r.y);
            r.z = fmaf(kv, s[i].z, r.z); r.w = fmaf(kv, s[i].w, r.w);
            pq.x = fmaf(qv, s[i].x, pq.x); pq.y = fmaf(qv, s[i].y, pq.y);
            pq.z = fmaf(qv, s[i].z, pq.z); pq.w = fmaf(qv, s[i].w, pq.w);
        }
        // partial sums in the buffer of this token's parity: the one of the token before is
        // still being read, the one of two tokens before is free (a barrier lies between)
        red[t & 1][0][rg][cg] = r;
        red[t & 1][1][rg][cg] = pq;
        __syncthreads();
        r = make_float4(0.f, 0.f, 0.f, 0.f);
        pq = r;
#pragma unroll
        for (int j = 0; j < RG; ++j) {
            const float4 a = red[t & 1][0][j][cg], b = red[t & 1][1][j][cg];
            r.x += a.x; r.y += a.y; r.z += a.z; r.w += a.w;
            pq.x += b.x; pq.y += b.y; pq.z += b.z; pq.w += b.w;
        }
        const float4 x = *reinterpret_cast<const float4*>(&sx[t][4 * cg]);
        float* Ss = kMulti && p.S_steps ? p.S_steps + (row * p.h_v + h) * DK * DV : nullptr;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int rw = rg + RG * i;
            const float e = -se[t][rw], kv = sk[t][rw];
            s[i].x = fmaf(kv, x.x, fmaf(e, r.x, s[i].x));
            s[i].y = fmaf(kv, x.y, fmaf(e, r.y, s[i].y));
            s[i].z = fmaf(kv, x.z, fmaf(e, r.z, s[i].z));
            s[i].w = fmaf(kv, x.w, fmaf(e, r.w, s[i].w));
            if (!kMulti) __stcs(reinterpret_cast<float4*>(S + (size_t)rw * DV) + cg, s[i]);
            if (Ss) __stcs(reinterpret_cast<float4*>(Ss + (size_t)rw * DV) + cg, s[i]);
        }
        if (rg == 0) {
            const float qe = dots[t][0], qk = dots[t][1];
            TO* o = static_cast<TO*>(p.o) + tv * DV + 4 * cg;
            o[0] = from_f32<TO>(pq.x - qe * r.x + qk * x.x);
            o[1] = from_f32<TO>(pq.y - qe * r.y + qk * x.y);
            o[2] = from_f32<TO>(pq.z - qe * r.z + qk * x.z);
            o[3] = from_f32<TO>(pq.w - qe * r.w + qk * x.w);
        }
    }
    if (kMulti) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) __stcs(reinterpret_cast<float4*>(S + (size_t)(rg + RG * i) * DV) + cg, s[i]);
    }
}

template <int DK, int DV, typename T, typename TO, bool kPro>
cudaError_t launch_dec_p(const Params& p, cudaStream_t st) {
    if (p.n_tok > 1 || p.S_steps)
        decode_kernel<DK, DV, T, TO, true, kPro><<<p.n_seq * p.h_v, kThreads, 0, st>>>(p);
    else
        decode_kernel<DK, DV, T, TO, false, kPro><<<p.n_seq * p.h_v, kThreads, 0, st>>>(p);
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

cudaError_t launch_decode(const Params& p, gdn2_dtype dt, gdn2_dtype odt, cudaStream_t s) {
    if (dt == GDN2_F32)
        return odt == GDN2_F32 ? launch_dec_t<float, float>(p, s) : launch_dec_t<float, __nv_bfloat16>(p, s);
    return odt == GDN2_F32 ? launch_dec_t<__nv_bfloat16, float>(p, s)
                           : launch_dec_t<__nv_bfloat16, __nv_bfloat16>(p, s);
}

}  // namespace gdn2
