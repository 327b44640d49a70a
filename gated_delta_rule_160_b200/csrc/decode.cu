// decode.cu -- one decode step: one new token per sequence, state updated in place.
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

template <int DK, int DV, typename T, typename TO>
__global__ void __launch_bounds__(kThreads) decode_kernel(Params p) {
    constexpr int TPR = DV / 4;          // threads per state row
    constexpr int RG = kThreads / TPR;   // row groups
    constexpr int RPT = DK / RG;         // rows per thread
    __shared__ float sa[DK], sk[DK], sq[DK], se[DK], sx[DV];
    __shared__ float4 red[2][RG][TPR];
    __shared__ float dots[2];

    const int item = blockIdx.x;  // n * h_v + h
    const int n = item / p.h_v;
    const int h = item % p.h_v;
    const int g = h / (p.h_v / p.h_qk);
    const int cg = threadIdx.x % TPR;
    const int rg = threadIdx.x / TPR;
    float* S = p.S_T + (size_t)item * DK * DV;

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(rg + RG * i) * DV) + cg);

    const size_t tq = (size_t)n * p.h_qk + g;  // token n of sequence n
    const size_t tv = (size_t)n * p.h_v + h;
    for (int c = threadIdx.x; c < DK; c += kThreads) {
        const float kv = to_f32(static_cast<const T*>(p.k)[tq * DK + c]);
        sk[c] = kv;
        sq[c] = to_f32(static_cast<const T*>(p.q)[tq * DK + c]);
        sa[c] = expf(p.log_alpha[tv * DK + c]);
        se[c] = to_f32(static_cast<const T*>(p.b)[tv * DK + c]) * kv;
    }
    for (int c = threadIdx.x; c < DV; c += kThreads)
        sx[c] = to_f32(static_cast<const T*>(p.w)[tv * DV + c]) *
                to_f32(static_cast<const T*>(p.v)[tv * DV + c]);
    __syncthreads();
    if (threadIdx.x < 32) {
        float d1 = 0.f, d2 = 0.f;
        for (int c = threadIdx.x; c < DK; c += 32) {
            d1 += sq[c] * se[c];
            d2 += sq[c] * sk[c];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            d1 += __shfl_xor_sync(0xffffffffu, d1, off);
            d2 += __shfl_xor_sync(0xffffffffu, d2, off);
        }
        if (threadIdx.x == 0) {
            dots[0] = d1;
            dots[1] = d2;
        }
    }

    float4 r = make_float4(0.f, 0.f, 0.f, 0.f), pq = r;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = rg + RG * i;
        const float a = sa[row], kv = sk[row], qv = sq[row];
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
    const float4 x = *reinterpret_cast<const float4*>(sx + 4 * cg);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = rg + RG * i;
        const float e = -se[row], kv = sk[row];
        float4 t = s[i];
        t.x = fmaf(kv, x.x, fmaf(e, r.x, t.x));
        t.y = fmaf(kv, x.y, fmaf(e, r.y, t.y));
        t.z = fmaf(kv, x.z, fmaf(e, r.z, t.z));
        t.w = fmaf(kv, x.w, fmaf(e, r.w, t.w));
        __stcs(reinterpret_cast<float4*>(S + (size_t)row * DV) + cg, t);
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

template <int DK, int DV, typename T, typename TO>
cudaError_t launch_dec(const Params& p, cudaStream_t st) {
    decode_kernel<DK, DV, T, TO><<<p.n_seq * p.h_v, kThreads, 0, st>>>(p);
    return cudaGetLastError();
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
