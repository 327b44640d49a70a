// recurrent.cu -- token-sequential kernel for gdn2_chunk_fwd: the fp32 path.
//
// Each CTA owns one (sequence, value head, 32-column slice of the value axis). The value
// columns of the state evolve independently (the transition acts on the key axis only),
// so slices need no communication. Lane j of every warp owns value column j of the slice;
// warp w owns key rows [w*DK/4, (w+1)*DK/4), so the state lives in registers, DK/4 floats
// per thread. Per token:
//   decay      s *= alpha                (alpha = exp(log_alpha), key axis)
//   key read   r = sum_rows k * s        (partial per warp, summed through shared memory)
//   query read p = sum_rows q * s        (same pass, on the decayed old state)
//   edit       s += -(b*k) r + k (w*v)
//   output     o = p - (q.(b*k)) r + (q.k)(w*v)   == (edited state)^T q
// Inputs are staged 16 tokens at a time in shared memory as fp32, with alpha and b*k
// precomputed. All arithmetic is fp32.
#include "internal.cuh"

namespace gdn2 {
namespace {

constexpr int kCols = 32;   // value columns per CTA, one per lane
constexpr int kSplit = 4;   // warps per CTA, each owning DK/kSplit key rows
constexpr int kStage = 16;  // tokens staged per pass

template <int DK>
struct RecSmem {
    float k[kStage][DK];
    float q[kStage][DK];
    float a[kStage][DK];  // alpha = exp(log_alpha)
    float e[kStage][DK];  // b (.) k
    float x[kStage][kCols];
    float qe[kStage];
    float qk[kStage];
    float red[2][2][kSplit][kCols];  // [token parity][r | p][warp][column]
};

// Device status word of this file's kernel (kStatus* bits), read and cleared by
// gdn2_device_status.
__device__ unsigned int g_status_rec = 0;

template <int DK, typename T, typename TO>
__global__ void __launch_bounds__(kCols * kSplit) recurrent_kernel(Params p) {
    __shared__ RecSmem<DK> sm;
    constexpr int RPT = DK / kSplit;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int slice = blockIdx.x;
    const int h = blockIdx.y;
    const int n = p.order ? p.order[blockIdx.z] : (int)blockIdx.z;
    if ((unsigned)n >= (unsigned)p.n_seq) {  // a stale order entry: skip the item, touch nothing
        if (threadIdx.x == 0) atomicOr(&g_status_rec, kStatusBadOrder);
        return;
    }
    const int g = h / (p.h_v / p.h_qk);
    const int col = slice * kCols + lane;
    const int row0 = warp * RPT;
    const int dv = p.dv;

    int t0, t1;
    seq_bounds(p, n, t0, t1);
    const size_t soff = ((size_t)n * p.h_v + h) * DK * dv;

    float s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = p.S0 ? p.S0[soff + (size_t)(row0 + i) * dv + col] : 0.f;

    const T* qp = static_cast<const T*>(p.q);
    const T* kp = static_cast<const T*>(p.k);
    const T* vp = static_cast<const T*>(p.v);
    const T* bp = static_cast<const T*>(p.b);
    const T* wp = static_cast<const T*>(p.w);
    TO* op = static_cast<TO*>(p.o);

    for (int base = t0; base < t1; base += kStage) {
        const int nt = min(kStage, t1 - base);
        __syncthreads();  // the previous stage is fully consumed
        for (int idx = threadIdx.x; idx < nt * DK; idx += blockDim.x) {
            const int tt = idx / DK, c = idx % DK;
            const size_t t = (size_t)(base + tt);
            const float kv = to_f32(kp[(t * p.h_qk + g) * DK + c]);
            const float qv = to_f32(qp[(t * p.h_qk + g) * DK + c]);
            const float la = p.log_alpha[(t * p.h_v + h) * DK + c];
            const float bv = to_f32(bp[(t * p.h_v + h) * DK + c]);
            sm.k[tt][c] = kv;
            sm.q[tt][c] = qv;
            sm.a[tt][c] = expf(la);
            sm.e[tt][c] = bv * kv;
        }
        for (int idx = threadIdx.x; idx < nt * kCols; idx += blockDim.x) {
            const int tt = idx / kCols, c = idx % kCols;
            const size_t t = (size_t)(base + tt);
            const size_t off = (t * p.h_v + h) * dv + slice * kCols + c;
            sm.x[tt][c] = to_f32(wp[off]) * to_f32(vp[off]);
        }
        __syncthreads();
        for (int tt = warp; tt < nt; tt += kSplit) {
            float d1 = 0.f, d2 = 0.f;
            for (int c = lane; c < DK; c += 32) {
                d1 += sm.q[tt][c] * sm.e[tt][c];
                d2 += sm.q[tt][c] * sm.k[tt][c];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                d1 += __shfl_xor_sync(0xffffffffu, d1, off);
                d2 += __shfl_xor_sync(0xffffffffu, d2, off);
            }
            if (lane == 0) {
                sm.qe[tt] = d1;
                sm.qk[tt] = d2;
            }
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            float r = 0.f, pq = 0.f;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                s[i] *= sm.a[tt][row0 + i];
                r = fmaf(sm.k[tt][row0 + i], s[i], r);
                pq = fmaf(sm.q[tt][row0 + i], s[i], pq);
            }
            const int par = tt & 1;
            sm.red[par][0][warp][lane] = r;
            sm.red[par][1][warp][lane] = pq;
            __syncthreads();
            r = 0.f;
            pq = 0.f;
#pragma unroll
            for (int w = 0; w < kSplit; ++w) {
                r += sm.red[par][0][w][lane];
                pq += sm.red[par][1][w][lane];
            }
            const float x = sm.x[tt][lane];
#pragma unroll
            for (int i = 0; i < RPT; ++i)
                s[i] = fmaf(sm.k[tt][row0 + i], x, fmaf(-sm.e[tt][row0 + i], r, s[i]));
            if (warp == (tt % kSplit)) {
                const float o = pq - sm.qe[tt] * r + sm.qk[tt] * x;
                op[((size_t)(base + tt) * p.h_v + h) * dv + col] = from_f32<TO>(o);
            }
        }
    }
    if (p.S_T) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) p.S_T[soff + (size_t)(row0 + i) * dv + col] = s[i];
    }
}

template <int DK, typename T, typename TO>
cudaError_t launch_rec(const Params& p, cudaStream_t st) {
    dim3 grid(p.dv / kCols, p.h_v, p.n_seq);
    recurrent_kernel<DK, T, TO><<<grid, kCols * kSplit, 0, st>>>(p);
    return cudaGetLastError();
}

template <typename T, typename TO>
cudaError_t launch_rec_dk(const Params& p, cudaStream_t s) {
    return p.dk == 128 ? launch_rec<128, T, TO>(p, s) : launch_rec<64, T, TO>(p, s);
}

}  // namespace

cudaError_t read_clear_status_recurrent(unsigned int* out, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_status_rec, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    static const unsigned int zero = 0;
    return cudaMemcpyToSymbolAsync(g_status_rec, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
}

cudaError_t launch_recurrent(const Params& p, gdn2_dtype dt, gdn2_dtype odt, cudaStream_t s) {
    if (dt == GDN2_F32)
        return odt == GDN2_F32 ? launch_rec_dk<float, float>(p, s) : launch_rec_dk<float, __nv_bfloat16>(p, s);
    return odt == GDN2_F32 ? launch_rec_dk<__nv_bfloat16, float>(p, s)
                           : launch_rec_dk<__nv_bfloat16, __nv_bfloat16>(p, s);
}

}  // namespace gdn2
