// internal.cuh -- declarations shared by the libgdn2 translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn2.h"

namespace gdn2 {

// Everything a kernel needs about one call; pointers are device pointers.
struct Params {
    int n_seq, T_total, h_qk, h_v, dk, dv;
    int T_fixed;               // tokens per sequence when cu_seqlens is NULL, else 0
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const void* b;
    const void* w;
    const float* S0;           // nullable
    const int32_t* cu_seqlens; // nullable
    void* o;
    float* S_T;                // nullable (decode: the in/out state)
    const int32_t* order;      // nullable: sequences longest first (varlen scheduling)
    // decode only
    int n_tok;                 // tokens per sequence and step (1..8)
    const int32_t* slots;      // nullable: state slot of each sequence in S_T's pool
    int n_slots;               // states in the pool
    float* S_steps;            // nullable: state after each token [n_seq, n_tok, h_v, dk, dv]
    // fused pre-processing: q, k, b, w are raw projections and log_alpha is replaced by the
    // decay pre-activation a_raw (dtype, same layout): q, k <- L2-normalised, log_alpha <-
    // -softplus(a_raw), b, w <- sigmoid
    int prologue;
    const void* a_raw;
    // bounded waits (tensor-core prefill, multi-token decode): a wait longer than wait_ns is
    // a fault; the CTA records it in the device status word, releases its tensor memory (if
    // any) and returns
    unsigned long long wait_ns;
    // testing only: the prefill's producer never issues the first chunk's loads, and the
    // multi-token decode never issues its first state load, so the CTA's waits run out
    // (nothing asynchronous is in flight when it gives up)
    int test_withhold_loads;
};

// Device status word bits (see gdn2_device_status in gdn2.h).
constexpr unsigned int kStatusWaitTimeout = GDN2_DEVICE_WAIT_TIMEOUT;
constexpr unsigned int kStatusBadSeqlens = GDN2_DEVICE_BAD_SEQLENS;
constexpr unsigned int kStatusBadOrder = GDN2_DEVICE_BAD_ORDER;
constexpr unsigned int kStatusDecayRange = GDN2_DEVICE_DECAY_RANGE;
constexpr unsigned long long kDefaultWaitNs = 4000000000ull;

// Pieces of the fused pre-processing, in fp32, on the special-function unit. Their errors
// are absolute ~1e-7 (softplus: summed into log-decays) and relative ~1e-6 (sigmoid), far
// below what the bf16 operands of the recurrence carry.
__device__ __forceinline__ float sigmoid_f(float x) {
    // 1 / (1 + e^-x); the exponent is capped where the quotient is already ~1e-35
    return __fdividef(1.f, 1.f + __expf(fminf(-x, 80.f)));
}
__device__ __forceinline__ float softplus_f(float x) {  // log(1 + e^x), without overflow
    return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)));
}
// softplus(x) log2(e) = max(x, 0) log2(e) + log2(1 + 2^(-|x| log2(e))), in base 2 throughout
// (two special-function operations, no conversions between the bases)
__device__ __forceinline__ float softplus_log2e_f(float x) {
    constexpr float kL2e = 1.4426950408889634f;
    float e, l;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-fabsf(x) * kL2e));
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.f + e));
    return fmaf(fmaxf(x, 0.f), kL2e, l);
}
// sigmoid from one special-function operation: 1/2 + tanh(x / 2) / 2, with tanh.approx's
// relative error of about 2^-11 (absolute error of the result below 2.5e-4). Used only where
// the value is rounded to a plain bf16 operand next (2^-9), never where a hi / lo split
// carries it.
__device__ __forceinline__ float sigmoid_tanh_f(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
constexpr float kL2NormEps = 1e-12f;  // q and k are divided by max(|x|_2, eps)

// 16-byte asynchronous copies global -> shared (cp.async, cached in L2 only), completed per
// thread by cp_async_wait_all (copies made visible to other threads by a barrier after it).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Packed two-wide fp32 arithmetic (sm_100): one instruction for two lanes' fma / mul / add,
// each rounded to nearest like fmaf / __fmul_rn / __fadd_rn, so a pairwise rewrite of scalar
// code gives the same bits.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 dup2(float x) { return make_float2(x, x); }

// Token range [t0, t1) of sequence n.
__device__ __forceinline__ void seq_bounds(const Params& p, int n, int& t0, int& t1) {
    if (p.cu_seqlens) {
        // clamped, so malformed offsets cannot send a kernel outside the token range
        t0 = min(max(p.cu_seqlens[n], 0), p.T_total);
        t1 = min(max(p.cu_seqlens[n + 1], t0), p.T_total);
    } else {
        t0 = n * p.T_fixed;
        t1 = t0 + p.T_fixed;
    }
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_recurrent(const Params& p, gdn2_dtype dt, gdn2_dtype odt, cudaStream_t s);
cudaError_t launch_decode(const Params& p, gdn2_dtype dt, gdn2_dtype odt, cudaStream_t s);
cudaError_t launch_varlen_order(const Params& p, int32_t* order, cudaStream_t s);
bool chunk_tc_supported(const Params& p, gdn2_dtype dt);
cudaError_t launch_chunk_tc(const Params& p, gdn2_dtype odt, cudaStream_t s);  // honours p.prologue
// Each translation unit that can flag a device-side error keeps its own status word; these
// queue, on stream s, a read of the word into *out (host) followed by clearing it.
cudaError_t read_clear_status_chunk_tc(unsigned int* out, cudaStream_t s);
cudaError_t read_clear_status_recurrent(unsigned int* out, cudaStream_t s);
cudaError_t read_clear_status_schedule(unsigned int* out, cudaStream_t s);
cudaError_t read_clear_status_decode(unsigned int* out, cudaStream_t s);
// cuTensorMapEncodeTiled from the driver (as a void*; NULL if unavailable)
void* tensor_map_encoder();
// Validate cu_seqlens on the device (flags kStatusBadSeqlens); used where no order kernel runs.
cudaError_t launch_check_seqlens(const Params& p, cudaStream_t s);
// Backward (gradients of the recurrence).
size_t bwd_workspace_bytes(const gdn2_shape* sh);
cudaError_t launch_bwd(const Params& p, gdn2_dtype dt, const float* dO, const float* dS_T, float* dq, float* dk,
                       float* dv, float* dla, float* db, float* dw, float* dS0, void* workspace, cudaStream_t s);
// Record a failure in the calling thread's error string and return st.
gdn2_status report_error(gdn2_status st, const char* msg);

}  // namespace gdn2
