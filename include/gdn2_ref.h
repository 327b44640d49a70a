/*
 * gdn2_ref.h -- C ABI of the fp64 CPU oracle for the Gated DeltaNet-2 recurrence.
 *
 * TEST INFRASTRUCTURE. The oracle lives in oracle/ and is built into its own shared
 * library (oracle/libgdn2_ref.so). It shares no code, header, table or helper with the
 * CUDA library described by gdn2.h; only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.
 *
 * What it computes (per sequence n and value head h, tokens t in order):
 *   S'_t = Diag(alpha_t) S_{t-1}                  alpha_t = exp(log_alpha_t), key axis
 *   r_t  = S'_t^T k_t                             read with the key, before the edit
 *   S_t  = S'_t - (b_t (.) k_t) r_t^T             erase along the key axis (gate b_t)
 *             + k_t (w_t (.) v_t)^T              write along the value axis (gate w_t)
 *   o_t  = S_t^T q_t                              read with the query, after the edit
 * Sources: the tilnote.io note on Gated DeltaNet-2, section "Gated DeltaNet-2 design
 * point" (channel-wise erase gate b_t on the key axis, channel-wise write gate w_t on the
 * value axis, the KDA channel-wise decay, and the order decay -> remove key-side component
 * -> add value-side component); the ai-systems-engineering.com post "Delta rule:
 * correcting the state's associations toward the new Value", sections "Why read with the
 * Key, why with the Query" (key read of the old state, query read of the updated state)
 * and "Recording the difference between the read value and the new Value" (r^T = k^T S,
 * state rows = key channels, columns = value channels).
 *
 * Layouts (all row-major, C order, innermost index last):
 *   q, k        [T_total, h_qk, dk]   dtype (GDN2_REF_F32: float, GDN2_REF_BF16: uint16 bf16 bits)
 *   v, w        [T_total, h_v,  dv]   dtype
 *   log_alpha   [T_total, h_v,  dk]   float (always fp32)
 *   b           [T_total, h_v,  dk]   dtype
 *   S0          [n_seq, h_v, dk, dv]  float, or NULL for a zero initial state
 *   o   (out)   [T_total, h_v,  dv]   double
 *   S_T (out)   [n_seq, h_v, dk, dv]  double, or NULL if not wanted
 *   cu_seqlens  [n_seq + 1] int32, cu_seqlens[0] = 0, non-decreasing, last = T_total;
 *               or NULL, in which case every sequence has T_total / n_seq tokens.
 * Value head h reads query/key head  h / (h_v / h_qk)  (consecutive groups).
 *
 * Ownership: all pointers are host memory owned by the caller; the oracle allocates only
 * per-thread scratch and frees it before returning.
 * Threads: OpenMP over (sequence, value head); n_threads <= 0 uses the OpenMP default.
 * Errors: returns GDN2_REF_OK, or GDN2_REF_EINVAL (nothing written) when a pointer that
 * must be set is NULL, a size is non-positive, h_v is not a multiple of h_qk, the dtype is
 * unknown, or cu_seqlens is malformed; GDN2_REF_ENOMEM if scratch allocation failed.
 */
#ifndef GDN2_REF_H
#define GDN2_REF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { GDN2_REF_F32 = 0, GDN2_REF_BF16 = 1 };
enum { GDN2_REF_OK = 0, GDN2_REF_EINVAL = 1, GDN2_REF_ENOMEM = 2 };

int gdn2_fwd_ref(int n_seq, int T_total, const int32_t* cu_seqlens,
                 int h_qk, int h_v, int dk, int dv, int dtype,
                 const void* q, const void* k, const void* v,
                 const float* log_alpha, const void* b, const void* w,
                 const float* S0, double* o, double* S_T, int n_threads);

/* Number of OpenMP threads a call with n_threads <= 0 would use. */
int gdn2_ref_max_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_REF_H */
