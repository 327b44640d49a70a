/*
 * gdn2_ref.c -- the oracle: a plain, sequential, fp64 CPU statement of the Gated
 * DeltaNet-2 state recurrence, one token at a time.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. It shares no code with the CUDA library.
 *
 * The recurrence, per sequence and value head (see include/gdn2_ref.h for layouts):
 *   decay   S <- Diag(alpha_t) S                      (KDA channel-wise decay on the key axis)
 *   read    r <- S^T k_t                               (read the old state with the key)
 *   erase   S <- S - (b_t (.) k_t) r^T                 (erase gate b_t on the key axis)
 *   write   S <- S + k_t (w_t (.) v_t)^T               (write gate w_t on the value axis)
 *   output  o_t <- S^T q_t                             (read the updated state with the query)
 * Sources: tilnote.io note on Gated DeltaNet-2, section "Gated DeltaNet-2 design point"
 * (separate channel-wise erase gate b_t on the key axis and write gate w_t on the value
 * axis; the decayed previous state loses its key-side component, then gains the
 * value-side one); ai-systems-engineering.com "Delta rule" post, sections "Why read with
 * the Key, why with the Query" (old state read with the key, updated state read with the
 * query) and "Recording the difference ..." (r^T = k^T S; rows are key channels, columns
 * value channels); news.hamidun.com "NVIDIA Presente Gated DeltaNet-2", section "Comment
 * DeltaNet-2 a Repense l'Architecture" (two independent channel-wise gates).
 *
 * Every step is written out as the loop it is; there is no blocking or reordering. The
 * only library routine used is exp() from libm.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "../include/gdn2_ref.h"

/* Read element i of a buffer holding fp32 or bf16 values, widened exactly to double. */
static double elem(const void* p, size_t i, int dtype) {
    if (dtype == GDN2_REF_F32) return (double)((const float*)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int gdn2_ref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int gdn2_fwd_ref(int n_seq, int T_total, const int32_t* cu_seqlens,
                 int h_qk, int h_v, int dk, int dv, int dtype,
                 const void* q, const void* k, const void* v,
                 const float* log_alpha, const void* b, const void* w,
                 const float* S0, double* o, double* S_T, int n_threads) {
    if (n_seq <= 0 || T_total < 0 || h_qk <= 0 || h_v <= 0 || dk <= 0 || dv <= 0)
        return GDN2_REF_EINVAL;
    if (h_v % h_qk != 0) return GDN2_REF_EINVAL;
    if (dtype != GDN2_REF_F32 && dtype != GDN2_REF_BF16) return GDN2_REF_EINVAL;
    if (T_total > 0 && (!q || !k || !v || !log_alpha || !b || !w || !o)) return GDN2_REF_EINVAL;
    if (cu_seqlens) {
        if (cu_seqlens[0] != 0 || cu_seqlens[n_seq] != T_total) return GDN2_REF_EINVAL;
        for (int n = 0; n < n_seq; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return GDN2_REF_EINVAL;
    } else if (T_total % n_seq != 0) {
        return GDN2_REF_EINVAL;
    }

    const int group = h_v / h_qk;
    const long pairs = (long)n_seq * h_v;
    int failed = 0;

#ifdef _OPENMP
    int nt = n_threads > 0 ? n_threads : omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : failed)
#endif
    for (long pair = 0; pair < pairs; ++pair) {
        const int n = (int)(pair / h_v);
        const int h = (int)(pair % h_v);
        const int g = h / group;                      /* query/key head shared by this value head */
        const long t0 = cu_seqlens ? cu_seqlens[n] : (long)n * (T_total / n_seq);
        const long t1 = cu_seqlens ? cu_seqlens[n + 1] : t0 + T_total / n_seq;

        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* r = (double*)malloc(sizeof(double) * (size_t)dv);
        if (!S || !r) {
            free(S);
            free(r);
            failed = 1;
            continue;
        }

        /* Initial state: S0 for this (sequence, head), else zero. */
        for (long i = 0; i < (long)dk * dv; ++i)
            S[i] = S0 ? (double)S0[((size_t)n * h_v + h) * dk * dv + i] : 0.0;

        for (long t = t0; t < t1; ++t) {
            const size_t qk_base = ((size_t)t * h_qk + g) * dk;   /* q, k    [t, g, :] */
            const size_t kd_base = ((size_t)t * h_v + h) * dk;    /* la, b   [t, h, :] */
            const size_t vd_base = ((size_t)t * h_v + h) * dv;    /* v, w, o [t, h, :] */

            /* decay: each key-channel row of S is scaled by alpha = exp(log_alpha) */
            for (int i = 0; i < dk; ++i) {
                const double alpha = exp((double)log_alpha[kd_base + i]);
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= alpha;
            }
            /* read with the key: r = S^T k */
            for (int j = 0; j < dv; ++j) r[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double ki = elem(k, qk_base + i, dtype);
                for (int j = 0; j < dv; ++j) r[j] += ki * S[(size_t)i * dv + j];
            }
            /* erase: S -= (b (.) k) r^T */
            for (int i = 0; i < dk; ++i) {
                const double ei = elem(b, kd_base + i, dtype) * elem(k, qk_base + i, dtype);
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] -= ei * r[j];
            }
            /* write: S += k (w (.) v)^T */
            for (int i = 0; i < dk; ++i) {
                const double ki = elem(k, qk_base + i, dtype);
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] +=
                        ki * (elem(w, vd_base + j, dtype) * elem(v, vd_base + j, dtype));
            }
            /* output: o = S^T q, read from the updated state */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i)
                    acc += elem(q, qk_base + i, dtype) * S[(size_t)i * dv + j];
                o[vd_base + j] = acc;
            }
        }

        if (S_T)
            memcpy(S_T + ((size_t)n * h_v + h) * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(r);
    }
    return failed ? GDN2_REF_ENOMEM : GDN2_REF_OK;
}
