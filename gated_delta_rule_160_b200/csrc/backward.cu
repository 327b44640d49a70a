// backward.cu -- gradients of the recurrence (gdn2_chunk_bwd).
//
// For each token, with e = b (.) k, x = w (.) v, S' = Diag(alpha) S_prev, r = S'^T k,
// S = S' - e r^T + k x^T, o = S^T q, and the adjoint dS of S (from later tokens and dS_T):
//   dS  += q dO^T                                   (o's contribution)
//   dx   = dS^T k,  dr = -dS^T e                    (column sums over key channels)
//   de   = -dS r,   dk = dS x + Diag(alpha) S_prev dr + de (.) b,   db = de (.) k
//   dS'  = dS + k dr^T
//   dalpha = rowsum(dS' (.) S_prev),  dlog_alpha = dalpha (.) alpha
//   dq   = S dO = Diag(alpha) S_prev dO - e (r . dO) + k (x . dO)
//   dw   = dx (.) v,  dv = dx (.) w,  and the adjoint of S_prev is Diag(alpha) dS'.
//
// Every value column of the state evolves on its own: the forward update and the adjoint of
// column m read only column m and the token's key-side vectors. So one CTA per (sequence,
// value head) gives each warp 8 value columns and keeps that dk x 8 slice of S_prev and of
// dS in registers (lane l holds key rows l, l + 32, ...): 16 warps for dv = 128, four per
// scheduler. Column sums (r, dx, dr) are a warp reduction; the per-row gradients (dq, dk,
// db, dlog_alpha) are sums over all columns, so each warp writes its partial row sums to
// shared memory and, after one barrier per token, the CTA adds the warps' partials and
// writes the outputs.
//
// Forward, then backward, over sub-chunks of kL tokens: a first pass stores the state at the
// start of every sub-chunk (checkpoints); then, from the last sub-chunk, the sub-chunk's states
// are recomputed from its checkpoint into a per-CTA scratch area (small enough to stay in L2)
// and its tokens are walked backwards. Each thread stores and reloads only its own slice of a
// state, in its own register order, so these copies need no synchronisation; the next token's
// S_prev is fetched with cp.async into shared memory while the current token is processed.
// A sub-chunk's inputs are staged in shared memory with cp.async (double-buffered) and then
// turned, once, into the fp32 operands every pass reads: alpha k, b k, k, alpha, q, b per key
// row and w v, dO per value column. A query/key head's dq, dk sum over the value heads that
// read it: with groups of several value heads they are accumulated with atomics into outputs
// the host zeroed first.
#include "internal.cuh"

namespace gdn2 {
namespace {

constexpr int kL = 8;        // tokens per sub-chunk (checkpoint interval)
constexpr int kMC = 8;       // value columns per warp
constexpr int kQ = kMC / 4;  // float4 per key row of a warp's slice

struct BwdParams {
    Params f;                // the forward's arguments
    const float* dO;         // [T, h_v, dv]
    const float* dS_T;       // nullable [N, h_v, dk, dv]
    float *dq, *dk, *dv, *dla, *db, *dw, *dS0;  // dS0 nullable
    float4* ckpt;            // [slots, h_v, dk * dv / 4]; slot = n + t0 / kL + sub-chunk
    float4* scratch;         // [N * h_v, kL - 1, dk * dv / 4]
    int atomic_qk;           // dq, dk accumulate (groups of value heads)
};

// kMC consecutive fp32 values (16-byte aligned); a warp reading one address broadcasts.
__device__ __forceinline__ void ldc(const float* p, float (&o)[kMC]) {
#pragma unroll
    for (int i = 0; i < kQ; ++i) {
        const float4 u = reinterpret_cast<const float4*>(p)[i];
        o[4 * i] = u.x; o[4 * i + 1] = u.y; o[4 * i + 2] = u.z; o[4 * i + 3] = u.w;
    }
}

// Sums of a[v][0..7] over the warp's 32 lanes, NV vectors at once: each of the first three
// steps hands half of the remaining columns to the partner lane (4 + 2 + 1 shuffles), two
// more add the partners that hold the same column, leaving in a[v][0] the full sum of
// column (lane >> 2).
template <int NV>
__device__ __forceinline__ void col_reduce(float (&a)[NV][kMC], int lane) {
#pragma unroll
    for (int st = 0; st < 3; ++st) {
        const int half = 4 >> st, xm = 16 >> st;
        const bool up = lane & xm;
#pragma unroll
        for (int v = 0; v < NV; ++v)
#pragma unroll
            for (int i = 0; i < half; ++i) {
                const float send = up ? a[v][i] : a[v][i + half];
                const float keep = up ? a[v][i + half] : a[v][i];
                a[v][i] = keep + __shfl_xor_sync(0xffffffffu, send, xm);
            }
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        a[v][0] += __shfl_xor_sync(0xffffffffu, a[v][0], 2);
        a[v][0] += __shfl_xor_sync(0xffffffffu, a[v][0], 1);
    }
}

template <int DK, int DV, typename T>
struct Cfg {
    static constexpr int NW = DV / kMC, NT = 32 * NW, RJ = DK / 32;
    static constexpr int ES = sizeof(T);
    // one token's raw inputs in shared memory: k, q, b, v, w (dtype), log_alpha, dO (fp32)
    static constexpr int OFF_K = 0, OFF_Q = DK * ES, OFF_B = 2 * DK * ES, OFF_V = 3 * DK * ES;
    static constexpr int OFF_W = OFF_V + DV * ES, OFF_LA = OFF_W + DV * ES, OFF_DO = OFF_LA + 4 * DK;
    static constexpr int REC = OFF_DO + 4 * DV;
    static constexpr int CK = DK * ES / 16, CV = DV * ES / 16, CLA = DK / 4, CDO = DV / 4;
    static constexpr int CPT = 3 * CK + 2 * CV + CLA + CDO;  // 16-byte pieces per token
    // one token's prepared fp32 operands: per key row {alpha k, b k, k, alpha} and {q, b};
    // per value column w v and dO
    static constexpr int PR_A = 0, PR_B = 16 * DK, PR_X = 24 * DK, PR_DO = PR_X + 4 * DV;
    static constexpr int PREC = PR_DO + 4 * DV;
    static constexpr int S4 = DK * DV / 4;                   // float4 per state
    // shared memory (bytes)
    static constexpr int SM_TOK = 0;                              // [2][kL][REC] raw inputs
    static constexpr int SM_PREP = SM_TOK + 2 * kL * REC;         // [kL][PREC] prepared operands
    static constexpr int SM_SP = SM_PREP + kL * PREC;             // [S4] float4: S_prev
    static constexpr int SM_PART = SM_SP + S4 * 16;               // [2][NW][4][DK] f32: row partials
    static constexpr int SM_COL = SM_PART + 2 * NW * 4 * DK * 4;  // [NW][2][kMC] f32: r, dr
    static constexpr int SM_R = SM_COL + NW * 2 * kMC * 4;        // [kL][DV] f32: r of each token
    static constexpr int SMEM = SM_R + kL * DV * 4;
};

// Queue (cp.async) the raw inputs of tokens [ts, ts + len) into a token buffer.
template <int DK, int DV, typename T>
__device__ void issue_tokens(const BwdParams& bp, uint8_t* dst, int ts, int len, int g, int h, bool with_dO) {
    using C = Cfg<DK, DV, T>;
    const Params& p = bp.f;
    const int total = len * C::CPT;
    for (int u = threadIdx.x; u < total; u += C::NT) {
        const int i = u / C::CPT, r = u - i * C::CPT;
        const size_t tok = (size_t)ts + i, rq = tok * p.h_qk + g, rv = tok * p.h_v + h;
        const char* src;
        if (r < 3 * C::CK) {
            const int seg = r / C::CK, off = r - seg * C::CK;
            const void* base = seg == 0 ? p.k : (seg == 1 ? p.q : p.b);
            src = static_cast<const char*>(base) + (seg < 2 ? rq : rv) * (DK * C::ES) + off * 16;
        } else if (r < 3 * C::CK + 2 * C::CV) {
            const int r2 = r - 3 * C::CK, seg = r2 / C::CV, off = r2 - seg * C::CV;
            src = static_cast<const char*>(seg == 0 ? p.v : p.w) + rv * (DV * C::ES) + off * 16;
        } else if (r < 3 * C::CK + 2 * C::CV + C::CLA) {
            src = reinterpret_cast<const char*>(p.log_alpha + rv * DK) + (r - 3 * C::CK - 2 * C::CV) * 16;
        } else {
            if (!with_dO) continue;
            src = reinterpret_cast<const char*>(bp.dO + rv * DV) + (r - 3 * C::CK - 2 * C::CV - C::CLA) * 16;
        }
        cp_async16(dst + i * C::REC + r * 16, src);
    }
}

// Raw inputs of len tokens -> their prepared fp32 operands (one exp per key row and token).
template <int DK, int DV, typename T>
__device__ void prepare(const uint8_t* raw, uint8_t* prep, int len, bool with_dO) {
    using C = Cfg<DK, DV, T>;
    for (int u = threadIdx.x; u < len * (DK + DV); u += C::NT) {
        const int i = u / (DK + DV), c = u - i * (DK + DV);
        const uint8_t* rec = raw + i * C::REC;
        uint8_t* pr = prep + i * C::PREC;
        if (c < DK) {
            const float k = to_f32(reinterpret_cast<const T*>(rec + C::OFF_K)[c]);
            const float q = to_f32(reinterpret_cast<const T*>(rec + C::OFF_Q)[c]);
            const float b = to_f32(reinterpret_cast<const T*>(rec + C::OFF_B)[c]);
            const float al = expf(reinterpret_cast<const float*>(rec + C::OFF_LA)[c]);
            reinterpret_cast<float4*>(pr + C::PR_A)[c] = make_float4(al * k, b * k, k, al);
            reinterpret_cast<float2*>(pr + C::PR_B)[c] = make_float2(q, b);
        } else {
            const int m = c - DK;
            const float v = to_f32(reinterpret_cast<const T*>(rec + C::OFF_V)[m]);
            const float w = to_f32(reinterpret_cast<const T*>(rec + C::OFF_W)[m]);
            reinterpret_cast<float*>(pr + C::PR_X)[m] = w * v;
            reinterpret_cast<float*>(pr + C::PR_DO)[m] =
                with_dO ? reinterpret_cast<const float*>(rec + C::OFF_DO)[m] : 0.f;
        }
    }
}

// One forward token on this thread's slice S (key rows lane + 32 j, the warp's kMC columns).
template <int DK, int DV, typename T>
__device__ __forceinline__ void fwd_step(float (&S)[DK / 32][kMC], const uint8_t* pr, float* col, int lane,
                                         int warp, float* rkeep = nullptr) {
    using C = Cfg<DK, DV, T>;
    const float4* A = reinterpret_cast<const float4*>(pr + C::PR_A);
    float4 rw[C::RJ];  // alpha k, e, k, alpha of this lane's rows
#pragma unroll
    for (int j = 0; j < C::RJ; ++j) rw[j] = A[lane + 32 * j];
    // column pairs (mm, mm + 1) in packed two-wide arithmetic
    float a[1][kMC];
#pragma unroll
    for (int pp = 0; pp < kMC / 2; ++pp) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < C::RJ; ++j) acc = ffma2(dup2(rw[j].x), make_float2(S[j][2 * pp], S[j][2 * pp + 1]), acc);
        a[0][2 * pp] = acc.x;
        a[0][2 * pp + 1] = acc.y;
    }
    col_reduce<1>(a, lane);
    __syncwarp();
    if (!(lane & 3)) {
        col[lane >> 2] = a[0][0];
        if (rkeep) rkeep[kMC * warp + (lane >> 2)] = a[0][0];  // the token's r, kept for its adjoint
    }
    __syncwarp();
    float r[kMC], x[kMC];
    ldc(col, r);
    ldc(reinterpret_cast<const float*>(pr + C::PR_X) + kMC * warp, x);
#pragma unroll
    for (int j = 0; j < C::RJ; ++j)
#pragma unroll
        for (int pp = 0; pp < kMC / 2; ++pp) {
            const float2 sj = fmul2(dup2(rw[j].w), make_float2(S[j][2 * pp], S[j][2 * pp + 1]));
            const float2 sn = ffma2(dup2(rw[j].z), make_float2(x[2 * pp], x[2 * pp + 1]),
                                    ffma2(dup2(-rw[j].y), make_float2(r[2 * pp], r[2 * pp + 1]), sj));
            S[j][2 * pp] = sn.x;
            S[j][2 * pp + 1] = sn.y;
        }
}

// A thread's slice of a state in its own order: float4 index of (row group j, column quad qq).
template <int DK>
__device__ __forceinline__ int sidx(int warp, int lane, int j, int qq) {
    return warp * (DK / 32) * kQ * 32 + (j * kQ + qq) * 32 + lane;
}
template <int DK>
__device__ __forceinline__ void put_slice(float4* dst, const float (&S)[DK / 32][kMC], int warp, int lane) {
#pragma unroll
    for (int j = 0; j < DK / 32; ++j)
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq)
            dst[sidx<DK>(warp, lane, j, qq)] =
                make_float4(S[j][4 * qq], S[j][4 * qq + 1], S[j][4 * qq + 2], S[j][4 * qq + 3]);
}
template <int DK>
__device__ __forceinline__ void get_slice(float (&S)[DK / 32][kMC], const float4* src, int warp, int lane) {
#pragma unroll
    for (int j = 0; j < DK / 32; ++j)
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq) {
            const float4 u = src[sidx<DK>(warp, lane, j, qq)];
            S[j][4 * qq] = u.x; S[j][4 * qq + 1] = u.y; S[j][4 * qq + 2] = u.z; S[j][4 * qq + 3] = u.w;
        }
}
template <int DK>
__device__ __forceinline__ void copy_slice_async(float4* dst, const float4* src, int warp, int lane) {
#pragma unroll
    for (int j = 0; j < DK / 32; ++j)
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq) {
            const int i = sidx<DK>(warp, lane, j, qq);
            cp_async16(dst + i, src + i);
        }
}
// The same slice in a [dk][dv] row-major state (S0, dS_T, dS0).
template <int DV>
__device__ __forceinline__ int gidx(int warp, int lane, int j, int qq) {
    return ((lane + 32 * j) * DV + kMC * warp + 4 * qq) / 4;
}
template <int DK, int DV>
__device__ __forceinline__ void load_rowmajor(float (&S)[DK / 32][kMC], const float* src, int warp, int lane) {
#pragma unroll
    for (int j = 0; j < DK / 32; ++j)
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq) {
            const float4 u = src ? reinterpret_cast<const float4*>(src)[gidx<DV>(warp, lane, j, qq)]
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            S[j][4 * qq] = u.x; S[j][4 * qq + 1] = u.y; S[j][4 * qq + 2] = u.z; S[j][4 * qq + 3] = u.w;
        }
}

template <int DK, int DV, typename T>
__global__ void __launch_bounds__(Cfg<DK, DV, T>::NT, 1) chunk_bwd_kernel(const __grid_constant__ BwdParams bp) {
    using C = Cfg<DK, DV, T>;
    constexpr int RJ = C::RJ;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* tok = smem + C::SM_TOK;
    uint8_t* prep = smem + C::SM_PREP;
    float4* spb = reinterpret_cast<float4*>(smem + C::SM_SP);
    float* part = reinterpret_cast<float*>(smem + C::SM_PART);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* col = reinterpret_cast<float*>(smem + C::SM_COL) + warp * 2 * kMC;  // r, dr of the warp's columns
    float* rkeep = reinterpret_cast<float*>(smem + C::SM_R);                    // [kL][DV]: r of each token

    const Params& p = bp.f;
    const int item = blockIdx.x;
    const int n = item / p.h_v, h = item % p.h_v, g = h / (p.h_v / p.h_qk);
    int t0, t1;
    seq_bounds(p, n, t0, t1);
    const int nsub = (t1 - t0 + kL - 1) / kL;
    const size_t soff = ((size_t)n * p.h_v + h) * DK * DV;
    const size_t slot0 = (size_t)n + t0 / kL;  // distinct per sub-chunk over all sequences
    auto ckpt = [&](int s) { return bp.ckpt + ((slot0 + s) * p.h_v + h) * C::S4; };
    auto scr = [&](int i) { return bp.scratch + ((size_t)item * (kL - 1) + i) * C::S4; };

    float S[RJ][kMC];
    load_rowmajor<DK, DV>(S, p.S0 ? p.S0 + soff : nullptr, warp, lane);

    // Phases k = 0 .. nsub-2 are the checkpointing pass over sub-chunks 0 .. nsub-2; phases
    // nsub-1 .. 2 nsub-2 are the backward over sub-chunks nsub-1 .. 0. Phase k's raw inputs
    // are in token buffer k & 1, queued during phase k - 1.
    const int K = nsub > 0 ? 2 * nsub - 1 : 0;
    auto sub_of = [&](int k) { return k < nsub - 1 ? k : 2 * (nsub - 1) - k; };
    auto queue = [&](int k) {
        const int s = sub_of(k), ts = t0 + s * kL;
        issue_tokens<DK, DV, T>(bp, tok + (k & 1) * kL * C::REC, ts, min(kL, t1 - ts), g, h, k >= nsub - 1);
    };
    // wait for phase k's inputs, queue phase k + 1's, prepare phase k's operands
    auto start_phase = [&](int k, int len, bool with_dO) {
        cp_async_wait_all();
        __syncthreads();
        if (k + 1 < K) queue(k + 1);
        cp_async_commit();
        prepare<DK, DV, T>(tok + (k & 1) * kL * C::REC, prep, len, with_dO);
        __syncthreads();
    };
    if (K > 0) queue(0);
    cp_async_commit();
    for (int k = 0; k + 1 < nsub; ++k) {
        start_phase(k, kL, false);
        put_slice<DK>(ckpt(k), S, warp, lane);
        for (int i = 0; i < kL; ++i) fwd_step<DK, DV, T>(S, prep + i * C::PREC, col, lane, warp);
    }
    if (nsub > 0) {
        put_slice<DK>(ckpt(nsub - 1), S, warp, lane);
        put_slice<DK>(spb, S, warp, lane);  // the last sub-chunk's start state
    }
    float dS[RJ][kMC];
    load_rowmajor<DK, DV>(dS, bp.dS_T ? bp.dS_T + soff : nullptr, warp, lane);
    int pb = 0;
    for (int k = max(nsub - 1, 0); k < K; ++k) {
        const int s = sub_of(k), ts = t0 + s * kL, len = min(kL, t1 - ts);
        start_phase(k, len, true);
        const uint8_t* tb = tok + (k & 1) * kL * C::REC;
        // ---- backward over sub-chunk s: its start state (in the S_prev buffer: put there
        // before this loop or fetched by the previous sub-chunk's last token); recompute the
        // states after tokens ts .. ts + len - 2 into scratch, the last of them straight
        // into the S_prev buffer for token ts + len - 1.
        get_slice<DK>(S, spb, warp, lane);
        for (int i = 0; i + 1 < len; ++i) {
            fwd_step<DK, DV, T>(S, prep + i * C::PREC, col, lane, warp, rkeep + i * DV);
            if (i + 2 < len) put_slice<DK>(scr(i), S, warp, lane);
        }
        put_slice<DK>(spb, S, warp, lane);
        {   // r of the last token, from its S_prev (in S now)
            const float4* A = reinterpret_cast<const float4*>(prep + (len - 1) * C::PREC + C::PR_A);
            float a[1][kMC];
#pragma unroll
            for (int pp = 0; pp < kMC / 2; ++pp) {
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < RJ; ++j)
                    acc = ffma2(dup2(A[lane + 32 * j].x), make_float2(S[j][2 * pp], S[j][2 * pp + 1]), acc);
                a[0][2 * pp] = acc.x;
                a[0][2 * pp + 1] = acc.y;
            }
            col_reduce<1>(a, lane);
            if (!(lane & 3)) rkeep[(len - 1) * DV + kMC * warp + (lane >> 2)] = a[0][0];
        }
        // S_prev of token ts + i (i < len - 1): the checkpoint for i = 0, else scratch state i - 1
        auto sprev = [&](int i) -> const float4* { return i == 0 ? ckpt(s) : scr(i - 1); };
        for (int i = len - 1; i >= 0; --i) {
            const uint8_t* pr = prep + i * C::PREC;
            const float4* A = reinterpret_cast<const float4*>(pr + C::PR_A);  // alpha k, e, k, alpha
            const float2* B = reinterpret_cast<const float2*>(pr + C::PR_B);  // q, b
            const size_t t = (size_t)ts + i;
            cp_async_wait_all();
            float SP[RJ][kMC];
            get_slice<DK>(SP, spb, warp, lane);
            float dO[kMC];
            ldc(reinterpret_cast<const float*>(pr + C::PR_DO) + kMC * warp, dO);
            // dS += q dO^T; column sums dx = dS^T k, dr = -dS^T e
            // (r = S'^T k of this token was kept by the recompute)
            float a[2][kMC];
            float4 rws[RJ];  // alpha k, e, k, alpha of this lane's rows, for both loops
#pragma unroll
            for (int j = 0; j < RJ; ++j) rws[j] = A[lane + 32 * j];
            {
                float2 acc[2][kMC / 2];
#pragma unroll
                for (int pp = 0; pp < kMC / 2; ++pp) acc[0][pp] = acc[1][pp] = make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < RJ; ++j) {
                    const float4 rw = rws[j];
                    const float2 qj = dup2(B[lane + 32 * j].x), kk = dup2(rw.z), ne = dup2(-rw.y);
#pragma unroll
                    for (int pp = 0; pp < kMC / 2; ++pp) {
                        const float2 d = ffma2(qj, make_float2(dO[2 * pp], dO[2 * pp + 1]),
                                               make_float2(dS[j][2 * pp], dS[j][2 * pp + 1]));
                        dS[j][2 * pp] = d.x;
                        dS[j][2 * pp + 1] = d.y;
                        acc[0][pp] = ffma2(kk, d, acc[0][pp]);
                        acc[1][pp] = ffma2(ne, d, acc[1][pp]);
                    }
                }
#pragma unroll
                for (int v = 0; v < 2; ++v)
#pragma unroll
                    for (int pp = 0; pp < kMC / 2; ++pp) {
                        a[v][2 * pp] = acc[v][pp].x;
                        a[v][2 * pp + 1] = acc[v][pp].y;
                    }
            }
            // every S_prev value has been consumed: fetch the next token's into the buffer
            if (i > 0) copy_slice_async<DK>(spb, sprev(i - 1), warp, lane);
            else if (s > 0) copy_slice_async<DK>(spb, ckpt(s - 1), warp, lane);
            cp_async_commit();
            col_reduce<2>(a, lane);
            __syncwarp();
            if (!(lane & 3)) {
                const int mc = lane >> 2, m = kMC * warp + mc;
                col[kMC + mc] = a[1][0];
                const size_t tv = t * p.h_v + h;
                bp.dw[tv * DV + m] = a[0][0] * to_f32(reinterpret_cast<const T*>(tb + i * C::REC + C::OFF_V)[m]);
                bp.dv[tv * DV + m] = a[0][0] * to_f32(reinterpret_cast<const T*>(tb + i * C::REC + C::OFF_W)[m]);
            }
            __syncwarp();
            float r[kMC], dr[kMC], x[kMC];
            ldc(rkeep + i * DV + kMC * warp, r);
            ldc(col + kMC, dr);
            ldc(reinterpret_cast<const float*>(pr + C::PR_X) + kMC * warp, x);
            float rdo = 0.f, xdo = 0.f;
#pragma unroll
            for (int mm = 0; mm < kMC; ++mm) {
                rdo = fmaf(r[mm], dO[mm], rdo);
                xdo = fmaf(x[mm], dO[mm], xdo);
            }
            // row sums over the warp's columns; dS <- Diag(alpha) (dS + k dr^T)
            float* pw = part + ((size_t)pb * C::NW + warp) * 4 * DK;
#pragma unroll
            for (int j = 0; j < RJ; ++j) {
                const float4 rw = rws[j];
                const float bj = B[lane + 32 * j].y;
                const float2 kk = dup2(rw.z), al = dup2(rw.w);
                float2 pde2 = make_float2(0.f, 0.f), pdk2 = pde2, pdr2 = pde2, pda2 = pde2, psd2 = pde2;
#pragma unroll
                for (int pp = 0; pp < kMC / 2; ++pp) {
                    const float2 d = make_float2(dS[j][2 * pp], dS[j][2 * pp + 1]);
                    const float2 sp = make_float2(SP[j][2 * pp], SP[j][2 * pp + 1]);
                    const float2 dr2 = make_float2(dr[2 * pp], dr[2 * pp + 1]);
                    const float2 dsp = ffma2(kk, dr2, d);
                    pde2 = ffma2(d, make_float2(r[2 * pp], r[2 * pp + 1]), pde2);
                    pdk2 = ffma2(d, make_float2(x[2 * pp], x[2 * pp + 1]), pdk2);
                    pdr2 = ffma2(sp, dr2, pdr2);
                    pda2 = ffma2(dsp, sp, pda2);
                    psd2 = ffma2(sp, make_float2(dO[2 * pp], dO[2 * pp + 1]), psd2);
                    const float2 nd = fmul2(al, dsp);
                    dS[j][2 * pp] = nd.x;
                    dS[j][2 * pp + 1] = nd.y;
                }
                const float pde = pde2.x + pde2.y, pdk = pdk2.x + pdk2.y, pdr = pdr2.x + pdr2.y;
                const float pda = pda2.x + pda2.y, psd = psd2.x + psd2.y;
                const int c = lane + 32 * j;
                pw[c] = fmaf(rw.w, psd, fmaf(-rw.y, rdo, rw.z * xdo));  // dq
                pw[DK + c] = fmaf(rw.w, pdr, fmaf(-bj, pde, pdk));      // dk
                pw[2 * DK + c] = -rw.z * pde;                            // db
                pw[3 * DK + c] = rw.w * pda;                             // dlog_alpha
            }
            __syncthreads();
            const float* pr_sum = part + (size_t)pb * C::NW * 4 * DK;
            for (int o = threadIdx.x; o < 4 * DK; o += C::NT) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < C::NW; ++w) sum += pr_sum[w * 4 * DK + o];
                const int which = o / DK, c = o - which * DK;
                const size_t iq = (t * p.h_qk + g) * DK + c, iv = (t * p.h_v + h) * DK + c;
                if (which == 0) {
                    if (bp.atomic_qk) atomicAdd(bp.dq + iq, sum); else bp.dq[iq] = sum;
                } else if (which == 1) {
                    if (bp.atomic_qk) atomicAdd(bp.dk + iq, sum); else bp.dk[iq] = sum;
                } else if (which == 2) {
                    bp.db[iv] = sum;
                } else {
                    bp.dla[iv] = sum;
                }
            }
            pb ^= 1;
        }
    }
    cp_async_wait_all();
    if (bp.dS0) {
        float4* dst = reinterpret_cast<float4*>(bp.dS0 + soff);
#pragma unroll
        for (int j = 0; j < RJ; ++j)
#pragma unroll
            for (int qq = 0; qq < kQ; ++qq)
                dst[gidx<DV>(warp, lane, j, qq)] =
                    make_float4(dS[j][4 * qq], dS[j][4 * qq + 1], dS[j][4 * qq + 2], dS[j][4 * qq + 3]);
    }
}

template <int DK, int DV, typename T>
cudaError_t launch_bwd_t(const BwdParams& bp, cudaStream_t s) {
    using C = Cfg<DK, DV, T>;
    static_assert(C::SMEM <= 227 * 1024, "backward shared memory");
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<DK, DV, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    chunk_bwd_kernel<DK, DV, T><<<bp.f.n_seq * bp.f.h_v, C::NT, C::SMEM, s>>>(bp);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bwd_d(const BwdParams& bp, cudaStream_t s) {
    if (bp.f.dk == 128) return bp.f.dv == 128 ? launch_bwd_t<128, 128, T>(bp, s) : launch_bwd_t<128, 64, T>(bp, s);
    return bp.f.dv == 128 ? launch_bwd_t<64, 128, T>(bp, s) : launch_bwd_t<64, 64, T>(bp, s);
}

// Checkpoint slots: n + t0 / kL + s is below this for every sub-chunk s of every sequence n.
size_t ckpt_slots(int T_total, int n_seq) { return (size_t)(T_total + kL - 1) / kL + (size_t)n_seq; }

}  // namespace

size_t bwd_workspace_bytes(const gdn2_shape* sh) {
    const size_t SZ = (size_t)sh->dk * sh->dv * sizeof(float);
    return ckpt_slots(sh->T_total, sh->n_seq) * sh->h_v * SZ + (size_t)sh->n_seq * sh->h_v * (kL - 1) * SZ;
}

cudaError_t launch_bwd(const Params& p, gdn2_dtype dt, const float* dO, const float* dS_T, float* dq, float* dk,
                       float* dv, float* dla, float* db, float* dw, float* dS0, void* workspace, cudaStream_t s) {
    BwdParams bp{};
    bp.f = p;
    bp.dO = dO; bp.dS_T = dS_T;
    bp.dq = dq; bp.dk = dk; bp.dv = dv; bp.dla = dla; bp.db = db; bp.dw = dw; bp.dS0 = dS0;
    const size_t S4 = (size_t)p.dk * p.dv / 4;
    bp.ckpt = static_cast<float4*>(workspace);
    bp.scratch = bp.ckpt + ckpt_slots(p.T_total, p.n_seq) * p.h_v * S4;
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
