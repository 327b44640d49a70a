// chunk_tc.cu -- chunkwise-parallel prefill on the tcgen05 tensor cores (bf16 inputs,
// dk = dv = 128, chunks of C = 64 tokens). One CTA owns one (sequence, value head) and
// walks its chunks in order; the fp32 state lives in tensor memory.
//
// Chunk algebra (per chunk, state S on entry; e = b(.)k, x = w(.)v, G = inclusive cumsum
// of log_alpha over the chunk, per key channel). Every decayed operand is taken relative
// to a per-channel reference Gref = (G_first + G_last) / 2, so that the factors
// exp(+-(G - Gref)) stay within about e^+-(half the chunk's decay):
//   Kh = K exp(G-Gref)   Qh = Q exp(G-Gref)   Kb = K exp(Gref-G)   Eb = E exp(Gref-G)
//   Gram:  B_ij = Kh_i.Kb_j (j<i)  A_ij = Kh_i.Eb_j (j<i)  P_ij = Qh_i.Kb_j (j<=i)
//          Qm_ij = Qh_i.Eb_j (j<=i)
//   T = (I + A)^-1                                  (the gated UT transform)
//   Y = Kh Sref + B X,  R = T Y                     (key reads of the decayed old state)
//   O = Qh Sref + P X - Qm R                        (query reads of the updated state)
//   U = Sref + Kb^T X - Eb^T R,   S' = exp(G_last - Gref) (.) U
// with Sref = exp(Gref) (.) S. Everything runs transposed (value channel m = row = tensor
// memory lane) so that every MMA has M = 128.
//
// Precision: bf16 operands round to 8 significant bits, and the outputs of this
// recurrence have max|o| / rms(o) of 10 to 15, so one rounding on a dominant term costs
// more than the 2e-2 * rms(o) error budget. The terms that carry the output and the
// state -- P (query/key Gram block), P X, Kb^T X and Qh Sref -- are therefore computed with
// both operands split into bf16 hi + lo parts (three MMAs: hi*hi + lo*hi + hi*lo, about 16
// significant bits); the erase path (A, B, Qm, T, Y, R) stays in plain bf16. (Qh Sref
// carries the whole output when the state dominates it: a long history, a large S0.)
//
// Phases per chunk. Sixteen SIMT warps take part in each (thread t serves tensor-memory
// lane t % 128 and column quarter t / 128): the phases are chains of dependent
// shared-memory, tensor-memory and special-function operations, and four warps per
// scheduler hide their latency where two did not. A seventeenth warp only issues the MMA
// groups, each as soon as the SIMT warps signal that its operands are written, so no SIMT
// warp waits behind the tensor pipe; an eighteenth issues the TMA loads of the next chunk's
// raw rows as soon as their space is free. Work that does not need the state is placed
// under the MMAs that do:
//   1 prep    q, k, b rows (staged by TMA) -> Kh, Qh hi/lo, Kb hi/lo, Eb tiles; MMA Gram
//   2 X = w (.) v tiles and the state epilogue (U <- f (.) U, Sref^T bf16 hi / lo into
//     tensor memory), both under the Gram MMAs; MMAs Y^T = Sref^T Kh^T,
//     O^T = Sref^T Qh^T (hi / lo), U += X^T Kb (hi / lo)
//   3 Gram epilogue (B, A, Qm); MMA Y^T += X^T B^T
//   4 UT solve T = (I + A)^-1 (16 -> 32 -> 64), the P block (after its cross terms) beside
//     its first level; MMA O^T += X^T P^T
//   5 Y^T (bf16, tensor memory); MMA R^T = Y^T T^T
//   6 -R^T (bf16, tensor memory); MMAs O^T -= R^T Qm^T, U -= R^T Eb
//   7 under those MMAs: the next chunk's cumulative log-decays and frame factors
//   8 o epilogue (full fp32 chunks: staged in the X tiles, TMA-stored in the next chunk's
//     prep; else plain stores)
// Sref^T, Y^T and -R^T are A operands read from tensor memory; the others come from shared
// memory.
// The next chunk's raw rows are staged by TMA (and prefetched into L2 one chunk earlier)
// while the current one is processed.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "tc_ptx.cuh"

namespace gdn2 {
namespace {

using namespace tc;

constexpr int CH = 64;   // chunk length
constexpr int D = 128;   // dk = dv
constexpr int NS = 512;           // SIMT threads (warps 0..15): prep, epilogues, solve
constexpr int kIssuer = NS / 32;       // warp 16 issues every MMA
constexpr int kProducer = kIssuer + 1;  // warp 17 issues every TMA load of raw chunk rows
constexpr int NT = NS + 64;             // threads per CTA
constexpr float kLog2e = 1.4426950408889634f;  // cumulative log-decays are kept in base 2
// Largest |G - Gref| (base 2) for which the decay factors, times operands of order one and
// the state's own scale, stay inside fp32's normal range with margin: a chunk whose
// cumulative log-decay varies more than that on some channel is flagged (kStatusDecayRange)
constexpr float kMaxFactorExp2 = 120.f;

// ---- shared memory map (bytes). Tiles written by the prep are token-major, K-major, with
// row groups outermost (LBO = 128 B, SBO = 2048 B): element (row r, channel c) at
//   (r/8)*2048 + (c/8)*128 + (r%8)*16 + (c%8)*2.
constexpr uint32_t kTile = CH * D * 2;   // 16384
constexpr uint32_t OFF_KH = 0;           // Kh      } rows 0..127 of the Gram B operand
constexpr uint32_t OFF_QH = 1 * kTile;   // Qh hi   }
constexpr uint32_t OFF_QL = 2 * kTile;   // Qh lo
constexpr uint32_t OFF_KBH = 3 * kTile;  // Kb hi   } rows 0..127 of the Gram A operand
constexpr uint32_t OFF_E = 4 * kTile;    // Eb      }
constexpr uint32_t OFF_KBL = 5 * kTile;  // Kb lo   (rows 64..127 of its operand are masked out)
constexpr uint32_t OFF_XH = 6 * kTile;   // X hi
constexpr uint32_t OFF_XL = 7 * kTile;   // X lo
// Raw chunk inputs, copied by TMA in boxes of 64 tokens x 128 bytes (64 bf16 or 32 fp32
// channels) with the 128-byte swizzle: within each 8-row group the 16-byte chunk c of
// row r sits at chunk c ^ (r % 8), so the prep's reads (8 rows, same columns) hit distinct
// banks. A bf16 [64][128] tile is 2 boxes (8 KB each), an fp32 one 4 boxes.
//   group A: log_alpha, v, w -> the reused region, free once the previous chunk's
//            X^T P^T MMAs are done;
//   group B: q, k, b         -> over Kh / Qh / Ql, free once its state read is done.
constexpr uint32_t OFF_RAW_Q = 0;            // bf16, 16 KB each
constexpr uint32_t OFF_RAW_K = 1 * kTile;
constexpr uint32_t OFF_RAW_B = 2 * kTile;
// The o tile of a full chunk is staged as fp32 [32 tokens][128 channels] halves over X hi
// and X lo (free once the X^T Kb, X^T B^T and X^T P^T MMAs are done; rewritten after the
// next chunk's Gram has been issued) and written by two TMA stores.
constexpr uint32_t OFF_OST0 = OFF_XH;        // tokens 0..31, fp32, 16 KB
constexpr uint32_t OFF_OST1 = OFF_XL;        // tokens 32..63
// [64][64] bf16 tiles. MN-major B operands B[n=i][k=j] written by the Gram epilogue:
//   (i/8)*1024 + (j/8)*128 + (j%8)*16 + (i%8)*2     (SBO = 1024, LBO = 128)
constexpr uint32_t kSmall = CH * CH * 2;  // 8192
constexpr uint32_t OFF_QM = 8 * kTile;     // Qm
constexpr uint32_t OFF_T = OFF_QM + kSmall;  // T, K-major [i][j]: (j/8)*1024 + (i/8)*128 + (i%8)*16 + (j%8)*2
constexpr uint32_t OFF_REG = OFF_T + kSmall;  // 64 KB reused by phases 3 / 5-6 / 7-10
constexpr uint32_t OFF_B = OFF_REG;             // B
constexpr uint32_t OFF_PH = OFF_REG + kSmall;   // P hi
constexpr uint32_t OFF_PL = OFF_REG + 2 * kSmall;
constexpr int WS = 68;                                // fp32 row stride (16-byte aligned rows)
constexpr uint32_t OFF_WA = OFF_REG + 3 * kSmall;      // fp32 A [64][WS]
constexpr uint32_t OFF_WT = OFF_WA + 64 * WS * 4;     // fp32 T [64][WS]
constexpr uint32_t OFF_WM = OFF_WT + 64 * WS * 4;     // fp32 scratch [32][33]
constexpr uint32_t OFF_RAW_LA = OFF_REG;              // fp32, 32 KB  (group A)
constexpr uint32_t OFF_RAW_A = OFF_REG + kTile;       // bf16 decay pre-activations (fused pre-processing)
constexpr uint32_t OFF_RAW_V = OFF_REG + 2 * kTile;   // bf16, 16 KB
constexpr uint32_t OFF_RAW_W = OFF_REG + 3 * kTile;   // bf16, 16 KB
// float gref[2][128], glast[2][128], frame factors f[2][128], quarter-chunk log-decay
// totals [4][128]
constexpr uint32_t OFF_SCAL = OFF_REG + 4 * kTile;
constexpr uint32_t OFF_MBAR = OFF_SCAL + 10 * 128 * 4;
constexpr uint32_t OFF_TSLOT = OFF_MBAR + 24 * 8;  // tensor-memory base; +4: decay-range flag
// fused pre-processing: 1 / max(|q|, eps) of the chunk's tokens at [0, 64), of k at [64, 128)
constexpr uint32_t OFF_RN = OFF_TSLOT + 16;
constexpr uint32_t SMEM_BYTES = OFF_RN + 128 * 4;
static_assert(OFF_WM + 32 * 33 * 4 <= OFF_REG + 4 * kTile, "solve workspace overflows its region");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- tensor memory columns
constexpr uint32_t TM_G = 0;     // Gram (transposed): lanes [Kb j ; Eb j], cols [Kh i ; Qh i]
constexpr uint32_t TM_D1 = 128;  // [Y^T | O^T]
constexpr uint32_t TM_R = 256;   // R^T
constexpr uint32_t TM_U = 384;   // state, lanes m (value channel), cols c (key channel)
constexpr uint32_t TM_S = 320;   // Sref^T hi as a bf16 A operand (packed pairs), 64 columns
// Sref^T lo, over the R^T columns: R^T of the previous chunk is dead once its U -= R^T Eb
// MMAs are done (before the state epilogue writes this), and R^T of this chunk is written
// after the Sref MMAs are done
constexpr uint32_t TM_SL = TM_R;
// Y^T and -R^T also serve as bf16 A operands from tensor memory, packed over the first 32
// columns of their own fp32 accumulators (TM_D1, TM_R).

// MB_*: MMA groups done (committed by the issuer warp) and raw rows landed (TMA);
// RDY_*: operands of an MMA group written (one arrival from the SIMT warps).
// RDY_RAWA: the SIMT warps are done with the region that the next log_alpha / v / w rows
// land in.
enum {
    MB_G = 0, MB_2B, MB_2A, MB_2P, MB_3, MB_45O, MB_45, MB_RAWA, MB_RAWB, MB_GX,
    RDY_G, RDY_2B, RDY_2A, RDY_2P, RDY_3, RDY_45, RDY_RAWA, kNumMbar
};
static_assert(kNumMbar <= 24, "mbarrier slots");

// Tensor maps of the six per-token inputs: 3-d {channel, head, token}, 128-byte boxes of
// 64 tokens with the 128-byte swizzle.
struct RawMaps {
    CUtensorMap la, q, k, b, v, w;
    CUtensorMap o;  // fp32 output, used for full chunks (box {128, 1, 32}, no swizzle)
};

// Device status word of this file's kernels (kStatus* bits), read and cleared by
// gdn2_device_status.
__device__ unsigned int g_status_tc = 0;

__device__ __forceinline__ uint32_t off_rowmajor(int r, int c) {  // prep tiles, 128 channels
    return (uint32_t)((r >> 3) * 2048 + (c >> 3) * 128 + (r & 7) * 16 + (c & 7) * 2);
}

// Byte offsets of (token i, channel c) in the swizzled raw tiles (see the map above).
__device__ __forceinline__ uint32_t raw_off_bf16(int i, int c) {
    return (uint32_t)((c >> 6) * 8192 + i * 128 + ((((c & 63) >> 3) ^ (i & 7)) << 4) + (c & 7) * 2);
}
__device__ __forceinline__ uint32_t raw_off_f32(int i, int c) {
    return (uint32_t)((c >> 5) * 8192 + i * 128 + ((((c & 31) >> 2) ^ (i & 7)) << 4) + (c & 3) * 4);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// Split 2 fp32 values into bf16 hi (packed) and bf16 lo = x - hi (packed): hi + lo carries
// about 16 significant bits.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(a, b);
    // a - hi(a), b - hi(b) in one packed FMA; both differences are exact in fp32
    const float2 r = ffma2(make_float2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u)),
                           make_float2(-1.f, -1.f), make_float2(a, b));
    lo = pack_bf16(r.x, r.y);
}

// 4 consecutive bf16 values (8 bytes) widened to fp32.
__device__ __forceinline__ void unpack4_bf16(uint2 u, float (&f)[4]) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x), b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    f[0] = __low2float(a);
    f[1] = __high2float(a);
    f[2] = __low2float(b);
    f[3] = __high2float(b);
}

__device__ __forceinline__ void store4_bf16(uint8_t* smem, uint32_t off, const float (&f)[4]) {
    *reinterpret_cast<uint2*>(smem + off) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
}

// 8 fp32 values as 8 bf16 in one 16-byte shared store.
__device__ __forceinline__ void store8_bf16(uint8_t* smem, uint32_t off, const float* f) {
    *reinterpret_cast<uint4*>(smem + off) =
        make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}

template <typename TO>
constexpr bool kTmaStoreO = sizeof(TO) == 4;  // the o tensor map is fp32

// ---- token-by-token recomputation of one (sequence, value head)
// A CTA whose decay left the chunk frame's range (kMaxFactorExp2) finishes its chunk walk
// (results unusable, S_T not written) and then runs the recurrence itself over the whole
// sequence in fp32, from S0, overwriting that pair's o and writing S_T: per token, decay
// the state by alpha, read r = S'^T k and p = S'^T q, edit S = S' - (b k) r^T + k (w v)^T,
// and emit o = p - (q.(b k)) r + (q.k) (w v), which is the updated state's read by q.
// The 512 SIMT threads hold the state in registers: warp w takes value column
// 32 (w / 4) + lane and key rows 32 (w % 4) .. + 31; the four partial reads of a column
// are added through shared memory after one barrier per token. Inputs are staged 16
// tokens at a time in shared memory as fp32, with the fused pre-processing applied for
// kPro (L2 norms of q and k, alpha = e^(-softplus(a)) = sigmoid(-a), sigmoid gates).
constexpr int kRedoStage = 16;
struct RedoSmem {
    float k[kRedoStage][D];
    float q[kRedoStage][D];
    float a[kRedoStage][D];  // alpha
    float e[kRedoStage][D];  // b (.) k
    float x[kRedoStage][D];  // w (.) v
    float qe[kRedoStage];    // q . (b (.) k)
    float qk[kRedoStage];    // q . k
    float red[2][2][4][D];   // [token parity][r | p][row quarter][value column]
};
static_assert(sizeof(RedoSmem) <= OFF_MBAR, "recomputation staging overlaps the barriers");

template <typename TO, bool kPro>
__device__ __forceinline__ void redo_tokens(const Params& p, int h, int g, int t0, int t1, size_t soff,
                                         uint8_t* smem_raw, int tid) {
    RedoSmem& sm = *reinterpret_cast<RedoSmem*>(smem_raw);
    const int warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3;
    const int col = 32 * (warp >> 2) + lane;
    const int row0 = 32 * quarter;
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(p.q);
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(p.k);
    const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(p.v);
    const __nv_bfloat16* bp = static_cast<const __nv_bfloat16*>(p.b);
    const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(p.w);
    const __nv_bfloat16* ap = static_cast<const __nv_bfloat16*>(p.a_raw);
    TO* op = static_cast<TO*>(p.o);

    float s[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) s[i] = p.S0 ? p.S0[soff + (size_t)(row0 + i) * D + col] : 0.f;

    for (int base = t0; base < t1; base += kRedoStage) {
        const int nt = min(kRedoStage, t1 - base);
        bar_sync_1<NS>();  // the previous stage is consumed
        for (int idx = tid; idx < nt * D; idx += NS) {
            const int tt = idx / D, c = idx % D;
            const size_t t = (size_t)(base + tt);
            const size_t oqk = (t * p.h_qk + g) * D + c, ov = (t * p.h_v + h) * D + c;
            float bv = to_f32(bp[ov]), wv = to_f32(wp[ov]);
            float av;
            if (kPro) {
                av = sigmoid_f(-to_f32(ap[ov]));
                bv = sigmoid_f(bv);
                wv = sigmoid_f(wv);
            } else {
                av = expf(p.log_alpha[ov]);
            }
            sm.k[tt][c] = to_f32(kp[oqk]);
            sm.q[tt][c] = to_f32(qp[oqk]);
            sm.a[tt][c] = av;
            sm.e[tt][c] = bv;  // times k below
            sm.x[tt][c] = wv * to_f32(vp[ov]);
        }
        bar_sync_1<NS>();
        if (warp < nt) {  // warp tt: q and k normalised (kPro), b (.) k, q . e and q . k
            const int tt = warp;
            float kv[4], qv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kv[j] = sm.k[tt][lane + 32 * j];
                qv[j] = sm.q[tt][lane + 32 * j];
            }
            if (kPro) {
                float sk = 0.f, sq = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sk = fmaf(kv[j], kv[j], sk);
                    sq = fmaf(qv[j], qv[j], sq);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, o);
                    sq += __shfl_xor_sync(0xffffffffu, sq, o);
                }
                const float rk = rsqrtf(fmaxf(sk, kL2NormEps * kL2NormEps));
                const float rq = rsqrtf(fmaxf(sq, kL2NormEps * kL2NormEps));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    kv[j] *= rk;
                    qv[j] *= rq;
                    sm.k[tt][lane + 32 * j] = kv[j];
                    sm.q[tt][lane + 32 * j] = qv[j];
                }
            }
            float d1 = 0.f, d2 = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float e = sm.e[tt][lane + 32 * j] * kv[j];
                sm.e[tt][lane + 32 * j] = e;
                d1 = fmaf(qv[j], e, d1);
                d2 = fmaf(qv[j], kv[j], d2);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                d1 += __shfl_xor_sync(0xffffffffu, d1, o);
                d2 += __shfl_xor_sync(0xffffffffu, d2, o);
            }
            if (lane == 0) {
                sm.qe[tt] = d1;
                sm.qk[tt] = d2;
            }
        }
        bar_sync_1<NS>();
        for (int tt = 0; tt < nt; ++tt) {
            float r = 0.f, pq = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s[i] *= sm.a[tt][row0 + i];
                r = fmaf(sm.k[tt][row0 + i], s[i], r);
                pq = fmaf(sm.q[tt][row0 + i], s[i], pq);
            }
            const int par = tt & 1;
            sm.red[par][0][quarter][col] = r;
            sm.red[par][1][quarter][col] = pq;
            bar_sync_1<NS>();  // (a buffer is rewritten two tokens later, after the next barrier)
            r = 0.f;
            pq = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                r += sm.red[par][0][w][col];
                pq += sm.red[par][1][w][col];
            }
            const float x = sm.x[tt][col];
#pragma unroll
            for (int i = 0; i < 32; ++i) s[i] = fmaf(sm.k[tt][row0 + i], x, fmaf(-sm.e[tt][row0 + i], r, s[i]));
            if (quarter == (tt & 3))
                op[((size_t)(base + tt) * p.h_v + h) * D + col] = from_f32<TO>(pq - sm.qe[tt] * r + sm.qk[tt] * x);
        }
    }
    if (p.S_T) {
#pragma unroll
        for (int i = 0; i < 32; ++i) p.S_T[soff + (size_t)(row0 + i) * D + col] = s[i];
    }
}

// kPro: fused pre-processing. The raw q, k are L2-normalised per token (norms over the 128
// channels, reduced across the eight warps of a token through shared memory), log_alpha is
// -softplus of the bf16 decay pre-activation (staged as a bf16 tile beside the cumulative
// decay), b and w are sigmoids of their raw values.
template <typename TO, bool kPro>
__global__ void __launch_bounds__(NT, 1) chunk_tc_kernel(const __grid_constant__ Params p,
                                                          const __grid_constant__ RawMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int L = tid & 127;   // tensor-memory lane served by this thread
    const int cp = tid >> 7;   // column quarter (SIMT threads)
    const uint32_t sbase = smem_u32(smem);
    const uint32_t lane_bits = (uint32_t)(L & 96) << 16;
    float* scal = reinterpret_cast<float*>(smem + OFF_SCAL);  // [0..255] gref, [256..511] glast (base 2)
    float* fscal = scal + 512;  // [2][128] state frame factors (applied one after the other)
    float* qtot = scal + 768;  // [4][128] sums of log_alpha over tokens 16q .. 16q + 15
    float* WA = reinterpret_cast<float*>(smem + OFF_WA);
    float* WT = reinterpret_cast<float*>(smem + OFF_WT);
    float* WM = reinterpret_cast<float*>(smem + OFF_WM);
    const uint32_t mbar0 = sbase + OFF_MBAR;
    auto mbar = [&](int i) { return mbar0 + 8u * (uint32_t)i; };

    const int item = blockIdx.x;
    const int n = p.order ? p.order[item / p.h_v] : item / p.h_v;
    const int h = item % p.h_v;
    if ((unsigned)n >= (unsigned)p.n_seq) {  // a stale order entry: skip the item, touch nothing
        if (tid == 0) atomicOr(&g_status_tc, kStatusBadOrder);
        return;
    }
    const uint64_t kWaitNs = p.wait_ns;
    const int g = h / (p.h_v / p.h_qk);
    int t0, t1;
    seq_bounds(p, n, t0, t1);
    const int nchunks = (t1 - t0 + CH - 1) / CH;
    const size_t soff = ((size_t)n * p.h_v + h) * D * D;

    TO* op = static_cast<TO*>(p.o);

    if (nchunks == 0) {  // empty sequence: S_T = S0
        if (p.S_T)
            for (int i = tid; i < D * D; i += NT) p.S_T[soff + i] = p.S0 ? p.S0[soff + i] : 0.f;
        return;
    }

    if (tid == 0) {
        for (int i = 0; i < kNumMbar; ++i) mbar_init(mbar(i), 1);
        fence_mbar_init();
        *reinterpret_cast<uint32_t*>(smem + OFF_TSLOT + 4) = 0u;
    }
    if (warp == 0) tmem_alloc(sbase + OFF_TSLOT, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TSLOT);
    bool fault = false;

    // prep mapping: warp w owns channels [16(w % 8), +16) and tokens [32 th, +32) with
    // th = w / 8; lane = (channel quad, token in a block of 8)
    const int th = (warp >> 3) & 1;
    const int ti0 = 32 * th + (lane & 7);
    const int c0 = 16 * (warp & 7) + 4 * (lane >> 3);

    // raw inputs of a chunk in two groups, each issued as soon as its space frees up
    auto issue_raw_a = [&](int ts) {  // log_alpha (or its bf16 pre-activation), v, w
        mbar_expect_tx(mbar(MB_RAWA), kPro ? 3 * kTile : 4 * kTile);
        if (kPro) {
#pragma unroll
            for (int x = 0; x < 2; ++x)
                tma_load_3d(sbase + OFF_RAW_A + x * 8192, &maps.la, 64 * x, h, ts, mbar(MB_RAWA));
        } else {
#pragma unroll
            for (int x = 0; x < 4; ++x)
                tma_load_3d(sbase + OFF_RAW_LA + x * 8192, &maps.la, 32 * x, h, ts, mbar(MB_RAWA));
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_load_3d(sbase + OFF_RAW_V + x * 8192, &maps.v, 64 * x, h, ts, mbar(MB_RAWA));
            tma_load_3d(sbase + OFF_RAW_W + x * 8192, &maps.w, 64 * x, h, ts, mbar(MB_RAWA));
        }
    };
    auto issue_raw_b = [&](int ts) {  // q, k, b
        mbar_expect_tx(mbar(MB_RAWB), 3 * kTile);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_load_3d(sbase + OFF_RAW_Q + x * 8192, &maps.q, 64 * x, g, ts, mbar(MB_RAWB));
            tma_load_3d(sbase + OFF_RAW_K + x * 8192, &maps.k, 64 * x, g, ts, mbar(MB_RAWB));
            tma_load_3d(sbase + OFF_RAW_B + x * 8192, &maps.b, 64 * x, h, ts, mbar(MB_RAWB));
        }
    };
    auto prefetch_raw = [&](int ts) {  // every raw row of the chunk at token ts, into L2
#pragma unroll
        for (int x = 0; x < (kPro ? 2 : 4); ++x) tma_prefetch_3d(&maps.la, (kPro ? 64 : 32) * x, h, ts);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            tma_prefetch_3d(&maps.q, 64 * x, g, ts);
            tma_prefetch_3d(&maps.k, 64 * x, g, ts);
            tma_prefetch_3d(&maps.b, 64 * x, h, ts);
            tma_prefetch_3d(&maps.v, 64 * x, h, ts);
            tma_prefetch_3d(&maps.w, 64 * x, h, ts);
        }
    };
    if (warp == kProducer) {
        // One thread of the producer warp stages every chunk's raw rows: q, k, b as soon as
        // the Sref MMAs of the previous chunk have read the tiles they land on, log_alpha,
        // v, w once the previous chunk's X^T P^T MMAs and its UT solve are done with theirs.
        if (lane == 0 && !p.test_withhold_loads) {
            issue_raw_a(t0);
            issue_raw_b(t0);
            if (nchunks > 1) prefetch_raw(t0 + CH);
            for (int ci = 0; ci + 1 < nchunks; ++ci) {
                const uint32_t par = (uint32_t)(ci & 1);
                const int ts = t0 + (ci + 1) * CH;
                // the chunk after the next one reaches L2 while this chunk is processed, so its
                // loads, issued once their space frees up, do not wait for HBM
                if (ci + 2 < nchunks) prefetch_raw(ts + CH);
                if (!mbar_wait(mbar(MB_2A), par, kWaitNs)) { fault = true; break; }
                issue_raw_b(ts);
                if (!mbar_wait(mbar(MB_2P), par, kWaitNs) || !mbar_wait(mbar(RDY_RAWA), par, kWaitNs)) {
                    fault = true;
                    break;
                }
                issue_raw_a(ts);
            }
        }
        __syncwarp();
    }

    if (warp == kIssuer) {
        // One thread of the issuer warp waits for each MMA group's operands, issues the group
        // and commits it to the group's completion barrier, chunk after chunk, so that no
        // SIMT warp stalls behind the tensor pipe. If the SIMT warps stop early (a fault), the
        // next wait here runs out and this warp stops too.
        if (lane == 0) {
            const uint32_t sbase_k = sbase, tmem_k = tmem;
            for (int ci = 0; ci < nchunks; ++ci) {
                const uint32_t par = (uint32_t)(ci & 1);
                // addresses re-derived every chunk: kept live across the loop, the ~80 operand
                // descriptors would take the registers the SIMT warps need
                const uint32_t sbase = opaque_u32(sbase_k), tmem = opaque_u32(tmem_k);
                if (!mbar_wait(mbar(RDY_G), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // Gram: [Kb; Eb] x [Kh; Qh]^T, then the P cross terms
                    const uint32_t id128 = idesc_bf16(128, 128, false, false);
                    const uint32_t id64 = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t kofs = ks * 256;
                        mma_bf16(tmem + TM_G, sdesc(sbase + OFF_KBH + kofs, 128, 2048),
                                 sdesc(sbase + OFF_KH + kofs, 128, 2048), id128, ks > 0);
                    }
                    mma_commit(mbar(MB_G));
                    // P cross terms (lanes 0..63 hold Kb rows; lanes 64..127 are masked out)
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t kofs = ks * 256;
                        mma_bf16(tmem + TM_G + 64, sdesc(sbase + OFF_KBL + kofs, 128, 2048),
                                 sdesc(sbase + OFF_QH + kofs, 128, 2048), id64, 1u, 0u, 0u, 0xffffffffu, 0xffffffffu);
                        mma_bf16(tmem + TM_G + 64, sdesc(sbase + OFF_KBH + kofs, 128, 2048),
                                 sdesc(sbase + OFF_QL + kofs, 128, 2048), id64, 1u, 0u, 0u, 0xffffffffu, 0xffffffffu);
                    }
                    mma_commit(mbar(MB_GX));
                }
                if (!mbar_wait(mbar(RDY_2A), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // Y^T = Sref^T Kh^T, O^T = Sref^T Qh^T (hi / lo); then U += X^T Kb (no state read)
                    const uint32_t id64 = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t a = tmem + TM_S + ks * 8, al = tmem + TM_SL + ks * 8;
                        const uint64_t qh = sdesc(sbase + OFF_QH + ks * 256, 128, 2048);
                        mma_bf16_ts(tmem + TM_D1, a, sdesc(sbase + OFF_KH + ks * 256, 128, 2048), id64, ks > 0);
                        mma_bf16_ts(tmem + TM_D1 + 64, a, qh, id64, ks > 0);
                        mma_bf16_ts(tmem + TM_D1 + 64, a, sdesc(sbase + OFF_QL + ks * 256, 128, 2048), id64, 1u);
                        mma_bf16_ts(tmem + TM_D1 + 64, al, qh, id64, 1u);
                    }
                    mma_commit(mbar(MB_2A));
                    const uint32_t id_xx = idesc_bf16(128, 128, true, true);
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks) {
                        const uint64_t xh = sdesc(sbase + OFF_XH + ks * 4096, 2048, 128);
                        const uint64_t xl = sdesc(sbase + OFF_XL + ks * 4096, 2048, 128);
                        mma_bf16(tmem + TM_U, xh, sdesc(sbase + OFF_KBH + ks * 4096, 2048, 128), id_xx, 1u);
                        mma_bf16(tmem + TM_U, xl, sdesc(sbase + OFF_KBH + ks * 4096, 2048, 128), id_xx, 1u);
                        mma_bf16(tmem + TM_U, xh, sdesc(sbase + OFF_KBL + ks * 4096, 2048, 128), id_xx, 1u);
                    }
                }
                if (!mbar_wait(mbar(RDY_2B), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // Y^T += X^T B^T
                    const uint32_t id64 = idesc_bf16(128, 64, true, true);
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks)
                        mma_bf16(tmem + TM_D1, sdesc(sbase + OFF_XH + ks * 4096, 2048, 128),
                                 sdesc(sbase + OFF_B + ks * 256, 128, 1024), id64, 1u);
                    mma_commit(mbar(MB_2B));
                }
                if (!mbar_wait(mbar(RDY_2P), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // O^T += X^T P^T (hi / lo)
                    const uint32_t id64 = idesc_bf16(128, 64, true, true);
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks) {
                        const uint64_t xh = sdesc(sbase + OFF_XH + ks * 4096, 2048, 128);
                        const uint64_t xl = sdesc(sbase + OFF_XL + ks * 4096, 2048, 128);
                        mma_bf16(tmem + TM_D1 + 64, xh, sdesc(sbase + OFF_PH + ks * 256, 128, 1024), id64, 1u);
                        mma_bf16(tmem + TM_D1 + 64, xl, sdesc(sbase + OFF_PH + ks * 256, 128, 1024), id64, 1u);
                        mma_bf16(tmem + TM_D1 + 64, xh, sdesc(sbase + OFF_PL + ks * 256, 128, 1024), id64, 1u);
                    }
                    mma_commit(mbar(MB_2P));
                }
                if (!mbar_wait(mbar(RDY_3), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // R^T = Y^T T^T
                    const uint32_t id64 = idesc_bf16(128, 64, false, false);
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks)
                        mma_bf16_ts(tmem + TM_R, tmem + TM_D1 + ks * 8, sdesc(sbase + OFF_T + ks * 2048, 1024, 128),
                                    id64, ks > 0);
                    mma_commit(mbar(MB_3));
                }
                if (!mbar_wait(mbar(RDY_45), par, kWaitNs)) { fault = true; break; }
                tc_fence_after();
                {  // O^T -= R^T Qm^T (committed on its own: the o epilogue waits for it only);
                   // U -= R^T Eb
                    const uint32_t id_o = idesc_bf16(128, 64, false, true);
                    const uint32_t id_rx = idesc_bf16(128, 128, false, true);
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks)
                        mma_bf16_ts(tmem + TM_D1 + 64, tmem + TM_R + ks * 8, sdesc(sbase + OFF_QM + ks * 256, 128, 1024),
                                    id_o, 1u);
                    mma_commit(mbar(MB_45O));
#pragma unroll
                    for (int ks = 0; ks < CH / 16; ++ks)
                        mma_bf16_ts(tmem + TM_U, tmem + TM_R + ks * 8, sdesc(sbase + OFF_E + ks * 4096, 2048, 128),
                                    id_rx, 1u);
                    mma_commit(mbar(MB_45));
                }
            }
        }
        __syncwarp();
    }
    // Cumulative log-decays G of chunk cs, in base 2 (G log2(e)), in place over its staged
    // log_alpha rows (tokens past the sequence end count as zero): thread (channel c, quarter
    // cp) sums tokens 16cp .. 16cp + 15 of channel c; the totals of the earlier quarters are
    // added where G is read. Runs for chunk 0 before the loop and for chunk c + 1 while chunk
    // c's last MMAs run (its rows are loaded once chunk c's UT solve is done, so by then they
    // have arrived). Returns false if its wait for the rows ran out.
    auto scan_cumsum = [&](int cs) -> bool {
        const int nv = min(CH, t1 - (t0 + cs * CH));
        const bool ok = mbar_wait(mbar(MB_RAWA), (uint32_t)(cs & 1), kWaitNs);
        const int c = L;
        if (kPro) {
            // bf16 pre-activations a (upper half of the area), read completely before the
            // cumulative decay overwrites the area
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int i = 16 * cp + r;
                x[r] = i < nv ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                                    smem + OFF_RAW_A + raw_off_bf16(i, c)))
                              : 0.f;
            }
            bar_sync_1<NS>();
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int i = 16 * cp + r;
                if (i < nv) acc -= softplus_log2e_f(x[r]);
                *reinterpret_cast<float*>(smem + OFF_RAW_LA + raw_off_f32(i, c)) = acc;
            }
            qtot[128 * cp + c] = acc;
        } else {
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int i = 16 * cp + r;
                float* gp = reinterpret_cast<float*>(smem + OFF_RAW_LA + raw_off_f32(i, c));
                acc = fmaf(i < nv ? *gp : 0.f, kLog2e, acc);
                *gp = acc;
            }
            qtot[128 * cp + c] = acc;
        }
        bar_sync_1<NS>();
        return ok;
    };
    // Reference frame of chunk cs (Gref, G_last) and the factors that take the state from
    // chunk cs - 1's frame into it: exp(G_last' - Gref') (to the state itself), then
    // exp(Gref). Two factors, not their product: with strong decay the product underflows
    // where the scaled state does not. (S0 takes exp(Gref) alone.) After scan_cumsum(cs),
    // while chunk cs - 1's last MMAs run; read after the next barrier.
    auto scan_frame = [&](int cs) {
        if (tid < D) {
            const int c = tid, bs = cs & 1;
            const float glast = (qtot[c] + qtot[128 + c]) + (qtot[256 + c] + qtot[384 + c]);
            const float g0 = *reinterpret_cast<const float*>(smem + OFF_RAW_LA + raw_off_f32(0, c));
            const float gref = 0.5f * (g0 + glast);
            // the factors 2^(G - Gref) reach 2^(+-|G_last - G_0| / 2) when the decays of the
            // chunk have one sign (log_alpha <= 0): outside [2^-120, 2^120] the chunk is flagged
            // in shared memory (nothing kept live across the chunks), posted at the end
            if (fabsf(glast - g0) > 2.f * kMaxFactorExp2) *reinterpret_cast<volatile uint32_t*>(smem + OFF_TSLOT + 4) = 1u;
            fscal[c] = exp2f(cs == 0 ? gref : scal[256 + (bs ^ 1) * 128 + c] - scal[(bs ^ 1) * 128 + c]);
            fscal[128 + c] = exp2f(gref);
            scal[bs * 128 + c] = gref;
            scal[256 + bs * 128 + c] = glast;
        }
    };
    // Fused pre-processing: 1 / max(|q|, eps) and 1 / max(|k|, eps) of every token of chunk
    // cs, for its prep, into OFF_RN. Thread u of nthr (256 or 512) takes row u / (nthr / 128)
    // (q rows of tokens 0..63, then k rows) and sums the squares of its share of the 128
    // channels, in swizzled 16-byte pieces. Rows past the sequence end get zero (the prep
    // zeroes those tokens anyway). Returns false if the wait for the rows ran out.
    auto scan_norms = [&](int cs, int u, int nthr) -> bool {
        const bool ok = mbar_wait(mbar(MB_RAWB), (uint32_t)(cs & 1), kWaitNs);
        const int per = nthr / 128, r = u / per, s = u % per, i = r & 63, npc = 16 / per;
        const uint8_t* row = smem + (r < 64 ? OFF_RAW_Q : OFF_RAW_K) + i * 128;
        float ss = 0.f;
        for (int j = 0; j < npc; ++j) {
            const int pc = s * npc + j;  // 16-byte piece: box pc / 8, piece pc % 8 of the row
            const uint4 v = *reinterpret_cast<const uint4*>(row + (pc >> 3) * 8192 + (((pc & 7) ^ (i & 7)) << 4));
            float f[4], g[4];
            unpack4_bf16(make_uint2(v.x, v.y), f);
            unpack4_bf16(make_uint2(v.z, v.w), g);
#pragma unroll
            for (int e = 0; e < 4; ++e) ss = fmaf(f[e], f[e], fmaf(g[e], g[e], ss));
        }
        for (int off = 1; off < per; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        // 1 / max(|x|, eps) as one reciprocal square root (relative error ~2^-22)
        if (s == 0)
            reinterpret_cast<float*>(smem + OFF_RN)[r] =
                i < min(CH, t1 - (t0 + cs * CH)) ? rsqrtf(fmaxf(ss, kL2NormEps * kL2NormEps)) : 0.f;
        return ok;
    };
    const int simt_chunks = warp < kIssuer ? nchunks : 0;
    if (simt_chunks > 0) {
        if (kPro) fault |= !scan_norms(0, tid, NS);
        fault |= !scan_cumsum(0);  // its barriers publish the norms too
        scan_frame(0);
    }

    for (int ci = 0; ci < simt_chunks; ++ci) {
        const int tc0 = t0 + ci * CH;
        const int nvalid = min(CH, t1 - tc0);
        const int buf = ci & 1;
        const uint32_t par = (uint32_t)(ci & 1);

        // ------------------------------------------------------------ 1. prep
        {
            // group B: q, k, b; the tiles below overwrite these rows and the staged o tile
            uint2 qq[4], kq[4], bq[4];
            fault |= !mbar_wait(mbar(MB_RAWB), par, kWaitNs);
#pragma unroll
            for (int pss = 0; pss < 4; ++pss) {
                const int i = ti0 + 8 * pss;
                const bool valid = i < nvalid;
                const uint32_t o = raw_off_bf16(i, c0);
                const uint2 z = make_uint2(0u, 0u);
                qq[pss] = valid ? *reinterpret_cast<const uint2*>(smem + OFF_RAW_Q + o) : z;
                kq[pss] = valid ? *reinterpret_cast<const uint2*>(smem + OFF_RAW_K + o) : z;
                bq[pss] = valid ? *reinterpret_cast<const uint2*>(smem + OFF_RAW_B + o) : z;
            }
            // the tiles below overwrite Eb, which the previous chunk's U -= R^T Eb MMAs read
            if (ci > 0) fault |= !mbar_wait(mbar(MB_45), par ^ 1u, kWaitNs);
            if (bar_or_1<NS>(fault)) {
                fault = true;
                break;
            }
            // the previous (full) chunk's o tile, staged in the X tiles before this barrier;
            // its reads must be done before the X tiles are rewritten, after the Gram's issue
            if (kTmaStoreO<TO> && ci > 0 && tid == 0) {
                tma_store_3d(&maps.o, sbase + OFF_OST0, 0, h, tc0 - CH);
                tma_store_3d(&maps.o, sbase + OFF_OST1, 0, h, tc0 - CH / 2);
                bulk_commit();
            }
            // G - Gref: this thread's tokens lie in quarters 2th and 2th + 1, whose offsets
            // are the totals of the quarters before them
            float dlo[4], dhi[4];
            {
                const float4 gr4 = *reinterpret_cast<const float4*>(scal + buf * 128 + c0);
                const float gr[4] = {gr4.x, gr4.y, gr4.z, gr4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float t0q = qtot[c0 + e], t1q = qtot[128 + c0 + e], t2q = qtot[256 + c0 + e];
                    dlo[e] = (th ? t0q + t1q : 0.f) - gr[e];
                    dhi[e] = (th ? (t0q + t1q) + t2q : t0q) - gr[e];
                }
            }
#pragma unroll
            for (int pss = 0; pss < 4; ++pss) {
                const int i = ti0 + 8 * pss;
                const float4 g4 = *reinterpret_cast<const float4*>(smem + OFF_RAW_LA + raw_off_f32(i, c0));
                const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
                float qf[4], kf[4], bf[4];
                unpack4_bf16(qq[pss], qf);
                unpack4_bf16(kq[pss], kf);
                unpack4_bf16(bq[pss], bf);
                if (kPro) {
                    // 1 / |q|, 1 / |k| of this token (taken during the previous chunk's solve)
                    const float* rn = reinterpret_cast<const float*>(smem + OFF_RN);
                    const float rqv = rn[i], rkv = rn[64 + i];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        qf[e] *= rqv;
                        kf[e] *= rkv;
                        bf[e] = sigmoid_tanh_f(bf[e]);  // b only reaches the plain bf16 Eb tile
                    }
                }
                float kh[4], qv[4], kb[4], eb[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // (G - Gref) log2(e); the special-function unit's 2^x is far more accurate
                    // than the 2^-16 carried by the hi/lo operand splits
                    const float d = gv[e] + (pss < 2 ? dlo[e] : dhi[e]);
                    const float ge = ex2_approx(d);
                    const float gi = ex2_approx(-d);
                    kh[e] = kf[e] * ge;
                    qv[e] = qf[e] * ge;
                    kb[e] = kf[e] * gi;
                    eb[e] = bf[e] * kb[e];
                }
                uint2 qh, ql, kbh, kbl;
                split2(qv[0], qv[1], qh.x, ql.x);
                split2(qv[2], qv[3], qh.y, ql.y);
                split2(kb[0], kb[1], kbh.x, kbl.x);
                split2(kb[2], kb[3], kbh.y, kbl.y);
                const uint32_t o = off_rowmajor(i, c0);
                store4_bf16(smem, OFF_KH + o, kh);
                store4_bf16(smem, OFF_E + o, eb);
                *reinterpret_cast<uint2*>(smem + OFF_QH + o) = qh;
                *reinterpret_cast<uint2*>(smem + OFF_QL + o) = ql;
                *reinterpret_cast<uint2*>(smem + OFF_KBH + o) = kbh;
                *reinterpret_cast<uint2*>(smem + OFF_KBL + o) = kbl;
            }
        }
        fence_proxy_async_smem();
        if (tid == 0) bulk_wait_read0();  // the staged o tile has been read out
        if (bar_or_1<NS>(fault)) { fault = true; break; }

        // ------------------------------------------------------------ 2. Gram MMAs
        if (tid == 0) mbar_arrive(mbar(RDY_G));
        // X = w (.) v tiles while the Gram MMAs run (their space holds nothing raw; the
        // epilogue below overwrites the raw v / w rows, after the next barrier)
#pragma unroll
        for (int pss = 0; pss < 4; ++pss) {
            const int i = ti0 + 8 * pss;
            const bool valid = i < nvalid;
            const uint32_t ro = raw_off_bf16(i, c0);
            const uint2 z = make_uint2(0u, 0u);
            float vf[4], wf[4];
            unpack4_bf16(valid ? *reinterpret_cast<const uint2*>(smem + OFF_RAW_V + ro) : z, vf);
            unpack4_bf16(valid ? *reinterpret_cast<const uint2*>(smem + OFF_RAW_W + ro) : z, wf);
            if (kPro) {
#pragma unroll
                for (int e = 0; e < 4; ++e) wf[e] = sigmoid_f(wf[e]);
            }
            uint2 xh, xl;
            const float2 x01 = fmul2(make_float2(wf[0], wf[1]), make_float2(vf[0], vf[1]));
            const float2 x23 = fmul2(make_float2(wf[2], wf[3]), make_float2(vf[2], vf[3]));
            split2(x01.x, x01.y, xh.x, xl.x);
            split2(x23.x, x23.y, xh.y, xl.y);
            const uint32_t o = off_rowmajor(i, c0);
            *reinterpret_cast<uint2*>(smem + OFF_XH + o) = xh;
            *reinterpret_cast<uint2*>(smem + OFF_XL + o) = xl;
        }
        fence_proxy_async_smem();  // the X tiles are operands of the MMAs signalled below
        // ------------------------------------------------------------ 3. state epilogue (under the Gram MMAs)
        // Thread (lane L, quarter cp) takes key channels 32cp .. 32cp + 31.
        {
            const int cb = 32 * cp;
            float u[32];
            if (ci == 0) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = cb + e;
                    u[e] = (p.S0 ? p.S0[soff + (size_t)c * D + L] : 0.f) * fscal[c];
                }
            } else {
                tmem_ld32_wait(tmem + lane_bits + TM_U + cb, u);
                const float4* f4 = reinterpret_cast<const float4*>(fscal + cb);
                const float4* g4 = reinterpret_cast<const float4*>(fscal + 128 + cb);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {  // (u f) g, two columns per packed multiply
                    const float4 f = f4[e4], gg = g4[e4];
                    const float2 a = fmul2(fmul2(make_float2(u[4 * e4], u[4 * e4 + 1]), make_float2(f.x, f.y)),
                                           make_float2(gg.x, gg.y));
                    const float2 b = fmul2(fmul2(make_float2(u[4 * e4 + 2], u[4 * e4 + 3]), make_float2(f.z, f.w)),
                                           make_float2(gg.z, gg.w));
                    u[4 * e4] = a.x;
                    u[4 * e4 + 1] = a.y;
                    u[4 * e4 + 2] = b.x;
                    u[4 * e4 + 3] = b.y;
                }
            }
            tmem_st32(tmem + lane_bits + TM_U + cb, u);
            // Sref^T as bf16 hi / lo A operands: key channels cb .. cb + 31 in columns
            // cb/2 .. +15 of TM_S (hi) and TM_SL (lo)
            uint32_t pk[16], pl[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) split2(u[2 * e], u[2 * e + 1], pk[e], pl[e]);
            tmem_st16(tmem + lane_bits + TM_S + 16 * cp, pk);
            tmem_st16(tmem + lane_bits + TM_SL + 16 * cp, pl);
            tmem_wait_st();
        }
        tc_fence_before();
        bar_sync_1<NS>();

        // ------------------------------------------------------------ 4. MMAs Y^T = Sref^T Kh^T, O^T = Sref^T Qh^T, U += X^T Kb
        if (tid == 0) mbar_arrive(mbar(RDY_2A));

        fault |= !mbar_wait(mbar(MB_G), par, kWaitNs);
        if (bar_or_1<NS>(fault)) { fault = true; break; }
        tc_fence_after();

        // ------------------------------------------------------------ 5. Gram epilogue
        // Thread (lane L, quarter cp) takes Gram columns 32cp .. 32cp + 31: lanes 0..63 are
        // Kb rows (B, then P), lanes 64..127 Eb rows (A, then Qm); column i, row j = L % 64.
        {
            // (lanes 0..63 of the P block, which the cross terms still update, are read after
            // the UT solve)
            float v[32];
            tmem_ld32_wait(tmem + lane_bits + TM_G + 32 * cp, v);
            const int j = L & 63;
            const int ib = 32 * (cp & 1);  // first i of this thread
            if (L < 64 && cp < 2) {  // B_ij, j < i
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = (ib + 8 * q + e > j) ? v[8 * q + e] : 0.f;
                    store8_bf16(smem, OFF_B + (ib / 8 + q) * 1024 + (j >> 3) * 128 + (j & 7) * 16, f);
                }
            } else if (L < 64) {
                // P: after the UT solve
            } else if (cp < 2) {  // A_ij, j < i, fp32 for the solve
#pragma unroll
                for (int e = 0; e < 32; ++e) WA[(ib + e) * WS + j] = (ib + e > j) ? v[e] : 0.f;
            } else {  // Qm_ij, j <= i
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = (ib + 8 * q + e >= j) ? v[8 * q + e] : 0.f;
                    store8_bf16(smem, OFF_QM + (ib / 8 + q) * 1024 + (j >> 3) * 128 + (j & 7) * 16, f);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (bar_or_1<NS>(fault)) { fault = true; break; }

        // ------------------------------------------------------------ 6. MMA Y^T += X^T B^T
        if (tid == 0) mbar_arrive(mbar(RDY_2B));
        // ------------------------------------------------------------ 3b. UT solve, while the MMAs above run
        // T = (I + A)^-1 in three levels. Level 1: the four 16 x 16 diagonal blocks by
        // column-wise forward substitution. Levels 2 and 3 join diagonal blocks of 16 into 32
        // and of 32 into 64 with T_21 = -T_22 (A_21 T_11). Rows of A and T are read as float4
        // (the same row for many lanes: broadcast), columns as consecutive floats.
        // Level 1 runs on warps 2 and 3 (schedulers 2 and 3), so that the P block, whose
        // tensor-memory lanes only warps on schedulers 0 and 1 can read, is written beside it.
        if (tid >= 64 && tid < 128) {
            // column jj of block bI, right-looking: once x_l is final, every later row takes
            // its term, so the chain from one row to the next is a single FMA
            const int bI = (tid - 64) >> 4, jj = tid & 15, col = 16 * bI + jj;
            const float* ablk = WA + 16 * bI * WS + 16 * bI;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = 0.f;
#pragma unroll
            for (int l = 0; l < 16; ++l) {
                x[l] = l < jj ? 0.f : (l == jj ? 1.f : x[l]);
                WT[(16 * bI + l) * WS + col] = x[l];
#pragma unroll
                for (int r = l + 1; r < 16; ++r) x[r] = fmaf(-ablk[r * WS + l], x[l], x[r]);
            }
        } else {
            for (int idx = tid < 64 ? tid : tid - 64; idx < 64 * 64; idx += NS - 64) {
                const int r = idx >> 6, c = idx & 63;
                if ((c >> 4) > (r >> 4)) WT[r * WS + c] = 0.f;
            }
            // ---------------------------------------------------------- 3c. P block of the Gram
            // P_ij (j <= i; lanes j = 0..63, columns 64 + i), split hi / lo, beside level 1.
            // The cross terms that complete it ran behind the main Gram MMAs; its own MMAs
            // (O^T += X^T P^T) run during the rest of the solve.
            if (L < 64 && cp >= 2) {
                if (!mbar_wait(mbar(MB_GX), par, kWaitNs)) fault = true;
                tc_fence_after();
                float v[32];
                tmem_ld32_wait(tmem + lane_bits + TM_G + 32 * cp, v);
                const int j = L, ib = 32 * (cp & 1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = (ib + 8 * q + e >= j) ? v[8 * q + e] : 0.f;
                    uint4 hi, lo;
                    split2(x[0], x[1], hi.x, lo.x);
                    split2(x[2], x[3], hi.y, lo.y);
                    split2(x[4], x[5], hi.z, lo.z);
                    split2(x[6], x[7], hi.w, lo.w);
                    const uint32_t o = (ib / 8 + q) * 1024 + (j >> 3) * 128 + (j & 7) * 16;
                    *reinterpret_cast<uint4*>(smem + OFF_PH + o) = hi;
                    *reinterpret_cast<uint4*>(smem + OFF_PL + o) = lo;
                }
                fence_proxy_async_smem();
                tc_fence_before();
            }
        }
        bar_sync_1<NS>();
        if (tid == 0) mbar_arrive(mbar(RDY_2P));
        {   // level 2, step 1: M = A_10 T_00 for the two 32-blocks (512 outputs, 1 per thread)
            const int blk = tid >> 8, base = 32 * blk, r = (tid >> 4) & 15, c = tid & 15;
            const float* a0 = WA + (base + 16 + r) * WS + base;
            float m = 0.f;
#pragma unroll
            for (int l4 = 0; l4 < 16; l4 += 4) {
                const float4 x0 = *reinterpret_cast<const float4*>(a0 + l4);
                m = fmaf(x0.x, WT[(base + l4) * WS + base + c], m);
                m = fmaf(x0.y, WT[(base + l4 + 1) * WS + base + c], m);
                m = fmaf(x0.z, WT[(base + l4 + 2) * WS + base + c], m);
                m = fmaf(x0.w, WT[(base + l4 + 3) * WS + base + c], m);
            }
            WM[(blk * 16 + r) * 33 + c] = m;
        }
        bar_sync_1<NS>();
        {   // level 2, step 2: T_10 = -T_11 M
            const int blk = tid >> 8, base = 32 * blk, r = (tid >> 4) & 15, c = tid & 15;
            const float* Mb = WM + blk * 16 * 33;
            const float* t0r = WT + (base + 16 + r) * WS + base + 16;
            float t = 0.f;
#pragma unroll
            for (int l4 = 0; l4 < 16; l4 += 4) {
                const float4 y0 = *reinterpret_cast<const float4*>(t0r + l4);  // upper triangle: zeros
                t = fmaf(y0.x, Mb[(l4) * 33 + c], t);
                t = fmaf(y0.y, Mb[(l4 + 1) * 33 + c], t);
                t = fmaf(y0.z, Mb[(l4 + 2) * 33 + c], t);
                t = fmaf(y0.w, Mb[(l4 + 3) * 33 + c], t);
            }
            WT[(base + 16 + r) * WS + base + c] = -t;
        }
        bar_sync_1<NS>();
        if (warp < 8) {
            // level 3 on warps 0..7: T_BA = -T_BB (A_BA T_AA), lane c = column c, four rows
            // per warp, so every value read from shared memory feeds four FMAs
            const int c = lane, rb = 4 * warp;
            float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int l4 = 0; l4 < 32; l4 += 4) {  // M = A_BA T_AA (rows rb .. rb + 3)
                float tv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) tv[u] = WT[(l4 + u) * WS + c];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 a = *reinterpret_cast<const float4*>(WA + (32 + rb + k) * WS + l4);
                    m[k] += a.x * tv[0] + a.y * tv[1] + a.z * tv[2] + a.w * tv[3];
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) WM[(rb + k) * 33 + c] = m[k];
            bar_sync_n<2, 256>();
            // T_BA rows rb .. rb + 3 = -T_BB M; T_BB is lower triangular, so only its columns
            // up to rb + 3 contribute
            float t[4] = {0.f, 0.f, 0.f, 0.f};
            for (int l4 = 0; l4 <= rb; l4 += 4) {
                float mv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) mv[u] = WM[(l4 + u) * 33 + c];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 a = *reinterpret_cast<const float4*>(WT + (32 + rb + k) * WS + 32 + l4);
                    t[k] += a.x * mv[0] + a.y * mv[1] + a.z * mv[2] + a.w * mv[3];
                }
            }
            // into the bf16 T tile (K-major [i][j]): T[32 + rb + k][c]
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = 32 + rb + k;
                *reinterpret_cast<__nv_bfloat16*>(smem + OFF_T + (c >> 3) * 1024 + (i >> 3) * 128 + (i & 7) * 16 +
                                                  (c & 7) * 2) = __float2bfloat16_rn(-t[k]);
            }
        } else {
            // meanwhile warps 8..15 store the parts of T complete after level 2 as the K-major
            // bf16 B operand [i][j]: rows 0..31 (all columns), rows 32..63 columns 32..63
            const int u = tid - 256, i = u & 31, jg = u >> 5;
            store8_bf16(smem, OFF_T + jg * 1024 + (i >> 3) * 128 + (i & 7) * 16, &WT[i * WS + 8 * jg]);
            if (u < 128) {
                const int i2 = 32 + i, jg2 = 4 + jg;
                store8_bf16(smem, OFF_T + jg2 * 1024 + (i2 >> 3) * 128 + (i2 & 7) * 16, &WT[i2 * WS + 8 * jg2]);
            }
            // then the next chunk's q and k norms (its q, k rows have landed by now: they are
            // loaded once this chunk's Sref MMAs are done)
            if (kPro && ci + 1 < nchunks) fault |= !scan_norms(ci + 1, u, 256);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        bar_sync_1<NS>();
        if (tid == 0) mbar_arrive(mbar(RDY_RAWA));  // the solve's workspace is dead

        fault |= !mbar_wait(mbar(MB_2B), par, kWaitNs);
        fault |= !mbar_wait(mbar(MB_2A), par, kWaitNs);
        if (bar_or_1<NS>(fault)) { fault = true; break; }
        tc_fence_after();

        // ------------------------------------------------------------ 7. Y^T as a bf16 A operand
        // Thread (lane L, quarter cp) takes tokens 16cp .. 16cp + 15 (fp32 columns), packed
        // into columns 8cp .. 8cp + 7.
        {
            float y[16];
            tmem_ld16_wait(tmem + lane_bits + TM_D1 + 16 * cp, y);
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(y[2 * e], y[2 * e + 1]);
            bar_sync_1<NS>();  // every quarter has read its fp32 columns before any are overwritten
            tmem_st8(tmem + lane_bits + TM_D1 + 8 * cp, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        bar_sync_1<NS>();

        // ------------------------------------------------------------ 8. R^T = Y^T T^T
        if (tid == 0) mbar_arrive(mbar(RDY_3));
        fault |= !mbar_wait(mbar(MB_3), par, kWaitNs);
        if (bar_or_1<NS>(fault)) { fault = true; break; }
        tc_fence_after();

        // ------------------------------------------------------------ 9. -R^T as a bf16 A operand
        {
            float r[16];
            tmem_ld16_wait(tmem + lane_bits + TM_R + 16 * cp, r);
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(-r[2 * e], -r[2 * e + 1]);
            bar_sync_1<NS>();  // every quarter has read its fp32 columns before any are overwritten
            tmem_st8(tmem + lane_bits + TM_R + 8 * cp, pk);
            tmem_wait_st();
        }
        tc_fence_before();
        bar_sync_1<NS>();

        // ------------------------------------------------------------ 10. output and state MMAs
        if (tid == 0) mbar_arrive(mbar(RDY_45));
        if (ci + 1 < nchunks) {  // the next chunk's scan, under the O and U MMAs
            fault |= !scan_cumsum(ci + 1);
            scan_frame(ci + 1);
        }
        fault |= !mbar_wait(mbar(MB_45O), par, kWaitNs);
        if (bar_or_1<NS>(fault)) { fault = true; break; }
        tc_fence_after();

        // ------------------------------------------------------------ 11. o
        // Thread (lane L = value channel, quarter cp) takes tokens 16cp .. 16cp + 15.
        {
            float ov[16];
            tmem_ld16_wait(tmem + lane_bits + TM_D1 + 64 + 16 * cp, ov);
            if (kTmaStoreO<TO> && nvalid == CH) {
                // stage the fp32 tile [token][channel] in two halves over X hi / lo (free:
                // every MMA that reads them ran before the ones just waited for; Eb, which
                // the U -= R^T Eb MMAs may still read, is untouched); TMA stores write them
                // after the next barrier (the next chunk's first, or the one after the loop)
                float* ost = reinterpret_cast<float*>(smem + (cp < 2 ? OFF_OST0 : OFF_OST1));
#pragma unroll
                for (int e = 0; e < 16; ++e) ost[(16 * (cp & 1) + e) * D + L] = ov[e];
                fence_proxy_async_smem();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i = 16 * cp + e;
                    if (i < nvalid) op[((size_t)(tc0 + i) * p.h_v + h) * D + L] = from_f32<TO>(ov[e]);
                }
            }
        }
        tc_fence_before();
    }
    // redo: some chunk's decay left the frame's range (the flag is set before a barrier the
    // SIMT warps have all passed); this pair is then recomputed token by token below
    bool redo = false;
    if (warp < kIssuer) {
        bar_sync_1<NS>();
        redo = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TSLOT + 4) != 0u;
        const int tcl = t0 + (nchunks - 1) * CH;
        if (kTmaStoreO<TO> && !fault && t1 - tcl == CH && tid == 0) {  // the last chunk's staged o
            tma_store_3d(&maps.o, sbase + OFF_OST0, 0, h, tcl);
            tma_store_3d(&maps.o, sbase + OFF_OST1, 0, h, tcl + CH / 2);
            bulk_commit();
        }
        // the staged o tile must be read out before shared memory is released or rewritten,
        // and, when o is recomputed, written out before the recomputation's stores
        if (tid == 0) {
            if (redo) bulk_wait_all0();
            else bulk_wait_read0();
        }
        if (!fault) fault = !mbar_wait(mbar(MB_45), (uint32_t)((nchunks - 1) & 1), kWaitNs);
        fault = bar_or_1<NS>(fault);  // one decision for all SIMT warps
        redo = redo && !fault;
    }

    if (!fault && !redo && p.S_T && warp < kIssuer) {  // S_T[c][m] = exp(G_last - Gref) (.) U[m][c]
        const int buf = (nchunks - 1) & 1;
        tc_fence_after();
        const int cb = 32 * cp;
        float u[32];
        tmem_ld32_wait(tmem + lane_bits + TM_U + cb, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int c = cb + e;
            p.S_T[soff + (size_t)c * D + L] = u[e] * exp2f(scal[256 + buf * 128 + c] - scal[buf * 128 + c]);
        }
    }
    if (fault && (tid == 0 || tid == NS || tid == NS + 32)) atomicOr(&g_status_tc, kStatusWaitTimeout);
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && redo) atomicOr(&g_status_tc, kStatusDecayRange);  // recomputed below
    if (warp == 0) tmem_dealloc(tmem, 512);
    if (redo) redo_tokens<TO, kPro>(p, h, g, t0, t1, soff, smem, tid);  // SIMT warps only
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // looked up once (a function-local static is initialised once, whichever threads call)
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

// Rows of one head of a [T, heads, 128] tensor, in boxes of box_rows tokens. swizzled:
// boxes of 128 bytes per row (64 bf16 / 32 fp32 channels) with the 128-byte swizzle; else
// whole rows.
bool encode_rows(PFN_cuTensorMapEncodeTiled_v12000 fn, CUtensorMap* m, const void* base, bool fp32, int heads,
                 int T, bool swizzled, int box_rows = CH) {
    const cuuint64_t es = fp32 ? 4 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)heads * D * es};
    cuuint32_t box[3] = {swizzled ? (cuuint32_t)(128 / es) : (cuuint32_t)D, 1u, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TO, bool kPro>
cudaError_t launch_tc_t(const Params& p, cudaStream_t s) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    RawMaps maps;
    const bool la_ok = kPro ? encode_rows(fn, &maps.la, p.a_raw, false, p.h_v, p.T_total, true)
                            : encode_rows(fn, &maps.la, p.log_alpha, true, p.h_v, p.T_total, true);
    if (!la_ok ||
        !encode_rows(fn, &maps.q, p.q, false, p.h_qk, p.T_total, true) ||
        !encode_rows(fn, &maps.k, p.k, false, p.h_qk, p.T_total, true) ||
        !encode_rows(fn, &maps.b, p.b, false, p.h_v, p.T_total, true) ||
        !encode_rows(fn, &maps.v, p.v, false, p.h_v, p.T_total, true) ||
        !encode_rows(fn, &maps.w, p.w, false, p.h_v, p.T_total, true))
        return cudaErrorInvalidValue;
    if (sizeof(TO) == 4) {
        if (!encode_rows(fn, &maps.o, p.o, true, p.h_v, p.T_total, false, CH / 2)) return cudaErrorInvalidValue;
    } else {
        maps.o = maps.la;  // unused: bf16 outputs take plain stores
    }
    // set on every launch: the attribute is per device and the call costs microseconds
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<TO, kPro>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<TO, kPro><<<p.n_seq * p.h_v, NT, SMEM_BYTES, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

void* tensor_map_encoder() { return reinterpret_cast<void*>(encode_fn()); }

bool chunk_tc_supported(const Params& p, gdn2_dtype dt) {
    return dt == GDN2_BF16 && p.dk == D && p.dv == D && p.T_total > 0;
}

cudaError_t launch_chunk_tc(const Params& p, gdn2_dtype odt, cudaStream_t s) {
    if (p.prologue) return odt == GDN2_F32 ? launch_tc_t<float, true>(p, s) : launch_tc_t<__nv_bfloat16, true>(p, s);
    return odt == GDN2_F32 ? launch_tc_t<float, false>(p, s) : launch_tc_t<__nv_bfloat16, false>(p, s);
}

cudaError_t read_clear_status_chunk_tc(unsigned int* out, cudaStream_t s) {
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_status_tc, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    static const unsigned int zero = 0;
    return cudaMemcpyToSymbolAsync(g_status_tc, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s);
}

}  // namespace gdn2
