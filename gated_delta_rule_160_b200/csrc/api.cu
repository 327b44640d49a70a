// api.cu -- the C ABI of libgdn2 (include/gdn2.h): argument checks and kernel dispatch.
//
// Every check runs on the host before anything is queued; a rejected call queues
// nothing. Error text is kept per calling thread.
#include <stdarg.h>
#include <stdio.h>

#include <atomic>

#include "internal.cuh"

namespace gdn2 {
namespace {

thread_local char g_err[512] = "";

// Testing hook (gdn2_testing_set_wait_limit): limit of the prefill's bounded waits, and
// whether its producer withholds the first loads.
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_withhold{0};

gdn2_status fail(gdn2_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

gdn2_status ok() {
    g_err[0] = '\0';
    return GDN2_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// A pointer the GPU can dereference as device memory (plain or managed allocations).
bool is_device_ptr(const void* ptr) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error this query may leave
        return false;
    }
    return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

gdn2_status check_shape(const gdn2_shape* sh) {
    if (!sh) return fail(GDN2_ERR_INVALID_ARG, "shape is NULL");
    if (sh->n_seq < 1 || sh->n_seq > 65535)
        return fail(GDN2_ERR_INVALID_ARG, "n_seq = %d outside [1, 65535]", sh->n_seq);
    if (sh->T_total < 0) return fail(GDN2_ERR_INVALID_ARG, "T_total = %d is negative", sh->T_total);
    if (sh->h_qk < 1 || sh->h_v < 1)
        return fail(GDN2_ERR_INVALID_ARG, "head counts must be positive (h_qk=%d, h_v=%d)", sh->h_qk, sh->h_v);
    if (sh->h_v % sh->h_qk != 0)
        return fail(GDN2_ERR_INVALID_ARG, "h_v = %d is not a multiple of h_qk = %d", sh->h_v, sh->h_qk);
    if (sh->h_v > 65535) return fail(GDN2_ERR_UNSUPPORTED, "h_v = %d above 65535", sh->h_v);
    if ((long long)sh->n_seq * sh->h_v > 0x7fffffffLL)  // one CTA per (sequence, value head)
        return fail(GDN2_ERR_UNSUPPORTED, "n_seq * h_v = %lld (sequence, head) pairs above 2^31 - 1",
                    (long long)sh->n_seq * sh->h_v);
    if (sh->dtype != GDN2_F32 && sh->dtype != GDN2_BF16)
        return fail(GDN2_ERR_INVALID_ARG, "unknown dtype %d", (int)sh->dtype);
    if (sh->o_dtype != GDN2_F32 && sh->o_dtype != GDN2_BF16)
        return fail(GDN2_ERR_INVALID_ARG, "unknown o_dtype %d", (int)sh->o_dtype);
    if ((sh->dk != 64 && sh->dk != 128) || (sh->dv != 64 && sh->dv != 128))
        return fail(GDN2_ERR_UNSUPPORTED, "dk = %d, dv = %d: only 64 and 128 are supported", sh->dk, sh->dv);
    return GDN2_OK;
}

struct NamedPtr {
    const char* name;
    const void* ptr;
    bool required;
};

gdn2_status check_ptrs(const NamedPtr* ps, int n) {
    for (int i = 0; i < n; ++i) {
        if (!ps[i].ptr) {
            if (ps[i].required) return fail(GDN2_ERR_INVALID_ARG, "%s is NULL", ps[i].name);
            continue;
        }
        if (!aligned16(ps[i].ptr))
            return fail(GDN2_ERR_INVALID_ARG, "%s = %p is not 16-byte aligned", ps[i].name, ps[i].ptr);
        if (!is_device_ptr(ps[i].ptr))
            return fail(GDN2_ERR_INVALID_ARG, "%s = %p is not device memory", ps[i].name, ps[i].ptr);
    }
    return GDN2_OK;
}

Params make_params(const gdn2_shape* sh, const void* q, const void* k, const void* v,
                   const float* la, const void* b, const void* w, const float* S0,
                   const int32_t* cu, void* o, float* S_T) {
    Params p{};
    p.n_seq = sh->n_seq;
    p.T_total = sh->T_total;
    p.h_qk = sh->h_qk;
    p.h_v = sh->h_v;
    p.dk = sh->dk;
    p.dv = sh->dv;
    p.T_fixed = cu ? 0 : sh->T_total / sh->n_seq;
    p.q = q; p.k = k; p.v = v; p.log_alpha = la; p.b = b; p.w = w;
    p.S0 = S0; p.cu_seqlens = cu; p.o = o; p.S_T = S_T; p.order = nullptr;
    p.n_tok = 1; p.slots = nullptr; p.n_slots = sh->n_seq; p.S_steps = nullptr;
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    p.test_withhold_loads = g_withhold.load(std::memory_order_relaxed);
    return p;
}

}  // namespace

gdn2_status report_error(gdn2_status st, const char* msg) { return fail(st, "%s", msg); }

}  // namespace gdn2

using namespace gdn2;

extern "C" {

const char* gdn2_last_error_string(void) { return g_err; }

int gdn2_version(void) { return 200; }

gdn2_status gdn2_device_status(unsigned int* flags, gdn2_stream_t stream) {
    if (!flags) return fail(GDN2_ERR_INVALID_ARG, "flags is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned int w[4] = {0u, 0u, 0u, 0u};
    cudaError_t e = cudaStreamSynchronize(s);  // the work queued so far has run
    if (e == cudaSuccess) e = read_clear_status_chunk_tc(&w[0], s);
    if (e == cudaSuccess) e = read_clear_status_recurrent(&w[1], s);
    if (e == cudaSuccess) e = read_clear_status_schedule(&w[2], s);
    if (e == cudaSuccess) e = read_clear_status_decode(&w[3], s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // the reads have landed in w
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "device status: %s", cudaGetErrorString(e));
    *flags = w[0] | w[1] | w[2] | w[3];
    return ok();
}

void gdn2_testing_set_wait_limit(unsigned long long wait_ns, int withhold_first_load) {
    g_wait_ns.store(wait_ns ? wait_ns : kDefaultWaitNs, std::memory_order_relaxed);
    g_withhold.store(withhold_first_load ? 1 : 0, std::memory_order_relaxed);
}

size_t gdn2_chunk_fwd_workspace_size(const gdn2_shape* shape, int varlen) {
    if (!shape || !varlen || shape->n_seq < 1) return 0;
    // the longest-first order of the sequences, 256-byte rounded
    return ((size_t)shape->n_seq * sizeof(int32_t) + 255) & ~(size_t)255;
}

}  // extern "C"

namespace {

// gdn2_chunk_fwd and gdn2_chunk_fwd_prologue: with prologue, la is the dtype decay
// pre-activation instead of fp32 log_alpha.
gdn2_status chunk_fwd(bool prologue, const gdn2_shape* shape, const void* q, const void* k, const void* v,
                      const void* la, const void* b, const void* w, const float* S0, const int32_t* cu_seqlens,
                      void* o, float* S_T, void* workspace, size_t workspace_bytes, gdn2_stream_t stream) {
    gdn2_status st = check_shape(shape);
    if (st != GDN2_OK) return st;
    const bool any_tokens = shape->T_total > 0;
    const NamedPtr ps[] = {
        {"q", q, any_tokens}, {"k", k, any_tokens}, {"v", v, any_tokens},
        {prologue ? "a" : "log_alpha", la, any_tokens}, {"b", b, any_tokens}, {"w", w, any_tokens},
        {"o", o, any_tokens}, {"S0", S0, false}, {"S_T", S_T, false},
        {"cu_seqlens", cu_seqlens, false}, {"workspace", workspace, false},
    };
    st = check_ptrs(ps, (int)(sizeof ps / sizeof ps[0]));
    if (st != GDN2_OK) return st;
    if (!cu_seqlens && shape->T_total % shape->n_seq != 0)
        return fail(GDN2_ERR_INVALID_ARG, "T_total = %d is not a multiple of n_seq = %d (and no cu_seqlens)",
                    shape->T_total, shape->n_seq);
    const size_t need = gdn2_chunk_fwd_workspace_size(shape, cu_seqlens != nullptr);
    if (need && (!workspace || workspace_bytes < need))
        return fail(GDN2_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(GDN2_ERR_INVALID_ARG, "workspace is not 256-byte aligned");

    Params p = make_params(shape, q, k, v, prologue ? nullptr : static_cast<const float*>(la), b, w, S0,
                           cu_seqlens, o, S_T);
    p.prologue = prologue;
    p.a_raw = prologue ? la : nullptr;
    if (prologue && any_tokens && !chunk_tc_supported(p, shape->dtype))
        return fail(GDN2_ERR_UNSUPPORTED, "the fused pre-processing needs bf16 inputs with dk = dv = 128");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cu_seqlens) {
        int32_t* order = static_cast<int32_t*>(workspace);
        cudaError_t e = launch_varlen_order(p, order, s);
        if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "order kernel: %s", cudaGetErrorString(e));
        p.order = order;
    }
    cudaError_t e = chunk_tc_supported(p, shape->dtype) ? launch_chunk_tc(p, shape->o_dtype, s)
                                                        : launch_recurrent(p, shape->dtype, shape->o_dtype, s);
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "chunk kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // namespace

extern "C" {

gdn2_status gdn2_chunk_fwd(const gdn2_shape* shape, const void* q, const void* k, const void* v,
                           const float* log_alpha, const void* b, const void* w, const float* S0,
                           const int32_t* cu_seqlens, void* o, float* S_T, void* workspace,
                           size_t workspace_bytes, gdn2_stream_t stream) {
    return chunk_fwd(false, shape, q, k, v, log_alpha, b, w, S0, cu_seqlens, o, S_T, workspace, workspace_bytes,
                     stream);
}

gdn2_status gdn2_chunk_fwd_prologue(const gdn2_shape* shape, const void* q_raw, const void* k_raw, const void* v,
                                    const void* a_raw, const void* b_raw, const void* w_raw, const float* S0,
                                    const int32_t* cu_seqlens, void* o, float* S_T, void* workspace,
                                    size_t workspace_bytes, gdn2_stream_t stream) {
    return chunk_fwd(true, shape, q_raw, k_raw, v, a_raw, b_raw, w_raw, S0, cu_seqlens, o, S_T, workspace,
                     workspace_bytes, stream);
}

gdn2_status gdn2_decode_step(const gdn2_shape* shape, const void* q, const void* k, const void* v,
                             const float* log_alpha, const void* b, const void* w, float* S, void* o,
                             gdn2_stream_t stream) {
    gdn2_status st = check_shape(shape);
    if (st != GDN2_OK) return st;
    if (shape->T_total != shape->n_seq)
        return fail(GDN2_ERR_INVALID_ARG, "decode takes one token per sequence: T_total = %d, n_seq = %d",
                    shape->T_total, shape->n_seq);
    if ((long long)shape->n_seq * shape->h_v > 0x7fffffffLL)
        return fail(GDN2_ERR_UNSUPPORTED, "n_seq * h_v too large for one launch");
    const NamedPtr ps[] = {
        {"q", q, true}, {"k", k, true}, {"v", v, true}, {"log_alpha", log_alpha, true},
        {"b", b, true}, {"w", w, true}, {"S", S, true}, {"o", o, true},
    };
    st = check_ptrs(ps, (int)(sizeof ps / sizeof ps[0]));
    if (st != GDN2_OK) return st;
    Params p = make_params(shape, q, k, v, log_alpha, b, w, nullptr, nullptr, o, S);
    cudaError_t e = launch_decode(p, shape->dtype, shape->o_dtype, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "decode kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"

namespace {

gdn2_status decode_multi(bool prologue, const gdn2_shape* shape, int n_tok, const int32_t* slots, const void* q,
                         const void* k, const void* v, const void* la, const void* b, const void* w, float* S_pool,
                         int n_slots, void* o, float* S_steps, gdn2_stream_t stream) {
    gdn2_status st = check_shape(shape);
    if (st != GDN2_OK) return st;
    if (n_tok < 1 || n_tok > GDN2_DECODE_MAX_TOKENS)
        return fail(GDN2_ERR_INVALID_ARG, "n_tok = %d outside 1..%d", n_tok, GDN2_DECODE_MAX_TOKENS);
    if ((long long)shape->n_seq * n_tok != shape->T_total)
        return fail(GDN2_ERR_INVALID_ARG, "T_total = %d is not n_seq * n_tok = %d * %d", shape->T_total,
                    shape->n_seq, n_tok);
    if (n_slots < 1 || (!slots && n_slots < shape->n_seq))
        return fail(GDN2_ERR_INVALID_ARG, "n_slots = %d too small (n_seq = %d, slots %s)", n_slots, shape->n_seq,
                    slots ? "given" : "NULL");
    if ((long long)shape->n_seq * shape->h_v > 0x7fffffffLL || (long long)n_slots * shape->h_v > 0x7fffffffLL)
        return fail(GDN2_ERR_UNSUPPORTED, "n_seq * h_v or n_slots * h_v too large for one launch");
    if ((long long)n_slots * shape->h_v * shape->dk > 0x7fffffffLL)  // state rows, addressed by TMA
        return fail(GDN2_ERR_UNSUPPORTED, "n_slots * h_v * dk = %lld state rows, above 2^31 - 1",
                    (long long)n_slots * shape->h_v * shape->dk);
    const NamedPtr ps[] = {
        {"q", q, true}, {"k", k, true}, {"v", v, true}, {prologue ? "a" : "log_alpha", la, true}, {"b", b, true},
        {"w", w, true}, {"S_pool", S_pool, true}, {"o", o, true}, {"slots", slots, false},
        {"S_steps", S_steps, false},
    };
    st = check_ptrs(ps, (int)(sizeof ps / sizeof ps[0]));
    if (st != GDN2_OK) return st;
    Params p = make_params(shape, q, k, v, prologue ? nullptr : static_cast<const float*>(la), b, w, nullptr,
                           nullptr, o, S_pool);
    p.prologue = prologue;
    p.a_raw = prologue ? la : nullptr;
    p.n_tok = n_tok;
    p.slots = slots;
    p.n_slots = n_slots;
    p.S_steps = S_steps;
    cudaError_t e = launch_decode(p, shape->dtype, shape->o_dtype, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "decode kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // namespace

extern "C" {

gdn2_status gdn2_decode_multi(const gdn2_shape* shape, int n_tok, const int32_t* slots, const void* q,
                              const void* k, const void* v, const float* log_alpha, const void* b, const void* w,
                              float* S_pool, int n_slots, void* o, float* S_steps, gdn2_stream_t stream) {
    return decode_multi(false, shape, n_tok, slots, q, k, v, log_alpha, b, w, S_pool, n_slots, o, S_steps, stream);
}

gdn2_status gdn2_decode_multi_prologue(const gdn2_shape* shape, int n_tok, const int32_t* slots, const void* q_raw,
                                       const void* k_raw, const void* v, const void* a_raw, const void* b_raw,
                                       const void* w_raw, float* S_pool, int n_slots, void* o, float* S_steps,
                                       gdn2_stream_t stream) {
    return decode_multi(true, shape, n_tok, slots, q_raw, k_raw, v, a_raw, b_raw, w_raw, S_pool, n_slots, o, S_steps,
                        stream);
}

size_t gdn2_chunk_bwd_workspace_size(const gdn2_shape* shape) {
    if (!shape || shape->n_seq < 1 || shape->T_total < 0 || shape->h_v < 1 || shape->dk < 1 || shape->dv < 1) return 0;
    return (bwd_workspace_bytes(shape) + 255) & ~(size_t)255;
}

gdn2_status gdn2_chunk_bwd(const gdn2_shape* shape, const void* q, const void* k, const void* v,
                           const float* log_alpha, const void* b, const void* w, const float* S0,
                           const int32_t* cu_seqlens, const float* dO, const float* dS_T, float* dq, float* dk,
                           float* dv, float* dlog_alpha, float* db, float* dw, float* dS0, void* workspace,
                           size_t workspace_bytes, gdn2_stream_t stream) {
    gdn2_status st = check_shape(shape);
    if (st != GDN2_OK) return st;
    const bool any = shape->T_total > 0;
    const NamedPtr ps[] = {
        {"q", q, any}, {"k", k, any}, {"v", v, any}, {"log_alpha", log_alpha, any}, {"b", b, any},
        {"w", w, any}, {"dO", dO, any}, {"dq", dq, any}, {"dk", dk, any}, {"dv", dv, any},
        {"dlog_alpha", dlog_alpha, any}, {"db", db, any}, {"dw", dw, any}, {"S0", S0, false},
        {"cu_seqlens", cu_seqlens, false}, {"dS_T", dS_T, false}, {"dS0", dS0, false},
        {"workspace", workspace, false},
    };
    st = check_ptrs(ps, (int)(sizeof ps / sizeof ps[0]));
    if (st != GDN2_OK) return st;
    if (!cu_seqlens && shape->T_total % shape->n_seq != 0)
        return fail(GDN2_ERR_INVALID_ARG, "T_total = %d is not a multiple of n_seq = %d (and no cu_seqlens)",
                    shape->T_total, shape->n_seq);
    const size_t need = gdn2_chunk_bwd_workspace_size(shape);
    if (!workspace || workspace_bytes < need)
        return fail(GDN2_ERR_INVALID_ARG, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(GDN2_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    Params p = make_params(shape, q, k, v, log_alpha, b, w, S0, cu_seqlens, nullptr, nullptr);
    if (cu_seqlens) {
        cudaError_t ec = launch_check_seqlens(p, reinterpret_cast<cudaStream_t>(stream));
        if (ec != cudaSuccess) return fail(GDN2_ERR_CUDA, "cu_seqlens check kernel: %s", cudaGetErrorString(ec));
    }
    cudaError_t e = launch_bwd(p, shape->dtype, dO, dS_T, dq, dk, dv, dlog_alpha, db, dw, dS0, workspace,
                               reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(GDN2_ERR_CUDA, "backward kernel launch: %s", cudaGetErrorString(e));
    return ok();
}

}  // extern "C"
