// extern "C" entry points of include/arops.h: argument validation, dispatch to
// the kernel launchers, status codes and the thread-local error string.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <atomic>

#include "common.cuh"

namespace arops {

namespace {

thread_local char g_last_error[512] = "";
std::atomic<int> g_pdl{0};
std::atomic<int> g_streaming{0};
std::atomic<int> g_topk_cluster{1};
std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];  // 0 = not queried yet

arops_status fail(arops_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

arops_status ok()
{
    g_last_error[0] = '\0';
    return AROPS_OK;
}

arops_status from_cuda(cudaError_t err, const char* op)
{
    if (err == cudaSuccess)
        return ok();
    return fail(AROPS_ERR_CUDA, "%s: CUDA error %d (%s): %s", op, (int)err, cudaGetErrorName(err),
                cudaGetErrorString(err));
}

bool valid_dtype(arops_dtype d)
{
    return d == AROPS_F32 || d == AROPS_BF16;
}

}  // namespace

// The device error word: kernels that abandon their work (a bounded wait ran
// out) OR a bit into it; arops_device_errors reads and clears it.
__device__ unsigned int g_device_errors = 0;

// Looked up on every call rather than cached per device ordinal: a __device__
// variable has one instance per CUDA context, and the caller's current context
// need not be the one a cached address came from (a context of its own, or a
// primary context reset and created anew).
cudaError_t device_error_word(unsigned** word)
{
    return cudaGetSymbolAddress(reinterpret_cast<void**>(word), g_device_errors);
}

cudaError_t current_device_info(DeviceInfo* info)
{
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    int sms = (dev >= 0 && dev < kMaxDevices) ? g_sm_count[dev].load(std::memory_order_relaxed) : 0;
    if (sms == 0) {
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess)
            return err;
        if (dev >= 0 && dev < kMaxDevices)
            g_sm_count[dev].store(sms, std::memory_order_relaxed);
    }
    info->sm_count = sms;
    return cudaSuccess;
}

bool pdl_enabled()
{
    return g_pdl.load(std::memory_order_relaxed) != 0;
}

bool streaming_enabled()
{
    return g_streaming.load(std::memory_order_relaxed) != 0;
}

int topk_cluster_mode()
{
    return g_topk_cluster.load(std::memory_order_relaxed);
}

void count_launch()
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
}

}  // namespace arops

using namespace arops;

namespace {

// Shared validation and dispatch of the four norm entry points.
arops_status norm_entry(const char* name, const void* x, const void* residual_in,
                        void* residual_out, const void* gamma, const void* beta, void* y,
                        int64_t rows, int64_t hidden, float eps, arops_dtype dtype, void* stream,
                        bool add, bool ln)
{
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "%s: unknown dtype %d", name, (int)dtype);
    if (rows < 0 || hidden <= 0 || hidden > INT32_MAX)
        return fail(AROPS_ERR_INVALID, "%s: bad shape rows=%lld hidden=%lld", name,
                    (long long)rows, (long long)hidden);
    if (!(eps >= 0.0f) || isinf(eps))
        return fail(AROPS_ERR_INVALID, "%s: eps must be finite and >= 0", name);
    if (rows == 0)
        return ok();
    if (!x || !gamma || !y || (add && (!residual_in || !residual_out)) || (ln && !beta))
        return fail(AROPS_ERR_INVALID, "%s: null pointer", name);
    if (add && y == residual_out)
        return fail(AROPS_ERR_INVALID, "%s: y and residual_out are one buffer", name);
    return from_cuda(launch_norm(x, add ? residual_in : nullptr, add ? residual_out : nullptr,
                                 gamma, ln ? beta : nullptr, y, rows, hidden, eps, dtype,
                                 static_cast<cudaStream_t>(stream)),
                     name);
}

}  // namespace

extern "C" {

AROPS_API arops_status arops_rmsnorm(const void* x, const void* gamma, void* y, int64_t rows,
                                     int64_t hidden, float eps, arops_dtype dtype, void* stream)
{
    return norm_entry("arops_rmsnorm", x, nullptr, nullptr, gamma, nullptr, y, rows, hidden, eps,
                      dtype, stream, false, false);
}

AROPS_API arops_status arops_add_rmsnorm(const void* x, const void* residual_in,
                                         void* residual_out, const void* gamma, void* y,
                                         int64_t rows, int64_t hidden, float eps,
                                         arops_dtype dtype, void* stream)
{
    return norm_entry("arops_add_rmsnorm", x, residual_in, residual_out, gamma, nullptr, y, rows,
                      hidden, eps, dtype, stream, true, false);
}

AROPS_API arops_status arops_layernorm(const void* x, const void* gamma, const void* beta, void* y,
                                       int64_t rows, int64_t hidden, float eps, arops_dtype dtype,
                                       void* stream)
{
    return norm_entry("arops_layernorm", x, nullptr, nullptr, gamma, beta, y, rows, hidden, eps,
                      dtype, stream, false, true);
}

AROPS_API arops_status arops_add_layernorm(const void* x, const void* residual_in,
                                           void* residual_out, const void* gamma,
                                           const void* beta, void* y, int64_t rows,
                                           int64_t hidden, float eps, arops_dtype dtype,
                                           void* stream)
{
    return norm_entry("arops_add_layernorm", x, residual_in, residual_out, gamma, beta, y, rows,
                      hidden, eps, dtype, stream, true, true);
}

AROPS_API arops_status arops_mrope_qk(const void* q, const void* k, void* q_out, void* k_out,
                                      const int32_t* pos, int64_t tokens, int32_t n_q_heads,
                                      int32_t n_k_heads, int32_t head_dim,
                                      const int32_t* sections, float theta, arops_dtype dtype,
                                      void* stream)
{
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: unknown dtype %d", (int)dtype);
    if (tokens < 0 || n_q_heads < 0 || n_k_heads < 0)
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: negative size");
    if (head_dim <= 0 || head_dim % 2 != 0)
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: head_dim must be even and > 0 (got %d)",
                    (int)head_dim);
    if (head_dim > 512)
        return fail(AROPS_ERR_UNSUPPORTED, "arops_mrope_qk: head_dim %d > 512", (int)head_dim);
    if (!sections)
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: sections is null");
    if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 ||
        (int64_t)sections[0] + sections[1] + sections[2] != head_dim / 2)
        return fail(AROPS_ERR_INVALID,
                    "arops_mrope_qk: sections [%d,%d,%d] must be >= 0 and sum to head_dim/2 = %d",
                    (int)sections[0], (int)sections[1], (int)sections[2], (int)head_dim / 2);
    if (!(theta > 0.0f) || isinf(theta))
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: theta must be finite and > 0");
    if (tokens == 0 || n_q_heads + n_k_heads == 0)
        return ok();
    if (!pos || (n_q_heads > 0 && (!q || !q_out)) || (n_k_heads > 0 && (!k || !k_out)))
        return fail(AROPS_ERR_INVALID, "arops_mrope_qk: null pointer");
    MropeArgs a;
    a.q = q;
    a.k = k;
    a.q_out = q_out;
    a.k_out = k_out;
    a.pos = pos;
    a.tokens = tokens;
    a.n_q_heads = n_q_heads;
    a.n_k_heads = n_k_heads;
    a.head_dim = head_dim;
    a.sections[0] = sections[0];
    a.sections[1] = sections[1];
    a.sections[2] = sections[2];
    a.theta = theta;
    return from_cuda(launch_mrope(a, dtype, static_cast<cudaStream_t>(stream)), "arops_mrope_qk");
}

AROPS_API arops_status arops_mrope_kv_append(const void* q, const void* k, const void* v,
                                             void* q_out, void* k_cache, void* v_cache,
                                             const int32_t* pos, const int32_t* cache_loc,
                                             int64_t tokens, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, int64_t cache_rows, int64_t max_seq,
                                             const int32_t* sections, float theta,
                                             arops_dtype dtype, void* stream)
{
    const char* name = "arops_mrope_kv_append";
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "%s: unknown dtype %d", name, (int)dtype);
    if (tokens < 0 || n_q_heads < 0 || n_kv_heads < 0 || cache_rows < 0 || max_seq < 0)
        return fail(AROPS_ERR_INVALID, "%s: negative size", name);
    if (head_dim <= 0 || head_dim % 2 != 0)
        return fail(AROPS_ERR_INVALID, "%s: head_dim must be even and > 0 (got %d)", name,
                    (int)head_dim);
    if (head_dim > 512)
        return fail(AROPS_ERR_UNSUPPORTED, "%s: head_dim %d > 512", name, (int)head_dim);
    if (!sections)
        return fail(AROPS_ERR_INVALID, "%s: sections is null", name);
    if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 ||
        (int64_t)sections[0] + sections[1] + sections[2] != head_dim / 2)
        return fail(AROPS_ERR_INVALID, "%s: sections [%d,%d,%d] must be >= 0 and sum to %d", name,
                    (int)sections[0], (int)sections[1], (int)sections[2], (int)head_dim / 2);
    if (!(theta > 0.0f) || isinf(theta))
        return fail(AROPS_ERR_INVALID, "%s: theta must be finite and > 0", name);
    if (tokens == 0 || n_q_heads + n_kv_heads == 0)
        return ok();
    if (!pos || (n_q_heads > 0 && (!q || !q_out)) ||
        (n_kv_heads > 0 && (!k || !v || !k_cache || !v_cache || !cache_loc)))
        return fail(AROPS_ERR_INVALID, "%s: null pointer", name);
    if (k_cache == v_cache && n_kv_heads > 0)
        return fail(AROPS_ERR_INVALID, "%s: k_cache and v_cache are one buffer", name);
    MropeArgs a;
    a.q = q;
    a.k = k;
    a.q_out = q_out;
    a.k_out = nullptr;
    a.pos = pos;
    a.tokens = tokens;
    a.n_q_heads = n_q_heads;
    a.n_k_heads = n_kv_heads;
    a.head_dim = head_dim;
    a.sections[0] = sections[0];
    a.sections[1] = sections[1];
    a.sections[2] = sections[2];
    a.theta = theta;
    AppendArgs x;
    x.v = v;
    x.k_cache = k_cache;
    x.v_cache = v_cache;
    x.cache_loc = cache_loc;
    x.cache_rows = cache_rows;
    x.max_seq = max_seq;
    return from_cuda(launch_mrope_append(a, x, dtype, static_cast<cudaStream_t>(stream)), name);
}

AROPS_API arops_status arops_swiglu(const void* gate, const void* up, void* out, int64_t rows,
                                    int64_t inter, arops_dtype dtype, void* stream)
{
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "arops_swiglu: unknown dtype %d", (int)dtype);
    if (rows < 0 || inter <= 0 || (rows > 0 && inter > INT64_MAX / rows))
        return fail(AROPS_ERR_INVALID, "arops_swiglu: bad shape rows=%lld inter=%lld",
                    (long long)rows, (long long)inter);
    if (rows == 0)
        return ok();
    if (!gate || !up || !out)
        return fail(AROPS_ERR_INVALID, "arops_swiglu: null pointer");
    return from_cuda(launch_swiglu(gate, up, out, rows * inter, dtype,
                                   static_cast<cudaStream_t>(stream)),
                     "arops_swiglu");
}

}  // extern "C"

namespace {

arops_status topk_check(const char* name, int64_t rows, int64_t vocab, int32_t top_k,
                        float temperature)
{
    if (rows < 0 || vocab <= 0)
        return fail(AROPS_ERR_INVALID, "%s: bad shape rows=%lld vocab=%lld", name,
                    (long long)rows, (long long)vocab);
    if (top_k < 1 || top_k > vocab)
        return fail(AROPS_ERR_INVALID, "%s: top_k %d must be in [1, vocab]", name, (int)top_k);
    if (top_k > topk_max_k() || vocab > (int64_t)topk_max_slices() * 4096 || rows > 65535)
        return fail(AROPS_ERR_UNSUPPORTED,
                    "%s: supported top_k <= %d, vocab <= %d, rows <= 65535", name, topk_max_k(),
                    topk_max_slices() * 4096);
    if (!(temperature > 0.0f) || isinf(temperature))
        return fail(AROPS_ERR_INVALID, "%s: temperature must be finite and > 0", name);
    return AROPS_OK;
}

}  // namespace

extern "C" {

AROPS_API arops_status arops_topk_sample_workspace(int64_t rows, int64_t vocab, int32_t top_k,
                                                   size_t* bytes)
{
    if (!bytes)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample_workspace: bytes is null");
    const arops_status st = topk_check("arops_topk_sample_workspace", rows, vocab, top_k, 1.0f);
    if (st != AROPS_OK)
        return st;
    *bytes = topk_counter_bytes() +
             (size_t)rows * (size_t)topk_slices(vocab) * (size_t)top_k * sizeof(uint64_t);
    return ok();
}

AROPS_API arops_status arops_topk_sample_prepare(void* workspace, size_t workspace_bytes,
                                                 void* stream)
{
    if (!workspace)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample_prepare: workspace is null");
    if (workspace_bytes < topk_counter_bytes())
        return fail(AROPS_ERR_INVALID,
                    "arops_topk_sample_prepare: workspace of %zu bytes < the %zu bytes of counters",
                    workspace_bytes, topk_counter_bytes());
    return from_cuda(cudaMemsetAsync(workspace, 0, topk_counter_bytes(),
                                     static_cast<cudaStream_t>(stream)),
                     "arops_topk_sample_prepare");
}

AROPS_API arops_status arops_topk_sample(const void* logits, const float* gumbel,
                                         int32_t* token_out, float* prob_out, int64_t rows,
                                         int64_t vocab, int32_t top_k, float temperature,
                                         arops_dtype dtype, void* workspace,
                                         size_t workspace_bytes, void* stream)
{
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "arops_topk_sample: unknown dtype %d", (int)dtype);
    const arops_status st = topk_check("arops_topk_sample", rows, vocab, top_k, temperature);
    if (st != AROPS_OK)
        return st;
    if (rows == 0)
        return ok();
    if (!logits || !gumbel || !token_out || !prob_out || !workspace)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample: null pointer");
    const size_t need =
        topk_counter_bytes() + (size_t)rows * (size_t)topk_slices(vocab) * (size_t)top_k * 8u;
    if (workspace_bytes < need)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample: workspace of %zu bytes < %zu needed",
                    workspace_bytes, need);
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample: workspace not 16-byte aligned");
    return from_cuda(launch_topk_sample(logits, gumbel, token_out, prob_out, rows, vocab, top_k,
                                        temperature, dtype, workspace,
                                        static_cast<cudaStream_t>(stream)),
                     "arops_topk_sample");
}

AROPS_API arops_status arops_topk_sample_noalloc(const void* logits, const float* gumbel,
                                                 int32_t* token_out, float* prob_out,
                                                 int64_t rows, int64_t vocab, int32_t top_k,
                                                 float temperature, arops_dtype dtype,
                                                 void* stream)
{
    if (!valid_dtype(dtype))
        return fail(AROPS_ERR_INVALID, "arops_topk_sample_noalloc: unknown dtype %d", (int)dtype);
    const arops_status st =
        topk_check("arops_topk_sample_noalloc", rows, vocab, top_k, temperature);
    if (st != AROPS_OK)
        return st;
    const size_t need = (size_t)rows * (size_t)topk_slices(vocab) * (size_t)top_k * 8u;
    if (need > topk_noalloc_scratch_bytes())
        return fail(AROPS_ERR_UNSUPPORTED,
                    "arops_topk_sample_noalloc: this shape needs %zu bytes of scratch "
                    "(rows x ceil(vocab/4096) x top_k x 8) but the built-in array holds %zu; "
                    "use arops_topk_sample with a caller workspace",
                    need, topk_noalloc_scratch_bytes());
    // resolved before the rows == 0 return, so that a call with no rows is the
    // set-up call: it makes the current context load this code and its array
    void* scratch = nullptr;
    cudaError_t err = topk_noalloc_scratch(&scratch);
    if (err != cudaSuccess)
        return from_cuda(err, "arops_topk_sample_noalloc (scratch address)");
    if (rows == 0)
        return ok();
    if (!logits || !gumbel || !token_out || !prob_out)
        return fail(AROPS_ERR_INVALID, "arops_topk_sample_noalloc: null pointer");
    return from_cuda(launch_topk_sample(logits, gumbel, token_out, prob_out, rows, vocab, top_k,
                                        temperature, dtype, scratch,
                                        static_cast<cudaStream_t>(stream)),
                     "arops_topk_sample_noalloc");
}

AROPS_API arops_status arops_device_errors(uint32_t* errors, int clear)
{
    if (!errors)
        return fail(AROPS_ERR_INVALID, "arops_device_errors: errors is null");
    unsigned v = 0;
    cudaError_t err = cudaMemcpyFromSymbol(&v, g_device_errors, sizeof(v));
    if (err == cudaSuccess && clear) {
        const unsigned zero = 0;
        err = cudaMemcpyToSymbol(g_device_errors, &zero, sizeof(zero));
    }
    if (err != cudaSuccess)
        return from_cuda(err, "arops_device_errors");
    *errors = v;
    return ok();
}

AROPS_API arops_status arops_selftest_wait_timeout(uint64_t timeout_ns, int32_t* waited_out,
                                                   void* stream)
{
    if (!waited_out)
        return fail(AROPS_ERR_INVALID, "arops_selftest_wait_timeout: waited_out is null");
    if (timeout_ns == 0 || timeout_ns > 2000000000ull)
        return fail(AROPS_ERR_INVALID, "arops_selftest_wait_timeout: timeout must be in (0, 2 s]");
    return from_cuda(launch_wait_timeout_selftest(timeout_ns, waited_out,
                                                  static_cast<cudaStream_t>(stream)),
                     "arops_selftest_wait_timeout");
}

AROPS_API int arops_set_pdl(int enable)
{
    return g_pdl.exchange(enable ? 1 : 0);
}

AROPS_API int arops_set_streaming(int enable)
{
    return g_streaming.exchange(enable ? 1 : 0);
}

AROPS_API int arops_set_topk_cluster(int mode)
{
    return g_topk_cluster.exchange(mode < 0 ? 0 : (mode > 3 ? 3 : mode));
}

AROPS_API uint64_t arops_launch_count(void)
{
    return g_launches.load(std::memory_order_relaxed);
}

AROPS_API const char* arops_status_string(arops_status status)
{
    switch (status) {
    case AROPS_OK: return "ok";
    case AROPS_ERR_INVALID: return "invalid argument";
    case AROPS_ERR_UNSUPPORTED: return "unsupported size";
    case AROPS_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

AROPS_API const char* arops_last_error(void)
{
    return g_last_error;
}

AROPS_API int arops_version(void)
{
    return AROPS_VERSION;
}

}  // extern "C"
