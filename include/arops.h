/*
 * arops.h: per-token operators of autoregressive speech-model decode, as a C ABI.
 *
 * Four operators, each one hand-written CUDA kernel for NVIDIA B200 (sm_100a):
 *
 *   arops_rmsnorm      y = gamma * x / sqrt(mean(x^2) + eps)
 *                      ("Optimising autoregressive speech models", §09
 *                      "LayerNorm -> RMSNorm": the RMSNorm equation and module)
 *   arops_add_rmsnorm  residual_out = x + residual_in (rounded to the dtype);
 *                      y = RMSNorm(residual_out)
 *                      ("Norm+Residual" in section 3 of the Triton kernel-fusion
 *                      post for Qwen3-TTS, news.hada.io topic 27742)
 *   arops_mrope_qk     multi-section rotary embedding of q and k
 *                      ("M-RoPE" in the same section; rotation of q/k in the
 *                      complex plane per forpes.ru post 233929, "Stage 2")
 *   arops_swiglu       out = silu(gate) * up, silu(g) = g / (1 + e^-g)
 *                      ("SwiGLU" in the same section)
 *
 * Conventions shared by every call:
 *   - All tensor pointers are caller-owned DEVICE memory, dense and row-major.
 *     The library allocates and frees nothing and keeps no pointer after the
 *     call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Every call is asynchronous on that stream: it validates its
 *     arguments on the host, enqueues one kernel and returns; it never
 *     synchronises.  Faults inside a kernel surface at the caller's next
 *     synchronisation, as with any CUDA library.
 *   - The device is the caller's current CUDA device.
 *   - A zero-sized problem (rows == 0, tokens == 0) is a no-op returning
 *     AROPS_OK; its pointers are not inspected.
 *   - Argument errors (null pointer, bad dtype, bad shape, eps < 0, ...) return
 *     AROPS_ERR_INVALID (or AROPS_ERR_UNSUPPORTED for valid but unimplemented
 *     sizes) before anything is launched.  A failed launch returns
 *     AROPS_ERR_CUDA.  arops_last_error() then gives a one-line reason.
 *   - Arithmetic is fp32 in registers whatever the storage dtype; each output
 *     is rounded once, round-to-nearest-even, to the storage dtype.
 *   - Pointers need not be aligned: 16-byte-aligned buffers whose row length is
 *     a multiple of 16 bytes take the vectorised kernels, anything else takes an
 *     element-wise kernel on the GPU with the same results.
 *   - An output may be the same buffer as an input of the same shape (in-place);
 *     partially overlapping buffers are undefined.
 *   - No C++ exception crosses this boundary.
 */
#ifndef AROPS_H
#define AROPS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define AROPS_API __attribute__((visibility("default")))
#else
#define AROPS_API
#endif

typedef enum {
    AROPS_OK = 0,
    AROPS_ERR_INVALID = 1,     /* bad argument; nothing was launched */
    AROPS_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim > 512) */
    AROPS_ERR_CUDA = 3         /* the CUDA runtime reported an error at launch */
} arops_status;

typedef enum {
    AROPS_F32 = 0,  /* IEEE binary32 storage */
    AROPS_BF16 = 1  /* bfloat16 storage */
} arops_dtype;

/*
 * RMSNorm over the last dimension ("Optimising autoregressive speech models",
 * §09: gamma * x / sqrt(mean(x^2) + eps), eps inside the root, the mean over the
 * row, a per-channel weight).
 *   x     [rows, hidden]  dtype      input
 *   gamma [hidden]        dtype      per-channel weight
 *   y     [rows, hidden]  dtype      output (may be x)
 *   eps >= 0 (1e-6 in the pages' module).  A zero row gives y = 0 for eps > 0;
 *   eps == 0 on a zero row gives NaN, as the formula does.
 * The sum of squares is accumulated in fp32.
 */
AROPS_API arops_status arops_rmsnorm(const void* x, const void* gamma, void* y,
                                     int64_t rows, int64_t hidden, float eps,
                                     arops_dtype dtype, void* stream);

/*
 * Fused residual add + RMSNorm ("Norm+Residual", Triton kernel-fusion post for
 * Qwen3-TTS, section 3), in one pass over memory:
 *   residual_out = round_dtype(x + residual_in)
 *   y            = RMSNorm(residual_out) with weight gamma
 * i.e. exactly "add, then normalise" on dtype tensors: the norm sees the
 * rounded residual that is written back.
 *   x, residual_in, residual_out, y: [rows, hidden] dtype; gamma: [hidden] dtype.
 *   residual_out may be residual_in (the usual in-place update of the residual
 *   stream); y may be x.
 */
AROPS_API arops_status arops_add_rmsnorm(const void* x, const void* residual_in,
                                         void* residual_out, const void* gamma, void* y,
                                         int64_t rows, int64_t hidden, float eps,
                                         arops_dtype dtype, void* stream);

/*
 * LayerNorm over the last dimension ("Optimising autoregressive speech models",
 * §09, the LayerNorm equation): y = gamma * (x - mean) / sqrt(var + eps) + beta,
 * mean and population variance over the row.  The variance is taken from the
 * row's deviations (a second reduction over the row held in registers), not
 * from E[x^2] - E[x]^2.  Layout and conventions as arops_rmsnorm; beta is
 * [hidden] dtype.  This is the norm that the pages' §09 replaces by RMSNorm;
 * it is here to measure that swap.
 */
AROPS_API arops_status arops_layernorm(const void* x, const void* gamma, const void* beta, void* y,
                                       int64_t rows, int64_t hidden, float eps,
                                       arops_dtype dtype, void* stream);

/*
 * Residual add + LayerNorm: residual_out = round_dtype(x + residual_in),
 * y = LayerNorm(residual_out) (the LayerNorm counterpart of arops_add_rmsnorm).
 */
AROPS_API arops_status arops_add_layernorm(const void* x, const void* residual_in,
                                           void* residual_out, const void* gamma,
                                           const void* beta, void* y, int64_t rows,
                                           int64_t hidden, float eps, arops_dtype dtype,
                                           void* stream);

/*
 * Multi-section rotary embedding (M-RoPE) of q and k, rotate-half pairing.
 * ("M-RoPE" in the Triton kernel-fusion post, section 3; RoPE as a rotation of
 * Q and K in the complex plane, forpes.ru post 233929, "Stage 2".)
 *
 * For every token t, head h and pair index j in [0, head_dim/2):
 *   row  = 0 if j < sections[0], 1 if j < sections[0] + sections[1], else 2
 *   p    = pos[row * tokens + t]                      (rows t, h, w of the ids)
 *   phi  = p * theta^(-2 j / head_dim)
 *   (a, b) = (x[j], x[j + head_dim/2])
 *   out[j] = a cos(phi) - b sin(phi),  out[j + head_dim/2] = b cos(phi) + a sin(phi)
 *
 *   q, q_out [tokens, n_q_heads, head_dim] dtype (q_out may be q)
 *   k, k_out [tokens, n_k_heads, head_dim] dtype (k_out may be k)
 *   pos      [3, tokens] int32 device array (rows t, h, w)
 *   sections HOST array of 3 non-negative int32 summing to head_dim / 2
 *   head_dim even, 2 <= head_dim <= 512; theta > 0 and finite.
 *   n_k_heads may be 0 (k, k_out ignored); likewise n_q_heads.
 * The angle is formed and reduced modulo 2*pi in fp64, then cos/sin are taken
 * in fp32, per (token, j), in registers: no cos/sin table is read.
 */
AROPS_API arops_status arops_mrope_qk(const void* q, const void* k, void* q_out, void* k_out,
                                      const int32_t* pos, int64_t tokens,
                                      int32_t n_q_heads, int32_t n_k_heads, int32_t head_dim,
                                      const int32_t* sections, float theta,
                                      arops_dtype dtype, void* stream);

/*
 * M-RoPE fused with the KV-cache append ("Optimising autoregressive speech
 * models", "Custom Triton kernels", item 3: insert the new K, V of a token at
 * its position in a cache laid out [head, position, head_dim] per sequence).
 * In one pass: q is rotated into q_out exactly as arops_mrope_qk does; k is
 * rotated the same way and written straight into its cache slot; v is copied
 * into its slot.  Token t's slot is (cache_loc[t], cache_loc[tokens + t]) =
 * (cache row, position).
 *   q, q_out      [tokens, n_q_heads, head_dim] dtype
 *   k, v          [tokens, n_kv_heads, head_dim] dtype
 *   k_cache, v_cache [cache_rows, n_kv_heads, max_seq, head_dim] dtype
 *   pos           [3, tokens] int32 (rows t, h, w); cache_loc [2, tokens] int32
 *   sections/theta/head_dim as for arops_mrope_qk.
 * A token whose cache row or position is out of range writes no cache slot
 * (its q is still rotated) and sets AROPS_DEVICE_ERR_BAD_INDEX in the device
 * error word.  Slots not named by cache_loc are left untouched.  Two tokens
 * naming one slot race.
 */
#define AROPS_DEVICE_ERR_BAD_INDEX 2u
AROPS_API arops_status arops_mrope_kv_append(const void* q, const void* k, const void* v,
                                             void* q_out, void* k_cache, void* v_cache,
                                             const int32_t* pos, const int32_t* cache_loc,
                                             int64_t tokens, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, int64_t cache_rows, int64_t max_seq,
                                             const int32_t* sections, float theta,
                                             arops_dtype dtype, void* stream);

/*
 * SwiGLU activation ("SwiGLU" in the Triton kernel-fusion post, section 3):
 *   out = silu(gate) * up,  silu(g) = g / (1 + e^-g), computed in fp32.
 *   gate, up, out: [rows, inter] dtype, separate tensors (out may be gate or up).
 */
AROPS_API arops_status arops_swiglu(const void* gate, const void* up, void* out,
                                    int64_t rows, int64_t inter,
                                    arops_dtype dtype, void* stream);

/*
 * Fused softmax + top-k sampling ("Optimising autoregressive speech models",
 * "Custom Triton kernels", item 2: scale logits by 1/temperature, softmax,
 * sample from the top k; done in one pass over the logits).
 *
 * For each row: the candidates are the top_k largest logits, ordered by logit
 * (descending) then index (ascending); candidate j (0 = largest) is given the
 * caller's Gumbel(0,1) draw gumbel[row * top_k + j]; the sampled token is the
 * candidate with the largest fl32(fl32(logit / temperature) + draw) (ties to
 * the lower j).  That is Gumbel-max sampling from softmax(logits/temperature)
 * restricted to the top_k candidates; the caller owns the randomness.
 *   logits     [rows, vocab] dtype (no NaNs)
 *   gumbel     [rows, top_k] float32 device array
 *   token_out  [rows] int32: vocabulary index of the sampled token
 *   prob_out   [rows] float32: its probability under the restricted softmax
 *   1 <= top_k <= min(64, vocab), vocab <= 262144, rows <= 65535,
 *   temperature > 0 and finite.
 *   workspace  device scratch of at least arops_topk_sample_workspace() bytes
 *              (16-byte aligned, caller-owned).  It starts with 256 KiB of
 *              per-row arrival counters that must be zero when a call begins:
 *              clear them once after allocating the workspace, with
 *              arops_topk_sample_prepare (or any zero fill of the first 256
 *              KiB); every call leaves them zero again, for any later shape.
 *              The rest holds candidates and needs no initialisation.  Two
 *              calls in flight at once must not share one workspace.
 * One kernel is enqueued on `stream`, by default (arops_set_topk_cluster) a
 * single-pass cluster kernel: a thread-block cluster per row whose CTAs
 * select the row's top_k together through each other's shared memory, the
 * cluster's first CTA ranking them and taking the decision, touching no
 * workspace byte.  A call whose rows' clusters of up to 16 CTAs all fit on
 * the device at once (a few rows: 7 of 151936 logits on a B200) holds the
 * logits in registers; larger calls use clusters of up to 8 CTAs holding
 * chunks of up to ~76 KB of logits in shared memory, many rows at once.
 * Calls with more rows than a quarter of the device's SMs whose rows start on
 * 16-byte boundaries and hold whole 16-byte vectors take the streaming
 * kernel instead: one CTA a row (a grid of at most one CTA an SM walking the
 * rows), the row read once through shared memory by bulk copies against a
 * running floor, no workspace byte touched either.
 * Where none can run (or arops_set_topk_cluster(0)) it is the slice
 * kernel: each 4096-logit slice's CTA writes its top_k candidates to the
 * workspace, and the last CTA of a row to finish (counted on the row's
 * arrival counter) merges them and takes the decision; no CTA waits for
 * another.  All four give identical results.  A bulk copy of the streaming
 * kernel that does not land within a second sets AROPS_DEVICE_ERR_TIMEOUT
 * (bit 1 of the device error word) and its CTA abandons its rows.  A counter found non-zero at the start of a slice-kernel call (a
 * workspace that was not cleared) sets AROPS_DEVICE_ERR_WORKSPACE in the
 * device error word, and that row's outputs are then undefined.
 */
#define AROPS_DEVICE_ERR_WORKSPACE 4u
AROPS_API arops_status arops_topk_sample_workspace(int64_t rows, int64_t vocab, int32_t top_k,
                                                   size_t* bytes);
/* Clears the arrival counters of a new workspace (a zero fill of its first
 * 256 KiB enqueued on `stream`); workspace_bytes must cover them. */
AROPS_API arops_status arops_topk_sample_prepare(void* workspace, size_t workspace_bytes,
                                                 void* stream);
AROPS_API arops_status arops_topk_sample(const void* logits, const float* gumbel,
                                         int32_t* token_out, float* prob_out, int64_t rows,
                                         int64_t vocab, int32_t top_k, float temperature,
                                         arops_dtype dtype, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * arops_topk_sample without a workspace argument: the same computation and
 * results, with the scratch taken from an array that the library itself holds
 * in device memory (a file-scope __device__ array of 1.25 MiB: 256 KiB of
 * arrival counters, zero when the library's device code is loaded, then 1 MiB
 * of candidates; every GPU that loads the library keeps it until the process
 * exits).  The paper has no
 * counterpart: it is here for callers that cannot allocate device memory,
 * such as code running inside a host application's real-time audio or
 * streaming callback, where cudaMalloc is not allowed because it can block
 * and synchronise the device, or a plugin that only receives buffers from a
 * host that owns all device memory.  This entry point calls no cudaMalloc,
 * cudaFree or other allocating routine (the one-time module load of the
 * set-up call below aside).
 *   - Limit: rows * ceil(vocab / 4096) * top_k * 8 bytes must not exceed 1 MiB
 *     (e.g. vocab 151936, top_k 50: up to 68 rows); larger shapes return
 *     AROPS_ERR_UNSUPPORTED with the numbers in arops_last_error(), before
 *     anything is launched.
 *   - The array has one instance per CUDA context.  Every call looks up its
 *     address in the caller's current context (cudaGetSymbolAddress), so a
 *     context the caller created itself, or a primary context that was reset
 *     and created anew, gets its own instance.
 *   - Set-up: a call with rows == 0 launches nothing but performs that lookup;
 *     the first lookup in a context loads the library's device code there
 *     (CUDA loads modules lazily by default), which reserves the array and may
 *     synchronise the device.  Callers whose later calls run where that is not
 *     allowed (a real-time callback) make one such call per context at set-up,
 *     outside that path and before any stream capture.  After it, calls
 *     allocate nothing and call no allocating routine.
 *   - All calls share the one array and it keeps the previous call's contents:
 *     the counters start at zero and every call leaves them zero, and every
 *     candidate slot a call reads is written earlier in that same call.  Calls
 *     whose kernels overlap on the GPU (different streams, different host
 *     threads) race on the array: serialise them, e.g. by issuing them on one
 *     stream.
 */
AROPS_API arops_status arops_topk_sample_noalloc(const void* logits, const float* gumbel,
                                                 int32_t* token_out, float* prob_out,
                                                 int64_t rows, int64_t vocab, int32_t top_k,
                                                 float temperature, arops_dtype dtype,
                                                 void* stream);

/*
 * Library controls and diagnostics follow.  They are this library's own
 * mechanisms; the pages define no such calls.
 *
 * Programmatic dependent launch.  The Triton kernel-fusion post for Qwen3-TTS
 * (section 3) reaches its end-to-end result by pairing its fused kernels with a
 * CUDA-graph decoder; this is the launch-level counterpart for chains of small
 * kernels.  When enabled (process-wide, default off), every kernel is launched
 * with the programmatic-stream-serialisation attribute so that it can be
 * scheduled while the previous kernel on the stream drains; each kernel waits
 * for its predecessor's memory before it reads activations or writes anything,
 * so results and stream-order semantics are unchanged.  It only shortens the
 * gaps between back-to-back launches (decode steps).
 * Contract while enabled: some read-only parameters are read before that
 * wait, so they must not be written by the kernel launched immediately before
 * on the same stream (kernels launched earlier have completed by then): gamma
 * and beta of the norms, and pos of arops_mrope_qk.  Model weights, and
 * position ids written ahead of a decode step, meet it.  Returns the old
 * setting.
 */
AROPS_API int arops_set_pdl(int enable);

/*
 * Kernel family selection (process-wide).  Disabled (the default), every
 * operator runs its register kernel: 16-byte coalesced loads straight into
 * registers.  Enabled, 16-byte-aligned rows go to the streaming kernels, which
 * stage data through shared memory with bulk asynchronous copies (TMA) under
 * time-bounded mbarrier waits.  Both families compute the same results within
 * the stated tolerance (the norm kernels may differ in the last bit, as their
 * sums of squares are accumulated in a different order); on B200 the register
 * kernels measured as fast or faster for every operator, so streaming is kept
 * as an option for measurement.  Returns the old setting.
 */
AROPS_API int arops_set_streaming(int enable);

/*
 * Top-k sampling kernel selection (process-wide): 0 = the slice kernel for
 * every call; 1 (the default) = the cluster kernels as described at
 * arops_topk_sample (registers for few rows, shared memory for many); 2 = the
 * shared-memory cluster kernel for every call; 3 = the streaming kernel (one
 * CTA a row, the row streamed once through shared memory) for every call
 * whose rows are 16-byte aligned, else as 2.  Other values are clamped.
 * Every kernel gives identical results; the control exists for measurement
 * and testing.  Returns the old setting.
 */
AROPS_API int arops_set_topk_cluster(int mode);

/*
 * Device-side error bits of the current device, OR-ed by kernels that abandon
 * part of their work: AROPS_DEVICE_ERR_TIMEOUT means a bulk copy into shared
 * memory did not complete within a second (the kernel's outputs are then
 * undefined); AROPS_DEVICE_ERR_BAD_INDEX (see arops_mrope_kv_append) means a
 * token's cache slot was out of range and was not written;
 * AROPS_DEVICE_ERR_WORKSPACE (see arops_topk_sample) means a sampling
 * workspace's counters were not cleared.  The call
 * synchronises the device (it is a plain copy from device memory) and, if
 * `clear` is non-zero, resets the bits.  Healthy runs always read 0.
 */
#define AROPS_DEVICE_ERR_TIMEOUT 1u
AROPS_API arops_status arops_device_errors(uint32_t* errors, int clear);

/*
 * Self-test of the bounded waits used by the streaming kernels: launches one
 * thread that waits, with limit `timeout_ns` (at most 2 s), for 16 bytes of a
 * bulk copy that is never issued.  The wait must run out: the kernel writes 1
 * to *waited_out (a device int32), sets AROPS_DEVICE_ERR_TIMEOUT and returns,
 * and the context stays usable.  Nothing else is launched or touched.
 */
AROPS_API arops_status arops_selftest_wait_timeout(uint64_t timeout_ns, int32_t* waited_out,
                                                   void* stream);

/* Number of kernels this library has launched in this process (all devices). */
AROPS_API uint64_t arops_launch_count(void);

/* Static string for a status code; never NULL. */
AROPS_API const char* arops_status_string(arops_status status);

/* Reason for the last non-OK status returned on the calling thread ("" if none). */
AROPS_API const char* arops_last_error(void);

/* ABI version of this header: major * 10000 + minor * 100 + patch. */
AROPS_API int arops_version(void);

#define AROPS_VERSION 20200

#ifdef __cplusplus
}
#endif

#endif /* AROPS_H */
