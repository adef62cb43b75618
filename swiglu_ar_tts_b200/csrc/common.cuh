// Shared device helpers for the decode-operator kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <string>

#include "arops.h"

namespace arops {

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PDL).  griddepcontrol.wait blocks until the
// preceding grid on the stream has completed and its memory is visible; it is
// a no-op when the kernel was launched without the PDL attribute.
// griddepcontrol.launch_dependents lets the next PDL kernel be scheduled early.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_allow_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Hint to bring [p, p + bytes) into L2 (one bulk prefetch; p and bytes must be
// multiples of 16).  Issued before pdl_wait() to overlap a kernel's first DRAM
// reads with its predecessor: L2 is the point of coherence for global memory,
// so a prefetch can never make a later load see stale data.  (No L1 prefetch is
// ever issued before the wait, since L1 is not coherent.)
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Hint to bring the 128-byte line holding p into L2 (any alignment).
__device__ __forceinline__ void prefetch_l2_line(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ORs `bits` into the library's device error word (a file-scope __device__
// variable whose address kernels receive as a parameter; device_error_word()).
__device__ __forceinline__ void record_device_error(unsigned* word, unsigned bits)
{
    atomicOr(word, bits);
}

// ---------------------------------------------------------------------------
// 16-byte vectors of the storage type, unpacked to / packed from fp32.
// ---------------------------------------------------------------------------
template <typename T>
struct Vec;

template <>
struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f)
    {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* f)
    {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

// bf16 is the top half of an fp32 word, so widening is a shift; narrowing is
// the hardware round-to-nearest-even conversion of two floats at once.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4& v, float* f)
    {
        f[0] = __uint_as_float(v.x << 16);
        f[1] = __uint_as_float(v.x & 0xFFFF0000u);
        f[2] = __uint_as_float(v.y << 16);
        f[3] = __uint_as_float(v.y & 0xFFFF0000u);
        f[4] = __uint_as_float(v.z << 16);
        f[5] = __uint_as_float(v.z & 0xFFFF0000u);
        f[6] = __uint_as_float(v.w << 16);
        f[7] = __uint_as_float(v.w & 0xFFFF0000u);
    }
    __device__ __forceinline__ static uint4 pack(const float* f)
    {
        return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
};

// Scalar element access for the unaligned / ragged kernels.
__device__ __forceinline__ float load_elem(const float* p) { return *p; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ float round_to(float v, const float*) { return v; }
__device__ __forceinline__ float round_to(float v, const __nv_bfloat16*)
{
    return __bfloat162float(__float2bfloat16_rn(v));
}

// Streaming 16-byte loads/stores: data is touched once, so ask the caches to
// evict it first.  These are coherent loads (not the read-only path) because
// outputs may alias inputs.
__device__ __forceinline__ uint4 ld_stream(const void* p)
{
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void st_stream(void* p, const uint4& v)
{
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// Output store of a kernel that streams (STREAM) or of a latency-bound launch
// of a few KB to a few MB whose output the next kernel reads at once: there a
// plain write-back store measured ~3% less time per launch on B200 than the
// evict-first one in chains of dependent decode-size launches.
template <bool STREAM>
__device__ __forceinline__ void st_out(void* p, const uint4& v)
{
    if constexpr (STREAM)
        __stcs(reinterpret_cast<uint4*>(p), v);
    else
        *reinterpret_cast<uint4*>(p) = v;
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
struct DeviceInfo {
    int sm_count;
};

// SM count of the current device (queried once per device).
cudaError_t current_device_info(DeviceInfo* info);

// Device address of the library's error word in the current context (looked
// up with cudaGetSymbolAddress on every call).
cudaError_t device_error_word(unsigned** word);

// Whether kernels are launched with the PDL attribute.
bool pdl_enabled();

// Whether the shared-memory streaming (bulk-copy) kernels may be chosen.
bool streaming_enabled();

// Counts one launch.
void count_launch();

// Launches `kernel` on `stream`, with the PDL attribute when enabled.
template <typename... Params, typename... Args>
cudaError_t launch(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl_enabled()) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 1;
    }
    cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
    if (err == cudaSuccess)
        count_launch();
    return err;
}

inline bool aligned16(const void* p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline int64_t ceil_div(int64_t a, int64_t b)
{
    return (a + b - 1) / b;
}

__host__ __device__ inline uint32_t round_up(uint32_t a, uint32_t b)
{
    return (a + b - 1) / b * b;
}

// Shared memory an SM offers to one CTA / to all its CTAs (B200: 227 / 228 KB).
constexpr uint32_t kMaxSmemPerCta = 227u * 1024u;
constexpr uint32_t kSmemPerSm = 228u * 1024u;

// Resident CTAs per SM for `kernel` at this block size and dynamic smem.  For
// kernels that use dynamic shared memory it first raises the kernel's limit
// (above the 48 KB default) and asks for the largest shared-memory carveout:
// otherwise the driver may configure only as much shared memory as one CTA
// needs, and the CTAs the grid was sized for would run in waves.
template <typename K>
cudaError_t resident_ctas(K kernel, int threads, size_t smem, int* ctas)
{
    if (smem > 0) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess)
            return e;
    }
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, kernel, threads, smem);
}

// CTAs of `Kernel` (at `threads` threads per CTA, no dynamic shared memory)
// that `waves` full waves fill on a device of `sm_count` SMs.  The resident
// CTAs per SM are looked up once per kernel (every device this library runs on
// is the same part); a failed lookup counts one per SM.
template <auto Kernel>
int64_t wave_ctas(int threads, int sm_count, int waves)
{
    static std::atomic<int> per_sm{0};
    int v = per_sm.load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, Kernel, threads, 0) != cudaSuccess ||
            v < 1)
            v = 1;
        per_sm.store(v, std::memory_order_relaxed);
    }
    return (int64_t)v * sm_count * waves;
}

// Launchers (one per operator), called after argument validation.
// residual_in == nullptr: no residual add; beta == nullptr: RMSNorm, else LayerNorm.
cudaError_t launch_norm(const void* x, const void* residual_in, void* residual_out,
                        const void* gamma, const void* beta, void* y, int64_t rows,
                        int64_t hidden, float eps, arops_dtype dtype, cudaStream_t stream);

cudaError_t launch_swiglu(const void* gate, const void* up, void* out, int64_t n,
                          arops_dtype dtype, cudaStream_t stream);

struct MropeArgs {
    const void* q;
    const void* k;
    void* q_out;
    void* k_out;
    const int32_t* pos;
    int64_t tokens;
    int32_t n_q_heads;
    int32_t n_k_heads;
    int32_t head_dim;
    int32_t sections[3];
    float theta;
};

cudaError_t launch_mrope(const MropeArgs& a, arops_dtype dtype, cudaStream_t stream);

// M-RoPE fused with the KV-cache append (mrope.cu).
struct AppendArgs {
    const void* v;
    void* k_cache;  // [cache_rows, n_k_heads, max_seq, head_dim]
    void* v_cache;
    const int32_t* cache_loc;  // [2, tokens]: cache row, position
    int64_t cache_rows;
    int64_t max_seq;
};
cudaError_t launch_mrope_append(const MropeArgs& a, const AppendArgs& x, arops_dtype dtype,
                                cudaStream_t stream);

// Fused softmax + top-k sampling (topk.cu).  The workspace starts with
// topk_counter_bytes() of per-row arrival counters (zero between calls), then
// rows x slices x k candidate keys of 8 bytes.
int topk_slices(int64_t vocab);
int topk_max_k();
int topk_max_slices();
size_t topk_counter_bytes();
cudaError_t launch_topk_sample(const void* logits, const float* gumbel, int32_t* token_out,
                               float* prob_out, int64_t rows, int64_t vocab, int k,
                               float temperature, arops_dtype dtype, void* workspace,
                               cudaStream_t stream);
// Self-test of the bounded mbarrier wait (selftest.cu).
cudaError_t launch_wait_timeout_selftest(uint64_t timeout_ns, int* waited_out,
                                         cudaStream_t stream);

// The allocation-free variant's built-in scratch array: the candidate bytes it
// holds (after its counters), and its device address in the current context.
size_t topk_noalloc_scratch_bytes();
cudaError_t topk_noalloc_scratch(void** ptr);

}  // namespace arops
