// Fused softmax + top-k sampling over a row of logits (sm_100a).
//
// "Optimising autoregressive speech models", "Custom Triton kernels", item 2:
// every decode step ends in softmax and sampling; fusing them reads the logits
// once.  Per row: the candidates are the k largest logits ordered by (logit
// desc, index asc); rank j gets the caller's Gumbel(0,1) draw g[j]; the token
// is the candidate with the largest fl(fl(logit / T) + g[j]) (ties to the lower
// rank): Gumbel-max sampling from softmax(logits / T) restricted to the top k.
// prob_out is that token's probability under the same restricted softmax.
//
// Two kernels:
//   topk_slice_kernel   grid (slices, rows): a CTA turns its 4096-logit slice
//                       into 64-bit keys (order-preserving bits of the value,
//                       then the inverted index, so that larger keys are larger
//                       logits and, among equal logits, lower indices), sorts
//                       them in shared memory (bitonic network) and writes its
//                       k best keys to the workspace.
//   topk_sample_kernel  grid (rows): merges the slices' candidates the same
//                       way, then takes the sampling decision and the
//                       probability for its row.
// The workspace holds rows x slices x k keys; every slot is written before it
// is read, so it needs no clearing.
#include <math.h>

#include <atomic>

#include "common.cuh"

namespace arops {
namespace {

constexpr int kSlice = 4096;        // logits per slice
constexpr int kSliceThreads = 256;  // 16 logits per thread
constexpr int kMaxTopK = 64;
constexpr int kMaxSlices = 64;  // merged candidates: kMaxSlices * kMaxTopK = 4096 keys
constexpr int kMergeThreads = 512;

// IEEE float bits, reordered so that unsigned comparison follows the value.
__device__ __forceinline__ uint32_t order_bits(float v)
{
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float value_of(uint64_t key)
{
    const uint32_t o = (uint32_t)(key >> 32);
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

__device__ __forceinline__ int64_t index_of(uint64_t key)
{
    return (int64_t)(uint32_t)~(uint32_t)key;
}

__device__ __forceinline__ uint64_t make_key(float v, int64_t idx)
{
    return ((uint64_t)order_bits(v) << 32) | (uint64_t)(uint32_t)~(uint32_t)idx;
}

// Bitonic sort of n (a power of two) keys in shared memory, descending.
__device__ void sort_desc(uint64_t* keys, int n)
{
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
                // the pair (lo, hi) of comparator i at this stage
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = ((lo & size) == 0);
                const uint64_t a = keys[lo], b = keys[hi];
                if ((a < b) == desc) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
        }
    }
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kSliceThreads)
topk_slice_kernel(const T* __restrict__ logits, int64_t vocab, int k, int slices,
                  uint64_t* __restrict__ work)
{
    __shared__ uint64_t keys[kSlice];
    const int64_t row = blockIdx.y;
    const int64_t first = (int64_t)blockIdx.x * kSlice;
    const T* lr = logits + row * vocab;
    // the slice into L2 while the previous kernel drains, one line per thread
    {
        constexpr int kPerLine = 128 / sizeof(T);
        const int64_t n = (vocab - first < kSlice) ? vocab - first : kSlice;
        if ((int64_t)threadIdx.x * kPerLine < n)
            prefetch_l2_line(lr + first + (int64_t)threadIdx.x * kPerLine);
    }
    pdl_wait();
    pdl_allow_dependents();
    for (int i = threadIdx.x; i < kSlice; i += kSliceThreads) {
        const int64_t idx = first + i;
        keys[i] = (idx < vocab) ? make_key(load_elem(lr + idx), idx) : 0ull;  // 0: below any logit
    }
    sort_desc(keys, kSlice);
    uint64_t* out = work + (row * slices + blockIdx.x) * (int64_t)k;
    for (int j = threadIdx.x; j < k; j += kSliceThreads)
        out[j] = keys[j];
}

__global__ void __launch_bounds__(kMergeThreads)
topk_sample_kernel(const uint64_t* __restrict__ work, int slices, int k,
                   const float* __restrict__ gumbel, float temperature,
                   int32_t* __restrict__ token_out, float* __restrict__ prob_out)
{
    __shared__ uint64_t keys[kMaxSlices * kMaxTopK];
    __shared__ float e[kMaxTopK];
    const int64_t row = blockIdx.x;
    const int n = slices * k;
    int np2 = 1;
    while (np2 < n)
        np2 <<= 1;
    pdl_wait();
    pdl_allow_dependents();
    for (int i = threadIdx.x; i < np2; i += kMergeThreads)
        keys[i] = (i < n) ? work[row * n + i] : 0ull;
    sort_desc(keys, np2);

    // exp((l_j - l_0) / T) for the k candidates
    const float l0 = value_of(keys[0]);
    for (int j = threadIdx.x; j < k; j += kMergeThreads)
        e[j] = expf((value_of(keys[j]) - l0) / temperature);
    __syncthreads();
    if (threadIdx.x == 0) {
        int best = 0;
        float best_score = 0.f, z = 0.f;
        for (int j = 0; j < k; ++j) {
            // fl(fl(l / T) + g), two correctly rounded operations
            const float score = __fadd_rn(__fdiv_rn(value_of(keys[j]), temperature),
                                          gumbel[row * k + j]);
            if (j == 0 || score > best_score) {
                best = j;
                best_score = score;
            }
            z += e[j];
        }
        token_out[row] = (int32_t)index_of(keys[best]);
        prob_out[row] = e[best] / z;
    }
}

}  // namespace

int topk_slices(int64_t vocab)
{
    return (int)ceil_div(vocab, kSlice);
}

int topk_max_k()
{
    return kMaxTopK;
}

int topk_max_slices()
{
    return kMaxSlices;
}

cudaError_t launch_topk_sample(const void* logits, const float* gumbel, int32_t* token_out,
                               float* prob_out, int64_t rows, int64_t vocab, int k,
                               float temperature, arops_dtype dtype, uint64_t* work,
                               cudaStream_t stream)
{
    const int slices = topk_slices(vocab);
    const dim3 grid1((unsigned)slices, (unsigned)rows);
    cudaError_t err;
    if (dtype == AROPS_BF16)
        err = launch(topk_slice_kernel<__nv_bfloat16>, grid1, dim3(kSliceThreads), 0, stream,
                     static_cast<const __nv_bfloat16*>(logits), vocab, k, slices, work);
    else
        err = launch(topk_slice_kernel<float>, grid1, dim3(kSliceThreads), 0, stream,
                     static_cast<const float*>(logits), vocab, k, slices, work);
    if (err != cudaSuccess)
        return err;
    return launch(topk_sample_kernel, dim3((unsigned)rows), dim3(kMergeThreads), 0, stream,
                  (const uint64_t*)work, slices, k, gumbel, temperature, token_out, prob_out);
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the workspace lives in this file-scope device
// array instead of caller memory.  It exists for callers that cannot allocate
// device memory themselves, e.g. code running inside a host application's
// real-time audio or streaming callback, where cudaMalloc is off limits
// because it can block and synchronise the device, or a plugin that is handed
// buffers by a host application that owns all device memory.  Every GPU that
// loads the library holds this array until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB

static __device__ __align__(256) uint64_t g_topk_scratch[kNoAllocScratchBytes / sizeof(uint64_t)];

namespace {
constexpr int kScratchDevices = 64;
std::atomic<uint64_t*> g_topk_scratch_addr[kScratchDevices];
}  // namespace

size_t topk_noalloc_scratch_bytes()
{
    return kNoAllocScratchBytes;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
cudaError_t topk_noalloc_scratch(uint64_t** ptr)
{
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess)
        return err;
    if (dev < 0 || dev >= kScratchDevices)
        return cudaErrorInvalidDevice;
    uint64_t* p = g_topk_scratch_addr[dev].load();
    if (p == nullptr) {
        err = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_topk_scratch);
        if (err != cudaSuccess)
            return err;
        g_topk_scratch_addr[dev].store(p);
    }
    *ptr = p;
    return cudaSuccess;
}

}  // namespace arops
