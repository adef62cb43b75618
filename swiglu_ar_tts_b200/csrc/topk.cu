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
// One kernel, grid (slices, rows).  A CTA turns its 4096-logit slice into
// keys (order-preserving bits of the value, then the inverted position, so
// that larger keys are larger logits and, among equal logits, lower indices:
// every key is distinct; 32 bits for bf16, 48 for fp32), finds its k largest
// with a block-wide select in registers and shared memory (select_top_k
// below), and writes them to the workspace as (value bits, inverted 24-bit
// vocabulary index) keys.  It then arrives on its row's counter; the CTA that
// arrives last (it sees slices - 1 earlier arrivals) resets the counter to 0,
// selects the row's k largest among the slices' candidates the same way, ranks
// those k by counting, and takes the sampling decision and the probability.
// No CTA waits for another: the others simply exit.
//
// Workspace: a fixed region of per-row arrival counters (kCounterBytes; they
// must be zero before a workspace's first call and every call leaves the ones
// it used at zero), then rows x slices x k candidate keys, every one written
// before it is read.
#include <math.h>

#include <type_traits>

#include "common.cuh"

namespace arops {
namespace {

constexpr int kSlice = 4096;        // logits per slice
constexpr int kSliceThreads = 512;  // 8 logits per thread
constexpr int kMaxTopK = 64;
constexpr int kMaxSlices = 64;  // merged candidates: kMaxSlices * kMaxTopK = 4096 keys
constexpr int kMergeThreads = kSliceThreads;  // the last slice CTA of a row merges
constexpr int kMaxRows = 65535;                 // grid y
// Arrival counters at the start of the workspace, one per row up to kMaxRows
// (so every shape finds them at the same place), padded to 256 KiB.
constexpr size_t kCounterBytes = size_t(1) << 18;
static_assert(kCounterBytes >= sizeof(unsigned) * kMaxRows, "a counter per row");
constexpr unsigned kDeviceErrWorkspace = 4u;  // a counter was not zero when a call began

// atomicAdd with release and acquire semantics at GPU scope.
__device__ __forceinline__ unsigned atomic_add_acq_rel_gpu(unsigned* p, unsigned v)
{
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// IEEE float bits, reordered so that unsigned comparison follows the value.
__device__ __forceinline__ uint32_t order_bits(float v)
{
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float from_order_bits(uint32_t o)
{
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Keys of the storage type T: the value's order bits, of which a bf16 needs
// only the top 16 (its low 16 are 0 for positive and 1 for negative values).
template <typename T>
struct KeyBits;
template <>
struct KeyBits<float> {
    static constexpr int V = 32;
    __device__ static uint32_t of(float v) { return order_bits(v); }
    __device__ static float value(uint32_t k) { return from_order_bits(k); }
};
template <>
struct KeyBits<__nv_bfloat16> {
    static constexpr int V = 16;
    __device__ static uint32_t of(float v) { return order_bits(v) >> 16; }
    __device__ static float value(uint32_t k)
    {
        return from_order_bits((k << 16) | ((k & 0x8000u) ? 0u : 0xFFFFu));
    }
};

// Candidate keys: value bits above the inverted vocabulary index (24 bits:
// vocab <= 2^18 < 2^24), so larger keys are larger logits and, among equal
// logits, lower indices; every key is distinct and 0 is below every logit.
constexpr int kIndexBits = 24;
template <typename T>
__device__ __forceinline__ uint64_t cand_key(float v, int64_t idx)
{
    return ((uint64_t)KeyBits<T>::of(v) << kIndexBits) |
           (uint64_t)((1u << kIndexBits) - 1u - (uint32_t)idx);
}
template <typename T>
__device__ __forceinline__ float cand_value(uint64_t key)
{
    return KeyBits<T>::value((uint32_t)(key >> kIndexBits));
}
__device__ __forceinline__ int64_t cand_index(uint64_t key)
{
    return (int64_t)((1u << kIndexBits) - 1u - (uint32_t)(key & ((1u << kIndexBits) - 1u)));
}

// Shared state of one block-wide select.
constexpr int kSmallBin = 64;  // boundary bins up to this size are ranked directly

struct SelectState {
    uint32_t hist[256];
    uint32_t warp_top[32];
    uint64_t bin_keys[kSmallBin];
    uint32_t bin_top;  // leading 16 bits of the boundary bin's keys
    int bin_size;
    int bin_filled;
    uint64_t tau;   // digits of the k-th largest key found so far
    int need;       // how many keys still to take from the current bin
    int shift;      // the select ends at this digit: keys with (key >> shift) >= (tau >> shift)
    int done;
    int window;     // the first round found the bin of the k-th largest key
    int count;      // output slots handed out
};

// Select of the k largest among the block's BITS-bit keys, all distinct: every
// thread passes its M keys (`valid` marks real ones).  On return every thread
// can test a key with selected().
//
// First round: the keys' leading 16 bits (the value's sign, exponent and
// leading mantissa bits) are measured as a distance d below the block's
// largest, and keys with d < 256 are histogrammed by d.  The k largest keys of
// a row of logits lie within that window (within two binades of the largest
// value) unless the row is flatter than any logit distribution, so this round
// usually finds the bin of the k-th largest key at once, and only the keys
// near the top touch the histogram.  An 8-bit digit of the raw bits instead
// puts most values into a handful of exponent bins, where shared-memory
// atomics on one address serialise.  When the window holds fewer than k keys,
// the select starts over on the raw bits.
// Further rounds (most significant 8-bit digit first) histogram the digit of
// the keys that share the bits fixed so far; the bin holding the k-th largest
// key becomes the next prefix; the select stops once that bin is taken whole,
// which always happens by the last digit because keys are distinct.  They are
// needed only for a boundary bin of more than kSmallBin keys (or after a
// window that held fewer than k): a smaller one is gathered into shared
// memory and its keys ranked by counting, and the key of rank `need` becomes
// the threshold.
template <int BITS, typename K, int M>
__device__ void select_top_k(const K (&key)[M], const bool (&valid)[M], int k, SelectState& st)
{
    static_assert(BITS % 8 == 0 && BITS >= 32 && BITS <= 8 * (int)sizeof(K),
                  "keys are whole 8-bit digits that fit the key type");
    constexpr int VS = BITS - 16;  // shift of the leading 16 bits
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int warps = (int)(blockDim.x >> 5);

    // largest leading 16 bits in the block
    uint32_t top = 0;
#pragma unroll
    for (int m = 0; m < M; ++m)
        if (valid[m])
            top = max(top, (uint32_t)(key[m] >> VS));
    top = __reduce_max_sync(0xFFFFFFFFu, top);
    if (lane == 0)
        st.warp_top[warp] = top;
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        st.hist[i] = 0;
    if (threadIdx.x == 0) {
        st.done = 0;
        st.window = 0;
        st.shift = 0;
        st.count = 0;  // output slots, handed out by the caller after the select
    }
    __syncthreads();
    top = 0;
    for (int w = 0; w < warps; ++w)
        top = max(top, st.warp_top[w]);
#pragma unroll
    for (int m = 0; m < M; ++m) {
        if (valid[m]) {
            const uint32_t d = top - (uint32_t)(key[m] >> VS);
            if (d < 256u)
                atomicAdd(&st.hist[d], 1u);
        }
    }
    __syncthreads();
    if (warp == 0) {
        // bins [8 lane, 8 lane + 8), nearest the top first
        uint32_t local = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b)
            local += st.hist[8 * lane + b];
        uint32_t upto = local;  // keys in this lane's bins and every nearer bin
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, upto, o);
            if (lane >= o)
                upto += v;
        }
        const uint32_t nearer = upto - local;
        if (nearer < (uint32_t)k && upto >= (uint32_t)k) {
            uint32_t run = nearer;
            for (int b = 0; b < 8; ++b) {
                const uint32_t h = st.hist[8 * lane + b];
                if (run + h >= (uint32_t)k) {
                    const int rest = k - (int)run;
                    st.tau = (uint64_t)(top - (uint32_t)(8 * lane + b)) << VS;
                    st.need = rest;
                    st.window = 1;
                    st.bin_top = top - (uint32_t)(8 * lane + b);
                    st.bin_size = (int)h;
                    st.bin_filled = 0;
                    if ((uint32_t)rest == h) {  // the whole bin is taken
                        st.done = 1;
                        st.shift = VS;
                    }
                    break;
                }
                run += h;
            }
        }
    }
    __syncthreads();
    if (st.done)
        return;
    if (st.window && st.bin_size <= kSmallBin) {
        const uint32_t bin_top = st.bin_top;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (valid[m] && (uint32_t)(key[m] >> VS) == bin_top)
                st.bin_keys[atomicAdd(&st.bin_filled, 1)] = (uint64_t)key[m];
        }
        __syncthreads();
        const int size = st.bin_size;
        if ((int)threadIdx.x < size) {
            const uint64_t mine = st.bin_keys[threadIdx.x];
            int larger = 0;
            for (int j = 0; j < size; ++j)
                larger += st.bin_keys[j] > mine;
            if (larger == st.need - 1) {  // keys are distinct: exactly one thread
                st.tau = mine;
                st.shift = 0;
                st.done = 1;
            }
        }
        __syncthreads();
        return;
    }
    int first = VS - 8;  // the bin's leading 16 bits are fixed
    if (!st.window) {
        first = BITS - 8;
        if (threadIdx.x == 0) {
            st.tau = 0;
            st.need = k;
        }
    }
    for (int shift = first; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x)
            st.hist[i] = 0;
        __syncthreads();
        const K high_mask = (shift + 8 >= BITS) ? K(0) : (K(~K(0)) << (shift + 8));
        const K prefix = (K)st.tau & high_mask;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (valid[m] && ((key[m] & high_mask) == prefix))
                atomicAdd(&st.hist[(uint32_t)(key[m] >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // bins [8 lane, 8 lane + 8); counts from the top down
            uint32_t local = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b)
                local += st.hist[8 * lane + b];
            uint32_t above = local;  // keys in this lane's bins and every higher bin
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, above, o);
                if (lane + o < 32)
                    above += v;
            }
            const uint32_t higher = above - local;  // keys in higher lanes' bins
            const int need = st.need;
            if (higher < (uint32_t)need && above >= (uint32_t)need) {
                uint32_t run = higher;
                for (int b = 7; b >= 0; --b) {
                    const uint32_t h = st.hist[8 * lane + b];
                    if (run + h >= (uint32_t)need) {
                        const int rest = need - (int)run;
                        st.tau |= (uint64_t)(8 * lane + b) << shift;
                        st.need = rest;
                        if ((uint32_t)rest == h) {  // the whole bin is taken
                            st.done = 1;
                            st.shift = shift;
                        }
                        break;
                    }
                    run += h;
                }
            }
        }
        __syncthreads();
        if (st.done)
            break;
    }
}

template <typename K>
__device__ __forceinline__ bool selected(K key, const SelectState& st)
{
    return (key >> st.shift) >= ((K)st.tau >> st.shift);
}

// First output slot of this thread's `count` selected keys: the block's
// selected keys are laid out warp by warp and, within a warp, lane by lane (a
// warp scan and one barrier; `warp_tot` holds one count per warp).  Every
// thread of the block must call it.
__device__ __forceinline__ int selected_offset(int count, int* warp_tot)
{
    const int lane = (int)(threadIdx.x & 31);
    const int warp = (int)(threadIdx.x >> 5);
    int incl = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o)
            incl += v;
    }
    if (lane == 31)
        warp_tot[warp] = incl;
    __syncthreads();
    int base = incl - count;
    for (int w = 0; w < warp; ++w)
        base += warp_tot[w];
    return base;
}

constexpr int kPerThread = kSlice / kSliceThreads;  // 8

// In-slice keys: value bits above the inverted 16-bit position in the slice
// (32 bits in all for bf16, 48 for fp32).
template <typename T>
struct LocalKey {
    using type = typename std::conditional<KeyBits<T>::V + 16 <= 32, uint32_t, uint64_t>::type;
    static constexpr int BITS = KeyBits<T>::V + 16;
};

constexpr int kMergePerThread = kMaxSlices * kMaxTopK / kMergeThreads;  // 8

// The row's merge and decision, run by the CTA that arrived last: the k
// largest of the slices' n = slices * k candidate keys (read through L2: other
// CTAs wrote them), ranked by counting, then the sampling decision.
template <typename T>
__device__ void merge_and_sample(const uint64_t* cand, int n, int k, const float* __restrict__ g,
                                 float temperature, int32_t* token_out, float* prob_out,
                                 SelectState& st, uint64_t* sel, uint64_t* ranked)
{
    // warp 0's Gumbel draws (two ranks per lane), loaded with the keys so that
    // their latency is not paid again at the decision
    float gdraw[2] = {0.f, 0.f};
    if (threadIdx.x < 32) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
            if ((int)threadIdx.x + 32 * r < k)
                gdraw[r] = __ldg(g + threadIdx.x + 32 * r);
    }
    uint64_t key[kMergePerThread];
    bool valid[kMergePerThread];
#pragma unroll
    for (int m = 0; m < kMergePerThread; ++m) {
        const int i = threadIdx.x + m * kMergeThreads;
        // padding keys (0) of short slices are not candidates
        key[m] = (i < n) ? __ldcg(cand + i) : 0ull;
        valid[m] = key[m] != 0ull;
    }
    select_top_k<KeyBits<T>::V + kIndexBits>(key, valid, k, st);
    {
        int count = 0;
#pragma unroll
        for (int m = 0; m < kMergePerThread; ++m)
            count += valid[m] && selected(key[m], st);
        int slot = selected_offset(count, reinterpret_cast<int*>(st.warp_top));
#pragma unroll
        for (int m = 0; m < kMergePerThread; ++m)
            if (valid[m] && selected(key[m], st)) {
                if (slot < k)
                    sel[slot] = key[m];
                ++slot;
            }
    }
    __syncthreads();
    // order the k candidates by counting: rank = number of larger keys
    if ((int)threadIdx.x < k) {
        const uint64_t mine = sel[threadIdx.x];
        int rank = 0;
        for (int j = 0; j < k; ++j)
            rank += sel[j] > mine;
        ranked[rank] = mine;
    }
    __syncthreads();

    // Warp 0 takes the decision, two ranks per lane (k <= 64).  Per rank j:
    // e_j = exp((l_j - l_0) / T) and the score fl(fl(l_j / T) + g_j), two
    // correctly rounded operations.  The token is the first rank with the
    // largest score, as a scan in rank order that moves on only to a strictly
    // larger score finds it: NaN scores after rank 0 never win, a NaN at rank 0
    // always does.
    if (threadIdx.x >= 32)
        return;
    const int lane = threadIdx.x;
    const float l0 = cand_value<T>(ranked[0]);
    float ej[2], bs = 0.f, z = 0.f;
    int bj = k;  // none yet
    float s0 = 0.f;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        ej[r] = 0.f;
        if (j < k) {
            const float l = cand_value<T>(ranked[j]);
            ej[r] = expf((l - l0) / temperature);
            const float sc = __fadd_rn(__fdiv_rn(l, temperature), gdraw[r]);
            if (j == 0)
                s0 = sc;
            if (!isnan(sc) && (bj == k || sc > bs)) {
                bs = sc;
                bj = j;
            }
            z += ej[r];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(0xFFFFFFFFu, bs, o);
        const int oj = __shfl_xor_sync(0xFFFFFFFFu, bj, o);
        if (oj < k && (bj == k || os > bs || (os == bs && oj < bj))) {
            bs = os;
            bj = oj;
        }
        z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
    }
    s0 = __shfl_sync(0xFFFFFFFFu, s0, 0);
    const int best = isnan(s0) ? 0 : bj;
    const float eb = __shfl_sync(0xFFFFFFFFu, best < 32 ? ej[0] : ej[1], best & 31);
    if (lane == 0) {
        *token_out = (int32_t)cand_index(ranked[best]);
        *prob_out = eb / z;
    }
}

// VEC: rows start on 16-byte boundaries, so a thread loads its 16 logits as
// 16-byte vectors (positions (v * 256 + thread) * E + e); otherwise one
// element at a time (positions thread + 256 m).  Either way every position of
// the slice is read exactly once.
// Two CTAs (32 warps) per SM: many-row calls run several waves, and a slice's
// 16 warps hide each other's latency (512 threads measured 8.2 -> 6.8 us
// against 256 for 5 x 151936 on B200).
template <typename T, bool VEC>
__global__ void __launch_bounds__(kSliceThreads, 2)
topk_sample_kernel(const T* __restrict__ logits, int64_t vocab, int k, int slices,
                   unsigned* __restrict__ counters, uint64_t* __restrict__ work,
                   const float* __restrict__ gumbel, float temperature,
                   int32_t* __restrict__ token_out, float* __restrict__ prob_out,
                   unsigned* err_word)
{
    using K = typename LocalKey<T>::type;
    constexpr int E = Vec<T>::N;
    __shared__ SelectState st;
    __shared__ uint64_t sel[kMaxTopK];
    __shared__ uint64_t ranked[kMaxTopK];
    __shared__ int last;
    const int64_t row = blockIdx.y;
    const int64_t first = (int64_t)blockIdx.x * kSlice;
    const T* lr = logits + row * vocab;
    const int n = (int)((vocab - first < kSlice) ? vocab - first : kSlice);
    // the slice into L2 while the previous kernel drains, one line per thread
    {
        constexpr int kPerLine = 128 / sizeof(T);
        if (threadIdx.x * kPerLine < n)
            prefetch_l2_line(lr + first + threadIdx.x * kPerLine);
    }
    pdl_wait();
    pdl_allow_dependents();
    K key[kPerThread];
    float val[kPerThread];
    bool valid[kPerThread];
    int pos[kPerThread];
    if constexpr (VEC) {
#pragma unroll
        for (int v = 0; v < kPerThread / E; ++v) {
            const int p0 = (v * kSliceThreads + (int)threadIdx.x) * E;
            float f[E];
            if (p0 + E <= n) {
                Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(lr + first + p0)), f);
            } else {
#pragma unroll
                for (int j = 0; j < E; ++j)
                    f[j] = (p0 + j < n) ? load_elem(lr + first + p0 + j) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < E; ++j) {
                val[v * E + j] = f[j];
                pos[v * E + j] = p0 + j;
            }
        }
    } else {
#pragma unroll
        for (int m = 0; m < kPerThread; ++m) {
            pos[m] = (int)threadIdx.x + m * kSliceThreads;
            val[m] = (pos[m] < n) ? load_elem(lr + first + pos[m]) : 0.f;
        }
    }
#pragma unroll
    for (int m = 0; m < kPerThread; ++m) {
        valid[m] = pos[m] < n;
        key[m] = valid[m] ? (((K)KeyBits<T>::of(val[m]) << 16) | (K)(0xFFFFu - (uint32_t)pos[m]))
                          : K(0);
    }
    uint64_t* row_cand = work + row * slices * (int64_t)k;
    uint64_t* out = row_cand + blockIdx.x * (int64_t)k;
    if (n <= k) {
        // the whole slice is a candidate; the unused slots get keys below any logit
#pragma unroll
        for (int m = 0; m < kPerThread; ++m) {
            if (pos[m] < k)
                out[pos[m]] = valid[m] ? cand_key<T>(val[m], first + pos[m]) : 0ull;
        }
    } else {
        select_top_k<LocalKey<T>::BITS>(key, valid, k, st);
        int count = 0;
#pragma unroll
        for (int m = 0; m < kPerThread; ++m)
            count += valid[m] && selected(key[m], st);
        int slot = selected_offset(count, reinterpret_cast<int*>(st.warp_top));
#pragma unroll
        for (int m = 0; m < kPerThread; ++m)
            if (valid[m] && selected(key[m], st)) {
                if (slot < k)  // exactly k are selected; the test only guards the bound
                    out[slot] = cand_key<T>(val[m], first + pos[m]);
                ++slot;
            }
    }
    // Arrival: the barrier orders every thread's candidate stores before thread
    // 0's count, an atomic add with release and acquire semantics at GPU scope
    // (release is cumulative: it covers the stores the barrier ordered before
    // it), so the CTA that counts last sees every other CTA's stores, and
    // merges.
    __syncthreads();
    if (threadIdx.x == 0) {
        // release: the CTA's stores, ordered by the barrier, before the count;
        // acquire: the other CTAs' stores before this CTA's reads
        const unsigned before = atomic_add_acq_rel_gpu(counters + row, 1u);
        if (before >= (unsigned)slices)  // the counter was not zero when the call began
            record_device_error(err_word, kDeviceErrWorkspace);
        last = before == (unsigned)slices - 1u;
        if (last)
            counters[row] = 0;  // every CTA of the row has arrived: ready for the next call
    }
    __syncthreads();
    if (!last)
        return;
    merge_and_sample<T>(row_cand, slices * k, k, gumbel + row * k, temperature, token_out + row,
                        prob_out + row, st, sel, ranked);
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

size_t topk_counter_bytes()
{
    return kCounterBytes;
}

cudaError_t launch_topk_sample(const void* logits, const float* gumbel, int32_t* token_out,
                               float* prob_out, int64_t rows, int64_t vocab, int k,
                               float temperature, arops_dtype dtype, void* workspace,
                               cudaStream_t stream)
{
    const int slices = topk_slices(vocab);
    const dim3 grid((unsigned)slices, (unsigned)rows);
    const size_t esize = dtype == AROPS_BF16 ? 2 : 4;
    const bool vec = aligned16(logits) && (vocab * esize) % 16 == 0;
    unsigned* counters = static_cast<unsigned*>(workspace);
    uint64_t* work = reinterpret_cast<uint64_t*>(static_cast<unsigned char*>(workspace) +
                                                 kCounterBytes);
    unsigned* word = nullptr;
    cudaError_t err = device_error_word(&word);
    if (err != cudaSuccess)
        return err;
    if (dtype == AROPS_BF16) {
        const auto* lg = static_cast<const __nv_bfloat16*>(logits);
        return vec ? launch(topk_sample_kernel<__nv_bfloat16, true>, grid, dim3(kSliceThreads), 0,
                            stream, lg, vocab, k, slices, counters, work, gumbel, temperature,
                            token_out, prob_out, word)
                   : launch(topk_sample_kernel<__nv_bfloat16, false>, grid, dim3(kSliceThreads), 0,
                            stream, lg, vocab, k, slices, counters, work, gumbel, temperature,
                            token_out, prob_out, word);
    }
    const auto* lg = static_cast<const float*>(logits);
    return vec ? launch(topk_sample_kernel<float, true>, grid, dim3(kSliceThreads), 0, stream, lg,
                        vocab, k, slices, counters, work, gumbel, temperature, token_out,
                        prob_out, word)
               : launch(topk_sample_kernel<float, false>, grid, dim3(kSliceThreads), 0, stream, lg,
                        vocab, k, slices, counters, work, gumbel, temperature, token_out,
                        prob_out, word);
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the workspace lives in this file-scope device
// array instead of caller memory.  It exists for callers that cannot allocate
// device memory themselves, e.g. code running inside a host application's
// real-time audio or streaming callback, where cudaMalloc is off limits
// because it can block and synchronise the device, or a plugin that is handed
// buffers by a host application that owns all device memory.  Every GPU that
// loads the library holds this array until the process exits.  It holds the
// arrival counters (zero when the module is loaded, as every __device__
// variable without an initialiser is, and left zero by every call) and then
// 1 MiB of candidate keys.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB of candidates

static __device__ __align__(256) uint64_t
    g_topk_scratch[(kCounterBytes + kNoAllocScratchBytes) / sizeof(uint64_t)];

size_t topk_noalloc_scratch_bytes()
{
    return kNoAllocScratchBytes;
}

// Device address of the scratch array in the current context.  In host code
// the array's name is only a stand-in, so the address is looked up with
// cudaGetSymbolAddress, on every call: the array has one instance per CUDA
// context, and a cached address could belong to another context than the
// caller's current one (a context the caller created itself, or a primary
// context that was reset and created anew).  Once this code is loaded in the
// context the lookup allocates nothing; the first lookup in a context loads it
// (with lazy module loading, the CUDA default), which reserves the array.
cudaError_t topk_noalloc_scratch(void** ptr)
{
    return cudaGetSymbolAddress(ptr, g_topk_scratch);
}

}  // namespace arops
