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
// Four kernels give the same results.  The cluster kernels (second half of
// this file) run a row per thread-block cluster with the selection exchanged
// through distributed shared memory: logits in registers on clusters of up
// to 16 CTAs while every row's cluster is resident at once (a few rows), in
// shared memory on clusters of up to 8 for more rows.  The streaming kernel
// (after them) runs a row per CTA for calls with many rows, streaming it
// through shared memory against a running floor.  The slice kernel serves
// calls where no cluster launch is possible: grid (slices, rows).  A CTA turns
// its 4096-logit slice into
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
#include "tma.cuh"

namespace arops {
// Which kernels sampling calls may take (api.cu, arops_set_topk_cluster): 0
// the slice kernel only; 1 the cluster kernels (registers for few rows, shared
// memory for many); 2 the shared-memory cluster kernel for every call.
int topk_cluster_mode();
}  // namespace arops

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

// The sampling decision, taken by warp 0 of the calling CTA (every thread
// may call it; the others return at once).  ranked[0..k) holds the row's k
// candidate keys from the largest down; gdraw holds the Gumbel draws of ranks
// lane and lane + 32 in warp 0.
template <typename T>
__device__ __forceinline__ void sample_decision(const uint64_t* ranked, int k,
                                                const float (&gdraw)[2], float temperature,
                                                int32_t* token_out, float* prob_out)
{
    // Two ranks per lane (k <= 64).  Per rank j:
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

// The k largest of the block's candidate keys (row keys, cand_key; each
// thread passes M of them, `valid` marking real ones; at least k valid in
// all), ordered by counting (rank = number of larger keys), then the sampling
// decision.  Every thread of the block must call it.
template <typename T, int M>
__device__ void rank_and_sample(const uint64_t (&key)[M], const bool (&valid)[M], int k,
                                const float (&gdraw)[2], float temperature, int32_t* token_out,
                                float* prob_out, SelectState& st, uint64_t* sel, uint64_t* ranked)
{
    select_top_k<KeyBits<T>::V + kIndexBits>(key, valid, k, st);
    {
        int count = 0;
#pragma unroll
        for (int m = 0; m < M; ++m)
            count += valid[m] && selected(key[m], st);
        int slot = selected_offset(count, reinterpret_cast<int*>(st.warp_top));
#pragma unroll
        for (int m = 0; m < M; ++m)
            if (valid[m] && selected(key[m], st)) {
                if (slot < k)
                    sel[slot] = key[m];
                ++slot;
            }
    }
    __syncthreads();
    if ((int)threadIdx.x < k) {
        const uint64_t mine = sel[threadIdx.x];
        int rank = 0;
        for (int j = 0; j < k; ++j)
            rank += sel[j] > mine;
        ranked[rank] = mine;
    }
    __syncthreads();
    sample_decision<T>(ranked, k, gdraw, temperature, token_out, prob_out);
}

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
    rank_and_sample<T>(key, valid, k, gdraw, temperature, token_out, prob_out, st, sel, ranked);
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

// ---------------------------------------------------------------------------
// Single-pass variants on a thread-block cluster: one cluster of `ncta` CTAs
// per row, each CTA holding a contiguous chunk of the row's logits, in
// registers (up to 16 CTAs) or in shared memory (up to 8).  The select runs
// over the whole row at once: every CTA first drops the keys below a floor
// that at least k of its keys reach (so none of the dropped ones can be among
// the row's k largest), histograms the rest in its shared memory and sends
// the histogram to its peers' shared memory (distributed shared memory)
// before a cluster barrier, and every CTA sums the cluster's, so all CTAs
// reach the same decision without any exchange through global memory.  Once the boundary bin holds at
// most kSmallBin keys, every CTA pushes its keys from that bin up (at most
// k - 1 + kSmallBin in all, the row's k largest among them) into the shared
// memory of the cluster's first CTA, which ranks them by counting and takes
// the sampling decision.  Two cluster barriers in the common case; a row whose
// boundary bin is larger (ties, flat rows) takes further 8-bit digit rounds of
// one barrier each.  Nothing is read or written outside the logits, the draws
// and the outputs.
// ---------------------------------------------------------------------------
constexpr int kClThreads = 512;
constexpr int kClWarps = kClThreads / 32;
constexpr int kClMaxCtas = 16;                       // non-portable cluster size
constexpr int kClPushSlots = 128;                   // >= kMaxTopK - 1 + kSmallBin
static_assert(kMaxTopK - 1 + kSmallBin <= kClPushSlots, "room for every pushed key");
static_assert(4 * kClPushSlots <= kClThreads, "four threads rank each pushed key");
static_assert(kClWarps * 4 >= kMaxTopK, "at most four keys a warp make the floor");

// Largest value over the warp.
template <typename K>
__device__ __forceinline__ K warp_max(K v)
{
    if constexpr (sizeof(K) == 4) {
        return __reduce_max_sync(0xFFFFFFFFu, v);
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const K u = __shfl_xor_sync(0xFFFFFFFFu, v, o);
            v = u > v ? u : v;
        }
        return v;
    }
}

// Distributed shared memory: the address of this CTA's shared variable `p` in
// the shared memory of cluster CTA `rank`, and accesses through it.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank)
{
    const uint32_t local = (uint32_t)__cvta_generic_to_shared(p);
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    return remote;
}

// (No memory clobber: the cluster barriers order these loads; without it the
// loads of one thread are issued together instead of one round trip each.)
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void st_cluster_u64(uint32_t addr, uint64_t v)
{
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, const uint4& v)
{
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_v2(uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b)
                 : "memory");
}

__device__ __forceinline__ uint32_t atom_add_cluster_u32(uint32_t addr, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "r"(addr), "r"(v)
                 : "memory");
    return old;
}

// Barrier of all threads of the cluster: shared-memory writes before it (this
// CTA's and remote ones) are visible to every thread of the cluster after it.
__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

struct ClusterSelect {
    alignas(16) uint32_t hist[2][256];  // this CTA's histogram of a round (alternating buffers)
    // first round: every CTA's histogram bins [0, span) as sent by that CTA,
    // and its (largest leading bits, span)
    alignas(16) uint32_t inbox[kClMaxCtas][256];
    uint2 inbox_meta[kClMaxCtas];
    uint32_t ghist[256];    // the cluster's, summed from every CTA's
    uint32_t warp_top[32];  // per-warp counts of the push
    uint64_t warp_key[32];  // per-warp largest key
    uint64_t warp_floor[32];  // per-warp r-th largest lane maximum
    uint64_t tau;           // bits of the boundary bin fixed so far (global-key layout)
    int shift;              // the bin is the keys with (key >> shift) == (tau >> shift)
    int need;               // keys still to take from the bin
    int binsz;              // keys in the bin, over the whole row
    int window;             // the first round found the bin
    int64_t first;          // the chunk's first vocabulary index
    uint32_t ncomp;         // keys listed by the shared-memory kernel
    uint32_t ctop;          // the row's largest leading bits
    uint32_t push_cnt[kClMaxCtas];  // keys each CTA pushes (when the first round decides)
    uint32_t push_base;
    // the first CTA's: keys pushed by the cluster, their count, their ranking
    uint32_t push_count;
    uint64_t cand[kClPushSlots];
    uint64_t ranked[kMaxTopK];
};

// Row-wide key (cand_key's layout) of a CTA-local key of the chunk at `first`.
template <typename T>
__device__ __forceinline__ uint64_t row_key(typename LocalKey<T>::type lk, int64_t first)
{
    const uint64_t vbits = (uint64_t)(lk >> 16);
    const uint32_t p = 0xFFFFu - (uint32_t)(lk & 0xFFFFu);
    return (vbits << kIndexBits) |
           (uint64_t)((1u << kIndexBits) - 1u - (uint32_t)(first + (int64_t)p));
}

// The smallest local key (as a 64-bit number) of the chunk at `first` whose
// row key is at least `t`.  Within a chunk the map from local to row keys
// keeps the order (the row key's index bits are the local ones plus
// 2^24 - 2^16 - first), so `local >= threshold` tests `row key >= t` without
// forming the row key.
template <typename T>
__device__ __forceinline__ uint64_t local_threshold(uint64_t t, int64_t first)
{
    const uint64_t vt = t >> kIndexBits;
    const int64_t it = (int64_t)(t & ((1ull << kIndexBits) - 1ull));
    const int64_t below = it - ((int64_t)(1 << kIndexBits) - 0x10000 - first);
    if (below <= 0)
        return vt << 16;
    if (below > 0xFFFF)
        return (vt + 1) << 16;
    return (vt << 16) | (uint64_t)below;
}

// Warp 0, first round: the bin of the k-th largest key in the cluster's
// histogram of distances below the row's largest leading 16 bits `ctop`.
// Leaves window = 0 when the 256 bins hold fewer than k keys.
__device__ __forceinline__ void cluster_window_scan(ClusterSelect& st, uint32_t ctop, int k, int gs)
{
    const int lane = threadIdx.x & 31;
    uint32_t local = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b)
        local += st.ghist[8 * lane + b];
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
            const uint32_t h = st.ghist[8 * lane + b];
            if (run + h >= (uint32_t)k) {
                st.tau = (uint64_t)(ctop - (uint32_t)(8 * lane + b)) << gs;
                st.shift = gs;
                st.need = k - (int)run;
                st.binsz = (int)h;
                st.window = 1;
                break;
            }
            run += h;
        }
    }
}

// Warp 0, a digit round: the bin of the need-th largest key among the keys of
// the current bin, by the 8-bit digit at `shift`.
__device__ __forceinline__ void cluster_digit_scan(ClusterSelect& st, int shift)
{
    const int lane = threadIdx.x & 31;
    uint32_t local = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b)
        local += st.ghist[8 * lane + b];
    uint32_t above = local;  // keys in this lane's bins and every higher bin
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, above, o);
        if (lane + o < 32)
            above += v;
    }
    const uint32_t higher = above - local;
    const int need = st.need;
    if (higher < (uint32_t)need && above >= (uint32_t)need) {
        uint32_t run = higher;
        for (int b = 7; b >= 0; --b) {
            const uint32_t h = st.ghist[8 * lane + b];
            if (run + h >= (uint32_t)need) {
                st.tau |= (uint64_t)(8 * lane + b) << shift;
                st.shift = shift;
                st.need = need - (int)run;
                st.binsz = (int)h;
                break;
            }
            run += h;
        }
    }
}

// Sum over the cluster's CTAs of bin threadIdx.x of a digit round's
// histogram buffer `h` (read from every CTA's shared memory; threads 0..255).
__device__ __forceinline__ uint32_t cluster_hist_sum(const uint32_t* h, uint32_t ncta)
{
    const uint32_t bin = threadIdx.x;
    // all remote loads first, then the sum: one round trip in all
    uint32_t v[kClMaxCtas];
#pragma unroll
    for (uint32_t c = 0; c < (uint32_t)kClMaxCtas; ++c)
        v[c] = c < ncta ? ld_cluster_u32(cluster_addr(h + bin, c)) : 0u;
    uint32_t tot = 0;
#pragma unroll
    for (int c = 0; c < kClMaxCtas; ++c)
        tot += v[c];
    return tot;
}

// This thread's keys of its chunk, as the select walks them:
//   max_key()        a key no smaller than the smallest key of the thread's
//                    largest value and no larger than its largest key (0 if
//                    the thread holds no position of the chunk);
//   each_from(lo, f) f(key) for every key >= lo (lo > 0).
// RegKeys holds the keys in registers (M a thread).  SmemKeys forms them from
// the chunk's values in shared memory (16-byte vectors tid, tid + 512, ...: a
// chunk too large for registers), testing the values first, two bf16 at a
// time, so that only the few keys at or above a threshold are ever formed.
template <typename K, int M>
struct RegKeys {
    static constexpr bool kCompact = false;
    K key[M];  // 0 marks a position past the chunk; no real key is 0
    __device__ __forceinline__ K max_key() const
    {
        K m = 0;
#pragma unroll
        for (int i = 0; i < M; ++i)
            m = max(m, key[i]);
        return m;
    }
    template <class F>
    __device__ __forceinline__ void each_from(uint64_t lo, F&& f) const
    {
#pragma unroll
        for (int i = 0; i < M; ++i)
            if ((uint64_t)key[i] >= lo)
                f(key[i]);
    }
};

// The keys of a CTA listed in shared memory (the compacted ones): thread tid
// takes entries tid, tid + 512, ...
template <typename K>
struct ListKeys {
    const K* list;
    int n;
    template <class F>
    __device__ __forceinline__ void each_from(uint64_t lo, F&& f) const
    {
        for (int i = (int)threadIdx.x; i < n; i += kClThreads) {
            const K x = list[i];
            if ((uint64_t)x >= lo)
                f(x);
        }
    }
};

// Keys from the floor up that the shared-memory kernel lists for its later
// passes (~130 a CTA for logit-like rows; a row that has more keeps walking
// its whole chunk).
constexpr int kCompactKeys = 2048;

template <typename T>
struct SmemKeys;

// Largest of each 16-bit half (a single instruction on sm_90 and later).
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Two bf16 in a 32-bit word, each turned into the 16 bits KeyBits orders by.
__device__ __forceinline__ uint32_t ordered_bf16x2(uint32_t w)
{
    const uint32_t sign = (w >> 15) & 0x00010001u;
    return w ^ 0x80008000u ^ (sign * 0x7FFFu);
}

template <>
struct SmemKeys<__nv_bfloat16> {
    static constexpr bool kCompact = true;
    const __nv_bfloat16* vals;  // 16-byte aligned, padded to whole vectors
    int n;
    uint32_t* list;             // kCompactKeys entries for the compacted keys
    __device__ __forceinline__ uint32_t max_key() const
    {
        const int nv = (n + 7) / 8;
        uint32_t acc = 0;
        bool any = false;
        for (int v = (int)threadIdx.x; v < nv; v += kClThreads) {
            const uint4 x = reinterpret_cast<const uint4*>(vals)[v];
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            if (v * 8 + 8 <= n) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    acc = max_u16x2(acc, ordered_bf16x2(w[i]));
            } else {  // the ragged last vector
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t o = ordered_bf16x2(w[i]);
                    if (v * 8 + 2 * i < n)
                        acc = max_u16x2(acc, o & 0xFFFFu);
                    if (v * 8 + 2 * i + 1 < n)
                        acc = max_u16x2(acc, o & 0xFFFF0000u);
                }
            }
            any = true;
        }
        const uint32_t m = max(acc & 0xFFFFu, acc >> 16);
        return any ? (m << 16) : 0u;  // (value, inverted position 0): the value's smallest key
    }
    template <class F>
    __device__ __forceinline__ void each_from(uint64_t lo, F&& f) const
    {
        if (lo > 0xFFFFFFFFull)
            return;
        const uint32_t lov = (uint32_t)(lo >> 16);
        // a half is at least lov when max(half, lov - 1) moves off lov - 1
        const uint32_t below2 = (lov ? lov - 1u : 0u) * 0x00010001u;
        const int nv = (n + 7) / 8;
        for (int v = (int)threadIdx.x; v < nv; v += kClThreads) {
            const uint4 x = reinterpret_cast<const uint4*>(vals)[v];
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t o = ordered_bf16x2(w[i]);
                if (lov == 0u || max_u16x2(o, below2) != below2) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int p = v * 8 + 2 * i + h;
                        if (((o >> (16 * h)) & 0xFFFFu) >= lov && p < n) {
                            const uint32_t key = (((o >> (16 * h)) & 0xFFFFu) << 16) |
                                                 (0xFFFFu - (uint32_t)p);
                            if (key >= (uint32_t)lo)
                                f(key);
                        }
                    }
                }
            }
        }
    }
};

template <>
struct SmemKeys<float> {
    static constexpr bool kCompact = true;
    const float* vals;  // 16-byte aligned, padded to whole vectors
    int n;
    uint64_t* list;     // kCompactKeys entries for the compacted keys
    __device__ __forceinline__ uint64_t max_key() const
    {
        uint32_t m = 0;
        bool any = false;
        for (int p = (int)threadIdx.x * 4; p < n; p += kClThreads * 4) {
            const float4 x = *reinterpret_cast<const float4*>(vals + p);
            const float e[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (p + j < n)
                    m = max(m, order_bits(e[j]));
            any = true;
        }
        return any ? ((uint64_t)m << 16) : 0ull;
    }
    template <class F>
    __device__ __forceinline__ void each_from(uint64_t lo, F&& f) const
    {
        if (lo > 0xFFFFFFFFFFFFull)
            return;
        const uint32_t lov = (uint32_t)(lo >> 16);
        for (int p = (int)threadIdx.x * 4; p < n; p += kClThreads * 4) {
            const float4 x = *reinterpret_cast<const float4*>(vals + p);
            const float e[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t o = order_bits(e[j]);
                if (o >= lov && p + j < n) {
                    const uint64_t key = ((uint64_t)o << 16) | (0xFFFFu - (uint32_t)(p + j));
                    if (key >= lo)
                        f(key);
                }
            }
        }
    }
};

// The rest of the select, from the histogram exchange on, and the sampling
// decision; `keys` walks this thread's keys from `floor` up.
template <typename T, class Keys>
__device__ __forceinline__ void cluster_finish(const Keys& keys, ClusterSelect& st,
                                               typename LocalKey<T>::type floor, uint32_t top,
                                               int64_t row, int64_t first, int k,
                                               const float (&gdraw)[2], float temperature,
                                               int32_t* token_out, float* prob_out)
{
    using K = typename LocalKey<T>::type;
    constexpr int VS = LocalKey<T>::BITS - 16;  // leading 16 bits of a local key
    constexpr int GB = KeyBits<T>::V + kIndexBits;
    constexpr int GS = GB - 16;                 // leading 16 bits of a row key
    const int tid = (int)threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const uint32_t crank = cluster_ctarank();
    const uint32_t ncta = cluster_nctarank();
    // Send the histogram to every CTA of the cluster (its row `crank` of their
    // inboxes) before the barrier, so that the sum after it reads only this
    // CTA's own shared memory.  The keys that take part lie within `span` bins
    // of the CTA's largest leading bits (the floor's are the lowest), so only
    // those bins go out, four to a store: a few dozen for logit-like rows.
    {
        const uint32_t flead = (uint32_t)(floor >> VS);
        const uint32_t span = floor ? min(256u, top - flead + 1u) : 256u;
        const uint32_t nv = (span + 3u) / 4u;
        for (uint32_t i = tid; i < nv * ncta; i += kClThreads) {
            const uint32_t c = i / nv;
            const uint32_t v = i - c * nv;
            st_cluster_v4(cluster_addr(&st.inbox[crank][4u * v], c),
                          *reinterpret_cast<const uint4*>(&st.hist[0][4u * v]));
        }
        if ((uint32_t)tid < ncta)
            st_cluster_v2(cluster_addr(&st.inbox_meta[crank], (uint32_t)tid), top, span);
    }
    cluster_barrier();  // every CTA's histogram has arrived everywhere

    // The row's histogram of distances below its largest leading bits: a CTA
    // whose own largest bits are delta below the row's contributes its bin
    // d - delta to bin d (its window covers the row's, from below).
    if (tid < 256) {
        const uint2 meta = (uint32_t)lane < ncta ? st.inbox_meta[lane] : make_uint2(0u, 0u);
        const uint32_t ctop = __reduce_max_sync(0xFFFFFFFFu, meta.x);
        uint32_t tot = 0;
#pragma unroll
        for (uint32_t c = 0; c < (uint32_t)kClMaxCtas; ++c) {
            const uint32_t delta = ctop - __shfl_sync(0xFFFFFFFFu, meta.x, c);
            const uint32_t span = __shfl_sync(0xFFFFFFFFu, meta.y, c);
            if (c < ncta && (uint32_t)tid >= delta && (uint32_t)tid - delta < span)
                tot += st.inbox[c][tid - delta];
        }
        st.ghist[tid] = tot;
        if (tid == 0) {
            st.tau = ctop;  // kept for warp 0's scan below
            st.ctop = ctop;
        }
    }
    __syncthreads();
    if (warp == 0)
        cluster_window_scan(st, (uint32_t)st.tau, k, GS);
    __syncthreads();

    // Digit rounds, only while the boundary bin is large and not taken whole
    // (or when the 256 nearest values held fewer than k keys).
    bool more = !st.window || (st.need != st.binsz && st.binsz > kSmallBin);
    const bool rounds = more;
    int shift = st.window ? GS - 8 : GB - 8;
    __syncthreads();  // every thread has read the first round's outcome
    if (tid == 0 && !st.window) {
        st.tau = 0;
        st.need = k;
    }
    for (int round = 1; more; ++round, shift -= 8) {
        uint32_t* h = st.hist[round & 1];
        for (int i = tid; i < 256; i += kClThreads)
            h[i] = 0;
        __syncthreads();
        const uint64_t high_mask = ~0ull << (shift + 8);
        const uint64_t prefix = st.tau & high_mask;
        // re-read each round, so that the row keys are formed here and not
        // kept in registers across rounds
        const int64_t f = *reinterpret_cast<volatile int64_t*>(&st.first);
        keys.each_from(floor ? (uint64_t)floor : 1ull, [&](K x) {
            const uint64_t g = row_key<T>(x, f);
            if ((g & high_mask) == prefix)
                atomicAdd(&h[(uint32_t)(g >> shift) & 255u], 1u);
        });
        cluster_barrier();
        if (tid < 256)
            st.ghist[tid] = cluster_hist_sum(h, ncta);
        __syncthreads();
        if (warp == 0)
            cluster_digit_scan(st, shift);
        __syncthreads();
        more = st.need != st.binsz && st.binsz > kSmallBin;
    }

    // Push: every key from the boundary bin up (k - need above the bin, binsz
    // in it: at most k - 1 + kSmallBin, or exactly k when the bin is taken
    // whole) into the first CTA's shared memory, CTA by CTA.  When the first
    // round decided, every CTA knows how many keys each CTA pushes (its bins
    // from the row's top down to the boundary bin, in the histograms it
    // received), so it finds its range without any exchange; after digit
    // rounds the range is reserved with one remote atomic per CTA.
    uint64_t lthr = local_threshold<T>(st.tau, first);  // the bin's low bits are 0
    lthr = max(lthr, (uint64_t)floor);
    int cnt = 0;
    keys.each_from(lthr ? lthr : 1ull, [&](K) { ++cnt; });
    int incl = cnt;  // warp-inclusive count: the thread's keys go after the lower lanes'
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o)
            incl += v;
    }
    if (lane == 31)
        st.warp_top[warp] = (uint32_t)incl;
    if (!rounds && (uint32_t)warp < ncta) {
        const uint32_t dbin = st.ctop - (uint32_t)(st.tau >> GS);
        const uint2 meta = st.inbox_meta[warp];
        const uint32_t delta = st.ctop - meta.x;
        uint32_t c = 0;
        if (dbin >= delta) {
            const uint32_t last = min(dbin - delta, meta.y - 1u);
            for (uint32_t i = lane; i <= last; i += 32)
                c += st.inbox[warp][i];
        }
        c = __reduce_add_sync(0xFFFFFFFFu, c);
        if (lane == 0)
            st.push_cnt[warp] = c;
    }
    __syncthreads();
    int off = incl - cnt;
    for (int w = 0; w < warp; ++w)
        off += (int)st.warp_top[w];
    uint32_t base;
    if (!rounds) {
        uint32_t b = 0, total = 0;
#pragma unroll
        for (uint32_t c = 0; c < (uint32_t)kClMaxCtas; ++c) {
            if (c < ncta) {
                total += st.push_cnt[c];
                if (c < crank)
                    b += st.push_cnt[c];
            }
        }
        base = b;
        if (crank == 0 && tid == 0)
            st.push_count = total;  // no CTA adds to it on this path
    } else {
        if (tid == kClThreads - 1) {
            const uint32_t total = (uint32_t)(off + cnt);
            st.push_base =
                total ? atom_add_cluster_u32(cluster_addr(&st.push_count, 0), total) : 0u;
        }
        __syncthreads();
        base = st.push_base;
    }
    {
        uint32_t slot = base + (uint32_t)off;
        const uint32_t cand0 = cluster_addr(&st.cand[0], 0);
        keys.each_from(lthr ? lthr : 1ull, [&](K x) {
            if (slot < (uint32_t)kClPushSlots)  // never reached: the bound only guards
                st_cluster_u64(cand0 + 8u * slot, row_key<T>(x, first));
            ++slot;
        });
    }
    cluster_barrier();  // every push has landed; no CTA touches another's memory after this
    if (crank != 0)
        return;

    // The first CTA: rank the pushed keys by counting, keep the k largest in
    // order, and take the sampling decision.
    // Four threads (adjacent lanes) per key, each counting the larger keys in a
    // quarter of the list.
    const int nc = min((int)st.push_count, kClPushSlots);
    {
        const int i = tid >> 2;
        const int q = tid & 3;
        const uint64_t mine = i < nc ? st.cand[i] : 0ull;
        int larger = 0;
        for (int j = q; j < nc; j += 4)
            larger += st.cand[j] > mine;
        larger += __shfl_xor_sync(0xFFFFFFFFu, larger, 1);
        larger += __shfl_xor_sync(0xFFFFFFFFu, larger, 2);
        if (i < nc && q == 0 && larger < k)
            st.ranked[larger] = mine;
    }
    __syncthreads();
    sample_decision<T>(st.ranked, k, gdraw, temperature, token_out + row, prob_out + row);
}

// The select and the sampling decision of one row's cluster, shared by the
// cluster kernels: `keys` walks this thread's keys of the chunk (KeySource
// below), `st` is the CTA's shared state (its first round's histogram zeroed
// and push_count, window and first set before the dependency wait).
template <typename T, class Keys>
__device__ __forceinline__ void cluster_select_sample(const Keys& keys, ClusterSelect& st,
                                                      int64_t row, int64_t first, int k,
                                                      const float (&gdraw)[2], float temperature,
                                                      int32_t* token_out, float* prob_out)
{
    using K = typename LocalKey<T>::type;
    constexpr int VS = LocalKey<T>::BITS - 16;  // leading 16 bits of a local key
    const int tid = (int)threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    // First round.  Each warp finds the r = ceil(k / 16) largest of its lanes'
    // largest keys; the smallest of the 16 warps' r-th values, `floor`, has at
    // least 16 r >= k of the CTA's keys at or above it, so the CTA's k-th
    // largest key, and with it the row's, is not below it: keys under `floor`
    // take no further part (typically all but a few dozen of the chunk's).
    // Then the CTA's largest leading 16 bits and its histogram of the
    // distances below them (the 256 nearest values) over the remaining keys.
    K floor;
    uint32_t top;
    {
        K cur = keys.max_key();
        const int r = (k + kClWarps - 1) / kClWarps;
        K wtop = 0, rth = 0;
        for (int i = 0; i < r; ++i) {
            const K w = warp_max(cur);
            if (i == 0)
                wtop = w;
            rth = w;
            if (cur == w)  // keys are distinct: the lane that holds it drops out
                cur = 0;
        }
        if (lane == 0) {
            st.warp_key[warp] = (uint64_t)wtop;
            st.warp_floor[warp] = (uint64_t)rth;
        }
        __syncthreads();
        uint64_t t = 0, f = ~0ull;
#pragma unroll
        for (int w = 0; w < kClWarps; ++w) {
            t = max(t, st.warp_key[w]);
            f = min(f, st.warp_floor[w]);
        }
        floor = (K)f;
        top = (uint32_t)(t >> VS);
    }
    keys.each_from(floor ? (uint64_t)floor : 1ull, [&](K x) {
        const uint32_t d = top - (uint32_t)(x >> VS);
        if (d < 256u)
            atomicAdd(&st.hist[0][d], 1u);
        if constexpr (Keys::kCompact) {  // the keys that take part, listed for the later passes
            const uint32_t slot = atomicAdd(&st.ncomp, 1u);
            if (slot < (uint32_t)kCompactKeys)
                keys.list[slot] = x;
        }
    });
    __syncthreads();  // the CTA's histogram (and list) is complete
    if constexpr (Keys::kCompact) {
        if (st.ncomp <= (uint32_t)kCompactKeys) {
            const ListKeys<K> listed{keys.list, (int)st.ncomp};
            cluster_finish<T>(listed, st, floor, top, row, first, k, gdraw, temperature,
                              token_out, prob_out);
            return;
        }
    }
    cluster_finish<T>(keys, st, floor, top, row, first, k, gdraw, temperature, token_out,
                      prob_out);
}

// What both cluster kernels do first: this CTA's chunk of its row into L2
// while the previous kernel drains, the first round's histogram zeroed and the
// shared state set, the dependency wait, and the first CTA's warp 0 loads the
// Gumbel draws of ranks lane and lane + 32.  Returns the chunk's first logit.
template <typename T>
__device__ __forceinline__ const T* cluster_prologue(ClusterSelect& st, const T* logits,
                                                     int64_t vocab, int chunk, int k,
                                                     const float* __restrict__ gumbel,
                                                     int64_t& first, int& n, float (&gdraw)[2])
{
    const int tid = (int)threadIdx.x;
    const uint32_t crank = cluster_ctarank();
    const int64_t row = blockIdx.y;
    first = (int64_t)crank * chunk;
    n = (int)(vocab - first < (int64_t)chunk ? (vocab - first > 0 ? vocab - first : 0)
                                              : (int64_t)chunk);
    const T* src = logits + row * vocab + first;
    {
        constexpr int kPerLine = 128 / sizeof(T);
        for (int i = tid * kPerLine; i < n; i += kClThreads * kPerLine)
            prefetch_l2_line(src + i);
    }
    for (int i = tid; i < 256; i += kClThreads)
        st.hist[0][i] = 0;
    if (tid == 0) {
        st.push_count = 0;
        st.window = 0;
        st.first = first;
        st.ncomp = 0;
    }
    pdl_wait();
    pdl_allow_dependents();
    gdraw[0] = gdraw[1] = 0.f;
    if (crank == 0 && tid < 32) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
            if (tid + 32 * r < k)
                gdraw[r] = __ldg(gumbel + row * k + tid + 32 * r);
    }
    return src;
}

// Grid (ncta, rows), clusters of ncta CTAs along x; CTA c of a row holds the
// row's logits [c * chunk, (c + 1) * chunk), M per thread in registers (chunk
// <= 512 M).  VEC: the chunk starts on a 16-byte boundary and thread t loads
// the 16-byte vectors at chunk positions (v * 512 + t) * E; otherwise one
// element at a time.
template <typename T, bool VEC, int M>
__global__ void __launch_bounds__(kClThreads, (sizeof(T) == 2 && M <= 16) ? 2 : 1)
topk_cluster_kernel(const T* __restrict__ logits, int64_t vocab, int chunk, int k,
                    const float* __restrict__ gumbel, float temperature,
                    int32_t* __restrict__ token_out, float* __restrict__ prob_out)
{
    using K = typename LocalKey<T>::type;
    constexpr int E = Vec<T>::N;
    static_assert(!VEC || M % E == 0, "whole vectors per thread");
    __shared__ ClusterSelect st;
    const int tid = (int)threadIdx.x;
    int64_t first;
    int n;
    float gdraw[2];
    const T* src = cluster_prologue<T>(st, logits, vocab, chunk, k, gumbel, first, n, gdraw);
    RegKeys<K, M> keys;
    if constexpr (VEC) {
#pragma unroll
        for (int v = 0; v < M / E; ++v) {
            const int p0 = (v * kClThreads + tid) * E;
            float f[E];
            if (p0 + E <= n) {
                Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(src + p0)), f);
            } else {
#pragma unroll
                for (int j = 0; j < E; ++j)
                    f[j] = (p0 + j < n) ? load_elem(src + p0 + j) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < E; ++j)
                keys.key[v * E + j] = (p0 + j < n) ? (((K)KeyBits<T>::of(f[j]) << 16) |
                                                      (K)(0xFFFFu - (uint32_t)(p0 + j)))
                                                   : K(0);
        }
    } else {
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const int p = tid + m * kClThreads;
            keys.key[m] = (p < n) ? (((K)KeyBits<T>::of(load_elem(src + p)) << 16) |
                                     (K)(0xFFFFu - (uint32_t)p))
                                  : K(0);
        }
    }
    cluster_select_sample<T>(keys, st, blockIdx.y, first, k, gdraw, temperature, token_out,
                             prob_out);
}

// Many-row variant: smaller clusters (up to 8 CTAs, so that many rows' clusters
// are resident at once) whose CTAs hold chunks too large for registers (up to
// ~76 KB of logits, 16-bit positions) in shared memory; the select walks them
// from there (SmemKeys).  VEC: 16-byte-aligned chunks copied with 16-byte
// loads, eight in flight per thread; otherwise one element at a time.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kClThreads, 2)
topk_cluster_smem_kernel(const T* __restrict__ logits, int64_t vocab, int chunk, int k,
                         const float* __restrict__ gumbel, float temperature,
                         int32_t* __restrict__ token_out, float* __restrict__ prob_out)
{
    constexpr int E = Vec<T>::N;
    extern __shared__ uint4 topk_chunk_smem[];  // the chunk, padded to whole vectors
    __shared__ ClusterSelect st;
    const int tid = (int)threadIdx.x;
    int64_t first;
    int n;
    float gdraw[2];
    const T* src = cluster_prologue<T>(st, logits, vocab, chunk, k, gumbel, first, n, gdraw);
    T* vals = reinterpret_cast<T*>(topk_chunk_smem);
    if constexpr (VEC) {
        constexpr int B = 8;
        const int nv = n / E;  // n is a multiple of E when rows are 16-byte aligned
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        for (int v0 = tid; v0 < nv; v0 += B * kClThreads) {
            uint4 r[B];
#pragma unroll
            for (int b = 0; b < B; ++b)
                if (v0 + b * kClThreads < nv)
                    r[b] = __ldg(s4 + v0 + b * kClThreads);
#pragma unroll
            for (int b = 0; b < B; ++b)
                if (v0 + b * kClThreads < nv)
                    topk_chunk_smem[v0 + b * kClThreads] = r[b];
        }
    } else {
        for (int p = tid; p < n; p += kClThreads)
            vals[p] = src[p];
    }
    __syncthreads();
    using K = typename LocalKey<T>::type;
    K* list = reinterpret_cast<K*>(topk_chunk_smem + (chunk * sizeof(T) + 15) / 16);
    const SmemKeys<T> keys{vals, n, list};
    cluster_select_sample<T>(keys, st, blockIdx.y, first, k, gdraw, temperature, token_out,
                             prob_out);
}

// ---------------------------------------------------------------------------
// Streaming variant for many rows: one CTA per row (a persistent grid of one
// CTA an SM walks the rows), the row streamed once through a ring of
// shared-memory stages filled by bulk copies (cp.async.bulk, mbarrier
// completion, every wait bounded).  Instead of a select over the whole row,
// the CTA keeps a running floor that at least k of the row's keys reach, so
// that no key under it can be among the k largest: first the smallest of the
// 16 warps' r-th largest lane maxima of the row's first stage (r = ceil(k /
// 16)), then, as keys are taken, the smallest of the warps' r-th largest lane
// values among the keys each lane appended.  Each 16-byte vector is tested
// against the floor's value with a few integer instructions; each warp lists
// its rare vectors holding a value at or above it and appends their keys (row
// keys, as cand_key) to a list in shared memory.  A list that would overflow
// is cut to its k largest (block select), which raises the floor, and the
// stage is taken again.  At the end of the row the list holds every key that
// can be among the k largest: the k largest of it are ranked and the decision
// taken as in the other kernels.  No exchange between CTAs and no global
// scratch.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr uint32_t kRowStage = 80 * 1024;                     // bytes a stage
constexpr int kRowStages = 2;                                 // stages in the ring
constexpr int kRowVecs = (int)(kRowStage / 16) / kRowThreads;  // vectors a thread a stage
constexpr int kRowListM = 9;                                  // list keys a thread at the end
constexpr uint32_t kRowList = kRowListM * kRowThreads;        // list capacity
constexpr size_t kRowSmem = (size_t)kRowStages * kRowStage + kRowList * sizeof(uint64_t);
static_assert(kRowWarps * 4 >= kMaxTopK, "at most four lanes a warp make the floor");
static_assert(kRowWarps % 4 == 0, "the warps' floors are read four at a time");
static_assert(kRowList >= (uint32_t)kMaxTopK + kRowThreads * 8, "a cut list takes a sub-round");

__device__ __forceinline__ uint32_t max_s16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Per-vector tests of the streaming kernel: the largest order value of a
// vector (vmax), whether a vector holds a value at or above the floor's
// (pass), and the order value of element e (ord; as KeyBits<T>::of).  While
// the floor's value is not negative (the usual case: the k-th largest logit
// is above zero), pass compares the raw bits as signed integers, which orders
// non-negative floats by value and puts every negative one below: two bf16 at
// a time with max.s16x2, three instructions for eight values.
template <typename T>
struct RowFilter;
template <>
struct RowFilter<__nv_bfloat16> {
    static constexpr int E = 8;
    uint32_t below2;  // order test: the floor's order value minus one, in both halves
    uint32_t sbelow2;  // signed test: the floor's raw bits minus one, in both halves
    bool all;          // floor order value 0: every vector passes
    bool pos;          // the floor's value is +0 or above: the signed test applies
    __device__ __forceinline__ void set(uint64_t floor)
    {
        const uint32_t fv = (uint32_t)(floor >> kIndexBits);
        all = fv == 0u;
        below2 = (fv - 1u) * 0x00010001u;
        pos = fv >= 0x8000u;
        sbelow2 = ((fv - 0x8000u - 1u) & 0xFFFFu) * 0x00010001u;
    }
    __device__ __forceinline__ static uint32_t max2(const uint4& x)
    {
        return max_u16x2(max_u16x2(ordered_bf16x2(x.x), ordered_bf16x2(x.y)),
                         max_u16x2(ordered_bf16x2(x.z), ordered_bf16x2(x.w)));
    }
    __device__ __forceinline__ static uint32_t vmax(const uint4& x)
    {
        const uint32_t m = max2(x);
        return max(m & 0xFFFFu, m >> 16);
    }
    template <bool POS>
    __device__ __forceinline__ bool pass(const uint4& x) const
    {
        if constexpr (POS) {
            const uint32_t m = max_s16x2(max_s16x2(x.x, x.y), max_s16x2(x.z, x.w));
            return max_s16x2(m, sbelow2) != sbelow2;
        } else {
            return all || max_u16x2(max2(x), below2) != below2;
        }
    }
    __device__ __forceinline__ static uint32_t ord(const uint4& x, int e)
    {
        const uint32_t w = e < 2 ? x.x : e < 4 ? x.y : e < 6 ? x.z : x.w;
        const uint32_t o = ordered_bf16x2(w);
        return (e & 1) ? (o >> 16) : (o & 0xFFFFu);
    }
};
template <>
struct RowFilter<float> {
    static constexpr int E = 4;
    uint32_t fv;
    int sfv;  // the floor's raw bits (signed test)
    bool pos;
    __device__ __forceinline__ void set(uint64_t floor)
    {
        fv = (uint32_t)(floor >> kIndexBits);
        pos = fv >= 0x80000000u;
        sfv = (int)(fv & 0x7FFFFFFFu);
    }
    __device__ __forceinline__ static uint32_t vmax(const uint4& x)
    {
        return max(max(order_bits(__uint_as_float(x.x)), order_bits(__uint_as_float(x.y))),
                   max(order_bits(__uint_as_float(x.z)), order_bits(__uint_as_float(x.w))));
    }
    template <bool POS>
    __device__ __forceinline__ bool pass(const uint4& x) const
    {
        if constexpr (POS)
            return max(max((int)x.x, (int)x.y), max((int)x.z, (int)x.w)) >= sfv;
        else
            return vmax(x) >= fv;
    }
    __device__ __forceinline__ static uint32_t ord(const uint4& x, int e)
    {
        const uint32_t w = e == 0 ? x.x : e == 1 ? x.y : e == 2 ? x.z : x.w;
        return order_bits(__uint_as_float(w));
    }
};

// Rows start on 16-byte boundaries and hold a whole number of vectors (the
// bulk copies need both).
template <typename T>
__global__ void __launch_bounds__(kRowThreads, 1)
topk_row_kernel(const T* __restrict__ logits, int64_t rows, int64_t vocab, int k,
                const float* __restrict__ gumbel, float temperature,
                int32_t* __restrict__ token_out, float* __restrict__ prob_out, unsigned* err_word)
{
    using F = RowFilter<T>;
    constexpr int E = F::E;
    constexpr uint32_t kStageVecs = kRowStage / 16;
    extern __shared__ uint4 topk_row_smem[];  // the ring of stages, then the list
    __shared__ SelectState st;
    __shared__ uint64_t sel[kMaxTopK];
    __shared__ uint64_t ranked[kMaxTopK];
    __shared__ __align__(8) uint64_t bars[kRowStages];
    __shared__ uint64_t s_floor;
    __shared__ uint32_t s_count;   // keys appended to the list (may run past its capacity)
    __shared__ int s_over;         // an append found the list full
    __shared__ uint16_t s_vlist[kStageVecs];  // per warp: its vectors at or above the floor
    __shared__ uint32_t s_wfloor[kRowWarps];
    __shared__ __align__(16) uint32_t s_wlv[kRowWarps];  // per warp: r-th largest of its lanes' appended values

    const int tid = (int)threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    uint64_t* list = reinterpret_cast<uint64_t*>(topk_row_smem + (size_t)kRowStages * kStageVecs);
    const uint32_t row_bytes = (uint32_t)vocab * (uint32_t)sizeof(T);
    const int nst = (int)((row_bytes + kRowStage - 1) / kRowStage);
    const int64_t my_rows =
        rows > (int64_t)blockIdx.x ? (rows - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t total = my_rows * nst;  // stages this CTA streams

    if (tid == 0) {
        for (int s = 0; s < kRowStages; ++s)
            mbar_init(smem_addr(&bars[s]), 1);
        mbar_init_fence();
    }
    // the first row into L2 while the previous kernel drains, a stage a thread
    if (my_rows > 0 && tid < nst) {
        const uint32_t off = (uint32_t)tid * kRowStage;
        prefetch_l2(reinterpret_cast<const unsigned char*>(logits + (int64_t)blockIdx.x * vocab) + off,
                    min(kRowStage, row_bytes - off));
    }
    __syncthreads();
    pdl_wait();
    pdl_allow_dependents();

    // The producer (thread 0) walks the same sequence of (row, stage, slot)
    // as the consumers, counters instead of divisions.
    int64_t issued = 0;  // stages requested (meaningful in thread 0 only)
    int64_t prow = blockIdx.x;
    int pst = 0, pslot = 0;
    auto issue = [&]() {
        const uint32_t off = (uint32_t)pst * kRowStage;
        const uint32_t bytes = min(kRowStage, row_bytes - off);
        const uint32_t bar = smem_addr(&bars[pslot]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(smem_addr(topk_row_smem + (size_t)pslot * kStageVecs),
                  reinterpret_cast<const unsigned char*>(logits + prow * vocab) + off, bytes, bar);
        ++issued;
        if (++pst == nst) {
            pst = 0;
            prow += gridDim.x;
        }
        if (++pslot == kRowStages)
            pslot = 0;
    };
    if (tid == 0)
        while (issued < kRowStages && issued < total)
            issue();

    F filt;
    uint64_t floor = 0;
    uint32_t lval = 0;  // largest order value among the keys this lane appended (this row)
    const int r = (k + kRowWarps - 1) / kRowWarps;
    float gdraw[2] = {0.f, 0.f};
    // list length when the stage began, read while no thread appends (after
    // the previous stage's last barrier, before the next stage's first)
    uint32_t cnt0 = 0;
    bool ok = true;
    int s = 0, buf = 0;
    uint32_t phase = 0;
    int64_t row = blockIdx.x;
    for (int64_t g = 0; g < total; ++g) {
        ok = ok && mbar_wait(smem_addr(&bars[buf]), phase);
        if (__syncthreads_or(!ok)) {
            // a copy did not land in time: record it, let this CTA's copies
            // still in flight finish (bounded), and give up
            if (tid == 0) {
                record_device_error(err_word, kDeviceErrTimeout);
                uint32_t ph = phase;
                for (int64_t q = g, b = buf; q < issued; ++q) {
                    mbar_wait(smem_addr(&bars[b]), ph);
                    if (++b == kRowStages) {
                        b = 0;
                        ph ^= 1u;
                    }
                }
            }
            return;
        }
        // every thread is done with stage g - 1: its slot takes stage g - 1 + stages
        if (tid == 0 && g >= 1 && issued < total)
            issue();
        const uint4* sb = topk_row_smem + (size_t)buf * kStageVecs;
        const int nvs = (int)(min(kRowStage, row_bytes - (uint32_t)s * kRowStage) / 16);
        const int64_t jbase = (int64_t)s * kStageVecs;  // row vector index of sb[0]

        if (s == 0) {
            // a new row: the floor from this stage's values
            uint32_t mx = 0;
#pragma unroll
            for (int i = 0; i < kRowVecs; ++i) {
                const int j = tid + i * kRowThreads;
                if (j < nvs)
                    mx = max(mx, F::vmax(sb[j]));
            }
            uint32_t cur = mx, rth = 0;
            for (int got = 0; got < r;) {
                const uint32_t w = __reduce_max_sync(0xFFFFFFFFu, cur);
                rth = w;
                if (w == 0u)
                    break;
                got += __popc(__ballot_sync(0xFFFFFFFFu, cur == w));
                if (cur == w)
                    cur = 0;
            }
            if (lane == 0) {
                s_wfloor[warp] = rth;
                s_wlv[warp] = 0;
            }
            lval = 0;
            if (tid == 0) {
                s_count = 0;
                s_over = 0;
            }
            if (tid < 32) {
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    if (tid + 32 * q < k)
                        gdraw[q] = __ldg(gumbel + row * k + tid + 32 * q);
            }
            __syncthreads();
            uint32_t fv = 0xFFFFFFFFu;
#pragma unroll
            for (int w = 0; w < kRowWarps; ++w)
                fv = min(fv, s_wfloor[w]);
            floor = (uint64_t)fv << kIndexBits;
            filt.set(floor);
            if (tid == 0)
                s_floor = floor;
            cnt0 = 0;
        }

        // The keys at or above the floor of entry q of this warp's list,
        // appended to the list (one atomic a vector; a handful of vectors a
        // warp and stage once the floor has risen).
        uint16_t* wlist = s_vlist + warp * (kRowVecs * 32);
        auto take = [&](uint32_t q) {
            const uint32_t fv = (uint32_t)(floor >> kIndexBits);
            const uint32_t flo = (uint32_t)floor & ((1u << kIndexBits) - 1u);
            const int j = wlist[q];
            const uint4 x = sb[j];
            const uint32_t inv0 = (1u << kIndexBits) - 1u - (uint32_t)((jbase + j) * E);
            uint32_t o[E], mask = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                o[e] = F::ord(x, e);
                if (o[e] > fv || (o[e] == fv && inv0 - (uint32_t)e >= flo)) {
                    mask |= 1u << e;
                    lval = max(lval, o[e]);
                }
            }
            if (mask == 0u)
                return;
            uint32_t slot = atomicAdd(&s_count, (uint32_t)__popc(mask));
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (mask & (1u << e)) {
                    if (slot < kRowList)
                        list[slot] = ((uint64_t)o[e] << kIndexBits) | (uint64_t)(inv0 - (uint32_t)e);
                    else
                        s_over = 1;
                    ++slot;
                }
        };
        // Each warp lists its vectors of the stage that hold a value at or
        // above the floor's (a ballot an iteration, into its own part of
        // s_vlist), then forms and appends their keys itself, a vector a
        // lane: no block barrier between the two.
        uint32_t wn = 0;  // vectors this warp listed
        auto scan = [&](auto pos) {
            // all of the thread's loads first (a full stage needs no bounds
            // test; the last one of a row reads stale but in-bounds slots
            // past its end, which the mask drops)
            uint4 v[kRowVecs];
#pragma unroll
            for (int i = 0; i < kRowVecs; ++i)
                v[i] = sb[tid + i * kRowThreads];
            uint32_t pm = 0;  // this thread's vectors that pass
#pragma unroll
            for (int i = 0; i < kRowVecs; ++i)
                if (filt.template pass<decltype(pos)::value>(v[i]) && tid + i * kRowThreads < nvs)
                    pm |= 1u << i;
            if (__any_sync(0xFFFFFFFFu, pm != 0u)) {  // rare once the floor has risen
#pragma unroll
                for (int i = 0; i < kRowVecs; ++i) {
                    const bool p = (pm >> i) & 1u;
                    const uint32_t b = __ballot_sync(0xFFFFFFFFu, p);
                    if (p)
                        wlist[wn + __popc(b & ((1u << lane) - 1u))] =
                            (uint16_t)(tid + i * kRowThreads);
                    wn += __popc(b);
                }
            }
        };
        if (filt.pos)
            scan(std::true_type{});
        else
            scan(std::false_type{});
        __syncwarp();
        for (uint32_t q = (uint32_t)lane; q < wn; q += 32)
            take(q);
        if (wn > 0u && s_wlv[warp] <= (uint32_t)(floor >> kIndexBits)) {
            // A second floor: the r-th largest of the warp's lanes' largest
            // appended values (each lane's keys are its own, so r of them are
            // at or above it in every warp, 16 r >= k in all).  It only rises
            // as the row goes on.  Only a warp whose value holds the floor
            // down updates it (the others' stay valid, if lower).
            uint32_t cur = lval, rth = 0;
            for (int got = 0; got < r;) {
                const uint32_t w = __reduce_max_sync(0xFFFFFFFFu, cur);
                rth = w;
                if (w == 0u)
                    break;
                got += __popc(__ballot_sync(0xFFFFFFFFu, cur == w));
                if (cur == w)
                    cur = 0;
            }
            if (lane == 0)
                s_wlv[warp] = rth;
        }
        __syncthreads();

        if (s_over) {
            // The list ran full in this stage: drop the stage's appends, and
            // take the listed vectors again, 32 a warp at a time, cutting the
            // list to its k largest (which raises the floor) whenever a round
            // might not fit.
            __syncthreads();  // every thread has read s_over
            if (tid == 0) {
                s_count = cnt0;
                s_over = 0;
            }
            __syncthreads();
            for (int i = 0; i < kRowVecs; ++i) {
                const uint32_t n = s_count;
                __syncthreads();  // every thread has read it before any appends
                if (n > kRowList - (uint32_t)(kRowThreads * E)) {
                    uint64_t key[kRowListM];
                    bool valid[kRowListM];
#pragma unroll
                    for (int m = 0; m < kRowListM; ++m) {
                        const uint32_t q = (uint32_t)(tid + m * kRowThreads);
                        valid[m] = q < n;
                        key[m] = valid[m] ? list[q] : 0ull;
                    }
                    select_top_k<KeyBits<T>::V + kIndexBits>(key, valid, k, st);
                    int c = 0;
#pragma unroll
                    for (int m = 0; m < kRowListM; ++m)
                        c += valid[m] && selected(key[m], st);
                    int slot = selected_offset(c, reinterpret_cast<int*>(st.warp_top));
#pragma unroll
                    for (int m = 0; m < kRowListM; ++m)
                        if (valid[m] && selected(key[m], st)) {
                            if (slot < k)
                                list[slot] = key[m];
                            ++slot;
                        }
                    if (tid == 0) {
                        const uint64_t t = (st.tau >> st.shift) << st.shift;
                        s_floor = max(s_floor, t);
                        s_count = (uint32_t)k;
                    }
                    __syncthreads();
                    floor = s_floor;
                    filt.set(floor);
                }
                if ((uint32_t)(32 * i + lane) < wn)
                    take((uint32_t)(32 * i + lane));
                __syncthreads();
            }
        }
        cnt0 = s_count;
        {
            // the floor rises to the smallest of the warps' second floors
            uint32_t fv2 = 0xFFFFFFFFu;
#pragma unroll
            for (int w = 0; w < kRowWarps; w += 4) {
                const uint4 v = *reinterpret_cast<const uint4*>(&s_wlv[w]);
                fv2 = min(fv2, min(min(v.x, v.y), min(v.z, v.w)));
            }
            const uint64_t nf = (uint64_t)fv2 << kIndexBits;
            if (nf > floor) {
                floor = nf;
                filt.set(floor);
                if (tid == 0)
                    s_floor = max(s_floor, nf);
            }
        }

        if (s == nst - 1) {
            // the row's last stage: the k largest of the list, ranked, and the decision
            const uint32_t n = min(s_count, kRowList);
            auto finish = [&](auto m_tag) {
                constexpr int M = decltype(m_tag)::value;
                uint64_t key[M];
                bool valid[M];
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const uint32_t q = (uint32_t)(tid + m * kRowThreads);
                    valid[m] = q < n;
                    key[m] = valid[m] ? list[q] : 0ull;
                }
                rank_and_sample<T>(key, valid, k, gdraw, temperature, token_out + row,
                                   prob_out + row, st, sel, ranked);
            };
            // usually a few hundred keys: two a thread
            if (n <= 2u * kRowThreads)
                finish(std::integral_constant<int, 2>{});
            else
                finish(std::integral_constant<int, kRowListM>{});
        }
        if (++s == nst) {
            s = 0;
            row += gridDim.x;
        }
        if (++buf == kRowStages) {
            buf = 0;
            phase ^= 1u;
        }
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

size_t topk_counter_bytes()
{
    return kCounterBytes;
}

namespace {

// Shape of the register launch for a vocabulary: the fewest CTAs per cluster
// (a power of two up to max_ncta) that hold the row at 8 logits a thread, else
// max_ncta CTAs; each CTA's chunk is a multiple of 8 logits (so every chunk of
// a 16-byte-aligned row starts on a 16-byte boundary) and M = logits a thread
// (a shape whose M has no instantiation is not launched).
struct ClusterShape {
    int ncta;
    int chunk;
    int m;
};

ClusterShape cluster_shape(int64_t vocab, int max_ncta)
{
    int ncta = 1;
    while (ncta < max_ncta && (int64_t)ncta * kClThreads * 8 < vocab)
        ncta *= 2;
    const int64_t chunk = (int64_t)round_up((uint32_t)ceil_div(vocab, ncta), 8u);
    const int m = (int)round_up((uint32_t)ceil_div(chunk, kClThreads), 8u);
    return {ncta, (int)chunk, m};
}

// Clusters of `ncta` CTAs of `Kernel` (with `smem` bytes of dynamic shared
// memory a CTA) that the current device holds at once (0 if it cannot run
// them; above 8 CTAs it first allows the non-portable cluster size on the
// kernel).  Looked up once per device and cluster size: every launcher passes
// one `smem` per kernel (its largest).
template <auto Kernel>
int cluster_capacity(int ncta, size_t smem = 0)
{
    constexpr int kMaxDevices = 64;
    constexpr int kSizes = 5;  // 1, 2, 4, 8, 16 CTAs
    static std::atomic<int> cache[kMaxDevices][kSizes];  // capacity + 1; 0 = not looked up
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 0;
    int slot = 0;
    while ((1 << slot) < ncta && slot < kSizes - 1)
        ++slot;
    int v = cache[dev][slot].load(std::memory_order_relaxed);
    if (v == 0) {
        int clusters = 0;
        const bool attrs_ok =
            (ncta <= 8 ||
             cudaFuncSetAttribute(Kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                 cudaSuccess) &&
            (smem <= 48 * 1024 ||
             cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem) == cudaSuccess);
        if (attrs_ok) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)ncta, 1);
            cfg.blockDim = dim3(kClThreads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)ncta;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&clusters, Kernel, &cfg) != cudaSuccess)
                clusters = 0;
        }
        (void)cudaGetLastError();  // a refused query leaves no sticky error behind
        v = clusters + 1;
        cache[dev][slot].store(v, std::memory_order_relaxed);
    }
    return v - 1;
}

// Kernel attributes a cluster launch needs (the non-portable cluster size
// above 8 CTAs, dynamic shared memory above 48 KB), set once per device: a
// call costs several microseconds on the host, as much as the kernel.  They
// belong to a CUDA context, so a launch that is refused (a context created
// after they were set) sets them again and retries once (launch_with_attrs).
template <auto Kernel>
cudaError_t set_cluster_attrs(int ncta, size_t smem, bool force)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<int> done[kMaxDevices];  // 1: set on that device
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices)
        dev = -1;
    if (!force && dev >= 0 && done[dev].load(std::memory_order_relaxed))
        return cudaSuccess;
    cudaError_t e = cudaSuccess;
    if (ncta > 8)
        e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess && smem > 48 * 1024)
        e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return e;
    }
    if (dev >= 0)
        done[dev].store(1, std::memory_order_relaxed);
    return cudaSuccess;
}

template <typename T, bool VEC, int M>
cudaError_t launch_cluster_t(const T* logits, const float* gumbel, int32_t* token_out,
                             float* prob_out, int64_t rows, int64_t vocab, int k,
                             float temperature, const ClusterShape& cs, cudaStream_t stream,
                             bool* launched)
{
    constexpr auto kernel = topk_cluster_kernel<T, VEC, M>;
    *launched = false;
    // Only while every row's cluster is resident at once: beyond that the
    // clusters run in waves and the slice kernel (many small CTAs) is faster
    // (5 rows of 151936 logits: 11.2 against 12.3 us a launch back to back on
    // B200; 8 rows: 18.4 against 14.7).
    if (rows > cluster_capacity<kernel>(cs.ncta))
        return cudaSuccess;
    // refused attributes: the slice kernel takes the call
    if (set_cluster_attrs<kernel>(kClMaxCtas, 0, false) != cudaSuccess)
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs.ncta, (unsigned)rows);
    cfg.blockDim = dim3(kClThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs.ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (pdl_enabled()) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    }
    *launched = true;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, logits, vocab, cs.chunk, k, gumbel,
                                         temperature, token_out, prob_out);
    if (err != cudaSuccess && cs.ncta > 8) {  // attributes of another context: set, retry
        (void)cudaGetLastError();
        if (set_cluster_attrs<kernel>(kClMaxCtas, 0, true) == cudaSuccess)
            err = cudaLaunchKernelEx(&cfg, kernel, logits, vocab, cs.chunk, k, gumbel,
                                     temperature, token_out, prob_out);
    }
    if (err == cudaSuccess)
        count_launch();
    return err;
}

template <typename T, bool VEC>
cudaError_t launch_cluster_m(const T* logits, const float* gumbel, int32_t* token_out,
                             float* prob_out, int64_t rows, int64_t vocab, int k,
                             float temperature, const ClusterShape& cs, cudaStream_t stream,
                             bool* launched)
{
    switch (cs.m) {
    case 8:
        return launch_cluster_t<T, VEC, 8>(logits, gumbel, token_out, prob_out, rows, vocab, k,
                                           temperature, cs, stream, launched);
    case 16:
        return launch_cluster_t<T, VEC, 16>(logits, gumbel, token_out, prob_out, rows, vocab, k,
                                            temperature, cs, stream, launched);
    case 24:
        return launch_cluster_t<T, VEC, 24>(logits, gumbel, token_out, prob_out, rows, vocab, k,
                                            temperature, cs, stream, launched);
    case 32:
        return launch_cluster_t<T, VEC, 32>(logits, gumbel, token_out, prob_out, rows, vocab, k,
                                            temperature, cs, stream, launched);
    case 40:
        return launch_cluster_t<T, VEC, 40>(logits, gumbel, token_out, prob_out, rows, vocab, k,
                                            temperature, cs, stream, launched);
    default:
        *launched = false;
        return cudaSuccess;
    }
}

// Shape of the many-row launch: the fewest CTAs per cluster (a power of two
// up to 8, the portable size) whose chunks hold at most ~76 KB of logits and
// 65,528 positions (16-bit local positions, multiples of 8 logits), so that
// two CTAs share an SM and many rows' clusters are resident at once; more
// CTAs when there are few rows.  ncta = 0 when no such shape exists.
struct SmemShape {
    int ncta;
    int chunk;
    size_t smem;  // dynamic shared memory a CTA: the chunk's values
};

constexpr size_t kSmemChunkTarget = 76 * 1024;
constexpr int kSmemMaxChunk = 65528;
constexpr size_t kSmemMaxBytes = 144 * 1024;  // fp32 rows of 262,144 logits over 8 CTAs

SmemShape smem_shape(int64_t vocab, size_t esize, int64_t rows, int sm_count)
{
    int ncta = 1;
    while (ncta < 8 && ((size_t)ceil_div(vocab, ncta) * esize > kSmemChunkTarget ||
                        ceil_div(vocab, ncta) > kSmemMaxChunk))
        ncta *= 2;
    // Few rows: twice the CTAs on half the chunk while the rows' CTAs would
    // fill at most half the SMs (8 rows of 151,936 bf16 logits: 10.9 against
    // 13.0 us back to back on B200 with 8 CTAs instead of 4; equal at 16
    // rows, slower at 32).
    while (ncta < 8 && rows * ncta * 2 <= sm_count && ceil_div(vocab, 2 * ncta) >= 4096)
        ncta *= 2;
    const int64_t chunk = (int64_t)round_up((uint32_t)ceil_div(vocab, ncta), 8u);
    if (chunk > kSmemMaxChunk || (size_t)chunk * esize + kCompactKeys * 8 > kSmemMaxBytes)
        return {0, 0, 0};
    const size_t key_bytes = esize == 2 ? 4 : 8;
    return {ncta, (int)chunk, (size_t)chunk * esize + kCompactKeys * key_bytes};
}

template <typename T, bool VEC>
cudaError_t launch_cluster_smem(const T* logits, const float* gumbel, int32_t* token_out,
                                float* prob_out, int64_t rows, int64_t vocab, int k,
                                float temperature, cudaStream_t stream, bool* launched)
{
    constexpr auto kernel = topk_cluster_smem_kernel<T, VEC>;
    *launched = false;
    DeviceInfo di;
    if (current_device_info(&di) != cudaSuccess)
        return cudaSuccess;
    const SmemShape ss = smem_shape(vocab, sizeof(T), rows, di.sm_count);
    if (ss.ncta == 0 || cluster_capacity<kernel>(ss.ncta, kSmemMaxBytes) < 1)
        return cudaSuccess;
    if (set_cluster_attrs<kernel>(8, kSmemMaxBytes, false) != cudaSuccess)
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ss.ncta, (unsigned)rows);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = ss.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ss.ncta;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (pdl_enabled()) {
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 2;
    }
    *launched = true;
    cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, logits, vocab, ss.chunk, k, gumbel,
                                         temperature, token_out, prob_out);
    if (err != cudaSuccess && ss.smem > 48 * 1024) {  // attributes of another context
        (void)cudaGetLastError();
        if (set_cluster_attrs<kernel>(8, kSmemMaxBytes, true) == cudaSuccess)
            err = cudaLaunchKernelEx(&cfg, kernel, logits, vocab, ss.chunk, k, gumbel,
                                     temperature, token_out, prob_out);
    }
    if (err == cudaSuccess)
        count_launch();
    return err;
}

// The streaming kernel on a persistent grid of one CTA an SM (its shared
// memory holds one); rows must be 16-byte aligned whole vectors.
template <typename T>
cudaError_t launch_row(const T* logits, const float* gumbel, int32_t* token_out, float* prob_out,
                       int64_t rows, int64_t vocab, int k, float temperature, cudaStream_t stream,
                       bool* launched)
{
    constexpr auto kernel = topk_row_kernel<T>;
    *launched = false;
    DeviceInfo di;
    if (current_device_info(&di) != cudaSuccess)
        return cudaSuccess;
    unsigned* word = nullptr;
    if (device_error_word(&word) != cudaSuccess) {
        (void)cudaGetLastError();
        return cudaSuccess;
    }
    if (set_cluster_attrs<kernel>(1, kRowSmem, false) != cudaSuccess)
        return cudaSuccess;
    const unsigned grid = (unsigned)std::min<int64_t>(rows, di.sm_count);
    *launched = true;
    cudaError_t err = launch(kernel, dim3(grid), dim3(kRowThreads), kRowSmem, stream, logits, rows,
                             vocab, k, gumbel, temperature, token_out, prob_out, word);
    if (err != cudaSuccess) {  // attributes of another context
        (void)cudaGetLastError();
        if (set_cluster_attrs<kernel>(1, kRowSmem, true) == cudaSuccess)
            err = launch(kernel, dim3(grid), dim3(kRowThreads), kRowSmem, stream, logits, rows,
                         vocab, k, gumbel, temperature, token_out, prob_out, word);
    }
    return err;
}

}  // namespace

cudaError_t launch_topk_sample(const void* logits, const float* gumbel, int32_t* token_out,
                               float* prob_out, int64_t rows, int64_t vocab, int k,
                               float temperature, arops_dtype dtype, void* workspace,
                               cudaStream_t stream)
{
    const size_t esize = dtype == AROPS_BF16 ? 2 : 4;
    const bool vec = aligned16(logits) && (vocab * esize) % 16 == 0;
    const int mode = topk_cluster_mode();
    // Many rows (more than a quarter as many as SMs): the streaming kernel, one
    // CTA a row.  151,936 bf16 logits on B200, back to back: 64 rows 16.1
    // against 18.3 us on the shared-memory cluster kernel, 128 rows 17.7
    // against 34.3, 256 rows 31.2 against 63.5; at 32 rows 16.0 against 15.1.
    bool many = false;
    if (mode == 1 && vec) {
        DeviceInfo di;
        many = current_device_info(&di) == cudaSuccess && rows * 4 > di.sm_count;
    }
    if ((mode == 3 || many) && vec) {
        bool launched = false;
        cudaError_t err =
            dtype == AROPS_BF16
                ? launch_row(static_cast<const __nv_bfloat16*>(logits), gumbel, token_out,
                             prob_out, rows, vocab, k, temperature, stream, &launched)
                : launch_row(static_cast<const float*>(logits), gumbel, token_out, prob_out,
                             rows, vocab, k, temperature, stream, &launched);
        if (launched)
            return err;
    }
    if (mode != 0) {
        bool launched = false;
        cudaError_t err = cudaSuccess;
        // Few rows: the register cluster kernel while every row's cluster is
        // resident at once (mode 1), on clusters of up to 16 CTAs, then of up
        // to 8 (more of them fit at once: 8 or 12 rows of 151,936 bf16 logits
        // measured 10.0 against 10.9 and 11.1 us back to back on B200 with the
        // shared-memory kernel, which takes every larger call).
        auto try_registers = [&](const ClusterShape& cs) {
            if (dtype == AROPS_BF16) {
                const auto* lg = static_cast<const __nv_bfloat16*>(logits);
                err = vec ? launch_cluster_m<__nv_bfloat16, true>(lg, gumbel, token_out, prob_out,
                                                                  rows, vocab, k, temperature, cs,
                                                                  stream, &launched)
                          : launch_cluster_m<__nv_bfloat16, false>(lg, gumbel, token_out, prob_out,
                                                                   rows, vocab, k, temperature,
                                                                   cs, stream, &launched);
            } else {
                const auto* lg = static_cast<const float*>(logits);
                err = vec ? launch_cluster_m<float, true>(lg, gumbel, token_out, prob_out, rows,
                                                          vocab, k, temperature, cs, stream,
                                                          &launched)
                          : launch_cluster_m<float, false>(lg, gumbel, token_out, prob_out, rows,
                                                           vocab, k, temperature, cs, stream,
                                                           &launched);
            }
        };
        if (mode == 1) {
            const ClusterShape wide = cluster_shape(vocab, kClMaxCtas);
            try_registers(wide);
            if (!launched) {
                const ClusterShape narrow = cluster_shape(vocab, 8);
                if (narrow.ncta < wide.ncta)
                    try_registers(narrow);
            }
        }
        if (!launched) {
            if (dtype == AROPS_BF16) {
                const auto* lg = static_cast<const __nv_bfloat16*>(logits);
                err = vec ? launch_cluster_smem<__nv_bfloat16, true>(lg, gumbel, token_out,
                                                                     prob_out, rows, vocab, k,
                                                                     temperature, stream,
                                                                     &launched)
                          : launch_cluster_smem<__nv_bfloat16, false>(lg, gumbel, token_out,
                                                                      prob_out, rows, vocab, k,
                                                                      temperature, stream,
                                                                      &launched);
            } else {
                const auto* lg = static_cast<const float*>(logits);
                err = vec ? launch_cluster_smem<float, true>(lg, gumbel, token_out, prob_out, rows,
                                                             vocab, k, temperature, stream,
                                                             &launched)
                          : launch_cluster_smem<float, false>(lg, gumbel, token_out, prob_out,
                                                              rows, vocab, k, temperature, stream,
                                                              &launched);
            }
        }
        if (launched)
            return err;
        // no cluster launch possible here: the slice kernel
    }
    const int slices = topk_slices(vocab);
    const dim3 grid((unsigned)slices, (unsigned)rows);
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
