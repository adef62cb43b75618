// RMSNorm, LayerNorm and their fused residual-add forms (sm_100a).
//
// RMSNorm: y = gamma * x / sqrt(mean(x^2) + eps) over each row
// ("Optimising autoregressive speech models", §09, the RMSNorm equation and
// module); LayerNorm: y = gamma * (x - mean) / sqrt(var + eps) + beta (same
// section).  Norm+Residual (Triton kernel-fusion post for Qwen3-TTS, section 3):
// residual_out = round(x + residual_in), y = norm(residual_out), in one pass.
//
// Two designs.  The register kernels (the default) keep the row in registers:
// a row of `hidden` elements is split into 16-byte vectors; a group of 32*GW
// threads owns the row and every thread holds VPL vectors, so global memory is
// read once and written once (x, residual -> residual_out, y) with fully
// coalesced 128-bit accesses.  The sum of squares is accumulated in fp32,
// reduced with warp shuffles and, for GW > 1 warps per row, one shared-memory
// step; rsqrtf of (sum * 1/hidden + eps) scales the row and x * r * gamma is
// rounded once to the storage type.  gamma (and beta) is read through the
// read-only path once per thread, before the dependency wait, so a row costs
// one memory round trip.  A problem of at most one vector per resident thread
// (a decode step's few rows) takes one vector per lane with the row spread
// over GW = hidden/256 warps; larger ones take 4 or 8 vectors per lane, one or
// two warps per row up to 2048 bf16 elements.  The streaming kernel (opt-in,
// arops_set_streaming) stages rows through shared memory with bulk copies
// instead; it measured slower on B200.
//
// Rows longer than 4096 vectors, and unaligned or ragged rows, take a looped
// kernel that makes a second pass over the row (served from L2).
#include "common.cuh"
#include "tma.cuh"

namespace arops {
namespace {

// ---------------------------------------------------------------------------
// Streaming kernel (opt-in: arops_set_streaming(1)).  A persistent CTA
// owns rows blockIdx.x, blockIdx.x + gridDim.x, ...  One thread keeps `stages`
// rows in flight as bulk copies (TMA) into a ring of shared-memory slots, each
// slot holding the row of x (and of the residual); gamma is copied once per
// CTA.  As a row lands, the CTA adds the residual, writes residual_out, reduces
// the sum of squares (warp shuffles, then one shared-memory step), and writes
// y.  With several CTAs per SM and 4 stages, an SM has its whole share of a
// 4096 x 2048 problem requested within the first microsecond.  On B200 it ran
// slower than the register kernels (21.0 vs 17.0 us for 4096 x 2048): the ring
// left too few warps for the arithmetic.
// ---------------------------------------------------------------------------
template <typename T, bool ADD, int THREADS>
__global__ void __launch_bounds__(THREADS)
norm_tma_kernel(const T* x, const T* residual_in, T* residual_out, const T* __restrict__ gamma,
                T* y, int64_t rows, int hidden, float eps, float inv_hidden, int stages,
                unsigned* err_word)
{
    constexpr int E = Vec<T>::N;
    constexpr int W = THREADS / 32;
    constexpr int NT = ADD ? 2 : 1;  // tensors streamed per row
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red[W];

    const int tid = threadIdx.x;
    const int nvec = hidden / E;
    const uint32_t row_bytes = (uint32_t)hidden * (uint32_t)sizeof(T);
    const uint32_t slot = round_up(row_bytes, 128);
    unsigned char* s_gamma = smem;
    unsigned char* s_ring = smem + slot;
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_ring + (size_t)stages * NT * slot);
    const uint32_t gamma_bar = smem_addr(&bars[stages]);
    const int64_t my_rows =
        rows > (int64_t)blockIdx.x ? (rows - 1 - (int64_t)blockIdx.x) / gridDim.x + 1 : 0;

    if (tid == 0) {
        for (int s = 0; s <= stages; ++s)
            mbar_init(smem_addr(&bars[s]), 1);
        mbar_init_fence();
    }
    __syncthreads();

    pdl_wait();
    pdl_allow_dependents();

    int64_t issued = 0;  // meaningful in thread 0 only
    auto issue = [&](int64_t j) {
        const int s = (int)(j % stages);
        const int64_t row = (int64_t)blockIdx.x + j * gridDim.x;
        const uint32_t bar = smem_addr(&bars[s]);
        unsigned char* dst = s_ring + (size_t)s * NT * slot;
        mbar_arrive_expect_tx(bar, NT * row_bytes);
        bulk_load(smem_addr(dst), x + row * hidden, row_bytes, bar);
        if constexpr (ADD)
            bulk_load(smem_addr(dst + slot), residual_in + row * hidden, row_bytes, bar);
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(gamma_bar, row_bytes);
        bulk_load(smem_addr(s_gamma), gamma, row_bytes, gamma_bar);
        for (; issued < stages && issued < my_rows; ++issued)
            issue(issued);
    }

    bool ok = mbar_wait(gamma_bar, 0);
    for (int64_t j = 0; j < my_rows; ++j) {
        const int s = (int)(j % stages);
        ok = ok && mbar_wait(smem_addr(&bars[s]), (uint32_t)((j / stages) & 1));
        if (__syncthreads_or(!ok)) {
            // a copy did not land in time: record it, let this CTA's copies
            // still in flight finish (bounded), and give up
            if (tid == 0) {
                record_device_error(err_word, kDeviceErrTimeout);
                mbar_wait(gamma_bar, 0);
                for (int64_t k = j; k < issued; ++k)
                    mbar_wait(smem_addr(&bars[k % stages]), (uint32_t)((k / stages) & 1));
            }
            return;
        }
        // every thread is past row j-1 (it reached the barrier above), so row
        // j-1's slot can take row j-1+stages; at j == 0 no slot is free yet
        if (tid == 0 && j >= 1 && issued < my_rows) {
            issue(issued);
            ++issued;
        }

        const int64_t row = (int64_t)blockIdx.x + j * gridDim.x;
        unsigned char* sx = s_ring + (size_t)s * NT * slot;
        float ss = 0.f;
        for (int v = tid; v < nvec; v += THREADS) {
            uint4 va = *reinterpret_cast<const uint4*>(sx + (size_t)v * 16);
            float a[E];
            if constexpr (ADD) {
                float b[E];
                Vec<T>::unpack(va, a);
                Vec<T>::unpack(*reinterpret_cast<const uint4*>(sx + slot + (size_t)v * 16), b);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    a[e] = a[e] + b[e];
                va = Vec<T>::pack(a);  // the residual rounded to T
                st_stream(residual_out + row * hidden + (int64_t)v * E, va);
                *reinterpret_cast<uint4*>(sx + (size_t)v * 16) = va;  // kept for the second pass
            }
            Vec<T>::unpack(va, a);
#pragma unroll
            for (int e = 0; e < E; ++e)
                ss = fmaf(a[e], a[e], ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        if ((tid & 31) == 0)
            red[tid >> 5] = ss;
        __syncthreads();
        ss = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w)
            ss += red[w];
        const float r = rsqrtf(ss * inv_hidden + eps);

        for (int v = tid; v < nvec; v += THREADS) {
            float a[E], g[E];
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(sx + (size_t)v * 16), a);
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(s_gamma + (size_t)v * 16), g);
#pragma unroll
            for (int e = 0; e < E; ++e)
                a[e] = a[e] * r * g[e];
            st_stream(y + row * hidden + (int64_t)v * E, Vec<T>::pack(a));
        }
    }
}

constexpr int kRowsPerSmallCta = 2;  // GW == 1: two warps, one row each

// Sum of v over the threads that own one row: shuffles, then (GW > 1) one
// shared-memory step.  `red` holds two buffers used alternately; every call
// flips `parity`, so one barrier per reduction is enough however many
// reductions a row takes (RMSNorm one, LayerNorm two).
template <int GW>
__device__ __forceinline__ float group_sum(float v, float (*red)[GW], int& parity, int tid)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if constexpr (GW > 1) {
        if ((tid & 31) == 0)
            red[parity][tid >> 5] = v;
        __syncthreads();
        v = 0.f;
#pragma unroll
        for (int w = 0; w < GW; ++w)
            v += red[parity][w];
        parity ^= 1;
    }
    return v;
}

// Value of thread 0 of the row's group, given to every thread of the group:
// a shuffle for one warp per row, shared memory and a barrier for several.
template <int GW>
__device__ __forceinline__ float row_broadcast(float v, float& slot, int tid)
{
    if constexpr (GW == 1) {
        return __shfl_sync(0xFFFFFFFFu, v, 0);
    } else {
        __syncthreads();  // the previous row is done with the slot
        if (tid == 0)
            slot = v;
        __syncthreads();
        return slot;
    }
}

// The mean of a sum is taken as sum * inv_hidden, inv_hidden = fl(1/hidden)
// computed by the host: a division at that point would sit between the
// reduction and the output on every row's critical path.
//
// LN = false: RMSNorm, y = x * rsqrt(mean(x^2) + eps) * gamma.
// LN = true:  LayerNorm, y = (x - mean) * rsqrt(mean((x - mean)^2) + eps) * gamma + beta,
//             the variance taken from the row held in registers (two reductions),
//             both sums taken over the row shifted by its first element.
// PF: the grid is capped (a prefill-size launch), so each group walks several
// rows and prefetches its next one.  Decode-size launches (one row per group)
// leave the prefetch out altogether: even as a branch that is never taken it
// measured 1.36 against 1.17 us a launch in chains of dependent 5 x 2048 launches.
// add+LayerNorm at prefill sizes is held to 64 registers, 8 CTAs an SM: 4096 x
// 2048 bf16 measured 10.9 against 12.0 us a launch back to back on B200 at the
// 72 it takes unbounded (plain LayerNorm measured slightly slower bounded).
template <typename T, bool ADD, bool LN, int VPL, int GW, bool PF>
__global__ void __launch_bounds__(GW == 1 ? 32 * kRowsPerSmallCta : 32 * GW,
                                  (ADD && LN && PF && GW == 4) ? 8 : 1)
norm_rows_kernel(const T* x, const T* residual_in, T* residual_out, const T* __restrict__ gamma,
                 const T* __restrict__ beta, T* y, int64_t rows, int hidden, float eps,
                 float inv_hidden)
{
    constexpr int E = Vec<T>::N;
    constexpr int G = 32 * GW;  // threads per row
    constexpr int ROWS_PER_CTA = (GW == 1) ? kRowsPerSmallCta : 1;
    // evict-first stores at every size: write-back ones measured no faster for
    // 5 decode rows and slower for 256 (1.68 -> 1.77 us a launch in a chain)
    constexpr bool kStream = true;
    const int nvec = hidden / E;
    const int tid = threadIdx.x;
    const int gt = (GW == 1) ? (tid & 31) : tid;
    const int group = (GW == 1) ? (tid >> 5) : 0;
    __shared__ float red[2][GW];
    __shared__ float shift;

    // The weights a thread applies are the same for every row it handles, so
    // they are loaded once, into registers, before the dependency wait: with
    // programmatic dependent launch the caller guarantees that gamma and beta
    // are not written by the kernel launched just before this one (every
    // earlier kernel has completed by the time this one starts).  This
    // group's first row goes into L2 while the previous kernel drains.
    uint4 gv[VPL], bv[LN ? VPL : 1];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int vi = gt + i * G;
        if (vi < nvec) {
            gv[i] = __ldg(reinterpret_cast<const uint4*>(gamma + (size_t)vi * E));
            if constexpr (LN)
                bv[i] = __ldg(reinterpret_cast<const uint4*>(beta + (size_t)vi * E));
        }
    }
    {
        const int64_t row0 = (int64_t)blockIdx.x * ROWS_PER_CTA + group;
        const uint32_t row_bytes = (uint32_t)hidden * sizeof(T);
        if (gt == 0 && row0 < rows) {
            prefetch_l2(x + (size_t)row0 * hidden, row_bytes);
            if constexpr (ADD)
                prefetch_l2(residual_in + (size_t)row0 * hidden, row_bytes);
        }
    }
    pdl_wait();
    pdl_allow_dependents();

    int parity = 0;
    const int64_t row_stride = (int64_t)gridDim.x * ROWS_PER_CTA;
    for (int64_t row = (int64_t)blockIdx.x * ROWS_PER_CTA + group; row < rows;
         row += row_stride) {
        const size_t base = (size_t)row * (size_t)hidden;
        // the group's next row into L2 while this one is worked on
        if (PF && gt == 0 && row + row_stride < rows) {
            const uint32_t row_bytes = (uint32_t)hidden * sizeof(T);
            prefetch_l2(x + base + (size_t)row_stride * hidden, row_bytes);
            if constexpr (ADD)
                prefetch_l2(residual_in + base + (size_t)row_stride * hidden, row_bytes);
        }
        uint4 v[VPL];
        float s1 = 0.f;  // sum of x^2 (RMSNorm) or of x (LayerNorm)
        if constexpr (ADD) {
            uint4 r[VPL];
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int vi = gt + i * G;
                if (vi < nvec) {
                    v[i] = ld_stream(x + base + (size_t)vi * E);
                    r[i] = ld_stream(residual_in + base + (size_t)vi * E);
                }
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int vi = gt + i * G;
                if (vi < nvec) {
                    float a[E], b[E];
                    Vec<T>::unpack(v[i], a);
                    Vec<T>::unpack(r[i], b);
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = a[e] + b[e];
                    v[i] = Vec<T>::pack(a);  // the residual, rounded to T
                    st_out<kStream>(residual_out + base + (size_t)vi * E, v[i]);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int vi = gt + i * G;
                if (vi < nvec)
                    v[i] = ld_stream(x + base + (size_t)vi * E);
            }
        }
        // LayerNorm sums the row shifted by its first element c: the mean's
        // rounding error then scales with the row's spread, not with its offset
        float c = 0.f;
        if constexpr (LN) {
            float a0[E];
            Vec<T>::unpack(v[0], a0);  // thread 0 of the group holds element 0
            c = row_broadcast<GW>(a0[0], shift, tid);
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int vi = gt + i * G;
            if (vi < nvec) {
                float a[E];
                Vec<T>::unpack(v[i], a);  // for add+norm: exactly what was written
#pragma unroll
                for (int e = 0; e < E; ++e)
                    s1 = LN ? s1 + (a[e] - c) : fmaf(a[e], a[e], s1);
            }
        }
        s1 = group_sum<GW>(s1, red, parity, tid);

        float mean = 0.f, r;  // for LayerNorm: the mean of the shifted row
        if constexpr (LN) {
            mean = s1 * inv_hidden;
            float s2 = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int vi = gt + i * G;
                if (vi < nvec) {
                    float a[E];
                    Vec<T>::unpack(v[i], a);
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const float d = (a[e] - c) - mean;
                        s2 = fmaf(d, d, s2);
                    }
                }
            }
            s2 = group_sum<GW>(s2, red, parity, tid);
            r = rsqrtf(s2 * inv_hidden + eps);
        } else {
            r = rsqrtf(s1 * inv_hidden + eps);
        }

#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int vi = gt + i * G;
            if (vi < nvec) {
                float a[E], g[E];
                Vec<T>::unpack(v[i], a);
                Vec<T>::unpack(gv[i], g);
                if constexpr (LN) {
                    float b[E];
                    Vec<T>::unpack(bv[i], b);
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = ((a[e] - c) - mean) * r * g[e] + b[e];
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = a[e] * r * g[e];
                }
                st_out<kStream>(y + base + (size_t)vi * E, Vec<T>::pack(a));
            }
        }
    }
}

// One CTA per row, passes over the row: RMSNorm two (sum of squares, output),
// LayerNorm three (sum, squared deviations, output); later passes are served
// from L2.  VEC: 16-byte vectors (aligned, hidden % E == 0); otherwise one
// element at a time.  Each thread touches the same elements in every pass, so
// later passes read back its own pass-1 writes of residual_out.
constexpr int kLoopThreads = 256;

template <typename T, bool ADD, bool LN, bool VEC>
__global__ void __launch_bounds__(kLoopThreads)
norm_looped_kernel(const T* x, const T* residual_in, T* residual_out, const T* __restrict__ gamma,
                   const T* __restrict__ beta, T* y, int64_t rows, int64_t hidden, float eps,
                   float inv_hidden)
{
    constexpr int E = Vec<T>::N;
    constexpr int W = kLoopThreads / 32;
    const int tid = threadIdx.x;
    __shared__ float red[2][W];

    pdl_wait();
    pdl_allow_dependents();

    __shared__ float shift;
    int parity = 0;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const size_t base = (size_t)row * (size_t)hidden;
        float s1 = 0.f;
        // LayerNorm: the row's first element (after the residual add), shifted
        // out of both sums as in the register kernel
        float c = 0.f;
        if constexpr (LN) {
            __syncthreads();  // the previous row is done with `shift`
            if (tid == 0) {
                float a0 = load_elem(x + base);
                if constexpr (ADD)
                    a0 = round_to(a0 + load_elem(residual_in + base), residual_out);
                shift = a0;
            }
            __syncthreads();
            c = shift;
        }
        if constexpr (VEC) {
            const int64_t nvec = hidden / E;
            for (int64_t vi = tid; vi < nvec; vi += kLoopThreads) {
                float a[E];
                uint4 va = ld_stream(x + base + vi * E);
                if constexpr (ADD) {
                    float b[E];
                    Vec<T>::unpack(va, a);
                    Vec<T>::unpack(ld_stream(residual_in + base + vi * E), b);
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = a[e] + b[e];
                    va = Vec<T>::pack(a);
                    st_stream(residual_out + base + vi * E, va);
                }
                Vec<T>::unpack(va, a);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    s1 = LN ? s1 + (a[e] - c) : fmaf(a[e], a[e], s1);
            }
        } else {
            for (int64_t i = tid; i < hidden; i += kLoopThreads) {
                float a = load_elem(x + base + i);
                if constexpr (ADD) {
                    a = round_to(a + load_elem(residual_in + base + i), residual_out);
                    store_elem(residual_out + base + i, a);
                }
                s1 = LN ? s1 + (a - c) : fmaf(a, a, s1);
            }
        }
        s1 = group_sum<W>(s1, red, parity, tid);

        const T* src = ADD ? residual_out : x;
        float mean = 0.f, r;
        if constexpr (LN) {
            mean = s1 * inv_hidden;
            float s2 = 0.f;
            if constexpr (VEC) {
                const int64_t nvec = hidden / E;
                for (int64_t vi = tid; vi < nvec; vi += kLoopThreads) {
                    float a[E];
                    Vec<T>::unpack(ld_stream(src + base + vi * E), a);
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const float d = (a[e] - c) - mean;
                        s2 = fmaf(d, d, s2);
                    }
                }
            } else {
                for (int64_t i = tid; i < hidden; i += kLoopThreads) {
                    const float d = (load_elem(src + base + i) - c) - mean;
                    s2 = fmaf(d, d, s2);
                }
            }
            s2 = group_sum<W>(s2, red, parity, tid);
            r = rsqrtf(s2 * inv_hidden + eps);
        } else {
            r = rsqrtf(s1 * inv_hidden + eps);
        }

        if constexpr (VEC) {
            const int64_t nvec = hidden / E;
            for (int64_t vi = tid; vi < nvec; vi += kLoopThreads) {
                float a[E], g[E];
                Vec<T>::unpack(ld_stream(src + base + vi * E), a);
                Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(gamma + vi * E)), g);
                if constexpr (LN) {
                    float b[E];
                    Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(beta + vi * E)), b);
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = ((a[e] - c) - mean) * r * g[e] + b[e];
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        a[e] = a[e] * r * g[e];
                }
                st_stream(y + base + vi * E, Vec<T>::pack(a));
            }
        } else {
            for (int64_t i = tid; i < hidden; i += kLoopThreads) {
                const float a = load_elem(src + base + i);
                if constexpr (LN)
                    store_elem(y + base + i,
                               ((a - c) - mean) * r * load_elem(gamma + i) + load_elem(beta + i));
                else
                    store_elem(y + base + i, a * r * load_elem(gamma + i));
            }
        }
    }
}

// Chooses block size and ring depth for the streaming kernel; returns
// cudaErrorNotSupported when two ring slots and gamma do not fit in one CTA's
// shared memory (very long rows), so that the register kernels take over.
template <typename T, bool ADD, int THREADS>
cudaError_t launch_norm_tma_t(const T* x, const T* ri, T* ro, const T* g, T* y, int64_t rows,
                              int hidden, float eps, cudaStream_t st, const DeviceInfo& di)
{
    constexpr int NT = ADD ? 2 : 1;
    const uint32_t slot = round_up((uint32_t)hidden * sizeof(T), 128);
    const uint32_t fixed = slot + 8 * 9 + 128;  // gamma, barriers, slack
    int stages = 4;
    while (stages > 2 && fixed + (uint32_t)stages * NT * slot > kMaxSmemPerCta)
        --stages;
    const uint32_t smem = fixed + (uint32_t)stages * NT * slot;
    if (smem > kMaxSmemPerCta)
        return cudaErrorNotSupported;
    auto kernel = norm_tma_kernel<T, ADD, THREADS>;
    int per_sm = 0;
    cudaError_t err = resident_ctas(kernel, THREADS, smem, &per_sm);
    if (err != cudaSuccess)
        return err;
    if (per_sm < 1)
        return cudaErrorNotSupported;
    unsigned* word = nullptr;
    err = device_error_word(&word);
    if (err != cudaSuccess)
        return err;
    const int64_t grid = std::min<int64_t>(rows, (int64_t)di.sm_count * per_sm);
    return launch(kernel, dim3((unsigned)grid), dim3(THREADS), smem, st, x, ri, ro, g, y, rows,
                  hidden, eps, 1.0f / (float)hidden, stages, word);
}

template <typename T, bool ADD>
cudaError_t launch_norm_tma(const T* x, const T* ri, T* ro, const T* g, T* y, int64_t rows,
                            int hidden, float eps, cudaStream_t st, const DeviceInfo& di)
{
    const int nvec = hidden / Vec<T>::N;
    if (nvec <= 64)
        return launch_norm_tma_t<T, ADD, 64>(x, ri, ro, g, y, rows, hidden, eps, st, di);
    if (nvec <= 128)
        return launch_norm_tma_t<T, ADD, 128>(x, ri, ro, g, y, rows, hidden, eps, st, di);
    return launch_norm_tma_t<T, ADD, 256>(x, ri, ro, g, y, rows, hidden, eps, st, di);
}

// Grids of the register kernels.  A decode-size launch (cap = SMs x 32, above
// its row count) has one row per group.  A larger one is capped at two waves of
// resident CTAs (kPrefillWaves): each group then walks a few rows, prefetching
// its next row into L2 while it works on the current one, which measured 10.6
// against 11.2 us for 4096 x 2048 add+RMSNorm back to back on B200 (one row per
// CTA, 4096 CTAs).
constexpr int kPrefillWaves = 2;

// VPL vectors per lane, GW warps per row (GW == 1: two one-warp groups per CTA).
template <typename T, bool ADD, bool LN, int VPL, int GW, bool PF>
cudaError_t launch_rows_t(const T* x, const T* ri, T* ro, const T* g, const T* b, T* y,
                          int64_t rows, int hidden, float eps, cudaStream_t st, int64_t cap,
                          int sm_count)
{
    constexpr int RPC = (GW == 1) ? kRowsPerSmallCta : 1;
    constexpr int THREADS = (GW == 1) ? 32 * kRowsPerSmallCta : 32 * GW;
    if constexpr (PF)
        cap = std::min<int64_t>(cap, wave_ctas<norm_rows_kernel<T, ADD, LN, VPL, GW, PF>>(
                                         THREADS, sm_count, kPrefillWaves));
    const int64_t grid = std::min<int64_t>(ceil_div(rows, RPC), cap);
    return launch(norm_rows_kernel<T, ADD, LN, VPL, GW, PF>, dim3((unsigned)grid), dim3(THREADS),
                  0, st, x, ri, ro, g, b, y, rows, hidden, eps, 1.0f / (float)hidden);
}

template <typename T, bool ADD, bool LN, int VPL, int GW>
cudaError_t launch_rows(const T* x, const T* ri, T* ro, const T* g, const T* b, T* y,
                        int64_t rows, int hidden, float eps, cudaStream_t st, int64_t cap,
                        int sm_count, bool prefill)
{
    if (prefill)
        return launch_rows_t<T, ADD, LN, VPL, GW, true>(x, ri, ro, g, b, y, rows, hidden, eps, st,
                                                        cap, sm_count);
    return launch_rows_t<T, ADD, LN, VPL, GW, false>(x, ri, ro, g, b, y, rows, hidden, eps, st,
                                                     cap, sm_count);
}

template <typename T, bool ADD, bool LN>
cudaError_t launch_norm_t(const void* xv, const void* riv, void* rov, const void* gv,
                          const void* bv, void* yv, int64_t rows, int64_t hidden, float eps,
                          cudaStream_t st)
{
    const T* x = static_cast<const T*>(xv);
    const T* ri = static_cast<const T*>(riv);
    T* ro = static_cast<T*>(rov);
    const T* g = static_cast<const T*>(gv);
    const T* b = static_cast<const T*>(bv);
    T* y = static_cast<T*>(yv);
    constexpr int E = Vec<T>::N;

    DeviceInfo di;
    cudaError_t err = current_device_info(&di);
    if (err != cudaSuccess)
        return err;
    const int64_t cap = (int64_t)di.sm_count * 32;
    const int sms = di.sm_count;

    const bool vec = (hidden % E == 0) && aligned16(x) && aligned16(g) && aligned16(y) &&
                     (!ADD || (aligned16(ri) && aligned16(ro))) && (!LN || aligned16(b));
    if constexpr (!LN) {
        if (vec && streaming_enabled()) {
            err = launch_norm_tma<T, ADD>(x, ri, ro, g, y, rows, (int)hidden, eps, st, di);
            if (err != cudaErrorNotSupported)
                return err;
        }
    }
    if (vec) {
        const int64_t nvec = hidden / E;
        const int h = (int)hidden;
        // A problem that fits one wave at one vector per thread (a decode step's
        // few rows) is latency-bound: after the dependency wait each warp then
        // has one load, a few flops and one store per tensor, and the row's
        // reduction runs across warps, instead of one warp walking the whole row.
        // Once every SM has a row of its own (256 decode rows), two vectors per
        // lane over half as many warps measured faster in chains of dependent
        // launches on B200 (1.78 against 1.85 us a launch for 256 x 2048), and
        // slower below that (1.43 against 1.36 us for 5 x 2048).
        if (rows * nvec <= (int64_t)di.sm_count * 2048 && rows >= di.sm_count && nvec > 64 &&
            nvec <= 1024) {
            if (nvec <= 128)
                return launch_rows<T, ADD, LN, 2, 2>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            if (nvec <= 256)
                return launch_rows<T, ADD, LN, 2, 4>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            if (nvec <= 512)
                return launch_rows<T, ADD, LN, 2, 8>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            return launch_rows<T, ADD, LN, 2, 16>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
        }
        if (rows * nvec <= (int64_t)di.sm_count * 2048 && nvec > 32) {
            if (nvec <= 64)
                return launch_rows<T, ADD, LN, 1, 2>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            if (nvec <= 128)
                return launch_rows<T, ADD, LN, 1, 4>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            if (nvec <= 256)
                return launch_rows<T, ADD, LN, 1, 8>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
            if (nvec <= 512)
                return launch_rows<T, ADD, LN, 1, 16>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, false);
        }
        const bool pre = rows * nvec > (int64_t)di.sm_count * 2048;  // beyond one wave
        if (nvec <= 32)
            return launch_rows<T, ADD, LN, 1, 1>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 64)
            return launch_rows<T, ADD, LN, 2, 1>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 128)
            return launch_rows<T, ADD, LN, 4, 1>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        // two vectors per lane over four warps (56 registers) rather than one
        // warp of 8 (160): 4096 x 2048 bf16 add+RMSNorm measured 10.6 against
        // 11.5 us a launch back to back on B200, with bit-identical residuals
        if (nvec <= 256)
            return launch_rows<T, ADD, LN, 2, 4>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 512)
            return launch_rows<T, ADD, LN, 8, 2>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 1024)
            return launch_rows<T, ADD, LN, 8, 4>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 2048)
            return launch_rows<T, ADD, LN, 8, 8>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
        if (nvec <= 4096)
            return launch_rows<T, ADD, LN, 8, 16>(x, ri, ro, g, b, y, rows, h, eps, st, cap, sms, pre);
    }
    const int64_t grid = std::min<int64_t>(rows, cap);
    if (vec)
        return launch(norm_looped_kernel<T, ADD, LN, true>, dim3((unsigned)grid),
                      dim3(kLoopThreads), 0, st, x, ri, ro, g, b, y, rows, hidden, eps,
                      1.0f / (float)hidden);
    return launch(norm_looped_kernel<T, ADD, LN, false>, dim3((unsigned)grid), dim3(kLoopThreads),
                  0, st, x, ri, ro, g, b, y, rows, hidden, eps, 1.0f / (float)hidden);
}

template <typename T>
cudaError_t launch_norm_dt(const void* x, const void* ri, void* ro, const void* g, const void* b,
                           void* y, int64_t rows, int64_t hidden, float eps, cudaStream_t st)
{
    const bool add = ri != nullptr;
    const bool ln = b != nullptr;
    if (add && ln)
        return launch_norm_t<T, true, true>(x, ri, ro, g, b, y, rows, hidden, eps, st);
    if (add)
        return launch_norm_t<T, true, false>(x, ri, ro, g, nullptr, y, rows, hidden, eps, st);
    if (ln)
        return launch_norm_t<T, false, true>(x, nullptr, nullptr, g, b, y, rows, hidden, eps, st);
    return launch_norm_t<T, false, false>(x, nullptr, nullptr, g, nullptr, y, rows, hidden, eps,
                                          st);
}

}  // namespace

cudaError_t launch_norm(const void* x, const void* residual_in, void* residual_out,
                        const void* gamma, const void* beta, void* y, int64_t rows,
                        int64_t hidden, float eps, arops_dtype dtype, cudaStream_t stream)
{
    if (dtype == AROPS_BF16)
        return launch_norm_dt<__nv_bfloat16>(x, residual_in, residual_out, gamma, beta, y, rows,
                                             hidden, eps, stream);
    return launch_norm_dt<float>(x, residual_in, residual_out, gamma, beta, y, rows, hidden, eps,
                                 stream);
}

}  // namespace arops
