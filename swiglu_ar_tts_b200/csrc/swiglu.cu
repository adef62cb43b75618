// SwiGLU: out = silu(gate) * up with silu(g) = g / (1 + e^-g), fp32 math
// ("SwiGLU" in section 3 of the Triton kernel-fusion post for Qwen3-TTS).
//
// Pure streaming work (two reads, one write per element, ~1 flop per byte), so
// the kernel is shaped for HBM: 16-byte coalesced accesses, U independent
// vectors of each input in flight per thread before any math, evict-first
// cache hints, one chunk of U vectors per thread per CTA on a grid the
// hardware schedules as SMs free up.  Decode-size problems (at most one vector
// per resident thread) take one vector per thread in CTAs of 128 or 512
// threads, with plain stores.  The ragged tail (n % 8 elements) is handled by
// block 0 in the same launch.  A streaming kernel that stages chunks through
// shared memory with bulk copies is opt-in (arops_set_streaming) and measured
// slower on B200.
#include "common.cuh"
#include "tma.cuh"

namespace arops {
namespace {

constexpr int kThreads = 256;

// silu(g) = g / (1 + e^-g).  For g < -80 the quotient form would need a
// denominator beyond 2^126, where the fast divide returns 0 although the true
// result can still be a normal number.  There silu(g) = g e^g / (1 + e^g)
// = g e^g to fp32 precision (e^g < 2e-35 vanishes next to 1), and it is taken as
// -exp(g + ln(-g)) so that the one rounding happens in the final result, not in
// a subnormal e^g.
// bf16 storage uses the fast exponential and divide (relative error ~1e-6, far
// below half a bf16 ulp); fp32 storage uses expf and an IEEE divide so that its
// error stays well inside the 1e-5 relative bound.
template <typename T>
__device__ __forceinline__ float silu_quotient(float g)
{
    if constexpr (sizeof(T) == 2)
        return __fdividef(g, 1.0f + __expf(-g));
    else
        return g / (1.0f + expf(-g));
}

template <typename T>
__device__ __forceinline__ float silu(float g)
{
    if (g < -80.0f)
        return -expf(g + logf(-g));
    return silu_quotient<T>(g);
}

// out = silu(gate) * up over one vector.  The g < -80 form is taken only by a
// vector that holds such a g: evaluated element by element, its exp and log
// would otherwise be paid for every element.
template <typename T, int E>
__device__ __forceinline__ void silu_mul(float (&a)[E], const float (&b)[E])
{
    float lo = a[0];
#pragma unroll
    for (int e = 1; e < E; ++e)
        lo = fminf(lo, a[e]);
    if (lo < -80.0f) {
#pragma unroll
        for (int e = 0; e < E; ++e)
            a[e] = silu<T>(a[e]) * b[e];
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e)
            a[e] = silu_quotient<T>(a[e]) * b[e];
    }
}

// U = 1 only for decode-size launches, whose output takes a plain store.
template <typename T, int U, int THREADS>
__global__ void __launch_bounds__(THREADS)
swiglu_vec_kernel(const T* gate, const T* up, T* out, int64_t n)
{
    constexpr int E = Vec<T>::N;
    const int64_t nvec = n / E;
    const int64_t chunk = (int64_t)THREADS * U;

    // the CTA's first chunk of gate and up into L2 while the previous kernel drains
    if (threadIdx.x == 0) {
        const int64_t v0 = (int64_t)blockIdx.x * chunk;
        if (v0 < nvec) {
            const int64_t nv = (nvec - v0 < chunk) ? nvec - v0 : chunk;
            prefetch_l2(gate + v0 * E, (uint32_t)(nv * 16));
            prefetch_l2(up + v0 * E, (uint32_t)(nv * 16));
        }
    }
    pdl_wait();
    pdl_allow_dependents();

    for (int64_t base = (int64_t)blockIdx.x * chunk + threadIdx.x; base < nvec;
         base += (int64_t)gridDim.x * chunk) {
        uint4 g[U], u[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int64_t vi = base + (int64_t)i * THREADS;
            if (vi < nvec) {
                g[i] = ld_stream(gate + vi * E);
                u[i] = ld_stream(up + vi * E);
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int64_t vi = base + (int64_t)i * THREADS;
            if (vi < nvec) {
                float a[E], b[E];
                Vec<T>::unpack(g[i], a);
                Vec<T>::unpack(u[i], b);
                silu_mul<T>(a, b);
                st_out<(U > 1)>(out + vi * E, Vec<T>::pack(a));
            }
        }
    }
    // ragged tail: fewer than E elements after the last full vector
    if (blockIdx.x == 0) {
        const int64_t i = nvec * E + threadIdx.x;
        if (i < n)
            store_elem(out + i, silu<T>(load_elem(gate + i)) * load_elem(up + i));
    }
}

// ---------------------------------------------------------------------------
// Streaming kernel (opt-in: arops_set_streaming(1), for 16-byte-aligned
// buffers with n % 8 == 0).  The
// flat array is cut into chunks of kChunk elements; warp gw of the grid owns
// chunks gw, gw + nw, ... and a ring of `slots` shared-memory slots, each
// holding one chunk of gate and of up.  Lane 0 keeps `slots` chunks in flight
// as bulk copies (TMA); the warp computes a chunk as soon as it lands and
// stores it with coalesced 16-byte stores.  No thread ever waits on another
// warp, and an SM keeps ~190 KB of reads outstanding at all times.
// ---------------------------------------------------------------------------
constexpr int kChunk = 2048;  // elements per chunk and tensor
constexpr int kTmaWarps = 4;

template <typename T>
__global__ void __launch_bounds__(32 * kTmaWarps)
swiglu_tma_kernel(const T* gate, const T* up, T* out, int64_t n, int slots, unsigned* err_word)
{
    constexpr int E = Vec<T>::N;
    constexpr uint32_t kBytes = kChunk * sizeof(T);
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    unsigned char* ring = smem + (size_t)warp * slots * 2 * kBytes;
    uint64_t* bars =
        reinterpret_cast<uint64_t*>(smem + (size_t)kTmaWarps * slots * 2 * kBytes) + warp * slots;
    const int64_t gw = (int64_t)blockIdx.x * kTmaWarps + warp;
    const int64_t nw = (int64_t)gridDim.x * kTmaWarps;
    const int64_t chunks = (n + kChunk - 1) / kChunk;
    const int64_t my = chunks > gw ? (chunks - 1 - gw) / nw + 1 : 0;

    if (lane == 0) {
        for (int i = 0; i < slots; ++i)
            mbar_init(smem_addr(&bars[i]), 1);
        mbar_init_fence();
    }
    __syncwarp();

    pdl_wait();
    pdl_allow_dependents();

    int64_t issued = 0;  // lane 0 only
    auto issue = [&](int64_t j) {
        const int64_t c = gw + j * nw;
        const int64_t base = c * kChunk;
        const int64_t left = n - base;
        const uint32_t bytes = (uint32_t)((left < kChunk ? left : kChunk) * sizeof(T));
        const int sidx = (int)(j % slots);
        const uint32_t bar = smem_addr(&bars[sidx]);
        unsigned char* dst = ring + (size_t)sidx * 2 * kBytes;
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_load(smem_addr(dst), gate + base, bytes, bar);
        bulk_load(smem_addr(dst + kBytes), up + base, bytes, bar);
    };
    if (lane == 0)
        for (; issued < slots && issued < my; ++issued)
            issue(issued);

    for (int64_t j = 0; j < my; ++j) {
        const int sidx = (int)(j % slots);
        const bool ok = mbar_wait(smem_addr(&bars[sidx]), (uint32_t)((j / slots) & 1));
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            if (lane == 0) {
                record_device_error(err_word, kDeviceErrTimeout);
                for (int64_t k = j; k < issued; ++k)
                    mbar_wait(smem_addr(&bars[k % slots]), (uint32_t)((k / slots) & 1));
            }
            return;
        }
        const int64_t base = (gw + j * nw) * kChunk;
        const int64_t left = n - base;
        const int nv = (int)((left < kChunk ? left : kChunk) / E);
        const unsigned char* sg = ring + (size_t)sidx * 2 * kBytes;
#pragma unroll 4
        for (int v = lane; v < nv; v += 32) {
            float a[E], b[E];
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(sg + (size_t)v * 16), a);
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(sg + kBytes + (size_t)v * 16), b);
            silu_mul<T>(a, b);
            st_stream(out + base + (int64_t)v * E, Vec<T>::pack(a));
        }
        __syncwarp();  // the slot has been read; it can take the next copy
        if (lane == 0 && issued < my) {
            issue(issued);
            ++issued;
        }
    }
}

// Unaligned buffers: one element per thread per iteration.
template <typename T>
__global__ void __launch_bounds__(kThreads)
swiglu_scalar_kernel(const T* gate, const T* up, T* out, int64_t n)
{
    pdl_wait();
    pdl_allow_dependents();
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * kThreads)
        store_elem(out + i, silu<T>(load_elem(gate + i)) * load_elem(up + i));
}

// Two 16-byte vectors of each input per thread and one chunk per CTA (a grid of
// n / 4096 CTAs that the hardware schedules as SMs free up) measured fastest on
// B200: 49.5 us for 8192 x 6144, against 53.5 us for 4 vectors on a persistent
// grid and 51-78 us for shared-memory rings fed by bulk copies.
constexpr int kUnroll = 2;

template <typename T>
cudaError_t launch_swiglu_t(const void* gv, const void* uv, void* ov, int64_t n, cudaStream_t st)
{
    const T* g = static_cast<const T*>(gv);
    const T* u = static_cast<const T*>(uv);
    T* o = static_cast<T*>(ov);
    DeviceInfo di;
    cudaError_t err = current_device_info(&di);
    if (err != cudaSuccess)
        return err;
    constexpr int E = Vec<T>::N;
    const bool aligned = aligned16(g) && aligned16(u) && aligned16(o);
    if (aligned && n % E == 0 && streaming_enabled()) {
        // 3 slots of 8 KB per warp: 96 KB per CTA, two CTAs per SM
        const int slots = 3;
        const uint32_t smem = kTmaWarps * slots * (2 * kChunk * sizeof(T) + 8) + 128;
        auto kernel = swiglu_tma_kernel<T>;
        int per_sm = 0;
        err = resident_ctas(kernel, 32 * kTmaWarps, smem, &per_sm);
        if (err != cudaSuccess)
            return err;
        unsigned* word = nullptr;
        err = device_error_word(&word);
        if (err != cudaSuccess)
            return err;
        const int64_t chunks = ceil_div(n, kChunk);
        const int64_t grid = std::min<int64_t>(ceil_div(chunks, kTmaWarps),
                                               (int64_t)di.sm_count * std::max(per_sm, 1));
        return launch(kernel, dim3((unsigned)grid), dim3(32 * kTmaWarps), smem, st, g, u, o, n,
                      slots, word);
    }
    if (aligned) {
        const int64_t nvec = n / E;
        // a problem that fits one wave at one vector per thread (decode batches)
        // is latency-bound: one vector per thread.  CTAs of 128 threads (a few
        // CTAs' worth of vectors per SM at most) or else 512 measured fastest
        // on B200 for 5 x 6144 and 256 x 6144 in chains of dependent launches.
        if (nvec <= (int64_t)di.sm_count * 2048) {
            if (nvec <= (int64_t)di.sm_count * 256) {
                const int64_t grid = std::max<int64_t>(1, ceil_div(nvec, 128));
                return launch(swiglu_vec_kernel<T, 1, 128>, dim3((unsigned)grid), dim3(128), 0,
                              st, g, u, o, n);
            }
            const int64_t grid = ceil_div(nvec, 512);
            return launch(swiglu_vec_kernel<T, 1, 512>, dim3((unsigned)grid), dim3(512), 0, st, g,
                          u, o, n);
        }
        const int64_t want = ceil_div(nvec, (int64_t)kThreads * kUnroll);
        const int64_t grid = std::min<int64_t>(want, (int64_t)INT32_MAX);
        return launch(swiglu_vec_kernel<T, kUnroll, kThreads>, dim3((unsigned)grid),
                      dim3(kThreads), 0, st, g, u, o, n);
    }
    const int64_t grid = std::min<int64_t>(ceil_div(n, kThreads), (int64_t)di.sm_count * 8);
    return launch(swiglu_scalar_kernel<T>, dim3((unsigned)grid), dim3(kThreads), 0, st, g, u, o, n);
}

}  // namespace

cudaError_t launch_swiglu(const void* gate, const void* up, void* out, int64_t n,
                          arops_dtype dtype, cudaStream_t stream)
{
    if (dtype == AROPS_BF16)
        return launch_swiglu_t<__nv_bfloat16>(gate, up, out, n, stream);
    return launch_swiglu_t<float>(gate, up, out, n, stream);
}

}  // namespace arops
