// SwiGLU: out = silu(gate) * up with silu(g) = g / (1 + e^-g), fp32 math
// ("SwiGLU" in section 3 of the Triton kernel-fusion post for Qwen3-TTS).
//
// Pure streaming work (two reads, one write per element, ~1 flop per byte), so
// the kernel is shaped for HBM: 16-byte coalesced accesses, U independent
// vectors of each input in flight per thread before any math, evict-first
// cache hints, and a grid-stride loop over a grid sized to the SM count.  The
// ragged tail (n % 8 elements) is handled by block 0 in the same launch.
#include "common.cuh"

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
__device__ __forceinline__ float silu(float g)
{
    if (g < -80.0f)
        return -expf(g + logf(-g));
    if constexpr (sizeof(T) == 2)
        return __fdividef(g, 1.0f + __expf(-g));
    else
        return g / (1.0f + expf(-g));
}

template <typename T, int U>
__global__ void __launch_bounds__(kThreads)
swiglu_vec_kernel(const T* gate, const T* up, T* out, int64_t n)
{
    constexpr int E = Vec<T>::N;
    const int64_t nvec = n / E;
    const int64_t chunk = (int64_t)kThreads * U;

    pdl_wait();
    pdl_allow_dependents();

    for (int64_t base = (int64_t)blockIdx.x * chunk + threadIdx.x; base < nvec;
         base += (int64_t)gridDim.x * chunk) {
        uint4 g[U], u[U];
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int64_t vi = base + (int64_t)i * kThreads;
            if (vi < nvec) {
                g[i] = ld_stream(gate + vi * E);
                u[i] = ld_stream(up + vi * E);
            }
        }
#pragma unroll
        for (int i = 0; i < U; ++i) {
            const int64_t vi = base + (int64_t)i * kThreads;
            if (vi < nvec) {
                float a[E], b[E];
                Vec<T>::unpack(g[i], a);
                Vec<T>::unpack(u[i], b);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    a[e] = silu<T>(a[e]) * b[e];
                st_stream(out + vi * E, Vec<T>::pack(a));
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

constexpr int kUnroll = 4;

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
    // 8 resident CTAs of 256 threads fill an SM's 2048 thread slots
    const int64_t resident = (int64_t)di.sm_count * 8;
    if (aligned16(g) && aligned16(u) && aligned16(o)) {
        const int64_t nvec = n / E;
        const int64_t want = std::max<int64_t>(1, ceil_div(nvec, (int64_t)kThreads * kUnroll));
        const int64_t grid = std::min<int64_t>(want, resident);
        return launch(swiglu_vec_kernel<T, kUnroll>, dim3((unsigned)grid), dim3(kThreads), 0, st,
                      g, u, o, n);
    }
    const int64_t grid = std::min<int64_t>(ceil_div(n, kThreads), resident);
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
