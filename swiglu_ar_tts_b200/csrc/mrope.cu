// Multi-section rotary embedding (M-RoPE) on q and k (sm_100a).
//
// "M-RoPE" is one of the four fused operators of the Triton kernel-fusion post
// for Qwen3-TTS (section 3); RoPE itself is a rotation of Q and K in the
// complex plane (forpes.ru post 233929, "Stage 2").  For pair index j of a head
// (rotate-half pairing: x[j] with x[j + D/2]) the angle is p * theta^(-2j/D),
// where the position p comes from row t, h or w of the int32 position ids
// according to the contiguous section that j falls in.
//
// Design: one warp per token.  cos/sin depend only on (token, j), not on the
// head, so a warp evaluates each of the token's D/2 angles once, spread over
// the lanes, and shares them with shuffles; no cos/sin table is streamed.  Lane
// `pv` of a head owns the 16-byte vector x[pv*E .. pv*E+E) of the first half
// and its partner vector of the second half; G = 32/P heads are covered per
// warp pass and up to U passes are loaded before any math, so each lane keeps
// 2*U 16-byte loads in flight.  The angle is formed in fp64 and reduced modulo
// 2*pi (|k * 2pi rounding| <= 1e-13 rad for the positions used here) before the
// fp32 sincosf, so cos/sin carry ~1e-7 absolute error at any position.
#include <math.h>

#include "common.cuh"

namespace arops {
namespace {

constexpr int kMaxHalf = 256;  // head_dim <= 512

struct MropeParams {
    int32_t sec0;   // pairs j < sec0 take row 0 (t)
    int32_t sec01;  // pairs sec0 <= j < sec01 take row 1 (h); the rest row 2 (w)
    double inv_freq[kMaxHalf];  // theta^(-2j/head_dim), j < head_dim/2
};

constexpr double kTwoPi = 6.283185307179586;
constexpr double kInvTwoPi = 0.15915494309189535;

__device__ __forceinline__ void rope_cos_sin(double inv_freq, int32_t p, float* c, float* s)
{
    const double phi = (double)p * inv_freq;
    const double k = rint(phi * kInvTwoPi);
    const double r = fma(-k, kTwoPi, phi);
    sincosf((float)r, s, c);
}

__device__ __forceinline__ int32_t position_of(int j, const MropeParams& prm, int32_t pt,
                                               int32_t ph, int32_t pw)
{
    return (j < prm.sec0) ? pt : ((j < prm.sec01) ? ph : pw);
}

constexpr int kWarpsPerCta = 4;

template <typename T, int P, int U>
__global__ void __launch_bounds__(32 * kWarpsPerCta)
mrope_vec_kernel(const T* q, const T* k, T* q_out, T* k_out, const int32_t* __restrict__ pos,
                 int64_t tokens, int hq, int hk, const __grid_constant__ MropeParams prm)
{
    constexpr int E = Vec<T>::N;
    constexpr int G = 32 / P;                // heads per warp pass
    constexpr int HALF = P * E;              // head_dim / 2
    constexpr int D = 2 * HALF;
    constexpr int F = (E >= G) ? E / G : 1;  // angles evaluated per lane
    const int lane = threadIdx.x & 31;
    const int pv = lane % P;
    const int hg = lane / P;
    const int j0 = pv * E;
    const int nh = hq + hk;

    pdl_wait();
    pdl_allow_dependents();

    for (int64_t t = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); t < tokens;
         t += (int64_t)gridDim.x * kWarpsPerCta) {
        const int32_t pt = __ldg(pos + t);
        const int32_t ph = __ldg(pos + tokens + t);
        const int32_t pw = __ldg(pos + 2 * tokens + t);

        // this lane's share of the E angles of block pv ...
        float cs[F], sn[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const int j = j0 + ((hg * F + f) % E);
            rope_cos_sin(prm.inv_freq[j], position_of(j, prm, pt, ph, pw), &cs[f], &sn[f]);
        }
        // ... gathered from the lanes that evaluated them
        float c[E], s[E];
#pragma unroll
        for (int m = 0; m < E; ++m) {
            const int src = pv + P * ((m / F) % G);
            c[m] = __shfl_sync(0xFFFFFFFFu, cs[m % F], src);
            s[m] = __shfl_sync(0xFFFFFFFFu, sn[m % F], src);
        }

        for (int h0 = hg; h0 < nh; h0 += G * U) {
            uint4 lo[U], hi[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = h0 + u * G;
                if (h < nh) {
                    const T* src = (h < hq) ? q + ((size_t)t * hq + h) * D
                                            : k + ((size_t)t * hk + (h - hq)) * D;
                    lo[u] = ld_stream(src + j0);
                    hi[u] = ld_stream(src + HALF + j0);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = h0 + u * G;
                if (h < nh) {
                    float a[E], b[E], oa[E], ob[E];
                    Vec<T>::unpack(lo[u], a);
                    Vec<T>::unpack(hi[u], b);
#pragma unroll
                    for (int m = 0; m < E; ++m) {
                        oa[m] = a[m] * c[m] - b[m] * s[m];
                        ob[m] = b[m] * c[m] + a[m] * s[m];
                    }
                    T* dst = (h < hq) ? q_out + ((size_t)t * hq + h) * D
                                      : k_out + ((size_t)t * hk + (h - hq)) * D;
                    st_stream(dst + j0, Vec<T>::pack(oa));
                    st_stream(dst + HALF + j0, Vec<T>::pack(ob));
                }
            }
        }
    }
}

// Any even head_dim, any alignment: one thread per (token, head, pair).
template <typename T>
__global__ void __launch_bounds__(256)
mrope_scalar_kernel(const T* q, const T* k, T* q_out, T* k_out, const int32_t* __restrict__ pos,
                    int64_t tokens, int hq, int hk, int half,
                    const __grid_constant__ MropeParams prm)
{
    pdl_wait();
    pdl_allow_dependents();
    const int nh = hq + hk;
    const int64_t total = tokens * nh * half;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(idx % half);
        const int h = (int)((idx / half) % nh);
        const int64_t t = idx / ((int64_t)half * nh);
        const int32_t p = position_of(j, prm, __ldg(pos + t), __ldg(pos + tokens + t),
                                      __ldg(pos + 2 * tokens + t));
        float c, s;
        rope_cos_sin(prm.inv_freq[j], p, &c, &s);
        const size_t off = (h < hq) ? ((size_t)t * hq + h) * 2 * half
                                    : ((size_t)t * hk + (h - hq)) * 2 * half;
        const T* src = (h < hq) ? q : k;
        T* dst = (h < hq) ? q_out : k_out;
        const float a = load_elem(src + off + j);
        const float b = load_elem(src + off + half + j);
        store_elem(dst + off + j, a * c - b * s);
        store_elem(dst + off + half + j, b * c + a * s);
    }
}

constexpr int kHeadUnroll = 8;

template <typename T, int P>
cudaError_t launch_vec(const MropeArgs& a, const MropeParams& prm, cudaStream_t st, int64_t cap)
{
    const int64_t grid = std::min<int64_t>(ceil_div(a.tokens, kWarpsPerCta), cap);
    return launch(mrope_vec_kernel<T, P, kHeadUnroll>, dim3((unsigned)grid),
                  dim3(32 * kWarpsPerCta), 0, st, static_cast<const T*>(a.q),
                  static_cast<const T*>(a.k), static_cast<T*>(a.q_out), static_cast<T*>(a.k_out),
                  a.pos, a.tokens, (int)a.n_q_heads, (int)a.n_k_heads, prm);
}

template <typename T>
cudaError_t launch_mrope_t(const MropeArgs& a, const MropeParams& prm, cudaStream_t st)
{
    DeviceInfo di;
    cudaError_t err = current_device_info(&di);
    if (err != cudaSuccess)
        return err;
    constexpr int E = Vec<T>::N;
    const int half = a.head_dim / 2;
    const bool aligned = aligned16(a.q) && aligned16(a.q_out) &&
                         (a.n_k_heads == 0 || (aligned16(a.k) && aligned16(a.k_out)));
    const int64_t cap = (int64_t)di.sm_count * 64;
    if (aligned && half % E == 0) {
        switch (half / E) {
        case 1: return launch_vec<T, 1>(a, prm, st, cap);
        case 2: return launch_vec<T, 2>(a, prm, st, cap);
        case 4: return launch_vec<T, 4>(a, prm, st, cap);
        case 8: return launch_vec<T, 8>(a, prm, st, cap);
        case 16: return launch_vec<T, 16>(a, prm, st, cap);
        case 32: return launch_vec<T, 32>(a, prm, st, cap);
        default: break;
        }
    }
    const int64_t total = a.tokens * (int64_t)(a.n_q_heads + a.n_k_heads) * half;
    const int64_t grid = std::min<int64_t>(ceil_div(total, 256), (int64_t)di.sm_count * 16);
    return launch(mrope_scalar_kernel<T>, dim3((unsigned)grid), dim3(256), 0, st,
                  static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                  static_cast<T*>(a.q_out), static_cast<T*>(a.k_out), a.pos, a.tokens,
                  (int)a.n_q_heads, (int)a.n_k_heads, half, prm);
}

}  // namespace

cudaError_t launch_mrope(const MropeArgs& a, arops_dtype dtype, cudaStream_t stream)
{
    MropeParams prm;
    const int half = a.head_dim / 2;
    prm.sec0 = a.sections[0];
    prm.sec01 = a.sections[0] + a.sections[1];
    // textbook RoPE inverse frequencies, formed in fp64 on the host
    for (int j = 0; j < kMaxHalf; ++j)
        prm.inv_freq[j] = (j < half) ? pow((double)a.theta, -2.0 * (double)j / (double)a.head_dim)
                                     : 0.0;
    if (dtype == AROPS_BF16)
        return launch_mrope_t<__nv_bfloat16>(a, prm, stream);
    return launch_mrope_t<float>(a, prm, stream);
}

}  // namespace arops
