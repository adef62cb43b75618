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
// 2*U 16-byte loads in flight.  A token's passes may be shared by `splits`
// warps (warp s of the token takes passes s, s + splits, ...): few tokens, as
// in a decode step, then spread over many warps instead of queueing every pass
// of a token behind one warp.  The angle is formed in fp64 and reduced modulo
// 2*pi (|k * 2pi rounding| <= 1e-13 rad for the positions used here) before the
// fp32 sincosf, so cos/sin carry ~1e-7 absolute error at any position.
#include <math.h>

#include "common.cuh"
#include "tma.cuh"

namespace arops {
namespace {

struct MropeParams {
    int32_t sec0;       // pairs j < sec0 take row 0 (t)
    int32_t sec01;      // pairs sec0 <= j < sec01 take row 1 (h); the rest row 2 (w)
    double freq_scale;  // 2 log2(theta) / head_dim: inverse frequency j is 2^(-j * freq_scale)
};

// theta^(-2j/head_dim) = 2^(-j * 2 log2(theta) / head_dim), the textbook RoPE
// inverse frequency, in fp64.
__device__ __forceinline__ double inv_freq_of(int j, const MropeParams& prm)
{
    return exp2(-(double)j * prm.freq_scale);
}

// Each CTA tabulates the head's inverse frequencies in shared memory once; this
// touches no global memory, so it runs before the dependency wait.
__device__ __forceinline__ void fill_inv_freq(double* table, int half, const MropeParams& prm)
{
    for (int j = threadIdx.x; j < half; j += blockDim.x)
        table[j] = inv_freq_of(j, prm);
    __syncthreads();
}

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

// cos/sin of the angles a lane applies, for token t: the lanes of pair block
// pv split the block's E angles between them (F each) and share them with
// shuffles, so every lane of the warp must take part.
template <int E, int P>
__device__ __forceinline__ void token_angles(int32_t pt, int32_t ph, int32_t pw,
                                             const double* inv_freq, const MropeParams& prm,
                                             int lane, float* c, float* s)
{
    constexpr int G = 32 / P;                // heads per warp pass
    constexpr int F = (E >= G) ? E / G : 1;  // angles evaluated per lane
    const int pv = lane % P;
    const int hg = lane / P;
    const int j0 = pv * E;
    float cs[F], sn[F];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        const int j = j0 + ((hg * F + f) % E);
        rope_cos_sin(inv_freq[j], position_of(j, prm, pt, ph, pw), &cs[f], &sn[f]);
    }
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int src = pv + P * ((m / F) % G);
        c[m] = __shfl_sync(0xFFFFFFFFu, cs[m % F], src);
        s[m] = __shfl_sync(0xFFFFFFFFu, sn[m % F], src);
    }
}

constexpr int kWarpsPerCta = 4;

// Token of warp unit `unit` and which of the token's `splits` warps it is.
// splits > 1 only for launches whose unit count fits 32 bits (at most one head
// pass per resident warp, or a KV append of under 2^30 tokens), so the
// division stays a 32-bit one.
__device__ __forceinline__ int64_t unit_token(int64_t unit, int splits, int& part)
{
    if (splits == 1) {
        part = 0;
        return unit;
    }
    const uint32_t u = (uint32_t)unit;
    part = (int)(u % (uint32_t)splits);
    return (int64_t)(u / (uint32_t)splits);
}

template <typename T, int P, int U>
__global__ void __launch_bounds__(32 * kWarpsPerCta)
mrope_vec_kernel(const T* q, const T* k, T* q_out, T* k_out, const int32_t* __restrict__ pos,
                 int64_t tokens, int hq, int hk, int splits, const __grid_constant__ MropeParams prm)
{
    constexpr int E = Vec<T>::N;
    constexpr int G = 32 / P;                // heads per warp pass
    constexpr int HALF = P * E;              // head_dim / 2
    constexpr int D = 2 * HALF;
    // evict-first stores, except with one pass per warp (U == 1: decode-size launches)
    constexpr bool kStream = U > 1;
    const int lane = threadIdx.x & 31;
    const int pv = lane % P;
    const int hg = lane / P;
    const int j0 = pv * E;
    const int nh = hq + hk;
    __shared__ double inv_freq[HALF];

    // this warp's first token (q and k heads, positions) into L2 while the
    // previous kernel drains; of the warps that share a token, the first asks
    const int64_t units = tokens * splits;
    const int64_t unit0 = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    {
        int part0 = 0;
        const int64_t t0 = unit_token(unit0, splits, part0);
        if (lane == 0 && unit0 < units && part0 == 0) {
            if (hq > 0)
                prefetch_l2(q + (size_t)t0 * hq * D, (uint32_t)(hq * D * sizeof(T)));
            if (hk > 0)
                prefetch_l2(k + (size_t)t0 * hk * D, (uint32_t)(hk * D * sizeof(T)));
            prefetch_l2_line(pos + t0);
            prefetch_l2_line(pos + tokens + t0);
            prefetch_l2_line(pos + 2 * tokens + t0);
        }
    }
    fill_inv_freq(inv_freq, HALF, prm);
    // Decode-size launches (U == 1: one unit per warp) issue their token's
    // position loads before the dependency wait, so that the loads complete
    // while the previous kernel drains (with programmatic dependent launch the
    // caller guarantees that the position ids are not written by the kernel
    // launched just before this one).  Only the loads move: evaluating the
    // angles there too measured slower, the window before the wait being
    // shorter than that work.
    int32_t pt0 = 0, ph0 = 0, pw0 = 0;
    if constexpr (U == 1) {
        if (unit0 < units) {
            int part0 = 0;
            const int64_t t0 = unit_token(unit0, splits, part0);
            pt0 = __ldg(pos + t0);
            ph0 = __ldg(pos + tokens + t0);
            pw0 = __ldg(pos + 2 * tokens + t0);
        }
    }
    pdl_wait();
    pdl_allow_dependents();

    const int64_t unit_stride = (int64_t)gridDim.x * kWarpsPerCta;
    for (int64_t unit = unit0; unit < units; unit += unit_stride) {
        int part = 0;
        const int64_t t = unit_token(unit, splits, part);
        const int h_first = hg + part * G * U;
        // the warp's next token into L2 while this one is worked on (a grid of
        // one wave walks several tokens per warp); decode-size launches (U ==
        // 1, one unit per warp) leave even the branch out, as the norm does
        if (U > 1 && lane == 0 && part == 0 && unit + unit_stride < units) {
            int part_n = 0;
            const int64_t tn = unit_token(unit + unit_stride, splits, part_n);
            if (hq > 0)
                prefetch_l2(q + (size_t)tn * hq * D, (uint32_t)(hq * D * sizeof(T)));
            if (hk > 0)
                prefetch_l2(k + (size_t)tn * hk * D, (uint32_t)(hk * D * sizeof(T)));
        }

        // the first batch of heads is loaded before the angles are evaluated, so
        // the q/k loads and the position loads share one memory latency
        uint4 lo[U], hi[U];
        auto load_batch = [&](int h0) {
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
        };
        load_batch(h_first);
        float c[E], s[E];
        if (U == 1 && unit == unit0)
            token_angles<E, P>(pt0, ph0, pw0, inv_freq, prm, lane, c, s);
        else
            token_angles<E, P>(__ldg(pos + t), __ldg(pos + tokens + t), __ldg(pos + 2 * tokens + t),
                               inv_freq, prm, lane, c, s);

        for (int h0 = h_first; h0 < nh; h0 += G * U * splits) {
            if (h0 != h_first)
                load_batch(h0);
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
                    st_out<kStream>(dst + j0, Vec<T>::pack(oa));
                    st_out<kStream>(dst + HALF + j0, Vec<T>::pack(ob));
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Streaming kernel (opt-in: arops_set_streaming(1), for 16-byte-aligned q/k;
// measured slower on B200 than the register kernel).  Each warp owns tokens
// gw, gw + nw, ... (gw = global warp index, nw = warps in the grid) and a ring
// of `slots` shared-memory slots, each holding one token's q and k heads.  Lane
// 0 keeps `slots` tokens in flight as bulk copies (TMA); the warp evaluates the
// token's angles (positions are fetched one token ahead) while its copy is in
// flight, then rotates the heads out of shared memory and stores them.  Warps
// never wait on each other, so an SM has ~30 tokens (~180 KB) requested at once.
// ---------------------------------------------------------------------------
constexpr int kTmaWarps = 4;

template <typename T, int P>
__global__ void __launch_bounds__(32 * kTmaWarps)
mrope_tma_kernel(const T* q, const T* k, T* q_out, T* k_out, const int32_t* __restrict__ pos,
                 int64_t tokens, int hq, int hk, int slots, const __grid_constant__ MropeParams prm,
                 unsigned* err_word)
{
    constexpr int E = Vec<T>::N;
    constexpr int G = 32 / P;
    constexpr int HALF = P * E;
    constexpr int D = 2 * HALF;
    constexpr int F = (E >= G) ? E / G : 1;
    extern __shared__ __align__(128) unsigned char smem[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pv = lane % P;
    const int hg = lane / P;
    const int j0 = pv * E;
    const int nh = hq + hk;
    const uint32_t q_bytes = (uint32_t)hq * D * sizeof(T);
    const uint32_t k_bytes = (uint32_t)hk * D * sizeof(T);
    const uint32_t slot = round_up(q_bytes + k_bytes, 128);
    unsigned char* ring = smem + (size_t)warp * slots * slot;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kTmaWarps * slots * slot) +
                     warp * slots;
    const int64_t gw = (int64_t)blockIdx.x * kTmaWarps + warp;
    const int64_t nw = (int64_t)gridDim.x * kTmaWarps;
    const int64_t my = tokens > gw ? (tokens - 1 - gw) / nw + 1 : 0;
    __shared__ double inv_freq[HALF];

    if (lane == 0) {
        for (int i = 0; i < slots; ++i)
            mbar_init(smem_addr(&bars[i]), 1);
        mbar_init_fence();
    }
    fill_inv_freq(inv_freq, HALF, prm);

    pdl_wait();
    pdl_allow_dependents();

    int64_t issued = 0;  // lane 0 only
    auto issue = [&](int64_t j) {
        const int64_t t = gw + j * nw;
        const int sidx = (int)(j % slots);
        const uint32_t bar = smem_addr(&bars[sidx]);
        unsigned char* dst = ring + (size_t)sidx * slot;
        mbar_arrive_expect_tx(bar, q_bytes + k_bytes);
        if (q_bytes)
            bulk_load(smem_addr(dst), q + t * hq * D, q_bytes, bar);
        if (k_bytes)
            bulk_load(smem_addr(dst + q_bytes), k + t * hk * D, k_bytes, bar);
    };
    if (lane == 0)
        for (; issued < slots && issued < my; ++issued)
            issue(issued);

    int32_t npt = 0, nph = 0, npw = 0;
    if (my > 0) {
        npt = __ldg(pos + gw);
        nph = __ldg(pos + tokens + gw);
        npw = __ldg(pos + 2 * tokens + gw);
    }
    for (int64_t j = 0; j < my; ++j) {
        const int64_t t = gw + j * nw;
        const int32_t pt = npt, ph = nph, pw = npw;
        if (j + 1 < my) {  // the next token's positions, one step ahead
            npt = __ldg(pos + t + nw);
            nph = __ldg(pos + tokens + t + nw);
            npw = __ldg(pos + 2 * tokens + t + nw);
        }
        float cs[F], sn[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const int jj = j0 + ((hg * F + f) % E);
            rope_cos_sin(inv_freq[jj], position_of(jj, prm, pt, ph, pw), &cs[f], &sn[f]);
        }
        float c[E], s[E];
#pragma unroll
        for (int m = 0; m < E; ++m) {
            const int src = pv + P * ((m / F) % G);
            c[m] = __shfl_sync(0xFFFFFFFFu, cs[m % F], src);
            s[m] = __shfl_sync(0xFFFFFFFFu, sn[m % F], src);
        }

        const int sidx = (int)(j % slots);
        const bool ok = mbar_wait(smem_addr(&bars[sidx]), (uint32_t)((j / slots) & 1));
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            if (lane == 0) {
                record_device_error(err_word, kDeviceErrTimeout);
                for (int64_t kk = j; kk < issued; ++kk)
                    mbar_wait(smem_addr(&bars[kk % slots]), (uint32_t)((kk / slots) & 1));
            }
            return;
        }
        const unsigned char* src = ring + (size_t)sidx * slot;
        for (int h = hg; h < nh; h += G) {
            float a[E], b[E], oa[E], ob[E];
            const unsigned char* hp = src + (size_t)h * D * sizeof(T);
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(hp + j0 * sizeof(T)), a);
            Vec<T>::unpack(*reinterpret_cast<const uint4*>(hp + (HALF + j0) * sizeof(T)), b);
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
        __syncwarp();  // every lane has read the slot; it can take the next copy
        if (lane == 0 && issued < my) {
            issue(issued);
            ++issued;
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
        rope_cos_sin(inv_freq_of(j, prm), p, &c, &s);
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

// ---------------------------------------------------------------------------
// M-RoPE fused with the KV-cache append ("Custom Triton kernels", item 3:
// new K, V of a token written into cache[head, position, :]).  One warp per
// token as in mrope_vec_kernel, over hq + 2*hkv "heads": q heads are rotated
// into q_out, k heads are rotated straight into their cache slot, v heads are
// copied into theirs; the rotated k never makes a round trip through memory.
// A token whose (cache row, position) lies outside the cache writes no cache
// slot and sets kDeviceErrBadIndex in the library's error word.
// ---------------------------------------------------------------------------
constexpr unsigned kDeviceErrBadIndex = 2u;

struct CacheArgs {
    const int32_t* loc;  // [2, tokens]: cache row, position
    int64_t rows;
    int64_t max_seq;
};

template <typename T, int P, int U>
__global__ void __launch_bounds__(32 * kWarpsPerCta)
mrope_append_kernel(const T* q, const T* k, const T* v, T* q_out, T* k_cache, T* v_cache,
                    const int32_t* __restrict__ pos, int64_t tokens, int hq, int hk, int splits,
                    const __grid_constant__ MropeParams prm, const __grid_constant__ CacheArgs ca,
                    unsigned* err_word)
{
    constexpr int E = Vec<T>::N;
    constexpr int G = 32 / P;
    constexpr int HALF = P * E;
    constexpr int D = 2 * HALF;
    // evict-first stores, except with one pass per warp (U == 1: decode-size launches)
    constexpr bool kStream = U > 1;
    const int lane = threadIdx.x & 31;
    const int pv = lane % P;
    const int hg = lane / P;
    const int j0 = pv * E;
    const int nh = hq + 2 * hk;
    __shared__ double inv_freq[HALF];

    const int64_t units = tokens * splits;
    const int64_t unit0 = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    {
        int part0 = 0;
        const int64_t t0 = unit_token(unit0, splits, part0);
        if (lane == 0 && unit0 < units && part0 == 0) {
            if (hq > 0)
                prefetch_l2(q + (size_t)t0 * hq * D, (uint32_t)(hq * D * sizeof(T)));
            if (hk > 0) {
                prefetch_l2(k + (size_t)t0 * hk * D, (uint32_t)(hk * D * sizeof(T)));
                prefetch_l2(v + (size_t)t0 * hk * D, (uint32_t)(hk * D * sizeof(T)));
                prefetch_l2_line(ca.loc + t0);
                prefetch_l2_line(ca.loc + tokens + t0);
            }
            prefetch_l2_line(pos + t0);
            prefetch_l2_line(pos + tokens + t0);
            prefetch_l2_line(pos + 2 * tokens + t0);
        }
    }
    fill_inv_freq(inv_freq, HALF, prm);
    pdl_wait();
    pdl_allow_dependents();

    const int64_t unit_stride = (int64_t)gridDim.x * kWarpsPerCta;
    for (int64_t unit = unit0; unit < units; unit += unit_stride) {
        int part = 0;
        const int64_t t = unit_token(unit, splits, part);
        const int h_first = hg + part * G * U;
        // the warp's next token into L2 while this one is worked on
        if (U > 1 && lane == 0 && part == 0 && unit + unit_stride < units) {
            int part_n = 0;
            const int64_t tn = unit_token(unit + unit_stride, splits, part_n);
            if (hq > 0)
                prefetch_l2(q + (size_t)tn * hq * D, (uint32_t)(hq * D * sizeof(T)));
            if (hk > 0) {
                prefetch_l2(k + (size_t)tn * hk * D, (uint32_t)(hk * D * sizeof(T)));
                prefetch_l2(v + (size_t)tn * hk * D, (uint32_t)(hk * D * sizeof(T)));
            }
        }
        int64_t cb = -1, cs = -1;
        if (hk > 0) {
            cb = __ldg(ca.loc + t);
            cs = __ldg(ca.loc + tokens + t);
        }
        const bool in_cache = cb >= 0 && cb < ca.rows && cs >= 0 && cs < ca.max_seq;
        if (hk > 0 && !in_cache && lane == 0)
            record_device_error(err_word, kDeviceErrBadIndex);

        uint4 lo[U], hi[U];
        auto src_of = [&](int h) -> const T* {
            if (h < hq)
                return q + ((size_t)t * hq + h) * D;
            if (h < hq + hk)
                return k + ((size_t)t * hk + (h - hq)) * D;
            return v + ((size_t)t * hk + (h - hq - hk)) * D;
        };
        auto load_batch = [&](int h0) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = h0 + u * G;
                if (h < nh) {
                    const T* src = src_of(h);
                    lo[u] = ld_stream(src + j0);
                    hi[u] = ld_stream(src + HALF + j0);
                }
            }
        };
        load_batch(h_first);
        float c[E], s[E];
        token_angles<E, P>(__ldg(pos + t), __ldg(pos + tokens + t), __ldg(pos + 2 * tokens + t),
                           inv_freq, prm, lane, c, s);

        for (int h0 = h_first; h0 < nh; h0 += G * U * splits) {
            if (h0 != h_first)
                load_batch(h0);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int h = h0 + u * G;
                if (h >= nh)
                    continue;
                if (h >= hq + hk) {  // v: copied unrotated into its cache slot
                    if (in_cache) {
                        T* dst = v_cache + (((size_t)cb * hk + (h - hq - hk)) * ca.max_seq + cs) * D;
                        st_out<kStream>(dst + j0, lo[u]);
                        st_out<kStream>(dst + HALF + j0, hi[u]);
                    }
                    continue;
                }
                float a[E], b[E], oa[E], ob[E];
                Vec<T>::unpack(lo[u], a);
                Vec<T>::unpack(hi[u], b);
#pragma unroll
                for (int m = 0; m < E; ++m) {
                    oa[m] = a[m] * c[m] - b[m] * s[m];
                    ob[m] = b[m] * c[m] + a[m] * s[m];
                }
                T* dst;
                if (h < hq) {
                    dst = q_out + ((size_t)t * hq + h) * D;
                } else {
                    if (!in_cache)
                        continue;
                    dst = k_cache + (((size_t)cb * hk + (h - hq)) * ca.max_seq + cs) * D;
                }
                st_out<kStream>(dst + j0, Vec<T>::pack(oa));
                st_out<kStream>(dst + HALF + j0, Vec<T>::pack(ob));
            }
        }
    }
}

// Any even head_dim, any alignment: one thread per (token, head, pair).
template <typename T>
__global__ void __launch_bounds__(256)
mrope_append_scalar_kernel(const T* q, const T* k, const T* v, T* q_out, T* k_cache, T* v_cache,
                           const int32_t* __restrict__ pos, int64_t tokens, int hq, int hk,
                           int half, const __grid_constant__ MropeParams prm,
                           const __grid_constant__ CacheArgs ca, unsigned* err_word)
{
    pdl_wait();
    pdl_allow_dependents();
    const int nh = hq + 2 * hk;
    const int64_t total = tokens * nh * half;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(idx % half);
        const int h = (int)((idx / half) % nh);
        const int64_t t = idx / ((int64_t)half * nh);
        const int64_t d2 = 2 * (int64_t)half;
        if (h < hq + hk) {
            const int32_t p = position_of(j, prm, __ldg(pos + t), __ldg(pos + tokens + t),
                                          __ldg(pos + 2 * tokens + t));
            float c, s;
            rope_cos_sin(inv_freq_of(j, prm), p, &c, &s);
            const T* src = (h < hq) ? q + ((size_t)t * hq + h) * d2 : k + ((size_t)t * hk + (h - hq)) * d2;
            const float a = load_elem(src + j);
            const float b = load_elem(src + half + j);
            T* dst;
            if (h < hq) {
                dst = q_out + ((size_t)t * hq + h) * d2;
            } else {
                const int64_t cb = __ldg(ca.loc + t), cs = __ldg(ca.loc + tokens + t);
                if (cb < 0 || cb >= ca.rows || cs < 0 || cs >= ca.max_seq) {
                    if (j == 0)
                        record_device_error(err_word, kDeviceErrBadIndex);
                    continue;
                }
                dst = k_cache + (((size_t)cb * hk + (h - hq)) * ca.max_seq + cs) * d2;
            }
            store_elem(dst + j, a * c - b * s);
            store_elem(dst + half + j, b * c + a * s);
        } else {
            const int64_t cb = __ldg(ca.loc + t), cs = __ldg(ca.loc + tokens + t);
            if (cb < 0 || cb >= ca.rows || cs < 0 || cs >= ca.max_seq)
                continue;
            const T* src = v + ((size_t)t * hk + (h - hq - hk)) * d2;
            T* dst = v_cache + (((size_t)cb * hk + (h - hq - hk)) * ca.max_seq + cs) * d2;
            dst[j] = src[j];
            dst[half + j] = src[half + j];
        }
    }
}

constexpr int kHeadUnroll = 8;

template <typename T, int P, int U>
cudaError_t launch_vec_u(const MropeArgs& a, const MropeParams& prm, cudaStream_t st, int64_t cap,
                         int splits = 1)
{
    const int64_t grid = std::min<int64_t>(ceil_div(a.tokens * splits, kWarpsPerCta), cap);
    return launch(mrope_vec_kernel<T, P, U>, dim3((unsigned)grid), dim3(32 * kWarpsPerCta), 0, st,
                  static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                  static_cast<T*>(a.q_out), static_cast<T*>(a.k_out), a.pos, a.tokens,
                  (int)a.n_q_heads, (int)a.n_k_heads, splits, prm);
}

// A problem with at most one pass for every warp the GPU holds at once (a
// decode step: a few tokens) is latency-bound: one pass per warp, the token's
// passes spread over as many warps.
inline bool one_pass_per_warp(int64_t tokens, int passes, int64_t cap)
{
    return tokens * passes <= cap;
}

// Otherwise one warp per token with every pass's heads in flight at once (U =
// passes, so no registers are held for absent heads), on a grid of one wave of
// resident CTAs: each warp walks several tokens and prefetches its next token
// into L2 while it works on the current one.  4096 tokens of 16 + 8 heads of
// 128 measured 8.1 us a launch back to back on B200, against 9.2 us with one
// warp per token and 1,024 CTAs, and 8.5 us with two warps per token.
constexpr int kPrefillWaves = 1;

template <typename T, int P, int U>
cudaError_t launch_vec_wave(const MropeArgs& a, const MropeParams& prm, cudaStream_t st,
                            int64_t cap, int sm_count)
{
    cap = std::min<int64_t>(
        cap, wave_ctas<mrope_vec_kernel<T, P, U>>(32 * kWarpsPerCta, sm_count, kPrefillWaves));
    return launch_vec_u<T, P, U>(a, prm, st, cap);
}

template <typename T, int P>
cudaError_t launch_vec(const MropeArgs& a, const MropeParams& prm, cudaStream_t st, int64_t cap,
                       int sm_count)
{
    constexpr int G = 32 / P;
    const int passes = (int)ceil_div(a.n_q_heads + a.n_k_heads, G);
    if (one_pass_per_warp(a.tokens, passes, cap))
        return launch_vec_u<T, P, 1>(a, prm, st, cap, passes);
    if (passes <= 2)
        return launch_vec_wave<T, P, 2>(a, prm, st, cap, sm_count);
    if (passes <= 4)
        return launch_vec_wave<T, P, 4>(a, prm, st, cap, sm_count);
    if (passes <= 6)
        return launch_vec_wave<T, P, 6>(a, prm, st, cap, sm_count);
    return launch_vec_wave<T, P, kHeadUnroll>(a, prm, st, cap, sm_count);
}

// Streaming launch; cudaErrorNotSupported when two slots per warp do not fit.
template <typename T, int P>
cudaError_t launch_tma(const MropeArgs& a, const MropeParams& prm, cudaStream_t st,
                       const DeviceInfo& di)
{
    const uint32_t tok = (uint32_t)(a.n_q_heads + a.n_k_heads) * a.head_dim * sizeof(T);
    const uint32_t slot = round_up(tok, 128);
    // ~96 KB of slots per CTA lets two CTAs (8 warps) share an SM
    int slots = (int)std::min<uint32_t>(8, (96u * 1024u) / (kTmaWarps * slot));
    slots = std::max(slots, 2);
    const uint32_t smem = (uint32_t)kTmaWarps * slots * (slot + 8) + 128;
    if (smem > kMaxSmemPerCta)
        return cudaErrorNotSupported;
    auto kernel = mrope_tma_kernel<T, P>;
    int per_sm = 0;
    cudaError_t err = resident_ctas(kernel, 32 * kTmaWarps, smem, &per_sm);
    if (err != cudaSuccess)
        return err;
    if (per_sm < 1)
        return cudaErrorNotSupported;
    unsigned* word = nullptr;
    err = device_error_word(&word);
    if (err != cudaSuccess)
        return err;
    const int64_t grid =
        std::min<int64_t>(ceil_div(a.tokens, kTmaWarps), (int64_t)di.sm_count * per_sm);
    return launch(kernel, dim3((unsigned)grid), dim3(32 * kTmaWarps), smem, st,
                  static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                  static_cast<T*>(a.q_out), static_cast<T*>(a.k_out), a.pos, a.tokens,
                  (int)a.n_q_heads, (int)a.n_k_heads, slots, prm, word);
}

template <typename T>
cudaError_t try_tma(const MropeArgs& a, const MropeParams& prm, cudaStream_t st,
                    const DeviceInfo& di, int p)
{
    switch (p) {
    case 1: return launch_tma<T, 1>(a, prm, st, di);
    case 2: return launch_tma<T, 2>(a, prm, st, di);
    case 4: return launch_tma<T, 4>(a, prm, st, di);
    case 8: return launch_tma<T, 8>(a, prm, st, di);
    case 16: return launch_tma<T, 16>(a, prm, st, di);
    case 32: return launch_tma<T, 32>(a, prm, st, di);
    default: return cudaErrorNotSupported;
    }
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
    if (aligned && half % E == 0 && streaming_enabled()) {
        err = try_tma<T>(a, prm, st, di, half / E);
        if (err != cudaErrorNotSupported)
            return err;
    }
    if (aligned && half % E == 0) {
        switch (half / E) {
        case 1: return launch_vec<T, 1>(a, prm, st, cap, di.sm_count);
        case 2: return launch_vec<T, 2>(a, prm, st, cap, di.sm_count);
        case 4: return launch_vec<T, 4>(a, prm, st, cap, di.sm_count);
        case 8: return launch_vec<T, 8>(a, prm, st, cap, di.sm_count);
        case 16: return launch_vec<T, 16>(a, prm, st, cap, di.sm_count);
        case 32: return launch_vec<T, 32>(a, prm, st, cap, di.sm_count);
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

template <typename T, int P, int U>
cudaError_t launch_append_u(const MropeArgs& a, const AppendArgs& x, const MropeParams& prm,
                            const CacheArgs& ca, unsigned* word, cudaStream_t st, int64_t cap,
                            int splits = 1)
{
    const int64_t grid = std::min<int64_t>(ceil_div(a.tokens * splits, kWarpsPerCta), cap);
    return launch(mrope_append_kernel<T, P, U>, dim3((unsigned)grid), dim3(32 * kWarpsPerCta), 0,
                  st, static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                  static_cast<const T*>(x.v), static_cast<T*>(a.q_out),
                  static_cast<T*>(x.k_cache), static_cast<T*>(x.v_cache), a.pos, a.tokens,
                  (int)a.n_q_heads, (int)a.n_k_heads, splits, prm, ca, word);
}

template <typename T, int P, int U>
cudaError_t launch_append_wave(const MropeArgs& a, const AppendArgs& x, const MropeParams& prm,
                               const CacheArgs& ca, unsigned* word, cudaStream_t st, int64_t cap,
                               int sm_count)
{
    cap = std::min<int64_t>(
        cap, wave_ctas<mrope_append_kernel<T, P, U>>(32 * kWarpsPerCta, sm_count, kPrefillWaves));
    return launch_append_u<T, P, U>(a, x, prm, ca, word, st, cap);
}

template <typename T, int P>
cudaError_t launch_append_p(const MropeArgs& a, const AppendArgs& x, const MropeParams& prm,
                            const CacheArgs& ca, unsigned* word, cudaStream_t st, int64_t cap,
                            int sm_count)
{
    constexpr int G = 32 / P;
    const int passes = (int)ceil_div(a.n_q_heads + 2 * a.n_k_heads, G);
    if (one_pass_per_warp(a.tokens, passes, cap))
        return launch_append_u<T, P, 1>(a, x, prm, ca, word, st, cap, passes);
    // as in launch_vec: one warp per token, one wave of resident CTAs
    if (passes <= 2)
        return launch_append_wave<T, P, 2>(a, x, prm, ca, word, st, cap, sm_count);
    if (passes <= 4)
        return launch_append_wave<T, P, 4>(a, x, prm, ca, word, st, cap, sm_count);
    if (passes <= 6)
        return launch_append_wave<T, P, 6>(a, x, prm, ca, word, st, cap, sm_count);
    // More passes: two warps per token, four passes in flight each (4096
    // tokens of 16 q + 8 k + 8 v heads of 128: 12.0 against 12.8 us a launch
    // back to back on B200 with one warp and all eight passes; plain M-RoPE's
    // six passes measured slower split).  The split's unit index is 32-bit.
    if (a.tokens * 2 > (int64_t)INT32_MAX)
        return launch_append_wave<T, P, kHeadUnroll>(a, x, prm, ca, word, st, cap, sm_count);
    cap = std::min<int64_t>(
        cap, wave_ctas<mrope_append_kernel<T, P, 4>>(32 * kWarpsPerCta, sm_count, kPrefillWaves));
    return launch_append_u<T, P, 4>(a, x, prm, ca, word, st, cap, 2);
}

template <typename T>
cudaError_t launch_append_t(const MropeArgs& a, const AppendArgs& x, const MropeParams& prm,
                            cudaStream_t st)
{
    DeviceInfo di;
    cudaError_t err = current_device_info(&di);
    if (err != cudaSuccess)
        return err;
    unsigned* word = nullptr;
    err = device_error_word(&word);
    if (err != cudaSuccess)
        return err;
    CacheArgs ca;
    ca.loc = x.cache_loc;
    ca.rows = x.cache_rows;
    ca.max_seq = x.max_seq;
    constexpr int E = Vec<T>::N;
    const int half = a.head_dim / 2;
    const bool aligned = aligned16(a.q) && aligned16(a.q_out) &&
                         (a.n_k_heads == 0 || (aligned16(a.k) && aligned16(x.v) &&
                                               aligned16(x.k_cache) && aligned16(x.v_cache)));
    const int64_t cap = (int64_t)di.sm_count * 64;
    if (aligned && half % E == 0) {
        switch (half / E) {
        case 1: return launch_append_p<T, 1>(a, x, prm, ca, word, st, cap, di.sm_count);
        case 2: return launch_append_p<T, 2>(a, x, prm, ca, word, st, cap, di.sm_count);
        case 4: return launch_append_p<T, 4>(a, x, prm, ca, word, st, cap, di.sm_count);
        case 8: return launch_append_p<T, 8>(a, x, prm, ca, word, st, cap, di.sm_count);
        case 16: return launch_append_p<T, 16>(a, x, prm, ca, word, st, cap, di.sm_count);
        case 32: return launch_append_p<T, 32>(a, x, prm, ca, word, st, cap, di.sm_count);
        default: break;
        }
    }
    const int64_t total = a.tokens * (int64_t)(a.n_q_heads + 2 * a.n_k_heads) * half;
    const int64_t grid = std::min<int64_t>(ceil_div(total, 256), (int64_t)di.sm_count * 16);
    return launch(mrope_append_scalar_kernel<T>, dim3((unsigned)grid), dim3(256), 0, st,
                  static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                  static_cast<const T*>(x.v), static_cast<T*>(a.q_out),
                  static_cast<T*>(x.k_cache), static_cast<T*>(x.v_cache), a.pos, a.tokens,
                  (int)a.n_q_heads, (int)a.n_k_heads, half, prm, ca, word);
}

}  // namespace

cudaError_t launch_mrope_append(const MropeArgs& a, const AppendArgs& x, arops_dtype dtype,
                                cudaStream_t stream)
{
    MropeParams prm;
    prm.sec0 = a.sections[0];
    prm.sec01 = a.sections[0] + a.sections[1];
    prm.freq_scale = 2.0 * log2((double)a.theta) / (double)a.head_dim;
    if (dtype == AROPS_BF16)
        return launch_append_t<__nv_bfloat16>(a, x, prm, stream);
    return launch_append_t<float>(a, x, prm, stream);
}

cudaError_t launch_mrope(const MropeArgs& a, arops_dtype dtype, cudaStream_t stream)
{
    MropeParams prm;
    prm.sec0 = a.sections[0];
    prm.sec01 = a.sections[0] + a.sections[1];
    prm.freq_scale = 2.0 * log2((double)a.theta) / (double)a.head_dim;
    if (dtype == AROPS_BF16)
        return launch_mrope_t<__nv_bfloat16>(a, prm, stream);
    return launch_mrope_t<float>(a, prm, stream);
}

}  // namespace arops
