// Cross-entropy against probability (soft) targets.
//
// MLX PR #4188 ("Shift by the max in cross_entropy") states the loss of a row
// as its log-sum-exp minus the target-weighted logits, assembled from values
// shifted by the row max. With a target distribution t (label smoothing mixes
// it with the uniform one, t' = (1-eps) t + eps/V):
//     loss = sum_j t'_j (lse - z_j) = L T' - sum_j t'_j (z_j - m),
//     L = log sum_j exp(z_j - m),  T' = sum_j t'_j = (1-eps) T + eps,
//     dz_j = g (p_j T' - t'_j),  p_j = exp(z_j - lse).
// Besides the online (m, s) of Ineshin, "A fused linear cross-entropy
// forward kernel for Apple GPUs", section 1, each lane carries D = sum t_j
// (z_j - m) and T = sum t_j (and, with eps, U = sum (z_j - m) and the count
// K); when m grows to m', D gains T (m - m') and U gains K (m - m'). A class
// with t_j = 0 adds nothing to D, even at z_j = -inf (0 log 0 = 0).
//
// G lanes share a row (G = 1..32, the smallest group whose one step of U
// vectors per lane covers the row; longer rows loop with G = 32), 32 / G rows
// per warp, rows in a grid-stride loop over 64-bit indices.
#include "ce_device.cuh"
#include "ce_launch.h"

namespace ceb {

struct SoftState {
    float m, s, d, t, u;
    int k;
};

template <typename T, int n>
__device__ __forceinline__ void load_n(const T* p, int64_t col, int64_t s_col, float (&out)[n]) {
    if constexpr (n == 1) {
        out[0] = to_f32(p[col * s_col]);
    } else {
        static_assert((n * sizeof(T)) % 16 == 0, "whole 16-byte words");
        constexpr int W = (int)(n * sizeof(T) / 16);
        constexpr int PER = 16 / (int)sizeof(T);
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const uint4 r = __ldcs(reinterpret_cast<const uint4*>(p + col) + w);
            unpack_words<T>(r, out + w * PER);
        }
    }
}

template <bool EPS>
__device__ __forceinline__ void soft_rescale(SoftState& st, float mn) {
    if (st.m != mn) {
        const float dm = st.m - mn;  // -inf when the state was empty
        st.s *= ex2(dm * kLog2e);
        if (st.t != 0.f) st.d += st.t * dm;
        if constexpr (EPS) {
            if (st.k != 0) st.u += (float)st.k * dm;
        }
        st.m = mn;
    }
}

// Folds n (z, t) pairs, all valid.
template <int n, bool EPS>
__device__ __forceinline__ void soft_fold(SoftState& st, const float (&z)[n], const float (&t)[n]) {
    float cm = z[0];
#pragma unroll
    for (int i = 1; i < n; ++i) cm = fmaxf(cm, z[i]);
    soft_rescale<EPS>(st, fmaxf(st.m, cm));
    const float ms = st.m == -INFINITY ? 0.f : st.m;
    float s = 0.f, d = 0.f, tt = 0.f, u = 0.f;
#pragma unroll
    for (int i = 0; i < n; ++i) {
        const float x = z[i] - ms;
        s += ex2(x * kLog2e);
        if (t[i] != 0.f) d = fmaf(t[i], x, d);
        tt += t[i];
        if constexpr (EPS) u += x;
    }
    st.s += s;
    st.d += d;
    st.t += tt;
    if constexpr (EPS) {
        st.u += u;
        st.k += n;
    }
}

template <int G, bool EPS>
__device__ __forceinline__ void soft_group_reduce(SoftState& st) {
    if constexpr (G > 1) {
        float M = st.m;
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        soft_rescale<EPS>(st, M);
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
            st.s += __shfl_xor_sync(0xffffffffu, st.s, off);
            st.d += __shfl_xor_sync(0xffffffffu, st.d, off);
            st.t += __shfl_xor_sync(0xffffffffu, st.t, off);
            if constexpr (EPS) {
                st.u += __shfl_xor_sync(0xffffffffu, st.u, off);
                st.k += __shfl_xor_sync(0xffffffffu, st.k, off);
            }
        }
    }
}

template <typename TZ, typename TT, int VEC, int G, int U, bool EPS, int MINB>
__global__ void __launch_bounds__(256, MINB) k_soft_fwd(SoftArgs a) {
    const TZ* __restrict__ z = reinterpret_cast<const TZ*>(a.z);
    const TT* __restrict__ tg = reinterpret_cast<const TT*>(a.t);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const float eps = a.eps;

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        const bool active = r < a.N;
        SoftState st{-INFINITY, 0.f, 0.f, 0.f, 0.f, 0};
        const TZ* zr = z;
        const TT* tr = tg;
        if (active) {
            zr = z + row_offset(a.lz, r, a.N);
            tr = tg + row_offset(a.lt, r, a.N);
        }
        for (int64_t vb = 0; vb < nvec; vb += (int64_t)G * U) {
            Raw<TZ, VEC> rz[U];
            Raw<TT, VEC> rt[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + u * G + gl;
                ok[u] = active && vi < nvec;
                if (ok[u]) {
                    load_raw<TZ, VEC>(zr, vi * VEC, a.lz.s_col, rz[u]);
                    load_raw<TT, VEC>(tr, vi * VEC, a.lt.s_col, rt[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float zv[VEC], tv[VEC];
                unpack_raw<TZ, VEC>(rz[u], zv);
                unpack_raw<TT, VEC>(rt[u], tv);
                soft_fold<VEC, EPS>(st, zv, tv);
            }
        }
        if (active) {
            for (int q = gl; q < tail; q += G) {
                float zx[1], tx[1];
                load_n<TZ, 1>(zr, nvec * VEC + q, a.lz.s_col, zx);
                load_n<TT, 1>(tr, nvec * VEC + q, a.lt.s_col, tx);
                soft_fold<1, EPS>(st, zx, tx);
            }
        }
        soft_group_reduce<G, EPS>(st);
        if (active && gl == 0) {
            OnlineState os = empty_state();
            os.m = st.m;
            os.s = st.s;
            float L, hi, lo;
            lse_pair(os, L, hi, lo);
            a.lse[r] = hi;
            if (a.lse_lo) a.lse_lo[r] = lo;
            if (a.tsum) a.tsum[r] = st.t;
            float loss;
            if (st.m == -INFINITY || st.m != st.m) {
                loss = __int_as_float(0x7fc00000);
            } else {
                const float Tp = (1.f - eps) * st.t + eps;
                float dot = (1.f - eps) * st.d;
                if constexpr (EPS) dot += (eps / (float)a.V) * st.u;
                loss = L * Tp - dot;
            }
            a.loss[r] = loss;
        }
    }
}

template <typename TZ, typename TT, typename TO, int VEC, int G, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) k_soft_bwd(SoftArgs a) {
    const TZ* z = reinterpret_cast<const TZ*>(a.z);
    const TT* __restrict__ tg = reinterpret_cast<const TT*>(a.t);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const float eps = a.eps, eps_v = a.eps / (float)a.V;

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        if (r >= a.N) continue;
        const TZ* zr = z + row_offset(a.lz, r, a.N);
        const TT* tr = tg + row_offset(a.lt, r, a.N);
        TO* dr = dz + row_offset(a.ld, r, a.N);
        const float g = a.g[r * a.g_stride];
        const float hi = a.lse[r];
        const float c_lo = (a.lse_lo ? a.lse_lo[r] : 0.f) * kLog2e;
        const float Tp = a.tsum ? (1.f - eps) * a.tsum[r] + eps : 1.f;
        const float gT = g * Tp, g1 = g * (1.f - eps), ge = g * eps_v;
        for (int64_t vb = gl; vb < nvec; vb += (int64_t)G * U) {
            Raw<TZ, VEC> rz[U];
            Raw<TT, VEC> rt[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + (int64_t)u * G;
                ok[u] = vi < nvec;
                if (ok[u]) {
                    load_raw<TZ, VEC>(zr, vi * VEC, a.lz.s_col, rz[u]);
                    load_raw<TT, VEC>(tr, vi * VEC, a.lt.s_col, rt[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float zv[VEC], tv[VEC], o[VEC];
                unpack_raw<TZ, VEC>(rz[u], zv);
                unpack_raw<TT, VEC>(rt[u], tv);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float p = ex2(fmaf(zv[e] - hi, kLog2e, -c_lo));
                    o[e] = fmaf(gT, p, -fmaf(g1, tv[e], ge));
                }
                store_vec<TO, VEC>(dr, (vb + (int64_t)u * G) * VEC, a.ld.s_col, o);
            }
        }
        for (int q = gl; q < tail; q += G) {
            const int64_t col = nvec * VEC + q;
            float zx[1], tx[1];
            load_n<TZ, 1>(zr, col, a.lz.s_col, zx);
            load_n<TT, 1>(tr, col, a.lt.s_col, tx);
            const float p = ex2(fmaf(zx[0] - hi, kLog2e, -c_lo));
            cvt_store1(dr + col * a.ld.s_col, fmaf(gT, p, -fmaf(g1, tx[0], ge)));
        }
    }
}

// ---------------------------------------------------------------------------
// Vectors per lane per step and resident blocks: raw words keep four
// vectors of logits and targets in flight per lane within a 64-register
// budget (four blocks per SM; three for the backward of 16-bit logits,
// whose eight-wide vectors need more registers); the scalar path keeps eight.
// The planner's lane grouping uses the same U (plan_soft).
template <typename TZ, typename TT, int VEC, bool BWD = false> struct SoftShape {
    // float targets of 16-bit logits take twice the words: two vectors
    static constexpr int U = VEC == 1 ? 8 : (sizeof(TT) > sizeof(TZ) ? 2 : 4);
    static constexpr int MINB = VEC == 1 ? 2 : ((BWD && VEC == 8) ? 3 : 4);
};

template <typename TZ, typename TT, int VEC, bool EPS>
static cudaError_t launch_soft_fwd_v(const SoftPlan& p, const SoftArgs& a, cudaStream_t s) {
    constexpr int U = SoftShape<TZ, TT, VEC>::U, MB = SoftShape<TZ, TT, VEC>::MINB;
#define CEB_SOFT(GG)                                                              \
    if (p.G == GG) {                                                              \
        k_soft_fwd<TZ, TT, VEC, GG, U, EPS, MB><<<p.grid, 256, 0, s>>>(a);        \
        return cudaGetLastError();                                                \
    }
    CEB_SOFT(1) CEB_SOFT(2) CEB_SOFT(4) CEB_SOFT(8) CEB_SOFT(16) CEB_SOFT(32)
#undef CEB_SOFT
    return cudaErrorInvalidValue;
}

template <typename TZ, typename TT, typename TO, int VEC>
static cudaError_t launch_soft_bwd_v(const SoftPlan& p, const SoftArgs& a, cudaStream_t s) {
    constexpr int U = SoftShape<TZ, TT, VEC, true>::U, MB = SoftShape<TZ, TT, VEC, true>::MINB;
#define CEB_SOFT(GG)                                                              \
    if (p.G == GG) {                                                              \
        k_soft_bwd<TZ, TT, TO, VEC, GG, U, MB><<<p.grid, 256, 0, s>>>(a);         \
        return cudaGetLastError();                                                \
    }
    CEB_SOFT(1) CEB_SOFT(2) CEB_SOFT(4) CEB_SOFT(8) CEB_SOFT(16) CEB_SOFT(32)
#undef CEB_SOFT
    return cudaErrorInvalidValue;
}

template <typename TZ, typename TT>
static cudaError_t soft_fwd_t(const SoftPlan& p, const SoftArgs& a, cudaStream_t s) {
    constexpr int V8 = ElemTraits<TZ>::kVec;
    const bool e = a.eps != 0.f;
    if (p.vec == 1)
        return e ? launch_soft_fwd_v<TZ, TT, 1, true>(p, a, s) : launch_soft_fwd_v<TZ, TT, 1, false>(p, a, s);
    return e ? launch_soft_fwd_v<TZ, TT, V8, true>(p, a, s) : launch_soft_fwd_v<TZ, TT, V8, false>(p, a, s);
}

template <typename TZ, typename TT, typename TO>
static cudaError_t soft_bwd_t(const SoftPlan& p, const SoftArgs& a, cudaStream_t s) {
    constexpr int V8 = ElemTraits<TZ>::kVec;
    if (p.vec == 1) return launch_soft_bwd_v<TZ, TT, TO, 1>(p, a, s);
    return launch_soft_bwd_v<TZ, TT, TO, V8>(p, a, s);
}

// dtypes: 0 f32, 1 bf16, 2 f16; targets in the logits' dtype or f32; the
// gradient in the logits' dtype or f32.
cudaError_t launch_soft_forward(const SoftPlan& p, const SoftArgs& a, int dz_t, int dt_t,
                                cudaStream_t s) {
    switch (dz_t * 3 + dt_t) {
        case 0: return soft_fwd_t<float, float>(p, a, s);
        case 3: return soft_fwd_t<__nv_bfloat16, float>(p, a, s);
        case 4: return soft_fwd_t<__nv_bfloat16, __nv_bfloat16>(p, a, s);
        case 6: return soft_fwd_t<__half, float>(p, a, s);
        case 8: return soft_fwd_t<__half, __half>(p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_soft_backward(const SoftPlan& p, const SoftArgs& a, int dz_t, int dt_t, int do_t,
                                 cudaStream_t s) {
    const bool f = do_t == 0;
    switch (dz_t * 3 + dt_t) {
        case 0: return soft_bwd_t<float, float, float>(p, a, s);
        case 3: return f ? soft_bwd_t<__nv_bfloat16, float, float>(p, a, s)
                         : soft_bwd_t<__nv_bfloat16, float, __nv_bfloat16>(p, a, s);
        case 4: return f ? soft_bwd_t<__nv_bfloat16, __nv_bfloat16, float>(p, a, s)
                         : soft_bwd_t<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(p, a, s);
        case 6: return f ? soft_bwd_t<__half, float, float>(p, a, s)
                         : soft_bwd_t<__half, float, __half>(p, a, s);
        case 8: return f ? soft_bwd_t<__half, __half, float>(p, a, s)
                         : soft_bwd_t<__half, __half, __half>(p, a, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ceb
