// Device-side building blocks of the row cross-entropy kernels (sm_100a).
//
// The per-row statistic is the online log-sum-exp state of Ineshin, "A fused
// linear cross-entropy forward kernel for Apple GPUs", section 1: a running
// maximum m and the sum s of exp(z - m), rescaled whenever m grows. We carry
// two more numbers so the loss can be assembled from max-shifted values as in
// MLX PR #4188 ("Shift by the max in cross_entropy"): t, the sum of (z - m)
// over the k elements seen so far (the label-smoothing term needs the mean
// logit, and the mean moves with the shift), and k itself.
//
// Merging two states is associative and is done with one operator everywhere
// (lane shuffles, the one shared-memory exchange per CTA, the split merge):
//   (m1,s1,t1,k1) + (m2,s2,t2,k2) = (M, s1 e^{m1-M} + s2 e^{m2-M},
//                                    t1 + k1 (m1-M) + t2 + k2 (m2-M), k1+k2)
// with M = max(m1, m2). A side whose m equals M takes factor 1 and shift 0, so
// an empty side (m = -inf) merges as the identity and never produces
// exp(-inf - (-inf)) = NaN.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ce_launch.h"

namespace ceb {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Element offset of logical row r. A plain matrix (one outer block) needs no
// division.
__device__ __forceinline__ int64_t row_offset(const Layout& L, int64_t r, int64_t N) {
    if (L.inner >= N) return r * L.s_inner;
    const int64_t o = r / L.inner;
    return o * L.s_outer + (r - o * L.inner) * L.s_inner;
}

// max of three floats in one instruction; like fmaxf, a NaN operand is
// dropped unless all are NaN.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Hardware base-2 exponential (MUFU); exp(x) = ex2(x * log2 e).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------
// Loads. VEC = 16 / sizeof(T) elements per 16-byte load on the vector path,
// VEC = 1 on the scalar path. Streaming loads (evict-first) for data read once.
template <typename T> struct ElemTraits;
template <> struct ElemTraits<float> { static constexpr int kVec = 4; };
template <> struct ElemTraits<__nv_bfloat16> { static constexpr int kVec = 8; };
template <> struct ElemTraits<__half> { static constexpr int kVec = 8; };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ void unpack_words(const uint4& r, float* out);

template <>
__device__ __forceinline__ void unpack_words<float>(const uint4& r, float* out) {
    out[0] = __uint_as_float(r.x);
    out[1] = __uint_as_float(r.y);
    out[2] = __uint_as_float(r.z);
    out[3] = __uint_as_float(r.w);
}

template <>
__device__ __forceinline__ void unpack_words<__nv_bfloat16>(const uint4& r, float* out) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        out[2 * k] = __uint_as_float(w[k] << 16);
        out[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
}

template <>
__device__ __forceinline__ void unpack_words<__half>(const uint4& r, float* out) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
        float2 f = __half22float2(h);
        out[2 * k] = f.x;
        out[2 * k + 1] = f.y;
    }
}

// Loads VEC consecutive (VEC > 1, s_col = 1, 16-byte aligned) or one
// (VEC = 1, any stride) element(s) starting at column `col` of `row`.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* row, int64_t col, int64_t s_col, float* out) {
    if constexpr (VEC == 1) {
        out[0] = to_f32(row[col * s_col]);
    } else {
        const uint4 r = __ldcs(reinterpret_cast<const uint4*>(row + col));
        unpack_words<T>(r, out);
    }
}

// Plain (coherent) loads for kernels whose output may alias the input.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec_coherent(const T* row, int64_t col, int64_t s_col,
                                                  float* out) {
    if constexpr (VEC == 1) {
        out[0] = to_f32(row[col * s_col]);
    } else {
        const uint4 r = *reinterpret_cast<const uint4*>(row + col);
        unpack_words<T>(r, out);
    }
}

// ---------------------------------------------------------------------------
// Stores of n = VEC floats converted to T (round to nearest even).
__device__ __forceinline__ void cvt_store1(float* p, float v) { __stcs(p, v); }
__device__ __forceinline__ void cvt_store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void cvt_store1(__half* p, float v) { *p = __float2half_rn(v); }

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16*, float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack2(__half*, float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <typename TO, int VEC>
__device__ __forceinline__ void store_vec(TO* row, int64_t col, int64_t s_col, const float* v) {
    if constexpr (VEC == 1) {
        cvt_store1(row + col * s_col, v[0]);
    } else if constexpr (sizeof(TO) == 4) {
        // VEC floats = VEC*4 bytes: one or two 16-byte stores
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
            uint4 w = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                 __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
            __stcs(reinterpret_cast<uint4*>(row + col) + q, w);
        }
    } else {
        static_assert(VEC == 8, "16-bit outputs are stored 8 at a time");
        uint4 w = make_uint4(pack2((TO*)nullptr, v[0], v[1]), pack2((TO*)nullptr, v[2], v[3]),
                             pack2((TO*)nullptr, v[4], v[5]), pack2((TO*)nullptr, v[6], v[7]));
        __stcs(reinterpret_cast<uint4*>(row + col), w);
    }
}

// VEC elements of T held as raw 16-byte words (VEC > 1) or one float (VEC =
// 1) between the load and the use, so that many loads can be in flight in
// few registers.
template <typename T, int VEC>
struct Raw {
    static constexpr int W = VEC == 1 ? 1 : (int)(VEC * sizeof(T) / 16);
    uint4 w[W];
};

template <typename T, int VEC>
__device__ __forceinline__ void load_raw(const T* p, int64_t col, int64_t s_col, Raw<T, VEC>& r) {
    if constexpr (VEC == 1) {
        r.w[0].x = __float_as_uint(to_f32(p[col * s_col]));
    } else {
#pragma unroll
        for (int w = 0; w < Raw<T, VEC>::W; ++w) r.w[w] = __ldcs(reinterpret_cast<const uint4*>(p + col) + w);
    }
}

template <typename T, int VEC>
__device__ __forceinline__ void unpack_raw(const Raw<T, VEC>& r, float (&out)[VEC]) {
    if constexpr (VEC == 1) {
        out[0] = __uint_as_float(r.w[0].x);
    } else {
        constexpr int PER = 16 / (int)sizeof(T);
#pragma unroll
        for (int w = 0; w < Raw<T, VEC>::W; ++w) unpack_words<T>(r.w[w], out + w * PER);
    }
}

// ---------------------------------------------------------------------------
// Online state: running max m, s = sum_j exp(z_j - m) and t = sum_j (z_j - m)
// over the k elements seen. Every term is formed from the difference z_j - m
// first (exact when z_j is near m, by Sterbenz's lemma), then scaled by
// log2 e for the hardware base-2 exponential: the gap between z_j and m
// survives at any magnitude (a fused z log2 e - m log2 e would carry the
// rounding error of m log2 e, which is huge for |m| ~ 1e36). Pairs of
// elements go through packed f32x2 arithmetic.
struct OnlineState {
    float m;  // running max (never NaN: fmaxf drops NaN operands)
    float s;  // sum of exp(z - m)
    float t;  // sum of (z - m)
    int k;    // elements seen
    float av; // argmax value (NaN beats everything; first NaN wins)
    int ai;   // argmax index, -1 = empty
};

__device__ __forceinline__ OnlineState empty_state() {
    OnlineState st;
    st.m = -INFINITY;
    st.s = 0.f;
    st.t = 0.f;
    st.k = 0;
    st.av = -INFINITY;
    st.ai = -1;
    return st;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// True when candidate (bv, bi) should replace (av, ai) as the argmax: a NaN
// beats any number, a larger value wins, and equal values (or two NaNs) go to
// the lower index.
__device__ __forceinline__ bool argmax_better(float bv, int bi, float av, int ai) {
    if (bi < 0) return false;
    if (ai < 0) return true;
    const bool bn = bv != bv, an = av != av;
    if (bn != an) return bn;
    if (!bn && bv != av) return bv > av;
    return bi < ai;
}

// Rescale the state to a new max mn >= st.m (st.m = -inf gives factor 0).
// Without WITH_T the state carries only (m, s): t and k are left untouched.
template <bool WITH_T = true>
__device__ __forceinline__ void rescale_to(OnlineState& st, float mn) {
    if (st.m != mn) {
        st.s *= ex2((st.m - mn) * kLog2e);
        if constexpr (WITH_T) {
            if (st.k != 0) st.t += (float)st.k * (st.m - mn);
        }
        st.m = mn;
    }
}

// Adds exp(x - ms) and (x - ms) for an even number n of values, two at a
// time in packed f32x2 arithmetic.
template <int n>
__device__ __forceinline__ void accumulate2(const float* x, float ms, float2& sa, float2& ta) {
    static_assert(n % 2 == 0, "pairs");
    const float2 l2 = make_float2(kLog2e, kLog2e);
    const float2 nm = make_float2(-ms, -ms);
#pragma unroll
    for (int i = 0; i < n; i += 2) {
        const float2 d = __fadd2_rn(make_float2(x[i], x[i + 1]), nm);
        const float2 d2 = __fmul2_rn(d, l2);
        sa = __fadd2_rn(sa, make_float2(ex2(d2.x), ex2(d2.y)));
        ta = __fadd2_rn(ta, d);
    }
}

// Folds n values (all valid) into the state: one max, one rescale, then one
// exponential per element. Columns are col0 + i*dcol (used for argmax only).
template <int n, bool ARGMAX>
__device__ __forceinline__ void fold(OnlineState& st, const float* v, int col0, int dcol) {
    float cm = v[0];
#pragma unroll
    for (int i = 1; i < n; ++i) cm = fmaxf(cm, v[i]);
    rescale_to(st, fmaxf(st.m, cm));
    const float ms = (st.m == -INFINITY) ? 0.f : st.m;
    if constexpr (n % 2 == 0) {
        float2 sa = make_float2(0.f, 0.f), ta = make_float2(0.f, 0.f);
        accumulate2<n>(v, ms, sa, ta);
        st.s += sa.x + sa.y;
        st.t += ta.x + ta.y;
    } else {
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float d = v[i] - ms;
            st.s += ex2(d * kLog2e);
            st.t += d;
        }
    }
    st.k += n;
    if constexpr (ARGMAX) {
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float x = v[i];
            const bool take = (st.ai < 0) | (x > st.av) | ((x != x) & (st.av == st.av));
            if (take) {
                st.av = x;
                st.ai = col0 + i * dcol;
            }
        }
    }
}

// Folds U vectors of VEC values, of which only those with ok[u] set are
// valid (MASKED) or all (not MASKED): one max, one rescale, one exponential
// per valid element.
template <int U, int VEC, bool MASKED>
__device__ __forceinline__ void fold_vecs(OnlineState& st, const float (&v)[U][VEC],
                                          const bool (&ok)[U]) {
    // max as a shallow tree: one partial per vector, then across vectors
    float pm[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        pm[u] = -INFINITY;
        if (MASKED && !ok[u]) continue;
        if constexpr (VEC == 8) {
            pm[u] = fmaxf(fmax3(v[u][0], v[u][1], v[u][2]),
                          fmax3(v[u][3], v[u][4], fmax3(v[u][5], v[u][6], v[u][7])));
        } else if constexpr (VEC == 4) {
            pm[u] = fmax3(v[u][0], v[u][1], fmaxf(v[u][2], v[u][3]));
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) pm[u] = fmaxf(pm[u], v[u][e]);
        }
    }
#pragma unroll
    for (int w = U; w > 1; w = (w + 2) / 3) {
#pragma unroll
        for (int i = 0; i < (w + 2) / 3; ++i) {
            const float a = pm[3 * i];
            const float b = 3 * i + 1 < w ? pm[3 * i + 1] : -INFINITY;
            const float c = 3 * i + 2 < w ? pm[3 * i + 2] : -INFINITY;
            pm[i] = fmax3(a, b, c);
        }
    }
    rescale_to(st, fmaxf(st.m, pm[0]));
    const float ms = (st.m == -INFINITY) ? 0.f : st.m;
    int n = 0;
    if constexpr (VEC % 2 == 0) {
        // one partial pair per vector, then a sum over vectors: short
        // dependency chains for the adds
        float2 sa = make_float2(0.f, 0.f), ta = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (MASKED && !ok[u]) continue;
            float2 su = make_float2(0.f, 0.f), tu = make_float2(0.f, 0.f);
            accumulate2<VEC>(v[u], ms, su, tu);
            sa = __fadd2_rn(sa, su);
            ta = __fadd2_rn(ta, tu);
            n += VEC;
        }
        st.s += sa.x + sa.y;
        st.t += ta.x + ta.y;
    } else {
        float sa = 0.f, ta = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (MASKED && !ok[u]) continue;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float d = v[u][e] - ms;
                sa += ex2(d * kLog2e);
                ta += d;
            }
            n += VEC;
        }
        st.s += sa;
        st.t += ta;
    }
    st.k += n;
}

// ---- 16-bit rows folded from their raw words -----------------------------------
// The max is taken with packed 16-bit max instructions on the stored words
// (exact: every 16-bit value is a float), and the words are widened to float
// pairs only when their exponentials are formed, so a lane holds its 16-bit
// data in half the registers. Packed 16-bit max returns the number when one
// operand is NaN, like fmaxf; the NaN still reaches the sum.
template <typename T> struct Raw16;
template <> struct Raw16<__nv_bfloat16> {
    static constexpr uint32_t kNegInf2 = 0xff80ff80u;
    static __device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) {
        __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a),
                                   *reinterpret_cast<__nv_bfloat162*>(&b));
        return *reinterpret_cast<uint32_t*>(&r);
    }
    static __device__ __forceinline__ float2 widen(uint32_t w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
};
template <> struct Raw16<__half> {
    static constexpr uint32_t kNegInf2 = 0xfc00fc00u;
    static __device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) {
        __half2 r = __hmax2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
        return *reinterpret_cast<uint32_t*>(&r);
    }
    static __device__ __forceinline__ float2 widen(uint32_t w) {
        return __half22float2(*reinterpret_cast<__half2*>(&w));
    }
};

// Folds U 16-byte words of 8 16-bit values (valid where ok[u], or all when
// not MASKED). WITH_T = false skips sum (z - m), which only label smoothing
// reads.
template <typename T, int U, bool MASKED, bool WITH_T>
__device__ __forceinline__ void fold_raw16(OnlineState& st, const uint4 (&w)[U],
                                           const bool (&ok)[U]) {
    using R = Raw16<T>;
    uint32_t mx = R::kNegInf2;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (MASKED && !ok[u]) continue;
        mx = R::max2(mx, R::max2(R::max2(w[u].x, w[u].y), R::max2(w[u].z, w[u].w)));
    }
    const float2 m2 = R::widen(mx);
    rescale_to<WITH_T>(st, fmaxf(st.m, fmaxf(m2.x, m2.y)));
    const float ms = (st.m == -INFINITY) ? 0.f : st.m;
    const float2 l2 = make_float2(kLog2e, kLog2e);
    const float2 nm = make_float2(-ms, -ms);
    float2 sa = make_float2(0.f, 0.f), ta = make_float2(0.f, 0.f);
    int n = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (MASKED && !ok[u]) continue;
        const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        float2 su = make_float2(0.f, 0.f), tu = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 d = __fadd2_rn(R::widen(ws[k]), nm);
            const float2 d2 = __fmul2_rn(d, l2);
            su = __fadd2_rn(su, make_float2(ex2(d2.x), ex2(d2.y)));
            if constexpr (WITH_T) tu = __fadd2_rn(tu, d);
        }
        sa = __fadd2_rn(sa, su);
        if constexpr (WITH_T) ta = __fadd2_rn(ta, tu);
        n += 8;
    }
    st.s += sa.x + sa.y;
    if constexpr (WITH_T) {
        st.t += ta.x + ta.y;
        st.k += n;
    }
}

// ---- folding against a fixed reference ------------------------------------------
// Once a lane's state has a finite running max m (its first part folded the
// exact way), later parts need neither their max nor a rescale: any
// reference point gives the same log-sum-exp, lse = m + log sum_j exp(z_j - m),
// as long as no term overflows. Each element then costs one fused
// multiply-add for its exponent,
//     a_j = z_j log2 e - mL,   mL = m log2 e rounded to float,
// and one base-2 exponential. The product m log2 e is not exact: with the
// exact residual r = m log2 e - mL (an fma recovers it), z_j log2 e - mL =
// (z_j - m) log2 e + r, so the part's sum carries the common factor 2^r,
// removed once per part by c = 2^-r. The reference is used only while
// |m| <= 2^23, where |r| <= 1/2 and the single rounding of a_j costs no more
// than the two roundings of (z_j - m) log2 e. A part whose sum exceeds 2^100
// (a term far above the reference) or is not a number is refused, and the
// caller folds it the exact way, which rescales the state to the part's max.
struct FoldRef {
    float mL;  // m log2 e rounded to float
    float c;   // 2^-(m log2 e - mL)
    bool ok;   // the reference may be used
};

__device__ __forceinline__ FoldRef fold_ref(const OnlineState& st) {
    FoldRef f;
    f.ok = fabsf(st.m) <= 8388608.f;  // false for an infinite or NaN max
    f.mL = f.ok ? st.m * kLog2e : 0.f;
    f.c = f.ok ? ex2(-fmaf(st.m, kLog2e, -f.mL)) : 1.f;
    return f;
}

// Folds U 16-byte words of 8 16-bit values (all valid) into (m, s) against the
// reference f. Returns false, leaving the state unchanged, when the part must
// be folded the exact way instead. t and k are not kept (no label smoothing).
template <typename T, int U>
__device__ __forceinline__ bool fold_raw16_ref(OnlineState& st, const uint4 (&w)[U],
                                               const FoldRef& f) {
    using R = Raw16<T>;
    const float2 l2 = make_float2(kLog2e, kLog2e);
    const float2 nmL = make_float2(-f.mL, -f.mL);
    float2 sa = make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        float2 su = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 a = __ffma2_rn(R::widen(ws[k]), l2, nmL);
            su = __fadd2_rn(su, make_float2(ex2(a.x), ex2(a.y)));
        }
        sa = __fadd2_rn(sa, su);
    }
    const float sp = sa.x + sa.y;
    if (!(sp <= 1.2676506e30f)) return false;  // 2^100; NaN fails too
    st.s = fmaf(sp, f.c, st.s);
    return true;
}

// A whole row of NV 16-byte words (n = NV * VEC values, all valid) folded in
// one piece: its max first, then the sum of exponentials, with no running
// state to rescale. The sums go per vector, then across vectors: the order
// of fold_vecs, so kernels that fold the same row either way get the same
// bits. The values are returned in x.
template <typename T, int VEC, int NV, bool ARGMAX, bool WITH_T>
__device__ __forceinline__ OnlineState fold_whole_row(const uint4 (&w)[NV], float (&x)[NV * VEC]) {
    constexpr int n = NV * VEC;
#pragma unroll
    for (int v = 0; v < NV; ++v) unpack_words<T>(w[v], x + v * VEC);
    float m = fmaxf(x[0], x[1]);
#pragma unroll
    for (int i = 2; i + 1 < n; i += 2) m = fmax3(m, x[i], x[i + 1]);
    OnlineState st = empty_state();
    st.m = m;
    const float ms = m == -INFINITY ? 0.f : m;
    const float2 nm = make_float2(-ms, -ms), l2 = make_float2(kLog2e, kLog2e);
    float2 sa = make_float2(0.f, 0.f), ta = make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
        float2 su = make_float2(0.f, 0.f), tu = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = v * VEC; i < (v + 1) * VEC; i += 2) {
            const float2 d = __fadd2_rn(make_float2(x[i], x[i + 1]), nm);
            const float2 d2 = __fmul2_rn(d, l2);
            su = __fadd2_rn(su, make_float2(ex2(d2.x), ex2(d2.y)));
            if constexpr (WITH_T) tu = __fadd2_rn(tu, d);
        }
        sa = __fadd2_rn(sa, su);
        if constexpr (WITH_T) ta = __fadd2_rn(ta, tu);
    }
    st.s = sa.x + sa.y;
    st.t = ta.x + ta.y;
    st.k = n;
    if constexpr (ARGMAX) {
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float xi = x[i];
            if ((st.ai < 0) | (xi > st.av) | ((xi != xi) & (st.av == st.av))) {
                st.av = xi;
                st.ai = i;
            }
        }
    }
    return st;
}

// x[idx] for a power-of-two n by a tree of selects on the bits of idx (no
// indexed register access).
template <int n>
__device__ __forceinline__ float select_tree(const float (&x)[n], int idx) {
    static_assert((n & (n - 1)) == 0, "power of two");
    float v[n];
#pragma unroll
    for (int i = 0; i < n; ++i) v[i] = x[i];
#pragma unroll
    for (int w = n / 2, b = 1; w >= 1; w >>= 1, b <<= 1) {
        const bool hi = (idx & b) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) v[i] = hi ? v[2 * i + 1] : v[2 * i];
    }
    return v[0];
}

// Argmax over U vectors whose first columns are col0[u], in increasing
// column order per thread (a strict comparison keeps the first of equals).
template <int U, int VEC, bool MASKED>
__device__ __forceinline__ void argmax_vecs(OnlineState& st, const float (&v)[U][VEC],
                                            const bool (&ok)[U], const int (&col0)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (MASKED && !ok[u]) continue;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const float x = v[u][e];
            const bool take = (st.ai < 0) | (x > st.av) | ((x != x) & (st.av == st.av));
            if (take) {
                st.av = x;
                st.ai = col0[u] + e;
            }
        }
    }
}

template <bool ARGMAX>
__device__ __forceinline__ void merge(OnlineState& a, const OnlineState& b) {
    const float M = fmaxf(a.m, b.m);
    const float fa = (a.m == M) ? 1.f : ex2((a.m - M) * kLog2e);
    const float fb = (b.m == M) ? 1.f : ex2((b.m - M) * kLog2e);
    const float ta = (a.k == 0 || a.m == M) ? 0.f : (float)a.k * (a.m - M);
    const float tb = (b.k == 0 || b.m == M) ? 0.f : (float)b.k * (b.m - M);
    a.s = a.s * fa + b.s * fb;
    a.t = (a.t + ta) + (b.t + tb);
    a.k += b.k;
    a.m = M;
    if constexpr (ARGMAX) {
        if (argmax_better(b.av, b.ai, a.av, a.ai)) {
            a.av = b.av;
            a.ai = b.ai;
        }
    }
}

template <bool ARGMAX>
__device__ __forceinline__ OnlineState shfl_xor_state(const OnlineState& st, int off) {
    OnlineState o;
    o.m = __shfl_xor_sync(0xffffffffu, st.m, off);
    o.s = __shfl_xor_sync(0xffffffffu, st.s, off);
    o.t = __shfl_xor_sync(0xffffffffu, st.t, off);
    o.k = __shfl_xor_sync(0xffffffffu, st.k, off);
    if constexpr (ARGMAX) {
        o.av = __shfl_xor_sync(0xffffffffu, st.av, off);
        o.ai = __shfl_xor_sync(0xffffffffu, st.ai, off);
    } else {
        o.av = 0.f;
        o.ai = -1;
    }
    return o;
}

// Reduction over groups of G lanes (G a power of two <= 32). Every lane of
// the warp must call it. Addition and multiplication commute exactly, so
// every lane of a group ends with the same bits.
//
// With argmax, states are merged pairwise along a butterfly. Without, the
// group takes its max first, every lane rescales its own (s, t) to it once,
// and the rescaled terms are summed along the butterfly: the same merge
// operator, with one exponential per lane instead of two per round. WITH_T =
// false reduces (m, s) only (t and k are left as they are); WITH_K = false
// leaves the count k unreduced, for a last merge whose caller reads only t.
template <int G, bool ARGMAX, bool WITH_T = true, bool WITH_K = true>
__device__ __forceinline__ void group_reduce(OnlineState& st) {
    if constexpr (ARGMAX) {
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
            OnlineState o = shfl_xor_state<ARGMAX>(st, off);
            merge<ARGMAX>(st, o);
        }
    } else if constexpr (G > 1) {
        float M = st.m;
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float s = st.s, t = st.t;
        int k = st.k;
        if (st.m != M) {
            s *= ex2((st.m - M) * kLog2e);
            if constexpr (WITH_T) {
                if (k != 0) t += (float)k * (st.m - M);
            }
        }
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
            s += __shfl_xor_sync(0xffffffffu, s, off);
            if constexpr (WITH_T) {
                t += __shfl_xor_sync(0xffffffffu, t, off);
                if constexpr (WITH_K) k += __shfl_xor_sync(0xffffffffu, k, off);
            }
        }
        st.m = M;
        st.s = s;
        if constexpr (WITH_T) {
            st.t = t;
            st.k = k;
        }
    }
}

// ---------------------------------------------------------------------------
// Targets.
__device__ __forceinline__ int64_t load_target(const void* y, int tdt, int64_t off) {
    return tdt == 0 ? (int64_t)(reinterpret_cast<const int32_t*>(y)[off])
                    : reinterpret_cast<const int64_t*>(y)[off];
}

// ---------------------------------------------------------------------------
// Finalisation of one row from its complete state, with L = log s (hardware
// base-2 logarithm times ln 2):
//   lse  = m + L, written as a float pair (hi, lo) with hi + lo = m + L to
//          about 48 bits (two-sum of m and L);
//   loss = L - (1-eps)(z_y - m) - eps t/V   (t = sum_j (z_j - m))
// ignore_index rows: loss 0. Out-of-range targets: loss NaN and error bit 1.
struct RowOut {
    float* loss;
    float* lse;
    float* lse_lo;
    int32_t* argmax;
    unsigned int* err;
};

// L = log sum_j exp(z_j - m) and the float pair (hi, lo) of m + L. Explicit
// round-to-nearest operations (never contracted into fmas), so every kernel
// that derives the pair from the same state gets the same bits.
__device__ __forceinline__ void lse_pair(const OnlineState& st, float& L, float& hi, float& lo) {
    L = __fmul_rn(lg2(st.s), kLn2);
    hi = __fadd_rn(st.m, L);
    lo = 0.f;
    if (isfinite(hi)) {
        const float bv = __fsub_rn(hi, st.m);
        const float av = __fsub_rn(hi, bv);
        lo = __fadd_rn(__fsub_rn(st.m, av), __fsub_rn(L, bv));
    }
}

__device__ __forceinline__ void finalize_row(const OnlineState& st, float zy, int64_t y,
                                             int64_t ignore, int64_t V, float eps,
                                             const RowOut& o, int64_t r, bool write_argmax) {
    float L, hi, lo;
    lse_pair(st, L, hi, lo);
    o.lse[r] = hi;
    if (o.lse_lo) o.lse_lo[r] = lo;
    float loss;
    if (y == ignore) {
        loss = 0.f;
    } else if (y < 0 || y >= V) {
        loss = __int_as_float(0x7fc00000);
        atomicOr(o.err, 1u);
    } else {
        loss = L - (1.f - eps) * (zy - st.m);
        // t / V as t times 1/V: a kernel's rows share the reciprocal
        if (eps != 0.f) loss -= eps * (st.t * (1.0f / (float)V));
    }
    o.loss[r] = loss;
    if (write_argmax) o.argmax[r] = st.ai < 0 ? 0 : st.ai;
}

}  // namespace ceb
