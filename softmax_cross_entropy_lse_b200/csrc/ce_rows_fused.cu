// Fused forward + VJP for short rows: one read of the logits, one write of
// the gradient.
//
// When the upstream gradient g is known before the forward runs (a mean or a
// sum of the per-row losses, the usual training case), the VJP needs nothing
// the forward has not just computed: a group of lanes holds the whole row in
// registers, folds it into the online (max, scaled sum) state of Ineshin, "A
// fused linear cross-entropy forward kernel for Apple GPUs", section 1,
// reduces, writes loss/lse, and turns the same registers into
//     dz_j = g (exp(z_j - lse) - (1 - eps)[j = y] - eps/V)
// without reading the row again. HBM traffic drops from three passes over the
// logits (forward read, backward read and write) to two.
//
// Every lane of a group derives (hi, lo) from the identical reduced state
// with the same operations as the forward's finalisation, and the gradient
// uses the same formula as the stand-alone VJP: where the forward plan groups
// the lanes the same way (4-byte rows) loss, lse and argmax are bit-identical
// to ce_forward, and the gradient agrees with ce_backward to a few ulps.
#include "ce_device.cuh"
#include "ce_launch.h"

namespace ceb {

template <typename TI, typename TO, int VEC, int G, int U, bool ARGMAX, int MINB>
__global__ void __launch_bounds__(256, MINB) k_fwdbwd_rows(FusedArgs fa) {
    const FwdArgs& a = fa.f;
    const TI* __restrict__ z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(fa.dz);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const bool full = nvec == (int64_t)G * U;  // every lane's every vector is in the row
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    const float inv_v = 1.f / (float)a.V;
    const float nan = __int_as_float(0x7fc00000);

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        const bool act = r < a.N;
        const TI* row = z;
        TO* drow = dz;
        int64_t y = a.ignore;
        float g = 0.f;
        if (act) {
            row = z + row_offset(a.lz, r, a.N);
            drow = dz + row_offset(fa.ld, r, a.N);
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            g = fa.g[r * fa.g_stride];
        }
        // the whole row: one step of U vectors per lane (the plan guarantees it)
        float v[U][VEC];
        bool ok[U];
        int c0[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t vi = (int64_t)u * G + gl;
            ok[u] = act && vi < nvec;
            c0[u] = (int)(vi * VEC);
            if (ok[u]) load_vec_coherent<TI, VEC>(row, vi * VEC, a.lz.s_col, v[u]);
        }
        const int yc = (y >= 0 && y < a.V && y != a.ignore) ? (int)y : -1;
        OnlineState st = empty_state();
        float zy = 0.f;
        if (act) {
            if (full) {  // every vector valid: the unpredicated fold (same bits)
                fold_vecs<U, VEC, false>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, false>(st, v, ok, c0);
            } else {
                fold_vecs<U, VEC, true>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, true>(st, v, ok, c0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const unsigned dy = (unsigned)(yc - c0[u]);
                if (ok[u] && dy < (unsigned)VEC) {
#pragma unroll
                    for (int e = 0; e < VEC; ++e)
                        if ((unsigned)e == dy) zy = v[u][e];
                }
            }
            for (int q = gl; q < tail; q += G) {
                float x;
                const int col = (int)(nvec * VEC + q);
                load_vec_coherent<TI, 1>(row, col, 1, &x);
                fold<1, ARGMAX>(st, &x, col, 0);
                if (col == yc) zy = x;
            }
        }
        group_reduce<G, ARGMAX>(st);
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) zy += __shfl_xor_sync(0xffffffffu, zy, off);
        if (!act) continue;
        if (gl == 0) finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);

        // (hi, lo) exactly as finalize_row writes them
        float L, hi, lo;
        lse_pair(st, L, hi, lo);
        const bool zero = y == a.ignore;
        const bool bad = !zero && (y < 0 || y >= a.V);
        const float c_lo = lo * kLog2e, c_eps = g * a.eps * inv_v, c_tgt = g * (1.f - a.eps);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!ok[u]) continue;
            float o[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float p = ex2(fmaf(v[u][e] - hi, kLog2e, -c_lo));
                o[e] = (zero || bad) ? (bad ? nan : 0.f) : fmaf(g, p, -c_eps);
            }
            const unsigned dy = (unsigned)(yc - c0[u]);
            if (dy < (unsigned)VEC) {
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    if ((unsigned)e == dy) o[e] -= c_tgt;
            }
            store_vec<TO, VEC>(drow, c0[u], fa.ld.s_col, o);
        }
        for (int q = gl; q < tail; q += G) {
            const int64_t col = nvec * VEC + q;
            float d;
            if (zero || bad) {
                d = bad ? nan : 0.f;
            } else {
                float x;
                load_vec_coherent<TI, 1>(row, col, 1, &x);
                d = fmaf(g, ex2(fmaf(x - hi, kLog2e, -c_lo)), -c_eps);
                if (col == y) d -= c_tgt;
            }
            cvt_store1(drow + col, d);
        }
    }
}

// Tiny rows (one or two 16-byte vectors, no ragged tail): one lane per row
// and R rows per lane per step, every load of the step issued before any is
// used. The row is folded in one piece exactly as the tiny-row forward folds
// it (same bits for loss, lse and argmax), and the gradient comes from the
// same registers.
template <typename TI, typename TO, int NV, int R, bool ARGMAX, bool WITH_T, int MINB>
__global__ void __launch_bounds__(256, MINB) k_fwdbwd_tiny(FusedArgs fa) {
    constexpr int VEC = ElemTraits<TI>::kVec;
    constexpr int n = NV * VEC;
    const FwdArgs& a = fa.f;
    const TI* z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(fa.dz);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    const float inv_v = 1.f / (float)a.V;
    const float nan = __int_as_float(0x7fc00000);

    for (int64_t base = warp * 32 * R; base < a.N; base += nwarps * 32 * R) {
        uint4 w[R][NV];
        int64_t y[R];
        float g[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            y[k] = a.ignore;
            g[k] = 0.f;
            if (r < a.N) {
                const TI* row = z + row_offset(a.lz, r, a.N);
                y[k] = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
                g[k] = fa.g[r * fa.g_stride];
#pragma unroll
                for (int v = 0; v < NV; ++v) w[k][v] = __ldcs(reinterpret_cast<const uint4*>(row) + v);
            }
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            if (r >= a.N) continue;
            float x[n];
            const OnlineState st = fold_whole_row<TI, VEC, NV, ARGMAX, WITH_T>(w[k], x);
            const int64_t yk = y[k];
            finalize_row(st, select_tree<n>(x, (int)(yk & (n - 1))), yk, a.ignore, a.V, a.eps, out, r,
                         ARGMAX);
            float L, hi, lo;
            lse_pair(st, L, hi, lo);
            const bool zero = yk == a.ignore;
            const bool bad = !zero && (yk < 0 || yk >= a.V);
            const float gk = g[k];
            const float c_lo = lo * kLog2e, c_eps = gk * a.eps * inv_v, c_tgt = gk * (1.f - a.eps);
            float o[n];
#pragma unroll
            for (int i = 0; i < n; ++i) {
                const float p = ex2(fmaf(x[i] - hi, kLog2e, -c_lo));
                o[i] = (zero || bad) ? (bad ? nan : 0.f) : fmaf(gk, p, -c_eps);
            }
            if (!zero && !bad) {
#pragma unroll
                for (int i = 0; i < n; ++i)
                    if (i == yk) o[i] -= c_tgt;
            }
            TO* drow = dz + row_offset(fa.ld, r, a.N);
#pragma unroll
            for (int v = 0; v < NV; ++v) store_vec<TO, VEC>(drow, v * VEC, 1, o + v * VEC);
        }
    }
}

template <typename TI, typename TO, bool ARGMAX, bool WITH_T>
static cudaError_t launch_fused_tiny(const FusedPlan& p, const FusedArgs& a, cudaStream_t s) {
    // register budgets: 64 per thread, 80 for two 16-bit vectors per row
    if (p.U == 1)
        k_fwdbwd_tiny<TI, TO, 1, kTinyRows, ARGMAX, WITH_T, 4><<<p.grid, 256, 0, s>>>(a);
    else if constexpr (sizeof(TI) == 4)
        k_fwdbwd_tiny<TI, TO, 2, kTinyRows, ARGMAX, WITH_T, 4><<<p.grid, 256, 0, s>>>(a);
    else
        k_fwdbwd_tiny<TI, TO, 2, kTinyRows, ARGMAX, WITH_T, 3><<<p.grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename TI, typename TO, int VEC, bool ARGMAX>
static cudaError_t launch_fused_v(const FusedPlan& p, const FusedArgs& a, cudaStream_t s) {
    constexpr int kU = VEC == 1 ? 8 : 32 / VEC;
    constexpr int kMinB = sizeof(TI) == 4 ? 3 : 2;
#define CEB_FUSED(GG, UU, MB)                                                      \
    if (p.G == GG && p.U == UU) {                                                  \
        k_fwdbwd_rows<TI, TO, VEC, GG, UU, ARGMAX, MB><<<p.grid, 256, 0, s>>>(a);  \
        return cudaGetLastError();                                                 \
    }
    CEB_FUSED(1, 2, 4)
    CEB_FUSED(1, kU, kMinB)
    CEB_FUSED(2, kU, kMinB)
    CEB_FUSED(4, kU, kMinB)
    CEB_FUSED(8, kU, kMinB)
    CEB_FUSED(16, kU, kMinB)
    CEB_FUSED(32, kU, kMinB)
#undef CEB_FUSED
    return cudaErrorInvalidValue;
}

template <typename TI, typename TO>
static cudaError_t launch_fused_t(const FusedPlan& p, const FusedArgs& a, cudaStream_t s) {
    const bool am = a.f.argmax != nullptr;
    if (p.tiny) {
        const bool t = a.f.eps != 0.f;
        if (am)
            return t ? launch_fused_tiny<TI, TO, true, true>(p, a, s) : launch_fused_tiny<TI, TO, true, false>(p, a, s);
        return t ? launch_fused_tiny<TI, TO, false, true>(p, a, s) : launch_fused_tiny<TI, TO, false, false>(p, a, s);
    }
    if (p.vec == 1)
        return am ? launch_fused_v<TI, TO, 1, true>(p, a, s) : launch_fused_v<TI, TO, 1, false>(p, a, s);
    constexpr int V8 = ElemTraits<TI>::kVec;
    return am ? launch_fused_v<TI, TO, V8, true>(p, a, s) : launch_fused_v<TI, TO, V8, false>(p, a, s);
}

cudaError_t launch_fused(const FusedPlan& p, const FusedArgs& a, int dt_in, int dt_out,
                         cudaStream_t s) {
    if (dt_in == 0 && dt_out == 0) return launch_fused_t<float, float>(p, a, s);
    if (dt_in == 1 && dt_out == 1) return launch_fused_t<__nv_bfloat16, __nv_bfloat16>(p, a, s);
    if (dt_in == 1 && dt_out == 0) return launch_fused_t<__nv_bfloat16, float>(p, a, s);
    if (dt_in == 2 && dt_out == 2) return launch_fused_t<__half, __half>(p, a, s);
    if (dt_in == 2 && dt_out == 0) return launch_fused_t<__half, float>(p, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ceb
