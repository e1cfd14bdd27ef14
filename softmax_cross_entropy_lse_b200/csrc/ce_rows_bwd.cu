// Row cross-entropy VJP for sm_100a:
//     dz_ij = g_i (exp(z_ij - lse_i) - (1 - eps)[j = y_i] - eps/V)
// from the saved lse (MLX issue #4686 describes this VJP and the strided
// view x[:, :-1] it must handle without a hidden copy; Ineshin, "A fused
// linear cross-entropy forward kernel for Apple GPUs", section 1: the
// backward regenerates what it needs from the saved log-sum-exp).
//
// Elementwise given four per-row scalars, so the kernel is a pure HBM stream:
// one read and one write per element. Work units are (row, column chunk);
// a group of G lanes walks one unit with 16-byte loads and stores. Short rows
// are one unit handled by a group of a few lanes (several rows per warp);
// long rows are cut into chunks so that every SM has many units.
//
// exp(z - lse) is evaluated as exp((z - hi) - lo) from the float pair
// (hi, lo) the forward writes: z - hi is exact when z is near lse, which
// keeps the softmax right at magnitudes where float lse alone has lost the
// gap (equal logits at 1e8 give [-1/2, 1/2], as MLX PR #4188 requires).
//
// dlogits may be the logits buffer itself: every element is loaded by the
// thread that later stores it, and the loads are plain coherent loads.
#include "ce_device.cuh"
#include "ce_launch.h"

namespace ceb {

template <typename TI, typename TO, int VEC, int G, int U>
__global__ void __launch_bounds__(256) k_bwd(BwdArgs a) {
    const TI* z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    const int64_t group = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / G;
    const int64_t ngroups = ((int64_t)gridDim.x * blockDim.x) / G;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const int64_t units = a.N * a.nchunks;
    const float inv_v = 1.f / (float)a.V;

    for (int64_t u = group; u < units; u += ngroups) {
        const int64_t r = a.nchunks == 1 ? u : u / a.nchunks;
        const int64_t c = a.nchunks == 1 ? 0 : u - r * a.nchunks;
        const TI* row = z + row_offset(a.lz, r, a.N);
        TO* drow = dz + row_offset(a.ld, r, a.N);
        const int64_t y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
        const float g = a.g[r * a.g_stride];
        const float hi = a.lse[r];
        const float lo = a.lse_lo ? a.lse_lo[r] : 0.f;
        const int64_t v0 = c * a.vec_per_chunk;
        const int64_t v1 = min(nvec, v0 + a.vec_per_chunk);
        const bool last = c == a.nchunks - 1;

        if (y == a.ignore || y < 0 || y >= a.V) {
            // ignored row: zeros, without reading the logits; bad target: NaN
            const bool bad = y != a.ignore;
            if (bad && gl == 0 && c == 0) atomicOr(a.err, 1u);
            float fill[VEC];
#pragma unroll
            for (int q = 0; q < VEC; ++q) fill[q] = bad ? __int_as_float(0x7fc00000) : 0.f;
            for (int64_t vi = v0 + gl; vi < v1; vi += G) store_vec<TO, VEC>(drow, vi * VEC, a.ld.s_col, fill);
            if (last)
                for (int q = gl; q < tail; q += G) cvt_store1(drow + (nvec * VEC + q), fill[0]);
            continue;
        }

        // dz = g p - g eps/V - [j = y] g (1 - eps)
        const float c0 = g * a.eps * inv_v;
        const float c1 = g * (1.f - a.eps);
        for (int64_t vb = v0; vb < v1; vb += (int64_t)G * U) {
            float v[U][VEC];
            bool ok[U];
#pragma unroll
            for (int q = 0; q < U; ++q) {
                const int64_t vi = vb + q * G + gl;
                ok[q] = vi < v1;
                if (ok[q]) load_vec_coherent<TI, VEC>(row, vi * VEC, a.lz.s_col, v[q]);
            }
#pragma unroll
            for (int q = 0; q < U; ++q) {
                if (!ok[q]) continue;
                const int64_t col0 = (vb + q * G + gl) * VEC;
                float o[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float p = ex2(((v[q][e] - hi) - lo) * kLog2e);
                    float d = fmaf(g, p, -c0);
                    if (col0 + e == y) d -= c1;
                    o[e] = d;
                }
                store_vec<TO, VEC>(drow, col0, a.ld.s_col, o);
            }
        }
        if (last) {
            for (int q = gl; q < tail; q += G) {
                const int64_t col = nvec * VEC + q;
                float x;
                load_vec_coherent<TI, 1>(row, col, 1, &x);
                const float p = ex2(((x - hi) - lo) * kLog2e);
                float d = fmaf(g, p, -c0);
                if (col == y) d -= c1;
                cvt_store1(drow + col, d);
            }
        }
    }
}

template <typename TI, typename TO, int VEC>
static cudaError_t launch_bwd_v(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
#define CEB_BWD(GG, UU)                                                  \
    if (p.G == GG && p.U == UU) {                                        \
        k_bwd<TI, TO, VEC, GG, UU><<<p.grid, 256, 0, s>>>(a);            \
        return cudaGetLastError();                                       \
    }
    CEB_BWD(1, 2)
    CEB_BWD(1, 8)
    CEB_BWD(2, 8)
    CEB_BWD(4, 8)
    CEB_BWD(8, 8)
    CEB_BWD(16, 8)
    CEB_BWD(32, 8)
    CEB_BWD(32, 4)
#undef CEB_BWD
    return cudaErrorInvalidValue;
}

template <typename TI, typename TO>
static cudaError_t launch_bwd_t(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
    if (p.vec == 1) return launch_bwd_v<TI, TO, 1>(p, a, s);
    return launch_bwd_v<TI, TO, ElemTraits<TI>::kVec>(p, a, s);
}

cudaError_t launch_backward(const BwdPlan& p, const BwdArgs& a, int dt_in, int dt_out,
                            cudaStream_t s) {
    if (dt_in == 0 && dt_out == 0) return launch_bwd_t<float, float>(p, a, s);
    if (dt_in == 1 && dt_out == 1) return launch_bwd_t<__nv_bfloat16, __nv_bfloat16>(p, a, s);
    if (dt_in == 1 && dt_out == 0) return launch_bwd_t<__nv_bfloat16, float>(p, a, s);
    if (dt_in == 2 && dt_out == 2) return launch_bwd_t<__half, __half>(p, a, s);
    if (dt_in == 2 && dt_out == 0) return launch_bwd_t<__half, float>(p, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ceb
