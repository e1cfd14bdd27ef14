// Row cross-entropy forward kernels for sm_100a.
//
// Two shapes of work, both HBM-bound streams over the logits:
//  * packed rows (short rows, V * elem <= 4 KB): a group of G lanes owns one
//    row, several rows per warp; each lane folds its slice into an online
//    (m, s, t, k) state and the group merges with lane shuffles;
//  * CTA rows (long rows): one CTA folds one row, or one vocabulary split of
//    a row, with 16-byte streaming loads, merges its warps through a single
//    shared-memory exchange, and either finalises the row or writes a partial
//    state that a second launch merges in a fixed order.
// Both walk their work in grid-stride loops over 64-bit row (unit) indices,
// so the grid never has to cover N (MLX PR #4776: rows beyond a truncated
// grid were silently skipped).
//
// The loss is assembled from max-shifted values (MLX PR #4188, "Shift by the
// max in cross_entropy"); the running state is the online log-sum-exp of
// Ineshin, "A fused linear cross-entropy forward kernel for Apple GPUs", §1.
#include "ce_device.cuh"
#include "ce_launch.h"

namespace ceb {

// ---------------------------------------------------------------------------
// Packed rows: G lanes per row, U vectors of VEC elements per lane per step.
template <typename T, int VEC, int G, int U, bool ARGMAX>
__global__ void __launch_bounds__(256) k_fwd_packed(FwdArgs a) {
    const T* __restrict__ z = reinterpret_cast<const T*>(a.z);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerWarp = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};

    for (int64_t base = warp * kRowsPerWarp; base < a.N; base += nwarps * kRowsPerWarp) {
        const int64_t r = base + lane / G;
        const bool active = r < a.N;
        OnlineState st = empty_state();
        int64_t y = 0;
        const T* row = z;
        if (active) {
            row = z + row_offset(a.lz, r, a.N);
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            for (int64_t vb = 0; vb < nvec; vb += (int64_t)G * U) {
                float v[U][VEC];
                bool ok[U];
                int c0[U];
                const bool full = vb + (int64_t)G * U <= nvec;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t vi = vb + u * G + gl;
                    ok[u] = full || vi < nvec;
                    c0[u] = (int)(vi * VEC);
                    if (ok[u]) load_vec<T, VEC>(row, vi * VEC, a.lz.s_col, v[u]);
                }
                if (full) {
                    fold_vecs<U, VEC, false>(st, v, ok);
                    if constexpr (ARGMAX) argmax_vecs<U, VEC, false>(st, v, ok, c0);
                } else {
                    fold_vecs<U, VEC, true>(st, v, ok);
                    if constexpr (ARGMAX) argmax_vecs<U, VEC, true>(st, v, ok, c0);
                }
            }
            // ragged tail: the last V % VEC columns, one per lane
            for (int q = gl; q < tail; q += G) {
                float x;
                load_vec<T, 1>(row, nvec * VEC + q, 1, &x);
                fold<1, ARGMAX>(st, &x, (int)(nvec * VEC + q), 0);
            }
        }
        group_reduce<G, ARGMAX>(st);
        if (active && gl == 0) {
            float zy = 0.f;
            if (y != a.ignore && y >= 0 && y < a.V) zy = to_f32(row[y * a.lz.s_col]);
            finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);
        }
    }
}

// ---------------------------------------------------------------------------
// CTA rows. Unit u = (row, split) with split-major order inside a row.
constexpr int kCtaThreads = 512;
constexpr int kCtaMinBlocks = 2;
constexpr int kCtaWarps = kCtaThreads / 32;

template <typename T, int VEC, int U, bool ARGMAX>
__global__ void __launch_bounds__(kCtaThreads, kCtaMinBlocks) k_fwd_cta(FwdArgs a) {
    // One exchange of warp states per unit. The slots alternate between two
    // buffers on successive units, so a warp that races ahead into the next
    // unit never overwrites a slot warp 0 may still be reading: between two
    // writes of the same buffer every thread has passed the barrier of the
    // unit in between (the slot-reuse race of "One barrier short" cannot occur).
    __shared__ OnlineState slots[2][kCtaWarps];
    const T* __restrict__ z = reinterpret_cast<const T*>(a.z);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const int64_t units = a.N * a.splits;
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    int parity = 0;

    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, parity ^= 1) {
        const int64_t r = a.splits == 1 ? u : u / a.splits;
        const int sp = a.splits == 1 ? 0 : (int)(u - r * a.splits);
        const T* row = z + row_offset(a.lz, r, a.N);
        const int64_t v0 = (int64_t)sp * a.vec_per_split;
        const int64_t v1 = min(nvec, v0 + a.vec_per_split);
        // the finalising thread fetches the target and its logit up front
        int64_t y = 0;
        float zy = 0.f;
        if (a.splits == 1 && tid == 0) {
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            if (y != a.ignore && y >= 0 && y < a.V) zy = to_f32(row[y * a.lz.s_col]);
        }

        OnlineState st = empty_state();
        // every step issues U 16-byte loads per thread before using any of
        // them; only the last step of a unit needs predicates
        for (int64_t vb = v0; vb < v1; vb += (int64_t)kCtaThreads * U) {
            float v[U][VEC];
            bool ok[U];
            int c0[U];
            const bool full = vb + (int64_t)kCtaThreads * U <= v1;
#pragma unroll
            for (int q = 0; q < U; ++q) {
                const int64_t vi = vb + q * kCtaThreads + tid;
                ok[q] = full || vi < v1;
                c0[q] = (int)(vi * VEC);
                if (ok[q]) load_vec<T, VEC>(row, vi * VEC, a.lz.s_col, v[q]);
            }
            if (full) {
                fold_vecs<U, VEC, false>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, false>(st, v, ok, c0);
            } else {
                fold_vecs<U, VEC, true>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, true>(st, v, ok, c0);
            }
        }
        if (sp == a.splits - 1) {
            for (int q = tid; q < tail; q += kCtaThreads) {
                float x;
                load_vec<T, 1>(row, nvec * VEC + q, 1, &x);
                fold<1, ARGMAX>(st, &x, (int)(nvec * VEC + q), 0);
            }
        }

        group_reduce<32, ARGMAX>(st);
        if (lane == 0) slots[parity][wid] = st;
        __syncthreads();
        if (wid == 0) {
            st = lane < kCtaWarps ? slots[parity][lane] : empty_state();
            group_reduce<32, ARGMAX>(st);
            if (lane == 0) {
                if (a.splits == 1) {
                    finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);
                } else {
                    float4 rec;
                    rec.x = st.m;
                    rec.y = st.s;
                    rec.z = st.t;
                    const unsigned nanbit = (ARGMAX && st.av != st.av) ? 0x80000000u : 0u;
                    rec.w = __uint_as_float((unsigned)max(st.ai, 0) | nanbit);
                    a.part[(int64_t)sp * a.N + r] = rec;
                }
            }
        }
    }
}

// Merge of split partials, in split order, one thread per row.
template <typename T, bool ARGMAX>
__global__ void __launch_bounds__(256) k_fwd_merge(FwdArgs a) {
    const T* z = reinterpret_cast<const T*>(a.z);
    const int64_t nvec = a.V / ElemTraits<T>::kVec;
    const int vec = a.vec_is_scalar ? 1 : ElemTraits<T>::kVec;
    const int64_t nv = a.vec_is_scalar ? a.V : nvec;
    const int tail = a.vec_is_scalar ? 0 : (int)(a.V - nvec * vec);
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < a.N;
         r += (int64_t)gridDim.x * blockDim.x) {
        const int64_t y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
        const T* row = z + row_offset(a.lz, r, a.N);
        float zy = 0.f;
        if (y != a.ignore && y >= 0 && y < a.V) zy = to_f32(row[y * a.lz.s_col]);
        OnlineState st = empty_state();
        for (int sp = 0; sp < a.splits; ++sp) {
            const float4 rec = a.part[(int64_t)sp * a.N + r];
            const int64_t v0 = (int64_t)sp * a.vec_per_split;
            const int64_t v1 = min(nv, v0 + a.vec_per_split);
            OnlineState o;
            o.m = rec.x;
            o.s = rec.y;
            o.t = rec.z;
            o.k = (int)((v1 > v0 ? v1 - v0 : 0) * vec) + (sp == a.splits - 1 ? tail : 0);
            const unsigned w = __float_as_uint(rec.w);
            o.ai = (int)(w & 0x7fffffffu);
            o.av = (w & 0x80000000u) ? __int_as_float(0x7fc00000) : rec.x;
            if (o.k == 0) o.ai = -1;
            merge<ARGMAX>(st, o);
        }
        finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers.

template <typename T, int VEC, bool ARGMAX>
static cudaError_t launch_packed(const FwdArgs& a, int G, int U, int grid, cudaStream_t s) {
#define CEB_PACKED(GG, UU)                                                        \
    if (G == GG && U == UU) {                                                     \
        k_fwd_packed<T, VEC, GG, UU, ARGMAX><<<grid, 256, 0, s>>>(a);             \
        return cudaGetLastError();                                                \
    }
    CEB_PACKED(1, 2)
    CEB_PACKED(1, 8)
    CEB_PACKED(2, 8)
    CEB_PACKED(4, 8)
    CEB_PACKED(8, 8)
    CEB_PACKED(16, 8)
    CEB_PACKED(32, 8)
#undef CEB_PACKED
    return cudaErrorInvalidValue;
}

template <typename T, bool ARGMAX>
static cudaError_t launch_fwd_t(const FwdPlan& p, const FwdArgs& a, cudaStream_t s) {
    constexpr int V8 = ElemTraits<T>::kVec;
    if (p.kind == FwdPlan::kPacked) {
        return p.vec == 1 ? launch_packed<T, 1, ARGMAX>(a, p.G, p.U, p.grid, s)
                          : launch_packed<T, V8, ARGMAX>(a, p.G, p.U, p.grid, s);
    }
    if (p.vec == 1)
        k_fwd_cta<T, 1, 8, ARGMAX><<<p.grid, kCtaThreads, 0, s>>>(a);
    else
        k_fwd_cta<T, V8, 4, ARGMAX><<<p.grid, kCtaThreads, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.splits == 1) return e;
    k_fwd_merge<T, ARGMAX><<<p.merge_grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_forward(const FwdPlan& p, const FwdArgs& a, int dtype, cudaStream_t s) {
    const bool am = a.argmax != nullptr;
    switch (dtype) {
        case 0: return am ? launch_fwd_t<float, true>(p, a, s) : launch_fwd_t<float, false>(p, a, s);
        case 1:
            return am ? launch_fwd_t<__nv_bfloat16, true>(p, a, s)
                      : launch_fwd_t<__nv_bfloat16, false>(p, a, s);
        case 2: return am ? launch_fwd_t<__half, true>(p, a, s) : launch_fwd_t<__half, false>(p, a, s);
    }
    return cudaErrorInvalidValue;
}

int cta_threads_forward() { return kCtaThreads; }

}  // namespace ceb
