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
#include "ce_sm100.cuh"

namespace ceb {

// ---------------------------------------------------------------------------
// Packed rows: G lanes per row, U vectors of VEC elements per lane per step,
// 32/G rows per warp. The group's first lane, which finalises the row, loads
// z_y itself as soon as the target is known; the load overlaps the fold, and
// the other lanes spend nothing on it.
template <typename T, int VEC, int G, int U, bool ARGMAX, int MINB>
__global__ void __launch_bounds__(256, MINB) k_fwd_packed(FwdArgs a) {
    const T* __restrict__ z = reinterpret_cast<const T*>(a.z);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        const bool active = r < a.N;
        OnlineState st = empty_state();
        int64_t y = a.ignore;
        const T* row = z;
        if (active) {
            row = z + row_offset(a.lz, r, a.N);
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
        }
        float zy = 0.f;
        if (active && gl == 0 && y >= 0 && y < a.V && y != a.ignore) zy = to_f32(row[y * a.lz.s_col]);
        for (int64_t vb = 0; vb < nvec; vb += (int64_t)G * U) {
            float v[U][VEC];
            bool ok[U];
            int c0[U];
            const bool full = vb + (int64_t)G * U <= nvec;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + u * G + gl;
                ok[u] = active && (full || vi < nvec);
                c0[u] = (int)(vi * VEC);
                if (ok[u]) load_vec<T, VEC>(row, vi * VEC, a.lz.s_col, v[u]);
            }
            if (active) {
                if (full) {
                    fold_vecs<U, VEC, false>(st, v, ok);
                    if constexpr (ARGMAX) argmax_vecs<U, VEC, false>(st, v, ok, c0);
                } else {
                    fold_vecs<U, VEC, true>(st, v, ok);
                    if constexpr (ARGMAX) argmax_vecs<U, VEC, true>(st, v, ok, c0);
                }
            }
        }
        // ragged tail: the last V % VEC columns, one per lane
        if (active) {
            for (int q = gl; q < tail; q += G) {
                float x;
                const int col = (int)(nvec * VEC + q);
                load_vec<T, 1>(row, col, 1, &x);
                fold<1, ARGMAX>(st, &x, col, 0);
            }
        }
        group_reduce<G, ARGMAX>(st);
        if (active && gl == 0) finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);
    }
}

// ---------------------------------------------------------------------------
// Packed rows that one step covers (nvec <= G U, whole 16-byte vectors, no
// tail), pipelined across row groups: while a warp folds its current group
// of 32/G rows, the next group's vectors are already streaming into its
// shared-memory slot (cp.async, two stages per warp). Each lane reads back
// only the slots it filled, so no barrier is needed and the slot layout
// [u][lane] is free of bank conflicts.
constexpr int kPipeWarps = 8;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(smem)),
                 "l"(reinterpret_cast<uint64_t>(gmem))
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int n>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory");
}

template <typename T, int VEC, int G, int U, bool ARGMAX, int MINB>
__global__ void __launch_bounds__(kPipeWarps * 32, MINB) k_fwd_packed_pipe(FwdArgs a) {
    extern __shared__ __align__(16) uint4 pipe_smem[];  // [2][kPipeWarps][U][32]
    const T* __restrict__ z = reinterpret_cast<const T*>(a.z);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t step = nwarps * kRowsPerStep;
    const int64_t nvec = a.V / VEC;
    const bool full = nvec == (int64_t)G * U;  // every lane's every slot holds a vector
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    auto slot = [&](int s, int u) { return pipe_smem + ((s * kPipeWarps + wid) * U + u) * 32 + lane; };
    auto issue = [&](int64_t base, int s) {
        const int64_t r = base + lane / G;
        if (r < a.N) {
            const T* row = z + row_offset(a.lz, r, a.N);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = u * G + gl;
                if (vi < nvec) cp_async16(slot(s, u), row + vi * VEC);
            }
        }
        cp_async_commit();  // one group per row group, empty or not
    };

    int s = 0;
    int64_t base = warp * kRowsPerStep;
    if (base < a.N) issue(base, 0);
    for (; base < a.N; base += step, s ^= 1) {
        issue(base + step, s ^ 1);
        const int64_t r = base + lane / G;
        const bool active = r < a.N;
        int64_t y = a.ignore;
        float zy = 0.f;
        if (active) {
            const T* row = z + row_offset(a.lz, r, a.N);
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            if (gl == 0 && y >= 0 && y < a.V && y != a.ignore) zy = to_f32(row[y * a.lz.s_col]);
        }
        cp_async_wait<1>();  // this row group's copies have landed
        OnlineState st = empty_state();
        if (active) {
            float v[U][VEC];
            bool ok[U];
            int c0[U];
            if (full) {
                // every slot holds a vector: no predicates in the fold (the same
                // operations in the same order as the masked fold, so the same bits)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    ok[u] = true;
                    c0[u] = (u * G + gl) * VEC;
                    unpack_words<T>(*slot(s, u), v[u]);
                }
                fold_vecs<U, VEC, false>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, false>(st, v, ok, c0);
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t vi = u * G + gl;
                    ok[u] = vi < nvec;
                    c0[u] = (int)(vi * VEC);
                    if (ok[u]) unpack_words<T>(*slot(s, u), v[u]);
                }
                fold_vecs<U, VEC, true>(st, v, ok);
                if constexpr (ARGMAX) argmax_vecs<U, VEC, true>(st, v, ok, c0);
            }
        }
        // the last merge of the row: finalize_row reads t, not the count
        group_reduce<G, ARGMAX, true, false>(st);
        if (active && gl == 0) finalize_row(st, zy, y, a.ignore, a.V, a.eps, out, r, ARGMAX);
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Tiny rows: one or two 16-byte vectors and no ragged tail (for instance 8
// floats). One lane per row and R rows per lane per step, with every load of
// the step issued before any is used. The whole row sits in registers, so it
// is folded in one piece: its max first (three-operand max instructions),
// then the sum of exponentials, with no running state to rescale. z_y is
// picked from the registers by a select tree on the bits of the target.
template <typename T, int VEC, int NV, int R, bool ARGMAX, bool WITH_T, int MINB>
__global__ void __launch_bounds__(256, MINB) k_fwd_tiny(FwdArgs a) {
    constexpr int n = NV * VEC;
    const T* __restrict__ z = reinterpret_cast<const T*>(a.z);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};

    // rows lie back to back in memory when the layout is a plain matrix
    const bool dense = a.lz.inner >= a.N && a.lz.s_inner == (int64_t)n;
    for (int64_t base = warp * 32 * R; base < a.N; base += nwarps * 32 * R) {
        uint4 w[R][NV];
        int64_t y[R];
        if (dense && lane == 0) {
            // the warp's next step (32 R rows) starts moving into L2 now
            const int64_t bn = base + nwarps * 32 * R;
            if (bn < a.N) {
                const int64_t rows = min((int64_t)32 * R, a.N - bn);
                sm100::bulk_prefetch_l2(z + bn * n, (uint32_t)(rows * n * sizeof(T)));
            }
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            y[k] = a.ignore;
            if (r < a.N) {
                const T* row = z + row_offset(a.lz, r, a.N);
                y[k] = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
#pragma unroll
                for (int v = 0; v < NV; ++v) w[k][v] = __ldcs(reinterpret_cast<const uint4*>(row) + v);
            }
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            if (r >= a.N) continue;
            float x[n];
            const OnlineState st = fold_whole_row<T, VEC, NV, ARGMAX, WITH_T>(w[k], x);
            const int64_t yk = y[k];
            const float zy = select_tree<n>(x, (int)(yk & (n - 1)));
            finalize_row(st, zy, yk, a.ignore, a.V, a.eps, out, r, ARGMAX);
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
            st = slots[parity][lane & (kCtaWarps - 1)];
            group_reduce<kCtaWarps, ARGMAX>(st);
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

// ---------------------------------------------------------------------------
// Long rows through per-warp bulk-copy rings. One CTA of kRingWarps warps
// folds one (row, split) unit, as in k_fwd_cta, but the row reaches shared
// memory through the tensor-memory-access engine: every warp owns a ring of
// kRingStages buffers of kRingVecs 16-byte vectors, its lane 0 keeps the ring
// full with 1-D bulk copies issued kRingStages chunks ahead (across unit
// boundaries), and the lanes fold each chunk straight from shared memory. The
// bytes in flight per SM are set by the rings (up to 192 KB), not by the
// registers of the folding threads. Four warps with 8 KB stages (three CTAs,
// twelve warps per SM) measured ahead of eight warps with 4 KB stages: the
// per-chunk wait, fence and refill and the per-unit exchange are paid over
// twice the elements, and each lane folds 64 values per part. Chunk c of a unit belongs to warp
// c % kRingWarps; the warps of a unit meet once, in one exchange of states:
// each warp writes its state to a slot and arrives on a named barrier without
// waiting, and only the unit's finaliser (a role that rotates over the warps)
// waits for all of them, merges and writes the row. Slots alternate between
// two sets; the finaliser releases its set through a second named barrier,
// which the other warps pass before they write that set again two units
// later (so no slot is rewritten before it is read: the race of "One barrier
// short" cannot occur), and the warps of a CTA stay within two units of each
// other, streaming neighbouring parts of the same rows.
constexpr int kRingWarps = 4;
constexpr int kRingStages = 2;
constexpr int kRingVecs = 512;  // 8 KB per stage
constexpr int kRingPart = 256;  // vectors folded at a time (8 per lane)
constexpr size_t kRingSmem = (size_t)kRingWarps * kRingStages * kRingVecs * 16;
static_assert((kRingStages & (kRingStages - 1)) == 0 && (kRingWarps & (kRingWarps - 1)) == 0,
              "stage and warp counts are powers of two");

struct RingUnit {
    const uint8_t* src;  // first byte of the unit's vectors
    int64_t v0, nv;      // first vector index in the row, vector count
    int nch;             // chunks
};

template <typename T>
__device__ __forceinline__ RingUnit ring_unit(const FwdArgs& a, int64_t u, int64_t nvec) {
    RingUnit ru;
    const int64_t r = a.splits == 1 ? u : u / a.splits;
    const int64_t sp = a.splits == 1 ? 0 : u - r * a.splits;
    ru.v0 = sp * a.vec_per_split;
    const int64_t v1 = min(nvec, ru.v0 + a.vec_per_split);
    ru.nv = v1 > ru.v0 ? v1 - ru.v0 : 0;
    ru.nch = (int)((ru.nv + kRingVecs - 1) / kRingVecs);
    ru.src = reinterpret_cast<const uint8_t*>(reinterpret_cast<const T*>(a.z) +
                                              row_offset(a.lz, r, a.N)) +
             ru.v0 * 16;
    return ru;
}

// The sequence of (unit, chunk) pairs one warp consumes, in order.
template <typename T>
struct RingCursor {
    int64_t u;
    int j;
    RingUnit ru;
    __device__ __forceinline__ void settle(const FwdArgs& a, int64_t units, int64_t nvec, int w) {
        while (u < units && j >= ru.nch) {
            u += gridDim.x;
            j = w;
            if (u < units) ru = ring_unit<T>(a, u, nvec);
        }
    }
    __device__ __forceinline__ void start(const FwdArgs& a, int64_t units, int64_t nvec, int w) {
        u = blockIdx.x;
        j = w;
        ru.nch = 0;
        if (u < units) ru = ring_unit<T>(a, u, nvec);
        settle(a, units, nvec, w);
    }
    __device__ __forceinline__ void next(const FwdArgs& a, int64_t units, int64_t nvec, int w) {
        j += kRingWarps;
        settle(a, units, nvec, w);
    }
    __device__ __forceinline__ bool valid(int64_t units) const { return u < units; }
    __device__ __forceinline__ uint32_t bytes() const {
        const int64_t left = ru.nv - (int64_t)j * kRingVecs;
        return (uint32_t)((left < kRingVecs ? left : kRingVecs) * 16);
    }
    __device__ __forceinline__ const uint8_t* src() const {
        return ru.src + (int64_t)j * kRingVecs * 16;
    }
};

template <typename T, bool ARGMAX, bool WITH_T>
__global__ void __launch_bounds__(kRingWarps * 32, 3) k_fwd_ring(FwdArgs a) {
    using namespace sm100;
    constexpr int VEC = ElemTraits<T>::kVec;
    constexpr int kPerLane = kRingPart / 32;
    extern __shared__ __align__(128) uint8_t ring_smem[];
    __shared__ __align__(8) uint64_t full_bar[kRingWarps][kRingStages];
    __shared__ OnlineState slots[2][kRingWarps];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const int64_t units = a.N * a.splits;
    const RowOut out{a.loss, a.lse, a.lse_lo, a.argmax, a.err};
    uint8_t* ring = ring_smem + (size_t)wid * kRingStages * kRingVecs * 16;

    if (lane == 0)
        for (int q = 0; q < kRingStages; ++q) mbar_init(smem_u32(&full_bar[wid][q]), 1);
    if (tid == 0) abort_flag = 0;
    if (lane == 0) mbar_fence_init();
    __syncthreads();

    // prologue: the first kRingStages chunks of this warp's sequence
    RingCursor<T> iss;
    iss.start(a, units, nvec, wid);
    // 32-bit counters: stage = count % kRingStages and parity = (count /
    // kRingStages) % 2 stay exact across wraparound (powers of two divide 2^32)
    uint32_t issued = 0;
    // (a starved launch, a testing mode, issues no copies: its waits run out)
    for (int q = 0; q < kRingStages && iss.valid(units); ++q) {
        if (!a.starve) {
            if (lane == 0) {
                const uint32_t bar = smem_u32(&full_bar[wid][q]);
                mbar_expect_tx(bar, iss.bytes());
                bulk_load(smem_u32(ring + q * kRingVecs * 16), iss.src(), iss.bytes(), bar);
            }
            ++issued;
        }
        iss.next(a, units, nvec, wid);
    }

    uint32_t consumed = 0, waited = 0;
    bool dead = false;
    int parity = 0;
    uint32_t it = 0;  // units of this CTA so far
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, parity ^= 1, ++it) {
        const RingUnit ru = ring_unit<T>(a, u, nvec);
        const int64_t r = a.splits == 1 ? u : u / a.splits;
        const int sp = a.splits == 1 ? 0 : (int)(u - r * a.splits);
        const T* row = reinterpret_cast<const T*>(a.z) + row_offset(a.lz, r, a.N);
        // the unit's finaliser rotates over the warps; it fetches the target
        // and its logit up front
        const int fin = (int)(it % kRingWarps);
        int64_t y = 0;
        float zy = 0.f;
        if (a.splits == 1 && wid == fin && lane == 0) {
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            if (y != a.ignore && y >= 0 && y < a.V) zy = to_f32(row[y]);
        }
        OnlineState st = empty_state();
        FoldRef ref;
        ref.ok = false;  // the unit's first part is folded the exact way
        for (int j = wid; j < ru.nch; j += kRingWarps) {
            const int stage = (int)(consumed & (kRingStages - 1));
            const uint32_t bar = smem_u32(&full_bar[wid][stage]);
            if (!dead) {
                if (mbar_wait(bar, (consumed / kRingStages) & 1u, &abort_flag, a.wait_ns))
                    ++waited;
                else
                    dead = true;
            }
            if (!dead) {
                const int64_t left = ru.nv - (int64_t)j * kRingVecs;
                const int nvc = (int)(left < kRingVecs ? left : kRingVecs);
                // the chunk is folded in parts of kRingPart vectors
#pragma unroll 1
                for (int h = 0; h < kRingVecs / kRingPart && h * kRingPart < nvc; ++h) {
                    const uint4* buf =
                        reinterpret_cast<const uint4*>(ring + stage * kRingVecs * 16) + h * kRingPart;
                    const int nvh = min(kRingPart, nvc - h * kRingPart);
                    if constexpr (sizeof(T) == 2 && !ARGMAX) {
                        // raw 16-bit words: packed max, widened pairwise for the sum
                        uint4 w[kPerLane];
                        bool ok[kPerLane];
#pragma unroll
                        for (int q = 0; q < kPerLane; ++q) {
                            const int vi = q * 32 + lane;
                            ok[q] = vi < nvh;
                            if (ok[q]) w[q] = buf[vi];
                        }
                        if (nvh == kRingPart) {
                            // without label smoothing, parts after the first
                            // fold against the lane's reference max
                            bool done = false;
                            if constexpr (!WITH_T) {
                                if (ref.ok) done = fold_raw16_ref<T, kPerLane>(st, w, ref);
                            }
                            if (!done) {
                                fold_raw16<T, kPerLane, false, WITH_T>(st, w, ok);
                                if constexpr (!WITH_T) ref = fold_ref(st);
                            }
                        } else {
                            fold_raw16<T, kPerLane, true, WITH_T>(st, w, ok);
                            if constexpr (!WITH_T) ref = fold_ref(st);
                        }
                    } else {
                        float v[kPerLane][VEC];
                        bool ok[kPerLane];
                        int c0[kPerLane];
#pragma unroll
                        for (int q = 0; q < kPerLane; ++q) {
                            const int vi = q * 32 + lane;
                            ok[q] = vi < nvh;
                            c0[q] = (int)((ru.v0 + (int64_t)j * kRingVecs + h * kRingPart + vi) * VEC);
                            if (ok[q]) unpack_words<T>(buf[vi], v[q]);
                        }
                        if (nvh == kRingPart) {
                            fold_vecs<kPerLane, VEC, false>(st, v, ok);
                            if constexpr (ARGMAX) argmax_vecs<kPerLane, VEC, false>(st, v, ok, c0);
                        } else {
                            fold_vecs<kPerLane, VEC, true>(st, v, ok);
                            if constexpr (ARGMAX) argmax_vecs<kPerLane, VEC, true>(st, v, ok, c0);
                        }
                    }
                }
            }
            // the buffer is read: hand it back to the copy engine
            fence_proxy_async_smem();
            __syncwarp();
            if (iss.valid(units) && !dead && !a.starve) {
                if (lane == 0) {
                    mbar_expect_tx(bar, iss.bytes());
                    bulk_load(smem_u32(ring + stage * kRingVecs * 16), iss.src(), iss.bytes(), bar);
                }
                ++issued;
            }
            iss.next(a, units, nvec, wid);
            ++consumed;
        }
        if (wid == 0 && sp == a.splits - 1) {
            for (int q = lane; q < tail; q += 32) {
                float x;
                load_vec<T, 1>(row, nvec * VEC + q, 1, &x);
                fold<1, ARGMAX>(st, &x, (int)(nvec * VEC + q), 0);
            }
        }
        group_reduce<32, ARGMAX, WITH_T>(st);
        // slot[parity] was last read by the finaliser of unit it - 2; every
        // other warp waits for its release before overwriting it
        if (it >= 2 && wid != (int)((it - 2) % kRingWarps)) named_bar_sync(3 + parity, kRingWarps * 32);
        if (lane == 0) slots[parity][wid] = st;
        if (wid != fin) {
            named_bar_arrive(1 + parity, kRingWarps * 32);
        } else {
            named_bar_sync(1 + parity, kRingWarps * 32);
            st = slots[parity][lane & (kRingWarps - 1)];
            group_reduce<kRingWarps, ARGMAX, WITH_T>(st);
            // the slots are read: release them for unit it + 2, if this CTA has one
            if ((int64_t)u + 2 * (int64_t)gridDim.x < units) named_bar_arrive(3 + parity, kRingWarps * 32);
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
    if (dead || abort_flag) {
        if (lane == 0) atomicOr(a.err, kErrTimeout);
        // let every copy this warp started land before the CTA exits
        if (lane == 0) {
            volatile int never = 0;
            for (uint32_t e = waited; e != issued; ++e)
                mbar_wait(smem_u32(&full_bar[wid][e & (kRingStages - 1)]), (e / kRingStages) & 1u,
                          &never);
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
    // 32 values per lane per step (8 loads of 4-byte, 4 of 2-byte types);
    // register budgets for four (4-byte) or two (2-byte) blocks per SM: the
    // 4-byte rows are latency-bound and gain more from resident warps than
    // they lose to a few spilled registers (argmax needs three blocks' room)
    constexpr int kU = sizeof(T) == 4 ? 8 : 4;
    constexpr int kMinB = sizeof(T) == 4 ? (ARGMAX ? 3 : 4) : 2;
    constexpr int kMinBTiny = sizeof(T) == 4 ? 5 : 4;
#define CEB_PACKED(GG, UU, MB)                                                    \
    if (G == GG && U == UU) {                                                     \
        k_fwd_packed<T, VEC, GG, UU, ARGMAX, MB><<<grid, 256, 0, s>>>(a);         \
        return cudaGetLastError();                                                \
    }
    CEB_PACKED(1, 2, kMinBTiny)  // tiny rows: latency-bound, so as many warps as fit
    CEB_PACKED(1, kU, (sizeof(T) == 4 ? 3 : 2))  // fewer rows per warp: more registers
    CEB_PACKED(2, kU, (sizeof(T) == 4 ? 3 : 2))
    CEB_PACKED(4, kU, kMinB)
    CEB_PACKED(8, kU, kMinB)
    CEB_PACKED(16, kU, kMinB)
    CEB_PACKED(32, kU, kMinB)
#undef CEB_PACKED
    return cudaErrorInvalidValue;
}

template <typename T, bool ARGMAX, bool WITH_T>
static cudaError_t launch_ring(const FwdPlan& p, const FwdArgs& a, cudaStream_t s) {
    cudaError_t e = ensure_smem_limit((const void*)k_fwd_ring<T, ARGMAX, WITH_T>, (int)kRingSmem);
    if (e != cudaSuccess) return e;
    k_fwd_ring<T, ARGMAX, WITH_T><<<p.grid, kRingWarps * 32, kRingSmem, s>>>(a);
    return cudaGetLastError();
}

template <typename T, int VEC>
static cudaError_t launch_pipe(const FwdPlan& p, const FwdArgs& a, cudaStream_t s) {
    constexpr int U = 8;
    constexpr size_t smem = (size_t)2 * kPipeWarps * U * 32 * 16;  // 64 KB
#define CEB_PIPE(GG)                                                                            \
    if (p.G == GG) {                                                                            \
        cudaError_t e =                                                                         \
            ensure_smem_limit((const void*)k_fwd_packed_pipe<T, VEC, GG, U, false, 3>, (int)smem); \
        if (e != cudaSuccess) return e;                                                         \
        k_fwd_packed_pipe<T, VEC, GG, U, false, 3><<<p.grid, kPipeWarps * 32, smem, s>>>(a);    \
        return cudaGetLastError();                                                              \
    }
    CEB_PIPE(2) CEB_PIPE(4) CEB_PIPE(8) CEB_PIPE(16) CEB_PIPE(32)
#undef CEB_PIPE
    return cudaErrorInvalidValue;
}

template <typename T, bool ARGMAX, bool WITH_T>
static cudaError_t launch_tiny(const FwdPlan& p, const FwdArgs& a, cudaStream_t s) {
    constexpr int V8 = ElemTraits<T>::kVec;
    // register budgets: 51 per thread for one vector per row, 64 for two
    if (p.U == 1)
        k_fwd_tiny<T, V8, 1, kTinyRows, ARGMAX, WITH_T, 5><<<p.grid, 256, 0, s>>>(a);
    else
        k_fwd_tiny<T, V8, 2, kTinyRows, ARGMAX, WITH_T, 4><<<p.grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T, bool ARGMAX>
static cudaError_t launch_fwd_t(const FwdPlan& p, const FwdArgs& a, cudaStream_t s) {
    constexpr int V8 = ElemTraits<T>::kVec;
    if (p.kind == FwdPlan::kTiny)
        return a.eps != 0.f ? launch_tiny<T, ARGMAX, true>(p, a, s) : launch_tiny<T, ARGMAX, false>(p, a, s);
    if constexpr (sizeof(T) == 4 && !ARGMAX) {
        // (with argmax, the plain packed kernel below takes the same plan)
        if (p.kind == FwdPlan::kPacked && p.pipe) return launch_pipe<T, V8>(p, a, s);
    }
    if (p.kind == FwdPlan::kPacked) {
        return p.vec == 1 ? launch_packed<T, 1, ARGMAX>(a, p.G, p.U, p.grid, s)
                          : launch_packed<T, V8, ARGMAX>(a, p.G, p.U, p.grid, s);
    }
    if (!p.ring) {
        if (p.vec == 1)
            k_fwd_cta<T, 1, 8, ARGMAX><<<p.grid, kCtaThreads, 0, s>>>(a);
        else
            k_fwd_cta<T, V8, 4, ARGMAX><<<p.grid, kCtaThreads, 0, s>>>(a);
    } else if (a.eps != 0.f) {
        cudaError_t e = launch_ring<T, ARGMAX, true>(p, a, s);
        if (e != cudaSuccess) return e;
    } else {
        cudaError_t e = launch_ring<T, ARGMAX, false>(p, a, s);
        if (e != cudaSuccess) return e;
    }
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

}  // namespace ceb
