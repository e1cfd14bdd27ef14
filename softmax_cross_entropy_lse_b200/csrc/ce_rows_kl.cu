// KL divergence of a student distribution from a teacher's, fused.
//
// Suryavanshi, "One barrier short", describes the fused KL loss of mlx-lm:
// for teacher logits zp and student logits zq of a row, p = softmax(zp) and
// q = softmax(zq),
//     loss = sum_j p_j (log p_j - log q_j),   dzq_j = g (q_j - p_j),
// computed in one pass with an online log-sum-exp per distribution. With
// (mq, sq) and (mp, sp) the running max and scaled sum of each, and
//     W = sum_j exp(zp_j - mp) (zp_j - zq_j),
// rescaled by exp(mp - mp') together with sp whenever mp grows to mp',
//     loss = W / sp - (lse_p - lse_q).
// A class with p_j = 0 adds nothing to W, even where zq_j is -inf too
// (0 log 0 = 0). The backward recomputes q_j and p_j from the two saved
// (lse, lse_lo) pairs.
//
// G lanes share a row (a whole warp, looping, for long rows), 32 / G rows
// per warp, grid-stride over rows; both rows stay in flight as raw 16-byte
// words. The cross-lane merge takes each maximum first, so the exchange has
// no slot to reuse (the race that "One barrier short" is about cannot occur).
#include "ce_device.cuh"
#include "ce_launch.h"
#include "ce_sm100.cuh"

#include <mutex>

namespace ceb {

struct KlState {
    float mq, sq, mp, sp, w;
};

__device__ __forceinline__ void kl_rescale(KlState& st, float mq, float mp) {
    if (st.mq != mq) {
        st.sq *= ex2((st.mq - mq) * kLog2e);
        st.mq = mq;
    }
    if (st.mp != mp) {
        const float f = ex2((st.mp - mp) * kLog2e);
        st.sp *= f;
        st.w *= f;
        st.mp = mp;
    }
}

template <int n>
__device__ __forceinline__ void kl_fold(KlState& st, const float (&zq)[n], const float (&zp)[n]) {
    float cq = zq[0], cp = zp[0];
#pragma unroll
    for (int i = 1; i < n; ++i) {
        cq = fmaxf(cq, zq[i]);
        cp = fmaxf(cp, zp[i]);
    }
    kl_rescale(st, fmaxf(st.mq, cq), fmaxf(st.mp, cp));
    const float msq = st.mq == -INFINITY ? 0.f : st.mq;
    const float msp = st.mp == -INFINITY ? 0.f : st.mp;
    float sq = 0.f, sp = 0.f, w = 0.f;
#pragma unroll
    for (int i = 0; i < n; ++i) {
        sq += ex2((zq[i] - msq) * kLog2e);
        const float ep = ex2((zp[i] - msp) * kLog2e);
        sp += ep;
        if (ep != 0.f) w = fmaf(ep, zp[i] - zq[i], w);
    }
    st.sq += sq;
    st.sp += sp;
    st.w += w;
}

template <int G>
__device__ __forceinline__ void kl_group_reduce(KlState& st) {
    if constexpr (G > 1) {
        float Mq = st.mq, Mp = st.mp;
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
            Mq = fmaxf(Mq, __shfl_xor_sync(0xffffffffu, Mq, off));
            Mp = fmaxf(Mp, __shfl_xor_sync(0xffffffffu, Mp, off));
        }
        kl_rescale(st, Mq, Mp);
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
            st.sq += __shfl_xor_sync(0xffffffffu, st.sq, off);
            st.sp += __shfl_xor_sync(0xffffffffu, st.sp, off);
            st.w += __shfl_xor_sync(0xffffffffu, st.w, off);
        }
    }
}

// loss and the two lse pairs of row r from its complete state
__device__ __forceinline__ void kl_finalize(const KlArgs& a, const KlState& st, int64_t r) {
    OnlineState oq = empty_state(), op = empty_state();
    oq.m = st.mq;
    oq.s = st.sq;
    op.m = st.mp;
    op.s = st.sp;
    float Lq, hq, lq, Lp, hp, lp;
    lse_pair(oq, Lq, hq, lq);
    lse_pair(op, Lp, hp, lp);
    a.lse_q[r] = hq;
    a.lse_p[r] = hp;
    if (a.lse_q_lo) a.lse_q_lo[r] = lq;
    if (a.lse_p_lo) a.lse_p_lo[r] = lp;
    float loss = __int_as_float(0x7fc00000);
    if (isfinite(hq) && isfinite(hp)) loss = st.w / st.sp - (st.mp - st.mq) - (Lp - Lq);
    a.loss[r] = loss;
}

template <typename T, int VEC, int G, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) k_kl_fwd(KlArgs a) {
    const T* __restrict__ zs = reinterpret_cast<const T*>(a.zq);
    const T* __restrict__ zt = reinterpret_cast<const T*>(a.zp);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        const bool active = r < a.N;
        KlState st{-INFINITY, 0.f, -INFINITY, 0.f, 0.f};
        const T* qr = zs;
        const T* pr = zt;
        if (active) {
            qr = zs + row_offset(a.lq, r, a.N);
            pr = zt + row_offset(a.lp, r, a.N);
        }
        for (int64_t vb = 0; vb < nvec; vb += (int64_t)G * U) {
            Raw<T, VEC> rq[U], rp[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + u * G + gl;
                ok[u] = active && vi < nvec;
                if (ok[u]) {
                    load_raw<T, VEC>(qr, vi * VEC, a.lq.s_col, rq[u]);
                    load_raw<T, VEC>(pr, vi * VEC, a.lp.s_col, rp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float q[VEC], p[VEC];
                unpack_raw<T, VEC>(rq[u], q);
                unpack_raw<T, VEC>(rp[u], p);
                kl_fold<VEC>(st, q, p);
            }
        }
        if (active) {
            for (int c = gl; c < tail; c += G) {
                const int64_t col = nvec * VEC + c;
                const float q[1] = {to_f32(qr[col * a.lq.s_col])};
                const float p[1] = {to_f32(pr[col * a.lp.s_col])};
                kl_fold<1>(st, q, p);
            }
        }
        kl_group_reduce<G>(st);
        if (active && gl == 0) kl_finalize(a, st, r);
    }
}

template <typename T, typename TO, int VEC, int G, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) k_kl_bwd(KlArgs a) {
    const T* zs = reinterpret_cast<const T*>(a.zq);
    const T* __restrict__ zt = reinterpret_cast<const T*>(a.zp);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        if (r >= a.N) continue;
        const T* qr = zs + row_offset(a.lq, r, a.N);
        const T* pr = zt + row_offset(a.lp, r, a.N);
        TO* dr = dz + row_offset(a.ld, r, a.N);
        const float g = a.g[r * a.g_stride];
        const float hq = a.lse_q[r], hp = a.lse_p[r];
        const float cq = (a.lse_q_lo ? a.lse_q_lo[r] : 0.f) * kLog2e;
        const float cp = (a.lse_p_lo ? a.lse_p_lo[r] : 0.f) * kLog2e;
        // a row whose lse is not finite has no distribution: NaN gradient
        const bool bad = !isfinite(hq) || !isfinite(hp);
        for (int64_t vb = gl; vb < nvec; vb += (int64_t)G * U) {
            Raw<T, VEC> rq[U], rp[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + (int64_t)u * G;
                ok[u] = vi < nvec;
                if (ok[u]) {
                    load_raw<T, VEC>(qr, vi * VEC, a.lq.s_col, rq[u]);
                    load_raw<T, VEC>(pr, vi * VEC, a.lp.s_col, rp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float q[VEC], p[VEC], o[VEC];
                unpack_raw<T, VEC>(rq[u], q);
                unpack_raw<T, VEC>(rp[u], p);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float qe = ex2(fmaf(q[e] - hq, kLog2e, -cq));
                    const float pe = ex2(fmaf(p[e] - hp, kLog2e, -cp));
                    o[e] = bad ? __int_as_float(0x7fc00000) : g * (qe - pe);
                }
                store_vec<TO, VEC>(dr, (vb + (int64_t)u * G) * VEC, a.ld.s_col, o);
            }
        }
        for (int c = gl; c < tail; c += G) {
            const int64_t col = nvec * VEC + c;
            const float qe = ex2(fmaf(to_f32(qr[col * a.lq.s_col]) - hq, kLog2e, -cq));
            const float pe = ex2(fmaf(to_f32(pr[col * a.lp.s_col]) - hp, kLog2e, -cp));
            cvt_store1(dr + col * a.ld.s_col, bad ? __int_as_float(0x7fc00000) : g * (qe - pe));
        }
    }
}

// ---------------------------------------------------------------------------
// Long rows, few of them (the page's 512 x 151,936): a CTA of 8 warps per row
// for the forward, the warp states meeting once in shared memory. The slots
// alternate between two sets on successive rows, so no slot is rewritten
// before every warp has passed the barrier of the row in between (the
// slot-reuse race of "One barrier short" cannot occur).
constexpr int kKlCtaWarps = 8;

template <typename T, int VEC, int U, int MINB>
__global__ void __launch_bounds__(kKlCtaWarps * 32, MINB) k_kl_fwd_cta(KlArgs a) {
    __shared__ KlState slots[2][kKlCtaWarps];
    const T* __restrict__ zs = reinterpret_cast<const T*>(a.zq);
    const T* __restrict__ zt = reinterpret_cast<const T*>(a.zp);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    constexpr int kThreads = kKlCtaWarps * 32;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    int parity = 0;
    for (int64_t r = blockIdx.x; r < a.N; r += gridDim.x, parity ^= 1) {
        const T* qr = zs + row_offset(a.lq, r, a.N);
        const T* pr = zt + row_offset(a.lp, r, a.N);
        KlState st{-INFINITY, 0.f, -INFINITY, 0.f, 0.f};
        for (int64_t vb = tid; vb < nvec; vb += (int64_t)kThreads * U) {
            Raw<T, VEC> rq[U], rp[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + (int64_t)u * kThreads;
                ok[u] = vi < nvec;
                if (ok[u]) {
                    load_raw<T, VEC>(qr, vi * VEC, a.lq.s_col, rq[u]);
                    load_raw<T, VEC>(pr, vi * VEC, a.lp.s_col, rp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float q[VEC], p[VEC];
                unpack_raw<T, VEC>(rq[u], q);
                unpack_raw<T, VEC>(rp[u], p);
                kl_fold<VEC>(st, q, p);
            }
        }
        for (int c = tid; c < tail; c += kThreads) {
            const int64_t col = nvec * VEC + c;
            const float q[1] = {to_f32(qr[col * a.lq.s_col])};
            const float p[1] = {to_f32(pr[col * a.lp.s_col])};
            kl_fold<1>(st, q, p);
        }
        kl_group_reduce<32>(st);
        if (lane == 0) slots[parity][wid] = st;
        __syncthreads();
        if (wid == 0) {
            st = slots[parity][lane & (kKlCtaWarps - 1)];
            kl_group_reduce<kKlCtaWarps>(st);
            if (lane == 0) kl_finalize(a, st, r);
        }
    }
}

// Long rows split across a thread-block cluster of CL CTAs: CTA k of the
// cluster folds vectors [k S, (k+1) S) of the row (S = vec_per_cta) with the
// 8-warp loop above, reduces its warps in shared memory, and stores its
// (mq, sq, mp, sp, w) state into slot [parity][k] of the cluster's first CTA,
// which merges the CL states in rank order and writes the row. A batch of a
// few hundred rows then fills every CTA slot of the GPU (a CTA per row left
// the last wave part-empty: 512 rows over 592 slots).
//
// One cluster barrier per row orders the exchange, split in halves so that
// no CTA waits at it: after storing its state of row i a CTA arrives (with
// release), folds row i + 1, then waits (with acquire) for row i's arrivals
// before storing its state of row i + 1 into the other slot set. The first
// CTA reads row i's slots after that wait and before arriving for row i + 1;
// a slot set is written again only for row i + 2, after the wait for row
// i + 1, which needs that arrival. No slot is rewritten before it is read
// (the race "One barrier short" describes cannot occur).
template <typename T, int VEC, int U, int CL, int MINB>
__global__ void __launch_bounds__(kKlCtaWarps * 32, MINB) k_kl_fwd_cluster(KlArgs a,
                                                                           int64_t vec_per_cta) {
    using namespace sm100;
    __shared__ KlState wslots[2][kKlCtaWarps];
    __shared__ __align__(16) float cslots[2][CL][8];  // in the first CTA: (mq, sq, mp, sp, w)
    const T* __restrict__ zs = reinterpret_cast<const T*>(a.zq);
    const T* __restrict__ zt = reinterpret_cast<const T*>(a.zp);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    constexpr int kThreads = kKlCtaWarps * 32;
    const uint32_t rank = cluster_ctarank();
    const int64_t cid = cluster_id_x(), ncl = cluster_count_x();
    const int64_t nvec = a.V / VEC;
    const int tail = rank == CL - 1 ? (int)(a.V - nvec * VEC) : 0;
    const int64_t v0 = (int64_t)rank * vec_per_cta;
    const int64_t v1 = min(nvec, v0 + vec_per_cta);
    // this CTA's two slots in the first CTA's shared memory
    const uint32_t dst[2] = {mapa_shared(smem_u32(&cslots[0][rank][0]), 0),
                             mapa_shared(smem_u32(&cslots[1][rank][0]), 0)};

    // the first CTA merges the CL states of row r (slot set par) and writes it
    auto finish = [&](int64_t r, int par) {
        if (rank == 0 && wid == 0) {
            KlState st{-INFINITY, 0.f, -INFINITY, 0.f, 0.f};
            if (lane < CL) {
                const float* c = cslots[par][lane];
                st = KlState{c[0], c[1], c[2], c[3], c[4]};
            }
            kl_group_reduce<CL>(st);  // lanes >= CL hold the empty state
            if (lane == 0) kl_finalize(a, st, r);
        }
    };

    int it = 0;
    int64_t prev = -1;
    for (int64_t r = cid; r < a.N; r += ncl, ++it) {
        const int par = it & 1;
        const T* qr = zs + row_offset(a.lq, r, a.N);
        const T* pr = zt + row_offset(a.lp, r, a.N);
        KlState st{-INFINITY, 0.f, -INFINITY, 0.f, 0.f};
        for (int64_t vb = v0 + tid; vb < v1; vb += (int64_t)kThreads * U) {
            Raw<T, VEC> rq[U], rp[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + (int64_t)u * kThreads;
                ok[u] = vi < v1;
                if (ok[u]) {
                    load_raw<T, VEC>(qr, vi * VEC, a.lq.s_col, rq[u]);
                    load_raw<T, VEC>(pr, vi * VEC, a.lp.s_col, rp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float q[VEC], p[VEC];
                unpack_raw<T, VEC>(rq[u], q);
                unpack_raw<T, VEC>(rp[u], p);
                kl_fold<VEC>(st, q, p);
            }
        }
        for (int c = tid; c < tail; c += kThreads) {
            const int64_t col = nvec * VEC + c;
            const float q[1] = {to_f32(qr[col * a.lq.s_col])};
            const float p[1] = {to_f32(pr[col * a.lp.s_col])};
            kl_fold<1>(st, q, p);
        }
        kl_group_reduce<32>(st);
        if (lane == 0) wslots[par][wid] = st;
        __syncthreads();
        if (wid == 0) {
            st = wslots[par][lane & (kKlCtaWarps - 1)];
            kl_group_reduce<kKlCtaWarps>(st);
        }
        // row it - 1: every CTA's state has arrived; the first CTA writes it
        if (it > 0) {
            cluster_wait_acquire();
            finish(prev, par ^ 1);
        }
        if (wid == 0 && lane == 0) {
            st_cluster_v4(dst[par], st.mq, st.sq, st.mp, st.sp);
            st_cluster_f32(dst[par] + 16, st.w);
        }
        cluster_arrive_release();
        prev = r;
    }
    if (it > 0) {
        cluster_wait_acquire();
        finish(prev, (it - 1) & 1);
    }
}

// The backward needs no reduction: the rows are cut into chunks of
// kKlChunkVecs vectors, one warp per (row, chunk) unit.
constexpr int64_t kKlChunkVecs = 1024;

template <typename T, typename TO, int VEC, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) k_kl_bwd_chunks(KlArgs a) {
    const T* zs = reinterpret_cast<const T*>(a.zq);
    const T* __restrict__ zt = reinterpret_cast<const T*>(a.zp);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const int64_t nch = (nvec + kKlChunkVecs - 1) / kKlChunkVecs > 0 ? (nvec + kKlChunkVecs - 1) / kKlChunkVecs : 1;
    for (int64_t unit = warp; unit < a.N * nch; unit += nwarps) {
        const int64_t r = unit / nch;
        const int64_t ch = unit - r * nch;
        const T* qr = zs + row_offset(a.lq, r, a.N);
        const T* pr = zt + row_offset(a.lp, r, a.N);
        TO* dr = dz + row_offset(a.ld, r, a.N);
        const float g = a.g[r * a.g_stride];
        const float hq = a.lse_q[r], hp = a.lse_p[r];
        const float cq = (a.lse_q_lo ? a.lse_q_lo[r] : 0.f) * kLog2e;
        const float cp = (a.lse_p_lo ? a.lse_p_lo[r] : 0.f) * kLog2e;
        const bool bad = !isfinite(hq) || !isfinite(hp);
        const int64_t v1 = min(nvec, (ch + 1) * kKlChunkVecs);
        for (int64_t vb = ch * kKlChunkVecs + lane; vb < v1; vb += (int64_t)32 * U) {
            Raw<T, VEC> rq[U], rp[U];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + (int64_t)u * 32;
                ok[u] = vi < v1;
                if (ok[u]) {
                    load_raw<T, VEC>(qr, vi * VEC, a.lq.s_col, rq[u]);
                    load_raw<T, VEC>(pr, vi * VEC, a.lp.s_col, rp[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                float q[VEC], p[VEC], o[VEC];
                unpack_raw<T, VEC>(rq[u], q);
                unpack_raw<T, VEC>(rp[u], p);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float qe = ex2(fmaf(q[e] - hq, kLog2e, -cq));
                    const float pe = ex2(fmaf(p[e] - hp, kLog2e, -cp));
                    o[e] = bad ? __int_as_float(0x7fc00000) : g * (qe - pe);
                }
                store_vec<TO, VEC>(dr, (vb + (int64_t)u * 32) * VEC, a.ld.s_col, o);
            }
        }
        if (ch == nch - 1) {
            for (int c = lane; c < tail; c += 32) {
                const int64_t col = nvec * VEC + c;
                const float qe = ex2(fmaf(to_f32(qr[col * a.lq.s_col]) - hq, kLog2e, -cq));
                const float pe = ex2(fmaf(to_f32(pr[col * a.lp.s_col]) - hp, kLog2e, -cp));
                cvt_store1(dr + col * a.ld.s_col, bad ? __int_as_float(0x7fc00000) : g * (qe - pe));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Four vectors of each row in flight per lane (eight on the scalar path) at
// three blocks per SM: two rows' words take the registers of four blocks'
// worth. The planner's lane grouping uses the same U.
template <int VEC, bool BWD = false> struct KlShape {
    static constexpr int U = VEC == 1 ? 8 : 4;
    static constexpr int MINB = VEC == 1 ? 2 : 3;
};

template <typename T, int VEC, int CL>
static cudaError_t launch_kl_cluster(const KlPlan& p, const KlArgs& a, cudaStream_t s) {
    constexpr int U = KlShape<VEC>::U;
    constexpr int MB = VEC == 1 ? 2 : (VEC == 8 ? 3 : 4);
    auto kern = k_kl_fwd_cluster<T, VEC, U, CL, MB>;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.blockDim = dim3(kKlCtaWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CL;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    // co-resident clusters, cached per device
    static std::mutex mu;
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int clusters;
    {
        std::lock_guard<std::mutex> lock(mu);
        clusters = cached[dev];
        if (clusters == 0) {
            cfg.gridDim = dim3(CL * p.sms);
            const cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
            if (e != cudaSuccess) return e;
            if (clusters < 1) return cudaErrorInvalidConfiguration;
            cached[dev] = clusters;
        }
    }
    const int64_t want = a.N < clusters ? a.N : clusters;
    cfg.gridDim = dim3((unsigned)(want * CL));
    return cudaLaunchKernelEx(&cfg, kern, a, p.vec_per_cta);
}

template <typename T, int VEC>
static cudaError_t kl_fwd_v(const KlPlan& p, const KlArgs& a, cudaStream_t s) {
    constexpr int U = KlShape<VEC>::U, MB = KlShape<VEC>::MINB;
    if (p.cta && p.cl > 1) {
        switch (p.cl) {
            case 2: return launch_kl_cluster<T, VEC, 2>(p, a, s);
            case 4: return launch_kl_cluster<T, VEC, 4>(p, a, s);
            case 8: return launch_kl_cluster<T, VEC, 8>(p, a, s);
        }
        return cudaErrorInvalidValue;
    }
    if (p.cta) {
        // four CTAs per SM for 4-byte rows: 592 rows in flight on a 148-SM
        // part, so a batch of a few hundred long rows runs in one wave
        // (16-bit rows need three CTAs' registers)
        k_kl_fwd_cta<T, VEC, U, (VEC == 1 ? 2 : (VEC == 8 ? 3 : 4))><<<p.grid, kKlCtaWarps * 32, 0, s>>>(a);
        return cudaGetLastError();
    }
#define CEB_KL(GG)                                                          \
    if (p.G == GG) {                                                        \
        k_kl_fwd<T, VEC, GG, U, MB><<<p.grid, 256, 0, s>>>(a);              \
        return cudaGetLastError();                                          \
    }
    CEB_KL(1) CEB_KL(2) CEB_KL(4) CEB_KL(8) CEB_KL(16) CEB_KL(32)
#undef CEB_KL
    return cudaErrorInvalidValue;
}

template <typename T, typename TO, int VEC>
static cudaError_t kl_bwd_v(const KlPlan& p, const KlArgs& a, cudaStream_t s) {
    constexpr int U = KlShape<VEC, true>::U, MB = KlShape<VEC, true>::MINB;
    if (p.cta) {
        k_kl_bwd_chunks<T, TO, VEC, U, MB><<<p.grid_bwd, 256, 0, s>>>(a);
        return cudaGetLastError();
    }
#define CEB_KL(GG)                                                          \
    if (p.G == GG) {                                                        \
        k_kl_bwd<T, TO, VEC, GG, U, MB><<<p.grid, 256, 0, s>>>(a);          \
        return cudaGetLastError();                                          \
    }
    CEB_KL(1) CEB_KL(2) CEB_KL(4) CEB_KL(8) CEB_KL(16) CEB_KL(32)
#undef CEB_KL
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t kl_fwd_t(const KlPlan& p, const KlArgs& a, cudaStream_t s) {
    if (p.vec == 1) return kl_fwd_v<T, 1>(p, a, s);
    return kl_fwd_v<T, ElemTraits<T>::kVec>(p, a, s);
}

template <typename T, typename TO>
static cudaError_t kl_bwd_t(const KlPlan& p, const KlArgs& a, cudaStream_t s) {
    if (p.vec == 1) return kl_bwd_v<T, TO, 1>(p, a, s);
    return kl_bwd_v<T, TO, ElemTraits<T>::kVec>(p, a, s);
}

cudaError_t launch_kl_forward(const KlPlan& p, const KlArgs& a, int dt, cudaStream_t s) {
    switch (dt) {
        case 0: return kl_fwd_t<float>(p, a, s);
        case 1: return kl_fwd_t<__nv_bfloat16>(p, a, s);
        case 2: return kl_fwd_t<__half>(p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_kl_backward(const KlPlan& p, const KlArgs& a, int dt, int ddt, cudaStream_t s) {
    if (dt == 0) return kl_bwd_t<float, float>(p, a, s);
    if (dt == 1) return ddt == 0 ? kl_bwd_t<__nv_bfloat16, float>(p, a, s)
                                 : kl_bwd_t<__nv_bfloat16, __nv_bfloat16>(p, a, s);
    if (dt == 2) return ddt == 0 ? kl_bwd_t<__half, float>(p, a, s) : kl_bwd_t<__half, __half>(p, a, s);
    return cudaErrorInvalidValue;
}

}  // namespace ceb
