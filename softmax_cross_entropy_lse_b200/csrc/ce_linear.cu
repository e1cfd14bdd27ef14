// Fused-linear cross-entropy on sm_100a tensor cores.
//
// Source: Ineshin, "A fused linear cross-entropy forward kernel for Apple
// GPUs", section 1: with H (N x D) and W (V x D), the logits Z = H W^T are
// produced tile by tile, each vocabulary tile is folded into the running
// (max, scaled sum) state of every row, the target logit is captured when its
// tile passes, and the (N, V) matrix never exists. The backward regenerates
// the logits tile by tile from the saved log-sum-exp.
//
// Design for B200 (not the page's Metal kernel):
//  * one persistent GEMM engine, K in 64-element (128-byte) steps: a TMA
//    producer warp fills a shared-memory ring, one thread issues tcgen05.mma
//    into a double-buffered f32 accumulator in tensor memory (2 x 256
//    columns), and four epilogue warps read the accumulator with tcgen05.ld,
//    one TMEM lane (= one output row) per thread. The forward runs one CTA
//    per 128 x 256 tile (4 stages); the backward runs CTA pairs on 256 x 256
//    tiles (6 stages, cta_group::2);
//  * the CTAs in flight work on consecutive units. Row tiles run fastest, so
//    the row operand A stays in L2 (H in the forward and in GEMM 1); in GEMMs
//    2 and 3, when A (G_c, 134 MB at N = 8192) is the larger operand, column
//    units run fastest instead and B's lines (H, or W_c) carry an evict_last
//    L2 policy, so each B panel crosses DRAM once per launch;
//  * forward epilogue: the online log-sum-exp of each row over a unit of
//    consecutive vocabulary tiles, kept in registers, then a partial state
//    per (unit, row) merged in unit order by a second launch;
//  * backward: for each vocabulary chunk, GEMM 1 recomputes Z_c = H W_c^T and
//    its epilogue writes G_c = g (softmax - (1-eps) onehot - eps/V) in bf16;
//    GEMM 2 forms dW_c = G_c^T H; GEMM 3 adds G_c W_c into a float dH
//    accumulator. Each dW row belongs to one chunk, so dW needs no
//    accumulation across chunks. GEMM 2 reads both its operands, and GEMM 3
//    its B operand, in their stored orientation: the tiles are loaded
//    MN-major (the output index contiguous) and the MMA descriptors say so,
//    so no transposed copy of H, W or G_c is ever made.
// Every pipeline wait is bounded in time; on expiry the CTA raises an error
// bit, drains its own copies and MMAs, frees its tensor memory and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "ce_b200.h"
#include "ce_device.cuh"
#include "ce_launch.h"
#include "ce_linear.h"
#include "ce_sm100.cuh"

namespace ceb {
using namespace sm100;

// TMA loads with an L2 cache policy for the source lines (the engine marks the
// operand that should stay in L2), and the policy itself.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

// An L2 policy under which the lines it marks are evicted after normal ones.
__device__ __forceinline__ uint64_t l2_policy_keep() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap* map,
                                                      uint32_t bar_cluster, int c0, int c1,
                                                      uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr uint32_t kABytes = kBM * kBK * 2;  // one CTA's A rows of a stage
constexpr int kGemmThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr uint32_t kTmemCols = 2 * kBN;
// An MN-major operand tile arrives as boxes of 64 (M or N) x kBK (K) elements,
// 8 KB each, stacked along M/N.
constexpr int kMnBox = 64;
constexpr uint32_t kMnBoxBytes = kMnBox * kBK * 2;

// Shapes of the engine for one CTA (CG = 1) or a CTA pair (CG = 2). A pair
// computes 256 x 256 output tiles: each CTA holds 128 rows of A and 128 rows
// of B per stage and receives its 128 rows of the accumulator, so a stage is
// 32 KB instead of 48 KB and six stages fit where four did.
template <int CG>
struct GemmCfg {
    static constexpr int kRowsB = kBN / CG;  // B rows per CTA and stage
    static constexpr uint32_t kBBytes = kRowsB * kBK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = CG == 1 ? 4 : 6;
    static constexpr int kTileM = kBM * CG;  // output rows per unit tile
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 256;
    // Reach of one MMA's MN-major descriptor: its start moves 2 KB per K step
    // of 16, it spans the tile's boxes along M/N (leading offset) and two 1 KB
    // K groups (stride offset). The last byte must stay inside the stage.
    static_assert((kBK / 16 - 1) * 2048 + (kBM / kMnBox - 1) * kMnBoxBytes + 2048 <= kABytes,
                  "an MN-major A descriptor reaches past its stage");
    static_assert((kBK / 16 - 1) * 2048 + (kRowsB / kMnBox - 1) * kMnBoxBytes + 2048 <= kBBytes,
                  "an MN-major B descriptor reaches past its stage");
    static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

enum EpiKind { kEpiCeFwd = 0, kEpiCeGrad = 1, kEpiStore = 2, kEpiAccum = 3 };

struct GemmArgs {
    int M, Nn, K;              // output rows, output columns, reduction length
    int n_mb, n_nb, nkb;       // tile counts
    int tiles_per_unit;        // consecutive column tiles handled as one unit
    int n_units_n;             // ceil(n_nb / tiles_per_unit)
    int64_t units;             // n_mb * n_units_n
    // unit order: row tiles fastest (0), or column units fastest (1), in which
    // case B's lines are kept in L2 ahead of normal ones (see launch_gemm)
    int n_fast;
    int kA0, kB0;              // K origin of A and B in their tensor maps
    unsigned int* err;
    unsigned long long wait_ns;  // limit of every pipeline wait
    int starve;                  // testing: the producer issues no copies
    // cross-entropy epilogues
    const void* y;
    int tdt;
    int64_t V;
    float eps;
    int64_t ignore;
    int64_t col_base;          // vocabulary index of output column 0
    float4* part;              // forward partials [n_units_n][M]
    const float* g;
    int64_t g_stride;
    const float* lse;
    __nv_bfloat16* G;          // gradient chunk, row-major, ld = ldG
    int64_t ldG;
    // store / accumulate epilogues
    void* C;                   // output rows start here
    int64_t ldc;
    int c_f32;
    float* acc;                // float accumulator (may equal C when c_f32)
    int64_t ld_acc;
    int acc_first, acc_last;
};

// ---------------------------------------------------------------------------
// Epilogue helpers.

// Folds the first nv of 32 values (nv < 32 only in a ragged last tile).
__device__ __forceinline__ void fold_prefix(OnlineState& st, const float (&v)[32], int nv) {
    float cm = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j)
        if (j < nv) cm = fmaxf(cm, v[j]);
    rescale_to(st, fmaxf(st.m, cm));
    const float ms = (st.m == -INFINITY) ? 0.f : st.m;
    float sa = 0.f, ta = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        if (j < nv) {
            const float d = v[j] - ms;
            sa += ex2(d * kLog2e);
            ta += d;
        }
    }
    st.s += sa;
    st.t += ta;
    st.k += nv;
}

__device__ __forceinline__ void store_row32(void* base, int64_t ld, int64_t row, int64_t col,
                                            const float (&v)[32], int f32, int ncols) {
    if (f32) {
        float* p = reinterpret_cast<float*>(base) + row * ld + col;
        if (ncols == 32) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
                reinterpret_cast<float4*>(p)[q] =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < ncols) p[j] = v[j];
        }
    } else {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(base) + row * ld + col;
        if (ncols == 32) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack2((__nv_bfloat16*)nullptr, v[8 * q], v[8 * q + 1]);
                w.y = pack2((__nv_bfloat16*)nullptr, v[8 * q + 2], v[8 * q + 3]);
                w.z = pack2((__nv_bfloat16*)nullptr, v[8 * q + 4], v[8 * q + 5]);
                w.w = pack2((__nv_bfloat16*)nullptr, v[8 * q + 6], v[8 * q + 7]);
                reinterpret_cast<uint4*>(p)[q] = w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < ncols) p[j] = __float2bfloat16_rn(v[j]);
        }
    }
}

// ---------------------------------------------------------------------------
// The persistent GEMM: C[M x Nn] = A[M x K] * B[Nn x K]^T, bf16 operands
// through TMA tensor maps, f32 accumulation in tensor memory. An operand is
// K-major (its K index contiguous in memory: A as M x K, B as Nn x K, loaded
// in 64-wide boxes of K) or, with AMN / BMN, MN-major (its M or Nn index
// contiguous: A stored K x M, B stored K x Nn, loaded in 64 x 64 boxes).
//
// With CG = 2 the kernel runs as clusters of two CTAs on neighbouring SMs
// that share each 256 x 256 tile: both load their halves of A and B, the
// even CTA's MMA thread issues pair MMAs that read both halves, and each
// CTA's epilogue reads its 128 accumulator rows from its own tensor memory.
// Both CTAs' copies complete on the even CTA's stage barrier; its MMA commits
// arrive on the stage-free and accumulator-full barriers of both CTAs; both
// epilogues arrive on the even CTA's accumulator-free barrier.
template <int EPI, bool AMN, bool BMN, int CG>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           const GemmArgs a) {
    using Cfg = GemmCfg<CG>;
    constexpr int kStages = Cfg::kStages;
    constexpr uint32_t kBBytes = Cfg::kBBytes;
    constexpr uint32_t kIdesc = idesc_bf16_f32(Cfg::kTileM, kBN, AMN, BMN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * Cfg::kStageBytes);
    // barrier slots: full[kStages], empty[kStages], tfull[2], tempty[2], drain
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CG == 1 ? 0u : cluster_ctarank();
    const bool lead = rank == 0;
    const int64_t u_first = CG == 1 ? (int64_t)blockIdx.x : (int64_t)cluster_id_x();
    const int64_t u_step = CG == 1 ? (int64_t)gridDim.x : (int64_t)cluster_count_x();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 128 * CG);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_cg<CG>(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_cg<CG>();
    }
    tc_fence_before();
    // (a pair: both CTAs' barriers and tensor memory exist before either uses
    // the other's)
    if constexpr (CG == 2)
        cluster_sync();
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the even CTA's stage and accumulator-free barriers, as this CTA addresses them
    const uint32_t lead_full0 = CG == 1 ? full_bar(0) : mapa_shared(full_bar(0), 0);
    const uint32_t lead_tempty0 = CG == 1 ? tempty_bar(0) : mapa_shared(tempty_bar(0), 0);

    if (warp == 0) {
        // ---------------- TMA producer (each CTA loads its own halves) ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, last_ph = 0;  // per stage: has a load, its phase
            const uint64_t pol_keep = l2_policy_keep();
            bool ok = true;
            for (int64_t u = u_first; u < a.units && ok; u += u_step) {
                const int mb = a.n_fast ? (int)(u / a.n_units_n) : (int)(u % a.n_mb);
                const int un = a.n_fast ? (int)(u % a.n_units_n) : (int)(u / a.n_mb);
                const int nb0 = un * a.tiles_per_unit;
                const int nb1 = min(a.n_nb, nb0 + a.tiles_per_unit);
                const int rowA = mb * Cfg::kTileM + (int)rank * kBM;
                for (int nb = nb0; nb < nb1 && ok; ++nb) {
                    const int rowB = nb * kBN + (int)rank * Cfg::kRowsB;
                    for (int kb = 0; kb < a.nkb; ++kb) {
                        if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, a.wait_ns)) {
                            ok = false;
                            break;
                        }
                        // (a starved launch, a testing mode, issues no copies:
                        // the MMA thread's wait for this stage runs out)
                        if (!a.starve) {
                            if (lead) mbar_expect_tx(full_bar(s), CG * Cfg::kStageBytes);
                            const uint32_t fb = lead_full0 + 8u * s;
                            auto load = [&](uint32_t dst, const CUtensorMap* map, int c0, int c1) {
                                if (a.n_fast && map == &tmB) {
                                    if constexpr (CG == 1)
                                        tma_load_2d_hint(dst, map, fb, c0, c1, pol_keep);
                                    else
                                        tma_load_2d_pair_hint(dst, map, fb, c0, c1, pol_keep);
                                } else {
                                    if constexpr (CG == 1)
                                        tma_load_2d(dst, map, fb, c0, c1);
                                    else
                                        tma_load_2d_pair(dst, map, fb, c0, c1);
                                }
                            };
                            const int k0a = a.kA0 + kb * kBK, k0b = a.kB0 + kb * kBK;
                            if constexpr (AMN) {
#pragma unroll
                                for (int h = 0; h < kBM / kMnBox; ++h)
                                    load(smem_u32(sA + s * kABytes + h * kMnBoxBytes), &tmA,
                                         rowA + h * kMnBox, k0a);
                            } else {
                                load(smem_u32(sA + s * kABytes), &tmA, k0a, rowA);
                            }
                            if constexpr (BMN) {
#pragma unroll
                                for (int h = 0; h < Cfg::kRowsB / kMnBox; ++h)
                                    load(smem_u32(sB + s * kBBytes + h * kMnBoxBytes), &tmB,
                                         rowB + h * kMnBox, k0b);
                            } else {
                                load(smem_u32(sB + s * kBBytes), &tmB, k0b, rowB);
                            }
                            issued_mask |= 1u << s;
                            last_ph = (last_ph & ~(1u << s)) | (ph << s);
                        }
                        if (++s == kStages) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                }
            }
            if (!ok) {
                atomicOr(a.err, kErrTimeout);
                // let every copy this thread started land before the CTA exits:
                // on this CTA's own stage barriers, or, for the odd CTA of a
                // pair (whose copies complete on the even CTA's barriers), for
                // a bounded time
                volatile int never = 0;
                if (CG == 1 || lead) {
                    for (int q = 0; q < kStages; ++q)
                        if (issued_mask & (1u << q))
                            mbar_wait(full_bar(q), (last_ph >> q) & 1u, &never);
                } else if (issued_mask) {
                    const unsigned long long t0 = globaltimer();
                    while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread of the even CTA) ----------------
        if (lane == 0 && lead) {
            int s = 0;
            uint32_t ph = 0, it = 0;
            bool ok = true;
            for (int64_t u = u_first; u < a.units && ok; u += u_step) {
                const int un = a.n_fast ? (int)(u % a.n_units_n) : (int)(u / a.n_mb);
                const int nb0 = un * a.tiles_per_unit;
                const int nb1 = min(a.n_nb, nb0 + a.tiles_per_unit);
                for (int nb = nb0; nb < nb1 && ok; ++nb, ++it) {
                    const uint32_t acc = it & 1u;
                    if (!mbar_wait(tempty_bar(acc), ((it >> 1) & 1u) ^ 1u, abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem_base + acc * kBN;
                    for (int kb = 0; kb < a.nkb; ++kb) {
                        if (!mbar_wait(full_bar(s), ph, abort_flag, a.wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(sA + s * kABytes);
                        const uint32_t b0 = smem_u32(sB + s * kBBytes);
                        // K steps of 16: 32 bytes along a K-major row, two
                        // 8-row K groups (2 KB) down an MN-major atom column
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint64_t da = AMN ? desc_mnmajor_sw128(a0 + kk * 2048, kMnBoxBytes)
                                                    : desc_kmajor_sw128(a0 + kk * 32);
                            const uint64_t db = BMN ? desc_mnmajor_sw128(b0 + kk * 2048, kMnBoxBytes)
                                                    : desc_kmajor_sw128(b0 + kk * 32);
                            if constexpr (CG == 1)
                                umma_bf16(d, da, db, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                            else
                                umma_bf16_pair(d, da, db, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        if constexpr (CG == 1)
                            umma_commit(empty_bar(s));
                        else
                            umma_commit_pair(empty_bar(s), 3);
                        if (++s == kStages) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                    if (ok) {
                        if constexpr (CG == 1)
                            umma_commit(tfull_bar(acc));
                        else
                            umma_commit_pair(tfull_bar(acc), 3);
                    }
                }
            }
            if (!ok) atomicOr(a.err, kErrTimeout);
            // every MMA this thread issued has completed once `drain` flips
            if constexpr (CG == 1)
                umma_commit(drain_bar);
            else
                umma_commit_pair(drain_bar, 1);
            volatile int never = 0;
            mbar_wait(drain_bar, 0, &never);
        }
    } else {
        // ---------------- epilogue: warps 2..5, TMEM lane quadrant warp % 4 ----
        const int q = warp & 3;
        const int r_in_tile = 32 * q + lane;
        const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        bool ok = true;
        for (int64_t u = u_first; u < a.units && ok; u += u_step) {
            const int mb = a.n_fast ? (int)(u / a.n_units_n) : (int)(u % a.n_mb);
            const int un = a.n_fast ? (int)(u % a.n_units_n) : (int)(u / a.n_mb);
            const int nb0 = un * a.tiles_per_unit;
            const int nb1 = min(a.n_nb, nb0 + a.tiles_per_unit);
            const int64_t m = (int64_t)mb * Cfg::kTileM + (int64_t)rank * kBM + r_in_tile;
            const bool row_ok = m < a.M;
            // per-row state of the cross-entropy epilogues
            OnlineState st = empty_state();
            int64_t y = 0;
            float zy = 0.f, gl = 0.f, lse = 0.f, c_eps = 0.f, c_tgt = 0.f;
            bool live = false;
            if constexpr (EPI == kEpiCeFwd || EPI == kEpiCeGrad) {
                if (row_ok) y = load_target(a.y, a.tdt, m);
            }
            if constexpr (EPI == kEpiCeGrad) {
                if (row_ok) {
                    const bool bad = y != a.ignore && (y < 0 || y >= a.V);
                    live = y != a.ignore && !bad;
                    if (bad && a.col_base == 0) atomicOr(a.err, 1u);
                    gl = a.g[m * a.g_stride];
                    lse = a.lse[m];
                    c_eps = gl * a.eps / (float)a.V;
                    c_tgt = gl * (1.f - a.eps);
                }
            }

            for (int nb = nb0; nb < nb1; ++nb, ++it) {
                const uint32_t acc = it & 1u;
                if (!mbar_wait(tfull_bar(acc), (it >> 1) & 1u, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t0 = tmem_base + lane_addr + acc * kBN;
                const int64_t col0 = (int64_t)nb * kBN;  // output column of chunk 0
                int valid = (int)min((int64_t)kBN, (int64_t)a.Nn - col0);
#pragma unroll 1
                for (int ch = 0; ch < kBN / 32; ++ch) {
                    if (ch * 32 >= valid) break;
                    uint32_t r[32];
                    tmem_ld32(t0 + ch * 32, r);
                    tmem_wait_ld();
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                    const int nv = min(32, valid - ch * 32);
                    const int64_t c = col0 + ch * 32;  // output column of v[0]
                    if constexpr (EPI == kEpiCeFwd) {
                        if (nv == 32)
                            fold<32, false>(st, v, 0, 0);
                        else
                            fold_prefix(st, v, nv);
                        const int64_t dy = y - (a.col_base + c);
                        if (row_ok && dy >= 0 && dy < 32) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (j == dy) zy = v[j];
                        }
                    } else if constexpr (EPI == kEpiCeGrad) {
                        // G = g (exp(z - lse) - eps/V) - g (1 - eps)[col = y]
                        const int64_t dy = y - (a.col_base + c);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            float gv = 0.f;
                            if (live && j < nv) {
                                gv = fmaf(gl, ex2((v[j] - lse) * kLog2e), -c_eps);
                                if (j == dy) gv -= c_tgt;
                            }
                            v[j] = gv;
                        }
                        if (row_ok) store_row32(a.G, a.ldG, m, c, v, 0, nv);
                    } else if constexpr (EPI == kEpiStore) {
                        if (row_ok) store_row32(a.C, a.ldc, m, c, v, a.c_f32, nv);
                    } else {  // kEpiAccum
                        if (row_ok) {
                            float* p = a.acc + m * a.ld_acc + c;
                            if (!a.acc_first) {
                                if (nv == 32) {
#pragma unroll
                                    for (int q4 = 0; q4 < 8; ++q4) {
                                        const float4 o = reinterpret_cast<const float4*>(p)[q4];
                                        v[4 * q4] += o.x;
                                        v[4 * q4 + 1] += o.y;
                                        v[4 * q4 + 2] += o.z;
                                        v[4 * q4 + 3] += o.w;
                                    }
                                } else {
#pragma unroll
                                    for (int j = 0; j < 32; ++j)
                                        if (j < nv) v[j] += p[j];
                                }
                            }
                            if (a.acc_last)
                                store_row32(a.C, a.ldc, m, c, v, a.c_f32, nv);
                            else
                                store_row32(a.acc, a.ld_acc, m, c, v, 1, nv);
                        }
                    }
                }
                tc_fence_before();
                if constexpr (CG == 1)
                    mbar_arrive(tempty_bar(acc));
                else
                    mbar_arrive_cluster(lead_tempty0 + 8u * acc);
            }
            if constexpr (EPI == kEpiCeFwd) {
                if (ok && row_ok) a.part[(int64_t)un * a.M + m] = make_float4(st.m, st.s, st.t, zy);
            }
        }
        if (!ok) atomicOr(a.err, kErrTimeout);
    }

    tc_fence_before();
    // (a pair: neither CTA frees its tensor memory, or leaves, while the even
    // CTA's MMAs may still write the odd CTA's accumulator or the odd CTA's
    // epilogue may still arrive on the even CTA's barriers)
    if constexpr (CG == 2)
        cluster_sync();
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_cg<CG>(tmem_base, kTmemCols);
    }
}

// Merge of the forward partials, in unit order, one thread per row.
__global__ void __launch_bounds__(256) k_linear_merge(const float4* part, int64_t N, int64_t V,
                                                      int tile_cols_per_unit, int n_units,
                                                      const void* y_ptr, int tdt, float eps,
                                                      int64_t ignore, float* loss, float* lse,
                                                      unsigned int* err) {
    const RowOut out{loss, lse, nullptr, nullptr, err};
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < N;
         r += (int64_t)gridDim.x * blockDim.x) {
        const int64_t y = load_target(y_ptr, tdt, r);
        const int64_t uy = (y >= 0 && y < V) ? y / tile_cols_per_unit : -1;
        OnlineState st = empty_state();
        float zy = 0.f;
        for (int un = 0; un < n_units; ++un) {
            const float4 rec = part[(int64_t)un * N + r];
            const int64_t c0 = (int64_t)un * tile_cols_per_unit;
            const int64_t c1 = min(V, c0 + tile_cols_per_unit);
            OnlineState o;
            o.m = rec.x;
            o.s = rec.y;
            o.t = rec.z;
            o.k = (int)(c1 - c0);
            o.av = 0.f;
            o.ai = -1;
            merge<false>(st, o);
            if (un == uy) zy = rec.w;
        }
        finalize_row(st, zy, y, ignore, V, eps, out, r, false);
    }
}

// ---------------------------------------------------------------------------
// Host side.

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map of a row-major bf16 matrix (rows x cols, row stride ld elements)
// loaded in boxes of 64 columns x box_rows rows with 128-byte swizzle (the
// row of a box is 128 bytes, one swizzle row). Out-of-range elements read as
// zero.
static bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                     int box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// CTAs per output tile. The backward GEMMs run as pairs sharing 256 x 256
// tiles (measured 7.7% faster than single CTAs on the 8192 x 151,936 x 4096
// backward); the forward keeps one CTA per 128 x 256 tile, which measured
// 2.5% faster there. The maps of K-major B operands are cut into boxes of
// kBoxB rows, one CTA's share of a tile.
constexpr int kCgFwd = 1, kCgBwd = 2;
template <int CG>
constexpr int kBoxB = GemmCfg<CG>::kRowsB;

template <int EPI, int CG, bool AMN = false, bool BMN = false>
static cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, GemmArgs a, int sms,
                               cudaStream_t s) {
    constexpr int kCG = CG;
    using Cfg = GemmCfg<kCG>;
    auto kern = k_gemm<EPI, AMN, BMN, kCG>;
    cudaError_t e = ensure_smem_limit((const void*)kern, (int)Cfg::kSmem);
    if (e != cudaSuccess) return e;
    const WaitPolicy wp = wait_policy();
    a.wait_ns = wp.limit_ns;
    a.starve = wp.starve;
    a.n_mb = (a.M + Cfg::kTileM - 1) / Cfg::kTileM;
    a.n_nb = (a.Nn + kBN - 1) / kBN;
    a.nkb = (a.K + kBK - 1) / kBK;
    if (a.tiles_per_unit < 1) a.tiles_per_unit = 1;
    a.n_units_n = (a.n_nb + a.tiles_per_unit - 1) / a.tiles_per_unit;
    a.units = (int64_t)a.n_mb * a.n_units_n;
    if constexpr (kCG == 1) {
        const int grid = (int)(a.units < sms ? a.units : sms);
        kern<<<grid, kGemmThreads, Cfg::kSmem, s>>>(ta, tb, a);
        return cudaGetLastError();
    } else {
        // one pair per two SMs (one CTA per SM), persistent over the tiles
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = Cfg::kSmem;
        cfg.stream = s;
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = kCG;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int pairs_max = 0;
        e = max_active_clusters((const void*)kern, cfg, &pairs_max);
        if (e != cudaSuccess) return e;
        const int64_t pairs = a.units < pairs_max ? a.units : pairs_max;
        cfg.gridDim = dim3((unsigned)(pairs * kCG));
        return cudaLaunchKernelEx(&cfg, kern, ta, tb, a);
    }
}

// Vocabulary tiles per forward unit: a few, so the W tiles in use by all CTAs
// at once stay in L2 next to H.
static constexpr int kFwdTilesPerUnit = 4;
// Vocabulary columns per backward chunk (a multiple of the 256-column tile).
#ifndef CE_BWD_CHUNK
#define CE_BWD_CHUNK 8192
#endif
static constexpr int64_t kBwdChunk = CE_BWD_CHUNK;
static_assert(kBwdChunk % kBN == 0, "whole output tiles per chunk");

static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

static bool linear_shapes_ok(int64_t N, int64_t V, int64_t D, int64_t ld_h, int64_t ld_w) {
    return N >= 1 && V >= 1 && V <= INT32_MAX && D >= kBK && D % kBK == 0 && ld_h >= D &&
           ld_w >= D && ld_h % 8 == 0 && ld_w % 8 == 0 && N <= INT32_MAX;
}

static size_t fwd_ws(int64_t N, int64_t V) {
    const int64_t n_nb = (V + kBN - 1) / kBN;
    const int64_t units = (n_nb + kFwdTilesPerUnit - 1) / kFwdTilesPerUnit;
    return (size_t)units * (size_t)N * sizeof(float4);
}

// Backward workspace: one vocabulary chunk of the logits' gradient (bf16,
// row-major N x vc) and the float dH accumulator (N x D; not needed when dH
// itself is float).
struct BwdLayout {
    size_t off_g, off_acc, total;
    int64_t vc;
};

static BwdLayout bwd_layout(int64_t N, int64_t V, int64_t D) {
    BwdLayout L{};
    L.vc = V < kBwdChunk ? round_up(V, kBN) : kBwdChunk;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (size_t)round_up((int64_t)(off + bytes), 256);
        return o;
    };
    L.off_g = take((size_t)N * L.vc * 2);
    L.off_acc = take((size_t)N * D * 4);
    L.total = off;
    return L;
}

}  // namespace ceb

using namespace ceb;

extern "C" {

size_t linear_ce_workspace_size(int64_t N, int64_t V, int64_t D, int num_sms) {
    (void)num_sms;
    (void)D;
    if (N <= 0 || V <= 0) return 0;
    return fwd_ws(N, V);
}

ce_status linear_ce_forward(const void* H, int64_t ld_h, const void* W, int64_t ld_w,
                            const void* targets, ce_index_dtype tdt, int64_t N, int64_t V,
                            int64_t D, float label_smoothing, int64_t ignore_index, float* loss,
                            float* lse, void* workspace, size_t ws_bytes, void* cuda_stream) {
    if (!linear_shapes_ok(N, V, D, ld_h, ld_w)) return CE_EINVAL;
    if (tdt != CE_I32 && tdt != CE_I64) return CE_EINVAL;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (!H || !W || !targets || !loss || !lse) return CE_EINVAL;
    if ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(W)) % 16) return CE_EINVAL;
    const size_t need = fwd_ws(N, V);
    if (!workspace || ws_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 16)
        return CE_EWORKSPACE;
    unsigned int* err = error_word();
    if (!err) return CE_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    const int sms = device_sms(0);

    CUtensorMap ta, tb;
    if (!make_map(&ta, H, N, D, ld_h, kBM) || !make_map(&tb, W, V, D, ld_w, kBoxB<kCgFwd>))
        return CE_ECUDA;
    GemmArgs a{};
    a.M = (int)N;
    a.Nn = (int)V;
    a.K = (int)D;
    a.tiles_per_unit = kFwdTilesPerUnit;
    a.err = err;
    a.y = targets;
    a.tdt = tdt == CE_I32 ? 0 : 1;
    a.V = V;
    a.eps = label_smoothing;
    a.ignore = ignore_index;
    a.col_base = 0;
    a.part = static_cast<float4*>(workspace);
    if (launch_gemm<kEpiCeFwd, kCgFwd>(ta, tb, a, sms, s) != cudaSuccess) return CE_ECUDA;
    const int64_t n_nb = (V + kBN - 1) / kBN;
    const int n_units = (int)((n_nb + kFwdTilesPerUnit - 1) / kFwdTilesPerUnit);
    const int64_t mg = (N + 255) / 256;
    k_linear_merge<<<(int)(mg < (int64_t)sms * 8 ? mg : (int64_t)sms * 8), 256, 0, s>>>(
        static_cast<const float4*>(workspace), N, V, kFwdTilesPerUnit * kBN, n_units, targets,
        a.tdt, label_smoothing, ignore_index, loss, lse, err);
    return cudaGetLastError() == cudaSuccess ? CE_OK : CE_ECUDA;
}

size_t linear_ce_backward_workspace_size(int64_t N, int64_t V, int64_t D, int num_sms) {
    (void)num_sms;
    if (N <= 0 || V <= 0 || D <= 0) return 0;
    return bwd_layout(N, V, D).total;
}

ce_status linear_ce_backward(const float* grad_out, int64_t grad_stride, const void* H,
                             int64_t ld_h, const void* W, int64_t ld_w, const void* targets,
                             ce_index_dtype tdt, const float* lse, int64_t N, int64_t V,
                             int64_t D, float label_smoothing, int64_t ignore_index, void* dH,
                             ce_dtype dH_dt, void* dW, ce_dtype dW_dt, void* workspace,
                             size_t ws_bytes, void* cuda_stream) {
    if (!linear_shapes_ok(N, V, D, ld_h, ld_w)) return CE_EINVAL;
    if (tdt != CE_I32 && tdt != CE_I64) return CE_EINVAL;
    if ((dH_dt != CE_BF16 && dH_dt != CE_F32) || (dW_dt != CE_BF16 && dW_dt != CE_F32))
        return CE_EINVAL;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (!grad_out || !H || !W || !targets || !lse || !dH || !dW) return CE_EINVAL;
    if ((reinterpret_cast<uintptr_t>(H) | reinterpret_cast<uintptr_t>(W) |
         reinterpret_cast<uintptr_t>(dH) | reinterpret_cast<uintptr_t>(dW)) % 16)
        return CE_EINVAL;
    const BwdLayout L = bwd_layout(N, V, D);
    if (!workspace || ws_bytes < L.total || reinterpret_cast<uintptr_t>(workspace) % 256)
        return CE_EWORKSPACE;
    unsigned int* err = error_word();
    if (!err) return CE_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    const int sms = device_sms(0);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto* G = reinterpret_cast<__nv_bfloat16*>(ws + L.off_g);
    float* dH_acc = dH_dt == CE_F32 ? static_cast<float*>(dH) : reinterpret_cast<float*>(ws + L.off_acc);

    // H as the K-major A operand of GEMM 1 and as the MN-major B operand of
    // GEMM 2 (its rows are the reduction index there)
    CUtensorMap mH, mHmn;
    if (!make_map(&mH, H, N, D, ld_h, kBM) || !make_map(&mHmn, H, N, D, ld_h, kMnBox))
        return CE_ECUDA;

    const int64_t nchunks = (V + L.vc - 1) / L.vc;
    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t v0 = c * L.vc;
        const int64_t vcv = (V - v0) < L.vc ? (V - v0) : L.vc;  // valid columns
        const __nv_bfloat16* Wc = static_cast<const __nv_bfloat16*>(W) + v0 * ld_w;
        // GEMM 1: Z_c = H W_c^T, epilogue writes G_c (stream order keeps the
        // previous chunk's GEMMs, which read G_c, ahead of this overwrite)
        {
            CUtensorMap mWc;
            if (!make_map(&mWc, Wc, vcv, D, ld_w, kBoxB<kCgBwd>)) return CE_ECUDA;
            GemmArgs a{};
            a.M = (int)N;
            a.Nn = (int)vcv;
            a.K = (int)D;
            a.tiles_per_unit = 1;
            a.err = err;
            a.y = targets;
            a.tdt = tdt == CE_I32 ? 0 : 1;
            a.V = V;
            a.eps = label_smoothing;
            a.ignore = ignore_index;
            a.col_base = v0;
            a.g = grad_out;
            a.g_stride = grad_stride;
            a.lse = lse;
            a.G = G;
            a.ldG = L.vc;
            if (launch_gemm<kEpiCeGrad, kCgBwd>(mH, mWc, a, sms, s) != cudaSuccess) return CE_ECUDA;
        }
        // GEMM 2: dW[v0:v0+vcv] = G_c^T H (M = vcv, K = N): A is G_c read with
        // its vocabulary index contiguous, B is H read with D contiguous, both
        // MN-major. The maps stop at vcv columns, so the stale columns of the
        // last, narrower chunk read as zero.
        {
            CUtensorMap mGmn;
            if (!make_map(&mGmn, G, N, vcv, L.vc, kMnBox)) return CE_ECUDA;
            GemmArgs a{};
            a.M = (int)vcv;
            a.Nn = (int)D;
            a.K = (int)N;
            a.tiles_per_unit = 1;
            a.err = err;
            const int esz = dW_dt == CE_F32 ? 4 : 2;
            a.C = static_cast<uint8_t*>(dW) + (size_t)v0 * D * esz;
            a.ldc = D;
            a.c_f32 = dW_dt == CE_F32;
            // the smaller operand stays in L2 while the other streams: H (B)
            // when G_c (A, vcv x N) is the larger
            a.n_fast = vcv > D ? 1 : 0;
            if (launch_gemm<kEpiStore, kCgBwd, true, true>(mGmn, mHmn, a, sms, s) != cudaSuccess)
                return CE_ECUDA;
        }
        // GEMM 3: dH (+)= G_c W_c (K = vcv): A is G_c K-major, B is W_c read
        // with D contiguous (MN-major)
        {
            CUtensorMap mG, mWmn;
            if (!make_map(&mG, G, N, vcv, L.vc, kBM) || !make_map(&mWmn, Wc, vcv, D, ld_w, kMnBox))
                return CE_ECUDA;
            GemmArgs a{};
            a.M = (int)N;
            a.Nn = (int)D;
            a.K = (int)vcv;
            a.kA0 = 0;
            a.kB0 = 0;
            a.tiles_per_unit = 1;
            a.err = err;
            a.acc = dH_acc;
            a.ld_acc = D;
            a.acc_first = c == 0;
            a.acc_last = c == nchunks - 1;
            a.C = dH;
            a.ldc = D;
            a.c_f32 = dH_dt == CE_F32;
            // W_c (B, vcv x D) stays in L2 when G_c (A, N x vcv) is the larger
            a.n_fast = N > D ? 1 : 0;
            if (launch_gemm<kEpiAccum, kCgBwd, false, true>(mG, mWmn, a, sms, s) != cudaSuccess)
                return CE_ECUDA;
        }
    }
    return CE_OK;
}

}  // extern "C"
