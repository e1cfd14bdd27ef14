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
// exp(z - lse) is evaluated from the float pair (hi, lo) the forward writes
// (see RowGrad): z - hi is exact near the max, which keeps the softmax right
// at magnitudes where a float lse alone has lost the gap (equal logits at 1e8
// give [-1/2, 1/2], as MLX PR #4188 requires).
//
// dlogits may be the logits buffer itself: every element is loaded by the
// thread that later stores it, and the loads are plain coherent loads.
#include "ce_device.cuh"
#include "ce_launch.h"
#include "ce_sm100.cuh"

namespace ceb {

// Per-row constants of the VJP. With (hi, lo) the float pair of lse,
// exp(z - lse) = 2^((z - hi) log2 e - lo log2 e): z - hi is exact near the
// max (Sterbenz), so the gap survives at any magnitude, and the rest is one
// fma (c_lo = lo log2 e).
struct RowGrad {
    float g, c_hi, c_lo, c_eps, c_tgt;  // c_hi = hi
    int64_t y;
    bool zero, bad;
};

template <typename TI, typename TO, int VEC, int G, int U, int R>
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
    const float nan = __int_as_float(0x7fc00000);

    // a group takes R units per step: u, u + ngroups, ... (R > 1 for tiny rows)
    for (int64_t u0 = group; u0 < units; u0 += ngroups * R) {
        RowGrad rg[R];
        const TI* row[R];
        TO* drow[R];
        int64_t v0[R], v1[R];
        bool act[R], last[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int64_t u = u0 + (int64_t)i * ngroups;
            act[i] = u < units;
            const int64_t r = !act[i] ? 0 : (a.nchunks == 1 ? u : u / a.nchunks);
            const int64_t c = !act[i] ? 0 : (a.nchunks == 1 ? 0 : u - r * a.nchunks);
            row[i] = z + row_offset(a.lz, r, a.N);
            drow[i] = dz + row_offset(a.ld, r, a.N);
            v0[i] = c * a.vec_per_chunk;
            v1[i] = act[i] ? min(nvec, v0[i] + a.vec_per_chunk) : v0[i];
            last[i] = act[i] && c == a.nchunks - 1;
            RowGrad& q = rg[i];
            q.y = act[i] ? load_target(a.y, a.tdt, row_offset(a.ly, r, a.N)) : a.ignore;
            q.zero = q.y == a.ignore;
            q.bad = !q.zero && (q.y < 0 || q.y >= a.V);
            q.g = 0.f;
            q.c_hi = q.c_lo = q.c_eps = q.c_tgt = 0.f;
            if (act[i] && !q.zero && !q.bad) {
                q.g = a.g[r * a.g_stride];
                const float hi = a.lse[r];
                const float lo = a.lse_lo ? a.lse_lo[r] : 0.f;
                q.c_hi = hi;
                q.c_lo = lo * kLog2e;
                q.c_eps = q.g * a.eps * inv_v;
                q.c_tgt = q.g * (1.f - a.eps);
            }
            if (act[i] && q.bad && gl == 0 && c == 0) atomicOr(a.err, 1u);
        }

        // steps of U vectors per lane; every unit of the step is loaded before
        // any is computed
        int64_t span = 0;
#pragma unroll
        for (int i = 0; i < R; ++i) span = max(span, v1[i] - v0[i]);
        for (int64_t off = 0; off < span; off += (int64_t)G * U) {
            float v[R][U][VEC];
            bool ok[R][U];
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const bool need = act[i] && !rg[i].zero && !rg[i].bad;
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    const int64_t vi = v0[i] + off + q * G + gl;
                    ok[i][q] = act[i] && vi < v1[i];
                    if (ok[i][q] && need) load_vec_coherent<TI, VEC>(row[i], vi * VEC, a.lz.s_col, v[i][q]);
                }
            }
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const RowGrad& q = rg[i];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!ok[i][u]) continue;
                    const int64_t col0 = (v0[i] + off + u * G + gl) * VEC;
                    float o[VEC];
                    if (q.zero || q.bad) {
#pragma unroll
                        for (int e = 0; e < VEC; ++e) o[e] = q.bad ? nan : 0.f;
                    } else {
                        // scalar arithmetic here: registers, not issue slots,
                        // bound this register-staged kernel
#pragma unroll
                        for (int e = 0; e < VEC; ++e) {
                            const float p = ex2(fmaf(v[i][u][e] - q.c_hi, kLog2e, -q.c_lo));
                            o[e] = fmaf(q.g, p, -q.c_eps);
                        }
                        const int64_t dy = q.y - col0;
                        if (dy >= 0 && dy < VEC) {
#pragma unroll
                            for (int e = 0; e < VEC; ++e)
                                if (e == dy) o[e] -= q.c_tgt;
                        }
                    }
                    store_vec<TO, VEC>(drow[i], col0, a.ld.s_col, o);
                }
            }
        }
        // ragged tail: the last V % VEC columns of the last chunk
#pragma unroll
        for (int i = 0; i < R; ++i) {
            if (!last[i]) continue;
            const RowGrad& q = rg[i];
            for (int t = gl; t < tail; t += G) {
                const int64_t col = nvec * VEC + t;
                float d;
                if (q.zero || q.bad) {
                    d = q.bad ? nan : 0.f;
                } else {
                    float x;
                    load_vec_coherent<TI, 1>(row[i], col, 1, &x);
                    d = fmaf(q.g, ex2(fmaf(x - q.c_hi, kLog2e, -q.c_lo)), -q.c_eps);
                    if (col == q.y) d -= q.c_tgt;
                }
                cvt_store1(drow[i] + col, d);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Tiny rows (one or two 16-byte vectors, no ragged tail): one lane per row
// and R rows per lane per step, with every load of the step issued before
// any is used, and the warp's next step of rows sent into L2 ahead of time
// when the rows lie back to back. The gradient is the one k_bwd_rows forms.
template <typename TI, typename TO, int NV, int R, int MINB>
__global__ void __launch_bounds__(256, MINB) k_bwd_tiny(BwdArgs a) {
    constexpr int VEC = ElemTraits<TI>::kVec;
    constexpr int n = NV * VEC;
    const TI* z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float inv_v = 1.f / (float)a.V;
    const float nan = __int_as_float(0x7fc00000);
    const bool dense = a.lz.inner >= a.N && a.lz.s_inner == (int64_t)n;

    for (int64_t base = warp * 32 * R; base < a.N; base += nwarps * 32 * R) {
        if (dense && lane == 0) {
            const int64_t bn = base + nwarps * 32 * R;
            if (bn < a.N) {
                const int64_t rows = min((int64_t)32 * R, a.N - bn);
                sm100::bulk_prefetch_l2(z + bn * n, (uint32_t)(rows * n * sizeof(TI)));
            }
        }
        uint4 w[R][NV];
        int64_t y[R];
        float hi[R], lo[R], g[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            y[k] = a.ignore;
            hi[k] = lo[k] = g[k] = 0.f;
            if (r < a.N) {
                const TI* row = z + row_offset(a.lz, r, a.N);
                y[k] = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
                hi[k] = a.lse[r];
                lo[k] = a.lse_lo ? a.lse_lo[r] : 0.f;
                g[k] = a.g[r * a.g_stride];
#pragma unroll
                for (int v = 0; v < NV; ++v) w[k][v] = *(reinterpret_cast<const uint4*>(row) + v);
            }
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int64_t r = base + 32 * k + lane;
            if (r >= a.N) continue;
            const bool zero = y[k] == a.ignore;
            const bool bad = !zero && (y[k] < 0 || y[k] >= a.V);
            const int yc = (zero || bad) ? -1 : (int)y[k];  // column of the target, if any
            const float c_lo = lo[k] * kLog2e, c_eps = g[k] * a.eps * inv_v, c_tgt = g[k] * (1.f - a.eps);
            TO* drow = dz + row_offset(a.ld, r, a.N);
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                float x[VEC], o[VEC];
                unpack_words<TI>(w[k][v], x);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float p = ex2(fmaf(x[e] - hi[k], kLog2e, -c_lo));
                    o[e] = (zero || bad) ? (bad ? nan : 0.f) : fmaf(g[k], p, -c_eps);
                    if (yc == v * VEC + e) o[e] -= c_tgt;
                }
                store_vec<TO, VEC>(drow, v * VEC, 1, o);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Short rows: G lanes per row, 32/G rows per warp, U vectors per lane per
// step. Every load of a row (target, lse pair, g and the logits of the first
// step) is issued before any of them is used, so a group waits on memory
// once per row; ignored rows read their logits too (a few percent more bytes
// for a shorter dependency chain) and write zeros.
template <typename TI, typename TO, int VEC, int G, int U, int MINB>
__global__ void __launch_bounds__(256, MINB) k_bwd_rows(BwdArgs a) {
    const TI* z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int lane = threadIdx.x & 31;
    const int gl = lane & (G - 1);
    constexpr int kRowsPerStep = 32 / G;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const float inv_v = 1.f / (float)a.V;
    const float nan = __int_as_float(0x7fc00000);

    for (int64_t base = warp * kRowsPerStep; base < a.N; base += nwarps * kRowsPerStep) {
        const int64_t r = base + lane / G;
        const bool act = r < a.N;
        const TI* row = z;
        TO* drow = dz;
        int64_t y = a.ignore;
        float hi = 0.f, lo = 0.f, g = 0.f;
        if (act) {
            row = z + row_offset(a.lz, r, a.N);
            drow = dz + row_offset(a.ld, r, a.N);
            y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
            hi = a.lse[r];
            lo = a.lse_lo ? a.lse_lo[r] : 0.f;
            g = a.g[r * a.g_stride];
        }
        for (int64_t vb = 0; vb < nvec; vb += (int64_t)G * U) {
            float v[U][VEC];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t vi = vb + u * G + gl;
                ok[u] = act && vi < nvec;
                if (ok[u]) load_vec_coherent<TI, VEC>(row, vi * VEC, a.lz.s_col, v[u]);
            }
            const bool zero = y == a.ignore;
            const bool bad = !zero && (y < 0 || y >= a.V);
            const int yc = (zero || bad) ? -1 : (int)y;
            const float c_lo = lo * kLog2e, c_eps = g * a.eps * inv_v, c_tgt = g * (1.f - a.eps);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!ok[u]) continue;
                const int col0 = (int)((vb + u * G + gl) * VEC);
                float o[VEC];
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float p = ex2(fmaf(v[u][e] - hi, kLog2e, -c_lo));
                    o[e] = (zero || bad) ? (bad ? nan : 0.f) : fmaf(g, p, -c_eps);
                }
                const unsigned dy = (unsigned)(yc - col0);
                if (dy < (unsigned)VEC) {
#pragma unroll
                    for (int e = 0; e < VEC; ++e)
                        if ((unsigned)e == dy) o[e] -= c_tgt;
                }
                store_vec<TO, VEC>(drow, col0, a.ld.s_col, o);
            }
        }
        if (act) {
            const bool zero = y == a.ignore;
            const bool bad = !zero && (y < 0 || y >= a.V);
            for (int t = gl; t < tail; t += G) {
                const int64_t col = nvec * VEC + t;
                float d;
                if (zero || bad) {
                    d = bad ? nan : 0.f;
                } else {
                    float x;
                    load_vec_coherent<TI, 1>(row, col, 1, &x);
                    d = fmaf(g, ex2(fmaf(x - hi, kLog2e, -lo * kLog2e)), -g * a.eps * inv_v);
                    if (col == y) d -= g * (1.f - a.eps);
                }
                cvt_store1(drow + col, d);
            }
            if (bad && gl == 0) atomicOr(a.err, 1u);
        }
    }
}

// ---------------------------------------------------------------------------
// dz of the vectors p * 32 + lane (p < P; all of them when FULL) of one
// chunk staged in shared memory; TGT: the target column lies in the chunk,
// dyc columns after its start.
template <typename TI, typename TO, int P, bool FULL, bool TGT>
__device__ __forceinline__ void ring_grad(const uint4* buf, int nvc, int lane, TO* dchunk, float2 nh,
                                          float2 l2, float2 nl, float2 gg, float2 ne, float c_tgt,
                                          int dyc) {
    constexpr int VEC = ElemTraits<TI>::kVec;
#pragma unroll
    for (int p = 0; p < P; ++p) {
        const int vi = p * 32 + lane;
        if (!FULL && vi >= nvc) continue;
        float v[VEC], o[VEC];
        unpack_words<TI>(buf[vi], v);
#pragma unroll
        for (int e = 0; e < VEC; e += 2) {
            float2 d = __fadd2_rn(make_float2(v[e], v[e + 1]), nh);
            d = __ffma2_rn(d, l2, nl);
            const float2 pp = make_float2(ex2(d.x), ex2(d.y));
            const float2 r2 = __ffma2_rn(gg, pp, ne);
            o[e] = r2.x;
            o[e + 1] = r2.y;
        }
        if constexpr (TGT) {
            const int dy = dyc - vi * VEC;
#pragma unroll
            for (int e = 0; e < VEC; ++e)
                if (dy == e) o[e] -= c_tgt;
        }
        store_vec<TO, VEC>(dchunk, (int64_t)vi * VEC, 1, o);
    }
}

// ---------------------------------------------------------------------------
// Long rows through per-warp bulk-copy rings. A unit is (row, chunk of
// vec_per_chunk vectors) and belongs to one warp; the warp's lane 0 keeps a
// ring of kBRingStages 2 KB buffers filled with 1-D bulk copies issued ahead
// across its units, and the lanes turn each buffer into dz with 16-byte
// stores. The bytes in flight per SM come from the rings, not the registers.
constexpr int kBRingWarps = 8;
constexpr int kBRingStages = 6;
constexpr int kBRingVecs = 128;
constexpr size_t kBRingSmem = (size_t)kBRingWarps * kBRingStages * kBRingVecs * 16;

struct BRingCursor {
    int64_t u;
    int64_t j, nel;
    const uint8_t* src;
    int64_t nv;
    __device__ __forceinline__ void load_unit(const BwdArgs& a, int64_t units, int64_t nvec,
                                              int vec) {
        nel = 0;
        if (u >= units) return;
        const int64_t r = a.nchunks == 1 ? u : u / a.nchunks;
        const int64_t c = a.nchunks == 1 ? 0 : u - r * a.nchunks;
        const int64_t v0 = c * a.vec_per_chunk;
        const int64_t v1 = min(nvec, v0 + a.vec_per_chunk);
        nv = v1 > v0 ? v1 - v0 : 0;
        nel = (nv + kBRingVecs - 1) / kBRingVecs;
        src = reinterpret_cast<const uint8_t*>(a.z) +
              (row_offset(a.lz, r, a.N) + v0 * vec) * (16 / vec);
    }
    __device__ __forceinline__ void settle(const BwdArgs& a, int64_t units, int64_t nvec, int vec,
                                           int64_t stride) {
        while (u < units && j >= nel) {
            u += stride;
            j = 0;
            load_unit(a, units, nvec, vec);
        }
    }
    __device__ __forceinline__ bool valid(int64_t units) const { return u < units; }
    __device__ __forceinline__ uint32_t bytes() const {
        const int64_t left = nv - j * kBRingVecs;
        return (uint32_t)((left < kBRingVecs ? left : kBRingVecs) * 16);
    }
};

template <typename TI, typename TO>
__global__ void __launch_bounds__(kBRingWarps * 32, 2) k_bwd_ring(BwdArgs a) {
    using namespace sm100;
    constexpr int VEC = ElemTraits<TI>::kVec;
    constexpr int kPerLane = kBRingVecs / 32;
    extern __shared__ __align__(128) uint8_t ring_smem[];
    __shared__ __align__(8) uint64_t full_bar[kBRingWarps][kBRingStages];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const TI* z = reinterpret_cast<const TI*>(a.z);
    TO* dz = reinterpret_cast<TO*>(a.dz);
    const int64_t nvec = a.V / VEC;
    const int tail = (int)(a.V - nvec * VEC);
    const int64_t units = a.N * a.nchunks;
    const int64_t gw = (int64_t)blockIdx.x * kBRingWarps + wid;
    const int64_t stride = (int64_t)gridDim.x * kBRingWarps;
    const float inv_v = 1.f / (float)a.V;
    const float nan = __int_as_float(0x7fc00000);
    uint8_t* ring = ring_smem + (size_t)wid * kBRingStages * kBRingVecs * 16;

    if (lane == 0)
        for (int q = 0; q < kBRingStages; ++q) mbar_init(smem_u32(&full_bar[wid][q]), 1);
    if (tid == 0) abort_flag = 0;
    if (lane == 0) mbar_fence_init();
    __syncthreads();

    BRingCursor iss;
    iss.u = gw;
    iss.j = 0;
    iss.load_unit(a, units, nvec, VEC);
    iss.settle(a, units, nvec, VEC, stride);
    int64_t issued = 0;
    for (int q = 0; q < kBRingStages && iss.valid(units); ++q) {
        if (lane == 0) {
            const uint32_t bar = smem_u32(&full_bar[wid][q]);
            mbar_expect_tx(bar, iss.bytes());
            bulk_load(smem_u32(ring + q * kBRingVecs * 16), iss.src + iss.j * kBRingVecs * 16,
                      iss.bytes(), bar);
        }
        ++issued;
        ++iss.j;
        iss.settle(a, units, nvec, VEC, stride);
    }

    int64_t consumed = 0, waited = 0;
    bool dead = false;
    for (int64_t u = gw; u < units; u += stride) {
        const int64_t r = a.nchunks == 1 ? u : u / a.nchunks;
        const int64_t c = a.nchunks == 1 ? 0 : u - r * a.nchunks;
        const int64_t v0 = c * a.vec_per_chunk;
        const int64_t v1 = min(nvec, v0 + a.vec_per_chunk);
        const int64_t nv = v1 > v0 ? v1 - v0 : 0;
        const int64_t nel = (nv + kBRingVecs - 1) / kBRingVecs;
        const TI* row = z + row_offset(a.lz, r, a.N);
        TO* drow = dz + row_offset(a.ld, r, a.N);
        RowGrad q;
        q.y = load_target(a.y, a.tdt, row_offset(a.ly, r, a.N));
        q.zero = q.y == a.ignore;
        q.bad = !q.zero && (q.y < 0 || q.y >= a.V);
        q.g = 0.f;
        q.c_hi = q.c_lo = q.c_eps = q.c_tgt = 0.f;
        if (!q.zero && !q.bad) {
            q.g = a.g[r * a.g_stride];
            const float hi = a.lse[r];
            const float lo = a.lse_lo ? a.lse_lo[r] : 0.f;
            q.c_hi = hi;
            q.c_lo = lo * kLog2e;
            q.c_eps = q.g * a.eps * inv_v;
            q.c_tgt = q.g * (1.f - a.eps);
        }
        if (q.bad && lane == 0 && c == 0) atomicOr(a.err, 1u);
        const float2 l2 = make_float2(kLog2e, kLog2e);
        const float2 nh = make_float2(-q.c_hi, -q.c_hi);
        const float2 nl = make_float2(-q.c_lo, -q.c_lo);
        const float2 gg = make_float2(q.g, q.g);
        const float2 ne = make_float2(-q.c_eps, -q.c_eps);

        for (int64_t j = 0; j < nel; ++j) {
            const int stage = (int)(consumed % kBRingStages);
            const uint32_t bar = smem_u32(&full_bar[wid][stage]);
            if (!dead) {
                if (mbar_wait(bar, (uint32_t)((consumed / kBRingStages) & 1), &abort_flag))
                    ++waited;
                else
                    dead = true;
            }
            if (!dead) {
                const int64_t left = nv - j * kBRingVecs;
                const int nvc = (int)(left < kBRingVecs ? left : kBRingVecs);
                const uint4* buf = reinterpret_cast<const uint4*>(ring + stage * kBRingVecs * 16);
                const int64_t cc = (v0 + j * kBRingVecs) * VEC;  // first column of the chunk
                TO* dchunk = drow + cc;
                // the chunk that holds the target (one per row) takes its own
                // warp-uniform branch; the others pay nothing for its term
                const int64_t dyc = q.y - cc;
                if (q.zero || q.bad) {
                    float o[VEC];
#pragma unroll
                    for (int e = 0; e < VEC; ++e) o[e] = q.bad ? nan : 0.f;
#pragma unroll
                    for (int p = 0; p < kPerLane; ++p) {
                        const int vi = p * 32 + lane;
                        if (vi < nvc) store_vec<TO, VEC>(dchunk, (int64_t)vi * VEC, 1, o);
                    }
                } else if (dyc >= 0 && dyc < (int64_t)nvc * VEC) {
                    ring_grad<TI, TO, kPerLane, false, true>(buf, nvc, lane, dchunk, nh, l2, nl, gg, ne,
                                                            q.c_tgt, (int)dyc);
                } else if (nvc == kBRingVecs) {
                    ring_grad<TI, TO, kPerLane, true, false>(buf, nvc, lane, dchunk, nh, l2, nl, gg, ne,
                                                            q.c_tgt, 0);
                } else {
                    ring_grad<TI, TO, kPerLane, false, false>(buf, nvc, lane, dchunk, nh, l2, nl, gg, ne,
                                                             q.c_tgt, 0);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (iss.valid(units) && !dead) {
                if (lane == 0) {
                    mbar_expect_tx(bar, iss.bytes());
                    bulk_load(smem_u32(ring + stage * kBRingVecs * 16),
                              iss.src + iss.j * kBRingVecs * 16, iss.bytes(), bar);
                }
                ++issued;
            }
            ++iss.j;
            iss.settle(a, units, nvec, VEC, stride);
            ++consumed;
        }
        // ragged tail of the row, in its last chunk
        if (c == a.nchunks - 1) {
            for (int t = lane; t < tail; t += 32) {
                const int64_t col = nvec * VEC + t;
                float d;
                if (q.zero || q.bad) {
                    d = q.bad ? nan : 0.f;
                } else {
                    float x;
                    load_vec_coherent<TI, 1>(row, col, 1, &x);
                    d = fmaf(q.g, ex2(fmaf(x - q.c_hi, kLog2e, -q.c_lo)), -q.c_eps);
                    if (col == q.y) d -= q.c_tgt;
                }
                cvt_store1(drow + col, d);
            }
        }
    }
    if (dead || abort_flag) {
        if (lane == 0) {
            atomicOr(a.err, kErrTimeout);
            volatile int never = 0;
            for (int64_t e = waited; e < issued; ++e)
                mbar_wait(smem_u32(&full_bar[wid][e % kBRingStages]),
                          (uint32_t)((e / kBRingStages) & 1), &never);
        }
    }
}

template <typename TI, typename TO>
static cudaError_t launch_bwd_ring(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
    cudaError_t e = ensure_smem_limit((const void*)k_bwd_ring<TI, TO>, (int)kBRingSmem);
    if (e != cudaSuccess) return e;
    k_bwd_ring<TI, TO><<<p.grid, kBRingWarps * 32, kBRingSmem, s>>>(a);
    return cudaGetLastError();
}

template <typename TI, typename TO, int VEC>
static cudaError_t launch_bwd_v(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
#define CEB_BWD(GG, UU, RR)                                              \
    if (p.G == GG && p.U == UU && p.R == RR) {                           \
        k_bwd<TI, TO, VEC, GG, UU, RR><<<p.grid, 256, 0, s>>>(a);        \
        return cudaGetLastError();                                       \
    }
    // long rows without a bulk-copy ring: one warp per (row, chunk) unit
    constexpr int kU = VEC == 1 ? 8 : 4;
    CEB_BWD(32, kU, 1)
#undef CEB_BWD
    return cudaErrorInvalidValue;
}

template <typename TI, typename TO, int VEC>
static cudaError_t launch_bwd_rows(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
    constexpr int kU = VEC == 1 ? 8 : 32 / VEC;
    constexpr int kMinB = sizeof(TI) == 4 ? 3 : 2;
#define CEB_BWDR(GG, UU)                                                   \
    if (p.G == GG && p.U == UU) {                                          \
        k_bwd_rows<TI, TO, VEC, GG, UU, kMinB><<<p.grid, 256, 0, s>>>(a);  \
        return cudaGetLastError();                                         \
    }
    if (p.G == 1 && p.U == 2) {  // tiny rows: latency-bound, so as many warps as fit
        k_bwd_rows<TI, TO, VEC, 1, 2, sizeof(TI) == 4 ? 6 : 4><<<p.grid, 256, 0, s>>>(a);
        return cudaGetLastError();
    }
    CEB_BWDR(1, kU)
    CEB_BWDR(2, kU)
    CEB_BWDR(4, kU)
    CEB_BWDR(8, kU)
    CEB_BWDR(16, kU)
    CEB_BWDR(32, kU)
#undef CEB_BWDR
    return cudaErrorInvalidValue;
}

template <typename TI, typename TO>
static cudaError_t launch_bwd_t(const BwdPlan& p, const BwdArgs& a, cudaStream_t s) {
    if (p.tiny) {
        // register budgets: 64 per thread for one vector per row, 85 for two
        if (p.U == 1)
            k_bwd_tiny<TI, TO, 1, kTinyRows, 4><<<p.grid, 256, 0, s>>>(a);
        else
            k_bwd_tiny<TI, TO, 2, kTinyRows, 3><<<p.grid, 256, 0, s>>>(a);
        return cudaGetLastError();
    }
    if (p.ring) return launch_bwd_ring<TI, TO>(p, a, s);
    if (p.rows) {
        if (p.vec == 1) return launch_bwd_rows<TI, TO, 1>(p, a, s);
        return launch_bwd_rows<TI, TO, ElemTraits<TI>::kVec>(p, a, s);
    }
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
