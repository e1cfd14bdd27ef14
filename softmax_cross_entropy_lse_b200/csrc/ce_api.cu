// C ABI of the fused softmax cross-entropy library: argument validation,
// workspace sizing, kernel planning and launches. No allocation, no
// synchronisation on the hot path.
#include <atomic>
#include <mutex>
#include <vector>

#include "ce_b200.h"
#include "ce_launch.h"
#include "ce_linear.h"
#include "ce_sm100.cuh"

namespace ceb {

// One error word per device; kernels receive its address as an argument.
static __device__ unsigned int g_ce_error_word;

static constexpr int kMaxDevices = 64;
static std::mutex g_dev_mutex;
static unsigned int* g_err_ptr[kMaxDevices];
static int g_num_sms[kMaxDevices];

static int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

unsigned int* error_word() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ce_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned int*>(p);
    }
    return g_err_ptr[dev];
}

// SM count of device `dev`, cached; the caller holds g_dev_mutex.
static int device_sms_locked(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (!g_num_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

int device_sms(int num_sms) {
    if (num_sms > 0) return num_sms;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    return device_sms_locked(dev);
}

// Settings of the testing hook ce_testing_set_wait.
static std::atomic<unsigned long long> g_wait_limit_ns{0};  // 0: the default
static std::atomic<int> g_wait_starve{0};

WaitPolicy wait_policy() {
    const unsigned long long ns = g_wait_limit_ns.load(std::memory_order_relaxed);
    return WaitPolicy{ns ? ns : sm100::kWaitTimeoutNs, g_wait_starve.load(std::memory_order_relaxed)};
}

// (kernel, device) pairs whose shared-memory limit has been raised, with the
// bytes it was raised to.
struct SmemLimit {
    const void* kernel;
    int device, bytes;
};
static std::vector<SmemLimit> g_smem_limits;

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    for (const SmemLimit& l : g_smem_limits)
        if (l.kernel == kernel && l.device == dev && l.bytes >= bytes) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    g_smem_limits.push_back(SmemLimit{kernel, dev, bytes});
    return cudaSuccess;
}

struct ClusterOcc {
    const void* kernel;
    int device, clusters;
};
static std::vector<ClusterOcc> g_cluster_occ;

cudaError_t max_active_clusters(const void* kernel, const cudaLaunchConfig_t& cfg, int* clusters) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    for (const ClusterOcc& o : g_cluster_occ)
        if (o.kernel == kernel && o.device == dev) {
            *clusters = o.clusters;
            return cudaSuccess;
        }
    cudaLaunchConfig_t c = cfg;
    c.gridDim = dim3((unsigned)(cfg.attrs && cfg.numAttrs ? cfg.attrs[0].val.clusterDim.x : 1) *
                     (unsigned)device_sms_locked(dev));
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kernel, &c);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    g_cluster_occ.push_back(ClusterOcc{kernel, dev, n});
    *clusters = n;
    return cudaSuccess;
}

int elem_size(int dt) { return dt == CE_F32 ? 4 : 2; }

// Byte range [lo, hi) that a layout can touch for N rows of V columns: a
// conservative box over the outer, inner and column index ranges.
struct Extent {
    uintptr_t lo, hi;
};

static Extent layout_extent(const void* base, const Layout& L, int64_t N, int64_t V, int esz) {
    const int64_t nouter = (N + L.inner - 1) / L.inner;
    const int64_t ninner = N < L.inner ? N : L.inner;
    int64_t mn = 0, mx = 0;
    auto span = [&](int64_t count, int64_t stride) {
        if (count <= 1) return;
        const int64_t d = (count - 1) * stride;
        if (d < 0) mn += d; else mx += d;
    };
    span(nouter, L.s_outer);
    span(ninner, L.s_inner);
    span(V, L.s_col);
    const uintptr_t b = reinterpret_cast<uintptr_t>(base);
    return {b + (uintptr_t)(mn * esz), b + (uintptr_t)((mx + 1) * esz)};
}

static Extent flat_extent(const void* base, int64_t count, int esz) {
    const uintptr_t b = reinterpret_cast<uintptr_t>(base);
    return {b, b + (uintptr_t)(count * esz)};
}

static bool overlap(const Extent& a, const Extent& b) { return a.lo < b.hi && b.lo < a.hi; }

// True when every row starts on a 16-byte boundary and columns are unit-stride.
static bool vectorizable(const void* base, const Layout& L, int64_t N, int esz) {
    if (L.s_col != 1) return false;
    if (reinterpret_cast<uintptr_t>(base) % 16) return false;
    if (N > L.inner && (L.s_outer * esz) % 16) return false;
    if (N > 1 && L.inner > 1 && (L.s_inner * esz) % 16) return false;
    return true;
}

static Layout to_layout(const ce_layout& l) { return Layout{l.inner, l.s_outer, l.s_inner, l.s_col}; }

static bool layout_ok(const ce_layout& l) { return l.inner >= 1; }

// ---- forward planning --------------------------------------------------------
static constexpr int kPackedMaxRowBytes = 4096;
static constexpr int64_t kMinSplitVecs = 2048;  // one full step of a 512-thread CTA x 4 vectors

static int packed_lanes(int64_t nvec) {
    int G = 1;
    while (G < 32 && nvec > 8 * (int64_t)G) G *= 2;
    return G;
}

static bool use_packed(int64_t V, int esz) { return V * esz <= kPackedMaxRowBytes; }

// Number of vocabulary splits per row for the CTA kernel: the smallest power
// of two whose unit count fills the machine's CTA slots to >= 90% in the last
// wave, keeping every split at least one full CTA step long.
static int plan_splits(int64_t N, int64_t V, int esz, int sms) {
    if (use_packed(V, esz) || N <= 0) return 1;
    const int64_t nvec = V / (16 / esz);
    const int64_t slots = (int64_t)sms * 2;
    const int64_t max_splits = nvec / kMinSplitVecs > 1 ? nvec / kMinSplitVecs : 1;
    int best = 1;
    double best_eff = -1.0;
    for (int64_t s = 1; s <= 256 && s <= max_splits; s *= 2) {
        const int64_t units = N * s;
        const int64_t waves = (units + slots - 1) / slots;
        const double eff = (double)units / (double)(waves * slots);
        if (eff >= 0.9) return (int)s;
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = (int)s;
        }
    }
    return best;
}

static FwdPlan plan_forward(int64_t N, int64_t V, int esz, bool vec_ok, int sms) {
    FwdPlan p{};
    const int vecw = 16 / esz;
    p.vec = vec_ok ? vecw : 1;
    p.splits = 1;
    p.vec_per_split = 0;
    if (vec_ok && V % vecw == 0 && V / vecw <= 2) {
        // one or two whole vectors per row: a lane per row
        p.kind = FwdPlan::kTiny;
        p.G = 1;
        p.U = (int)(V / vecw);
        p.R = kTinyRows;
        const int64_t rows_per_block = 256 * (int64_t)kTinyRows;
        const int64_t want = (N + rows_per_block - 1) / rows_per_block;
        const int64_t cap = (int64_t)sms * (p.U == 1 ? 5 : 4);  // every block resident
        p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
        return p;
    }
    if (use_packed(V, esz) || (!vec_ok && V <= 256)) {
        p.kind = FwdPlan::kPacked;
        const int64_t nvec = V / p.vec;
        p.G = packed_lanes(nvec);
        p.U = (p.G == 1 && nvec <= 2) ? 2 : (esz == 4 ? 8 : 4);
        p.R = 1;
        const int64_t rows_per_block = 8 * (32 / p.G) * p.R;
        const int64_t want = (N + rows_per_block - 1) / rows_per_block;
        const int64_t cap = (int64_t)sms * 16;
        p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
        // whole-vector 4-byte rows that one step covers: pipelined through
        // shared memory, three resident blocks per SM, every block resident;
        // only when every warp gets at least two row groups (with fewer there
        // is nothing to overlap, and the kernel above takes the batch in one
        // wave of up to four blocks per SM)
        const int64_t capp = (int64_t)sms * 3;
        if (vec_ok && esz == 4 && p.G >= 2 && V % p.vec == 0 && nvec <= (int64_t)p.G * 8 &&
            want >= 2 * capp) {
            p.pipe = 1;
            p.grid = (int)capp;
        }
        return p;
    }
    p.kind = FwdPlan::kCta;
    // 2-byte rows fold at twice the elements per byte: their loads go through
    // bulk-copy rings so that bytes in flight do not depend on registers;
    // 4-byte rows keep register-staged 16-byte loads, which measured faster
    p.ring = (vec_ok && esz == 2) ? 1 : 0;
    p.splits = plan_splits(N, V, esz, sms);
    const int64_t nvec = V / p.vec;
    int64_t vps = (nvec + p.splits - 1) / p.splits;
    if (vps < 1) vps = 1;
    p.splits = (int)((nvec + vps - 1) / vps);
    if (p.splits < 1) p.splits = 1;
    p.vec_per_split = vps;
    const int64_t units = N * p.splits;
    const int64_t cap = (int64_t)sms * (p.ring ? 3 : 2);
    p.grid = (int)(units < cap ? units : cap);
    const int64_t mg = (N + 255) / 256;
    p.merge_grid = (int)(mg < (int64_t)sms * 8 ? mg : (int64_t)sms * 8);
    if (p.merge_grid < 1) p.merge_grid = 1;
    return p;
}

static size_t forward_workspace(int64_t N, int64_t V, int esz, int sms) {
    const int splits = plan_splits(N, V, esz, sms);
    if (splits <= 1) return 0;
    // the realised split count can only shrink (vectors per split rounded up)
    return (size_t)splits * (size_t)N * sizeof(float4);
}

// ---- backward planning -------------------------------------------------------
static constexpr int64_t kBwdChunkVecs = 2048;

static BwdPlan plan_backward(int64_t N, int64_t V, int esz_in, bool vec_ok, int sms,
                             int64_t* nchunks, int64_t* vpc) {
    BwdPlan p{};
    p.vec = vec_ok ? 16 / esz_in : 1;
    const int64_t nvec = V / p.vec;
    p.R = 1;
    p.ring = 0;
    p.rows = 0;
    const int kU = p.vec == 1 ? 8 : 32 / p.vec;
    if (vec_ok && V % p.vec == 0 && nvec <= 2) {
        // one or two whole vectors per row: a lane per row, every block resident
        p.tiny = 1;
        p.G = 1;
        p.U = (int)nvec;
        *nchunks = 1;
        *vpc = nvec;
        const int64_t rows_per_block = 256 * (int64_t)kTinyRows;
        const int64_t want = (N + rows_per_block - 1) / rows_per_block;
        const int64_t cap = (int64_t)sms * (p.U == 1 ? 4 : 3);
        p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
        return p;
    }
    if (nvec <= 256) {
        p.rows = 1;
        p.G = packed_lanes(nvec);
        p.U = (p.G == 1 && nvec <= 2) ? 2 : kU;
        *nchunks = 1;
        *vpc = nvec > 0 ? nvec : 1;
    } else {
        // long rows: one warp per (row, chunk) unit; aligned 2-byte rows stream
        // through bulk-copy rings, other layouts through register loads
        p.G = 32;
        p.U = p.vec == 1 ? 8 : 4;
        p.ring = (vec_ok && esz_in == 2) ? 1 : 0;
        *vpc = kBwdChunkVecs;
        *nchunks = (nvec + kBwdChunkVecs - 1) / kBwdChunkVecs;
    }
    if (p.ring) {
        const int64_t want = (N * *nchunks + 7) / 8;  // 8 warps per CTA
        const int64_t cap = (int64_t)sms * 2;
        p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
        return p;
    }
    const int64_t groups_per_block = 256 / p.G;
    const int64_t want = (N * *nchunks + groups_per_block * p.R - 1) / (groups_per_block * p.R);
    const int64_t cap = (int64_t)sms * 16;
    p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    return p;
}

}  // namespace ceb

using namespace ceb;

extern "C" {

size_t ce_workspace_size(int64_t N, int64_t V, ce_dtype dt, int num_sms) {
    if (N <= 0 || V <= 0 || (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16)) return 0;
    return forward_workspace(N, V, elem_size(dt), device_sms(num_sms));
}

ce_status ce_forward(const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                     const void* targets, ce_index_dtype tdt, ce_layout tg,
                     float label_smoothing, int64_t ignore_index,
                     float* loss, float* lse, float* lse_lo, int32_t* argmax,
                     void* workspace, size_t ws_bytes, void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return CE_EINVAL;
    if (tdt != CE_I32 && tdt != CE_I64) return CE_EINVAL;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!logits || !targets || !loss || !lse) return CE_EINVAL;
    if (!layout_ok(lg) || !layout_ok(tg)) return CE_EINVAL;
    const int esz = elem_size(dt);
    const int tsz = tdt == CE_I32 ? 4 : 8;
    const Layout L = to_layout(lg), T = to_layout(tg);

    // outputs must not overlap inputs or each other
    const Extent ez = layout_extent(logits, L, N, V, esz);
    const Extent et = layout_extent(targets, Layout{T.inner, T.s_outer, T.s_inner, 0}, N, 1, tsz);
    Extent outs[4];
    int nout = 0;
    outs[nout++] = flat_extent(loss, N, 4);
    outs[nout++] = flat_extent(lse, N, 4);
    if (lse_lo) outs[nout++] = flat_extent(lse_lo, N, 4);
    if (argmax) outs[nout++] = flat_extent(argmax, N, 4);
    for (int i = 0; i < nout; ++i) {
        if (overlap(outs[i], ez) || overlap(outs[i], et)) return CE_EALIAS;
        for (int j = 0; j < i; ++j)
            if (overlap(outs[i], outs[j])) return CE_EALIAS;
    }

    const int sms = device_sms(0);
    const bool vec_ok = vectorizable(logits, L, N, esz);
    FwdPlan plan = plan_forward(N, V, esz, vec_ok, sms);
    FwdArgs a{};
    if (plan.kind == FwdPlan::kCta && plan.splits > 1) {
        const size_t need = (size_t)plan.splits * (size_t)N * sizeof(float4);
        if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 16))
            return CE_EWORKSPACE;
        const Extent ew = flat_extent(workspace, (int64_t)need, 1);
        if (overlap(ew, ez) || overlap(ew, et)) return CE_EALIAS;
        for (int i = 0; i < nout; ++i)
            if (overlap(ew, outs[i])) return CE_EALIAS;
        a.part = static_cast<float4*>(workspace);
    }
    a.z = logits;
    a.N = N;
    a.V = V;
    a.y = targets;
    a.tdt = tdt == CE_I32 ? 0 : 1;
    a.eps = label_smoothing;
    a.ignore = ignore_index;
    a.loss = loss;
    a.lse = lse;
    a.lse_lo = lse_lo;
    a.argmax = argmax;
    a.err = error_word();
    if (!a.err) return CE_ECUDA;
    a.splits = plan.splits;
    a.vec_is_scalar = plan.vec == 1;
    a.vec_per_split = plan.vec_per_split;
    a.lz = L;
    a.ly = T;
    const WaitPolicy wp = wait_policy();
    a.wait_ns = wp.limit_ns;
    a.starve = wp.starve;
    cudaError_t e = launch_forward(plan, a, (int)dt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

ce_status ce_backward(const float* grad_out, int64_t grad_stride, const void* logits,
                      ce_dtype dt, ce_layout lg, int64_t N, int64_t V, const void* targets,
                      ce_index_dtype tdt, ce_layout tg, const float* lse, const float* lse_lo,
                      float label_smoothing, int64_t ignore_index, void* dlogits, ce_dtype ddt,
                      ce_layout dl, void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return CE_EINVAL;
    if (ddt != CE_F32 && ddt != dt) return CE_ENOTSUP;
    if (tdt != CE_I32 && tdt != CE_I64) return CE_EINVAL;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!grad_out || !logits || !targets || !lse || !dlogits) return CE_EINVAL;
    if (!layout_ok(lg) || !layout_ok(tg) || !layout_ok(dl)) return CE_EINVAL;
    const int esz = elem_size(dt), dsz = elem_size(ddt);
    const int tsz = tdt == CE_I32 ? 4 : 8;
    const Layout L = to_layout(lg), T = to_layout(tg), D = to_layout(dl);

    const Extent ez = layout_extent(logits, L, N, V, esz);
    const Extent ed = layout_extent(dlogits, D, N, V, dsz);
    const Extent et = layout_extent(targets, Layout{T.inner, T.s_outer, T.s_inner, 0}, N, 1, tsz);
    const Extent eg = grad_stride == 0 ? flat_extent(grad_out, 1, 4)
                                       : layout_extent(grad_out, Layout{N, 0, grad_stride, 0}, N, 1, 4);
    const Extent el = flat_extent(lse, N, 4);
    const bool in_place = dlogits == logits && ddt == dt && L.inner == D.inner &&
                          L.s_outer == D.s_outer && L.s_inner == D.s_inner && L.s_col == D.s_col;
    if (!in_place && overlap(ed, ez)) return CE_EALIAS;
    if (overlap(ed, et) || overlap(ed, eg) || overlap(ed, el)) return CE_EALIAS;
    if (lse_lo && overlap(ed, flat_extent(lse_lo, N, 4))) return CE_EALIAS;

    const int sms = device_sms(0);
    // vector path: both operands row-aligned with unit column stride
    const bool vec_ok = vectorizable(logits, L, N, esz) && vectorizable(dlogits, D, N, dsz);
    int64_t nchunks = 1, vpc = 1;
    BwdPlan plan = plan_backward(N, V, esz, vec_ok, sms, &nchunks, &vpc);
    BwdArgs a{};
    a.g = grad_out;
    a.g_stride = grad_stride;
    a.z = logits;
    a.N = N;
    a.V = V;
    a.y = targets;
    a.tdt = tdt == CE_I32 ? 0 : 1;
    a.lse = lse;
    a.lse_lo = lse_lo;
    a.eps = label_smoothing;
    a.ignore = ignore_index;
    a.dz = dlogits;
    a.err = error_word();
    if (!a.err) return CE_ECUDA;
    a.nchunks = nchunks;
    a.vec_per_chunk = vpc;
    a.lz = L;
    a.ly = T;
    a.ld = D;
    cudaError_t e = launch_backward(plan, a, (int)dt, (int)ddt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

// ---- probability (soft) targets -------------------------------------------------
static SoftPlan plan_soft(int64_t N, int64_t V, int esz, int tsz, bool vec_ok, int sms) {
    SoftPlan p{};
    p.vec = vec_ok ? 16 / esz : 1;
    // vectors per lane per step, as the kernels take them
    const int U = p.vec == 1 ? 8 : (tsz > esz ? 2 : 4);
    const int64_t nvec = V / p.vec;
    int G = 1;
    while (G < 32 && nvec > (int64_t)U * G) G *= 2;
    p.G = G;
    const int64_t rows_per_block = 8 * (32 / G);
    const int64_t want = (N + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * 16;
    p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    return p;
}

static bool soft_dtypes_ok(ce_dtype dt, ce_dtype tdt) {
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return false;
    return tdt == dt || tdt == CE_F32;
}

ce_status ce_soft_forward(const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                          const void* target_probs, ce_dtype tdt, ce_layout tl,
                          float label_smoothing, float* loss, float* lse, float* lse_lo,
                          float* target_sum, void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (!soft_dtypes_ok(dt, tdt)) return CE_ENOTSUP;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!logits || !target_probs || !loss || !lse) return CE_EINVAL;
    if (!layout_ok(lg) || !layout_ok(tl)) return CE_EINVAL;
    const int esz = elem_size(dt), tsz = elem_size(tdt);
    const Layout L = to_layout(lg), T = to_layout(tl);
    const Extent ez = layout_extent(logits, L, N, V, esz);
    const Extent et = layout_extent(target_probs, T, N, V, tsz);
    Extent outs[4];
    int nout = 0;
    outs[nout++] = flat_extent(loss, N, 4);
    outs[nout++] = flat_extent(lse, N, 4);
    if (lse_lo) outs[nout++] = flat_extent(lse_lo, N, 4);
    if (target_sum) outs[nout++] = flat_extent(target_sum, N, 4);
    for (int i = 0; i < nout; ++i) {
        if (overlap(outs[i], ez) || overlap(outs[i], et)) return CE_EALIAS;
        for (int j = 0; j < i; ++j)
            if (overlap(outs[i], outs[j])) return CE_EALIAS;
    }
    const bool vec_ok = vectorizable(logits, L, N, esz) && vectorizable(target_probs, T, N, tsz);
    SoftPlan p = plan_soft(N, V, esz, tsz, vec_ok, device_sms(0));
    SoftArgs a{};
    a.z = logits;
    a.t = target_probs;
    a.N = N;
    a.V = V;
    a.eps = label_smoothing;
    a.loss = loss;
    a.lse = lse;
    a.lse_lo = lse_lo;
    a.tsum = target_sum;
    a.lz = L;
    a.lt = T;
    cudaError_t e = launch_soft_forward(p, a, (int)dt, (int)tdt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

ce_status ce_soft_backward(const float* grad_out, int64_t grad_stride, const void* logits, ce_dtype dt,
                           ce_layout lg, int64_t N, int64_t V, const void* target_probs, ce_dtype tdt,
                           ce_layout tl, const float* lse, const float* lse_lo, const float* target_sum,
                           float label_smoothing, void* dlogits, ce_dtype ddt, ce_layout dl,
                           void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (!soft_dtypes_ok(dt, tdt)) return CE_ENOTSUP;
    if (ddt != CE_F32 && ddt != dt) return CE_ENOTSUP;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!grad_out || !logits || !target_probs || !lse || !dlogits) return CE_EINVAL;
    if (!layout_ok(lg) || !layout_ok(tl) || !layout_ok(dl)) return CE_EINVAL;
    const int esz = elem_size(dt), tsz = elem_size(tdt), dsz = elem_size(ddt);
    const Layout L = to_layout(lg), T = to_layout(tl), D = to_layout(dl);
    const Extent ez = layout_extent(logits, L, N, V, esz);
    const Extent et = layout_extent(target_probs, T, N, V, tsz);
    const Extent ed = layout_extent(dlogits, D, N, V, dsz);
    const Extent eg = grad_stride == 0 ? flat_extent(grad_out, 1, 4)
                                       : layout_extent(grad_out, Layout{N, 0, grad_stride, 0}, N, 1, 4);
    const bool in_place = dlogits == logits && ddt == dt && L.inner == D.inner &&
                          L.s_outer == D.s_outer && L.s_inner == D.s_inner && L.s_col == D.s_col;
    if (!in_place && overlap(ed, ez)) return CE_EALIAS;
    if (overlap(ed, et) || overlap(ed, eg) || overlap(ed, flat_extent(lse, N, 4))) return CE_EALIAS;
    if (lse_lo && overlap(ed, flat_extent(lse_lo, N, 4))) return CE_EALIAS;
    if (target_sum && overlap(ed, flat_extent(target_sum, N, 4))) return CE_EALIAS;
    const bool vec_ok = vectorizable(logits, L, N, esz) && vectorizable(target_probs, T, N, tsz) &&
                        vectorizable(dlogits, D, N, dsz);
    SoftPlan p = plan_soft(N, V, esz, tsz, vec_ok, device_sms(0));
    SoftArgs a{};
    a.z = logits;
    a.t = target_probs;
    a.N = N;
    a.V = V;
    a.eps = label_smoothing;
    a.lse = const_cast<float*>(lse);
    a.lse_lo = const_cast<float*>(lse_lo);
    a.tsum = const_cast<float*>(target_sum);
    a.g = grad_out;
    a.g_stride = grad_stride;
    a.dz = dlogits;
    a.lz = L;
    a.lt = T;
    a.ld = D;
    cudaError_t e = launch_soft_backward(p, a, (int)dt, (int)tdt, (int)ddt,
                                         static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

// ---- KL divergence of a student from a teacher -------------------------------------
// Rows that need a whole warp (G = 32) and number fewer than the resident
// warps of the GPU take a CTA each in the forward and (row, 1024-vector
// chunk) units in the backward.
static KlPlan plan_kl(int64_t N, int64_t V, int esz, bool vec_ok, int sms) {
    KlPlan p = plan_soft(N, V, esz, esz, vec_ok, sms);
    p.cta = 0;
    p.cl = 1;
    p.sms = sms;
    if (p.G == 32 && N < (int64_t)sms * 24) {
        p.cta = 1;
        const int64_t cap = (int64_t)sms * 4;
        p.grid = (int)(N < cap ? (N > 0 ? N : 1) : cap);
        // rows split over a cluster of CL CTAs when that fills the CTA slots
        // better (4 per SM for 4-byte rows, 3 for 16-bit): the CL with the
        // fullest last wave, each CTA keeping at least 1024 vectors
        const int64_t nv = V / p.vec;
        const int64_t slots = (int64_t)sms * (esz == 4 && p.vec > 1 ? 4 : (p.vec == 1 ? 2 : 3));
        double best = 0.0;
        for (int cl = 1; cl <= 8; cl *= 2) {
            if (cl > 1 && nv / cl < 1024) break;
            const int64_t ncl = slots / cl;
            const int64_t waves = (N + ncl - 1) / ncl;
            const double eff = (double)N / (double)(waves * ncl);
            if (eff > best + 0.02) {
                best = eff;
                p.cl = cl;
            }
        }
        p.vec_per_cta = (nv + p.cl - 1) / p.cl;
        const int64_t nvec = V / p.vec;
        const int64_t nch = nvec > 0 ? (nvec + 1023) / 1024 : 1;
        const int64_t want = (N * nch + 7) / 8;
        const int64_t capb = (int64_t)sms * 12;
        p.grid_bwd = (int)(want < capb ? (want > 0 ? want : 1) : capb);
    }
    return p;
}

ce_status ce_kl_forward(const void* student, const void* teacher, ce_dtype dt, ce_layout ls,
                        ce_layout lt, int64_t N, int64_t V, float* loss, float* lse_student,
                        float* lse_student_lo, float* lse_teacher, float* lse_teacher_lo,
                        void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!student || !teacher || !loss || !lse_student || !lse_teacher) return CE_EINVAL;
    if (!layout_ok(ls) || !layout_ok(lt)) return CE_EINVAL;
    const int esz = elem_size(dt);
    const Layout Q = to_layout(ls), P = to_layout(lt);
    const Extent eq = layout_extent(student, Q, N, V, esz);
    const Extent ep = layout_extent(teacher, P, N, V, esz);
    Extent outs[5];
    int nout = 0;
    outs[nout++] = flat_extent(loss, N, 4);
    outs[nout++] = flat_extent(lse_student, N, 4);
    outs[nout++] = flat_extent(lse_teacher, N, 4);
    if (lse_student_lo) outs[nout++] = flat_extent(lse_student_lo, N, 4);
    if (lse_teacher_lo) outs[nout++] = flat_extent(lse_teacher_lo, N, 4);
    for (int i = 0; i < nout; ++i) {
        if (overlap(outs[i], eq) || overlap(outs[i], ep)) return CE_EALIAS;
        for (int j = 0; j < i; ++j)
            if (overlap(outs[i], outs[j])) return CE_EALIAS;
    }
    const bool vec_ok = vectorizable(student, Q, N, esz) && vectorizable(teacher, P, N, esz);
    KlPlan p = plan_kl(N, V, esz, vec_ok, device_sms(0));
    KlArgs a{};
    a.zq = student;
    a.zp = teacher;
    a.N = N;
    a.V = V;
    a.loss = loss;
    a.lse_q = lse_student;
    a.lse_q_lo = lse_student_lo;
    a.lse_p = lse_teacher;
    a.lse_p_lo = lse_teacher_lo;
    a.lq = Q;
    a.lp = P;
    cudaError_t e = launch_kl_forward(p, a, (int)dt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

ce_status ce_kl_backward(const float* grad_out, int64_t grad_stride, const void* student,
                         const void* teacher, ce_dtype dt, ce_layout ls, ce_layout lt, int64_t N,
                         int64_t V, const float* lse_student, const float* lse_student_lo,
                         const float* lse_teacher, const float* lse_teacher_lo, void* dstudent,
                         ce_dtype ddt, ce_layout dl, void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return CE_EINVAL;
    if (ddt != CE_F32 && ddt != dt) return CE_ENOTSUP;
    if (N == 0) return CE_OK;
    if (!grad_out || !student || !teacher || !lse_student || !lse_teacher || !dstudent) return CE_EINVAL;
    if (!layout_ok(ls) || !layout_ok(lt) || !layout_ok(dl)) return CE_EINVAL;
    const int esz = elem_size(dt), dsz = elem_size(ddt);
    const Layout Q = to_layout(ls), P = to_layout(lt), D = to_layout(dl);
    const Extent eq = layout_extent(student, Q, N, V, esz);
    const Extent ep = layout_extent(teacher, P, N, V, esz);
    const Extent ed = layout_extent(dstudent, D, N, V, dsz);
    const Extent eg = grad_stride == 0 ? flat_extent(grad_out, 1, 4)
                                       : layout_extent(grad_out, Layout{N, 0, grad_stride, 0}, N, 1, 4);
    const bool in_place = dstudent == student && ddt == dt && Q.inner == D.inner &&
                          Q.s_outer == D.s_outer && Q.s_inner == D.s_inner && Q.s_col == D.s_col;
    if (!in_place && overlap(ed, eq)) return CE_EALIAS;
    if (overlap(ed, ep) || overlap(ed, eg) || overlap(ed, flat_extent(lse_student, N, 4)) ||
        overlap(ed, flat_extent(lse_teacher, N, 4)))
        return CE_EALIAS;
    if (lse_student_lo && overlap(ed, flat_extent(lse_student_lo, N, 4))) return CE_EALIAS;
    if (lse_teacher_lo && overlap(ed, flat_extent(lse_teacher_lo, N, 4))) return CE_EALIAS;
    const bool vec_ok = vectorizable(student, Q, N, esz) && vectorizable(teacher, P, N, esz) &&
                        vectorizable(dstudent, D, N, dsz);
    KlPlan p = plan_kl(N, V, esz, vec_ok, device_sms(0));
    KlArgs a{};
    a.zq = student;
    a.zp = teacher;
    a.N = N;
    a.V = V;
    a.lse_q = const_cast<float*>(lse_student);
    a.lse_q_lo = const_cast<float*>(lse_student_lo);
    a.lse_p = const_cast<float*>(lse_teacher);
    a.lse_p_lo = const_cast<float*>(lse_teacher_lo);
    a.g = grad_out;
    a.g_stride = grad_stride;
    a.dz = dstudent;
    a.lq = Q;
    a.lp = P;
    a.ld = D;
    cudaError_t e = launch_kl_backward(p, a, (int)dt, (int)ddt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

ce_status ce_forward_backward(const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                              const void* targets, ce_index_dtype tdt, ce_layout tg,
                              float label_smoothing, int64_t ignore_index, const float* grad_out,
                              int64_t grad_stride, float* loss, float* lse, float* lse_lo,
                              int32_t* argmax, void* dlogits, ce_dtype ddt, ce_layout dl,
                              void* workspace, size_t ws_bytes, void* cuda_stream) {
    if (N < 0 || V < 1 || V > INT32_MAX) return CE_EINVAL;
    if (dt != CE_F32 && dt != CE_BF16 && dt != CE_F16) return CE_EINVAL;
    if (ddt != CE_F32 && ddt != dt) return CE_ENOTSUP;
    if (tdt != CE_I32 && tdt != CE_I64) return CE_EINVAL;
    if (!(label_smoothing >= 0.f && label_smoothing <= 1.f)) return CE_EINVAL;
    if (N == 0) return CE_OK;
    if (!logits || !targets || !loss || !lse || !grad_out || !dlogits) return CE_EINVAL;
    if (!layout_ok(lg) || !layout_ok(tg) || !layout_ok(dl)) return CE_EINVAL;
    const int esz = elem_size(dt), dsz = elem_size(ddt);
    const Layout L = to_layout(lg), T = to_layout(tg), D = to_layout(dl);
    // the gradient must not overlap the per-row outputs or the upstream gradient
    const Extent ed = layout_extent(dlogits, D, N, V, dsz);
    const Extent eg = grad_stride == 0 ? flat_extent(grad_out, 1, 4)
                                       : layout_extent(grad_out, Layout{N, 0, grad_stride, 0}, N, 1, 4);
    if (overlap(ed, flat_extent(loss, N, 4)) || overlap(ed, flat_extent(lse, N, 4)) || overlap(ed, eg))
        return CE_EALIAS;
    if (lse_lo && overlap(ed, flat_extent(lse_lo, N, 4))) return CE_EALIAS;
    if (argmax && overlap(ed, flat_extent(argmax, N, 4))) return CE_EALIAS;
    if (overlap(eg, flat_extent(loss, N, 4)) || overlap(eg, flat_extent(lse, N, 4))) return CE_EALIAS;

    const bool vec_ok = vectorizable(logits, L, N, esz) && vectorizable(dlogits, D, N, dsz);
    const int vec = vec_ok ? 16 / esz : 1;
    const int64_t nvec = V / vec;
    const int kU = vec == 1 ? 8 : 32 / vec;
    int G = 1;
    while (G < 32 && nvec > (int64_t)kU * G) G *= 2;
    const int sms = device_sms(0);
    // rows beyond one warp's registers: one slice per CTA, held in shared
    // memory when the row fits one CTA's 112 KB, else re-read through L2 by a
    // cluster of the fewest CTAs (up to 8) whose slices are at most 128 KB.
    // Both need 16-byte rows, and enough rows to give every SM a CTA; else a
    // forward, then the VJP.
    SliceRowPlan sp{};
    if (nvec > (int64_t)kU * G && vec_ok) {
        if (nvec <= (int64_t)kSliceSmemMaxChunks * 128) {
            if (N >= sms) {
                sp.cl = 1;
                sp.nch = (int)((nvec + 127) / 128);
                sp.vec_per_cta = nvec;
                sp.sms = sms;
                sp.l2 = 0;
            }
        } else {
            for (int cl = 1; cl <= 8; cl *= 2) {
                const int64_t per = (nvec + cl - 1) / cl;
                if (per * 16 <= kSliceL2MaxBytes) {
                    if (N * cl >= sms) {
                        sp.cl = cl;
                        sp.nch = (int)((per + 127) / 128);
                        sp.vec_per_cta = per;
                        sp.sms = sms;
                        sp.l2 = 1;
                    }
                    break;
                }
            }
        }
    }
    if (nvec > (int64_t)kU * G && sp.cl == 0) {
        // rows longer than one register step of a warp: forward, then the VJP
        // (which re-reads the logits)
        ce_status st = ce_forward(logits, dt, lg, N, V, targets, tdt, tg, label_smoothing,
                                  ignore_index, loss, lse, lse_lo, argmax, workspace, ws_bytes,
                                  cuda_stream);
        if (st != CE_OK) return st;
        return ce_backward(grad_out, grad_stride, logits, dt, lg, N, V, targets, tdt, tg, lse, lse_lo,
                           label_smoothing, ignore_index, dlogits, ddt, dl, cuda_stream);
    }
    // the same checks as the two separate calls
    {
        const int tsz = tdt == CE_I32 ? 4 : 8;
        const Extent ez = layout_extent(logits, L, N, V, esz);
        const Extent et = layout_extent(targets, Layout{T.inner, T.s_outer, T.s_inner, 0}, N, 1, tsz);
        Extent outs[4];
        int nout = 0;
        outs[nout++] = flat_extent(loss, N, 4);
        outs[nout++] = flat_extent(lse, N, 4);
        if (lse_lo) outs[nout++] = flat_extent(lse_lo, N, 4);
        if (argmax) outs[nout++] = flat_extent(argmax, N, 4);
        for (int i = 0; i < nout; ++i) {
            if (overlap(outs[i], ez) || overlap(outs[i], et)) return CE_EALIAS;
            for (int j = 0; j < i; ++j)
                if (overlap(outs[i], outs[j])) return CE_EALIAS;
        }
        const bool in_place = dlogits == logits && ddt == dt && L.inner == D.inner &&
                              L.s_outer == D.s_outer && L.s_inner == D.s_inner && L.s_col == D.s_col;
        if (!in_place && overlap(ed, ez)) return CE_EALIAS;
        if (overlap(ed, et)) return CE_EALIAS;
    }
    FusedPlan p{};
    p.vec = vec;
    p.G = G;
    p.U = (G == 1 && nvec <= 2) ? 2 : kU;
    const int64_t rows_per_block = 8 * (32 / G);
    const int64_t want = (N + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * 16;
    p.grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    if (vec_ok && V % vec == 0 && nvec <= 2) {
        // one or two whole vectors per row: a lane per row, every block resident
        p.tiny = 1;
        p.U = (int)nvec;
        const int64_t rows_tiny = 256 * (int64_t)kTinyRows;
        const int64_t want_t = (N + rows_tiny - 1) / rows_tiny;
        const int64_t cap_t = (int64_t)sms * ((nvec == 2 && esz == 2) ? 3 : 4);
        p.grid = (int)(want_t < cap_t ? (want_t > 0 ? want_t : 1) : cap_t);
    }
    FusedArgs a{};
    a.f.z = logits;
    a.f.N = N;
    a.f.V = V;
    a.f.y = targets;
    a.f.tdt = tdt == CE_I32 ? 0 : 1;
    a.f.eps = label_smoothing;
    a.f.ignore = ignore_index;
    a.f.loss = loss;
    a.f.lse = lse;
    a.f.lse_lo = lse_lo;
    a.f.argmax = argmax;
    a.f.err = error_word();
    if (!a.f.err) return CE_ECUDA;
    a.f.splits = 1;
    a.f.lz = L;
    a.f.ly = T;
    a.f.wait_ns = wait_policy().limit_ns;
    a.g = grad_out;
    a.g_stride = grad_stride;
    a.dz = dlogits;
    a.ld = D;
    cudaError_t e = sp.cl > 0
                        ? launch_fused_slices(sp, a, (int)dt, (int)ddt, static_cast<cudaStream_t>(cuda_stream))
                        : launch_fused(p, a, (int)dt, (int)ddt, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? CE_OK : CE_ECUDA;
}

ce_status ce_get_error(void* cuda_stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return CE_ECUDA;
    unsigned int w = 0;
    if (cudaMemcpyFromSymbol(&w, g_ce_error_word, sizeof(w)) != cudaSuccess) return CE_ECUDA;
    if (w) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_ce_error_word, &zero, sizeof(zero)) != cudaSuccess) return CE_ECUDA;
        // a wait that ran out invalidates whole launches: it outranks a bad target
        return (w & kErrTimeout) ? CE_ETIMEOUT : CE_ETARGET;
    }
    return CE_OK;
}

ce_status ce_testing_set_wait(uint64_t limit_ns, int starve) {
    if (starve != 0 && starve != 1) return CE_EINVAL;
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    g_wait_starve.store(starve, std::memory_order_relaxed);
    return CE_OK;
}

const char* ce_status_string(ce_status s) {
    switch (s) {
        case CE_OK: return "ok";
        case CE_EINVAL: return "invalid argument (size, pointer, dtype or layout)";
        case CE_EALIAS: return "an output overlaps an input";
        case CE_EWORKSPACE: return "workspace missing, misaligned or too small";
        case CE_ECUDA: return "CUDA runtime error";
        case CE_ETARGET: return "a target outside [0, V) that is not ignore_index";
        case CE_ENOTSUP: return "configuration not supported";
        case CE_ETIMEOUT: return "a kernel gave up a bounded wait; the outputs of that launch are not valid";
    }
    return "unknown status";
}

}  // extern "C"
