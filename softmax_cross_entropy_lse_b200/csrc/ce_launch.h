// Internal launch interface between the C ABI (ce_api.cu) and the kernel
// translation units. Not part of the public header.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ceb {

// Bit of the device error word raised by a kernel that gave up a bounded
// pipeline wait (bit 0 flags an out-of-range target).
constexpr unsigned kErrTimeout = 2u;

// Time limit of the bounded pipeline waits and the copy-starving switch of
// the testing hook ce_testing_set_wait (defaults: 2 s, off). Read at launch
// time and passed to the kernels that wait on mbarriers for their copies.
struct WaitPolicy {
    unsigned long long limit_ns;
    int starve;  // 1: producers issue no copies, so every wait for data runs out
};
WaitPolicy wait_policy();

// Raises the dynamic shared-memory limit of `kernel` to `bytes` on the
// current device, once per (kernel, device); safe from several threads.
cudaError_t ensure_smem_limit(const void* kernel, int bytes);

// Clusters of `kernel` that can be resident at once on the current device
// for the block, cluster and shared-memory shape of `cfg` (its grid is
// ignored), cached per (kernel, device).
cudaError_t max_active_clusters(const void* kernel, const cudaLaunchConfig_t& cfg, int* clusters);

// Two-level row addressing: row r starts at (r / inner) * s_outer +
// (r % inner) * s_inner elements, column j a further j * s_col on.
struct Layout {
    int64_t inner, s_outer, s_inner, s_col;
};

// ---- row forward -------------------------------------------------------------
struct FwdArgs {
    const void* z;
    int64_t N, V;
    const void* y;
    int tdt;
    float eps;
    int64_t ignore;
    float* loss;
    float* lse;
    float* lse_lo;
    int32_t* argmax;
    unsigned int* err;
    float4* part;           // split partials [splits][N]
    int splits;
    int vec_is_scalar;
    int64_t vec_per_split;  // in units of the kernel's vector width
    Layout lz, ly;
    unsigned long long wait_ns;  // limit of the bulk-copy ring's waits
    int starve;                  // testing: the ring issues no copies
};

struct FwdPlan {
    enum Kind { kPacked = 0, kCta = 1, kTiny = 2 } kind;
    int vec;        // 1 (scalar path) or the 16-byte vector width of the dtype
    int G, U;       // packed: lanes per row, vectors per lane per step; tiny: U vectors per row
    int R;          // packed: rows per group per step
    int ring;       // long rows through per-warp bulk-copy rings
    int pipe;       // packed 4-byte rows of one step, pipelined through shared memory
    int grid;
    int merge_grid;
    int splits;
    int64_t vec_per_split;
};

cudaError_t launch_forward(const FwdPlan& p, const FwdArgs& a, int dtype, cudaStream_t s);

// rows per lane per step of the tiny-row forward
constexpr int kTinyRows = 2;

// ---- row backward ------------------------------------------------------------
struct BwdArgs {
    const float* g;
    int64_t g_stride;
    const void* z;
    int64_t N, V;
    const void* y;
    int tdt;
    const float* lse;
    const float* lse_lo;
    float eps;
    int64_t ignore;
    void* dz;
    unsigned int* err;
    int64_t nchunks;
    int64_t vec_per_chunk;
    Layout lz, ly, ld;
};

struct BwdPlan {
    int vec;
    int G, U;
    int R;     // units per group per step
    int ring;  // long rows through per-warp bulk-copy rings
    int rows;  // short rows, one unit per row (k_bwd_rows)
    int tiny;  // one or two whole vectors per row: a lane per row (k_bwd_tiny)
    int grid;
};

cudaError_t launch_backward(const BwdPlan& p, const BwdArgs& a, int dt_in, int dt_out,
                            cudaStream_t s);

// ---- fused forward + backward (short rows) ---------------------------------
struct FusedArgs {
    FwdArgs f;
    const float* g;
    int64_t g_stride;
    void* dz;
    Layout ld;
};

struct FusedPlan {
    int vec;
    int G, U;   // tiny: U vectors per row
    int tiny;   // one lane per row (one or two whole vectors per row)
    int grid;
};

cudaError_t launch_fused(const FusedPlan& p, const FusedArgs& a, int dt_in, int dt_out,
                         cudaStream_t s);

// ---- fused forward + backward of long rows, one slice per CTA ---------------
// A row is split over a cluster of `cl` CTAs, vec_per_cta 16-byte vectors
// (nch 2 KB chunks) each. The slice is held in shared memory (l2 = 0; one CTA
// per row, up to kSliceSmemMaxChunks chunks), or read twice from global
// memory with the second read served by L1/L2 (l2 = 1; slices up to
// kSliceL2MaxBytes, clusters of 1 to 8).
constexpr int kSliceSmemMaxChunks = 56;           // 112 KB per CTA: two CTAs per SM
constexpr int64_t kSliceL2MaxBytes = 128 * 1024;  // 148 SMs x 4 CTAs: 76 MB of L2

struct SliceRowPlan {
    int cl;
    int nch;
    int64_t vec_per_cta;
    int sms;
    int l2;
};

cudaError_t launch_fused_slices(const SliceRowPlan& p, const FusedArgs& a, int dt_in, int dt_out,
                                cudaStream_t s);

// ---- probability (soft) targets ---------------------------------------------
struct SoftArgs {
    const void* z;
    const void* t;
    int64_t N, V;
    float eps;
    float* loss;
    float* lse;
    float* lse_lo;
    float* tsum;        // forward: sum_j t_j per row (nullable)
    const float* g;     // backward
    int64_t g_stride;
    void* dz;
    Layout lz, lt, ld;
};

struct SoftPlan {
    int vec;
    int G;
    int grid;
    int cta;       // KL: long rows, too few of them for a warp each to fill the GPU
    int grid_bwd;  // KL backward over (row, chunk) units
    int cl;        // KL forward of long rows: CTAs per row (a cluster), 1, 2, 4 or 8
    int64_t vec_per_cta;  // vectors of a row each CTA of the cluster folds
    int sms;
};

cudaError_t launch_soft_forward(const SoftPlan& p, const SoftArgs& a, int dz_t, int dt_t,
                                cudaStream_t s);
cudaError_t launch_soft_backward(const SoftPlan& p, const SoftArgs& a, int dz_t, int dt_t, int do_t,
                                 cudaStream_t s);

// ---- KL divergence of a student (q) from a teacher (p) ----------------------
struct KlArgs {
    const void* zq;   // student logits
    const void* zp;   // teacher logits
    int64_t N, V;
    float* loss;
    float* lse_q;
    float* lse_q_lo;
    float* lse_p;
    float* lse_p_lo;
    const float* g;   // backward
    int64_t g_stride;
    void* dz;
    Layout lq, lp, ld;
};

using KlPlan = SoftPlan;

cudaError_t launch_kl_forward(const KlPlan& p, const KlArgs& a, int dt, cudaStream_t s);
cudaError_t launch_kl_backward(const KlPlan& p, const KlArgs& a, int dt, int ddt, cudaStream_t s);

}  // namespace ceb
