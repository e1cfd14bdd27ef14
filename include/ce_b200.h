/*
 * ce_b200.h -- fused softmax cross-entropy on one NVIDIA B200 (sm_100a).
 *
 * C ABI. Plain pointers and sizes; no framework types. All device pointers
 * refer to memory of the device that is current on the calling thread; the
 * `cuda_stream` argument is a cudaStream_t (NULL = the legacy default stream).
 *
 * Ownership. The caller owns every buffer, the workspace and the stream. The
 * library allocates no device memory per call and writes nothing but the
 * outputs named in each call and the workspace handed to it. Library-owned
 * device state: a per-device error word (see ce_get_error) and the scratch
 * array of ce_forward_noalloc.
 *
 * Completion. Calls are asynchronous: they validate their arguments on the
 * host, enqueue kernels on `cuda_stream` and return. Every output element is
 * written on every call that returns CE_OK, including rows that are ignored
 * (a stale buffer content never survives a successful call).
 *
 * Errors. Problems the host can see (a null pointer, a bad size, dtype or
 * layout, an output overlapping an input, a short workspace) are returned as
 * a status before anything is enqueued. A target outside [0, V) that is not
 * ignore_index is only seen on the device: that row's loss (and, in the
 * backward, its gradient row) is written as NaN and the device error word is
 * set; ce_get_error reports it.
 *
 * Row addressing (ce_layout). Logical row r of an operand, 0 <= r < N, starts
 * at element offset
 *     (r / inner) * s_outer + (r % inner) * s_inner
 * from the base pointer, and its column j sits a further j * s_col elements
 * on. Offsets are in elements, 64-bit. A plain (N, V) matrix with row stride
 * ld is {inner = N, s_outer = 0, s_inner = ld, s_col = 1}. A view x[:, :-1]
 * of a (B, L, V) tensor is {inner = L - 1, s_outer = L*V, s_inner = V,
 * s_col = 1} with N = B*(L-1); the matching targets t[:, 1:] of a (B, L)
 * tensor are base t + 1 with {inner = L - 1, s_outer = L, s_inner = 1}.
 * Views are read in place: the library never makes a contiguous copy (MLX
 * issue #4686: the VJP went wrong through exactly such a hidden copy whose
 * output aliased it). Loads are vectorised to 16 bytes when s_col = 1 and
 * every row starts on a 16-byte boundary; other layouts take a scalar path.
 *
 * Rows are counted in 64 bits and every launch walks its rows in a
 * grid-stride loop, so no grid dimension limits N (MLX PR #4776: a grid
 * truncated past 2^32 threads silently skipped rows from 2^27 rows up).
 */
#ifndef CE_B200_H
#define CE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { CE_F32 = 0, CE_BF16 = 1, CE_F16 = 2 } ce_dtype;
typedef enum { CE_I32 = 0, CE_I64 = 1 } ce_index_dtype;

typedef struct {
    int64_t inner;   /* rows per outer block, >= 1 */
    int64_t s_outer; /* element stride between outer blocks */
    int64_t s_inner; /* element stride between rows of one block */
    int64_t s_col;   /* element stride between columns (unused for targets) */
} ce_layout;

typedef enum {
    CE_OK = 0,
    CE_EINVAL = 1,     /* bad size, pointer, dtype or layout */
    CE_EALIAS = 2,     /* an output overlaps an input (other than the allowed in-place) */
    CE_EWORKSPACE = 3, /* workspace missing or smaller than the *_workspace_size query */
    CE_ECUDA = 4,      /* a CUDA runtime call failed (launch, attribute query) */
    CE_ETARGET = 5,    /* device flag: a target outside [0, V) that is not ignore_index */
    CE_ENOTSUP = 6,    /* a configuration the library does not implement */
    CE_ETIMEOUT = 7    /* device flag: a kernel gave up a bounded wait (outputs invalid) */
} ce_status;

/* ------------------------------------------------------------------------ *
 * Row cross-entropy over an (N, V) logits operand.
 * ------------------------------------------------------------------------ */

/* Bytes of workspace ce_forward needs for this shape. Long rows on few rows
 * are split across several CTAs whose partial (max, scaled sum) states are
 * merged by a second launch; the workspace holds those partials. Returns 0
 * when no split is used. `num_sms` is the device's multiprocessor count, or
 * <= 0 to query the current device. */
size_t ce_workspace_size(int64_t N, int64_t V, ce_dtype dt, int num_sms);

/* Forward. For each row i with target y_i (ignore_index rows excepted):
 *     m_i   = max_j z_ij
 *     lse_i = m_i + log sum_j exp(z_ij - m_i)            (online, one pass)
 *     loss_i = (lse_i - m_i) - (1 - eps)(z_i,y_i - m_i) - eps (mean_j z_ij - m_i)
 * i.e. (1-eps)(lse - z_y) + eps(lse - mean z), assembled from max-shifted
 * values so that the gaps between logits survive at any magnitude.
 * Sources: Ineshin, "A fused linear cross-entropy forward kernel for Apple
 * GPUs", section 1 (the running (m, s) state and logsumexp = m + log s);
 * MLX PR #4188 "Shift by the max in cross_entropy" (the shifted assembly and
 * the label-smoothing term, which subtracts the mean logit).
 *
 * logits   N x V values of dtype `dt`, addressed through `lg`.
 * targets  N class indices of type `tdt`, addressed through `tg` (column 0).
 * label_smoothing  eps in [0, 1]; eps/V goes to every class.
 * ignore_index     rows whose target equals it get loss 0 (lse still written).
 * loss     N floats, contiguous. Out-of-range target: NaN (and the error word).
 * lse      N floats, contiguous: lse_i rounded to float.
 * lse_lo   N floats or NULL: lse_i minus the float `lse_i`, rounded to float
 *          (the pair carries lse to about 48 bits; ce_backward uses it to keep
 *          the softmax exact when |logits| is so large that float lse loses
 *          the gap, e.g. equal logits at 1e8).
 * argmax   N int32 or NULL: the lowest index attaining the row max (the first
 *          NaN if the row has one).
 * workspace, ws_bytes  at least ce_workspace_size(N, V, dt, sms) bytes,
 *          16-byte aligned; may be NULL when that size is 0.
 * Special rows: an all -inf row gives lse = -inf and loss NaN; a NaN in the
 * row gives lse and loss NaN.
 * Outputs must not overlap each other, the logits or the targets. */
ce_status ce_forward(const void* logits, ce_dtype dt, ce_layout lg,
                     int64_t N, int64_t V,
                     const void* targets, ce_index_dtype tdt, ce_layout tg,
                     float label_smoothing, int64_t ignore_index,
                     float* loss, float* lse, float* lse_lo, int32_t* argmax,
                     void* workspace, size_t ws_bytes, void* cuda_stream);

/* Backward (VJP of sum_i g_i loss_i with respect to the logits):
 *     dz_ij = g_i (exp(z_ij - lse_i) - (1 - eps)[j = y_i] - eps/V)
 * from the saved lse (and lse_lo when given); ignore_index rows get a zero
 * row, out-of-range targets a NaN row and the error word.
 * Sources: MLX issue #4686 (the fast.cross_entropy VJP, including the strided
 * view x[:, :-1]); Ineshin section 1 (the backward regenerates what it needs
 * from the saved log-sum-exp).
 *
 * grad_out     g: N floats read at grad_out[i * grad_stride]; grad_stride = 0
 *              broadcasts one scalar (e.g. 1/count for a mean reduction).
 * lse, lse_lo  as written by ce_forward (lse_lo may be NULL: taken as 0).
 * dlogits      N x V values of dtype `ddt` through layout `dl`. It may be the
 *              logits themselves (same pointer, same dtype, same layout:
 *              each element is read before it is overwritten by the same
 *              thread); any other overlap with an input is CE_EALIAS. */
ce_status ce_backward(const float* grad_out, int64_t grad_stride,
                      const void* logits, ce_dtype dt, ce_layout lg,
                      int64_t N, int64_t V,
                      const void* targets, ce_index_dtype tdt, ce_layout tg,
                      const float* lse, const float* lse_lo,
                      float label_smoothing, int64_t ignore_index,
                      void* dlogits, ce_dtype ddt, ce_layout dl,
                      void* cuda_stream);

/* Forward and backward in one call, for when the upstream gradient g is
 * known before the forward runs (a mean or sum of the per-row losses: g =
 * 1/count or 1 with grad_stride 0). Writes what ce_forward and ce_backward
 * write, with the same definitions, readings and errors (argument meanings as
 * there). The logits cross HBM once instead of twice wherever a row fits on
 * chip: rows of up to 1024 elements stay in the registers of the lanes that
 * fold them. Longer rows need 16-byte aligned, unit-stride rows (logits and
 * dlogits): rows of up to 112 KB are copied into one CTA's shared memory and
 * differentiated from there; rows of up to 8 x 128 KB are split into slices
 * over a cluster of 1 to 8 CTAs, whose partial states meet once in
 * distributed shared memory, and each slice is read a second time from L1/L2
 * for the gradient. Those rows need at least (number of SMs / cluster size)
 * rows per call; otherwise, and for longer or unaligned rows, the call runs
 * the forward, then the backward.
 * Sources: Ineshin, "A fused linear cross-entropy forward kernel for Apple
 * GPUs", section 1 (the backward needs only the row's log-sum-exp, which
 * the forward has just produced); MLX issue #4686 (the VJP).
 * dlogits may be the logits themselves (same pointer, dtype and layout); it
 * must not overlap the per-row outputs or grad_out. The workspace is the
 * one ce_forward needs for the same shape (only used on the long-row path). */
ce_status ce_forward_backward(const void* logits, ce_dtype dt, ce_layout lg,
                              int64_t N, int64_t V,
                              const void* targets, ce_index_dtype tdt, ce_layout tg,
                              float label_smoothing, int64_t ignore_index,
                              const float* grad_out, int64_t grad_stride,
                              float* loss, float* lse, float* lse_lo, int32_t* argmax,
                              void* dlogits, ce_dtype ddt, ce_layout dl,
                              void* workspace, size_t ws_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Probability (soft) targets. Source: MLX PR #4188, "Shift by the max in
 * cross_entropy" (the loss is the row's log-sum-exp minus the
 * target-weighted logits, assembled from values shifted by the row max).
 * With a target distribution t per row and label smoothing eps (which mixes
 * t with the uniform distribution: t' = (1-eps) t + eps/V):
 *     loss_i = sum_j t'_ij (lse_i - z_ij),
 *     dz_ij  = g_i (p_ij T'_i - t'_ij),   T'_i = sum_j t'_ij = (1-eps) T_i + eps,
 * which is lse - sum_j t_j z_j and p - t when the rows of t sum to 1.
 * t is used as given (not renormalised). A class whose t'_ij is 0 adds
 * nothing, even at z_ij = -inf. NaN in a row, or a row of z that is all -inf,
 * gives a NaN loss and a NaN gradient row. There is no ignore_index.
 * Logits in f32, bf16 or f16; targets in the logits' dtype or f32 (else
 * CE_ENOTSUP), N x V through their own layout `tl` (all four fields used).
 * Each row of logits and of targets is read once per call; rows are not split
 * across CTAs, so the calls want at least a few hundred rows to fill the GPU.
 * ------------------------------------------------------------------------ */

/* Forward: loss, lse (and lse_lo, as ce_forward; nullable) and, when
 * target_sum is not NULL, T_i = sum_j t_ij per row (N floats) for the
 * backward. No workspace. */
ce_status ce_soft_forward(const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                          const void* target_probs, ce_dtype tdt, ce_layout tl,
                          float label_smoothing, float* loss, float* lse, float* lse_lo,
                          float* target_sum, void* cuda_stream);

/* Backward (VJP of sum_i g_i loss_i): dz as above from the saved lse (and
 * lse_lo) and target_sum; target_sum NULL means every row of t sums to 1.
 * grad_out, grad_stride and dlogits (dtype ddt: the logits' dtype or f32;
 * in place on the logits allowed, same pointer, dtype and layout) as for
 * ce_backward. */
ce_status ce_soft_backward(const float* grad_out, int64_t grad_stride,
                           const void* logits, ce_dtype dt, ce_layout lg, int64_t N, int64_t V,
                           const void* target_probs, ce_dtype tdt, ce_layout tl,
                           const float* lse, const float* lse_lo, const float* target_sum,
                           float label_smoothing, void* dlogits, ce_dtype ddt, ce_layout dl,
                           void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * KL divergence of a student distribution from a teacher's, fused. Source:
 * Suryavanshi, "One barrier short" (the fused KL loss of mlx-lm, forward and
 * backward in one pass over both rows, an online log-sum-exp for each). With
 * teacher logits zp and student logits zq of a row, p = softmax(zp) and
 * q = softmax(zq):
 *     loss_i = sum_j p_ij (log p_ij - log q_ij),   dzq_ij = g_i (q_ij - p_ij).
 * Only the student gets a gradient (the teacher is a fixed target). A class
 * with p_ij = 0 adds nothing, even where zq_ij is -inf too; a student -inf
 * under teacher mass gives +inf. NaN in either row, or a row of either that
 * is all -inf, gives a NaN loss and a NaN gradient row. Both inputs have
 * dtype dt (f32, bf16, f16), N x V through their own layouts. The result
 * depends on the inputs alone: repeated calls give the same bytes (the
 * cross-lane exchange reuses no scratch, so the race "One barrier short"
 * describes cannot occur).
 * ------------------------------------------------------------------------ */

/* Forward: loss, the student's and the teacher's lse (each with its lo
 * part, nullable, as in ce_forward). N floats each. No workspace. */
ce_status ce_kl_forward(const void* student, const void* teacher, ce_dtype dt, ce_layout ls,
                        ce_layout lt, int64_t N, int64_t V, float* loss, float* lse_student,
                        float* lse_student_lo, float* lse_teacher, float* lse_teacher_lo,
                        void* cuda_stream);

/* Backward: dstudent (dtype ddt: dt or f32; may be the student logits
 * themselves, same pointer, dtype and layout) from the saved lse pairs.
 * grad_out and grad_stride as for ce_backward. */
ce_status ce_kl_backward(const float* grad_out, int64_t grad_stride, const void* student,
                         const void* teacher, ce_dtype dt, ce_layout ls, ce_layout lt, int64_t N,
                         int64_t V, const float* lse_student, const float* lse_student_lo,
                         const float* lse_teacher, const float* lse_teacher_lo, void* dstudent,
                         ce_dtype ddt, ce_layout dl, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Fused-linear cross-entropy: logits Z = H W^T are never stored.
 * Source: Ineshin, "A fused linear cross-entropy forward kernel for Apple
 * GPUs", section 1 (Z = H W^T streamed over vocabulary tiles into the running
 * (m, s) state, the target logit captured when its tile passes; the backward
 * regenerates the logits tile by tile from the saved log-sum-exp).
 * H: N x D bf16, row stride ld_h elements; W: V x D bf16, row stride ld_w.
 * D must be a multiple of 64 and ld_h, ld_w multiples of 8 (16-byte rows for
 * the tensor-memory-access engine); H and W 16-byte aligned.
 * ------------------------------------------------------------------------ */

/* Workspace bytes for linear_ce_forward (per-row partial states of the
 * vocabulary splits). `num_sms` <= 0 queries the current device. */
size_t linear_ce_workspace_size(int64_t N, int64_t V, int64_t D, int num_sms);

/* loss and lse of Z = H W^T rows, same definitions as ce_forward.
 * targets: N indices of type tdt, contiguous. loss, lse: N floats. */
ce_status linear_ce_forward(const void* H, int64_t ld_h, const void* W, int64_t ld_w,
                            const void* targets, ce_index_dtype tdt,
                            int64_t N, int64_t V, int64_t D,
                            float label_smoothing, int64_t ignore_index,
                            float* loss, float* lse,
                            void* workspace, size_t ws_bytes, void* cuda_stream);

/* Workspace bytes for linear_ce_backward: one vocabulary chunk of the
 * gradient of the logits (bf16, N x 8192) and the float dH accumulator
 * (268 MB at N = 8192, V = 151,936, D = 4096). No transposed copy of H, W or
 * the gradient is made. */
size_t linear_ce_backward_workspace_size(int64_t N, int64_t V, int64_t D, int num_sms);

/* dH = G W and dW = G^T H with G_ij = g_i (exp(Z_ij - lse_i) - (1-eps)[j=y_i]
 * - eps/V), Z recomputed chunk by chunk of the vocabulary from H and W and
 * the saved lse. dH: N x D, dW: V x D, contiguous, dtype CE_BF16 or CE_F32
 * (accumulation is float either way). */
ce_status linear_ce_backward(const float* grad_out, int64_t grad_stride,
                             const void* H, int64_t ld_h, const void* W, int64_t ld_w,
                             const void* targets, ce_index_dtype tdt, const float* lse,
                             int64_t N, int64_t V, int64_t D,
                             float label_smoothing, int64_t ignore_index,
                             void* dH, ce_dtype dH_dt, void* dW, ce_dtype dW_dt,
                             void* workspace, size_t ws_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Forward without a caller-provided workspace.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory or pass a workspace: plugins inside a host
 * application that owns all device memory through its own pool (a raw
 * allocation would bypass its accounting), loops with a memory budget fixed
 * at start-up that must not run out of memory halfway, and C callers without
 * an allocator (cudaMalloc may also synchronise the device).
 *
 * Same arguments, results and errors as ce_forward, without workspace and
 * ws_bytes. The scratch for the vocabulary split lives in a library-owned
 * array of CE_NOALLOC_SCRATCH_BYTES (64 KiB) in device memory, one per device
 * that loads the library, held until the process exits. On a 148-SM B200
 * that holds the split partials of every shape whose rows are at most
 * 128 KB (32768 fp32 or 65536 bf16 classes) and of longer rows for up to 32
 * rows (and many larger counts); a shape whose ce_workspace_size exceeds it
 * returns CE_EWORKSPACE and enqueues nothing.
 * The call allocates nothing. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current) and caches
 * it; make that first call before any stream capture begins. All calls on a
 * device share the one array and it keeps the last call's partial states:
 * calls whose kernels can overlap on the GPU (different streams, no ordering
 * between them) race on it and must be serialised by the caller. Nothing in
 * the array needs to start at zero: each call writes every slot it reads.
 * ------------------------------------------------------------------------ */
#define CE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 10)

ce_status ce_forward_noalloc(const void* logits, ce_dtype dt, ce_layout lg,
                             int64_t N, int64_t V,
                             const void* targets, ce_index_dtype tdt, ce_layout tg,
                             float label_smoothing, int64_t ignore_index,
                             float* loss, float* lse, float* lse_lo, int32_t* argmax,
                             void* cuda_stream);

/* ------------------------------------------------------------------------ */

/* Waits for `cuda_stream`, then reads and clears the current device's error
 * word: CE_ETIMEOUT if any launch since the last call gave up a bounded wait
 * (the outputs of that launch, and of the launches that consumed them, are
 * not valid), else CE_ETARGET if any launch saw an out-of-range target,
 * CE_ECUDA if the wait itself failed, CE_OK otherwise.
 *
 * Bounded waits. The kernels that stream their operands through mbarrier
 * pipelines (the tensor-core GEMM engine of linear_ce_forward and
 * linear_ce_backward, and the bulk-copy rings of the long-row kernels) give up
 * any wait after a time limit (2 s by default; a correct pipeline waits
 * microseconds): the CTA raises the timeout flag, lets the copies and
 * tensor-core operations it started complete, frees its tensor memory and
 * returns, so a broken pipeline ends with an error status instead of a hung
 * GPU, and the context stays usable. */
ce_status ce_get_error(void* cuda_stream);

/* Testing hook for the bounded waits; the pages have no counterpart. Sets the
 * wait limit of the GEMM engine, of the long-row forward's bulk-copy ring and
 * of ce_forward_backward's long-row slices for the launches this process makes
 * afterwards (limit_ns = 0 restores the default of 2 s). With starve = 1 those
 * launches issue none of their copies (and the slices push no state to their
 * cluster peers), so every wait for data runs out after the limit: tests use it to check that
 * a wait that runs out ends the kernel with CE_ETIMEOUT and leaves the
 * context and the next call correct. starve = 0 is normal operation; any
 * other value is CE_EINVAL. Not for production use: a starved launch writes
 * invalid outputs. */
ce_status ce_testing_set_wait(uint64_t limit_ns, int starve);

/* Static text for a status code. */
const char* ce_status_string(ce_status s);

#ifdef __cplusplus
}
#endif

#endif /* CE_B200_H */
