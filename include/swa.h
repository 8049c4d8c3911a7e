/*
 * swa.h -- C ABI of libswa.so: the fused softmax-weighted average on B200
 * (sm_100a).  Two instances of one operation, "a softmax-weighted average
 * whose scores come from a join":
 *
 *   causal attention   out_i = sum_{j in J(i)} softmax_j(q_i . k_j * scale) v_j
 *   Nadaraya-Watson    out_p = sum_q w_pq v_q / sum_q w_pq,
 *                      w_pq = exp(-|t_p - s_q|^2 / h^2)
 *
 * Definitions: "Show HN: Automatic deduction of FlashAttention kernel from
 * ~25 lines of SQL" (page 2), demo script 01_attention.py -- views
 * ATTENTION_WINDOW / ATTENTION_GROUP_BY (forward), query GRADIENT (backward
 * of loss = 1/2 sum out^2), query NADARAYA_WATSON (regrid), and
 * check_masks_are_absent_rows (mask semantics).
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.  Every pointer must be
 *     16-byte aligned.
 *   - Attention tensors are contiguous row-major [B, H, N, D] ("(t, d)"
 *     matrices per head, ordered by t then d as the FORWARD query orders
 *     them); lse and delta are [B, H, N] float32.
 *   - J(i) = {0 .. i} when causal != 0 (the join predicate q.t >= k.t,
 *     diagonal included), else {0 .. N-1}.  scale = 1/sqrt(D) = 1/8 at D = 64.
 *   - Masked pairs are absent: a pair (i, j) with j > i is never used in a
 *     product.  A +inf (or -inf, NaN) in V therefore reaches exactly the
 *     queries i with j in J(i), per IEEE rules, and never turns into a NaN
 *     elsewhere.  Q and K must be finite.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream).  Argument errors are detected on the
 *     host and returned before anything is enqueued.  A device-side
 *     failure (a bounded wait that ran out) is recorded in a device error
 *     word and reported by swa_get_device_error().
 *   - Workspaces are caller-owned device buffers of at least the size the
 *     matching *_workspace_size() returns (0 means none is needed, and
 *     `workspace` may then be NULL).  Their contents on entry do not matter;
 *     they must not be shared by calls that can run concurrently.
 *   - Thread safety: entry points may be called from several host threads
 *     on different streams; swa_last_error_message() is per host thread.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SWA_OK = 0,
    SWA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size, small workspace */
    SWA_ERR_UNSUPPORTED = 2,      /* a valid request this build does not implement */
    SWA_ERR_CUDA = 3,             /* a CUDA runtime call failed (message has details) */
    SWA_ERR_DEVICE_TIMEOUT = 4    /* a kernel's bounded wait ran out (device error word) */
} swa_status;

typedef enum {
    SWA_F32 = 0,  /* float32 storage, float32 arithmetic on CUDA cores */
    SWA_BF16 = 1  /* bfloat16 storage, tensor cores with float32 accumulation */
} swa_dtype;

/*
 * Bytes of workspace swa_attn_fwd needs: for bf16, four int32 of per-head
 * information, a 128-bit mask per 128-row tile of V (its rows that hold an
 * infinity or NaN) and an f16 copy of V ([B,H,N,D]), each rounded up to 256
 * bytes; 0 for float32.
 */
size_t swa_attn_fwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                   swa_dtype dtype);

/*
 * Attention forward (views ATTENTION_WINDOW / ATTENTION_GROUP_BY; the
 * FlashAttention plan the demo's docstring names: keys streamed past query
 * blocks under a running row max and row sum, the N x N scores never
 * stored).
 *   q, k, v  [B,H,N,D] of `dtype`         (in)
 *   out      [B,H,N,D] of `dtype`         (out)  out_i = sum_j P_ij v_j
 *   lse      [B,H,N] float32              (out)  m_i + ln z_i (natural log)
 *   B, H >= 1; N >= 1; D == 64.
 * The bf16 path runs every head on the tensor cores.  A prep pass over V
 * writes its f16 copy into the workspace and finds the heads that hold an
 * infinity or NaN: for those the kernel replaces every non-finite V entry by
 * 0 before its products and gives each output entry the IEEE class of the
 * sum over its existing pairs (every weight > 0), so a masked pair never
 * multiplies a value.  The same pass decides the operand type of P V: f16
 * (P and the f16 copy of V) when every finite |V| < 2^15, else bf16.
 * float32 inputs run on CUDA cores in float32.
 */
swa_status swa_attn_fwd(const void* q, const void* k, const void* v, void* out,
                        float* lse, int64_t B, int64_t H, int64_t N, int64_t D,
                        int causal, swa_dtype dtype, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace swa_attn_bwd needs: per-head information (four int32),
 * for bf16 a 128-bit mask per 128-row tile of V (rows holding an infinity or
 * NaN; the gradient call's forward reads it), delta and lse * log2(e) as
 * float32 [B,H,Npad] each (Npad = N rounded up to 128) and, for bf16, f16
 * copies of q, k, v and dout ([B,H,N,D] each); each part rounded up to 256
 * bytes.
 */
size_t swa_attn_bwd_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                   swa_dtype dtype);

/*
 * Attention backward (query GRADIENT: the gradient of a loss with respect
 * to every value of q, k and v in one pass; with loss = 1/2 sum out^2 the
 * upstream gradient dout equals out).
 *   q, k, v, out, dout  [B,H,N,D] of `dtype`   (in)  out/lse from swa_attn_fwd
 *   lse                 [B,H,N] float32        (in)
 *   dq, dk, dv          [B,H,N,D] of `dtype`   (out)
 * P_ij = exp(s_ij - lse_i); delta_i = sum_d dout_id out_id;
 * dS_ij = P_ij (dout_i . v_j - delta_i); dq_i = scale sum_j dS_ij k_j;
 * dk_j = scale sum_i dS_ij q_i; dv_j = sum_i P_ij dout_i (existing pairs only).
 * bf16: tensor cores for every head, with f16 operands (copies made by a prep
 * pass) when every finite |q|, |k|, |v|, |dout| < 2^15, else bf16.  V and
 * dout may hold infinities or NaN: every product over existing pairs is the
 * IEEE one, and no masked pair multiplies a value (dV of a diagonal block
 * reads a copy of dout with its non-finite entries replaced by 0, and those
 * entries' classes are merged back).  float32: CUDA cores, float32.
 */
swa_status swa_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        int64_t B, int64_t H, int64_t N, int64_t D, int causal,
                        swa_dtype dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * swa_attn_bwd that ADDS dq, dk, dv to float32 sums instead of writing them
 * (sequence sharding: a query chunk's dq, and a key chunk's dk and dv, are
 * sums over the chunk pairs computed by several calls; a bf16 rounding of
 * each partial dq would lose the cancellation in sum_j dS_ij k_j).
 *   dq_acc, dk_acc, dv_acc  [B,H,N,D] float32   (in/out)  += this call's terms
 * Other arguments, workspace (swa_attn_bwd_workspace_size) and errors as
 * swa_attn_bwd; bf16 inputs only (else SWA_ERR_UNSUPPORTED).  Each row of
 * the sums is read and written once per call, without atomics: calls that
 * share a sum must run one after another (one stream).
 */
swa_status swa_attn_bwd_acc(const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, float* dq_acc, float* dk_acc,
                            float* dv_acc, int64_t B, int64_t H, int64_t N, int64_t D,
                            int causal, swa_dtype dtype, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Bytes of workspace swa_attn_grad needs (as swa_attn_bwd_workspace_size). */
size_t swa_attn_grad_workspace_size(int64_t B, int64_t H, int64_t N, int64_t D,
                                    swa_dtype dtype);

/*
 * Forward and gradient in one call: the query GRADIENT of "Show HN: Automatic
 * deduction of FlashAttention kernel from ~25 lines of SQL" (page 2) --
 * loss = 1/2 sum out^2 over the attention view, and its gradient with
 * respect to every value of q, k and v in one backward pass.
 *   q, k, v     [B,H,N,D] of `dtype`   (in)
 *   out         [B,H,N,D] of `dtype`   (out)  as swa_attn_fwd
 *   lse         [B,H,N] float32        (out)  as swa_attn_fwd
 *   dq, dk, dv  [B,H,N,D] of `dtype`   (out)  gradient of 1/2 sum out^2
 * Same as swa_attn_fwd followed by swa_attn_bwd with dout = out, except that
 * for bf16 the backward's upstream gradient is the forward's float32 output
 * (kept as an f16 copy in the workspace; delta_i = |out_i|^2 in float32), not
 * the bf16 `out`: the gradient of rows whose dq nearly cancels (rows that see
 * few keys) is then not limited by the bf16 rounding of out.
 * Workspace: swa_attn_grad_workspace_size() bytes.  Errors as swa_attn_bwd.
 */
swa_status swa_attn_grad(const void* q, const void* k, const void* v, void* out, float* lse,
                         void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t N,
                         int64_t D, int causal, swa_dtype dtype, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * swa_attn_fwd without a workspace, for callers that cannot allocate device
 * memory (a plugin whose host application owns every device allocation and
 * passes it only inputs and outputs; a latency-critical path that must not
 * pay for cudaMalloc/cudaFree and their implicit synchronisation).  The
 * pages have no counterpart: this is an interface convenience.
 * Same arguments, results and errors as swa_attn_fwd minus the workspace.
 * With no room for an f16 copy of V, P V takes bf16 operands for every
 * head (out within the same tolerance, but not bitwise equal to
 * swa_attn_fwd's).  The forward's scratch (four int32 of information per
 * head) lives in a
 * static device array for 4096 heads (64 KB, held by every GPU that loads
 * the library until exit); B*H > 4096 returns SWA_ERR_UNSUPPORTED.  The first call on
 * each device looks up the array's device address (make it before any
 * stream capture).  All calls share the array: calls that overlap on the
 * GPU race.  Allocates nothing.
 */
swa_status swa_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                float* lse, int64_t B, int64_t H, int64_t N, int64_t D,
                                int causal, swa_dtype dtype, void* stream);

/* Bytes of workspace swa_nw_regrid needs for M targets and S sources. */
size_t swa_nw_workspace_size(int64_t M, int64_t S);

/*
 * Nadaraya-Watson regrid (query NADARAYA_WATSON; "bandwidth h = 0.5" with
 * divisor 0.25 = h^2):
 *   targets [M,2] float32 (x, y)   sources [S,2] float32 (x, y)   vals [S] float32
 *   out     [M] float32            out_p = sum_q w_pq v_q / sum_q w_pq
 *   w_pq = exp(-((tx-sx)^2 + (ty-sy)^2) / h^2), h > 0.  M, S >= 1.
 * If every weight of a target underflows, out_p is NaN (0/0).
 */
swa_status swa_nw_regrid(const float* targets, int64_t M, const float* sources,
                         const float* vals, int64_t S, float h, float* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * The regrid with points of `dims` coordinates (1, 2 or 3; dims = 2 is
 * swa_nw_regrid): the NADARAYA_WATSON view with the squared distance summed
 * over every coordinate column of the point tables.
 *   targets [M,dims] float32   sources [S,dims] float32   vals [S] float32
 *   out     [M] float32        out_p = sum_q w_pq v_q / sum_q w_pq,
 *   w_pq = exp(-sum_c (t_pc - s_qc)^2 / h^2).  Workspace: swa_nw_workspace_size.
 * Other dims return SWA_ERR_UNSUPPORTED.
 */
swa_status swa_nw_regrid_nd(const float* targets, int64_t M, const float* sources,
                            const float* vals, int64_t S, int dims, float h, float* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace swa_nw_regrid_bwd needs. */
size_t swa_nw_regrid_bwd_workspace_size(int64_t M, int64_t S, int dims);

/*
 * Gradient of the regrid (the GRADIENT query's backward pass applied to the
 * NADARAYA_WATSON view: the same softmax-weighted average over a join, with
 * weights P_pq = w_pq / sum_q w_pq) for an upstream gradient gout = dL/dout:
 *   gout      [M] float32        (in)
 *   dtargets  [M,dims] float32   (out)  dL/dt_p = (-2/h^2) sum_q (gout_p / Z_p)
 *                                        w_pq (v_q - out_p) (t_p - s_q)
 *   dsources  [S,dims] float32   (out)  dL/ds_q = (+2/h^2) sum_p (same terms)
 *   dvals     [S] float32        (out)  dL/dv_q = sum_p gout_p P_pq
 * with Z_p = sum_q w_pq and out_p recomputed (the forward's output is not an
 * input).  Two passes over the pair grid (per target, then per source) with
 * deterministic partial sums.  Arguments and errors as swa_nw_regrid_nd.
 */
swa_status swa_nw_regrid_bwd(const float* targets, int64_t M, const float* sources,
                             const float* vals, int64_t S, int dims, float h, const float* gout,
                             float* dtargets, float* dsources, float* dvals, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * The projection in front of attention ("Wiki notes", page 5, mini_attention:
 * Q = x Wq, K = x Wk, V = x Wv), written straight into attention's layout.
 *   x        [B*N, C] bf16 (token rows, b major)      (in)
 *   w        [3*H*D, C] bf16: one row per output feature -- q's features
 *            h*D + d, then k's, then v's (a linear layer's weight layout)
 *   q, k, v  [B,H,N,D] bf16                             (out)
 * q[b,h,n,d] = sum_c x[b*N+n, c] w[h*D+d, c] (k, v: rows H*D.., 2*H*D..),
 * float32 accumulation on the tensor cores, one rounding to bf16.
 * D == 64, C a positive multiple of 64 (else SWA_ERR_UNSUPPORTED); bf16 only.
 */
swa_status swa_qkv_proj(const void* x, const void* w, void* q, void* k, void* v, int64_t B,
                        int64_t N, int64_t C, int64_t H, int64_t D, swa_dtype dtype,
                        void* stream);

/*
 * Merges a partial attention result over a set of keys into an accumulator
 * over a disjoint set (sequence sharding: a rank's queries meet the other
 * ranks' key blocks one at a time).  The view ATTENTION_WINDOW's average
 * splits exactly ("Show HN ...", page 2): with lse = max + ln z of each set,
 *   lse = ln(e^lse_acc + e^lse_part)
 *   out = e^(lse_acc - lse) out_acc + e^(lse_part - lse) out_part
 * (a set with lse = -inf contributes nothing).
 *   out_part   [rows][D] of `dtype`    (in)   partial output (swa_attn_fwd's out)
 *   lse_part   [rows] float32          (in)   its lse (natural log)
 *   out_acc    [rows][D] float32       (in/out; input ignored when `first`)
 *   lse_acc    [rows] float32          (in/out; input ignored when `first`)
 *   out_final  [rows][D] of `dtype` or NULL   (out) the merged rows, rounded
 * rows = B*H*N of the row-major [B,H,N,D] tensors; D == 64.  One kernel,
 * asynchronous on `stream`; out_final may be out_part.
 * Errors: SWA_ERR_INVALID_ARGUMENT (null or misaligned pointer, rows outside
 * [1, 2^31], unknown dtype), SWA_ERR_UNSUPPORTED (D != 64).
 */
swa_status swa_attn_merge(const void* out_part, const float* lse_part, float* out_acc,
                          float* lse_acc, void* out_final, int64_t rows, int64_t D, int first,
                          swa_dtype dtype, void* stream);

/*
 * dst[i] = bf16(src[i]) (round to nearest even) for i < n: float32 sums
 * (swa_attn_merge's accumulator, swa_attn_bwd_acc's) to bf16 tensors.
 * n a positive multiple of 8; src, dst 16-byte aligned (else
 * SWA_ERR_INVALID_ARGUMENT).  One kernel on `stream`.
 */
swa_status swa_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream);

/*
 * Synchronises `stream`, then reads and clears this device's error word.
 * Returns SWA_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since
 * the last call, SWA_ERR_CUDA if the synchronisation failed, else SWA_OK.
 */
swa_status swa_get_device_error(void* stream);

/*
 * Diagnostic of the device-side failure path: enqueues on `stream` one small
 * kernel whose bounded waits (both forms the tensor-core kernels use: parked
 * with a suspend hint, and polling) run out, since nothing arrives at the
 * barriers they wait on.
 * The kernel exits normally after about 2 s of SM clock; a following
 * swa_get_device_error() reports SWA_ERR_DEVICE_TIMEOUT and clears the
 * word, and the context stays usable.  Returns SWA_OK once enqueued, or
 * SWA_ERR_CUDA.
 */
swa_status swa_selftest_wait_timeout(void* stream);

/* Static string naming a status code. */
const char* swa_status_string(swa_status status);

/* Detail of the last failure on this host thread ("" if none). */
const char* swa_last_error_message(void);

/* Kernel launches the last successful call on this host thread enqueued. */
int swa_last_launch_count(void);

/* Main kernels that swa_profile_kernel can bracket with events. */
typedef enum {
    SWA_KERNEL_NONE = 0,
    SWA_KERNEL_ATTN_FWD = 1, /* swa_attn_fwd, swa_attn_grad: the tensor-core forward */
    SWA_KERNEL_ATTN_BWD = 2, /* swa_attn_bwd, swa_attn_grad: the tensor-core backward */
    SWA_KERNEL_NW = 3,       /* swa_nw_regrid(_nd): both kernels (pair grid and final sum) */
    SWA_KERNEL_NW_BWD = 4,   /* swa_nw_regrid_bwd: its four kernels */
    SWA_KERNEL_QKV = 5       /* swa_qkv_proj */
} swa_kernel;

/*
 * Timing hook for this host thread: every later call that launches kernel
 * `which` records `start_event` on its stream just before that launch and
 * `stop_event` just after it (both are cudaEvent_t created by the caller).
 * SWA_KERNEL_NONE (or NULL events) turns the hook off.  Never fails.
 */
void swa_profile_kernel(swa_kernel which, void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
