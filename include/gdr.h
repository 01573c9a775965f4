/*
 * gdr.h -- C ABI of the gated delta-rule mixer library (libgdr.so, NVIDIA B200 / sm_100a).
 *
 * The operation. Per head, with state S in R^{d_v x d_k} (value-by-key, read as o = S q):
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t / sqrt(d_k)                     (read after the token's write)
 *
 * alpha_t = exp(g_t): 1 for DeltaNet, a per-head scalar for Gated DeltaNet, a per-key-channel
 * vector for Kimi Delta Attention. Sources: "linear attention and its gated descendants",
 * sections DeltaNet, Gated DeltaNet and Kimi Delta Attention (update rules and the
 * key-dimension decay); "Linear Attention Architectures: Mechanisms, Trade-offs, and
 * Cross-Layer Routing", Sec. 3 (the diagonal decay multiplies the memory on the right, along
 * the key-feature dimension); "Linear Attention & DeltaNet", How it works, items 3-4. The
 * 1/sqrt(d_k) read scale is fixed by this library (the pages read o = S q unscaled).
 *
 * Conventions shared by every entry point:
 *  - All pointers are DEVICE pointers unless stated, owned by the caller, contiguous
 *    row-major, and 16-byte aligned. The library keeps no pointer after a call returns.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *    the call returns without waiting. Calls on one stream run in order.
 *  - Return value: GDR_OK (0) or a negative gdr_status. Argument errors are detected on the
 *    host before anything is enqueued; the message is available from gdr_last_error() on
 *    the calling thread. Errors found on the device (a bounded wait that expired) are
 *    recorded in a per-device status word and reported by gdr_sync_status(). Nothing in
 *    the library traps, aborts or exits.
 *  - No entry point allocates device memory on the call path: scratch space is the
 *    caller's `workspace`. The status word is a statically sized device variable.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = -1,  /* null pointer, non-positive size, bad enum, S_T overlaps an input */
    GDR_ERR_UNSUPPORTED = -2,  /* shape outside what the kernels implement (see each entry point) */
    GDR_ERR_MISALIGNED = -3,   /* a pointer not 16-byte aligned */
    GDR_ERR_WORKSPACE = -4,    /* workspace missing or smaller than *_workspace_bytes() */
    GDR_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed (message has the CUDA error) */
    GDR_ERR_TIMEOUT = -6,      /* a device-side bounded wait expired (reported by gdr_sync_status) */
    GDR_ERR_DEVICE = -7,       /* the current device is not an sm_100 part */
    GDR_ERR_RANGE = -8         /* device-side: a value left the range a kernel supports (kept for
                                  ABI stability; no current kernel reports it) */
} gdr_status;

typedef enum {
    GDR_DECAY_NONE = 0,     /* DeltaNet: alpha = 1, g unused (may be NULL) */
    GDR_DECAY_SCALAR = 1,   /* Gated DeltaNet: g is [.., H] (one log-decay per head and token) */
    GDR_DECAY_CHANNEL = 2   /* Kimi Delta Attention: g is [.., H, d_k] (per key channel) */
} gdr_decay_mode;

typedef enum {
    GDR_F32 = 0,   /* float32 */
    GDR_BF16 = 1   /* bfloat16 */
} gdr_dtype;

/* Element types: `dtype` is the type of q, k, v; `o_dtype` the type of the output o. Supported
 * pairs: (F32, F32), (BF16, F32) and (BF16, BF16). Arithmetic is fp32 (fp32 accumulation, fp32
 * state) in every case. A bf16 output adds its own rounding (up to 2^-8 relative per element)
 * on top of the computation's error. */

/*
 * gdr_chunk_fwd -- chunkwise-parallel forward over a whole sequence (training / prefill form).
 *
 * Defined by: "linear attention and its gated descendants", Chunkwise Parallel Form (state
 * carried across chunk boundaries, a masked intra-chunk part, chunk size C) generalised to the
 * delta rule through the compact WY/UT form of a chunk of updates ("Linear Attention &
 * DeltaNet", item 3): per chunk, T = (I + strictly_lower(diag(beta) (K*gamma)(K/gamma)^T))^-1,
 * W = T diag(beta)(K*gamma), U = T diag(beta) V, Delta = U - W S^T,
 * O = [(Q*gamma) S^T + (M * (Q*gamma)(K/gamma)^T) Delta] / sqrt(d_k) with M causal including
 * the diagonal, and S <- S Diag(gamma_C) + Delta^T (K * gamma_C/gamma), where gamma_r is the
 * exponential of the inclusive cumulative log-decay inside the chunk. The result equals the
 * token-by-token recurrence above up to rounding.
 *
 *   q, k      [B, T, H, d_k]   dtype            queries and keys (the caller applies any
 *                                               feature map / normalisation)
 *   v         [B, T, H, d_v]   dtype            values
 *   g         fp32 log-decay (<= 0 for a decay): [B, T, H] for SCALAR, [B, T, H, d_k] for
 *             CHANNEL, ignored (may be NULL) for NONE. alpha = exp(g).
 *   beta      [B, T, H]        fp32             write strength, normally in [0, 1]
 *   S0        [B, H, d_v, d_k] fp32, or NULL for a zero initial state
 *   o         [B, T, H, d_v]   o_dtype          output (written)
 *   S_T       [B, H, d_v, d_k] fp32, or NULL; the state after the last token. It may be the
 *             same pointer as S0 (in-place carry); any other overlap with an input is an error.
 *   B, T, H   batch, tokens, heads (T may be any value >= 1; a ragged last chunk is masked)
 *   dtype, o_dtype  element types of q/k/v and of o (see gdr_dtype).
 *   d_k, d_v  head dims. Supported: bf16 with d_k = d_v = 128 and chunk = 64 runs on the
 *             tensor cores (tcgen05); otherwise d_k, d_v in {32, 64, 128} run on an fp32
 *             CUDA-core path (fp32 accumulation, no TF32). Anything else: GDR_ERR_UNSUPPORTED.
 *   chunk     chunk size C; 64 is the supported value.
 *   Decay range: any g <= 0 (alpha in [0, 1]), including alpha = 0 (g far below zero). On the
 *             tensor-core path the channel gate folds its decay factors into fp16 operands around a
 *             mid-chunk reference for the key channels whose cumulative log-decay stays within a
 *             narrow band inside the chunk; the other channels' terms are added exactly on the CUDA
 *             cores (slower when many channels decay strongly, never out of range).
 *   workspace device scratch of at least gdr_chunk_fwd_workspace_bytes(...) bytes (may be
 *             NULL when that is 0). Contents on entry do not matter; the library does not
 *             keep it after the enqueued work completes. Two calls in flight at the same time
 *             must not share one workspace.
 * Launches (tensor-core path): B * H <= 100 run as one cooperative kernel with one CTA per SM, in
 * which the per-chunk factor pipelines hand their blocks to the per-head state passes through a
 * ring in the workspace: eight blocks per head (0.6 MB per head) up to 56 heads, 17 for the channel
 * gate (but few heads with long sequences run the segment scan of gdr_chunk_fwd_scan; see
 * gdr_chunk_fwd_plan). Above that a prep kernel on every SM first writes the blocks of the leading
 * chunks of each head to the workspace, and the ring has a slot for every later chunk. The
 * workspace then holds one block (73 KB) per chunk of every head. More than 100 heads use two
 * kernels that exchange every block through the workspace. gdr_chunk_fwd_plan reports which.
 */
int gdr_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const float* S0, void* o, float* S_T, int B, int T, int H, int d_k, int d_v,
                  int chunk, int mode, int dtype, int o_dtype, void* workspace,
                  size_t workspace_bytes, void* stream);

/* Bytes of device workspace gdr_chunk_fwd needs for this problem (0 if none). Returns 0 for
 * arguments gdr_chunk_fwd would reject. Host-only; enqueues nothing. */
size_t gdr_chunk_fwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int mode,
                                     int dtype, int o_dtype);

/*
 * gdr_chunk_fwd_ex -- gdr_chunk_fwd with the mixer layer's input steps done inside the kernels.
 *
 * Defined by: "Linear Attention & DeltaNet", minimal pseudocode (recurrent reference form): before
 * the recurrence, q and k pass through a feature map, the write strength is beta = sigmoid of a
 * projection, and the decay gate is a squashed projection. Each step below is applied, in fp32, to
 * the values as the kernels read them, so that no separate pass writes and re-reads them:
 *
 *   GDR_PRO_L2NORM_QK     q and k hold raw vectors: each (b, t, h) vector of q and of k is divided
 *                         by its Euclidean norm (no epsilon). An all-zero vector stays zero, and so
 *                         does one whose squared norm underflows fp32 (norm below about 1e-19).
 *   GDR_PRO_BETA_SIGMOID  beta holds logits x; the write strength is 1 / (1 + e^-x).
 *   GDR_PRO_GATE_SOFTPLUS g holds gate logits a (same shape as g); the log-decay is
 *                         g = -A_h softplus(a) = -A_h log(1 + e^a), with A = gate_scale [H] fp32
 *                         (NULL: A_h = 1). A_h >= 0 keeps g <= 0. A_h = 0.05 gives the decay
 *                         exp(-0.05 softplus(.)) of the small Gated DeltaNet workload; A_h = 1 with
 *                         a = -x gives alpha = sigmoid(x), the pseudocode's gate. Needs mode SCALAR
 *                         or CHANNEL.
 *
 *   prologue    bitwise OR of gdr_prologue flags (0 = gdr_chunk_fwd).
 *   gate_scale  device pointer, [H] fp32, 16-byte aligned, or NULL; read only with
 *               GDR_PRO_GATE_SOFTPLUS.
 * Every other argument, the paths and the errors are as gdr_chunk_fwd; a prologue bit outside the
 * three above is GDR_ERR_INVALID_ARG. The workspace size and the plan do not depend on `prologue`.
 */
typedef enum {
    GDR_PRO_NONE = 0,
    GDR_PRO_L2NORM_QK = 1,
    GDR_PRO_BETA_SIGMOID = 2,
    GDR_PRO_GATE_SOFTPLUS = 4
} gdr_prologue;

int gdr_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     const float* S0, void* o, float* S_T, int B, int T, int H, int d_k, int d_v,
                     int chunk, int mode, int dtype, int o_dtype, int prologue,
                     const float* gate_scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdr_decode_step -- one recurrent step for a batch of states (the decoding view).
 *
 * Defined by: "linear attention and its gated descendants", Recurrent Linear Attention for
 * Inference (constant-size state, fixed cost per token) and the update rules above; "Linear
 * Attention & DeltaNet", minimal pseudocode (one update then one read per token).
 * Per (b, h) and per row j of S:  s_bar = s_j * alpha;  p = s_bar . k;  a = s_bar . q;
 * delta = beta (v_j - p);  o_j = (a + delta (k . q)) / sqrt(d_k);  s_j <- s_bar + delta k.
 * S is read once and written once.
 *
 *   q, k   [B, H, d_k] dtype;  v [B, H, d_v] dtype;  beta [B, H] fp32
 *   g      [B, H] (SCALAR) or [B, H, d_k] (CHANNEL) fp32, ignored for NONE
 *   S      [B, H, d_v, d_k] fp32, updated in place
 *   o      [B, H, d_v] o_dtype (written); dtype / o_dtype pairs as for gdr_chunk_fwd
 *   d_k in {32, 64, 128, 256}, d_v >= 1.
 */
int gdr_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                    float* S, void* o, int B, int H, int d_k, int d_v, int mode, int dtype,
                    int o_dtype, void* stream);

/* gdr_decode_step with the prologue steps of gdr_chunk_fwd_ex applied to q, k (per (b, h) vector),
 * beta and g in-kernel; arguments and errors otherwise as gdr_decode_step. */
int gdr_decode_step_ex(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       float* S, void* o, int B, int H, int d_k, int d_v, int mode, int dtype,
                       int o_dtype, int prologue, const float* gate_scale, void* stream);

/*
 * gdr_chunk_fwd_scan -- gdr_chunk_fwd with each sequence split into n_seg segments that run in
 * parallel (sequence-level parallelism for few heads and long sequences).
 *
 * Defined by: "linear attention and its gated descendants", Hardware Performance (with few
 * sequences x heads there is not enough parallel work; sequence-level parallelism) and the closing
 * summary of the gated variants (the update is a transition plus a write, S_t = S_{t-1} A_t + B_t,
 * with A_t = Diag(alpha_t)(I - beta_t k_t k_t^T) and B_t = beta_t v_t k_t^T in this library's
 * orientation, and such maps compose associatively). With segments of T / n_seg tokens, M(i) the
 * product of the A_t of segment i and ^0 a run from a zero state:
 *     S_in(i + 1) = S_in(i) M(i) + S_end^0(i),   S_in(0) = S0,   S_T = S_in(n_seg),
 *     o_t = o_t^0 + S_in(i) (scale * prod_{u <= t in segment i} A_u) q_t.
 * The library computes o^0 and S_end^0 by the chunked forward on the [B * n_seg, T / n_seg, H] view
 * of the inputs, M(i) and the per-token read-outs by the same forward with v = 0 from the identity
 * state, then the carry (n_seg steps per head) and the correction on warp MMAs (tf32 operands,
 * fp32 accumulation). The result equals gdr_chunk_fwd's up to rounding.
 *
 * Arguments as gdr_chunk_fwd, plus n_seg >= 2. Supported: the tensor-core shapes (bf16 q/k/v,
 * d_k = d_v = 128, chunk 64), any decay mode, T a multiple of n_seg * 64; otherwise
 * GDR_ERR_UNSUPPORTED. S_T may be S0. workspace: gdr_chunk_fwd_scan_workspace_bytes(...) bytes
 * (the forward's workspace for the view, a zero value tensor, the per-token read-outs in fp32 and
 * four states per segment; plus an fp32 copy of o when o is bf16).
 */
int gdr_chunk_fwd_scan(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       const float* S0, void* o, float* S_T, int B, int T, int H, int d_k, int d_v,
                       int chunk, int mode, int dtype, int o_dtype, int n_seg, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace of gdr_chunk_fwd_scan (0 for arguments it would reject). Host-only. */
size_t gdr_chunk_fwd_scan_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int mode,
                                          int dtype, int o_dtype, int n_seg);

/*
 * gdr_chunk_fwd_gdn2 / gdr_decode_step_gdn2 -- Gated DeltaNet-2: separate channel-wise erase and
 * write gates in place of the single write strength beta.
 *
 * Defined by: "Linear Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer Routing",
 * Sec. 3 (Gated DeltaNet-2 and the gate definitions before it): the decay-adjusted memory
 * S_bar = S_{t-1} Diag(alpha_t), a gated erase direction e_t (.) k_t on the key side, a gated write
 * target w_t (.) v_t on the value side, and one residual written along k_t:
 *
 *     S_t = S_bar + (w_t (.) v_t - S_bar (e_t (.) k_t)) k_t^T ,   o_t = S_t q_t / sqrt(d_k).
 *
 * The page's formulas are stripped; this reading keeps a single rank-one residual per token and
 * reduces to gdr_chunk_fwd for e_t = beta_t 1, w_t = beta_t 1 (Kimi Delta Attention with the channel
 * decay, Gated DeltaNet with the scalar one), as the page states.
 *
 *   erase   [B, T, H, d_k] fp32 (decode: [B, H, d_k]); usually in [0, 1]
 *   write   [B, T, H, d_v] fp32 (decode: [B, H, d_v]); usually in [0, 1]
 *   the other arguments as gdr_chunk_fwd / gdr_decode_step (no beta; any decay mode).
 * In the chunk form the erase direction E = e (.) K takes the place of diag(beta) K on the left of the
 * Gram matrix and in W, and w (.) V that of diag(beta) V in U:
 * A_ri = sum_c E_rc k_ic exp(Gamma_rc - Gamma_ic) (i < r), W = T (E * gamma), U = T (w (.) V).
 * With the channel decay at the tensor-core shapes (bf16, d_k = d_v = 128, chunk 64) it runs on the
 * channel gate's tensor-core plans and needs gdr_chunk_fwd_gdn2_workspace_bytes(...) of
 * workspace; otherwise on the fp32 CUDA-core kernels with no workspace (d_k, d_v in {32, 64, 128},
 * chunk 64). Decode: as gdr_decode_step. Errors as gdr_chunk_fwd / gdr_decode_step.
 */
int gdr_chunk_fwd_gdn2(const void* q, const void* k, const void* v, const float* g, const float* erase,
                       const float* write, const float* S0, void* o, float* S_T, int B, int T, int H,
                       int d_k, int d_v, int chunk, int mode, int dtype, int o_dtype, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace of gdr_chunk_fwd_gdn2 (0 when it runs on the CUDA cores or would be rejected). */
size_t gdr_chunk_fwd_gdn2_workspace_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int mode,
                                          int dtype, int o_dtype);

int gdr_decode_step_gdn2(const void* q, const void* k, const void* v, const float* g, const float* erase,
                         const float* write, float* S, void* o, int B, int H, int d_k, int d_v, int mode,
                         int dtype, int o_dtype, void* stream);

/*
 * gdr_chunk_bwd -- gradients of gdr_chunk_fwd (the training backward pass).
 *
 * Defined by: the forward above (its value is the token recurrence of "Linear Attention & DeltaNet",
 * How it works, items 3-4, with the decay of "linear attention and its gated descendants", Gated
 * DeltaNet and Kimi Delta Attention), differentiated in reverse mode. For a loss L with dO = dL/do
 * and dS_T = dL/dS_T, the call returns dL/dq, dL/dk, dL/dv, dL/dg, dL/dbeta and dL/dS0, where g, beta,
 * q, k are the values gdr_chunk_fwd reads (no prologue). Per row j of the state, in reverse token
 * order (s_bar = s (.) alpha, p = s_bar . k, delta = beta (v_j - p), s' = s_bar + delta k):
 *     ds' = ds + scale do_j q;  ddelta = ds' . k;  dv_j = beta ddelta;  ds_bar = ds' - beta ddelta k;
 *     ds = ds_bar (.) alpha;  dq += scale do_j s';  dk += delta ds' - beta ddelta s_bar;
 *     dbeta += ddelta (v_j - p);  dg += ds_bar (.) s_bar  (summed over channels for SCALAR).
 *
 *   q, k, v, g, beta, S0  the forward's inputs, as for gdr_chunk_fwd (S0 may be NULL: zero)
 *   dO        [B, T, H, d_v] dtype (the type of q, k, v)
 *   dS_T      [B, H, d_v, d_k] fp32, or NULL (zero)
 *   dq, dk    [B, T, H, d_k] fp32 (written);  dv [B, T, H, d_v] fp32 (written)
 *   dg        fp32 in the shape of g (written; NULL for NONE);  dbeta [B, T, H] fp32 (written)
 *   dS0       [B, H, d_v, d_k] fp32 (written), or NULL
 *   d_k, d_v  in {32, 64, 128}; dtype F32 or BF16; arithmetic fp32 on the CUDA cores.
 *   workspace at least gdr_chunk_bwd_workspace_bytes(...) bytes: the state before every token,
 *             B * H * T * d_v * d_k * 4 bytes (the reverse sweep reads it back instead of
 *             recomputing). Not kept after the enqueued work completes.
 * Launches: two kernels, one CTA of 512 threads per (b, h). No output may overlap an input, another
 * output or the workspace. Errors as gdr_chunk_fwd.
 */
int gdr_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const float* S0, const void* dO, const float* dS_T, float* dq, float* dk, float* dv,
                  float* dg, float* dbeta, float* dS0, int B, int T, int H, int d_k, int d_v, int mode,
                  int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace gdr_chunk_bwd needs (0 for arguments it would reject). Host-only. */
size_t gdr_chunk_bwd_workspace_bytes(int B, int T, int H, int d_k, int d_v, int mode, int dtype);

/* Number of kernel launches one gdr_chunk_fwd call makes for this problem (0 if it would be
 * rejected). Host-only. */
int gdr_chunk_fwd_launches(int B, int T, int H, int d_k, int d_v, int chunk, int mode, int dtype,
                           int o_dtype);

/* How gdr_chunk_fwd runs a problem (no counterpart in the method; host-only). */
typedef enum {
    GDR_PLAN_INVALID = 0,      /* the call would be rejected */
    GDR_PLAN_CUDA_CORE = 1,    /* one fp32 CUDA-core kernel */
    GDR_PLAN_TWO_PASS = 2,     /* tensor cores: prep kernel (all chunks), then state kernel */
    GDR_PLAN_FUSED = 3,        /* tensor cores: one cooperative kernel (prep and state passes) */
    GDR_PLAN_PREP_FUSED = 4,   /* tensor cores: prep kernel for the first chunks of every head, then
                                  the cooperative kernel for the rest */
    GDR_PLAN_SCAN = 5          /* tensor cores: segment scan (see gdr_chunk_fwd_scan): prep kernel, one
                                  state kernel for the segments' data and transition chains, carry,
                                  output correction */
} gdr_plan;

/* The plan gdr_chunk_fwd uses for this problem (a gdr_plan value). For GDR_PLAN_PREP_FUSED,
 * *precomputed_chunks (if not NULL) receives the number of leading chunks per head the first
 * kernel prepares (gdr_chunk_fwd_ex with prologue flags prepares a few more, its prep tasks being
 * longer, inside the same workspace); for GDR_PLAN_SCAN, the number of segments; 0 otherwise. Chosen from the shape
 * alone: at most 16 heads with at least 256 chunks each run the segment scan, with s segments, the
 * largest power of two in 2 .. 16 with B * H * s <= 64, at least 16 chunks per segment and T a
 * multiple of 64 s (4 segments for 16 heads, 16 for 1-4 heads); otherwise B * H <= 56 heads run
 * fused (the chains are the bound), 57-100 heads
 * prepare the first chunks on every SM so that the fused kernel's remaining prep CTAs keep up with
 * the chains (the channel gate at any head count where they would not), more than 100 heads run two
 * passes. gdr_chunk_fwd_noalloc never uses the segment scan. */
int gdr_chunk_fwd_plan(int B, int T, int H, int d_k, int d_v, int chunk, int mode, int dtype,
                       int o_dtype, int* precomputed_chunks);

/* Diagnostics (no counterpart in the method): per-kernel timing of the next chunked forward or
 * backward. The next gdr_chunk_fwd(_ex, _scan), gdr_chunk_fwd_noalloc or gdr_chunk_bwd call made on
 * the calling host thread records
 * events[i] on its stream right after it enqueues its i-th kernel, for i < min(n_events,
 * launches), then forgets the events; a call that fails validation forgets them too.
 *   events    n_events cudaEvent_t handles created by the caller (owned by the caller; timing
 *             events if durations are wanted). An event recorded by the caller before the call
 *             and events[0] bracket the first kernel, events[i-1] and events[i] the i-th one.
 *   n_events  0 .. 8; 0 clears a pending request.
 * Returns GDR_OK, or GDR_ERR_INVALID_ARG for n_events outside 0 .. 8 or a NULL events array
 * with n_events > 0. Host-only; enqueues nothing by itself. */
int gdr_profile_next_call(void* const* events, int n_events);

/*
 * gdr_chunk_fwd_host -- gdr_chunk_fwd on host-resident tensors, copies overlapped with the work.
 *
 * No counterpart in the method: a transfer schedule for callers whose inputs and outputs live
 * in host memory. Arguments as gdr_chunk_fwd, except that q, k, v, g, beta, S0 (inputs) and o,
 * S_T (outputs) are HOST pointers, and `staging` is caller-owned device memory of at least
 * gdr_chunk_fwd_host_staging_bytes(...) bytes (16-byte aligned) in place of the workspace.
 * The batch is processed in pieces of consecutive sequences (at most 8 pieces): the inputs of
 * piece i are copied in on one internal stream while piece i-1 computes on `stream` and the
 * outputs of piece i-2 are copied out on another internal stream; staging holds two pieces.
 * Page-locked host memory lets the copies run asynchronously and overlap (pageable memory
 * works but serialises). The call returns once everything is enqueued; all of it is ordered
 * after the work already on `stream`, and `stream` waits for the last copy: when `stream` has
 * completed, o and S_T hold the results. The host buffers and staging must stay valid until
 * then. Two calls in flight at the same time must not share `staging`. The two internal streams
 * and a few events are created on the first call on each device and kept; they are shared by all
 * calls on the device, so calls made from several host threads at once are serialised while they
 * enqueue (a per-device lock), and their work is ordered as enqueued.
 * Errors: as gdr_chunk_fwd (validated before anything is enqueued), plus GDR_ERR_WORKSPACE for
 * a staging area that is missing or too small.
 */
int gdr_chunk_fwd_host(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       const float* S0, void* o, float* S_T, int B, int T, int H, int d_k, int d_v,
                       int chunk, int mode, int dtype, int o_dtype, void* staging, size_t staging_bytes,
                       void* stream);

/* Device staging gdr_chunk_fwd_host needs for this problem (bytes; 0 if it would be rejected). */
size_t gdr_chunk_fwd_host_staging_bytes(int B, int T, int H, int d_k, int d_v, int chunk, int mode,
                                        int dtype, int o_dtype);

/* Size of the scratch area built into the library for gdr_chunk_fwd_noalloc: 32 MiB of device
 * memory on every GPU that loads the library, held until the process exits. */
#define GDR_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * gdr_chunk_fwd_noalloc -- gdr_chunk_fwd for callers that cannot allocate device memory.
 *
 * The pages have no counterpart; this is a convenience of this library. Some callers cannot
 * call cudaMalloc for a workspace: a plugin inside a host program that owns all device memory
 * and hands the plugin only its inputs and outputs; code running in a loop where an allocation
 * (which may synchronise the device) is not allowed; a program that must not grow its device
 * footprint after start-up. This entry point takes the same arguments as gdr_chunk_fwd minus the
 * workspace and uses a fixed scratch area compiled into the library instead
 * (GDR_NOALLOC_SCRATCH_BYTES). DeltaNet and the scalar gate with B * H <= 56 (the channel gate:
 * <= 17) need a ring of eight hand-off blocks per head, which fits at any T. Larger problems need
 * one block per chunk of every head and are accepted while the total fits (see
 * gdr_chunk_fwd_workspace_bytes). It allocates nothing on any call.
 *
 *  - Shapes: only those that need scratch (bf16 q/k/v, d_k = d_v = 128, chunk = 64); other
 *    shapes need none and are rejected with GDR_ERR_UNSUPPORTED (call gdr_chunk_fwd with a null
 *    workspace for them). A problem needing more scratch than the area holds is rejected with
 *    GDR_ERR_UNSUPPORTED and a message giving both sizes; nothing is enqueued.
 *  - Set-up: the first call on each device looks up the area's device address (once per device,
 *    with that device current). Make that first call before any stream capture.
 *  - Sharing: every call on a device uses the same area, which keeps the last call's contents.
 *    Nothing in it needs to start at zero: every byte a call reads there is written earlier by
 *    the same call, in stream order. Calls whose execution overlaps on the GPU (for example on two
 *    streams) race on the area and produce wrong results; serialise them.
 * Errors and everything else: as gdr_chunk_fwd.
 */
int gdr_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* S0, void* o, float* S_T, int B, int T,
                          int H, int d_k, int d_v, int chunk, int mode, int dtype, int o_dtype,
                          void* stream);

/* Waits for `stream`, then reads and clears the calling device's status word. Returns
 * GDR_OK, GDR_ERR_TIMEOUT (a kernel's bounded wait expired; its outputs are invalid),
 * GDR_ERR_RANGE (a value out of a kernel's range) or GDR_ERR_CUDA (the stream reported a CUDA
 * error). */
int gdr_sync_status(void* stream);

/* Message for the last non-zero return on the calling thread ("" if none). The pointer stays
 * valid until the next gdr_* call on the same thread. */
const char* gdr_last_error(void);

/* Self-test of the device-side bounded waits (no counterpart in the method; a diagnostic). Runs one
 * small kernel whose roles are laid out like the state pass's -- a copy role waiting on a ring flag,
 * an MMA-issue role waiting on the copy role, epilogue warps waiting on the issue role -- where the
 * ring flag is one that nothing ever sets. The copy role's wait is bounded by limit_us microseconds
 * (instead of the kernels' 2 s), the other roles' by 100 times that: the copy role's wait expires,
 * records GDR_ERR_TIMEOUT and releases the other roles through the CTA's abort flag, so the run ends
 * after about limit_us. Synchronous: waits for `stream` before and after, clears the status
 * word, and returns what gdr_sync_status returns for the run (GDR_ERR_TIMEOUT when the bounded waits
 * work). *elapsed_ns (if not NULL) receives the kernel's own measure of how long its roles waited.
 * limit_us must be in 1 .. 1000000. Nothing faults or traps; the stream stays usable. */
int gdr_selftest_bounded_wait(unsigned limit_us, unsigned long long* elapsed_ns, void* stream);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
