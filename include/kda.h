/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library.
 *
 * The operation (Kimi Delta Attention, "KDA"), per head with a d_k x d_v state S
 * (d_k = d_v = 128 here), for tokens t = 1..T of one sequence:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T (scale * q_t)
 *
 * with a per-channel decay alpha_t = exp(g_t) in [0,1]^{d_k} and a scalar write
 * strength beta_t.  Source: "Kimi Linear: An Expressive, Efficient Attention
 * Architecture" (research notes on arXiv 2510.26692), section Method, "From
 * Linear Attention to KDA", eq. KDA and its residual reading
 * S~ = Diag(alpha_t) S_{t-1}, S_t = S~ + beta_t k_t (v_t - S~^T k_t)^T.
 * The state's rows are key channels (Diag(alpha) scales rows); scale = 1 is the
 * pages' o_t = S_t^T q_t.
 *
 * Conventions for every entry point below:
 *  - All tensor pointers are DEVICE pointers owned by the caller (allocated by
 *    whatever allocator it uses); the library never allocates, frees or keeps
 *    them.  Scratch memory comes only from the caller's `workspace`.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Arguments are validated on the host before any launch;
 *    a rejected call launches nothing and returns a status code.  No entry
 *    point throws, aborts or prints.
 *  - Token tensors are row-major with the head dim fastest: [B, T, H, 128]
 *    (dense) or [1, Ttot, H, 128] (packed, with cu_seqlens).  States are fp32
 *    [N, H, 128 (key channel), 128 (value channel)], value channel fastest.
 *  - Pointers must be 16-byte aligned.  Outputs must not alias inputs except
 *    where stated (the decode state is updated in place).
 *  - Device-side waits are bounded: a kernel that waits too long gives up,
 *    records KDA_ERR_TIMEOUT in a device status word and exits cleanly; read it
 *    with kda_device_status() (which synchronises `stream`).
 *  - The caller's current CUDA device must be the device that holds the
 *    pointers.
 */
#ifndef KDA_B200_H_
#define KDA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* NULL where not allowed, bad size, misaligned pointer */
    KDA_ERR_UNSUPPORTED = 2,  /* valid request this library does not implement (e.g. head dim != 128) */
    KDA_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than the matching *_workspace() query */
    KDA_ERR_CUDA = 4,         /* a CUDA runtime / driver call or kernel launch failed */
    KDA_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (see kda_device_status) */
} kda_status;

typedef enum {
    KDA_BF16 = 0,
    KDA_FP32 = 1
} kda_dtype;

/* Human-readable name of a status code (static storage; never NULL). */
const char *kda_status_string(int status);

/* Head dimension this library supports (d_k = d_v): 128. */
int kda_head_dim(void);

/* Detail of the last host-side rejection or CUDA error on this thread
 * (static thread-local storage; empty string when none). */
const char *kda_last_error(void);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device: KDA_OK, or KDA_ERR_TIMEOUT if any kernel of this library gave
 * up a bounded wait since the last call, or KDA_ERR_CUDA if the sync failed. */
int kda_device_status(void *stream);

/* Testing hook for the failure path of the bounded device-side waits (no
 * counterpart on the pages).  wait_limit_cycles > 0 sets the bound of every
 * later device-side wait of this library on the current device, in SM cycles;
 * <= 0 restores the default of 2^31 (about a second).  skip_chunk >= 0 makes
 * every later launch of the chunk kernels' map/whole-sequence pass skip the
 * q/k/g load of that chunk (counted inside the launch's sequence segment) of
 * each (sequence, head): the wait for it then gives up, the kernel records
 * KDA_ERR_TIMEOUT in the device status word and exits cleanly, without a trap
 * or a hang, and that call's results are undefined.  skip_chunk < 0 turns the
 * skip off.  The settings are global to the device: change them only while no
 * call of this library runs.  Synchronous (legacy default stream).  Production
 * code never needs it. */
int kda_debug_fault_injection(long long wait_limit_cycles, int skip_chunk);

/* Optional tracing hook for kda_chunk_fwd.  When `events` is non-NULL it must
 * point to 5 cudaEvent_t created by the caller on the current device; every
 * later kda_chunk_fwd call on this thread records them on its stream around
 * its kernels: [0] before the plan kernel, [1] after it, [2] after the first
 * phase (the segments' maps; same as [1] when the sequences are not
 * segmented), [3] after the combine pass, [4] after the segments' outputs (or
 * after the only launch, unsegmented).  They are recorded with
 * cudaEventRecordExternal, so a call captured into a CUDA graph records them
 * as event nodes each time the graph runs.  Pass NULL to stop.  The events
 * stay owned by the caller. */
int kda_set_trace_events(void *events, int n_events);

/* ------------------------------------------------------------------------
 * kda_chunk_fwd -- chunkwise-parallel prefill.
 *
 * Computes o and the final state of the recurrence above over whole sequences
 * (chunks of 64 tokens; "Kimi Linear: An Expressive, Efficient Attention
 * Architecture", section "Chunkwise Algorithm": per-channel decay and rank-1
 * corrections unrolled inside a chunk, WY representation, UT transform, only
 * the fixed-size state crossing chunks; the inverse (I + A)^{-1} by forward
 * substitution, "Kimi Linear" news rewrite, section on the hardware-efficient
 * chunkwise algorithm).  The result is the recurrence's, up to rounding.
 *
 *   q, k      [B,T,H,128] (dense) or [1,Ttot,H,128] (packed); dtype bf16 or fp32.
 *             With l2norm_qk != 0 each (token, head) row of q and k is first
 *             normalised to unit L2 norm (x / sqrt(sum x^2 + 1e-6)).
 *   v         same shape and dtype as q.
 *   g         fp32, same shape: log of the per-channel decay (alpha = exp(g)),
 *             expected <= 0.  Values below -1e4 are treated as -1e4 (alpha = 0
 *             in fp32).
 *   beta      fp32 [B,T,H] (or [1,Ttot,H]).
 *   initial_state  fp32 [N,H,128,128] or NULL (zero state).
 *   final_state    fp32 [N,H,128,128] or NULL (not written).  May alias
 *                  initial_state.
 *   o         output, same shape and dtype as q.
 *   cu_seqlens     NULL for dense input (N = B sequences of T tokens; then
 *                  num_seqs must be 0), or a device int32 [num_seqs+1] of
 *                  non-decreasing token offsets with cu_seqlens[0] = 0 and
 *                  cu_seqlens[num_seqs] = T (T = total packed tokens); then B
 *                  must be 1 and N = num_seqs >= 1.  Empty sequences are allowed.
 *                  The offsets are read on the device only (never copied back).
 *   scale     multiplies q (1.0 = o_t = S_t^T q_t).
 *   workspace      device scratch of at least kda_chunk_fwd_workspace_min(...)
 *                  bytes (kda_chunk_fwd_workspace(...) for the fastest
 *                  schedule), 256-byte aligned; contents need not be
 *                  initialised and are clobbered.
 *
 * Tensor cores compute the chunk contractions with bf16 operands and fp32
 * accumulation; the state is carried in fp32.  fp32 inputs are rounded to
 * bf16 where they feed the tensor cores.  Rounding: a bf16 o is rounded from
 * its fp32 accumulator once, to nearest with ties to even; the bf16 operands
 * the kernels form on chip (gated keys and queries, W, U~, the state copy) are
 * rounded to nearest with ties away from zero.
 */
/* How a kda_chunk_fwd call with these sizes on the current device is split:
 * 0 when every (sequence, head) runs in one CTA; otherwise the length in tokens
 * of each sequence's first segment, with the length of the following segments
 * (the last one holds the rest) in *middle_tokens when that is not NULL.  A
 * segmented call runs the segments' maps in one launch, then the combine pass,
 * then the segments' outputs in a second launch.
 * -1 (and -1 in *middle_tokens) when the cuts depend on the sequence lengths:
 * packed calls (cu_seqlens) with num_seqs <= 64 whose (sequence, head) pairs
 * outnumber a third of the SMs and whose total length exceeds 16 chunks.  Their
 * plan, made on the device from cu_seqlens, cuts each sequence at a common
 * target length chosen to balance the SMs (short sequences stay whole);
 * segment 0 then runs its output in the first launch, from the initial state,
 * and the later segments run their maps there and their outputs in the second.
 * kda_chunk_fwd_plan_items reports the cuts after a call.
 * Informational (profiling); it never changes what is computed. */
int kda_chunk_fwd_segment_tokens(int B, int T, int H, int num_seqs, int *middle_tokens);

/* The segment table that the last kda_chunk_fwd or kda_gdn_chunk_fwd call with
 * these sizes left at the start of `workspace`: copies up to max_rows rows of
 * five ints (sequence, first token, end token, segment index g, segment count
 * G) into the host array `rows` and returns the number of segments, or -1 on a
 * CUDA error.  Synchronous (it waits for the device).  Informational: tests and
 * profiling. */
int kda_chunk_fwd_plan_items(const void *workspace, int B, int T, int H, int num_seqs, int *rows, int max_rows);

/* Workspace bytes for a kda_chunk_fwd call with the same B, T, H, num_seqs
 * (0 = dense), dtype and l2norm_qk, on the current device. */
size_t kda_chunk_fwd_workspace(int B, int T, int H, int num_seqs, int dtype, int l2norm_qk);

/* The smallest workspace kda_chunk_fwd accepts for the same arguments.  With a
 * workspace of at least kda_chunk_fwd_workspace() bytes a segmented call keeps
 * each segment map pass's per-chunk products (about 66 KB per chunk and head,
 * e.g. ~1.2 GB at B=1 H=16 T=65536) and its output pass reads them back instead
 * of recomputing them; with less (but at least this many) bytes it recomputes
 * them.  Both give bit-identical results; the first is faster.
 * Calls that take the balanced plan (kda_chunk_fwd_segment_tokens() == -1) also
 * need per-segment states, up to (num_seqs + ceil((T/64 + num_seqs) / 16)) x H
 * x 192 KiB.  With a workspace smaller than that (but at least this many bytes)
 * they run unsegmented, one CTA per (sequence, head): slower, and equal to the
 * segmented results only up to rounding. */
size_t kda_chunk_fwd_workspace_min(int B, int T, int H, int num_seqs, int dtype, int l2norm_qk);

int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                  const float *initial_state, float *final_state, void *o, const int32_t *cu_seqlens,
                  int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk,
                  void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * kda_gdn_chunk_fwd -- chunkwise prefill with a per-head scalar decay (gated
 * DeltaNet).
 *
 * The same recurrence with alpha_t = exp(g_t) * (1, ..., 1): one forgetting
 * rate per head and token, shared by every key channel.  "Kimi Linear: An
 * Expressive, Efficient Attention Architecture", section Method, "From Linear
 * Attention to KDA": GDN adds a per-head scalar forgetting rate; KDA makes it a
 * per-channel vector.  With g broadcast over the 128 channels, kda_chunk_fwd
 * computes the same result; this entry point reads 4 bytes of gate per
 * (token, head) instead of 512 and computes the decay factors once per token
 * instead of once per (token, channel).
 *
 *   g         fp32 [B,T,H] (or [1,Ttot,H] with cu_seqlens): log of the per-head
 *             decay, expected <= 0 (values below -1e4 are treated as -1e4).
 *   Every other argument, the layouts, the workspace (size it with
 *   kda_chunk_fwd_workspace() of the same arguments), the numerics and the
 *   error behaviour are those of kda_chunk_fwd.
 */
int kda_gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      const float *initial_state, float *final_state, void *o, const int32_t *cu_seqlens,
                      int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk,
                      void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * kda_dplr_chunk_fwd -- chunkwise prefill of the general (untied) DPLR
 * recurrence, the comparison point for KDA.
 *
 *     S_t = (I - a_t b_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T (scale * q_t),
 * with a_t, b_t free vectors per (token, head).  "Kimi Linear: An Expressive,
 * Efficient Attention Architecture", section "Chunkwise Algorithm": KDA is the
 * constrained DPLR transition whose low-rank pair is tied to the key (a = beta k,
 * b = k here), which halves the gated gram matrices per chunk (four become two)
 * and is what the pages' 64K kernel timing compares against.  This entry point
 * computes the untied form with the same chunk size, tiling and numerics as
 * kda_chunk_fwd, so the two can be timed against each other.
 *
 *   q, k, v, a, b  [B,T,H,128] (or [1,Ttot,H,128] with cu_seqlens), bf16 or fp32.
 *   g              fp32, same shape: log decay (<= 0; below -1e4 treated as -1e4).
 *   beta           fp32 [B,T,H].
 *   initial_state, final_state, o, cu_seqlens, num_seqs, scale: as in
 *   kda_chunk_fwd (no in-kernel L2 norm: normalise a, b, k, q beforehand).
 *   workspace      at least kda_dplr_chunk_fwd_workspace(B, T, H, num_seqs, dtype)
 *                  bytes, 256-byte aligned.
 * Each (sequence, head) runs in one CTA, chunk after chunk: unlike
 * kda_chunk_fwd there is no segment scan, so few long sequences use few SMs.
 * Up to 65535 sequences and 65535 heads.
 */
size_t kda_dplr_chunk_fwd_workspace(int B, int T, int H, int num_seqs, int dtype);

int kda_dplr_chunk_fwd(const void *q, const void *k, const void *v, const void *a, const void *b, const float *g,
                       const float *beta, const float *initial_state, float *final_state, void *o,
                       const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int dtype, float scale,
                       void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate.
 *
 * No counterpart on the pages: this is a library convenience.  Some callers
 * cannot provide a device workspace -- e.g. a plugin inside a runtime that
 * owns all device memory and gives it no allocator, or a serving loop that
 * must not call cudaMalloc (which may synchronise the device) mid-step.  This
 * entry point takes the same arguments as kda_chunk_fwd minus the workspace and
 * runs the same kernels, with its scratch in a static 64 MiB device array that
 * every GPU loading the library reserves until the process exits.  It never
 * allocates.
 *   - It uses kda_chunk_fwd_workspace() bytes when they fit in 64 MiB; else the
 *     kda_chunk_fwd_workspace_min() bytes, which run the same segments
 *     recomputing the chunk products (same bits, slower); B=1, H=16, T=65536
 *     bf16 needs about 31 MB that way.  A call needing more than 64 MiB even
 *     then returns KDA_ERR_UNSUPPORTED without launching; use kda_chunk_fwd.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress: a host-side lookup once the library's device code
 *     is loaded there, and still right after a device reset).  The first call
 *     on a device loads that code; make it before any stream capture.
 *   - All calls share the array: calls whose kernels can overlap on the GPU
 *     (e.g. on two unordered streams) race and corrupt each other's results.
 *     Calls ordered on one stream are safe; nothing needs clearing between them.
 */
int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g, const float *beta,
                          const float *initial_state, float *final_state, void *o, const int32_t *cu_seqlens,
                          int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk,
                          void *stream);

/* ------------------------------------------------------------------------
 * kda_decode_step -- one recurrent step for B sequences (one token each).
 *
 * Residual form, "Kimi Linear: An Expressive, Efficient Attention
 * Architecture", section Method (S~ = Diag(alpha) S; S = S~ + beta k (v - S~^T
 * k)^T) and section "Code Verification" (the naive recurrence multiplies by
 * exp(g), then writes the residual); decode uses this recurrent form (section
 * "Training and Inference").  Each head's state is read once and written once.
 *
 *   q, k, v   [B,H,128], dtype bf16 or fp32 (l2norm_qk as for kda_chunk_fwd).
 *   g         fp32 [B,H,128] log decay;  beta fp32 [B,H].
 *   state     fp32 [B,H,128,128], updated IN PLACE.
 *   o         [B,H,128], same dtype as q; o = S_new^T (scale * q).
 * All arithmetic is fp32 on CUDA cores.  No workspace.
 */
int kda_decode_step(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    float *state, void *o, int B, int H, int dtype, float scale, int l2norm_qk,
                    void *stream);

/* ------------------------------------------------------------------------
 * kda_recurrent_fwd -- fused recurrent segments: T tokens per sequence, the
 * state read once and written once.
 *
 * "Kimi Linear: An Expressive, Efficient Attention Architecture", section
 * "Training and Inference": long prompts take the chunk kernel, single steps and
 * segments of at most 64 tokens take a fused recurrent kernel, with a fixed
 * recurrent state cached between calls.  This is that kernel: the residual
 * form of kda_decode_step applied token by token, with each head's state held
 * on chip across the segment.  Any T >= 0 is accepted.  T = 1 computes what
 * kda_decode_step computes.  Its cost grows with T (~50 us per token at B=256,
 * H=32 on a B200) while one kda_chunk_fwd call costs ~0.75 ms for any T <= 64
 * there: from about 16 tokens the chunk call is faster, at bf16 tensor-core
 * operand precision instead of this kernel's fp32.
 *
 *   q, k, v   [B,T,H,128], dtype bf16 or fp32 (l2norm_qk as for kda_chunk_fwd).
 *   g         fp32 [B,T,H,128] log decay;  beta fp32 [B,T,H].
 *   state     fp32 [B,H,128,128], updated IN PLACE (the state after token T).
 *   o         [B,T,H,128], same dtype as q; o_t = S_t^T (scale * q_t).  Must not
 *             alias q, k or v.
 * All arithmetic is fp32 on CUDA cores.  No workspace.
 */
int kda_recurrent_fwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      float *state, void *o, int B, int T, int H, int dtype, float scale, int l2norm_qk,
                      void *stream);

/* ------------------------------------------------------------------------
 * kda_recurrent_bwd -- gradients of the operator (reverse mode).
 *
 * For a loss L with dL/do = d_o and dL/dS_T = d_final_state, computes dL/dq,
 * dL/dk, dL/dv, dL/dg, dL/dbeta and dL/dS_0 of the recurrence above.  Training
 * needs them ("Kimi Linear: An Expressive, Efficient Attention Architecture",
 * section "Training and Inference"; the pages' public-code audit lists
 * q/k/v/g/beta and initial-state gradient tests).  The reverse of each
 * recurrent step is evaluated exactly in fp32 on CUDA cores.  The recurrence
 * never mixes value columns, so each (sequence, head) runs as 16 one-warp CTAs of
 * 8 value columns (lane l holds key rows 4l..4l+3): each runs the forward storing its state
 * slice every 16 tokens, then walks the 16-token sub-chunks backwards,
 * recomputing their states in shared memory.  The slices' partial sums of dq,
 * dk, dg and dbeta are added by a second kernel in a fixed order, so results are
 * deterministic.  A chunked tensor-core backward is not part of this library.
 *
 *   q, k, v, d_o   [B,T,H,128], dtype bf16 or fp32 (q, k not normalised here).
 *   g              fp32 [B,T,H,128];  beta fp32 [B,T,H].
 *   initial_state  fp32 [B,H,128,128] or NULL (zero);  d_final_state likewise.
 *   dq, dk, dv, dg fp32 [B,T,H,128];  dbeta fp32 [B,T,H];
 *   d_initial_state fp32 [B,H,128,128] or NULL (not written).
 *   workspace      at least kda_recurrent_bwd_workspace(B, T, H) bytes, 256-byte
 *                  aligned: per (sequence, head), 64 KiB of state checkpoints per
 *                  16 tokens plus 16 x (3 x 128 + 1) x 4 bytes of partial sums per
 *                  token (about 28 KiB per token in all).
 * Dense batches only (no cu_seqlens).
 */
size_t kda_recurrent_bwd_workspace(int B, int T, int H);

int kda_recurrent_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                      const float *initial_state, const void *d_o, const float *d_final_state, float *dq,
                      float *dk, float *dv, float *dg, float *dbeta, float *d_initial_state, int B, int T, int H,
                      int dtype, float scale, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * kda_layer_fwd -- the KDA layer around the operator (forward).
 *
 * "Kimi Linear: An Expressive, Efficient Attention Architecture", section
 * "Neural Parameterization" and "Code Verification": bias-free Q/K/V
 * projections; depthwise causal ShortConv (kernel 4) then SiLU on q, k, v;
 * L2 norm of q and k; per-channel decay alpha = exp(-softplus(W_aup W_adown x))
 * (rank-128 low-rank projection); beta = sigmoid(W_b x); KDA (scale 1); per-head
 * RMSNorm (eps 1e-5, weight norm_w) times sigmoid(W_gup W_gdown x); output
 * projection.  Packed sequences: the convolution of each sequence starts from
 * its cached history (conv_state_in) or, when that is NULL, from zero history.
 *
 * All weights are bf16 row-major "out x in" (y = x W^T) except conv_* and
 * norm_w:
 *   W_in    [3*H*128 + 2*rank + H, d_model]: rows are, in order, W_q, W_k, W_v
 *           (H*128 each), W_adown (rank), W_gdown (rank), W_b (H).
 *   W_aup   [H*128, rank];  W_gup [H*128, rank];
 *   conv_w  bf16 [3*H*128, 4]: depthwise taps for the q, k, v channels; tap j
 *           multiplies x[t-3+j];
 *   norm_w  fp32 [128];     W_o [d_model, H*128].
 *   x       bf16 [total_tokens, d_model];  y bf16 [total_tokens, d_model].
 *   cu_seqlens  device int32 [num_seqs+1] (required);
 *   initial_state / final_state as in kda_chunk_fwd (N = num_seqs).
 *   conv_state_in / conv_state_out  bf16 [num_seqs, 3, 3*H*128] or NULL: the
 *           ShortConv cache, i.e. the last three convolution inputs (the q, k, v
 *           projections, in W_in's row order) before / at the end of each
 *           sequence, oldest first.  A sequence shorter than three tokens keeps
 *           the tail of its incoming history.  conv_state_out may equal
 *           conv_state_in.  Together with final_state this is the fixed-size
 *           cache the pages describe ("Training and Inference": KDA caches the
 *           short-convolution state and the recurrent state).
 * Every step runs in this library's kernels: the projections on the tensor
 * cores (kda_linear_bf16's GEMM, bf16 operands, fp32 accumulation), with beta,
 * the log decay g = -softplus(.) and the RMSNorm x sigmoid(gate) computed in
 * the epilogues of the GEMMs that produce their inputs; the operator's output
 * o stays fp32 up to the RMSNorm.  Intermediate activations (the projections,
 * q, k, v after the convolution, the normed output) are bf16.
 */
/* ------------------------------------------------------------------------
 * kda_linear_bf16 -- one projection of the KDA layer: y = x W^T.
 *
 * "Kimi Linear: An Expressive, Efficient Attention Architecture", section
 * "Neural Parameterization": the layer's Q/K/V, gate and output projections
 * are bias-free linear maps.  kda_layer_fwd runs all of them on this GEMM
 * (tcgen05 tensor cores, TMA-fed, fp32 accumulation in tensor memory); this
 * entry point exposes the plain form.
 *
 *   x   bf16 [M, K] row-major, row stride ldx elements;
 *   W   bf16 [N, K] row-major ("out x in"), row stride ldw;
 *   y   bf16 [M, N] row-major, row stride ldy; rounded from the fp32
 *       accumulator to nearest, ties to even.  Must not alias x or W.
 * Pointers 16-byte aligned and row strides multiples of 8 elements.  Any
 * M, N, K >= 1.  No workspace.
 */
int kda_linear_bf16(const void *x, int ldx, const void *W, int ldw, void *y, int ldy, int M, int N, int K,
                    void *stream);

typedef struct {
    const void *W_in;
    const void *W_aup;
    const void *W_gup;
    const void *conv_w;
    const float *norm_w;
    const void *W_o;
    int d_model;
    int H;
    int rank;
} kda_layer_weights;

size_t kda_layer_fwd_workspace(int total_tokens, int d_model, int H, int rank, int num_seqs);

int kda_layer_fwd(const void *x, const kda_layer_weights *w, const int32_t *cu_seqlens, int num_seqs,
                  int total_tokens, const float *initial_state, float *final_state,
                  const void *conv_state_in, void *conv_state_out, void *y,
                  void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------------
 * kda_layer_decode -- the layer on T new tokens per sequence from its cache.
 *
 * The inference path of "Kimi Linear" ("Training and Inference": single steps
 * and segments of at most 64 tokens take the fused recurrent kernel; the KDA
 * layer caches the short-convolution state and the recurrent state).  Same
 * pipeline as kda_layer_fwd for B sequences of T tokens each, with the
 * convolution reading its history from conv_state and the operator run by the
 * fused recurrent kernel (kda_recurrent_fwd) on state; both caches are updated
 * in place, so repeated calls continue the sequences.  After a kda_layer_fwd
 * prefill, its final_state and conv_state_out are the caches to pass here.
 *
 *   x           bf16 [B, T, d_model];   y bf16 [B, T, d_model].
 *   conv_state  bf16 [B, 3, 3*H*128], in place (layout as in kda_layer_fwd).
 *   state       fp32 [B, H, 128, 128], in place.
 *   workspace   at least kda_layer_decode_workspace(B, T, d_model, H, rank)
 *               bytes, 256-byte aligned.
 */
size_t kda_layer_decode_workspace(int B, int T, int d_model, int H, int rank);

int kda_layer_decode(const void *x, const kda_layer_weights *w, void *conv_state, float *state, void *y,
                     int B, int T, void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H_ */
