/*
 * ittt.h — C ABI of the In-Place TTT fast-weight MLP layer forward (prefill)
 * for NVIDIA B200 (sm_100a).
 *
 * The method (Feng et al., "In-Place Test-Time Training"; web pages cited
 * per entry point below):
 *
 *   Z      = silu(H W_gate^T) * (H W_up^T)            gated-MLP activations
 *   Y[t,c] = sum_j conv[c,j] X0[t+j, c]                depthwise look-ahead conv
 *   Vhat   = Y W_target                                LM-aligned value target
 *   chunk i of C tokens:  O_i = Z_i W^(i)^T            apply with the current state
 *                         W^(i+1) = W^(i) + eta Vhat_i^T Z_i   then update
 *   W_down_final = W^(n),  W^(0) = W_down0 for every sequence of the batch
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  Inputs are
 *   read only; outputs are fully overwritten.  The library allocates no
 *   device memory on any compute path: scratch space is the caller's
 *   workspace (size from ittt_workspace_size).
 * - Row-major layouts, element type given by ittt_problem.dtype:
 *     H, X0   [B, T, d]     O [B, T, d]   (X0 [B, T + k - 1, d] with
 *                           ITTT_FLAG_X0_LOOKAHEAD)
 *     W_gate, W_up [f, d]   (nn.Linear "out x in" layout: the method uses H W^T)
 *     W_down0 [d, f]        shared initial fast weight of all B sequences
 *     conv_kernel [d, k]    tap j of channel c multiplies X0[t + j, c]
 *     W_target [d, d]       applied untransposed: Vhat = Y W_target
 *     W_down_final [B, d, f] always float32
 * - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *   performs no host synchronisation.  Argument errors are reported before any
 *   launch.  Launch errors return ITTT_ERR_CUDA.  Device-side failures (a
 *   bounded wait that ran out, an index check) set a per-device flag that
 *   ittt_get_last_error() reports after synchronising the stream.
 * - bf16 path: bf16 storage of inputs, Z, Vhat, W^(i) and O; fp32 tensor-core
 *   accumulation; fp32 W_down_final.  Requirements: d % 8 == 0, f % 8 == 0,
 *   C % 128 == 0, T % C == 0, every pointer 16-byte aligned.
 * - f32 path: fp32 everywhere (CUDA-core FMA); any d, f >= 1, T % C == 0.
 * - p->clip > 0 applies update-norm clipping in ittt_fast_mlp_forward (and
 *   in ittt_fast_weight_scan on the f32 path; the bf16 scan entry point
 *   expects targets already clipped by ittt_clip_update_targets).
 * - Concurrent calls on different streams are safe; they must not share a
 *   workspace.
 */
#ifndef ITTT_H
#define ITTT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ITTT_OK = 0,
  ITTT_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum, ...        */
  ITTT_ERR_UNSUPPORTED = 2,   /* valid but not handled: T % C != 0, alignment, ... */
  ITTT_ERR_WORKSPACE = 3,     /* workspace pointer null or smaller than required  */
  ITTT_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed     */
  ITTT_ERR_TIMEOUT = 5,       /* a device-side bounded wait ran out                */
  ITTT_ERR_DEVICE_FAULT = 6   /* a device-side consistency check failed            */
} ittt_status;

typedef enum { ITTT_F32 = 0, ITTT_BF16 = 1 } ittt_dtype;

/* Which algebraic form computes the chunk recurrence.  All forms give the
 * same result in exact arithmetic.  AUTO picks by problem shape (see
 * ittt_resolve_form).
 *   PREFIX: the effective weight of every chunk is stored (the pages'
 *           Algorithm 1, deltas and prefix sum fused) and applied;
 *   DUAL:   O_i = Z_i W_down0^T + eta sum_{j<i} (Z_i Z_j^T) Vhat_j, no stored weight;
 *   HYBRID: chunks in groups of m (m = max(2, 1024 / C); C a multiple of 256
 *           and at least two whole groups, else the prefix form runs): only the weight at each group's
 *           start is stored (n / m weights instead of n - 1), the dual form runs
 *           inside each group.  The smallest workspace at long T; at C = 256
 *           also the fastest form for long sequences (AUTO picks it there).
 * The dual and hybrid forms are bf16 only; fp32 problems run the prefix form.
 * The form applies to ittt_fast_mlp_forward; the step entry points
 * (ittt_fast_weight_scan, ittt_apply, ...) compute their own step whatever it says. */
typedef enum {
  ITTT_FORM_AUTO = 0,
  ITTT_FORM_PREFIX = 1,
  ITTT_FORM_DUAL = 2,
  ITTT_FORM_HYBRID = 3
} ittt_form;

/* Bits of ittt_problem.flags. */
/* The conv's look-ahead stops at the end of each chunk (X0 taken as zero past
 * it), so a chunk's targets read no token of a later chunk (iplexlaw review,
 * section 6: chunk boundaries manage the padding).  Default: zero past the
 * end of the sequence only. */
#define ITTT_FLAG_PAD_CHUNK_END 1
/* X0 is [B, T + k - 1, d]: after each sequence's T rows come the first k - 1
 * rows of the next segment of the same document, read by the look-ahead of the
 * last tokens (segment continuation with sequence-end padding; together with
 * W_down0 = the previous segment's W_down_final the split is exact). */
#define ITTT_FLAG_X0_LOOKAHEAD 2

typedef struct {
  int64_t B;       /* independent sequences, each starting from W_down0      */
  int64_t T;       /* tokens per sequence                                     */
  int64_t d;       /* model width                                             */
  int64_t f;       /* MLP hidden width                                        */
  int32_t C;       /* chunk size (tokens per fast-weight update)              */
  int32_t k;       /* conv taps, 1..16                                        */
  float eta;       /* update step size, finite; 0 = plain MLP.  f32 path: any
                      finite value.  bf16 path: 0 or |eta| >= 1e-30, else
                      ITTT_ERR_UNSUPPORTED (the fused scan accumulates from
                      W_down0 / eta in fp32 and multiplies by eta on output;
                      entries of W_down0 with |w| / |eta| above the fp32 range,
                      3.4e38, are not checked and come out inf or NaN)          */
  int32_t dtype;   /* ittt_dtype                                              */
  int32_t form;    /* ittt_form                                               */
  int32_t flags;   /* ITTT_FLAG_* bits, others must be 0                      */
  float clip;      /* update-norm clipping: every chunk's delta eta Vhat_i^T Z_i
                      is rescaled to Frobenius norm <= clip; 0 = off           */
  int32_t reserved;/* must be 0                                               */
} ittt_problem;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int ittt_version(void);

/* Human-readable name of a status code (static string). */
const char* ittt_status_string(ittt_status s);

/* Bytes of workspace ittt_fast_mlp_forward needs for problem *p.
 * Validates *p like the forward call (pointer checks aside). */
ittt_status ittt_workspace_size(const ittt_problem* p, size_t* bytes);

/* The form ittt_fast_mlp_forward takes for problem *p: ITTT_FORM_PREFIX,
 * ITTT_FORM_DUAL or ITTT_FORM_HYBRID, never ITTT_FORM_AUTO (AUTO takes the
 * dual form when C <= 256 and T C (d + f) <= 170 d f, else the hybrid form
 * when C = 256, T d >= 2^24 and the hybrid's groups fit, else the prefix form:
 * rules fitted to the forms' measured times on B200; HYBRID without whole
 * groups and every fp32 problem resolve to PREFIX).  Host only, no device work; validates *p like
 * ittt_workspace_size.  *form is written only on ITTT_OK. */
ittt_status ittt_resolve_form(const ittt_problem* p, int32_t* form);

/* The whole layer forward (prefill): O and W_down_final.
 *
 * Pages: deep-read notes "论文精读：In-Place Test-Time Training", sections
 * "In-Place 设计" (gated MLP, W_down as fast weight), "Chunk-Wise 更新机制"
 * (update equation) and "LM-Aligned 目标函数" (target equation); iplexlaw
 * review of "In-Place Test-Time Training", section 3 (apply then update) and
 * section 6 (Algorithm 1: parallel deltas, exclusive prefix sum, parallel
 * apply); forum summary "In-Place TTT: ByteDance Seed's Test-Time Training
 * Framework ...", "Three Core Designs" item 3 (kernel [0,1,0,...] with
 * W_target = I is exact next-token prediction).
 *
 * workspace: device memory of at least ittt_workspace_size() bytes, 256-byte
 * aligned; its contents on entry are ignored and on exit are unspecified.
 * O: [B, T, d] of dtype.  W_down_final: [B, d, f] float32. */
ittt_status ittt_fast_mlp_forward(const ittt_problem* p,
                                  const void* H, const void* X0,
                                  const void* W_gate, const void* W_up,
                                  const void* W_down0, const void* conv_kernel,
                                  const void* W_target,
                                  void* O, float* W_down_final,
                                  void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Step 1 alone: Z = silu(H W_gate^T) * (H W_up^T), Z [B*T, f] of dtype.
 * Pages: deep-read notes, "In-Place 设计" gated-MLP equation; iplexlaw review
 * section 2. */
ittt_status ittt_gated_activations(const ittt_problem* p, const void* H, const void* W_gate,
                                   const void* W_up, void* Z, void* stream);

/* Step 2a alone: Y = depthwise look-ahead Conv1D of X0, Y [B, T, d] of dtype,
 * zero padding past each sequence's end.  Pages: forum summary "Three Core
 * Designs" item 3; iplexlaw review section 4 (Conv1D over X0). */
ittt_status ittt_lookahead_conv(const ittt_problem* p, const void* X0, const void* conv_kernel,
                                void* Y, void* stream);

/* Step 2 alone: Vhat = Conv1D(X0) W_target, Vhat [B*T, d] of dtype.
 * workspace: at least ittt_workspace_size() bytes (holds Y).
 * Pages: deep-read notes "LM-Aligned 目标函数" equation; iplexlaw review
 * section 4. */
ittt_status ittt_lm_target(const ittt_problem* p, const void* X0, const void* conv_kernel,
                           const void* W_target, void* Vhat, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Steps 3+4 alone (update deltas and their exclusive prefix sum):
 *   W_stack[b, i-1] = W_down0 + eta * sum_{j<i} Vhat_j^T Z_j   for i = 1..n-1
 *   W_down_final[b] = W_down0 + eta * sum_{j<n} Vhat_j^T Z_j
 * Vhat [B*T, d], Z [B*T, f], W_down0 [d, f] of dtype; W_stack
 * [B, n-1, d, f] of dtype (may be NULL when n == 1); W_down_final float32.
 * Pages: iplexlaw review section 6 (Algorithm 1 steps 1-3); deep-read notes
 * "Chunk-Wise 更新机制" update equation. */
ittt_status ittt_fast_weight_scan(const ittt_problem* p, const void* Vhat, const void* Z,
                                  const void* W_down0, void* W_stack, float* W_down_final,
                                  void* stream);

/* Step 5 alone: O_i = Z_i W^(i)^T for every chunk i, W^(0) = W_down0 and
 * W^(i) = W_stack[b, i-1].  Pages: iplexlaw review section 3 (a chunk's
 * output uses its pre-update state) and section 6 (Algorithm 1 step 4). */
ittt_status ittt_apply(const ittt_problem* p, const void* Z, const void* W_down0,
                       const void* W_stack, void* O, void* stream);

/* Steps 3-5 together, the chunk recurrence: O and W_down_final from Z, Vhat
 * and W_down0, in the form ittt_fast_mlp_forward takes for *p (see
 * ittt_resolve_form; clipping is not applied here: pass targets already
 * clipped by ittt_clip_update_targets).  On the bf16 prefix form this is one
 * persistent kernel in which the fused update scan and the apply share one
 * work queue (an apply unit starts once its d-tile's effective weight is
 * stored).  Z [B*T, f], Vhat [B*T, d], W_down0 [d, f] of dtype; O [B, T, d] of
 * dtype; W_down_final [B, d, f] float32.  workspace: ittt_workspace_size()
 * bytes (only its stack, form and scheduling regions are used).
 * Pages: iplexlaw review sections 3 and 6 (Algorithm 1); deep-read notes
 * "Chunk-Wise 更新机制". */
ittt_status ittt_chunk_recurrence(const ittt_problem* p, const void* Z, const void* Vhat,
                                  const void* W_down0, void* O, float* W_down_final,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Update-norm clipping step: for every sequence b and chunk i, computes
 * norms[b, i] = ||eta Vhat_i^T Z_i||_F (before clipping) and, where it exceeds
 * p->clip > 0, scales the chunk's rows of Vhat by p->clip / norms[b, i] in
 * place, so that the later steps see clipped deltas.  Z [B*T, f], Vhat
 * [B*T, d] (read and rewritten) of dtype; norms [B, T/C] float32, written.
 * bf16: the norm comes from ||Vhat_i^T Z_i||_F^2 = sum((Z_i Z_i^T) *
 * (Vhat_i Vhat_i^T)) on the tensor cores, without forming the delta.
 * Pages: iplexlaw review section 6 (the Frobenius norm of the update delta
 * is limited to a threshold; each chunk's delta is clipped on its own). */
ittt_status ittt_clip_update_targets(const ittt_problem* p, const void* Z, void* Vhat,
                                     float* norms, void* stream);

/* ----------------------------------------------------------------- decode
 * Token-by-token decoding of B sequences in lockstep.  Token pos of every
 * sequence gets O = Z W^ᵀ with the fast weight of its chunk (the state after
 * the updates of all earlier chunks), and after the last token of a chunk the
 * state takes that chunk's update (clipped if p->clip > 0):
 *   W += eta Vhat_i^T Z_i, Vhat_i = Conv1D(X0_i) W_target.
 * This is the prefill recurrence of ittt_fast_mlp_forward with chunk-end
 * padding, processed one token at a time.  Decoding requires
 * ITTT_FLAG_PAD_CHUNK_END: with sequence-end padding the update of chunk i
 * would need X0 of tokens of chunk i+1 that are not generated yet, which is
 * the leak the chunk-boundary padding of the pages (iplexlaw review,
 * section 6) rules out.  Pages: iplexlaw review sections 3 (apply then
 * update) and 6; deep-read notes "Chunk-Wise 更新机制".
 *
 * p: B (1..8), d, f, C, k, eta, clip, dtype as for the forward; T must equal
 * C; flags must contain ITTT_FLAG_PAD_CHUNK_END.
 * pos: index of this token in the sequences (0, 1, 2, ...; one call each).
 * H_tok, X0_tok: [B, d]; O_tok: [B, d] (dtype).
 * W_state: [B, d, f] float32, the fast weight; set to W_down0 before pos 0;
 *   updated in place after every chunk's last token.
 * Z_buf [B, C, f], X0_buf [B, C, d] (dtype): the current chunk's rows,
 *   written at slot pos % C; caller-owned, contents kept between calls.
 * workspace: ittt_decode_workspace_size() bytes.  On the bf16 path it holds,
 *   between calls, the state rounded to bf16 (the operand of the per-token
 *   GEMV, as the prefill applies bf16 weights); it is rebuilt from W_state at
 *   the first token of every chunk, so pass the same workspace to every step
 *   of a chunk and change W_state only before a chunk's first token. */
ittt_status ittt_decode_workspace_size(const ittt_problem* p, size_t* bytes);
ittt_status ittt_decode_step(const ittt_problem* p, int64_t pos, const void* H_tok,
                             const void* X0_tok, const void* W_gate, const void* W_up,
                             const void* conv_kernel, const void* W_target, float* W_state,
                             void* Z_buf, void* X0_buf, void* O_tok, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ------------------------------------------------------- context parallel
 * One sequence split into G contiguous segments of whole chunks, segment r
 * on rank r.  The chunk updates are additive, so the recurrence splits into
 * three steps around one exchange between ranks (the prefix-sum scheme of the
 * pages: the forum summary, "Three Core Designs", item 2, and the iplexlaw
 * review, section 6, Algorithm 1 — per-chunk deltas in parallel, exclusive
 * prefix sum, parallel application; here a rank plays the part of a chunk):
 *
 *   ittt_cp_delta    the segment's (clipped) chunk deltas eta Vhat_i^T Z_i
 *                    summed from zero: S_r, their total, and (kept in the
 *                    workspace with Z) the running sums L_i before each chunk;
 *   (caller)         bring the S_q of all ranks together (NCCL);
 *   ittt_cp_prefix   P_r = sum_{q < r} S_q, the exclusive prefix over ranks;
 *   ittt_cp_apply    the segment's effective weights W_down0 + P_r + L_i, O of
 *                    its chunks, and W_end = W_down0 + P_r + S_r, the state
 *                    after the segment (on the last rank: W_down_final).
 *
 * The concatenated O and the last rank's W_end equal one ittt_fast_mlp_forward
 * of the whole sequence up to rounding (bf16: the running sums L_i are stored
 * in bf16, then each effective weight is rounded once from the fp32 sum).
 * With sequence-end padding every rank but the
 * last passes X0 with the next segment's first k - 1 rows appended
 * (ITTT_FLAG_X0_LOOKAHEAD); with ITTT_FLAG_PAD_CHUNK_END no rows cross ranks.
 *
 * p describes this rank's segment: T = its token count (a multiple of C), B
 * sequences (segment r of each), everything else as for the forward (the
 * form is ignored).  The same workspace, of ittt_cp_workspace_size() bytes,
 * must be passed to ittt_cp_delta and then to ittt_cp_apply of the same
 * segment, unchanged in between; ittt_cp_apply turns the running sums into
 * the effective weights in place, so it runs once per ittt_cp_delta.
 * S: [B, d, f] float32, written by ittt_cp_delta, read by ittt_cp_apply.
 * P: [B, d, f] float32, read by ittt_cp_apply (zeros on rank 0).
 * O: [B, T, d] dtype; W_end: [B, d, f] float32, written by ittt_cp_apply. */
ittt_status ittt_cp_workspace_size(const ittt_problem* p, size_t* bytes);
ittt_status ittt_cp_delta(const ittt_problem* p, const void* H, const void* X0,
                          const void* W_gate, const void* W_up, const void* conv_kernel,
                          const void* W_target, float* S, void* workspace,
                          size_t workspace_bytes, void* stream);
ittt_status ittt_cp_apply(const ittt_problem* p, const void* W_down0, const float* P,
                          const float* S, void* O, float* W_end, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Exclusive prefix sum along the leading axis of G rows of n float32:
 * P_all[g, e] = sum over q < g of S_all[q, e]: row 0 is zeros and row g
 * holds S_all[0, e] + ... + S_all[g-1, e], summed in that order.
 * S_all, P_all: [G, n] float32 device arrays (they must not overlap).  With
 * the all-to-all exchange, rank q calls it on slice q of every rank's S and
 * sends row r back to rank r.  G >= 1, n >= 0. */
ittt_status ittt_cp_prefix(const float* S_all, int64_t G, int64_t n, float* P_all, void* stream);

/* Buffer checks (a debugging aid, off by default).  level 1: every compute
 * entry point first verifies that each device buffer it reads or writes lies
 * inside one device allocation from its start to the end the problem implies
 * (cuMemGetAddressRange), and returns ITTT_ERR_INVALID_ARG instead of
 * launching when one does not (too small, host memory, or freed).  Costs one
 * driver query per buffer per call.  level 0: off.  Process-wide. */
ittt_status ittt_set_checks(int level);

/* The check itself: ITTT_OK if [ptr, ptr + bytes) lies inside one device
 * allocation known to the driver, ITTT_ERR_INVALID_ARG otherwise (null, host
 * memory, or past the allocation's end).  Launches nothing. */
ittt_status ittt_check_buffer(const void* ptr, size_t bytes);

/* ---------------------------------------------------------- timing probe
 * A measurement aid with no counterpart in the method.  After
 * ittt_probe_start(n), the next n calls of ittt_fast_mlp_forward on the
 * calling thread record a CUDA event on the caller's stream right before and
 * right after they launch the gate/up GEMM (step 1) and right before and after
 * the chunk recurrence (steps 3-5).  ittt_probe_read() waits for those events,
 * writes each call's gate/up GEMM time in milliseconds to ms[0 .. *got - 1]
 * (at most `capacity`), and turns the probe off.  Recording an event pair
 * costs the bracketed launch its programmatic overlap with its neighbours
 * (about a microsecond per call).
 * n: 1 .. 65536; ittt_probe_start while a probe is on discards it. */
ittt_status ittt_probe_start(int n);
ittt_status ittt_probe_read(float* ms, int capacity, int* got);
/* Both probed times of each call: the gate/up GEMM's and the chunk
 * recurrence's (the launches of step 3-5: on the prefix form the one
 * persistent scan-and-apply kernel), each between events on the caller's
 * stream.  Either array may be NULL (not written); turns the probe off. */
ittt_status ittt_probe_read2(float* gate_up_ms, float* recurrence_ms, int capacity, int* got);

/* Synchronises `stream`, then returns and clears the first device-side
 * failure recorded since the last call (ITTT_ERR_TIMEOUT /
 * ITTT_ERR_DEVICE_FAULT), or ITTT_ERR_CUDA for a pending CUDA error, or
 * ITTT_OK. */
ittt_status ittt_get_last_error(void* stream);

/* Upper bound, in nanoseconds, of every device-side wait in later launches
 * on the calling thread's current device (default 4e9).  A wait that runs
 * out sets ITTT_ERR_TIMEOUT and the kernel returns early. */
ittt_status ittt_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded-wait path: launches one tiny kernel that waits
 * on a barrier nobody signals, for at most `ns` nanoseconds, then returns.
 * ittt_get_last_error() afterwards reports ITTT_ERR_TIMEOUT. */
ittt_status ittt_selftest_wait_timeout(uint64_t ns, void* stream);

/* Self-test of the device-side index checks (no counterpart in the method):
 * runs ittt_apply on the caller's buffers (same arguments and layouts) with
 * the kernel told that W_stack holds one d x f slice fewer than it does.  The
 * apply kernel checks every work unit's slice index against the stack's
 * extent before it loads anything, so the units of the last sequence's last
 * chunk are skipped (those rows of O are left as they were, no memory outside
 * the buffers is touched) and ittt_get_last_error() afterwards reports
 * ITTT_ERR_DEVICE_FAULT; every other row of O is computed as by ittt_apply.
 * bf16 only, B (T / C - 1) >= 2. */
ittt_status ittt_selftest_device_check(const ittt_problem* p, const void* Z, const void* W_down0,
                                       const void* W_stack, void* O, void* stream);

/* Size of the built-in scratch array used by ittt_lm_target_noalloc. */
#define ITTT_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* ittt_lm_target without a caller workspace.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory,
 * such as plugins whose host framework owns every byte of device memory
 * through its own pool, or latency-critical loops in which the implicit
 * device synchronisation of cudaMalloc is not acceptable, and that have no
 * workspace of their own to hand over.
 *
 * Same arguments, layouts and result as ittt_lm_target minus the workspace:
 * Vhat [B*T, d] = Conv1D(X0) W_target.  The intermediate Y (B*T*d elements
 * of dtype) lives in a file-scope __device__ array of
 * ITTT_NOALLOC_SCRATCH_BYTES (16 MiB), which every GPU that loads the library
 * holds until the process exits; problems needing more return
 * ITTT_ERR_WORKSPACE before any launch.  No cudaMalloc, cudaFree or other
 * allocating call is made.  Every call looks up the array's device address
 * (cudaGetSymbolAddress) on the current device, so the address always belongs
 * to the device's current context, also after the application has reset the
 * device; the first call on a device also loads the library's device code
 * there, so make that first call before any stream capture.  All calls on a
 * device share the one
 * array and it keeps the last call's contents (every element this entry point
 * reads is written first in the same call): calls whose kernels may overlap
 * on the GPU, e.g. on two streams, race on it and must be serialised by the
 * caller. */
ittt_status ittt_lm_target_noalloc(const ittt_problem* p, const void* X0, const void* conv_kernel,
                                   const void* W_target, void* Vhat, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ITTT_H */
