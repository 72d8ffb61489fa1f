/*
 * kda.h -- C ABI of libkda.so, the B200 (sm_100a) Kimi Delta Attention operator.
 *
 * The operator (per sequence b, head h; state S is d_k x d_v, fp32):
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t,            alpha_t = exp(log_alpha_t) in (0, 1]^{d_k}
 * Sources: "Kimi Linear's 75% KV cache cut comes from making three of every
 * four layers recurrent" (theclarity.today), third paragraph (per-channel
 * decay, removal of the old projection onto the key, write of the new pair)
 * and fourth paragraph (chunked kernels with the WY representation: a chunk's
 * rank-1 updates become triangular solves and tensor-core matrix products);
 * "Kimi Linear wlasnie pokonal pelna uwage na wlasnych warunkach" (remio.ai),
 * section "Jak Kimi Linear wykorzystuje inteligentniejsza pamiec
 * rekurencyjna" (delta rule, finer-grained gates than Gated DeltaNet,
 * blockwise algorithm with a diagonal-plus-low-rank transition, fixed-size
 * recurrent state).
 *
 * Padding: a position whose pad_mask entry is 0 neither decays nor writes the
 * state and its output is exactly 0, whatever its gate and input values
 * ("Transformers Community Reports Kimi Linear Cache Bug: Padding May Change
 * Subsequent Inference State", ainews, paragraphs on the reproduction and the
 * follow-up investigation).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, owned by the caller, on the
 *     current CUDA device.  The library allocates no device memory.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Nothing is synchronised.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched; no output is touched in that case.
 *   - Errors found on the device (an invalid cu_seqlens, a bounded wait that
 *     ran out) are latched in a per-device library word and reported by
 *     kda_get_device_status().  Kernels that follow a failed check on the same
 *     stream return without writing.
 *   - No C++ exception crosses the ABI.
 *   - Every launch is stream-ordered, so the calls can be captured into a CUDA
 *     graph; the first call on each device looks up the library's device error
 *     word (cudaGetSymbolAddress), so make one call before capturing.  The
 *     library keeps those device addresses for the life of the process: after
 *     a cudaDeviceReset(), unload and reload the library before calling it.
 *   - Layouts are row-major and contiguous.  N = total packed tokens,
 *     B = sequences (prefill) or rows (decode), H = heads.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,    /* bad pointer, size, alignment, overlap, dtype */
  KDA_ERR_UNSUPPORTED = 2,    /* valid but not built: head dims, chunk size */
  KDA_ERR_CUDA = 3,           /* a CUDA runtime call failed (launch, attribute) */
  KDA_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait gave up */
  KDA_ERR_DEVICE_CHECK = 5    /* a device-side argument check failed */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/*
 * Layout of log_alpha.  KDA_GATE_CHANNEL: one decay per key channel, [.., H, dk]
 * (Kimi Delta Attention).  KDA_GATE_HEAD: one decay per token and head, [.., H],
 * applied to every channel of the state: the head-wise gate of Gated DeltaNet,
 * the coarser special case KDA refines ("Kimi Linear's 75% KV cache cut ...",
 * theclarity.today, third paragraph; "Kimi Linear wlasnie pokonal ...",
 * remio.ai, section "Jak Kimi Linear wykorzystuje inteligentniejsza pamiec
 * rekurencyjna").  The result equals the per-channel operator with the gate
 * broadcast over d_k; the head-wise layout reads 4 bytes of gate per token and
 * head instead of 4 * dk.
 */
typedef enum { KDA_GATE_CHANNEL = 0, KDA_GATE_HEAD = 1 } kda_gate;

/*
 * Chunkwise prefill over a packed variable-length batch.
 *
 * Fields (all device pointers, caller-owned):
 *   dtype        type of q, k, v and o.  log_alpha, beta and the states are
 *                always fp32.
 *   num_seqs     B >= 0 sequences; total_tokens N >= 0; H >= 1 heads;
 *   dk, dv       head dimensions, each 64 or 128.
 *   q, k         [N, H, dk]; v [N, H, dv]; 16-byte aligned.
 *   log_alpha    [N, H, dk] fp32 (gate = KDA_GATE_CHANNEL, 16-byte aligned) or
 *                [N, H] fp32 (gate = KDA_GATE_HEAD, 4-byte aligned): natural
 *                log of the forget gate; finite and <= 0 (values outside that
 *                range are not checked and give unspecified results).
 *   beta         [N, H] fp32, finite.
 *   cu_seqlens   [B+1] int32: cu[0] = 0, non-decreasing, cu[B] = N; sequence b
 *                owns packed rows [cu[b], cu[b+1]).  Checked on the device
 *                (KDA_ERR_DEVICE_CHECK, nothing written).
 *   pad_mask     [N] uint8, 1 = valid, 0 = pad; NULL = all valid.  A pad is an
 *                identity step with o = 0.  Pads at the two ends of a sequence
 *                are skipped outright, so a run with edge pads is bit-identical
 *                to the unpadded run; pads between valid tokens are identity
 *                steps inside a chunk (equal to the unpadded run up to
 *                rounding).  Requires a workspace.
 *   init_state   [B, H, dk, dv] fp32 (dv contiguous), 16-byte aligned; NULL = 0.
 *   o            [N, H, dv] of dtype; must not overlap any input.
 *   final_state  [B, H, dk, dv] fp32 or NULL (not written).  It may be the same
 *                pointer as init_state (in-place update) but may not otherwise
 *                overlap an input.
 *   chunk        0 (default: 64 for bf16, 16 for fp32), 16, 32 or 64; 128 or
 *                256 for bf16 with d_k = d_v = 128 and the full workspace (the
 *                tensor-core path merges 64-row chunks into longer ones: the
 *                pages' chunk of 256, "Kimi Linear's 75% KV cache cut ...",
 *                theclarity.today, fourth paragraph), else KDA_ERR_UNSUPPORTED.
 *                The result is defined by the recurrence and does not depend on
 *                the chunk size beyond rounding.
 *   workspace    device scratch, 256-byte aligned.  kda_prefill_workspace_size()
 *                bytes select the fastest path (for bf16, d_k = d_v = 128,
 *                chunk 64: a two-kernel path that stores each chunk's
 *                intermediate tiles, about 73 KB per 64 tokens and head; chunk
 *                128 / 256 also store the merged chunk items, about 2.5 / 3 KB
 *                per token and head in all).  A
 *                smaller workspace selects a fused single-kernel path; a pad
 *                mask needs at least 16 bytes per sequence (rounded up to 256).
 *                May be NULL when pad_mask is NULL.
 *   gate         layout of log_alpha (kda_gate); 0 = per channel.  With
 *                KDA_GATE_HEAD the single-kernel tensor-core path is not used
 *                (a small workspace selects the CUDA-core path).
 * Numerics: bf16 inputs take the tensor-core path (bf16 operands, fp32
 * accumulation, fp32 state); fp32 inputs take an fp32 CUDA-core path.  o is
 * rounded once (round to nearest even) to its dtype.
 */
typedef struct {
  kda_dtype dtype;
  int num_seqs;
  int total_tokens;
  int H;
  int dk;
  int dv;
  const void *q;
  const void *k;
  const void *v;
  const float *log_alpha;
  const float *beta;
  const int32_t *cu_seqlens;
  const uint8_t *pad_mask;
  const float *init_state;
  void *o;
  float *final_state;
  int chunk;
  void *workspace;
  size_t workspace_bytes;
  kda_gate gate;
} kda_prefill_args;

/* Bytes of workspace for the fastest path of kda_prefill() with these
 * arguments (reads only dtype, sizes and chunk).  Returns 0 if args is NULL. */
size_t kda_prefill_workspace_size(const kda_prefill_args *args);

/* Enqueue one prefill.  Returns KDA_OK or an argument/launch error. */
kda_status kda_prefill(const kda_prefill_args *args, void *stream);

/*
 * kda_prefill without a workspace argument.  The pages have no counterpart to
 * this call: it serves callers that cannot call cudaMalloc where they run the
 * operator (an engine whose device memory is owned up front by a host
 * framework that passes operators only their tensors, or a serving loop in
 * which cudaMalloc/cudaFree are not allowed because they may synchronise the
 * device).  Same arguments as kda_prefill; args->workspace and
 * args->workspace_bytes are ignored.  Its 64 KiB of scratch holds the span
 * table of the pad pre-pass but not the per-chunk items of the two-kernel
 * tensor-core path, so it runs the single-kernel tensor-core path (bf16,
 * d_k = 128, d_v a multiple of 64, chunk 64, per-channel gate) or the
 * CUDA-core path (everything else): its results equal kda_prefill's up to
 * rounding (within the same tolerances against the exact recurrence), not bit
 * for bit, and it is slower than kda_prefill with a full workspace.  The
 * scratch comes from a fixed device
 * array inside the library, sized for KDA_NOALLOC_MAX_SEQS sequences (64 KiB,
 * held by every GPU that loads the library until exit); a batch with more
 * sequences returns KDA_ERR_INVALID_ARG and launches nothing.  All calls on a
 * device share that array: calls whose kernels may overlap on the GPU race and
 * must be ordered by the caller.  The first call on each device looks up the
 * array's device address; make it before any stream capture.  Allocates no
 * memory.
 */
#define KDA_NOALLOC_MAX_SEQS 4096
kda_status kda_prefill_noalloc(const kda_prefill_args *args, void *stream);

/*
 * One decode step: one new token for each of B independent rows, all heads.
 *   q, k [B, H, dk]; v [B, H, dv] of dtype; log_alpha [B, H, dk] fp32, or
 *   [B, H] fp32 with gate = KDA_GATE_HEAD; beta [B, H] fp32; mask [B] uint8 (1 = active, NULL = all active);
 *   state [B, H, dk, dv] fp32, updated in place, 16-byte aligned;
 *   o [B, H, dv] of dtype, must not overlap any other argument.
 * A masked row's state is neither read nor written and its o is written as 0.
 * The step is: S' = Diag(alpha) S; p = S'^T k; S = S' + k (beta (v - p))^T;
 * o = S^T q.
 */
typedef struct {
  kda_dtype dtype;
  int B;
  int H;
  int dk;
  int dv;
  const void *q;
  const void *k;
  const void *v;
  const float *log_alpha;
  const float *beta;
  const uint8_t *mask;
  float *state;
  void *o;
  kda_gate gate;
} kda_decode_args;

kda_status kda_decode(const kda_decode_args *args, void *stream);

/*
 * Short causal convolution of the layer's inputs, padding-correct, with a
 * carried convolution state (the convolution window a cached continuation
 * keeps besides the recurrent state: "Transformers Community Reports Kimi
 * Linear Cache Bug", ainews, paragraphs on the reproduction and the follow-up
 * investigation -- padded entries must neither enter the window nor advance the
 * convolution state).  Depthwise, per channel c of sequence b, over the
 * sequence's VALID positions only:
 *   y_t[c] = bias[c] + sum_{i<W} weight[c*W + i] * u_i[c]
 * where u_0 .. u_{W-2} are the W-1 valid inputs before t (oldest first) and
 * u_{W-1} = x_t; before the sequence's first valid inputs the window holds the
 * incoming state.  A pad position has y = 0 and changes nothing.  No activation
 * is applied.  Fields (device pointers, caller-owned):
 *   dtype        type of x and y (KDA_BF16 or KDA_F32); everything else fp32.
 *   num_seqs     B >= 0; total_tokens N >= 0; D >= 8 channels, a multiple of 8.
 *   width        W in 1..4.
 *   x, y         [N, D], 16-byte aligned; y must not overlap any input.
 *   weight       [D, W]; bias [D] or NULL (zeros).
 *   cu_seqlens   [B+1] int32, as for kda_prefill (checked on the device).
 *   pad_mask     [N] uint8 (1 = valid) or NULL.
 *   state_in     [B, W-1, D] (oldest row first), 16-byte aligned, or NULL (zeros).
 *   state_out    [B, W-1, D]: the last W-1 valid inputs of each sequence
 *                (completed from state_in when the sequence has fewer), or
 *                NULL.  May be the same pointer as state_in (in-place update),
 *                may not otherwise overlap an input.
 * A decode step is a call with one token per sequence.  Allocates nothing.
 */
typedef struct {
  kda_dtype dtype;
  int num_seqs;
  int total_tokens;
  int D;
  int width;
  const void *x;
  const float *weight;
  const float *bias;
  const int32_t *cu_seqlens;
  const uint8_t *pad_mask;
  const float *state_in;
  float *state_out;
  void *y;
} kda_conv_args;

kda_status kda_short_conv(const kda_conv_args *args, void *stream);

/*
 * Backward pass of kda_prefill (training): the gradients of <o, grad_o> +
 * <final_state, grad_final_state> with respect to q, k, v, log_alpha, beta and
 * init_state, by the blockwise algorithm ("Kimi Linear wlasnie pokonal ...",
 * remio.ai, section "Jak Kimi Linear wykorzystuje inteligentniejsza pamiec
 * rekurencyjna": the chunked form serves training as well as inference).  Chunks
 * of 64 rows: the chunk quantities (pairwise decay products, so exact for any
 * log_alpha <= 0) and every gradient of a chunk's rows are computed for all
 * chunks in parallel; only the state at each chunk start (forward) and its
 * gradient at each chunk end (backward) are chained over a sequence's chunks.
 * fp32 accuracy throughout: the gradient kernel's dense products run on the tensor
 * cores with each fp32 operand split into two tf32 parts (three products), the
 * rest on CUDA cores in fp32.
 * Fields (device pointers, caller-owned):
 *   dtype, num_seqs, total_tokens, H, dk, dv, q, k, v, log_alpha, beta,
 *   cu_seqlens, pad_mask, init_state, gate   as for kda_prefill (chunk is not
 *                used; the result does not depend on it).
 *   grad_o           [N, H, dv] fp32.
 *   grad_final_state [B, H, dk, dv] fp32 or NULL (zero).
 *   grad_q, grad_k   [N, H, dk] fp32; grad_v [N, H, dv] fp32;
 *   grad_log_alpha   fp32, the layout of log_alpha; grad_beta [N, H] fp32;
 *   grad_init_state  [B, H, dk, dv] fp32 or NULL (not written).
 *                All outputs 16-byte aligned and not overlapping any input or
 *                each other; pad positions get zero gradients; rows outside
 *                every sequence are not written.
 *   workspace    kda_prefill_backward_workspace_size() bytes, 256-byte aligned:
 *                per 64-row chunk and head the chunk quantities, the state at
 *                the chunk start and its gradient at the chunk end, about
 *                5 KB per token and head for d_k = d_v = 128.
 */
typedef struct {
  kda_dtype dtype;
  int num_seqs;
  int total_tokens;
  int H;
  int dk;
  int dv;
  const void *q;
  const void *k;
  const void *v;
  const float *log_alpha;
  const float *beta;
  const int32_t *cu_seqlens;
  const uint8_t *pad_mask;
  const float *init_state;
  kda_gate gate;
  const float *grad_o;
  const float *grad_final_state;
  float *grad_q;
  float *grad_k;
  float *grad_v;
  float *grad_log_alpha;
  float *grad_beta;
  float *grad_init_state;
  void *workspace;
  size_t workspace_bytes;
} kda_backward_args;

size_t kda_prefill_backward_workspace_size(const kda_backward_args *args);
kda_status kda_prefill_backward(const kda_backward_args *args, void *stream);

/* Synchronise `stream`, then return and clear the error latched on the
 * current device by earlier kernels (KDA_OK if none). */
kda_status kda_get_device_status(void *stream);

/*
 * Test hook for failure detection without a GPU fault (the pages have no
 * counterpart).  Every device-side wait of the prefill kernels is bounded;
 * when one runs out the kernel drains what it has in flight, releases its
 * tensor memory, latches KDA_ERR_DEVICE_TIMEOUT and returns, so the context
 * stays usable.  This hook lets a test make that happen on purpose:
 *   fault        0 (normal operation) or KDA_FAULT_STARVE_STATE_LOADS: the
 *                state pass of the workspace-backed tensor-core prefill issues
 *                none of its item loads, so its waits run out; nothing is read
 *                or written out of bounds and the call's outputs are left
 *                unspecified.
 *   wait_cycles  the limit, in SM clock cycles, of every bounded wait in later
 *                prefill calls; <= 0 restores the default (about 2 s).
 * Process-wide and read at each kda_prefill call; meant for tests only.
 * Returns KDA_ERR_INVALID_ARG for an unknown fault bit.
 */
#define KDA_FAULT_STARVE_STATE_LOADS 1
kda_status kda_debug_set_fault(int fault, long long wait_cycles);

/*
 * Which bounded wait ran out first on the current device since the last call
 * (0: none): a diagnostic beside KDA_ERR_DEVICE_TIMEOUT.  Synchronises
 * `stream`, then returns and clears the code; -1 if a CUDA call failed.
 * Codes: workspace-backed tensor-core prefill, intra-chunk kernel: 1 Gram
 * products, 2 V tile, 3 W and U_v products, 4 staged log_alpha rows; its state
 * pass: 11 item load,
 * 12 first product group of a chunk, 13 second product group, 14 buffer
 * release (loading side); single-kernel tensor-core prefill: 21-26 (its six
 * waits in program order); chunks of 128 / 256: the state pass uses 11-14 as
 * above (11 any item tile) and 16 for the U_v block, the merge kernels 31
 * (operand loads), 32 and 33 (their two product groups).
 */
int kda_debug_timeout_site(void *stream);

/* Static string for a status code; never NULL. */
const char *kda_status_string(kda_status status);

/* ABI version: (major << 16) | minor. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
