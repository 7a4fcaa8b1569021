/*
 * rlk.h -- C ABI of librlk: the bitwise batch-invariant linear-logp operator
 * (LM head GEMM -> temperature -> full-vocab logsumexp, target log-prob and
 * entropy, plus its backward to dHidden and dW) for NVIDIA B200 (sm_100a).
 *
 * The operation.  The RL-Kernel pages name a linear-logp route,
 * "rlkernel.linear_logp.bitwise.v1" (h100-cp-gradient.json,
 * runs[].validation.runtime_readbacks.frameworks.{megatron/training,
 * vllm/rollout}.modules.logp), that stands in for VIME's native
 * calculate_log_probs_and_entropy (VIME Qwen3-8B TP4/CP2 dense page,
 * "User-facing operator matrix") and whose train and rollout results must be
 * bitwise equal (same page, "Required gates": zero bitwise mismatches, no
 * fallback; h100-cp-gradient.json runs[0].validation.train_rollout_logprob:
 * bitwise_equal, 0 mismatches over 8192 elements).  The pages print no
 * formula; this library computes, for each row t and the whole vocabulary,
 *
 *   z[t,v]     = (sum_h hidden[t,h] * W[v,h]) / temperature
 *   lse[t]     = log sum_v exp(z[t,v])
 *   logp[t]    = z[t,targets[t]] - lse[t]
 *   entropy[t] = lse[t] - sum_v p[t,v] z[t,v],       p = exp(z - lse)
 *
 * and, given upstream gradients dlogp[t] and dentropy[t],
 *
 *   dx[t,v]      = (dlogp[t] (1[v = targets[t]] - p[t,v])
 *                   - dentropy[t] p[t,v] (z[t,v] - (lse[t] - entropy[t]))) / temperature
 *   dHidden[t,:] = sum_v dx[t,v] W[v,:]
 *   dW[v,:]      = sum_t dx[t,v] hidden[t,:]
 *
 * The T x V logits are never written to memory.
 *
 * Determinism contract.  For a given (H, V, temperature), every per-row output
 * (logp, entropy, lse and the dHidden row) depends only on that row's hidden
 * vector, target and gradient seeds: it is bitwise the same for any T, any
 * position of the row in the batch and any other rows in the batch, and
 * bitwise the same run to run.  (Batches of at most 128 rows run a second
 * forward kernel, with the operands of the tensor-core product swapped; it
 * computes every logit and every online-softmax update with the same
 * arithmetic in the same order, and the test suite holds it to the long-batch
 * kernel bit for bit.)  dW (a sum over rows) is bitwise repeatable for
 * identical inputs: fixed summation order, no atomics.
 *
 * Conventions for every entry point below.
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    contiguous.  bf16 tensors are passed as rlk_bf16 (the raw 16-bit
 *    pattern).  hidden, W, dHidden and dW must be 16-byte aligned, the
 *    workspace 256-byte aligned; the float and int64 vectors need their
 *    natural alignment.
 *  - The library allocates no memory and keeps no per-call state; everything
 *    is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    with no host synchronisation.  Kernel launch parameters are fixed at
 *    enqueue time, so a call can be captured into a CUDA graph.
 *  - Errors are fail-closed: bad arguments are rejected with a status before
 *    anything is enqueued and there is no fallback route of any kind.
 *  - Supported shapes: 64 <= H <= 2^20, H % 64 == 0; 1 <= V < 2^31;
 *    0 <= T < 2^31.
 *    T == 0 is a successful no-op (bwd still zeroes dW).
 *  - Device faults are reported, never trapped: a target outside [0, V)
 *    yields NaN logp for that row (its dHidden row omits the one-hot term)
 *    and sets RLK_DEVERR_TARGET in the workspace's error word; an internal
 *    pipeline wait that exceeds its time bound sets RLK_DEVERR_TIMEOUT and
 *    the kernel exits.  Read (and clear) the word with
 *    rlk_read_device_error.
 */
#ifndef RLK_H_
#define RLK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t rlk_bf16;

typedef enum {
  RLK_OK = 0,
  RLK_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad temperature */
  RLK_ERR_UNSUPPORTED_SHAPE = 2,  /* H % 64 != 0, sizes out of range            */
  RLK_ERR_MISALIGNED = 3,         /* pointer alignment below the stated minimum  */
  RLK_ERR_WORKSPACE_TOO_SMALL = 4,
  RLK_ERR_UNSUPPORTED_DEVICE = 5, /* current device is not compute capability 10.0 */
  RLK_ERR_CUDA = 6                /* a CUDA runtime/driver call or launch failed */
} rlk_status;

/* Bits of the device error word at the start of the workspace. */
#define RLK_DEVERR_TARGET 0x1u
#define RLK_DEVERR_TIMEOUT 0x2u
#define RLK_DEVERR_SCALE 0x4u   /* a transition std s_b was not a positive finite number */

/* Bytes of workspace that rlk_linear_logp_fwd (for_backward == 0) or both
 * rlk_linear_logp_fwd and rlk_linear_logp_bwd (for_backward != 0) need for
 * these sizes.  Returns 0 for unsupported sizes.  The first 256 bytes hold
 * the device error word: zero them once when the workspace is allocated (or
 * call rlk_read_device_error once); the library never clears it on its own. */
size_t rlk_linear_logp_workspace_bytes(int64_t T, int64_t H, int64_t V, int for_backward);

/* Forward.  hidden [T,H] bf16, W [V,H] bf16 (the LM head, one row per vocab
 * entry), targets [T] int64 in [0, V), temperature > 0 and finite.  Writes
 * logp, entropy and lse, each [T] fp32 (natural log, lse of the temperature-
 * scaled logits).  Uses the workspace for per-(row, vocab split) partials. */
rlk_status rlk_linear_logp_fwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                               int64_t T, int64_t H, int64_t V, float temperature, float* logp,
                               float* entropy, float* lse, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Backward.  Same hidden, W, targets, sizes and temperature as the forward;
 * lse and entropy are the forward's outputs for these rows; dlogp and
 * dentropy [T] fp32 are the upstream gradients of logp and entropy.
 * Overwrites dHidden [T,H] bf16 and dW [V,H] fp32 (no accumulation into
 * existing contents).  The logits are recomputed one vocab chunk at a time;
 * the chunk's dlogits are rounded to bf16 in the workspace before the two
 * gradient GEMMs. */
rlk_status rlk_linear_logp_bwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                               int64_t T, int64_t H, int64_t V, float temperature,
                               const float* lse, const float* entropy, const float* dlogp,
                               const float* dentropy, rlk_bf16* dHidden, float* dW,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Forward with no workspace argument and no allocation anywhere.  The pages
 * have no counterpart: this entry exists for callers that cannot allocate
 * device memory -- code running inside a host framework that owns every
 * device byte (a serving engine with a pre-reserved memory pool, a plugin
 * host that forbids allocation calls) or that cannot size a workspace ahead
 * of time.  Arguments and results are those of rlk_linear_logp_fwd.
 *  - Scratch (error word and per-split partials) lives in a file-scope device
 *    array of 32 MiB that every GPU which loads the library holds until the
 *    process exits.  Sizes needing more than that (more than about 9400 rows
 *    at V = 151936) are rejected with RLK_ERR_WORKSPACE_TOO_SMALL before
 *    anything is enqueued.
 *  - The first call on a device looks up the array's device address with that
 *    device current (cudaGetSymbolAddress); make that first call before any
 *    stream capture.  The address is kept together with the id of the
 *    context it belongs to: after the context is destroyed and created again
 *    (cudaDeviceReset, or a host that releases and re-retains the primary
 *    context) the next call looks the address up again, so that call too
 *    belongs before any capture.  Host threads may call concurrently.
 *  - Every call shares the one array: calls whose kernels overlap on the GPU
 *    (for instance on two streams) race and corrupt each other's results.
 *    Each call clears the error word itself; an out-of-range target gives NaN
 *    logp for its row, and a timed-out internal wait turns all outputs NaN.
 *  - Calls no allocation routine of CUDA or of any other library.
 *  - Counted by rlk_call_count(0), like rlk_linear_logp_fwd. */
rlk_status rlk_linear_logp_fwd_noalloc(const rlk_bf16* hidden, const rlk_bf16* W,
                                       const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                       float temperature, float* logp, float* entropy,
                                       float* lse, void* stream);

/* Vocab-parallel (tensor-parallel) forward, invariant to the TP degree.  The
 * pages train the same model under TP2/CP4 and TP4/CP2 layouts and find the
 * weights, gradient norms and tokens bitwise equal across the two runs
 * (h100-cp-gradient.json, all_parameter_hash_comparisons[].bitwise_equal,
 * gradient_norm_comparisons[].exactly_equal, tokens_equal).  Here each rank
 * holds a contiguous shard of W whose first row v0 is a multiple of
 * rlk_fwd_split_width() (512): the forward's vocab splits then fall wholly in
 * one shard and every shard computes exactly the single-GPU split triples, so
 * merging the gathered splits in global order gives logp / entropy / lse bit
 * for bit equal to rlk_linear_logp_fwd, for any number of shards.
 *
 * rlk_linear_logp_fwd_shard: hidden [T,H] bf16, W_shard [V_shard,H] bf16 =
 * rows v0 .. v0+V_shard-1 of the full [V,H] head, targets [T] (global vocab
 * indices).  Writes the first ceil(V_shard / 512) columns of part_m, part_s,
 * part_b, each [T][Gs] fp32 (row stride Gs, with ceil(V_shard / 512) <= Gs <=
 * ceil(V / 512); give every shard the same Gs so that the buffers concatenate
 * into the combine's layout), and ytgt[t] for the rows whose target lies in
 * the shard (other rows of ytgt are left untouched).  The workspace holds only
 * the device error word (256 bytes).  v0 not a multiple of 512, or V_shard
 * not one either for a shard that does not end at V, gives
 * RLK_ERR_UNSUPPORTED_SHAPE; a shard outside [0, V) or Gs out of range gives
 * RLK_ERR_INVALID_ARG.
 *
 * rlk_linear_logp_combine: part_* laid out [nshards][T][Gs] (the shards' part_
 * buffers one after another, as an all-gather delivers them), the last shard's
 * unused columns ignored, (nshards-1)*Gs < ceil(V/512) <= nshards*Gs; ytgt [T] holds every row's target logit (each row's from the
 * shard that owns its target).  Writes logp, entropy, lse [T] as
 * rlk_linear_logp_fwd does; out-of-range targets give NaN logp and set
 * RLK_DEVERR_TARGET in the workspace. */
int64_t rlk_fwd_split_width(void);
rlk_status rlk_linear_logp_fwd_shard(const rlk_bf16* hidden, const rlk_bf16* W_shard,
                                     const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                     int64_t v0, int64_t V_shard, float temperature,
                                     float* part_m, float* part_s, float* part_b, int64_t Gs,
                                     float* ytgt, void* workspace, size_t workspace_bytes,
                                     void* stream);
rlk_status rlk_linear_logp_combine(const float* part_m, const float* part_s, const float* part_b,
                                   int64_t nshards, int64_t Gs, const float* ytgt,
                                   const int64_t* targets, int64_t T, int64_t V, float* logp,
                                   float* entropy, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Vocab-parallel backward, invariant to the TP degree (same pages and fields
 * as the vocab-parallel forward above).  The single-GPU backward adds the
 * dHidden products of its vocab chunks (rlk_bwd_chunk_width(V) rows each, the
 * last one ragged) in ascending chunk order in fp32 and rounds the sum to
 * bf16 once.  A shard whose first row v0 is a multiple of the chunk width, and
 * whose length is too unless it ends at V, holds whole chunks of the full
 * head; it writes each chunk's fp32 product on its own, and
 * rlk_dhidden_combine adds the products of all shards in global chunk order
 * with the same additions and rounding.  dHidden and dW therefore equal
 * rlk_linear_logp_bwd's bit for bit for any number of shards.
 *
 * rlk_bwd_chunk_width: vocab rows per backward chunk for a V-row head
 * (min(8192, V rounded up to 256)); 0 for V outside [1, 2^31).
 *
 * rlk_linear_logp_bwd_shard: hidden, targets (global indices), lse, entropy,
 * dlogp, dentropy as for rlk_linear_logp_bwd (lse, entropy of the full
 * vocabulary, e.g. from rlk_linear_logp_combine); W_shard [V_shard,H] bf16 =
 * rows v0 .. v0+V_shard-1 of the head.  Writes dW_shard [V_shard,H] fp32 (the
 * shard's rows of dW) and the shard's chunk products into dh_parts, fp32 laid
 * out [S][part_chunks][part_rows][H] with S = ceil(T / part_rows): the product
 * of local chunk k for row t sits at slice t / part_rows, slot k, row
 * t % part_rows (slots past the shard's chunks and rows past T are not
 * written).  part_rows = T gives plain [chunk][T][H]; part_rows =
 * ceil(T / ranks) puts each rank's row slice in one contiguous block, ready for
 * an all-to-all.  part_chunks in [ceil(V_shard / width), ceil(V / width)].
 * Workspace: rlk_linear_logp_workspace_bytes(T, H, V, 1) bytes (full V),
 * 256-byte aligned.  Errors: v0 or V_shard off the chunk grid
 * RLK_ERR_UNSUPPORTED_SHAPE; shard outside [0, V), part_rows < 1 or
 * part_chunks out of range RLK_ERR_INVALID_ARG; otherwise as
 * rlk_linear_logp_bwd.  T = 0 zeroes dW_shard.
 *
 * rlk_dhidden_combine: dh_parts [nparts][count] fp32 (16-byte aligned), the
 * chunk products in global chunk order; writes out[i] = bf16 of
 * ((p_0[i] + p_1[i]) + ...) + p_{nparts-1}[i], out [count] bf16 (8-byte
 * aligned).  count must be a multiple of 4 (RLK_ERR_UNSUPPORTED_SHAPE). */
int64_t rlk_bwd_chunk_width(int64_t V);
rlk_status rlk_linear_logp_bwd_shard(const rlk_bf16* hidden, const rlk_bf16* W_shard,
                                     const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                     int64_t v0, int64_t V_shard, float temperature,
                                     const float* lse, const float* entropy, const float* dlogp,
                                     const float* dentropy, float* dh_parts, int64_t part_rows,
                                     int64_t part_chunks, float* dW_shard, void* workspace,
                                     size_t workspace_bytes, void* stream);
rlk_status rlk_dhidden_combine(const float* dh_parts, int64_t nparts, int64_t count,
                               rlk_bf16* out, void* stream);

/* Diffusion transition step and its log-probability.  The RL-Kernel B200
 * report's transition gate (h3-runtime-integration-b200 report.json,
 * transition[]: shapes B3 x 257x96, B4 x 4096x96, B2 x 8192x32; prev_sample and
 * mean bitwise, logp within 5.8e-6 .. 1.5e-4 of a torch mean, batch invariant,
 * scoring reproduces the sampling logprob) checks such an operator but gives
 * no formula; this library takes the plainest reading, a Gaussian transition
 * with an affine mean, per sample b of n = L * D elements:
 *     mean = a_b x + c_b v,   prev = mean + s_b eps,
 *     logp_b = mean over the n elements of log N(prev; mean, s_b^2)
 *            = -(sum (prev - mean)^2) / (2 s_b^2 n) - ln s_b - ln(2 pi) / 2.
 * x (latent), v (model output), eps (standard normal draw), prev: fp32
 * [B][n] row-major, 16-byte aligned; a, c, s: fp32 [B]; mean_out (may be
 * NULL) and prev_out fp32 [B][n], 16-byte aligned; logp fp32 [B].
 * Elementwise results are single fp32 operations rounded to nearest (a x,
 * c v, their sum; s eps, mean + that), so mean and prev equal plain fp32
 * tensor arithmetic bit for bit.  The residual sum of a sample runs over fixed
 * 4096-element chunks in a fixed order and then over the chunks in order:
 * logp is bitwise independent of B and of the other samples, and
 * rlk_transition_logp on a recorded prev reproduces rlk_transition_sample's
 * logp bit for bit.
 * Sizes: n % 4 == 0, n <= 2^24, B <= 65535 (else RLK_ERR_UNSUPPORTED_SHAPE);
 * B = 0 or n = 0 is a no-op.  Workspace: rlk_transition_workspace_bytes(B, n)
 * bytes, 256-byte aligned, caller-owned, ZERO-FILLED ONCE before its first use
 * (every call leaves its counters at zero again; calls sharing a workspace
 * must not overlap on the GPU).  Its first word is the device error word,
 * rewritten by every call: a non-positive or non-finite s_b gives NaN logp_b
 * and sets RLK_DEVERR_SCALE.  One kernel is enqueued on `stream`; nothing is
 * allocated. */
size_t rlk_transition_workspace_bytes(int64_t B, int64_t n);
rlk_status rlk_transition_sample(const float* x, const float* v, const float* eps,
                                 const float* a, const float* c, const float* s, int64_t B,
                                 int64_t n, float* mean_out, float* prev_out, float* logp,
                                 void* workspace, size_t workspace_bytes, void* stream);
rlk_status rlk_transition_logp(const float* x, const float* v, const float* prev,
                               const float* a, const float* c, const float* s, int64_t B,
                               int64_t n, float* mean_out, float* logp, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Batch-invariant deterministic dense GEMM on the same tensor-core mainloop as
 * every kernel above (also its self-check): C[M,N] fp32 = sum_k A[m,k] B[n,k]
 * with bf16 inputs and fp32 accumulation, each row of C bitwise independent of
 * the other rows of A and repeatable.  The pages run such a route for the
 * dense FFN and LoRA linear ("rlkernel.ffn.qwen3.deterministic.v1",
 * h100-cp-gradient.json runtime readbacks; lora_gate, h3-runtime-integration-
 * b200 report).  a_mn_major == 0: A is stored [M,K] (K contiguous); != 0:
 * stored [K,M].  b_mn_major == 0: B is stored [N,K]; != 0: stored [K,N].
 * M, N, K >= 1; K and N multiples of 8, and M too when a_mn_major.  Needs a
 * workspace of rlk_gemm_workspace_bytes() bytes for its error word.  With
 * row-major A and B and M <= 224 it runs the short-batch forward kernel's
 * mainloop (operands swapped) with a plain store, for M <= 128 and N <= 8192
 * in a half-height form (64 rows of B per CTA on twice the CTAs);
 * every element is the same K-ordered dot product on every path, so C's bits
 * do not depend on M. */
size_t rlk_gemm_workspace_bytes(void);
rlk_status rlk_gemm_bf16_f32(const rlk_bf16* A, const rlk_bf16* B, int64_t M, int64_t N,
                             int64_t K, int a_mn_major, int b_mn_major, float* C,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Backward that publishes each vocab chunk's completion, so that the
 * data-parallel exchange of dW (the one exchange of a token-sharded step; the
 * pages' deterministic collectives: VIME Qwen3-8B TP4/CP2 page, "Required
 * gates") can start on a chunk's rows while later chunks still compute.
 * Arguments, layouts, results and errors are those of rlk_linear_logp_bwd,
 * plus: chunk_done, a caller-owned device array of
 * ceil(V / rlk_bwd_chunk_width(V)) 32-bit words, and seq >= 1.  Chunk c
 * covers W rows [c * width, (c + 1) * width); its word is set to seq (a
 * system-scope release store) once its dW rows (and its dHidden terms) are
 * written.  Give every call a larger seq than the last one on the same words
 * (the words are never cleared).  After a timed-out internal wait every word
 * is set to seq as well, so waiters are released; rlk_read_device_error then
 * reports RLK_DEVERR_TIMEOUT and the results are not to be used.  T = 0:
 * dW is zeroed and the words set in stream order.  chunk_done null or
 * seq = 0: RLK_ERR_INVALID_ARG. */
rlk_status rlk_linear_logp_bwd_signal(const rlk_bf16* hidden, const rlk_bf16* W,
                                      const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                      float temperature, const float* lse, const float* entropy,
                                      const float* dlogp, const float* dentropy,
                                      rlk_bf16* dHidden, float* dW, void* workspace,
                                      size_t workspace_bytes, uint32_t* chunk_done, uint32_t seq,
                                      void* stream);

/* Makes `stream` wait (on the device, no host sync) until *chunk_word >= seq:
 * a stream memory wait on a word rlk_linear_logp_bwd_signal publishes.  Work
 * enqueued on `stream` afterwards sees the chunk's dW rows.  chunk_word
 * device memory, 4-byte aligned; seq >= 1. */
rlk_status rlk_stream_wait_chunk(const uint32_t* chunk_word, uint32_t seq, void* stream);

/* Fixed-order sum out[i] = ((parts[0][i] + parts[1][i]) + parts[2][i]) + ...
 * over nparts (1..64) equally sized fp32 device buffers of `count` elements;
 * `parts` is a HOST array of device pointers.  The data-parallel exchange of
 * dW uses it: every rank's partial dW slice reaches the slice's owner, which
 * adds them in rank order, so the result is bitwise the same whatever order
 * the slices arrive in.  (The pages' deterministic TP collectives stage
 * through CUDA-IPC buffers: VIME Qwen3-8B TP4/CP2 page, "Required gates".)
 * out may alias parts[0].  Enqueued on `stream`; no allocation. */
rlk_status rlk_sum_ordered(const float* const* parts, int nparts, float* out, int64_t count,
                           void* stream);

/* Provenance readback, in the spirit of the pages' per-module runtime
 * readbacks (h100-cp-gradient.json, runs[].validation.runtime_readbacks:
 * backend_ids, call_count).  rlk_backend_id() names this implementation;
 * rlk_call_count(0) / (1) / (2) count successfully enqueued forward
 * (rlk_linear_logp_fwd and rlk_linear_logp_fwd_noalloc) / backward /
 * self-check GEMM calls in this process. */
const char* rlk_backend_id(void);
uint64_t rlk_call_count(int which);

/* Copies the device error word (RLK_DEVERR_* bits) of `workspace` to *flags,
 * then clears it.  Synchronises `stream`. */
rlk_status rlk_read_device_error(void* workspace, uint32_t* flags, void* stream);

/* Test hook for the fail-closed path; not for production use.  The pages' runs
 * require an error status rather than a hang when the operator cannot finish
 * (VIME Qwen3-8B TP4/CP2 page, "Required gates"; h3-runtime-integration-b200
 * report, runtime mode fail_on_fallback).  Every wait inside the kernels is
 * bounded; when one gives up, the kernel sets RLK_DEVERR_TIMEOUT in the
 * workspace's error word, lets its in-flight copies and MMAs finish, frees its
 * tensor memory and returns, and the outputs are not to be used.
 * rlk_test_linear_logp_bwd_stall is rlk_linear_logp_bwd (same arguments,
 * layouts and ownership) with more: wait_limit_ns bounds every wait of the
 * launch (1 ms .. 2 s; the production entry points use 2 s); stall != 0
 * makes the first dHidden unit wait for one more recompute tile than exists,
 * a dependency nothing ever meets; chunk_done / seq, when chunk_done is not
 * null, publish vocab-chunk completion as rlk_linear_logp_bwd_signal does
 * (so the release of the words after a timeout can be tested).  With stall set the call still returns
 * RLK_OK (the launch is enqueued); rlk_read_device_error then reports
 * RLK_DEVERR_TIMEOUT, and later calls on the same workspace and stream behave
 * as on a fresh one.  T = 0 or a limit outside the range: RLK_ERR_INVALID_ARG. */
rlk_status rlk_test_linear_logp_bwd_stall(const rlk_bf16* hidden, const rlk_bf16* W,
                                          const int64_t* targets, int64_t T, int64_t H,
                                          int64_t V, float temperature, const float* lse,
                                          const float* entropy, const float* dlogp,
                                          const float* dentropy, rlk_bf16* dHidden, float* dW,
                                          void* workspace, size_t workspace_bytes,
                                          uint64_t wait_limit_ns, int stall,
                                          uint32_t* chunk_done, uint32_t seq, void* stream);

/* Test hook of the short-batch forward's fail-closed path: rlk_linear_logp_fwd
 * (same arguments, layouts and ownership) for 1 <= T <= 256 rows, the sizes
 * that run the short-batch kernel, with more: wait_limit_ns bounds every wait
 * of the kernel (1 ms .. 2 s; the production entry points use 2 s); stall != 0
 * makes the first CTA of every cluster wait for a second arrival on its first
 * accumulator's "full" barrier, which never comes, so that its epilogue, the
 * chain of the other CTAs and the MMA issuer all run out their waits and
 * unwind.  The call returns RLK_OK (the launches are enqueued); the results
 * are not to be used; rlk_read_device_error then reports RLK_DEVERR_TIMEOUT,
 * and later calls on the same workspace and stream behave as on a fresh one.
 * T outside 1 .. 256 or a limit outside the range: RLK_ERR_INVALID_ARG. */
rlk_status rlk_test_linear_logp_fwd_stall(const rlk_bf16* hidden, const rlk_bf16* W,
                                          const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                          float temperature, float* logp, float* entropy,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          uint64_t wait_limit_ns, int stall, void* stream);

/* Human-readable name of a status code (static string). */
const char* rlk_status_string(rlk_status status);

#ifdef __cplusplus
}
#endif

#endif /* RLK_H_ */
