/*
 * kda.h -- C ABI of libkda: the Kimi Delta Attention (KDA) recurrence on one
 * NVIDIA B200 (sm_100a), in its two schedules.
 *
 * The operation (sources are web pages, cited by title and section):
 *   per token t, per (sequence, head), with the state S in R^{dk x dv}
 *   (row = key channel, column = value channel), g_t = log(alpha_t) in R^dk,
 *   beta_t in (0, 1]:
 *     S~  = Diag(alpha_t) S_{t-1}        decay per key channel
 *     v^  = S~^T k_t                     prediction from the key
 *     e_t = beta_t (v_t - v^)            error
 *     S_t = S~ + k_t e_t^T               write along the key
 *     o_t = S_t^T q_t                    read with the query
 *   "Kimi K3 notes 1: KDA" section 4 (projection form of the update) and
 *   section 5 (boxed summary, decay then delta correction); "Deriving Kimi
 *   Delta Attention from scratch" sections 3-5 (predict, error, write) and
 *   section 6 (the fused recurrent mode for decode and the chunked mode for
 *   prefill are two schedules of this one formula).  No output scale and no
 *   normaliser are applied; q and k are used as given (a caller that wants
 *   L2-normalised q, k or a 1/sqrt(dk) scale applies it beforehand).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers, row-major, densely packed.
 *     Alignment: kda_chunk_fwd needs 16-byte aligned q, k, v, g, o, S0, S_out
 *     and workspace and 4-byte aligned beta and cu_seqlens (kda_gdn_chunk_fwd:
 *     the same, with a 4-byte aligned g); kda_recurrent_step and
 *     kda_gdn_recurrent_step need a 16-byte aligned S and element-aligned q, k,
 *     v, o, g, beta.  The caller owns every buffer and the stream; the
 *     library never allocates, frees or synchronises (except
 *     kda_device_error, which synchronises the given stream by design).
 *   - Calls are asynchronous on `stream`.  The return value reports argument
 *     errors and launch errors; execution errors appear at the caller's next
 *     synchronisation.  On any non-KDA_OK return, kda_last_error() holds a
 *     message for the calling thread.
 *   - dtype selects the element type of q, k, v and o (bf16 or fp32).  g, beta
 *     and the state are always fp32.
 *   - Supported head sizes: dk == dv in {32, 64, 128}; anything else returns
 *     KDA_ERR_UNSUPPORTED.
 *   - Thread safety: no global mutable state is shared between calls apart
 *     from a device-side error word (see kda_device_error).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,    /* null pointer, negative size, bad cu_seqlens */
  KDA_ERR_UNSUPPORTED = 2,    /* head size / chunk size / dtype not built   */
  KDA_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned           */
  KDA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  KDA_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed       */
  KDA_ERR_DEVICE_TIMEOUT = 6  /* a bounded device-side wait gave up         */
} kda_status_t;

typedef enum { KDA_BF16 = 0, KDA_F32 = 1 } kda_dtype_t;

/*
 * Bytes of device workspace kda_chunk_fwd needs for these sizes (0 is a
 * valid answer).  For packed inputs (num_seqs > 0) the bound assumes T total
 * tokens split into num_seqs sequences.  Arguments as for kda_chunk_fwd.
 */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                    int chunk_size, kda_dtype_t dtype);

/*
 * Chunkwise-parallel prefill ("Deriving Kimi Delta Attention from scratch"
 * section 6, chunked mode; "Linear / sparse attention" tutorial section 6.2
 * chunk skeleton and section 5.3 WY representation): C tokens per chunk
 * become dense matrix products plus one unit-lower-triangular solve that
 * corrects each token's provisional error; the dk x dv fp32 state is carried
 * from chunk to chunk.  The result equals the token-by-token recurrence up to
 * rounding and does not depend on chunk_size.
 *
 *   q, k  : [B, T, H, dk]  (dtype)          g : [B, T, H, dk] fp32, log alpha <= 0
 *   v     : [B, T, H, dv]  (dtype)       beta : [B, T, H]     fp32
 *   S0    : [N, H, dk, dv] fp32, or NULL for a zero initial state
 *   o     : [B, T, H, dv]  (dtype), written; must not alias an input
 *   S_out : [N, H, dk, dv] fp32, or NULL; may alias S0
 *   cu_seqlens : device int32 [num_seqs + 1] (packed varlen layout, B == 1,
 *           T == total tokens, cu_seqlens[0] == 0, non-decreasing,
 *           cu_seqlens[num_seqs] == T) or NULL, in which case num_seqs must
 *           be 0 and N = B.  The values live on the device, so they are
 *           checked there: a table that breaks these rules sets the device
 *           error word (kda_device_error reports KDA_ERR_INVALID_ARG) and no
 *           read or write leaves the buffers' bounds.  The tensor-core path
 *           then writes nothing at all (o and S_out keep their contents); the
 *           fp32 path treats each sequence whose own range [cu[n], cu[n+1])
 *           is not inside [0, T] as empty (its S_out is its S0).
 *   chunk_size : 16, 32 or 64.  The tensor-core path (bf16, dk == dv == 128)
 *           runs with 64; other combinations run the fp32-arithmetic path.
 *   workspace : device buffer of at least kda_chunk_fwd_workspace_size(...)
 *           bytes (may be NULL when that size is 0); contents are scratch.
 * Numerics: the tensor-core path takes bf16 operands with fp32 accumulation
 * and an fp32 state; it is exact (no overflow) as long as every key channel's
 * log-decay over any 16 consecutive tokens of a chunk is >= -80 (implied by
 * per-token log alpha >= -5).  Chunks whose every channel decays by no more
 * than 80 over the whole chunk use one decay reference per chunk, the others
 * one per 16-token block; both give the same result up to rounding.  The fp32
 * path has no such restriction.
 */
kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, void* o, float* S_out,
                           const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                           int dk, int dv, int chunk_size, kda_dtype_t dtype,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Fused recurrent step, one token for each of N sequences ("Deriving Kimi
 * Delta Attention from scratch" section 6, recurrent mode for decode): each
 * (sequence, head) state is read once and written once, in place.
 *
 *   q, k : [N, H, dk] (dtype)    v : [N, H, dv] (dtype)
 *   g    : [N, H, dk] fp32       beta : [N, H] fp32
 *   S    : [N, H, dk, dv] fp32, updated in place
 *   o    : [N, H, dv] (dtype), written
 */
kda_status_t kda_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* S, void* o, int N, int H, int dk,
                                int dv, kda_dtype_t dtype, cudaStream_t stream);

/*
 * Gated DeltaNet: the same recurrence with one decay per token and head
 * instead of one per key channel, alpha_t a scalar ("Kimi K3 notes 1: KDA"
 * section 3; "Linear / sparse attention" tutorial section 5.2).  It is KDA
 * with every key channel's gate equal, and runs the same kernels with g
 * broadcast over dk.
 *
 * kda_gdn_chunk_fwd: arguments as kda_chunk_fwd except
 *   g : [B, T, H] fp32, log alpha <= 0, 4-byte aligned.
 * It takes the same workspace (kda_chunk_fwd_workspace_size), chunk sizes,
 * paths and exactness domain (log alpha over any 16 tokens >= -80).
 * kda_gdn_recurrent_step: arguments as kda_recurrent_step except
 *   g : [N, H] fp32.
 */
kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* S0, void* o, float* S_out,
                               const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                               int dk, int dv, int chunk_size, kda_dtype_t dtype,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);
kda_status_t kda_gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, float* S, void* o, int N, int H, int dk,
                                    int dv, kda_dtype_t dtype, cudaStream_t stream);

/*
 * KDA from raw projections, with the input preparation fused into the
 * kernels' load phase ("Kimi K3 notes 1: KDA" section 4: q and k are
 * L2-normalised; "Linear / sparse attention" tutorial section 10: beta and
 * the decay come from bounded activations, sigmoid / softplus).  Per token and
 * head, before the recurrence:
 *   q <- q / max(|q|_2, 1e-12),  k <- k / max(|k|_2, 1e-12)   (over dk, fp32)
 *   log alpha = -softplus(a) = -log(1 + e^a)                   (per key channel)
 *   beta = sigmoid(b) = 1 / (1 + e^-b)
 * Arguments as kda_chunk_fwd / kda_recurrent_step except
 *   a : raw gate logits, same layout as g ([B, T, H, dk] / [N, H, dk]), in
 *       a_dtype (KDA_F32 or KDA_BF16: bf16 halves the largest input);
 *       kda_chunk_fwd_prep needs it 16-byte aligned, the decode step
 *       element-aligned;
 *   b : raw beta logits, fp32, same layout as beta.
 * q and k are read as given (unnormalised); nothing is written back to them.
 * Same workspace, paths and exactness domain as kda_chunk_fwd.
 */
kda_status_t kda_chunk_fwd_prep(const void* q, const void* k, const void* v, const void* a,
                                kda_dtype_t a_dtype, const float* b, const float* S0, void* o,
                                float* S_out, const int32_t* cu_seqlens, int num_seqs, int B, int T,
                                int H, int dk, int dv, int chunk_size, kda_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream);
kda_status_t kda_recurrent_step_prep(const void* q, const void* k, const void* v, const void* a,
                                     kda_dtype_t a_dtype, const float* b, float* S, void* o, int N,
                                     int H, int dk, int dv, kda_dtype_t dtype, cudaStream_t stream);

/*
 * Backward pass of the prefill: the gradients of a scalar loss with respect
 * to q, k, v, g (= log alpha, per key channel), beta and the initial state,
 * given dO (the loss's gradient with respect to o) and, optionally, dS_T
 * (with respect to the final state).  The pages describe only the forward;
 * this is the adjoint of the chunked algebra of "Deriving Kimi Delta
 * Attention from scratch" section 6 and the "Linear / sparse attention"
 * tutorial sections 5.3 and 6.2, run chunk by chunk in reverse with the state
 * gradient carried across chunks.  All arithmetic is fp32 and every decay
 * factor is e^x with x <= 0, so it is exact for any gate.
 *
 *   q, k, v, dout : as kda_chunk_fwd's q, k, v and o (dtype), dout the gradient of o
 *   g, beta, S0   : as kda_chunk_fwd (S0 may be NULL: zero initial state)
 *   dS_T          : [N, H, dk, dv] fp32 or NULL (no loss term on the final state)
 *   dq, dk, dv, dg: [B, T, H, d] fp32, written;  dbeta : [B, T, H] fp32, written
 *   dS0           : [N, H, dk, dv] fp32 or NULL, written
 *   cu_seqlens, num_seqs, B, T, H, dk, dv: as kda_chunk_fwd
 *   workspace     : at least kda_chunk_bwd_workspace_size(...) bytes: the state
 *                   at the start of every 16-token chunk, fp32.
 * Alignment: every pointer element-aligned.  No output may alias an input,
 * the workspace or another output (KDA_ERR_INVALID_ARG for identical
 * pointers; partial overlaps are the caller's to avoid).  One CTA per
 * (sequence, head).
 */
size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs);
kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, const void* dout, const float* dS_T, float* dq, float* dk,
                           float* dv, float* dg, float* dbeta, float* dS0, const int32_t* cu_seqlens,
                           int num_seqs, int B, int T, int H, int dk_, int dv_, kda_dtype_t dtype,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass of the Gated DeltaNet prefill (kda_gdn_chunk_fwd: one decay
 * alpha_t = e^{g_t} per token and head, "Kimi K3 notes 1: KDA" section 3;
 * "Linear / sparse attention" tutorial section 5.2).  Arguments, workspace
 * (kda_chunk_bwd_workspace_size), alignment, aliasing rules and errors as
 * kda_chunk_bwd except
 *   g  : [B, T, H] fp32 log alpha, one per token and head;
 *   dg : [B, T, H] fp32, written: dL/dg_t, which is the sum over the key
 *        channels of the per-channel gradient (every channel decays by g_t).
 */
kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                               const float* S0, const void* dout, const float* dS_T, float* dq, float* dk,
                               float* dv, float* dg, float* dbeta, float* dS0, const int32_t* cu_seqlens,
                               int num_seqs, int B, int T, int H, int dk_, int dv_, kda_dtype_t dtype,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward pass of the prefill from raw projections (kda_chunk_fwd_prep: q, k
 * L2-normalised per token and head, log alpha = -softplus(a), beta =
 * sigmoid(b); "Kimi K3 notes 1: KDA" section 4 and the "Linear / sparse
 * attention" tutorial section 10 for the preparation).  The gradients are
 * those of kda_chunk_bwd, taken on the prepared inputs in fp32, composed
 * with the preparation's Jacobians:
 *   dq = (dq^ - q^ (q^ . dq^)) / |q|  (dq^ / 1e-12 where |q| < 1e-12), dk alike,
 *   da = -sigmoid(a) dg,  db = beta (1 - beta) dbeta.
 * Arguments as kda_chunk_bwd except
 *   q, k           : the raw (unnormalised) projections, dtype;
 *   a, a_dtype     : raw gate logits [B, T, H, dk], KDA_F32 or KDA_BF16, element-aligned;
 *   b              : raw beta logits [B, T, H] fp32;
 *   dq, dk         : [B, T, H, dk] fp32, written: gradients of the RAW q, k;
 *   da             : [B, T, H, dk] fp32, written: gradient of a;
 *   db             : [B, T, H] fp32, written: gradient of b;
 *   workspace      : at least kda_chunk_bwd_prep_workspace_size(...) bytes: the
 *                    checkpoints of kda_chunk_bwd, then fp32 copies of the
 *                    prepared q, k, of v, dO and of the gates (20 B per
 *                    token, head and channel, and 12 B per token-head row, more).
 * Three launches: the preparation, the backward kernel, the chain rule.
 */
size_t kda_chunk_bwd_prep_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs);
kda_status_t kda_chunk_bwd_prep(const void* q, const void* k, const void* v, const void* a, kda_dtype_t a_dtype,
                                const float* b, const float* S0, const void* dout, const float* dS_T, float* dq,
                                float* dk, float* dv, float* da, float* db, float* dS0, const int32_t* cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk_, int dv_, kda_dtype_t dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_chunk_fwd from HOST buffers (library plumbing around the prefill of
 * "Deriving Kimi Delta Attention from scratch" section 6, chunked mode; the
 * pages have no host interface).  q, k, v, g, beta, S0 (or NULL), cu_seqlens
 * (or NULL) are read from host memory and o, S_out (or NULL) written to host
 * memory, with the layouts, sizes and meaning of kda_chunk_fwd (KDA gates, one
 * per key channel).  Use page-locked (pinned) host memory: with pageable
 * memory the copies still happen but do not overlap anything.
 *
 * The batch is processed in `pieces` groups of rows (packed inputs: one
 * group): the host->device copies of group p+1 run on `copy_in`, the prefill
 * of group p on `compute` and the device->host copies of group p-1 on
 * `copy_out`, so both copy directions and the kernels work at once.  The three
 * streams may be the same stream (no overlap then).  Ordering: the copies
 * start after the work already queued on `compute`, and `compute` waits for
 * the last copy back, so synchronising `compute` covers the whole call.
 *
 *   device_buffer : device memory of at least kda_chunk_fwd_host_buffer_size
 *     (same sizes, same pieces) bytes, 256-byte aligned; the library keeps the
 *     device copies of every tensor and the prefill's workspace there.  Its
 *     contents are scratch; it must not be used by anything else until
 *     `compute` has passed the call.
 * Errors: as kda_chunk_fwd (KDA_ERR_WORKSPACE when device_buffer is too
 * small).  The host buffers must stay valid until `compute` has passed the
 * call.  Uses three CUDA events per host thread and device, created on the
 * first call and kept.
 */
size_t kda_chunk_fwd_host_buffer_size(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size,
                                      kda_dtype_t dtype, int pieces);
kda_status_t kda_chunk_fwd_host(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* S0, void* o, float* S_out,
                                const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                                int dv, int chunk_size, kda_dtype_t dtype, int pieces,
                                void* device_buffer, size_t device_buffer_bytes, cudaStream_t compute,
                                cudaStream_t copy_in, cudaStream_t copy_out);

/*
 * kda_chunk_fwd for callers that cannot allocate device memory: the same
 * prefill, same arguments minus the workspace.  (Library plumbing: the pages
 * have no counterpart.)  Some callers get only input and output pointers
 * from a host framework that owns the whole device memory pool, or must not
 * call cudaMalloc because it synchronises the device; this entry point needs
 * no allocation from them and makes none itself.
 *
 * Its scratch is a fixed array inside the library, KDA_NOALLOC_SCRATCH_BYTES
 * bytes on every GPU that loads the library, held until process exit.  Sizes
 * whose kda_chunk_fwd_workspace_size(...) exceeds it are rejected with
 * KDA_ERR_WORKSPACE, except that where the automatic sequence segments
 * (kda_set_segment_chunks, left at 0) make the difference, the call runs
 * without them.  The single-pass tensor-core prefill (see
 * kda_set_prefill_path) needs 256 + 4 * (num_seqs + N * H) bytes, the
 * fp32-arithmetic path none; the two-kernel path keeps a per-chunk image and
 * can exceed it: 64 MiB hold 903 of its (chunk, head) pairs, e.g. B=1, H=8,
 * T=7168.
 * The first call on each device looks up the array's device address (with
 * that device current) and remembers it together with the CUDA context that
 * was current; a call from another context on that device (a driver-API
 * context, or the primary context re-created after cudaDeviceReset) looks it
 * up again.  Make the first call in each context before any stream capture.
 * All calls share the one array: calls whose executions overlap on the GPU
 * (other streams, other threads) race and corrupt each other's results.
 * Nothing in it has to start at zero: each call writes every byte it reads.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* S0, void* o, float* S_out,
                                   const int32_t* cu_seqlens, int num_seqs, int B, int T, int H,
                                   int dk, int dv, int chunk_size, kda_dtype_t dtype,
                                   cudaStream_t stream);

/* Message describing the calling thread's last failure ("" if none). */
const char* kda_last_error(void);

/*
 * Reads and clears the device-side error word.  Kernels set it, never trap:
 * KDA_ERR_DEVICE_TIMEOUT when a bounded wait gives up, KDA_ERR_INVALID_ARG
 * when a cu_seqlens table fails its device-side check (see kda_chunk_fwd).
 * The first error since the last read is kept.  Synchronises `stream` first.
 * *code receives 0 when nothing was raised.
 */
kda_status_t kda_device_error(int* code, cudaStream_t stream);

/*
 * Self-check of the failure detection (library plumbing: the pages have no
 * counterpart).  Launches one small kernel on `stream` whose single waiting
 * thread uses the kernels' own bounded mbarrier wait on a barrier that nothing
 * ever completes: after limit_ns (1 .. 1e9) of wall time the wait gives up,
 * sets the device error word to KDA_ERR_DEVICE_TIMEOUT and the kernel returns
 * normally.  A following kda_device_error() reports and clears it; the
 * context stays usable.  Nothing faults, traps or hangs.
 */
kda_status_t kda_selftest_bounded_wait(unsigned long long limit_ns, cudaStream_t stream);

/*
 * Sequence parallelism of the tensor-core prefill (across the chunks of one
 * sequence).  The state pass is linear in the state, so a segment of L chunks
 * maps its entry state as S -> M S + N ("Linear / sparse attention" tutorial
 * section 6.2: the state handed from chunk to chunk; composing those hand-offs
 * is exact algebra).  When the (sequence, head) units are too few to fill the
 * GPU and the sequences are long (64 chunks or more, when a wave-count model
 * of the two schedules says it pays), kda_chunk_fwd (and its _gdn / _prep forms)
 * splits each sequence into segments: the maps of all segments are formed in
 * parallel, chained from S0 in fp32, and every segment is then run from its
 * entry state.  Packed (cu_seqlens) inputs are not split.  The workspace size
 * accounts for it.
 *
 * kda_set_segment_chunks: for the calling thread's later calls (including
 * kda_chunk_fwd_workspace_size), 0 = choose automatically (default), L > 0 =
 * segments of L chunks whenever a sequence has more than L chunks, < 0 = never
 * split.  kda_segment_chunks returns the choice for these sizes on the
 * current device (0 = not split).
 */
kda_status_t kda_set_segment_chunks(int chunks);
int kda_segment_chunks(int B, int T, int H, int num_seqs);

/*
 * Which kernel forms the per-chunk operands of the tensor-core prefill
 * ("Deriving Kimi Delta Attention from scratch", section 6: everything of a
 * chunk that does not involve the carried state).  Two kernels compute the
 * same result: a warp-specialised one (one CTA per SM; one warp group builds
 * the decay-scaled operands of a chunk while the other inverts the previous
 * chunk's I + A; inputs arrive by tensor-map TMA) and a two-CTA-per-SM one.
 * For the calling thread's later calls (kda_chunk_fwd, kda_gdn_chunk_fwd,
 * kda_chunk_fwd_prep on the tensor-core path): 0 (default) uses the
 * warp-specialised kernel (packed sequences: after a one-CTA kernel has built
 * a chunk table from cu_seqlens in the workspace), with the two-CTA kernel for
 * the chunks whose log-decay over the chunk falls below -80 on some channel;
 * 1 = the two-CTA kernel always.  Other values: KDA_ERR_INVALID_ARG, setting
 * unchanged.
 */
kda_status_t kda_set_local_kernel(int variant);

/*
 * Which tensor-core prefill runs (bf16, dk == dv == 128, chunk 64), for the
 * calling thread's later calls (kda_chunk_fwd, kda_gdn_chunk_fwd,
 * kda_chunk_fwd_prep, their workspace sizes and kda_chunk_fwd_phases).  Both
 * compute the chunked form of "Deriving Kimi Delta Attention from scratch"
 * section 6:
 *   1 = single pass: one persistent kernel, one CTA per SM, each CTA taking
 *       whole (sequence, head) units (packed sequences longest first) and
 *       carrying the state from chunk to chunk in tensor memory; nothing of a
 *       chunk goes to HBM but its outputs; its workspace is a few hundred bytes;
 *   2 = two kernels: every chunk's operands built in parallel into a per-chunk
 *       workspace image, then a state pass over the chunks of each unit (the
 *       path that also splits long sequences into segments);
 *   0 = automatic (default): the single pass for packed sequences with at
 *       least one (sequence, head) unit per SM (it balances unequal lengths
 *       longest first) and for batches whose units fill their waves (one
 *       unit per SM) to at least 80% (on 148 SMs: 128 or 256 units, e.g.
 *       B8 H32), with at least 16 chunks per sequence; the two kernels
 *       otherwise.
 * The single pass runs a plain instance and then a precise one, which
 * recomputes only the units where the plain one met near-parallel keys (some
 * |A_rj| >= 0.5) and returns at once when there are none.
 * The two-kernel path keeps U and E in bf16 and T diag(beta) without its lo
 * part, which is accurate unless a chunk has near-parallel keys (some
 * |A_rj| >= 0.5, e.g. a key repeated within a chunk): its chunk-local kernels
 * then raise a flag in the workspace, its state pass does nothing, and the
 * single-pass kernel, launched last in every two-kernel call (it returns at
 * once when the flag is clear), recomputes the whole call in its precise form.
 * Other values: KDA_ERR_INVALID_ARG, setting unchanged.
 */
kda_status_t kda_set_prefill_path(int path);

/*
 * Phases of one kda_chunk_fwd call with these sizes on the current device and
 * the calling thread's settings: 1 for the fp32-arithmetic path and for the
 * single-pass tensor-core prefill, 2 for the two-kernel one (the chunk-local
 * phase, then the state pass).  kda_profile_events records one event before
 * the call and one after each phase.
 */
int kda_chunk_fwd_phases(int B, int T, int H, int num_seqs, int dk, int dv, int chunk_size, kda_dtype_t dtype);

/*
 * Largest number of phases any kda_chunk_fwd call with these head and chunk
 * sizes can run: 1 for the fp32-arithmetic path (one kernel); 2 for the
 * tensor-core path, whose two-kernel form runs the chunk-local phase (the
 * precise fallback's set-up kernel, then one kernel, or two when the
 * warp-specialised kernel hands its steep chunks to the two-CTA kernel, see
 * kda_set_local_kernel) and then the state pass (one kernel, or three when the
 * sequences are split into segments) followed by the precise fallback's
 * single-pass kernel (see kda_set_prefill_path).
 */
int kda_chunk_fwd_launches(int dk, int dv, int chunk_size, kda_dtype_t dtype);

/*
 * Measurement hook.  While set (events != NULL), each later kda_chunk_fwd,
 * kda_gdn_chunk_fwd or kda_chunk_fwd_prep call made by the calling thread
 * records events[0] before its first kernel launch and events[i] after its
 * i-th phase, on the call's stream; count must be at least
 * kda_chunk_fwd_phases(...) + 1 for the call's sizes (kda_chunk_fwd_launches(...) + 1
 * always suffices) or the call fails with KDA_ERR_INVALID_ARG.
 * The caller owns the events.  Pass NULL, 0 to stop.
 */
kda_status_t kda_profile_events(cudaEvent_t* events, int count);

/* Library version, major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
