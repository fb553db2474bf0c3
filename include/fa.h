/*
 * fa.h -- C ABI of the exact tiled-attention library for NVIDIA B200 (sm_100a).
 *
 * The library computes exact softmax attention
 *     O = softmax(scale * Q K^T  [+ causal mask]) V
 * tile by tile with the online-softmax recurrence (running maximum m, running
 * normaliser l, running output rescaled by exp(m_old - m_new)), so the N x N
 * score matrix never reaches device memory, and the training backward that
 * keeps only O and the per-row log-sum-exp and recomputes the score tiles.
 * Sources for the method:
 *   - fanfani.net "FlashAttention": "Do not materialize the matrix" (tiling),
 *     "A pinch of math: making the softmax work in pieces" (the recurrence and
 *     the single division by l at the end), "The backward pass, and where the
 *     memory saving comes from" (keep per-row statistics, recompute blocks);
 *   - mentria.ai "Exact attention, sped up by never writing the giant grid
 *     down": block score equation (S_ij = Q_i K_j^T / sqrt(d)), safe-softmax
 *     equation, running-max recurrence;
 *   - synthetic.wiki "FlashAttention: attention's bottleneck is the wire, not
 *     the maths": "The backward pass buys memory with recompute"; "Versions,
 *     and what the numbers say" (head dimensions up to 256, MQA/GQA).
 *
 * Conventions shared by every entry point
 *   Layout   dense row-major "BHND": Q, O, dO, dQ are [B][Hq][N][d];
 *            K, V, dK, dV are [B][Hkv][N][d]; LSE is float [B][Hq][N].
 *   Heads    grouped-query attention: query head h reads KV head
 *            h / (Hq / Hkv) (contiguous groups); Hkv == Hq is plain multi-head,
 *            Hkv == 1 is multi-query.
 *   Mask     causal != 0 hides key j from query i when j > i (square,
 *            top-left aligned). The pages name "the mask" without defining
 *            it; this is the reading the library implements.
 *   LSE      natural-log log-sum-exp of the scaled scores of each row:
 *            LSE_i = m_i + ln(l_i). It stands in for the two numbers per query
 *            (m, l) that the pages keep: P = exp(scale*S - LSE) rebuilds the
 *            weights without a second pass.
 *   Pointers device pointers (cudaMalloc / torch CUDA tensors), each 16-byte
 *            aligned. The caller owns every buffer; the library allocates no
 *            device memory and keeps no per-call state, except the fixed
 *            scratch array that fa_bwd_noalloc uses (see there).
 *   Streams  every call enqueues its kernels on `stream` (0 = legacy default
 *            stream) and returns without synchronising.
 *   Errors   arguments are checked, and every launch of the call is planned
 *            (tensor maps encoded, grid sizes checked), before anything is
 *            launched; on a non-zero return other than FA_ERR_CUDA nothing
 *            was launched and no output was written. FA_ERR_CUDA from a
 *            failed launch may follow earlier launches of the same call.
 *            Kernels that hit a bounded wait limit record FA_ERR_TIMEOUT in a
 *            per-device status word, read (and cleared) by
 *            fa_last_device_status().
 *   Empty    B == 0 or N == 0 is a valid empty problem: FA_OK, no launch.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that the header
 * does not need the CUDA headers. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID = 1,      /* bad argument: null/misaligned pointer, bad size */
    FA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    FA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
    FA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out */
    FA_ERR_WORKSPACE = 5     /* workspace missing or smaller than required */
} fa_status;

typedef enum {
    FA_BF16 = 0,  /* bfloat16 tensors, float32 accumulation (tensor cores) */
    FA_F32 = 1    /* float32 tensors, float32 arithmetic (CUDA cores) */
} fa_dtype;

/*
 * fa_fwd -- forward pass: O and LSE.
 *
 *   q [B][Hq][N][d], k/v [B][Hkv][N][d]   inputs, element type `dtype`
 *   o [B][Hq][N][d]                        output, element type `dtype`
 *   lse [B][Hq][N]                         output, float32, natural log
 *   d in {64, 128, 256}; Hq % Hkv == 0; B, N >= 0; Hq, Hkv >= 1
 *   scale: the factor applied to Q K^T (1/sqrt(d) gives the pages' scores)
 *   causal: 0 or 1
 *   dtype: FA_BF16 (all d) or FA_F32 (all d)
 * Computes, per (batch, query head), the fused tiled pass of "Do not
 * materialize the matrix" with the recurrence of "A pinch of math", dividing
 * by l once at the end. Returns fa_status.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
           int dtype, fa_stream_t stream);

/*
 * fa_fwd_partial -- fa_fwd over one block of a longer sequence, for attention
 * sharded over the sequence dimension.
 *
 *   arguments as fa_fwd; dtype FA_BF16 only (FA_F32 returns
 *   FA_ERR_UNSUPPORTED)
 *   diag_offset: with causal = 1, query row i sees key row j iff
 *                j <= i + diag_offset (0 gives fa_fwd; values beyond +-N
 *                act as +-N); ignored when causal = 0
 * A row that sees no key (causal, i + diag_offset < 0) gets O = 0 and
 * LSE = -inf. The outputs are the block's own softmax, normalised over its
 * keys, with the LSE that fa_merge_partials needs to combine blocks: the
 * pages name parallelism over the sequence dimension (synthetic.wiki
 * "FlashAttention: attention's bottleneck is the wire, not the maths",
 * "Versions, and what the numbers say") and the rescale rule that makes
 * the merge exact ("A pinch of math"). With the striped assignment (token t
 * on device t mod W), device r's queries against device c's keys are this
 * call with diag_offset 0 for c <= r and -1 for c > r. Returns fa_status.
 */
FA_API int fa_fwd_partial(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   int diag_offset, int dtype, fa_stream_t stream);

/*
 * fa_merge_partials -- combine normalised outputs of disjoint key sets.
 *
 *   o_parts [n_parts][rows][d]   input (bf16): part p's output for each row
 *   lse_parts [n_parts][rows]    input, float32: part p's LSE (-inf: the
 *                                part saw no key of that row)
 *   o [rows][d]                  output (bf16)
 *   lse [rows]                   output, float32, natural log
 *   n_parts >= 1, rows >= 0, d in {64, 128, 256}, dtype FA_BF16
 * With M = max_p LSE_p: L = sum_p exp(LSE_p - M), O = sum_p exp(LSE_p - M)
 * O_p / L, LSE = M + ln L, in float32 ("A pinch of math": the rescale of
 * the running state, applied to states already divided by l). Rows whose
 * parts are all -inf get O = 0, LSE = -inf. rows counts (batch, head,
 * query) triples, so an fa_fwd_partial output [B][Hq][N][d] is
 * rows = B * Hq * N. The outputs may not overlap the inputs
 * (FA_ERR_INVALID). Returns fa_status.
 */
FA_API int fa_merge_partials(const void* o_parts, const float* lse_parts, int n_parts,
                      long long rows, void* o, float* lse, int d, int dtype,
                      fa_stream_t stream);

/*
 * fa_fwd_varlen -- forward pass over a packed batch of sequences of
 * different lengths, or over strided "BNHD" tensors.
 *
 *   q [total_q][Hq][d], k, v [total_k][Hkv][d]   inputs (bf16), tokens of all
 *                                                sequences one after another
 *   o [total_q][Hq][d]                           output (bf16)
 *   lse [total_q][Hq]                            output, float32, natural log
 *   cu_seqlens_q, cu_seqlens_k                   device int32 arrays of batch+1
 *                                                non-decreasing offsets from 0:
 *                                                sequence s owns query tokens
 *                                                cu_seqlens_q[s] .. [s+1]-1 and
 *                                                key tokens cu_seqlens_k[s] ..
 *                                                [s+1]-1
 *   max_seqlen_q                                 the longest query sequence
 *   total_q, total_k                             tokens in q and in k, v
 * Attention runs within each sequence and nothing crosses sequences. A
 * sequence may have fewer queries than keys (a continued prefill, a draft):
 * its queries are then its last positions, and with causal = 1 query i of
 * the sequence sees its keys 0 .. (keys - queries) + i. The pages say nothing
 * on layouts ("the softmax attention you asked for", synthetic.wiki
 * "FlashAttention: attention's bottleneck is the wire, not the maths", "Where
 * to be careful"); this is the plain reading. A dense [B][N][H][d] tensor is
 * the packed layout with offsets 0, N, 2N, ..., BN, so the same call serves
 * BNHD inputs. Supports dtype FA_BF16 with d in {64, 128}; other cases return
 * FA_ERR_UNSUPPORTED. The offsets live on the device, so their consistency
 * (lengths >= 0, at most max_seqlen_q queries, no more queries than keys,
 * inside total_q and total_k) is checked by the kernel: a sequence that
 * fails it is skipped and FA_ERR_INVALID is recorded in the device status
 * word (fa_last_device_status). batch == 0 or total_q == 0 is a no-op.
 */
FA_API int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                  int max_seqlen_q, int total_q, int total_k, int Hq, int Hkv,
                  int d, float scale, int causal, int dtype, fa_stream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs: the
 * per-row term D = rowsum(dO * O) and the log2-scaled LSE, both float32 and
 * padded to a multiple of 128 rows per head, plus a float32 dQ accumulator
 * [B][Hq][N][d]: 4 * (2 * B * Hq * Npad + B * Hq * N * d) bytes, Npad = N
 * rounded up to 128. When B * Hkv * ceil(N / T) < 592, with key tiles of
 * T = 128 keys (64 at d = 256), the backward splits each group's query
 * heads over several CTAs (the smallest divisor s of Hq / Hkv with that
 * product times s >= 592, else Hq / Hkv) and the workspace also holds
 * float32 dK and dV accumulators [B][Hkv][N][d].
 * Linear in N: nothing N x N is ever allocated. Returns 0 for invalid sizes.
 */
FA_API size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * fa_bwd -- backward pass: dQ, dK, dV from Q, K, V, O, LSE and dO.
 *
 *   q, o, dO [B][Hq][N][d], k, v [B][Hkv][N][d]   inputs (bf16)
 *   lse [B][Hq][N] float32                          input, as written by fa_fwd
 *   dq [B][Hq][N][d], dk, dv [B][Hkv][N][d]         outputs (bf16); dk and dv
 *                                                   sum over each KV head's
 *                                                   group of query heads
 *   workspace, workspace_bytes                      scratch owned by the caller,
 *                                                   >= fa_bwd_workspace_size()
 *                                                   bytes, 16-byte aligned;
 *                                                   contents on entry ignored
 * Recomputes every score tile from Q and K and the stored LSE ("The backward
 * pass, and where the memory saving comes from"): P = exp(scale*S - LSE),
 * dV = P^T dO, dP = dO V^T, dS = P * (dP - D), dQ = scale dS K,
 * dK = scale dS^T Q. Supports dtype FA_BF16 with d in {64, 128, 256};
 * FA_F32 returns FA_ERR_UNSUPPORTED. Three kernels run in stream order:
 * D and LSE preparation (and zeroing of the dQ accumulator), the main
 * recompute kernel (one CTA per 128-key tile, 64-key at d = 256: dK and dV,
 * and each dQ tile added into the f32 accumulator), and the dQ conversion; with split query
 * heads (see fa_bwd_workspace_size) the main stage also zeroes the dK/dV
 * accumulators before, and rounds them to dk, dv after, its kernel. dq is
 * summed in whatever order the key tiles finish, so it can differ in the
 * last bit from run to run; dk and dv are bit-for-bit repeatable unless the
 * query heads are split.
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o,
           const float* lse, const void* dO, void* dq, void* dk, void* dv,
           void* workspace, size_t workspace_bytes,
           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
           int dtype, fa_stream_t stream);

/*
 * The three stages of fa_bwd as separate calls, for callers that want to
 * time or schedule them one by one. Calling them in this order on one
 * stream, with the same sizes and workspace, is exactly fa_bwd. Arguments
 * mean what they mean for fa_bwd; the same checks and error codes apply.
 *
 * fa_bwd_prep -- writes D = rowsum(dO * O) and LSE * log2(e) into the
 *   workspace (128-row padded per head; padding rows get D = 0 and an
 *   infinite LSE, i.e. zero weight) and zeroes the f32 dQ accumulator.
 *   Reads o, lse, dO.
 * fa_bwd_main -- the recompute kernel: per 128-key tile of each KV head it
 *   rebuilds P from Q, K and the padded LSE, and forms dV, dP, dS, dK (written
 *   to dk, dv, through f32 accumulators when the query heads are split) and
 *   adds each dQ tile into the accumulator. Needs fa_bwd_prep to have run on
 *   the same workspace.
 * fa_bwd_dq -- converts the f32 dQ accumulator to dq (bf16).
 */
FA_API int fa_bwd_prep(const void* o, const float* lse, const void* dO,
                void* workspace, size_t workspace_bytes,
                int B, int Hq, int Hkv, int N, int d, int dtype,
                fa_stream_t stream);
FA_API int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO,
                void* dk, void* dv, void* workspace, size_t workspace_bytes,
                int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                int dtype, fa_stream_t stream);
FA_API int fa_bwd_dq(void* dq, void* workspace, size_t workspace_bytes,
              int B, int Hq, int Hkv, int N, int d, int dtype,
              fa_stream_t stream);

/*
 * fa_bwd_noalloc -- fa_bwd for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot hand fa_bwd a workspace: code running where the device allocator
 * must not be touched (a locked caching allocator, a fixed memory arena
 * planned ahead of time, a runtime that forbids cudaMalloc once it has
 * started) and plain C callers with no allocator of their own.
 *
 * Same arguments, results and checks as fa_bwd, without workspace and
 * workspace_bytes. The scratch is a fixed device array of
 * FA_NOALLOC_SCRATCH_BYTES bytes inside the library, present on every GPU
 * that loads the library until the process exits. Problems whose
 * fa_bwd_workspace_size() exceeds it return FA_ERR_WORKSPACE without
 * launching anything. The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) and keeps it for the life of the
 * process; make that first call before any stream capture, and do not reset
 * the device afterwards. All calls share the one array: the call rewrites
 * every scratch byte it reads before reading it (it zeroes the dQ
 * accumulator itself), but two calls whose kernels
 * overlap on the GPU (different streams, no ordering between them) race on
 * it and give wrong results. Order such calls on one stream.
 */
#define FA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
FA_API int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                   const float* lse, const void* dO, void* dq, void* dk, void* dv,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   int dtype, fa_stream_t stream);

/*
 * fa_bwd_partial -- one key block's share of the backward, for attention
 * sharded over the sequence (the backward of fa_fwd_partial's blocks).
 *
 *   q, dO [B][Hq][N][d], k, v [B][Hkv][N][d]   inputs (bf16): this rank's
 *                                               queries, a key block
 *   dk_acc, dv_acc [B][Hkv][N][d]               float32 accumulators of the
 *                                               key block's dK, dV: added to,
 *                                               never cleared
 *   workspace                                   as for fa_bwd, after
 *                                               fa_bwd_prep on this rank's O,
 *                                               dO and the LSE of its whole
 *                                               rows (every key block); the
 *                                               block's dQ is added into its
 *                                               f32 dQ accumulator
 *   diag_offset                                 as for fa_fwd_partial: with
 *                                               causal = 1 query i sees key j
 *                                               iff j <= i + diag_offset
 * With the full rows' LSE and D, the block's weights are P = exp(scale S -
 * LSE) and its share of the gradient is dQ += scale dS K, dK += scale dS^T Q,
 * dV += P^T dO, dS = P (dP - D) ("The backward pass, and where the memory
 * saving comes from"); summed over the key blocks it is fa_bwd's result.
 * Call fa_bwd_prep once, fa_bwd_partial once per key block, then fa_bwd_dq
 * for dQ and fa_f32_to_bf16 for dK and dV. dtype FA_BF16 with d in {64, 128};
 * other cases return FA_ERR_UNSUPPORTED. Returns fa_status.
 */
FA_API int fa_bwd_partial(const void* q, const void* k, const void* v, const void* dO,
                   float* dk_acc, float* dv_acc, void* workspace, size_t workspace_bytes,
                   int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                   int diag_offset, int dtype, fa_stream_t stream);

/*
 * fa_f32_to_bf16 -- dst[i] = bf16(src[i]) (round to nearest even) for
 * i < n; n a multiple of 4, both pointers 16-byte aligned device memory
 * (FA_ERR_INVALID otherwise). For the dK, dV accumulators of
 * fa_bwd_partial. Returns fa_status.
 */
FA_API int fa_f32_to_bf16(const float* src, void* dst, size_t n, fa_stream_t stream);

/*
 * fa_bwd_varlen_workspace_size -- bytes of device workspace fa_bwd_varlen
 * needs: 4 * (2 * Hq * P + total_q * Hq * d + A), where P = the multiple
 * of 128 at or above 4 * ceil(total_q / 4) + 4 * batch + 128 (per query
 * head, the D and LSE rows of every sequence, each starting on a 16-byte
 * boundary, with a 128-row tail) and A = 2 * total_k * Hkv * d when the
 * group's query heads are split over several CTAs per key tile (the same
 * rule as fa_bwd_workspace_size with B = 1, N = total_k), else 0. A pure
 * function of the sizes. Returns 0 for invalid sizes.
 */
FA_API size_t fa_bwd_varlen_workspace_size(int batch, int total_q, int total_k, int Hq,
                                           int Hkv, int d);

/*
 * fa_bwd_varlen -- backward pass over a packed batch of sequences of
 * different lengths (or strided BNHD tensors), the gradient of fa_fwd_varlen.
 *
 *   q, o, dO [total_q][Hq][d]        inputs (bf16); o and lse from
 *   lse [total_q][Hq]                fa_fwd_varlen on the same q, k, v
 *   k, v [total_k][Hkv][d]           inputs (bf16)
 *   dq [total_q][Hq][d]              output (bf16)
 *   dk, dv [total_k][Hkv][d]         outputs (bf16): dK, dV summed over the
 *                                    query heads of each KV head's group
 *   cu_seqlens_q, cu_seqlens_k, batch, max_seqlen_q, total_q, total_k:
 *                                    as fa_fwd_varlen; max_seqlen_k the
 *                                    longest key sequence
 *   workspace                        device memory, at least
 *                                    fa_bwd_varlen_workspace_size bytes,
 *                                    16-byte aligned; overwritten
 * Each sequence is its own problem with its queries at its last positions,
 * as in the forward; the formulas are fa_bwd's ("The backward pass, and
 * where the memory saving comes from": scores recomputed from Q and K, the
 * weights rebuilt from the stored LSE). Keys that no query sees, and every
 * key of a sequence with no queries, get zero gradients. dtype FA_BF16 with
 * d in {64, 128}; other cases return FA_ERR_UNSUPPORTED. As in the forward,
 * the offsets' consistency is checked on the device (FA_ERR_INVALID in the
 * device status word; the sequence is skipped). dQ is accumulated with f32
 * atomics, so its last bit may differ between runs. batch == 0 or
 * total_k == 0 is a no-op. Returns fa_status.
 */
FA_API int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                  const float* lse, const void* dO, void* dq, void* dk, void* dv,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                  int Hq, int Hkv, int d, float scale, int causal, void* workspace,
                  size_t workspace_bytes, int dtype, fa_stream_t stream);

/*
 * fa_fwd_kvcache_workspace_size -- bytes of device workspace fa_fwd_kvcache
 * needs, a pure function of the sizes (0 for invalid sizes): per key split,
 * the split's normalised output rows (bf16) and LSE (float32) of all
 * B * Hq * Nq query rows, S * B * Hq * Nq * (2 d + 4) bytes, and 0 when
 * S = 1. The keys are cut into S splits of T tiles of 128 keys; (S, T)
 * minimise ceil(B * Hkv * S / 148) * (T + 2) over S = 1 .. min(tiles, 128),
 * T = ceil(tiles / S), S then reduced to ceil(tiles / T).
 */
FA_API size_t fa_fwd_kvcache_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d);

/*
 * fa_fwd_kvcache -- forward pass of Nq new queries against Nk >= Nq cached
 * keys (decoding, or a short chunk of prefill, over a KV cache).
 *
 *   q [B][Hq][Nq][d], k, v [B][Hkv][Nk][d]   inputs (bf16)
 *   o [B][Hq][Nq][d]                         output (bf16)
 *   lse [B][Hq][Nq]                          output, float32, natural log of
 *                                            the scaled scores
 *   workspace, workspace_bytes               scratch owned by the caller,
 *                                            >= fa_fwd_kvcache_workspace_size()
 *                                            bytes, 16-byte aligned
 *   scale, causal                            as for fa_fwd; query i is at key
 *                                            position Nk - Nq + i, and with
 *                                            causal = 1 it sees keys 0 .. Nk - Nq + i
 * The pages name the KV cache as what now limits serving (fanfani.net
 * "FlashAttention", "The backward pass, and where the memory saving comes
 * from") and define the running-state rescale this uses to merge key splits
 * ("A pinch of math: making the softmax work in pieces"). Two kernels run in
 * stream order: one CTA per (batch, KV head, key split) computes each split's
 * result for all R = (Hq / Hkv) * Nq query rows of the KV head (K and V are
 * read from HBM once), then a merge kernel writes O and LSE (with one split
 * the first kernel writes them itself). The first kernel runs on the tensor
 * cores with the R rows as one 128-row tile. Supports dtype FA_BF16 with d in
 * {64, 128, 256} and R <= 128; other cases return FA_ERR_UNSUPPORTED. Nq > Nk or Nq < 1 returns FA_ERR_INVALID; B == 0 is a
 * no-op. The workspace may be null when its size is 0. On error nothing is
 * written.
 */
FA_API int fa_fwd_kvcache(const void* q, const void* k, const void* v, void* o, float* lse,
                   void* workspace, size_t workspace_bytes,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   int dtype, fa_stream_t stream);

/* Human-readable name of a fa_status value (static string, never NULL). */
FA_API const char* fa_status_string(int status);

/*
 * fa_last_device_status -- synchronises `stream`, returns the current
 * device's status word and clears it: FA_OK, or the first problem a kernel
 * recorded since the last call -- FA_ERR_TIMEOUT (a bounded wait gave up),
 * FA_ERR_INVALID (sequence offsets of fa_fwd_varlen inconsistent with its
 * sizes) or FA_ERR_UNSUPPORTED (a kernel found its shared memory laid out in
 * a way it cannot use). FA_ERR_CUDA if the synchronisation itself fails.
 */
FA_API int fa_last_device_status(fa_stream_t stream);

/*
 * fa_set_wait_timeout_ns -- limit, in nanoseconds, on every spin-wait inside
 * the kernels launched after this call (default 2e9 = 2 s). Values <= 0
 * restore the default. Process-wide.
 */
FA_API void fa_set_wait_timeout_ns(long long timeout_ns);

/*
 * fa_selftest_wait_timeout -- launches one block that waits on a barrier
 * nothing ever arrives at, with a limit of `timeout_ns`, so that the bounded
 * wait runs out and records FA_ERR_TIMEOUT in the status word (read it with
 * fa_last_device_status). Exercises the failure path without faulting or
 * hanging the GPU. Returns FA_ERR_INVALID for timeout_ns outside (0, 1e10].
 */
FA_API int fa_selftest_wait_timeout(long long timeout_ns, fa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
