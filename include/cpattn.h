/*
 * cpattn.h -- C-ABI of libcpattn.so, the B200 (sm_100a) hot path of
 * context-parallel attention for diffusion transformers.
 *
 * What the calls compute, by source page and section:
 *
 *   diffusers context-parallelism guide (optimization/context_parallelism),
 *     §Ring Attention        -- each rank attends its local Q to every K/V
 *                               block as the blocks go round the ring; after a
 *                               full round it has seen every token.
 *     §Ring Anything         -- any sequence length; K/V blocks are trimmed to
 *                               their true (uneven) length before attention.
 *     §Ulysses Attention     -- all-to-all from sequence shards to head
 *                               shards, attention per head subset, and the
 *                               inverse all-to-all.
 *     §Unified Attention     -- all-to-all, then Ring Attention, then the
 *                               inverse all-to-all on a 2-D rank grid.
 *   diffusers parallelism API page (api/parallel), §ContextParallelConfig
 *     convert_to_fp32        -- per-block output and LSE are combined in fp32.
 *     rotate_method          -- "allgather": every K/V block is present before
 *                               the walk, which is what a chunk list models.
 *
 * The pages give no C interface, tensor layout or merge equation; the layout
 * and the equations below are the plain reading of those passages.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are described by cp_tensor: a DEVICE pointer, a dtype, a rank and
 *    per-dimension sizes and strides counted in ELEMENTS (a tensor with no
 *    elements may carry a NULL pointer).  The caller owns all
 *    memory; the library never allocates, frees or retains a pointer past the
 *    call (it builds TMA descriptors per call on the host).
 *  - q/k/v/out are [B, S, H, D] ("BSHD"); the last dimension must be
 *    contiguous (stride 1).  lse is [B, H, S] float32 in natural log.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  The return value reports argument
 *    and launch errors only; device-side faults surface on the stream.
 *  - scale: pass 0 or NaN for the default 1/sqrt(D).
 *  - Attention is non-causal with no mask (Ring Anything forbids masks).
 *  - Supported: D in {64, 128}; q/k/v all CP_BF16 (tcgen05 tensor-core path,
 *    fp32 accumulation) or all CP_F32 (exact fp32 FFMA path); out CP_F32 or
 *    CP_BF16; lse always CP_F32.  TMA needs 16-byte-aligned base pointers and
 *    strides for bf16 inputs.
 *  - Empty key sets give out = 0 and lse = -inf (the merge identity).
 *  - The bf16 attention runs on a persistent grid (one CTA per SM) that takes
 *    its work units from a device counter pair owned by the library; each
 *    launch takes the next of 64 pairs per device and leaves it at zero.  So
 *    at most 64 of these launches may execute at the same time on one device
 *    (from different streams); more could share a pair and skip work.
 */
#ifndef CPATTN_H_
#define CPATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CP_MAX_DIMS 6
#define CP_MAX_CHUNKS 512

typedef enum { CP_F32 = 0, CP_BF16 = 1 } cp_dtype;

typedef struct {
  void*   data;                    /* device pointer                     */
  int32_t dtype;                   /* cp_dtype                           */
  int32_t ndim;                    /* number of dimensions in use        */
  int64_t shape[CP_MAX_DIMS];
  int64_t stride[CP_MAX_DIMS];     /* element strides                    */
} cp_tensor;

/* Status codes (0 = success, negative = error). */
enum {
  CP_OK = 0,
  CP_ERR_NULL = -1,      /* a required pointer or tensor is NULL            */
  CP_ERR_DTYPE = -2,     /* unsupported or mismatched dtypes                */
  CP_ERR_SHAPE = -3,     /* bad rank, mismatched B/H/D, D not 64/128, ...   */
  CP_ERR_ALIGN = -4,     /* base/stride not 16-byte aligned, or inner dim
                            not contiguous                                   */
  CP_ERR_OFFSETS = -5,   /* chunk offsets not monotone, not starting at 0,
                            not ending at S_kv, or too many chunks; chunk
                            lengths outside [0, L] or a bad skip_chunk     */
  CP_ERR_DEGREE = -6,    /* Ulysses/ring degree does not divide S or H      */
  CP_ERR_CUDA = -7,      /* a CUDA runtime/driver call failed               */
  CP_ERR_TIMEOUT = -8,   /* a bounded device-side wait gave up              */
  CP_ERR_WORKSPACE = -9, /* workspace missing or too small                  */
  CP_ERR_ALIAS = -10,    /* an output overlaps an input it must not alias,
                            or maps two of its own elements to one address
                            (a zero stride, or dims that interleave)        */
  CP_ERR_BOUNDS = -11    /* a device-side bounds check failed (debug build,
                            libcpattn_debug.so, compiled with CP_DEBUG)     */
};

/*
 * cp_attn_partial -- one ring step (§Ring Attention): attention of the local
 * query block against ONE K/V chunk, normalised within the chunk.
 *   q       [B, S_q, H, D]    k_chunk, v_chunk [B, S_c, H, D]
 *   out     [B, S_q, H, D]    (CP_F32 or CP_BF16)  = softmax(scale q k^T) v
 *   lse     [B, H, S_q] f32   = ln sum_j exp(scale q.k_j)   (natural log)
 * S_c may be 0 (empty chunk): out = 0, lse = -inf.  Rows past the chunk are
 * never read (the chunk extent bounds every load).
 */
int cp_attn_partial(const cp_tensor* q, const cp_tensor* k_chunk,
                    const cp_tensor* v_chunk, float scale, cp_tensor* out,
                    cp_tensor* lse, void* stream);

/*
 * cp_attn_partial_merge -- one ring step with the merge fused into its
 * epilogue: the partial of q against this K/V chunk is folded into the fp32
 * accumulator (out_acc, lse_acc) in place, with the same log-sum-exp merge
 * as cp_lse_merge.  This is the call a ring rank makes as each chunk
 * arrives; it writes no separate partial and needs no merge pass.
 *   out_acc [B, S_q, H, D] f32 (in/out)   lse_acc [B, H, S_q] f32 (in/out)
 * Start from (0, -inf).  An empty chunk leaves the accumulator unchanged.
 */
int cp_attn_partial_merge(const cp_tensor* q, const cp_tensor* k_chunk,
                          const cp_tensor* v_chunk, float scale,
                          cp_tensor* out_acc, cp_tensor* lse_acc,
                          void* stream);

/*
 * cp_lse_merge -- fold one partial into an fp32 accumulator, in place
 * (ContextParallelConfig.convert_to_fp32).  Per row, with a = lse_acc and
 * b = lse_i:
 *   lse' = max(a,b) + log1p(exp(-|a-b|))
 *   out' = exp(a - lse') * out_acc + exp(b - lse') * out_i
 * (out_acc = 0, lse_acc = -inf) is the identity; when a = b = -inf the
 * accumulator is left unchanged.
 *   out_acc [B, S, H, D] f32 (in/out)   lse_acc [B, H, S] f32 (in/out)
 *   out_i   [B, S, H, D] f32 or bf16    lse_i   [B, H, S] f32
 */
int cp_lse_merge(cp_tensor* out_acc, cp_tensor* lse_acc,
                 const cp_tensor* out_i, const cp_tensor* lse_i, void* stream);

/*
 * cp_ring_attention -- the whole ring walk on one GPU (§Ring Attention with
 * rotate_method="allgather"; §Ring Anything for uneven chunks).  Chunk c is
 * keys [chunk_offsets[c], chunk_offsets[c+1]) of k/v.  The per-chunk partials
 * and their fp32 LSE merge are fused: each chunk's running statistics are
 * folded into one fp32 accumulator at the chunk boundary, so the result is
 * exactly the merge of the per-chunk partials (up to rounding).
 *   chunk_offsets: HOST array of n_chunks+1 int64, [0] = 0, non-decreasing,
 *                  [n_chunks] = S_kv; 1 <= n_chunks <= CP_MAX_CHUNKS.
 *                  Empty chunks are allowed and contribute nothing.
 *   out [B, S_q, H, D] f32 or bf16; lse [B, H, S_q] f32 (may be NULL).
 */
int cp_ring_attention(const cp_tensor* q, const cp_tensor* k,
                      const cp_tensor* v, const int64_t* chunk_offsets,
                      int n_chunks, float scale, cp_tensor* out,
                      cp_tensor* lse, void* stream);

/*
 * cp_ring_attention_gathered -- the ring over the slots of a padded K/V
 * all-gather (§Ring Anything: every rank pads its K/V to the longest local
 * length, the padded shards are all-gathered, and the padding is trimmed
 * before attention).  Here the trim is part of the chunk walk: chunk c is
 * rows [0, chunk_lengths[c]) of slot c, read in place, and the padding rows
 * are never attended.
 *   q          [B, S_q, H, D]        bf16 or f32
 *   k_gathered [R, B, L, H, D]       same dtype as q; R = n_chunks slots of
 *   v_gathered [R, B, L, H, D]       L >= every chunk length (rank order)
 *   chunk_lengths: HOST array of n_chunks int64 in [0, L].
 *   skip_chunk: a chunk to leave out (-1: none), typically the caller's own
 *               chunk when it has already been folded in from local memory.
 *   accumulate: 0 writes (out, lse) like cp_ring_attention (lse may be
 *               NULL); 1 folds the result into the fp32 accumulator
 *               (out f32, lse required) like cp_attn_partial_merge, and is
 *               a no-op when no chunk remains.
 * The padding rows of k and v may hold any value, NaN and Inf included:
 * the bf16 path loads a chunk's last 128-row tile whole, masks the scores
 * of the padded keys to -inf and zeroes the padded v rows in shared memory
 * before P V reads them; the f32 path never loads them.
 */
int cp_ring_attention_gathered(const cp_tensor* q, const cp_tensor* k_gathered,
                               const cp_tensor* v_gathered,
                               const int64_t* chunk_lengths, int n_chunks,
                               int skip_chunk, float scale, int accumulate,
                               cp_tensor* out, cp_tensor* lse, void* stream);

/*
 * cp_ulysses_permute -- the Ulysses all-to-all as an on-GPU layout
 * permutation (§Ulysses Attention).  U = degree.
 *   dir 0 (sequence shards -> head shards):
 *     x [U, B, S/U, H, D]  ->  y [U, B, S, H/U, D]
 *     y[q, b, p*S/U + s, h', d] = x[p, b, s, q*H/U + h', d]
 *   dir 1 (head shards -> sequence shards): the exact inverse,
 *     x [U, B, S, H/U, D]  ->  y [U, B, S/U, H, D]
 * Bit-exact copy of CP_F32 or CP_BF16 elements (x and y same dtype).  The
 * (H or H/U, D) dimensions of both tensors must be packed; the other strides
 * are free, so y may be a strided view into a larger buffer.  H % U == 0 and
 * S % U == 0 (the Ulysses rule of the guide's variant table), else
 * CP_ERR_DEGREE.  x and y must not overlap.
 */
int cp_ulysses_permute(const cp_tensor* x, cp_tensor* y, int degree, int dir,
                       void* stream);

/*
 * cp_usp_attention -- unified sequence parallelism (§Unified Attention)
 * emulated on one GPU for a ring_degree R x ulysses_degree U grid.  Rank
 * g = r*U + u (ring outer, Ulysses inner: the mesh dimension order of
 * ContextParallelConfig.mesh) holds sequence shard g.
 *   q/k/v_shards, out_shards: [R*U, B, S/(R*U), H, D]
 *   lse: [B, H, S] f32 in token order (may be NULL)
 * Steps: Ulysses permute inside every group r; ring attention with R
 * chunks per head group u; inverse permute.  R = 1 is plain Ulysses.
 * For bf16 inputs with D in {64, 128}, 16-byte-aligned strides and a shard
 * length S/(R*U) that is a multiple of 128, the permutations are folded into
 * the attention kernel's tensor maps: one launch reads q/k/v and writes out
 * in the shard layout, and the workspace is not used (may be NULL).
 * Otherwise the intermediates live in the caller's workspace
 * (cp_usp_workspace_bytes).
 */
int cp_usp_attention(const cp_tensor* q_shards, const cp_tensor* k_shards,
                     const cp_tensor* v_shards, int ring_degree,
                     int ulysses_degree, float scale, void* workspace,
                     size_t workspace_bytes, cp_tensor* out_shards,
                     cp_tensor* lse, void* stream);

/* Workspace bytes cp_usp_attention needs for contiguous tensors of these
 * sizes: 0 when the permutations fold into the attention kernel (see above)
 * or on bad input.  in_dtype is the q/k/v dtype, out_dtype the out_shards
 * dtype. */
size_t cp_usp_workspace_bytes(int64_t B, int64_t S, int64_t H, int64_t D,
                              int in_dtype, int out_dtype, int ring_degree,
                              int ulysses_degree);

/*
 * cp_usp_attention_static -- cp_usp_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart to this call: it
 * exists for hosts such as another engine's plugin hook, where a cudaMalloc
 * would synchronise the device and is not allowed, or a plain-C program with
 * no CUDA allocator of its own.  The caller still passes inputs and outputs
 * (same arguments and results as cp_usp_attention); the workspace is a
 * fixed device array of CP_USP_STATIC_SCRATCH_BYTES inside the library,
 * which every GPU that loads this part of the library holds until the
 * process exits.  The call allocates nothing.
 *   - Sizes whose workspace (cp_usp_workspace_bytes) exceeds
 *     CP_USP_STATIC_SCRATCH_BYTES are rejected with CP_ERR_WORKSPACE before
 *     any GPU work.
 *   - Arguments are checked exactly as by cp_usp_attention and give the
 *     same error codes.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current).  With CUDA's lazy
 *     module loading that lookup also loads this part of the library and
 *     reserves the array, and it may synchronise the device.  So make one
 *     call per device before any stream capture or latency-critical hook: a
 *     call with an empty problem (B = 0) does only this set-up and launches
 *     nothing.
 *   - Every call shares the one array and it keeps the last call's contents
 *     (all of it is rewritten before it is read, so nothing needs clearing):
 *     calls whose GPU work overlaps -- other streams, other threads -- race.
 */
#define CP_USP_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
int cp_usp_attention_static(const cp_tensor* q_shards,
                            const cp_tensor* k_shards,
                            const cp_tensor* v_shards, int ring_degree,
                            int ulysses_degree, float scale,
                            cp_tensor* out_shards, cp_tensor* lse,
                            void* stream);

/*
 * cp_ulysses_anything_permute -- the Ulysses all-to-all when the degree U
 * divides neither the sequence length nor the head count (§Ulysses Anything
 * Attention; ContextParallelConfig.ulysses_anything).  Rank p holds tokens
 * [seq_offsets[p], seq_offsets[p+1]), rank q heads [head_offsets[q],
 * head_offsets[q+1]) (HOST arrays of U+1 int64: 0, non-decreasing, ending
 * at S and H; cp_ring_chunk_offsets gives the ceil split).  Every rank's
 * buffer is contiguous, so both sides are flat 1-D buffers of B*S*H*D
 * elements, the rank buffers concatenated in rank order:
 *   sequence side: rank p holds [B, s_p, H, D]
 *   head side:     rank q holds [B, S, h_q, D] (every token, in order)
 *   dir 0: y[q][b, off_p + s, h', d] = x[p][b, s, hoff_q + h', d]
 *   dir 1: the exact inverse.
 * Bit-exact copy; x and y same dtype, contiguous, not overlapping.
 * 1 <= U <= CP_MAX_CHUNKS; empty ranks are allowed.
 */
int cp_ulysses_anything_permute(const cp_tensor* x, cp_tensor* y, int64_t B,
                                int64_t H, int64_t D, int degree,
                                const int64_t* seq_offsets,
                                const int64_t* head_offsets, int dir,
                                void* stream);

/*
 * cp_ulysses_anything_attention -- Ulysses Anything (ring_degree 1): the
 * uneven all-to-all above, attention of every head group over the whole
 * sequence, and the inverse all-to-all.  q/k/v/out are flat sequence-side
 * buffers as above (out f32 or bf16); lse is [B, H, S] f32 in token order
 * (may be NULL).  On one GPU all head groups share the device, so the data
 * is moved only as far as one attention launch over all heads needs: for
 * B = 1 the rank buffers already form [1, S, H, D] and are read in place
 * (no workspace); for B > 1 the sequence is gathered into the caller's
 * workspace of cp_ulysses_anything_workspace_bytes bytes (256-byte
 * aligned) and the output scattered back.
 */
int cp_ulysses_anything_attention(const cp_tensor* q, const cp_tensor* k,
                                  const cp_tensor* v, int64_t B, int64_t H,
                                  int64_t D, int degree,
                                  const int64_t* seq_offsets,
                                  const int64_t* head_offsets, float scale,
                                  void* workspace, size_t workspace_bytes,
                                  cp_tensor* out, cp_tensor* lse, void* stream);
size_t cp_ulysses_anything_workspace_bytes(int64_t B, int64_t S, int64_t H,
                                           int64_t D, int in_dtype,
                                           int out_dtype);

/*
 * cp_ring_chunk_offsets -- the Ring Anything split of S tokens over R ranks:
 * ceil(S/R) tokens per rank, the last ranks holding the rest (possibly
 * nothing).  Writes R+1 offsets to the HOST array `offsets`.
 */
int cp_ring_chunk_offsets(int64_t S, int R, int64_t* offsets);

/* Static text for a status code. */
const char* cp_status_string(int status);

/*
 * cp_last_device_error -- synchronises `stream`, returns CP_ERR_TIMEOUT if a
 * bounded device-side wait in any kernel of this library gave up since the
 * last call, CP_ERR_BOUNDS if a device-side bounds check of the debug build
 * failed first (else CP_OK, or CP_ERR_CUDA if the stream reports an error),
 * and clears the flag.
 */
int cp_last_device_error(void* stream);

/*
 * cp_selftest_wait_timeout -- launches one block that waits on an mbarrier
 * nothing will ever complete, with a spin limit of `spin_limit` polls; the
 * wait gives up, sets the device error flag and the kernel returns.  Used by
 * the tests to check that bounded waits surface as CP_ERR_TIMEOUT without
 * hanging or faulting the GPU.
 */
int cp_selftest_wait_timeout(int spin_limit, void* stream);

/*
 * cp_selftest_bounds_check -- launches one thread whose single bounds check
 * fails on purpose (an index one past a one-element range).  The debug build
 * (libcpattn_debug.so, CP_DEBUG) records it, so the next
 * cp_last_device_error returns CP_ERR_BOUNDS; the release build compiles the
 * check away and records nothing.  The guarded store goes to the block's own
 * shared memory in either build.  Used by the tests to check that the debug
 * build's checks are live and surface without a GPU fault.
 */
int cp_selftest_bounds_check(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CPATTN_H_ */
