/* dsa.h -- C ABI of the B200 (sm_100a) DSA sparse-attention prefill library.
 *
 * One call processes one prefill chunk of n_q queries against a cache that
 * already holds the chunk's own rows. Query i sits at absolute position
 * t = q_pos0 + i and sees cache rows s = 0..t.
 *
 * Where the operations come from. The feedman.me post feedman.me/posts/wy2HU
 * (an M3 Ultra + M5 Ultra prefill/decode split for GLM-5.3-Flash) profiles the
 * layer in its per-component prefill table (rows "DSA indexer" and "DSA
 * sparse-attention core"), calls the attention step a per-query top-2048
 * gather kernel (paragraph after the table), describes it as gathering each
 * query's 2,048 keys for dot products (paragraph "Two levers fell out of
 * this"), and gives the 512-wide latent KV ("Why the hand-off is cheap"). The
 * pages print no formula; the definitions below are the plainest reading of
 * DeepSeek-style sparse attention that agrees with them.
 *
 * Conventions shared by every entry point
 *  - bf16 tensors are passed as uint16_t bit patterns; float tensors are IEEE
 *    float32; every tensor is dense, row-major, in device memory, and its base
 *    address is 16-byte aligned.
 *  - The caller owns all memory, including the workspace. The library never
 *    allocates or frees memory and never synchronizes the stream, except
 *    dsa_device_status(), which exists to do exactly that.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream). The returned status covers argument
 *    checks and kernel launch only. A device-side failure (a bounded wait that
 *    gave up, or an index out of range) is recorded in the workspace's status
 *    word and reported by dsa_device_status(). Every call clears that word
 *    first, so it always describes the latest call that used the workspace.
 *  - Calls that share a workspace must not overlap on the GPU (use one stream,
 *    or one workspace per stream).
 *  - Argument errors are returned before anything is launched; outputs are
 *    then left untouched.
 *  - n_q == 0 is valid and launches nothing.
 *  - Inputs must be finite (no NaN or Inf).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Shapes of one prefill chunk. */
typedef struct dsa_dims {
  int32_t n_q;         /* queries in the chunk, >= 0                                  */
  int32_t q_pos0;      /* absolute position of query 0, >= 0                          */
  int32_t ctx_len;     /* cache rows T, q_pos0 + n_q <= T <= DSA_MAX_CTX              */
  int32_t n_heads;     /* attention heads H                                           */
  int32_t d_latent;    /* latent width Dc (the attention value is the latent row)     */
  int32_t d_rope;      /* rotary width Dr (keys only; already rotated)                */
  int32_t n_idx_heads; /* indexer heads H_I (query side; one shared key per row)      */
  int32_t d_idx;       /* indexer head width D_I                                      */
  int32_t top_k;       /* keys kept per query, 1..DSA_MAX_TOPK                        */
  float softmax_scale; /* multiplies the attention logits                             */
  uint32_t flags;      /* 0, or the DSA_FLAG_* options below where a call accepts them */
} dsa_dims;

/* dims.flags: the whole-layer calls (dsa_prefill_layer, dsa_decode_layer,
 * dsa_prefill_layer_host, dsa_prefill_layer_noalloc) score with the FP8
 * indexer: q_idx and k_idx are taken to their e4m3 form (dsa_quantize_fp8,
 * in the workspace), scored by dsa_index_scores_fp8, and the exact top-k
 * orders keys by the float64 contract of dsa_topk_select on the dequantized
 * rows. Calls other than those named here require flags == 0. */
#define DSA_FLAG_FP8_INDEXER 1u
/* dims.flags: dsa_sparse_attn_prefill and the prefill-layer calls run the
 * attention on SM pairs (a thread-block cluster of two CTAs per query, each
 * gathering half of every selected key's dims, so that two tiles fit in
 * flight; the halves of S and P cross between the pair through distributed
 * shared memory). Shapes without that kernel (the 4-head shape) and the
 * decode calls ignore it. Outputs agree with the one-SM kernel within
 * rounding; selections are unaffected. */
#define DSA_FLAG_ATTN_PAIR 2u
/* dims.flags: dsa_prefill_layer_host does not order itself after the work
 * that earlier calls left on its streams; the caller orders it instead. With
 * two sets of device tensors used in turn, each set reused only after an
 * event recorded on streams[2] at the end of the call that last used it,
 * the copy-in of one chunk then overlaps the layers and the copy-out of the
 * previous one. The other calls reject it (DSA_ERR_DIMS). */
#define DSA_FLAG_HOST_UNORDERED 4u
/* dims.flags: dsa_prefill_layer scores and selects over query sub-blocks
 * whose float32 scores fit 64 MiB (a multiple of 64 rows, at least 64: 960
 * rows at a 17,408-token context), one sub-block after the other. The score
 * matrix then stays in L2 between the indexer that writes it and the top-k
 * that reads it, instead of making a round trip through HBM. The workspace
 * (dsa_workspace_size with the same dims) holds one sub-block's scores.
 * Selections, outputs and lse are bit-identical to the default schedule.
 * dsa_prefill_layer_noalloc accepts it too (its scratch then holds the
 * sub-block workspace). Not with DSA_FLAG_FP8_INDEXER; the other calls reject
 * it (DSA_ERR_DIMS). */
#define DSA_FLAG_L2_SCORES 8u

/* Supported shapes (anything else returns DSA_ERR_DIMS; there is no fallback):
 *   (n_heads, d_latent, d_rope)  in {(4, 64, 16), (32, 512, 64)}
 *   (n_idx_heads, d_idx)         in {(2, 32), (32, 128)}
 *   1 <= top_k <= 2048, ctx_len <= 131072                                      */
#define DSA_MAX_TOPK 2048
#define DSA_MAX_CTX 131072

typedef int32_t dsa_status;
#define DSA_OK 0
#define DSA_ERR_NULL (-1)      /* a required pointer is NULL                          */
#define DSA_ERR_ALIGN (-2)     /* a pointer is not 16-byte aligned, or ld % 4 != 0    */
#define DSA_ERR_DIMS (-3)      /* unsupported or inconsistent shape, or flags != 0     */
#define DSA_ERR_CAUSAL (-4)    /* q_pos0 + n_q > ctx_len                               */
#define DSA_ERR_WORKSPACE (-5) /* workspace NULL or smaller than dsa_workspace_size()  */
#define DSA_ERR_TIMEOUT (-6)   /* a device-side bounded wait gave up                   */
#define DSA_ERR_CUDA (-7)      /* CUDA runtime or launch error                         */
#define DSA_ERR_DEVICE (-8)    /* current device is not sm_100 (B200)                  */
#define DSA_ERR_RANGE (-9)     /* device found a selected index outside 0..t           */
#define DSA_ERR_SCRATCH_LIMIT (-10) /* dsa_prefill_layer_noalloc: the chunk needs more
                                       scratch than DSA_NOALLOC_SCRATCH_BYTES             */
#define DSA_ERR_LAYOUT (-11)   /* dsa_selftest_mma_layout: a tensor-core product differed */

/* Which call a workspace is for. */
#define DSA_WS_INDEX_SCORES 0
#define DSA_WS_TOPK 1
#define DSA_WS_ATTN 2
#define DSA_WS_LAYER 3
#define DSA_WS_DECODE_ATTN 4
#define DSA_WS_DECODE_LAYER 5
#define DSA_WS_BLOCK_ATTN 6

/* Bytes of device workspace the call `which` needs for these dims (0 on bad
 * arguments). The first 256 bytes of every workspace hold the device status
 * word and per-call scalars; dsa_prefill_layer adds the float32 score matrix
 * [n_q, round_up(ctx_len, 128)] and an int32 selection [n_q, top_k] after
 * them. When the chunk's last query sees more than 49,152 keys
 * (q_pos0 + n_q > 49152) the top-k selects in two passes -- the top_k of
 * each of n_seg = ceil((q_pos0 + n_q) / 32768) key segments, then the top_k
 * of those candidates -- and dsa_topk_select and the layer calls add an
 * int32 candidate buffer [n_q, n_seg, top_k]. Workspace contents need no
 * initialisation and are not preserved between calls. */
size_t dsa_workspace_size(const dsa_dims* dims, int32_t which);

/* Lightning-indexer scores (component-table row "DSA indexer" of the feedman.me
 * post). For query row i at position t and cache row s <= t:
 *     I[i,s] = sum_j w_idx[i,j] * ReLU( sum_c q_idx[i,j,c] * k_idx[s,c] )
 * computed with bf16 products, float32 accumulation on tensor cores and a
 * float32 head sum.
 *   q_idx   bf16  [n_q, n_idx_heads, d_idx]
 *   k_idx   bf16  [ctx_len, d_idx]        one key per cache row, shared by heads
 *   w_idx   f32   [n_q, n_idx_heads]
 *   scores  f32   [n_q, ld_scores], ld_scores >= ctx_len, ld_scores % 4 == 0.
 *           Row i holds I[i,s] for s <= t; entries s > t are not written.
 * Errors: DSA_ERR_NULL, _ALIGN, _DIMS, _CAUSAL, _WORKSPACE, _DEVICE, _CUDA. */
dsa_status dsa_index_scores(const dsa_dims* dims, const uint16_t* q_idx, const uint16_t* k_idx,
                            const float* w_idx, float* scores, int64_t ld_scores,
                            void* workspace, size_t workspace_bytes, void* stream);

/* FP8 (e4m3) form of bf16 rows for the FP8 indexer (an 8-bit form of the
 * "DSA indexer" row of the feedman.me post's component table; the pages
 * describe no FP8 indexer, these are this library's rules). For each of the
 * `rows` rows of `cols` (1..128) values:
 *   scale[r] = the smallest power of two s with max_c |x[r,c]| <= 448 s
 *              (1 for an all-zero row; 448 is the largest finite e4m3 value);
 *   x8[r,c]  = x[r,c] / s rounded to the nearest e4m3 value, ties to even
 *              (the bit pattern; the sign of a zero is kept);
 *   xhat[r,c]= x8[r,c] * s as bf16 (exact).
 *   x     bf16 [rows, cols]     x8    uint8 [rows, cols]
 *   scale f32  [rows]           xhat  bf16  [rows, cols]
 * Indexer rows are k_idx [ctx_len, d_idx] and q_idx [n_q * n_idx_heads,
 * d_idx]. Errors: DSA_ERR_DIMS, _NULL, _ALIGN, _DEVICE, _CUDA. */
dsa_status dsa_quantize_fp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* x8,
                            float* scale, uint16_t* xhat, void* stream);

/* Lightning-indexer scores from e4m3 operands (tensor cores, kind::f8f6f4,
 * float32 accumulation): for s <= t,
 *     I[i,s] = s_k[s] * sum_j w_idx[i,j] * s_q[i,j] * ReLU( sum_c q8[i,j,c] * k8[s,c] )
 * which is the score of dsa_index_scores on the dequantized rows (xhat) up to
 * float32 rounding, within the same error bound, so dsa_topk_select given the
 * dequantized rows orders these scores exactly.
 *   q8 uint8 [n_q, n_idx_heads, d_idx], q_scale f32 [n_q, n_idx_heads],
 *   k8 uint8 [ctx_len, d_idx], k_scale f32 [ctx_len] (from dsa_quantize_fp8);
 *   w_idx, scores, ld_scores and the workspace as in dsa_index_scores.
 * Errors: those of dsa_index_scores. */
dsa_status dsa_index_scores_fp8(const dsa_dims* dims, const uint8_t* q8, const float* q_scale,
                                const uint8_t* k8, const float* k_scale, const float* w_idx,
                                float* scores, int64_t ld_scores, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Per-query top-k selection (the "per-query top-2048" step of the feedman.me
 * post, paragraph after the component table). Among s = 0..t, keys are
 * ordered by score descending and then index ascending; the first
 * min(top_k, t+1) are kept and written in ascending index order, the unused
 * tail of the row holding -1.
 *   scores  f32   [n_q, ld_scores] as written by dsa_index_scores (only
 *                 entries s <= t are read)
 *   idx     int32 [n_q, top_k] (output)
 * With q_idx, k_idx and w_idx all NULL the order is that of the given float32
 * scores. With all three given, the order is that of the float64 definition
 *     d_j = sum_c q*k (float64, in c order), r_j = max(d_j, +0),
 *     score = sum_j w_j * r_j (float64, in j order, no fused multiply-add)
 * which the kernel reproduces exactly: float32 scores within a proven error
 * bound decide every key except those whose bound straddles the k-th score,
 * and those are re-scored in float64 in that order. Giving only some of the
 * three is DSA_ERR_NULL.
 * Errors: DSA_ERR_NULL, _ALIGN, _DIMS, _CAUSAL, _WORKSPACE, _DEVICE, _CUDA. */
dsa_status dsa_topk_select(const dsa_dims* dims, const float* scores, int64_t ld_scores,
                           const uint16_t* q_idx, const uint16_t* k_idx, const float* w_idx,
                           int32_t* idx, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Sparse MLA-style attention over the selected keys (component-table row "DSA
 * sparse-attention core" of the feedman.me post). For query row i, head h and
 * the keys S listed in idx[i,:] (entries < 0 are skipped):
 *     z_s = softmax_scale * ( q[i,h,:Dc] . latent[s,:] + q[i,h,Dc:] . rope[s,:] )
 *     out[i,h,:] = sum_{s in S} softmax(z)_s * latent[s,:]
 *     lse[i,h]   = log sum_{s in S} exp(z_s)
 * bf16 operands, float32 accumulation, bf16 output rounded to nearest even.
 * A row with no valid key gets out = 0 and lse = -inf.
 *   q      bf16  [n_q, n_heads, d_latent + d_rope]
 *   latent bf16  [ctx_len, d_latent]
 *   rope   bf16  [ctx_len, d_rope]
 *   idx    int32 [n_q, top_k], every valid entry of row i in 0..t, t = q_pos0 + i
 *          (the keys a causal query may see)
 *   out    bf16  [n_q, n_heads, d_latent] (output)
 *   lse    f32   [n_q, n_heads] (output) or NULL
 * An index past t (a future token, or past the cache) is not read; it sets
 * DSA_ERR_RANGE in the workspace status and that key is skipped.
 * Errors: DSA_ERR_NULL, _ALIGN, _DIMS, _CAUSAL, _WORKSPACE, _DEVICE, _CUDA. */
dsa_status dsa_sparse_attn_prefill(const dsa_dims* dims, const uint16_t* q,
                                   const uint16_t* latent, const uint16_t* rope,
                                   const int32_t* idx, uint16_t* out, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* The whole layer on one stream: indexer scores -> exact top-k (float64
 * order, as in dsa_topk_select with the indexer inputs given) -> sparse
 * attention. idx_out ([n_q, top_k]) and lse may be NULL. The float32 score
 * matrix lives in the workspace. */
dsa_status dsa_prefill_layer(const dsa_dims* dims, const uint16_t* q, const uint16_t* latent,
                             const uint16_t* rope, const uint16_t* q_idx,
                             const uint16_t* k_idx, const float* w_idx, uint16_t* out,
                             float* lse, int32_t* idx_out, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Decode-side attention: dsa_sparse_attn_prefill for chunks of few queries (a
 * decode step is n_q = 1). The per-query kernel runs one query per SM, so a
 * chunk smaller than the GPU would leave most SMs idle; here each query's
 * selected keys are cut into up to ceil(top_k / 128) ranges of 128-key tiles
 * (n_split = min(ceil(top_k / 128), SMs / n_q), at least 1) that run on
 * different SMs, each writing its unnormalised partial output, reference
 * maximum and row sum to the workspace; a combine pass then merges them
 * (flash-decoding style: out = sum_j 2^(m_j - M) O_j / sum_j 2^(m_j - M) l_j).
 * Same definition, arguments, layouts and errors as dsa_sparse_attn_prefill,
 * with a workspace of dsa_workspace_size(dims, DSA_WS_DECODE_ATTN) bytes.
 * Results agree with dsa_sparse_attn_prefill within rounding (the sums are
 * grouped differently), and depend on n_q through n_split. The feedman.me
 * post profiles prefill only; this call is the decode side of the same
 * layer (its component table lists decode throughput for the same model). */
dsa_status dsa_sparse_attn_decode(const dsa_dims* dims, const uint16_t* q,
                                  const uint16_t* latent, const uint16_t* rope,
                                  const int32_t* idx, uint16_t* out, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* The whole layer for a decode step (few queries): dsa_prefill_layer with the
 * attention of dsa_sparse_attn_decode. The indexer spreads a small chunk's key
 * tiles over all SMs in either call. Workspace: dsa_workspace_size(dims,
 * DSA_WS_DECODE_LAYER) bytes. Selections are those of dsa_prefill_layer (bit
 * for bit); outputs agree with it within rounding. */
dsa_status dsa_decode_layer(const dsa_dims* dims, const uint16_t* q, const uint16_t* latent,
                            const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                            const float* w_idx, uint16_t* out, float* lse, int32_t* idx_out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Block-sparse attention (the feedman.me post's proposed fix, paragraph "Two
 * levers fell out of this": share gathered keys across neighbouring queries
 * and use the matrix units). Queries are taken in groups of block_queries
 * (1 or 2) neighbours; each group gathers the union of its queries' selected
 * keys once, in ascending key order, and runs QK^T and PV for all of the
 * group's heads on it, a key outside a query's own selection being masked
 * (p = 0) for that query. Same definition, arguments, layouts and errors as
 * dsa_sparse_attn_prefill, with each valid key listed at most once per idx
 * row (as every selection is); entries past t are reported as DSA_ERR_RANGE
 * and skipped. Workspace: dsa_workspace_size(dims, DSA_WS_BLOCK_ATTN) bytes
 * (the union lists and masks). block_queries = 1 runs the same kernel per
 * query. This kernel runs its steps one after another (a tile of the union
 * and the group's q rows fill shared memory); dsa_sparse_attn_prefill, which
 * pipelines the gather under the tensor-core work, is the faster path on the
 * measured workloads, and this call exists to measure the union against it.
 * Errors: those of dsa_sparse_attn_prefill, DSA_ERR_DIMS for block_queries
 * outside 1..DSA_MAX_BLOCK_QUERIES. */
#define DSA_MAX_BLOCK_QUERIES 2
dsa_status dsa_sparse_attn_block(const dsa_dims* dims, const uint16_t* q, const uint16_t* latent,
                                 const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                 float* lse, int32_t block_queries, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Device copies of the layer's tensors for dsa_prefill_layer_host, owned by
 * the caller, each of the full size given under dsa_prefill_layer and 16-byte
 * aligned. lse and idx may be NULL when the matching host output is NULL. */
typedef struct {
  uint16_t* q;
  uint16_t* latent;
  uint16_t* rope;
  uint16_t* q_idx;
  uint16_t* k_idx;
  float* w_idx;
  uint16_t* out;
  float* lse;
  int32_t* idx;
} dsa_device_tensors;

/* The whole layer on host buffers, with the host<->device copies overlapped
 * with the compute. Query rows are independent given the cache, so the chunk
 * is cut into n_sub consecutive sub-chunks of ceil(n_q / n_sub) rows. The call
 * enqueues:
 *   streams[0]: the cache (latent, rope, k_idx) into dev, then each
 *               sub-chunk's q, q_idx and w_idx rows;
 *   streams[1]: dsa_prefill_layer on each sub-chunk once its rows are in
 *               (the workspace is shared by the sub-chunks, in order);
 *   streams[2]: each sub-chunk's out (and lse, idx when given) back to the
 *               host once its layer is done;
 * so the copy-in of sub-chunk s+1, the layer on s and the copy-out of s-1 run
 * together. events[0..1] are the caller's CUDA events (timing may be
 * disabled) that the call records and waits on; streams and events are
 * passed as cudaStream_t / cudaEvent_t cast to void*.
 * Host inputs and outputs are the tensors of dsa_prefill_layer in host
 * memory; page-locked memory is needed for the copies to run asynchronously.
 * The outputs are complete once streams[2] has finished the work this call
 * enqueued; the device status of the layer calls is read with
 * dsa_device_status(workspace, streams[1]). Results are bit-identical to one
 * dsa_prefill_layer call on the whole chunk. Unless dims.flags holds
 * DSA_FLAG_HOST_UNORDERED, the call first orders its copies after the layers
 * and its layers after the copy-outs that earlier calls left on the streams,
 * so that back-to-back calls on the same device tensors never overwrite a
 * buffer still in use.
 * Errors: those of dsa_prefill_layer, DSA_ERR_NULL for a missing stream,
 * event or device tensor, DSA_ERR_DIMS for n_sub < 1. */
dsa_status dsa_prefill_layer_host(const dsa_dims* dims, const uint16_t* q, const uint16_t* latent,
                                  const uint16_t* rope, const uint16_t* q_idx,
                                  const uint16_t* k_idx, const float* w_idx, uint16_t* out,
                                  float* lse, int32_t* idx_out, const dsa_device_tensors* dev,
                                  void* workspace, size_t workspace_bytes, void* const streams[3],
                                  void* const events[2], int32_t n_sub);

/* The whole layer, as dsa_prefill_layer, for callers that cannot allocate
 * device memory: code that runs inside another engine's plugin or callback and
 * is handed only its input and output buffers, or code that must not touch the
 * device allocator while a memory pool is shared or being captured. The pages
 * have no counterpart to this call; it exists for such callers only.
 *
 * The scratch (score rows, selections, status word) lives in a static device
 * array of DSA_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU which loads the
 * library holds until the process exits. The call allocates nothing:
 *  - chunks whose dsa_workspace_size(dims, DSA_WS_LAYER), i.e.
 *        256 + n_q * (round_up(ctx_len, 128) + top_k) * 4 bytes,
 *    exceeds DSA_NOALLOC_SCRATCH_BYTES return DSA_ERR_SCRATCH_LIMIT (e.g.
 *    1,024 queries at top_k 2048 fit up to a 6,016-token context; split larger
 *    chunks). The selection region counts even when idx_out is given;
 *  - the first call on each device looks up the array's device address with
 *    that device current, and so does the first call after the device's
 *    context was destroyed and created anew (cudaDeviceReset, or the primary
 *    context released and retained again); make those calls before any stream
 *    capture;
 *  - all calls on a device share the array, and it keeps the last call's
 *    contents: calls that overlap on the GPU (other streams, other threads)
 *    race on it. Each call clears the status word and scalars it relies on.
 * device_status (device memory, 4-byte aligned, may be NULL) receives this
 * call's device status word, asynchronously on `stream`: 0 on success,
 * 1 a bounded device wait gave up, 2 an index was out of range, 3 an internal
 * consistency check failed.
 * Other arguments and errors are those of dsa_prefill_layer. */
#define DSA_NOALLOC_SCRATCH_BYTES (32u << 20)
dsa_status dsa_prefill_layer_noalloc(const dsa_dims* dims, const uint16_t* q,
                                     const uint16_t* latent, const uint16_t* rope,
                                     const uint16_t* q_idx, const uint16_t* k_idx,
                                     const float* w_idx, uint16_t* out, float* lse,
                                     int32_t* idx_out, uint32_t* device_status, void* stream);

/* Multi-GPU prefill of one chunk: splits its queries into n_parts contiguous
 * ranges, one per rank, with nearly equal useful work. Row i (position t)
 * costs (t+1) * 2 * n_idx_heads * d_idx multiply-adds in the indexer and
 * min(top_k, t+1) * 2 * n_heads * (2 d_latent + d_rope) in the attention, so
 * later rows are dearer and equal row counts would overload the last rank.
 * Part p takes rows starts[p] .. starts[p+1]-1; rank p then calls
 * dsa_prefill_layer with n_q = starts[p+1] - starts[p], q_pos0 advanced by
 * starts[p] and its row slices of q, q_idx, w_idx, out, lse and idx, against
 * the whole cache. Boundaries are multiples of the smallest row count that
 * keeps every per-row tensor offset 16-byte aligned (1 for the 32-head shapes
 * at a top_k that is a multiple of 4, at most 8); a part may be empty.
 *   starts  host int32 [n_parts + 1] (output), starts[0] = 0, starts[n_parts] = n_q
 * Host arithmetic only: no device is touched and nothing is allocated on one.
 * Errors: DSA_ERR_NULL, _DIMS (n_parts < 1 or a nonpositive size), _CAUSAL. */
dsa_status dsa_partition_queries(const dsa_dims* dims, int32_t n_parts, int32_t* starts);

/* Self-test of the failure path every kernel of the library shares: each
 * device wait is bounded, and a wait that gives up records DSA_ERR_TIMEOUT
 * (with the failing site) in the workspace status and makes the CTA's other
 * waits give up too, so the CTA exits and the context stays usable. This
 * launches one CTA of two warps that wait on barriers nothing ever signals:
 * warp 0 with a limit of about 0.5 ms, warp 1 with the kernels' own limit
 * (about one second), which it can only beat by following warp 0's abort.
 * No memory outside the workspace header and `cycles` is touched.
 *   workspace  >= dsa_workspace_size(any dims, DSA_WS_ATTN) bytes; its header
 *              is cleared first, then receives the timeout
 *   cycles     device int64 [2] (may be NULL): each warp's wait in SM clock
 *              cycles
 * Read the outcome with dsa_device_status(workspace, stream), which returns
 * DSA_ERR_TIMEOUT. Errors: DSA_ERR_WORKSPACE, _ALIGN, _DEVICE, _CUDA. */
dsa_status dsa_selftest_bounded_wait(void* workspace, size_t workspace_bytes, int64_t* cycles,
                                     void* stream);

/* Start-up self-test of the tensor-core operand layouts the kernels use (the
 * TensorFold issue #743 page, "Pre-M5 kernel checks": a load-time check of the
 * matrix-fragment layout that a transposed operand got through). One CTA
 * multiplies small-integer matrices that are not symmetric, each laid out in
 * shared memory as the kernels' own copies lay it out and multiplied with the
 * kernels' descriptor conventions, and compares every accumulator element
 * with a sum of the same integers on the CUDA cores; both are exact in
 * float32, so any difference means a transposed operand or a wrong swizzle,
 * stride, descriptor field or tensor-memory mapping. Forms, in order:
 *   0 the indexer's bf16 MMA (M 128, N 256, K 128, K-major, 128-byte swizzle)
 *   1 the attention's QK^T (M 128 keys, N 32 heads, K-major)
 *   2 the attention's PV (latent pair read MN-major, P in 64-byte swizzled
 *     rows, N 32)
 *   3 the FP8 indexer's e4m3 MMA (kind::f8f6f4, M 128, N 256, K 128)
 *   workspace   >= 288 bytes (16-byte aligned); its header is cleared first;
 *               bytes 256..271 receive the four counts and 272..287 the four
 *               timings on the device
 *   mismatches  host int32 [4] (may be NULL): wrong accumulator elements of
 *               each form (all 0 when the layouts hold; -1 when an MMA did
 *               not complete within the kernels' wait limit)
 *   cycles_per_mma  host float [4] (may be NULL): each form's MMAs issued 32
 *               times back to back on one SM, SM clock cycles per MMA from
 *               the first issue to the last completion (-1 as above)
 * When either host array is given, the call synchronizes `stream` and copies
 * the results back.
 * A wrong element also records DSA_ERR_LAYOUT (site = the first bad form) in
 * the workspace status, read by dsa_device_status. Run it once per device
 * before the first layer call. Errors: DSA_ERR_WORKSPACE, _ALIGN, _DEVICE,
 * _CUDA. */
dsa_status dsa_selftest_mma_layout(void* workspace, size_t workspace_bytes, int32_t* mismatches,
                                   float* cycles_per_mma, void* stream);

/* Synchronizes `stream`, returns the device status word of `workspace`
 * (DSA_OK, DSA_ERR_TIMEOUT, DSA_ERR_RANGE or DSA_ERR_LAYOUT) and clears it. */
dsa_status dsa_device_status(void* workspace, void* stream);

/* Static text for a status code. */
const char* dsa_status_string(dsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
