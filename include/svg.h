/*
 * svg.h -- C ABI of libsvg, a B200 (sm_100a) implementation of the hot path of
 * Sparse VideoGen (SVG 1) spatial/temporal sparse 3D attention.
 *
 * Source of the method: "Sparse VideoGen: Accelerating Video Diffusion
 * Transformers with Spatial-Temporal Sparsity" (arXiv 2502.01776), abstract:
 * attention heads of a video diffusion transformer are classified online as
 * spatial heads (output dominated by tokens of the query's own and nearby
 * frames) or temporal heads (dominated by tokens at the same in-frame position
 * across frames); a hardware-efficient tensor layout transformation and
 * customised kernels turn either pattern into contiguous block-sparse work.
 * The project article "Sparse-VideoGen and the sparsity hiding inside video
 * diffusion attention" (section "Three generations of the same idea", and the
 * install section on block sparse attention with varied block sizes) restates
 * the same pieces. The pages fix no interface; this one is derived from that
 * description.
 *
 * Conventions shared by every call
 * --------------------------------
 *  Tensors   Q, K, V, O are [B, H, N, d] bf16 (raw bit patterns, svg_bf16),
 *            contiguous, base address 16-byte aligned, N = T*P + n_text.
 *            Video token (frame f, position p) is row f*P + p in frame-major
 *            order and row p*T + f in position-major order; the n_text text
 *            tokens follow the video tokens in both orders and are global.
 *  Memory    All pointers marked "device" are caller-owned device memory; the
 *            library allocates no device memory and frees nothing. Each
 *            attention/profiling CTA allocates and frees its own tensor memory.
 *  Streams   Every call that takes a stream enqueues its work on that stream
 *            (a cudaStream_t passed as void*; NULL = legacy default stream)
 *            and returns without synchronising.
 *  Errors    Every call returns an svg_status. Arguments are validated on the
 *            host before anything is launched; on any error nothing is
 *            launched and outputs are untouched. Nothing aborts, traps or
 *            prints. Device-side waits are bounded: one that runs out sets a
 *            status bit read by svg_get_device_status.
 *  Devices   The current CUDA device at call time must be an sm_100 GPU
 *            (SVG_ERR_UNSUPPORTED otherwise).
 */
#ifndef SVG_H_
#define SVG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svg_status {
  SVG_OK = 0,
  SVG_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned tensor, bad kind */
  SVG_ERR_UNSUPPORTED = 2,   /* head_dim not in {64,128}, block size not in {64,128},
                                not an sm_100 device */
  SVG_ERR_CAPACITY = 3,      /* caller buffer too small (col_capacity, workspace) */
  SVG_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  SVG_ERR_DEVICE_TIMEOUT = 5 /* a device-side bounded wait ran out (see svg_get_device_status) */
} svg_status;

/* Head labels (one int8 per (b, h), index b*H + h). */
enum { SVG_HEAD_SPATIAL = 0, SVG_HEAD_TEMPORAL = 1 };

/* Block-mask kinds. SPATIAL lives in frame-major order, TEMPORAL in
 * position-major order, DENSE (all blocks) in either. */
enum { SVG_MASK_SPATIAL = 0, SVG_MASK_TEMPORAL = 1, SVG_MASK_DENSE = 2 };

typedef uint16_t svg_bf16; /* raw bf16 bits */
typedef void* svg_stream_t; /* a cudaStream_t */

/* Geometry of one attention layer. */
typedef struct svg_geom {
  int32_t B, H;            /* batch, heads (>= 1) */
  int32_t T, P;            /* frames, tokens per frame (>= 1) */
  int32_t n_text;          /* text tokens after the T*P video tokens (>= 0) */
  int32_t head_dim;        /* d: 64 or 128 */
  int32_t block_q;         /* query block rows of the block mask: 64 or 128 */
  int32_t block_k;         /* key block columns of the block mask: 64 or 128 */
  int32_t spatial_band;    /* s >= 0: spatial mask keeps key frames with |f(i)-f(j)| <= s */
  int32_t temporal_width;  /* w >= 0: temporal mask keeps in-frame positions |p(i)-p(j)| <= w */
  float scale;             /* softmax scale applied to q.k (normally 1/sqrt(d)); finite, > 0 */
} svg_geom;

/* ---------------------------------------------------------------------------
 * svg_mask_nnz -- host only, exact.
 * Number of (query block, key block) pairs of the block mask `kind` (the
 * length col_idx must have for svg_build_block_mask). Block (r, c) is on iff
 * some token pair of the block pair is allowed by the token mask in the
 * pattern's layout (SVG abstract: spatial heads attend within nearby frames,
 * temporal heads across frames at nearby positions; text tokens are global).
 *   nnz  out, host pointer.
 * Errors: INVALID_ARG (null, bad geometry, bad kind).
 */
svg_status svg_mask_nnz(const svg_geom* geom, int32_t kind, int64_t* nnz);

/* ---------------------------------------------------------------------------
 * svg_build_block_mask -- the block mask of `kind` as CSR.
 *   row_ptr   device int32 [nQB + 1], nQB = ceil(N / block_q); row_ptr[0] = 0.
 *   col_idx   device int32 [col_capacity]; key-block indices of each row,
 *             ascending; nnz = row_ptr[nQB] = svg_mask_nnz(...).
 * Built in closed form: a query block's video tokens span an integer interval
 * of frames (spatial) or positions (temporal), so each row is one contiguous
 * run of key blocks plus the text key blocks. Depends only on the geometry;
 * callers build it once and reuse it across layers and steps.
 * Errors: INVALID_ARG, CAPACITY (col_capacity < nnz), CUDA.
 */
svg_status svg_build_block_mask(const svg_geom* geom, int32_t kind, int32_t* row_ptr,
                                int32_t* col_idx, int64_t col_capacity, svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_profile_workspace_bytes -- host only: device workspace svg_profile_heads
 * needs for n_samples sampled rows: the per-tile partial sums of the MSE
 * reduction and, when each (head, tile of 128 sampled rows) is split over up
 * to 4 key ranges to fill a B200's 148 SMs, the unnormalised fp32 partial
 * outputs and (base, sum) pairs of every split (B*H*tiles*splits*3*(d+2)*128
 * floats). Depends only on the geometry and n_samples.
 */
svg_status svg_profile_workspace_bytes(const svg_geom* geom, int32_t n_samples, size_t* bytes);

/* ---------------------------------------------------------------------------
 * svg_profile_heads -- online profiling (SVG abstract: "online profiling
 * strategy to capture the dynamic sparse patterns and predict the type of
 * attention head").
 * For every (b, h) and every sampled query row i, computes full attention,
 * spatial-masked attention (|f(i)-f(j)| <= s, text global) and
 * temporal-masked attention (|p(i)-p(j)| <= w, text global), all token-level
 * in frame-major order, then
 *   mse_X = mean over rows x channels of (O_X - O_full)^2,
 *   label = SVG_HEAD_TEMPORAL iff mse_temporal < mse_spatial (tie: spatial).
 *   q, k, v      device bf16 [B, H, N, d], frame-major.
 *   sample_idx   device int32 [n_samples], distinct video rows in [0, T*P);
 *                the same rows serve every (b, h).
 *   labels       device int8 [B*H], out.
 *   mse          device float [B*H*2] out ({spatial, temporal} per head), or NULL.
 *   workspace    device, >= svg_profile_workspace_bytes(...), 256-byte aligned.
 * Deterministic for a given geometry and n_samples: fixed-order reductions,
 * no atomics in the arithmetic.
 * Errors: INVALID_ARG, UNSUPPORTED, CAPACITY (workspace too small), CUDA.
 * A sample index outside [0, T*P) sets the device bounds bit (row skipped).
 */
svg_status svg_profile_heads(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                             const svg_bf16* v, const int32_t* sample_idx, int32_t n_samples,
                             int8_t* labels, float* mse, void* workspace,
                             size_t workspace_bytes, svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_profile_heads_noalloc -- svg_profile_heads without a caller workspace.
 * No counterpart on the pages: this is an interface convenience, not part of
 * the method. Some callers cannot allocate device memory when they call the
 * library: a plugin inside an inference engine that plans every buffer up
 * front and forbids allocation in its execute path, a latency-critical loop
 * that cannot afford cudaMalloc's implicit device synchronisation, or code
 * that simply has no allocator at hand. This entry point takes the same
 * arguments as svg_profile_heads minus the workspace and keeps the MSE
 * partial sums in a fixed array inside the library instead; it calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   Limit      the partial sums need B*H*2*ceil(n_samples/128)*4 bytes (one
 *              key range per tile of 128 sampled rows: unlike
 *              svg_profile_heads it never splits the key range); more than
 *              256 KiB (that is, B*H*ceil(n_samples/128) > 32768) returns
 *              SVG_ERR_CAPACITY before anything is launched.
 *   Results    the same labels as svg_profile_heads; the MSE values agree up
 *              to the rounding of the summation order when svg_profile_heads
 *              splits the key ranges.
 *   Memory     every GPU that loads the library holds the 256 KiB array
 *              until the process exits.
 *   Set-up     the first call on a device looks up that device's copy of
 *              the array (cudaGetSymbolAddress) with the device current;
 *              make that first call before any stream capture. A device
 *              reset (cudaDeviceReset) loads the library's device code again
 *              at another address: the next call notices the new context and
 *              looks the address up again, so after a reset, too, make one
 *              call before any stream capture.
 *   Sharing    all calls share the one array and it keeps the last call's
 *              contents (every slot is written before it is read, so no
 *              clearing is needed); calls that overlap on the GPU (e.g. on
 *              two streams) race and must be serialised by the caller.
 * Errors: as svg_profile_heads (CAPACITY as above).
 */
svg_status svg_profile_heads_noalloc(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                     const svg_bf16* v, const int32_t* sample_idx,
                                     int32_t n_samples, int8_t* labels, float* mse,
                                     svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_permute / svg_unpermute -- the layout transformation (SVG abstract:
 * "hardware-efficient tensor layout transformation").
 *   permute:    out[b,h,pi(i),:] = in[b,h,i,:]   (frame-major -> position-major)
 *   unpermute:  out[b,h,i,:]     = in[b,h,pi(i),:]
 * with pi(f*P + p) = p*T + f for video rows and pi(i) = i for text rows.
 *   in, out   device bf16 [B, H, N, d]; must not overlap.
 *   labels    device int8 [B*H]: only heads labelled SVG_HEAD_TEMPORAL are
 *             written (others untouched); NULL = every head.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
svg_status svg_permute(const svg_geom* geom, const svg_bf16* in, svg_bf16* out,
                       const int8_t* labels, svg_stream_t stream);
svg_status svg_unpermute(const svg_geom* geom, const svg_bf16* in, svg_bf16* out,
                         const int8_t* labels, svg_stream_t stream);

/* svg_permute_qkv -- svg_permute of Q, K and V in one launch. q and qp may
 * both be NULL: then only K and V are permuted (the input of
 * svg_sparse_attention_fused with position-major K/V copies). */
svg_status svg_permute_qkv(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                           const svg_bf16* v, svg_bf16* qp, svg_bf16* kp, svg_bf16* vp,
                           const int8_t* labels, svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_sparse_attention -- block-sparse flash attention over per-head block
 * masks (SVG abstract: "customized kernel implementations"; the project
 * article's block sparse attention).
 * Head (b, h) with label l works in layout L(l): frame-major for spatial
 * heads (reads q, k, v; CSR row_ptr_s/col_idx_s; writes o), position-major
 * for temporal heads (reads qp, kp, vp; CSR row_ptr_t/col_idx_t; writes op).
 * For each query row i of the head:
 *   O[i] = sum_{j < N, BM[i/block_q][j/block_k] = 1} softmax_j(scale * q_i.k_j) v_j
 * (block-granular: every token pair of a listed block pair is attended),
 * accumulated in fp32, rounded to bf16. Rows whose CSR row is empty get O = 0.
 *   q,k,v,o        device bf16 [B,H,N,d] (frame-major).
 *   qp,kp,vp,op    device bf16 [B,H,N,d] (position-major); may be NULL when
 *                  labels is NULL or no head is temporal (then a temporal
 *                  label sets the device bounds bit and the head is skipped).
 *   labels         device int8 [B*H]; NULL = every head spatial.
 *   row_ptr_*, col_idx_*  device CSR as built by svg_build_block_mask (any CSR
 *                  with ascending, in-range column indices is accepted;
 *                  out-of-range indices set the bounds bit and are skipped).
 *                  The temporal CSR may be NULL when labels is NULL.
 *   lse            device float [B,H,N] out (natural-log sum of exp of the
 *                  scaled logits over attended keys, in the head's layout;
 *                  -inf for empty rows), or NULL.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
svg_status svg_sparse_attention(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                const svg_bf16* v, const svg_bf16* qp, const svg_bf16* kp,
                                const svg_bf16* vp, const int8_t* labels,
                                const int32_t* row_ptr_s, const int32_t* col_idx_s,
                                const int32_t* row_ptr_t, const int32_t* col_idx_t,
                                svg_bf16* o, svg_bf16* op, float* lse, svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_sparse_attention_fused -- svg_sparse_attention with the layout
 * transformation folded into the attention kernel (SVG abstract: the
 * "hardware-efficient tensor layout transformation"): no permuted copy of Q
 * or O is written, and optionally none of K and V either.
 * Every head reads q in frame-major order. A head labelled temporal still
 * attends in position-major order over the temporal CSR: its query tiles are
 * assembled row by row in that order (TMA tile::gather4 row gathers,
 * frame-major row pi^-1(j) for position-major row j) and each output row is
 * stored at its frame-major place. Its key/value tiles come either from
 * position-major copies kp, vp (plain tiled loads) or, with kp = vp = NULL,
 * are gathered row by row from k, v like the queries (no copy at all, but
 * row gathers move far fewer bytes per cycle than tiled loads, so this form is
 * slower on long key lists). The result equals
 *   svg_permute_qkv -> svg_sparse_attention -> svg_unpermute
 * bit for bit (same arithmetic in the same order), with lse, if given, also
 * in frame-major rows.
 *   q,k,v,o        device bf16 [B,H,N,d], frame-major, every head.
 *   kp,vp          device bf16 [B,H,N,d], position-major copies of k and v
 *                  for the temporal heads (svg_permute_qkv with q = qp =
 *                  NULL), or both NULL.
 *   labels         device int8 [B*H] (required).
 *   row_ptr_s, col_idx_s, row_ptr_t, col_idx_t  device CSR of both masks
 *                  (required), as for svg_sparse_attention.
 *   lse            device float [B,H,N] out (frame-major rows) or NULL.
 * Errors: INVALID_ARG (NULL or misaligned pointer, only one of kp/vp, bad
 *   geometry),
 *   UNSUPPORTED (block_q != 128, B*H*N >= 2^31 rows, or a device where the
 *   paired-tile kernel cannot run), CUDA.
 */
svg_status svg_sparse_attention_fused(const svg_geom* geom, const svg_bf16* q,
                                      const svg_bf16* k, const svg_bf16* v,
                                      const svg_bf16* kp, const svg_bf16* vp,
                                      const int8_t* labels, const int32_t* row_ptr_s,
                                      const int32_t* col_idx_s, const int32_t* row_ptr_t,
                                      const int32_t* col_idx_t, svg_bf16* o, float* lse,
                                      svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_quantize_v_e4m3 -- V for the FP8 PV product of
 * svg_sparse_attention_fp8pv. The project article "Sparse-VideoGen and the
 * sparsity hiding inside video diffusion attention" (section "Publication
 * record and the road ahead") lists FP8 attention as open; the pages fix no
 * scheme, so this one is stated here. One scale per (b, h, channel):
 *   amax_c     = max over the head's N rows of |v[b,h,j,c]|,
 *   v8[b,h,j,c] = e4m3(v[b,h,j,c] * (448 / amax_c))  (fp32 product, round to
 *                nearest even, saturating; E4M3 "fn": bias 7, max 448),
 *   v_scale[b,h,c] = amax_c / 448, so v ~= v8 * v_scale
 * (an all-zero channel gets scale 0 and codes 0). Each head is read in the
 * layout it attends in: from v (frame-major) when labelled spatial or when
 * labels is NULL, from vp (position-major) when labelled temporal.
 *   v, vp      device bf16 [B,H,N,128]; vp may be NULL when labels is NULL.
 *   labels     device int8 [B*H] or NULL.
 *   v8         device uint8 [B,H,N,128] out (e4m3 codes), 16-byte aligned.
 *   v_scale    device float [B*H*128] out.
 * Errors: INVALID_ARG, UNSUPPORTED (head_dim != 128), CUDA.
 */
svg_status svg_quantize_v_e4m3(const svg_geom* geom, const svg_bf16* v, const svg_bf16* vp,
                               const int8_t* labels, uint8_t* v8, float* v_scale,
                               svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_sparse_attention_fp8pv -- svg_sparse_attention with the PV product in
 * FP8 (tcgen05 kind::f8f6f4): the softmax probabilities are rounded to e4m3
 * (scaled by 2^6, which the row sum carries too, so it cancels) and multiplied
 * with the e4m3 V of svg_quantize_v_e4m3; the fp32 accumulator is scaled back
 * per channel by v_scale before the division by the row sum. Q K^T, the
 * softmax and the output stay as in svg_sparse_attention, so the result is the
 * same block-sparse attention up to e4m3 rounding of P and V (unit roundoff
 * 2^-4 each): a looser tolerance than the bf16 product's.
 *   q, k, qp, kp, labels, CSR, o, op, lse   as for svg_sparse_attention
 *                  (qp, kp, op NULL together when no head is temporal).
 *   v8, v_scale    from svg_quantize_v_e4m3 with the same labels (every head
 *                  in its own layout).
 * Errors: INVALID_ARG, UNSUPPORTED (head_dim != 128, block_q != 128, or a
 *   device where the paired-tile kernel cannot run), CUDA.
 */
svg_status svg_sparse_attention_fp8pv(const svg_geom* geom, const svg_bf16* q, const svg_bf16* k,
                                      const svg_bf16* qp, const svg_bf16* kp, const uint8_t* v8,
                                      const float* v_scale, const int8_t* labels,
                                      const int32_t* row_ptr_s, const int32_t* col_idx_s,
                                      const int32_t* row_ptr_t, const int32_t* col_idx_t,
                                      svg_bf16* o, svg_bf16* op, float* lse,
                                      svg_stream_t stream);

/* ===========================================================================
 * Semantic-aware permutation (Sparse VideoGen 2)
 * The project article "Sparse-VideoGen and the sparsity hiding inside video
 * diffusion attention", section "Three generations of the same idea": the
 * second generation clusters tokens by meaning (a batched, "flash" k-means),
 * permutes them so each cluster is contiguous, and runs a dynamic block-sparse
 * attention over the permuted layout; the install section names block sparse
 * attention with varied block sizes. The pages give no formula; the rules of
 * each call below are stated with it. Every tensor is per (b, h) = bh, heads
 * stacked: x [BH, N, d] bf16, centroids [BH, C, d] fp32, assign/order
 * [BH, N] int32, offsets [BH, C+1] int32. All device memory is the caller's.
 * ------------------------------------------------------------------------ */

/* svg2_kmeans_workspace_bytes -- host only: device workspace (256-byte
 * aligned) svg2_kmeans and svg2_kmeans_step need. Errors: INVALID_ARG,
 * UNSUPPORTED (d not 64/128; C not a multiple of 16 in [16, 256]). */
svg_status svg2_kmeans_workspace_bytes(int32_t BH, int32_t N, int32_t d, int32_t C,
                                       size_t* bytes);

/* svg2_kmeans -- Lloyd's k-means of every head's N rows of x (the query or the
 * key vectors of a layer) into C clusters, `iters` iterations:
 *   init        centroid c = row floor(c * N / C) of the head;
 *   assignment  every row to the centroid of least squared Euclidean distance,
 *               the centroids rounded to bf16 for the distance (a tcgen05
 *               product X C^T, fp32 accumulation), ties to the smaller index;
 *   update      each centroid = the fp32 mean of its members (an empty
 *               cluster keeps its centroid), summed in a fixed order: the
 *               sorted positions are cut into chunks of 256; the members in
 *               each chunk are added in order, then the chunks' sums in
 *               chunk order.
 * Outputs the final centroids, the last iteration's assignment (the one the
 * centroids are the means of) and its stable cluster order: order[bh, pos] =
 * row at sorted position pos (rows sorted by cluster, ties by row index),
 * offsets[bh, c] = first sorted position of cluster c, offsets[bh, C] = N.
 * With iters = 0: the initial centroids, their assignment and its order.
 * Deterministic (fixed-order sums, integer atomics only).
 * Errors: INVALID_ARG (null, misaligned: x and centroids 16-byte, workspace
 * 256-byte), UNSUPPORTED (d, C), CAPACITY (workspace), CUDA. */
svg_status svg2_kmeans(int32_t BH, int32_t N, int32_t d, int32_t C, int32_t iters,
                       const svg_bf16* x, float* centroids, int32_t* assign, int32_t* order,
                       int32_t* offsets, void* workspace, size_t workspace_bytes,
                       svg_stream_t stream);

/* svg2_kmeans_step -- one iteration of svg2_kmeans from given centroids:
 * assignment with centroids_in, its stable cluster order and offsets, and
 * centroids_out = the members' means (centroids_in for empty clusters).
 * centroids_out must not be centroids_in. Errors: as svg2_kmeans. */
svg_status svg2_kmeans_step(int32_t BH, int32_t N, int32_t d, int32_t C, const svg_bf16* x,
                            const float* centroids_in, float* centroids_out, int32_t* assign,
                            int32_t* order, int32_t* offsets, void* workspace,
                            size_t workspace_bytes, svg_stream_t stream);

/* svg2_select_clusters -- the key clusters each query cluster attends. For
 * query cluster a of head bh, key cluster b weighs
 *   w_b = softmax_b( scale * cq[bh,a] . ck[bh,b] + log |b| ),  |b| =
 *   offsets_k[bh,b+1] - offsets_k[bh,b]  (empty clusters weigh 0),
 * and a keeps the fewest clusters, taken in descending weight (ties to the
 * smaller index), whose weights add up to at least top_p (0 < top_p <= 1).
 * With disp != NULL (SVG-EAR's error-aware routing; the project article's
 * section "Three generations of the same idea": high-error blocks are computed
 * exactly, the rest compensated), a skipped cluster is kept as well when its
 * error estimate w_b * disp[bh, b] exceeds tau (disp from
 * svg2_cluster_value_stats: the spread of what its centroid would stand in for).
 *   cq [BH, Cq, d], ck [BH, Ck, d] fp32 centroids; offsets_k [BH, Ck+1].
 *   disp  fp32 [BH, Ck] or NULL; tau >= 0 (ignored when disp is NULL).
 *   sel   out, uint32 [BH, Cq, ceil(Ck/32)]: bit b%32 of word b/32 = kept.
 * fp32 arithmetic; a cluster whose preceding weight lies within rounding of
 * top_p (or whose estimate lies within rounding of tau) may go either way.
 * Errors: INVALID_ARG (Ck > 1024, bad scale/top_p/tau), CUDA. */
svg_status svg2_select_clusters(int32_t BH, int32_t d, int32_t Cq, int32_t Ck, float scale,
                                float top_p, const float* cq, const float* ck,
                                const int32_t* offsets_k, const float* disp, float tau,
                                uint32_t* sel, svg_stream_t stream);

/* svg2_cluster_value_stats -- SVG-EAR statistics of every key cluster, over
 * its members (summed in a fixed order: four consecutive runs of the
 * cluster's sorted members, each in order, then the four run sums in order):
 * vbar[bh, b] = the fp32 mean of their values,
 * disp[bh, b] = sqrt(mean over members and channels of (v - vbar)^2); an
 * empty cluster gets zeros. v bf16 [BH, N, d] (original order), order_k and
 * offsets_k from svg2_kmeans of the keys; vbar fp32 [BH, Ck, d] (16-byte
 * aligned), disp fp32 [BH, Ck]. Errors: INVALID_ARG, UNSUPPORTED (d), CUDA. */
svg_status svg2_cluster_value_stats(int32_t BH, int32_t N, int32_t d, int32_t Ck,
                                    const svg_bf16* v, const int32_t* order_k,
                                    const int32_t* offsets_k, float* vbar, float* disp,
                                    svg_stream_t stream);

/* svg2_ear_workspace_bytes -- host only: the workspace of svg2_ear_compensate
 * (bf16 copies of the centroids and value means). */
svg_status svg2_ear_workspace_bytes(int32_t BH, int32_t d, int32_t Ck, size_t* bytes);

/* svg2_ear_compensate -- SVG-EAR's centroid compensation ("parameter-free
 * centroid compensation" of the skipped blocks, the same section), in place
 * on the block-sparse output of svg2_sparse_attention. For sorted query row i
 * of query tile r of head bh: every key outside the computed key tiles of row
 * r of the CSR is stood in for by its cluster: n_b(r) uncovered keys of key
 * cluster b add n_b(r) * exp(scale * q_i . kbar_b) to the softmax's
 * denominator and the same times vbar_b to its numerator (kbar_b, vbar_b
 * rounded to bf16, the tensor-core operand format), so
 *   O_i = (O_s,i e^{lse_i} + sum_b n_b e^{scale q_i.kbar_b} vbar_b)
 *         / (e^{lse_i} + sum_b n_b e^{scale q_i.kbar_b}).
 *   qs         bf16 [BH, N, d] sorted queries (as given to the attention).
 *   kbar       fp32 [BH, Ck, d] key centroids (svg2_kmeans of the keys).
 *   vbar       fp32 [BH, Ck, d] (svg2_cluster_value_stats).
 *   offsets_k  [BH, Ck+1]; row_ptr, col_idx the CSR the attention used
 *              (block_q = 128, block_k).
 *   os         bf16 [BH, N, d] in: the attention's output, out: compensated.
 *   lse        fp32 [BH, N], the attention's log-sum-exp (natural log).
 *   workspace  >= svg2_ear_workspace_bytes, 256-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED (d, block_k, Ck not a multiple of 16 in
 * [16, 256], more than 4096 key tiles), CAPACITY, CUDA. */
svg_status svg2_ear_compensate(int32_t BH, int32_t N, int32_t d, int32_t Ck, int32_t block_k,
                               float scale, const svg_bf16* qs, const float* kbar,
                               const float* vbar, const int32_t* offsets_k,
                               const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                               const float* lse, void* workspace, size_t workspace_bytes,
                               svg_stream_t stream);

/* svg2_build_tile_csr -- the tile pairs of the sorted layouts to compute, one
 * CSR per head: query tile r (sorted query positions [r*block_q, ...)) lists,
 * ascending, every key tile holding a key of a cluster kept (sel) by a query
 * cluster present in tile r. Row bh*nQB + r of the stacked CSR; row_ptr
 * [BH*nQB + 1] (row_ptr[0] = 0), col_idx [col_capacity] (at most
 * BH*nQB*nKB entries are written; beyond col_capacity an entry is dropped
 * and the device bounds bit set). counts [BH*nQB] int32 is scratch.
 * Errors: INVALID_ARG, UNSUPPORTED (blocks not 64/128, more than 4096 key
 * tiles), CUDA. */
svg_status svg2_build_tile_csr(int32_t BH, int32_t N, int32_t Cq, int32_t Ck, int32_t block_q,
                               int32_t block_k, const int32_t* offsets_q, const int32_t* offsets_k,
                               const uint32_t* sel, int32_t* row_ptr, int32_t* col_idx,
                               int64_t col_capacity, int32_t* counts, svg_stream_t stream);

/* svg2_gather_rows / svg2_scatter_rows -- the token permutation:
 *   gather   y[bh, pos]            = x[bh, order[bh, pos]]   (into sorted order)
 *   scatter  y[bh, order[bh, pos]] = y_sorted[bh, pos]       (back)
 * x, y bf16 [BH, N, d] (d 64 or 128), 16-byte aligned, not overlapping. An
 * order entry outside [0, N) sets the device bounds bit and is skipped. */
svg_status svg2_gather_rows(int32_t BH, int32_t N, int32_t d, const svg_bf16* x,
                            const int32_t* order, svg_bf16* y, svg_stream_t stream);
svg_status svg2_scatter_rows(int32_t BH, int32_t N, int32_t d, const svg_bf16* y_sorted,
                             const int32_t* order, svg_bf16* y, svg_stream_t stream);

/* svg2_sparse_attention -- block-sparse flash attention over the sorted
 * layouts with one CSR per head (from svg2_build_tile_csr with block_q =
 * 128): for sorted query row i of head bh,
 *   O[i] = sum over keys j of listed tiles of softmax_j(scale * q_i . k_j) v_j
 * (queries sorted by their cluster order, keys and values by theirs; the same
 * kernel as svg_sparse_attention). qs, ks, vs, os bf16 [BH, N, d]; lse fp32
 * [BH, N] (natural log, sorted query rows) or NULL.
 * Errors: INVALID_ARG, UNSUPPORTED (d or block_k), CUDA. */
svg_status svg2_sparse_attention(int32_t BH, int32_t N, int32_t d, int32_t block_k, float scale,
                                 const svg_bf16* qs, const svg_bf16* ks, const svg_bf16* vs,
                                 const int32_t* row_ptr, const int32_t* col_idx, svg_bf16* os,
                                 float* lse, svg_stream_t stream);

/* ---------------------------------------------------------------------------
 * svg_get_device_status -- synchronises `stream`, then reads and clears the
 * device status bits of the current device (1 = a bounded wait ran out,
 * 2 = an out-of-range index from caller memory was skipped) into *bits
 * (may be NULL). Returns SVG_ERR_DEVICE_TIMEOUT if bit 1 was set,
 * SVG_ERR_INVALID_ARG if only bit 2 was set, SVG_ERR_CUDA on a CUDA error
 * (including errors of earlier asynchronous launches), SVG_OK otherwise.
 */
svg_status svg_get_device_status(svg_stream_t stream, int32_t* bits);

/* ---------------------------------------------------------------------------
 * svg_selftest_wait_timeout -- failure-detection self-test. Launches one CTA
 * whose thread waits, through the same bounded wait the kernels use, on a
 * shared-memory barrier that nothing ever completes, with a limit of
 * limit_cycles SM clock cycles (1 .. 2^31). The wait runs out, sets the
 * timeout status bit and the kernel returns normally; no fault, trap or hang.
 */
svg_status svg_selftest_wait_timeout(int64_t limit_cycles, svg_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char* svg_status_string(svg_status status);

/* Library version (major*10000 + minor*100 + patch). */
int32_t svg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVG_H_ */
