/*
 * bsa.h -- C ABI of libbsa.so: block-sparse 3D spatio-temporal attention for
 * video-DiT tokens on NVIDIA B200 (sm_100a).
 *
 * The library computes the data-parallel path the sparse video-attention pages
 * describe:
 *   (a) a 3D tile permute of a T x H x W token grid (and its inverse),
 *   (b) block masks: the static Sliding-Tile window, the static radial
 *       (energy-decay) mask, and the dynamic per-head NABLA top-p mask,
 *   (c) compaction of a block mask into per-row kept-block lists,
 *   (d) the attention forward that visits only kept (query block, key block)
 *       pairs, with an online softmax, producing O and the log-sum-exp,
 *   (e) its backward (dQ, dK, dV) over the same kept pairs,
 *   (f) SPADE scheme generation (SICS per block for a menu of 3D slice shapes
 *       and the per-head choice), and
 *   (g) a paged key/value cache with persistent anchors for autoregressive
 *       chunk decoding (page writes, block means, page importance, keep/evict,
 *       attention through the page table).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them and keeps no per-call state.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  A return of BSA_OK means the work was enqueued.
 *   - Arguments are validated on the host before anything is enqueued.  Invalid
 *     arguments return BSA_ERR_INVALID_ARG, shapes outside what the kernels
 *     implement return BSA_ERR_UNSUPPORTED; neither enqueues work.  There is no
 *     fallback path of any kind.
 *   - Token tensors are bfloat16, layout [B, N, heads, head_dim] with
 *     head_dim contiguous (one token row = heads * head_dim elements), 16-byte
 *     aligned base addresses.  Calls that take a row stride also accept token
 *     rows that are a slice of wider rows: consecutive rows lie row_stride
 *     elements apart (0 = the dense heads * head_dim; otherwise at least that
 *     and a multiple of 8) and batches N * row_stride apart.  That runs a range
 *     of heads of a [B, N, H_total, head_dim] tensor in place (pass the pointer
 *     to the first head of the range, heads = the range's size, row_stride =
 *     H_total * head_dim), or Q, K and V straight out of a fused
 *     [B, N, 3, H, head_dim] projection (row_stride = 3 * H * head_dim).
 *   - Masks are uint8, one byte per (query block, key block), 0 = dropped,
 *     nonzero = kept, row-major [rows][KB].
 *   - Errors never abort the process.  Errors detected on the device (a
 *     malformed kept list, a pipeline wait that ran out of time) are recorded
 *     in the workspace's status word; read it with bsa_read_status().
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad kept list */
  BSA_ERR_UNSUPPORTED = 2,   /* valid request outside the implemented shapes   */
  BSA_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_size()   */
  BSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed      */
  BSA_ERR_TIMEOUT = 5        /* a device-side pipeline wait ran out of time      */
} bsa_status;

/* Human-readable name of a status code (static string). */
const char* bsa_status_string(int status);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* bsa_last_error_message(void);

/* Library version as major*10000 + minor*100 + patch. */
int bsa_version(void);

/* ---------------------------------------------------------------------------
 * (a) Tile permute.
 * Source: "Fast Video Generation with Sliding Tile Attention" explainer
 * (aibr.jp/archives/60739), section 3: the video latent is a 3D
 * (time, height, width) token grid and the work is organised in 3D tiles.
 *
 * The grid T x H x W (raster order: w fastest) is cut into tT x tH x tW tiles.
 * The permuted sequence lists the tiles in raster order over the tile grid and,
 * inside each tile, its tokens in raster order.  Edge tiles may be smaller
 * (ragged); they are not padded.  Positions N .. n_pad-1 (N = T*H*W) of the
 * output are written with zeros so the sequence fills whole blocks.
 *
 *   x    : [batch, N] input rows in raster order (any element type)
 *   y    : [batch, n_pad] output rows in tile order
 *   row_bytes : bytes moved per token row (heads * head_dim * 2 for bf16),
 *               multiple of 16
 *   x_row_stride_bytes, y_row_stride_bytes : bytes from one row of x / y to the
 *               next (0 = row_bytes; else >= row_bytes, multiple of 16), so a
 *               row may be a slice (e.g. a range of heads) of a wider row
 *   n_pad >= N.  x and y must not overlap.
 * bsa_tile_untile is the inverse: reads y (tile order, n_pad rows), writes the
 * N raster-order rows of x; the zero tail of y is not read.
 * ------------------------------------------------------------------------- */
int bsa_tile_permute(const void* x, void* y, int batch, int T, int H, int W,
                     int tT, int tH, int tW, int row_bytes, int n_pad, int x_row_stride_bytes,
                     int y_row_stride_bytes, void* stream);
int bsa_tile_untile(const void* y, void* x, int batch, int T, int H, int W,
                    int tT, int tH, int tW, int row_bytes, int n_pad, int y_row_stride_bytes,
                    int x_row_stride_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (a') Tile permute fused with per-block mean pooling.
 * Sources: STA explainer section 3 (tile order) and the NABLA explainer
 * (aibr.jp/archives/124678), section 3 (Q and K are mean-pooled per block).
 *
 * Same permutation as bsa_tile_permute for bf16 rows of heads * head_dim
 * elements, with n_pad a multiple of `block` (1..1024).  While the rows are
 * moved, the mean of every `block` consecutive output rows is taken per head over
 * the rows that hold tokens (the zero tail is excluded), so the NABLA mask needs
 * no second pass over Q and K.
 *   pooled : [batch, heads, n_pad / block, head_dim] float32, written completely.
 *   x_row_stride, y_row_stride : token row strides of x and y in elements (0 =
 *            heads * head_dim; else >= that and a multiple of 8).
 * ------------------------------------------------------------------------- */
int bsa_tile_permute_pool(const void* x, void* y, int batch, int T, int H, int W, int tT,
                          int tH, int tW, int heads, int head_dim, int n_pad, int block,
                          float* pooled, int x_row_stride, int y_row_stride, void* stream);

/* ---------------------------------------------------------------------------
 * (a'') Tile permute with a slice shape per (batch, head).
 * Source: SPADE summary (gist.science/ja/paper/2608.03335), solution part 1 (a
 * menu of ways to cut the T x H x W cube, the best one picked for the video),
 * part 2 (the pick by SICS, bsa_sics_scheme) and part 3 (head-wise sparse
 * attention on the result).
 *
 * Head h of batch b is permuted like bsa_tile_permute with the tile
 * shapes[choice[b * heads + h]], so each head of y has its own token order; the
 * attention, masks and compaction then run on y unchanged (they are per head).
 *   shapes : HOST int array [n_shapes][3] (tT, tH, tW), 1 <= n_shapes <= 8,
 *            e.g. the menu given to bsa_sics_scheme.
 *   choice : DEVICE int32 [batch][heads] (4-byte aligned), e.g. bsa_sics_scheme's
 *            choice output.
 *            An entry outside [0, n_shapes) is not a host error (the host does
 *            not read it): that head's rows of y (and its pooled means) are
 *            zero and BSA_ERR_INVALID_ARG is written to *device_status (a device
 *            int, may be NULL, not cleared by the call).
 *   x, y   : bf16 [batch, N, heads, head_dim] raster / [batch, n_pad, heads,
 *            head_dim] in per-head tile order, zero tail; row strides in
 *            elements as in bsa_tile_permute_pool.  head_dim a multiple of 8,
 *            at most 1024.
 *   pooled : optional (NULL: no pooling) float32 [batch, heads, n_pad / block,
 *            head_dim], the mean of every `block` consecutive rows of y per head
 *            over the rows that hold tokens; n_pad a multiple of block, block <=
 *            1024.  Without pooled, block only sets the rows per CTA (0 = 64).
 * bsa_scheme_untile: the inverse, y (per-head tile order) -> x (raster); the
 *   zero tail of y is not read.  A head with a choice outside the menu gets zero
 *   rows in x and the same device status.
 * ------------------------------------------------------------------------- */
int bsa_scheme_permute(const void* x, void* y, int batch, int T, int H, int W,
                       const int* shapes, int n_shapes, const int* choice, int heads,
                       int head_dim, int n_pad, int block, float* pooled, int x_row_stride,
                       int y_row_stride, int* device_status, void* stream);
int bsa_scheme_untile(const void* y, void* x, int batch, int T, int H, int W, const int* shapes,
                      int n_shapes, const int* choice, int heads, int head_dim, int n_pad,
                      int y_row_stride, int x_row_stride, int* device_status, void* stream);

/* ---------------------------------------------------------------------------
 * (b1) Sliding Tile Attention mask.
 * Source: STA explainer (aibr.jp/archives/60739), sections 2-3: each query tile
 * attends to a window of neighbouring tiles; the window is counted in tiles.
 *
 * Tile grid nT x nH x nW (tiles in raster order = blocks of the permuted
 * sequence when the block size equals the tile volume), window wT x wH x wW
 * tiles.  shift = 0: the window covers offsets -floor((w-1)/2)..+ceil((w-1)/2)
 * around the query tile on each axis, clipped at the grid edge.  shift = 1:
 * the window keeps its full width and slides inward at the edges.
 *   mask : [n_tiles][n_tiles] uint8, n_tiles = nT*nH*nW, written completely.
 * ------------------------------------------------------------------------- */
int bsa_sta_mask(int nT, int nH, int nW, int wT, int wH, int wW, int shift,
                 uint8_t* mask, void* stream);

/* ---------------------------------------------------------------------------
 * (b2) Radial (energy-decay) mask.
 * Source: "Radial Attention" explainer (aibr.jp/archives/112136), sections 1-3:
 * a static mask, dense for temporally close tokens, whose spatial window shrinks
 * as the temporal distance grows, for O(n log n) kept pairs.
 *
 * Tokens in raster order, S = tokens_per_frame, token i is (frame i / S,
 * in-frame index i % S).  Token pair (query, key) at frame distance d and
 * in-frame distance ds is kept iff d <= 1, or, with r = floor(log2 d):
 *   if S >= block * 2^r : ds < S / 2^(r+1)
 *   else                : d % 2^c == 0 and ds < block / 2,
 *                         c = smallest integer with S * 2^c >= block * 2^r.
 * A block pair is kept iff any of its token pairs is kept.
 *   mask : [NB][NB] uint8, NB = ceil(n_tokens / block), written completely.
 * ------------------------------------------------------------------------- */
int bsa_radial_mask(int n_tokens, int tokens_per_frame, int block, uint8_t* mask,
                    void* stream);

/* ---------------------------------------------------------------------------
 * (b3) NABLA dynamic mask (optionally with forced-on key ranges).
 * Source: "NABLA" explainer (aibr.jp/archives/124678), section 3: mean-pool Q
 * and K per block, compute full attention on the pooled tokens, threshold each
 * row by its cumulative distribution, apply the binary mask at block level.
 * Forced ranges: "Sparse Forcing" summary (gist.science/ja/paper/2604.21221),
 * part 2 -- persistent anchor frames and recent frames kept, sparse selection
 * elsewhere.
 *
 *   q : [batch, nq, heads, head_dim] bf16 (tile order); k : [batch, nk, ...];
 *   row_stride : token row stride of q and k in elements (0 = heads * head_dim)
 *   Blocks of `block` tokens; the last block of q / k may be partial and is
 *   averaged over its valid tokens only.  QB = ceil(nq/block), KB = ceil(nk/block).
 *   Row (b, h, qb): logits z_c = mean_q . mean_k[c] * scale (scale <= 0 means
 *   1/sqrt(head_dim)) over key blocks c in [kb_begin, kb_end); softmax over that
 *   range; the kept set is the smallest set of largest probabilities (ties to the
 *   lower index) whose sum reaches p (p >= 1 keeps the whole range).  Key blocks
 *   outside [kb_begin, kb_end) are written as force_outside (0 or 1).
 *   mask : [batch][heads][QB][KB] uint8, written completely.
 *   near_count : device int, overwritten with the number of rows whose cut lies
 *                within 1e-5 of p (rows a float64 evaluation may decide
 *                differently); may be NULL.
 *   ws : device workspace of at least bsa_nabla_workspace_size() bytes.
 *   head_dim in {64, 128}; block a multiple of 16 in [16, 1024].
 * ------------------------------------------------------------------------- */
size_t bsa_nabla_workspace_size(int batch, int heads, int nq, int nk, int head_dim, int block);
int bsa_nabla_mask(const void* q, const void* k, int batch, int heads, int nq, int nk,
                   int head_dim, int row_stride, int block, float p, float scale, int kb_begin,
                   int kb_end, int force_outside, uint8_t* mask, int* near_count, void* ws,
                   size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (b4) NABLA selection from pooled means, optionally united with a fixed mask.
 * Sources: NABLA explainer section 3 (softmax over pooled logits, CDF cut);
 * sections 1-2 (NABLA combines with Sliding Tile Attention and other sparse
 * patterns); Sparse Forcing summary part 2 (forced anchor / recent ranges).
 *
 * The selection step of bsa_nabla_mask on caller-provided means:
 *   qbar : [batch, heads, QB, head_dim] float32, kbar : [batch, heads, KB, head_dim]
 * (as written by bsa_tile_permute_pool or by the pooling of bsa_nabla_mask).
 * Semantics of p, scale, kb_begin, kb_end, force_outside, mask and near_count
 * as for bsa_nabla_mask.  base_mask (may be NULL): [QB][KB] uint8 shared by all
 * batches and heads, OR-ed into every row of the result -- with a Sliding-Tile
 * mask this gives the NABLA-plus-window hybrid.  key_allowed (may be NULL):
 * [batch][KB] uint8; key blocks with 0 (e.g. evicted from a paged cache, see
 * bsa_kv_resident_blocks) leave the softmax of [kb_begin, kb_end) and are never
 * selected there.  head_dim in {64, 128}.
 * ------------------------------------------------------------------------- */
int bsa_nabla_select(const float* qbar, const float* kbar, int batch, int heads, int QB, int KB,
                     int head_dim, float p, float scale, int kb_begin, int kb_end,
                     int force_outside, const uint8_t* base_mask, const uint8_t* key_allowed,
                     uint8_t* mask, int* near_count, void* stream);

/* ---------------------------------------------------------------------------
 * (c) Mask compaction into per-row kept-block lists (CSR).
 * Source: the NABLA explainer (aibr.jp/archives/124678), section 3, and the STA
 * explainer, section 3: the binary block mask decides which block pairs are
 * computed; listing the kept blocks per row is this library's step (no
 * counterpart in the pages).
 *   mask    : [rows][KB] uint8
 *   row_ptr : [rows + 1] int32, written; row_ptr[rows] = number of kept blocks
 *   col_idx : int32 with room for rows*KB entries (worst case), written with the
 *             kept key-block indices of each row in ascending order.
 * ------------------------------------------------------------------------- */
int bsa_mask_compact(const uint8_t* mask, int rows, int KB, int* row_ptr, int* col_idx,
                     void* stream);

/* ---------------------------------------------------------------------------
 * (d) Block-sparse attention forward.
 * Sources: STA explainer section 3 (hardware-aware tile attention kernel),
 * SPADE summary (gist.science/ja/paper/2608.03335), solution part 3 (head-wise
 * sparse attention), NABLA explainer section 3 (mask applied at block level).
 *
 *   O[b, i, h, :] = softmax_j( Q[b,i,h,:] . K[b,j,h,:] * scale ) V[b, j, h, :]
 *   over keys j < nk whose block pair (i / block_q, j / block_k) is kept in the
 *   list of mask head m = (list_heads == 1 ? 0 : b * heads + h).
 *   LSE[b, h, i] = natural-log sum of exp(scores) over the same keys.
 *   A row with no kept key gets O = 0 and LSE = -inf.
 *
 *   q : [batch, nq, heads, head_dim] bf16; k, v : [batch, nk, heads, head_dim]
 *   o : [batch, nq, heads, head_dim] bf16 (rows >= nq are never written)
 *   qkv_row_stride : token row stride of q, k and v in elements; o_row_stride :
 *       that of o (each 0 = heads * head_dim; see the conventions above)
 *   lse : [batch, heads, nq] float32 (dense, for the heads of this call)
 *   row_ptr, col_idx : CSR over rows m * QB + qb (QB = ceil(nq/block_q)),
 *                      col_idx ascending within a row, values < KB = ceil(nk/block_k)
 *                      (as written by bsa_mask_compact).  Malformed lists set
 *                      BSA_ERR_INVALID_ARG in the status word and are skipped.
 *   list_heads : 1 (one list for every batch and head) or batch * heads
 *   scale : <= 0 means 1/sqrt(head_dim)
 *   head_dim in {64, 128}; block_q, block_k each 64 or a multiple of 128.
 *   ws : device workspace of at least bsa_attn_workspace_size() bytes; its
 *        status word is cleared at the start of every call.
 * ------------------------------------------------------------------------- */
size_t bsa_attn_workspace_size(int batch, int heads, int nq, int nk, int block_q, int block_k,
                               int list_heads);
int bsa_attn_fwd(const void* q, const void* k, const void* v, int batch, int heads, int nq,
                 int nk, int head_dim, int qkv_row_stride, int o_row_stride, int block_q,
                 int block_k, const int* row_ptr, const int* col_idx, int list_heads,
                 float scale, void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (e) Block-sparse attention backward.
 * Sources: Radial explainer (aibr.jp/archives/112136) section 4 (training cost
 * falls with the sparse mask), NABLA explainer (aibr.jp/archives/124678)
 * section 4 (training and inference speed-up), Sparse Forcing summary
 * (gist.science/ja/paper/2604.21221): the sparse attention is trained through.
 *
 *   Gradients of bsa_attn_fwd with respect to q, k and v, for the same kept
 *   block pairs: with P the forward's probabilities (recomputed from lse),
 *   Delta[i] = sum_d dO[i,d] * O[i,d],
 *     dV[j] = sum_i P[i,j] dO[i]
 *     dS[i,j] = P[i,j] * (dO[i] . V[j] - Delta[i])
 *     dQ[i] = scale * sum_j dS[i,j] K[j],   dK[j] = scale * sum_i dS[i,j] Q[i]
 *   q, k, v, row_ptr, col_idx, list_heads, scale : as passed to bsa_attn_fwd
 *   o, lse : that call's outputs; dout : dL/dO, same layout as o (bf16)
 *   dq : [batch, nq, heads, head_dim] bf16, written (rows with no kept key: 0)
 *   dk, dv : [batch, nk, heads, head_dim] bf16, written (keys no row keeps: 0)
 *   qkv_row_stride : token row stride (elements) of q, k, v, dq, dk and dv;
 *   o_row_stride : that of o and dout (each 0 = heads * head_dim)
 *   head_dim in {64, 128}; block_q, block_k each 64 or a multiple of 128.
 *   ws : device workspace of at least bsa_attn_bwd_workspace_size() bytes (its
 *        status word, read with bsa_read_status, is cleared by every call).
 *   Two kernel passes, no atomics: dK/dV per 128-key tile over the transposed
 *   kept lists, then dQ per 128-query tile.  Pointer arguments must be 16-byte
 *   aligned; errors as for bsa_attn_fwd.
 * ------------------------------------------------------------------------- */
size_t bsa_attn_bwd_workspace_size(int batch, int heads, int nq, int nk, int block_q,
                                   int block_k, int list_heads);
int bsa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, int batch, int heads, int nq, int nk, int head_dim,
                 int qkv_row_stride, int o_row_stride, int block_q, int block_k,
                 const int* row_ptr, const int* col_idx, int list_heads, float scale, void* dq,
                 void* dk, void* dv, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (d') Block-sparse attention forward that allocates nothing.
 * No counterpart in the pages: this is a library convenience, not part of the
 * method.
 *
 * For callers that cannot provide or allocate a workspace -- e.g. code running
 * inside a host framework that owns every device allocation through its own
 * pre-reserved pool, or a serving loop where a cudaMalloc (which may
 * synchronise the device) is not permitted.  Same arguments and results as
 * bsa_attn_fwd with dense token rows (both row strides 0), without ws /
 * ws_bytes: the workspace is a fixed 8 MiB device array inside libbsa.so,
 * which every GPU that loads the library holds until the process exits.
 *   - Shapes whose bsa_attn_workspace_size() exceeds 8 MiB are rejected with
 *     BSA_ERR_WORKSPACE (see bsa_last_error_message()) before any work.
 *   - Arguments are checked as bsa_attn_fwd checks them, in the same order and
 *     with the same codes, before the size check.
 *   - The first call made with a given device current looks up that device's
 *     array address (cudaGetSymbolAddress); make that first call before any
 *     stream capture.  The address is looked up again when the calling
 *     thread's current context differs from the one it was taken in (e.g.
 *     after cudaDeviceReset), so the first call after such a reset also belongs
 *     before any capture.
 *   - All calls share the one array per device: calls that can overlap on the
 *     GPU (different streams without ordering) race and must be serialised by
 *     the caller.  Everything the call needs zeroed is cleared by the call.
 *   - device_status (optional device int, may be NULL) receives the call's
 *     device-side status word (a bsa_status value) when the work completes.
 *   The library itself calls no allocator in this entry point.
 * ------------------------------------------------------------------------- */
int bsa_attn_fwd_noalloc(const void* q, const void* k, const void* v, int batch, int heads,
                         int nq, int nk, int head_dim, int block_q, int block_k,
                         const int* row_ptr, const int* col_idx, int list_heads, float scale,
                         void* o, float* lse, int* device_status, void* stream);

/* ---------------------------------------------------------------------------
 * (f) SPADE scheme generation: SICS and the per-head slicing choice.
 * Source: SPADE summary (gist.science/ja/paper/2608.03335), solution part 1 (a
 * menu of 3D slice shapes: wide and flat, tall and thin, mixed) and part 2
 * (scheme generation by SICS, the sum of intra-block cosine similarities, from Q
 * and K alone, per head).
 *
 * bsa_sics_blocks: for every tile of shape tT x tH x tW (tiles in raster order
 *   over the tile grid, ragged at the far edges) and every head,
 *     out[b][h][tile] = sum over ordered token pairs (i, j) of the tile of
 *                       cos(x[b, i, h, :], x[b, j, h, :])   (i == j included;
 *                       a zero vector contributes 0).
 *   x : [batch, T*H*W, heads, head_dim] bf16, raster token order, 16-byte aligned;
 *       row_stride: token row stride in elements (0 = heads * head_dim), as in the
 *       conventions above (bsa_sics_scheme: shared by q and k)
 *   out : float32 [batch][heads][ceil(T/tT)*ceil(H/tH)*ceil(W/tW)], written
 *   head_dim in {64, 128}; heads * head_dim <= 8192; tT*tH*tW <= 4096 tokens.
 *
 * bsa_sics_scheme: runs bsa_sics_blocks on q and k for every shape of the menu
 *   shapes (HOST array of n_shapes x {tT, tH, tW}, 1 <= n_shapes <= 16) and writes
 *     scores[b][h][s] = (sum_tiles SICS_q + sum_tiles SICS_k) / (2 * sum_tiles n^2)
 *   (n = the tile's token count: the mean intra-block cosine similarity) and
 *     choice[b][h] = the first s with the highest score (int32).
 *   ws : device workspace of at least bsa_sics_workspace_size() bytes.
 * A tile may be larger than the grid along an axis (one ragged tile there).
 * Errors: BSA_ERR_INVALID_ARG (null / misaligned pointers, a non-positive
 * extent), BSA_ERR_UNSUPPORTED (head_dim, heads * head_dim or tile volume out of
 * range), BSA_ERR_WORKSPACE.
 * ------------------------------------------------------------------------- */
int bsa_sics_blocks(const void* x, int batch, int T, int H, int W, int tT, int tH, int tW,
                    int heads, int head_dim, int row_stride, float* out, void* stream);
size_t bsa_sics_workspace_size(int batch, int heads, int T, int H, int W, const int* shapes,
                               int n_shapes);
int bsa_sics_scheme(const void* q, const void* k, int batch, int T, int H, int W, int heads,
                    int head_dim, int row_stride, const int* shapes, int n_shapes,
                    float* scores, int* choice, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * (g) Paged KV cache with persistent anchors (autoregressive chunk decoding).
 * Source: Sparse Forcing summary (gist.science/ja/paper/2604.21221), part 2
 * (anchors kept as persistent memory, recent frames looked at closely, only the
 * important points of the past stored) and part 4 (memory use down 42 %).
 *
 * Pages hold 128 consecutive tokens of the key sequence (one attention k-tile)
 * with the [token][heads][head_dim] bf16 row layout.  A pool of n_pool_pages
 * pages is shared by the batch; page_table [batch][pages_per_batch] int32 maps
 * logical page lp (tokens 128*lp .. 128*lp+127) to a physical page, -1 when
 * evicted.  The pool must be allocated initialised (e.g. zeros): rows past the
 * end of the sequence in its last page are read and must be finite.
 *
 * bsa_kv_write: rows [batch, n_new, heads, head_dim] bf16 go to logical tokens
 *   first_token .. first_token+n_new-1 of each batch; their pages must be
 *   assigned.  A row whose page is -1 or out of range is skipped and
 *   BSA_ERR_INVALID_ARG is written to *device_status (a device int, may be NULL).
 * bsa_block_pool: out[b][h][first_block + i][:] = mean of tokens
 *   [block*(first_block+i), min(block*(first_block+i+1), n_tokens)) of x, for
 *   i < n_blocks; x is [batch, n_tokens, heads, head_dim] (page_table NULL) or a
 *   paged pool; out is float32 [batch][heads][out_blocks][head_dim].
 * bsa_kv_resident_blocks: allowed[b][kb] = 1 iff the page of key block kb
 *   (block tokens, 128 % block == 0) is resident.
 * bsa_kv_page_scores: scores[b][page] = sum over heads h and query blocks qb of
 *   softmax_kb(qbar[b,h,qb] . kbar[b,h,kb] * scale) over the allowed kb in
 *   [kb_begin, kb_end), summed over the blocks kb of that page (zeroed first).
 * bsa_kv_keep_pages: scores [batch][n_pages]; page_table rows of
 *   pages_per_batch >= n_pages entries.  Per batch, pages < anchor_pages and
 *   >= recent_begin are kept; of the resident pages in between the `budget` highest scores are kept
 *   (ties: the lower page) and every other one is evicted: its page_table entry
 *   becomes -1 and its physical page is appended to freed[] at index
 *   atomicAdd(freed_count, 1).  *freed_count is not cleared by the call, so
 *   freed[] needs room for batch * (recent_begin - anchor_pages - budget) ints
 *   past its current value (zero it first to start at freed[0]).
 *   recent_begin - anchor_pages <= 8192.
 * bsa_attn_fwd_paged: bsa_attn_fwd with K and V read through the page table
 *   from one-batch pools [n_pool_pages * 128, heads, head_dim]; key blocks on
 *   evicted pages are dropped from the kept lists.  block_k in {64, 128};
 *   pages_per_batch >= ceil(nk / 128); list_heads == batch * heads unless
 *   batch == 1.
 * ------------------------------------------------------------------------- */
int bsa_kv_write(const void* src, int batch, int n_new, int heads, int head_dim, int first_token,
                 const int* page_table, int pages_per_batch, void* pool, int n_pool_pages,
                 int* device_status, void* stream);
int bsa_block_pool(const void* x, const int* page_table, int pages_per_batch, int batch,
                   int n_tokens, int heads, int head_dim, int block, int first_block,
                   int n_blocks, float* out, int out_blocks, void* stream);
int bsa_kv_resident_blocks(const int* page_table, int batch, int pages_per_batch, int block,
                           int KB, uint8_t* allowed, void* stream);
int bsa_kv_page_scores(const float* qbar, const float* kbar, int batch, int heads, int QB, int KB,
                       int head_dim, float scale, int kb_begin, int kb_end,
                       const uint8_t* key_allowed, int block, int n_pages, float* scores,
                       void* stream);
int bsa_kv_keep_pages(const float* scores, int batch, int n_pages, int anchor_pages,
                      int recent_begin, int budget, int* page_table, int pages_per_batch,
                      int* freed, int* freed_count, void* stream);
int bsa_attn_fwd_paged(const void* q, const void* k_pool, const void* v_pool, int n_pool_pages,
                       const int* page_table, int pages_per_batch, int batch, int heads, int nq,
                       int nk, int head_dim, int block_q, int block_k, const int* row_ptr,
                       const int* col_idx, int list_heads, float scale, void* o, float* lse,
                       void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Self-test of the bounded device-side waits (failure detection).
 * No counterpart in the pages.  Launches one thread that waits, through the
 * same bounded wait the attention pipeline uses, on a barrier phase that never
 * completes; after timeout_ns (1 ns .. 10 s) it writes BSA_ERR_TIMEOUT to
 * *device_status (a device int, cleared first) and returns.  Used by the tests
 * to show that a stuck pipeline ends with a status instead of hanging the GPU.
 * ------------------------------------------------------------------------- */
int bsa_wait_selftest(int* device_status, unsigned long long timeout_ns, void* stream);

/* ---------------------------------------------------------------------------
 * Device status word of a workspace (attention or NABLA; no counterpart in the
 * pages): synchronises `stream`,
 * copies the word to *status (a bsa_status value) and clears it.
 * ------------------------------------------------------------------------- */
int bsa_read_status(void* ws, int* status, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* BSA_H_ */
