/*
 * bsa.h - C ABI of libbsa: radial block-sparse softmax attention, forward pass,
 * for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (page title, section):
 *  - "Radial Attention: O(nlog n) Sparse Attention with Energy Decay for Long
 *    Video Generation" skill page (skillsmp.com, radial-attention-video),
 *    Step 1 (radial mask: frame-major tokens, log2 temporal bands, decay) and
 *    Step 2 (RadialAttention.forward: softmax(Q K^T * head_dim^-0.5 + mask) V,
 *    layout [batch, heads, n, head_dim]).
 *  - "Radial Attention: A Breakthrough in Efficient Long Video Generation"
 *    (thismoment.ai), "How Radial Attention Works": density halves as temporal
 *    distance doubles, a spatial window that shrinks for distant frames, and
 *    128x128 block sparsity.
 *  - Sparse-vDiT skill page (skillsmp.com), "Sparse attention patterns", and
 *    the Compact Attention abstract (zhuanzhiai.com): per-head tile masks,
 *    passed to bsa_attn_fwd as per-head block lists.
 *
 * Conventions for every entry point:
 *  - Every function returns a bsa_status value (0 = BSA_OK).
 *  - Device pointers are plain CUDA device addresses owned by the caller; the
 *    library never frees or keeps them. The library allocates no device
 *    memory; scratch memory is the caller's `workspace`.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). All work
 *    is stream-ordered and asynchronous unless a function says it
 *    synchronises.
 *  - Errors found on the host (bad argument, unsupported shape, launch
 *    failure) are returned directly and nothing is launched. Errors found on
 *    the device (a bounded wait that ran out, a list entry out of range, an
 *    output buffer too small) are recorded in a per-device status word and
 *    reported by bsa_get_device_status().
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *bsa_stream_t; /* same type as cudaStream_t */

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, inconsistent sizes, aliasing */
  BSA_ERR_UNSUPPORTED = 2,    /* head_dim, block or device not supported */
  BSA_ERR_CUDA = 3,           /* a CUDA runtime call failed; see bsa_last_cuda_error() */
  BSA_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait ran out; results are invalid */
  BSA_ERR_BAD_LISTS = 5,      /* block lists not monotone / sorted / in range */
  BSA_ERR_CAPACITY = 6,       /* col_idx capacity smaller than the list size */
  BSA_ERR_SCRATCH_LIMIT = 7   /* problem too large for bsa_attn_fwd_noalloc's fixed scratch */
} bsa_status;

/*
 * Per-query-block key-block lists in CSR form (device memory).
 *
 * num_lists     1 (one list shared by every head) or `heads` (head h uses
 *               list h, whose rows start at h * num_q_blocks).
 * num_q_blocks  ceil(n / block); num_k_blocks is the same value.
 * block         tile edge in tokens: 64 or 128.
 * row_ptr       int32[num_lists * num_q_blocks + 1], row_ptr[0] = 0,
 *               non-decreasing.
 * col_idx       int32[nnz], each row strictly increasing, entries in
 *               [0, num_k_blocks).
 * nnz           entries in col_idx (= row_ptr[last]). Kernels clamp every row
 *               bound into [0, nnz] and every entry into [0, num_k_blocks), so
 *               malformed lists give wrong results, never an out-of-bounds
 *               access; bsa_validate_lists() detects them.
 *
 * A query in query block qb attends to every key j < n of every key block the
 * row lists (block granularity, thismoment.ai page: 128x128 block sparsity).
 */
typedef struct {
  int32_t num_lists;
  int32_t num_q_blocks;
  int32_t num_k_blocks;
  int32_t block;
  int32_t nnz;
  const int32_t *row_ptr;
  const int32_t *col_idx;
} bsa_block_lists;

/*
 * Build the radial block lists for `frames` x `tokens_per_frame` tokens
 * (n = frames * tokens_per_frame, frame-major) at tile size `block`.
 *
 * Rule (skillsmp radial-attention-video Step 1; thismoment.ai "How Radial
 * Attention Works"): temporal distance d = |f_i - f_j| has band
 * r = floor(log2(max(d, 1))); band r keeps a window of S >> min(r, r*) keys
 * (S = tokens_per_frame, r* = the last band whose window still holds `block`
 * keys, 0 if S < block) centred on the query's in-frame index and clamped into
 * the frame; bands beyond r* keep only frames with d % 2^(r - r*) == 0. A key
 * block is listed for a query block when any admitted token pair falls in it.
 *
 * row_ptr      device int32[ceil(n/block) + 1], written.
 * col_idx      device int32[col_capacity], or NULL to compute row_ptr only.
 * col_capacity entries available in col_idx (ignored when col_idx is NULL).
 * nnz_out      host int64*, or NULL. When given, the call synchronises
 *              `stream`, writes the list size and returns BSA_ERR_CAPACITY if
 *              col_idx was given and is too small (nothing beyond the capacity
 *              is written). When NULL the call is asynchronous and an
 *              overflow is reported by bsa_get_device_status().
 * Limits: 1 <= frames, 1 <= tokens_per_frame, n < 2^31, block in {64, 128},
 * ceil(n/block) <= 262144.
 */
int bsa_radial_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t block,
                          int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int64_t *nnz_out, bsa_stream_t stream);

/*
 * bsa_radial_mask_build for a joint sequence of video and text tokens: the
 * frames * tokens_per_frame video tokens (frame-major) followed by
 * text_tokens text tokens, n = frames * tokens_per_frame + text_tokens.
 * The pages describe video tokens only; the reading taken for the text that
 * video DiTs attend jointly with the video: the radial rule applies between
 * video tokens; a text query attends to every token and every query attends
 * to every text key. Blocks are cut over the whole sequence from token 0, so
 * a block may hold both the last video and the first text tokens; a query
 * block holding any text token lists every key block, and every row lists
 * the key blocks from (frames * tokens_per_frame) / block on.
 * text_tokens = 0 gives bsa_radial_mask_build's lists. Other arguments,
 * limits, synchronisation and errors as bsa_radial_mask_build
 * (text_tokens < 0 is BSA_ERR_INVALID_ARG).
 */
int bsa_joint_mask_build(int32_t frames, int32_t tokens_per_frame, int32_t text_tokens,
                         int32_t block, int32_t *row_ptr, int32_t *col_idx,
                         int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream);

/*
 * Block lists of a variable-length batch: item b is a video of frames[b] x
 * tokens_per_frame[b] tokens followed by text_tokens[b] text tokens (NULL:
 * none), with the joint rule of bsa_joint_mask_build. The pages describe one
 * video at a time and say nothing of batches; batching items of different
 * lengths (prompts with different text lengths, clips with different frame
 * counts) in one launch is this library's reading, and each item keeps
 * exactly its own lists.
 * The lists of the items are concatenated: item b's nqb_b = ceil(n_b / block)
 * query-block rows follow those of items 0..b-1 (row_ptr holds
 * sum_b nqb_b + 1 entries, values are offsets into one col_idx), and its
 * column indices count key blocks from 0 inside the item. The result is the
 * bsa_block_lists of bsa_attn_fwd_varlen with num_lists = 1,
 * num_q_blocks = sum_b nqb_b and num_k_blocks = max_b nqb_b.
 * num_items in [1, 64]; frames, tokens_per_frame, text_tokens are host
 * arrays of num_items entries. Other arguments, synchronisation and errors
 * as bsa_joint_mask_build.
 */
int bsa_joint_mask_build_varlen(int32_t num_items, const int32_t *frames,
                                const int32_t *tokens_per_frame, const int32_t *text_tokens,
                                int32_t block, int32_t *row_ptr, int32_t *col_idx,
                                int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream);

#define BSA_TILE_PATTERN_MAX_BANDS 16

/*
 * One head's tile pattern: the union of its terms over tiles (query block qb,
 * key block kb, rel = kb - qb). It covers the families of the Sparse-vDiT
 * skill page, "Sparse attention patterns" (diagonal window |rel| <= w;
 * multi-diagonal bands at chosen offsets; vertical stripes, fixed key columns
 * in every row; mixed = their union), and the dual window (local plus axial)
 * of the Compact Attention abstract.
 *
 * num_bands        0..BSA_TILE_PATTERN_MAX_BANDS band terms: band t holds
 *                  band_lo[t] <= rel <= band_hi[t] (empty when lo > hi).
 * axial_period     0 (no axial term) or P >= 1: the term holds when rel is
 *                  congruent modulo P to some t with |t| <= axial_halfwidth
 *                  (the axial window read on a video's tile sequence: tiles
 *                  about a whole number of frame periods away).
 * axial_halfwidth  >= 0.
 * columns_begin,   this pattern's vertical-stripe key blocks are
 * columns_end      columns[columns_begin .. columns_end) of the shared
 *                  `columns` array (any order, repeats allowed).
 * Key blocks outside [0, num_q_blocks) do not exist; a row may be empty.
 */
typedef struct {
  int32_t num_bands;
  int32_t band_lo[BSA_TILE_PATTERN_MAX_BANDS];
  int32_t band_hi[BSA_TILE_PATTERN_MAX_BANDS];
  int32_t axial_period;
  int32_t axial_halfwidth;
  int32_t columns_begin;
  int32_t columns_end;
} bsa_tile_pattern;

/*
 * Expand one tile pattern per list into CSR block lists on the device
 * (num_k_blocks = num_q_blocks): list h's rows start at h * num_q_blocks and
 * each row holds its key blocks in ascending order, as bsa_attn_fwd takes
 * them with num_lists = heads.
 *
 * patterns     device bsa_tile_pattern[num_lists].
 * columns      device int32[num_columns], the stripe columns of every
 *              pattern; NULL when num_columns is 0.
 * row_ptr      device int32[num_lists * num_q_blocks + 1], written.
 * col_idx, col_capacity, nnz_out: as bsa_radial_mask_build (NULL col_idx =
 *              count only; nnz_out given = synchronise and check capacity).
 * Limits: num_lists >= 1, 1 <= num_q_blocks <= 262144,
 * num_lists * num_q_blocks < 2^31 - 1. A malformed pattern (num_bands
 * outside [0, 16], negative period or half-width, a column range outside
 * [0, num_columns]) or a stripe column outside [0, num_q_blocks) is found on
 * the device: its rows (for a bad column, just that column) are left out and
 * bsa_get_device_status() reports BSA_ERR_INVALID_ARG.
 */
int bsa_tile_pattern_lists_build(int32_t num_lists, int32_t num_q_blocks,
                                 const bsa_tile_pattern *patterns, const int32_t *columns,
                                 int64_t num_columns, int32_t *row_ptr, int32_t *col_idx,
                                 int64_t col_capacity, int64_t *nnz_out, bsa_stream_t stream);

/*
 * Bytes of device scratch memory bsa_attn_fwd needs for this problem (the
 * longest-row-first work order of every list and a work counter the kernel's
 * CTAs take items from; at block 64 also the lists merged into 128-row tile
 * lists, about 5 bytes per list entry, on which block-64 problems run).
 * Returns 0 for invalid lists.
 */
size_t bsa_attn_fwd_workspace_bytes(int32_t batch, int32_t heads, const bsa_block_lists *lists);

/*
 * Block-sparse softmax attention forward (skillsmp radial-attention-video
 * Step 2, RadialAttention.forward, restricted to the listed blocks):
 *   out[b,h,i,:] = sum_j softmax_j(scale * <q[b,h,i], k[b,h,j]>) v[b,h,j,:]
 * over the keys j < n of the blocks listed for i's query block;
 *   lse[b,h,i]   = natural log of sum_j exp(scale * <q[b,h,i], k[b,h,j]>).
 * A row with an empty list gets out = 0 and lse = -inf.
 *
 * q, k, v       device bf16 [batch, heads, n, head_dim], contiguous, 16-byte
 *               aligned. They may alias each other.
 * head_dim      64 or 128.
 * softmax_scale <= 0 selects head_dim^-0.5.
 * lists         host pointer to the list descriptor (its arrays on device).
 * out           device bf16 [batch, heads, n, head_dim]; must not overlap q/k/v.
 * lse           device float [batch, heads, n], or NULL.
 * workspace     device scratch of at least bsa_attn_fwd_workspace_bytes(),
 *               16-byte aligned; overwritten.
 * Runs on the tensor cores (tcgen05, TMEM accumulators, TMA-staged tiles) of
 * an sm_100 device; returns BSA_ERR_UNSUPPORTED elsewhere. Asynchronous.
 */
int bsa_attn_fwd(const void *q, const void *k, const void *v,
                 int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                 float softmax_scale, const bsa_block_lists *lists,
                 void *out, float *lse, void *workspace, size_t workspace_bytes,
                 bsa_stream_t stream);

/*
 * Bytes of device workspace bsa_attn_fwd_host needs: device copies of q, k,
 * v, out and lse plus bsa_attn_fwd's own scratch. Returns 0 for invalid
 * arguments.
 */
size_t bsa_attn_fwd_host_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                         int32_t head_dim, const bsa_block_lists *lists);

/*
 * bsa_attn_fwd on HOST buffers: q_host, k_host, v_host (bf16 [batch, heads,
 * n, head_dim], contiguous) are copied to the device, the attention runs, and
 * out_host (same layout) and lse_host (float [batch, heads, n], or NULL) are
 * copied back. The problem is cut into about eight groups of whole heads
 * (never across batch items); group g's inputs are copied in on an internal
 * stream while group g-1 computes on `stream` and group g-2's results are
 * copied out on a second internal stream, so with pinned (page-locked) host
 * memory the copies in both directions overlap the kernels; pageable memory
 * works but serialises.
 * lists        device lists as for bsa_attn_fwd (already built, or built
 *              earlier on `stream`: the call orders after the work already
 *              enqueued on `stream`).
 * workspace    device memory of bsa_attn_fwd_host_workspace_bytes(),
 *              256-byte aligned; holds the device copies.
 * Asynchronous: the host buffers must stay valid, and out_host / lse_host
 * must not be read, until `stream` has been synchronised (work enqueued on
 * `stream` afterwards also orders after the last copy back). Calls are
 * serialised on the internal streams (one staging area per call). Errors as
 * bsa_attn_fwd; an error from a group's launch is returned after the groups
 * before it were enqueued (their results are then incomplete).
 */
int bsa_attn_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                      int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                      float softmax_scale, const bsa_block_lists *lists, void *out_host,
                      float *lse_host, void *workspace, size_t workspace_bytes,
                      bsa_stream_t stream);

/*
 * Strides of a [batch, heads, n, head_dim] bf16 tensor view, in elements; the
 * head_dim axis is contiguous. The contiguous layout of bsa_attn_fwd is
 * {heads*n*head_dim, n*head_dim, head_dim}. The token-major output of a fused
 * q/k/v projection, [batch, n, 3, heads, head_dim] (the skill page's
 * RadialAttention.forward projects x with q_proj, k_proj, v_proj and views the
 * result as [batch, n, heads, head_dim] before transposing), gives q, k and v
 * the layout {3*n*heads*head_dim, head_dim, 3*heads*head_dim} at offsets 0,
 * heads*head_dim and 2*heads*head_dim; an output in [batch, n, heads,
 * head_dim] order (what out_proj reads after the page's transpose back) is
 * {n*heads*head_dim, head_dim, heads*head_dim}.
 */
typedef struct {
  int64_t batch_stride;
  int64_t head_stride;
  int64_t token_stride;
} bsa_layout;

/*
 * bsa_attn_fwd on strided views: the same operation and results, with q, k,
 * v and out addressed as ptr + b*batch_stride + h*head_stride + i*token_stride
 * + d. The kernels read the views directly (the TMA descriptors carry the
 * strides) and write out in place, so no transpose runs before or after.
 *
 * Layout rules (BSA_ERR_INVALID_ARG otherwise): every stride of an axis
 * longer than 1 is positive, a multiple of 8 and below 2^39; the pointers are
 * 16-byte aligned; out's rows are pairwise disjoint; the span of out (first to
 * last addressed element) overlaps none of the spans of q, k and v (which may
 * overlap each other, e.g. as three slices of one projection buffer).
 * lse stays [batch, heads, n] contiguous (or NULL). Other arguments,
 * workspace and errors as bsa_attn_fwd. Asynchronous.
 */
int bsa_attn_fwd_strided(const void *q, const bsa_layout *q_layout,
                         const void *k, const bsa_layout *k_layout,
                         const void *v, const bsa_layout *v_layout,
                         int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                         float softmax_scale, const bsa_block_lists *lists,
                         void *out, const bsa_layout *out_layout, float *lse,
                         void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Rows generated inside the attention kernel. The two entries below compute
 * bsa_attn_fwd's operation over lists that are never written out: each
 * query-block row's key blocks are generated by the attention kernel's
 * producer from the analytic description (the Sparse-vDiT skill page, "CUDA
 * kernel invocation (pseudo-code)", dispatches pattern-specialised kernels;
 * the Compact Attention abstract's tile-aligned windows; the radial rule of
 * the "Radial Attention" skill page, Step 1, and the thismoment.ai blog, "How
 * Radial Attention Works"). Only the row lengths are computed first (the
 * builders' count pass), for the work order and the softmax; no column list
 * exists. Results are bit-identical to bsa_attn_fwd on the lists that
 * bsa_tile_pattern_lists_build / bsa_joint_mask_build would build. Block
 * 128; q, k, v, out contiguous bf16 [batch, heads, n, head_dim] as for
 * bsa_attn_fwd, lse fp32 [batch, heads, n] or NULL; other limits and errors
 * as bsa_attn_fwd. Asynchronous.
 */

/* Bytes of device scratch bsa_attn_fwd_patterns needs (row lengths, work
 * order, work counter); 0 for invalid arguments. */
size_t bsa_attn_fwd_patterns_workspace_bytes(int32_t num_patterns, int32_t num_q_blocks);

/*
 * Per-head tile patterns generated in the kernel. patterns: device array of
 * num_patterns descriptors (as for bsa_tile_pattern_lists_build, whose
 * columns array and num_columns they index). head_pattern: device int32
 * [heads], the pattern of each head (heads sharing a pattern share one set of
 * row lengths and one work order: Sparse-vDiT's head fusion), or NULL when
 * num_patterns is 1 (every head) or heads (head h uses pattern h); entries are
 * clamped into [0, num_patterns). num_patterns in [1, 4096]. A malformed
 * descriptor or out-of-range column is reported through
 * bsa_get_device_status() (BSA_ERR_INVALID_ARG), as by the list builder.
 */
int bsa_attn_fwd_patterns(const void *q, const void *k, const void *v,
                          int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                          float softmax_scale, int32_t num_patterns,
                          const bsa_tile_pattern *patterns, const int32_t *columns,
                          int64_t num_columns, const int32_t *head_pattern,
                          void *out, float *lse, void *workspace, size_t workspace_bytes,
                          bsa_stream_t stream);

/* Bytes of device scratch bsa_attn_fwd_radial needs; 0 for invalid
 * arguments. */
size_t bsa_attn_fwd_radial_workspace_bytes(int32_t frames, int32_t tokens_per_frame,
                                           int32_t text_tokens);

/*
 * The joint radial mask (bsa_joint_mask_build's rule; text_tokens = 0 is the
 * plain radial mask) generated in the kernel, shared by every head:
 * n = frames * tokens_per_frame + text_tokens. tokens_per_frame at most
 * 8063 (a key frame then touches at most 64 key blocks, the generator's
 * window), BSA_ERR_UNSUPPORTED beyond.
 */
int bsa_attn_fwd_radial(const void *q, const void *k, const void *v,
                        int32_t batch, int32_t heads, int32_t frames,
                        int32_t tokens_per_frame, int32_t text_tokens, int32_t head_dim,
                        float softmax_scale, void *out, float *lse, void *workspace,
                        size_t workspace_bytes, bsa_stream_t stream);

/*
 * Bytes of device scratch bsa_attn_fwd_varlen needs (the per-item work order
 * and the work counter; for block-64 lists also the items' 128-row tile
 * lists: offsets, entries and quarter masks); 0 for invalid arguments.
 */
size_t bsa_attn_fwd_varlen_workspace_bytes(int32_t num_items, const int32_t *cu_seqlens,
                                           int32_t heads, const bsa_block_lists *lists);

/*
 * bsa_attn_fwd's operation on a variable-length batch in one launch: the
 * items' tokens are packed one after another, item b owning tokens
 * [cu_seqlens[b], cu_seqlens[b+1]) of q, k, v and out, and attention runs
 * inside each item only, over that item's block lists (the pages treat one
 * sequence at a time; batching sequences of different lengths is this
 * library's reading).
 * q, k, v, out  device bf16 views of [1, heads, total, head_dim] described by
 *        their bsa_layout (batch_stride unused), total = cu_seqlens[num_items];
 *        e.g. packed [total, heads, head_dim] (token_stride = heads*head_dim,
 *        head_stride = head_dim) or [heads, total, head_dim]. Layout rules as
 *        bsa_attn_fwd_strided. Every element must be finite (an item's last
 *        key block may read the next item's tokens, which enter with weight 0).
 * num_items, cu_seqlens  number of items in [1, 64] and a host array of
 *        num_items + 1 token offsets: cu_seqlens[0] = 0, non-decreasing, total
 *        >= 1 (empty items are allowed).
 * lists  the items' lists concatenated as bsa_joint_mask_build_varlen writes
 *        them: block 64 or 128; num_q_blocks = sum_b ceil(n_b / block);
 *        num_k_blocks = max_b ceil(n_b / block); num_lists 1 (each item's list
 *        shared by its heads) or heads (item b's rows hold its lists for heads
 *        0..heads-1, one after another, nqb_b rows each); column indices count
 *        key blocks inside the item. Block-64 lists run, item by item, as
 *        128-row tiles with a mask of their listed 64 x 64 quarters (built in
 *        the workspace), like bsa_attn_fwd's.
 * lse    device fp32 [heads, total] (natural log, -inf for a row without
 *        keys), or NULL.
 * workspace  bsa_attn_fwd_varlen_workspace_bytes() bytes of device scratch.
 * Results for each item equal bsa_attn_fwd on that item alone, bit for bit.
 * Returns BSA_ERR_UNSUPPORTED for a block other than 64 / 128 or head_dim
 * other than 64 / 128; other errors as bsa_attn_fwd. Asynchronous.
 */
int bsa_attn_fwd_varlen(const void *q, const bsa_layout *q_layout,
                        const void *k, const bsa_layout *k_layout,
                        const void *v, const bsa_layout *v_layout,
                        int32_t num_items, const int32_t *cu_seqlens,
                        int32_t heads, int32_t head_dim, float softmax_scale,
                        const bsa_block_lists *lists,
                        void *out, const bsa_layout *out_layout, float *lse,
                        void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Bytes of device scratch bsa_attn_module_fwd needs: the projected q/k/v
 * [batch*n, 3*heads*head_dim] bf16, the attention output [batch*n,
 * heads*head_dim] bf16, its lse and the attention's work order. Returns 0
 * for invalid arguments.
 */
size_t bsa_attn_module_workspace_bytes(int32_t batch, int32_t n, int32_t heads,
                                       int32_t head_dim, const bsa_block_lists *lists);

/*
 * The radial attention module forward ("Radial Attention" skill page, Step 2,
 * RadialAttention.forward):
 *   q, k, v = q_proj(x), k_proj(x), v_proj(x), split into heads;
 *   o = block-sparse attention of q, k, v (bsa_attn_fwd's operation);
 *   y = out_proj(o with the heads merged back).
 * With C = heads * head_dim:
 * x      device bf16 [batch, n, C], row-major.
 * w_qkv  device bf16 [3C, C]: rows [0, C) q_proj.weight, [C, 2C)
 *        k_proj.weight, [2C, 3C) v_proj.weight (nn.Linear's [out, in]).
 * b_qkv  device bf16 [3C] (the three biases in the same order), or NULL.
 * w_out  device bf16 [C, C] out_proj.weight; b_out bf16 [C] or NULL.
 * y      device bf16 [batch, n, C]; must not overlap x, the weights or the
 *        workspace.
 * workspace  device scratch of bsa_attn_module_workspace_bytes(); the
 *        projected q/k/v, the attention output and its lse stay there after
 *        the call (bsa_attn_module_bwd reads them).
 * Head h of the split is columns [h*head_dim, (h+1)*head_dim) of each
 * projection (the page's view(batch, n, heads, head_dim)). The projections
 * run on the library's tcgen05 GEMM (bsa_gemm_bf16: bf16 in, fp32
 * accumulate, bias in the epilogue, bf16 out); the attention reads q, k, v in
 * place from the projection output and
 * writes o in [batch, n, heads, head_dim] order, out_proj's input layout, so
 * no transpose runs. Pointers 16-byte aligned; other limits and errors as
 * bsa_attn_fwd. Asynchronous.
 */
int bsa_attn_module_fwd(const void *x, const void *w_qkv, const void *b_qkv,
                        const void *w_out, const void *b_out,
                        int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                        float softmax_scale, const bsa_block_lists *lists, void *y,
                        void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Bytes of device scratch bsa_attn_module_bwd needs: the attention output's
 * gradient [batch*n, C] and the q/k/v gradients [batch*n, 3C] (bf16), the
 * attention backward's workspace and the bias-gradient partial sums. Returns
 * 0 for invalid arguments.
 */
size_t bsa_attn_module_bwd_workspace_bytes(int32_t batch, int32_t n, int32_t heads,
                                           int32_t head_dim, const bsa_block_lists *lists);

/*
 * Backward of bsa_attn_module_fwd: given dy = dL/dy (bf16 [batch, n, C]),
 * the gradients of x and of the four nn.Linear layers' weights and biases
 * (the LoRA fine-tuning of the "Radial Attention" skill page, Step 4, runs
 * loss.backward() through this module). With the forward's A = the attention
 * output, heads merged ([batch*n, C]) and QKV = the stacked projection:
 *   dA = dy w_out,            dw_out = dy^T A,        db_out = column sums of dy,
 *   dQKV = attention backward (bsa_attn_bwd's operation) of dA, laid out as
 *          QKV's q / k / v column slices,
 *   dw_qkv = dQKV^T x,        db_qkv = column sums of dQKV,   dx = dQKV w_qkv.
 * x, w_qkv, w_out, lists, softmax_scale: exactly as given to the forward.
 * fwd_workspace: the forward call's workspace, unchanged since (q/k/v, A and
 *   lse are read from it).
 * dx [batch, n, C], dw_qkv [3C, C], dw_out [C, C]: bf16 outputs; db_qkv [3C]
 *   and db_out [C]: bf16 outputs or NULL (not computed). No output may
 *   overlap an input, a workspace or another output.
 * workspace: bsa_attn_module_bwd_workspace_bytes() of device scratch.
 * GEMMs on the library's tcgen05 GEMM (bsa_gemm_bf16: bf16 in, fp32
 * accumulate, bf16 out; each output element is summed in one fixed order);
 * bias gradients by a fixed-order two-pass column sum (fp32), so the whole
 * backward is deterministic. 16-byte aligned pointers; limits and errors as bsa_attn_bwd.
 * Asynchronous.
 */
int bsa_attn_module_bwd(const void *x, const void *w_qkv, const void *w_out, const void *dy,
                        int32_t batch, int32_t n, int32_t heads, int32_t head_dim,
                        float softmax_scale, const bsa_block_lists *lists,
                        const void *fwd_workspace, size_t fwd_workspace_bytes,
                        void *dx, void *dw_qkv, void *db_qkv, void *dw_out, void *db_out,
                        void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Dense bf16 matrix product of the module's linear layers ("Radial Attention"
 * skill page, Step 2: q_proj, k_proj, v_proj and out_proj are nn.Linear
 * layers, y = x W^T + b; the backward multiplies by W and by the transposed
 * activations):
 *   D[m, n] = A[m, k] B[k, n] (+ bias[n] on every row),
 * bf16 operands, fp32 accumulation on the tensor cores (tcgen05, TMEM
 * accumulators), rounded to bf16 once on output.
 * a, lda, a_mn_major  A stored row-major as [m][k] (a_mn_major = 0, row stride
 *        lda >= k) or as its transpose [k][m] (a_mn_major = 1, lda >= m).
 * b, ldb, b_mn_major  B stored as [n][k] (b_mn_major = 0, ldb >= k: an
 *        nn.Linear weight [out, in], giving x W^T) or as [k][n]
 *        (b_mn_major = 1, ldb >= n).
 * bias   device bf16 [n] or NULL.
 * d, ldd device bf16 output [m][n], row stride ldd >= n; must not overlap a,
 *        b or bias.
 * Device pointers 16-byte aligned; lda, ldb, ldd and n multiples of 8;
 * m, n, k in [1, 2^31 - 256]. Every output element is the sum over k in one
 * fixed order (results are reproducible bit for bit). Returns
 * BSA_ERR_INVALID_ARG for bad arguments (nothing launched),
 * BSA_ERR_UNSUPPORTED on a device other than sm_100, BSA_ERR_CUDA on a launch
 * error; a device-side wait that runs out is reported through
 * bsa_get_device_status(). Asynchronous on `stream`.
 */
int bsa_gemm_bf16(const void *a, int64_t lda, int32_t a_mn_major,
                  const void *b, int64_t ldb, int32_t b_mn_major,
                  const void *bias, void *d, int64_t ldd,
                  int64_t m, int64_t n, int64_t k, bsa_stream_t stream);

/*
 * Same operation, same arguments (no workspace), computed by a plain fp32
 * CUDA-core kernel that scores every key of every listed block with scalar
 * arithmetic. It is the full-tensor checker for sizes where the CPU oracle
 * can only sample rows. Asynchronous.
 */
int bsa_attn_dense_masked_ref(const void *q, const void *k, const void *v,
                              int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                              float softmax_scale, const bsa_block_lists *lists,
                              void *out, float *lse, bsa_stream_t stream);

/*
 * Backward pass of bsa_attn_fwd: the gradients dq, dk, dv of the attention
 * output with respect to q, k and v, given the output's gradient dout. The
 * pages fine-tune the radial attention module with LoRA for longer
 * sequences ("Radial Attention" skill page, Step 4, `loss.backward()`);
 * this is the derivative of the forward definition, which the pages do not
 * print:
 *   P = softmax(Q K^T * scale over the listed blocks),  dV = P^T dO,
 *   dP = dO V^T,  delta_i = sum_d dO_id O_id,  dS = P * (dP - delta),
 *   dQ = dS K * scale,  dK = dS^T Q * scale.
 *
 * Arguments: q, k, v, out (the forward's output) and dout: bf16
 * [batch, heads, n, head_dim] contiguous, 16-byte aligned device pointers; lse:
 * the forward's fp32 [batch, heads, n] log-sum-exp (required); lists and
 * softmax_scale exactly as given to the forward call; dq, dk, dv: bf16
 * [batch, heads, n, head_dim] outputs, 16-byte aligned, written in full (rows
 * of query blocks with no key block get dq = 0, keys no query block lists get
 * dk = dv = 0), and not overlapping any input. workspace: device scratch of
 * at least bsa_attn_bwd_workspace_bytes() bytes, 16-byte aligned, owned by the
 * caller. Supported: block 64 or 128, head_dim 64 or 128 (block-64 lists
 * run as 128-row tiles with a mask of the listed 64 x 64 quarters).
 * Two kernels: dK/dV per key block, then dQ per query block (which
 * recomputes S and dP). Deterministic: every output row is written by one
 * CTA, no atomics. Asynchronous on `stream`; device timeouts are reported
 * through bsa_get_device_status(). Returns BSA_OK or an argument / CUDA error.
 */
int bsa_attn_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
                 const float *lse, int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                 float softmax_scale, const bsa_block_lists *lists, void *dq, void *dk, void *dv,
                 void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * bsa_attn_bwd on strided views (bsa_layout, as for bsa_attn_fwd_strided):
 * the same gradients, with q, k, v, out, dout read and dq, dk, dv written
 * through their strides (the kernels' TMA descriptors and stores carry
 * them), so the gradients of a fused projection's q / k / v slices land in
 * one [batch, n, 3, heads, head_dim] buffer without a transpose. lse stays
 * [batch, heads, n] contiguous.
 * Layout rules (BSA_ERR_INVALID_ARG otherwise): those of
 * bsa_attn_fwd_strided for every view; each gradient's rows pairwise
 * disjoint; the gradients share no element with each other (disjoint spans,
 * or identical token-major layouts offset inside a token row by at least the
 * row's head footprint, like three column slices of one buffer) and their
 * spans overlap no input span, lse or the workspace. Workspace, limits,
 * determinism and errors as bsa_attn_bwd. Asynchronous.
 */
int bsa_attn_bwd_strided(const void *q, const bsa_layout *q_layout,
                         const void *k, const bsa_layout *k_layout,
                         const void *v, const bsa_layout *v_layout,
                         const void *out, const bsa_layout *out_layout,
                         const void *dout, const bsa_layout *dout_layout,
                         const float *lse, int32_t batch, int32_t heads, int32_t n,
                         int32_t head_dim, float softmax_scale, const bsa_block_lists *lists,
                         void *dq, const bsa_layout *dq_layout,
                         void *dk, const bsa_layout *dk_layout,
                         void *dv, const bsa_layout *dv_layout,
                         void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Bytes of device scratch bsa_attn_bwd_varlen needs: lse * log2(e) and delta
 * for every item's query rows padded to whole 128-row blocks, per head (2 x 4
 * bytes each), the transposed lists of all items (num_lists * sum_b nt_b + 1
 * offsets, nnz entries; nt_b = ceil(n_b / 128)) and two work counters; for
 * block-64 lists also the items' tile lists and one mask byte per tile and
 * per transposed entry. 0 for invalid arguments.
 */
size_t bsa_attn_bwd_varlen_workspace_bytes(int32_t num_items, const int32_t *cu_seqlens,
                                           int32_t heads, const bsa_block_lists *lists);

/*
 * bsa_attn_bwd on a variable-length batch packed as for bsa_attn_fwd_varlen:
 * item b owns tokens [cu_seqlens[b], cu_seqlens[b+1]) of q, k, v, out, dout,
 * dq, dk and dv, and its gradients are those of bsa_attn_bwd on that item
 * alone with its own lists (the pages treat one sequence at a time; batching
 * sequences of different lengths is this library's reading).
 * q, k, v, out, dout, dq, dk, dv  device bf16 views of [1, heads, total,
 *        head_dim] (batch_stride unused), total = cu_seqlens[num_items]; layout
 *        rules as bsa_attn_bwd_strided with batch 1 and n = total.
 * lse    the forward's fp32 [heads, total] log-sum-exp (required), as
 *        bsa_attn_fwd_varlen writes it.
 * num_items, cu_seqlens, lists  as for bsa_attn_fwd_varlen (block 64 or 128;
 *        block-64 lists run as 128-row tiles with quarter masks, like
 *        bsa_attn_bwd's).
 * workspace  bsa_attn_bwd_varlen_workspace_bytes() bytes of device scratch,
 *        16-byte aligned, overlapping no view and not lse.
 * Per item a prep launch (delta, lse * log2(e)) and the item's columns of
 * the transposed lists (count, fill; one scan over all items between them),
 * then ONE dK/dV and ONE dQ launch serve every item (their work items are
 * (item, head, block), decoded from a per-item table). Tokens of empty items
 * are not touched. Each item's gradients are bit-identical to bsa_attn_bwd
 * on that item alone. Every element of the views must be finite (an item's
 * last blocks read the next item's tokens, which enter with weight 0).
 * Deterministic. Returns BSA_ERR_UNSUPPORTED for a block other than 64 /
 * 128 or head_dim other than 64 / 128; other errors as bsa_attn_bwd_strided.
 * Asynchronous.
 */
int bsa_attn_bwd_varlen(const void *q, const bsa_layout *q_layout,
                        const void *k, const bsa_layout *k_layout,
                        const void *v, const bsa_layout *v_layout,
                        const void *out, const bsa_layout *out_layout,
                        const void *dout, const bsa_layout *dout_layout,
                        const float *lse, int32_t num_items, const int32_t *cu_seqlens,
                        int32_t heads, int32_t head_dim, float softmax_scale,
                        const bsa_block_lists *lists,
                        void *dq, const bsa_layout *dq_layout,
                        void *dk, const bsa_layout *dk_layout,
                        void *dv, const bsa_layout *dv_layout,
                        void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Workspace bytes bsa_attn_bwd needs: per query row of every (batch, head),
 * lse * log2(e) and delta, padded to whole 128-row tiles (2 x 4 bytes), plus
 * the transposed lists (num_lists * ceil(n / 128) + 1 offsets, nnz entries);
 * at block 64 also the 128-row tile lists (offsets, entries) and one mask
 * byte per tile and per transposed entry. 0 when the arguments are invalid.
 */
size_t bsa_attn_bwd_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                    const bsa_block_lists *lists);

/*
 * Bytes of device scratch bsa_attn_bwd_one_pass needs: bsa_attn_bwd's, plus
 * each transposed entry's position in its query row (nnz ints), four dQ part
 * counters per (batch, head, query block) and an fp32 dQ accumulator row of
 * 128 floats per padded query row (512 bytes: the largest head_dim). 0 for
 * invalid arguments or block 64.
 */
size_t bsa_attn_bwd_one_pass_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                             const bsa_block_lists *lists);

/*
 * bsa_attn_bwd's gradients from ONE kernel (block 128): per (batch*head, key
 * block) it computes S, dP, dV, dK and this key block's part of dQ for each
 * listed query block once (five block products per listed pair instead of
 * seven), and the dQ parts of a query block are added in the order of its
 * row's key blocks: a counter per (query block, 32 rows) admits them one by
 * one into an fp32 accumulator row in the workspace, the last part writes
 * dq. Deterministic (the same sum in the same order on every call); dk, dv
 * are bit-identical to bsa_attn_bwd, dq equal up to rounding order. On a B200
 * it is slower than bsa_attn_bwd on the radial workloads: the ordered dQ
 * parts are 64 KB of fp32 per listed block pair through L2 (measured on Wan:
 * 84.8 ms against 32.5 ms; 50.1 ms with unordered atomic adds, 27.7 ms
 * without any dQ accumulation). Lists must be well formed
 * (bsa_validate_lists): with a duplicated or out-of-range entry a row's
 * counter may never reach a part's turn and the call ends with
 * BSA_ERR_DEVICE_TIMEOUT after the wait limit. Arguments as bsa_attn_bwd,
 * workspace bsa_attn_bwd_one_pass_workspace_bytes(); BSA_ERR_UNSUPPORTED for
 * block 64. Asynchronous.
 */
int bsa_attn_bwd_one_pass(const void *q, const void *k, const void *v, const void *out,
                          const void *dout, const float *lse, int32_t batch, int32_t heads,
                          int32_t n, int32_t head_dim, float softmax_scale,
                          const bsa_block_lists *lists, void *dq, void *dk, void *dv,
                          void *workspace, size_t workspace_bytes, bsa_stream_t stream);

/*
 * Bytes of device workspace bsa_attn_bwd_host needs: device copies of q, k,
 * v, out, dout, lse, dq, dk and dv plus bsa_attn_bwd's own scratch for the
 * largest head group. Returns 0 for invalid arguments.
 */
size_t bsa_attn_bwd_host_workspace_bytes(int32_t batch, int32_t heads, int32_t n,
                                         int32_t head_dim, const bsa_block_lists *lists);

/*
 * bsa_attn_bwd on HOST buffers: q_host, k_host, v_host, out_host, dout_host
 * (bf16 [batch, heads, n, head_dim], contiguous) and lse_host (float
 * [batch, heads, n], required) are copied to the device, the backward runs,
 * and dq_host, dk_host, dv_host (bf16, same layout; not overlapping any
 * input) are copied back. Head groups and streams as bsa_attn_fwd_host:
 * group g's inputs are copied in on an internal stream while group g-1's
 * backward runs on `stream` (one bsa_attn_bwd call per group, on that
 * group's heads and lists) and group g-2's gradients are copied out on a
 * second internal stream. The gradients are bit-identical to one
 * bsa_attn_bwd call on the whole problem: every (batch, head) slice is
 * computed by the same kernels in the same order either way.
 * lists        device lists as for bsa_attn_bwd (built, or enqueued on
 *              `stream` before this call).
 * workspace    device memory of bsa_attn_bwd_host_workspace_bytes(),
 *              256-byte aligned; holds the device copies.
 * Asynchronous, with the same rules as bsa_attn_fwd_host: host buffers stay
 * valid and the gradients unread until `stream` has been synchronised; calls
 * of both host entries are serialised on the internal streams. Errors as
 * bsa_attn_bwd; an error from a group's launch is returned after the groups
 * before it were enqueued (their results are then incomplete).
 */
int bsa_attn_bwd_host(const void *q_host, const void *k_host, const void *v_host,
                      const void *out_host, const void *dout_host, const float *lse_host,
                      int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                      float softmax_scale, const bsa_block_lists *lists, void *dq_host,
                      void *dk_host, void *dv_host, void *workspace, size_t workspace_bytes,
                      bsa_stream_t stream);

/*
 * Check `lists`: row_ptr starts at 0, is non-decreasing and ends at nnz; each
 * row is strictly increasing and in [0, num_k_blocks). Reads no col_idx entry
 * at or beyond nnz. Synchronises `stream`. Returns BSA_OK, BSA_ERR_BAD_LISTS
 * or BSA_ERR_INVALID_ARG (null pointers, sizes out of range).
 */
int bsa_validate_lists(const bsa_block_lists *lists, bsa_stream_t stream);

/*
 * Synchronise `stream`, then return and clear the current device's status
 * word (BSA_OK, BSA_ERR_DEVICE_TIMEOUT, BSA_ERR_BAD_LISTS or BSA_ERR_CAPACITY).
 */
int bsa_get_device_status(bsa_stream_t stream);

/*
 * Where the first device-side wait that ran out gave up, for diagnosis:
 * out4[0] role (1 producer, 2 MMA issuer, 3 softmax), out4[1] barrier id,
 * out4[2] pipeline counter, out4[3] CTA index. Synchronous; not cleared by
 * bsa_get_device_status().
 */
int bsa_get_timeout_detail(int32_t *out4);

/* Static description of a status code. */
const char *bsa_status_string(int status);

/* Text of the last CUDA error seen by this thread in the library ("" if none). */
const char *bsa_last_cuda_error(void);

/*
 * Test hooks. `wait_limit_ns` bounds every device-side wait of bsa_attn_fwd
 * (0 restores the default of 2 s). `fault_flags` bit 0 makes the next
 * bsa_attn_fwd launch skip its first K-tile load, so that the consumer's
 * bounded wait runs out and the call reports BSA_ERR_DEVICE_TIMEOUT through
 * bsa_get_device_status(); the flag clears itself after one launch.
 * `fault_flags` bit 1 (sticky until the next call) runs every problem on the
 * one-tile kernel instead of the two-tile kernel (block 128 directly, block
 * 64 without packing its blocks into 128-row tiles), so that tests can compare
 * the two schedules; it changes no result beyond rounding order.
 */
int bsa_set_test_hooks(int64_t wait_limit_ns, int32_t fault_flags);

/*
 * Self-test of the exponentials the attention softmax uses. For each of the n
 * (even) device floats x, writes 2^x from the FMA-pipe polynomial path
 * (y_poly), from the hardware ex2.approx path (y_mufu) and from CUDA's exp2f
 * (y_ref). Not part of the computation; used by the tests to bound the
 * polynomial's error. Asynchronous.
 */
int bsa_selftest_exp2(const float *x, float *y_poly, float *y_mufu, float *y_ref, int32_t n,
                      bsa_stream_t stream);

/*
 * Allocation-free variant of bsa_attn_fwd. The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory, such as a
 * plugin that its host framework hands only input and output buffers and no
 * allocator, or a runtime whose memory plan is fixed at start-up and forbids
 * later allocations. Those callers cannot provide bsa_attn_fwd's workspace.
 *
 * Same operation, arguments and results as bsa_attn_fwd, minus the workspace
 * (block-64 problems run on the one-tile kernel here, without the tile
 * lists that would need more scratch):
 * the scratch it needs (the longest-first work order and the work counter)
 * lives in a fixed array compiled into the library, of
 * BSA_NOALLOC_MAX_ORDER_ENTRIES + 64 int32 entries (256 KiB + 256 B). The work
 * order takes one int32 per query block per list at block 64 and one per pair
 * of query blocks (ceil(num_q_blocks / 2) per list) at block 128; the limit
 * below is checked against the larger of the two, so at block 128 it is
 * conservative by a factor of two. Every GPU that loads the library holds
 * that array until the process exits.
 *
 * - Returns BSA_ERR_SCRATCH_LIMIT, launching nothing, when
 *   lists->num_lists * lists->num_q_blocks exceeds the maximum.
 * - Calls no cudaMalloc, cudaFree or other allocating routine.
 * - The first call on each device resolves the array's device address
 *   (cudaGetSymbolAddress) with that device current and keeps it for the
 *   rest of the process; make that first call before any stream capture.
 *   A device reset (cudaDeviceReset) unloads the library's device code and
 *   leaves the kept address stale: do not call this entry point on a device
 *   after resetting it in the same process.
 * - All calls share the one array and each call overwrites the entries it
 *   uses (nothing in it has to start at zero). Calls whose kernels overlap on
 *   the GPU (for example on two streams at once) race on it; serialise them.
 */
#define BSA_NOALLOC_MAX_ORDER_ENTRIES 65536
int bsa_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                         int32_t batch, int32_t heads, int32_t n, int32_t head_dim,
                         float softmax_scale, const bsa_block_lists *lists,
                         void *out, float *lse, bsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
