/*
 * msa.h -- C ABI of the MiniMax Sparse Attention (MSA) hot path on B200
 * (sm_100a).
 *
 * The method (page "MSA 稀疏注意力三国杀：NSA / DSA / MoBA / MSA 四方案深度对比",
 * section "MSA 架构：粗筛 + 精算"; page "稀疏注意力速览（Sparse Attention，
 * 2019 ~ 2026）", section 4, entry
 * "MiniMax Sparse Attention (MSA)"):
 *   1. an index branch scores every causal (query, key token) pair with one
 *      index query head per GQA group and a shared index key head;
 *   2. token scores are max-pooled over 128-token KV blocks and each query
 *      keeps 16 blocks per group, its own block always among them;
 *   3. the main branch runs exact softmax attention over the 16 x 128 = 2048
 *      selected tokens.
 * Step 3 runs KV-block-outer ("Kernel 创新：Outer Gather Q" section of the
 * first page): each selected KV block is read once and every query row that
 * chose it is gathered into one tensor-core tile; the per-(query, block)
 * softmax pieces are then merged by log-sum-exp.
 *
 * Beside the path: an 8-bit (e4m3) index branch, the selection recall / KL
 * alignment target of the index branch, token-level selection at the same
 * key budget, and the backward of the attention (dq, dk, dv) for training
 * through the sparse attention.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer.  The library never allocates, frees or synchronises; each call
 *     validates its arguments on the host, then enqueues its kernels on
 *     `stream` (a cudaStream_t; NULL = legacy default stream) and returns.
 *   - A non-OK status is returned before anything is enqueued, except
 *     MSA_ERR_CUDA, which reports a launch error.
 *   - `dev_err` (may be NULL) is a device int32 the caller zeroes; a kernel
 *     that detects a problem at run time (an out-of-range block id, a wait
 *     that ran past its time limit) stores an MSA_DEVERR_* code there and
 *     returns early.  Nothing traps.
 *   - Results are deterministic: bit-identical from run to run.
 *   - Fixed sizes: block B_k = 128 tokens, top-k = 16 blocks (own included),
 *     head_dim = 128, d_idx in {64, 128}.
 *   - Layouts are given as [outer, ..., inner]; the innermost dimension is
 *     contiguous, the other strides are element strides in msa_tensor.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#define MSA_BLOCK_TOKENS 128
#define MSA_TOPK_BLOCKS 16
#define MSA_HEAD_DIM 128

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,        /* null pointer, bad size, inconsistent dims */
  MSA_ERR_UNSUPPORTED = 2,        /* valid but not implemented (e.g. d_idx 96) */
  MSA_ERR_ALIGNMENT = 3,          /* pointer or stride not 16-byte aligned (32 where
                                     an entry point says so) */
  MSA_ERR_WORKSPACE_TOO_SMALL = 4,
  MSA_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
  MSA_ERR_SCRATCH_LIMIT = 6       /* needs more than the built-in scratch of the
                                     allocation-free entry point */
} msa_status;

/* device-side error codes written to *dev_err */
#define MSA_DEVERR_TIMEOUT 1      /* a bounded wait on a barrier ran out */
#define MSA_DEVERR_BAD_BLOCK 2    /* a selected block id outside [0, own] */
#define MSA_DEVERR_BAD_ENTRY 3    /* a block->query entry or entry position out of range */

/* Problem sizes.  Query i of batch b sits at absolute position
 * t = q_pos0 + i and may attend keys j <= t; keys are 0 .. n_kv-1 and
 * q_pos0 + n_q <= n_kv.  Prefill: q_pos0 = 0, n_q = n_kv.  Decode: n_q = 1,
 * q_pos0 = n_kv - 1.  Chunked prefill: q_pos0 = length of the cached prefix.
 * G = h_kv GQA groups; h_q / h_kv query heads per group (a power of two
 * <= 128); head h belongs to group h / (h_q / h_kv).  h_kidx is 1 (one index
 * key head shared by all groups) or h_kv (one per group).  scale multiplies
 * q.k in the main branch (1/sqrt(128) for the textbook softmax).
 * q_window is a layout choice of the block->query lists, not of the method:
 * the query indices are cut into windows of q_window consecutive queries
 * and each block's list is split by window (see msa_build_block_query_lists).
 * 0 selects the default (msa_query_window); otherwise a positive multiple of
 * 128.  Results other than the lists' layout do not depend on it. */
typedef struct {
  int64_t batch, n_q, n_kv, q_pos0;
  int32_t h_q, h_kv, h_kidx, d_idx;
  float scale;
  int32_t q_window;
} msa_dims;

/* A strided bf16 tensor: element strides of the batch, token and head
 * dimensions; the innermost (feature) dimension is contiguous.  ptr and
 * every stride * 2 bytes must be multiples of 16 bytes. */
typedef struct {
  const void* ptr;
  int64_t s_batch, s_tok, s_head;
} msa_tensor;

/* Number of KV blocks, ceil(n_kv / 128). */
MSA_API int64_t msa_num_blocks(const msa_dims* dims);

/* Number of (query, selected block) pairs over the whole problem:
 * batch * h_kv * sum_i min(16, own(q_pos0 + i) + 1), own(t) = t / 128.
 * It sizes the `entries` array of msa_build_block_query_lists. */
MSA_API int64_t msa_num_entries(const msa_dims* dims);

/* The query window W of the block->query lists: dims->q_window when it is
 * positive, else the largest power of two W >= 128 with
 * W * (h_q / h_kv) * 256 <= 32 MiB (the bf16 query rows one window gathers
 * for one group: about a quarter of B200's L2).  0 for invalid dims. */
MSA_API int64_t msa_query_window(const msa_dims* dims);

/* Number of segments of the block->query lists,
 * batch * h_kv * ceil(n_q / W) * msa_num_blocks(dims); blk_offsets holds one
 * more value.  0 for invalid dims. */
MSA_API int64_t msa_num_segments(const msa_dims* dims);

/* Step 1+2a: index scores and causal block max-pool
 * (first page, "第一步：粗筛" items 1-2: score each token, a block's score is
 * its highest token score; "稀疏注意力速览" page, MSA entry: one index query head per
 * GQA group, shared index key head, block max-pool).
 *   q_idx  [B, n_q, G, d_idx]            bf16
 *   k_idx  [B, h_kidx, n_kv, d_idx]      bf16 (s_head = stride between index key heads)
 *   pooled [B, G, n_q, pooled_row_stride] fp32, written for every block
 *          c < own(t): pooled = max_{j in block c} sum_k q_idx[t,g,k] k_idx[j,k],
 *          accumulated in fp32 from the exact bf16 products.  Entries
 *          c >= own(t) are left untouched.  The n_q x n_kv score matrix is
 *          never stored.
 * pooled_row_stride >= msa_num_blocks(dims) and a multiple of 4. */
MSA_API msa_status msa_index_score_maxpool(const msa_dims* dims, msa_tensor q_idx, msa_tensor k_idx,
                                   float* pooled, int64_t pooled_row_stride,
                                   int32_t* dev_err, void* stream);

/* Step 2b: block selection (first page, "第一步：粗筛" item 3: 16 blocks, the
 * current position's block always taken, the rest by score; "稀疏注意力速览" page:
 * top-k per GQA group with the local block kept).
 *   pooled [B, G, n_q, pooled_row_stride] fp32 as written above
 *   sel    [B, G, n_q, 16] int32: own(t) plus the min(15, own(t)) best blocks
 *          c < own(t) ranked by (score descending, block index ascending;
 *          -0.0 equals +0.0), in ascending block order, padded with -1 to 16.
 * No other block (first block, sink, window) is forced. */
MSA_API msa_status msa_topk_blocks(const msa_dims* dims, const float* pooled, int64_t pooled_row_stride,
                           int32_t* sel, int32_t* dev_err, void* stream);

/* Bytes of device workspace msa_build_block_query_lists needs. */
MSA_API size_t msa_block_query_lists_workspace(const msa_dims* dims);

/* Step 3a: inversion of the query->block lists into block->query lists, the
 * index a KV-block-outer kernel walks (first page, "Kernel 创新：Outer Gather
 * Q": the queries that chose a block are gathered and computed together).
 * Each block's list is split by query window (W = msa_query_window(dims)
 * consecutive query indices): the attention kernel walks the segments in
 * order, so at any time it gathers the query rows of one window, which stay
 * in L2, while each K/V block is still read once per window.
 *   sel         [B, G, n_q, 16] int32 (as written by msa_topk_blocks; any
 *               valid selection works)
 *   blk_offsets [msa_num_segments(dims) + 1] int32: segment
 *               s = ((b * G + g) * nwin + w) * nblk + c, nwin = ceil(n_q / W),
 *               holds entries[blk_offsets[s] .. blk_offsets[s+1]), the
 *               queries i of window w (w * W <= i < (w + 1) * W) that chose c
 *   entries     [msa_num_entries(dims)] int32: (i << 4) | slot for each query
 *               index i (within its batch) and the slot of c in sel[b,g,i,:],
 *               ascending in i inside a segment (deterministic counting sort)
 *   entry_pos   [B, G, n_q, 16] int32 (the shape of sel): the position in
 *               entries of (b, g, i, slot), -1 for an empty slot.  The
 *               attention writes the piece of the entry at position p in
 *               piece rows p * R .. p * R + R - 1, and the merge finds it here.
 *   ws          device workspace of at least msa_block_query_lists_workspace()
 *               bytes, 16-byte aligned; contents on entry do not matter. */
MSA_API msa_status msa_build_block_query_lists(const msa_dims* dims, const int32_t* sel,
                                       int32_t* blk_offsets, int32_t* entries,
                                       int32_t* entry_pos, void* ws, size_t ws_bytes,
                                       int32_t* dev_err, void* stream);

/* Size of the device scratch array behind msa_build_block_query_lists_noalloc
 * (32 MiB per device on which that entry point has run, kept until the
 * process exits). */
#define MSA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* Allocation-free variant of msa_build_block_query_lists (the paper has no
 * counterpart: it is a convenience of this library).  It is meant for callers
 * that cannot call cudaMalloc or any allocating routine where they build the
 * lists -- e.g. a plugin inside a serving process whose host owns all device
 * memory through its own pool, or a latency-critical loop that must not
 * allocate.  Same arguments, results and status codes as
 * msa_build_block_query_lists, minus the workspace: the scratch is a
 * file-scope device array of MSA_NOALLOC_SCRATCH_BYTES, and problems needing
 * more (msa_block_query_lists_workspace(dims) > MSA_NOALLOC_SCRATCH_BYTES) are
 * rejected with MSA_ERR_SCRATCH_LIMIT before anything is enqueued.  For
 * example the 32K prefill (8 groups), the 64 x 256K decode and an 8192-query
 * chunk after a 1M-token cache fit; a 128K-token prefill with 8 groups does not.
 *   - The array is committed on a device when the library's module that holds
 *     it is loaded there.  Under CUDA's default lazy module loading that is the
 *     first call of this entry point on the device (under
 *     CUDA_MODULE_LOADING=EAGER, the creation of the context).  A host that
 *     reserves device memory for its own pool should make that first call
 *     before the reservation; otherwise the call can fail with MSA_ERR_CUDA.
 *   - The first call in a context looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current); so does the first call
 *     after the device's context changed (e.g. after cudaDeviceReset).  Make
 *     that first call before any stream capture.
 *   - Nothing is allocated or freed.  Every call shares the one array, which
 *     keeps the previous call's contents; its contents on entry do not matter
 *     (every word is written before it is read).  Calls that overlap on the
 *     GPU (on different streams without ordering) race on the array. */
MSA_API msa_status msa_build_block_query_lists_noalloc(const msa_dims* dims, const int32_t* sel,
                                                       int32_t* blk_offsets, int32_t* entries,
                                                       int32_t* entry_pos, int32_t* dev_err,
                                                       void* stream);

/* Step 3b: KV-block-outer sparse attention (first page "第二步：精算": full
 * attention over the selected blocks only; "稀疏注意力速览" page: exact softmax
 * attention; softmax(Q K^T * scale) V from the "稀疏注意力架构革命" page, section 1.1).  For every
 * segment (b, g, window, c) each K/V block is brought into shared memory once and the
 * R = h_q / h_kv head rows of every listed query are gathered into 128-row
 * tensor-core tiles.  For each list entry (query i, group g, slot) at position
 * p of entries and each head r of the group (head h = g * R + r) it writes the
 * piece over the tokens j of block c with j <= t into row p * R + r:
 *   part_ml [msa_num_entries(dims), R, 2] fp32: m = max_j scale * q.k_j,
 *                                               l = sum_j e^{scale q.k_j - m}
 *   part_acc[msa_num_entries(dims), R, 128] fp32: sum_j e^{scale q.k_j - m} v_j
 * Pieces follow the lists' order, so the rows of one 128-row tile of entries
 * are adjacent in memory and leave in a few large stores; entry_pos (from the
 * list builder) maps (b, g, i, slot) back to p.  Rows past the listed entries
 * are not written.
 * (l sums the fp32 weights e^{...}; they are rounded to bf16 only where they
 * multiply V, as in standard flash attention).  With one query per sequence
 * (n_q = 1) and R <= 8 the work runs on warp-level tiles instead; same output.
 *   q [B, n_q, h_q, 128] bf16; k, v [B, h_kv, n_kv, 128] bf16
 *   (msa_tensor strides; for k/v s_head is the stride between KV heads). */
MSA_API msa_status msa_sparse_attn_fwd(const msa_dims* dims, msa_tensor q, msa_tensor k, msa_tensor v,
                               const int32_t* blk_offsets, const int32_t* entries,
                               float* part_ml, float* part_acc,
                               int32_t* dev_err, void* stream);

/* Step 3b with compact pieces (an opt-in of this library; the pages fix no
 * piece format, and the default above keeps every piece in fp32).  Same
 * arguments and part_ml as msa_sparse_attn_fwd, but part_acc_bf16 is
 * [msa_num_entries(dims), R, 128] bf16 and holds acc / l: the piece's weighted mean
 * of the V rows, a convex combination of them, so it cannot overflow; it is
 * rounded to bf16 once.  This halves the bytes the pieces move (264 instead
 * of 520 per (query, head, block)); merge with msa_merge_partials_compact.
 * One query per sequence with h_q / h_kv <= 8 (the warp-level decode kernel)
 * returns MSA_ERR_UNSUPPORTED: use the fp32 pieces there. */
MSA_API msa_status msa_sparse_attn_fwd_compact(const msa_dims* dims, msa_tensor q, msa_tensor k,
                                               msa_tensor v, const int32_t* blk_offsets,
                                               const int32_t* entries, float* part_ml,
                                               void* part_acc_bf16, int32_t* dev_err,
                                               void* stream);

/* Step 3c: log-sum-exp merge of the pieces, in slot order:
 *   M = max_s m_s, L = sum_s l_s e^{m_s - M}, o = sum_s acc_s e^{m_s - M} / L,
 *   lse = M + ln L, over the slots s with p_s = entry_pos[b, g, i, s] >= 0,
 *   the piece of slot s and head r being row p_s * R + r of the pieces.
 *   entry_pos [B, G, n_q, 16] int32, as written by the list builder; a
 *             position >= msa_num_entries(dims) sets MSA_DEVERR_BAD_ENTRY in
 *             *dev_err and counts as an empty slot
 *   out [B, n_q, h_q, 128] bf16 contiguous; lse [B, n_q, h_q] fp32. */
MSA_API msa_status msa_merge_partials(const msa_dims* dims, const int32_t* entry_pos,
                              const float* part_ml, const float* part_acc,
                              void* out, float* lse, int32_t* dev_err, void* stream);

/* Step 3c on compact pieces (msa_sparse_attn_fwd_compact): with
 * accn_s = part_acc_bf16 of slot s, o = sum_s l_s e^{m_s - M} accn_s / L and
 * lse as in msa_merge_partials. */
MSA_API msa_status msa_merge_partials_compact(const msa_dims* dims, const int32_t* entry_pos,
                                              const float* part_ml, const void* part_acc_bf16,
                                              void* out, float* lse, int32_t* dev_err,
                                              void* stream);

/* Backward of step 3b/3c for training through the sparse attention ("MSA 稀疏
 * 注意力三国杀" page, section "MSA 能力不掉：3T token 对照实验": a model trained
 * with MSA from the start, MSA-PT, and a dense one converted by continued
 * training, MSA-CPT; section "索引分支训练：KL 对齐": the index branch learns
 * only through its KL term, so the selection is fixed here).  For every
 * (query t, head h) of group g and its selected causal tokens J (the same
 * block->query lists as the forward):
 *   p_j = exp(scale q.k_j - lse),  D = dO.o,  dS_j = p_j (dO.v_j - D),
 *   dq = scale sum_j dS_j k_j,  dk_j = scale sum dS_j q,  dv_j = sum p_j dO,
 * the last two summed over every (query, head) whose set holds j.
 *   q, o, d_o   [B, n_q, h_q, 128] bf16 (msa_tensor strides); o and lse are
 *               the forward's results (msa_merge_partials)
 *   k, v        [B, h_kv, n_kv, 128] bf16
 *   lse         [B, n_q, h_q] fp32
 *   delta       [B, n_q, h_q] fp32 device scratch (receives D)
 *   part_dq     [B, n_q, h_kv, 16, R, 128] fp32 device scratch (a forward
 *               piece buffer of B * n_q * h_kv * 16 rows of R x 128 fp32 may
 *               be reused; the forward itself needs msa_num_entries rows)
 *   dq          [B, n_q, h_q, 128] fp32, contiguous (its memory also holds
 *               the call's work order until the result overwrites it)
 *   dk, dv      [B, h_kv, n_kv, 128] fp32, contiguous; zeroed by the call
 *   (part_dq, dk and dv 32-byte aligned, the others 16-byte aligned:
 *   MSA_ERR_ALIGNMENT otherwise)
 * Blocks and keys that no query selected get zero gradients.  dq is summed in
 * slot order; each KV block's dk and dv are accumulated by the one block of
 * threads that owns the block (all its query windows) and stored once, so all
 * three are bit-identical from run to run.  Lists with fewer entries than the
 * sizes imply set MSA_DEVERR_BAD_ENTRY. */
MSA_API msa_status msa_sparse_attn_bwd(const msa_dims* dims, msa_tensor q, msa_tensor k,
                                       msa_tensor v, msa_tensor o, msa_tensor d_o,
                                       const float* lse, const int32_t* blk_offsets,
                                       const int32_t* entries, float* delta, float* part_dq,
                                       float* dq, float* dk, float* dv, int32_t* dev_err,
                                       void* stream);

/* 8-bit (e4m3) index branch, an opt-in variant of step 1 that the MSA pages do
 * not describe: the "推理系统基础设施手记（三）" page (sections "4. CSA：先压缩，
 * 再稀疏选择" and "8. 常见坑") reports a low-precision indexer that makes selection
 * cheap and warns that its inputs must be clamped to the format's range.
 * msa_quantize_e4m3: n bf16 values x (device, contiguous) -> n e4m3 codes
 * (device, contiguous bytes) with one per-tensor scale: amax = max |x|,
 * scale = amax / 448 (1 when amax is 0), code = e4m3 nearest to x / scale
 * (ties to even; magnitudes past 448 saturate).  scale points to 2 device
 * floats: scale[0] receives the scale, scale[1] is scratch for amax. */
MSA_API msa_status msa_quantize_e4m3(const void* x_bf16, int64_t n, void* codes, float* scale,
                                     void* stream);

/* Step 1 on e4m3 codes (d_idx = 128 only): pooled[b, g, i, c] =
 * scale_q[0] * scale_k[0] * max over keys j of block c of sum_k code_q . code_k,
 * for c < own(t), tcgen05 kind::f8f6f4 tiles.  q_idx8 [B, n_q, G, 128] and
 * k_idx8 [B, h_kidx, n_kv, 128] are uint8 codes (msa_tensor strides in bytes,
 * multiples of 16); the scales are device floats from msa_quantize_e4m3.
 * Feed `pooled` to msa_topk_blocks as usual. */
MSA_API msa_status msa_index_score_maxpool_e4m3(const msa_dims* dims, msa_tensor q_idx8,
                                                msa_tensor k_idx8, const float* scale_q,
                                                const float* scale_k, float* pooled,
                                                int64_t pooled_row_stride, int32_t* dev_err,
                                                void* stream);

/* Selection recall and the index branch's alignment target, for sampled query
 * rows ("MSA 稀疏注意力三国杀" page, section "索引分支训练：KL 对齐": the index
 * branch learns the main branch's attention distribution through a KL
 * divergence with the teacher's gradient stopped, and its chosen blocks hold
 * most of the main branch's weight; "稀疏注意力速览" page, section 4, MSA entry).
 * For sampled row rows[i] = b * n_q + qi (position t = q_pos0 + qi) and group
 * g, over blocks c = 0 .. t / 128 and keys j <= t:
 *   teacher P(c) = mean over the group's R heads of the full causal softmax
 *                  mass of block c, softmax over all j <= t of scale * q.k_j
 *   student Q(c) = softmax over c of z(c) = max_{j in c} q_idx[g] . k_idx[j]
 *   recall = sum of P over the blocks sel[b, g, qi, :] selects
 *   kl_pq = sum_c P log(P / Q), kl_qp = sum_c Q log(Q / P)
 * Outputs (device, fp32): block_mass [n_rows, G, mass_stride] (P, 0 beyond the
 * causal blocks), recall, kl_pq, kl_qp [n_rows, G], and, when lse_full is not
 * NULL, lse_full [n_rows, H]: each head's log sum_{j <= t} exp(scale * q.k_j),
 * the full causal attention's log-normaliser.  rows: device int64
 * [n_rows]; sel: [B, G, n_q, 16] as from msa_topk_blocks.  Needs R = h_q/h_kv
 * <= 8 (else MSA_ERR_UNSUPPORTED), mass_stride >= the block count, and a
 * device workspace of msa_selection_recall_workspace(dims, n_rows) bytes
 * (16-byte aligned).  A row outside [0, B * n_q) sets MSA_DEVERR_BAD_ENTRY. */
MSA_API size_t msa_selection_recall_workspace(const msa_dims* dims, int64_t n_rows);
MSA_API msa_status msa_selection_recall(const msa_dims* dims, msa_tensor q, msa_tensor k,
                                        msa_tensor q_idx, msa_tensor k_idx,
                                        const int32_t* sel, const int64_t* rows, int64_t n_rows,
                                        float* block_mass, int64_t mass_stride, float* recall,
                                        float* kl_pq, float* kl_qp, float* lse_full, void* ws,
                                        size_t ws_bytes, int32_t* dev_err, void* stream);

/* Token-level selection at the same key budget, for sampled query rows: the
 * selection granularity the pages set against MSA's 128-token blocks ("MSA 稀疏
 * 注意力三国杀" page, section "分歧一：颗粒度——token 级还是块级？"; "稀疏注意力速览"
 * page, section 4; "Sparse attention · DSA và MSA chọn vị trí" page), here with
 * MSA's own index branch as the scorer.  For sampled row rows[i] = b * n_q + qi
 * (position t = q_pos0 + qi) and group g:
 *   score(j) = q_idx[b, qi, g] . k_idx[b, g or 0, j] for every key j <= t (fp32),
 *   T = the min(budget, t + 1) keys of highest score, the lower index first
 *       among equal scores, written ascending to tokens[i, g, :] (int32,
 *       [n_rows, G, budget], -1 after the last),
 *   out[i, h] = sum_{j in T} softmax_{j in T}(scale * q_h.k_j) v_j and
 *   lse[i, h] = log sum_{j in T} exp(scale * q_h.k_j) for the group's heads h
 *   (device fp32, [n_rows, H, 128] and [n_rows, H]).
 * exp(lse - lse_full) (lse_full from msa_selection_recall) is the share of the
 * full attention mass the tokens hold, the token-level counterpart of recall.
 * budget >= 1 (2048 spends the 16 x 128 keys of the block selection); R =
 * h_q/h_kv <= 8 (else MSA_ERR_UNSUPPORTED); a device workspace of
 * msa_token_select_workspace(dims, n_rows) bytes (16-byte aligned; it holds
 * the score rows).  A row outside [0, B * n_q) sets MSA_DEVERR_BAD_ENTRY. */
MSA_API size_t msa_token_select_workspace(const msa_dims* dims, int64_t n_rows);
MSA_API msa_status msa_token_select_attention(const msa_dims* dims, msa_tensor q, msa_tensor k,
                                              msa_tensor v, msa_tensor q_idx, msa_tensor k_idx,
                                              const int64_t* rows, int64_t n_rows,
                                              int64_t budget, int32_t* tokens, float* out,
                                              float* lse, void* ws, size_t ws_bytes,
                                              int32_t* dev_err, void* stream);

/* Debug setting (the pages have no counterpart): the time limit, in
 * nanoseconds, of every barrier wait inside the kernels that
 * msa_sparse_attn_fwd and msa_sparse_attn_fwd_compact launch from now on, in
 * this process (2 s by default; 0 restores the default, larger values are
 * capped at it).  A wait that runs out stops its block: the block drains the
 * loads and tensor-core work it has in flight, frees its tensor memory,
 * stores MSA_DEVERR_TIMEOUT in *dev_err and returns, leaving the outputs
 * incomplete.  A tiny limit (e.g. 1000) makes a valid call time out, which is
 * how the tests exercise that path without a fault.  Returns the previous
 * limit.  Not thread-safe against concurrent attention calls. */
MSA_API uint64_t msa_debug_set_attn_wait_limit_ns(uint64_t ns);

/* Human-readable name of a status code (static storage). */
MSA_API const char* msa_status_string(msa_status status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
