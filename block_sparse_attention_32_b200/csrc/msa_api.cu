// C ABI of the MSA hot path: host-side argument checks, TMA tensor-map
// encoding and kernel dispatch.  Every call validates first and enqueues on
// the caller's stream; nothing here allocates, frees or synchronises.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace msa {
cudaError_t launch_index_score_prefill(const CUtensorMap&, const CUtensorMap&, int, int64_t,
                                       int64_t, int64_t, int32_t, int32_t, float*, int64_t,
                                       int32_t*, cudaStream_t);
cudaError_t launch_index_score_decode(const CUtensorMap&, const void*, int64_t, int64_t,
                                      int64_t, int64_t, int32_t, float*, int64_t, int32_t*,
                                      cudaStream_t);
cudaError_t launch_topk_blocks(const float*, int64_t, int64_t, int64_t, int64_t, int32_t*,
                               cudaStream_t);
size_t block_lists_workspace(int64_t, int64_t, int64_t, int64_t);
cudaError_t launch_block_lists(const int32_t*, int64_t, int64_t, int64_t, int64_t, int64_t,
                               int32_t*, int32_t*, int32_t*, int64_t, void*, int32_t*,
                               cudaStream_t);
cudaError_t launch_sparse_attn(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                               const CUtensorMap&, const CUtensorMap&, const void*, int64_t,
                               int64_t, int64_t, const int32_t*, const int32_t*, int64_t,
                               int64_t, int64_t, int64_t, int32_t, int32_t, int32_t, int32_t,
                               float, float*, void*, bool, int32_t*, cudaStream_t);
cudaError_t launch_sparse_attn_decode(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                      const int32_t*, const int32_t*, int64_t, int64_t, int64_t,
                                      int32_t, int32_t, int32_t, float, float*, float*, int32_t*,
                                      cudaStream_t);
size_t recall_workspace(int64_t, int32_t, int32_t, int32_t);
cudaError_t launch_selection_recall(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const int64_t*, int64_t, const void*, int64_t, int64_t,
                                    int64_t, int64_t, int64_t, int64_t, int32_t, int32_t,
                                    int32_t, int32_t, int32_t, float, const int32_t*, float*,
                                    int64_t, float*, float*, float*, float*, void*, int32_t*,
                                    cudaStream_t);
cudaError_t launch_sparse_attn_bwd(const CUtensorMap&, const CUtensorMap&, const void*, int64_t,
                                   int64_t, int64_t, const void*, int64_t, int64_t, int64_t,
                                   const void*, int64_t, int64_t, int64_t, const float*,
                                   const int32_t*, const int32_t*, int64_t, int64_t, int64_t,
                                   int64_t, int64_t, int32_t, int32_t, int32_t, int32_t, float,
                                   float*, float*, float*, float*, float*, int32_t*,
                                   cudaStream_t);
size_t token_select_workspace(int64_t, int32_t, int64_t);
cudaError_t launch_token_select_attention(const CUtensorMap&, const int64_t*, int64_t,
                                          const void*, int64_t, int64_t, int64_t, const void*,
                                          int64_t, int64_t, int64_t, const void*, int64_t,
                                          int64_t, int64_t, const void*, int64_t, int64_t,
                                          int64_t, int64_t, int64_t, int64_t, int64_t, int32_t,
                                          int32_t, int32_t, int32_t, float, int64_t, int32_t*,
                                          float*, float*, void*, int32_t*, cudaStream_t);
cudaError_t launch_index_score_e4m3(const CUtensorMap&, const CUtensorMap&, int64_t, int64_t,
                                   int64_t, int32_t, int32_t, float*, int64_t, const float*,
                                   const float*, int32_t*, cudaStream_t);
cudaError_t launch_quantize_e4m3(const void*, int64_t, void*, float*, cudaStream_t);
uint64_t set_attn_wait_limit(uint64_t);
cudaError_t launch_merge(const int32_t*, const float*, const void*, bool, void*, float*,
                         int64_t, int64_t, int32_t, int32_t, int64_t, int32_t*, cudaStream_t);
}  // namespace msa

namespace {

constexpr int64_t kMaxBlocks = 50000;   // shared-memory histogram bound of the inversion

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

// Query window of the block->query lists: dims->q_window when positive, else
// the largest power of two W >= 128 whose gathered query rows of one group,
// W * (h_q / h_kv) * 256 bytes, fit in 32 MiB (about a quarter of L2).
int64_t query_window(const msa_dims* d) {
  if (d->q_window > 0) return d->q_window;
  const int64_t R = d->h_q / d->h_kv;
  int64_t w = MSA_BLOCK_TOKENS;
  while (2 * w * R * 256 <= (int64_t(32) << 20)) w *= 2;
  return w;
}

int64_t num_windows(const msa_dims* d) {
  const int64_t w = query_window(d);
  return (d->n_q + w - 1) / w;
}

msa_status check_dims(const msa_dims* d) {
  if (d == nullptr) return MSA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_q < 1 || d->n_kv < 1 || d->q_pos0 < 0) return MSA_ERR_INVALID_ARG;
  if (d->q_pos0 + d->n_q > d->n_kv) return MSA_ERR_INVALID_ARG;
  if (d->h_kv < 1 || d->h_q < 1 || d->h_q % d->h_kv != 0) return MSA_ERR_INVALID_ARG;
  if (d->h_kidx != 1 && d->h_kidx != d->h_kv) return MSA_ERR_INVALID_ARG;
  if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return MSA_ERR_INVALID_ARG;
  const int64_t R = d->h_q / d->h_kv;
  if (!is_pow2(R) || R > 16) return MSA_ERR_UNSUPPORTED;
  if (d->d_idx != 64 && d->d_idx != 128) return MSA_ERR_UNSUPPORTED;
  const int64_t nblk = (d->n_kv + MSA_BLOCK_TOKENS - 1) / MSA_BLOCK_TOKENS;
  if (nblk > kMaxBlocks) return MSA_ERR_UNSUPPORTED;
  if (d->n_kv > (int64_t(1) << 31) - 1) return MSA_ERR_UNSUPPORTED;
  if (d->n_q > (int64_t(1) << 26)) return MSA_ERR_UNSUPPORTED;   // entries pack i << 4
  if (d->batch > 65535 || d->batch * d->h_kv > 65535) return MSA_ERR_UNSUPPORTED;
  if (d->n_q / 128 + 1 > 65535) return MSA_ERR_UNSUPPORTED;
  if (d->q_window < 0 || d->q_window % MSA_BLOCK_TOKENS != 0) return MSA_ERR_INVALID_ARG;
  if (d->batch * d->h_kv * num_windows(d) > 65535) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

msa_status check_tensor(const msa_tensor& t) {
  if (t.ptr == nullptr) return MSA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return MSA_ERR_ALIGNMENT;
  if (t.s_batch < 0 || t.s_tok < 0 || t.s_head < 0) return MSA_ERR_INVALID_ARG;
  if ((t.s_batch % 8) || (t.s_tok % 8) || (t.s_head % 8)) return MSA_ERR_ALIGNMENT;
  return MSA_OK;
}

// total (query, selected block) pairs of one (batch, group)
int64_t entries_per_bg(const msa_dims* d) {
  int64_t total = 0;
  // queries with own(t) >= 15 contribute 16; earlier ones own + 1
  const int64_t t0 = d->q_pos0, t1 = d->q_pos0 + d->n_q;   // [t0, t1)
  const int64_t full_from = 15 * MSA_BLOCK_TOKENS;           // first t with own >= 15
  const int64_t a = t0, bnd = std::min(t1, std::max(t0, full_from));
  for (int64_t t = a; t < bnd; ++t) total += t / MSA_BLOCK_TOKENS + 1;
  if (t1 > bnd) total += (t1 - bnd) * MSA_TOPK_BLOCKS;
  return total;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D bf16 map: dims {inner, d1, d2, d3} with byte strides of d1..d3, box
// {64, b1, b2, 1}, 128-byte swizzle, zero fill out of bounds.
msa_status make_map(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t d1, uint64_t d2,
                    uint64_t d3, int64_t s1, int64_t s2, int64_t s3, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (fn == nullptr) return MSA_ERR_CUDA;
  cuuint64_t dims[4] = {inner, d1, d2, d3};
  cuuint64_t strides[3] = {(cuuint64_t)s1 * 2, (cuuint64_t)s2 * 2, (cuuint64_t)s3 * 2};
  // a dimension of extent 1 still needs a legal stride
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0) strides[i] = 16;
  cuuint32_t box[4] = {64, b1, b2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

// 3-D map over the pieces' rows of 128 values (fp32: 512-byte rows; bf16:
// 256-byte rows) seen as {128 bytes of a row, rows, 128-byte panels of a row},
// box {128 bytes, box_rows, panels}: one store writes box_rows consecutive
// rows (an entry's heads) across `panels` panels, from shared memory staged
// [panel][row][128 B] with the 128-byte swizzle.
msa_status make_map_piece_rows(CUtensorMap* map, void* ptr, uint64_t rows, bool bf16,
                               uint32_t box_rows, uint32_t panels) {
  auto fn = encode_fn();
  if (fn == nullptr) return MSA_ERR_CUDA;
  const uint64_t row_bytes = bf16 ? 256 : 512;
  cuuint64_t dims[3] = {bf16 ? 64u : 32u, rows, row_bytes / 128};
  cuuint64_t strides[2] = {row_bytes, 128};
  cuuint32_t box[3] = {bf16 ? 64u : 32u, box_rows, panels};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  3, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

msa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// 5-D bf16 view of q [B, n_q, H, 128] for the attention kernel's gather: dims
// {64 columns, H heads, 2 panels of 64 columns, n_q, B} with byte strides
// {head, 128, token, batch}; box {64, 8, 2, 1, 1} = eight heads of one query,
// both panels, 2 KB, landing as [panel][8 rows][128 B] (128-byte swizzle).
msa_status make_map_q_groups(CUtensorMap* map, const msa_dims* d, const msa_tensor& q) {
  auto fn = encode_fn();
  if (fn == nullptr) return MSA_ERR_CUDA;
  cuuint64_t dims[5] = {64, (cuuint64_t)d->h_q, 2, (cuuint64_t)d->n_q, (cuuint64_t)d->batch};
  cuuint64_t strides[4] = {(cuuint64_t)q.s_head * 2, 128, (cuuint64_t)q.s_tok * 2,
                           (cuuint64_t)q.s_batch * 2};
  for (int i = 0; i < 4; ++i)
    if (strides[i] == 0) strides[i] = 16;      // a dimension of extent 1 still needs a stride
  cuuint32_t box[5] = {64, 8, 2, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(q.ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

// 4-D uint8 map (e4m3 codes): dims {inner, d1, d2, d3}, byte strides, box
// {128, b1, b2, 1}, 128-byte swizzle, zero fill out of bounds.
msa_status make_map_u8(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t d1,
                       uint64_t d2, uint64_t d3, int64_t s1, int64_t s2, int64_t s3, uint32_t b1,
                       uint32_t b2) {
  auto fn = encode_fn();
  if (fn == nullptr) return MSA_ERR_CUDA;
  cuuint64_t dims[4] = {inner, d1, d2, d3};
  cuuint64_t strides[3] = {(cuuint64_t)s1, (cuuint64_t)s2, (cuuint64_t)s3};
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0) strides[i] = 16;
  cuuint32_t box[4] = {128, b1, b2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MSA_OK : MSA_ERR_CUDA;
}

msa_status check_tensor_u8(const msa_tensor& t) {
  if (t.ptr == nullptr) return MSA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return MSA_ERR_ALIGNMENT;
  if (t.s_batch < 0 || t.s_tok < 0 || t.s_head < 0) return MSA_ERR_INVALID_ARG;
  if ((t.s_batch % 16) || (t.s_tok % 16) || (t.s_head % 16)) return MSA_ERR_ALIGNMENT;
  return MSA_OK;
}



}  // namespace

namespace msa {
// the dims check of every entry point, for the allocation-free list builder
// (library-internal: hidden like everything but the C ABI)
msa_status validate_dims(const msa_dims* d) { return check_dims(d); }
}  // namespace msa

extern "C" {

int64_t msa_num_blocks(const msa_dims* d) {
  if (d == nullptr || d->n_kv < 1) return 0;
  return (d->n_kv + MSA_BLOCK_TOKENS - 1) / MSA_BLOCK_TOKENS;
}

int64_t msa_num_entries(const msa_dims* d) {
  if (check_dims(d) != MSA_OK) return 0;
  return d->batch * d->h_kv * entries_per_bg(d);
}

int64_t msa_query_window(const msa_dims* d) {
  if (check_dims(d) != MSA_OK) return 0;
  return query_window(d);
}

int64_t msa_num_segments(const msa_dims* d) {
  if (check_dims(d) != MSA_OK) return 0;
  return d->batch * d->h_kv * num_windows(d) * msa_num_blocks(d);
}

msa_status msa_index_score_maxpool(const msa_dims* d, msa_tensor q_idx, msa_tensor k_idx,
                                   float* pooled, int64_t pooled_row_stride, int32_t* dev_err,
                                   void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if ((s = check_tensor(q_idx)) != MSA_OK) return s;
  if ((s = check_tensor(k_idx)) != MSA_OK) return s;
  if (pooled == nullptr) return MSA_ERR_INVALID_ARG;
  if (!aligned16(pooled)) return MSA_ERR_ALIGNMENT;
  const int64_t nblk = msa_num_blocks(d);
  if (pooled_row_stride < nblk || pooled_row_stride % 4 != 0) return MSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int32_t G = d->h_kv;
  if (d->n_q == 1 && d->h_kidx == 1 && d->d_idx == 128 && G <= 8) {
    // k_idx [B, 1, n_kv, 128]: dims {128, n_kv, 1, B}, box {64, 128, 1, 1} (one key block
    // per pair of loads)
    CUtensorMap tk;
    if ((s = make_map(&tk, k_idx.ptr, d->d_idx, d->n_kv, d->h_kidx, d->batch, k_idx.s_tok,
                      k_idx.s_head, k_idx.s_batch, 128, 1)) != MSA_OK)
      return s;
    return from_cuda(msa::launch_index_score_decode(tk, q_idx.ptr, q_idx.s_batch, q_idx.s_head,
                                                    d->batch, d->q_pos0, G, pooled,
                                                    pooled_row_stride, dev_err, st));
  }
  CUtensorMap tq, tk;
  // q_idx [B, n_q, G, d_idx]: dims {d_idx, G, n_q, B}, box {64, 1, 128, 1}
  if ((s = make_map(&tq, q_idx.ptr, d->d_idx, G, d->n_q, d->batch, q_idx.s_head, q_idx.s_tok,
                    q_idx.s_batch, 1, 128)) != MSA_OK)
    return s;
  // k_idx [B, h_kidx, n_kv, d_idx]: dims {d_idx, n_kv, h_kidx, B}, box {64, 256, 1, 1}
  // (two key blocks per load)
  if ((s = make_map(&tk, k_idx.ptr, d->d_idx, d->n_kv, d->h_kidx, d->batch, k_idx.s_tok,
                    k_idx.s_head, k_idx.s_batch, 256, 1)) != MSA_OK)
    return s;
  return from_cuda(msa::launch_index_score_prefill(tq, tk, d->d_idx, d->batch, d->n_q,
                                                   d->q_pos0, G, d->h_kidx, pooled,
                                                   pooled_row_stride, dev_err, st));
}

msa_status msa_topk_blocks(const msa_dims* d, const float* pooled, int64_t pooled_row_stride,
                           int32_t* sel, int32_t* dev_err, void* stream) {
  (void)dev_err;
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if (pooled == nullptr || sel == nullptr) return MSA_ERR_INVALID_ARG;
  if (!aligned16(pooled) || !aligned16(sel)) return MSA_ERR_ALIGNMENT;
  if (pooled_row_stride < msa_num_blocks(d) || pooled_row_stride % 4 != 0)
    return MSA_ERR_INVALID_ARG;
  const int64_t n_rows = d->batch * d->h_kv * d->n_q;
  return from_cuda(msa::launch_topk_blocks(pooled, pooled_row_stride, n_rows, d->n_q, d->q_pos0,
                                           sel, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_block_query_lists_workspace(const msa_dims* d) {
  if (check_dims(d) != MSA_OK) return 0;
  return msa::block_lists_workspace(d->batch * d->h_kv, d->n_q, msa_num_blocks(d),
                                   query_window(d));
}

msa_status msa_build_block_query_lists(const msa_dims* d, const int32_t* sel,
                                       int32_t* blk_offsets, int32_t* entries,
                                       int32_t* entry_pos, void* ws, size_t ws_bytes,
                                       int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if (sel == nullptr || blk_offsets == nullptr || entries == nullptr || entry_pos == nullptr ||
      ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(sel) || !aligned16(ws)) return MSA_ERR_ALIGNMENT;
  if (ws_bytes < msa_block_query_lists_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  const int64_t total = msa_num_entries(d);
  if (total >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return from_cuda(msa::launch_block_lists(sel, d->batch * d->h_kv, d->n_q, d->q_pos0,
                                           msa_num_blocks(d), query_window(d), blk_offsets,
                                           entries, entry_pos, total, ws, dev_err,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

msa_status sparse_attn_fwd(const msa_dims* d, msa_tensor q, msa_tensor k, msa_tensor v,
                           const int32_t* blk_offsets, const int32_t* entries, float* part_ml,
                           void* part_acc, bool compact, int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if ((s = check_tensor(q)) != MSA_OK) return s;
  if ((s = check_tensor(k)) != MSA_OK) return s;
  if ((s = check_tensor(v)) != MSA_OK) return s;
  if (blk_offsets == nullptr || entries == nullptr || part_ml == nullptr || part_acc == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(part_ml) || !aligned16(part_acc)) return MSA_ERR_ALIGNMENT;
  const int64_t nblk = msa_num_blocks(d);
  const int64_t nwin = num_windows(d);
  const int64_t n_seg = d->batch * d->h_kv * nwin * nblk;
  const int64_t total = msa_num_entries(d);
  if (total >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  const int64_t R = d->h_q / d->h_kv;
  // one query per sequence with R <= 8 runs on the warp-level decode kernel,
  // which writes fp32 pieces only
  const bool decode = d->n_q == 1 && R <= 8;
  if (compact && decode) return MSA_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  // k, v [B, h_kv, n_kv, 128]: dims {128, n_kv, h_kv, B}, box {64, 128, 1, 1}
  if ((s = make_map(&tk, k.ptr, MSA_HEAD_DIM, d->n_kv, d->h_kv, d->batch, k.s_tok, k.s_head,
                    k.s_batch, 128, 1)) != MSA_OK)
    return s;
  if ((s = make_map(&tv, v.ptr, MSA_HEAD_DIM, d->n_kv, d->h_kv, d->batch, v.s_tok, v.s_head,
                    v.s_batch, 128, 1)) != MSA_OK)
    return s;
  // part_acc [entries, R, 128] as rows of 128-byte panels; for R >= 8 a
  // warp's 32 adjacent rows are written by TMA stores of 32 rows x 2 panels
  // (fp32: half rows; bf16: whole rows), a partly covered warp's by 8-row,
  // one-panel stores
  CUtensorMap to, to8, tq;
  std::memset(&to, 0, sizeof(to));
  std::memset(&to8, 0, sizeof(to8));
  std::memset(&tq, 0, sizeof(tq));
  if (decode) {
    // one query per sequence: warp-level tiles, heads as the 8-wide side.
    // q [B, 1, H, 128]: dims {128, H, 1, B}, box {64, R, 1, 1} (the query's heads of a group)
    if ((s = make_map(&tq, q.ptr, MSA_HEAD_DIM, d->h_q, d->n_q, d->batch, q.s_head, q.s_tok,
                      q.s_batch, (uint32_t)R, 1)) != MSA_OK)
      return s;
    return from_cuda(msa::launch_sparse_attn_decode(
        tq, tk, tv, blk_offsets, entries, d->batch * d->h_kv, d->n_q, d->q_pos0, d->h_kv,
        d->h_q, (int32_t)nblk, d->scale, part_ml, reinterpret_cast<float*>(part_acc), dev_err,
        reinterpret_cast<cudaStream_t>(stream)));
  }
  if (R >= 8) {
    // q: one box per group of eight heads of an entry (both 64-column panels)
    if ((s = make_map_q_groups(&tq, d, q)) != MSA_OK) return s;
    const int64_t rows = total * R;
    if (rows >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
    s = make_map_piece_rows(&to, part_acc, (uint64_t)rows, compact, 32, 2);
    if (s != MSA_OK) return s;
    s = make_map_piece_rows(&to8, part_acc, (uint64_t)rows, compact, 8, 1);
    if (s != MSA_OK) return s;
  }
  return from_cuda(msa::launch_sparse_attn(
      tq, tk, tv, to, to8, q.ptr, q.s_batch, q.s_tok, q.s_head, blk_offsets, entries, n_seg, total,
      d->n_q, d->q_pos0, d->h_kv, d->h_q, (int32_t)nblk, (int32_t)nwin, d->scale, part_ml,
      part_acc, compact, dev_err, reinterpret_cast<cudaStream_t>(stream)));
}

msa_status merge_partials(const msa_dims* d, const int32_t* entry_pos, const float* part_ml,
                          const void* part_acc, bool compact, void* out, float* lse,
                          int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if (entry_pos == nullptr || part_ml == nullptr || part_acc == nullptr || out == nullptr ||
      lse == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(part_ml) || !aligned16(part_acc) || !aligned16(out))
    return MSA_ERR_ALIGNMENT;
  const int64_t n_rows = d->batch * d->n_q * d->h_q;
  return from_cuda(msa::launch_merge(entry_pos, part_ml, part_acc, compact, out, lse, n_rows,
                                     d->n_q, d->h_q, d->h_kv, msa_num_entries(d), dev_err,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

msa_status msa_sparse_attn_fwd(const msa_dims* d, msa_tensor q, msa_tensor k, msa_tensor v,
                               const int32_t* blk_offsets, const int32_t* entries,
                               float* part_ml, float* part_acc, int32_t* dev_err,
                               void* stream) {
  return sparse_attn_fwd(d, q, k, v, blk_offsets, entries, part_ml, part_acc, false, dev_err,
                         stream);
}

msa_status msa_sparse_attn_fwd_compact(const msa_dims* d, msa_tensor q, msa_tensor k,
                                       msa_tensor v, const int32_t* blk_offsets,
                                       const int32_t* entries, float* part_ml,
                                       void* part_acc_bf16, int32_t* dev_err, void* stream) {
  return sparse_attn_fwd(d, q, k, v, blk_offsets, entries, part_ml, part_acc_bf16, true,
                         dev_err, stream);
}

msa_status msa_merge_partials(const msa_dims* d, const int32_t* entry_pos, const float* part_ml,
                              const float* part_acc, void* out, float* lse, int32_t* dev_err,
                              void* stream) {
  return merge_partials(d, entry_pos, part_ml, part_acc, false, out, lse, dev_err, stream);
}

msa_status msa_merge_partials_compact(const msa_dims* d, const int32_t* entry_pos,
                                      const float* part_ml, const void* part_acc_bf16,
                                      void* out, float* lse, int32_t* dev_err, void* stream) {
  return merge_partials(d, entry_pos, part_ml, part_acc_bf16, true, out, lse, dev_err, stream);
}

msa_status msa_quantize_e4m3(const void* x, int64_t n, void* codes, float* scale,
                             void* stream) {
  if (n < 0) return MSA_ERR_INVALID_ARG;
  if (scale == nullptr || (n > 0 && (x == nullptr || codes == nullptr))) return MSA_ERR_INVALID_ARG;
  return from_cuda(msa::launch_quantize_e4m3(x, n, codes, scale,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_index_score_maxpool_e4m3(const msa_dims* d, msa_tensor q_idx8, msa_tensor k_idx8,
                                        const float* scale_q, const float* scale_k,
                                        float* pooled, int64_t pooled_row_stride,
                                        int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if (d->d_idx != 128) return MSA_ERR_UNSUPPORTED;   // one 128-byte row per index vector
  if ((s = check_tensor_u8(q_idx8)) != MSA_OK) return s;
  if ((s = check_tensor_u8(k_idx8)) != MSA_OK) return s;
  if (pooled == nullptr || scale_q == nullptr || scale_k == nullptr) return MSA_ERR_INVALID_ARG;
  if (!aligned16(pooled)) return MSA_ERR_ALIGNMENT;
  if (pooled_row_stride < msa_num_blocks(d) || pooled_row_stride % 4 != 0)
    return MSA_ERR_INVALID_ARG;
  CUtensorMap tq, tk;
  // q_idx codes [B, n_q, G, 128]: dims {128, G, n_q, B}, box {128, 1, 128, 1}
  if ((s = make_map_u8(&tq, q_idx8.ptr, 128, d->h_kv, d->n_q, d->batch, q_idx8.s_head,
                       q_idx8.s_tok, q_idx8.s_batch, 1, 128)) != MSA_OK)
    return s;
  // k_idx codes [B, h_kidx, n_kv, 128]: dims {128, n_kv, h_kidx, B}, box {128, 256, 1, 1}
  if ((s = make_map_u8(&tk, k_idx8.ptr, 128, d->n_kv, d->h_kidx, d->batch, k_idx8.s_tok,
                       k_idx8.s_head, k_idx8.s_batch, 256, 1)) != MSA_OK)
    return s;
  return from_cuda(msa::launch_index_score_e4m3(tq, tk, d->batch, d->n_q, d->q_pos0, d->h_kv,
                                                d->h_kidx, pooled, pooled_row_stride, scale_q,
                                                scale_k, dev_err,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_selection_recall_workspace(const msa_dims* d, int64_t n_rows) {
  if (check_dims(d) != MSA_OK || n_rows < 0) return 0;
  return msa::recall_workspace(n_rows, d->h_kv, d->h_q / d->h_kv, (int32_t)msa_num_blocks(d));
}

msa_status msa_selection_recall(const msa_dims* d, msa_tensor q, msa_tensor k, msa_tensor q_idx,
                                msa_tensor k_idx, const int32_t* sel, const int64_t* rows,
                                int64_t n_rows, float* block_mass, int64_t mass_stride,
                                float* recall, float* kl_pq, float* kl_qp, float* lse_full,
                                void* ws,
                                size_t ws_bytes, int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if ((s = check_tensor(q)) != MSA_OK) return s;
  if ((s = check_tensor(k)) != MSA_OK) return s;
  if ((s = check_tensor(q_idx)) != MSA_OK) return s;
  if ((s = check_tensor(k_idx)) != MSA_OK) return s;
  if (n_rows < 0) return MSA_ERR_INVALID_ARG;
  if (n_rows == 0) return MSA_OK;
  if (sel == nullptr || rows == nullptr || block_mass == nullptr || recall == nullptr ||
      kl_pq == nullptr || kl_qp == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MSA_ERR_ALIGNMENT;
  const int64_t nblk = msa_num_blocks(d);
  const int64_t R = d->h_q / d->h_kv;
  if (R > 8) return MSA_ERR_UNSUPPORTED;            // heads are the 8-wide side of the tiles
  if (mass_stride < nblk) return MSA_ERR_INVALID_ARG;
  if (n_rows * d->h_kv > 0x7FFFFFFF) return MSA_ERR_UNSUPPORTED;
  if (ws_bytes < msa_selection_recall_workspace(d, n_rows)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  CUtensorMap tq, tk, tki;
  // q [B, n_q, H, 128]: box {64, R, 1, 1} (one query's heads of a group)
  if ((s = make_map(&tq, q.ptr, MSA_HEAD_DIM, d->h_q, d->n_q, d->batch, q.s_head, q.s_tok,
                    q.s_batch, (uint32_t)R, 1)) != MSA_OK)
    return s;
  // k [B, h_kv, n_kv, 128] and k_idx [B, h_kidx, n_kv, d_idx]: one 128-token block per box
  if ((s = make_map(&tk, k.ptr, MSA_HEAD_DIM, d->n_kv, d->h_kv, d->batch, k.s_tok, k.s_head,
                    k.s_batch, 128, 1)) != MSA_OK)
    return s;
  if ((s = make_map(&tki, k_idx.ptr, d->d_idx, d->n_kv, d->h_kidx, d->batch, k_idx.s_tok,
                    k_idx.s_head, k_idx.s_batch, 128, 1)) != MSA_OK)
    return s;
  return from_cuda(msa::launch_selection_recall(
      tq, tk, tki, rows, n_rows, q_idx.ptr, q_idx.s_batch, q_idx.s_tok, q_idx.s_head, d->batch,
      d->n_q, d->q_pos0, d->h_kv, d->h_q, d->d_idx, d->h_kidx, (int32_t)nblk, d->scale, sel,
      block_mass, mass_stride, recall, kl_pq, kl_qp, lse_full, ws, dev_err,
      reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_sparse_attn_bwd(const msa_dims* d, msa_tensor q, msa_tensor k, msa_tensor v,
                               msa_tensor o, msa_tensor d_o, const float* lse,
                               const int32_t* blk_offsets, const int32_t* entries, float* delta,
                               float* part_dq, float* dq, float* dk, float* dv, int32_t* dev_err,
                               void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if ((s = check_tensor(q)) != MSA_OK) return s;
  if ((s = check_tensor(k)) != MSA_OK) return s;
  if ((s = check_tensor(v)) != MSA_OK) return s;
  if ((s = check_tensor(o)) != MSA_OK) return s;
  if ((s = check_tensor(d_o)) != MSA_OK) return s;
  if (lse == nullptr || blk_offsets == nullptr || entries == nullptr || delta == nullptr ||
      part_dq == nullptr || dq == nullptr || dk == nullptr || dv == nullptr)
    return MSA_ERR_INVALID_ARG;
  // dq pieces, dk and dv leave in 32-byte stores
  if (!aligned32(part_dq) || !aligned16(dq) || !aligned32(dk) || !aligned32(dv))
    return MSA_ERR_ALIGNMENT;
  const int64_t nblk = msa_num_blocks(d);
  const int64_t total = msa_num_entries(d);
  if (total >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  // k, v [B, h_kv, n_kv, 128]: dims {128, n_kv, h_kv, B}, box {64, 128, 1, 1}
  if ((s = make_map(&tk, k.ptr, MSA_HEAD_DIM, d->n_kv, d->h_kv, d->batch, k.s_tok, k.s_head,
                    k.s_batch, 128, 1)) != MSA_OK)
    return s;
  if ((s = make_map(&tv, v.ptr, MSA_HEAD_DIM, d->n_kv, d->h_kv, d->batch, v.s_tok, v.s_head,
                    v.s_batch, 128, 1)) != MSA_OK)
    return s;
  return from_cuda(msa::launch_sparse_attn_bwd(
      tk, tv, q.ptr, q.s_batch, q.s_tok, q.s_head, o.ptr, o.s_batch, o.s_tok, o.s_head, d_o.ptr,
      d_o.s_batch, d_o.s_tok, d_o.s_head, lse, blk_offsets, entries, total, d->batch, d->n_q,
      d->n_kv, d->q_pos0, d->h_kv, d->h_q, (int32_t)nblk, (int32_t)num_windows(d), d->scale,
      delta, part_dq, dq, dk, dv, dev_err, reinterpret_cast<cudaStream_t>(stream)));
}

size_t msa_token_select_workspace(const msa_dims* d, int64_t n_rows) {
  if (check_dims(d) != MSA_OK || n_rows < 0) return 0;
  return msa::token_select_workspace(n_rows, d->h_kv, d->n_kv);
}

msa_status msa_token_select_attention(const msa_dims* d, msa_tensor q, msa_tensor k,
                                      msa_tensor v, msa_tensor q_idx, msa_tensor k_idx,
                                      const int64_t* rows, int64_t n_rows, int64_t budget,
                                      int32_t* tokens, float* out, float* lse, void* ws,
                                      size_t ws_bytes, int32_t* dev_err, void* stream) {
  msa_status s = check_dims(d);
  if (s != MSA_OK) return s;
  if ((s = check_tensor(q)) != MSA_OK) return s;
  if ((s = check_tensor(k)) != MSA_OK) return s;
  if ((s = check_tensor(v)) != MSA_OK) return s;
  if ((s = check_tensor(q_idx)) != MSA_OK) return s;
  if ((s = check_tensor(k_idx)) != MSA_OK) return s;
  if (n_rows < 0 || budget < 1 || budget > 0x7FFFFFFF) return MSA_ERR_INVALID_ARG;
  if (n_rows == 0) return MSA_OK;
  if (rows == nullptr || tokens == nullptr || out == nullptr || lse == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(ws) || !aligned16(out)) return MSA_ERR_ALIGNMENT;
  const int64_t R = d->h_q / d->h_kv;
  if (R > 8) return MSA_ERR_UNSUPPORTED;            // heads are the 8-wide side of the tiles
  if (n_rows * d->h_kv > 0x7FFFFFFF) return MSA_ERR_UNSUPPORTED;
  if (ws_bytes < msa_token_select_workspace(d, n_rows)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  CUtensorMap tki;
  // k_idx [B, h_kidx, n_kv, d_idx]: one 128-token block of 64 dims per box
  if ((s = make_map(&tki, k_idx.ptr, d->d_idx, d->n_kv, d->h_kidx, d->batch, k_idx.s_tok,
                    k_idx.s_head, k_idx.s_batch, 128, 1)) != MSA_OK)
    return s;
  return from_cuda(msa::launch_token_select_attention(
      tki, rows, n_rows, q.ptr, q.s_batch, q.s_tok, q.s_head, q_idx.ptr, q_idx.s_batch,
      q_idx.s_tok, q_idx.s_head, k.ptr, k.s_batch, k.s_tok, k.s_head, v.ptr, v.s_batch, v.s_tok,
      v.s_head, d->batch, d->n_q, d->n_kv, d->q_pos0, d->h_kv, d->h_q, d->d_idx, d->h_kidx,
      d->scale, budget, tokens, out, lse, ws, dev_err, reinterpret_cast<cudaStream_t>(stream)));
}

uint64_t msa_debug_set_attn_wait_limit_ns(uint64_t ns) {
  if (ns == 0) ns = msa::kWaitLimitNs;
  if (ns > msa::kWaitLimitNs) ns = msa::kWaitLimitNs;
  return msa::set_attn_wait_limit(ns);
}

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_ALIGNMENT: return "MSA_ERR_ALIGNMENT";
    case MSA_ERR_WORKSPACE_TOO_SMALL: return "MSA_ERR_WORKSPACE_TOO_SMALL";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
    case MSA_ERR_SCRATCH_LIMIT: return "MSA_ERR_SCRATCH_LIMIT";
  }
  return "MSA_ERR_UNKNOWN";
}

}  // extern "C"
