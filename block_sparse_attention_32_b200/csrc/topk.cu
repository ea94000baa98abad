// Block selection: per (query, group) the own block plus the best 15 of the
// candidate blocks c < own, ranked by (score descending, block index
// ascending), written in ascending block order.
//
// Source: page "MSA 稀疏注意力三国杀", section "MSA 架构：粗筛 + 精算", first
// step item 3 (16 blocks, the current position's block always taken, the rest
// by score); sparse-attention survey page, MSA entry (per-group top-k with the
// local block kept).  The tie rule is the stated reading where the pages are
// silent.
//
// One warp per row.  The 15th-best score is found by an exact radix select on
// order-preserving 32-bit keys (4 passes of 8 bits, warp-aggregated shared
// histograms); candidates strictly above it are taken, and among those equal
// to it the lowest block indices fill the remaining places.  The row is read
// from global memory once per pass (L1-resident after the first).
#include "common.cuh"

namespace msa {

constexpr int kTopkWarps = 8;

// float -> uint32 whose unsigned order is the float order; -0.0 maps like +0.0
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkWarps * 32)
    topk_blocks_kernel(const float* __restrict__ pooled, int64_t stride, int64_t n_rows,
                       int64_t n_q, int64_t q_pos0, int32_t* __restrict__ sel) {
  __shared__ uint32_t hist_all[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* hist = hist_all[warp];
  const uint32_t lt_mask = (1u << lane) - 1u;

  for (int64_t r = (int64_t)blockIdx.x * kTopkWarps + warp; r < n_rows;
       r += (int64_t)gridDim.x * kTopkWarps) {
    const int64_t q = r % n_q;
    const int64_t own = (q_pos0 + q) / kBlock;
    int32_t* out = sel + r * kTopK;
    if (own < kTopK) {                          // every block 0..own is taken
      if (lane < kTopK) out[lane] = (lane <= own) ? lane : -1;
      continue;
    }
    const float* row = pooled + r * stride;
    const int n = (int)own;

    // radix select: threshold key T and how many keys equal to T to take
    uint32_t prefix = 0, mask = 0;
    int k = kTopK - 1;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = lane; i < 256; i += 32) hist[i] = 0;
      __syncwarp();
      for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        bool act = false;
        uint32_t bin = 0;
        if (i < n) {
          const uint32_t u = order_key(row[i]);
          act = (u & mask) == prefix;
          bin = (u >> shift) & 255u;
        }
        const uint32_t am = __ballot_sync(0xffffffffu, act);
        if (act) {
          const uint32_t peers = __match_any_sync(am, bin);
          if ((peers & lt_mask) == 0) atomicAdd(&hist[bin], __popc(peers));
        }
      }
      __syncwarp();
      // lane l owns bins 8l .. 8l+7; count of keys in higher lanes' bins
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) mine += hist[8 * lane + j];
      uint32_t above = 0;   // sum over lanes > lane
      {
        uint32_t incl = mine;   // inclusive suffix sum
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += v;
        }
        above = incl - mine;
      }
      int digit = -1;
      uint32_t cum_at = 0;
      uint32_t cum = above;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const uint32_t h = hist[8 * lane + j];
        if (digit < 0 && cum < (uint32_t)k && cum + h >= (uint32_t)k) {
          digit = 8 * lane + j;
          cum_at = cum;
        }
        cum += h;
      }
      const uint32_t found = __ballot_sync(0xffffffffu, digit >= 0);
      const int src = __ffs(found) - 1;
      digit = __shfl_sync(0xffffffffu, digit, src);
      cum_at = __shfl_sync(0xffffffffu, cum_at, src);
      prefix |= (uint32_t)digit << shift;
      mask |= 255u << shift;
      k -= (int)cum_at;
      __syncwarp();
    }
    const uint32_t T = prefix;   // the 15th-best key; k keys equal to T are taken

    // emit selected candidates in ascending index order, then the own block
    int written = 0, ties = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      uint32_t u = 0;
      if (i < n) u = order_key(row[i]);
      const bool eq = (i < n) && (u == T);
      const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
      const int tie_rank = ties + __popc(eqm & lt_mask);
      ties += __popc(eqm);
      const bool take = (i < n) && (u > T || (eq && tie_rank < k));
      const uint32_t tm = __ballot_sync(0xffffffffu, take);
      if (take) out[written + __popc(tm & lt_mask)] = i;
      written += __popc(tm);
    }
    if (lane == 0) out[kTopK - 1] = n;
    __syncwarp();
  }
}

cudaError_t launch_topk_blocks(const float* pooled, int64_t stride, int64_t n_rows,
                               int64_t n_q, int64_t q_pos0, int32_t* sel, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  int64_t blocks = (n_rows + kTopkWarps - 1) / kTopkWarps;
  if (blocks > 148 * 64) blocks = 148 * 64;
  topk_blocks_kernel<<<(unsigned)blocks, kTopkWarps * 32, 0, st>>>(pooled, stride, n_rows, n_q,
                                                                   q_pos0, sel);
  return cudaGetLastError();
}

}  // namespace msa
