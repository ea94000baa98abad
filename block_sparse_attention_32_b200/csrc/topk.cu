// Block selection: per (query, group) the own block plus the best 15 of the
// candidate blocks c < own, ranked by (score descending, block index
// ascending), written in ascending block order.
//
// Source: page "MSA 稀疏注意力三国杀", section "MSA 架构：粗筛 + 精算", first
// step item 3 (16 blocks, the current position's block always taken, the rest
// by score); page "稀疏注意力速览", section 4, MSA entry (per-group top-k with the
// local block kept).  The tie rule is the stated reading where the pages are
// silent.
//
// One warp per row; keys are (score, block) pairs ordered by score, then lower
// block first (a 64-bit key: order-preserving score bits over the complemented
// block index).  The row is scanned in chunks of 32 x 32 candidates:
//   1. every lane takes the maximum of its 32 scores; the 15th largest lane
//      maximum is a lower bound for the 15th-best score (15 distinct
//      candidates reach it), and so is the current 15th-best of the row;
//   2. the candidates at or above the larger of the two bounds (usually a few
//      dozen) are compacted by a warp prefix sum into a shared buffer next to
//      the current best 15 and sorted by a warp bitonic network (one key per
//      lane when they fit in 32, else two); the first 15 are the new best.
// If more than 64 keys pass the bound (many equal scores), the row falls back
// to an exact radix select over the whole row (4 passes of 8 bits with
// warp-aggregated shared histograms).  Both give the same set.
#include "common.cuh"

namespace msa {

constexpr int kTopkWarps = 8;

// float -> uint32 whose unsigned order is the float order; -0.0 maps like +0.0
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exact radix select over a row of n candidates: the 15 best in ascending
// block order into out[0..14]
__device__ __noinline__ void select_row_radix(const float* __restrict__ row, int n, int32_t* out,
                                              uint32_t* hist, int lane) {
  const uint32_t lt_mask = (1u << lane) - 1u;
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
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) mine += hist[8 * lane + j];
    uint32_t incl = mine;   // inclusive suffix sum over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += v;
    }
    int digit = -1;
    uint32_t cum_at = 0, cum = incl - mine;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
      const uint32_t h = hist[8 * lane + j];
      if (digit < 0 && cum < (uint32_t)k && cum + h >= (uint32_t)k) {
        digit = 8 * lane + j;
        cum_at = cum;
      }
      cum += h;
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, digit >= 0)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    cum_at = __shfl_sync(0xffffffffu, cum_at, src);
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
    k -= (int)cum_at;
    __syncwarp();
  }
  const uint32_t T = prefix;   // the 15th-best score key; k keys equal to T are taken
  int written = 0, ties = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t u = (i < n) ? order_key(row[i]) : 0u;
    const bool eq = (i < n) && (u == T);
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const int tie_rank = ties + __popc(eqm & lt_mask);
    ties += __popc(eqm);
    const bool take = (i < n) && (u > T || (eq && tie_rank < k));
    const uint32_t tm = __ballot_sync(0xffffffffu, take);
    if (take) out[written + __popc(tm & lt_mask)] = i;
    written += __popc(tm);
  }
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// Sorts the 64 keys held as (a: position lane, b: position lane + 32)
// descending with a bitonic network.
__device__ __forceinline__ void bitonic64_desc(uint64_t& a, uint64_t& b, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {                        // partners within the lane (last stage only)
        const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
        a = hi;
        b = lo;
      } else {
        const uint64_t oa = shfl_xor_u64(a, j), ob = shfl_xor_u64(b, j);
        const bool lower = (lane & j) == 0;
        const bool desc_a = (lane & k) == 0;          // position lane
        const bool desc_b = ((lane + 32) & k) == 0;   // position lane + 32
        a = (lower == desc_a) ? (a > oa ? a : oa) : (a < oa ? a : oa);
        b = (lower == desc_b) ? (b > ob ? b : ob) : (b < ob ? b : ob);
      }
    }
  }
}

// Sorts one 64-bit key per lane descending over the warp.
__device__ __forceinline__ uint64_t bitonic32_desc(uint64_t a, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const uint64_t o = shfl_xor_u64(a, j);
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
      a = keep_max ? (a > o ? a : o) : (a < o ? a : o);
    }
  }
  return a;
}

// Sorts one 32-bit value per lane ascending over lanes 0..15 (lanes 16..31
// take part with values that sort after).
__device__ __forceinline__ int32_t bitonic16_asc(int32_t v, int lane) {
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int32_t o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool lower = (lane & j) == 0;
      const bool asc = (lane & k) == 0;
      v = (lower == asc) ? min(v, o) : max(v, o);
    }
  }
  return v;
}

__global__ void __launch_bounds__(kTopkWarps * 32, 3)
    topk_blocks_kernel(const float* __restrict__ pooled, int64_t stride, int64_t n_rows,
                       int64_t n_q, int64_t q_pos0, int32_t* __restrict__ sel) {
  __shared__ uint32_t hist_all[kTopkWarps][256];
  __shared__ uint64_t cand_all[kTopkWarps][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* hist = hist_all[warp];
  uint64_t* cand = cand_all[warp];

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
    {
      // pull the warp's next row toward L2 while this one is processed (one
      // 128-byte line per lane covers rows of up to 1024 candidates)
      const int64_t rn = r + (int64_t)gridDim.x * kTopkWarps;
      if (rn < n_rows && lane * 32 < n)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(pooled + rn * stride + lane * 32));
    }

    // best 15 so far, descending, in lanes 0..14 (0 = empty, below every key)
    uint64_t best = 0;
    bool overflow = false;
    for (int c0 = 0; c0 < n; c0 += 1024) {
      float v[32];
      float lmax = -INFINITY;
#pragma unroll
      for (int s = 0; s < 32; ++s) {
        const int i = c0 + s * 32 + lane;
        v[s] = (i < n) ? __ldg(row + i) : -INFINITY;
        lmax = fmaxf(lmax, v[s]);
      }
      // 15th largest lane maximum: bitonic sort of the 32 maxima, descending
      float sm = lmax;
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
          const float o = __shfl_xor_sync(0xffffffffu, sm, j);
          const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
          sm = keep_max ? fmaxf(sm, o) : fminf(sm, o);
        }
      }
      float T = __shfl_sync(0xffffffffu, sm, 14);
      if (c0 > 0) {
        // the 15th best so far, back from its order-preserving key
        const uint32_t kb = (uint32_t)(__shfl_sync(0xffffffffu, best, 14) >> 32);
        const float tb = __uint_as_float((kb & 0x80000000u) ? (kb & 0x7FFFFFFFu) : ~kb);
        T = fmaxf(T, tb);
      }
      // candidates: score >= T (ties at T included), compacted by a prefix sum
      int cnt = 0;
#pragma unroll
      for (int s = 0; s < 32; ++s) cnt += (c0 + s * 32 + lane < n && v[s] >= T) ? 1 : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      const int nbest = (c0 > 0) ? kTopK - 1 : 0;
      if (total + nbest > 64) {
        overflow = true;
        break;
      }
      // raw (score bits, block) pairs; the sort keys are formed after the compaction
      uint2* raw = reinterpret_cast<uint2*>(cand);
      int pos = incl - cnt;
#pragma unroll
      for (int s = 0; s < 32; ++s) {
        const int i = c0 + s * 32 + lane;
        if (i < n && v[s] >= T) raw[pos++] = make_uint2(__float_as_uint(v[s]), (uint32_t)i);
      }
      __syncwarp();
      const int m = total + nbest;
      // key j of the merged list: compacted candidates first, then the best so far
      // (the shuffle runs on every lane, whichever side its j falls on)
      auto key_at = [&](int j) -> uint64_t {
        const uint64_t bk = shfl_u64(best, (j - total) & 31);
        if (j < total) {
          const uint2 c = raw[j];
          return ((uint64_t)order_key(__uint_as_float(c.x)) << 32) |
                 (uint32_t)(0xFFFFFFFFu - c.y);
        }
        return (j < m) ? bk : 0;
      };
      if (m <= 32) {
        uint64_t k1 = key_at(lane);
        k1 = bitonic32_desc(k1, lane);
        best = (lane < kTopK - 1) ? k1 : 0;
      } else {
        uint64_t a = key_at(lane), b = key_at(lane + 32);
        bitonic64_desc(a, b, lane);
        best = (lane < kTopK - 1) ? a : 0;
      }
      __syncwarp();
    }
    if (overflow) {
      select_row_radix(row, n, out, hist, lane);
    } else {
      // the 15 block ids ascending, then the own block
      int32_t id = (lane < kTopK - 1) ? (int32_t)(0xFFFFFFFFu - (uint32_t)best) : 0x7FFFFFFF;
      id = bitonic16_asc(id, lane);
      if (lane < kTopK - 1) out[lane] = id;
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
