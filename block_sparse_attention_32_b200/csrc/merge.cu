// Log-sum-exp merge of the per-(query, head, block) softmax pieces written by
// the KV-block-outer attention kernel, in fixed slot order (deterministic):
//   M = max_s m_s, L = sum_s l_s e^{m_s-M}, o = sum_s acc_s e^{m_s-M} / L,
//   lse = M + ln L.
// Softmax over a union of disjoint token sets factors this way, which is
// what lets the "Outer Gather Q" scheme (page "MSA 稀疏注意力三国杀", section
// "Kernel 创新：Outer Gather Q") compute each selected block separately.
//
// Pieces are in the block->query lists' order: the piece of (b, g, i, slot)
// and head r of the group is row entry_pos[b, g, i, slot] * R + r; an empty
// slot has entry_pos -1, and a position past the lists' entries is reported
// (MSA_DEVERR_BAD_ENTRY) and read as an empty slot.
//
// One warp per (batch, query, head); lane l owns output dims 4l .. 4l+3.
// HBM-bound: it reads each piece once.  Compact pieces hold accn_s = acc_s /
// l_s in bf16; then o = sum_s (l_s e^{m_s-M}) accn_s / L.
#include "common.cuh"

namespace msa {

template <bool kCompact>
__global__ void __launch_bounds__(256)
    merge_partials_kernel(const int32_t* __restrict__ entry_pos, const float* __restrict__ part_ml,
                          const void* __restrict__ part_acc, __nv_bfloat16* __restrict__ out,
                          float* __restrict__ lse, int64_t n_rows, int64_t n_q, int32_t H,
                          int32_t G, int64_t n_ent, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (r >= n_rows) return;
  const int32_t R = H / G;
  const int32_t h = (int32_t)(r % H);
  const int64_t bq = r / H;            // b * n_q + qi
  const int64_t b = bq / n_q, qi = bq - b * n_q;
  const int32_t g = h / R;
  const int32_t* prow = entry_pos + ((b * G + g) * n_q + qi) * kTopK;
  const int32_t hr = h - g * R;

  // lane s < 16: the piece row of slot s for this head
  float m = -INFINITY, l = 0.f;
  bool v = false;
  int64_t row = 0;
  if (lane < kTopK) {
    int32_t p = prow[lane];
    if (p >= n_ent) {
      report(err, MSA_DEVERR_BAD_ENTRY);
      p = -1;
    }
    v = p >= 0;
    if (v) {
      row = (int64_t)p * R + hr;
      const float2 ml = *reinterpret_cast<const float2*>(part_ml + row * 2);
      m = ml.x;
      l = ml.y;
    }
  }
  const uint32_t vmask = __ballot_sync(0xffffffffu, v);
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w = v ? expf(m - M) : 0.f;
  float L = w * l;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (kCompact) {
    // weight of piece s: l_s e^{m_s - M}
    const float wl = w * l;
    const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(part_acc) + 4 * lane;
#pragma unroll
    for (int s = 0; s < kTopK; ++s) {
      const float ws = __shfl_sync(0xffffffffu, wl, s);
      const int64_t rs = __shfl_sync(0xffffffffu, row, s);
      if ((vmask >> s) & 1u) {
        const uint2 u = *reinterpret_cast<const uint2*>(pa + rs * kHeadDim);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        acc.x = fmaf(ws, lo.x, acc.x);
        acc.y = fmaf(ws, lo.y, acc.y);
        acc.z = fmaf(ws, hi.x, acc.z);
        acc.w = fmaf(ws, hi.y, acc.w);
      }
    }
  } else {
    const float* pa = reinterpret_cast<const float*>(part_acc) + 4 * lane;
#pragma unroll
    for (int s = 0; s < kTopK; ++s) {
      const float ws = __shfl_sync(0xffffffffu, w, s);
      const int64_t rs = __shfl_sync(0xffffffffu, row, s);
      if ((vmask >> s) & 1u) {
        const float4 a = *reinterpret_cast<const float4*>(pa + rs * kHeadDim);
        acc.x = fmaf(ws, a.x, acc.x);
        acc.y = fmaf(ws, a.y, acc.y);
        acc.z = fmaf(ws, a.z, acc.z);
        acc.w = fmaf(ws, a.w, acc.w);
      }
    }
  }
  const float inv = 1.0f / L;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 packed;
  packed.x = *reinterpret_cast<const uint32_t*>(&lo);
  packed.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + r * kHeadDim + 4 * lane) = packed;
  if (lane == 0) lse[r] = M + logf(L);
}

cudaError_t launch_merge(const int32_t* entry_pos, const float* part_ml, const void* part_acc,
                         bool compact, void* out, float* lse, int64_t n_rows, int64_t n_q,
                         int32_t H, int32_t G, int64_t n_ent, int32_t* err, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int64_t threads = n_rows * 32;
  const unsigned grid = (unsigned)((threads + 255) / 256);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  if (compact)
    merge_partials_kernel<true><<<grid, 256, 0, st>>>(entry_pos, part_ml, part_acc, o, lse, n_rows,
                                                      n_q, H, G, n_ent, err);
  else
    merge_partials_kernel<false><<<grid, 256, 0, st>>>(entry_pos, part_ml, part_acc, o, lse, n_rows,
                                                       n_q, H, G, n_ent, err);
  return cudaGetLastError();
}

}  // namespace msa
