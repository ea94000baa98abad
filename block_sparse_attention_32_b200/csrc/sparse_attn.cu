// KV-block-outer sparse attention: for every (batch, group, KV block) segment
// of the block->query lists, the block's K and V tiles are loaded into shared
// memory by TMA once, the query rows that chose it are gathered into 128-row
// tiles, and S = Q K^T, the softmax piece and O = P V run on the tcgen05 tensor
// cores with fp32 accumulators in TMEM.  Each (query, head, slot) gets a
// piece (m, l, acc) that the merge kernel combines.
//
// Source: page "MSA 稀疏注意力三国杀", section "MSA 架构：粗筛 + 精算" (main
// branch: full attention over the selected blocks only) and section "Kernel
// 创新：Outer Gather Q" (the KV block is the outer loop, all queries that chose
// it are computed together so the block is read once); sparse-attention
// survey page, MSA entry (exact softmax attention); chenxutan page, standard
// attention softmax(Q K^T / sqrt(d_k)) V.
//
// Tile shapes: a 128-row tile holds 128 / R query entries x R heads of the
// group (R = h_q / h_kv).  Shared memory (per CTA, 96 KB, two CTAs per SM):
//   sq: Q tile, later overwritten by P (bf16, 128 x 128, K-major, 128B swizzle)
//   sk: K block (keys x dims, K-major for S = Q K^T)
//   sv: V block (keys x dims, N(dims)-major for O = P V)
// TMEM: columns [0,128) hold S, [128,256) hold O.
#include "common.cuh"

namespace msa {

constexpr int kAttnThreads = 128;
constexpr int kAttnChunksPerItem = 8;
constexpr int kAttnSmemBytes = 1024 + 3 * 32768 + 256 + 128 * 4;

template <int R>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __nv_bfloat16* __restrict__ q, int64_t qs_b, int64_t qs_t,
                           int64_t qs_h, const int32_t* __restrict__ blk_offsets,
                           const int32_t* __restrict__ entries, int64_t n_seg,
                           int64_t n_entries, int64_t n_q, int64_t q_pos0, int32_t G,
                           int32_t H, int32_t nblk, float scale, float* __restrict__ part_ml,
                           float* __restrict__ part_acc, int32_t* err) {
  constexpr int CH = 128 / R;                       // query entries per 128-row tile
  constexpr int W = CH * kAttnChunksPerItem;        // entries per CTA
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 1);
  const float scale_log2 = scale * 1.4426950408889634f;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk = base + 32768;
  uint8_t* sv = base + 65536;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + 98304);
  uint64_t* kv_full = bars;
  uint64_t* mma_done = bars + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* ent_s = reinterpret_cast<int32_t*>(base + 98304 + 256);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t e0 = (int64_t)blockIdx.x * W;
  const int64_t e1 = min64(e0 + W, n_entries);

  if (tid == 0) {
    mbar_init(kv_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t sq_a = smem_u32(sq), sk_a = smem_u32(sk), sv_a = smem_u32(sv);

  uint32_t kv_phase = 0, mma_phase = 0;
  int64_t pos = e0;
  while (pos < e1) {
    if (__syncthreads_or(*abort_flag != 0)) break;
    // segment holding entry `pos`: the last s with blk_offsets[s] <= pos
    int64_t lo = 0, hi = n_seg;   // invariant: offsets[lo] <= pos < offsets[hi]
    while (hi - lo > 1) {
      const int64_t mid = (lo + hi) >> 1;
      if (blk_offsets[mid] <= pos) lo = mid; else hi = mid;
    }
    const int64_t seg = lo;
    const int64_t pend = min64(e1, blk_offsets[seg + 1]);
    if (pend <= pos) {               // fewer entries listed than expected
      if (tid == 0) report(err, MSA_DEVERR_BAD_ENTRY);
      break;
    }
    const int64_t bg = seg / nblk;
    const int32_t c = (int32_t)(seg - bg * nblk);
    const int32_t b = (int32_t)(bg / G), g = (int32_t)(bg - (int64_t)b * G);

    if (tid == 0) {
      mbar_arrive_expect_tx(kv_full, 65536);
      tma_load_4d(sk, &tm_k, kv_full, 0, c * kBlock, g, b);
      tma_load_4d(sk + 16384, &tm_k, kv_full, 64, c * kBlock, g, b);
      tma_load_4d(sv, &tm_v, kv_full, 0, c * kBlock, g, b);
      tma_load_4d(sv + 16384, &tm_v, kv_full, 64, c * kBlock, g, b);
    }

    for (int64_t cpos = pos; cpos < pend; cpos += CH) {
      const int cnt = (int)min64(CH, pend - cpos);
      if (tid < CH) ent_s[tid] = (tid < cnt) ? entries[cpos + tid] : -1;
      if (__syncthreads_or(*abort_flag != 0)) break;

      // gather the Q rows of this tile (zero rows past the entry count)
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int idx = it * kAttnThreads + tid;
        const int row = idx >> 4, ch = idx & 15;
        const int e = ent_s[row / R];
        const int hr = row % R;
        const int64_t qi = (int64_t)(e >> 4);
        const bool ok = (e >= 0) && (qi < n_q);
        const __nv_bfloat16* src =
            ok ? q + (int64_t)b * qs_b + qi * qs_t + (int64_t)(g * R + hr) * qs_h + ch * 8 : q;
        uint8_t* dst = sq + (ch >> 3) * 16384 + row * 128 + ((((ch & 7) ^ (row & 7))) << 4);
        cp_async_16(dst, src, ok ? 16u : 0u);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncthreads();

      // S = Q K^T
      if (tid == 0) {
        bool ok = true;
        if (cpos == pos) ok = mbar_wait(kv_full, kv_phase, abort_flag, err);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem, smem_desc_sw128(sq_a + off, 16, 1024),
                      smem_desc_sw128(sk_a + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(mma_done);
        }
      }
      mbar_wait(mma_done, mma_phase, abort_flag, err);
      mma_phase ^= 1;
      tc_fence_after();

      // softmax piece of row `tid`
      const int row = tid;
      const int e = ent_s[row / R];
      const int hr = row % R;
      const int64_t qi = (int64_t)(e >> 4);
      const int slot = e & 15;
      bool valid = (e >= 0) && (qi < n_q);
      int lim = 127;   // last key offset inside the block visible to the row
      if (valid) {
        const int64_t t = q_pos0 + qi;
        const int64_t rel = t - (int64_t)c * kBlock;
        if (rel < 0) {
          valid = false;
          report(err, MSA_DEVERR_BAD_ENTRY);
        } else if (rel < 127) {
          lim = (int)rel;
        }
      }
      float sv_[128];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_base + j * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) sv_[j * 32 + x] = u2f(r[x]);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int x = 0; x < 128; ++x)
        if (x <= lim) mx = fmaxf(mx, sv_[x]);
      if (!valid) mx = 0.f;
      const float mneg = -mx * scale_log2;
      float l = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int k0 = j * 8 + 2 * x;
          float p0 = (valid && k0 <= lim) ? exp2f(fmaf(sv_[k0], scale_log2, mneg)) : 0.f;
          float p1 = (valid && k0 + 1 <= lim) ? exp2f(fmaf(sv_[k0 + 1], scale_log2, mneg)) : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          l += __low2float(h2) + __high2float(h2);
          w[x] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        uint8_t* dst = sq + (j >> 3) * 16384 + row * 128 + ((((j & 7) ^ (row & 7))) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();

      // O = P V
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16(tmem + 128, smem_desc_sw128(sq_a + aoff, 16, 1024),
                    smem_desc_sw128(sv_a + kk * 2048, 16384, 1024), kIdescPV, kk > 0 ? 1u : 0u);
        }
        umma_commit(mma_done);
      }
      mbar_wait(mma_done, mma_phase, abort_flag, err);
      mma_phase ^= 1;
      tc_fence_after();

      // write the piece
      const int64_t pidx =
          valid ? ((((int64_t)b * n_q + qi) * H + (g * R + hr)) * kTopK + slot) : 0;
      if (valid) {
        *reinterpret_cast<float2*>(part_ml + pidx * 2) = make_float2(mx * scale, l);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_base + 128 + j * 32, r);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(part_acc + pidx * kHeadDim + j * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            dst[x] = make_float4(u2f(r[4 * x]), u2f(r[4 * x + 1]), u2f(r[4 * x + 2]),
                                 u2f(r[4 * x + 3]));
        }
      }
      tc_fence_before();
    }
    kv_phase ^= 1;
    pos = pend;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int R>
static cudaError_t launch_attn_r(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                                 int64_t qs_b, int64_t qs_t, int64_t qs_h,
                                 const int32_t* blk_offsets, const int32_t* entries,
                                 int64_t n_seg, int64_t n_entries, int64_t n_q, int64_t q_pos0,
                                 int32_t G, int32_t H, int32_t nblk, float scale, float* part_ml,
                                 float* part_acc, int32_t* err, cudaStream_t st) {
  constexpr int W = (128 / R) * kAttnChunksPerItem;
  auto k = sparse_attn_fwd_kernel<R>;
  cudaError_t e =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t items = (n_entries + W - 1) / W;
  if (items == 0) return cudaSuccess;
  k<<<(unsigned)items, kAttnThreads, kAttnSmemBytes, st>>>(
      tm_k, tm_v, reinterpret_cast<const __nv_bfloat16*>(q), qs_b, qs_t, qs_h, blk_offsets,
      entries, n_seg, n_entries, n_q, q_pos0, G, H, nblk, scale, part_ml, part_acc, err);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                               int64_t qs_b, int64_t qs_t, int64_t qs_h,
                               const int32_t* blk_offsets, const int32_t* entries,
                               int64_t n_seg, int64_t n_entries, int64_t n_q, int64_t q_pos0,
                               int32_t G, int32_t H, int32_t nblk, float scale, float* part_ml,
                               float* part_acc, int32_t* err, cudaStream_t st) {
  const int R = H / G;
#define MSA_ATTN_CASE(RR)                                                                     \
  case RR:                                                                                    \
    return launch_attn_r<RR>(tm_k, tm_v, q, qs_b, qs_t, qs_h, blk_offsets, entries, n_seg,    \
                             n_entries, n_q, q_pos0, G, H, nblk, scale, part_ml, part_acc, err, \
                             st);
  switch (R) {
    MSA_ATTN_CASE(1)
    MSA_ATTN_CASE(2)
    MSA_ATTN_CASE(4)
    MSA_ATTN_CASE(8)
    MSA_ATTN_CASE(16)
    default:
      return cudaErrorInvalidValue;
  }
#undef MSA_ATTN_CASE
}

}  // namespace msa
