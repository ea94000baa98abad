// Index branch: token scores q_idx . k_idx and causal block max-pool, without
// ever storing the score matrix.
//
// Source: page "MSA 稀疏注意力三国杀", section "MSA 架构：粗筛 + 精算", first
// step items 1-2 (score every token of a 128-token block, the block's score is
// its highest token score); page "稀疏注意力速览", section 4, MSA entry (one index
// query head per GQA group, shared index key head, block max-pool).
//
// Two kernels:
//  * index_score_maxpool_kernel -- prefill / chunked prefill.  A 128-query x
//    256-key tile of scores is one tcgen05 MMA (M=128, N=256, K=d_idx) whose
//    fp32 accumulator lives in TMEM; the block max is the row max of that
//    tile, read back with tcgen05.ld (one thread per query row).  Each MMA
//    step covers two key blocks (N = 256, halving shared-memory operand
//    traffic per FLOP).  Warp roles: warp 0 issues TMA loads (the q_idx tile
//    once, pairs of k_idx blocks through a 3-5 stage ring), warp 1 issues the
//    MMAs into two 256-column TMEM accumulators, warps 2-9 take the row maxima
//    (one warp per TMEM lane quarter and block of the pair, all 128 columns in
//    one round of loads) and store them.
//  * index_score_decode_kernel -- one query per sequence (decode): a
//    streaming scan of k_idx, HBM-bound.  TMA streams 32 KB key blocks
//    through a shared-memory ring; consumer warps multiply them by the
//    G <= 8 index queries of the sequence with mma.sync (m16n8k16: keys x
//    groups) and keep each group's block maximum.
#include "common.cuh"

namespace msa {

template <int D, bool F8 = false>
struct IdxCfg {
  static constexpr int kEsz = F8 ? 1 : 2;            // bytes per element
  static constexpr int kHalves = D * kEsz / 128;     // 128-byte column panels
  static constexpr int kPanelElems = 128 / kEsz;     // elements per panel row
  static constexpr int kQBytes = 128 * D * kEsz;     // 128 query rows
  static constexpr int kPairBytes = 256 * D * kEsz;  // two key blocks (256 key rows)
  static constexpr int kKSteps = D * kEsz / 32;      // MMA steps of 32 bytes along K
  static constexpr int kStages = (kPairBytes == 65536) ? 3 : 5;   // k_idx ring depth (pairs)
  static constexpr int kChunkPairs = 64;             // key-block pairs per CTA
  static constexpr int kThreads = 320;               // TMA, MMA, 8 epilogue warps
  static constexpr int kBars = 2 * kStages + 1 + 4;
  static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kPairBytes + kBars * 8 + 16;
};

template <int D, bool F8 = false>
__global__ void __launch_bounds__(320, 1)
    index_score_maxpool_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k, int64_t n_q,
                               int64_t q_pos0, int32_t G, int32_t h_kidx, int32_t n_qtiles,
                               float* __restrict__ pooled, int64_t stride, int32_t* err,
                               const float* __restrict__ scale_q,
                               const float* __restrict__ scale_k) {
  using C = IdxCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk = base + C::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sk + C::kStages * C::kPairBytes);
  uint64_t* full = bars;                        // [kStages] key pair loaded
  uint64_t* empty = bars + C::kStages;          // [kStages] key pair consumed by the MMAs
  uint64_t* qfull = bars + 2 * C::kStages;      // q tile loaded
  uint64_t* accfull = qfull + 1;                // [2] accumulator ready
  uint64_t* accempty = qfull + 3;               // [2] accumulator drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % G;
  const int kc = blockIdx.x / G;
  const int qt = n_qtiles - 1 - (int)blockIdx.y;   // longest rows first
  const int b = blockIdx.z;
  const int64_t q0 = (int64_t)qt * 128;
  const int64_t q_last = min64(q0 + 127, n_q - 1);
  const int64_t nb_tile = (q_pos0 + q_last) / kBlock;   // candidates of the tile's last row
  const int64_t c0 = (int64_t)kc * 2 * C::kChunkPairs;
  if (c0 >= nb_tile) return;                            // uniform: nothing to score
  const int nb = (int)min64(2 * C::kChunkPairs, nb_tile - c0);
  const int np = (nb + 1) >> 1;                         // MMA steps of 256 keys
  const int hk = (h_kidx == 1) ? 0 : g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(accfull + i, 1);
      mbar_init(accempty + i, 8);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      mbar_arrive_expect_tx(qfull, C::kQBytes);
      for (int h = 0; h < C::kHalves; ++h)
        tma_load_4d(sq + h * 16384, &tm_q, qfull, h * C::kPanelElems, g, (int32_t)q0, b);
      for (int i = 0; i < np; ++i) {
        const int s = i % C::kStages;
        if (i >= C::kStages &&
            !mbar_wait(empty + s, ((i / C::kStages) - 1) & 1, abort_flag, err))
          break;
        mbar_arrive_expect_tx(full + s, C::kPairBytes);
        // one box of 256 key rows per 64-column panel (rows past n_kv read as 0)
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_4d(sk + s * C::kPairBytes + h * 32768, &tm_k, full + s, h * C::kPanelElems,
                      (int32_t)((c0 + 2 * i) * kBlock), hk, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(128, 256) : idesc_bf16_f32(128, 256, 0);
      const uint32_t qa = smem_u32(sq);
      bool ok = mbar_wait(qfull, 0, abort_flag, err);
      for (int i = 0; ok && i < np; ++i) {
        const int s = i % C::kStages, a = i & 1;
        if (!mbar_wait(full + s, (i / C::kStages) & 1, abort_flag, err)) break;
        if (i >= 2 && !mbar_wait(accempty + a, ((i >> 1) - 1) & 1, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(sk + s * C::kPairBytes);
#pragma unroll
        for (int kk = 0; kk < C::kKSteps; ++kk) {
          const uint64_t ad = smem_desc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(ka + (kk >> 2) * 32768 + (kk & 3) * 32, 16, 1024);
          if constexpr (F8)
            umma_e4m3(tmem + a * 256, ad, bd, idesc, kk > 0 ? 1u : 0u);
          else
            umma_bf16(tmem + a * 256, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(empty + s);
        umma_commit(accfull + a);
      }
    }
  } else {
    // epilogue: thread = query row; warps 2-5 take columns [0,128) of each
    // accumulator (block c), warps 6-9 columns [128,256) (block c+1)
    const int quarter = warp & 3;
    const int hb = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int64_t q = q0 + row;
    const int64_t own = (q_pos0 + q) / kBlock;
    float* prow = pooled + (((int64_t)b * G + g) * n_q + q) * stride;
    // 8-bit inputs: the codes' product times both tensors' scales
    const float sc = F8 ? scale_q[0] * scale_k[0] : 1.0f;
    for (int i = 0; i < np; ++i) {
      const int a = i & 1;
      if (!mbar_wait(accfull + a, (i >> 1) & 1, abort_flag, err)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t col = tmem + lane_base + a * 256 + hb * 128;
      tmem_ld_32x32b_x32(col, r0);
      tmem_ld_32x32b_x32(col + 32, r1);
      tmem_ld_32x32b_x32(col + 64, r2);
      tmem_ld_32x32b_x32(col + 96, r3);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty + a);
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        m4[0] = fmaxf(m4[0], u2f(r0[x]));
        m4[1] = fmaxf(m4[1], u2f(r1[x]));
        m4[2] = fmaxf(m4[2], u2f(r2[x]));
        m4[3] = fmaxf(m4[3], u2f(r3[x]));
      }
      float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      if (F8) m *= sc;
      const int64_t c = c0 + 2 * i + hb;
      if (q < n_q && c < own && 2 * i + hb < nb) prow[c] = m;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// decode: one query per sequence, d_idx = 128, shared index key head, G <= 8
// ---------------------------------------------------------------------------
// A streaming scan of k_idx.  The units are the (sequence, candidate block)
// pairs, split into one contiguous range per CTA (persistent grid, one CTA
// per SM).  Warp 0 streams each unit's 32 KB key block into a ring of
// shared-memory stages with TMA (two 64-column boxes, 128-byte swizzle), so
// that up to kDecStages x 32 KB per SM are in flight.  Each consumer warp
// owns the stages s with s % kDecConsumers == its index (one consumer per
// stage keeps the barrier phases unambiguous) and multiplies the block by the
// sequence's G <= 8 index queries with mma.sync m16n8k16: A = 16 keys x 16
// dims through ldmatrix, B = the queries held in registers; the block score
// of group g is the maximum of column g over the 128 keys.
constexpr int kDecStages = 6;
constexpr int kDecConsumers = 3;
static_assert(kDecStages % kDecConsumers == 0, "a stage must always have the same consumer");
constexpr int kDecThreads = 32 * (1 + kDecConsumers);
constexpr int kDecStageBytes = kBlock * 128 * 2;    // 128 keys x 128 dims bf16
constexpr int kDecSmemBytes = 1024 + kDecStages * kDecStageBytes + 2 * kDecStages * 8 + 16;

__global__ void __launch_bounds__(kDecThreads, 1)
    index_score_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                              const __nv_bfloat16* __restrict__ q_idx, int64_t qs_b,
                              int64_t qs_h, int64_t batch, int64_t q_pos0, int32_t G,
                              float* __restrict__ pooled, int64_t stride, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kDecStages * kDecStageBytes);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t own = q_pos0 / kBlock;                  // candidates per sequence
  const int64_t total = batch * own;
  const int64_t u0 = total * blockIdx.x / gridDim.x;
  const int n = (int)(total * (blockIdx.x + 1) / gridDim.x - u0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      int i = 0;
      for (; i < n; ++i) {
        const int s = i % kDecStages;
        if (i >= kDecStages &&
            !mbar_wait(empty + s, ((i / kDecStages) - 1) & 1, abort_flag, err))
          break;
        const int64_t u = u0 + i;
        const int64_t b = u / own, c = u - b * own;
        uint8_t* dst = base + s * kDecStageBytes;
        mbar_arrive_expect_tx(full + s, kDecStageBytes);
        tma_load_4d(dst, &tm_k, full + s, 0, (int32_t)(c * kBlock), 0, (int32_t)b);
        tma_load_4d(dst + kDecStageBytes / 2, &tm_k, full + s, 64, (int32_t)(c * kBlock), 0,
                    (int32_t)b);
      }
      // no copy may still be writing this block's shared memory when it exits
      for (int j = (i > kDecStages ? i - kDecStages : 0); j < i; ++j)
        mbar_drain(full + j % kDecStages, (j / kDecStages) & 1, err);
    }
  } else {
    const int cw = warp - 1;
    const int gq = lane >> 2, tq = lane & 3;
    // ldmatrix row of this lane inside a 16-key tile, and its 128-byte swizzle phase
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int hi = lane >> 4;                          // second 8 dims of a k-step
    uint32_t bq[16];
    int64_t qb = -1;
    for (int i = cw; i < n; i += kDecConsumers) {
      const int s = i % kDecStages;
      const int64_t u = u0 + i;
      const int64_t b = u / own, c = u - b * own;
      if (b != qb) {
        // B fragments: k pairs (16 ks + 2 tq, +1) and (16 ks + 8 + 2 tq, +1) of group gq
        const __nv_bfloat16* qp = q_idx + b * qs_b + (int64_t)gq * qs_h + 2 * tq;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          bq[2 * ks] = gq < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks) : 0u;
          bq[2 * ks + 1] = gq < G ? *reinterpret_cast<const uint32_t*>(qp + 16 * ks + 8) : 0u;
        }
        qb = b;
      }
      if (!mbar_wait(full + s, (i / kDecStages) & 1, abort_flag, err)) break;
      const uint32_t sbase = smem_u32(base + s * kDecStageBytes);
      float acc[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        // 16-byte chunk of this lane's row, swizzled by the row (row & 7 == lane & 7)
        const uint32_t chunk = (uint32_t)((2 * (ks & 3) + hi) ^ (lane & 7));
        const uint32_t kaddr = sbase + (ks >> 2) * (kDecStageBytes / 2) + lrow * 128 + chunk * 16;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(kaddr + mt * 16 * 128, a0, a1, a2, a3);
          mma_bf16_16816(acc[mt], a0, a1, a2, a3, bq[2 * ks], bq[2 * ks + 1]);
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;   // groups 2 tq and 2 tq + 1
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        mx0 = fmaxf(mx0, fmaxf(acc[mt][0], acc[mt][2]));
        mx1 = fmaxf(mx1, fmaxf(acc[mt][1], acc[mt][3]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (gq == 0) {
        const int g0 = 2 * tq, g1 = 2 * tq + 1;
        if (g0 < G) pooled[(b * G + g0) * stride + c] = mx0;
        if (g1 < G) pooled[(b * G + g1) * stride + c] = mx1;
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// host launchers (called from the C ABI after validation)
// ---------------------------------------------------------------------------
cudaError_t launch_index_score_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                       int d_idx, int64_t batch, int64_t n_q, int64_t q_pos0,
                                       int32_t G, int32_t h_kidx, float* pooled,
                                       int64_t stride, int32_t* err, cudaStream_t st) {
  const int64_t n_qtiles = (n_q + 127) / 128;
  const int64_t max_nb = (q_pos0 + n_q - 1) / kBlock;
  if (max_nb == 0) return cudaSuccess;
  const int64_t per_cta = 2 * IdxCfg<128>::kChunkPairs;
  const int64_t n_chunks = (max_nb + per_cta - 1) / per_cta;
  dim3 grid((unsigned)(n_chunks * G), (unsigned)n_qtiles, (unsigned)batch);
  if (d_idx == 128) {
    auto k = index_score_maxpool_kernel<128, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         IdxCfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
    k<<<grid, IdxCfg<128>::kThreads, IdxCfg<128>::kSmemBytes, st>>>(
        tm_q, tm_k, n_q, q_pos0, G, h_kidx, (int32_t)n_qtiles, pooled, stride, err, nullptr,
        nullptr);
  } else {
    auto k = index_score_maxpool_kernel<64, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         IdxCfg<64>::kSmemBytes);
    if (e != cudaSuccess) return e;
    k<<<grid, IdxCfg<64>::kThreads, IdxCfg<64>::kSmemBytes, st>>>(
        tm_q, tm_k, n_q, q_pos0, G, h_kidx, (int32_t)n_qtiles, pooled, stride, err, nullptr,
        nullptr);
  }
  return cudaGetLastError();
}

// 8-bit (e4m3) index scores: d_idx = 128, maps over uint8 codes, box {128, ...}.
cudaError_t launch_index_score_e4m3(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                   int64_t batch, int64_t n_q, int64_t q_pos0, int32_t G,
                                   int32_t h_kidx, float* pooled, int64_t stride,
                                   const float* scale_q, const float* scale_k, int32_t* err,
                                   cudaStream_t st) {
  using C = IdxCfg<128, true>;
  const int64_t n_qtiles = (n_q + 127) / 128;
  const int64_t max_nb = (q_pos0 + n_q - 1) / kBlock;
  if (max_nb == 0) return cudaSuccess;
  const int64_t per_cta = 2 * C::kChunkPairs;
  const int64_t n_chunks = (max_nb + per_cta - 1) / per_cta;
  dim3 grid((unsigned)(n_chunks * G), (unsigned)n_qtiles, (unsigned)batch);
  auto k = index_score_maxpool_kernel<128, true>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  k<<<grid, C::kThreads, C::kSmemBytes, st>>>(tm_q, tm_k, n_q, q_pos0, G, h_kidx,
                                               (int32_t)n_qtiles, pooled, stride, err, scale_q,
                                               scale_k);
  return cudaGetLastError();
}

// Per-tensor e4m3 quantisation: amax of |x| (atomic max on the float bits of
// non-negative values), scale = amax / 448 (1 when amax is 0), codes = x /
// scale rounded to the nearest e4m3 value (ties to even, saturating at 448).
__global__ void __launch_bounds__(256)
    amax_bf16_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, uint32_t* amax_bits) {
  float m = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(x[i])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__global__ void __launch_bounds__(256)
    quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x, int64_t n,
                         const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                         float* __restrict__ scale_out) {
  const float amax = __uint_as_float(*amax_bits);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = scale;
  for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const float y0 = __fdiv_rn(__bfloat162float(x[i]), scale);
    const float y1 = (i + 1 < n) ? __fdiv_rn(__bfloat162float(x[i + 1]), scale) : 0.f;
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(y1), "f"(y0));
    codes[i] = (uint8_t)(pair & 0xFF);
    if (i + 1 < n) codes[i + 1] = (uint8_t)(pair >> 8);
  }
}

cudaError_t launch_quantize_e4m3(const void* x, int64_t n, void* codes, float* scale,
                                 cudaStream_t st) {
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(scale + 1);
  cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  if (n == 0) {
    quantize_e4m3_kernel<<<1, 32, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x), 0,
                                           amax_bits, reinterpret_cast<uint8_t*>(codes), scale);
    return cudaGetLastError();
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks = min64((n + 511) / 512, (int64_t)sms * 8);
  amax_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                                     n, amax_bits);
  quantize_e4m3_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), n, amax_bits, reinterpret_cast<uint8_t*>(codes),
      scale);
  return cudaGetLastError();
}

cudaError_t launch_index_score_decode(const CUtensorMap& tm_k, const void* q_idx, int64_t qs_b,
                                      int64_t qs_h, int64_t batch, int64_t q_pos0, int32_t G,
                                      float* pooled, int64_t stride, int32_t* err,
                                      cudaStream_t st) {
  const int64_t total = batch * (q_pos0 / kBlock);
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto k = index_score_decode_kernel;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kDecSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t grid = min64(total, sms);
  k<<<(unsigned)grid, kDecThreads, kDecSmemBytes, st>>>(
      tm_k, reinterpret_cast<const __nv_bfloat16*>(q_idx), qs_b, qs_h, batch, q_pos0, G, pooled,
      stride, err);
  return cudaGetLastError();
}

}  // namespace msa
