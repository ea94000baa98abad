// KV-block-outer sparse attention for one query per sequence (decode).
//
// Same computation and output as sparse_attn_fwd_kernel: for every selected
// (batch, group, KV block) the block's K and V are read once and the query
// rows that chose it -- here the R heads of the single query of the sequence
// -- get a softmax piece (m, l, acc) in fp32.  Source: page
// "MSA 稀疏注意力三国杀", sections "MSA 架构：粗筛 + 精算" and "Kernel 创新：Outer
// Gather Q"; page "稀疏注意力架构革命", section 1.1 (softmax(Q K^T / sqrt(d_k)) V).
//
// With one query per segment a 128-row tensor-core tile would be 1/16 full, so
// this kernel works on warp-level tiles instead (mma.sync m16n8k16, heads as
// the 8-wide N side) and spends its resources on keeping many K/V blocks in
// flight, the decode bound:
//   * work units are (batch x group, half of the selected slots); warp 0
//     finds a unit's selected segments with one coalesced scan of the block
//     offsets and streams each block's K, V (32 KB each) and the query's R
//     head rows by TMA into a 3-stage ring (about 200 KB in flight per SM);
//   * consumer warp w owns stage w: S^T = K Q^T (keys x heads; K through
//     ldmatrix), the causal mask on the query's own block, the per-head
//     softmax piece, P^T through shared memory, O^T = V^T P^T (V through
//     ldmatrix.trans), and the R rows of acc leave by one bulk copy.
// P is rounded to bf16 for the P V product; l sums the fp32 weights.
#include "common.cuh"

namespace msa {

constexpr int kDaStages = 3;
constexpr int kDaConsumers = kDaStages;           // consumer warp 1 + s owns stage s
constexpr int kDaThreads = 32 * (1 + kDaConsumers);
constexpr int kDaSlotsPerUnit = 8;                // selected slots per work unit
constexpr int kDaOffK = 0, kDaOffV = 32768, kDaOffQ = 65536;
constexpr int kDaStageBytes = 65536 + 2048;       // K, V, Q (2 panels x 8 rows x 128 B)
constexpr int kDaOffCons = kDaStages * kDaStageBytes;
constexpr int kDaConsP = 0;                       // P^T [8 heads][128 keys] bf16
constexpr int kDaConsO = 2048;                    // O^T [8 heads][128 dims] fp32
constexpr int kDaConsBytes = 2048 + 4096;
constexpr int kDaOffDesc = kDaOffCons + kDaConsumers * kDaConsBytes;
constexpr int kDaOffBar = kDaOffDesc + kDaStages * 16;
constexpr int kDaSmemBytes = 1024 + kDaOffBar + 2 * kDaStages * 8 + 16;
static_assert(kDaStageBytes % 1024 == 0, "TMA boxes with 128-byte swizzle need 1 KB alignment");

struct DecodeAttnArgs {
  const int32_t* blk_offsets;
  const int32_t* entries;
  int64_t n_bg;                 // batch x groups
  int64_t n_q, q_pos0;
  int32_t G, nblk;
  float scale;
  float* part_ml;
  float* part_acc;
  int32_t* err;
};

struct alignas(16) DecodeDesc {
  int32_t b, g, c, e;           // e < 0: no more work; else the entry's index in `entries`
};

template <int R>
__global__ void __launch_bounds__(kDaThreads, 1)
    sparse_attn_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ DecodeAttnArgs a) {
  static_assert(R >= 1 && R <= 8, "heads of a group are the N = 8 side of the tiles");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  DecodeDesc* desc = reinterpret_cast<DecodeDesc*>(base + kDaOffDesc);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kDaOffBar);
  uint64_t* empty = full + kDaStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDaStages);
  int32_t* err = a.err;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Q panels start zeroed: head rows R..7 of a stage are never loaded
  for (int i = threadIdx.x; i < kDaStages * 128; i += kDaThreads) {
    const int s = i >> 7, k = i & 127;
    reinterpret_cast<uint4*>(base + s * kDaStageBytes + kDaOffQ)[k] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDaStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------- producer: find the unit's segments, stream K, V, Q ----------------
    int64_t n = 0;                       // pieces published so far
    bool ok = true;
    // lane 0 claims the next stage and publishes piece (b, g, c, e)
    auto publish = [&](int32_t b, int32_t g, int32_t c, int32_t e) {
      const int s = (int)(n % kDaStages);
      bool r = true;
      if (lane == 0) {
        if (n >= kDaStages && !mbar_wait(empty + s, (uint32_t)(((n / kDaStages) - 1) & 1),
                                         abort_flag, err)) {
          r = false;
        } else {
          desc[s] = DecodeDesc{b, g, c, e};
          uint8_t* st = base + s * kDaStageBytes;
          if (e >= 0) {
            const int32_t qi = a.entries[e] >> 4;
            mbar_arrive_expect_tx(full + s, 65536 + 2 * R * 128);
            for (int p = 0; p < 2; ++p) {
              tma_load_4d(st + kDaOffK + p * 16384, &tm_k, full + s, p * 64, c * kBlock, g, b);
              tma_load_4d(st + kDaOffV + p * 16384, &tm_v, full + s, p * 64, c * kBlock, g, b);
              tma_load_4d(st + kDaOffQ + p * 1024, &tm_q, full + s, p * 64, g * R, qi, b);
            }
          } else {
            mbar_arrive(full + s);
          }
        }
      }
      ++n;
      return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
    };
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
    }
    const int64_t n_units = a.n_bg * 2;
    for (int64_t u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const int64_t bg = u >> 1;
      const int lo = (int)(u & 1) * kDaSlotsPerUnit, hi = lo + kDaSlotsPerUnit;
      const int32_t b = (int32_t)(bg / a.G), g = (int32_t)(bg - (int64_t)b * a.G);
      const int32_t* off = a.blk_offsets + bg * a.nblk;
      const int32_t first = off[0];
      // segments are ascending in the block index and hold one entry each, so
      // the entry of block c has rank off[c] - first among the query's blocks.
      // The offsets are read 512 blocks at a time, 16 independent loads per lane.
      constexpr int kBatch = 16;
      for (int cb = 0; ok && cb < a.nblk; cb += 32 * kBatch) {
        int32_t v[kBatch + 1];
#pragma unroll
        for (int j = 0; j <= kBatch; ++j) {
          const int c = cb + 32 * j + lane;
          v[j] = (c <= a.nblk) ? off[c] : 0x7FFFFFFF;
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int c = cb + 32 * j + lane;
          const int32_t cur = v[j];
          // off[c + 1]: the next lane's value, or lane 0's of the next row
          const int32_t up = __shfl_down_sync(0xffffffffu, cur, 1);
          const int32_t wrap = __shfl_sync(0xffffffffu, v[j + 1], 0);
          const int32_t nxt = (lane < 31) ? up : wrap;
          const int rank = cur - first;
          const bool take = (c < a.nblk) && nxt > cur && rank >= lo && rank < hi;
          uint32_t m = __ballot_sync(0xffffffffu, take);
          while (ok && m) {
            const int l = __ffs(m) - 1;
            m &= m - 1;
            ok = publish(b, g, cb + 32 * j + l, __shfl_sync(0xffffffffu, cur, l));
          }
        }
        // every later block has a higher rank
        if (__shfl_sync(0xffffffffu, v[kBatch], 0) - first >= hi) break;
      }
    }
    // one end marker per stage
    for (int s = 0; ok && s < kDaStages; ++s) ok = publish(0, 0, 0, -1);
    // no copy may still be writing shared memory when the block exits
    if (lane == 0) {
      for (int64_t j = (n > kDaStages ? n - kDaStages : 0); j < n; ++j)
        mbar_drain(full + j % kDaStages, (uint32_t)((j / kDaStages) & 1), err);
    }
  } else {
    // ---------------- consumers ----------------
    const int s = warp - 1;
    uint8_t* st = base + s * kDaStageBytes;
    uint8_t* cons = base + kDaOffCons + s * kDaConsBytes;
    __nv_bfloat16* ps = reinterpret_cast<__nv_bfloat16*>(cons + kDaConsP);
    float* os = reinterpret_cast<float*>(cons + kDaConsO);
    const uint32_t k_s = smem_u32(st + kDaOffK), v_s = smem_u32(st + kDaOffV);
    const uint8_t* q_s = st + kDaOffQ;
    const int gq = lane >> 2, tq = lane & 3;
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;   // ldmatrix row inside a 16-row tile
    const int hi16 = lane >> 4;
    const float scale_log2 = a.scale * 1.4426950408889634f;
    for (int64_t it = 0;; ++it) {
      if (!mbar_wait(full + s, (uint32_t)(it & 1), abort_flag, err)) break;
      const DecodeDesc d = desc[s];
      if (d.e < 0) break;
      const int32_t ent = a.entries[d.e];
      const int64_t qi = ent >> 4;
      const int64_t lim64 = a.q_pos0 + qi - (int64_t)d.c * kBlock;   // last visible key
      if (qi >= a.n_q || lim64 < 0) {
        report(err, MSA_DEVERR_BAD_ENTRY);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        continue;
      }
      const int lim = (int)min64(lim64, 127);

      // S^T = K Q^T: keys 16 mt + (gq, gq + 8) x heads (2 tq, 2 tq + 1)
      float acc[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int j0 = 2 * (ks & 3);
        const uint8_t* qrow = q_s + (ks >> 2) * 1024 + gq * 128 + 4 * tq;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qrow + ((j0 ^ (gq & 7)) << 4));
        const uint32_t b1 =
            *reinterpret_cast<const uint32_t*>(qrow + (((j0 + 1) ^ (gq & 7)) << 4));
        const uint32_t kaddr = k_s + (ks >> 2) * 16384 + lrow * 128 +
                               (((uint32_t)(j0 + hi16) ^ (uint32_t)(lane & 7)) << 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(kaddr + mt * 2048, a0, a1, a2, a3);
          mma_bf16_16816(acc[mt], a0, a1, a2, a3, b0, b1);
        }
      }
      // causal mask on the query's own block, then the per-head maxima
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        if (16 * mt + gq > lim) acc[mt][0] = acc[mt][1] = -INFINITY;
        if (16 * mt + gq + 8 > lim) acc[mt][2] = acc[mt][3] = -INFINITY;
        m0 = fmaxf(m0, fmaxf(acc[mt][0], acc[mt][2]));
        m1 = fmaxf(m1, fmaxf(acc[mt][1], acc[mt][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      const float n0 = -m0 * scale_log2, n1 = -m1 * scale_log2;
      float l0 = 0.f, l1 = 0.f;
      __nv_bfloat16* p0 = ps + (2 * tq) * 128;
      __nv_bfloat16* p1 = ps + (2 * tq + 1) * 128;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const float e0 = ex2_approx(fmaf(acc[mt][0], scale_log2, n0));
        const float e1 = ex2_approx(fmaf(acc[mt][1], scale_log2, n1));
        const float e2 = ex2_approx(fmaf(acc[mt][2], scale_log2, n0));
        const float e3 = ex2_approx(fmaf(acc[mt][3], scale_log2, n1));
        l0 += e0 + e2;
        l1 += e1 + e3;
        p0[16 * mt + gq] = __float2bfloat16_rn(e0);
        p1[16 * mt + gq] = __float2bfloat16_rn(e1);
        p0[16 * mt + gq + 8] = __float2bfloat16_rn(e2);
        p1[16 * mt + gq + 8] = __float2bfloat16_rn(e3);
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      __syncwarp();

      // O^T = V^T P^T: dims 16 mt + (gq, gq + 8) x heads (2 tq, 2 tq + 1)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      const __nv_bfloat16* prow = ps + gq * 128 + 2 * tq;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(prow + 16 * ks);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(prow + 16 * ks + 8);
        const int kr = 16 * ks + (lane & 7) + 8 * hi16;          // key row of this lane
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const uint32_t chunk = (uint32_t)(2 * (mt & 3) + ((lane >> 3) & 1));
          const uint32_t vaddr =
              v_s + (mt >> 2) * 16384 + kr * 128 + ((chunk ^ (uint32_t)(kr & 7)) << 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(vaddr, a0, a1, a2, a3);
          mma_bf16_16816(acc[mt], a0, a1, a2, a3, b0, b1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);          // K, V and Q of the stage are consumed

      // pieces in list order: the R head rows of the entry at position d.e
      const int64_t prow0 = (int64_t)d.e * R;
      if (lane == 0) bulk_wait_read();                 // the previous piece left the staging
      __syncwarp();
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        os[(2 * tq) * 128 + 16 * mt + gq] = acc[mt][0];
        os[(2 * tq + 1) * 128 + 16 * mt + gq] = acc[mt][1];
        os[(2 * tq) * 128 + 16 * mt + gq + 8] = acc[mt][2];
        os[(2 * tq + 1) * 128 + 16 * mt + gq + 8] = acc[mt][3];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        bulk_store_s2g(a.part_acc + prow0 * kHeadDim, os, R * kHeadDim * 4);
        bulk_commit();
      }
      if (gq == 0) {
        if (2 * tq < R)
          *reinterpret_cast<float2*>(a.part_ml + (prow0 + 2 * tq) * 2) =
              make_float2(m0 * a.scale, l0);
        if (2 * tq + 1 < R)
          *reinterpret_cast<float2*>(a.part_ml + (prow0 + 2 * tq + 1) * 2) =
              make_float2(m1 * a.scale, l1);
      }
    }
    if (lane == 0) bulk_wait_all();                    // every piece has landed
  }
  __syncthreads();
}

template <int R>
static cudaError_t launch_decode_r(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                   const CUtensorMap& tm_v, const DecodeAttnArgs& a,
                                   cudaStream_t st) {
  auto k = sparse_attn_decode_kernel<R>;
  cudaError_t e =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kDaSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = min64(a.n_bg * 2, sms);
  k<<<(unsigned)grid, kDaThreads, kDaSmemBytes, st>>>(tm_q, tm_k, tm_v, a);
  return cudaGetLastError();
}

// One query per sequence and R <= 8 heads per group; the caller checked both.
cudaError_t launch_sparse_attn_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                      const CUtensorMap& tm_v, const int32_t* blk_offsets,
                                      const int32_t* entries, int64_t n_bg, int64_t n_q,
                                      int64_t q_pos0, int32_t G, int32_t H, int32_t nblk,
                                      float scale, float* part_ml, float* part_acc,
                                      int32_t* err, cudaStream_t st) {
  if (n_bg == 0) return cudaSuccess;
  DecodeAttnArgs a;
  a.blk_offsets = blk_offsets;
  a.entries = entries;
  a.n_bg = n_bg;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.G = G;
  a.nblk = nblk;
  a.scale = scale;
  a.part_ml = part_ml;
  a.part_acc = part_acc;
  a.err = err;
  switch (H / G) {
    case 1: return launch_decode_r<1>(tm_q, tm_k, tm_v, a, st);
    case 2: return launch_decode_r<2>(tm_q, tm_k, tm_v, a, st);
    case 4: return launch_decode_r<4>(tm_q, tm_k, tm_v, a, st);
    case 8: return launch_decode_r<8>(tm_q, tm_k, tm_v, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace msa
