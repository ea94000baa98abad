// Selection recall and the index branch's alignment target, for sampled query
// rows: the main branch's full causal attention mass per 128-token block (the
// teacher), the share of it the chosen blocks hold (recall), and the KL
// divergences between the teacher and the index branch's block softmax (the
// student).  Source: page "MSA 稀疏注意力三国杀", section "索引分支训练：KL 对齐"
// (the index branch learns the main branch's attention distribution through a
// KL divergence, teacher gradient stopped; its blocks hold most of the main
// branch's weight); page "稀疏注意力速览", section 4, MSA entry (KL loss that
// aligns the index distribution to the main branch's probabilities).
//
// For row (b, t) and group g, over blocks c = 0 .. own(t) and keys j <= t:
//   teacher P(c) = mean over the group's R heads h of
//                  sum_{j in c} softmax_h(j), softmax over all j <= t of s_h(j)
//   student Q(c) = softmax over c of z(c) = max_{j in c} q_idx[g] . k_idx[j]
//   recall = sum of P over the selected blocks; kl_pq = KL(P || Q), kl_qp = KL(Q || P)
//
// Two kernels:
//  * block_logmass_kernel -- one CTA per (sampled row, group): warp 0 streams
//    every causal block's K, k_idx and the query's R head rows by TMA into a
//    3-stage ring; consumer warp w owns stage w and writes, per block, each
//    head's log-mass a_h(c) = log sum_{j in c} exp(s_h(j)) (S^T = K Q^T by
//    mma.sync, heads as the 8-wide side) and the block's index score z(c)
//    (k_idx times the index query, mma.sync with one live column);
//  * recall_reduce_kernel -- one warp per (row, group): lse_h = log sum_c
//    exp(a_h(c)), P(c) = mean_h exp(a_h(c) - lse_h), Q from z, recall, KL,
//    and (optionally) lse_h itself, the full causal attention's log-normaliser.
#include "common.cuh"

namespace msa {

constexpr int kRcStages = 3;
constexpr int kRcThreads = 32 * (1 + kRcStages);
constexpr int kRcOffK = 0, kRcOffKi = 32768, kRcOffQ = 65536;
constexpr int kRcStageBytes = 65536 + 2048;      // K, k_idx (<= 32 KB), Q (2 panels x 8 rows)
constexpr int kRcOffBar = kRcStages * kRcStageBytes;
constexpr int kRcSmemBytes = 1024 + kRcOffBar + 2 * kRcStages * 8 + kRcStages * 8 + 16;

struct RecallArgs {
  const int64_t* rows;          // sampled rows: b * n_q + qi
  const __nv_bfloat16* q_idx;   // [B, n_q, G, d_idx]
  int64_t qis_b, qis_t, qis_h;
  int64_t n_rows, n_q, q_pos0, batch;
  int32_t G, d_idx, h_kidx, nblk;
  float scale;
  float* logmass;               // [n_rows, G, nblk, R]
  float* zblk;                  // [n_rows, G, nblk]
  int32_t* err;
};

template <int R>
__global__ void __launch_bounds__(kRcThreads, 1)
    block_logmass_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_ki,
                         const __grid_constant__ RecallArgs a) {
  static_assert(R >= 1 && R <= 8, "heads of a group are the N = 8 side of the tiles");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kRcOffBar);
  uint64_t* empty = full + kRcStages;
  int32_t* stage_c = reinterpret_cast<int32_t*>(empty + kRcStages);   // block of each stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(stage_c + 2 * kRcStages);
  int32_t* err = a.err;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t unit = blockIdx.x;                 // (sampled row, group)
  const int64_t row = a.rows[unit / a.G];
  if (row < 0 || row >= a.batch * a.n_q) {         // uniform for the block
    if (threadIdx.x == 0) report(err, MSA_DEVERR_BAD_ENTRY);
    return;
  }
  const int32_t g = (int32_t)(unit % a.G);
  const int64_t b = row / a.n_q, qi = row - b * a.n_q;
  const int64_t t = a.q_pos0 + qi;
  const int32_t nb = (int32_t)(t / kBlock) + 1;    // causal blocks 0 .. own
  const int hk = (a.h_kidx == 1) ? 0 : g;
  const int kpanels = a.d_idx / 64;

  for (int i = threadIdx.x; i < kRcStages * 128; i += kRcThreads) {
    const int s = i >> 7, k = i & 127;
    reinterpret_cast<uint4*>(base + s * kRcStageBytes + kRcOffQ)[k] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRcStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_ki);
      int32_t n = 0;
      for (; n < nb + kRcStages; ++n) {              // blocks, then one end marker per stage
        const int s = n % kRcStages;
        if (n >= kRcStages &&
            !mbar_wait(empty + s, (uint32_t)(((n / kRcStages) - 1) & 1), abort_flag, err))
          break;
        uint8_t* st = base + s * kRcStageBytes;
        if (n < nb) {
          stage_c[s] = n;
          mbar_arrive_expect_tx(full + s, 32768 + kpanels * 16384 + 2 * R * 128);
          for (int p = 0; p < 2; ++p) {
            tma_load_4d(st + kRcOffK + p * 16384, &tm_k, full + s, p * 64, n * kBlock, g, (int32_t)b);
            tma_load_4d(st + kRcOffQ + p * 1024, &tm_q, full + s, p * 64, g * R, (int32_t)qi,
                        (int32_t)b);
          }
          for (int p = 0; p < kpanels; ++p)
            tma_load_4d(st + kRcOffKi + p * 16384, &tm_ki, full + s, p * 64, n * kBlock, hk,
                        (int32_t)b);
        } else {
          stage_c[s] = -1;
          mbar_arrive(full + s);
        }
      }
      for (int32_t j = (n > kRcStages ? n - kRcStages : 0); j < n; ++j)
        mbar_drain(full + j % kRcStages, (uint32_t)((j / kRcStages) & 1), err);
    }
  } else {
    const int s = warp - 1;
    uint8_t* st = base + s * kRcStageBytes;
    const uint32_t k_s = smem_u32(st + kRcOffK), ki_s = smem_u32(st + kRcOffKi);
    const uint8_t* q_s = st + kRcOffQ;
    const int gq = lane >> 2, tq = lane & 3;
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int hi16 = lane >> 4;
    const float scale_log2 = a.scale * 1.4426950408889634f;
    // index query fragments: column 0 of B holds q_idx (lanes with gq == 0)
    const __nv_bfloat16* qip = a.q_idx + b * a.qis_b + qi * a.qis_t + (int64_t)g * a.qis_h;
    uint32_t bi[16];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const bool live = gq == 0 && ks < a.d_idx / 16;
      bi[2 * ks] = live ? *reinterpret_cast<const uint32_t*>(qip + 16 * ks + 2 * tq) : 0u;
      bi[2 * ks + 1] = live ? *reinterpret_cast<const uint32_t*>(qip + 16 * ks + 8 + 2 * tq) : 0u;
    }
    const int64_t unit_base = unit * (int64_t)a.nblk;
    for (int64_t it = 0;; ++it) {
      if (!mbar_wait(full + s, (uint32_t)(it & 1), abort_flag, err)) break;
      const int32_t c = stage_c[s];
      if (c < 0) break;
      const int lim = (int)min64(t - (int64_t)c * kBlock, 127);   // last causal key of the block

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
      // z: index scores of the block's keys (column 0 of the product)
      float zac[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) zac[mt][0] = zac[mt][1] = zac[mt][2] = zac[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        if (ks < a.d_idx / 16) {
          const uint32_t kiaddr =
              ki_s + (ks >> 2) * 16384 + lrow * 128 +
              (((uint32_t)(2 * (ks & 3) + hi16) ^ (uint32_t)(lane & 7)) << 4);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(kiaddr + mt * 2048, a0, a1, a2, a3);
            mma_bf16_16816(zac[mt], a0, a1, a2, a3, bi[2 * ks], bi[2 * ks + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);        // the stage's K, k_idx and Q are consumed

      float m0 = -INFINITY, m1 = -INFINITY, zm = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const bool v0 = 16 * mt + gq <= lim, v1 = 16 * mt + gq + 8 <= lim;
        if (!v0) acc[mt][0] = acc[mt][1] = -INFINITY;
        if (!v1) acc[mt][2] = acc[mt][3] = -INFINITY;
        m0 = fmaxf(m0, fmaxf(acc[mt][0], acc[mt][2]));
        m1 = fmaxf(m1, fmaxf(acc[mt][1], acc[mt][3]));
        zm = fmaxf(zm, fmaxf(v0 ? zac[mt][0] : -INFINITY, v1 ? zac[mt][2] : -INFINITY));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        zm = fmaxf(zm, __shfl_xor_sync(0xffffffffu, zm, o));
      }
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        l0 += ex2_approx((acc[mt][0] - m0) * scale_log2) + ex2_approx((acc[mt][2] - m0) * scale_log2);
        l1 += ex2_approx((acc[mt][1] - m1) * scale_log2) + ex2_approx((acc[mt][3] - m1) * scale_log2);
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      // a_h(c) = log sum_{j in c} exp(s_h(j)) = m scale + log l
      float* lm = a.logmass + (unit_base + c) * R;
      if (gq == 0) {
        if (2 * tq < R) lm[2 * tq] = m0 * a.scale + logf(l0);
        if (2 * tq + 1 < R) lm[2 * tq + 1] = m1 * a.scale + logf(l1);
      }
      if (lane == 0) a.zblk[unit_base + c] = zm;     // column 0 lives in lanes with tq == 0
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256)
    recall_reduce_kernel(const RecallArgs a, int32_t R, const int32_t* __restrict__ sel,
                         float* __restrict__ block_mass, int64_t mass_stride,
                         float* __restrict__ recall, float* __restrict__ kl_pq,
                         float* __restrict__ kl_qp, float* __restrict__ lse_full) {
  const int lane = threadIdx.x & 31;
  const int64_t unit = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (unit >= a.n_rows * a.G) return;
  const int64_t row = a.rows[unit / a.G];
  if (row < 0 || row >= a.batch * a.n_q) return;   // reported by the first kernel
  const int32_t g = (int32_t)(unit % a.G);
  const int64_t b = row / a.n_q, qi = row - b * a.n_q;
  const int32_t nb = (int32_t)((a.q_pos0 + qi) / kBlock) + 1;
  const float* lm = a.logmass + unit * (int64_t)a.nblk * R;
  const float* z = a.zblk + unit * (int64_t)a.nblk;
  float* P = block_mass + unit * mass_stride;

  auto wmax = [](float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
  };
  auto wsum = [](float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  };
  // per-head normaliser over all causal blocks
  float lse[8];
  for (int h = 0; h < R; ++h) {
    float m = -INFINITY;
    for (int c = lane; c < nb; c += 32) m = fmaxf(m, lm[(int64_t)c * R + h]);
    m = wmax(m);
    float s = 0.f;
    for (int c = lane; c < nb; c += 32) s += expf(lm[(int64_t)c * R + h] - m);
    lse[h] = m + logf(wsum(s));
  }
  // student normaliser
  float zmax = -INFINITY;
  for (int c = lane; c < nb; c += 32) zmax = fmaxf(zmax, z[c]);
  zmax = wmax(zmax);
  float zs = 0.f;
  for (int c = lane; c < nb; c += 32) zs += expf(z[c] - zmax);
  const float zlog = zmax + logf(wsum(zs));
  float kpq = 0.f, kqp = 0.f;
  for (int c = lane; c < nb; c += 32) {
    float p = 0.f;
    for (int h = 0; h < R; ++h) p += expf(lm[(int64_t)c * R + h] - lse[h]);
    p /= (float)R;
    P[c] = p;
    const float logq = z[c] - zlog;
    const float logp = logf(p);
    if (p > 0.f) kpq += p * (logp - logq);
    kqp += expf(logq) * (logq - logp);
  }
  for (int64_t c = nb + lane; c < mass_stride; c += 32) P[c] = 0.f;
  kpq = wsum(kpq);
  kqp = wsum(kqp);
  __syncwarp();
  float rc = 0.f;
  if (lane < kTopK) {
    const int32_t c = sel[((b * a.G + g) * a.n_q + qi) * kTopK + lane];
    if (c >= 0 && c < nb) rc = P[c];
  }
  rc = wsum(rc);
  if (lane == 0) {
    recall[unit] = rc;
    kl_pq[unit] = kpq;
    kl_qp[unit] = kqp;
    if (lse_full != nullptr)                       // [n_rows, H], head g R + h
      for (int h = 0; h < R; ++h) lse_full[unit * R + h] = lse[h];
  }
}

template <int R>
static cudaError_t launch_recall_r(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                   const CUtensorMap& tm_ki, const RecallArgs& a,
                                   cudaStream_t st) {
  auto k = block_logmass_kernel<R>;
  cudaError_t e =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kRcSmemBytes);
  if (e != cudaSuccess) return e;
  k<<<(unsigned)(a.n_rows * a.G), kRcThreads, kRcSmemBytes, st>>>(tm_q, tm_k, tm_ki, a);
  return cudaGetLastError();
}

size_t recall_workspace(int64_t n_rows, int32_t G, int32_t R, int32_t nblk) {
  return (size_t)n_rows * G * nblk * (R + 1) * sizeof(float);
}

cudaError_t launch_selection_recall(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                    const CUtensorMap& tm_ki, const int64_t* rows,
                                    int64_t n_rows, const void* q_idx, int64_t qis_b,
                                    int64_t qis_t, int64_t qis_h, int64_t batch, int64_t n_q,
                                    int64_t q_pos0, int32_t G, int32_t H, int32_t d_idx,
                                    int32_t h_kidx,
                                    int32_t nblk, float scale, const int32_t* sel,
                                    float* block_mass, int64_t mass_stride, float* recall,
                                    float* kl_pq, float* kl_qp, float* lse_full, void* ws,
                                    int32_t* err, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int32_t R = H / G;
  RecallArgs a;
  a.rows = rows;
  a.q_idx = reinterpret_cast<const __nv_bfloat16*>(q_idx);
  a.qis_b = qis_b;
  a.qis_t = qis_t;
  a.qis_h = qis_h;
  a.n_rows = n_rows;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.batch = batch;
  a.G = G;
  a.d_idx = d_idx;
  a.h_kidx = h_kidx;
  a.nblk = nblk;
  a.scale = scale;
  a.logmass = reinterpret_cast<float*>(ws);
  a.zblk = a.logmass + n_rows * G * (int64_t)nblk * R;
  a.err = err;
  cudaError_t e;
  switch (R) {
    case 1: e = launch_recall_r<1>(tm_q, tm_k, tm_ki, a, st); break;
    case 2: e = launch_recall_r<2>(tm_q, tm_k, tm_ki, a, st); break;
    case 4: e = launch_recall_r<4>(tm_q, tm_k, tm_ki, a, st); break;
    case 8: e = launch_recall_r<8>(tm_q, tm_k, tm_ki, a, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int64_t threads = n_rows * G * 32;
  recall_reduce_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
      a, R, sel, block_mass, mass_stride, recall, kl_pq, kl_qp, lse_full);
  return cudaGetLastError();
}

}  // namespace msa
