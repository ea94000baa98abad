// Token-level selection at the same budget, for sampled query rows: the top
// min(budget, t + 1) keys j <= t by index score q_idx[g] . k_idx[j] (score
// descending, lower index first among equal scores), and exact softmax
// attention over them for each head of the group.  This is the granularity of
// the other selection method the pages weigh MSA against (page "MSA 稀疏注意力
// 三国杀", section "分歧一：颗粒度——token 级还是块级？"; page "稀疏注意力速览",
// section 4; page "Sparse attention · DSA và MSA chọn vị trí"); with 2048
// tokens it spends the same key budget as 16 blocks of 128.  It serves to
// compare token- and block-level selection on the same inputs.
//
// Three kernels, one CTA per (sampled row, group) each:
//  * token_scores_kernel -- warp 0 streams the row's causal k_idx blocks by
//    TMA into a 4-stage ring; consumer warp w owns stage w and scores each
//    block's 128 keys against the index query (mma.sync, one live column)
//    into a score row of the workspace;
//  * token_topk_kernel -- exact radix select over order-preserving 32-bit
//    keys (4 passes of 8 bits, warp-aggregated shared histograms), then an
//    index-ordered compaction: every key above the threshold and the
//    lowest-index keys equal to it, written in ascending token order;
//  * token_attention_kernel<R> -- four warps, warp w over every fourth
//    64-token tile of the list: the tile's K and V rows gathered by cp.async
//    into swizzled shared memory, S^T = K Q^T and O^T += V^T P^T by mma.sync
//    (the group's R <= 8 heads are the 8-wide side), online softmax per head;
//    the four warps' states merge at the end into out and lse (fp32).
#include "common.cuh"

namespace msa {

struct TokenArgs {
  const int64_t* rows;          // sampled rows: b * n_q + qi
  const __nv_bfloat16* q;       // [B, n_q, H, 128]
  int64_t qs_b, qs_t, qs_h;
  const __nv_bfloat16* q_idx;   // [B, n_q, G, d_idx]
  int64_t qis_b, qis_t, qis_h;
  const __nv_bfloat16* k;       // [B, G, n_kv, 128]
  const __nv_bfloat16* v;
  int64_t ks_b, ks_t, ks_h, vs_b, vs_t, vs_h;
  int64_t n_rows, n_q, n_kv, q_pos0, batch, budget;
  int32_t G, H, d_idx, h_kidx;
  float scale;
  float* scores;                // [n_rows * G, n_kv] (workspace)
  int32_t* tokens;              // [n_rows * G, budget], ascending, -1 padded
  float* out;                   // [n_rows, H, 128]
  float* lse;                   // [n_rows, H]
  int32_t* err;
};

// (b, qi) of the unit's sampled row; false for a row outside [0, B * n_q)
__device__ __forceinline__ bool unit_row(const TokenArgs& a, int64_t unit, int64_t& b,
                                         int64_t& qi) {
  const int64_t row = a.rows[unit / a.G];
  if (row < 0 || row >= a.batch * a.n_q) return false;
  b = row / a.n_q;
  qi = row - b * a.n_q;
  return true;
}

// ---------------------------------------------------------------------------
// index scores of every causal key
// ---------------------------------------------------------------------------
constexpr int kTsStages = 4;
constexpr int kTsThreads = 32 * (1 + kTsStages);
constexpr int kTsStageBytes = 32768;               // 128 keys x <= 128 dims, bf16
constexpr int kTsOffBar = kTsStages * kTsStageBytes;
constexpr int kTsSmemBytes = 1024 + kTsOffBar + 2 * kTsStages * 8 + kTsStages * 4 + 16;

__global__ void __launch_bounds__(kTsThreads, 1)
    token_scores_kernel(const __grid_constant__ CUtensorMap tm_ki,
                        const __grid_constant__ TokenArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kTsOffBar);
  uint64_t* empty = full + kTsStages;
  int32_t* stage_c = reinterpret_cast<int32_t*>(empty + kTsStages);   // block of each stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(stage_c + kTsStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = blockIdx.x;
  int64_t b, qi;
  if (!unit_row(a, unit, b, qi)) {                 // uniform for the block
    if (threadIdx.x == 0) report(a.err, MSA_DEVERR_BAD_ENTRY);
    return;
  }
  const int32_t g = (int32_t)(unit % a.G);
  const int64_t t = a.q_pos0 + qi;
  const int32_t nb = (int32_t)(t / kBlock) + 1;    // causal blocks 0 .. own
  const int hk = (a.h_kidx == 1) ? 0 : g;
  const int kpanels = a.d_idx / 64;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTsStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_ki);
      // fills n = 0 .. nb - 1 carry block n; fills nb .. nb + 3 are end marks,
      // one per consumer
      int32_t n = 0;
      for (; n < nb + kTsStages; ++n) {
        const int s = n % kTsStages;
        if (n >= kTsStages &&
            !mbar_wait(empty + s, (uint32_t)(((n / kTsStages) - 1) & 1), abort_flag, a.err))
          break;
        if (n < nb) {
          stage_c[s] = n;
          mbar_arrive_expect_tx(full + s, (uint32_t)kpanels * 16384u);
          for (int p = 0; p < kpanels; ++p)
            tma_load_4d(base + s * kTsStageBytes + p * 16384, &tm_ki, full + s, p * 64,
                        n * kBlock, hk, (int32_t)b);
        } else {
          stage_c[s] = -1;
          mbar_arrive(full + s);
        }
      }
      for (int32_t j = (n > kTsStages ? n - kTsStages : 0); j < n; ++j)
        mbar_drain(full + j % kTsStages, (uint32_t)((j / kTsStages) & 1), a.err);
    }
  } else {
    const int w = warp - 1;                        // owns stage w: fills w, w + 4, ...
    const int gq = lane >> 2, tq = lane & 3;
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int hi16 = lane >> 4;
    const int ksteps = a.d_idx / 16;
    // index query as the B operand: column 0 live (lanes gq == 0), dims 16 ks + 2 tq (+ 8)
    const __nv_bfloat16* qip = a.q_idx + b * a.qis_b + qi * a.qis_t + (int64_t)g * a.qis_h;
    uint32_t bi[16];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const bool live = gq == 0 && ks < ksteps;
      bi[2 * ks] = live ? *reinterpret_cast<const uint32_t*>(qip + 16 * ks + 2 * tq) : 0u;
      bi[2 * ks + 1] = live ? *reinterpret_cast<const uint32_t*>(qip + 16 * ks + 8 + 2 * tq) : 0u;
    }
    float* srow = a.scores + unit * a.n_kv;
    const uint32_t ki_s = smem_u32(base + w * kTsStageBytes);
    for (int32_t n = w;; n += kTsStages) {
      if (!mbar_wait(full + w, (uint32_t)((n / kTsStages) & 1), abort_flag, a.err)) break;
      const int32_t c = stage_c[w];
      if (c < 0) break;
      float zac[8][4];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) zac[mt][0] = zac[mt][1] = zac[mt][2] = zac[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        if (ks < ksteps) {
          // rows 16 mt + lrow, 16-byte chunk 2 (ks % 4) + hi16 of panel ks / 4 (128-byte swizzle)
          const uint32_t kaddr = ki_s + (ks >> 2) * 16384 + lrow * 128 +
                                 (((uint32_t)(2 * (ks & 3) + hi16) ^ (uint32_t)(lane & 7)) << 4);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(kaddr + mt * 2048, a0, a1, a2, a3);
            mma_bf16_16816(zac[mt], a0, a1, a2, a3, bi[2 * ks], bi[2 * ks + 1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + w);
      if (tq == 0) {                               // column 0: keys 16 mt + gq and + 8
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int64_t j0 = (int64_t)c * kBlock + 16 * mt + gq;
          if (j0 < a.n_kv) srow[j0] = zac[mt][0];
          if (j0 + 8 < a.n_kv) srow[j0 + 8] = zac[mt][2];
        }
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// top-budget select
// ---------------------------------------------------------------------------
// order-preserving key: u(x) > u(y) exactly when x > y (-0 and +0 equal)
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTkThreads = 1024;

__global__ void __launch_bounds__(kTkThreads)
    token_topk_kernel(const __grid_constant__ TokenArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t wsum[kTkThreads / 32];
  __shared__ uint32_t sh_digit, sh_cum;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x;
  int64_t b, qi;
  if (!unit_row(a, unit, b, qi)) return;           // reported by the scores kernel
  const int64_t n = a.q_pos0 + qi + 1;             // causal keys 0 .. t
  const int64_t kk = min64(a.budget, n);
  const float* srow = a.scores + unit * a.n_kv;
  int32_t* out = a.tokens + unit * a.budget;
  const bool take_all = kk >= n;

  // threshold key T and the number k of keys equal to T that are taken
  uint32_t prefix = 0, mask = 0;
  int64_t k = kk;
  for (int shift = 24; shift >= 0 && !take_all; shift -= 8) {
    for (int i = tid; i < 256; i += kTkThreads) hist[i] = 0;
    __syncthreads();
    for (int64_t j0 = 0; j0 < n; j0 += kTkThreads) {
      const int64_t j = j0 + tid;
      uint32_t bin = 256;                          // no bin
      if (j < n) {
        const uint32_t u = score_key(srow[j]);
        if ((u & mask) == prefix) bin = (u >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane L covers bins 255 - 8 L .. 248 - 8 L; the bin where the running
      // count from the top first reaches k holds the threshold's digit
      uint32_t mine = 0;
      for (int q = 0; q < 8; ++q) mine += hist[255 - (8 * lane + q)];
      uint32_t incl = mine;
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      uint32_t cum = incl - mine;
      int found = -1;
      uint32_t cum_at = 0;
      for (int q = 0; q < 8; ++q) {
        const uint32_t h = hist[255 - (8 * lane + q)];
        if (found < 0 && cum < (uint32_t)k && cum + h >= (uint32_t)k) {
          found = 255 - (8 * lane + q);
          cum_at = cum;
        }
        cum += h;
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, found >= 0);
      if (bal != 0u && lane == __ffs(bal) - 1) {
        sh_digit = (uint32_t)found;
        sh_cum = cum_at;
      }
    }
    __syncthreads();
    prefix |= sh_digit << shift;
    mask |= 255u << shift;
    k -= sh_cum;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // index-ordered compaction: keys above T, then the first k keys equal to T
  uint32_t taken = 0, ties = 0;
  for (int64_t j0 = 0; j0 < n; j0 += kTkThreads) {
    const int64_t j = j0 + tid;
    bool gt = false, eq = false;
    if (j < n) {
      const uint32_t u = score_key(srow[j]);
      gt = take_all || u > T;
      eq = !take_all && u == T;
    }
    const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wsum[warp] = __popc(eqb);
    __syncthreads();
    uint32_t eq_before = ties + __popc(eqb & ((1u << lane) - 1u)), eq_total = 0;
    for (int w = 0; w < kTkThreads / 32; ++w) {
      if (w < warp) eq_before += wsum[w];
      eq_total += wsum[w];
    }
    __syncthreads();
    const bool take = gt || (eq && eq_before < (uint32_t)k);
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    if (lane == 0) wsum[warp] = __popc(tb);
    __syncthreads();
    uint32_t pos = taken + __popc(tb & ((1u << lane) - 1u)), take_total = 0;
    for (int w = 0; w < kTkThreads / 32; ++w) {
      if (w < warp) pos += wsum[w];
      take_total += wsum[w];
    }
    __syncthreads();
    if (take && pos < (uint32_t)a.budget) out[pos] = (int32_t)j;
    taken += take_total;
    ties += eq_total;
  }
  for (int64_t i = kk + tid; i < a.budget; i += kTkThreads) out[i] = -1;
}

// ---------------------------------------------------------------------------
// attention over the chosen tokens
// ---------------------------------------------------------------------------
constexpr int kTaWarps = 4;
constexpr int kTaTile = 64;                                    // tokens per tile
constexpr int kTaPanel = kTaTile * 128;                        // 64 dims of 64 rows, bytes
constexpr int kTaWarpBytes = 4 * kTaPanel + 8 * kTaTile * 2;   // K, V (2 panels each), P^T
constexpr int kTaRedFloats = 8 * 130;                          // per warp: 8 heads x (m, l, o[128])
constexpr int kTaSmemBytes = 1024 + kTaWarps * kTaWarpBytes;
static_assert(kTaWarps * kTaRedFloats * 4 <= kTaWarps * kTaWarpBytes, "merge area fits");

template <int R>
__global__ void __launch_bounds__(kTaWarps * 32, 1)
    token_attention_kernel(const __grid_constant__ TokenArgs a) {
  static_assert(R >= 1 && R <= 8, "heads of a group are the N = 8 side of the tiles");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = blockIdx.x;
  int64_t b, qi;
  if (!unit_row(a, unit, b, qi)) return;           // reported by the scores kernel
  const int64_t r_s = unit / a.G;                  // sample index
  const int32_t g = (int32_t)(unit % a.G);
  const int64_t ntok = min64(a.budget, a.q_pos0 + qi + 1);
  const int32_t* toks = a.tokens + unit * a.budget;
  uint8_t* ks = base + warp * kTaWarpBytes;        // [panel][row][128 B], 128-byte swizzle
  uint8_t* vs = ks + 2 * kTaPanel;
  __nv_bfloat16* ps = reinterpret_cast<__nv_bfloat16*>(vs + 2 * kTaPanel);   // P^T [8][64]
  const int gq = lane >> 2, tq = lane & 3;
  const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int hi16 = lane >> 4;
  const float scale_log2 = a.scale * 1.4426950408889634f;

  // Q^T as the B operand: head gq (< R), dims 16 s + 2 tq (+ 8)
  const __nv_bfloat16* qh =
      a.q + b * a.qs_b + qi * a.qs_t + (int64_t)(g * R + (gq < R ? gq : 0)) * a.qs_h;
  uint32_t bq[16];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    bq[2 * s] = gq < R ? *reinterpret_cast<const uint32_t*>(qh + 16 * s + 2 * tq) : 0u;
    bq[2 * s + 1] = gq < R ? *reinterpret_cast<const uint32_t*>(qh + 16 * s + 8 + 2 * tq) : 0u;
  }
  const __nv_bfloat16* kb = a.k + b * a.ks_b + (int64_t)g * a.ks_h;
  const __nv_bfloat16* vb = a.v + b * a.vs_b + (int64_t)g * a.vs_h;

  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads 2 tq and 2 tq + 1

  const int64_t ntiles = (ntok + kTaTile - 1) / kTaTile;
  for (int64_t tile = warp; tile < ntiles; tile += kTaWarps) {
    // gather: 16-byte chunk c of row r (token toks[64 tile + r]) goes to panel
    // c / 8, row r, position (c % 8) ^ (r % 8); lane handles chunk lane % 16 of
    // rows 2 it + lane / 16
    const int64_t t0 = tile * kTaTile;
    const int32_t tok_a = (t0 + lane < ntok) ? toks[t0 + lane] : -1;
    const int32_t tok_b = (t0 + 32 + lane < ntok) ? toks[t0 + 32 + lane] : -1;
    const int c = lane & 15;
#pragma unroll 4
    for (int it = 0; it < kTaTile / 2; ++it) {
      const int r = 2 * it + hi16;
      const int32_t ja = __shfl_sync(0xffffffffu, tok_a, r & 31);
      const int32_t jb = __shfl_sync(0xffffffffu, tok_b, r & 31);
      const int32_t j = r < 32 ? ja : jb;
      const bool ok = j >= 0 && j < a.n_kv;
      const uint32_t off = (uint32_t)((c >> 3) * kTaPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4));
      cp_async_16(ks + off, ok ? kb + (int64_t)j * a.ks_t + c * 8 : a.k, ok ? 16u : 0u);
      cp_async_16(vs + off, ok ? vb + (int64_t)j * a.vs_t + c * 8 : a.v, ok ? 16u : 0u);
    }
    cp_async_wait_all();
    __syncwarp();
    const uint32_t k_s = smem_u32(ks), v_s = smem_u32(vs);
    // S^T = K Q^T: tokens 16 mt + gq (and + 8) x heads 2 tq, 2 tq + 1
    float s4[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) s4[mt][0] = s4[mt][1] = s4[mt][2] = s4[mt][3] = 0.f;
#pragma unroll
    for (int kst = 0; kst < 8; ++kst) {
      const uint32_t kaddr = k_s + (kst >> 2) * kTaPanel + lrow * 128 +
                             (((uint32_t)(2 * (kst & 3) + hi16) ^ (uint32_t)(lane & 7)) << 4);
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(kaddr + mt * 2048, a0, a1, a2, a3);
        mma_bf16_16816(s4[mt], a0, a1, a2, a3, bq[2 * kst], bq[2 * kst + 1]);
      }
    }
    // tokens past the list carry no weight
    float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if (t0 + 16 * mt + gq >= ntok) s4[mt][0] = s4[mt][1] = -INFINITY;
      if (t0 + 16 * mt + gq + 8 >= ntok) s4[mt][2] = s4[mt][3] = -INFINITY;
      tm0 = fmaxf(tm0, fmaxf(s4[mt][0], s4[mt][2]));
      tm1 = fmaxf(tm1, fmaxf(s4[mt][1], s4[mt][3]));
    }
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, x));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, x));
    }
    // every tile holds at least one listed token, so the new maxima are finite
    const float nm0 = fmaxf(m0, tm0), nm1 = fmaxf(m1, tm1);
    const float c0 = (m0 == -INFINITY) ? 0.f : ex2_approx((m0 - nm0) * scale_log2);
    const float c1 = (m1 == -INFINITY) ? 0.f : ex2_approx((m1 - nm1) * scale_log2);
    m0 = nm0;
    m1 = nm1;
    l0 *= c0;
    l1 *= c1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o[mt][0] *= c0;
      o[mt][1] *= c1;
      o[mt][2] *= c0;
      o[mt][3] *= c1;
    }
    float tl0 = 0.f, tl1 = 0.f;
    __nv_bfloat16* p0 = ps + (2 * tq) * kTaTile;
    __nv_bfloat16* p1 = p0 + kTaTile;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const float e0 = ex2_approx((s4[mt][0] - m0) * scale_log2);
      const float e1 = ex2_approx((s4[mt][1] - m1) * scale_log2);
      const float e2 = ex2_approx((s4[mt][2] - m0) * scale_log2);
      const float e3 = ex2_approx((s4[mt][3] - m1) * scale_log2);
      tl0 += e0 + e2;
      tl1 += e1 + e3;
      p0[16 * mt + gq] = __float2bfloat16_rn(e0);
      p1[16 * mt + gq] = __float2bfloat16_rn(e1);
      p0[16 * mt + gq + 8] = __float2bfloat16_rn(e2);
      p1[16 * mt + gq + 8] = __float2bfloat16_rn(e3);
    }
#pragma unroll
    for (int x = 4; x < 32; x <<= 1) {
      tl0 += __shfl_xor_sync(0xffffffffu, tl0, x);
      tl1 += __shfl_xor_sync(0xffffffffu, tl1, x);
    }
    l0 += tl0;
    l1 += tl1;
    __syncwarp();
    // O^T += V^T P^T: dims 16 mt + gq (and + 8) x heads 2 tq, 2 tq + 1; V^T
    // fragments come from the token-major V tile by transposing loads
    const __nv_bfloat16* prow = ps + gq * kTaTile + 2 * tq;
#pragma unroll
    for (int kst = 0; kst < 4; ++kst) {
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(prow + 16 * kst);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(prow + 16 * kst + 8);
      const int kr = 16 * kst + (lane & 7) + 8 * hi16;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t chunk = (uint32_t)(2 * (mt & 3) + ((lane >> 3) & 1));
        const uint32_t vaddr = v_s + (mt >> 2) * kTaPanel + kr * 128 +
                               ((chunk ^ (uint32_t)(kr & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(vaddr, a0, a1, a2, a3);
        mma_bf16_16816(o[mt], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncwarp();
  }

  // merge the warps' states: (m, l, O) per head through shared memory (the
  // tiles' area, free once every warp is past its loop)
  __syncthreads();
  float* red = reinterpret_cast<float*>(base);
  float* mine = red + warp * kTaRedFloats;
  if (gq == 0) {
    mine[(2 * tq) * 130 + 0] = m0;
    mine[(2 * tq) * 130 + 1] = l0;
    mine[(2 * tq + 1) * 130 + 0] = m1;
    mine[(2 * tq + 1) * 130 + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    mine[(2 * tq) * 130 + 2 + 16 * mt + gq] = o[mt][0];
    mine[(2 * tq + 1) * 130 + 2 + 16 * mt + gq] = o[mt][1];
    mine[(2 * tq) * 130 + 2 + 16 * mt + gq + 8] = o[mt][2];
    mine[(2 * tq + 1) * 130 + 2 + 16 * mt + gq + 8] = o[mt][3];
  }
  __syncthreads();
  for (int hh = warp; hh < R; hh += kTaWarps) {    // lane: dims 4 lane .. 4 lane + 3
    float M = -INFINITY;
    for (int w = 0; w < kTaWarps; ++w) M = fmaxf(M, red[w * kTaRedFloats + hh * 130]);
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < kTaWarps; ++w) {
      const float* st = red + w * kTaRedFloats + hh * 130;
      const float f = (st[0] == -INFINITY) ? 0.f : ex2_approx((st[0] - M) * scale_log2);
      L += f * st[1];
#pragma unroll
      for (int x = 0; x < 4; ++x) acc[x] += f * st[2 + 4 * lane + x];
    }
    const int64_t h = (int64_t)g * R + hh;
    const float4 res = make_float4(acc[0] / L, acc[1] / L, acc[2] / L, acc[3] / L);
    reinterpret_cast<float4*>(a.out + (r_s * a.H + h) * kHeadDim)[lane] = res;
    if (lane == 0) a.lse[r_s * a.H + h] = M * a.scale + logf(L);
  }
}

size_t token_select_workspace(int64_t n_rows, int32_t G, int64_t n_kv) {
  return (size_t)n_rows * G * n_kv * sizeof(float);
}

cudaError_t launch_token_select_attention(
    const CUtensorMap& tm_ki, const int64_t* rows, int64_t n_rows, const void* q, int64_t qs_b,
    int64_t qs_t, int64_t qs_h, const void* q_idx, int64_t qis_b, int64_t qis_t, int64_t qis_h,
    const void* k, int64_t ks_b, int64_t ks_t, int64_t ks_h, const void* v, int64_t vs_b,
    int64_t vs_t, int64_t vs_h, int64_t batch, int64_t n_q, int64_t n_kv, int64_t q_pos0,
    int32_t G, int32_t H, int32_t d_idx, int32_t h_kidx, float scale, int64_t budget,
    int32_t* tokens, float* out, float* lse, void* ws, int32_t* err, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  TokenArgs a;
  a.rows = rows;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.qs_b = qs_b;
  a.qs_t = qs_t;
  a.qs_h = qs_h;
  a.q_idx = reinterpret_cast<const __nv_bfloat16*>(q_idx);
  a.qis_b = qis_b;
  a.qis_t = qis_t;
  a.qis_h = qis_h;
  a.k = reinterpret_cast<const __nv_bfloat16*>(k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.ks_b = ks_b;
  a.ks_t = ks_t;
  a.ks_h = ks_h;
  a.vs_b = vs_b;
  a.vs_t = vs_t;
  a.vs_h = vs_h;
  a.n_rows = n_rows;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.q_pos0 = q_pos0;
  a.batch = batch;
  a.budget = budget;
  a.G = G;
  a.H = H;
  a.d_idx = d_idx;
  a.h_kidx = h_kidx;
  a.scale = scale;
  a.tokens = tokens;
  a.out = out;
  a.lse = lse;
  a.err = err;
  const int64_t units = a.n_rows * a.G;
  const int32_t R = a.H / a.G;
  a.scores = reinterpret_cast<float*>(ws);
  cudaError_t e = cudaFuncSetAttribute(token_scores_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kTsSmemBytes);
  if (e != cudaSuccess) return e;
  token_scores_kernel<<<(unsigned)units, kTsThreads, kTsSmemBytes, st>>>(tm_ki, a);
  token_topk_kernel<<<(unsigned)units, kTkThreads, 0, st>>>(a);
  switch (R) {
#define MSA_TOKEN_ATTN_CASE(RR)                                                             \
  case RR: {                                                                                \
    auto kern = token_attention_kernel<RR>;                                                 \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,             \
                             kTaSmemBytes);                                                 \
    if (e != cudaSuccess) return e;                                                         \
    kern<<<(unsigned)units, kTaWarps * 32, kTaSmemBytes, st>>>(a);                          \
    break;                                                                                  \
  }
    MSA_TOKEN_ATTN_CASE(1)
    MSA_TOKEN_ATTN_CASE(2)
    MSA_TOKEN_ATTN_CASE(4)
    MSA_TOKEN_ATTN_CASE(8)
#undef MSA_TOKEN_ATTN_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace msa
