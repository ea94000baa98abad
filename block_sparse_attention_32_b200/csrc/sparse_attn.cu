// KV-block-outer sparse attention: for every (batch, group, KV block) segment
// of the block->query lists, the block's K and V tiles are loaded into shared
// memory by TMA once per work item, the query rows that chose the block are
// gathered into 128-row tiles, and S = Q K^T, the softmax piece and O = P V
// run on the tcgen05 tensor cores with fp32 accumulators in TMEM.  Each
// (query, head, slot) gets a piece (m, l, acc) that the merge kernel combines.
//
// Source: page "MSA 稀疏注意力三国杀", section "MSA 架构：粗筛 + 精算" (main
// branch: full attention over the selected blocks only) and section "Kernel
// 创新：Outer Gather Q" (the KV block is the outer loop, all queries that chose
// it are computed together so the block is read once); sparse-attention
// "稀疏注意力速览" page, section 4, MSA entry (exact softmax attention); page
// "稀疏注意力架构革命", section 1.1 (standard attention softmax(Q K^T / sqrt(d_k)) V).
//
// A 128-row tile ("chunk") holds 128 / R query entries x R heads of one group
// (R = h_q / h_kv).  Work items are runs of W consecutive entries; an item
// splits into pieces (one per segment = one K/V block) and pieces into
// chunks.  The kernel is persistent (one CTA per SM) and warp-specialised so
// that consecutive chunks overlap:
//   warp 0      scheduler:    walks the CTA's items (32-ary search of the
//                             segment offsets) and publishes one descriptor
//                             per chunk -- (b, g, block, count, piece, flags)
//                             and its entries -- in an 8-deep shared ring
//   warp 1      MMA issuer:   S(n) = Q K^T, then O(n-1) = P V  (TMEM owner)
//   warp 2      TMA producer: K and V of each piece; K of the next piece is
//                             loaded as soon as the last S MMA of the current
//                             one is done, V as soon as its last P V is done
//   warps 3-6   gather:       cp.async of the chunk's Q rows into a 3-deep ring
//   warps 7-10  softmax:      S -> (m, l), P = bf16(e^{s-m}) written back into
//                             the first 64 columns of its S buffer in TMEM
//                             (the A operand of O = P V)
//   warps 11-14 epilogue:     O -> the (m, l, acc) pieces in global memory:
//                             each warp stages its 32 rows half a row (256 B)
//                             at a time in shared memory and reads them back
//                             transposed, so that one store instruction
//                             writes two whole half rows (coalesced)
// Shared memory: K 32 KB, V 32 KB, 3 x 32 KB Q tiles (128B-swizzled K-major;
// V is read N-major for P V), 34 KB output staging (half rows padded to 272
// bytes so a warp's row-per-thread writes spread over all banks).  TMEM: S/P
// in columns [0,256), O in [256,512), two buffers of 128 columns each; a Q
// tile is released as soon as its S MMA is done, and S(n+2) waits for
// O(n) = P(n) V, which reads P(n) from the same columns.
#include "common.cuh"

namespace msa {

constexpr int kAttnThreads = 480;
constexpr int kAttnMaxChunksPerItem = 8;
constexpr int kQRing = 3;              // Q/P tiles in flight
constexpr int kDescRing = 8;           // chunk descriptors in flight

struct alignas(16) ChunkDesc {
  int32_t b, g, c, cnt;                // cnt < 0: no more work
  int32_t piece, first, last, pad;
  int32_t ent[128];
};

constexpr int kOffK = 0;               // 32768: [K lo | K hi]
constexpr int kOffV = 32768;           // 32768: [V lo | V hi]
constexpr int kOffQP = 65536;          // kQRing x 32768: Q tile, then P
constexpr int kStageRow = 272;                           // staged half row (256 B + pad)
constexpr int kOffStage = kOffQP + kQRing * 32768;       // 128 staged rows
constexpr int kOffML = kOffStage + 128 * kStageRow;      // 2 x 128 float2: (m, l) per row
constexpr int kOffDesc = kOffML + 2048;                  // kDescRing descriptors
constexpr int kOffBar = kOffDesc + kDescRing * (int)sizeof(ChunkDesc);
constexpr int kNumBars = 4 + 3 * kQRing + 6 + 2 * kDescRing;
constexpr int kOffMisc = kOffBar + kNumBars * 8;         // TMEM base, abort flag
constexpr int kAttnSmemBytes = 1024 + kOffMisc + 64;

enum {
  BAR_K_FULL = 0, BAR_K_EMPTY = 1, BAR_V_FULL = 2, BAR_V_EMPTY = 3,
  BAR_Q_FULL = 4, BAR_QP_EMPTY = 4 + kQRing, BAR_P_FULL = 4 + 2 * kQRing,
  BAR_S_FULL = 4 + 3 * kQRing, BAR_O_FULL = BAR_S_FULL + 2, BAR_O_EMPTY = BAR_S_FULL + 4,
  BAR_D_FULL = BAR_S_FULL + 6, BAR_D_EMPTY = BAR_D_FULL + kDescRing
};

struct AttnArgs {
  const __nv_bfloat16* q;
  int64_t qs_b, qs_t, qs_h;
  const int32_t* blk_offsets;
  const int32_t* entries;
  int64_t n_seg, n_entries, n_items, W;
  int64_t n_q, q_pos0;
  int32_t G, H, nblk;
  float scale;
  float* part_ml;
  float* part_acc;
  int32_t* err;
};

// Largest s in [lo, n_seg) with off[s] <= pos, by a 32-ary search: each round
// the 31 probes of the warp split the range.  Called by a full warp.
__device__ __forceinline__ int64_t warp_find_segment(const int32_t* off, int64_t lo,
                                                     int64_t hi, int64_t pos, int lane) {
  while (hi - lo > 1) {
    const int64_t step = (hi - lo + 31) >> 5;
    const int64_t idx = lo + (int64_t)lane * step;
    const bool le = lane >= 1 && idx < hi && off[idx] <= pos;
    const int k = __popc(__ballot_sync(0xffffffffu, le));
    lo = lo + (int64_t)k * step;
    hi = min64(hi, lo + step);
  }
  return lo;
}

template <int R>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ AttnArgs a) {
  constexpr int CH = 128 / R;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + kOffBar);
  float2* ml_s = reinterpret_cast<float2*>(base + kOffML);
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(base + kOffDesc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar + BAR_K_FULL, 1);
    mbar_init(bar + BAR_K_EMPTY, 1);
    mbar_init(bar + BAR_V_FULL, 1);
    mbar_init(bar + BAR_V_EMPTY, 1);
    for (int i = 0; i < kQRing; ++i) {
      mbar_init(bar + BAR_Q_FULL + i, 128);
      mbar_init(bar + BAR_QP_EMPTY + i, 1);
      mbar_init(bar + BAR_P_FULL + i, 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + BAR_S_FULL + i, 1);
      mbar_init(bar + BAR_O_FULL + i, 1);
      mbar_init(bar + BAR_O_EMPTY + i, 128);
    }
    for (int i = 0; i < kDescRing; ++i) {
      mbar_init(bar + BAR_D_FULL + i, 1);
      mbar_init(bar + BAR_D_EMPTY + i, 128 + 1);   // epilogue threads + TMA producer
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
  int32_t* err = a.err;
  // ring of depth D: the n-th use is ready / the (n-D)-th use has been released
  auto Wuse = [&](int id, int depth, int64_t n) {
    return mbar_wait(bar + id + (int)(n % depth), (uint32_t)((n / depth) & 1), abort_flag, err);
  };
  auto Wfree = [&](int id, int depth, int64_t n) {
    return n < depth || mbar_wait(bar + id + (int)(n % depth),
                                  (uint32_t)(((n / depth) + 1) & 1), abort_flag, err);
  };

  if (warp == 0) {
    // ---------------- scheduler ----------------
    int64_t chunk = 0, piece = 0;
    bool ok = true;
    auto claim = [&](int64_t n) {      // lane 0 waits, the warp follows
      bool r = true;
      if (lane == 0) r = Wfree(BAR_D_EMPTY, kDescRing, n);
      return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
    };
    for (int64_t item = blockIdx.x; ok && item < a.n_items; item += gridDim.x) {
      const int64_t e0 = item * a.W;
      const int64_t e1 = min64(e0 + a.W, a.n_entries);
      int64_t pos = e0;
      int64_t seg = warp_find_segment(a.blk_offsets, 0, a.n_seg, pos, lane);
      while (pos < e1) {
        const int64_t pend = min64(e1, (int64_t)a.blk_offsets[seg + 1]);
        if (pend <= pos) {             // fewer entries listed than the sizes imply
          if (lane == 0) {
            report(err, MSA_DEVERR_BAD_ENTRY);
            *abort_flag = 1;
          }
          ok = false;
          break;
        }
        const int64_t bg = seg / a.nblk;
        const int32_t c = (int32_t)(seg - bg * a.nblk);
        const int32_t b = (int32_t)(bg / a.G), g = (int32_t)(bg - (int64_t)b * a.G);
        for (int64_t cpos = pos; cpos < pend; cpos += CH) {
          if (!claim(chunk)) {
            ok = false;
            break;
          }
          ChunkDesc& d = desc[chunk % kDescRing];
          const int cnt = (int)min64(CH, pend - cpos);
          for (int i = lane; i < CH; i += 32) d.ent[i] = (i < cnt) ? a.entries[cpos + i] : -1;
          if (lane == 0) {
            d.b = b;
            d.g = g;
            d.c = c;
            d.cnt = cnt;
            d.piece = (int32_t)piece;
            d.first = cpos == pos;
            d.last = cpos + CH >= pend;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar + BAR_D_FULL + (int)(chunk % kDescRing));
          ++chunk;
        }
        if (!ok) break;
        ++piece;
        pos = pend;
        if (pos < e1) seg = warp_find_segment(a.blk_offsets, seg + 1, a.n_seg, pos, lane);
      }
    }
    if (ok && claim(chunk)) {          // end marker
      if (lane == 0) {
        desc[chunk % kDescRing].cnt = -1;
        mbar_arrive(bar + BAR_D_FULL + (int)(chunk % kDescRing));
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // S(n) and the pending P V(n-1) are issued in whichever order their
    // inputs become ready (S(n) needs the gathered Q tile, P V(n-1) the
    // softmax of n-1); S(n+1) always waits for P V(n-1), which frees S buffer.
    if (lane == 0) {
      int64_t pn = -1, pp = 0, v_ready = -1, last_s_piece = -1;
      bool plast = false, ok = true;
      auto pv_ready = [&](int64_t n, int64_t p) {
        if (p != v_ready) {
          if (!mbar_try_wait(bar + BAR_V_FULL, (uint32_t)(p & 1))) return false;
          v_ready = p;
        }
        return mbar_try_wait(bar + BAR_P_FULL + (int)(n % kQRing),
                             (uint32_t)((n / kQRing) & 1));
      };
      auto issue_pv = [&](int64_t n, bool last) {
        const int ob = (int)(n & 1);
        tc_fence_after();
        const uint32_t va = smem_u32(base + kOffV);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem + 256 + ob * 128, tmem + ob * 128 + kk * 8,
                       smem_desc_sw128(va + kk * 2048, 16384, 1024), kIdescPV, kk > 0 ? 1u : 0u);
        umma_commit(bar + BAR_O_FULL + ob);
        if (last) umma_commit(bar + BAR_V_EMPTY);
      };
      for (int64_t n = 0;; ++n) {
        if (!Wuse(BAR_D_FULL, kDescRing, n)) { ok = false; break; }
        const ChunkDesc& d = desc[n % kDescRing];
        if (d.cnt < 0) break;
        const int64_t p = d.piece;
        const bool first = d.first != 0, last = d.last != 0;
        const int qb = (int)(n % kQRing), sb = (int)(n & 1);
        bool s_done = false, k_ok = !first, pv_done = pn < 0, o_ok = n < 2;
        const uint64_t t0 = global_timer_ns();
        while (!(s_done && pv_done)) {
          bool progress = false;
          if (!pv_done && pv_ready(pn, pp)) {
            issue_pv(pn, plast);
            pv_done = progress = true;
          }
          if (!s_done) {
            if (!k_ok) k_ok = mbar_try_wait(bar + BAR_K_FULL, (uint32_t)(p & 1));
            // S buffer sb holds P(n-2) until O(n-2) = P(n-2) V is complete
            if (!o_ok) o_ok = mbar_try_wait(bar + BAR_O_FULL + sb, (uint32_t)(((n - 2) >> 1) & 1));
            if (k_ok && o_ok &&
                mbar_try_wait(bar + BAR_Q_FULL + qb, (uint32_t)((n / kQRing) & 1))) {
              tc_fence_after();
              const uint32_t qa = smem_u32(base + kOffQP + qb * 32768);
              const uint32_t ka = smem_u32(base + kOffK);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                umma_bf16(tmem + sb * 128, smem_desc_sw128(qa + off, 16, 1024),
                          smem_desc_sw128(ka + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
              }
              umma_commit(bar + BAR_S_FULL + sb);
              umma_commit(bar + BAR_QP_EMPTY + qb);
              if (last) {
                umma_commit(bar + BAR_K_EMPTY);
                last_s_piece = p;
              }
              s_done = progress = true;
            }
          }
          if (!progress) {
            if (*abort_flag) { ok = false; break; }
            if (global_timer_ns() - t0 > kWaitLimitNs) {
              *abort_flag = 1;
              report(err, MSA_DEVERR_TIMEOUT);
              ok = false;
              break;
            }
            __nanosleep(32);
          }
        }
        if (!ok) break;
        pn = n;
        pp = p;
        plast = last;
      }
      if (ok && pn >= 0) {
        bool ready = false;
        if (pp != v_ready) ready = Wuse(BAR_V_FULL, 1, pp);
        else ready = true;
        if (ready && Wuse(BAR_P_FULL, kQRing, pn)) {
          issue_pv(pn, plast);
          // let the last completions land before the block can exit
          Wuse(BAR_QP_EMPTY, kQRing, pn);
          Wuse(BAR_O_FULL, 2, pn);
          if (plast) Wuse(BAR_V_EMPTY, 1, pp);
          if (last_s_piece >= 0) Wuse(BAR_K_EMPTY, 1, last_s_piece);
        }
      }
    }
  } else if (warp == 2) {
    // ---------------- TMA producer: K/V of every piece ----------------
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      for (int64_t n = 0;; ++n) {
        if (!Wuse(BAR_D_FULL, kDescRing, n)) break;
        const ChunkDesc& d = desc[n % kDescRing];
        if (d.cnt < 0) break;
        if (d.first) {
          const int64_t p = d.piece;
          const int32_t b = d.b, g = d.g, c = d.c;
          if (!Wfree(BAR_K_EMPTY, 1, p)) break;
          mbar_arrive_expect_tx(bar + BAR_K_FULL, 32768);
          tma_load_4d(base + kOffK, &tm_k, bar + BAR_K_FULL, 0, c * kBlock, g, b);
          tma_load_4d(base + kOffK + 16384, &tm_k, bar + BAR_K_FULL, 64, c * kBlock, g, b);
          if (!Wfree(BAR_V_EMPTY, 1, p)) break;
          mbar_arrive_expect_tx(bar + BAR_V_FULL, 32768);
          tma_load_4d(base + kOffV, &tm_v, bar + BAR_V_FULL, 0, c * kBlock, g, b);
          tma_load_4d(base + kOffV + 16384, &tm_v, bar + BAR_V_FULL, 64, c * kBlock, g, b);
        }
        mbar_arrive(bar + BAR_D_EMPTY + (int)(n % kDescRing));
      }
    }
  } else if (warp < 7) {
    // ---------------- gather: Q rows of each chunk ----------------
    const int gt = tid - 96;   // 0..127
    const int ch = gt & 15;
    for (int64_t n = 0;; ++n) {
      if (!Wuse(BAR_D_FULL, kDescRing, n)) break;
      const ChunkDesc& d = desc[n % kDescRing];
      if (d.cnt < 0) break;
      const int qb = (int)(n % kQRing);
      const int32_t b = d.b, g = d.g;
      if (!Wfree(BAR_QP_EMPTY, kQRing, n)) break;
      uint8_t* sq = base + kOffQP + qb * 32768;
      const __nv_bfloat16* qbase =
          a.q + (int64_t)b * a.qs_b + (int64_t)(g * R) * a.qs_h + ch * 8;
#pragma unroll 4
      for (int it = 0; it < 16; ++it) {
        const int row = it * 8 + (gt >> 4);
        const int e = d.ent[row / R];
        const int64_t qi = (int64_t)(e >> 4);
        const bool ok = (e >= 0) && (qi < a.n_q);
        const __nv_bfloat16* src = ok ? qbase + qi * a.qs_t + (int64_t)(row % R) * a.qs_h : a.q;
        uint8_t* dst = sq + (ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        cp_async_16(dst, src, ok ? 16u : 0u);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(bar + BAR_Q_FULL + qb);
    }
  } else if (warp < 11) {
    // ---------------- softmax: S -> P, (m, l) ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float scale_log2 = a.scale * 1.4426950408889634f;
    for (int64_t n = 0;; ++n) {
      if (!Wuse(BAR_D_FULL, kDescRing, n)) break;
      const ChunkDesc& d = desc[n % kDescRing];
      if (d.cnt < 0) break;
      const int qb = (int)(n % kQRing), sb = (int)(n & 1);
      const int e = d.ent[row / R];
      const int32_t c = d.c;
      if (!Wuse(BAR_S_FULL, 2, n)) break;
      tc_fence_after();
      const int64_t qi = (int64_t)(e >> 4);
      bool valid = (e >= 0) && (qi < a.n_q);
      int lim = 127;
      if (valid) {
        const int64_t rel = a.q_pos0 + qi - (int64_t)c * kBlock;
        if (rel < 0) {
          valid = false;
          report(err, MSA_DEVERR_BAD_ENTRY);
        } else if (rel < 127) {
          lim = (int)rel;
        }
      }
      const uint32_t s_addr = tmem + lane_base + sb * 128;
      float mx = -INFINITY;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(s_addr + j * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x)
          if (j * 32 + x <= lim) mx = fmaxf(mx, u2f(r[x]));
      }
      if (!valid) {
        mx = 0.f;
        lim = -1;                             // every weight of the row is zero
      }
      const float mneg = -mx * scale_log2;
      float lsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(s_addr + j * 32, r);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int k0 = j * 32 + 2 * x;
          // branch-free: exponentiate every key, then zero the ones past lim
          float p0 = ex2_approx(fmaf(u2f(r[2 * x]), scale_log2, mneg));
          float p1 = ex2_approx(fmaf(u2f(r[2 * x + 1]), scale_log2, mneg));
          p0 = (k0 <= lim) ? p0 : 0.f;
          p1 = (k0 + 1 <= lim) ? p1 : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          lsum[x & 3] += __low2float(h2) + __high2float(h2);
          w[x] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        // keys 32j..32j+31 -> columns 16j..16j+15 of this S buffer (already read)
        tmem_st_32x32b_x16(s_addr + j * 16, w);
      }
      tmem_st_wait();
      const float l = (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
      // (m, l) slot sb and O buffer sb are free once the epilogue of n-2 is done;
      // P V(n) is issued only after this arrival
      if (!Wfree(BAR_O_EMPTY, 2, n)) break;
      ml_s[sb * 128 + row] = make_float2(mx * a.scale, l);
      tc_fence_before();
      mbar_arrive(bar + BAR_P_FULL + qb);
    }
  } else {
    // ---------------- epilogue: O -> pieces ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    for (int64_t n = 0;; ++n) {
      if (!Wuse(BAR_D_FULL, kDescRing, n)) break;
      const ChunkDesc& d = desc[n % kDescRing];
      if (d.cnt < 0) break;
      const int ob = (int)(n & 1);
      const int e = d.ent[row / R];
      const int32_t b = d.b, g = d.g, c = d.c;
      if (!Wuse(BAR_O_FULL, 2, n)) break;
      if (!Wuse(BAR_P_FULL, kQRing, n)) break;   // acquire the softmax's (m, l)
      tc_fence_after();
      const int hr = row % R;
      const int64_t qi = (int64_t)(e >> 4);
      const bool valid = (e >= 0) && (qi < a.n_q) && (a.q_pos0 + qi >= (int64_t)c * kBlock);
      // piece row of (b, qi, g, slot, hr): the R head rows of one entry are adjacent
      const int64_t pidx =
          valid ? ((((int64_t)b * a.n_q + qi) * a.G + g) * kTopK + (e & 15)) * R + hr : 0;
      if (valid) *reinterpret_cast<float2*>(a.part_ml + pidx * 2) = ml_s[ob * 128 + row];
      uint8_t* srow = base + kOffStage + row * kStageRow;
      uint8_t* swarp = base + kOffStage + (quarter * 32) * kStageRow;
      const uint32_t o_addr = tmem + lane_base + 256 + ob * 128;
      float* acc = a.part_acc + pidx * kHeadDim;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(o_addr + half * 64, r0);
        tmem_ld_32x32b_x32(o_addr + half * 64 + 32, r1);
        tmem_ld_wait();
        if (half == 1) {
          tc_fence_before();
          mbar_arrive(bar + BAR_O_EMPTY + ob);
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          *reinterpret_cast<uint4*>(srow + x * 16) =
              make_uint4(r0[4 * x], r0[4 * x + 1], r0[4 * x + 2], r0[4 * x + 3]);
          *reinterpret_cast<uint4*>(srow + 128 + x * 16) =
              make_uint4(r1[4 * x], r1[4 * x + 1], r1[4 * x + 2], r1[4 * x + 3]);
        }
        __syncwarp();
        // two half rows per instruction: lanes 0-15 row 2i, lanes 16-31 row 2i+1
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int rr = 2 * i + (lane >> 4);
          const float* dst_row = (const float*)__shfl_sync(0xffffffffu, (unsigned long long)acc, rr);
          const bool rv = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
          const uint4 v = *reinterpret_cast<const uint4*>(swarp + rr * kStageRow + (lane & 15) * 16);
          if (rv)
            *reinterpret_cast<uint4*>(const_cast<float*>(dst_row) + half * 64 + (lane & 15) * 4) = v;
        }
        __syncwarp();
      }
      mbar_arrive(bar + BAR_D_EMPTY + (int)(n % kDescRing));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int R>
static cudaError_t launch_attn_r(const CUtensorMap& tm_k, const CUtensorMap& tm_v, AttnArgs a,
                                 cudaStream_t st) {
  constexpr int CH = 128 / R;
  auto k = sparse_attn_fwd_kernel<R>;
  cudaError_t e =
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // items of W consecutive entries: at most 8 tiles each, and enough items
  // (about 8 per SM) to keep every SM busy on small problems
  const int64_t target_items = (int64_t)sms * 8;
  int64_t W = (a.n_entries + target_items - 1) / target_items;
  W = max64(1, min64(W, (int64_t)CH * kAttnMaxChunksPerItem));
  a.W = W;
  a.n_items = (a.n_entries + W - 1) / W;
  if (a.n_items == 0) return cudaSuccess;
  const int64_t grid = min64(a.n_items, sms);
  k<<<(unsigned)grid, kAttnThreads, kAttnSmemBytes, st>>>(tm_k, tm_v, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                               int64_t qs_b, int64_t qs_t, int64_t qs_h,
                               const int32_t* blk_offsets, const int32_t* entries,
                               int64_t n_seg, int64_t n_entries, int64_t n_q, int64_t q_pos0,
                               int32_t G, int32_t H, int32_t nblk, float scale, float* part_ml,
                               float* part_acc, int32_t* err, cudaStream_t st) {
  AttnArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.qs_b = qs_b;
  a.qs_t = qs_t;
  a.qs_h = qs_h;
  a.blk_offsets = blk_offsets;
  a.entries = entries;
  a.n_seg = n_seg;
  a.n_entries = n_entries;
  a.n_items = 0;
  a.W = 1;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.G = G;
  a.H = H;
  a.nblk = nblk;
  a.scale = scale;
  a.part_ml = part_ml;
  a.part_acc = part_acc;
  a.err = err;
  switch (H / G) {
    case 1: return launch_attn_r<1>(tm_k, tm_v, a, st);
    case 2: return launch_attn_r<2>(tm_k, tm_v, a, st);
    case 4: return launch_attn_r<4>(tm_k, tm_v, a, st);
    case 8: return launch_attn_r<8>(tm_k, tm_v, a, st);
    case 16: return launch_attn_r<16>(tm_k, tm_v, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace msa
