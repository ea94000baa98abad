// KV-block-outer sparse attention: for every (batch, group, KV block) segment
// of the block->query lists, the block's K and V tiles are loaded into shared
// memory by TMA once per work item, the query rows that chose the block are
// gathered into 128-row tiles, and S = Q K^T, the softmax piece and O = P V
// run on the tcgen05 tensor cores with fp32 accumulators in TMEM.  Each
// (query, head, slot) gets a piece (m, l, acc) that the merge kernel combines;
// pieces are stored in the order of the lists' entries (the entry at position
// p owns rows p * R .. p * R + R - 1), so a chunk's pieces are adjacent.
// Pieces are fp32 by default; the compact form (an opt-in of the C ABI) keeps
// (m, l) in fp32 and stores acc / l rounded to bf16 (a convex combination of
// V rows, so it cannot overflow), which halves the piece traffic.
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
//   warp 1      MMA issuer:   S(n) = Q K^T, then O(n-1) = P V, in that fixed order
//   warp 2      TMA producer: K and V of each piece; K of the next piece is
//                             loaded as soon as the last S MMA of the current
//                             one is done, V as soon as its last P V is done
//   warp 3      idle (fills the control warpgroup)
//   warps 4-7   gather:       the chunk's Q rows into a 2-deep ring: for R >= 8
//                             warp 4 alone, one 2 KB TMA box per eight heads
//                             of an entry (both 64-column panels; a 5-D view
//                             of q), otherwise 16-byte cp.async by all four
//                             warps
//   warps 8-15  softmax:      two warpgroups, one per half of the keys; each
//                             holds its 64 S values of a row in registers,
//                             the halves exchange row maxima (and whether to
//                             go on) at a named barrier per quarter, and
//                             P = bf16(e^{s-m}) goes back into the first 64
//                             columns of the S buffer in TMEM (the A operand
//                             of O = P V)
//   warps 16-19 epilogue:     O from TMEM half a row at a time, then the
//                             (m, l, acc) pieces to global memory.  R >= 8:
//                             each warp stages its 32 rows in 128B-swizzled
//                             panels and writes them with one TMA tensor
//                             store per half row (fp32) or per chunk
//                             (compact); R < 8: staged rows are read back
//                             transposed so that one store instruction
//                             writes two whole half rows (coalesced)
// The five warpgroups split the register file unevenly (setmaxnreg).
// Shared memory: K 32 KB, V 32 KB, 2 x 32 KB Q tiles (128B-swizzled K-major;
// a Q tile gathered by TMA is laid out [8-row group][panel][8 rows][128 B] so
// that one box brings eight heads of an entry; V is read N-major for P V),
// 64 KB output staging (16 KB per epilogue warp), (m, l) slots and the row
// maxima the two softmax halves exchange.  TMEM: S/P in columns [0,256), O in
// [256,512), two buffers of 128 columns each; a Q tile is released as soon as
// its S MMA is done, S(n+2) waits for O(n) = P(n) V, which reads P(n) from
// the same columns, and P V(n+2) waits until the epilogue has read O(n).
// Every wait is bounded (a time limit, then the block winds down and reports
// MSA_DEVERR_TIMEOUT); whatever path a role leaves by, the loads it issued
// and the MMAs in flight are drained before TMEM is freed and the block exits.
#include <atomic>

#include "common.cuh"

namespace msa {

constexpr int kAttnThreads = 640;
// Registers per thread: 96 at launch (65536 / 640, rounded down to the
// allocation unit); the control and gather warpgroups give registers back,
// the two softmax warpgroups and the epilogue take them, and the five shares
// add up to exactly the launch allocation.  The launcher checks the compiled
// count before the first launch.
constexpr int kAttnRegsAtLaunch = 96;
constexpr int kRegsControl = 88, kRegsGather = 48, kRegsSoftmax = 120, kRegsEpilogue = 104;
static_assert(kRegsControl + kRegsGather + 2 * kRegsSoftmax + kRegsEpilogue ==
                  5 * kAttnRegsAtLaunch,
              "warpgroup register shares must add up to the launch allocation");
static_assert(kAttnThreads * kAttnRegsAtLaunch <= 65536, "register file");
constexpr int kAttnMaxChunksPerItem = 32;
constexpr int kQRing = 2;              // Q tiles in flight
constexpr int kDescRing = 8;           // chunk descriptors in flight

struct alignas(16) ChunkDesc {
  int32_t b, g, c, cnt;                // cnt < 0: no more work
  int32_t piece, first, last, pos0;   // pos0: position of ent[0] in the entries array
  int32_t ent[128];
};

constexpr int kOffK = 0;               // 32768: [K lo | K hi]
constexpr int kOffV = 32768;           // 32768: [V lo | V hi]
constexpr int kOffQP = 65536;          // kQRing x 32768: the gathered Q tiles
constexpr int kStageRow = 272;                           // staged half row (256 B + pad)
constexpr int kOffStage = kOffQP + kQRing * 32768;       // 4 warps x 16 KB of staged rows
constexpr int kStageBytes = 65536;
static_assert(128 * kStageRow <= kStageBytes, "padded rows of the R < 8 epilogue");
constexpr int kOffML = kOffStage + kStageBytes;          // [2 slots][2 halves][128] float2 (m, l)
constexpr int kOffMX = kOffML + 4096;                    // [2][2 halves][128] float row maxima
constexpr int kOffVerdict = kOffMX + 2048;               // [2][2 halves][4 quarters] int
constexpr int kOffDesc = kOffVerdict + 64;               // kDescRing descriptors
constexpr int kOffBar = kOffDesc + kDescRing * (int)sizeof(ChunkDesc);
constexpr int kNumBars = 4 + 3 * kQRing + 6 + 2 * kDescRing + 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;         // TMEM base, abort flag
constexpr int kAttnSmemBytes = 1024 + kOffMisc + 64;

enum {
  BAR_K_FULL = 0, BAR_K_EMPTY = 1, BAR_V_FULL = 2, BAR_V_EMPTY = 3,
  BAR_Q_FULL = 4, BAR_QP_EMPTY = 4 + kQRing, BAR_P_FULL = 4 + 2 * kQRing,
  BAR_S_FULL = 4 + 3 * kQRing, BAR_O_FULL = BAR_S_FULL + 2, BAR_O_EMPTY = BAR_S_FULL + 4,
  BAR_D_FULL = BAR_S_FULL + 6, BAR_D_EMPTY = BAR_D_FULL + kDescRing,
  BAR_ML_EMPTY = BAR_D_EMPTY + kDescRing,
  BAR_DRAIN = BAR_ML_EMPTY + 2      // the MMA issuer's last commit (all its MMAs done)
};

struct AttnArgs {
  const __nv_bfloat16* q;
  int64_t qs_b, qs_t, qs_h;
  const int32_t* blk_offsets;
  const int32_t* entries;
  int64_t n_seg, n_entries, n_items, W;
  int64_t n_q, q_pos0;
  int32_t G, H, nblk, nwin;   // segments are (batch, group, query window, block)
  float scale;
  float* part_ml;
  void* part_acc;             // fp32 rows, or bf16 rows of acc / l (compact pieces)
  int32_t* err;
  uint64_t wait_limit_ns;     // time limit of every barrier wait (drains excepted)
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

template <int R, bool kCompact>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ CUtensorMap tm_o,
                           const __grid_constant__ CUtensorMap tm_o8,
                           const __grid_constant__ AttnArgs a) {
  constexpr int CH = 128 / R;
  // R >= 8: an entry's R head rows (R x 256 contiguous bytes) arrive by TMA
  constexpr bool kTmaGather = R >= 8;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + kOffBar);
  float2* ml_s = reinterpret_cast<float2*>(base + kOffML);
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(base + kOffDesc);
  float* mx_x = reinterpret_cast<float*>(base + kOffMX);
  int* verdict = reinterpret_cast<int*>(base + kOffVerdict);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar + BAR_K_FULL, 1);
    mbar_init(bar + BAR_K_EMPTY, 1);
    mbar_init(bar + BAR_V_FULL, 1);
    mbar_init(bar + BAR_V_EMPTY, 1);
    for (int i = 0; i < kQRing; ++i) {
      mbar_init(bar + BAR_Q_FULL + i, kTmaGather ? 1 : 128);
      mbar_init(bar + BAR_QP_EMPTY + i, 1);
      mbar_init(bar + BAR_P_FULL + i, 256);       // both softmax warpgroups
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + BAR_S_FULL + i, 1);
      mbar_init(bar + BAR_O_FULL + i, 1);
      mbar_init(bar + BAR_O_EMPTY + i, 128);
      mbar_init(bar + BAR_ML_EMPTY + i, 128);
    }
    for (int i = 0; i < kDescRing; ++i) {
      mbar_init(bar + BAR_D_FULL + i, 1);
      mbar_init(bar + BAR_D_EMPTY + i, 128 + 1);   // epilogue threads + TMA producer
    }
    mbar_init(bar + BAR_DRAIN, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // Q tiles start zeroed: rows that no entry fills keep finite old data
  for (int i = tid; i < kQRing * 32768 / 16; i += kAttnThreads)
    reinterpret_cast<uint4*>(base + kOffQP)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
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
  const uint64_t wait_lim = a.wait_limit_ns;
  auto Wuse = [&](int id, int depth, int64_t n) {
    return mbar_wait(bar + id + (int)(n % depth), (uint32_t)((n / depth) & 1), abort_flag, err,
                     wait_lim);
  };
  auto Wfree = [&](int id, int depth, int64_t n) {
    return n < depth || mbar_wait(bar + id + (int)(n % depth),
                                  (uint32_t)(((n / depth) + 1) & 1), abort_flag, err, wait_lim);
  };
  // The same for roles whose whole warp goes on to warp-collective instructions
  // (tcgen05.ld/st .sync.aligned, votes, shuffles): every lane waits, then the
  // warp votes, so that after a timeout no lane carries on while another has
  // left (a lane still waiting returns once the abort flag is set).
  auto WuseW = [&](int id, int depth, int64_t n) {
    return __all_sync(0xffffffffu, Wuse(id, depth, n) ? 1 : 0) != 0;
  };
  auto WfreeW = [&](int id, int depth, int64_t n) {
    return __all_sync(0xffffffffu, Wfree(id, depth, n) ? 1 : 0) != 0;
  };

  // Roles by warpgroup; each warpgroup first resizes its registers (all four
  // of its warps execute the same setmaxnreg).
  if (warp < 4) {
    setmaxnreg_dec<kRegsControl>();
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
          const int64_t bgw = seg / a.nblk;
          const int32_t c = (int32_t)(seg - bgw * a.nblk);
          const int64_t bg = bgw / a.nwin;
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
              d.pos0 = (int32_t)cpos;
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
      // Fixed order S(0), S(1), P V(0), S(2), P V(1), ...: S(n) needs the
      // gathered Q tile, the piece's K and its S buffer back from P V(n-2);
      // P V(n-1) needs the softmax of n-1 and the piece's V.  Every wait
      // suspends in hardware (no polling).
      if (lane == 0) {
        int64_t pn = -1, pp = -1, v_ready = -1, last_s_piece = -1;
        bool plast = false, ok = true;
        // shared-memory descriptors of the operands' first slices
        const uint64_t kdesc0 = smem_desc_sw128(smem_u32(base + kOffK), 16, 1024);
        const uint64_t vdesc0 = smem_desc_sw128(smem_u32(base + kOffV), 16384, 1024);
        const uint64_t qdesc_ring0 =
            smem_desc_sw128(smem_u32(base + kOffQP), 16, kTmaGather ? 2048 : 1024);
        auto issue_pv = [&](int64_t n, int64_t p, bool last) {
          if (p != v_ready) {
            if (!Wuse(BAR_V_FULL, 1, p)) return false;
            v_ready = p;
          }
          if (!Wuse(BAR_P_FULL, kQRing, n)) return false;
          // O buffer n & 1 is free once the epilogue of n-2 has read it
          if (!Wfree(BAR_O_EMPTY, 2, n)) return false;
          const int ob = (int)(n & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ts(tmem + 256 + ob * 128, tmem + ob * 128 + kk * 8,
                         vdesc0 + (uint64_t)((kk * 2048) >> 4), kIdescPV, kk > 0 ? 1u : 0u);
          umma_commit(bar + BAR_O_FULL + ob);
          if (last) umma_commit(bar + BAR_V_EMPTY);
          return true;
        };
        int64_t k_ready = -1;
        for (int64_t n = 0;; ++n) {
          if (!Wuse(BAR_D_FULL, kDescRing, n)) { ok = false; break; }
          const ChunkDesc& d = desc[n % kDescRing];
          if (d.cnt < 0) break;
          const int64_t p = d.piece;
          const bool last = d.last != 0;
          const int qb = (int)(n % kQRing), sb = (int)(n & 1);
          if (p != k_ready) {
            if (!Wuse(BAR_K_FULL, 1, p)) { ok = false; break; }
            k_ready = p;
          }
          // S buffer sb holds P(n-2) until O(n-2) = P(n-2) V is complete
          if (n >= 2 && !Wuse(BAR_O_FULL, 2, n - 2)) { ok = false; break; }
          if (!Wuse(BAR_Q_FULL, kQRing, n)) { ok = false; break; }
          tc_fence_after();
          const uint64_t qdesc0 = qdesc_ring0 + (uint64_t)((qb * 32768) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K: [panel][128 rows][128 B] (8-row groups 1024 B apart); Q for R >= 8:
            // [8-row group][panel][8 rows][128 B] (groups 2048 B apart), else as K.
            // A descriptor's low 14 bits hold the address / 16, so the step to
            // the kk-th 16-column slice is a plain add.
            const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t qoff = kTmaGather ? (kk >> 2) * 1024 + (kk & 3) * 32 : koff;
            umma_bf16(tmem + sb * 128, qdesc0 + (uint64_t)(qoff >> 4),
                      kdesc0 + (uint64_t)(koff >> 4), kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar + BAR_S_FULL + sb);
          umma_commit(bar + BAR_QP_EMPTY + qb);
          if (last) {
            umma_commit(bar + BAR_K_EMPTY);
            last_s_piece = p;
          }
          if (pn >= 0 && !issue_pv(pn, pp, plast)) { ok = false; break; }
          pn = n;
          pp = p;
          plast = last;
        }
        if (ok && pn >= 0 && issue_pv(pn, pp, plast)) {
          // let the last completions land before the block can exit
          Wuse(BAR_QP_EMPTY, kQRing, pn);
          Wuse(BAR_O_FULL, 2, pn);
          if (plast) Wuse(BAR_V_EMPTY, 1, pp);
          if (last_s_piece >= 0) Wuse(BAR_K_EMPTY, 1, last_s_piece);
        }
        // On every exit path, also after an abort: one more commit arrives once
        // every MMA this thread issued has completed (commits complete in issue
        // order), so no MMA still reads shared memory or writes TMEM when the
        // block deallocates TMEM and exits.
        umma_commit(bar + BAR_DRAIN);
        mbar_drain(bar + BAR_DRAIN, 0, err);
      }
    } else if (warp == 2) {
      // ---------------- TMA producer: K/V of every piece ----------------
      if (lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        int64_t k_issued = -1, v_issued = -1;    // last piece whose K / V load was issued
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
            k_issued = p;
            if (!Wfree(BAR_V_EMPTY, 1, p)) break;
            mbar_arrive_expect_tx(bar + BAR_V_FULL, 32768);
            tma_load_4d(base + kOffV, &tm_v, bar + BAR_V_FULL, 0, c * kBlock, g, b);
            tma_load_4d(base + kOffV + 16384, &tm_v, bar + BAR_V_FULL, 64, c * kBlock, g, b);
            v_issued = p;
          }
          mbar_arrive(bar + BAR_D_EMPTY + (int)(n % kDescRing));
        }
        // the loads in flight land before the block exits (piece p is the p-th
        // phase of each full barrier)
        if (k_issued >= 0) mbar_drain(bar + BAR_K_FULL, (uint32_t)(k_issued & 1), err);
        if (v_issued >= 0) mbar_drain(bar + BAR_V_FULL, (uint32_t)(v_issued & 1), err);
      }
    }
    // warp 3: idle
  } else if (warp < 8) {
    // ---------------- gather: Q rows of each chunk ----------------
    setmaxnreg_dec<kRegsGather>();
    if constexpr (kTmaGather) {
      // warp 4 alone: lane 0 arms Q_FULL with the chunk's bytes, then lane l
      // issues the box of 8-row group l: eight heads of one entry, both
      // 64-column panels (2 KB), into [group][panel][8 rows][128 B] of the Q
      // tile.  One thread arms each phase, so on an abort it knows which loads
      // are in flight and drains exactly those.
      if (warp == 4) {
        constexpr int kGroups = R / 8;           // 8-row groups per entry
        int64_t armed = -1;                      // last chunk whose loads were issued
        for (int64_t n = 0;; ++n) {
          if (!WuseW(BAR_D_FULL, kDescRing, n)) break;
          const ChunkDesc& d = desc[n % kDescRing];
          if (d.cnt < 0) break;
          const int qb = (int)(n % kQRing);
          int ok = 1;
          if (lane == 0) {
            if (!Wfree(BAR_QP_EMPTY, kQRing, n)) {
              ok = 0;
            } else {
              uint32_t bytes = 0;
              for (int k = 0; k < CH; ++k) {
                const int e = d.ent[k];
                if (e >= 0 && (int64_t)(e >> 4) < a.n_q) bytes += R * 256;
              }
              mbar_arrive_expect_tx(bar + BAR_Q_FULL + qb, bytes);
            }
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
          armed = n;
          uint8_t* sq = base + kOffQP + qb * 32768;
          if (lane < 16) {                       // 16 groups of 8 rows per tile
            const int k = lane / kGroups, j = lane % kGroups;
            const int e = d.ent[k];
            if (e >= 0 && (int64_t)(e >> 4) < a.n_q)
              tma_load_5d(sq + lane * 2048, &tm_q, bar + BAR_Q_FULL + qb, 0, d.g * R + 8 * j, 0,
                          e >> 4, d.b);
          }
        }
        if (lane == 0 && armed >= 0)
          mbar_drain(bar + BAR_Q_FULL + (int)(armed % kQRing),
                     (uint32_t)((armed / kQRing) & 1), err);
      }
    } else {
      // thread = (row within an 8-row group, 16-byte column chunk); a warp
      // instruction copies two whole 256-byte rows
      const int gt = tid - 128;   // 0..127
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
          const __nv_bfloat16* src =
              ok ? qbase + qi * a.qs_t + (int64_t)(row % R) * a.qs_h : a.q;
          uint8_t* dst = sq + (ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
          cp_async_16(dst, src, ok ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(bar + BAR_Q_FULL + qb);
      }
    }
  } else if (warp < 16) {
    // ---------------- softmax: S -> P, (m, l) ----------------
    // Warpgroup h (0, 1) takes keys 64h .. 64h+63 of every row of every chunk
    // (thread = row = TMEM lane), so a chunk's softmax takes half the time of
    // a whole row's.  Per chunk every wait comes first; then the two warps of
    // a quarter (one per half) meet once at a named barrier, exchanging their
    // row maxima and their verdict (all waits done / end of work), and both
    // go on or both leave on the exchanged verdicts: after a timeout neither
    // half can be left waiting at the barrier for the other.
    setmaxnreg_inc<kRegsSoftmax>();
    const int h = (warp >> 2) - 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float scale_log2 = a.scale * 1.4426950408889634f;
    const uint64_t scale2 = pack_f32x2(__float_as_uint(scale_log2), __float_as_uint(scale_log2));
    for (int64_t n = 0;; ++n) {
      const int qb = (int)(n % kQRing), sb = (int)(n & 1);
      bool ok = WuseW(BAR_D_FULL, kDescRing, n);
      const ChunkDesc& d = desc[n % kDescRing];
      const bool end = ok && d.cnt < 0;
      if (ok && !end) ok = WuseW(BAR_S_FULL, 2, n);
      // the (m, l) slot sb is free once the epilogue of n-2 has read it
      if (ok && !end) ok = WfreeW(BAR_ML_EMPTY, 2, n);
      const bool work = ok && !end;
      const uint32_t s_addr = tmem + lane_base + sb * 128;
      bool valid = false;
      int lim = -1;
      uint32_t r0[32], r1[32];
      float mloc = -INFINITY;
      bool masked = false;
      if (work) {
        tc_fence_after();
        tmem_ld_32x32b_x32(s_addr + 64 * h, r0);
        tmem_ld_32x32b_x32(s_addr + 64 * h + 32, r1);
        const int e = d.ent[row / R];
        const int64_t qi = (int64_t)(e >> 4);
        valid = (e >= 0) && (qi < a.n_q);
        lim = 127;
        if (valid) {
          const int64_t rel = a.q_pos0 + qi - (int64_t)d.c * kBlock;
          if (rel < 0) {
            valid = false;
            if (h == 0) report(err, MSA_DEVERR_BAD_ENTRY);
          } else if (rel < 127) {
            lim = (int)rel;
          }
        }
        if (!valid) lim = -1;                 // every weight of the row is zero
        // only rows of the query's own block mask keys (past the query); a warp
        // with no such row skips every per-key compare
        masked = __any_sync(0xffffffffu, lim >= 0 && lim < 127);
        tmem_ld_wait();
        const int k0 = 64 * h;
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (!masked) {
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            m4[0] = fmax3f(m4[0], u2f(r0[x]), u2f(r0[x + 1]));
            m4[1] = fmax3f(m4[1], u2f(r0[x + 2]), u2f(r0[x + 3]));
            m4[2] = fmax3f(m4[2], u2f(r1[x]), u2f(r1[x + 1]));
            m4[3] = fmax3f(m4[3], u2f(r1[x + 2]), u2f(r1[x + 3]));
          }
        } else {
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            m4[0] = fmaxf(m4[0], k0 + x <= lim ? u2f(r0[x]) : -INFINITY);
            m4[1] = fmaxf(m4[1], k0 + x + 1 <= lim ? u2f(r0[x + 1]) : -INFINITY);
            m4[2] = fmaxf(m4[2], k0 + 32 + x <= lim ? u2f(r1[x]) : -INFINITY);
            m4[3] = fmaxf(m4[3], k0 + 33 + x <= lim ? u2f(r1[x + 1]) : -INFINITY);
          }
        }
        mloc = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      // exchange with the other half's warp of this quarter (by parity: the
      // partner reads a slot before it is written again two chunks later)
      float* mxn = mx_x + (int)(n & 1) * 256;
      mxn[h * 128 + row] = mloc;
      if (lane == 0) verdict[((int)(n & 1) * 2 + h) * 4 + quarter] = (ok ? 1 : 0) | (end ? 2 : 0);
      tc_fence_before();                       // this half's S reads precede the other's P writes
      named_bar_sync(1 + quarter, 64);
      tc_fence_after();
      const int pv = verdict[((int)(n & 1) * 2 + (1 - h)) * 4 + quarter];
      if (!work || !(pv & 1) || (pv & 2)) break;
      float mx = fmaxf(mloc, mxn[(1 - h) * 128 + row]);
      if (!valid) mx = 0.f;
      // e^{s-m} = 2^{s log2(e) scale - m log2(e) scale}; a row with no valid
      // key gets weight 2^-inf = 0 everywhere
      const float mneg = valid ? -mx * scale_log2 : -INFINITY;
      const uint64_t mneg2 = pack_f32x2(__float_as_uint(mneg), __float_as_uint(mneg));
      // two packed (f32x2) partial sums of the weights
      uint64_t lsum2[2] = {0ull, 0ull};
      // keys 32j..32j+31 -> columns 16j..16j+15 of this S buffer (already
      // read).  P is rounded to bf16 for the P V product; l sums the fp32
      // weights.  The exponents of a pair of keys are one packed FMA, their
      // weights one packed add into the row sum.
      auto exp_pack_store = [&](const uint32_t (&r)[32], int j, bool mask) {
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float x0, x1;
          unpack_f32x2(fma_f32x2(pack_f32x2(r[2 * x], r[2 * x + 1]), scale2, mneg2), x0, x1);
          float p0 = ex2_approx(x0);
          float p1 = ex2_approx(x1);
          if (mask) {
            const int kk = j * 32 + 2 * x;
            p0 = (kk <= lim) ? p0 : 0.f;
            p1 = (kk + 1 <= lim) ? p1 : 0.f;
          }
          lsum2[x & 1] =
              add_f32x2(lsum2[x & 1], pack_f32x2(__float_as_uint(p0), __float_as_uint(p1)));
          w[x] = pack_bf16x2(p0, p1);
        }
        tmem_st_32x32b_x16(s_addr + j * 16, w);
      };
      if (!masked) {
        exp_pack_store(r0, 2 * h, false);
        exp_pack_store(r1, 2 * h + 1, false);
      } else {
        exp_pack_store(r0, 2 * h, true);
        exp_pack_store(r1, 2 * h + 1, true);
      }
      tmem_st_wait();
      float la, lb, lc, ld;
      unpack_f32x2(lsum2[0], la, lb);
      unpack_f32x2(lsum2[1], lc, ld);
      ml_s[(sb * 2 + h) * 128 + row] = make_float2(mx * a.scale, (la + lb) + (lc + ld));
      tc_fence_before();
      mbar_arrive(bar + BAR_P_FULL + qb);      // P V(n) is issued once both halves arrive
    }
  } else {
    // ---------------- epilogue: O -> pieces ----------------
    setmaxnreg_inc<kRegsEpilogue>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // Pieces follow the lists' order: row r of a chunk is piece row
    // pos0 * R + r, so a warp's 32 rows are adjacent in memory.  R >= 8: each
    // warp stages [2 panels][32 rows][128 B] at a time (128-byte swizzle;
    // fp32: a half row's two 32-column panels, one buffer per half; compact:
    // the row's two 64-column halves in bf16, one buffer per chunk parity)
    // and one TMA store writes them (a 3-D view of the pieces: 128-byte
    // panels x rows x panels); a warp only partly covered by the chunk's
    // entries (the end of a block's list) stores its rows in 8-row groups,
    // one panel at a time.
    // R < 8: rows padded to 272 B, read back transposed, two half rows (fp32)
    // or four (compact) per store instruction.
    constexpr bool kTmaStore = R >= 8;
    // pieces are read back only by the merge kernel: keep them from displacing Q rows in L2
    const uint64_t pol_st = l2_policy_evict_first();
    uint8_t* stage = base + kOffStage + quarter * 16384;
    uint8_t* srow = base + kOffStage + row * kStageRow;
    uint8_t* swarp = base + kOffStage + (quarter * 32) * kStageRow;
    for (int64_t n = 0;; ++n) {
      if (!WuseW(BAR_D_FULL, kDescRing, n)) break;
      const ChunkDesc& d = desc[n % kDescRing];
      if (d.cnt < 0) break;
      const int ob = (int)(n & 1);
      const int e = d.ent[row / R];
      const int32_t c = d.c;
      if (!WuseW(BAR_O_FULL, 2, n)) break;
      if (!WuseW(BAR_P_FULL, kQRing, n)) break;  // acquire the softmax's (m, l)
      tc_fence_after();
      const float2 ml0 = ml_s[(ob * 2) * 128 + row];
      const float2 ml1 = ml_s[(ob * 2 + 1) * 128 + row];
      mbar_arrive(bar + BAR_ML_EMPTY + ob);      // (m, l) slot ob is free
      const int64_t qi = (int64_t)(e >> 4);
      const bool valid = (e >= 0) && (qi < a.n_q) && (a.q_pos0 + qi >= (int64_t)c * kBlock);
      // first piece row of this warp (piece rows < 2^31, checked by the
      // launcher), and how many of its 32 rows hold entries
      const int32_t wrow0 = d.pos0 * R + quarter * 32;
      const int wrows = max(0, min(32, d.cnt * R - quarter * 32));
      const int64_t pidx = (int64_t)wrow0 + lane;
      const float l_sum = ml0.y + ml1.y;
      if (valid) *reinterpret_cast<float2*>(a.part_ml + pidx * 2) = make_float2(ml0.x, l_sum);
      // compact pieces: acc / l (l >= 1 on a valid row: the row maximum's weight is 1)
      const float inv_l = (kCompact && valid && l_sum > 0.f) ? 1.0f / l_sum : 0.f;
      const uint32_t o_addr = tmem + lane_base + 256 + ob * 128;
      // two staged panels [2][32 rows][128 B] at src -> panels z0, z0 + 1 of
      // rows wrow0 .. wrow0 + wrows - 1: one store for a whole warp, else one
      // per 8-row group and panel (wrows is a multiple of R >= 8)
      uint8_t* sbuf = kCompact ? stage + (int)(n & 1) * 8192 : stage;
      auto store_rows = [&](uint8_t* src, int z0) {
        if (wrows == 32) {
          if (lane == 0) tma_store_3d_hint(&tm_o, src, 0, wrow0, z0, pol_st);
        } else if (lane < (wrows >> 3) * 2) {
          const int grp = lane >> 1, pan = lane & 1;
          tma_store_3d_hint(&tm_o8, src + pan * 4096 + grp * 1024, 0, wrow0 + grp * 8, z0 + pan,
                            pol_st);
        }
      };
      float* acc = reinterpret_cast<float*>(a.part_acc) + pidx * kHeadDim;
      __nv_bfloat16* acc16 = reinterpret_cast<__nv_bfloat16*>(a.part_acc) + pidx * kHeadDim;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(o_addr + half * 64, r0);
        tmem_ld_32x32b_x32(o_addr + half * 64 + 32, r1);
        tmem_ld_wait();
        if (half == 1) {
          tc_fence_before();
          mbar_arrive(bar + BAR_O_EMPTY + ob);   // O buffer ob is free
        }
        if constexpr (kCompact) {
          // the half row as 64 bf16 values = 128 bytes = 8 chunks of 16 bytes
          uint32_t w[32];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            w[x] = pack_bf16x2(u2f(r0[2 * x]) * inv_l, u2f(r0[2 * x + 1]) * inv_l);
            w[16 + x] = pack_bf16x2(u2f(r1[2 * x]) * inv_l, u2f(r1[2 * x + 1]) * inv_l);
          }
          if constexpr (kTmaStore) {
            // half `half` of the row is panel `half` of this chunk's staging
            // buffer [2 panels][32 rows][128 B] (two buffers, by chunk parity);
            // the buffer leaves by one store
            if (half == 0) {
              bulk_wait_read_1();                // the store of two chunks ago has read sbuf
              __syncwarp();
            }
            const int sw = lane & 7;
            uint8_t* mine = sbuf + lane * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(mine + half * 4096 + ((j ^ sw) << 4)) =
                  make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            if (half == 1) {
              fence_proxy_async_smem();
              __syncwarp();
              store_rows(sbuf, 0);
              bulk_commit();
            }
          } else {
#pragma unroll
            for (int x = 0; x < 8; ++x)
              *reinterpret_cast<uint4*>(srow + x * 16) =
                  make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
            __syncwarp();
            // four half rows (128 bytes each) per instruction: lane -> (row 4i + lane / 8,
            // 16-byte chunk lane % 8)
#pragma unroll 4
            for (int i = 0; i < 8; ++i) {
              const int rr = 4 * i + (lane >> 3);
              const __nv_bfloat16* dst_row = (const __nv_bfloat16*)__shfl_sync(
                  0xffffffffu, (unsigned long long)acc16, rr);
              const bool rv = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
              const uint4 v =
                  *reinterpret_cast<const uint4*>(swarp + rr * kStageRow + (lane & 7) * 16);
              if (rv)
                *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(dst_row) + half * 64 +
                                          (lane & 7) * 8) = v;
            }
            __syncwarp();
          }
        } else if constexpr (kTmaStore) {
          // the half row's two 32-column panels into its own staging buffer
          // [2 panels][32 rows][128 B] (one per half), written by one store
          // as soon as it is staged; a buffer is refilled once the store from
          // the same half of the previous chunk has read it
          bulk_wait_read_1();
          __syncwarp();
          const int sw = lane & 7;
          uint8_t* hbuf = sbuf + half * 8192;
          uint8_t* mine = hbuf + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            *reinterpret_cast<uint4*>(mine + ((j ^ sw) << 4)) =
                make_uint4(r0[4 * j], r0[4 * j + 1], r0[4 * j + 2], r0[4 * j + 3]);
            *reinterpret_cast<uint4*>(mine + 4096 + ((j ^ sw) << 4)) =
                make_uint4(r1[4 * j], r1[4 * j + 1], r1[4 * j + 2], r1[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          store_rows(hbuf, half * 2);
          bulk_commit();
        } else {
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
            const float* dst_row =
                (const float*)__shfl_sync(0xffffffffu, (unsigned long long)acc, rr);
            const bool rv = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
            const uint4 v =
                *reinterpret_cast<const uint4*>(swarp + rr * kStageRow + (lane & 15) * 16);
            if (rv)
              *reinterpret_cast<uint4*>(const_cast<float*>(dst_row) + half * 64 +
                                        (lane & 15) * 4) = v;
          }
          __syncwarp();
        }
      }
      mbar_arrive(bar + BAR_D_EMPTY + (int)(n % kDescRing));
    }
    if constexpr (kTmaStore) bulk_wait_all();    // every store has landed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Time limit of the attention kernel's barrier waits (a debug setting of the C
// ABI; 2 s by default).
static std::atomic<uint64_t> g_attn_wait_limit_ns{kWaitLimitNs};

uint64_t set_attn_wait_limit(uint64_t ns) { return g_attn_wait_limit_ns.exchange(ns); }

template <int R, bool kCompact>
static cudaError_t launch_attn_r(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                 const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                                 const CUtensorMap& tm_o8, AttnArgs a, cudaStream_t st) {
  constexpr int CH = 128 / R;
  auto k = sparse_attn_fwd_kernel<R, kCompact>;
  // the register split above is only safe with exactly this many registers
  // per thread at launch
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kAttnRegsAtLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttnSmemBytes);
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
  k<<<(unsigned)grid, kAttnThreads, kAttnSmemBytes, st>>>(tm_q, tm_k, tm_v, tm_o, tm_o8, a);
  return cudaGetLastError();
}

template <bool kCompact>
static cudaError_t launch_attn_c(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                 const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                                 const CUtensorMap& tm_o8, const AttnArgs& a, cudaStream_t st) {
  switch (a.H / a.G) {
    case 1: return launch_attn_r<1, kCompact>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
    case 2: return launch_attn_r<2, kCompact>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
    case 4: return launch_attn_r<4, kCompact>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
    case 8: return launch_attn_r<8, kCompact>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
    case 16: return launch_attn_r<16, kCompact>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sparse_attn(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                               const CUtensorMap& tm_v, const CUtensorMap& tm_o,
                               const CUtensorMap& tm_o8, const void* q,
                               int64_t qs_b, int64_t qs_t, int64_t qs_h,
                               const int32_t* blk_offsets, const int32_t* entries,
                               int64_t n_seg, int64_t n_entries, int64_t n_q, int64_t q_pos0,
                               int32_t G, int32_t H, int32_t nblk, int32_t nwin, float scale,
                               float* part_ml, void* part_acc, bool compact, int32_t* err,
                               cudaStream_t st) {
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
  a.nwin = nwin;
  a.scale = scale;
  a.part_ml = part_ml;
  a.part_acc = part_acc;
  a.err = err;
  a.wait_limit_ns = g_attn_wait_limit_ns.load();
  return compact ? launch_attn_c<true>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st)
                 : launch_attn_c<false>(tm_q, tm_k, tm_v, tm_o, tm_o8, a, st);
}

}  // namespace msa
