// Backward of the main branch's sparse attention, for training through MSA
// (page "MSA 稀疏注意力三国杀", section "MSA 能力不掉：3T token 对照实验": a
// model trained sparse from the start, MSA-PT, and a dense one converted by
// continued training, MSA-CPT; section "索引分支训练：KL 对齐": the index branch
// learns only through its KL term, so the selection is a fixed input here).
// For every (query t, head h) and its selected causal tokens J(t, g):
//   p_j = exp(scale q.k_j - lse),  dP_j = dO.v_j,  D = dO.o,
//   dS_j = p_j (dP_j - D),  dQ = scale sum_j dS_j k_j,
//   dK_j += scale dS_j q,  dV_j += p_j dO.
//
// Same KV-block-outer order as the forward ("Kernel 创新：Outer Gather Q"): a
// KV block's K and V are loaded once per piece and every query row that chose
// the block is gathered against it, so dK and dV of the block accumulate in
// TMEM; dQ leaves as one fp32 piece per (query, head, slot), summed in slot
// order by a second kernel (deterministic), exactly like the forward's
// (m, l, acc) pieces and merge.
//
// Three kernels:
//  * bwd_delta_kernel      -- D = dO.o per (query, head), one warp each;
//  * sparse_attn_bwd_tc_kernel<R> -- every (batch, group, KV block) is one
//    work item, owned by one CTA (items dealt to a grid of at most one CTA
//    per SM in snake order: round j gives CTA k item j * grid + k for even
//    j, j * grid + grid - 1 - k for odd j, which evens out the sizes, large
//    for early blocks).  A piece is an item with entries: its query-window
//    segments in window order, each cut into 128-row tiles (128 / R
//    entries x R heads).  Warp roles
//    (512 threads): a TMA warp loads each piece's K and V; four gather warps
//    bring each tile's Q and dO rows by cp.async into two buffers; an MMA
//    warp issues, per tile, S^T = K Q^T and dP^T = V dO^T (tcgen05, M = 128
//    keys, N = 128 rows), then -- once four softmax warps (thread = key) have
//    turned them into P^T and dS^T (bf16, back into TMEM, and dS^T also into
//    shared memory) -- dV += P^T dO and dK += dS^T Q with A read from TMEM,
//    and dQ = dS K with A read from shared memory; four epilogue warps store
//    the dQ pieces and, at the end of a piece, store the block's dK and dV
//    (one CTA owns a block: no atomics, bit-identical from run to run);
//  * bwd_dq_reduce_kernel  -- dQ = sum over the slots of the pieces, one warp
//    per (query, head).
#include "common.cuh"

namespace msa {

namespace {

struct BwdArgs {
  const __nv_bfloat16* q;     // [B, n_q, H, 128] (strided)
  int64_t qs_b, qs_t, qs_h;
  const __nv_bfloat16* dout;  // same layout as q
  int64_t ds_b, ds_t, ds_h;
  const float* lse;           // [B, n_q, H] (forward)
  const float* delta;         // [B, n_q, H] (bwd_delta_kernel)
  const int32_t* offsets;     // [nseg + 1]
  const int32_t* entries;     // (i << 4) | slot
  float* part_dq;             // [B, n_q, G, 16, R, 128]
  float* dk;                  // [B, G, n_kv, 128]
  float* dv;
  int64_t n_q, n_kv, q_pos0, nseg, total, nitems;   // items: (batch, group, block)
  const int32_t* perm;        // items largest first (null: in index order)
  int32_t G, H, nblk, nwin;   // segments are (batch, group, query window, block)
  float scale;
  int32_t* err;
};

// last segment s with offsets[s] <= e (non-empty, since offsets[s + 1] > e)
__device__ __forceinline__ int64_t segment_of(const int32_t* __restrict__ off, int64_t nseg,
                                              int64_t e) {
  int64_t lo = 0, hi = nseg;                     // answer in [lo, hi)
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (off[mid] <= e) lo = mid; else hi = mid;
  }
  return lo;
}

}  // namespace

__global__ void __launch_bounds__(256)
    bwd_delta_kernel(const __nv_bfloat16* __restrict__ o, int64_t os_b, int64_t os_t,
                     int64_t os_h, const __nv_bfloat16* __restrict__ dout, int64_t ds_b,
                     int64_t ds_t, int64_t ds_h, int64_t rows, int64_t n_q, int32_t H,
                     float* __restrict__ delta) {
  const int lane = threadIdx.x & 31;
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (r >= rows) return;
  const int64_t h = r % H, bt = r / H, b = bt / n_q, t = bt - b * n_q;
  const uint2 ov = *reinterpret_cast<const uint2*>(o + b * os_b + t * os_t + h * os_h + 4 * lane);
  const uint2 dv = *reinterpret_cast<const uint2*>(dout + b * ds_b + t * ds_t + h * ds_h + 4 * lane);
  const float2 o0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.x));
  const float2 o1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.y));
  const float2 d0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.x));
  const float2 d1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.y));
  float s = o0.x * d0.x + o0.y * d0.y + o1.x * d1.x + o1.y * d1.y;
#pragma unroll
  for (int x = 16; x > 0; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
  if (lane == 0) delta[r] = s;
}

// ---------------------------------------------------------------------------
// main kernel: 128-row tiles on tcgen05, accumulators in TMEM
// ---------------------------------------------------------------------------
// TMEM columns (lanes = keys unless noted): [0,128) S^T, then P^T as bf16 in
// [0,64); [128,256) dP^T, then dS^T as bf16 in [128,192), then dQ (lanes =
// rows); [256,384) dV; [384,512) dK.  S^T of the next tile of a piece goes in
// as soon as dV and dK have read P^T, while the epilogue still reads dQ.  Shared memory: K, V (32 KB each,
// TMA, 128B swizzle, two 64-column panels), two Q and two dO tiles (128
// gathered rows each, same layout, cp.async), dS^T [128 keys][128 rows] (the
// A operand of dQ = dS K, stored rows-contiguous: an MN-major operand), the
// tile's row data (t, lse, D), barriers.
namespace {
constexpr int kTcThreads = 512;
constexpr int kTcOffK = 0, kTcOffV = 32768;
constexpr int kTcOffQ = 65536;                   // 2 x 32 KB
constexpr int kTcOffDO = kTcOffQ + 2 * 32768;    // 2 x 32 KB
constexpr int kTcOffDS = kTcOffDO + 2 * 32768;   // 32 KB
constexpr int kTcOffMeta = kTcOffDS + 32768;     // t[128] (int32), lse[128], D[128]
constexpr int kTcOffBar = kTcOffMeta + 3 * 128 * 4;
enum {
  TB_KV_FULL = 0, TB_KV_EMPTY, TB_QDO_FULL0, TB_QDO_FULL1, TB_QDO_EMPTY0, TB_QDO_EMPTY1,
  TB_S_FULL, TB_P_FULL, TB_DVK_DONE, TB_DQ_FULL, TB_DQ_EMPTY, TB_DKV_FULL, TB_DKV_EMPTY,
  TB_COUNT
};
constexpr int kTcOffMisc = kTcOffBar + TB_COUNT * 8;
constexpr int kTcSmemBytes = 1024 + kTcOffMisc + 16;
static_assert(kTcSmemBytes <= 232448, "shared memory per block");
// kind::f16, bf16 A and B, fp32 D, M = N = 128; a_mn / b_mn: operand stored
// M- / N-contiguous
constexpr uint32_t idesc_tc(int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// The CTA's sequence of pieces: its items in snake order, skipping blocks no
// query selected.  Every role walks the same sequence.  With a.perm the items
// are dealt largest first (longest-processing-time order), which evens out
// the CTAs' loads; results do not depend on which CTA takes an item.
struct PieceWalk {
  int64_t round;
};
struct Piece {
  int64_t b, seg0, nt;   // seg0: the segment of window 0 (window w: seg0 + w * nblk)
  int32_t g, c;          // nt: 128-row tiles of the piece
};
// the tiles of one piece: window by window, kEnt entries each
struct TileWalk {
  int64_t e, e_end;
  int32_t w;
};
__device__ __forceinline__ void walk_start(PieceWalk& w) { w.round = 0; }
__device__ __forceinline__ bool walk_next(PieceWalk& w, const BwdArgs& a, Piece& pc, int kEnt) {
  for (;;) {
    const int64_t j = w.round++;
    const int64_t k = (j & 1) ? (int64_t)(gridDim.x - 1 - blockIdx.x) : (int64_t)blockIdx.x;
    const int64_t i0 = j * gridDim.x + k;                // grows with j: the last item ends it
    if (i0 >= a.nitems) return false;
    const int64_t i = a.perm != nullptr ? (int64_t)__ldg(a.perm + i0) : i0;
    const int64_t bg = i / a.nblk;
    const int32_t c = (int32_t)(i - bg * a.nblk);
    const int64_t seg0 = bg * a.nwin * a.nblk + c;
    int64_t nt = 0;
    for (int32_t win = 0; win < a.nwin; ++win) {
      const int64_t sg = seg0 + (int64_t)win * a.nblk;
      nt += ((int64_t)__ldg(a.offsets + sg + 1) - __ldg(a.offsets + sg) + kEnt - 1) / kEnt;
    }
    if (nt <= 0) continue;
    pc.b = bg / a.G;
    pc.g = (int32_t)(bg - pc.b * a.G);
    pc.c = c;
    pc.seg0 = seg0;
    pc.nt = nt;
    return true;
  }
}
__device__ __forceinline__ void tiles_start(TileWalk& t) {
  t.e = 0;
  t.e_end = 0;
  t.w = -1;
}
// entries [e0, e1) of the piece's next tile (called exactly pc.nt times)
__device__ __forceinline__ void tiles_next(TileWalk& t, const BwdArgs& a, const Piece& pc,
                                           int kEnt, int64_t& e0, int64_t& e1) {
  while (t.e >= t.e_end && t.w + 1 < a.nwin) {
    ++t.w;
    const int64_t sg = pc.seg0 + (int64_t)t.w * a.nblk;
    t.e = __ldg(a.offsets + sg);
    t.e_end = __ldg(a.offsets + sg + 1);
  }
  e0 = t.e;
  e1 = min64(t.e + kEnt, t.e_end);
  t.e = e1;
}
}  // namespace

template <int R>
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ BwdArgs a) {
  static_assert(R >= 1 && R <= 16 && (128 % R) == 0, "128 rows hold whole entries");
  constexpr int kEnt = 128 / R;                  // entries per tile
  constexpr uint32_t kIdKK = idesc_tc(0, 0);     // S^T = K Q^T, dP^T = V dO^T
  constexpr uint32_t kIdKN = idesc_tc(0, 1);     // dV += P^T dO, dK += dS^T Q (A in TMEM)
  constexpr uint32_t kIdNN = idesc_tc(1, 1);     // dQ = dS K
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + kTcOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kTcOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kTcOffMisc + 4);
  int32_t* m_t = reinterpret_cast<int32_t*>(base + kTcOffMeta);
  float* m_lse = reinterpret_cast<float*>(base + kTcOffMeta + 512);
  float* m_d = reinterpret_cast<float*>(base + kTcOffMeta + 1024);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* err = a.err;

  if (tid == 0) {
    mbar_init(bar + TB_KV_FULL, 1);
    mbar_init(bar + TB_KV_EMPTY, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + TB_QDO_FULL0 + i, 128);
      mbar_init(bar + TB_QDO_EMPTY0 + i, 1);
    }
    mbar_init(bar + TB_S_FULL, 1);
    mbar_init(bar + TB_P_FULL, 128);
    mbar_init(bar + TB_DVK_DONE, 1);
    mbar_init(bar + TB_DQ_FULL, 1);
    mbar_init(bar + TB_DQ_EMPTY, 128);
    mbar_init(bar + TB_DKV_FULL, 1);
    mbar_init(bar + TB_DKV_EMPTY, 128);
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
  // k-th completion of a barrier has parity k & 1
  auto W = [&](int id, int64_t k) {
    return mbar_wait(bar + id, (uint32_t)(k & 1), abort_flag, err);
  };
  PieceWalk wk;
  walk_start(wk);
  Piece pc;
  TileWalk tw;
  // lists with fewer entries than the sizes imply (a malformed selection): the
  // dq slot sums would read pieces nobody wrote
  if (blockIdx.x == 0 && tid == 0 && (int64_t)a.offsets[a.nseg] != a.total)
    report(err, MSA_DEVERR_BAD_ENTRY);

  if (warp == 0) {
    // ---------------- K, V of every piece by TMA ----------------
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      for (int64_t p = 0; walk_next(wk, a, pc, kEnt); ++p) {
        if (p > 0 && !W(TB_KV_EMPTY, p - 1)) break;
        mbar_arrive_expect_tx(bar + TB_KV_FULL, 65536u);
        for (int h = 0; h < 2; ++h) {
          tma_load_4d(base + kTcOffK + h * 16384, &tm_k, bar + TB_KV_FULL, h * 64, pc.c * kBlock,
                      pc.g, (int32_t)pc.b);
          tma_load_4d(base + kTcOffV + h * 16384, &tm_v, bar + TB_KV_FULL, h * 64, pc.c * kBlock,
                      pc.g, (int32_t)pc.b);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int64_t n = 0, p = 0;
      bool ok = true;
      const uint32_t ka = smem_u32(base + kTcOffK), va = smem_u32(base + kTcOffV);
      const uint32_t dsa = smem_u32(base + kTcOffDS);
      for (; ok && walk_next(wk, a, pc, kEnt); ++p) {
        if (!W(TB_KV_FULL, p)) { ok = false; break; }
        const int64_t nt = pc.nt;
        // S^T(n) = K Q(n)^T into [0,128): for the first tile of a piece here, for
        // the others right after dQ(n-1) (it only needs P^T(n-1) consumed)
        auto issue_s = [&](int64_t nn) {
          if (!W(TB_QDO_FULL0 + (int)(nn & 1), nn >> 1)) return false;
          tc_fence_after();
          const uint32_t qa = smem_u32(base + kTcOffQ + (int)(nn & 1) * 32768);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem, smem_desc_sw128(ka + off, 16, 1024), smem_desc_sw128(qa + off, 16, 1024),
                      kIdKK, kk > 0 ? 1u : 0u);
          }
          return true;
        };
        if (nt > 0 && !issue_s(n)) { ok = false; break; }
        for (int64_t t = 0; t < nt; ++t, ++n) {
          const int buf = (int)(n & 1);
          // dP^T(n) into [128,256), once the epilogue has read dQ(n-1) there
          if (n > 0 && !W(TB_DQ_EMPTY, n - 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qa = smem_u32(base + kTcOffQ + buf * 32768);
          const uint32_t da = smem_u32(base + kTcOffDO + buf * 32768);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem + 128, smem_desc_sw128(va + off, 16, 1024),
                      smem_desc_sw128(da + off, 16, 1024), kIdKK, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar + TB_S_FULL);
          if (!W(TB_P_FULL, n)) { ok = false; break; }
          if (t == 0 && p > 0 && !W(TB_DKV_EMPTY, p - 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
            umma_bf16_ts(tmem + 256, tmem + kk * 8, smem_desc_sw128(da + kk * 2048, 16384, 1024),
                         kIdKN, acc);
            umma_bf16_ts(tmem + 384, tmem + 128 + kk * 8,
                         smem_desc_sw128(qa + kk * 2048, 16384, 1024), kIdKN, acc);
          }
          umma_commit(bar + TB_QDO_EMPTY0 + buf);
          umma_commit(bar + TB_DVK_DONE);
          // dQ overwrites the columns dS^T was read from, and S^T(n+1) those of
          // P^T: wait for dV, dK first
          if (!W(TB_DVK_DONE, n)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tmem + 128, smem_desc_sw128(dsa + kk * 2048, 16384, 1024),
                      smem_desc_sw128(ka + kk * 2048, 16384, 1024), kIdNN, kk > 0 ? 1u : 0u);
          umma_commit(bar + TB_DQ_FULL);
          if (t + 1 == nt) {
            umma_commit(bar + TB_KV_EMPTY);
            umma_commit(bar + TB_DKV_FULL);
          } else if (!issue_s(n + 1)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && n > 0) {                         // let the last completions land
        W(TB_DQ_FULL, n - 1);
        W(TB_DKV_FULL, p - 1);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- gather: Q and dO rows of each tile ----------------
    const int gt = tid - 128;                    // 0..127
    const int ch = gt & 15;
    int64_t n = 0;
    bool ok = true;
    for (int64_t p = 0; ok && walk_next(wk, a, pc, kEnt); ++p) {
      const int64_t nt = pc.nt;
      tiles_start(tw);
      const __nv_bfloat16* qb = a.q + pc.b * a.qs_b + (int64_t)(pc.g * R) * a.qs_h + ch * 8;
      const __nv_bfloat16* db = a.dout + pc.b * a.ds_b + (int64_t)(pc.g * R) * a.ds_h + ch * 8;
      for (int64_t t = 0; t < nt; ++t, ++n) {
        const int buf = (int)(n & 1);
        if (n >= 2 && !W(TB_QDO_EMPTY0 + buf, (n >> 1) - 1)) { ok = false; break; }
        uint8_t* sq = base + kTcOffQ + buf * 32768;
        uint8_t* sd = base + kTcOffDO + buf * 32768;
        int64_t et, te;
        tiles_next(tw, a, pc, kEnt, et, te);
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
          const int row = it * 8 + (gt >> 4);
          const int64_t ei = et + row / R;
          const int32_t ent = ei < te ? __ldg(a.entries + ei) : -1;
          const bool v = ent >= 0 && (int64_t)(ent >> 4) < a.n_q;
          const int64_t qi = v ? (int64_t)(ent >> 4) : 0;
          const int64_t hoff = (int64_t)(row % R);
          const uint32_t off = (uint32_t)((ch >> 3) * 16384 + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
          cp_async_16(sq + off, v ? (const void*)(qb + qi * a.qs_t + hoff * a.qs_h) : (const void*)a.q,
                      v ? 16u : 0u);
          cp_async_16(sd + off, v ? (const void*)(db + qi * a.ds_t + hoff * a.ds_h) : (const void*)a.dout,
                      v ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(bar + TB_QDO_FULL0 + buf);
      }
    }
  } else if (warp >= 8 && warp < 12) {
    // ---------------- P^T and dS^T (thread = key) ----------------
    const int quarter = warp & 3;
    const int key = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float scale_log2 = a.scale * 1.4426950408889634f;
    const float log2e = 1.4426950408889634f;
    uint8_t* ds = base + kTcOffDS;
    int64_t n = 0;
    bool ok = true;
    for (int64_t p = 0; ok && walk_next(wk, a, pc, kEnt); ++p) {
      const int64_t nt = pc.nt;
      tiles_start(tw);
      const int64_t key_abs = (int64_t)pc.c * kBlock + key;
      for (int64_t t = 0; t < nt; ++t, ++n) {
        // this thread's row (row = key index) data for the tile
        int64_t et, te;
        tiles_next(tw, a, pc, kEnt, et, te);
        const int64_t ei = et + key / R;
        const int32_t ent = ei < te ? __ldg(a.entries + ei) : -1;
        int32_t trow = -1;
        float lse_r = 0.f, d_r = 0.f;
        if (ent >= 0 && (int64_t)(ent >> 4) < a.n_q) {
          const int64_t qi = (int64_t)(ent >> 4);
          const int64_t mrow = (pc.b * a.n_q + qi) * a.H + pc.g * R + (key % R);
          trow = (int32_t)(a.q_pos0 + qi);
          lse_r = __ldg(a.lse + mrow);
          d_r = __ldg(a.delta + mrow);
        }
        if (!W(TB_S_FULL, n)) { ok = false; break; }
        m_t[key] = trow;
        m_lse[key] = lse_r * log2e;
        m_d[key] = d_r;
        named_bar_sync(1, 128);
        tc_fence_after();
        const uint32_t taddr = tmem + lane_base;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t sr[32], dr[32];
          tmem_ld_32x32b_x32(taddr + 32 * cc, sr);
          tmem_ld_32x32b_x32(taddr + 128 + 32 * cc, dr);
          tmem_ld_wait();
          uint32_t pp[16], sp[16];
#pragma unroll
          for (int q = 0; q < 8; ++q) {            // rows 32 cc + 4 q .. + 3
            const int4 t4 = reinterpret_cast<const int4*>(m_t)[8 * cc + q];
            const float4 l4 = reinterpret_cast<const float4*>(m_lse)[8 * cc + q];
            const float4 d4 = reinterpret_cast<const float4*>(m_d)[8 * cc + q];
            const int32_t tv[4] = {t4.x, t4.y, t4.z, t4.w};
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
            float pv[4], sv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const bool live = key_abs <= (int64_t)tv[x];
              const float pr = live ? ex2_approx(u2f(sr[4 * q + x]) * scale_log2 - lv[x]) : 0.f;
              pv[x] = pr;
              sv[x] = live ? pr * (u2f(dr[4 * q + x]) - dv4[x]) : 0.f;
            }
            pp[2 * q] = pack_bf16x2(pv[0], pv[1]);
            pp[2 * q + 1] = pack_bf16x2(pv[2], pv[3]);
            sp[2 * q] = pack_bf16x2(sv[0], sv[1]);
            sp[2 * q + 1] = pack_bf16x2(sv[2], sv[3]);
          }
          tmem_st_32x32b_x16(taddr + 16 * cc, pp);
          tmem_st_32x32b_x16(taddr + 128 + 16 * cc, sp);
          // dS^T row `key`, rows 32 cc .. 32 cc + 31: panel cc / 2, 16-byte chunks
          // 4 (cc % 2) .. + 3, at chunk ^ (key % 8)
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chk = 4 * (cc & 1) + q4;
            uint4 v4 = make_uint4(sp[4 * q4], sp[4 * q4 + 1], sp[4 * q4 + 2], sp[4 * q4 + 3]);
            *reinterpret_cast<uint4*>(ds + (cc >> 1) * 16384 + key * 128 + ((chk ^ (key & 7)) << 4)) = v4;
          }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar + TB_P_FULL);
      }
    }
  } else if (warp >= 12) {
    // ---------------- epilogue: dQ pieces, then dK, dV of each piece ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;         // dQ: lane = row; dK, dV: lane = key
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    int64_t n = 0;
    bool ok = true;
    for (int64_t p = 0; ok && walk_next(wk, a, pc, kEnt); ++p) {
      const int64_t nt = pc.nt;
      tiles_start(tw);
      for (int64_t t = 0; t < nt; ++t, ++n) {
        int64_t et, te;
        tiles_next(tw, a, pc, kEnt, et, te);
        const int64_t ei = et + row / R;
        const int32_t ent = ei < te ? __ldg(a.entries + ei) : -1;
        float* dst = nullptr;
        if (ent >= 0 && (int64_t)(ent >> 4) < a.n_q) {
          const int64_t prow = ((pc.b * a.n_q + (ent >> 4)) * a.G + pc.g) * (int64_t)kTopK * R +
                               (int64_t)(ent & 15) * R + (row % R);
          dst = a.part_dq + prow * kHeadDim;
        }
        if (!W(TB_DQ_FULL, n)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_base + 128 + 32 * cc, r);
          tmem_ld_wait();
          if (dst != nullptr) {
            // 32-byte stores: each lane writes whole sectors of its own row
#pragma unroll
            for (int x = 0; x < 4; ++x)
              st_global_v8(dst + 32 * cc + 8 * x, a.scale * u2f(r[8 * x]),
                           a.scale * u2f(r[8 * x + 1]), a.scale * u2f(r[8 * x + 2]),
                           a.scale * u2f(r[8 * x + 3]), a.scale * u2f(r[8 * x + 4]),
                           a.scale * u2f(r[8 * x + 5]), a.scale * u2f(r[8 * x + 6]),
                           a.scale * u2f(r[8 * x + 7]));
          }
        }
        tc_fence_before();
        mbar_arrive(bar + TB_DQ_EMPTY);
        if (t + 1 == nt) {
          if (!W(TB_DKV_FULL, p)) { ok = false; break; }
          tc_fence_after();
          const int64_t key_abs = (int64_t)pc.c * kBlock + row;
          const bool live = key_abs < a.n_kv;
          const int64_t kb = ((pc.b * a.G + pc.g) * a.n_kv + key_abs) * kHeadDim;
#pragma unroll 1
          for (int which = 0; which < 2; ++which) {      // 0: dV, 1: dK (scaled)
            float* outp = which ? a.dk : a.dv;
            const float f = which ? a.scale : 1.f;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(tmem + lane_base + 256 + 128 * which + 32 * cc, r);
              tmem_ld_wait();
              if (live) {                // this CTA owns the block: plain stores
#pragma unroll
                for (int x = 0; x < 4; ++x)
                  st_global_v8(outp + kb + 32 * cc + 8 * x, f * u2f(r[8 * x]),
                               f * u2f(r[8 * x + 1]), f * u2f(r[8 * x + 2]),
                               f * u2f(r[8 * x + 3]), f * u2f(r[8 * x + 4]),
                               f * u2f(r[8 * x + 5]), f * u2f(r[8 * x + 6]),
                               f * u2f(r[8 * x + 7]));
              }
            }
          }
          tc_fence_before();
          mbar_arrive(bar + TB_DKV_EMPTY);
        }
      }
    }
  }
  // warps 2, 3: idle
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

__global__ void __launch_bounds__(256)
    bwd_dq_reduce_kernel(const float* __restrict__ part_dq, float* __restrict__ dq, int64_t rows,
                         int64_t n_q, int64_t q_pos0, int32_t H, int32_t G) {
  const int lane = threadIdx.x & 31;
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (r >= rows) return;
  const int32_t R = H / G;
  const int32_t h = (int32_t)(r % H), g = h / R;
  const int64_t bq = r / H;                       // b * n_q + i
  const int64_t i = bq % n_q;
  const int64_t nsel = min64(kTopK, (q_pos0 + i) / kBlock + 1);
  const float* p = part_dq + ((bq * G + g) * kTopK * R + (h - g * R)) * kHeadDim + 4 * lane;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t s = 0; s < nsel; ++s) {
    const float4 x = *reinterpret_cast<const float4*>(p + s * R * kHeadDim);
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  }
  *reinterpret_cast<float4*>(dq + r * kHeadDim + 4 * lane) = acc;
}

// ---------------------------------------------------------------------------
// work order: items by tile count, largest first (a counting sort over
// kOrderBuckets buckets; the order inside a bucket is whatever the atomics
// give, which changes only which CTA takes an item, never a result)
// ---------------------------------------------------------------------------
constexpr int kOrderBuckets = 1024;

__device__ __forceinline__ int item_bucket(const int32_t* __restrict__ offsets, int64_t i,
                                           int64_t nblk, int32_t nwin, int kEnt) {
  const int64_t bg = i / nblk;
  const int64_t seg0 = bg * nwin * nblk + (i - bg * nblk);
  int64_t nt = 0;
  for (int32_t w = 0; w < nwin; ++w) {
    const int64_t sg = seg0 + (int64_t)w * nblk;
    nt += ((int64_t)offsets[sg + 1] - offsets[sg] + kEnt - 1) / kEnt;
  }
  return (int)min64(nt, kOrderBuckets - 1);
}

__global__ void __launch_bounds__(256)
    bwd_item_hist_kernel(const int32_t* __restrict__ offsets, int64_t nitems, int64_t nblk,
                         int32_t nwin, int kEnt, int32_t* __restrict__ hist) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nitems;
       i += (int64_t)gridDim.x * blockDim.x)
    atomicAdd(hist + item_bucket(offsets, i, nblk, nwin, kEnt), 1);
}

// counts -> first position of each bucket, buckets in descending order
__global__ void __launch_bounds__(kOrderBuckets) bwd_item_scan_kernel(int32_t* hist) {
  __shared__ int32_t s[kOrderBuckets];
  const int t = threadIdx.x;
  s[t] = hist[kOrderBuckets - 1 - t];
  __syncthreads();
  for (int o = 1; o < kOrderBuckets; o <<= 1) {
    const int32_t v = t >= o ? s[t - o] : 0;
    __syncthreads();
    s[t] += v;
    __syncthreads();
  }
  hist[kOrderBuckets - 1 - t] = s[t] - hist[kOrderBuckets - 1 - t];   // exclusive
}

__global__ void __launch_bounds__(256)
    bwd_item_scatter_kernel(const int32_t* __restrict__ offsets, int64_t nitems, int64_t nblk,
                            int32_t nwin, int kEnt, int32_t* __restrict__ cursor,
                            int32_t* __restrict__ perm) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nitems;
       i += (int64_t)gridDim.x * blockDim.x)
    perm[atomicAdd(cursor + item_bucket(offsets, i, nblk, nwin, kEnt), 1)] = (int32_t)i;
}

template <int R>
static cudaError_t launch_bwd_tc_r(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                   const BwdArgs& a, int grid, cudaStream_t st) {
  auto k = sparse_attn_bwd_tc_kernel<R>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kTcSmemBytes);
  if (e != cudaSuccess) return e;
  k<<<grid, kTcThreads, kTcSmemBytes, st>>>(tm_k, tm_v, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn_bwd(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                   const void* q, int64_t qs_b, int64_t qs_t, int64_t qs_h,
                                   const void* o, int64_t os_b, int64_t os_t, int64_t os_h,
                                   const void* dout, int64_t ds_b, int64_t ds_t, int64_t ds_h,
                                   const float* lse, const int32_t* offsets,
                                   const int32_t* entries, int64_t total_entries, int64_t batch,
                                   int64_t n_q, int64_t n_kv, int64_t q_pos0, int32_t G,
                                   int32_t H, int32_t nblk, int32_t nwin, float scale,
                                   float* delta,
                                   float* part_dq, float* dq, float* dk, float* dv,
                                   int32_t* err, cudaStream_t st) {
  const int32_t R = H / G;
  const int64_t rows = batch * n_q * H;
  const size_t kv_bytes = (size_t)batch * G * n_kv * kHeadDim * sizeof(float);
  cudaError_t e = cudaMemsetAsync(dk, 0, kv_bytes, st);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, kv_bytes, st)) != cudaSuccess) return e;
  bwd_delta_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(o), os_b, os_t, os_h,
      reinterpret_cast<const __nv_bfloat16*>(dout), ds_b, ds_t, ds_h, rows, n_q, H, delta);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  BwdArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.qs_b = qs_b;
  a.qs_t = qs_t;
  a.qs_h = qs_h;
  a.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  a.ds_b = ds_b;
  a.ds_t = ds_t;
  a.ds_h = ds_h;
  a.lse = lse;
  a.delta = delta;
  a.offsets = offsets;
  a.entries = entries;
  a.part_dq = part_dq;
  a.dk = dk;
  a.dv = dv;
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.q_pos0 = q_pos0;
  a.nseg = batch * G * nwin * nblk;
  a.total = total_entries;
  a.G = G;
  a.H = H;
  a.nblk = nblk;
  a.nwin = nwin;
  a.scale = scale;
  a.err = err;
  // one item per (batch, group, KV block); at most one CTA per SM
  a.nitems = batch * G * (int64_t)nblk;
  a.perm = nullptr;
  const int grid = total_entries > 0 ? (int)min64(a.nitems, sms) : 0;
  // the largest-first order lives in dq's memory until the final reduction
  // overwrites it (when dq is large enough to hold it)
  if (grid > 0 && a.nitems > grid && a.nitems < (int64_t(1) << 31) &&
      (int64_t)kOrderBuckets + a.nitems <= rows * kHeadDim) {
    int32_t* hist = reinterpret_cast<int32_t*>(dq);
    int32_t* perm = hist + kOrderBuckets;
    const int kEnt = kBlock / R;
    if ((e = cudaMemsetAsync(hist, 0, kOrderBuckets * sizeof(int32_t), st)) != cudaSuccess)
      return e;
    const unsigned og = (unsigned)min64((a.nitems + 255) / 256, (int64_t)sms * 8);
    bwd_item_hist_kernel<<<og, 256, 0, st>>>(offsets, a.nitems, nblk, nwin, kEnt, hist);
    bwd_item_scan_kernel<<<1, kOrderBuckets, 0, st>>>(hist);
    bwd_item_scatter_kernel<<<og, 256, 0, st>>>(offsets, a.nitems, nblk, nwin, kEnt, hist,
                                                perm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.perm = perm;
  }
  if (grid > 0) {
    switch (R) {
      case 1: e = launch_bwd_tc_r<1>(tm_k, tm_v, a, grid, st); break;
      case 2: e = launch_bwd_tc_r<2>(tm_k, tm_v, a, grid, st); break;
      case 4: e = launch_bwd_tc_r<4>(tm_k, tm_v, a, grid, st); break;
      case 8: e = launch_bwd_tc_r<8>(tm_k, tm_v, a, grid, st); break;
      case 16: e = launch_bwd_tc_r<16>(tm_k, tm_v, a, grid, st); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  bwd_dq_reduce_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(part_dq, dq, rows,
                                                                              n_q, q_pos0, H, G);
  return cudaGetLastError();
}

}  // namespace msa
