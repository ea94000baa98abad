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
// registers; dQ leaves as one fp32 piece per (query, head, slot), summed in
// slot order by a second kernel (deterministic), exactly like the forward's
// (m, l, acc) pieces and merge.
//
// Three kernels:
//  * bwd_delta_kernel      -- D = dO.o per (query, head), one warp each;
//  * sparse_attn_bwd_kernel<R> -- 8 warps; the entries of the block->query
//    lists are cut into equal runs ("chunks", one CTA each, strided over a
//    grid of at most one CTA per SM), a chunk into pieces (one per segment =
//    KV block) and a piece into 32-row tiles (32 / R entries x R heads).
//    Per piece: K, V by TMA (128B swizzle).  Per tile: Q and dO rows and the
//    rows' lse and D by cp.async (double-buffered, the entries one tile
//    further ahead in registers); warp w owns keys 16w .. 16w+15 and forms
//    S^T = K Q^T and dP^T = V dO^T (mma.sync m16n8k16), P^T and dS^T in
//    registers, then dV += P^T dO and dK += dS^T Q from those registers;
//    dS^T goes to shared memory for dQ = dS K (warp w: 16 rows x 32 dims).
//    At the end of a piece dK and dV are added to fp32 accumulators in
//    global memory (one vector atomic per element pair: a block split over
//    several chunks sums its parts there);
//  * bwd_dq_reduce_kernel  -- dQ = sum over the slots of the pieces, one warp
//    per (query, head).
#include "common.cuh"

namespace msa {

namespace {

constexpr int kBwThreads = 256;
constexpr int kBwRows = 32;                      // gathered rows per tile
constexpr int kBwOffK = 0, kBwOffV = 32768;
constexpr int kBwOffQ = 65536;                   // 2 buffers x 8 KB (2 panels x 32 rows x 128 B)
constexpr int kBwOffDO = kBwOffQ + 2 * 8192;
constexpr int kBwOffDS = kBwOffDO + 2 * 8192;    // dS^T [128 keys][32 rows] bf16, 64 B per key
constexpr int kBwOffMeta = kBwOffDS + 8192;
// meta per buffer: lse[32], D[32] (fp32), ent[32] (int32)
constexpr int kBwMetaBytes = 3 * kBwRows * 4;
constexpr int kBwOffBar = kBwOffMeta + 2 * kBwMetaBytes;
constexpr int kBwSmemBytes = 1024 + kBwOffBar + 16;

__device__ __forceinline__ void cp_async_4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

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
  int64_t n_q, n_kv, q_pos0, nseg, total, chunk_entries;
  int32_t G, H, nblk;
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

template <int R>
__global__ void __launch_bounds__(kBwThreads, 1)
    sparse_attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const __grid_constant__ BwdArgs a) {
  static_assert(R >= 1 && R <= 16 && (kBwRows % R) == 0, "32 rows hold whole entries");
  constexpr int kEnt = kBwRows / R;              // entries per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* kv_bar = reinterpret_cast<uint64_t*>(base + kBwOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + kBwOffBar + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  const float log2e = 1.4426950408889634f;

  if (tid == 0) {
    mbar_init(kv_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  __syncthreads();

  const uint32_t k_s = smem_u32(base + kBwOffK), v_s = smem_u32(base + kBwOffV);
  const uint32_t ds_s = smem_u32(base + kBwOffDS);
  // prefetch role: row pr = tid / 8 of the tile, 16-byte chunks 2 (tid % 8) and + 1
  const int pr = tid >> 3, pc = (tid & 7) * 2;
  uint32_t kv_phase = 0;
  bool stop = false, kv_phase_used = false;

  const int64_t nchunks = (a.total + a.chunk_entries - 1) / a.chunk_entries;
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int64_t c_begin = chunk * a.chunk_entries;
    const int64_t c_end = min64(c_begin + a.chunk_entries, a.total);
    int64_t e = c_begin;
    int64_t seg = -1;
    while (e < c_end) {
      // the segment holding entry e: a few steps past the previous one, else a search
      {
        int64_t s2 = seg + 1;
        const int64_t lim = seg < 0 ? 0 : min64(seg + 5, a.nseg);
        while (s2 < lim && a.offsets[s2 + 1] <= e) ++s2;
        seg = (s2 < lim) ? s2 : segment_of(a.offsets, a.nseg, e);
      }
      const int64_t p_end = min64((int64_t)a.offsets[seg + 1], c_end);
      const int64_t p_begin = e;
      if (p_end <= p_begin) {                    // fewer entries listed than the sizes imply
        if (tid == 0) report(a.err, MSA_DEVERR_BAD_ENTRY);
        stop = true;                             // uniform: every thread read the same offsets
        break;
      }
      e = p_end;
      const int32_t c = (int32_t)(seg % a.nblk);
      const int64_t bg = seg / a.nblk;
      const int32_t g = (int32_t)(bg % a.G);
      const int64_t b = bg / a.G;
      const int64_t ntiles = (p_end - p_begin + kEnt - 1) / kEnt;

      __syncthreads();                           // K, V, the buffers and dS^T are free
      if (tid == 0) {
        mbar_arrive_expect_tx(kv_bar, 65536u);
        for (int p = 0; p < 2; ++p) {
          tma_load_4d(base + kBwOffK + p * 16384, &tm_k, kv_bar, p * 64, c * kBlock, g, (int32_t)b);
          tma_load_4d(base + kBwOffV + p * 16384, &tm_v, kv_bar, p * 64, c * kBlock, g, (int32_t)b);
        }
      }

      // the prefetch of tile n into buffer n & 1: this thread's row's entry
      // value for tile n is `ent_cur`; rows past the piece load zeros
      auto prefetch = [&](int64_t n, int32_t ent) {
        const int buf = (int)(n & 1);
        uint8_t* qd = base + kBwOffQ + buf * 8192;
        uint8_t* dd = base + kBwOffDO + buf * 8192;
        uint8_t* meta = base + kBwOffMeta + buf * kBwMetaBytes;
        const bool ok = ent >= 0;
        const int64_t qi = ok ? (ent >> 4) : 0;
        const int64_t h = (int64_t)g * R + (pr % R);
        const __nv_bfloat16* qrow = a.q + b * a.qs_b + qi * a.qs_t + h * a.qs_h;
        const __nv_bfloat16* drow = a.dout + b * a.ds_b + qi * a.ds_t + h * a.ds_h;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int ch = pc + x;
          const uint32_t off = (uint32_t)((ch >> 3) * 4096 + pr * 128 + (((ch & 7) ^ (pr & 7)) << 4));
          cp_async_16(qd + off, ok ? (const void*)(qrow + ch * 8) : (const void*)a.q, ok ? 16u : 0u);
          cp_async_16(dd + off, ok ? (const void*)(drow + ch * 8) : (const void*)a.dout, ok ? 16u : 0u);
        }
        if ((tid & 7) == 0) {
          const int64_t mrow = (b * a.n_q + qi) * a.H + h;
          cp_async_4(meta + pr * 4, ok ? (const void*)(a.lse + mrow) : (const void*)a.lse, ok ? 4u : 0u);
          cp_async_4(meta + 128 + pr * 4, ok ? (const void*)(a.delta + mrow) : (const void*)a.delta,
                     ok ? 4u : 0u);
          reinterpret_cast<int32_t*>(meta + 256)[pr] = ent;
        }
        cp_async_commit();
      };
      auto load_ent = [&](int64_t n) -> int32_t {
        const int64_t ei = p_begin + n * kEnt + pr / R;
        return (n < ntiles && ei < p_end) ? __ldg(a.entries + ei) : -1;
      };

      float dv_acc[16][4], dk_acc[16][4];
#pragma unroll
      for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int x = 0; x < 4; ++x) dv_acc[i][x] = dk_acc[i][x] = 0.f;

      int32_t ent_next = load_ent(0);
      prefetch(0, ent_next);
      ent_next = load_ent(1);
      bool kv_ok = true;
      for (int64_t n = 0; n < ntiles; ++n) {
        const int buf = (int)(n & 1);
        if (n + 1 < ntiles) {
          prefetch(n + 1, ent_next);
          ent_next = load_ent(n + 2);
          cp_async_wait_group<1>();
        } else {
          cp_async_wait_group<0>();
        }
        __syncthreads();                         // tile n in shared memory
        if (n == 0) {
          kv_ok = mbar_wait(kv_bar, kv_phase, abort_flag, a.err);
          kv_phase ^= 1u;
          kv_phase_used = true;
        }
        const uint32_t q_s = smem_u32(base + kBwOffQ + buf * 8192);
        const uint32_t do_s = smem_u32(base + kBwOffDO + buf * 8192);
        const float* m_lse = reinterpret_cast<const float*>(base + kBwOffMeta + buf * kBwMetaBytes);
        const float* m_d = m_lse + kBwRows;
        const int32_t* m_ent = reinterpret_cast<const int32_t*>(m_d + kBwRows);

        // S^T and dP^T: keys 16 warp + gq (+8) x rows 8 j + 2 tq (+1)
        float st[4][4], dpt[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int x = 0; x < 4; ++x) st[j][x] = dpt[j][x] = 0.f;
        {
          const int krow = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int qrow_l = (lane & 7) + 8 * (lane >> 4);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const int ach = 2 * ks + (lane >> 4);              // A: K / V rows
            const uint32_t aoff = (uint32_t)((ach >> 3) * 16384 + krow * 128 +
                                             (((ach & 7) ^ (krow & 7)) << 4));
            uint32_t ka0, ka1, ka2, ka3, va0, va1, va2, va3;
            ldmatrix_x4(k_s + aoff, ka0, ka1, ka2, ka3);
            ldmatrix_x4(v_s + aoff, va0, va1, va2, va3);
            const int bch = 2 * ks + ((lane >> 3) & 1);        // B: Q / dO rows
#pragma unroll
            for (int jp = 0; jp < 2; ++jp) {
              const int rr = 16 * jp + qrow_l;
              const uint32_t boff = (uint32_t)((bch >> 3) * 4096 + rr * 128 +
                                               (((bch & 7) ^ (rr & 7)) << 4));
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4(q_s + boff, b0, b1, b2, b3);
              mma_bf16_16816(st[2 * jp], ka0, ka1, ka2, ka3, b0, b1);
              mma_bf16_16816(st[2 * jp + 1], ka0, ka1, ka2, ka3, b2, b3);
              ldmatrix_x4(do_s + boff, b0, b1, b2, b3);
              mma_bf16_16816(dpt[2 * jp], va0, va1, va2, va3, b0, b1);
              mma_bf16_16816(dpt[2 * jp + 1], va0, va1, va2, va3, b2, b3);
            }
          }
        }
        // P^T and dS^T; rows with no entry carry t = -1, so every key masks them
        uint32_t pa[4][2], sa[4][2];             // bf16 pairs: [n-tile][key half]
        {
          const int64_t key0 = (int64_t)c * kBlock + 16 * warp + gq;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int row = 8 * j + 2 * tq;
            const float2 lse2 = *reinterpret_cast<const float2*>(m_lse + row);
            const float2 d2 = *reinterpret_cast<const float2*>(m_d + row);
            const int32_t e0 = m_ent[row], e1 = m_ent[row + 1];
            const int64_t t0 = e0 >= 0 ? a.q_pos0 + (e0 >> 4) : -1;
            const int64_t t1 = e1 >= 0 ? a.q_pos0 + (e1 >> 4) : -1;
            float p[4], s[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int64_t key = key0 + ((x >> 1) ? 8 : 0);
              const bool col1 = x & 1;
              const int64_t tt = col1 ? t1 : t0;
              const float lv = col1 ? lse2.y : lse2.x;
              const float dd = col1 ? d2.y : d2.x;
              p[x] = key <= tt ? ex2_approx(st[j][x] * scale_log2 - lv * log2e) : 0.f;
              s[x] = p[x] * (dpt[j][x] - dd);
            }
            pa[j][0] = pack_bf16x2(p[0], p[1]);
            pa[j][1] = pack_bf16x2(p[2], p[3]);
            sa[j][0] = pack_bf16x2(s[0], s[1]);
            sa[j][1] = pack_bf16x2(s[2], s[3]);
          }
        }
        // dS^T to shared memory: key row 64 B, 16-byte chunk j holds rows 8j .. 8j+7,
        // stored at chunk j ^ ((key >> 1) & 3)
        {
          const int k0 = 16 * warp + gq, k1 = k0 + 8;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t o0 = (uint32_t)(k0 * 64 + ((j ^ ((k0 >> 1) & 3)) << 4) + tq * 4);
            const uint32_t o1 = (uint32_t)(k1 * 64 + ((j ^ ((k1 >> 1) & 3)) << 4) + tq * 4);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ds_s + o0), "r"(sa[j][0]) : "memory");
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(ds_s + o1), "r"(sa[j][1]) : "memory");
          }
        }
        // dV += P^T dO and dK += dS^T Q: k-steps over the 32 rows, B by transposing loads
        {
          const int rrow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t pa0 = pa[2 * kk][0], pa1 = pa[2 * kk][1];
            const uint32_t pa2 = pa[2 * kk + 1][0], pa3 = pa[2 * kk + 1][1];
            const uint32_t sa0 = sa[2 * kk][0], sa1 = sa[2 * kk][1];
            const uint32_t sa2 = sa[2 * kk + 1][0], sa3 = sa[2 * kk + 1][1];
            const int rr = 16 * kk + rrow;
#pragma unroll
            for (int np = 0; np < 8; ++np) {               // dim tiles 2 np, 2 np + 1
              const int ch = 2 * np + (lane >> 4);
              const uint32_t off = (uint32_t)((ch >> 3) * 4096 + rr * 128 +
                                              (((ch & 7) ^ (rr & 7)) << 4));
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4_trans(do_s + off, b0, b1, b2, b3);
              mma_bf16_16816(dv_acc[2 * np], pa0, pa1, pa2, pa3, b0, b1);
              mma_bf16_16816(dv_acc[2 * np + 1], pa0, pa1, pa2, pa3, b2, b3);
              ldmatrix_x4_trans(q_s + off, b0, b1, b2, b3);
              mma_bf16_16816(dk_acc[2 * np], sa0, sa1, sa2, sa3, b0, b1);
              mma_bf16_16816(dk_acc[2 * np + 1], sa0, sa1, sa2, sa3, b2, b3);
            }
          }
        }
        const int32_t dq_ent0 = m_ent[16 * (warp & 1) + gq];
        const int32_t dq_ent1 = m_ent[16 * (warp & 1) + gq + 8];
        __syncthreads();                         // dS^T complete; buffer n & 1 read
        // dQ = scale dS K: warp -> rows 16 (warp & 1) + .., dims 32 (warp >> 1) + ..
        {
          float dq[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j) dq[j][0] = dq[j][1] = dq[j][2] = dq[j][3] = 0.f;
          const int mrow = warp & 1, dcol = warp >> 1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int key = 16 * kk + (lane & 7) + 8 * (lane >> 4);
            const int rch = 2 * mrow + ((lane >> 3) & 1);
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(ds_s + (uint32_t)(key * 64 + ((rch ^ ((key >> 1) & 3)) << 4)),
                              a0, a1, a2, a3);
            const int kkey = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int np = 0; np < 2; ++np) {
              const int ch = 4 * dcol + 2 * np + (lane >> 4);
              const uint32_t off = (uint32_t)((ch >> 3) * 16384 + kkey * 128 +
                                              (((ch & 7) ^ (kkey & 7)) << 4));
              uint32_t b0, b1, b2, b3;
              ldmatrix_x4_trans(k_s + off, b0, b1, b2, b3);
              mma_bf16_16816(dq[2 * np], a0, a1, a2, a3, b0, b1);
              mma_bf16_16816(dq[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
          }
          // rows 16 mrow + gq and + 8: piece row (b, i, g, slot, r) of [B, n_q, G, 16, R]
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int row = 16 * mrow + gq + 8 * hf;
            const int32_t ent = hf ? dq_ent1 : dq_ent0;
            if (ent >= 0 && kv_ok) {
              const int64_t prow = ((b * a.n_q + (ent >> 4)) * a.G + g) * (int64_t)kTopK * R +
                                   (int64_t)(ent & 15) * R + (row % R);
              float* dst = a.part_dq + prow * kHeadDim + 32 * dcol + 2 * tq;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float2*>(dst + 8 * j) =
                    make_float2(a.scale * dq[j][2 * hf], a.scale * dq[j][2 * hf + 1]);
            }
          }
        }
      }
      // the piece's dK, dV rows: keys 16 warp + gq (+8), dims 8 n + 2 tq (+1)
      if (kv_ok) {
        const int64_t kbase = ((b * a.G + g) * a.n_kv) * kHeadDim;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int64_t key = (int64_t)c * kBlock + 16 * warp + gq + 8 * hf;
          if (key < a.n_kv) {
            float* dkr = a.dk + kbase + key * kHeadDim + 2 * tq;
            float* dvr = a.dv + kbase + key * kHeadDim + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
              atomicAdd(reinterpret_cast<float2*>(dkr + 8 * nt),
                        make_float2(a.scale * dk_acc[nt][2 * hf], a.scale * dk_acc[nt][2 * hf + 1]));
              atomicAdd(reinterpret_cast<float2*>(dvr + 8 * nt),
                        make_float2(dv_acc[nt][2 * hf], dv_acc[nt][2 * hf + 1]));
            }
          }
        }
      }
      if (__syncthreads_or(*abort_flag != 0)) {
        stop = true;
        break;
      }
    }
    if (stop) break;
  }
  // after an abort, the last K/V load may still be in flight
  if (stop && kv_phase_used && tid == 0) mbar_drain(kv_bar, kv_phase ^ 1u, a.err);
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

template <int R>
static cudaError_t launch_bwd_r(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                const BwdArgs& a, int grid, cudaStream_t st) {
  auto k = sparse_attn_bwd_kernel<R>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kBwSmemBytes);
  if (e != cudaSuccess) return e;
  k<<<grid, kBwThreads, kBwSmemBytes, st>>>(tm_k, tm_v, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn_bwd(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                   const void* q, int64_t qs_b, int64_t qs_t, int64_t qs_h,
                                   const void* o, int64_t os_b, int64_t os_t, int64_t os_h,
                                   const void* dout, int64_t ds_b, int64_t ds_t, int64_t ds_h,
                                   const float* lse, const int32_t* offsets,
                                   const int32_t* entries, int64_t total_entries, int64_t batch,
                                   int64_t n_q, int64_t n_kv, int64_t q_pos0, int32_t G,
                                   int32_t H, int32_t nblk, float scale, float* delta,
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
  a.nseg = batch * G * nblk;
  a.total = total_entries;
  a.G = G;
  a.H = H;
  a.nblk = nblk;
  a.scale = scale;
  a.err = err;
  // equal runs of entries, whole tiles each, about 8 per SM
  const int64_t ent_per_tile = kBwRows / R;
  const int64_t tiles = (total_entries + ent_per_tile - 1) / ent_per_tile;
  const int64_t tiles_per_chunk = max64(16, (tiles + 8LL * sms - 1) / (8LL * sms));
  a.chunk_entries = tiles_per_chunk * ent_per_tile;
  const int64_t nchunks = (total_entries + a.chunk_entries - 1) / a.chunk_entries;
  const int grid = (int)min64(nchunks, sms);
  if (grid > 0) {
    switch (R) {
      case 1: e = launch_bwd_r<1>(tm_k, tm_v, a, grid, st); break;
      case 2: e = launch_bwd_r<2>(tm_k, tm_v, a, grid, st); break;
      case 4: e = launch_bwd_r<4>(tm_k, tm_v, a, grid, st); break;
      case 8: e = launch_bwd_r<8>(tm_k, tm_v, a, grid, st); break;
      case 16: e = launch_bwd_r<16>(tm_k, tm_v, a, grid, st); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  bwd_dq_reduce_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(part_dq, dq, rows,
                                                                              n_q, q_pos0, H, G);
  return cudaGetLastError();
}

}  // namespace msa
