// Inversion of the per-query block lists into per-block query lists (CSR),
// the index the KV-block-outer attention kernel walks.
//
// Source: page "MSA 稀疏注意力三国杀", section "Kernel 创新：Outer Gather Q":
// the KV block is the outer loop and all queries that chose it are gathered
// and computed together, so each block is read once.  The inversion itself is
// not spelled out on the pages; this is a deterministic counting sort.
//
// The query indices are cut into windows of W consecutive queries (W a
// multiple of the 128-query tile); segments are (batch, group, window, block)
// in that order, and inside a segment the entries (i << 4 | slot) are
// ascending in the query index i.  A KV-block-outer kernel that walks the
// segments in order then gathers, at any time, the query rows of one window
// only, which stay in L2.  Steps:
//   1. count:   per 128-query tile, a shared-memory histogram over blocks;
//   2. colscan: per (window, block), exclusive prefix over the window's tiles
//      (in place) + totals (coalesced two-pass form for many tiles, one
//      thread per column else);
//   3. offsets: exclusive scan of the totals over all segments (chunk sums,
//      scan of the chunk sums, chunk-local scans);
//   4. scatter: per tile, queries in ascending order claim consecutive slots
//      of each block's range, so the order never depends on timing; each
//      (query, slot) also records the position it claimed (entry_pos, the
//      shape of sel, -1 for an empty slot), which is where the attention
//      writes that entry's piece and where the merge finds it.
// Workspace: tile histograms [B*G, ntiles, nblk] + totals [B*G*nwin*nblk] +
// chunk sums [ceil(B*G*nwin*nblk / 4096)], int32.  One query per row (decode) takes a
// two-launch path that needs only the per-row counts.
#include <algorithm>

#include "common.cuh"

namespace msa {

constexpr int kCsrTile = 128;   // queries per tile

__global__ void __launch_bounds__(256)
    csr_count_kernel(const int32_t* __restrict__ sel, int64_t n_q, int64_t q_pos0,
                     int32_t nblk, int32_t ntiles, int32_t* __restrict__ tile_counts,
                     int32_t* err) {
  extern __shared__ int32_t hist[];
  const int tile = blockIdx.x;
  const int64_t bg = blockIdx.y;
  for (int c = threadIdx.x; c < nblk; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  const int64_t q0 = (int64_t)tile * kCsrTile;
  const int64_t nq = min64(kCsrTile, n_q - q0);
  const int32_t* srow = sel + (bg * n_q + q0) * kTopK;
  for (int idx = threadIdx.x; idx < nq * kTopK; idx += blockDim.x) {
    const int32_t c = srow[idx];
    if (c < 0) continue;
    const int64_t own = (q_pos0 + q0 + idx / kTopK) / kBlock;
    if (c > own || c >= nblk) {
      report(err, MSA_DEVERR_BAD_BLOCK);
      continue;
    }
    atomicAdd(&hist[c], 1);
  }
  __syncthreads();
  int32_t* dst = tile_counts + (bg * ntiles + tile) * (int64_t)nblk;
  for (int c = threadIdx.x; c < nblk; c += blockDim.x) dst[c] = hist[c];
}

// Column scan for few tiles per window: one thread per (batch-group, block),
// walking all tiles; the prefix restarts at every window boundary (tw tiles).
__global__ void __launch_bounds__(256)
    csr_colscan_small_kernel(int32_t* __restrict__ tile_counts, int32_t* __restrict__ totals,
                             int32_t nblk, int32_t ntiles, int32_t tw, int32_t nwin) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t bg = blockIdx.y;
  if (c >= nblk) return;
  int32_t* col = tile_counts + bg * ntiles * (int64_t)nblk + c;
  int32_t run = 0;
  int w = 0;
  for (int t = 0; t < ntiles; ++t) {
    if (t == (w + 1) * tw) {
      totals[(bg * nwin + w) * nblk + c] = run;
      run = 0;
      ++w;
    }
    const int32_t v = col[(int64_t)t * nblk];
    col[(int64_t)t * nblk] = run;
    run += v;
  }
  totals[(bg * nwin + w) * nblk + c] = run;
}

// Column scan, coalesced: a block takes 32 adjacent blocks (one per lane) of
// one (batch, group, window) and its 8 warps split the window's query tiles;
// each warp sums its tiles, the warps' partial sums give each warp its
// starting prefix, and a second pass writes the exclusive prefixes in place.
constexpr int kColWarps = 8;

__global__ void __launch_bounds__(kColWarps * 32)
    csr_colscan_kernel(int32_t* __restrict__ tile_counts, int32_t* __restrict__ totals,
                       int32_t nblk, int32_t ntiles, int32_t tw, int32_t nwin) {
  __shared__ int32_t part[kColWarps][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  const int64_t bgw = blockIdx.y;                 // (batch-group) * nwin + window
  const int64_t bg = bgw / nwin;
  const int win = (int)(bgw - bg * nwin);
  int32_t* col = tile_counts + bg * ntiles * (int64_t)nblk + c;
  const int wt0 = win * tw, wt1 = min(ntiles, wt0 + tw);
  const int per = (wt1 - wt0 + kColWarps - 1) / kColWarps;
  const int t0 = min(wt1, wt0 + w * per), t1 = min(wt1, t0 + per);
  int32_t s = 0;
  if (c < nblk) {
#pragma unroll 8
    for (int t = t0; t < t1; ++t) s += col[(int64_t)t * nblk];
  }
  part[w][lane] = s;
  __syncthreads();
  int32_t run = 0, total = 0;
#pragma unroll
  for (int k = 0; k < kColWarps; ++k) {
    run += (k < w) ? part[k][lane] : 0;
    total += part[k][lane];
  }
  if (c < nblk) {
#pragma unroll 8
    for (int t = t0; t < t1; ++t) {
      const int32_t v = col[(int64_t)t * nblk];
      col[(int64_t)t * nblk] = run;
      run += v;
    }
    if (w == 0) totals[bgw * nblk + c] = total;
  }
}

// Exclusive scan of the per-segment totals into offsets[0..n], in three
// steps over chunks of kScanChunk values: chunk sums, a scan of the chunk
// sums, then a block-local scan of each chunk plus its chunk prefix.
constexpr int kScanThreads = 1024;
constexpr int kScanPerThread = 4;
constexpr int kScanChunk = kScanThreads * kScanPerThread;

// inclusive block scan of one value per thread (1024 threads); returns the
// inclusive prefix, *block_total receives the sum
__device__ __forceinline__ int32_t block_scan_incl(int32_t v, int32_t* warp_sums,
                                                   int32_t* block_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int32_t r = incl + (warp > 0 ? warp_sums[warp - 1] : 0);
  *block_total = warp_sums[31];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kScanThreads)
    csr_chunk_sums_kernel(const int32_t* __restrict__ totals, int64_t n,
                          int32_t* __restrict__ chunk_sums) {
  __shared__ int32_t ws[32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk + threadIdx.x * kScanPerThread;
  int32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k)
    if (base + k < n) s += totals[base + k];
  int32_t tot;
  block_scan_incl(s, ws, &tot);
  if (threadIdx.x == 0) chunk_sums[blockIdx.x] = tot;
}

// single block: exclusive scan of the chunk sums in place; total to offsets[n]
__global__ void __launch_bounds__(kScanThreads)
    csr_chunk_scan_kernel(int32_t* __restrict__ chunk_sums, int64_t nchunks, int64_t n,
                          int32_t* __restrict__ offsets) {
  __shared__ int32_t ws[32];
  int32_t carry = 0;
  for (int64_t base = 0; base < nchunks; base += kScanThreads) {
    const int64_t i = base + threadIdx.x;
    const int32_t v = (i < nchunks) ? chunk_sums[i] : 0;
    int32_t tot;
    const int32_t incl = block_scan_incl(v, ws, &tot);
    if (i < nchunks) chunk_sums[i] = carry + incl - v;
    carry += tot;
  }
  if (threadIdx.x == 0) offsets[n] = carry;
}

__global__ void __launch_bounds__(kScanThreads)
    csr_chunk_apply_kernel(const int32_t* __restrict__ totals, int64_t n,
                           const int32_t* __restrict__ chunk_prefix,
                           int32_t* __restrict__ offsets) {
  __shared__ int32_t ws[32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk + threadIdx.x * kScanPerThread;
  int32_t v[kScanPerThread];
  int32_t s = 0;
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    v[k] = (base + k < n) ? totals[base + k] : 0;
    s += v[k];
  }
  int32_t tot;
  int32_t run = block_scan_incl(s, ws, &tot) - s + chunk_prefix[blockIdx.x];
#pragma unroll
  for (int k = 0; k < kScanPerThread; ++k) {
    if (base + k < n) offsets[base + k] = run;
    run += v[k];
  }
}

__global__ void __launch_bounds__(32)
    csr_scatter_kernel(const int32_t* __restrict__ sel, int64_t n_q, int64_t q_pos0,
                       int32_t nblk, int32_t ntiles, int32_t tw, int32_t nwin,
                       const int32_t* __restrict__ tile_counts,
                       const int32_t* __restrict__ offsets, int32_t* __restrict__ entries,
                       int32_t* __restrict__ entry_pos, int64_t cap) {
  extern __shared__ int32_t base[];
  const int tile = blockIdx.x;
  const int64_t bg = blockIdx.y;
  const int lane = threadIdx.x;
  const int32_t* tc = tile_counts + (bg * ntiles + tile) * (int64_t)nblk;
  const int32_t* off = offsets + (bg * nwin + tile / tw) * nblk;
  for (int c = lane; c < nblk; c += 32) base[c] = off[c] + tc[c];
  __syncwarp();
  const int64_t q0 = (int64_t)tile * kCsrTile;
  const int64_t nq = min64(kCsrTile, n_q - q0);
  for (int64_t i = 0; i < nq; ++i) {
    const int64_t qi = q0 + i;
    if (lane < kTopK) {
      const int64_t r = (bg * n_q + qi) * kTopK + lane;
      const int32_t c = sel[r];
      const int64_t own = (q_pos0 + qi) / kBlock;
      int32_t at = -1;
      if (c >= 0 && c <= own && c < nblk) {
        const int32_t p = base[c];
        base[c] = p + 1;                // blocks within one row are distinct
        if (p >= 0 && p < cap) {
          entries[p] = (int32_t)((qi << 4) | lane);
          at = p;
        }
      }
      entry_pos[r] = at;
    }
    __syncwarp();
  }
}

// One query per (batch, group) row (decode).  Each segment then holds at most
// one entry, and the lists follow from the rows directly: the offset of block
// c in row r is (entries of the rows before r) + (selected blocks of r below
// c), and each selected block gets its entry at that offset.  Two launches:
// per-row counts, then one warp per row writes its offsets and entries.
constexpr int kRowWarps = 8;

__global__ void __launch_bounds__(kRowWarps * 32)
    csr_rows_count_kernel(const int32_t* __restrict__ sel, int64_t n_rows, int64_t q_pos0,
                          int32_t nblk, int32_t* __restrict__ counts, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  const int64_t own = q_pos0 / kBlock;
  const int32_t c = (lane < kTopK) ? sel[r * kTopK + lane] : -1;
  const bool v = c >= 0 && c <= own && c < nblk;
  if (c >= 0 && !v) report(err, MSA_DEVERR_BAD_BLOCK);
  const int32_t cnt = __popc(__ballot_sync(0xffffffffu, v));
  if (lane == 0) counts[r] = cnt;
}

__global__ void __launch_bounds__(kRowWarps * 32)
    csr_rows_fill_kernel(const int32_t* __restrict__ sel, int64_t n_rows, int64_t q_pos0,
                         int32_t nblk, const int32_t* __restrict__ counts,
                         int32_t* __restrict__ offsets, int32_t* __restrict__ entries,
                         int32_t* __restrict__ entry_pos, int64_t cap) {
  __shared__ int32_t part[kRowWarps * 32];
  __shared__ int32_t row_base[kRowWarps + 1];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * kRowWarps;
  // entries of all rows before this block's first row
  int32_t s = 0;
  for (int64_t i = threadIdx.x; i < r0; i += blockDim.x) s += counts[i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t b = 0;
    for (int i = 0; i < kRowWarps * 32; ++i) b += part[i];
    for (int k = 0; k <= kRowWarps; ++k) {
      row_base[k] = b;
      if (r0 + k < n_rows) b += counts[r0 + k];
    }
  }
  __syncthreads();
  const int64_t r = r0 + w;
  if (r >= n_rows) return;
  const int64_t own = q_pos0 / kBlock;
  const int32_t base = row_base[w];
  const int32_t raw = (lane < kTopK) ? sel[r * kTopK + lane] : -1;
  const int32_t mine = (raw >= 0 && raw <= own && raw < nblk) ? raw : 0x7FFFFFFF;
  int32_t ck[kTopK];
#pragma unroll
  for (int k = 0; k < kTopK; ++k) ck[k] = __shfl_sync(0xffffffffu, mine, k);
  int32_t* off = offsets + r * nblk;
  for (int c = lane; c < nblk; c += 32) {
    int32_t below = 0;
#pragma unroll
    for (int k = 0; k < kTopK; ++k) below += (ck[k] < c) ? 1 : 0;
    off[c] = base + below;
  }
  if (lane < kTopK) {
    int32_t at = -1;
    if (mine != 0x7FFFFFFF) {
      int32_t below = 0;
#pragma unroll
      for (int k = 0; k < kTopK; ++k) below += (ck[k] < mine) ? 1 : 0;
      const int64_t p = (int64_t)base + below;
      if (p < cap) {
        entries[p] = lane;                   // query 0 of the row, slot `lane`
        at = (int32_t)p;
      }
    }
    entry_pos[r * kTopK + lane] = at;
  }
  if (r == n_rows - 1 && lane == 0) offsets[n_rows * nblk] = row_base[w + 1];
}

size_t block_lists_workspace(int64_t bgcount, int64_t n_q, int64_t nblk, int64_t window) {
  const int64_t ntiles = (n_q + kCsrTile - 1) / kCsrTile;
  const int64_t nwin = (n_q + window - 1) / window;
  const int64_t nseg = bgcount * nwin * nblk;
  const int64_t nchunks = (nseg + kScanChunk - 1) / kScanChunk;
  return (size_t)(bgcount * ntiles * nblk + nseg + nchunks) * sizeof(int32_t);
}

cudaError_t launch_block_lists(const int32_t* sel, int64_t bgcount, int64_t n_q,
                               int64_t q_pos0, int64_t nblk, int64_t window, int32_t* offsets,
                               int32_t* entries, int32_t* entry_pos, int64_t cap, void* ws,
                               int32_t* err, cudaStream_t st) {
  if (n_q == 1) {
    // one window: segment (bg, c) = bg * nblk + c
    int32_t* counts = reinterpret_cast<int32_t*>(ws);
    const unsigned grid = (unsigned)((bgcount + kRowWarps - 1) / kRowWarps);
    csr_rows_count_kernel<<<grid, kRowWarps * 32, 0, st>>>(sel, bgcount, q_pos0, (int32_t)nblk,
                                                           counts, err);
    csr_rows_fill_kernel<<<grid, kRowWarps * 32, 0, st>>>(sel, bgcount, q_pos0, (int32_t)nblk,
                                                          counts, offsets, entries, entry_pos,
                                                          cap);
    return cudaGetLastError();
  }
  const int64_t ntiles = (n_q + kCsrTile - 1) / kCsrTile;
  const int64_t nwin = (n_q + window - 1) / window;
  const int32_t tw = (int32_t)(window / kCsrTile);        // tiles per window
  int32_t* tile_counts = reinterpret_cast<int32_t*>(ws);
  int32_t* totals = tile_counts + bgcount * ntiles * nblk;
  const size_t hist_bytes = (size_t)nblk * sizeof(int32_t);
  cudaError_t e;
  if (hist_bytes > 48 * 1024) {
    e = cudaFuncSetAttribute(csr_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)hist_bytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(csr_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)hist_bytes);
    if (e != cudaSuccess) return e;
  }
  dim3 g1((unsigned)ntiles, (unsigned)bgcount);
  csr_count_kernel<<<g1, 256, hist_bytes, st>>>(sel, n_q, q_pos0, (int32_t)nblk,
                                                (int32_t)ntiles, tile_counts, err);
  if (std::min<int64_t>(tw, ntiles) < 4 * kColWarps) {
    dim3 g2((unsigned)((nblk + 255) / 256), (unsigned)bgcount);
    csr_colscan_small_kernel<<<g2, 256, 0, st>>>(tile_counts, totals, (int32_t)nblk,
                                                 (int32_t)ntiles, tw, (int32_t)nwin);
  } else {
    dim3 g2((unsigned)((nblk + 31) / 32), (unsigned)(bgcount * nwin));
    csr_colscan_kernel<<<g2, kColWarps * 32, 0, st>>>(tile_counts, totals, (int32_t)nblk,
                                                      (int32_t)ntiles, tw, (int32_t)nwin);
  }
  const int64_t nseg = bgcount * nwin * nblk;
  const int64_t nchunks = (nseg + kScanChunk - 1) / kScanChunk;
  int32_t* chunk_sums = totals + nseg;
  csr_chunk_sums_kernel<<<(unsigned)nchunks, kScanThreads, 0, st>>>(totals, nseg, chunk_sums);
  csr_chunk_scan_kernel<<<1, kScanThreads, 0, st>>>(chunk_sums, nchunks, nseg, offsets);
  csr_chunk_apply_kernel<<<(unsigned)nchunks, kScanThreads, 0, st>>>(totals, nseg, chunk_sums,
                                                                     offsets);
  csr_scatter_kernel<<<g1, 32, hist_bytes, st>>>(sel, n_q, q_pos0, (int32_t)nblk,
                                                 (int32_t)ntiles, tw, (int32_t)nwin,
                                                 tile_counts, offsets, entries, entry_pos,
                                                 cap);
  return cudaGetLastError();
}

}  // namespace msa
