/*
 * msa_oracle.c -- plain, slow, double-precision CPU definition of the
 * MiniMax Sparse Attention (MSA) hot path.  TEST INFRASTRUCTURE ONLY: the
 * tests, the smoke check and the CPU baseline of the benchmark call it; the
 * product path never does.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * Sources (page title, section):
 *  [P1] "MSA 稀疏注意力三国杀：NSA / DSA / MoBA / MSA 四方案深度对比",
 *       section "MSA 架构：粗筛 + 精算" (index branch: 128-token blocks, one
 *       score per token, block score = max over the block, 16 blocks with the
 *       query's own block always taken; main branch: full attention over the
 *       16 x 128 = 2048 selected tokens).
 *  [P3] "稀疏注意力速览（Sparse Attention，2019 ~ 2026）", section 4 (block
 *       级选择派), entry "MiniMax Sparse Attention（MSA）"
 *       (per GQA group one index query head and a shared index key head,
 *       block max-pool, per-group top-k with the local block kept, exact
 *       softmax attention on the selected blocks).
 *  [P5] "稀疏注意力架构革命：2026年长上下文大模型核心技术解析", section 1.1
 *       (标准Transformer Attention的O(n²)困境), formula
 *       softmax(Q K^T / sqrt(d_k)) V.
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes as well):
 *  - index score of (query t, key j) for group g is the raw dot product
 *    q_idx[t,g,:] . k_idx[j,:] (no scale, bias or activation);
 *  - a block's score is taken only over keys j <= t; blocks c < own(t) are
 *    whole, so only the own block would be cut, and it is forced anyway;
 *  - "16 blocks" counts the forced own block: own + 15 best candidates;
 *  - ranking is by score descending, ties to the lower block index, with
 *    -0.0 equal to +0.0 (C comparison of doubles already does this);
 *  - the attention scale is the caller's (1/sqrt(128) by default);
 *  - head h belongs to group h / (H / G).
 *
 * Every input array is contiguous in the layout stated beside it; bf16
 * values are passed as their raw uint16 bit patterns.  All arithmetic is
 * double precision; a bf16 value converts to double exactly, and so does a
 * product of two of them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MSA_BLOCK 128  /* B_k: tokens per KV block ([P1], [P3]) */
#define MSA_TOPK 16    /* blocks per query and group, own block included */
#define MSA_HEAD_DIM 128

static double bf16_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ---------------------------------------------------------------------- */
/* Step 1-2: token scores and block max-pooling ([P1] steps 1-2, [P3]).   */
/*                                                                        */
/* For each row r (absolute position t = row_pos[r], batch row_batch[r])  */
/* and group g: pooled[r,g,c] = max over keys j in block c of             */
/*   sum_k q_idx_rows[r,g,k] * k_idx[b, hk(g), j, k]                      */
/* for every block c < own(t) = t / 128.  Entries c >= own(t) are NaN.    */
/* hk(g) = 0 when h_kidx == 1 (shared index key head), else g.            */
/* ---------------------------------------------------------------------- */
void msa_oracle_index_pooled(int64_t n_rows, int32_t G, int32_t d_idx,
                             int64_t n_kv, int32_t h_kidx,
                             const uint16_t* q_idx_rows, /* [n_rows,G,d_idx] */
                             const int64_t* row_pos, const int64_t* row_batch,
                             const uint16_t* k_idx, /* [B',h_kidx,n_kv,d_idx] */
                             int64_t out_stride,    /* >= number of blocks */
                             double* pooled)        /* [n_rows,G,out_stride] */
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int32_t g = 0; g < G; ++g) {
      const int64_t t = row_pos[r];
      const int64_t own = t / MSA_BLOCK;
      const int32_t hk = (h_kidx == 1) ? 0 : g;
      const uint16_t* qv = q_idx_rows + (r * G + g) * (int64_t)d_idx;
      const uint16_t* kb =
          k_idx + ((row_batch[r] * h_kidx + hk) * n_kv) * (int64_t)d_idx;
      double* out = pooled + (r * G + g) * out_stride;
      double qd[256];
      for (int32_t k = 0; k < d_idx; ++k) qd[k] = bf16_to_f64(qv[k]);
      for (int64_t c = 0; c < out_stride; ++c) out[c] = NAN;
      for (int64_t c = 0; c < own; ++c) {
        double best = -INFINITY;
        for (int64_t j = c * MSA_BLOCK; j < (c + 1) * MSA_BLOCK; ++j) {
          const uint16_t* kv = kb + j * (int64_t)d_idx;
          double s = 0.0;
          for (int32_t k = 0; k < d_idx; ++k) s += qd[k] * bf16_to_f64(kv[k]);
          if (s > best) best = s;
        }
        out[c] = best;
      }
    }
  }
}

/* ---------------------------------------------------------------------- */
/* Step 3: block selection ([P1] step 3; [P3] per-group top-k with the    */
/* local block kept).  nsel = min(16, own+1).  The own block is always    */
/* in; the other nsel-1 are the best candidates c < own ranked by         */
/* (score descending, block index ascending).  Output is the selected     */
/* block ids in ascending order, padded with -1 to 16.                    */
/* ---------------------------------------------------------------------- */
typedef struct {
  double score;
  int32_t idx;
} cand_t;

static int cand_cmp(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int int_cmp(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

void msa_oracle_select_row(int64_t own, const double* scores, int32_t* sel) {
  int32_t out[MSA_TOPK];
  int32_t n = 0;
  if (own + 1 <= MSA_TOPK) {
    for (int32_t c = 0; c <= own; ++c) out[n++] = c;
  } else {
    cand_t* cands = (cand_t*)malloc(sizeof(cand_t) * (size_t)own);
    for (int64_t c = 0; c < own; ++c) {
      cands[c].score = scores[c];
      cands[c].idx = (int32_t)c;
    }
    qsort(cands, (size_t)own, sizeof(cand_t), cand_cmp);
    for (int32_t i = 0; i < MSA_TOPK - 1; ++i) out[n++] = cands[i].idx;
    out[n++] = (int32_t)own;
    free(cands);
    qsort(out, (size_t)n, sizeof(int32_t), int_cmp);
  }
  for (int32_t i = 0; i < MSA_TOPK; ++i) sel[i] = (i < n) ? out[i] : -1;
}

void msa_oracle_topk(int64_t n_rows, int32_t G, const int64_t* row_pos,
                     int64_t stride, const double* pooled, /* [n_rows,G,stride] */
                     int32_t* sel)                          /* [n_rows,G,16] */
{
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t r = 0; r < n_rows; ++r)
    for (int32_t g = 0; g < G; ++g)
      msa_oracle_select_row(row_pos[r] / MSA_BLOCK,
                            pooled + (r * G + g) * stride,
                            sel + (r * G + g) * MSA_TOPK);
}

/* Same selection on fp32 scores (the scores a caller hands to the select
 * step), so that a float-valued input is ranked exactly as given. */
void msa_oracle_topk_f32(int64_t n_rows, int64_t stride, const int64_t* own,
                         const float* pooled, int32_t* sel) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    double* tmp = (double*)malloc(sizeof(double) * (size_t)(own[r] + 1));
    for (int64_t c = 0; c < own[r]; ++c) tmp[c] = (double)pooled[r * stride + c];
    msa_oracle_select_row(own[r], tmp, sel + r * MSA_TOPK);
    free(tmp);
  }
}

/* ---------------------------------------------------------------------- */
/* Step 4: exact softmax attention over the selected tokens ([P1] main     */
/* branch, [P3] "exact softmax attention", [P5] softmax(QK^T/sqrt(d))V).   */
/* For row r, head h (group g = h / (H/G), KV head g): the token set is    */
/* the union of the selected blocks, restricted to j <= t.                 */
/*   o = sum_j p_j v_j,  p_j = exp(s_j - m) / l,  s_j = scale * q.k_j,     */
/*   m = max_j s_j, l = sum_j exp(s_j - m), lse = m + log(l).              */
/* ---------------------------------------------------------------------- */
void msa_oracle_attention(int64_t n_rows, int32_t H, int32_t G, int64_t n_kv,
                          const uint16_t* q_rows,   /* [n_rows,H,128] */
                          const int64_t* row_pos, const int64_t* row_batch,
                          const uint16_t* k, const uint16_t* v, /* [B',G,n_kv,128] */
                          const int32_t* sel,        /* [n_rows,G,16] */
                          double scale,
                          double* out,               /* [n_rows,H,128] */
                          double* lse)               /* [n_rows,H] */
{
  const int32_t R = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int32_t h = 0; h < H; ++h) {
      const int64_t t = row_pos[r];
      const int32_t g = h / R;
      const int32_t* srow = sel + (r * G + g) * MSA_TOPK;
      const uint16_t* qh = q_rows + (r * H + h) * (int64_t)MSA_HEAD_DIM;
      const int64_t kvbase = (row_batch[r] * G + g) * n_kv;
      double qd[MSA_HEAD_DIM];
      for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) qd[d] = bf16_to_f64(qh[d]);

      /* logits of every selected causal token */
      double logit[MSA_TOPK * MSA_BLOCK];
      int64_t tok[MSA_TOPK * MSA_BLOCK];
      int32_t n = 0;
      for (int32_t s = 0; s < MSA_TOPK; ++s) {
        const int32_t c = srow[s];
        if (c < 0) continue;
        for (int64_t j = (int64_t)c * MSA_BLOCK; j < (int64_t)(c + 1) * MSA_BLOCK; ++j) {
          if (j > t || j >= n_kv) break;
          const uint16_t* kj = k + (kvbase + j) * MSA_HEAD_DIM;
          double dot = 0.0;
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dot += qd[d] * bf16_to_f64(kj[d]);
          logit[n] = scale * dot;
          tok[n] = j;
          ++n;
        }
      }
      double m = -INFINITY;
      for (int32_t i = 0; i < n; ++i) if (logit[i] > m) m = logit[i];
      double l = 0.0;
      double o[MSA_HEAD_DIM];
      for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) o[d] = 0.0;
      for (int32_t i = 0; i < n; ++i) {
        const double p = exp(logit[i] - m);
        l += p;
        const uint16_t* vj = v + (kvbase + tok[i]) * MSA_HEAD_DIM;
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) o[d] += p * bf16_to_f64(vj[d]);
      }
      double* orow = out + (r * H + h) * (int64_t)MSA_HEAD_DIM;
      for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) orow[d] = o[d] / l;
      lse[r * H + h] = m + log(l);
    }
  }
}

/* ---------------------------------------------------------------------- */
/* Combination of per-block softmax pieces.  A piece s of one (query,      */
/* head) carries m_s (max logit of its tokens), l_s = sum exp(s_j - m_s)   */
/* and acc_s = sum exp(s_j - m_s) v_j.  Softmax over the union of the      */
/* pieces' tokens is                                                       */
/*   M = max_s m_s, L = sum_s l_s e^{m_s-M}, o = sum_s acc_s e^{m_s-M} / L, */
/*   lse = M + log L.                                                      */
/* Pieces with valid[s] == 0 are ignored.                                  */
/* ---------------------------------------------------------------------- */
void msa_oracle_merge(int64_t n, int32_t nslot, int32_t dim,
                      const int32_t* valid, /* [n,nslot] */
                      const double* m, const double* l, /* [n,nslot] */
                      const double* acc,                /* [n,nslot,dim] */
                      double* out, double* lse)         /* [n,dim], [n] */
{
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double M = -INFINITY;
    for (int32_t s = 0; s < nslot; ++s)
      if (valid[i * nslot + s] && m[i * nslot + s] > M) M = m[i * nslot + s];
    double L = 0.0;
    for (int32_t d = 0; d < dim; ++d) out[i * dim + d] = 0.0;
    for (int32_t s = 0; s < nslot; ++s) {
      if (!valid[i * nslot + s]) continue;
      const double w = exp(m[i * nslot + s] - M);
      L += w * l[i * nslot + s];
      for (int32_t d = 0; d < dim; ++d)
        out[i * dim + d] += w * acc[(i * nslot + s) * dim + d];
    }
    for (int32_t d = 0; d < dim; ++d) out[i * dim + d] /= L;
    lse[i] = M + log(L);
  }
}

/* ---------------------------------------------------------------------- */
/* Inversion of the query -> block lists into block -> query lists, the    */
/* data structure a KV-block-outer kernel walks ([P1] "Outer Gather Q":    */
/* all queries that chose a block are gathered and computed together).    */
/* The query range is cut into windows of `window` consecutive query       */
/* indices (window w holds q in [w*window, (w+1)*window)); segments are    */
/* ordered by (batch, group, window, block), and inside a segment the      */
/* entries are (q << 4) | slot with q ascending.  offsets has              */
/* B*G*nwin*nblk + 1 entries, nwin = ceil(n_q / window); offsets[seg] ..   */
/* offsets[seg+1] bound segment seg.                                       */
/* ---------------------------------------------------------------------- */
void msa_oracle_block_query_lists(int64_t B, int32_t G, int64_t n_q, int64_t nblk,
                                  int64_t window,
                                  const int32_t* sel, /* [B,G,n_q,16] */
                                  int64_t* offsets,   /* [B*G*nwin*nblk+1] */
                                  int32_t* entries)
{
  const int64_t nwin = (n_q + window - 1) / window;
  const int64_t nseg = B * G * nwin * nblk;
  int64_t* cursor = (int64_t*)calloc((size_t)nseg, sizeof(int64_t));
  for (int64_t i = 0; i <= nseg; ++i) offsets[i] = 0;
  for (int64_t bg = 0; bg < B * G; ++bg)
    for (int64_t q = 0; q < n_q; ++q)
      for (int32_t s = 0; s < MSA_TOPK; ++s) {
        const int32_t c = sel[(bg * n_q + q) * MSA_TOPK + s];
        if (c >= 0) offsets[(bg * nwin + q / window) * nblk + c + 1] += 1;
      }
  for (int64_t i = 0; i < nseg; ++i) offsets[i + 1] += offsets[i];
  for (int64_t i = 0; i < nseg; ++i) cursor[i] = offsets[i];
  for (int64_t bg = 0; bg < B * G; ++bg)
    for (int64_t q = 0; q < n_q; ++q)
      for (int32_t s = 0; s < MSA_TOPK; ++s) {
        const int32_t c = sel[(bg * n_q + q) * MSA_TOPK + s];
        if (c < 0) continue;
        entries[cursor[(bg * nwin + q / window) * nblk + c]++] = (int32_t)((q << 4) | s);
      }
  free(cursor);
}

/* ---------------------------------------------------------------------- */
/* Selection recall and the index branch's alignment target ([P1] section */
/* "索引分支训练：KL 对齐": the index branch learns from the main branch's   */
/* attention distribution through a KL divergence with the teacher's      */
/* gradient stopped, and its chosen blocks are reported to hold over 90 % */
/* of the main branch's attention weight; [P3] MSA entry: a KL loss       */
/* aligns the index distribution to the main branch's probabilities).     */
/* For row r (position t, own = t / 128) and group g, over blocks         */
/* c = 0 .. own and keys j <= t:                                          */
/*   teacher P(c) = (1/R) sum_{h in g} sum_{j in c} softmax_h(j), with    */
/*                  softmax_h over all keys j <= t of scale * q_h . k_j   */
/*   student Q(c) = softmax over c of z(c), z(c) = max_{j in c} of the    */
/*                  index score q_idx[g] . k_idx[j] (own block: j <= t)   */
/*   recall = sum of P(c) over the selected blocks                        */
/*   kl_pq = sum_c P(c) log(P(c) / Q(c)), kl_qp = sum_c Q(c) log(Q(c)/P(c)) */
/* block_mass[r,g,c] = P(c) for c <= own and 0 for own < c < stride.      */
/* The teacher of a group is the mean over its R heads (the group shares  */
/* one selection); the index logits are unscaled, as in step 1.           */
/* ---------------------------------------------------------------------- */
void msa_oracle_selection_recall(int64_t n_rows, int32_t H, int32_t G, int32_t d_idx,
                                 int64_t n_kv, int32_t h_kidx,
                                 const uint16_t* q_rows,     /* [n_rows,H,128] */
                                 const uint16_t* q_idx_rows, /* [n_rows,G,d_idx] */
                                 const int64_t* row_pos, const int64_t* row_batch,
                                 const uint16_t* k,          /* [B',G,n_kv,128] */
                                 const uint16_t* k_idx,      /* [B',h_kidx,n_kv,d_idx] */
                                 const int32_t* sel,         /* [n_rows,G,16] */
                                 double scale, int64_t stride,
                                 double* block_mass,         /* [n_rows,G,stride] */
                                 double* recall, double* kl_pq, double* kl_qp) /* [n_rows,G] */
{
  const int32_t R = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int32_t g = 0; g < G; ++g) {
      const int64_t t = row_pos[r];
      const int64_t own = t / MSA_BLOCK;
      const int64_t nb = own + 1;
      const int64_t kvbase = (row_batch[r] * G + g) * n_kv;
      const int64_t kibase = (row_batch[r] * h_kidx + (h_kidx == 1 ? 0 : g)) * n_kv;
      double* P = block_mass + (r * G + g) * stride;
      double* z = (double*)malloc((size_t)nb * sizeof(double));
      double* logit = (double*)malloc((size_t)(t + 1) * sizeof(double));
      for (int64_t c = 0; c < stride; ++c) P[c] = 0.0;
      /* teacher: each head's softmax over every key j <= t, summed per block */
      for (int32_t hr = 0; hr < R; ++hr) {
        const uint16_t* qh = q_rows + (r * H + g * R + hr) * (int64_t)MSA_HEAD_DIM;
        double qd[MSA_HEAD_DIM];
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) qd[d] = bf16_to_f64(qh[d]);
        double m = -INFINITY;
        for (int64_t j = 0; j <= t; ++j) {
          const uint16_t* kj = k + (kvbase + j) * MSA_HEAD_DIM;
          double dot = 0.0;
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dot += qd[d] * bf16_to_f64(kj[d]);
          logit[j] = scale * dot;
          if (logit[j] > m) m = logit[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j <= t; ++j) l += exp(logit[j] - m);
        for (int64_t j = 0; j <= t; ++j) P[j / MSA_BLOCK] += exp(logit[j] - m) / l / R;
      }
      /* student: softmax of the block-max index scores */
      const uint16_t* qi = q_idx_rows + (r * G + g) * (int64_t)d_idx;
      double zmax = -INFINITY;
      for (int64_t c = 0; c < nb; ++c) {
        double best = -INFINITY;
        for (int64_t j = c * MSA_BLOCK; j < (c + 1) * MSA_BLOCK && j <= t; ++j) {
          const uint16_t* kj = k_idx + (kibase + j) * d_idx;
          double dot = 0.0;
          for (int32_t d = 0; d < d_idx; ++d) dot += bf16_to_f64(qi[d]) * bf16_to_f64(kj[d]);
          if (dot > best) best = dot;
        }
        z[c] = best;
        if (best > zmax) zmax = best;
      }
      double zs = 0.0;
      for (int64_t c = 0; c < nb; ++c) zs += exp(z[c] - zmax);
      double kpq = 0.0, kqp = 0.0;
      for (int64_t c = 0; c < nb; ++c) {
        const double logq = z[c] - zmax - log(zs);
        const double q = exp(logq);
        if (P[c] > 0.0) kpq += P[c] * (log(P[c]) - logq);
        if (q > 0.0) kqp += q * (logq - log(P[c]));
      }
      double rc = 0.0;
      const int32_t* srow = sel + (r * G + g) * MSA_TOPK;
      for (int32_t s = 0; s < MSA_TOPK; ++s)
        if (srow[s] >= 0 && srow[s] <= own) rc += P[srow[s]];
      recall[r * G + g] = rc;
      kl_pq[r * G + g] = kpq;
      kl_qp[r * G + g] = kqp;
      free(z);
      free(logit);
    }
  }
}

/* ---------------------------------------------------------------------- */
/* FP8 (e4m3) index branch: the next scoped variant of steps 1-2, the     */
/* index scores computed from 8-bit copies of q_idx and k_idx.            */
/* e4m3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is   */
/* subnormal (2^-6 * m / 8); exponent 15 with mantissa 7 is NaN; there is */
/* no infinity, the largest finite magnitude is 448.                      */
/* Quantisation of a tensor x: amax = max |x|, scale = amax / 448 (fp32,  */
/* 1 when amax is 0), code(x) = e4m3 nearest to x / scale (fp32 division),*/
/* ties to the even code, magnitudes past 448 saturate to 448.            */
/* ---------------------------------------------------------------------- */
double msa_oracle_e4m3_value(uint8_t code) {
  const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -mag : mag;
}

static uint8_t e4m3_nearest(float y) {
  /* brute force over the 127 finite non-negative codes 0x00 .. 0x7E */
  const double a = fabs((double)y);
  uint8_t best = 0;
  double bd = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    const double d = fabs(msa_oracle_e4m3_value((uint8_t)c) - a);
    if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
      bd = d;
      best = (uint8_t)c;
    }
  }
  if (a >= 448.0) best = 0x7E;
  return (uint8_t)(best | (signbit(y) ? 0x80 : 0));   /* the sign survives rounding to zero */
}

void msa_oracle_quantize_e4m3(int64_t n, const uint16_t* x_bf16, float* scale_out,
                              uint8_t* codes) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    const float v = fabsf((float)bf16_to_f64(x_bf16[i]));
    if (v > amax) amax = v;
  }
  const float scale = (amax > 0.0f) ? amax / 448.0f : 1.0f;
  *scale_out = scale;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) codes[i] = e4m3_nearest((float)bf16_to_f64(x_bf16[i]) / scale);
}

/* Steps 1-2 on the codes: pooled[r,g,c] = s_q s_k max over keys j of block c */
/* of sum_k value(q_codes[r,g,k]) value(k_codes[b,hk(g),j,k]), c < own(t).   */
void msa_oracle_index_pooled_e4m3(int64_t n_rows, int32_t G, int32_t d_idx, int64_t n_kv,
                                  int32_t h_kidx,
                                  const uint8_t* q_codes,   /* [n_rows,G,d_idx] */
                                  const int64_t* row_pos, const int64_t* row_batch,
                                  const uint8_t* k_codes,   /* [B',h_kidx,n_kv,d_idx] */
                                  double s_q, double s_k, int64_t stride,
                                  double* out)              /* [n_rows,G,stride] */
{
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int32_t g = 0; g < G; ++g) {
      const int64_t own = row_pos[r] / MSA_BLOCK;
      const uint8_t* qr = q_codes + (r * G + g) * (int64_t)d_idx;
      const int64_t kb = (row_batch[r] * h_kidx + (h_kidx == 1 ? 0 : g)) * n_kv;
      double* o = out + (r * G + g) * stride;
      for (int64_t c = 0; c < stride; ++c) o[c] = NAN;
      for (int64_t c = 0; c < own; ++c) {
        double best = -INFINITY;
        for (int64_t j = c * MSA_BLOCK; j < (c + 1) * MSA_BLOCK && j < n_kv; ++j) {
          const uint8_t* kr = k_codes + (kb + j) * d_idx;
          double dot = 0.0;
          for (int32_t d = 0; d < d_idx; ++d)
            dot += msa_oracle_e4m3_value(qr[d]) * msa_oracle_e4m3_value(kr[d]);
          if (dot > best) best = dot;
        }
        o[c] = s_q * s_k * best;
      }
    }
  }
}

/* ---------------------------------------------------------------------- */
/* Token-level selection at the same budget: the top min(2048, t+1) keys  */
/* j <= t by index score q_idx[g] . k_idx[j] (score descending, lower      */
/* index first), the granularity the other selection-based method of the  */
/* pages (DSA) uses ([P1] section "分歧一：颗粒度——token 级还是块级？";   */
/* [P3] section 4; [P4] "Sparse attention · DSA và MSA chọn vị trí").      */
/* Exact softmax attention                                                */
/* over the chosen tokens, per head of the group, with its lse; and the   */
/* full causal attention's lse for the same heads.                        */
/* ---------------------------------------------------------------------- */
typedef struct { double s; int64_t j; } tok_t;

static int tok_cmp(const void* pa, const void* pb) {
  const tok_t* a = (const tok_t*)pa;
  const tok_t* b = (const tok_t*)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->j < b->j) ? -1 : (a->j > b->j);
}

static int i64_cmp(const void* pa, const void* pb) {
  const int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
  return (a > b) - (a < b);
}

void msa_oracle_token_select_attention(int64_t n_rows, int32_t H, int32_t G, int32_t d_idx,
                                       int64_t n_kv, int32_t h_kidx, int64_t budget,
                                       const uint16_t* q_rows,     /* [n_rows,H,128] */
                                       const uint16_t* q_idx_rows, /* [n_rows,G,d_idx] */
                                       const int64_t* row_pos, const int64_t* row_batch,
                                       const uint16_t* k, const uint16_t* v, /* [B',G,n_kv,128] */
                                       const uint16_t* k_idx,      /* [B',h_kidx,n_kv,d_idx] */
                                       double scale,
                                       int64_t* tokens,            /* [n_rows,G,budget], -1 pad */
                                       double* out,                /* [n_rows,H,128] */
                                       double* lse,                /* [n_rows,H] */
                                       double* lse_full)           /* [n_rows,H] */
{
  const int32_t R = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int32_t g = 0; g < G; ++g) {
      const int64_t t = row_pos[r];
      const int64_t kvbase = (row_batch[r] * G + g) * n_kv;
      const int64_t kibase = (row_batch[r] * h_kidx + (h_kidx == 1 ? 0 : g)) * n_kv;
      const uint16_t* qi = q_idx_rows + (r * G + g) * (int64_t)d_idx;
      tok_t* sc = (tok_t*)malloc((size_t)(t + 1) * sizeof(tok_t));
      for (int64_t j = 0; j <= t; ++j) {
        const uint16_t* kj = k_idx + (kibase + j) * d_idx;
        double dot = 0.0;
        for (int32_t d = 0; d < d_idx; ++d) dot += bf16_to_f64(qi[d]) * bf16_to_f64(kj[d]);
        sc[j].s = dot;
        sc[j].j = j;
      }
      qsort(sc, (size_t)(t + 1), sizeof(tok_t), tok_cmp);
      const int64_t m = (t + 1 < budget) ? t + 1 : budget;
      int64_t* tk = tokens + (r * G + g) * budget;
      for (int64_t i = 0; i < m; ++i) tk[i] = sc[i].j;
      qsort(tk, (size_t)m, sizeof(int64_t), i64_cmp);
      for (int64_t i = m; i < budget; ++i) tk[i] = -1;
      free(sc);
      for (int32_t hr = 0; hr < R; ++hr) {
        const int32_t h = g * R + hr;
        const uint16_t* qh = q_rows + (r * H + h) * (int64_t)MSA_HEAD_DIM;
        double qd[MSA_HEAD_DIM];
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) qd[d] = bf16_to_f64(qh[d]);
        double* logit = (double*)malloc((size_t)(t + 1) * sizeof(double));
        double mf = -INFINITY;
        for (int64_t j = 0; j <= t; ++j) {
          const uint16_t* kj = k + (kvbase + j) * MSA_HEAD_DIM;
          double dot = 0.0;
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dot += qd[d] * bf16_to_f64(kj[d]);
          logit[j] = scale * dot;
          if (logit[j] > mf) mf = logit[j];
        }
        double lf = 0.0;
        for (int64_t j = 0; j <= t; ++j) lf += exp(logit[j] - mf);
        lse_full[r * H + h] = mf + log(lf);
        double ms = -INFINITY;
        for (int64_t i = 0; i < m; ++i) if (logit[tk[i]] > ms) ms = logit[tk[i]];
        double ls = 0.0, o[MSA_HEAD_DIM];
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) o[d] = 0.0;
        for (int64_t i = 0; i < m; ++i) {
          const double p = exp(logit[tk[i]] - ms);
          ls += p;
          const uint16_t* vj = v + (kvbase + tk[i]) * MSA_HEAD_DIM;
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) o[d] += p * bf16_to_f64(vj[d]);
        }
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) out[(r * H + h) * (int64_t)MSA_HEAD_DIM + d] = o[d] / ls;
        lse[r * H + h] = ms + log(ls);
        free(logit);
      }
    }
  }
}

/* ---------------------------------------------------------------------- */
/* Backward of step 4 for sparse training ([P1] section "MSA 能力不掉：3T    */
/* token 对照实验": a model trained with MSA from the start (MSA-PT) and a   */
/* dense model converted by continued training (MSA-CPT), both of which    */
/* back-propagate through the main branch; [P1] section "索引分支训练：KL    */
/* 对齐": the index branch learns only through its own KL term, so the top-k */
/* selection is a fixed input here and carries no gradient).               */
/*                                                                        */
/* The gradients of o = sum_j p_j v_j, p = softmax_j(scale q.k_j) over the  */
/* selected causal tokens J(t, g) of the forward, for an upstream dO:      */
/*   dP_j = dO.v_j,  D = sum_j p_j dP_j (= dO.o),  dS_j = p_j (dP_j - D),   */
/*   dQ = scale sum_j dS_j k_j,  dK_j += scale dS_j q,  dV_j += p_j dO,     */
/* summed over every (query, head) whose token set holds j.                */
/* Inputs are doubles so that the finite-difference pins can perturb them; */
/* bf16 callers convert exactly.  All arrays contiguous:                   */
/*   q, dout, dq [B, n_q, H, 128];  k, v, dk, dv [B, G, n_kv, 128];         */
/*   sel [B, G, n_q, 16] (-1 = unused slot); query i sits at t = q_pos0+i. */
/* Two passes, each over independent units: (1) per (batch, query, head):  */
/* lse, D and dQ; (2) per (batch, group, KV block c): dK and dV of c's     */
/* tokens, summed over the queries that selected c in ascending order and  */
/* over the group's heads.                                                 */
/* ---------------------------------------------------------------------- */
static int32_t bwd_tokens(const int32_t* srow, int64_t t, int64_t n_kv, int64_t* tok) {
  int32_t n = 0;
  for (int32_t s = 0; s < MSA_TOPK; ++s) {
    const int32_t c = srow[s];
    if (c < 0) continue;
    for (int64_t j = (int64_t)c * MSA_BLOCK; j < (int64_t)(c + 1) * MSA_BLOCK; ++j) {
      if (j > t || j >= n_kv) break;
      tok[n++] = j;
    }
  }
  return n;
}

static double dot128(const double* a, const double* b) {
  double s = 0.0;
  for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) s += a[d] * b[d];
  return s;
}

void msa_oracle_attention_bwd(int64_t B, int64_t n_q, int64_t n_kv, int64_t q_pos0, int32_t H,
                              int32_t G, const double* q, const double* k, const double* v,
                              const double* dout, const int32_t* sel, double scale,
                              double* dq, double* dk, double* dv,
                              double* lse_out, double* delta_out) /* [B, n_q, H] each */
{
  const int32_t R = H / G;
  const int64_t nblk = (n_kv + MSA_BLOCK - 1) / MSA_BLOCK;
  /* pass 1: per (b, i, h) */
#pragma omp parallel for collapse(3) schedule(dynamic, 16)
  for (int64_t b = 0; b < B; ++b) {
    for (int64_t i = 0; i < n_q; ++i) {
      for (int32_t h = 0; h < H; ++h) {
        const int64_t t = q_pos0 + i;
        const int32_t g = h / R;
        const int64_t row = (b * n_q + i) * H + h;
        const double* qh = q + row * MSA_HEAD_DIM;
        const double* doh = dout + row * MSA_HEAD_DIM;
        const double* kb = k + (b * G + g) * n_kv * MSA_HEAD_DIM;
        const double* vb = v + (b * G + g) * n_kv * MSA_HEAD_DIM;
        int64_t tok[MSA_TOPK * MSA_BLOCK];
        double s[MSA_TOPK * MSA_BLOCK], p[MSA_TOPK * MSA_BLOCK], dp[MSA_TOPK * MSA_BLOCK];
        const int32_t n = bwd_tokens(sel + ((b * G + g) * n_q + i) * MSA_TOPK, t, n_kv, tok);
        double m = -INFINITY;
        for (int32_t a = 0; a < n; ++a) {
          s[a] = scale * dot128(qh, kb + tok[a] * MSA_HEAD_DIM);
          if (s[a] > m) m = s[a];
        }
        double l = 0.0;
        for (int32_t a = 0; a < n; ++a) l += exp(s[a] - m);
        const double lse = m + log(l);
        double D = 0.0;
        for (int32_t a = 0; a < n; ++a) {
          p[a] = exp(s[a] - lse);
          dp[a] = dot128(doh, vb + tok[a] * MSA_HEAD_DIM);
          D += p[a] * dp[a];
        }
        double* dqh = dq + row * MSA_HEAD_DIM;
        for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dqh[d] = 0.0;
        for (int32_t a = 0; a < n; ++a) {
          const double ds = p[a] * (dp[a] - D);
          const double* kj = kb + tok[a] * MSA_HEAD_DIM;
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dqh[d] += scale * ds * kj[d];
        }
        lse_out[row] = lse;
        delta_out[row] = D;
      }
    }
  }
  /* pass 2: per (b, g, c) */
#pragma omp parallel for collapse(3) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b) {
    for (int32_t g = 0; g < G; ++g) {
      for (int64_t c = 0; c < nblk; ++c) {
        const int64_t j0 = c * MSA_BLOCK;
        const int64_t j1 = (j0 + MSA_BLOCK < n_kv) ? j0 + MSA_BLOCK : n_kv;
        const double* kb = k + (b * G + g) * n_kv * MSA_HEAD_DIM;
        const double* vb = v + (b * G + g) * n_kv * MSA_HEAD_DIM;
        double* dkb = dk + (b * G + g) * n_kv * MSA_HEAD_DIM;
        double* dvb = dv + (b * G + g) * n_kv * MSA_HEAD_DIM;
        for (int64_t j = j0; j < j1; ++j)
          for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) dkb[j * MSA_HEAD_DIM + d] = dvb[j * MSA_HEAD_DIM + d] = 0.0;
        for (int64_t i = 0; i < n_q; ++i) {
          const int64_t t = q_pos0 + i;
          const int32_t* srow = sel + ((b * G + g) * n_q + i) * MSA_TOPK;
          int chosen = 0;
          for (int32_t s2 = 0; s2 < MSA_TOPK; ++s2) chosen |= (srow[s2] == (int32_t)c);
          if (!chosen || j0 > t) continue;
          for (int32_t r = 0; r < R; ++r) {
            const int64_t row = (b * n_q + i) * H + g * R + r;
            const double* qh = q + row * MSA_HEAD_DIM;
            const double* doh = dout + row * MSA_HEAD_DIM;
            for (int64_t j = j0; j < j1 && j <= t; ++j) {
              const double pj = exp(scale * dot128(qh, kb + j * MSA_HEAD_DIM) - lse_out[row]);
              const double ds = pj * (dot128(doh, vb + j * MSA_HEAD_DIM) - delta_out[row]);
              for (int32_t d = 0; d < MSA_HEAD_DIM; ++d) {
                dkb[j * MSA_HEAD_DIM + d] += scale * ds * qh[d];
                dvb[j * MSA_HEAD_DIM + d] += pj * doh[d];
              }
            }
          }
        }
      }
    }
  }
}
