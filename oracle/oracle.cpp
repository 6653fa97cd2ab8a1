// Oracle for the fused attention path: a plain, slow, fp64 CPU implementation.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or calls this
// file; only the test suite, the smoke check and the benchmark's CPU-baseline leg load it.
// It shares no code, header or constant with the CUDA path.
//
// What it computes, with the passage each part follows:
//
//  * Attention(Q,K,V) = softmax(Q K^T * scale) V  -- "FlashAttention on Ascend NPUs",
//    section on why attention is memory hungry (the formula softmax(QK^T/sqrt(d_k))V).
//    `oracle_attn_*_rows` evaluate exactly that definition one output row at a time:
//    scores of the allowed keys, their maximum, the exp-sum, the weighted sum of V rows.
//  * The naive multi-pass form that stores the whole S x S score matrix -- "Flash
//    Attention on Ascend: three techniques", section on the memory traffic of standard
//    attention (scores = QK^T, scale, softmax, probs @ V, each pass through memory).
//    `oracle_attn_brute` materialises every score matrix and the probability matrix.
//  * Tiled evaluation with an online softmax -- same page, sections "tiling" (Q blocks in the
//    outer loop, K/V blocks in the inner loop) and "online softmax" (keep only the running
//    maximum and running exp-sum; correct earlier partial results when the maximum grows);
//    "FlashAttention on Ascend NPUs", tiling section (local max and sum, corrected at the
//    end).  `oracle_attn_tiled` follows those steps with a settable block size.
//  * MHA/GQA/MQA head mapping -- "FlashAttention variants: GQA, MQA, sparse attention",
//    section on expanding KV: K and V are repeated along the head axis with
//    repeat_interleave(Hq/Hkv), so query head h reads KV head floor(h / (Hq/Hkv)).
//  * Causal and sliding-window masks -- same page, sliding-window section: each token sees
//    the nearest W tokens, itself included (the prose and the N*W connection count); the
//    causal mask is aligned to the bottom-right corner when Sq != Skv (the pages are
//    silent; this is the reading this project takes).  A row with no allowed key returns
//    O = 0 and LSE = -inf.
//  * INT8 KV cache used without decompressing it first -- "Flash Attention on Ascend: three
//    techniques", KV compression section.  The decode oracle evaluates attention over the
//    dequantised values k_code * k_scale (exact in fp64), one query token per sequence.
//    With num_splits > 1 it evaluates each key chunk separately and merges the partial
//    results through their log-sum-exp, the same correction step the online softmax uses.
//  * The backward pass -- "FlashAttention on Ascend NPUs", recomputation section: the attention
//    matrix is not stored; the backward pass recomputes it.  `oracle_attn_bwd` differentiates
//    L = sum(dO * O) through the definition for one (b, h) at a time with the probabilities of
//    the visible keys written out: D_i = sum_t dO_it O_it, dV_j = sum_i P_ij dO_i,
//    dP_ij = dO_i . v_j, dS_ij = P_ij (dP_ij - D_i), dQ_i = scale sum_j dS_ij k_j,
//    dK_j = scale sum_i dS_ij q_i; GQA sums dK, dV over the query heads of a KV head.
//  * An additive mask tensor and global + local attention -- "FlashAttention variants: GQA,
//    MQA, sparse attention", sliding-window section (the mask passed as atten_mask: -inf where a
//    key is dropped, added to the scaled scores) and global+local section (a few global tokens
//    attend to, and are attended by, every token; the others see their local window).  The
//    printed global+local code concatenates two outputs along the sequence; the reading taken
//    here is the union of the two key sets for each query, which is what merging the two
//    partial results through their log-sum-exp gives.  `oracle_attn_ext_rows` adds
//    M[b, h, i, j] (broadcast over b or h by a zero stride) to scale * q.k and, with G > 0
//    global tokens, lets query i see key j when j < G or i < G besides the causal / window rule.
//  * INT4 KV cache, the second format of the same KV-compression section ("INT8/INT4").  The
//    pages give no packing; this project stores two 4-bit two's-complement codes per byte (dim
//    2i in the low nibble, dim 2i+1 in the high nibble) with one fp32 scale per (token, KV head),
//    as for INT8.  `oracle_unpack_int4` writes the codes out as int8; the INT4 decode is then
//    the INT8 decode definition over those codes.
//  * Dynamic sequence lengths and a paged KV cache -- "Flash Attention on Ascend: three
//    techniques", version section (sequences of different lengths in one batch) and "Sparse
//    attention and MLA operators in ops-transformer", section 2.2 (KV cache pages addressed
//    through a block_table).  The paged decode
//    oracle gathers key j of sequence b from page block_table[b][j / P], row j % P, and then
//    evaluates the same definition over that sequence's own length.
//
// Inputs are bf16 bit patterns (widened exactly to fp64), fp64 arrays, or int8 codes with
// fp32 scales.  Layouts: Q [B, Sq, Hq, D], K/V [B, Skv, Hkv, D], scales [B, Hkv, Skv],
// O [B, Sq, Hq, D], LSE [B, Hq, Sq] (natural log).  Rows are addressed as (b, h, i) triples.
#include <omp.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <utility>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

struct Dims {
  long B, Hq, Hkv, Sq, Skv, D;
};

double widen_bf16(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Key j is visible to query row i.  Bottom-right aligned causal mask; a window of W keys
// that includes the query's own position.
bool allowed(const Dims& d, int causal, int window, long i, long j) {
  const long ip = i + d.Skv - d.Sq;
  if (j < 0 || j >= d.Skv) return false;
  if (causal && j > ip) return false;
  if (window > 0 && j <= ip - window) return false;
  return true;
}

long kv_head(const Dims& d, long h) { return h / (d.Hq / d.Hkv); }

long q_index(const Dims& d, long b, long i, long h) { return ((b * d.Sq + i) * d.Hq + h) * d.D; }
long kv_index(const Dims& d, long b, long j, long g) { return ((b * d.Skv + j) * d.Hkv + g) * d.D; }

// One output row by the definition.  Q(idx), K(idx), V(idx) return fp64 elements.
template <class QF, class KF, class VF>
void attn_row(const Dims& d, double scale, int causal, int window, long b, long h, long i,
              long j_begin, long j_end, QF Q, KF K, VF V, double* o, double* lse,
              std::vector<double>& x) {
  const long g = kv_head(d, h);
  x.assign(d.Skv, kNegInf);
  double m = kNegInf;
  bool any = false;
  for (long j = j_begin; j < j_end; ++j) {
    if (!allowed(d, causal, window, i, j)) continue;
    double dot = 0.0;
    const long qi = q_index(d, b, i, h), ki = kv_index(d, b, j, g);
    for (long t = 0; t < d.D; ++t) dot += Q(qi + t) * K(ki + t);
    x[j] = scale * dot;
    if (!any || x[j] > m) m = x[j];
    any = true;
  }
  for (long t = 0; t < d.D; ++t) o[t] = 0.0;
  if (!any) {
    *lse = kNegInf;
    return;
  }
  double l = 0.0;
  for (long j = j_begin; j < j_end; ++j) {
    if (x[j] == kNegInf) continue;
    const double p = std::exp(x[j] - m);
    l += p;
    const long vi = kv_index(d, b, j, g);
    for (long t = 0; t < d.D; ++t) o[t] += p * V(vi + t);
  }
  for (long t = 0; t < d.D; ++t) o[t] /= l;
  *lse = m + std::log(l);
}

bool dims_ok(const Dims& d) {
  return d.B > 0 && d.Hq > 0 && d.Hkv > 0 && d.Sq > 0 && d.Skv > 0 && d.D > 0 &&
         d.Hq % d.Hkv == 0;
}

template <class QF, class KF, class VF>
int rows_driver(const Dims& d, double scale, int causal, int window, const int64_t* rows,
                int64_t nrows, double* o, double* lse, int nthreads, QF Q, KF K, VF V) {
  if (!dims_ok(d) || nrows < 0 || (nrows > 0 && (!rows || !o || !lse))) return -1;
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= d.B || h < 0 || h >= d.Hq || i < 0 || i >= d.Sq) return -1;
  }
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
  {
    std::vector<double> x;
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
      attn_row(d, scale, causal, window, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], 0, d.Skv,
               Q, K, V, o + r * d.D, lse + r, x);
    }
  }
  return 0;
}

}  // namespace

extern "C" {

int oracle_max_threads() { return omp_get_max_threads(); }

// The definition, row by row, on bf16 inputs (bit patterns).  rows: nrows (b, h, i) triples;
// o: nrows x D; lse: nrows.  Returns 0, or -1 on a bad argument.
int oracle_attn_bf16_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                          int Hkv, int Sq, int Skv, int D, double scale, int causal, int window,
                          const int64_t* rows, int64_t nrows, double* o, double* lse,
                          int nthreads) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  auto Q = [q](long idx) { return widen_bf16(q[idx]); };
  auto K = [k](long idx) { return widen_bf16(k[idx]); };
  auto V = [v](long idx) { return widen_bf16(v[idx]); };
  return rows_driver(d, scale, causal, window, rows, nrows, o, lse, nthreads, Q, K, V);
}

// The same definition on fp64 inputs.
int oracle_attn_f64_rows(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                         int Sq, int Skv, int D, double scale, int causal, int window,
                         const int64_t* rows, int64_t nrows, double* o, double* lse,
                         int nthreads) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  auto Q = [q](long idx) { return q[idx]; };
  auto K = [k](long idx) { return k[idx]; };
  auto V = [v](long idx) { return v[idx]; };
  return rows_driver(d, scale, causal, window, rows, nrows, o, lse, nthreads, Q, K, V);
}

// The naive multi-pass form: for every (b, h) build the full Sq x Skv score matrix, scale it,
// mask it with -inf, softmax each row, multiply by V.  fp64 inputs; all outputs in full layout
// (O [B,Sq,Hq,D], LSE [B,Hq,Sq]); probs [B,Hq,Sq,Skv] may be null.  Meant for small shapes.
int oracle_attn_brute(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                      int Sq, int Skv, int D, double scale, int causal, int window, double* o,
                      double* lse, double* probs) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  if (!dims_ok(d) || !q || !k || !v || !o || !lse) return -1;
  std::vector<double> S(static_cast<size_t>(Sq) * Skv);
  for (long b = 0; b < B; ++b) {
    for (long h = 0; h < Hq; ++h) {
      const long g = kv_head(d, h);
      // pass 1: scores = Q K^T
      for (long i = 0; i < Sq; ++i)
        for (long j = 0; j < Skv; ++j) {
          double dot = 0.0;
          for (long t = 0; t < D; ++t) dot += q[q_index(d, b, i, h) + t] * k[kv_index(d, b, j, g) + t];
          S[i * Skv + j] = dot;
        }
      // pass 2: scale, then mask (-inf where a key is not visible)
      for (long i = 0; i < Sq; ++i)
        for (long j = 0; j < Skv; ++j) {
          S[i * Skv + j] *= scale;
          if (!allowed(d, causal, window, i, j)) S[i * Skv + j] = kNegInf;
        }
      // pass 3: row softmax (and the log of its normaliser)
      for (long i = 0; i < Sq; ++i) {
        double m = kNegInf;
        for (long j = 0; j < Skv; ++j) m = std::max(m, S[i * Skv + j]);
        double* lrow = lse + (b * Hq + h) * Sq + i;
        if (m == kNegInf) {
          for (long j = 0; j < Skv; ++j) S[i * Skv + j] = 0.0;
          *lrow = kNegInf;
          continue;
        }
        double l = 0.0;
        for (long j = 0; j < Skv; ++j) {
          S[i * Skv + j] = (S[i * Skv + j] == kNegInf) ? 0.0 : std::exp(S[i * Skv + j] - m);
          l += S[i * Skv + j];
        }
        for (long j = 0; j < Skv; ++j) S[i * Skv + j] /= l;
        *lrow = m + std::log(l);
      }
      if (probs)
        std::memcpy(probs + (b * Hq + h) * Sq * Skv, S.data(), sizeof(double) * Sq * Skv);
      // pass 4: output = P V
      for (long i = 0; i < Sq; ++i)
        for (long t = 0; t < D; ++t) {
          double acc = 0.0;
          for (long j = 0; j < Skv; ++j) acc += S[i * Skv + j] * v[kv_index(d, b, j, g) + t];
          o[q_index(d, b, i, h) + t] = acc;
        }
    }
  }
  return 0;
}

// Tiled evaluation: Q blocks of `tile` rows in the outer loop, K/V blocks of `tile` keys in
// the inner loop.  Per row only the running maximum m, the running exp-sum l and the
// unnormalised output are kept; when a block raises the maximum, l and the output are
// multiplied by exp(m_old - m_new).  fp64 inputs; full-layout outputs.
int oracle_attn_tiled(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                      int Sq, int Skv, int D, double scale, int causal, int window, int tile,
                      double* o, double* lse) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  if (!dims_ok(d) || tile <= 0 || !q || !k || !v || !o || !lse) return -1;
  std::vector<double> m(tile), l(tile), acc(static_cast<size_t>(tile) * D), x(tile);
  for (long b = 0; b < B; ++b) {
    for (long h = 0; h < Hq; ++h) {
      const long g = kv_head(d, h);
      for (long i0 = 0; i0 < Sq; i0 += tile) {
        const long ni = std::min<long>(tile, Sq - i0);
        for (long r = 0; r < ni; ++r) {
          m[r] = kNegInf;
          l[r] = 0.0;
          for (long t = 0; t < D; ++t) acc[r * D + t] = 0.0;
        }
        for (long j0 = 0; j0 < Skv; j0 += tile) {
          const long nj = std::min<long>(tile, Skv - j0);
          for (long r = 0; r < ni; ++r) {
            const long i = i0 + r;
            double m_blk = kNegInf;
            for (long c = 0; c < nj; ++c) {
              const long j = j0 + c;
              if (!allowed(d, causal, window, i, j)) {
                x[c] = kNegInf;
                continue;
              }
              double dot = 0.0;
              for (long t = 0; t < D; ++t) dot += q[q_index(d, b, i, h) + t] * k[kv_index(d, b, j, g) + t];
              x[c] = scale * dot;
              m_blk = std::max(m_blk, x[c]);
            }
            if (m_blk == kNegInf) continue;  // nothing visible in this block
            const double m_new = std::max(m[r], m_blk);
            const double corr = (m[r] == kNegInf) ? 0.0 : std::exp(m[r] - m_new);
            l[r] *= corr;
            for (long t = 0; t < D; ++t) acc[r * D + t] *= corr;
            for (long c = 0; c < nj; ++c) {
              if (x[c] == kNegInf) continue;
              const double p = std::exp(x[c] - m_new);
              l[r] += p;
              const long vi = kv_index(d, b, j0 + c, g);
              for (long t = 0; t < D; ++t) acc[r * D + t] += p * v[vi + t];
            }
            m[r] = m_new;
          }
        }
        for (long r = 0; r < ni; ++r) {
          const long i = i0 + r;
          double* orow = o + q_index(d, b, i, h);
          double* lrow = lse + (b * Hq + h) * Sq + i;
          if (m[r] == kNegInf) {
            for (long t = 0; t < D; ++t) orow[t] = 0.0;
            *lrow = kNegInf;
            continue;
          }
          for (long t = 0; t < D; ++t) orow[t] = acc[r * D + t] / l[r];
          *lrow = m[r] + std::log(l[r]);
        }
      }
    }
  }
  return 0;
}

// The definition with an additive mask and global tokens, row by row, on bf16 inputs.
// mask: fp32, element (b, h, i, j) at mask[b * mask_sb + h * mask_sh + i * Skv + j] (a zero
// stride broadcasts), or null.  n_global = G >= 0.  Key j is visible to query i when the
// causal / window rule admits it, or j < G, or i < G; its score is scale * q.k + mask, and a
// score of -inf (from the mask) drops the key.
int oracle_attn_ext_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                         int Hkv, int Sq, int Skv, int D, double scale, int causal, int window,
                         int n_global, const float* mask, int64_t mask_sb, int64_t mask_sh,
                         const int64_t* rows, int64_t nrows, double* o, double* lse,
                         int nthreads) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  if (!dims_ok(d) || n_global < 0 || nrows < 0 || (nrows > 0 && (!rows || !o || !lse)))
    return -1;
  if (!q || !k || !v || mask_sb < 0 || mask_sh < 0) return -1;
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Sq) return -1;
  }
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
  {
    std::vector<double> x(Skv);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
      const long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
      const long g = kv_head(d, h);
      double* orow = o + r * D;
      // scores of the visible keys, mask added
      double m = kNegInf;
      for (long j = 0; j < Skv; ++j) {
        const bool vis = allowed(d, causal, window, i, j) ||
                         (n_global > 0 && (j < n_global || i < n_global));
        x[j] = kNegInf;
        if (!vis) continue;
        double dot = 0.0;
        for (long t = 0; t < D; ++t)
          dot += widen_bf16(q[q_index(d, b, i, h) + t]) * widen_bf16(k[kv_index(d, b, j, g) + t]);
        x[j] = scale * dot;
        if (mask) x[j] += static_cast<double>(mask[b * mask_sb + h * mask_sh + i * Skv + j]);
        m = std::max(m, x[j]);
      }
      for (long t = 0; t < D; ++t) orow[t] = 0.0;
      if (m == kNegInf) {
        lse[r] = kNegInf;
        continue;
      }
      double l = 0.0;
      for (long j = 0; j < Skv; ++j) {
        if (x[j] == kNegInf) continue;
        const double pj = std::exp(x[j] - m);
        l += pj;
        for (long t = 0; t < D; ++t) orow[t] += pj * widen_bf16(v[kv_index(d, b, j, g) + t]);
      }
      for (long t = 0; t < D; ++t) orow[t] /= l;
      lse[r] = m + std::log(l);
    }
  }
  return 0;
}

// Gradients of the definition (causal / window rule) on bf16 inputs: q, do [B,Sq,Hq,D];
// k, v [B,Skv,Hkv,D].  Outputs fp64: dq [B,Sq,Hq,D], dk, dv [B,Skv,Hkv,D] (overwritten).
// P is recomputed exactly from the scores; O and D come from the same exact P.
int oracle_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                    int B, int Hq, int Hkv, int Sq, int Skv, int D, double scale, int causal,
                    int window, double* dq, double* dk, double* dv, int nthreads) {
  const Dims d{B, Hq, Hkv, Sq, Skv, D};
  if (!dims_ok(d) || !q || !k || !v || !dout || !dq || !dk || !dv) return -1;
  const size_t nq = static_cast<size_t>(B) * Sq * Hq * D, nk = static_cast<size_t>(B) * Skv * Hkv * D;
  for (size_t t = 0; t < nq; ++t) dq[t] = 0.0;
  for (size_t t = 0; t < nk; ++t) dk[t] = dv[t] = 0.0;
  if (nthreads <= 0) nthreads = omp_get_max_threads();
  const long G = Hq / Hkv;
  // one task per (b, KV head): its query heads write disjoint dq rows and share dk, dv rows
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
  for (long task = 0; task < static_cast<long>(B) * Hkv; ++task) {
    const long b = task / Hkv, g = task % Hkv;
    std::vector<double> P(static_cast<size_t>(Sq) * Skv), dS(static_cast<size_t>(Sq) * Skv);
    std::vector<double> Orow(D);
    for (long h = g * G; h < (g + 1) * G; ++h) {
      for (long i = 0; i < Sq; ++i) {
        // probabilities of row i (0 where a key is not visible)
        double* prow = P.data() + i * Skv;
        double m = kNegInf;
        for (long j = 0; j < Skv; ++j) {
          prow[j] = kNegInf;
          if (!allowed(d, causal, window, i, j)) continue;
          double dot = 0.0;
          for (long t = 0; t < D; ++t)
            dot += widen_bf16(q[q_index(d, b, i, h) + t]) * widen_bf16(k[kv_index(d, b, j, g) + t]);
          prow[j] = scale * dot;
          m = std::max(m, prow[j]);
        }
        double l = 0.0;
        for (long j = 0; j < Skv; ++j) {
          prow[j] = (prow[j] == kNegInf) ? 0.0 : std::exp(prow[j] - m);
          l += prow[j];
        }
        for (long j = 0; j < Skv; ++j) prow[j] = (l > 0.0) ? prow[j] / l : 0.0;
        // O_i and D_i = dO_i . O_i
        for (long t = 0; t < D; ++t) Orow[t] = 0.0;
        for (long j = 0; j < Skv; ++j)
          if (prow[j] != 0.0)
            for (long t = 0; t < D; ++t) Orow[t] += prow[j] * widen_bf16(v[kv_index(d, b, j, g) + t]);
        double Di = 0.0;
        for (long t = 0; t < D; ++t) Di += widen_bf16(dout[q_index(d, b, i, h) + t]) * Orow[t];
        // dS_ij = P_ij (dO_i . v_j - D_i)
        for (long j = 0; j < Skv; ++j) {
          double dp = 0.0;
          if (prow[j] != 0.0)
            for (long t = 0; t < D; ++t)
              dp += widen_bf16(dout[q_index(d, b, i, h) + t]) * widen_bf16(v[kv_index(d, b, j, g) + t]);
          dS[i * Skv + j] = prow[j] * (dp - Di);
        }
      }
      // dV_j += sum_i P_ij dO_i ; dK_j += scale sum_i dS_ij q_i ; dQ_i = scale sum_j dS_ij k_j
      for (long j = 0; j < Skv; ++j)
        for (long i = 0; i < Sq; ++i) {
          const double pij = P[i * Skv + j], sij = dS[i * Skv + j];
          if (pij == 0.0 && sij == 0.0) continue;
          for (long t = 0; t < D; ++t) {
            dv[kv_index(d, b, j, g) + t] += pij * widen_bf16(dout[q_index(d, b, i, h) + t]);
            dk[kv_index(d, b, j, g) + t] += scale * sij * widen_bf16(q[q_index(d, b, i, h) + t]);
          }
        }
      for (long i = 0; i < Sq; ++i)
        for (long t = 0; t < D; ++t) {
          double acc = 0.0;
          for (long j = 0; j < Skv; ++j)
            acc += dS[i * Skv + j] * widen_bf16(k[kv_index(d, b, j, g) + t]);
          dq[q_index(d, b, i, h) + t] = scale * acc;
        }
    }
  }
  return 0;
}

// Decode over an INT8 KV cache: one query token per sequence (Sq = 1), keys and values
// dequantised as code * scale.  rows: nrows (b, h) pairs; o: nrows x D; lse: nrows.
// num_splits = 1 evaluates the definition directly.  num_splits > 1 cuts the keys into
// chunks of ceil(Skv / num_splits), evaluates each chunk by the definition (giving a
// normalised partial output O_s and its log-sum-exp L_s) and merges them:
// L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
int oracle_decode_int8_rows(const uint16_t* q, const int8_t* k, const int8_t* v,
                            const float* k_scale, const float* v_scale, int B, int Hq, int Hkv,
                            int Skv, int D, double scale, int num_splits, const int64_t* rows,
                            int64_t nrows, double* o, double* lse, int nthreads) {
  const Dims d{B, Hq, Hkv, 1, Skv, D};
  if (!dims_ok(d) || num_splits < 1 || nrows < 0 || (nrows > 0 && (!rows || !o || !lse)))
    return -1;
  if (!q || !k || !v || !k_scale || !v_scale) return -1;
  for (int64_t r = 0; r < nrows; ++r) {
    if (rows[2 * r] < 0 || rows[2 * r] >= B || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Hq)
      return -1;
  }
  // Scale of element idx of K/V [B, Skv, Hkv, D] lives at [b, g, j] of [B, Hkv, Skv].
  auto scale_at = [&d](const float* s, long idx) {
    const long row = idx / d.D;  // (b * Skv + j) * Hkv + g
    const long g = row % d.Hkv, bj = row / d.Hkv;
    const long j = bj % d.Skv, b = bj / d.Skv;
    return static_cast<double>(s[(b * d.Hkv + g) * d.Skv + j]);
  };
  auto Q = [q](long idx) { return widen_bf16(q[idx]); };
  auto K = [&](long idx) { return static_cast<double>(k[idx]) * scale_at(k_scale, idx); };
  auto V = [&](long idx) { return static_cast<double>(v[idx]) * scale_at(v_scale, idx); };
  const long chunk = (Skv + num_splits - 1) / num_splits;
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
  {
    std::vector<double> x, part_o(static_cast<size_t>(num_splits) * D), part_l(num_splits);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
      const long b = rows[2 * r], h = rows[2 * r + 1];
      for (int s = 0; s < num_splits; ++s) {
        const long j0 = std::min<long>(Skv, s * chunk), j1 = std::min<long>(Skv, (s + 1) * chunk);
        attn_row(d, scale, 1, 0, b, h, 0, j0, j1, Q, K, V, part_o.data() + s * D, &part_l[s], x);
      }
      double mx = kNegInf;
      for (int s = 0; s < num_splits; ++s) mx = std::max(mx, part_l[s]);
      double* orow = o + r * D;
      for (long t = 0; t < D; ++t) orow[t] = 0.0;
      if (mx == kNegInf) {
        lse[r] = kNegInf;
        continue;
      }
      double sum = 0.0;
      for (int s = 0; s < num_splits; ++s)
        if (part_l[s] != kNegInf) sum += std::exp(part_l[s] - mx);
      const double L = mx + std::log(sum);
      for (int s = 0; s < num_splits; ++s) {
        if (part_l[s] == kNegInf) continue;
        const double w = std::exp(part_l[s] - L);
        for (long t = 0; t < D; ++t) orow[t] += w * part_o[s * D + t];
      }
      lse[r] = L;
    }
  }
  return 0;
}

// Decode over a paged INT8 KV cache with per-sequence lengths.  k/v pages: int8
// [num_pages, P, Hkv, D]; scales: fp32 [num_pages, Hkv, P]; block_table: int32 [B, max_pages];
// seqlens: int32 [B].  Key j < seqlens[b] of sequence b is row j % P of page
// block_table[b][j / P].  rows: (b, h) pairs.  num_splits cuts each sequence into chunks of
// ceil(seqlens[b] / num_splits) merged by log-sum-exp as in oracle_decode_int8_rows.  A sequence
// with no key (seqlens[b] == 0) gives O = 0 and LSE = -inf.  Entries of block_table past a
// sequence's last page are never read.
int oracle_decode_int8_paged_rows(const uint16_t* q, const int8_t* k, const int8_t* v,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, const int32_t* seqlens, int B,
                                  int Hq, int Hkv, int P, int max_pages, int num_pages, int D,
                                  double scale, int num_splits, const int64_t* rows,
                                  int64_t nrows, double* o, double* lse, int nthreads) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || P <= 0 || max_pages <= 0 ||
      num_pages <= 0 || D <= 0 || num_splits < 1 || nrows < 0)
    return -1;
  if (!q || !k || !v || !k_scale || !v_scale || !block_table || !seqlens) return -1;
  if (nrows > 0 && (!rows || !o || !lse)) return -1;
  for (int b = 0; b < B; ++b) {
    if (seqlens[b] < 0 || seqlens[b] > static_cast<long>(max_pages) * P) return -1;
    for (long pg = 0; pg < (seqlens[b] + P - 1) / P; ++pg) {
      const int id = block_table[static_cast<long>(b) * max_pages + pg];
      if (id < 0 || id >= num_pages) return -1;
    }
  }
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[2 * r] < 0 || rows[2 * r] >= B || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= Hq)
      return -1;
  const long G = Hq / Hkv;
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
  {
    std::vector<double> x, part_o(static_cast<size_t>(num_splits) * D), part_l(num_splits);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
      const long b = rows[2 * r], h = rows[2 * r + 1], g = h / G;
      const long S = seqlens[b];
      // key j of this sequence: element t of K or V, dequantised
      auto page_row = [&](long j) {
        const long pg = block_table[b * max_pages + j / P];
        return std::make_pair(pg, j % P);
      };
      auto kval = [&](long j, long t) {
        const auto pr = page_row(j);
        const long idx = ((pr.first * P + pr.second) * Hkv + g) * D + t;
        return static_cast<double>(k[idx]) *
               static_cast<double>(k_scale[(pr.first * Hkv + g) * P + pr.second]);
      };
      auto vval = [&](long j, long t) {
        const auto pr = page_row(j);
        const long idx = ((pr.first * P + pr.second) * Hkv + g) * D + t;
        return static_cast<double>(v[idx]) *
               static_cast<double>(v_scale[(pr.first * Hkv + g) * P + pr.second]);
      };
      const long chunk = (S + num_splits - 1) / num_splits;
      x.assign(S, kNegInf);
      for (int s = 0; s < num_splits; ++s) {
        const long j0 = std::min<long>(S, s * chunk), j1 = std::min<long>(S, (s + 1) * chunk);
        double* po = part_o.data() + static_cast<size_t>(s) * D;
        for (long t = 0; t < D; ++t) po[t] = 0.0;
        if (j0 >= j1) {
          part_l[s] = kNegInf;
          continue;
        }
        // the definition over keys [j0, j1): scores, their max, exp-sum, weighted V sum
        double m = kNegInf;
        for (long j = j0; j < j1; ++j) {
          double dot = 0.0;
          for (long t = 0; t < D; ++t) dot += widen_bf16(q[(b * Hq + h) * D + t]) * kval(j, t);
          x[j] = scale * dot;
          m = std::max(m, x[j]);
        }
        double l = 0.0;
        for (long j = j0; j < j1; ++j) {
          const double pj = std::exp(x[j] - m);
          l += pj;
          for (long t = 0; t < D; ++t) po[t] += pj * vval(j, t);
        }
        for (long t = 0; t < D; ++t) po[t] /= l;
        part_l[s] = m + std::log(l);
      }
      double mx = kNegInf;
      for (int s = 0; s < num_splits; ++s) mx = std::max(mx, part_l[s]);
      double sum = 0.0;
      for (int s = 0; s < num_splits; ++s)
        if (part_l[s] != kNegInf) sum += std::exp(part_l[s] - mx);
      const double L = mx + std::log(sum);
      double* orow = o + r * D;
      for (long t = 0; t < D; ++t) orow[t] = 0.0;
      for (int s = 0; s < num_splits; ++s) {
        if (part_l[s] == kNegInf) continue;
        const double w = std::exp(part_l[s] - L);
        for (long t = 0; t < D; ++t) orow[t] += w * part_o[static_cast<size_t>(s) * D + t];
      }
      lse[r] = L;
    }
  }
  return 0;
}

// Unpack INT4 codes: byte i of `packed` holds code 2i in bits 0-3 and code 2i+1 in bits 4-7,
// each a 4-bit two's-complement integer in [-8, 7].  Writes 2 * n_bytes int8 codes.
int oracle_unpack_int4(const uint8_t* packed, int64_t n_bytes, int8_t* codes) {
  if (n_bytes < 0 || (n_bytes > 0 && (!packed || !codes))) return -1;
  for (int64_t i = 0; i < n_bytes; ++i) {
    const int lo = packed[i] & 0xF, hi = (packed[i] >> 4) & 0xF;
    codes[2 * i] = static_cast<int8_t>(lo >= 8 ? lo - 16 : lo);
    codes[2 * i + 1] = static_cast<int8_t>(hi >= 8 ? hi - 16 : hi);
  }
  return 0;
}

}  // extern "C"
