// Plain fp64 C++ oracle of the MoBA hot path (OpenMP over rows / heads).
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// CPU legs of bench.py load this library (through oracle/moba_oracle_c.py).
// It shares no code, header, constant or helper with the CUDA library under
// block_sparse_long_key_b200/csrc, and includes nothing from it.
//
// Everything is computed in double precision from the (bf16) input values,
// one query row at a time, in the order the method's definition gives.  No
// blocking, fusion or reordering beyond a plain loop over the terms of each
// sum.  Source: "Optimizing Mixture of Block Attention" (Xiao, Guo,
// Mazaheri, Han), as summarised on the lowest.today pages (Italian and
// German); section names below are the Italian page's.
//
// Readings of points the pages leave open (the same as the numpy oracle,
// oracle/moba_oracle.py):
//  * a query at local position p (block b = p / B) scores only the strictly
//    earlier blocks j < b of its own sequence; its own block is always kept
//    and counts toward topk; with fewer than topk - 1 earlier blocks all are
//    kept; unused sel slots hold -1; rows are sorted ascending;
//  * exact score ties: the lower block index wins;
//  * router scores are the unscaled q . c_j; attention logits are scaled by
//    1/sqrt(d); LSE is the natural-log log-sum-exp of the scaled logits;
//  * GQA: query head h routes on its own against KV head h / (h_q / h_kv);
//  * varlen: blocks, causality and the key-conv zero padding restart at every
//    cu_seqlens boundary; a partial last block's centroid averages its real
//    tokens;
//  * key conv: k'_t = k_t + SiLU(sum_l w_l (.) k_{t-l}), no bias, rounded to
//    bf16 (nearest, ties to even); routing and attention both use k';
//  * backward: the selection is held fixed (top-k has no gradient).
//
// Array layouts (row-major): q, dout [T, hq, d]; k, v [T, hkv, d];
// cu int32 [batch + 1]; sel int64 [T, hq, topk]; centroids [hkv, nbt, d]
// where block j of sequence s is row blk_off[s] + j, blk_off[s] the number
// of blocks of the sequences before s and nbt the total.
#ifdef _OPENMP
#include <omp.h>
#endif

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <limits>
#include <utility>
#include <vector>

namespace {

typedef int64_t i64;

// Number of blocks of a sequence of L tokens (the last one may be partial).
i64 nblocks(i64 L, int B) { return (L + B - 1) / B; }

// First block of every sequence in the concatenated centroid table.
std::vector<i64> block_offsets(const int* cu, int batch, int B) {
  std::vector<i64> off(batch + 1, 0);
  for (int s = 0; s < batch; ++s) off[s + 1] = off[s] + nblocks((i64)cu[s + 1] - cu[s], B);
  return off;
}

// Sequence that holds token t: the largest s with cu[s] <= t.
int seq_of(const int* cu, int batch, i64 t) {
  int s = (int)(std::upper_bound(cu, cu + batch + 1, (int)t) - cu) - 1;
  // empty sequences share their start with the next one: upper_bound already
  // skipped them
  return std::min(std::max(s, 0), batch - 1);
}

// bf16 rounding: 8 significant bits, fp32 exponent range, ties to even.
// For x = m 2^e (0.5 <= |m| < 1) the spacing is 2^(e-8); below the smallest
// normal (2^-126) it stays 2^-133.
double round_bf16(double x) {
  if (std::isnan(x) || std::isinf(x) || x == 0.0) return x;
  int e;
  std::frexp(x, &e);
  if (e < -125) e = -125;
  const double q = std::ldexp(std::nearbyint(std::ldexp(x, 8 - e)), e - 8);
  const double bf16_max = (2.0 - std::ldexp(1.0, -7)) * std::ldexp(1.0, 127);
  if (std::fabs(q) > bf16_max) return std::copysign(std::numeric_limits<double>::infinity(), x);
  return q;
}

double silu(double x) { return x / (1.0 + std::exp(-x)); }

double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

// Visible tokens of query t (global index) under its selected blocks: every
// token of a selected earlier block, and the tokens of its own block up to
// and including t (section "Definizione del Compito": causal attention over
// the selected blocks only).
std::vector<i64> visible_tokens(const i64* sel_row, int topk, i64 t, i64 a, i64 b, int B) {
  std::vector<i64> blocks;
  for (int i = 0; i < topk; ++i)
    if (sel_row[i] >= 0) blocks.push_back(sel_row[i]);
  std::sort(blocks.begin(), blocks.end());
  std::vector<i64> vis;
  for (i64 j : blocks) {
    const i64 t0 = a + j * B, t1 = std::min(a + (j + 1) * B, b);
    for (i64 u = t0; u < std::min(t1, t + 1); ++u) vis.push_back(u);
  }
  return vis;
}

struct RowSoftmax {
  std::vector<i64> vis;
  std::vector<double> p;  // normalised probabilities over vis
  double lse;
};

// Softmax of one query over its visible tokens (max-subtracted, fp64).
RowSoftmax row_softmax(const double* qi, const double* k, int hkv, int kv, int d, const std::vector<i64>& vis) {
  RowSoftmax r;
  r.vis = vis;
  r.p.resize(vis.size());
  const double scale = 1.0 / std::sqrt((double)d);
  double m = -std::numeric_limits<double>::infinity();
  for (size_t u = 0; u < vis.size(); ++u) {
    r.p[u] = dot(qi, k + ((size_t)vis[u] * hkv + kv) * d, d) * scale;
    m = std::max(m, r.p[u]);
  }
  double l = 0.0;
  for (size_t u = 0; u < vis.size(); ++u) {
    r.p[u] = std::exp(r.p[u] - m);
    l += r.p[u];
  }
  for (size_t u = 0; u < vis.size(); ++u) r.p[u] /= l;
  r.lse = m + std::log(l);
  return r;
}

// Routing of one query row: section "Architettura del Modello Statistico" 1
// (score s_j = q . c_j) and "Definizione del Compito" (keep the top-k
// blocks).  The query at local position pos lives in block b = pos / B; it
// scores j < b, keeps the topk - 1 best (ties: lower j) and always b.
// Writes the selected blocks sorted ascending, -1 padded, and returns the
// relative gap between the last kept and the first rejected earlier-block
// score (+inf when nothing was rejected; 0 when both are 0).
double route_row(const double* qi, const double* cent_h, i64 pos, int d, int B, int topk, i64* out) {
  const i64 b = pos / B;
  for (int i = 0; i < topk; ++i) out[i] = -1;
  if (b == 0) {
    out[0] = 0;
    return std::numeric_limits<double>::infinity();
  }
  std::vector<std::pair<double, i64>> sc(b);
  for (i64 j = 0; j < b; ++j) sc[j] = {dot(qi, cent_h + (size_t)j * d, d), j};
  // best first: higher score, then lower index
  auto better = [](const std::pair<double, i64>& x, const std::pair<double, i64>& y) {
    return x.first > y.first || (x.first == y.first && x.second < y.second);
  };
  const i64 keep = std::min<i64>(topk - 1, b);
  double gap = std::numeric_limits<double>::infinity();
  if (b > keep && keep >= 1) {
    // positions keep-1 (last kept) and keep (first rejected) of the order
    std::partial_sort(sc.begin(), sc.begin() + keep + 1, sc.end(), better);
    const double s_in = sc[keep - 1].first, s_out = sc[keep].first;
    const double den = std::max(std::fabs(s_in), std::fabs(s_out));
    gap = den > 0 ? std::fabs(s_in - s_out) / den : 0.0;
  } else {
    std::sort(sc.begin(), sc.end(), better);
  }
  std::vector<i64> kept;
  for (i64 i = 0; i < keep; ++i) kept.push_back(sc[i].second);
  std::sort(kept.begin(), kept.end());
  for (size_t i = 0; i < kept.size(); ++i) out[i] = kept[i];
  out[kept.size()] = b;
  return gap;
}

// Backward of one row with the selection fixed (section "Progettazione del
// Kernel FlashMoBA", "Backward Pass: Ricalcolo": the probabilities are
// recomputed; the gradient is that of softmax attention).  With P the row's
// softmax, O = P V, D = dO . O, dS_t = P_t (dO . v_t - D):
//   dq = sum_t dS_t k_t / sqrt(d);  dk_t += dS_t q / sqrt(d);  dv_t += P_t dO.
// Calls `emit(token, dS_t, P_t)` for every visible token and fills dq.
template <typename Emit>
void backward_row(const double* q, const double* k, const double* v, const double* dout, const i64* sel_row,
                         const int* cu, int batch, int hq, int hkv, int d, int B, int topk, i64 t, int h, double* dq,
                         Emit emit) {
  const int g = hq / hkv;
  const int s = seq_of(cu, batch, t);
  const int kv = h / g;
  const double scale = 1.0 / std::sqrt((double)d);
  const double* qi = q + ((size_t)t * hq + h) * d;
  const double* doi = dout + ((size_t)t * hq + h) * d;
  const std::vector<i64> vis = visible_tokens(sel_row, topk, t, cu[s], cu[s + 1], B);
  const RowSoftmax sm = row_softmax(qi, k, hkv, kv, d, vis);
  std::vector<double> o(d, 0.0);
  for (size_t u = 0; u < vis.size(); ++u) {
    const double* vr = v + ((size_t)vis[u] * hkv + kv) * d;
    for (int c = 0; c < d; ++c) o[c] += sm.p[u] * vr[c];
  }
  const double D = dot(doi, o.data(), d);
  for (int c = 0; c < d; ++c) dq[c] = 0.0;
  for (size_t u = 0; u < vis.size(); ++u) {
    const double* kr = k + ((size_t)vis[u] * hkv + kv) * d;
    const double* vr = v + ((size_t)vis[u] * hkv + kv) * d;
    const double ds = sm.p[u] * (dot(doi, vr, d) - D);
    for (int c = 0; c < d; ++c) dq[c] += ds * kr[c] * scale;
    emit(vis[u], ds, sm.p[u]);
  }
}

}  // namespace

extern "C" {

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_round_bf16(const double* x, double* y, i64 n) {
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < n; ++i) y[i] = round_bf16(x[i]);
}

void orc_silu(const double* x, double* y, i64 n) {
#pragma omp parallel for schedule(static)
  for (i64 i = 0; i < n; ++i) y[i] = silu(x[i]);
}

// Section "Progettazione della Convoluzione delle Chiavi (Appendice B)",
// "Forma Formale": k'_t = k_t + SiLU(sum_{l=0}^{W-1} w_l (.) k_{t-l}), one
// filter per channel, zero padding before the sequence start; w [H, d, W],
// tap l multiplies k_{t-l}.
void orc_key_conv(const double* k, const double* w, int width, const int* cu, int batch, int T, int H, int d,
                  int round_output, double* out) {
#pragma omp parallel for schedule(static)
  for (i64 t = 0; t < T; ++t) {
    const int s = seq_of(cu, batch, t);
    const i64 a = cu[s];
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        double x = 0.0;
        for (int l = 0; l < width; ++l)
          if (t - l >= a) x += w[((size_t)h * d + c) * width + l] * k[((size_t)(t - l) * H + h) * d + c];
        const double y = k[((size_t)t * H + h) * d + c] + silu(x);
        out[((size_t)t * H + h) * d + c] = round_output ? round_bf16(y) : y;
      }
  }
}

// Section "Architettura del Modello Statistico" 1: a block's representative
// is the mean of its keys; blocks are consecutive runs of B tokens of a
// sequence (section "Definizione del Compito": n = N / B), the last one
// possibly partial (its mean is over its real tokens).
void orc_block_centroids(const double* k, const int* cu, int batch, int T, int H, int d, int B, double* cent) {
  (void)T;
  const std::vector<i64> off = block_offsets(cu, batch, B);
  const i64 nbt = off[batch];
#pragma omp parallel for schedule(dynamic, 16)
  for (i64 gb = 0; gb < nbt; ++gb) {
    const int s = (int)(std::upper_bound(off.begin(), off.end(), gb) - off.begin()) - 1;
    const i64 j = gb - off[s];
    const i64 t0 = cu[s] + j * B, t1 = std::min((i64)cu[s] + (j + 1) * B, (i64)cu[s + 1]);
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (i64 t = t0; t < t1; ++t) acc += k[((size_t)t * H + h) * d + c];
        cent[((size_t)h * nbt + gb) * d + c] = acc / (double)(t1 - t0);
      }
  }
}

// sel [T, hq, topk] and gap [T, hq] for every row; or, for the `nrows` rows
// (token, head) listed in `rows` ([nrows, 2]), sel [nrows, topk] and gap
// [nrows] in list order.
void orc_route(const double* q, const double* cent, const int* cu, int batch, int T, int hq, int hkv, int d, int B,
               int topk, const i64* rows, i64 nrows, i64* sel, double* gap) {
  const std::vector<i64> off = block_offsets(cu, batch, B);
  const i64 nbt = off[batch];
  const int g = hq / hkv;
  const i64 n = rows ? nrows : (i64)T * hq;
#pragma omp parallel for schedule(dynamic, 64)
  for (i64 r = 0; r < n; ++r) {
    const i64 t = rows ? rows[2 * r] : r / hq;
    const int h = rows ? (int)rows[2 * r + 1] : (int)(r % hq);
    const int s = seq_of(cu, batch, t);
    const double* cent_h = cent + ((size_t)(h / g) * nbt + off[s]) * d;
    const size_t o = rows ? (size_t)r : (size_t)t * hq + h;
    gap[o] = route_row(q + ((size_t)t * hq + h) * d, cent_h, t - cu[s], d, B, topk, sel + o * topk);
  }
}

// Section "Definizione del Compito": O_i = softmax(q_i K_V^T / sqrt(d)) V_V
// over the visible set V(i) of the selected blocks, and LSE_i.  sel, o and
// lse are indexed like orc_route's sel and gap: [T, hq, ...] for every row,
// [nrows, ...] in list order for listed rows.
void orc_attention(const double* q, const double* k, const double* v, const i64* sel, const int* cu, int batch,
                   int T, int hq, int hkv, int d, int B, int topk, const i64* rows, i64 nrows, double* o,
                   double* lse) {
  const int g = hq / hkv;
  const i64 n = rows ? nrows : (i64)T * hq;
#pragma omp parallel for schedule(dynamic, 64)
  for (i64 r = 0; r < n; ++r) {
    const i64 t = rows ? rows[2 * r] : r / hq;
    const int h = rows ? (int)rows[2 * r + 1] : (int)(r % hq);
    const int s = seq_of(cu, batch, t);
    const int kv = h / g;
    const size_t ro = rows ? (size_t)r : (size_t)t * hq + h;
    const std::vector<i64> vis = visible_tokens(sel + ro * topk, topk, t, cu[s], cu[s + 1], B);
    const RowSoftmax sm = row_softmax(q + ((size_t)t * hq + h) * d, k, hkv, kv, d, vis);
    double* orow = o + ro * d;
    for (int c = 0; c < d; ++c) orow[c] = 0.0;
    for (size_t u = 0; u < vis.size(); ++u) {
      const double* vr = v + ((size_t)vis[u] * hkv + kv) * d;
      for (int c = 0; c < d; ++c) orow[c] += sm.p[u] * vr[c];
    }
    lse[ro] = sm.lse;
  }
}

// dQ of the listed rows ([nrows, 2] (token, head)) -> dq_rows [nrows, d];
// sel holds the listed rows' selections, [nrows, topk].
void orc_backward_rows(const double* q, const double* k, const double* v, const double* dout, const i64* sel,
                       const int* cu, int batch, int T, int hq, int hkv, int d, int B, int topk, const i64* rows,
                       i64 nrows, double* dq_rows) {
  (void)T;
#pragma omp parallel for schedule(dynamic, 16)
  for (i64 r = 0; r < nrows; ++r)
    backward_row(q, k, v, dout, sel + (size_t)r * topk, cu, batch, hq, hkv, d, B, topk, rows[2 * r], (int)rows[2 * r + 1],
                 dq_rows + (size_t)r * d, [](i64, double, double) {});
}

// Dense backward of every row: dq [T, hq, d], dk, dv [T, hkv, d] (summed over
// the query heads of each KV head).  One KV head per thread at a time.
void orc_attention_backward(const double* q, const double* k, const double* v, const double* dout, const i64* sel,
                            const int* cu, int batch, int T, int hq, int hkv, int d, int B, int topk, double* dq,
                            double* dk, double* dv) {
  const int g = hq / hkv;
  const double scale = 1.0 / std::sqrt((double)d);
  for (size_t i = 0; i < (size_t)T * hkv * d; ++i) dk[i] = dv[i] = 0.0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int kv = 0; kv < hkv; ++kv)
    for (int h = kv * g; h < (kv + 1) * g; ++h)
      for (i64 t = 0; t < T; ++t) {
        const double* qi = q + ((size_t)t * hq + h) * d;
        const double* doi = dout + ((size_t)t * hq + h) * d;
        backward_row(q, k, v, dout, sel + ((size_t)t * hq + h) * topk, cu, batch, hq, hkv, d, B, topk, t, h,
                     dq + ((size_t)t * hq + h) * d,
                     [&](i64 u, double ds, double p) {
                       double* dkr = dk + ((size_t)u * hkv + kv) * d;
                       double* dvr = dv + ((size_t)u * hkv + kv) * d;
                       for (int c = 0; c < d; ++c) {
                         dkr[c] += ds * qi[c] * scale;
                         dvr[c] += p * doi[c];
                       }
                     });
      }
}

// dK, dV of individual key blocks: for each listed (kv head, global block)
// ([nblocks, 2]), the sum over every query row of the group that selected
// the block of that row's contribution to the block's tokens.  Outputs
// [nblocks, B, d] (rows past a partial block's end stay 0).
//
// Optional (non-null) dk_abs, dv_abs [nblocks, B, d]: magnitude sums the
// GPU tests use for their rounding tolerance, not part of the method:
// dk_abs = sum_i (|dS_it| + P_it U_i) |q_i| / sqrt(d) and dv_abs = sum_i P_it
// |dO_i| with U_i = sum_c |dO_ic O_ic|.
void orc_block_grads(const double* q, const double* k, const double* v, const double* dout, const i64* sel,
                     const int* cu, int batch, int T, int hq, int hkv, int d, int B, int topk, const i64* blocks,
                     i64 nblocks_req, double* dk_blk, double* dv_blk, double* dk_abs, double* dv_abs) {
  (void)T;
  const int g = hq / hkv;
  const double scale = 1.0 / std::sqrt((double)d);
  const std::vector<i64> off = block_offsets(cu, batch, B);
  const size_t nbd = (size_t)B * d;
  for (i64 r = 0; r < nblocks_req; ++r) {
    const int kv = (int)blocks[2 * r];
    const i64 gb = blocks[2 * r + 1];
    double* out[4] = {dk_blk + r * nbd, dv_blk + r * nbd, dk_abs ? dk_abs + r * nbd : nullptr,
                      dv_abs ? dv_abs + r * nbd : nullptr};
    for (int a = 0; a < 4; ++a)
      if (out[a])
        for (size_t i = 0; i < nbd; ++i) out[a][i] = 0.0;
    if (gb < 0 || gb >= off[batch] || kv < 0 || kv >= hkv) continue;  // no such block: zeros
    const int s = (int)(std::upper_bound(off.begin(), off.end(), gb) - off.begin()) - 1;
    const i64 j = gb - off[s];
    const i64 a = cu[s], b = cu[s + 1];
    const i64 t0 = a + j * B, t1 = std::min(a + (j + 1) * B, b);
    // the rows of the group that selected the block (only queries at or
    // after the block's start can)
    std::vector<std::pair<i64, int>> pickers;
    for (i64 t = t0; t < b; ++t)
      for (int h = kv * g; h < (kv + 1) * g; ++h) {
        const i64* row = sel + ((size_t)t * hq + h) * topk;
        for (int i = 0; i < topk; ++i)
          if (row[i] == j) {
            pickers.push_back({t, h});
            break;
          }
      }
#pragma omp parallel
    {
      std::vector<double> acc(4 * nbd, 0.0), dq(d), o(d);
#pragma omp for schedule(dynamic, 16)
      for (i64 n = 0; n < (i64)pickers.size(); ++n) {
        const i64 t = pickers[n].first;
        const int h = pickers[n].second;
        const i64* row = sel + ((size_t)t * hq + h) * topk;
        const double* qi = q + ((size_t)t * hq + h) * d;
        const double* doi = dout + ((size_t)t * hq + h) * d;
        std::vector<std::pair<i64, std::pair<double, double>>> mine;  // (token, (dS, P)) inside the block
        backward_row(q, k, v, dout, row, cu, batch, hq, hkv, d, B, topk, t, h, dq.data(),
                     [&](i64 u, double ds, double p) {
                       if (u >= t0 && u < t1) mine.push_back({u, {ds, p}});
                     });
        double U = 0.0;
        if (dk_abs) {
          // U_i from the row's output O_i = sum_t P_t v_t over its visible set
          const std::vector<i64> vis = visible_tokens(row, topk, t, a, b, B);
          const RowSoftmax sm = row_softmax(qi, k, hkv, kv, d, vis);
          for (int c = 0; c < d; ++c) o[c] = 0.0;
          for (size_t w = 0; w < vis.size(); ++w)
            for (int c = 0; c < d; ++c) o[c] += sm.p[w] * v[((size_t)vis[w] * hkv + kv) * d + c];
          for (int c = 0; c < d; ++c) U += std::fabs(doi[c] * o[c]);
        }
        for (const auto& e : mine) {
          const size_t u = (size_t)(e.first - t0) * d;
          const double ds = e.second.first, p = e.second.second;
          for (int c = 0; c < d; ++c) {
            acc[u + c] += ds * qi[c] * scale;
            acc[nbd + u + c] += p * doi[c];
            acc[2 * nbd + u + c] += (std::fabs(ds) + p * U) * std::fabs(qi[c]) * scale;
            acc[3 * nbd + u + c] += p * std::fabs(doi[c]);
          }
        }
      }
#pragma omp critical
      for (int a2 = 0; a2 < 4; ++a2)
        if (out[a2])
          for (size_t i = 0; i < nbd; ++i) out[a2][i] += acc[a2 * nbd + i];
    }
  }
}

// Backward of the key convolution (differentiating orc_key_conv with the
// bf16 rounding taken as the identity): with x_t = sum_l w_l (.) k_{t-l} and
// g_t = dK'_t (.) SiLU'(x_t), SiLU'(x) = s(x) (1 + x (1 - s(x))):
//   dK_t = dK'_t + sum_l w_l (.) g_{t+l}   (t + l inside the sequence)
//   dW_l = sum_t g_t (.) k_{t-l}.
void orc_key_conv_backward(const double* k, const double* w, int width, const int* cu, int batch, int T, int H, int d,
                           const double* dk_conv, double* dk, double* dw) {
  std::vector<double> gbuf((size_t)T * H * d);
#pragma omp parallel for schedule(static)
  for (i64 t = 0; t < T; ++t) {
    const int s = seq_of(cu, batch, t);
    const i64 a = cu[s];
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        double x = 0.0;
        for (int l = 0; l < width; ++l)
          if (t - l >= a) x += w[((size_t)h * d + c) * width + l] * k[((size_t)(t - l) * H + h) * d + c];
        const double sg = 1.0 / (1.0 + std::exp(-x));
        const size_t i = ((size_t)t * H + h) * d + c;
        gbuf[i] = dk_conv[i] * sg * (1.0 + x * (1.0 - sg));
      }
  }
#pragma omp parallel for schedule(static)
  for (i64 t = 0; t < T; ++t) {
    const int s = seq_of(cu, batch, t);
    const i64 b = cu[s + 1];
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        const size_t i = ((size_t)t * H + h) * d + c;
        double acc = dk_conv[i];
        for (int l = 0; l < width; ++l)
          if (t + l < b) acc += w[((size_t)h * d + c) * width + l] * gbuf[((size_t)(t + l) * H + h) * d + c];
        dk[i] = acc;
      }
  }
#pragma omp parallel for schedule(static)
  for (int hc = 0; hc < H * d; ++hc) {
    const int h = hc / d, c = hc % d;
    for (int l = 0; l < width; ++l) {
      double acc = 0.0;
      for (i64 t = 0; t < T; ++t) {
        const int s = seq_of(cu, batch, t);
        if (t - l >= cu[s]) acc += gbuf[((size_t)t * H + h) * d + c] * k[((size_t)(t - l) * H + h) * d + c];
      }
      dw[((size_t)h * d + c) * width + l] = acc;
    }
  }
}

// Key-block-major inversion of the picks (section "Progettazione del Kernel
// FlashMoBA", "Tre Kernel Fusi" 1, stage 3): bucket (kv head, global block)
// = kv * nbt + gb lists the row ids t * hq + h of every valid pick, in
// ascending order.  ptr [hkv * nbt + 1]; rows must hold every valid pick.
// Returns the number of picks.
i64 orc_block_index(const i64* sel, const int* cu, int batch, int T, int hq, int hkv, int B, int topk, i64* ptr,
                    i64* rows) {
  const std::vector<i64> off = block_offsets(cu, batch, B);
  const i64 nbt = off[batch];
  const int g = hq / hkv;
  const i64 nb = (i64)hkv * nbt;
  for (i64 i = 0; i <= nb; ++i) ptr[i] = 0;
  for (i64 t = 0; t < T; ++t) {
    const int s = seq_of(cu, batch, t);
    for (int h = 0; h < hq; ++h)
      for (int i = 0; i < topk; ++i) {
        const i64 j = sel[((size_t)t * hq + h) * topk + i];
        if (j >= 0) ptr[(i64)(h / g) * nbt + off[s] + j + 1] += 1;
      }
  }
  for (i64 i = 0; i < nb; ++i) ptr[i + 1] += ptr[i];
  std::vector<i64> cur(ptr, ptr + nb);
  for (i64 t = 0; t < T; ++t) {  // ascending row ids: every bucket comes out sorted
    const int s = seq_of(cu, batch, t);
    for (int h = 0; h < hq; ++h)
      for (int i = 0; i < topk; ++i) {
        const i64 j = sel[((size_t)t * hq + h) * topk + i];
        if (j >= 0) rows[cur[(i64)(h / g) * nbt + off[s] + j]++] = t * hq + h;
      }
  }
  return ptr[nb];
}

}  // extern "C"
