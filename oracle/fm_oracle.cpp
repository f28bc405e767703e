// Oracle for the mask-aware attention hot path (TEST INFRASTRUCTURE ONLY).
//
// Plain, slow, obviously-correct C++17 CPU code in double precision.  It shares
// no code, header, table or helper with the CUDA library; only the tests, the
// smoke check and the bench's CPU-baseline leg may call it.  Every function
// cites the passage of the FlashMask-3 pages it follows.  Pages cited:
//   [abstract]  acceptodds.com, "FlashMask-3: Efficient and Expressive
//               Mask-Aware Distributed Attention" (the paper abstract)
//   [explainer] learnaivisually.com, "FlashMask-3 sends each GPU its mask
//               without sending any mask" (paragraphs: "four numbers per
//               avenue", "clip-shift-max / Theorem 1", "fully masked, partly
//               masked or unmasked tiles")
//
// Conventions fixed by this build where the pages are silent (each is a stated
// reading, pinned by the tests against independent dense predicates):
//   * intervals are half-open and 0-based: key j masks row i iff
//       LTS[j] <= i < LTE[j]  or  UTS[j] <= i < UTE[j]
//   * a fully masked row has O = 0 and LSE = -inf
//   * LSE is a natural logarithm
//   * vectors are int32 [B, Hm, n_k], Hm in {1, H}; head h reads row hm = (Hm==1 ? 0 : h)
//   * Q, K, V, dO are [B, n, H, D] (row i of head h at ((b*n + i)*H + h)*D)
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

inline bool masked_at(int64_t i, int32_t lts, int32_t lte, int32_t uts, int32_t ute) {
  // [explainer] "four numbers per avenue": start and end of the stretch below
  // the diagonal (LTS, LTE) and of the stretch above it (UTS, UTE).
  return (lts <= i && i < lte) || (uts <= i && i < ute);
}

struct Vecs {
  const int32_t *lts, *lte, *uts, *ute;
  int32_t n_q;
  // NULL vector = canonical empty interval (lower: n_q, n_q; upper: 0, 0)
  int32_t LTS(int64_t j) const { return lts ? lts[j] : n_q; }
  int32_t LTE(int64_t j) const { return lte ? lte[j] : n_q; }
  int32_t UTS(int64_t j) const { return uts ? uts[j] : 0; }
  int32_t UTE(int64_t j) const { return ute ? ute[j] : 0; }
  bool masked(int64_t i, int64_t j) const { return masked_at(i, LTS(j), LTE(j), UTS(j), UTE(j)); }
};

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Dense expansion of the four vectors ([explainer] "four numbers per avenue":
// the n x n map of open/closed squares that the vectors replace).
// out[i*n_k + j] = 1 if (i, j) is masked.
// ---------------------------------------------------------------------------
void orc_dense_mask(int32_t n_q, int32_t n_k, const int32_t* lts, const int32_t* lte,
                    const int32_t* uts, const int32_t* ute, uint8_t* out) {
  Vecs v{lts, lte, uts, ute, n_q};
  for (int64_t i = 0; i < n_q; ++i)
    for (int64_t j = 0; j < n_k; ++j) out[i * n_k + j] = v.masked(i, j) ? 1 : 0;
}

// Unmasked (i, j) pairs by brute force over the dense definition.
int64_t orc_count_unmasked_dense(int32_t n_q, int32_t n_k, const int32_t* lts, const int32_t* lte,
                                 const int32_t* uts, const int32_t* ute) {
  Vecs v{lts, lte, uts, ute, n_q};
  int64_t c = 0;
  for (int64_t i = 0; i < n_q; ++i)
    for (int64_t j = 0; j < n_k; ++j) c += v.masked(i, j) ? 0 : 1;
  return c;
}

// Unmasked pairs per column from the interval lengths: n_q - |([LTS,LTE) U [UTS,UTE)) n [0,n_q)|.
int64_t orc_count_unmasked_intervals(int32_t n_q, int32_t n_k, const int32_t* lts, const int32_t* lte,
                                     const int32_t* uts, const int32_t* ute) {
  Vecs v{lts, lte, uts, ute, n_q};
  int64_t c = 0;
  for (int64_t j = 0; j < n_k; ++j) {
    int64_t a0 = std::max<int64_t>(v.LTS(j), 0), a1 = std::min<int64_t>(v.LTE(j), n_q);
    int64_t b0 = std::max<int64_t>(v.UTS(j), 0), b1 = std::min<int64_t>(v.UTE(j), n_q);
    int64_t la = a1 > a0 ? a1 - a0 : 0, lb = b1 > b0 ? b1 - b0 : 0;
    int64_t ov = 0;
    if (la > 0 && lb > 0) {
      int64_t o0 = std::max(a0, b0), o1 = std::min(a1, b1);
      ov = o1 > o0 ? o1 - o0 : 0;
    }
    c += n_q - (la + lb - ov);
  }
  return c;
}

// Unmasked (row, key) pairs per key chunk of chunk_len keys ([explainer] across-ranks
// paragraph: the all-gather skips key-value chunks that are fully masked; a chunk with
// zero pairs is one of them).  Plain: the per-column count above over each chunk's keys.
void orc_kv_chunk_pairs(int32_t n_q, int32_t n_k, int32_t chunk_len, const int32_t* lts, const int32_t* lte,
                        const int32_t* uts, const int32_t* ute, int64_t* out) {
  const int32_t n_chunks = (n_k + chunk_len - 1) / chunk_len;
  for (int32_t c = 0; c < n_chunks; ++c) {
    const int32_t j0 = c * chunk_len, j1 = std::min(j0 + chunk_len, n_k);
    out[c] = orc_count_unmasked_intervals(n_q, j1 - j0, lts ? lts + j0 : nullptr, lte ? lte + j0 : nullptr,
                                          uts ? uts + j0 : nullptr, ute ? ute + j0 : nullptr);
  }
}

// ---------------------------------------------------------------------------
// Tile classification and block lists ([explainer] "sort every tile of the
// score matrix as fully masked, partly masked or unmasked, using the maximum
// and minimum along the key axis"; "fully masked tiles are never loaded";
// "scans the marks and queues the valid blocks").
//
// Reading: for tile rows [r0, r1) and columns [c0, c1) take min and max of
// each vector over the columns; then
//   skip    = (maxLTS <= r0 && minLTE >= r1) || (maxUTS <= r0 && minUTE >= r1)
//   clear_L = (minLTS >= r1) || (maxLTE <= r0)
//   clear_U = (minUTS >= r1) || (maxUTE <= r0)
//   full    = !skip && clear_L && clear_U;     partial otherwise.
// Class codes 0 = skip, 1 = partial, 2 = full.  List entries are
// (tile << 1) | is_partial in ascending tile order.  Ragged last tiles use
// r1 = min(r0 + tile, n).
//   minmax[kt*8 + {0..7}] = minLTS, maxLTS, minLTE, maxLTE, minUTS, maxUTS, minUTE, maxUTE
// ---------------------------------------------------------------------------
void orc_tile_meta(int32_t n_q, int32_t n_k, int32_t tile_q, int32_t tile_k, const int32_t* lts,
                   const int32_t* lte, const int32_t* uts, const int32_t* ute, int32_t* minmax,
                   uint8_t* cls, int32_t* row_count, int32_t* row_entries, int32_t* col_count,
                   int32_t* col_entries) {
  Vecs v{lts, lte, uts, ute, n_q};
  const int32_t T_q = (n_q + tile_q - 1) / tile_q, T_k = (n_k + tile_k - 1) / tile_k;
  for (int32_t kt = 0; kt < T_k; ++kt) {
    int32_t mn[4], mx[4];
    for (int c = 0; c < 4; ++c) {
      mn[c] = std::numeric_limits<int32_t>::max();
      mx[c] = std::numeric_limits<int32_t>::min();
    }
    for (int64_t j = (int64_t)kt * tile_k; j < std::min<int64_t>((int64_t)(kt + 1) * tile_k, n_k); ++j) {
      int32_t val[4] = {v.LTS(j), v.LTE(j), v.UTS(j), v.UTE(j)};
      for (int c = 0; c < 4; ++c) {
        mn[c] = std::min(mn[c], val[c]);
        mx[c] = std::max(mx[c], val[c]);
      }
    }
    for (int c = 0; c < 4; ++c) {
      minmax[kt * 8 + 2 * c] = mn[c];
      minmax[kt * 8 + 2 * c + 1] = mx[c];
    }
  }
  for (int32_t qt = 0; qt < T_q; ++qt) {
    const int64_t r0 = (int64_t)qt * tile_q, r1 = std::min<int64_t>(r0 + tile_q, n_q);
    for (int32_t kt = 0; kt < T_k; ++kt) {
      const int32_t* m = minmax + kt * 8;
      const int64_t minLTS = m[0], maxLTS = m[1], minLTE = m[2], maxLTE = m[3];
      const int64_t minUTS = m[4], maxUTS = m[5], minUTE = m[6], maxUTE = m[7];
      bool skip = (maxLTS <= r0 && minLTE >= r1) || (maxUTS <= r0 && minUTE >= r1);
      bool clearL = (minLTS >= r1) || (maxLTE <= r0);
      bool clearU = (minUTS >= r1) || (maxUTE <= r0);
      cls[(int64_t)qt * T_k + kt] = skip ? 0 : ((clearL && clearU) ? 2 : 1);
    }
  }
  for (int32_t qt = 0; qt < T_q; ++qt) {
    int32_t c = 0;
    for (int32_t kt = 0; kt < T_k; ++kt) {
      uint8_t k = cls[(int64_t)qt * T_k + kt];
      if (k != 0) row_entries[(int64_t)qt * T_k + c++] = (kt << 1) | (k == 1 ? 1 : 0);
    }
    row_count[qt] = c;
  }
  for (int32_t kt = 0; kt < T_k; ++kt) {
    int32_t c = 0;
    for (int32_t qt = 0; qt < T_q; ++qt) {
      uint8_t k = cls[(int64_t)qt * T_k + kt];
      if (k != 0) col_entries[(int64_t)kt * T_q + c++] = (qt << 1) | (k == 1 ? 1 : 0);
    }
    col_count[kt] = c;
  }
}

// ---------------------------------------------------------------------------
// Localization to a context-parallel rank ([explainer] "clip-shift-max":
// clip each mark to a chunk, shift it into the rank's concatenated numbering,
// take the maximum across the rank's chunks; [abstract] "zero-communication
// clip-shift-max on the boundary vectors").
// The rank owns chunks k = 0..C-1 with global starts g[k], lengths L[k]
// (strictly increasing, non-overlapping); local offsets o[k] = sum_{k'<k} L[k'].
// Formula A (clip-shift-max, the pages' operation as read here):
//   v_loc = max(0, max_k clamp(v - g[k] + o[k], 0, o[k] + L[k]))
// Each of the n values in `in` is mapped independently (keys stay global).
// ---------------------------------------------------------------------------
void orc_localize_clip_shift_max(int64_t n, const int32_t* in, int32_t C, const int32_t* g,
                                 const int32_t* L, int32_t* out) {
  std::vector<int64_t> o(C);
  int64_t acc = 0;
  for (int32_t k = 0; k < C; ++k) {
    o[k] = acc;
    acc += L[k];
  }
  for (int64_t j = 0; j < n; ++j) {
    int64_t best = 0;
    for (int32_t k = 0; k < C; ++k) {
      int64_t x = (int64_t)in[j] - g[k] + o[k];
      int64_t hi = o[k] + L[k];
      x = x < 0 ? 0 : (x > hi ? hi : x);
      best = std::max(best, x);
    }
    out[j] = (int32_t)best;
  }
}

// Formula B (plain definition of the local row number of a global bound):
//   v_loc = #{ rank rows with global index < v } = sum_k clamp(v - g[k], 0, L[k]).
void orc_localize_count(int64_t n, const int32_t* in, int32_t C, const int32_t* g, const int32_t* L,
                        int32_t* out) {
  for (int64_t j = 0; j < n; ++j) {
    int64_t s = 0;
    for (int32_t k = 0; k < C; ++k) {
      int64_t x = (int64_t)in[j] - g[k];
      s += x < 0 ? 0 : (x > L[k] ? L[k] : x);
    }
    out[j] = (int32_t)s;
  }
}

// ---------------------------------------------------------------------------
// Exact masked softmax attention, forward and backward, in fp64.
// Forward (plain definition): U_i = {j : not masked(i, j)}, s_ij = scale q_i.k_j;
//   U_i empty -> O_i = 0, LSE_i = -inf; else m = max s, l = sum exp(s - m),
//   LSE_i = m + ln l, O_i = sum_j exp(s_ij - LSE_i) v_j.
// Backward (exact gradient of the forward, with the oracle's own O):
//   D_i = dO_i . O_i; P_ij = exp(s_ij - LSE_i) on U_i else 0;
//   dV_j = sum_i P_ij dO_i; dS_ij = P_ij (dO_i . v_j - D_i);
//   dQ_i = scale sum_j dS_ij k_j; dK_j = scale sum_i dS_ij q_i.
// The pages fix only that the method is exact attention restricted to the
// unmasked pairs ([abstract]; [explainer] tile paragraph); the formulas are
// the textbook softmax attention and its gradient.
//
// rows/cols select which query rows (O, LSE, dQ) and key columns (dK, dV) of
// head (b, h) are returned.  Column outputs need LSE_i and D_i of every row,
// so they trigger an all-rows statistics pass.
// ---------------------------------------------------------------------------
struct Problem {
  int32_t B, H, Hm, n_q, n_k, D;
  double scale;
  const float *q, *k, *v, *dout;
  const int32_t *lts, *lte, *uts, *ute;
  int32_t b, h;
  Vecs vecs() const {
    int64_t off = ((int64_t)b * Hm + (Hm == 1 ? 0 : h)) * n_k;
    return Vecs{lts ? lts + off : nullptr, lte ? lte + off : nullptr, uts ? uts + off : nullptr,
                ute ? ute + off : nullptr, n_q};
  }
  const float* Q(int64_t i) const { return q + (((int64_t)b * n_q + i) * H + h) * D; }
  const float* K(int64_t j) const { return k + (((int64_t)b * n_k + j) * H + h) * D; }
  const float* V(int64_t j) const { return v + (((int64_t)b * n_k + j) * H + h) * D; }
  const float* dO(int64_t i) const { return dout + (((int64_t)b * n_q + i) * H + h) * D; }
};

static double dot_f(const float* a, const float* b, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) s += (double)a[d] * (double)b[d];
  return s;
}

// One row: its scores s_ij = scale q_i.k_j on the unmasked keys are formed once
// into s[0, n_k) (entries of masked keys are left untouched and never read);
// then LSE_i and O_i (O written to o[D]) by the three passes of the definition:
// the maximum, the sum of exp(s - m), and the weighted sum of the V rows.
static double row_forward(const Problem& p, const Vecs& vv, int64_t i, double* s, double* o) {
  const int D = p.D;
  double m = -std::numeric_limits<double>::infinity();
  bool any = false;
  for (int64_t j = 0; j < p.n_k; ++j) {
    if (vv.masked(i, j)) continue;
    s[j] = p.scale * dot_f(p.Q(i), p.K(j), D);
    if (!any || s[j] > m) m = s[j];
    any = true;
  }
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (!any) return -std::numeric_limits<double>::infinity();
  double l = 0.0;
  for (int64_t j = 0; j < p.n_k; ++j) {
    if (vv.masked(i, j)) continue;
    l += std::exp(s[j] - m);
  }
  double lse = m + std::log(l);
  for (int64_t j = 0; j < p.n_k; ++j) {
    if (vv.masked(i, j)) continue;
    double pij = std::exp(s[j] - lse);
    const float* vj = p.V(j);
    for (int d = 0; d < D; ++d) o[d] += pij * (double)vj[d];
  }
  return lse;
}

// Returns 0 on success.
int orc_attention_head(int32_t B, int32_t H, int32_t Hm, int32_t n_q, int32_t n_k, int32_t D, double scale,
                       const float* q, const float* k, const float* v, const float* dout,
                       const int32_t* lts, const int32_t* lte, const int32_t* uts, const int32_t* ute,
                       int32_t b, int32_t h, int32_t n_rows, const int32_t* rows, int32_t n_cols,
                       const int32_t* cols, double* o_out, double* lse_out, double* dq_out,
                       double* dk_out, double* dv_out, int32_t nthreads) {
  if (b < 0 || b >= B || h < 0 || h >= H || D <= 0) return 1;
  if (Hm != 1 && Hm != H) return 1;
  Problem p{B, H, Hm, n_q, n_k, D, scale, q, k, v, dout, lts, lte, uts, ute, b, h};
  const Vecs vv = p.vecs();
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
  // sampled rows: O, LSE, dQ
#pragma omp parallel
  {
    std::vector<double> s(n_k), o(D), dq(D);
#pragma omp for schedule(dynamic, 1)
    for (int32_t r = 0; r < n_rows; ++r) {
      const int64_t i = rows[r];
      double lse = row_forward(p, vv, i, s.data(), o.data());
      for (int d = 0; d < D; ++d) o_out[(int64_t)r * D + d] = o[d];
      lse_out[r] = lse;
      if (dq_out) {
        for (int d = 0; d < D; ++d) dq[d] = 0.0;
        if (std::isfinite(lse)) {
          double Di = 0.0;
          for (int d = 0; d < D; ++d) Di += (double)p.dO(i)[d] * o[d];
          for (int64_t j = 0; j < n_k; ++j) {
            if (vv.masked(i, j)) continue;
            double pij = std::exp(s[j] - lse);
            double dsij = pij * (dot_f(p.dO(i), p.V(j), D) - Di);
            const float* kj = p.K(j);
            for (int d = 0; d < D; ++d) dq[d] += scale * dsij * (double)kj[d];
          }
        }
        for (int d = 0; d < D; ++d) dq_out[(int64_t)r * D + d] = dq[d];
      }
    }
  }
  if (n_cols <= 0) return 0;
  // all-rows statistics for the column outputs: LSE_i and D_i
  std::vector<double> lse_all(n_q), D_all(n_q);
#pragma omp parallel
  {
    std::vector<double> s(n_k), o(D);
#pragma omp for schedule(dynamic, 16)
    for (int64_t i = 0; i < n_q; ++i) {
      double lse = row_forward(p, vv, i, s.data(), o.data());
      lse_all[i] = lse;
      double Di = 0.0;
      for (int d = 0; d < D; ++d) Di += (double)p.dO(i)[d] * o[d];
      D_all[i] = Di;
    }
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t c = 0; c < n_cols; ++c) {
    const int64_t j = cols[c];
    std::vector<double> dk(D, 0.0), dv(D, 0.0);
    for (int64_t i = 0; i < n_q; ++i) {
      if (!std::isfinite(lse_all[i]) || vv.masked(i, j)) continue;
      double pij = std::exp(scale * dot_f(p.Q(i), p.K(j), D) - lse_all[i]);
      double dsij = pij * (dot_f(p.dO(i), p.V(j), D) - D_all[i]);
      const float* doi = p.dO(i);
      const float* qi = p.Q(i);
      for (int d = 0; d < D; ++d) {
        dv[d] += pij * (double)doi[d];
        dk[d] += scale * dsij * (double)qi[d];
      }
    }
    for (int d = 0; d < D; ++d) {
      if (dk_out) dk_out[(int64_t)c * D + d] = dk[d];
      if (dv_out) dv_out[(int64_t)c * D + d] = dv[d];
    }
  }
  return 0;
}

int orc_max_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
