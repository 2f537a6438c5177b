// CPU oracle for the DSA forward path: plain, slow, fp64.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
// CPU-baseline leg may load this library. The CUDA library never links,
// includes or calls it, and it shares no code with the CUDA library.
//
// What it computes (page "DeepseekV3.2 拆解", section "核心组件"):
//   * lightning indexer score, equation I_{t,s}:
//       I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]),  j = 1..H^I,
//     with q and k the dequantised FP8 vectors (code value * per-row scale);
//   * fine-grained token selection, equation u_t = Attn(h_t, {c_s | I_{t,s}
//     in Top-k(I_{t,:})}): the k keys with the largest score, ties broken by
//     the lower key index, fewer than k valid keys -> all of them, pad -1;
//   * the per-row FP8 encoding of the indexer inputs (scale = amax / 448,
//     nearest E4M3 value, ties to even, saturating);
//   * the indexer's dense warm-up loss KL(p || Softmax(I)) and its gradient
//     (section "预训练策略 / 密集预热阶段"), see oracle_indexer_kl;
//   * the attention over the selected latent rows c_s (MQA: every query head
//     reads the same row; K = all qk_dim dims, V = the first v_dim dims; the
//     latent width 576 = 512 + 64 follows the MLA section 1.1 of page
//     "DeepSeek architecture"), exact softmax in fp64.
// Everything is the definition written out: no blocking, no fusion, no
// reordering of the sums beyond the natural loop order.
//
// Parity pins live in tests/test_oracle.py (closed forms, library special
// cases, brute force, invariants); the pages print no worked example.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// OCP 8-bit floating point, E4M3 ("fn" flavour): 1 sign bit, 4 exponent bits
// with bias 7, 3 mantissa bits; exponent field 0 is subnormal; S.1111.111 is
// NaN; there is no infinity.
double e4m3_value(uint8_t code) {
  const int sign = (code >> 7) & 1;
  const int e = (code >> 3) & 0xF;
  const int m = code & 0x7;
  double mag;
  if (e == 0xF && m == 0x7) return std::numeric_limits<double>::quiet_NaN();
  if (e == 0) {
    mag = std::ldexp(static_cast<double>(m) / 8.0, 1 - 7);
  } else {
    mag = std::ldexp(1.0 + static_cast<double>(m) / 8.0, e - 7);
  }
  return sign ? -mag : mag;
}

// Encode a float into E4M3 "fn" by the definition: the finite code whose
// value is nearest to v (exact comparison in fp64), ties to the code with an
// even mantissa, magnitudes at or above 448 saturating to +-448, the sign of v
// (including -0) kept in bit 7. A NaN maps to the NaN code 0x7F.
uint8_t e4m3_encode(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  if (a >= 448.0) return sign | 0x7E;
  uint8_t best = 0;
  double best_d = std::numeric_limits<double>::infinity();
  for (int c = 0; c <= 0x7E; ++c) {   // every non-negative finite code
    const double d = std::fabs(a - e4m3_value(static_cast<uint8_t>(c)));
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best_d = d;
      best = static_cast<uint8_t>(c);
    }
  }
  return sign | best;
}

// bfloat16 is the upper half of an IEEE binary32.
double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return static_cast<double>(f);
}

template <class F>
void parallel_rows(int n_rows, int n_threads, F&& body) {
  if (n_threads <= 0) n_threads = static_cast<int>(std::thread::hardware_concurrency());
  if (n_threads <= 0) n_threads = 1;
  n_threads = std::min(n_threads, std::max(n_rows, 1));
  if (n_threads == 1) {
    for (int r = 0; r < n_rows; ++r) body(r);
    return;
  }
  std::vector<std::thread> pool;
  for (int th = 0; th < n_threads; ++th) {
    pool.emplace_back([&, th]() {
      for (int r = th; r < n_rows; r += n_threads) body(r);
    });
  }
  for (auto& t : pool) t.join();
}

}  // namespace

extern "C" {

int oracle_hardware_threads() {
  return static_cast<int>(std::thread::hardware_concurrency());
}

double oracle_e4m3_value(uint8_t code) { return e4m3_value(code); }

uint8_t oracle_e4m3_encode(float v) { return e4m3_encode(v); }

// Per-row FP8 quantisation of bf16 rows (the indexer's inputs: one scale per
// row of d^I values, scale = amax / 448, amax = 0 -> scale 1). The scale and
// each x / scale are computed in fp32 (the precision the GPU kernel decides
// the codes in); the code is then the definition's nearest E4M3 value.
//   x [rows, dim] bf16 bits -> codes [rows, dim], scales [rows]
void oracle_quantize_rows(long long rows, int dim, const uint16_t* x, uint8_t* codes,
                          float* scales) {
  for (long long r = 0; r < rows; ++r) {
    const uint16_t* xr = x + r * dim;
    float amax = 0.0f;
    for (int d = 0; d < dim; ++d)
      amax = std::max(amax, std::fabs(static_cast<float>(bf16_value(xr[d]))));
    const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    scales[r] = scale;
    for (int d = 0; d < dim; ++d) {
      float y = static_cast<float>(bf16_value(xr[d])) / scale;
      y = std::min(448.0f, std::max(-448.0f, y));
      codes[r * dim + d] = e4m3_encode(y);
    }
  }
}

// Indexer scores for n_rows query rows of ONE sequence.
//   q8   [n_rows, HI, DI] e4m3 codes,  qs [n_rows, HI] scale per (row, head)
//   w    [n_rows, HI]
//   k8   [S, DI] e4m3 codes,           ks [S] scale per key
//   pos  [n_rows] absolute query position of each row
//   kv_len: keys with index >= kv_len are invalid
//   out  [n_rows, S]: I[t,s] for valid s (s <= pos and s < kv_len), -inf else
void oracle_indexer_scores(int n_rows, int S, int HI, int DI,
                           const uint8_t* q8, const float* qs, const float* w,
                           const uint8_t* k8, const float* ks,
                           const int32_t* pos, int kv_len,
                           double* out, int n_threads) {
  const double neg_inf = -std::numeric_limits<double>::infinity();
  parallel_rows(n_rows, n_threads, [&](int r) {
    std::vector<double> qhat(static_cast<size_t>(HI) * DI);
    for (int j = 0; j < HI; ++j)
      for (int d = 0; d < DI; ++d)
        qhat[static_cast<size_t>(j) * DI + d] =
            e4m3_value(q8[(static_cast<size_t>(r) * HI + j) * DI + d]) *
            static_cast<double>(qs[static_cast<size_t>(r) * HI + j]);
    std::vector<double> khat(DI);
    double* row_out = out + static_cast<size_t>(r) * S;
    for (int s = 0; s < S; ++s) {
      if (s > pos[r] || s >= kv_len) {
        row_out[s] = neg_inf;
        continue;
      }
      for (int d = 0; d < DI; ++d)
        khat[d] = e4m3_value(k8[static_cast<size_t>(s) * DI + d]) *
                  static_cast<double>(ks[s]);
      double score = 0.0;
      for (int j = 0; j < HI; ++j) {
        double dot = 0.0;
        for (int d = 0; d < DI; ++d) dot += qhat[static_cast<size_t>(j) * DI + d] * khat[d];
        const double relu = dot > 0.0 ? dot : 0.0;
        score += static_cast<double>(w[static_cast<size_t>(r) * HI + j]) * relu;
      }
      row_out[s] = score;
    }
  });
}

// Top-k selection per row: sort the valid keys (finite score) by
// (score descending, index ascending) and keep the first min(k, #valid);
// remaining slots are -1.
//   scores [n_rows, S], out [n_rows, k]
void oracle_topk(int n_rows, int S, int k, const double* scores, int32_t* out,
                 int n_threads) {
  parallel_rows(n_rows, n_threads, [&](int r) {
    const double* row = scores + static_cast<size_t>(r) * S;
    std::vector<int32_t> cand;
    cand.reserve(S);
    for (int s = 0; s < S; ++s)
      if (std::isfinite(row[s])) cand.push_back(s);
    std::sort(cand.begin(), cand.end(), [row](int32_t a, int32_t b) {
      if (row[a] != row[b]) return row[a] > row[b];
      return a < b;
    });
    int32_t* o = out + static_cast<size_t>(r) * k;
    for (int i = 0; i < k; ++i)
      o[i] = i < static_cast<int>(cand.size()) ? cand[i] : -1;
  });
}

// Attention of n_rows query rows of ONE sequence over their selected latent
// rows.
//   q    [n_rows, H, Dqk] bf16 bits
//   kv   [S, Dqk] bf16 bits; K = kv[s, 0:Dqk], V = kv[s, 0:Dv]
//   idx  [n_rows, k] selected key indices, -1 = empty slot
//   o    [n_rows, H, Dv]; lse [n_rows, H] (natural log)
// A row with no selected key gets o = 0 and lse = -inf.
void oracle_sparse_attn(int n_rows, int S, int H, int Dqk, int Dv, int k,
                        double scale, const uint16_t* q, const uint16_t* kv,
                        const int32_t* idx, double* o, double* lse,
                        int n_threads) {
  parallel_rows(n_rows, n_threads, [&](int r) {
    const int32_t* sel = idx + static_cast<size_t>(r) * k;
    std::vector<int32_t> keys;
    for (int i = 0; i < k; ++i)
      if (sel[i] >= 0 && sel[i] < S) keys.push_back(sel[i]);
    const int n = static_cast<int>(keys.size());
    std::vector<double> z(n), qh(Dqk);
    for (int h = 0; h < H; ++h) {
      double* oh = o + (static_cast<size_t>(r) * H + h) * Dv;
      for (int d = 0; d < Dqk; ++d)
        qh[d] = bf16_value(q[(static_cast<size_t>(r) * H + h) * Dqk + d]);
      if (n == 0) {
        for (int d = 0; d < Dv; ++d) oh[d] = 0.0;
        lse[static_cast<size_t>(r) * H + h] = -std::numeric_limits<double>::infinity();
        continue;
      }
      double m = -std::numeric_limits<double>::infinity();
      for (int i = 0; i < n; ++i) {
        const uint16_t* c = kv + static_cast<size_t>(keys[i]) * Dqk;
        double dot = 0.0;
        for (int d = 0; d < Dqk; ++d) dot += qh[d] * bf16_value(c[d]);
        z[i] = scale * dot;
        m = std::max(m, z[i]);
      }
      double l = 0.0;
      for (int i = 0; i < n; ++i) {
        z[i] = std::exp(z[i] - m);
        l += z[i];
      }
      for (int d = 0; d < Dv; ++d) oh[d] = 0.0;
      for (int i = 0; i < n; ++i) {
        const uint16_t* c = kv + static_cast<size_t>(keys[i]) * Dqk;
        const double p = z[i] / l;
        for (int d = 0; d < Dv; ++d) oh[d] += p * bf16_value(c[d]);
      }
      lse[static_cast<size_t>(r) * H + h] = m + std::log(l);
    }
  });
}

// Indexer warm-up loss and its gradient for n_rows query rows of ONE
// sequence (page "DeepseekV3.2 拆解", section "预训练策略 / 密集预热阶段":
// the main model is frozen and the indexer alone is trained to match the
// dense attention distribution, L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:}))).
//
// Readings taken where the page is silent:
//   * p_{t,:} is the main attention's dense causal softmax over the visible
//     keys (s <= pos[t], s < kv_len), averaged over the H query heads (each
//     head's softmax sums to one, so the mean is one distribution per query);
//   * Softmax(I_{t,:}) runs over the same visible keys;
//   * gradients are taken with respect to w and to the dequantised indexer
//     vectors q^ = code * q_scale and k^ = code * k_scale (the FP8 encoding is
//     upstream of the indexer and passes the gradient through unchanged).
// With r_t = Softmax(I_{t,:}) and g[t,s] = r_t[s] - p[t,s] (the derivative of
// KL(p || Softmax(I)) with respect to I[t,s] when p sums to one), and
// x[t,j,s] = q^[t,j] . k^[s]:
//   dL/dw[t,j]  = sum_s g[t,s] ReLU(x[t,j,s])
//   dL/dq^[t,j] = sum_s g[t,s] w[t,j] [x[t,j,s] > 0] k^[s]
//   dL/dk^[s]   = sum_t sum_j g[t,s] w[t,j] [x[t,j,s] > 0] q^[t,j]
//   q8, qs, w, k8, ks, pos, kv_len  as oracle_indexer_scores
//   q   [n_rows, H, Dqk] bf16 bits (main attention queries), kv [S, Dqk] bf16
//   loss [n_rows] (KL of each row), dw [n_rows, HI], dq [n_rows, HI, DI],
//   dk [S, DI] (summed over the given rows; zero where no row sees the key)
void oracle_indexer_kl(int n_rows, int S, int HI, int DI, const uint8_t* q8, const float* qs,
                       const float* w, const uint8_t* k8, const float* ks, const int32_t* pos,
                       int kv_len, int H, int Dqk, double scale, const uint16_t* q,
                       const uint16_t* kv, double* loss, double* dw, double* dq, double* dk,
                       int n_threads) {
  std::vector<double> khat(static_cast<size_t>(S) * DI);
  for (int s = 0; s < S; ++s)
    for (int d = 0; d < DI; ++d)
      khat[static_cast<size_t>(s) * DI + d] =
          e4m3_value(k8[static_cast<size_t>(s) * DI + d]) * static_cast<double>(ks[s]);
  // per-row contributions to dk, summed after the parallel part
  std::vector<double> dk_rows(static_cast<size_t>(n_rows) * S * DI, 0.0);
  parallel_rows(n_rows, n_threads, [&](int r) {
    const int n_vis = std::max(0, std::min(pos[r] + 1, std::min(kv_len, S)));
    std::vector<double> qhat(static_cast<size_t>(HI) * DI);
    for (int j = 0; j < HI; ++j)
      for (int d = 0; d < DI; ++d)
        qhat[static_cast<size_t>(j) * DI + d] =
            e4m3_value(q8[(static_cast<size_t>(r) * HI + j) * DI + d]) *
            static_cast<double>(qs[static_cast<size_t>(r) * HI + j]);
    double* dw_r = dw + static_cast<size_t>(r) * HI;
    double* dq_r = dq + static_cast<size_t>(r) * HI * DI;
    for (int i = 0; i < HI; ++i) dw_r[i] = 0.0;
    for (int i = 0; i < HI * DI; ++i) dq_r[i] = 0.0;
    loss[r] = 0.0;
    if (n_vis == 0) return;
    // p: dense causal attention of each head over the visible keys, averaged
    std::vector<double> p(n_vis, 0.0), z(n_vis), qh(Dqk);
    for (int h = 0; h < H; ++h) {
      for (int d = 0; d < Dqk; ++d)
        qh[d] = bf16_value(q[(static_cast<size_t>(r) * H + h) * Dqk + d]);
      double m = -std::numeric_limits<double>::infinity();
      for (int s = 0; s < n_vis; ++s) {
        double dot = 0.0;
        for (int d = 0; d < Dqk; ++d)
          dot += qh[d] * bf16_value(kv[static_cast<size_t>(s) * Dqk + d]);
        z[s] = scale * dot;
        m = std::max(m, z[s]);
      }
      double l = 0.0;
      for (int s = 0; s < n_vis; ++s) {
        z[s] = std::exp(z[s] - m);
        l += z[s];
      }
      for (int s = 0; s < n_vis; ++s) p[s] += z[s] / l / static_cast<double>(H);
    }
    // indexer scores I and x kept for the gradient. x = q^ . k^ is formed
    // as (sum_d code_q code_k) * q_scale * k_scale: the code products are
    // exact in fp64 and so is their sum (at most 128 terms spanning 36 bits),
    // so the sign of x, which decides the ReLU and its mask, is exact.
    std::vector<double> x(static_cast<size_t>(n_vis) * HI), I(n_vis);
    for (int s = 0; s < n_vis; ++s) {
      double score = 0.0;
      for (int j = 0; j < HI; ++j) {
        double code_dot = 0.0;
        for (int d = 0; d < DI; ++d)
          code_dot += e4m3_value(q8[(static_cast<size_t>(r) * HI + j) * DI + d]) *
                      e4m3_value(k8[static_cast<size_t>(s) * DI + d]);
        const double dot = code_dot * static_cast<double>(qs[static_cast<size_t>(r) * HI + j]) *
                           static_cast<double>(ks[s]);
        x[static_cast<size_t>(s) * HI + j] = dot;
        score += static_cast<double>(w[static_cast<size_t>(r) * HI + j]) * (dot > 0.0 ? dot : 0.0);
      }
      I[s] = score;
    }
    // log Softmax(I) and the KL divergence
    double mi = -std::numeric_limits<double>::infinity();
    for (int s = 0; s < n_vis; ++s) mi = std::max(mi, I[s]);
    double li = 0.0;
    for (int s = 0; s < n_vis; ++s) li += std::exp(I[s] - mi);
    const double lse_i = mi + std::log(li);
    double kl = 0.0;
    for (int s = 0; s < n_vis; ++s)
      if (p[s] > 0.0) kl += p[s] * (std::log(p[s]) - (I[s] - lse_i));
    loss[r] = kl;
    // gradient
    double* dk_r = dk_rows.data() + static_cast<size_t>(r) * S * DI;
    for (int s = 0; s < n_vis; ++s) {
      const double g = std::exp(I[s] - lse_i) - p[s];
      for (int j = 0; j < HI; ++j) {
        const double xv = x[static_cast<size_t>(s) * HI + j];
        if (xv <= 0.0) continue;
        const double wj = static_cast<double>(w[static_cast<size_t>(r) * HI + j]);
        dw_r[j] += g * xv;
        for (int d = 0; d < DI; ++d) {
          dq_r[static_cast<size_t>(j) * DI + d] += g * wj * khat[static_cast<size_t>(s) * DI + d];
          dk_r[static_cast<size_t>(s) * DI + d] += g * wj * qhat[static_cast<size_t>(j) * DI + d];
        }
      }
    }
  });
  for (size_t i = 0; i < static_cast<size_t>(S) * DI; ++i) {
    double acc = 0.0;
    for (int r = 0; r < n_rows; ++r) acc += dk_rows[static_cast<size_t>(r) * S * DI + i];
    dk[i] = acc;
  }
}

}  // extern "C"
