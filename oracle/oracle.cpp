/*
 * oracle.cpp -- plain, slow CPU reference (double precision) for the
 * low-latency FP8 decode path.  TEST INFRASTRUCTURE ONLY: see oracle.h.
 *
 * Build: g++ -O2 -std=c++17 -fPIC -shared -ffp-contract=off (no fast-math).
 * -ffp-contract=off keeps the few float operations (amax/448, x*inv) as single
 * IEEE roundings, the way the method states them.
 */
#include "oracle.h"

#include <cmath>
#include <cstring>
#include <limits>
#include <vector>

namespace {

/* e4m3 value of each of the 256 codes, from the format definition:
 * exponent field e (4 bits), mantissa field f (3 bits), bias 7;
 * e == 0: subnormal f/8 * 2^-6; otherwise (1 + f/8) * 2^(e-7);
 * e == 15 && f == 7: NaN (the format has no infinities). */
struct E4m3Table {
  double v[256];
  E4m3Table() {
    for (int c = 0; c < 256; ++c) {
      const int s = (c >> 7) & 1, e = (c >> 3) & 15, f = c & 7;
      double mag;
      if (e == 15 && f == 7) {
        mag = std::numeric_limits<double>::quiet_NaN();
      } else if (e == 0) {
        mag = std::ldexp(f / 8.0, -6);
      } else {
        mag = std::ldexp(1.0 + f / 8.0, e - 7);
      }
      v[c] = s ? -mag : mag;
    }
  }
};
const E4m3Table kE4m3;

inline double silu(double g) { return g / (1.0 + std::exp(-g)); }

}  // namespace

extern "C" {

double oracle_bf16_to_f64(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;  // bf16 is the top half of a float
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

uint16_t oracle_f64_to_bf16(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const bool neg = std::signbit(v);
  double a = std::fabs(v);
  if (a == 0.0) return neg ? 0x8000 : 0x0000;
  // bf16: 8 significant bits, exponent range of float (min normal 2^-126,
  // subnormal step 2^-133).  Round |v| to that grid, ties to even.
  int e = std::ilogb(a);
  if (e < -126) e = -126;
  const double ulp = std::ldexp(1.0, e - 7);
  double r = std::nearbyint(a / ulp) * ulp;  // default mode: round half to even
  const double max_bf16 = std::ldexp(255.0, 127 - 7);  // 0x7F7F = (2 - 2^-7) * 2^127
  if (r > max_bf16) r = std::numeric_limits<double>::infinity();
  const float rf = static_cast<float>(r);  // exact: r lies on the bf16 grid
  uint32_t u;
  std::memcpy(&u, &rf, 4);
  uint16_t b = static_cast<uint16_t>(u >> 16);
  return neg ? static_cast<uint16_t>(b | 0x8000) : b;
}

double oracle_e4m3_to_f64(uint8_t code) { return kE4m3.v[code]; }

uint8_t oracle_f32_to_e4m3(float vf) {
  if (std::isnan(vf)) return 0x7F;
  const uint8_t sign = std::signbit(vf) ? 0x80 : 0x00;
  double a = std::fabs(static_cast<double>(vf));
  if (a >= 448.0) return sign | 0x7E;  // saturate: S.1111.110 = 448
  // subnormal range: below 2^-6, step 2^-9
  if (a < std::ldexp(1.0, -6)) {
    const double m = std::nearbyint(a / std::ldexp(1.0, -9));  // 0..8, ties to even
    // m == 8 is exactly the smallest normal 2^-6 = code 0x08, which the same
    // formula (exponent field 0, mantissa 8) encodes as 0x08 as well.
    return sign | static_cast<uint8_t>(m);
  }
  int e = std::ilogb(a);                       // a in [2^e, 2^(e+1))
  double frac = a / std::ldexp(1.0, e) - 1.0;  // [0, 1), exact
  double m = std::nearbyint(frac * 8.0);       // ties to even
  if (m == 8.0) { m = 0.0; e += 1; }
  // Here a < 448, so at e == 8 the fraction is below 0.75 and m <= 6: the
  // largest code reached is S.1111.110 (448), never the NaN pattern.
  const int ef = e + 7;
  return sign | static_cast<uint8_t>((ef << 3) | static_cast<int>(m));
}

void oracle_act_quant(const uint16_t* x, int M, int K, uint8_t* xq, float* s_x) {
  const long long n = static_cast<long long>(M) * K;
  float amax = 0.0f;
  for (long long i = 0; i < n; ++i) {
    const float a = std::fabs(static_cast<float>(oracle_bf16_to_f64(x[i])));
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) {
    *s_x = 1.0f;
    for (long long i = 0; i < n; ++i) xq[i] = 0;
    return;
  }
  volatile float num = 448.0f;  // keep each float operation a single rounding
  const float inv = num / amax;
  const float sx = amax / num;
  *s_x = sx;
  for (long long i = 0; i < n; ++i) {
    const float xv = static_cast<float>(oracle_bf16_to_f64(x[i]));
    volatile float prod = xv * inv;
    xq[i] = oracle_f32_to_e4m3(prod);
  }
}

void oracle_gemm_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                   int M, int N, int K, double* y) {
  const double scale = static_cast<double>(s_x) * static_cast<double>(s_w);
  std::vector<double> xd(static_cast<size_t>(K));
  for (int m = 0; m < M; ++m) {
    for (int k = 0; k < K; ++k) xd[k] = kE4m3.v[xq[static_cast<size_t>(m) * K + k]];
    for (int n = 0; n < N; ++n) {
      const uint8_t* wr = w + static_cast<size_t>(n) * K;
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xd[k] * kE4m3.v[wr[k]];
      y[static_cast<size_t>(m) * N + n] = acc * scale;
    }
  }
}

void oracle_fc13_swiglu_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                          int M, int K, int N2, double* out) {
  const int F = N2 / 2;
  std::vector<double> y(static_cast<size_t>(M) * N2);
  oracle_gemm_q(xq, s_x, w, s_w, M, N2, K, y.data());
  for (int m = 0; m < M; ++m) {
    for (int j = 0; j < F; ++j) {
      const double g = y[static_cast<size_t>(m) * N2 + j];
      const double u = y[static_cast<size_t>(m) * N2 + F + j];
      out[static_cast<size_t>(m) * F + j] = silu(g) * u;
    }
  }
}

void oracle_fc13_swiglu(const uint16_t* x, int M, int K, const uint8_t* w, float s_w,
                        int N2, double* out) {
  std::vector<uint8_t> xq(static_cast<size_t>(M) * K);
  float s_x = 0.0f;
  oracle_act_quant(x, M, K, xq.data(), &s_x);
  oracle_fc13_swiglu_q(xq.data(), s_x, w, s_w, M, K, N2, out);
}

void oracle_fc_qkv_scale_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                           int M, int K, int Hq, int Hkv, int d, float q_scale,
                           double* out) {
  const int N = (Hq + 2 * Hkv) * d;
  oracle_gemm_q(xq, s_x, w, s_w, M, N, K, out);
  const int qcols = Hq * d;
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < qcols; ++n) out[static_cast<size_t>(m) * N + n] *= static_cast<double>(q_scale);
}

void oracle_fc_qkv_scale(const uint16_t* x, int M, int K, const uint8_t* w, float s_w,
                         int Hq, int Hkv, int d, float q_scale, double* out) {
  std::vector<uint8_t> xq(static_cast<size_t>(M) * K);
  float s_x = 0.0f;
  oracle_act_quant(x, M, K, xq.data(), &s_x);
  oracle_fc_qkv_scale_q(xq.data(), s_x, w, s_w, M, K, Hq, Hkv, d, q_scale, out);
}

void oracle_moe_fc13_swiglu(const uint16_t* x, int T, int K, const int32_t* ids, int E,
                            const uint8_t* w, const float* s_w, int N2, double* out) {
  const int F = N2 / 2;
  std::vector<uint8_t> xq(static_cast<size_t>(T) * K);
  float s_x = 0.0f;
  oracle_act_quant(x, T, K, xq.data(), &s_x);
  for (int t = 0; t < T; ++t) {
    const int e = ids[t];
    if (e < 0 || e >= E) {  // not a valid route: leave a NaN row so a test sees it
      for (int j = 0; j < F; ++j) out[static_cast<size_t>(t) * F + j] = std::nan("");
      continue;
    }
    const uint8_t* we = w + static_cast<size_t>(e) * N2 * K;
    oracle_fc13_swiglu_q(xq.data() + static_cast<size_t>(t) * K, s_x, we, s_w[e], 1, K, N2,
                         out + static_cast<size_t>(t) * F);
  }
}

void oracle_quant_f32(const float* y, long long n, uint8_t* xq, float* s_x) {
  float amax = 0.0f;
  for (long long i = 0; i < n; ++i) {
    const float a = std::fabs(y[i]);
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) {
    *s_x = 1.0f;
    for (long long i = 0; i < n; ++i) xq[i] = 0;
    return;
  }
  volatile float num = 448.0f;  // single IEEE roundings, as in oracle_act_quant
  const float inv = num / amax;
  *s_x = amax / num;
  for (long long i = 0; i < n; ++i) {
    volatile float prod = y[i] * inv;
    xq[i] = oracle_f32_to_e4m3(prod);
  }
}

void oracle_linear(const uint16_t* x, int M, int K, const uint8_t* w, float s_w, int N,
                   double* out) {
  std::vector<uint8_t> xq(static_cast<size_t>(M) * K);
  float s_x = 0.0f;
  oracle_act_quant(x, M, K, xq.data(), &s_x);
  oracle_gemm_q(xq.data(), s_x, w, s_w, M, N, K, out);
}

void oracle_moe_linear(const uint16_t* x, int T, int K, const int32_t* ids, int E,
                       const uint8_t* w, const float* s_w, int N, double* out) {
  std::vector<uint8_t> xq(static_cast<size_t>(T) * K);
  float s_x = 0.0f;
  oracle_act_quant(x, T, K, xq.data(), &s_x);
  for (int t = 0; t < T; ++t) {
    const int e = ids[t];
    double* row = out + static_cast<size_t>(t) * N;
    if (e < 0 || e >= E) {
      for (int n = 0; n < N; ++n) row[n] = std::nan("");
      continue;
    }
    oracle_gemm_q(xq.data() + static_cast<size_t>(t) * K, s_x, w + static_cast<size_t>(e) * N * K,
                  s_w[e], 1, N, K, row);
  }
}

void oracle_add_rmsnorm(const uint16_t* x, const uint16_t* r, const uint16_t* gamma, int M,
                        int K, float eps, uint16_t* h_out, double* y) {
  std::vector<double> h(static_cast<size_t>(K));
  for (int m = 0; m < M; ++m) {
    const size_t base = static_cast<size_t>(m) * K;
    double ss = 0.0;
    for (int k = 0; k < K; ++k) {
      // the residual stream is bf16: the exact sum is rounded once to bf16
      uint16_t hb = x[base + k];
      if (r != nullptr) hb = oracle_f64_to_bf16(oracle_bf16_to_f64(x[base + k]) + oracle_bf16_to_f64(r[base + k]));
      h_out[base + k] = hb;
      h[k] = oracle_bf16_to_f64(hb);
      ss += h[k] * h[k];
    }
    const double inv_rms = 1.0 / std::sqrt(ss / K + static_cast<double>(eps));
    for (int k = 0; k < K; ++k) y[base + k] = h[k] * inv_rms * oracle_bf16_to_f64(gamma[k]);
  }
}

void oracle_spec_verify_greedy(const uint16_t* logits, int B, int T, int V, const int32_t* draft,
                               int32_t* target_ids, int32_t* n_accepted, int32_t* emitted) {
  for (int b = 0; b < B; ++b) {
    // the token the target model itself would emit after each input position
    for (int t = 0; t < T; ++t) {
      const uint16_t* row = logits + (static_cast<size_t>(b) * T + t) * static_cast<size_t>(V);
      int best = 0;
      double best_v = oracle_bf16_to_f64(row[0]);
      for (int v = 1; v < V; ++v) {
        const double x = oracle_bf16_to_f64(row[v]);
        if (x > best_v) {  // strict: the lowest index wins a tie
          best_v = x;
          best = v;
        }
      }
      target_ids[static_cast<size_t>(b) * T + t] = best;
    }
    // drafts are accepted while they equal the target's own token; the first
    // mismatch ends the run and the target's token there is emitted instead
    int n = 0;
    while (n < T - 1 && draft[static_cast<size_t>(b) * (T - 1) + n] == target_ids[static_cast<size_t>(b) * T + n]) ++n;
    n_accepted[b] = n;
    for (int t = 0; t < T; ++t)
      emitted[static_cast<size_t>(b) * T + t] = t <= n ? target_ids[static_cast<size_t>(b) * T + t] : -1;
  }
}

void oracle_attn_partial(const uint16_t* q, long long q_stride, int T, int Hq, int Hkv,
                         int d, const uint16_t* k, const uint16_t* v, int Lcap,
                         int b, int t, int h, int L, float scale, int key_lo, int key_hi,
                         double* m_out, double* l_out, double* o) {
  const int g = Hq / Hkv;
  const int hk = h / g;
  const uint16_t* qr = q + (static_cast<long long>(b) * T + t) * q_stride + static_cast<long long>(h) * d;
  const size_t head_off = (static_cast<size_t>(b) * Hkv + hk) * static_cast<size_t>(Lcap) * d;
  const int last_visible = L - T + t;  // inclusive
  int lo = key_lo < 0 ? 0 : key_lo;
  int hi = key_hi;
  if (hi > last_visible + 1) hi = last_visible + 1;
  std::vector<double> qd(static_cast<size_t>(d));
  for (int i = 0; i < d; ++i) qd[i] = oracle_bf16_to_f64(qr[i]);
  std::vector<double> s;
  for (int j = lo; j < hi; ++j) {
    const uint16_t* kr = k + head_off + static_cast<size_t>(j) * d;
    double dot = 0.0;
    for (int i = 0; i < d; ++i) dot += qd[i] * oracle_bf16_to_f64(kr[i]);
    s.push_back(static_cast<double>(scale) * dot);
  }
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  if (s.empty()) {
    *m_out = -std::numeric_limits<double>::infinity();
    *l_out = 0.0;
    return;
  }
  double mx = s[0];
  for (double sv : s) mx = sv > mx ? sv : mx;
  double l = 0.0;
  for (int j = lo; j < hi; ++j) {
    const double p = std::exp(s[static_cast<size_t>(j - lo)] - mx);
    l += p;
    const uint16_t* vr = v + head_off + static_cast<size_t>(j) * d;
    for (int i = 0; i < d; ++i) o[i] += p * oracle_bf16_to_f64(vr[i]);
  }
  *m_out = mx;
  *l_out = l;
}

void oracle_decode_attn(const uint16_t* q, long long q_stride, int B, int T, int Hq,
                        int Hkv, int d, const uint16_t* k, const uint16_t* v, int Lcap,
                        const int32_t* seq_lens, float scale, double* out) {
  std::vector<double> o(static_cast<size_t>(d));
  for (int b = 0; b < B; ++b) {
    const int L = seq_lens[b];
    for (int t = 0; t < T; ++t) {
      for (int h = 0; h < Hq; ++h) {
        double m = 0.0, l = 0.0;
        oracle_attn_partial(q, q_stride, T, Hq, Hkv, d, k, v, Lcap, b, t, h, L, scale, 0, L,
                            &m, &l, o.data());
        double* dst = out + ((static_cast<size_t>(b) * T + t) * Hq + h) * d;
        for (int i = 0; i < d; ++i) dst[i] = l > 0.0 ? o[i] / l : 0.0;
      }
    }
  }
}

void oracle_decode_attn_fp8kv(const uint16_t* q, long long q_stride, int B, int T, int Hq, int Hkv,
                              int d, const uint8_t* k, const uint8_t* v_t, int Lcap,
                              const int32_t* seq_lens, float scale, float s_k, float s_v,
                              double* out) {
  const int g = Hq / Hkv;
  std::vector<double> qd(static_cast<size_t>(d)), s, o(static_cast<size_t>(d));
  for (int b = 0; b < B; ++b) {
    const int L = seq_lens[b];
    for (int t = 0; t < T; ++t) {
      for (int h = 0; h < Hq; ++h) {
        const uint16_t* qr = q + (static_cast<long long>(b) * T + t) * q_stride + static_cast<long long>(h) * d;
        const size_t head = (static_cast<size_t>(b) * Hkv + h / g) * static_cast<size_t>(Lcap) * d;
        for (int i = 0; i < d; ++i) qd[i] = oracle_bf16_to_f64(qr[i]);
        const int visible = L - T + t + 1;  // keys 0 .. L-T+t
        s.assign(static_cast<size_t>(visible > 0 ? visible : 0), 0.0);
        double mx = -std::numeric_limits<double>::infinity();
        for (int j = 0; j < visible; ++j) {
          double dot = 0.0;  // the cache holds k = s_k * e4m3(code)
          for (int i = 0; i < d; ++i) dot += qd[i] * (static_cast<double>(s_k) * kE4m3.v[k[head + static_cast<size_t>(j) * d + i]]);
          s[j] = static_cast<double>(scale) * dot;
          mx = s[j] > mx ? s[j] : mx;
        }
        double l = 0.0;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (int j = 0; j < visible; ++j) {
          const double p = std::exp(s[j] - mx);
          l += p;
          for (int i = 0; i < d; ++i)  // v_t is [d][Lcap] per head: element (key j, dim i) at i*Lcap + j
            o[i] += p * (static_cast<double>(s_v) * kE4m3.v[v_t[head + static_cast<size_t>(i) * Lcap + j]]);
        }
        double* dst = out + ((static_cast<size_t>(b) * T + t) * Hq + h) * d;
        for (int i = 0; i < d; ++i) dst[i] = l > 0.0 ? o[i] / l : 0.0;
      }
    }
  }
}

void oracle_lse_combine(int S, const double* m, const double* l, const double* o_parts,
                        int d, double* out) {
  double mstar = -std::numeric_limits<double>::infinity();
  for (int i = 0; i < S; ++i)
    if (l[i] > 0.0 && m[i] > mstar) mstar = m[i];
  double lstar = 0.0;
  for (int j = 0; j < d; ++j) out[j] = 0.0;
  for (int i = 0; i < S; ++i) {
    if (!(l[i] > 0.0)) continue;  // empty or fully masked chunk: weight 0
    const double w = std::exp(m[i] - mstar);
    lstar += l[i] * w;
    for (int j = 0; j < d; ++j) out[j] += o_parts[static_cast<size_t>(i) * d + j] * w;
  }
  for (int j = 0; j < d; ++j) out[j] = lstar > 0.0 ? out[j] / lstar : 0.0;
}

}  // extern "C"
