// NF4 codebook, decision thresholds and the bin shortcut table, built on the host.
//
// Source: "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog), 贡献一
// 4-bit NormalFloat: 16 levels from standard-normal quantiles, 8 on the negative
// side and 9 on the positive side with the shared zero kept once (8 + 9 - 1 = 16),
// scaled into [-1, 1]. The probability grid runs evenly from
// P_MAX = 1 - (1/32 + 1/30)/2 down to 1/2 on each side.
//
// The inverse normal CDF is Wichura's algorithm AS 241 (PPND16, Applied Statistics
// 37(3), 1988), followed by Newton steps on Phi(z) = erfc(-z/sqrt 2)/2 so the
// result is accurate to the last bit of a double before the single rounding to fp32.
#include "tables.h"

#include <cmath>
#include <cstring>
#include <limits>
#include <mutex>

namespace qnf4 {
namespace {

double poly8(const double* c, double r) {
  double v = c[7];
  for (int i = 6; i >= 0; --i) v = v * r + c[i];
  return v;
}

// AS 241 (PPND16): z with Phi(z) = p, relative accuracy about 1e-16.
double ppnd16(double p) {
  static const double a[8] = {3.387132872796366608,   133.14166789178437745,
                              1971.5909503065514427,  13731.693765509461125,
                              45921.953931549871457,  67265.770927008700853,
                              33430.575583588128105,  2509.0809287301226727};
  static const double b[8] = {1.0,                    42.313330701600911252,
                              687.1870074920579083,   5394.1960214247511077,
                              21213.794301586595867,  39307.89580009271061,
                              28729.085735721942674,  5226.495278852545925};
  static const double c[8] = {1.42343711074968357734,  4.6303378461565452959,
                              5.7694972214606914055,   3.64784832476320460504,
                              1.27045825245236838258,  0.24178072517745061177,
                              0.0227238449892691845833, 7.7454501427834140764e-4};
  static const double d[8] = {1.0,                     2.05319162663775882187,
                              1.6763848301838038494,   0.68976733498510000455,
                              0.14810397642748007459,  0.0151986665636164571966,
                              5.475938084995344946e-4, 1.05075007164441684324e-9};
  static const double e[8] = {6.6579046435011037772,   5.4637849111641143699,
                              1.7848265399172913358,   0.29656057182850489123,
                              0.026532189526576123093, 0.0012426609473880784386,
                              2.71155556874348757815e-5, 2.01033439929228813265e-7};
  static const double f[8] = {1.0,                     0.59983220655588793769,
                              0.13692988092273580531,  0.0148753612908506148525,
                              7.868691311456132591e-4, 1.8463183175100546818e-5,
                              1.4215117583164458887e-7, 2.04426310338993978564e-15};
  const double q = p - 0.5;
  if (std::fabs(q) <= 0.425) {
    const double r = 0.180625 - q * q;
    return q * poly8(a, r) / poly8(b, r);
  }
  double r = q < 0 ? p : 1.0 - p;
  r = std::sqrt(-std::log(r));
  double z;
  if (r <= 5.0) {
    r -= 1.6;
    z = poly8(c, r) / poly8(d, r);
  } else {
    r -= 5.0;
    z = poly8(e, r) / poly8(f, r);
  }
  return q < 0 ? -z : z;
}

double phi_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

double inv_normal(double p) {
  if (p == 0.5) return 0.0;
  double z = ppnd16(p);
  const double inv_sqrt_2pi = 0.39894228040143267794;
  for (int it = 0; it < 3; ++it) {
    const double dens = inv_sqrt_2pi * std::exp(-0.5 * z * z);
    z -= (phi_cdf(z) - p) / dens;
  }
  return z;
}

void build(Nf4Tables& t) {
  const double p_max = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
  double vals[17];
  int nv = 0;
  // 9 probabilities from p_max to 1/2 (positive side) and 8 (negative side); the
  // grid point i is p_max + i * step with the last one exactly 1/2.
  for (int side = 0; side < 2; ++side) {
    const int n = side == 0 ? 9 : 8;
    const double step = (0.5 - p_max) / (n - 1);
    for (int i = 0; i < n - 1; ++i) {  // the median (zero) is added once below
      const double p = i * step + p_max;
      const double z = inv_normal(p);
      vals[nv++] = side == 0 ? z : -z;
    }
  }
  vals[nv++] = 0.0;
  // sort ascending (16 values)
  for (int i = 1; i < nv; ++i)
    for (int j = i; j > 0 && vals[j] < vals[j - 1]; --j) std::swap(vals[j], vals[j - 1]);
  const double zmax = inv_normal(p_max);
  for (int i = 0; i < 16; ++i) t.levels[i] = static_cast<float>(vals[i] / zmax);

  // Decision thresholds: smallest fp32 strictly above the exact midpoint.
  for (int k = 0; k < 15; ++k) {
    const double m = (static_cast<double>(t.levels[k]) + static_cast<double>(t.levels[k + 1])) * 0.5;
    float f = static_cast<float>(m);
    if (static_cast<double>(f) <= m) f = std::nextafter(f, std::numeric_limits<float>::infinity());
    t.thr[k] = f;
  }
  t.thr[15] = std::numeric_limits<float>::infinity();

  // Bin shortcut (see tables.h): the smallest H whose bins each hold at most one
  // threshold, every threshold at least 2^-16 from a bin edge.
  t.bin_h = 0;
  const double min_gap = 1.0 / 65536.0;
  for (int h = 16; h <= kMaxHalfBins; ++h) {
    bool ok = true;
    for (int k = 0; k < 15 && ok; ++k) {
      const double u = static_cast<double>(t.thr[k]) * h + h;  // bin units; edges at j + 0.5
      const double off = u - 0.5 - std::floor(u - 0.5);        // distance above the edge below
      if (off / h < min_gap || (1.0 - off) / h < min_gap) ok = false;
      if (k < 14) {
        const double u2 = static_cast<double>(t.thr[k + 1]) * h + h;
        if (std::floor(u2 + 0.5) == std::floor(u + 0.5)) ok = false;  // same bin
      }
    }
    if (!ok) continue;
    t.bin_h = h;
    for (int b = 0; b <= 2 * h; ++b) {
      const double lo = (b - 0.5) / h - 1.0;
      int c = 0;
      for (int k = 0; k < 15; ++k) c += static_cast<double>(t.thr[k]) <= lo ? 1 : 0;
      const float tk = c < 15 ? t.thr[c] : 2.0f;
      // entry = (t_k exactly, h'_k): h_k is half the fp32 spacing below t_k, so that
      // t_k - h_k is the midpoint under which RN(w / c) rounds below t_k; h'_k moves it by
      // 2^-15 h_k towards the side an exact tie rounds to (up when t_k's mantissa is even,
      // round half to even), and carries (c_k + 1) mod 16 in its 4 lowest mantissa bits
      // (a shift of at most 15 ulp, far inside that 2^-15 move)
      const double h = (static_cast<double>(tk) -
                        static_cast<double>(std::nextafter(tk, -std::numeric_limits<float>::infinity()))) * 0.5;
      uint32_t tbits;
      std::memcpy(&tbits, &tk, 4);
      const bool even = (tbits & 1u) == 0;
      const float hp = static_cast<float>(even ? h * (1.0 + 0x1p-15) : h * (1.0 - 0x1p-15));
      uint32_t hbits;
      std::memcpy(&hbits, &hp, 4);
      hbits = (hbits & ~15u) | static_cast<uint32_t>((c + 1) & 15);
      t.bin_th[2 * b] = tk;
      std::memcpy(&t.bin_th[2 * b + 1], &hbits, 4);
    }
    break;
  }
}

}  // namespace

const Nf4Tables& nf4_tables() {
  static Nf4Tables t;
  static std::once_flag once;
  std::call_once(once, [] {
    std::memset(&t, 0, sizeof(t));
    build(t);
  });
  return t;
}

}  // namespace qnf4
