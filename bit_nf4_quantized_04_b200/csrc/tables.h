// Host-side constant tables of the NF4 format (computed once per process).
#pragma once
#include <stdint.h>

namespace qnf4 {

constexpr int kMaxHalfBins = 128;

// Bin shortcut for the code search. With H = bin_h, a normalised value x in [-1, 1]
// falls in bin k = round(H x + H) (0 <= k <= 2H), which covers
// [(k - 0.5)/H - 1, (k + 0.5)/H - 1). H is chosen so that every bin holds at most one
// decision threshold and every threshold lies at least 2^-16 from a bin edge; then
// code(x) = c_k + (x >= t_k), where c_k counts the thresholds below the bin and t_k is
// the next threshold (2.0 past the last). bin_th[2k], bin_th[2k+1] hold t_k exactly and
// h'_k: half the fp32 spacing below t_k, moved by 2^-15 of itself towards the side an
// exact tie rounds to, with (c_k + 1) mod 16 written into its 4 lowest mantissa bits.
// For a block constant c (8 significant bits, as the absmax of bf16 values) the sign of
// s = fma(c, h'_k, fma(-c, t_k, w)) is exactly that of RN(w / c) - t_k (>= 0 when the
// quotient rounds to t_k or above): within 2^-18 c of c t_k the inner fma is exact (a
// multiple of 2^(e_c + e_t - 30) of at most 18 bits), and farther away c h'_k cannot
// change its sign. Subtracting [s < 0] from h'_k's bits leaves the code in the low 4 bits.
struct Nf4Tables {
  float levels[16];      // sorted NF4 levels, exact 0 at index 7, -1 / +1 at the ends
  float thr[16];         // 15 decision thresholds, thr[15] = +inf sentinel
  int bin_h;             // H above; 0 if no valid H was found (exact count only)
  float bin_th[2 * (2 * kMaxHalfBins + 1)];
};

// Builds the tables on first use (thread-safe). Never aborts; a failure to find a
// valid bin count leaves bin_h = 0 and the kernels use the plain threshold count.
const Nf4Tables& nf4_tables();

}  // namespace qnf4
