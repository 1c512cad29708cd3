// Host-side constant tables of the NF4 format (computed once per process).
#pragma once
#include <stdint.h>

namespace qnf4 {

constexpr int kMaxBins = 256;

struct Nf4Tables {
  float levels[16];      // sorted NF4 levels, exact 0 at index 7, -1 / +1 at the ends
  float thr[16];         // 15 decision thresholds, thr[15] = +inf sentinel
  int nbins;             // uniform bins over [-1, 1] used to shortcut the code search
  uint8_t bin_code[kMaxBins + 1];  // #{k : thr[k] <= lower edge of bin b}
};

// Builds the tables on first use (thread-safe). Aborts never; a failure to find a
// valid bin count leaves nbins = 0 and the kernels use the plain threshold count.
const Nf4Tables& nf4_tables();

}  // namespace qnf4
