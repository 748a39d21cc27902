// config_table.h -- tile configurations and the per-shape choice among them.
//
// The counterpart of the pages' compile-time parameter search: candidate
// tile shapes are enumerated, pruned by the shared-memory budget, timed, and
// the winner per shape class is written down ahead of time ("用Triton跨芯片
// 优化GEMM" section 3.3; the crowd-sourced tuning page, sections 3.2 and 5.2:
// median of several runs, results kept in a table).  The sweep script
// (dense_gemm_16_b200/sweep.py) rewrites the RULES block below from its
// measurements; until a rule matches, the fallback heuristic applies.
#pragma once

#include "dispatch.h"

namespace dg16 {

static const Config kConfigs[] = {
    // name                    kind          BN   stages group_m
    {"tc1_128x256_s4_g8", kKindSingle, 256, 4, 8},
    {"tc1_128x128_s6_g8", kKindSingle, 128, 6, 8},
    {"swap_128x16_s8", kKindSwap, 16, 8, 1},
    {"swap_128x32_s8", kKindSwap, 32, 8, 1},
};
static constexpr int kNumConfigs = static_cast<int>(sizeof(kConfigs) / sizeof(kConfigs[0]));

// One measured choice: problems inside the box [lo, hi] on M, N, K with the
// given B layout (-1 = either) and kind (0 dense, 1 grouped) use config `id`.
struct Rule {
  int m_lo, m_hi, n_lo, n_hi, k_lo, k_hi;
  int b_col;
  int grouped;
  int id;
};

// BEGIN RULES (written by the sweep)
static const Rule kRules[] = {
    {0, 0, 0, 0, 0, 0, -1, -1, -1},  // sentinel
};
// END RULES

inline int table_lookup(int M, int N, int K, bool b_col, bool grouped) {
  for (const Rule& r : kRules) {
    if (r.id < 0) continue;
    if (M < r.m_lo || M > r.m_hi || N < r.n_lo || N > r.n_hi || K < r.k_lo || K > r.k_hi) continue;
    if (r.b_col >= 0 && r.b_col != static_cast<int>(b_col)) continue;
    if (r.grouped != static_cast<int>(grouped)) continue;
    return r.id;
  }
  // Fallback: a few rows of A against a column-major B -> swapped operands so
  // the wide N fills the MMA rows; otherwise the widest tile that still puts
  // at least one tile on most SMs.
  if (!grouped && b_col && M <= 32) return M <= 16 ? 2 : 3;
  const long long tiles256 = static_cast<long long>((M + 127) / 128) * ((N + 255) / 256);
  if (N <= 128 || tiles256 < 96) return 1;
  return 0;
}

}  // namespace dg16
