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

// L2 policies: 0 normal, 1 evict-first, 2 evict-last.
static const Config kConfigs[] = {
    // name                     kind         BN  stages group_m splits pol_p pol_q
    {"tc1_128x256_s4_g8", kKindSingle, 256, 4, 8, 1, 2, 2},
    {"tc1_128x128_s6_g8", kKindSingle, 128, 6, 8, 1, 2, 2},
    {"swap_128x16_s8", kKindSwap, 16, 8, 1, 1, 1, 2},
    {"swap_128x32_s8", kKindSwap, 32, 8, 1, 1, 1, 2},
    {"pair_256x256_s6_g8", kKindPair, 256, 6, 8, 1, 2, 2},
    {"pair_256x128_s8_g8", kKindPair, 128, 8, 8, 1, 2, 2},
    {"swap_128x16_s8_k4", kKindSwap, 16, 8, 1, 4, 1, 2},
    {"swap_128x16_s8_k8", kKindSwap, 16, 8, 1, 8, 1, 2},
    {"tc1_128x128_s6_g8_k2", kKindSingle, 128, 6, 8, 2, 2, 2},
    {"tc1_128x128_s6_g8_k4", kKindSingle, 128, 6, 8, 4, 2, 2},
    {"tc1_128x256_s4_g8_k2", kKindSingle, 256, 4, 8, 2, 2, 2},
    {"pair_256x256_s6_g16", kKindPair, 256, 6, 16, 1, 2, 2},
    {"pair_256x512_s4_g8", kKindPair, 512, 4, 8, 1, 2, 2},
    {"pair_256x512_s4_g16", kKindPair, 512, 4, 16, 1, 2, 2},
    {"pair_256x512_s4_g8_pn", kKindPair, 512, 4, 8, 1, 0, 0},
    {"tc1_128x256_s4_g8_pn", kKindSingle, 256, 4, 8, 1, 0, 0},
    {"tc1_128x128_s6_g8_pn", kKindSingle, 128, 6, 8, 1, 0, 0},
    {"swap_128x16_s8_k16", kKindSwap, 16, 8, 1, 16, 1, 2},
    {"swap_128x16_s8_k32", kKindSwap, 16, 8, 1, 32, 1, 2},
    {"pair_256x512_s4_g16_pf", kKindPair, 512, 4, 16, 1, 2, 1},
    {"pair_256x512_s4_g32", kKindPair, 512, 4, 32, 1, 2, 2},
    {"swap_128x16_s8_sk", kKindSwap, 16, 8, 1, -1, 1, 2},
    {"swap_128x32_s8_sk", kKindSwap, 32, 8, 1, -1, 1, 2},
    {"tc1_128x128_s6_g8_sk", kKindSingle, 128, 6, 8, -1, 2, 2},
    {"tc1_128x256_s4_g8_sk", kKindSingle, 256, 4, 8, -1, 2, 2},
    {"gswap_128x256_s4", kKindGroupedSwap, 256, 4, 1, 1, 0, 0},
    {"gswap2_256x256_s6", kKindGroupedSwapPair, 256, 6, 1, 1, 0, 0},
    {"gswap2_256x256_s6_xl", kKindGroupedSwapPair, 256, 6, 1, 1, 0, 2},
    {"tc1_128x64_s8_g8", kKindSingle, 64, 8, 8, 1, 2, 2},
    {"tc1_128x64_s8_g8_sk", kKindSingle, 64, 8, 8, -1, 2, 2},
    {"tc1_128x64_s8_g8_k2", kKindSingle, 64, 8, 8, 2, 2, 2},
    {"csk_2x128x128_s4", kKindClusterSplitK, 128, 4, 8, 1, 2, 2},
    {"csk_2x128x64_s6", kKindClusterSplitK, 64, 6, 8, 1, 2, 2},
    {"cskswap_2x128x16_s10", kKindClusterSplitKSwap, 16, 10, 1, 1, 1, 2},
    {"tc1_128x256_s4_g8_hy", kKindSingle, 256, 4, 8, -2, 2, 2},
    {"tc1_128x128_s6_g8_hy", kKindSingle, 128, 6, 8, -2, 2, 2},
    {"pair_256x512_s4_g16_sk", kKindPair, 512, 4, 16, -1, 2, 2},
    {"pair_256x512_s4_g16_hy", kKindPair, 512, 4, 16, -2, 2, 2},
    {"pair_256x256_s6_g16_sk", kKindPair, 256, 6, 16, -1, 2, 2},
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
    {256, 256, 256, 256, 256, 256, 0, 0, 28},  // square256: tc1_128x64_s8_g8 3 TFLOP/s
    {1024, 1024, 1024, 1024, 2048, 2048, 0, 0, 31},  // m1024n1024k2048: csk_2x128x128_s4 233 TFLOP/s
    {2048, 2048, 2048, 2048, 2048, 2048, 0, 0, 0},  // square2048: tc1_128x256_s4_g8 749 TFLOP/s
    {4096, 4096, 4096, 4096, 4096, 4096, 0, 0, 13},  // square4096: pair_256x512_s4_g16 1398 TFLOP/s
    {8192, 8192, 8192, 8192, 8192, 8192, 0, 0, 13},  // square8192 (sustained): pair_256x512_s4_g16 1311 TFLOP/s
    {1000, 1000, 1000, 1000, 2000, 2000, 1, 0, 31},  // m1000n1000k2000_bcol: csk_2x128x128_s4 217 TFLOP/s
    {4096, 4096, 4096, 4096, 512, 512, 1, 0, 0},  // m4096n4096k512_bcol: tc1_128x256_s4_g8 684 TFLOP/s
    {16, 16, 8192, 8192, 8192, 8192, 1, 0, 21},  // m16n8192k8192_bcol: swap_128x16_s8_sk 62 TFLOP/s
    {8192, 8192, 1408, 1408, 4096, 4096, 0, 1, 0},  // moe32_n1408_k4096: tc1_128x256_s4_g8 669 TFLOP/s
    {16384, 16384, 4096, 4096, 4096, 4096, 0, 1, 12},  // moe8_n4096_k4096: pair_256x512_s4_g8 1288 TFLOP/s
    {8192, 8192, 768, 768, 2048, 2048, 0, 1, 11},  // moe64_n768_k2048: pair_256x256_s6_g16 405 TFLOP/s
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
  // Few tiles and a long K loop: a CTA pair per 128 x 128 tile, each CTA
  // one half of K, reduced in distributed shared memory
  const long long tiles128 = static_cast<long long>((M + 127) / 128) * ((N + 127) / 128);
  if (!grouped && tiles128 <= 64 && K >= 1024) return 31;
  const long long tiles256 = static_cast<long long>((M + 127) / 128) * ((N + 255) / 256);
  const long long pair_tiles = static_cast<long long>((M + 255) / 256) * ((N + 255) / 256);
  // CTA pairs halve the shared-memory operand traffic per MMA, which wins
  // once every pair gets about two tiles and the K loop is long
  const long long pair512_tiles = static_cast<long long>((M + 255) / 256) * ((N + 511) / 512);
  // Wide 256 x 512 pair tiles stage the fewest operand bytes per FLOP (the
  // most energy-efficient under the power cap) once there are ~4 waves of them
  if (!grouped && pair512_tiles >= 296 && K >= 2048) return 13;
  if (!grouped && pair_tiles >= 128 && K >= 1024) return 11;
  if (N <= 128 || tiles256 < 96) return 1;
  return 0;
}

}  // namespace dg16
