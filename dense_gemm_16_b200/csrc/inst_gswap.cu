// Kernel instances of the swapped-operand grouped GEMM (single CTA and CTA
// pair).  The ring is as deep as 227 KB of shared memory allows.
#include "dispatch.h"
#include "gemm_kernel_gswap.cuh"

namespace dg16 {

template <int TOK, int S, bool P_MN, bool BF16, bool F32>
static KernelEntry entry_gswap() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  return {reinterpret_cast<const void*>(&gemm_gswap_kernel<TOK, S, P_MN, BF16, Out>),
          gemm_gswap_smem_bytes<TOK, S>()};
}

template <int TOK, int S>
static KernelEntry pick_gswap(bool p_mn, bool bf16, bool out_f32) {
  const int key = (p_mn ? 4 : 0) | (bf16 ? 2 : 0) | (out_f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_gswap<TOK, S, false, false, false>();
    case 1: return entry_gswap<TOK, S, false, false, true>();
    case 2: return entry_gswap<TOK, S, false, true, false>();
    case 3: return entry_gswap<TOK, S, false, true, true>();
    case 4: return entry_gswap<TOK, S, true, false, false>();
    case 5: return entry_gswap<TOK, S, true, false, true>();
    case 6: return entry_gswap<TOK, S, true, true, false>();
    default: return entry_gswap<TOK, S, true, true, true>();
  }
}

template <int TOK, int S, bool P_MN, bool BF16, bool F32>
static KernelEntry entry_gswap2() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  return {reinterpret_cast<const void*>(&gemm_gswap2_kernel<TOK, S, P_MN, BF16, Out>),
          gemm_gswap2_smem_bytes<TOK, S>()};
}

template <int TOK, int S>
static KernelEntry pick_gswap2(bool p_mn, bool bf16, bool out_f32) {
  const int key = (p_mn ? 4 : 0) | (bf16 ? 2 : 0) | (out_f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_gswap2<TOK, S, false, false, false>();
    case 1: return entry_gswap2<TOK, S, false, false, true>();
    case 2: return entry_gswap2<TOK, S, false, true, false>();
    case 3: return entry_gswap2<TOK, S, false, true, true>();
    case 4: return entry_gswap2<TOK, S, true, false, false>();
    case 5: return entry_gswap2<TOK, S, true, false, true>();
    case 6: return entry_gswap2<TOK, S, true, true, false>();
    default: return entry_gswap2<TOK, S, true, true, true>();
  }
}

// tok = most rows per tile.  Only 256-row tiles are compiled: 192- and
// 128-row tiles (deeper rings: 5 and 6 stages single, 8 for the pair) were
// slower on every grouped shape swept.
// Pair form: per CTA and stage 16 KB of W plus 16 KB of X, 6 stages.
KernelEntry kernels_gswap2(int tok, bool p_mn, bool bf16, bool out_f32) {
  if (tok == 256) return pick_gswap2<256, 6>(p_mn, bf16, out_f32);
  return {nullptr, 0};
}

// Single CTA: per stage 16 KB of W plus up to 32 KB of X, 4 stages.
KernelEntry kernels_gswap(int tok, bool p_mn, bool bf16, bool out_f32) {
  if (tok == 256) return pick_gswap<256, 4>(p_mn, bf16, out_f32);
  return {nullptr, 0};
}

}  // namespace dg16
