// Kernel instances with 128 x 64 tiles (8-stage ring, 192 KB of operands): twice
// the tiles of 128 x 128 for problems too small to fill the SMs.
#include "dispatch.h"
#include "gemm_kernel.cuh"

namespace dg16 {

template <bool Q_MN, bool BF16, bool F32, bool GROUPED>
static KernelEntry entry64() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  constexpr int S = 8;
  return {reinterpret_cast<const void*>(&gemm_tc_kernel<64, S, Q_MN, BF16, Out, false, GROUPED>),
          gemm_smem_bytes<64, S, GROUPED>()};
}

KernelEntry kernels_bn64(bool q_mn, bool bf16, bool out_f32, bool grouped) {
  const int key = (q_mn ? 8 : 0) | (bf16 ? 4 : 0) | (out_f32 ? 2 : 0) | (grouped ? 1 : 0);
  switch (key) {
    case 0: return entry64<false, false, false, false>();
    case 1: return entry64<false, false, false, true>();
    case 2: return entry64<false, false, true, false>();
    case 3: return entry64<false, false, true, true>();
    case 4: return entry64<false, true, false, false>();
    case 5: return entry64<false, true, false, true>();
    case 6: return entry64<false, true, true, false>();
    case 7: return entry64<false, true, true, true>();
    case 8: return entry64<true, false, false, false>();
    case 9: return entry64<true, false, false, true>();
    case 10: return entry64<true, false, true, false>();
    case 11: return entry64<true, false, true, true>();
    case 12: return entry64<true, true, false, false>();
    case 13: return entry64<true, true, false, true>();
    case 14: return entry64<true, true, true, false>();
    default: return entry64<true, true, true, true>();
  }
}

}  // namespace dg16
