// Kernel instances of the CTA-pair GEMM for grouped problems: 256 x 512 pair
// tiles with a 4-deep ring and 256 x 256 pair tiles with a 6-deep ring.
// Grouped tiles store from registers, so the 32 KB epilogue staging area
// gives way to the group table.
#include "dispatch.h"
#include "gemm_kernel_pair.cuh"

namespace dg16 {

template <int BN, int NS, int S, bool Q_MN, bool BF16, bool F32>
static KernelEntry entry_pair_g() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  return {reinterpret_cast<const void*>(&gemm_tc2_kernel<BN, NS, S, Q_MN, BF16, Out, true>),
          gemm_pair_smem_bytes<BN, NS, S, true>()};
}

template <int BN, int NS, int S>
static KernelEntry pick_g(bool q_mn, bool bf16, bool f32) {
  const int key = (q_mn ? 4 : 0) | (bf16 ? 2 : 0) | (f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_pair_g<BN, NS, S, false, false, false>();
    case 1: return entry_pair_g<BN, NS, S, false, false, true>();
    case 2: return entry_pair_g<BN, NS, S, false, true, false>();
    case 3: return entry_pair_g<BN, NS, S, false, true, true>();
    case 4: return entry_pair_g<BN, NS, S, true, false, false>();
    case 5: return entry_pair_g<BN, NS, S, true, false, true>();
    case 6: return entry_pair_g<BN, NS, S, true, true, false>();
    default: return entry_pair_g<BN, NS, S, true, true, true>();
  }
}

// bn = output columns per pair tile (256 x bn)
KernelEntry kernels_pair_grouped(int bn, bool q_mn, bool bf16, bool out_f32) {
  if (bn == 512) return pick_g<256, 2, 4>(q_mn, bf16, out_f32);
  if (bn == 256) return pick_g<256, 1, 6>(q_mn, bf16, out_f32);
  return {nullptr, 0};
}

}  // namespace dg16
