// Kernel instances of the CTA-pair GEMM: 256 x 512 pair tiles (two N=256
// MMAs per K step, one 512-column accumulator) with a 4-deep ring of 48 KB
// stages; 256 x 256 pair tiles with a 6-deep ring (32 KB per stage per CTA);
// 256 x 128 pair tiles with an 8-deep ring.  Each ring plus the 32 KB
// epilogue staging area fits the 227 KB a block may use.
#include "dispatch.h"
#include "gemm_kernel_pair.cuh"

namespace dg16 {

template <int BN, int NS, int S, bool Q_MN, bool BF16, bool F32>
static KernelEntry entry_pair() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  return {reinterpret_cast<const void*>(&gemm_tc2_kernel<BN, NS, S, Q_MN, BF16, Out>),
          gemm_pair_smem_bytes<BN, NS, S>()};
}

template <int BN, int NS, int S>
static KernelEntry pick(bool q_mn, bool bf16, bool f32) {
  const int key = (q_mn ? 4 : 0) | (bf16 ? 2 : 0) | (f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_pair<BN, NS, S, false, false, false>();
    case 1: return entry_pair<BN, NS, S, false, false, true>();
    case 2: return entry_pair<BN, NS, S, false, true, false>();
    case 3: return entry_pair<BN, NS, S, false, true, true>();
    case 4: return entry_pair<BN, NS, S, true, false, false>();
    case 5: return entry_pair<BN, NS, S, true, false, true>();
    case 6: return entry_pair<BN, NS, S, true, true, false>();
    default: return entry_pair<BN, NS, S, true, true, true>();
  }
}

// bn = output columns per pair tile (256 x bn)
KernelEntry kernels_pair(int bn, int stages, bool q_mn, bool bf16, bool out_f32) {
  if (bn == 512) return pick<256, 2, 4>(q_mn, bf16, out_f32);
  if (bn == 256) return pick<256, 1, 6>(q_mn, bf16, out_f32);
  if (bn == 128) return pick<128, 1, 8>(q_mn, bf16, out_f32);
  return {nullptr, 0};
}

}  // namespace dg16
