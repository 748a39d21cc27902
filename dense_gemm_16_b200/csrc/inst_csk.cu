// Kernel instances of the CTA-pair split-K GEMM (one tile per pair, the two
// halves of K reduced through distributed shared memory).  Per CTA: the ring,
// the 32 KB epilogue staging and a 128 x BN fp32 receive buffer.
#include "dispatch.h"
#include "gemm_kernel_csk.cuh"

namespace dg16 {

template <int BN, int S, bool Q_MN, bool BF16, bool F32, bool SWAP = false>
static KernelEntry entry_csk() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  return {reinterpret_cast<const void*>(&gemm_csk_kernel<BN, S, Q_MN, BF16, Out, SWAP>),
          gemm_csk_smem_bytes<BN, S>()};
}

template <int BN, int S>
static KernelEntry pick_csk(bool q_mn, bool bf16, bool out_f32) {
  const int key = (q_mn ? 4 : 0) | (bf16 ? 2 : 0) | (out_f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_csk<BN, S, false, false, false>();
    case 1: return entry_csk<BN, S, false, false, true>();
    case 2: return entry_csk<BN, S, false, true, false>();
    case 3: return entry_csk<BN, S, false, true, true>();
    case 4: return entry_csk<BN, S, true, false, false>();
    case 5: return entry_csk<BN, S, true, false, true>();
    case 6: return entry_csk<BN, S, true, true, false>();
    default: return entry_csk<BN, S, true, true, true>();
  }
}

// 128 x 128 tiles: 4 stages (128 KB) + 32 KB staging + 64 KB receive buffer;
// 128 x 64 tiles: 6 stages (144 KB) + 32 KB + 32 KB.
KernelEntry kernels_csk(int bn, bool q_mn, bool bf16, bool out_f32) {
  if (bn == 128) return pick_csk<128, 4>(q_mn, bf16, out_f32);
  if (bn == 64) return pick_csk<64, 6>(q_mn, bf16, out_f32);
  return {nullptr, 0};
}

// Swapped (skinny, column-major B): 128 columns of B x 16 rows of A per
// tile, a 10-stage ring of 18 KB.
KernelEntry kernels_csk_swap(int bn, bool bf16, bool out_f32) {
  if (bn != 16) return {nullptr, 0};
  const int key = (bf16 ? 2 : 0) | (out_f32 ? 1 : 0);
  switch (key) {
    case 0: return entry_csk<16, 10, false, false, false, true>();
    case 1: return entry_csk<16, 10, false, false, true, true>();
    case 2: return entry_csk<16, 10, false, true, false, true>();
    default: return entry_csk<16, 10, false, true, true, true>();
  }
}

}  // namespace dg16
