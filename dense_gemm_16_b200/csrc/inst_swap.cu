// Kernel instances for skinny problems (few rows of A, column-major B):
// C^T = B^T . A^T with the wide N dimension on the 128 MMA rows and M on the
// MMA's N (16 or 32), an 8-deep ring to keep enough bytes in flight.
#include "dispatch.h"
#include "gemm_kernel.cuh"

namespace dg16 {

template <int BN, bool BF16, bool F32>
static KernelEntry entry_swap() {
  using In = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using Out = typename std::conditional<F32, float, In>::type;
  constexpr int S = 8;
  return {reinterpret_cast<const void*>(&gemm_tc_kernel<BN, S, false, BF16, Out, true, false>),
          gemm_smem_bytes<BN, S, false, true>()};
}

KernelEntry kernels_swap(int bn, bool bf16, bool out_f32) {
  const int key = (bf16 ? 2 : 0) | (out_f32 ? 1 : 0);
  if (bn == 16) {
    switch (key) {
      case 0: return entry_swap<16, false, false>();
      case 1: return entry_swap<16, false, true>();
      case 2: return entry_swap<16, true, false>();
      default: return entry_swap<16, true, true>();
    }
  }
  if (bn == 32) {
    switch (key) {
      case 0: return entry_swap<32, false, false>();
      case 1: return entry_swap<32, false, true>();
      case 2: return entry_swap<32, true, false>();
      default: return entry_swap<32, true, true>();
    }
  }
  return {nullptr, 0};
}

}  // namespace dg16
