// Kernel instances for fp32 inputs multiplied as tf32 (tcgen05 kind::tf32),
// fp32 accumulate, fp32 out: 128 x 256 tiles (4-stage ring) and 128 x 128
// tiles (6-stage ring), B row- or column-major.  A stage is 32 K elements
// (one 128-byte swizzle row), so the rings have the bytes of the 16-bit ones.
#include "dispatch.h"
#include "gemm_kernel.cuh"

namespace dg16 {

template <int BN, int S, bool Q_MN>
static KernelEntry entry_tf32() {
  return {reinterpret_cast<const void*>(
              &gemm_tc_kernel<BN, S, Q_MN, false, float, false, false, true>),
          gemm_smem_bytes<BN, S, false>()};
}

KernelEntry kernels_tf32(int bn, bool q_mn) {
  if (bn == 256) return q_mn ? entry_tf32<256, 4, true>() : entry_tf32<256, 4, false>();
  if (bn == 128) return q_mn ? entry_tf32<128, 6, true>() : entry_tf32<128, 6, false>();
  return {nullptr, 0};
}

}  // namespace dg16
