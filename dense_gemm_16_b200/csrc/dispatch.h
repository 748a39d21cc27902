// dispatch.h -- the compiled kernel instances and the tile-config table.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace dg16 {

// What a launch needs to know about one compiled kernel instance.
struct KernelEntry {
  const void* fn;  // __global__ function
  int smem;        // dynamic shared memory bytes
};

enum ConfigKind : int {
  kKindSingle = 0,  // one CTA per 128 x BN tile
  kKindSwap = 1,    // skinny problems: C^T = B^T A^T, N fills the MMA rows
  kKindPair = 2,    // two CTAs (cta_group::2) per 256 x BN tile
  kKindGroupedSwap = 3,  // grouped only: Y_g^T tiles of 128 columns x <= bn rows,
                         // sized per group, drawn from a dynamic tile queue
  kKindGroupedSwapPair = 4,  // the same with a CTA pair per 256 columns x <= bn rows
  kKindClusterSplitK = 5,    // dense, tiles <= SMs / 2: a CTA pair per 128 x bn tile,
                             // one half of K each, reduced in distributed shared memory
  kKindClusterSplitKSwap = 6,  // the same for skinny problems, operands swapped (C^T)
};

struct Config {
  const char* name;
  int kind;
  int bn;       // MMA N (Q rows per tile)
  int stages;   // operand ring depth
  int group_m;  // raster band height
  int splits;   // split-K factor (1 = whole K per tile; -1 = stream-K; -2 = hybrid
                //  stream-K over the last waves' tiles)
  int pol_p;    // L2 eviction policy of the 128-row operand's copies (kPolicy*)
  int pol_q;    // ... and of the BN-row operand's copies
};

// Instances, one getter per translation unit (so they compile in parallel).
// Each returns {nullptr, 0} for a combination that was not compiled.
KernelEntry kernels_bn256(bool q_mn, bool bf16, bool out_f32, bool grouped);
KernelEntry kernels_bn128(bool q_mn, bool bf16, bool out_f32, bool grouped);
KernelEntry kernels_bn64(bool q_mn, bool bf16, bool out_f32, bool grouped);
KernelEntry kernels_swap(int bn, bool bf16, bool out_f32);
KernelEntry kernels_pair(int bn, int stages, bool q_mn, bool bf16, bool out_f32);
KernelEntry kernels_pair_grouped(int bn, bool q_mn, bool bf16, bool out_f32);
KernelEntry kernels_tf32(int bn, bool q_mn);
KernelEntry kernels_gswap(int tok, bool p_mn, bool bf16, bool out_f32);
KernelEntry kernels_gswap2(int tok, bool p_mn, bool bf16, bool out_f32);
KernelEntry kernels_csk(int bn, bool q_mn, bool bf16, bool out_f32);
KernelEntry kernels_csk_swap(int bn, bool bf16, bool out_f32);

// NHWC im2col gather (im2col.cu): A[m][k] for M = batch*OH*OW, K = KH*KW*cin.
cudaError_t launch_im2col(const void* x, void* A, long long lda, int batch, int H, int W, int cin,
                          int KH, int KW, int sh, int sw, int ph, int pw, int dh, int dw, int OH,
                          int OW, int num_sms, cudaStream_t stream);

}  // namespace dg16
