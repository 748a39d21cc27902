// im2col.cu -- 2-D convolution on the GEMM core ("FlagOS众智跨芯算子优化实践"
// section 5.3: convolution becomes a GEMM through im2col and reuses its
// optimisations).
//
// conv2d_im2col gathers the sliding windows of an NHWC input into an
// M x K matrix (M = batch*OH*OW output pixels, K = KH*KW*cin taps, k running
// kh, kw, ci), then runs the tcgen05 GEMM of gemm_api.cu with the filter
// [KH][KW][cin][cout] as the K x N operand and the NHWC output as C, so bias
// and ReLU fuse into the GEMM's epilogue.  The gather is a memory-bound
// copy: one thread per 8 consecutive taps (16-byte loads and stores when
// cin is a multiple of 8), coalesced along K.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "dispatch.h"

namespace dg16 {

// A[m][k] (leading dimension lda) for output pixel m and tap k; 0 where the
// window falls into the zero padding.  VEC: cin % 8 == 0, so the 8 taps of a
// thread share (kh, kw) and are 8 consecutive input channels.
template <bool VEC>
__global__ void im2col_nhwc_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ A,
                                   long long lda, int batch, int H, int W, int cin, int KH, int KW,
                                   int sh, int sw, int ph, int pw, int dh, int dw, int OH, int OW) {
  const int K = KH * KW * cin;
  const int groups = (K + 7) / 8;  // 8-tap groups per row
  const long long total = static_cast<long long>(batch) * OH * OW * groups;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = i / groups;
    const int k0 = static_cast<int>(i - m * groups) * 8;
    const int n = static_cast<int>(m / (static_cast<long long>(OH) * OW));
    const int oh = static_cast<int>((m / OW) % OH);
    const int ow = static_cast<int>(m % OW);
    uint16_t* dst = A + m * lda + k0;
    if constexpr (VEC) {
      const int ci = k0 % cin;
      const int tap = k0 / cin;
      const int kh = tap / KW, kw = tap % KW;
      const int ih = oh * sh - ph + kh * dh, iw = ow * sw - pw + kw * dw;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (ih >= 0 && ih < H && iw >= 0 && iw < W)
        v = *reinterpret_cast<const uint4*>(x + ((static_cast<long long>(n) * H + ih) * W + iw) *
                                                    cin + ci);
      *reinterpret_cast<uint4*>(dst) = v;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = k0 + j;
        if (k >= K) break;
        const int ci = k % cin;
        const int tap = k / cin;
        const int kh = tap / KW, kw = tap % KW;
        const int ih = oh * sh - ph + kh * dh, iw = ow * sw - pw + kw * dw;
        uint16_t v = 0;
        if (ih >= 0 && ih < H && iw >= 0 && iw < W)
          v = x[((static_cast<long long>(n) * H + ih) * W + iw) * cin + ci];
        dst[j] = v;
      }
    }
  }
}

cudaError_t launch_im2col(const void* x, void* A, long long lda, int batch, int H, int W, int cin,
                          int KH, int KW, int sh, int sw, int ph, int pw, int dh, int dw, int OH,
                          int OW, int num_sms, cudaStream_t stream) {
  const long long total = static_cast<long long>(batch) * OH * OW * ((KH * KW * cin + 7) / 8);
  const int blocks = static_cast<int>(
      std::min<long long>((total + 255) / 256, static_cast<long long>(num_sms) * 16));
  if (cin % 8 == 0)
    im2col_nhwc_kernel<true><<<blocks, 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), static_cast<uint16_t*>(A), lda, batch, H, W, cin, KH, KW,
        sh, sw, ph, pw, dh, dw, OH, OW);
  else
    im2col_nhwc_kernel<false><<<blocks, 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), static_cast<uint16_t*>(A), lda, batch, H, W, cin, KH, KW,
        sh, sw, ph, pw, dh, dw, OH, OW);
  return cudaGetLastError();
}

}  // namespace dg16
