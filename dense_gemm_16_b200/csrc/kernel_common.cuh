// kernel_common.cuh -- pieces shared by the single-CTA and CTA-pair GEMM
// kernels: launch parameters, the bounded mbarrier wait, type conversions
// and the tile scheduler's coordinate mapping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "ptx.cuh"
#include "raster.h"

namespace dg16 {


constexpr int kBM = 128;         // MMA rows per CTA
constexpr int kBK = 64;          // K elements per stage = one 128-byte swizzle row
constexpr int kThreads = 192;    // 6 warps
constexpr int kMaxGroups = 1024; // grouped GEMM: groups per launch

// Device status word codes (first error wins).
enum : unsigned {
  kStatusOk = 0,
  kStatusTimeoutProducer = 1,
  kStatusTimeoutMma = 2,
  kStatusTimeoutEpilogue = 3,
  kStatusTimeoutSelftest = 4,
  kStatusBadGroups = 16,
};

struct KParams {
  int M, N, K;            // dense: problem size; grouped: total rows, N, K
  int num_p, num_q;       // dense tile grid (P blocks x Q blocks)
  int num_kb;             // K blocks of kBK
  int group_m;            // raster group height
  long long num_tiles;    // dense tile count
  void* C;
  long long ldc;
  const void* bias;
  int epi;                // bit0 bias, bit1 relu
  const int* group_rows;  // grouped: device counts
  int num_groups;
  unsigned* status;       // device status word
  unsigned long long timeout_ns;
  int pol_p, pol_q;       // L2 policy of the P / Q operand copies (kPolicy*)
  // split-K: each tile's K blocks are cut into `splits` ranges of kb_per_split
  // blocks; partial fp32 tiles go to `ws` and the last range to finish sums
  // them (in range order) and runs the epilogue.  splits == 1: no split.
  int splits, kb_per_split;
  float* ws;              // [tile][split][128][BN] fp32 partials
  unsigned* counters;     // [tile] arrivals, left at 0 after every launch
};

enum : int { kPolicyNormal = 0, kPolicyFirst = 1, kPolicyLast = 2 };

__device__ __forceinline__ uint64_t make_policy(int code) {
  return code == kPolicyLast ? policy_evict_last()
         : code == kPolicyFirst ? policy_evict_first() : policy_evict_normal();
}

// Barrier among the four epilogue warps only (named barrier 1).
__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

struct SharedCtl {
  int abort;
  unsigned tmem_base;
  int last;  // split-K: this block finishes the current tile
  int pad;
};

// Bounded wait on an mbarrier phase.  Returns false when the block is
// aborting (another warp gave up) or when this wait itself ran out, in which
// case it records `code` and raises the block's abort flag.
// CLUSTER selects cluster-scope acquire, for barriers that another CTA of
// the pair arrives on.
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, SharedCtl* ctl,
                                           const KParams& p, unsigned code) {
  auto try_once = [&]() {
    return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (try_once()) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (try_once()) return true;
    if ((n & 63u) == 0) {
      if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
      if (global_timer_ns() - t0 > p.timeout_ns) {
        atomicCAS(p.status, 0u, code);
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag: used only to drain a block's
// own asynchronous work on the way out.
__device__ __forceinline__ bool wait_phase_drain(uint32_t bar, uint32_t parity,
                                                 unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_timer_ns() - t0 > limit_ns) return false;
  return true;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Pack two fp32 values into the 32-bit pair of the output type (RNE).
template <typename OutT>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename OutT>
__device__ __forceinline__ OutT from_f32(float v);
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }

// Where a tile lives.
struct TileCoord {
  int p0;        // first P row (dense: global; grouped: global row of A)
  int q0;        // first Q row
  int group;     // grouped: group index (0 otherwise)
  int row_end;   // grouped: one past the group's last global row
  bool valid;
};

// Grouped-GEMM schedule: per-group tile prefix and row starts, in shared memory.
struct GroupTable {
  int tile_start[kMaxGroups + 1];
  int row_start[kMaxGroups + 1];
};

template <bool GROUPED>
__device__ __forceinline__ TileCoord tile_coord(long long t, const KParams& p, int num_q_blocks,
                                                const GroupTable* gt, int& gcursor) {
  TileCoord c;
  c.group = 0;
  c.valid = true;
  if constexpr (!GROUPED) {
    int pb, qb;
    raster_tile(t, p.num_p, p.num_q, p.group_m, pb, qb);
    c.p0 = pb * kBM;
    c.q0 = qb;  // caller scales by BN
    c.row_end = p.M;
  } else {
    // tiles are visited in increasing order by each role, so walk forward
    while (gcursor < p.num_groups && t >= gt->tile_start[gcursor + 1]) ++gcursor;
    if (gcursor >= p.num_groups) {
      c.valid = false;
      return c;
    }
    const int g = gcursor;
    const int local = static_cast<int>(t - gt->tile_start[g]);
    const int rows = gt->row_start[g + 1] - gt->row_start[g];
    const int mblocks = (rows + kBM - 1) / kBM;
    int mb, nb;
    raster_tile(local, mblocks, num_q_blocks, p.group_m, mb, nb);
    c.group = g;
    c.p0 = gt->row_start[g] + mb * kBM;
    c.q0 = nb;
    c.row_end = min(gt->row_start[g + 1], p.M);
  }
  return c;
}

// Epilogue for one accumulator row held by this thread: TMEM columns
// [0, BN) of lane `prow - p0` become output row `prow`, columns q0 .. q0+BN:
// fp32 -> (+ bias[col]) -> (ReLU) -> round to OutT -> store.  Called by all
// 32 lanes of an epilogue warp (the TMEM loads are warp-collective); rows at
// or past row_end and columns at or past N are not stored.
template <int BN, typename InT, typename OutT>
__device__ __forceinline__ void store_acc_rows(uint32_t taddr, int prow, int row_end, int q0,
                                               const KParams& p, const InT* bias_g, bool relu,
                                               OutT* C) {
  const bool row_ok = prow < row_end;
  OutT* crow = C + static_cast<long long>(prow) * p.ldc;
#pragma unroll 1
  for (int cc = 0; cc < BN; cc += 32) {
    const int col0 = q0 + cc;
    if (col0 >= p.N) break;  // warp-uniform
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + cc, v);
    tmem_ld_wait();
    float f[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float x = __uint_as_float(v[j]);
      if (bias_g != nullptr && col0 + j < p.N) x += to_f32<InT>(bias_g[col0 + j]);
      if (relu) x = fmaxf(x, 0.0f);
      f[j] = x;
    }
    if (row_ok) {
      if (col0 + 32 <= p.N) {
        if constexpr (sizeof(OutT) == 2) {
          uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack2<OutT>(f[8 * j + 0], f[8 * j + 1]),
                                pack2<OutT>(f[8 * j + 2], f[8 * j + 3]),
                                pack2<OutT>(f[8 * j + 4], f[8 * j + 5]),
                                pack2<OutT>(f[8 * j + 6], f[8 * j + 7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(crow + col0);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < p.N) crow[col0 + j] = from_f32<OutT>(f[j]);
      }
    }
  }
}

// Sum of 16 consecutive fp32 values over `splits` partial tiles `stride`
// floats apart, in split order (so the result does not depend on which
// block finished last).
__device__ __forceinline__ void sum_partials16(const float* src, int splits, long long stride,
                                               float (&f)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) f[j] = 0.0f;
  for (int s = 0; s < splits; ++s) {
    const float4* q = reinterpret_cast<const float4*>(src + s * stride);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = __ldcg(q + j);
      f[4 * j] += v.x;
      f[4 * j + 1] += v.y;
      f[4 * j + 2] += v.z;
      f[4 * j + 3] += v.w;
    }
  }
}

// Split-K finish for one output row: sum the partial rows (row-major
// [split][128][BN] fp32 starting at `base` for this row), then bias, ReLU,
// cast and store exactly like store_acc_rows.
template <int BN, typename InT, typename OutT>
__device__ __forceinline__ void store_partial_sums(const float* base, int splits, int prow,
                                                   int row_end, int q0, const KParams& p,
                                                   const InT* bias_g, bool relu, OutT* C) {
  const bool row_ok = prow < row_end;
  OutT* crow = C + static_cast<long long>(prow) * p.ldc;
  const long long stride = static_cast<long long>(kBM) * BN;
#pragma unroll 1
  for (int cc = 0; cc < BN; cc += 16) {
    const int col0 = q0 + cc;
    if (col0 >= p.N || !row_ok) break;
    float f[16];
    sum_partials16(base + cc, splits, stride, f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (bias_g != nullptr && col0 + j < p.N) f[j] += to_f32<InT>(bias_g[col0 + j]);
      if (relu) f[j] = fmaxf(f[j], 0.0f);
    }
    if (col0 + 16 <= p.N) {
      if constexpr (sizeof(OutT) == 2) {
        uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
        for (int j = 0; j < 2; ++j)
          dst[j] = make_uint4(pack2<OutT>(f[8 * j + 0], f[8 * j + 1]),
                              pack2<OutT>(f[8 * j + 2], f[8 * j + 3]),
                              pack2<OutT>(f[8 * j + 4], f[8 * j + 5]),
                              pack2<OutT>(f[8 * j + 6], f[8 * j + 7]));
      } else {
        float4* dst = reinterpret_cast<float4*>(crow + col0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (col0 + j < p.N) crow[col0 + j] = from_f32<OutT>(f[j]);
    }
  }
}

}  // namespace dg16
