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
  // Work distribution (see WorkIter):
  //   work_mode 0  whole tiles
  //   work_mode 1  split-K: each tile's K blocks in `splits` ranges of
  //                kb_per_split blocks
  //   work_mode 2  stream-K: block b takes iterations [b*sk_width,
  //                (b+1)*sk_width) of the (tile, K block) space
  //   work_mode 3  hybrid: stream-K over the tiles of the last waves, whole
  //                tiles for the rest (see WorkIter)
  // A tile computed in several pieces parks fp32 partial tiles in `ws`
  // (slot tile*slot_stride + piece) and the last piece to finish sums them
  // in piece order and runs the epilogue.
  int work_mode;
  int splits, kb_per_split;
  long long sk_width;
  int slot_stride;
  float* ws;              // [slot][BN/4][128][4] fp32 partials
  unsigned* counters;     // [tile] arrivals, left at 0 after every launch
  // 1: store output tiles with TMA (set only when a row of C ends on a
  // 16-byte boundary, N * sizeof(out) % 16 == 0: a TMA store writes whole
  // 16-byte granules, so a shorter row end would spill into the padding)
  int tma_store;
  // Strided batches (dense kernels): tile t belongs to batch t / tiles_per_batch.
  // The operand maps are 3-D with the batch as the third coordinate; an
  // operand shared by all batches (stride 0) has z_p or z_q == 0.
  long long tiles_per_batch;
  int z_p, z_q;           // 1: the P / Q operand advances with the batch
  long long stride_c;     // elements between batches' outputs
  long long stride_bias;  // elements between batches' bias vectors
  // Optional tracing: when non-null, blocks below trace_blocks write the
  // global timer at each event into trace[block * kTraceEvents + event].
  unsigned long long* trace;
  int trace_blocks;
};

// Trace events (the same numbering as the GEMM_TRACE_* constants of the C ABI).
enum : int {
  kTrEntry = 0, kTrSetup = 1, kTrFirstLoad = 2, kTrFirstData = 3,
  kTrLastMma = 4, kTrFirstEpi = 5, kTrEpiDone = 6, kTrExit = 7, kTraceEvents = 8
};

enum : int { kPolicyNormal = 0, kPolicyFirst = 1, kPolicyLast = 2 };

// Record the global timer for trace event `ev` of this block (one thread
// calls it; a no-op unless tracing is on).
__device__ __forceinline__ void trace_mark(const KParams& p, int ev) {
  if (p.trace != nullptr && static_cast<int>(blockIdx.x) < p.trace_blocks)
    p.trace[static_cast<long long>(blockIdx.x) * kTraceEvents + ev] = global_timer_ns();
}

__device__ __forceinline__ uint64_t make_policy(int code) {
  return code == kPolicyLast ? policy_evict_last()
         : code == kPolicyFirst ? policy_evict_first() : policy_evict_normal();
}

// Barrier among the four epilogue warps only (named barrier 1).
__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// The same barrier, returning whether `pred` held in any of the 128 threads:
// one answer for all of them, so the four warps always take the same branch.
__device__ __forceinline__ bool epilogue_bar_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

// One unit of work: K blocks [kb0, kb1) of output tile t, piece `idx` of
// the `count` pieces that together cover the tile's K range.
struct Work {
  long long t;
  int kb0, kb1;
  int idx, count;
};

// The sequence of work units one block processes, in the same order for the
// producer, the MMA issuer and the epilogue.
//   work_mode 0: whole tiles t = block, block + grid, ...
//   work_mode 1: split-K units (tile, split), strided the same way
//   work_mode 2: stream-K: block b takes iterations [b*W, (b+1)*W) of the
//                (tile, K block) space, W = sk_width
//   work_mode 3: hybrid: stream-K over the first sk_tiles tiles (the tiles
//                that do not fill whole waves, plus one wave), then whole
//                tiles sk_tiles + block, + grid, ... for the rest, so most
//                of the work keeps the raster's L2 locality
struct WorkIter {
  long long cursor, end, step;
  long long sk_width;  // stream-K: iterations per unit
  long long dp_cursor, dp_end;  // hybrid: the whole tiles after the stream-K part
  long long unit, units;        // this block (or CTA pair) and how many there are
  // width: the stream-K width, p.sk_width unless the kernel derived it from
  // a tile count it computed itself; sk_tiles: the hybrid's stream-K tiles;
  // unit / units: the worker index and count (default: the block and grid;
  // the CTA-pair kernel passes its pair index and pair count)
  __device__ __forceinline__ WorkIter(const KParams& p, long long num_tiles, long long width = 0,
                                      long long sk_tiles = 0, long long unit_ = -1,
                                      long long units_ = -1) {
    unit = unit_ >= 0 ? unit_ : static_cast<long long>(blockIdx.x);
    units = units_ > 0 ? units_ : static_cast<long long>(gridDim.x);
    sk_width = width > 0 ? width : p.sk_width;
    dp_cursor = 0;
    dp_end = 0;
    if (p.work_mode == 2 || p.work_mode == 3) {
      const long long total = (p.work_mode == 3 ? sk_tiles : num_tiles) * p.num_kb;
      cursor = unit * sk_width;
      end = min(total, cursor + sk_width);
      step = 0;
      if (p.work_mode == 3) {
        dp_cursor = sk_tiles + unit;
        dp_end = num_tiles;
      }
    } else {
      const long long n = p.work_mode == 1 ? num_tiles * p.splits : num_tiles;
      cursor = unit;
      end = n;
      step = units;
    }
  }
  __device__ __forceinline__ bool next(const KParams& p, Work& w) {
    if (cursor >= end) {
      if (p.work_mode != 3 || dp_cursor >= dp_end) return false;
      w.t = dp_cursor;
      w.idx = 0;
      w.count = 1;
      w.kb0 = 0;
      w.kb1 = p.num_kb;
      dp_cursor += units;
      return true;
    }
    if (p.work_mode >= 2) {
      const long long nkb = p.num_kb;
      w.t = cursor / nkb;
      w.kb0 = static_cast<int>(cursor - w.t * nkb);
      w.kb1 = static_cast<int>(min(nkb, static_cast<long long>(w.kb0) + (end - cursor)));
      const long long first = (w.t * nkb) / sk_width;
      const long long last = ((w.t + 1) * nkb - 1) / sk_width;
      w.idx = static_cast<int>(unit - first);
      w.count = static_cast<int>(last - first + 1);
      cursor += w.kb1 - w.kb0;
    } else if (p.work_mode == 1) {
      w.t = cursor / p.splits;
      w.idx = static_cast<int>(cursor - w.t * p.splits);
      w.count = p.splits;
      w.kb0 = w.idx * p.kb_per_split;
      w.kb1 = min(w.kb0 + p.kb_per_split, p.num_kb);
      cursor += step;
    } else {
      w.t = cursor;
      w.idx = 0;
      w.count = 1;
      w.kb0 = 0;
      w.kb1 = p.num_kb;
      cursor += step;
    }
    return true;
  }
};

// The hybrid split of work_mode 3 for `num_tiles` tiles on `workers` (the
// grid's blocks unless given; the CTA-pair kernel passes its pairs): the
// tiles past whole waves, plus one whole wave when there are two or more,
// go to stream-K (*sk_tiles, over which each block takes *sk_width
// iterations); the rest run as whole tiles.  Every role computes the same.
__device__ __forceinline__ void hybrid_split(long long num_tiles, int num_kb, long long* sk_tiles,
                                             long long* sk_width, long long workers = -1) {
  const long long g = workers > 0 ? workers : static_cast<long long>(gridDim.x);
  const long long waves = num_tiles / g;
  const long long dp = (num_tiles % g == 0) ? num_tiles : (waves >= 2 ? (waves - 1) * g : 0);
  *sk_tiles = num_tiles - dp;
  *sk_width = max(1ll, (*sk_tiles * num_kb + g - 1) / g);
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
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }

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
  int p0;        // first P row (dense: within the batch; grouped: global row of A)
  int q0;        // first Q block (caller scales by BN)
  int group;     // grouped: group index; dense: batch index
  int zp, zq;    // third TMA coordinate of the P and Q copies
  int row_end;   // one past the last output row this tile may store
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
    const long long b = t / p.tiles_per_batch;
    int pb, qb;
    raster_tile(t - b * p.tiles_per_batch, p.num_p, p.num_q, p.group_m, pb, qb);
    c.p0 = pb * kBM;
    c.q0 = qb;  // caller scales by BN
    c.group = static_cast<int>(b);
    c.zp = static_cast<int>(b) * p.z_p;
    c.zq = static_cast<int>(b) * p.z_q;
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
    c.zp = 0;
    c.zq = g;
    c.p0 = gt->row_start[g] + mb * kBM;
    c.q0 = nb;
    c.row_end = min(gt->row_start[g + 1], p.M);
  }
  return c;
}


// Scratch slot (in partial tiles) of piece s of split tile t, whose piece 0
// is processed by block first_block:
//   split-K: slot t * slot_stride + s;
//   stream-K: two slots per block, one for the tile its range starts inside
//   (a piece s > 0) and one for the tile its range ends inside (piece 0), so
//   the scratch is 2 x grid partial tiles whatever the tile count.
// With `ranks` CTAs per worker (the CTA pair: 2), each rank keeps its own
// slots: slot * ranks + rank.
__device__ __forceinline__ long long piece_slot(const KParams& p, long long t, int s,
                                                long long first_block, int rank = 0,
                                                int ranks = 1) {
  const long long base =
      p.work_mode >= 2 ? 2 * (first_block + s) + (s > 0 ? 0 : 1) : t * p.slot_stride + s;
  return base * ranks + rank;
}

// Partial tiles are laid out [BN/4][128 rows][4 floats] so that the 32
// lanes of a warp, which hold 32 consecutive rows, touch 512 contiguous
// bytes per float4 access.

// Write 16 raw fp32 accumulator values (columns cc .. cc+15 of this thread's
// row) into a partial tile.
__device__ __forceinline__ void put_partial16(float* tile, int row, int cc, const uint32_t (&v)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    __stcg(reinterpret_cast<float4*>(tile) + (static_cast<long long>(cc / 4 + j) * kBM + row),
           make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                       __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
}

// Epilogue for one accumulator row held by this thread, from any source of
// raw fp32 values: src.get<16>(cc, v) fills v[0..15] with columns cc .. cc+15
// of the row (a warp-collective TMEM load, or a partial-tile sum).  Output row
// `prow`, columns q0 .. q0+TILE_N: + bias[col] -> ReLU -> round to OutT ->
// store from registers.  Rows at or past row_end and columns at or past N are
// not stored.  Called by all 32 lanes of an epilogue warp.
template <int TILE_N, typename InT, typename OutT, typename Src>
__device__ __forceinline__ void store_rows_from(Src&& src, int prow, int row_end, int q0,
                                                const KParams& p, const InT* bias_g, bool relu,
                                                OutT* C) {
  const bool row_ok = prow < row_end;
  OutT* crow = C + static_cast<long long>(prow) * p.ldc;
#pragma unroll 1
  for (int cc = 0; cc < TILE_N; cc += 16) {
    const int col0 = q0 + cc;
    if (col0 >= p.N) break;  // warp-uniform
    // the bias loads go out before the accumulator read, so their latency overlaps it
    float bv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      bv[j] = (bias_g != nullptr && col0 + j < p.N) ? to_f32<InT>(bias_g[col0 + j]) : 0.0f;
    uint32_t v[16];
    src.template get<16>(cc, v);
    float f[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float x = __uint_as_float(v[j]);
      if (bias_g != nullptr) x += bv[j];
      if (relu) x = fmaxf(x, 0.0f);
      f[j] = x;
    }
    if (!row_ok) continue;
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

// Bytes of the epilogue staging area: 4 epilogue warps x 2 buffers x one
// 32-row box of 128-byte rows (4 KB).
constexpr uint32_t kEpiStageBytes = 4 * 2 * 4096;

// Epilogue through shared memory and TMA stores, for one warp's 32
// accumulator rows (TMEM lanes of this warp's quadrant, output rows
// row0 .. row0+31) and output columns q0 .. q0+TILE_N.  Each pass takes 128
// bytes of every row (64 16-bit or 32 fp32 outputs): TMEM -> registers ->
// bias, ReLU, round -> a 128B-swizzled 32 x 128 B staging buffer (16-byte
// chunk c of row r at chunk c ^ (r % 8), so the eight rows of a store phase hit
// eight different bank groups) -> one lane issues a TMA store of the box (at
// batch z of the 3-D output map), which clips rows >= M and columns >= N.  Two buffers per warp alternate;
// `count` carries the warp's store count across tiles.  Called by all 32
// lanes of the warp.
template <int TILE_N, typename InT, typename OutT, typename Src>
__device__ __forceinline__ void store_tma_from(Src&& src, int row0, int q0, int z,
                                               const KParams& p, const InT* bias, bool relu,
                                               uint32_t stage, uint32_t& count,
                                               const CUtensorMap* tmC) {
  constexpr int CH = 128 / static_cast<int>(sizeof(OutT));  // outputs per 128-byte row chunk
  const int lane = threadIdx.x & 31;
  // a box must start inside the tensor: a slab wholly below the last row
  // stores nothing (warp-uniform)
  if (row0 >= p.M) return;
#pragma unroll 1
  for (int c0 = 0; c0 < TILE_N; c0 += CH) {
    const int col0 = q0 + c0;
    if (col0 >= p.N) break;  // warp-uniform
    // the bias loads go out before the accumulator read, so their latency overlaps it
    float bv[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j)
      bv[j] = (bias != nullptr && col0 + j < p.N) ? to_f32<InT>(bias[col0 + j]) : 0.0f;
    uint32_t v[CH];
    src.template get<CH>(c0, v);
    uint32_t packed[32];
    if constexpr (sizeof(OutT) == 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x0 = __uint_as_float(v[2 * j]), x1 = __uint_as_float(v[2 * j + 1]);
        if (bias != nullptr) {
          x0 += bv[2 * j];
          x1 += bv[2 * j + 1];
        }
        if (relu) {
          x0 = fmaxf(x0, 0.0f);
          x1 = fmaxf(x1, 0.0f);
        }
        packed[j] = pack2<OutT>(x0, x1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x = __uint_as_float(v[j]);
        if (bias != nullptr) x += bv[j];
        if (relu) x = fmaxf(x, 0.0f);
        packed[j] = __float_as_uint(x);
      }
    }
    // the buffer written two stores ago must have been read by its TMA store
    if (count >= 2) {
      if (lane == 0) tma_store_wait_read<1>();
      __syncwarp();
    }
    const uint32_t buf = stage + (count & 1u) * 4096u;
    const uint32_t row_addr = buf + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t dst = row_addr + ((static_cast<uint32_t>(c) ^ (lane & 7u)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[4 * c]),
                   "r"(packed[4 * c + 1]), "r"(packed[4 * c + 2]), "r"(packed[4 * c + 3])
                   : "memory");
    }
    fence_proxy_async_shared();  // these generic writes -> the TMA (async proxy) read
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(tmC, buf, col0, row0, z);
      tma_store_commit();
    }
    ++count;
  }
}

// A tile's bias columns q0 .. q0+TILE_N held across the warp: lane l keeps
// columns q0+16l .. q0+16l+15 as raw values (16-bit types two to a word,
// fp32 one to a word; zero past N).  Loaded once per tile before the
// epilogue waits for the accumulator, so the load latency hides behind the
// tile's MMAs; the epilogue then reads any column pair by warp shuffle.
template <int TILE_N, typename InT>
struct BiasRegs {
  static_assert(TILE_N <= 512, "16 columns per lane");
  static constexpr bool F32 = sizeof(InT) == 4;
  static constexpr int WORDS = F32 ? 16 : 8;
  uint32_t w[WORDS];
  __device__ __forceinline__ void load(const InT* bias, int q0, int N) {
    const int lane = threadIdx.x & 31;
    const int col = q0 + 16 * lane;
#pragma unroll
    for (int i = 0; i < WORDS; ++i) w[i] = 0u;
    if (bias == nullptr || 16 * lane >= TILE_N || col >= N) return;
    const InT* src = bias + col;
    if (col + 16 <= N && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
#pragma unroll
      for (int i = 0; i < WORDS / 4; ++i) {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(src) + i);
        w[4 * i] = a.x;
        w[4 * i + 1] = a.y;
        w[4 * i + 2] = a.z;
        w[4 * i + 3] = a.w;
      }
    } else if constexpr (F32) {
      const uint32_t* s32 = reinterpret_cast<const uint32_t*>(src);
#pragma unroll
      for (int k = 0; k < 16; ++k) w[k] = col + k < N ? s32[k] : 0u;
    } else {
      const unsigned short* s16 = reinterpret_cast<const unsigned short*>(src);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint32_t h = col + k < N ? static_cast<uint32_t>(s16[k]) : 0u;
        w[k / 2] |= h << (16 * (k & 1));
      }
    }
  }
  // the bias of tile columns col, col+1 (col even); called by the whole warp
  __device__ __forceinline__ void pair(int col, float& lo, float& hi) const {
    if constexpr (F32) {
      lo = __uint_as_float(__shfl_sync(0xffffffffu, w[col & 15], col >> 4));
      hi = __uint_as_float(__shfl_sync(0xffffffffu, w[(col & 15) + 1], col >> 4));
    } else {
      const uint32_t x = __shfl_sync(0xffffffffu, w[(col & 15) >> 1], col >> 4);
      if constexpr (std::is_same<InT, __nv_bfloat16>::value) {
        lo = __uint_as_float(x << 16);
        hi = __uint_as_float(x & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&x));
        lo = f.x;
        hi = f.y;
      }
    }
  }
};

// store_tma_from with the chunk loop unrolled and the bias taken from
// registers loaded ahead of time (BIAS: add `br`), so each chunk's source
// read, rounding, staging and TMA store are straight-line code with no
// global load on the way.  Measured on the 256 x 512 pair tile, whose MMA
// waits for this store: 5 us per tile against 8.8 us for the generic loop.
template <int TILE_N, typename InT, typename OutT, bool BIAS, typename Src>
__device__ __forceinline__ void store_tile_from(const Src& src, int row0, int q0, int z,
                                                const KParams& p, const BiasRegs<TILE_N, InT>& br,
                                                bool relu, uint32_t stage, uint32_t& count,
                                                const CUtensorMap* tmC) {
  constexpr int CH = 128 / static_cast<int>(sizeof(OutT));  // outputs per 128-byte row chunk
  constexpr int NCH = TILE_N / CH;
  static_assert(TILE_N % CH == 0, "whole chunks");
  const int lane = threadIdx.x & 31;
  // chunks with columns inside the matrix; none for a slab wholly below the
  // last row (a box must start inside the tensor).  Warp-uniform.
  const int nch = row0 >= p.M ? 0 : max(0, min(NCH, (p.N - q0 + CH - 1) / CH));
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c >= nch) break;  // warp-uniform
    const int col0 = q0 + c * CH;
    uint32_t v[CH];
    src.template get<CH>(c * CH, v);
    uint32_t packed[32];
    if constexpr (sizeof(OutT) == 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x0 = __uint_as_float(v[2 * j]), x1 = __uint_as_float(v[2 * j + 1]);
        if constexpr (BIAS) {
          float b0, b1;
          br.pair(c * CH + 2 * j, b0, b1);
          x0 += b0;
          x1 += b1;
        }
        if (relu) {
          x0 = fmaxf(x0, 0.0f);
          x1 = fmaxf(x1, 0.0f);
        }
        packed[j] = pack2<OutT>(x0, x1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float x0 = __uint_as_float(v[j]), x1 = __uint_as_float(v[j + 1]);
        if constexpr (BIAS) {
          float b0, b1;
          br.pair(c * CH + j, b0, b1);
          x0 += b0;
          x1 += b1;
        }
        if (relu) {
          x0 = fmaxf(x0, 0.0f);
          x1 = fmaxf(x1, 0.0f);
        }
        packed[j] = __float_as_uint(x0);
        packed[j + 1] = __float_as_uint(x1);
      }
    }
    // the buffer written two stores ago must have been read by its TMA store
    if (count >= 2) {
      if (lane == 0) tma_store_wait_read<1>();
      __syncwarp();
    }
    const uint32_t buf = stage + (count & 1u) * 4096u;
    const uint32_t row_addr = buf + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t dst = row_addr + ((static_cast<uint32_t>(q) ^ (lane & 7u)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[4 * q]),
                   "r"(packed[4 * q + 1]), "r"(packed[4 * q + 2]), "r"(packed[4 * q + 3])
                   : "memory");
    }
    fence_proxy_async_shared();  // these generic writes -> the TMA (async proxy) read
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(tmC, buf, col0, row0, z);
      tma_store_commit();
    }
    ++count;
  }
}

// store_tile_from for tiles whose rows may end inside the warp's 32 (a
// grouped GEMM's last tile of a group): the same unrolled chunks, staged in
// one 4 KB swizzled buffer per warp, then read back row-contiguously so each
// vector store writes 16 bytes of a whole 128-byte row segment; rows at or
// past row_end and columns at or past N are masked.  No TMA and nothing to
// wait for.  Needs C 16-byte aligned and ldc and N multiples of 16 bytes.
template <int TILE_N, typename InT, typename OutT, bool BIAS, typename Src>
__device__ __forceinline__ void store_tile_rows(const Src& src, int row0, int row_end, int q0,
                                                const KParams& p, const BiasRegs<TILE_N, InT>& br,
                                                bool relu, uint32_t buf, OutT* C) {
  constexpr int CH = 128 / static_cast<int>(sizeof(OutT));  // outputs per 128-byte row chunk
  constexpr int NCH = TILE_N / CH;
  constexpr int EPV = 16 / static_cast<int>(sizeof(OutT));  // outputs per 16-byte vector
  static_assert(TILE_N % CH == 0, "whole chunks");
  const int lane = threadIdx.x & 31;
  const int nch = row0 >= row_end ? 0 : max(0, min(NCH, (p.N - q0 + CH - 1) / CH));
  const int sl = lane & 7;  // read-back: this lane's 16-byte slot of a row
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c >= nch) break;  // warp-uniform
    uint32_t v[CH];
    src.template get<CH>(c * CH, v);
    uint32_t packed[32];
    if constexpr (sizeof(OutT) == 2) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x0 = __uint_as_float(v[2 * j]), x1 = __uint_as_float(v[2 * j + 1]);
        if constexpr (BIAS) {
          float b0, b1;
          br.pair(c * CH + 2 * j, b0, b1);
          x0 += b0;
          x1 += b1;
        }
        if (relu) {
          x0 = fmaxf(x0, 0.0f);
          x1 = fmaxf(x1, 0.0f);
        }
        packed[j] = pack2<OutT>(x0, x1);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float x0 = __uint_as_float(v[j]), x1 = __uint_as_float(v[j + 1]);
        if constexpr (BIAS) {
          float b0, b1;
          br.pair(c * CH + j, b0, b1);
          x0 += b0;
          x1 += b1;
        }
        if (relu) {
          x0 = fmaxf(x0, 0.0f);
          x1 = fmaxf(x1, 0.0f);
        }
        packed[j] = __float_as_uint(x0);
        packed[j + 1] = __float_as_uint(x1);
      }
    }
    __syncwarp();  // the previous chunk's read-back of the buffer is done
    const uint32_t row_addr = buf + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t dst = row_addr + ((static_cast<uint32_t>(q) ^ (lane & 7u)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(packed[4 * q]),
                   "r"(packed[4 * q + 1]), "r"(packed[4 * q + 2]), "r"(packed[4 * q + 3])
                   : "memory");
    }
    __syncwarp();
    const int col = q0 + c * CH + sl * EPV;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + (lane >> 3);  // rows 4i .. 4i+3, eight lanes each
      uint32_t x0, x1, x2, x3;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                   : "r"(buf + static_cast<uint32_t>(r) * 128u +
                         ((static_cast<uint32_t>(sl) ^ static_cast<uint32_t>(r & 7)) << 4))
                   : "memory");
      if (row0 + r < row_end && col < p.N)
        *reinterpret_cast<uint4*>(C + static_cast<long long>(row0 + r) * p.ldc + col) =
            make_uint4(x0, x1, x2, x3);
    }
  }
}

// TMEM as a source of raw accumulator values for the epilogues above: the
// warp's 32 lanes x 16 consecutive columns starting at `taddr + cc`.
// get<W>(cc, v) fills v with W consecutive columns starting at cc; all
// loads of one call are in flight together and waited for once.
// With nacc > 1 the values are the in-order sum of nacc accumulators that
// sit acc_stride columns apart.
struct TmemSrc {
  uint32_t taddr;
  int nacc = 1;
  int acc_stride = 0;
  template <int W>
  __device__ __forceinline__ void get(int cc, uint32_t (&v)[W]) const {
    static_assert(W % 16 == 0, "whole 16-column groups");
    if (nacc > 1) {  // warp-uniform
#pragma unroll
      for (int h = 0; h < W; h += 16) {
        float f[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = 0.0f;
        for (int r = 0; r < nacc; ++r) {
          uint32_t u[16];
          tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(cc + h + r * acc_stride), u);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) f[j] += __uint_as_float(u[j]);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) v[h + j] = __float_as_uint(f[j]);
      }
      return;
    }
    if constexpr (W % 32 == 0) {
#pragma unroll
      for (int h = 0; h < W; h += 32)
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(cc + h),
                           *reinterpret_cast<uint32_t(*)[32]>(&v[h]));
    } else {
#pragma unroll
      for (int h = 0; h < W; h += 16)
        tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(cc + h),
                           *reinterpret_cast<uint32_t(*)[16]>(&v[h]));
    }
    tmem_ld_wait();
  }
};

// A partial-tile sum as a source (the last piece of a split tile).
// The sum of a split tile's pieces, for the piece that finishes it: piece
// `own` is this block's accumulator in tensor memory (`acc`), every other
// piece s is the fp32 partial tile in scratch slot piece_slot(t, s).  Columns cc ..
// cc+W-1 of this thread's row are summed in piece order, so the result does
// not depend on which piece finished last; all W/4 loads of one partial are
// issued before any is used (one memory round trip per piece, not W/4).
// Returned as raw fp32 bits.
struct PieceSumSrc {
  TmemSrc acc;
  const KParams* p;
  long long t, first_block;  // the tile, and the worker of its piece 0
  long long part;            // floats per partial tile
  int count, own, row;
  int rank = 0, ranks = 1;   // CTA pair: this CTA's rank and 2
  template <int W>
  __device__ __forceinline__ void get(int cc, uint32_t (&v)[W]) const {
    static_assert(W % 16 == 0, "whole 16-column groups");
    float f[W];
#pragma unroll
    for (int j = 0; j < W; ++j) f[j] = 0.0f;
    for (int s = 0; s < count; ++s) {  // warp-uniform
      if (s == own) {
        uint32_t t[W];
        acc.get<W>(cc, t);
#pragma unroll
        for (int j = 0; j < W; ++j) f[j] += __uint_as_float(t[j]);
        continue;
      }
      const float4* q =
          reinterpret_cast<const float4*>(p->ws + piece_slot(*p, t, s, first_block, rank, ranks) * part);
      float4 t[W / 4];
#pragma unroll
      for (int j = 0; j < W / 4; ++j)
        t[j] = __ldcg(q + (static_cast<long long>(cc / 4 + j) * kBM + row));
#pragma unroll
      for (int j = 0; j < W / 4; ++j) {
        f[4 * j] += t[j].x;
        f[4 * j + 1] += t[j].y;
        f[4 * j + 2] += t[j].z;
        f[4 * j + 3] += t[j].w;
      }
    }
#pragma unroll
    for (int j = 0; j < W; ++j) v[j] = __float_as_uint(f[j]);
  }
};

}  // namespace dg16
