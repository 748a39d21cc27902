// gemm_kernel_gswap.cuh -- grouped GEMM with swapped operands and a dynamic
// tile queue, for MoE layers whose experts hold a few hundred rows each.
//
// The grouped problem is Y_g = act(X_g . W_g + bias_g) for every group g
// ("用Triton跨芯片优化GEMM" section 2.3: the dozens of GEMMs of a MoE layer in
// one launch).  With 128-row tiles over the rows of X_g, a group of m_g rows
// pays for ceil(m_g / 128) * 128 rows, and an N that is not a multiple of the
// tile width pays for the rest of the last column block.  Here the MMA
// computes Y_g^T instead: the 128 MMA rows run over N (the weights' output
// columns) and the MMA's N runs over the group's rows, sized per tile at run
// time in steps of 16 (the instruction descriptor is a register operand).  A
// group is cut into ceil(m_g / TOK) row blocks of near-equal size (TOK = 128,
// 192 or 256), so the only padding is to the next multiple of 16 rows.
//
// Tiles differ in cost, so instead of a static stride the producer warp takes
// the next tile id from a global counter (one atomicAdd per tile) and hands it
// to the MMA and epilogue warps through a small shared-memory queue.  Every
// block takes ids until it draws one past the last tile; the block that draws
// the very last id of the launch (num_tiles + gridDim.x - 1) knows every other
// draw has happened and resets the counter to 0 for the next launch on the
// stream, also on the error path.
//
// Tile order inside a group: weight column block outer, row block inner, so
// the row blocks that read the same 128 columns of W_g are drawn together and
// share them in L2.
//
// Warp roles as in gemm_tc_kernel: warp 0 TMA producer, warp 1 TMEM owner and
// MMA issuer, warps 2..5 epilogue.  Every wait is bounded.
#pragma once

#include "kernel_common.cuh"

namespace dg16 {

constexpr int kGsQueue = 4;  // tile-id queue depth

// Row-operand tensor maps of the same matrix X with 128-, 64-, 32-, 16- and
// 8-row boxes: r rows (r a multiple of 8) are fetched with a few copies,
// largest first.
struct RowMaps {
  CUtensorMap m[5];
};

// Copy rows [r0, r0 + rows) of X (rows a multiple of `min_box`), K block kb,
// into consecutive 128-byte rows at dst, counting the bytes on `bar`.
template <bool PAIR>
__device__ __forceinline__ void load_rows(const RowMaps& tmX, uint32_t dst, int kb, int r0,
                                          int rows, uint32_t bar, uint64_t pol) {
  int off = 0;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int box = 128 >> i;
    while (rows - off >= box) {
      if constexpr (PAIR)
        tma_load_2d_pair(dst + off * 128, &tmX.m[i], kb * kBK, r0 + off, bar, pol);
      else
        tma_load_2d(dst + off * 128, &tmX.m[i], kb * kBK, r0 + off, bar, pol);
      off += box;
    }
  }
}

// Where a grouped-swap tile lives.
struct GsTile {
  int g;    // group
  int n0;   // first output column (the tile's first MMA row)
  int r0;   // first row of X / Y (global)
  int nr;   // rows in the tile (1 .. TOK)
};

// Tile t of the launch (groups cut into row blocks of at most TOK rows,
// output columns into blocks of COLS); t must be below the table's total.
// Tile ids reach each role in increasing order, so `gcursor` only walks
// forward.
template <int TOK, int COLS>
__device__ __forceinline__ GsTile gswap_tile(int t, const GroupTable* gt, int num_groups,
                                             int& gcursor) {
  while (gcursor < num_groups - 1 && t >= gt->tile_start[gcursor + 1]) ++gcursor;
  const int g = gcursor;
  const int rows = gt->row_start[g + 1] - gt->row_start[g];
  const int nblk = (rows + TOK - 1) / TOK;  // >= 1 for a group with tiles
  const int local = t - gt->tile_start[g];
  const int nb = local / nblk;
  const int rb = local - nb * nblk;
  const int base = rows / nblk, extra = rows - base * nblk;
  GsTile c;
  c.g = g;
  c.n0 = nb * COLS;
  c.r0 = gt->row_start[g] + rb * base + min(rb, extra);
  c.nr = base + (rb < extra ? 1 : 0);
  return c;
}

// Bounded wait by a whole warp; true only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, SharedCtl* ctl,
                                          const KParams& p, unsigned code) {
  const bool ok = wait_phase(bar, parity, ctl, p, code);
  return __all_sync(0xffffffffu, ok);
}

//   TOK     most group rows per tile (MMA N; 128, 192 or 256)
//   STAGES  operand ring depth (each stage: 128 x 64 of W, up to TOK x 64 of X)
//   P_MN    W is row-major ([g][K][N], N contiguous): the weight operand is
//           MN-major in shared memory; else W is [g][N][K] (K-major)
//   IN_BF16 inputs are bf16 (else fp16)
//   OutT    output element type
template <int TOK, int STAGES, bool P_MN, bool IN_BF16, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_gswap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ RowMaps tmX,
                      const __grid_constant__ KParams p) {
  using InT = typename std::conditional<IN_BF16, __nv_bfloat16, __half>::type;
  constexpr uint32_t W_BYTES = kBM * 128;        // 128 columns of W x 64 K
  static_assert(TOK % 64 == 0 && TOK >= 128 && TOK <= 256, "row blocks of 128..256 rows");
  constexpr uint32_t X_BYTES = TOK * 128;  // up to TOK rows of X x 64 K
  constexpr uint32_t ACC_COLS = TOK <= 128 ? 128 : 256;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  // M = 128; N is or-ed in per tile
  constexpr uint32_t IDESC_BASE = f16_idesc(kBM, 0, IN_BF16 ? 1u : 0u, P_MN ? 1u : 0u, 0u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + STAGES * X_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* accf_bar = bars + 2 * STAGES;
  uint64_t* acce_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint64_t* tqf_bar = bars + 2 * STAGES + 5;
  uint64_t* tqe_bar = tqf_bar + kGsQueue;
  int* tq = reinterpret_cast<int*>(tqe_bar + kGsQueue);
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(tq + kGsQueue);
  GroupTable* gt = reinterpret_cast<GroupTable*>(ctl + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) trace_mark(p, kTrEntry);
  const int num_nb = (p.N + kBM - 1) / kBM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&accf_bar[a]), 1);
      mbar_init(smem_u32(&acce_bar[a]), 4 * 32);
    }
    mbar_init(smem_u32(drain_bar), 1);
    for (int q = 0; q < kGsQueue; ++q) {
      mbar_init(smem_u32(&tqf_bar[q]), 1);
      mbar_init(smem_u32(&tqe_bar[q]), 1 + 4);  // the MMA lane + one lane per epilogue warp
    }
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    for (int i = 0; i < 5; ++i) tma_prefetch_desc(&tmX.m[i]);
  }
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<1>();
  }
  if (warp == 2 && lane == 0) {
    // per-group tile prefix from the device counts
    int tiles = 0, rows = 0;
    bool bad = false;
    for (int g = 0; g < p.num_groups; ++g) {
      int m = __ldg(&p.group_rows[g]);
      if (m < 0) {
        m = 0;
        bad = true;
      }
      gt->tile_start[g] = tiles;
      gt->row_start[g] = rows;
      const int usable = max(0, min(m, p.M - rows));  // rows past the total are never touched
      if (usable < m) bad = true;
      tiles += (usable + TOK - 1) / TOK * num_nb;
      rows += usable;
    }
    gt->tile_start[p.num_groups] = tiles;
    gt->row_start[p.num_groups] = rows;
    if (bad && blockIdx.x == 0) atomicCAS(p.status, 0u, kStatusBadGroups);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int num_tiles = gt->tile_start[p.num_groups];
  if (threadIdx.x == 0) trace_mark(p, kTrSetup);

  if (warp == 0) {
    // ------------------------------------------- tile queue + TMA producer
    if (lane == 0) {
      const uint64_t pol_w = make_policy(p.pol_p);
      const uint64_t pol_x = make_policy(p.pol_q);
      unsigned* const counter = p.counters;
      uint32_t it = 0;
      int gcur = 0;
      bool ok = true;
      // `held` is the latest id this block drew; the next tile's id is drawn
      // while the current one loads, so the atomic's latency stays hidden
      unsigned held = atomicAdd(counter, 1u);
      for (uint32_t local = 0;; ++local) {
        const unsigned drawn = held;
        const uint32_t q = local % kGsQueue;
        if (!wait_phase(smem_u32(&tqe_bar[q]), ((local / kGsQueue) & 1u) ^ 1u, ctl, p,
                        kStatusTimeoutProducer)) {
          ok = false;
          break;
        }
        const bool last = drawn >= static_cast<unsigned>(num_tiles);
        tq[q] = last ? -1 : static_cast<int>(drawn);
        mbar_arrive(smem_u32(&tqf_bar[q]));  // release: the id is visible to the waiters
        if (last) break;
        held = atomicAdd(counter, 1u);
        const GsTile c = gswap_tile<TOK, kBM>(static_cast<int>(drawn), gt, p.num_groups, gcur);
        const int rows16 = (c.nr + 15) & ~15;
        const uint32_t bytes = W_BYTES + static_cast<uint32_t>(rows16) * 128u;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase(smem_u32(&empty_bar[s]), ph ^ 1u, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t wdst = smem_u32(sW + s * W_BYTES);
          if constexpr (P_MN) {
            // two 64-column chunks, each 64 K rows of 128 bytes
            tma_load_3d(wdst, &tmW, c.n0, kb * kBK, c.g, fb, pol_w);
            tma_load_3d(wdst + kBK * 128, &tmW, c.n0 + 64, kb * kBK, c.g, fb, pol_w);
          } else {
            tma_load_3d(wdst, &tmW, kb * kBK, c.n0, c.g, fb, pol_w);
          }
          load_rows<false>(tmX, smem_u32(sX + s * X_BYTES), kb, c.r0, rows16, fb, pol_x);
        }
        if (!ok) break;
      }
      if (!ok) {
        // leave no copy in flight into this block's shared memory
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j)
          wait_phase_drain(smem_u32(&full_bar[j % STAGES]), (j / STAGES) & 1u, 50000000ull);
        // keep drawing so that the launch's draws still add up and the
        // counter is reset
        while (held < static_cast<unsigned>(num_tiles)) held = atomicAdd(counter, 1u);
      }
      if (held == static_cast<unsigned>(num_tiles) + gridDim.x - 1u) atomicExch(counter, 0u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      int gcur = 0;
      for (uint32_t local = 0;; ++local) {
        const uint32_t q = local % kGsQueue;
        if (!wait_phase(smem_u32(&tqf_bar[q]), (local / kGsQueue) & 1u, ctl, p, kStatusTimeoutMma))
          break;
        const int t = *reinterpret_cast<volatile int*>(&tq[q]);
        mbar_arrive(smem_u32(&tqe_bar[q]));
        if (t < 0) break;
        const GsTile c = gswap_tile<TOK, kBM>(t, gt, p.num_groups, gcur);
        const uint32_t rows16 = static_cast<uint32_t>((c.nr + 15) & ~15);
        const uint32_t idesc = IDESC_BASE | ((rows16 >> 3) << 17);
        const uint32_t a = local & 1u;
        if (!wait_phase(smem_u32(&acce_bar[a]), ((local >> 1) & 1u) ^ 1u, ctl, p,
                        kStatusTimeoutMma))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + a * ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (!wait_phase(smem_u32(&full_bar[s]), (it / STAGES) & 1u, ctl, p, kStatusTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wbase = smem_u32(sW + s * W_BYTES);
          const uint32_t xbase = smem_u32(sX + s * X_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // W: MN-major slices are 16 K rows of 128 B, the two 64-column
            // chunks 8 KB apart; K-major slices start 32 B further along each
            // swizzled row.  X is K-major.  8-row groups are 1024 B apart.
            const uint64_t wdesc = P_MN ? sw128_desc(wbase + k * 16 * 128, kBK * 128, 1024)
                                        : sw128_desc(wbase + k * 32, 16, 1024);
            const uint64_t xdesc = sw128_desc(xbase + k * 32, 16, 1024);
            mma_f16<1>(d, wdesc, xdesc, idesc, (kb != 0 || k != 0) ? 1u : 0u);
          }
          mma_commit<1>(smem_u32(&empty_bar[s]));
        }
        if (!ok) break;
        mma_commit<1>(smem_u32(&accf_bar[a]));
      }
      trace_mark(p, kTrLastMma);
      mma_commit<1>(smem_u32(drain_bar));
      wait_phase_drain(smem_u32(drain_bar), 0, 50000000ull);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int row_local = quad * 32 + lane;  // this thread's MMA row: output column n0 + row_local
    OutT* const C = reinterpret_cast<OutT*>(p.C);
    const InT* const bias = reinterpret_cast<const InT*>(p.bias);
    const bool has_bias = (p.epi & 1) != 0;
    const bool relu = (p.epi & 2) != 0;
    int gcur = 0;
    for (uint32_t local = 0;; ++local) {
      const uint32_t q = local % kGsQueue;
      if (!warp_wait(smem_u32(&tqf_bar[q]), (local / kGsQueue) & 1u, ctl, p,
                     kStatusTimeoutEpilogue))
        break;
      const int t = *reinterpret_cast<volatile int*>(&tq[q]);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tqe_bar[q]));
      if (t < 0) break;
      const GsTile c = gswap_tile<TOK, kBM>(t, gt, p.num_groups, gcur);
      const uint32_t a = local & 1u;
      if (!warp_wait(smem_u32(&accf_bar[a]), (local >> 1) & 1u, ctl, p, kStatusTimeoutEpilogue))
        break;
      tc_fence_after();
      const int n = c.n0 + row_local;
      const bool col_ok = n < p.N;
      const float b =
          (has_bias && col_ok) ? to_f32<InT>(bias[static_cast<long long>(c.g) * p.N + n]) : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * ACC_COLS;
      OutT* const out = C + static_cast<long long>(c.r0) * p.ldc + n;
#pragma unroll 1
      for (int cc = 0; cc < c.nr; cc += 16) {  // warp-uniform bound
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(cc), v);
        tmem_ld_wait();
        if (col_ok) {
          const int lim = min(16, c.nr - cc);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < lim) {
              float x = __uint_as_float(v[j]) + b;
              if (relu) x = fmaxf(x, 0.0f);
              out[static_cast<long long>(cc + j) * p.ldc] = from_f32<OutT>(x);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acce_bar[a]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0) trace_mark(p, kTrExit);
}

// ---------------------------------------------------------------------------
// Pair form.  Two CTAs (a cluster of 2) share one tile of 256 output columns
// by up to TOK rows: each CTA stages its own 128 columns of W and one half of
// the tile's rows of X, and the leader issues tcgen05.mma with M = 256, whose
// B operand (the rows) is split between the two CTAs' shared memory.  Per MMA
// each SM now stages 16 KB of W and at most 16 KB of X instead of 16 + 32 KB:
// the single-CTA form is bound by that shared-memory fill rate.
//
// Tile queue: only the leader's producer draws ids.  It writes each id into
// the queue slot of both CTAs (a cluster store into the peer) and arrives on
// both CTAs' slot barriers; the slot is free again once all ten readers (the
// leader's MMA lane, the peer's producer and the four epilogue warps of each
// CTA) have arrived on the leader's empty barrier.
//
// Barriers (same offsets in both CTAs):
//   full[s]  leader only; armed by the leader with both CTAs' bytes.
//   empty[s] per CTA; the leader's MMA lane commits to both.
//   accf[a]  per CTA; the leader's MMA lane commits to both.
//   acce[a]  leader only; one arrival per epilogue warp of either CTA (8).
//   tqf[q]   per CTA; the leader's producer arrives on both.
//   tqe[q]   leader only; 10 arrivals.
template <int TOK, int STAGES, bool P_MN, bool IN_BF16, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_gswap2_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ RowMaps tmX, const __grid_constant__ KParams p) {
  using InT = typename std::conditional<IN_BF16, __nv_bfloat16, __half>::type;
  static_assert(TOK % 64 == 0 && TOK >= 128 && TOK <= 256, "row blocks of 128..256 rows");
  constexpr int COLS = 2 * kBM;                     // output columns per pair tile
  constexpr uint32_t W_BYTES = kBM * 128;          // this CTA's 128 columns x 64 K
  constexpr uint32_t X_BYTES = (TOK / 2) * 128;    // its half of the rows x 64 K
  constexpr uint32_t ACC_COLS = TOK <= 128 ? 128 : 256;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  constexpr uint32_t IDESC_BASE = f16_idesc(2 * kBM, 0, IN_BF16 ? 1u : 0u, P_MN ? 1u : 0u, 0u);
  constexpr uint32_t kReaders = 1 + 4 + 1 + 4;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + STAGES * X_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* accf_bar = bars + 2 * STAGES;
  uint64_t* acce_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint64_t* tqf_bar = bars + 2 * STAGES + 5;
  uint64_t* tqe_bar = tqf_bar + kGsQueue;
  int* tq = reinterpret_cast<int*>(tqe_bar + kGsQueue);
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(tq + kGsQueue);
  GroupTable* gt = reinterpret_cast<GroupTable*>(ctl + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) trace_mark(p, kTrEntry);
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const uint32_t peer = rank ^ 1u;
  const int num_nb = (p.N + COLS - 1) / COLS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&accf_bar[a]), 1);
      mbar_init(smem_u32(&acce_bar[a]), 2 * 4);
    }
    mbar_init(smem_u32(drain_bar), 1);
    for (int q = 0; q < kGsQueue; ++q) {
      mbar_init(smem_u32(&tqf_bar[q]), 1);
      mbar_init(smem_u32(&tqe_bar[q]), kReaders);
    }
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    for (int i = 0; i < 5; ++i) tma_prefetch_desc(&tmX.m[i]);
  }
  if (warp == 1) {
    tmem_alloc<2>(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<2>();
  }
  if (warp == 2 && lane == 0) {
    // per-group tile prefix from the device counts (each CTA its own copy)
    int tiles = 0, rows = 0;
    bool bad = false;
    for (int g = 0; g < p.num_groups; ++g) {
      int m = __ldg(&p.group_rows[g]);
      if (m < 0) {
        m = 0;
        bad = true;
      }
      gt->tile_start[g] = tiles;
      gt->row_start[g] = rows;
      const int usable = max(0, min(m, p.M - rows));
      if (usable < m) bad = true;
      tiles += (usable + TOK - 1) / TOK * num_nb;
      rows += usable;
    }
    gt->tile_start[p.num_groups] = tiles;
    gt->row_start[p.num_groups] = rows;
    if (bad && blockIdx.x == 0) atomicCAS(p.status, 0u, kStatusBadGroups);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int num_tiles = gt->tile_start[p.num_groups];
  if (threadIdx.x == 0) trace_mark(p, kTrSetup);
  const uint32_t tqe_leader0 = map_shared_rank(smem_u32(&tqe_bar[0]), 0);

  if (warp == 0) {
    // ------------------------------- tile queue (leader) + TMA producer (both)
    if (lane == 0) {
      const uint64_t pol_w = make_policy(p.pol_p);
      const uint64_t pol_x = make_policy(p.pol_q);
      unsigned* const counter = p.counters;
      const uint32_t tq_peer0 = map_shared_rank(smem_u32(&tq[0]), peer);
      const uint32_t tqf_peer0 = map_shared_rank(smem_u32(&tqf_bar[0]), peer);
      uint32_t it = 0;
      int gcur = 0;
      bool ok = true;
      unsigned held = rank == 0 ? atomicAdd(counter, 1u) : 0u;
      for (uint32_t local = 0;; ++local) {
        const uint32_t q = local % kGsQueue;
        const uint32_t qph = (local / kGsQueue) & 1u;
        int t;
        if (rank == 0) {
          const unsigned drawn = held;
          if (!wait_phase<true>(smem_u32(&tqe_bar[q]), qph ^ 1u, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          t = drawn >= static_cast<unsigned>(num_tiles) ? -1 : static_cast<int>(drawn);
          tq[q] = t;
          st_shared_cluster_u32(tq_peer0 + q * 4u, static_cast<uint32_t>(t));
          mbar_arrive(smem_u32(&tqf_bar[q]));
          mbar_arrive_cluster(tqf_peer0 + q * 8u);  // release: the peer's copy of t first
          if (t < 0) break;
          held = atomicAdd(counter, 1u);  // the next id, drawn while this tile loads
        } else {
          if (!wait_phase<true>(smem_u32(&tqf_bar[q]), qph, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          t = *reinterpret_cast<volatile int*>(&tq[q]);
          mbar_arrive_cluster(tqe_leader0 + q * 8u);
          if (t < 0) break;
        }
        const GsTile c = gswap_tile<TOK, COLS>(t, gt, p.num_groups, gcur);
        const int rows16 = (c.nr + 15) & ~15;
        const int half = rows16 / 2;  // a multiple of 8
        const uint32_t bytes = 2 * W_BYTES + static_cast<uint32_t>(rows16) * 128u;
        const int wcol = c.n0 + static_cast<int>(rank) * kBM;
        const int xrow = c.r0 + static_cast<int>(rank) * half;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase<true>(smem_u32(&empty_bar[s]), ph ^ 1u, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb_leader = map_shared_rank(smem_u32(&full_bar[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), bytes);
          const uint32_t wdst = smem_u32(sW + s * W_BYTES);
          if constexpr (P_MN) {
            tma_load_3d_pair(wdst, &tmW, wcol, kb * kBK, c.g, fb_leader, pol_w);
            tma_load_3d_pair(wdst + kBK * 128, &tmW, wcol + 64, kb * kBK, c.g, fb_leader, pol_w);
          } else {
            tma_load_3d_pair(wdst, &tmW, kb * kBK, wcol, c.g, fb_leader, pol_w);
          }
          load_rows<true>(tmX, smem_u32(sX + s * X_BYTES), kb, xrow, half, fb_leader, pol_x);
        }
        if (!ok) break;
      }
      if (!ok) {
        if (rank == 0) {
          const uint32_t first = it > STAGES ? it - STAGES : 0;
          for (uint32_t j = first; j < it; ++j)
            wait_phase_drain(smem_u32(&full_bar[j % STAGES]), (j / STAGES) & 1u, 50000000ull);
        }
        // the peer cannot observe its copies' completion (they count on the
        // leader's barrier): give any copy in flight time to land
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
      }
      if (rank == 0) {
        if (!ok)  // keep drawing so that the launch's draws still add up
          while (held < static_cast<unsigned>(num_tiles)) held = atomicAdd(counter, 1u);
        if (held == static_cast<unsigned>(num_tiles) + (gridDim.x >> 1) - 1u)
          atomicExch(counter, 0u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      const uint32_t peer_empty0 = map_shared_rank(smem_u32(&empty_bar[0]), peer);
      const uint32_t peer_accf0 = map_shared_rank(smem_u32(&accf_bar[0]), peer);
      uint32_t it = 0;
      int gcur = 0;
      for (uint32_t local = 0;; ++local) {
        const uint32_t q = local % kGsQueue;
        if (!wait_phase<true>(smem_u32(&tqf_bar[q]), (local / kGsQueue) & 1u, ctl, p,
                              kStatusTimeoutMma))
          break;
        const int t = *reinterpret_cast<volatile int*>(&tq[q]);
        mbar_arrive(smem_u32(&tqe_bar[q]));
        if (t < 0) break;
        const GsTile c = gswap_tile<TOK, COLS>(t, gt, p.num_groups, gcur);
        const uint32_t rows16 = static_cast<uint32_t>((c.nr + 15) & ~15);
        const uint32_t idesc = IDESC_BASE | ((rows16 >> 3) << 17);
        const uint32_t a = local & 1u;
        if (!wait_phase<true>(smem_u32(&acce_bar[a]), ((local >> 1) & 1u) ^ 1u, ctl, p,
                              kStatusTimeoutMma))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + a * ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          if (!wait_phase<true>(smem_u32(&full_bar[s]), (it / STAGES) & 1u, ctl, p,
                                kStatusTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wbase = smem_u32(sW + s * W_BYTES);
          const uint32_t xbase = smem_u32(sX + s * X_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t wdesc = P_MN ? sw128_desc(wbase + k * 16 * 128, kBK * 128, 1024)
                                        : sw128_desc(wbase + k * 32, 16, 1024);
            const uint64_t xdesc = sw128_desc(xbase + k * 32, 16, 1024);
            mma_f16<2>(d, wdesc, xdesc, idesc, (kb != 0 || k != 0) ? 1u : 0u);
          }
          // stage s is free in both CTAs once these MMAs have read it
          mma_commit<2>(smem_u32(&empty_bar[s]));
          mma_commit<2>(peer_empty0 + s * 8u);
        }
        if (!ok) break;
        mma_commit<2>(smem_u32(&accf_bar[a]));
        mma_commit<2>(peer_accf0 + a * 8u);
      }
      trace_mark(p, kTrLastMma);
      mma_commit<2>(smem_u32(drain_bar));
      wait_phase_drain(smem_u32(drain_bar), 0, 50000000ull);
    }
    __syncwarp();
  } else {
    // --------------------------------------------- epilogue (both CTAs)
    const int quad = warp & 3;
    const int row_local = quad * 32 + lane;
    OutT* const C = reinterpret_cast<OutT*>(p.C);
    const InT* const bias = reinterpret_cast<const InT*>(p.bias);
    const bool has_bias = (p.epi & 1) != 0;
    const bool relu = (p.epi & 2) != 0;
    const uint32_t acce_leader0 = map_shared_rank(smem_u32(&acce_bar[0]), 0);
    int gcur = 0;
    for (uint32_t local = 0;; ++local) {
      const uint32_t q = local % kGsQueue;
      const bool got = wait_phase<true>(smem_u32(&tqf_bar[q]), (local / kGsQueue) & 1u, ctl, p,
                                        kStatusTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;
      const int t = *reinterpret_cast<volatile int*>(&tq[q]);
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tqe_leader0 + q * 8u);
      if (t < 0) break;
      const GsTile c = gswap_tile<TOK, COLS>(t, gt, p.num_groups, gcur);
      const uint32_t a = local & 1u;
      const bool ready = wait_phase<true>(smem_u32(&accf_bar[a]), (local >> 1) & 1u, ctl, p,
                                          kStatusTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const int n = c.n0 + static_cast<int>(rank) * kBM + row_local;
      const bool col_ok = n < p.N;
      const float b =
          (has_bias && col_ok) ? to_f32<InT>(bias[static_cast<long long>(c.g) * p.N + n]) : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * ACC_COLS;
      OutT* const out = C + static_cast<long long>(c.r0) * p.ldc + n;
#pragma unroll 1
      for (int cc = 0; cc < c.nr; cc += 16) {  // warp-uniform bound
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + static_cast<uint32_t>(cc), v);
        tmem_ld_wait();
        if (col_ok) {
          const int lim = min(16, c.nr - cc);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < lim) {
              float x = __uint_as_float(v[j]) + b;
              if (relu) x = fmaxf(x, 0.0f);
              out[static_cast<long long>(cc + j) * p.ldc] = from_f32<OutT>(x);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader0 + a * 8u);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<2>(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0) trace_mark(p, kTrExit);
}

template <int TOK, int STAGES>
constexpr int gemm_gswap2_smem_bytes() {
  return 1024 + STAGES * (kBM * 128 + (TOK / 2) * 128) +
         (2 * STAGES + 5 + 2 * kGsQueue) * 8 + kGsQueue * 4 +
         static_cast<int>(sizeof(SharedCtl)) + static_cast<int>(sizeof(GroupTable));
}

template <int TOK, int STAGES>
constexpr int gemm_gswap_smem_bytes() {
  return 1024 + STAGES * (kBM * 128 + TOK * 128) + (2 * STAGES + 5 + 2 * kGsQueue) * 8 +
         kGsQueue * 4 + static_cast<int>(sizeof(SharedCtl)) + static_cast<int>(sizeof(GroupTable));
}

}  // namespace dg16
