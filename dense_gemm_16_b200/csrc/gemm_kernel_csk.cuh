// gemm_kernel_csk.cuh -- split-K across a CTA pair, reduced in shared memory.
//
// For grids with fewer output tiles than SMs ("用Triton跨芯片优化GEMM" section
// 2.3's 1024 x 1024 x 2048 layer puts 64 tiles of 128 x 128 on 148 SMs) each
// tile goes to a cluster of two CTAs.  CTA rank r runs an ordinary
// single-CTA main loop (the warp roles of gemm_tc_kernel) over the r-th half
// of the K blocks into its own tensor-memory accumulator.  Rank 1 then writes
// its fp32 accumulator straight into rank 0's shared memory (distributed
// shared memory; no global-memory round trip) and arrives on a barrier there;
// rank 0 adds the two halves in rank order (deterministic), applies bias and
// ReLU, rounds and stores the tile.  Each CTA streams half of the tile's
// operands, so the main loop takes half as long; the reduction is one
// SM-to-SM transfer of 64 KB.
//
// One tile per pair: the launch has exactly two CTAs per tile, so it is used
// only where tiles <= SMs / 2.  No load is multicast.  The swapped form (the
// skinny 16 x 8192 x 8192 problem: 64 tiles of 128 columns of B) streams
// each half of B once and hands over 8 KB per tile.
#pragma once

#include "kernel_common.cuh"

namespace dg16 {

constexpr int kCskChunk = 32;  // columns per transfer chunk (one barrier each)

// Where rank 1's partial lands in rank 0: [BN/4][128 rows][4] fp32, so the
// 32 lanes of a warp (32 consecutive rows) touch 512 contiguous bytes.  It
// arrives in chunks of kCskChunk columns, each with its own barrier; rank 0
// loads its own accumulator columns first and waits for the matching chunks
// only then, so its epilogue overlaps the rest of the transfer.
template <int BN, int CH>
struct CskRecvSrc {
  TmemSrc acc;     // rank 0's accumulator
  uint32_t recv;   // shared-memory address of the received partial
  uint32_t bar0;   // shared-memory address of the first chunk's barrier
  int row;
  SharedCtl* ctl;
  const KParams* p;
  template <int W>
  __device__ __forceinline__ void get(int cc, uint32_t (&v)[W]) const {
    static_assert(W % CH == 0 || CH % W == 0, "whole chunks");
    uint32_t t[W];
    acc.get<W>(cc, t);
    // a chunk that never arrives leaves its values undefined; the bounded
    // wait has then recorded the error in the status word
    for (int c = cc / CH; c * CH < cc + W; ++c)
      (void)wait_phase<true>(bar0 + static_cast<uint32_t>(c) * 8u, 0, ctl, *p,
                             kStatusTimeoutEpilogue);
#pragma unroll
    for (int j = 0; j < W / 4; ++j) {
      const uint32_t a =
          recv + static_cast<uint32_t>(((cc / 4 + j) * kBM + row) * 16);
      float4 r;
      asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                   : "r"(a));
      v[4 * j] = __float_as_uint(__uint_as_float(t[4 * j]) + r.x);
      v[4 * j + 1] = __float_as_uint(__uint_as_float(t[4 * j + 1]) + r.y);
      v[4 * j + 2] = __float_as_uint(__uint_as_float(t[4 * j + 2]) + r.z);
      v[4 * j + 3] = __float_as_uint(__uint_as_float(t[4 * j + 3]) + r.w);
    }
  }
};

//   BN, STAGES, Q_MN, IN_BF16, OutT as in gemm_tc_kernel (dense tiles only)
//   SWAP    skinny problems: P = B stored N x K, Q = A, the accumulator holds
//           C^T (N on the 128 MMA rows, BN = 16 or 32 rows of A on MMA-N)
template <int BN, int STAGES, bool Q_MN, bool IN_BF16, typename OutT, bool SWAP = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_csk_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ KParams p) {
  using InT = typename std::conditional<IN_BF16, __nv_bfloat16, __half>::type;
  static_assert(SWAP ? ((BN == 16 || BN == 32) && !Q_MN)
                     : (BN % 64 == 0 && BN >= 64 && BN <= 256),
                "BN of 64..256 in whole 64-column chunks; swapped: 16 or 32, K-major A");
  constexpr int CH = BN < kCskChunk ? BN : kCskChunk;  // columns per transfer chunk
  constexpr uint32_t P_BYTES = kBM * 128;
  constexpr uint32_t Q_BYTES = BN * 128;
  constexpr uint32_t STAGE_BYTES = P_BYTES + Q_BYTES;
  constexpr uint32_t RECV_BYTES = kBM * BN * 4;
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t IDESC = f16_idesc(kBM, BN, IN_BF16 ? 1u : 0u, 0u, Q_MN ? 1u : 0u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sP = smem;
  uint8_t* sQ = smem + STAGES * P_BYTES;
  uint8_t* sStage = sQ + STAGES * Q_BYTES;   // epilogue staging (rank 0)
  uint8_t* sRecv = sStage + kEpiStageBytes;  // rank 1's partial (rank 0)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRecv + RECV_BYTES);
  constexpr int NCHUNK = BN / CH;
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* accf_bar = bars + 2 * STAGES;
  uint64_t* drain_bar = bars + 2 * STAGES + 1;
  uint64_t* recv_bar = bars + 2 * STAGES + 2;  // NCHUNK barriers
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(bars + 2 * STAGES + 2 + NCHUNK);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) trace_mark(p, kTrEntry);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    mbar_init(smem_u32(accf_bar), 1);
    for (int c = 0; c < NCHUNK; ++c)
      mbar_init(smem_u32(&recv_bar[c]), 4 * 32);  // every epilogue thread of rank 1
    mbar_init(smem_u32(drain_bar), 1);
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    if (rank == 0) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // rank 0's barriers exist before rank 1 can signal them
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  if (threadIdx.x == 0) trace_mark(p, kTrSetup);

  // this pair's tile and this CTA's half of the K blocks
  const long long t = blockIdx.x >> 1;
  GroupTable* const no_groups = nullptr;
  int gcur = 0;
  const TileCoord c = tile_coord<false>(t, p, p.num_q, no_groups, gcur);
  const int half = (p.num_kb + 1) / 2;
  const int kb0 = rank == 0 ? 0 : half;
  const int kb1 = rank == 0 ? half : p.num_kb;
  const bool have_tile = t < p.num_tiles && kb1 > kb0;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0 && have_tile) {
      const uint64_t pol_p = make_policy(p.pol_p);
      const uint64_t pol_q = make_policy(p.pol_q);
      const int q0 = c.q0 * BN;
      uint32_t it = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % STAGES;
        if (!wait_phase(smem_u32(&empty_bar[s]), ((it / STAGES) & 1u) ^ 1u, ctl, p,
                        kStatusTimeoutProducer)) {
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(fb, STAGE_BYTES);
        tma_load_3d(smem_u32(sP + s * P_BYTES), &tmP, kb * kBK, c.p0, c.zp, fb, pol_p);
        const uint32_t qdst = smem_u32(sQ + s * Q_BYTES);
        if constexpr (Q_MN) {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_3d(qdst + j * (kBK * 128), &tmQ, q0 + 64 * j, kb * kBK, c.zq, fb, pol_q);
        } else {
          tma_load_3d(qdst, &tmQ, kb * kBK, q0, c.zq, fb, pol_q);
        }
        if (it == 0) trace_mark(p, kTrFirstLoad);
      }
      if (!ok) {
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j)
          wait_phase_drain(smem_u32(&full_bar[j % STAGES]), (j / STAGES) & 1u, 50000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && have_tile) {
      uint32_t it = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % STAGES;
        if (!wait_phase(smem_u32(&full_bar[s]), (it / STAGES) & 1u, ctl, p, kStatusTimeoutMma)) {
          ok = false;
          break;
        }
        if (it == 0) trace_mark(p, kTrFirstData);
        tc_fence_after();
        const uint32_t pbase = smem_u32(sP + s * P_BYTES);
        const uint32_t qbase = smem_u32(sQ + s * Q_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t adesc = sw128_desc(pbase + k * 32, 16, 1024);
          const uint64_t bdesc = Q_MN ? sw128_desc(qbase + k * 16 * 128, kBK * 128, 1024)
                                      : sw128_desc(qbase + k * 32, 16, 1024);
          mma_f16<1>(tmem_base, adesc, bdesc, IDESC, (kb != kb0 || k != 0) ? 1u : 0u);
        }
        mma_commit<1>(smem_u32(&empty_bar[s]));
      }
      if (ok) mma_commit<1>(smem_u32(accf_bar));
      trace_mark(p, kTrLastMma);
      mma_commit<1>(smem_u32(drain_bar));
      wait_phase_drain(smem_u32(drain_bar), 0, 50000000ull);
    }
    __syncwarp();
  } else if (have_tile) {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int row_local = quad * 32 + lane;
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const TmemSrc tsrc{taddr};
    const bool ready = wait_phase(smem_u32(accf_bar), 0, ctl, p, kStatusTimeoutEpilogue);
    if (__all_sync(0xffffffffu, ready)) {
      if (warp == 2 && lane == 0) trace_mark(p, kTrFirstEpi);
      tc_fence_after();
      if (rank == 1) {
        // fp32 accumulator -> rank 0's receive buffer, then one arrival per
        // thread (release at cluster scope: the stores are visible first)
        const uint32_t recv0 = map_shared_rank(smem_u32(sRecv), 0);
        const uint32_t rbar0 = map_shared_rank(smem_u32(&recv_bar[0]), 0);
#pragma unroll 1
        for (int cc = 0; cc < BN; cc += CH) {
          uint32_t v[CH];
          tsrc.get<CH>(cc, v);
#pragma unroll
          for (int j = 0; j < CH / 4; ++j) {
            const uint32_t a =
                recv0 + static_cast<uint32_t>(((cc / 4 + j) * kBM + row_local) * 16);
            asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a),
                         "r"(v[4 * j]), "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3])
                         : "memory");
          }
          mbar_arrive_cluster(rbar0 + static_cast<uint32_t>(cc / CH) * 8u);
        }
      } else {
        // sum in rank order as rank 1's chunks arrive, bias, ReLU, store
        {
          const InT* bias = (p.epi & 1) ? reinterpret_cast<const InT*>(p.bias) +
                                              static_cast<long long>(c.group) * p.stride_bias
                                        : nullptr;
          const bool relu = (p.epi & 2) != 0;
          const CskRecvSrc<BN, CH> src{tsrc,     smem_u32(sRecv), smem_u32(&recv_bar[0]),
                                       row_local, ctl,      &p};
          const int q0 = c.q0 * BN;
          if constexpr (SWAP) {
            // accumulator row = output column n; its columns are output rows
            // q0 .. q0+BN
            const int n = c.p0 + row_local;
            const bool col_ok = n < p.N;
            const float b = (bias != nullptr && col_ok) ? to_f32<InT>(bias[n]) : 0.0f;
            OutT* const C =
                reinterpret_cast<OutT*>(p.C) + static_cast<long long>(c.group) * p.stride_c;
#pragma unroll 1
            for (int cc = 0; cc < BN; cc += 16) {
              const int row0 = q0 + cc;
              if (row0 >= p.M) break;  // warp-uniform
              uint32_t v[16];
              src.template get<16>(cc, v);
              if (col_ok) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  if (row0 + j < p.M) {
                    float x = __uint_as_float(v[j]) + b;
                    if (relu) x = fmaxf(x, 0.0f);
                    C[static_cast<long long>(row0 + j) * p.ldc + n] = from_f32<OutT>(x);
                  }
                }
              }
            }
          } else if (p.tma_store) {
            uint32_t stores = 0;
            const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>(warp - 2) * 8192u;
            store_tma_from<BN, InT, OutT>(src, c.p0 + quad * 32, q0, c.group, p, bias, relu,
                                          stage, stores, &tmC);
            if (lane == 0) tma_store_wait_read<0>();
          } else {
            OutT* const C = reinterpret_cast<OutT*>(p.C) + static_cast<long long>(c.group) * p.stride_c;
            store_rows_from<BN, InT, OutT>(src, c.p0 + row_local, c.row_end, q0, p, bias, relu, C);
          }
        }
      }
      if (warp == 2 && lane == 0) trace_mark(p, kTrEpiDone);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // rank 0 has read rank 1's partial; no CTA leaves before its peer is done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0) trace_mark(p, kTrExit);
}

template <int BN, int STAGES>
constexpr int gemm_csk_smem_bytes() {
  return 1024 + STAGES * (kBM * 128 + BN * 128) + static_cast<int>(kEpiStageBytes) +
         kBM * BN * 4 + (2 * STAGES + 2 + BN / (BN < kCskChunk ? BN : kCskChunk)) * 8 +
         static_cast<int>(sizeof(SharedCtl));
}

}  // namespace dg16
