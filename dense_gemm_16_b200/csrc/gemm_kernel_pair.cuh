// gemm_kernel_pair.cuh -- the CTA-pair (cta_group::2) variant of the GEMM.
//
// Two CTAs on neighbouring SMs (a cluster of 2) share one 256 x BN output
// tile.  Each CTA streams its own 128 rows of A and its own half (BN/2
// columns) of B into its own shared memory; the pair's leader issues
// tcgen05.mma with M = 256, which reads A and B from both CTAs and leaves
// each CTA's 128 x BN slice of the accumulator in that CTA's tensor memory.
// Per output element each SM now stages half as much of B as the single-CTA
// kernel, which halves the shared-memory operand traffic per MMA -- the
// limit the single-CTA kernel runs into at 128 x 256 tiles.
//
// No load is multicast: every CTA fetches its own operand halves.
//
// Synchronisation (barriers live in each CTA's shared memory):
//   full[s]   leader only; armed by the leader's producer with both CTAs'
//             bytes; both CTAs' TMA copies count their bytes on it.
//   empty[s]  one per CTA; the leader's MMA thread commits to both.
//   accf[a]   one per CTA; the leader's MMA thread commits to both.
//   acce[a]   leader only; one arrival per epilogue warp of either CTA (8).
#pragma once

#include "kernel_common.cuh"

namespace dg16 {

// BN      MMA N (each CTA loads BN/2 columns of B per MMA)
// NSUB    MMAs per K step, side by side in N: the pair tile is 256 x (BN*NSUB).
//         With NSUB = 2 and BN = 256 one accumulator fills all 512 TMEM
//         columns (no double buffering) but each SM stages 25% fewer operand
//         bytes per FLOP and the ring holds more time's worth of work.
// STAGES  ring depth
// Q_MN    B is row-major (MN-major operand)
// IN_BF16 / OutT as in the single-CTA kernel
// GROUPED grouped GEMM: pair tiles of 256 rows within one group (rows of A
//         sorted by group, B a [group][K][N] or [group][N][K] stack); the
//         tile prefix is built in shared memory from the device-side group
//         sizes, and stores are masked at the group's last row
template <int BN, int NSUB, int STAGES, bool Q_MN, bool IN_BF16, typename OutT,
          bool GROUPED = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ KParams p) {
  using InT = typename std::conditional<IN_BF16, __nv_bfloat16, __half>::type;
  constexpr int HALF_N = BN / 2;
  constexpr int TILE_N = BN * NSUB;                 // output columns per pair tile
  constexpr int ACC_BUFS = (2 * TILE_N <= 512) ? 2 : 1;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair MMA N must be 64..256");
  static_assert(TILE_N <= 512, "the accumulator must fit in 512 TMEM columns");
  static_assert(!Q_MN || HALF_N % 64 == 0, "MN-major B halves are whole 64-column rows");
  constexpr uint32_t P_BYTES = kBM * kBK * 2;              // this CTA's 128 rows of A
  constexpr uint32_t QSUB_BYTES = HALF_N * kBK * 2;        // its half of one MMA's B
  constexpr uint32_t Q_BYTES = NSUB * QSUB_BYTES;
  constexpr uint32_t STAGE_BYTES = P_BYTES + Q_BYTES;
  constexpr uint32_t TMEM_COLS = (ACC_BUFS * TILE_N <= 256) ? 256 : 512;
  // grouped tiles must not write past their group's last row: they stage
  // through one 4 KB buffer per epilogue warp and store masked rows
  constexpr uint32_t STAGE_EPI = GROUPED ? kEpiStageBytes / 2 : kEpiStageBytes;
  constexpr uint32_t IDESC = f16_idesc(2 * kBM, BN, IN_BF16 ? 1u : 0u, 0u, Q_MN ? 1u : 0u);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sP = smem;
  uint8_t* sQ = smem + STAGES * P_BYTES;
  uint8_t* sStage = sQ + STAGES * Q_BYTES;  // 1024-aligned epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStage + STAGE_EPI);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* accf_bar = bars + 2 * STAGES;
  uint64_t* acce_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  SharedCtl* ctl = reinterpret_cast<SharedCtl*>(bars + 2 * STAGES + 5);
  GroupTable* gt = reinterpret_cast<GroupTable*>(ctl + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const uint32_t peer = rank ^ 1u;
  // Every CTA of a pair shares the same smem layout, so a barrier's offset
  // names the same barrier role in either CTA.
  const long long pair_id = blockIdx.x >> 1;
  const long long num_pairs = gridDim.x >> 1;
  if (threadIdx.x == 0) trace_mark(p, kTrEntry);

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
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    if constexpr (!GROUPED) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc<2>(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<2>();
  }
  const int num_q_tiles = (p.N + TILE_N - 1) / TILE_N;
  if constexpr (GROUPED) {
    if (warp == 2 && lane == 0) {
      // per-group tile prefix (256-row blocks) from the device counts; each
      // CTA of the pair builds the same table
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
        tiles += (usable + 2 * kBM - 1) / (2 * kBM) * num_q_tiles;
        rows += usable;
      }
      gt->tile_start[p.num_groups] = tiles;
      gt->row_start[p.num_groups] = rows;
      if (bad && blockIdx.x == 0) atomicCAS(p.status, 0u, kStatusBadGroups);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const long long num_tiles = GROUPED ? gt->tile_start[p.num_groups] : p.num_tiles;
  // Work split over pairs: whole tiles (mode 0), or stream-K (2) / the
  // hybrid (3) over (tile, K block) iterations.  A piece of a split tile is
  // the same K range in both CTAs; each CTA fixes up its own 128 rows with
  // its own counter (2t + rank) and partial slots.
  long long sk_width = 0, sk_tiles = 0;
  if (p.work_mode == 3) hybrid_split(num_tiles, p.num_kb, &sk_tiles, &sk_width, num_pairs);
  if (threadIdx.x == 0) trace_mark(p, kTrSetup);

  // Where pair tile t lives: its first row (of the batch, or global for
  // grouped), its column block, the TMA batch/group coordinates, the batch
  // or group index and the end of the rows it may store.  Tile ids reach
  // each role in increasing order, so the group cursor only walks forward.
  struct PairTile {
    int p0, qb, zp, zq, b, row_end;
  };
  auto pair_tile = [&](long long t, int& gcur) {
    PairTile c;
    if constexpr (GROUPED) {
      while (gcur < p.num_groups - 1 && t >= gt->tile_start[gcur + 1]) ++gcur;
      const int g = gcur;
      const int local = static_cast<int>(t - gt->tile_start[g]);
      const int rows = gt->row_start[g + 1] - gt->row_start[g];
      int mb, nb;
      raster_tile(local, (rows + 2 * kBM - 1) / (2 * kBM), num_q_tiles, p.group_m, mb, nb);
      c.p0 = gt->row_start[g] + mb * 2 * kBM;
      c.qb = nb;
      c.zp = 0;
      c.zq = g;
      c.b = g;
      c.row_end = min(gt->row_start[g + 1], p.M);
    } else {
      const long long b = t / p.tiles_per_batch;
      int pb, qb;
      raster_tile(t - b * p.tiles_per_batch, p.num_p, p.num_q, p.group_m, pb, qb);
      c.p0 = pb * (2 * kBM);
      c.qb = qb;
      c.zp = static_cast<int>(b) * p.z_p;
      c.zq = static_cast<int>(b) * p.z_q;
      c.b = static_cast<int>(b);
      c.row_end = p.M;
    }
    return c;
  };

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint64_t pol_p = make_policy(p.pol_p);
      const uint64_t pol_q = make_policy(p.pol_q);
      uint32_t it = 0;
      bool ok = true;
      int gcur = 0;
      WorkIter wi(p, num_tiles, sk_width, sk_tiles, pair_id, num_pairs);
      Work w;
      while (ok && wi.next(p, w)) {
        const PairTile c = pair_tile(w.t, gcur);
        const int zp = c.zp, zq = c.zq;
        const int prow0 = c.p0 + static_cast<int>(rank) * kBM;
        // MMA j of the K step covers tile columns [j*BN, (j+1)*BN); this CTA
        // supplies the rank-th half of each
        const int qcol0 = c.qb * TILE_N + static_cast<int>(rank) * HALF_N;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase<true>(smem_u32(&empty_bar[s]), ph ^ 1u, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          // the leader's full barrier counts both CTAs' bytes
          const uint32_t fb_leader = map_shared_rank(smem_u32(&full_bar[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), 2 * STAGE_BYTES);
          tma_load_3d_pair(smem_u32(sP + s * P_BYTES), &tmP, kb * kBK, prow0, zp, fb_leader,
                           pol_p);
#pragma unroll
          for (int sub = 0; sub < NSUB; ++sub) {
            const uint32_t qdst = smem_u32(sQ + s * Q_BYTES + sub * QSUB_BYTES);
            const int qc = qcol0 + sub * BN;
            if constexpr (Q_MN) {
#pragma unroll
              for (int j = 0; j < HALF_N / 64; ++j)
                tma_load_3d_pair(qdst + j * (64 * kBK * 2), &tmQ, qc + 64 * j, kb * kBK, zq,
                                 fb_leader, pol_q);
            } else {
              tma_load_3d_pair(qdst, &tmQ, kb * kBK, qc, zq, fb_leader, pol_q);
            }
          }
          if (it == 0) trace_mark(p, kTrFirstLoad);
        }
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
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      uint32_t it = 0, local = 0;
      bool ok = true;
      const uint32_t peer_empty0 = map_shared_rank(smem_u32(&empty_bar[0]), peer);
      const uint32_t peer_accf0 = map_shared_rank(smem_u32(&accf_bar[0]), peer);
      WorkIter wi(p, num_tiles, sk_width, sk_tiles, pair_id, num_pairs);
      Work w;
      for (; ok && wi.next(p, w); ++local) {
        const uint32_t a = ACC_BUFS == 2 ? (local & 1u) : 0u;
        const uint32_t aph = ACC_BUFS == 2 ? ((local >> 1) & 1u) : (local & 1u);
        if (!wait_phase<true>(smem_u32(&acce_bar[a]), aph ^ 1u, ctl, p, kStatusTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + a * TILE_N;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase<true>(smem_u32(&full_bar[s]), ph, ctl, p, kStatusTimeoutMma)) {
            ok = false;
            break;
          }
          if (it == 0) trace_mark(p, kTrFirstData);
          tc_fence_after();
          const uint32_t pbase = smem_u32(sP + s * P_BYTES);
          const uint32_t qbase = smem_u32(sQ + s * Q_BYTES);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t adesc = sw128_desc(pbase + k * 32, 16, 1024);
#pragma unroll
            for (int sub = 0; sub < NSUB; ++sub) {
              const uint32_t qb_addr = qbase + sub * QSUB_BYTES;
              const uint64_t bdesc = Q_MN ? sw128_desc(qb_addr + k * 16 * 128, kBK * 128, 1024)
                                          : sw128_desc(qb_addr + k * 32, 16, 1024);
              mma_f16<2>(d + sub * BN, adesc, bdesc, IDESC, (kb != w.kb0 || k != 0) ? 1u : 0u);
            }
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
    const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>(warp - 2) * (STAGE_EPI / 4);
    uint32_t stores = 0;
    uint32_t local = 0;
    const InT* bias = (p.epi & 1) ? reinterpret_cast<const InT*>(p.bias) : nullptr;
    const bool relu = (p.epi & 2) != 0;
    const uint32_t acce_leader0 = map_shared_rank(smem_u32(&acce_bar[0]), 0);
    const int row_local = quad * 32 + lane;  // this thread's accumulator row in this CTA
    const bool pieces_possible = p.work_mode != 0;  // uniform for the launch
    constexpr long long PART = static_cast<long long>(kBM) * TILE_N;  // floats per CTA partial
    // this warp is done reading accumulator `a`
    auto free_acc = [&](uint32_t a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_leader0 + a * 8u);
    };
    int gcur = 0;
    WorkIter wi(p, num_tiles, sk_width, sk_tiles, pair_id, num_pairs);
    Work w;
    for (; wi.next(p, w); ++local) {
      const PairTile c = pair_tile(w.t, gcur);
      const long long b = c.b;
      const int qb = c.qb;
      const InT* const bias_t =
          bias ? bias + b * (GROUPED ? static_cast<long long>(p.N) : p.stride_bias) : nullptr;
      const uint32_t a = ACC_BUFS == 2 ? (local & 1u) : 0u;
      const uint32_t aph = ACC_BUFS == 2 ? ((local >> 1) & 1u) : (local & 1u);
      BiasRegs<TILE_N, InT> br;
      br.load(bias_t, qb * TILE_N, p.N);
      const bool ok = wait_phase<true>(smem_u32(&accf_bar[a]), aph, ctl, p, kStatusTimeoutEpilogue);
      if (pieces_possible) {
        // the piece path syncs the four epilogue warps: one answer for all
        if (epilogue_bar_any(!ok || *reinterpret_cast<volatile int*>(&ctl->abort))) break;
      } else if (!__all_sync(0xffffffffu, ok)) {
        break;
      }
      if (warp == 2 && lane == 0 && local == 0) trace_mark(p, kTrFirstEpi);
      tc_fence_after();
      const int row0 = c.p0 + static_cast<int>(rank) * kBM + quad * 32;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * TILE_N;
      const TmemSrc tsrc{taddr};
      const long long cidx = 2 * w.t + rank;  // this CTA's counter for the tile
      const long long first_pair = pair_id - w.idx;
      bool finish = true;
      if (w.count > 1) {
        // one piece of a split tile: arrive on the counter (low 16 bits);
        // the last to arrive sums, every other piece parks its partial and
        // counts it written (high 16 bits)
        epilogue_bar();
        if (row_local == 0) {
          const unsigned old = atomicAdd(&p.counters[cidx], 1u);
          ctl->last = ((old & 0xFFFFu) == static_cast<unsigned>(w.count - 1)) ? 1 : 0;
        }
        epilogue_bar();
        finish = ctl->last != 0;
        if (!finish) {
          float* part = p.ws + piece_slot(p, w.t, w.idx, first_pair, static_cast<int>(rank), 2) * PART;
          // up to 64 columns per tensor-memory round trip
          constexpr int PW = TILE_N < 64 ? TILE_N : 64;
#pragma unroll 1
          for (int cc = 0; cc < TILE_N; cc += PW) {
            uint32_t v[PW];
            tsrc.get<PW>(cc, v);
#pragma unroll
            for (int h = 0; h < PW; h += 16)
              put_partial16(part, row_local, cc + h, *reinterpret_cast<uint32_t(*)[16]>(&v[h]));
          }
          free_acc(a);  // the accumulator is free again
          __threadfence();
          epilogue_bar();
          if (row_local == 0) atomicAdd(&p.counters[cidx], 0x10000u);
        } else {
          bool gave_up = false;
          if (row_local == 0) {
            // every other piece has arrived and writes its partial without
            // waiting on anything: a bounded wait
            const unsigned need = static_cast<unsigned>(w.count - 1);
            const volatile unsigned* cnt = p.counters + cidx;
            const uint64_t t0 = global_timer_ns();
            while ((*cnt >> 16) < need) {
              if (global_timer_ns() - t0 > p.timeout_ns) {
                atomicCAS(p.status, 0u, kStatusTimeoutEpilogue);
                *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
                gave_up = true;
                break;
              }
            }
            __threadfence();
          }
          if (epilogue_bar_any(gave_up)) break;
        }
      }
      if (!finish) continue;
      if (w.count > 1) {
        const PieceSumSrc psrc{tsrc, &p, w.t, first_pair, PART, w.count, w.idx, row_local,
                               static_cast<int>(rank), 2};
        if (!GROUPED && p.tma_store) {
          if (bias_t != nullptr)
            store_tile_from<TILE_N, InT, OutT, true>(psrc, row0, qb * TILE_N, static_cast<int>(b),
                                                     p, br, relu, stage, stores, &tmC);
          else
            store_tile_from<TILE_N, InT, OutT, false>(psrc, row0, qb * TILE_N,
                                                      static_cast<int>(b), p, br, relu, stage,
                                                      stores, &tmC);
        } else
          store_rows_from<TILE_N, InT, OutT>(
              psrc, row0 + lane, c.row_end, qb * TILE_N, p, bias_t, relu,
              reinterpret_cast<OutT*>(p.C) + (GROUPED ? 0 : b * p.stride_c));
        if (row_local == 0) p.counters[cidx] = 0u;  // ready for the next launch
      } else if (!GROUPED && p.tma_store) {
        if (bias_t != nullptr)
          store_tile_from<TILE_N, InT, OutT, true>(tsrc, row0, qb * TILE_N, static_cast<int>(b),
                                                   p, br, relu, stage, stores, &tmC);
        else
          store_tile_from<TILE_N, InT, OutT, false>(tsrc, row0, qb * TILE_N,
                                                    static_cast<int>(b), p, br, relu, stage,
                                                    stores, &tmC);
      } else if (GROUPED && p.tma_store) {
        // grouped: masked at the group's last row (tma_store: N whole 16-byte vectors)
        OutT* const Cg = reinterpret_cast<OutT*>(p.C);
        if (bias_t != nullptr)
          store_tile_rows<TILE_N, InT, OutT, true>(tsrc, row0, c.row_end, qb * TILE_N, p, br, relu,
                                                   stage, Cg);
        else
          store_tile_rows<TILE_N, InT, OutT, false>(tsrc, row0, c.row_end, qb * TILE_N, p, br,
                                                    relu, stage, Cg);
      } else {
        store_rows_from<TILE_N, InT, OutT>(
            tsrc, row0 + lane, c.row_end, qb * TILE_N, p, bias_t, relu,
            reinterpret_cast<OutT*>(p.C) + (GROUPED ? 0 : b * p.stride_c));
      }
      free_acc(a);
    }
    if (!GROUPED && lane == 0) tma_store_wait_read<0>();  // staging read; writes finish with the grid
    if (warp == 2 && lane == 0) trace_mark(p, kTrEpiDone);
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

template <int BN, int NSUB, int STAGES, bool GROUPED = false>
constexpr int gemm_pair_smem_bytes() {
  return 1024 + STAGES * (kBM * kBK * 2 + NSUB * (BN / 2) * kBK * 2) +
         static_cast<int>(GROUPED ? kEpiStageBytes / 2 : kEpiStageBytes) + (2 * STAGES + 5) * 8 +
         static_cast<int>(sizeof(SharedCtl)) + (GROUPED ? static_cast<int>(sizeof(GroupTable)) : 0);
}

}  // namespace dg16
