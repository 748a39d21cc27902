// gemm_kernel.cuh -- the persistent, warp-specialised tcgen05 GEMM kernel.
//
// One CTA per SM loops over output tiles.  Its six warps split the work:
//   warp 0      TMA producer: streams 64-deep K slices of the two operands
//               into a STAGES-deep shared-memory ring (the counterpart of the
//               pages' num_stages software pipelining, "FlagOS众智跨芯算子优化
//               实践" section 2.2), 128-byte swizzled so the tensor core reads
//               them without bank conflicts (the pages' padding / XOR swizzle
//               of section 2.3, done here by the copy engine itself).
//   warp 1      allocates tensor memory, then one lane issues tcgen05.mma
//               (128 x BN x 16 per instruction) into an fp32 accumulator in
//               TMEM; two accumulators alternate so the epilogue of one tile
//               overlaps the main loop of the next.
//   warps 2..5  epilogue: tcgen05.ld the accumulator, add bias, ReLU, round
//               to the output type and store ("用Triton跨芯片优化GEMM" section
//               3.4: bias + ReLU fused after the GEMM, one trip to memory).
// Tiles are visited in grouped-M order ("Triton 学习笔记" 2.3.7) so that the
// tiles in flight on all SMs share operand panels in L2.
//
// Operand naming: the MMA computes D[p, q] = sum_k P[p, k] * Q[q, k] with P
// the 128-row operand and Q the BN-row operand.  For C = A.B, P = A (K-major)
// and Q = B (K-major when B is column-major, MN-major when row-major).  In
// the swapped ("skinny") form, P = B stored N x K and Q = A, so D = C^T and the
// wide N dimension fills the 128 MMA rows while the few rows of A become the
// MMA's N.
//
// Every wait is bounded (see wait_phase); on a time-out the block records an
// error in the device status word, drains its own asynchronous work, frees
// its tensor memory and returns.
#pragma once

#include "kernel_common.cuh"

namespace dg16 {

// The kernel.
//   BN      Q rows per tile = MMA N (multiple of 16; of 64 when Q is MN-major)
//   STAGES  depth of the operand ring
//   Q_MN    Q operand is MN-major in memory (row-major B)
//   IN_BF16 inputs are bf16 (else fp16); InT is the matching CUDA type
//   TF32    inputs are fp32, multiplied as tf32 (tcgen05 kind::tf32); one
//           128-byte swizzle row then holds 32 elements instead of 64
//   OutT    output element type (__half, __nv_bfloat16 or float)
//   SWAP    P = B (N x K), Q = A: the accumulator holds C^T
//   GROUPED grouped GEMM (Q tensor map is 3-D: [group][rows][K or N])
template <int BN, int STAGES, bool Q_MN, bool IN_BF16, typename OutT, bool SWAP, bool GROUPED,
          bool TF32 = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ KParams p) {
  using InT = typename std::conditional<
      TF32, float, typename std::conditional<IN_BF16, __nv_bfloat16, __half>::type>::type;
  constexpr int ELEM = TF32 ? 4 : 2;           // input bytes
  constexpr int KB_EL = 128 / ELEM;            // K elements per stage (one swizzle row)
  constexpr int MN_CHUNK = 128 / ELEM;         // MN elements per MN-major box row
  constexpr int MMA_K = 32 / ELEM;             // K per MMA instruction (32 bytes)
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N must be 16..256, step 16");
  static_assert(!Q_MN || BN % (128 / (TF32 ? 4 : 2)) == 0,
                "MN-major Q tiles are whole 128-byte swizzle rows");
  static_assert(!(SWAP && GROUPED), "grouped GEMM uses the plain operand order");
  constexpr uint32_t P_BYTES = kBM * 128;     // 128 rows x one 128-byte K row
  constexpr uint32_t Q_BYTES = BN * 128;
  constexpr uint32_t STAGE_BYTES = P_BYTES + Q_BYTES;
  // Swapped (skinny) tiles have a tiny MMA-N, so chaining a tile's MMAs into
  // one accumulator would pay each MMA's full latency: consecutive MMAs (the
  // 32-byte K slices, across K blocks) rotate over NACC independent
  // accumulators instead, summed in order by the epilogue.
  constexpr int NACC = SWAP ? (BN <= 16 ? 8 : 4) : 1;
  constexpr int ACC_COLS = NACC * BN;  // TMEM columns per accumulator buffer
  constexpr uint32_t TMEM_COLS = (2 * ACC_COLS <= 32) ? 32 : (2 * ACC_COLS <= 64) ? 64
                                 : (2 * ACC_COLS <= 128) ? 128 : (2 * ACC_COLS <= 256) ? 256 : 512;
  constexpr uint32_t IDESC =
      TF32 ? mma_idesc(kBM, BN, 2u, Q_MN ? 1u : 0u) : f16_idesc(kBM, BN, IN_BF16 ? 1u : 0u, 0u, Q_MN ? 1u : 0u);
  // dense tiles store through shared memory and TMA; grouped tiles must not
  // write past their group's last row and swapped tiles are transposed, so
  // those store from registers
  constexpr bool TMA_EPI = !GROUPED && !SWAP;
  constexpr uint32_t STAGE_EPI = TMA_EPI ? kEpiStageBytes : 0u;

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms (8 rows x 128 B)
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
  if (threadIdx.x == 0) trace_mark(p, kTrEntry);

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
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    if constexpr (TMA_EPI) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish<1>();
  }
  if constexpr (GROUPED) {
    if (warp == 2 && lane == 0) {
      // per-group tile prefix from the device counts (no host sync)
      int tiles = 0, rows = 0;
      const int nq = (p.N + BN - 1) / BN;
      bool bad = false;
      for (int g = 0; g < p.num_groups; ++g) {
        int m = __ldg(&p.group_rows[g]);
        if (m < 0) {
          m = 0;
          bad = true;
        }
        gt->tile_start[g] = tiles;
        gt->row_start[g] = rows;
        // rows past the stated total are never read or written
        const int usable = max(0, min(m, p.M - rows));
        if (usable < m) bad = true;
        tiles += (usable + kBM - 1) / kBM * nq;
        rows += usable;
      }
      gt->tile_start[p.num_groups] = tiles;
      gt->row_start[p.num_groups] = rows;
      if (bad && blockIdx.x == 0) atomicCAS(p.status, 0u, kStatusBadGroups);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  if (threadIdx.x == 0) trace_mark(p, kTrSetup);

  long long num_tiles = p.num_tiles;
  if constexpr (GROUPED) num_tiles = gt->tile_start[p.num_groups];
  // grouped stream-K: the width follows from the tile count computed above
  // (the host cannot know it); the hybrid mode derives its split here for
  // both kinds.  The same values in every role.
  long long sk_width = 0, sk_tiles = 0;
  if (p.work_mode == 3)
    hybrid_split(num_tiles, p.num_kb, &sk_tiles, &sk_width);
  else if (GROUPED && p.work_mode == 2)
    sk_width =
        max(1ll, (num_tiles * p.num_kb + gridDim.x - 1) / static_cast<long long>(gridDim.x));
  const int num_q_blocks = GROUPED ? (p.N + BN - 1) / BN : p.num_q;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_p = make_policy(p.pol_p);
      const uint64_t pol_q = make_policy(p.pol_q);
      uint32_t it = 0;
      int gcur = 0;
      bool ok = true;
      WorkIter wi(p, num_tiles, sk_width, sk_tiles);
      Work w;
      while (ok && wi.next(p, w)) {
        const TileCoord c = tile_coord<GROUPED>(w.t, p, num_q_blocks, gt, gcur);
        if (!c.valid) break;
        const int q0 = c.q0 * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase(smem_u32(&empty_bar[s]), ph ^ 1u, ctl, p, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          if constexpr (GROUPED)
            tma_load_2d(smem_u32(sP + s * P_BYTES), &tmP, kb * KB_EL, c.p0, fb, pol_p);
          else
            tma_load_3d(smem_u32(sP + s * P_BYTES), &tmP, kb * KB_EL, c.p0, c.zp, fb, pol_p);
          const uint32_t qdst = smem_u32(sQ + s * Q_BYTES);
          // Q is 3-D: [group][rows][cols] (grouped) or [batch][rows][cols]
          if constexpr (Q_MN) {
#pragma unroll
            for (int j = 0; j < BN / MN_CHUNK; ++j)
              tma_load_3d(qdst + j * (KB_EL * 128), &tmQ, q0 + MN_CHUNK * j, kb * KB_EL, c.zq,
                          fb, pol_q);
          } else {
            tma_load_3d(qdst, &tmQ, kb * KB_EL, q0, c.zq, fb, pol_q);
          }
          if (it == 0) trace_mark(p, kTrFirstLoad);
        }
      }
      if (!ok) {
        // leave no copy in flight into this block's shared memory
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j)
          wait_phase_drain(smem_u32(&full_bar[j % STAGES]), (j / STAGES) & 1u, 50000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      int gcur = 0;
      bool ok = true;
      WorkIter wi(p, num_tiles, sk_width, sk_tiles);
      Work w;
      for (; ok && wi.next(p, w); ++local) {
        const TileCoord c = tile_coord<GROUPED>(w.t, p, num_q_blocks, gt, gcur);
        if (!c.valid) break;
        const uint32_t a = local & 1u;
        const uint32_t aph = (local >> 1) & 1u;
        if (!wait_phase(smem_u32(&acce_bar[a]), aph ^ 1u, ctl, p, kStatusTimeoutMma)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + a * ACC_COLS;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase(smem_u32(&full_bar[s]), ph, ctl, p, kStatusTimeoutMma)) {
            ok = false;
            break;
          }
          if (it == 0) trace_mark(p, kTrFirstData);
          tc_fence_after();
          const uint32_t pbase = smem_u32(sP + s * P_BYTES);
          const uint32_t qbase = smem_u32(sQ + s * Q_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // four 32-byte K slices per 128-byte row
            // K-major: the k-th 16-element slice starts 32 bytes further
            // along each 128-byte swizzled row; 8-row groups are 1024 B apart.
            const uint64_t adesc = sw128_desc(pbase + k * 32, 16, 1024);
            // MN-major: MMA_K rows of 128 B per slice; 128-byte MN chunks are
            // KB_EL rows apart; K-row groups (8 rows; 4 rows for tf32, whose
            // 32-byte-atom swizzle repeats every 4 rows) 1024 / 512 B apart.
            const uint64_t bdesc =
                Q_MN ? (TF32 ? sw128_desc(qbase + k * MMA_K * 128, KB_EL * 128, 512, 1)
                             : sw128_desc(qbase + k * MMA_K * 128, KB_EL * 128, 1024))
                     : sw128_desc(qbase + k * 32, 16, 1024);
            // MMA number `step` of the tile goes to accumulator step % NACC;
            // the first NACC of them start their accumulator from zero
            const int step = (kb - w.kb0) * 4 + k;
            const uint32_t d = d0 + static_cast<uint32_t>((step % NACC) * BN);
            const uint32_t acc = step >= NACC ? 1u : 0u;
            if constexpr (TF32)
              mma_tf32<1>(d, adesc, bdesc, IDESC, acc);
            else
              mma_f16<1>(d, adesc, bdesc, IDESC, acc);
          }
          mma_commit<1>(smem_u32(&empty_bar[s]));  // frees the stage when read
        }
        if (!ok) break;
        mma_commit<1>(smem_u32(&accf_bar[a]));  // accumulator ready
      }
      trace_mark(p, kTrLastMma);
      // every MMA this thread issued has completed before tensor memory is freed
      mma_commit<1>(smem_u32(drain_bar));
      wait_phase_drain(smem_u32(drain_bar), 0, 50000000ull);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32*quad ..
    const int row_local = quad * 32 + lane;
    const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>(warp - 2) * 8192u;
    uint32_t stores = 0;  // this warp's TMA stores so far
    uint32_t local = 0;
    int gcur = 0;
    OutT* const C0 = reinterpret_cast<OutT*>(p.C);
    const InT* const bias = reinterpret_cast<const InT*>(p.bias);
    const bool has_bias = (p.epi & 1) != 0;
    const bool relu = (p.epi & 2) != 0;
    const bool pieces_possible = p.work_mode != 0;  // uniform for the launch
    constexpr long long PART = static_cast<long long>(kBM) * BN;  // floats per partial tile
    WorkIter wi(p, num_tiles, sk_width, sk_tiles);
    Work w;
    for (; wi.next(p, w); ++local) {
      const TileCoord c = tile_coord<GROUPED>(w.t, p, num_q_blocks, gt, gcur);
      if (!c.valid) break;
      const uint32_t a = local & 1u;
      const uint32_t aph = (local >> 1) & 1u;
      BiasRegs<BN, InT> br;
      if (!SWAP && TMA_EPI && has_bias)
        br.load(bias + static_cast<long long>(c.group) * (GROUPED ? p.N : p.stride_bias), c.q0 * BN,
                p.N);
      // every lane waits; the warp proceeds only if all saw the phase, so the
      // .sync.aligned TMEM loads below are always issued by the whole warp
      const bool ok = wait_phase(smem_u32(&accf_bar[a]), aph, ctl, p, kStatusTimeoutEpilogue);
      if (pieces_possible) {
        // the piece path below syncs the four epilogue warps, so they must
        // agree on leaving: one reduced answer for all 128 threads
        if (epilogue_bar_any(!ok || *reinterpret_cast<volatile int*>(&ctl->abort))) break;
      } else if (!__all_sync(0xffffffffu, ok)) {
        break;
      }
      if (warp == 2 && lane == 0 && local == 0) trace_mark(p, kTrFirstEpi);
      tc_fence_after();
      const int prow = c.p0 + row_local;  // this thread's accumulator row
      const int q0 = c.q0 * BN;
      // this tile's output and bias (grouped: the group's bias row; dense:
      // the batch's output and bias)
      OutT* const C = GROUPED ? C0 : C0 + static_cast<long long>(c.group) * p.stride_c;
      const InT* const bias_t =
          !has_bias ? nullptr
                    : (GROUPED ? bias + static_cast<long long>(c.group) * p.N
                               : bias + static_cast<long long>(c.group) * p.stride_bias);
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + a * ACC_COLS;
      const TmemSrc tsrc{taddr, min(NACC, 4 * (w.kb1 - w.kb0)), BN};
      bool finish = true;  // this block stores the tile
      if (w.count > 1) {
        // ---- one piece of a split tile.  The tile's counter holds arrivals
        // in its low 16 bits and written partials in its high 16 bits.  The
        // last piece to arrive waits for the others' partials and sums all
        // pieces (its own straight from tensor memory); every other piece
        // parks its partial and signals it.
        epilogue_bar();
        if (row_local == 0) {
          const unsigned old = atomicAdd(&p.counters[w.t], 1u);
          ctl->last = ((old & 0xFFFFu) == static_cast<unsigned>(w.count - 1)) ? 1 : 0;
        }
        epilogue_bar();
        finish = ctl->last != 0;
        if (!finish) {
          float* part =
              p.ws + piece_slot(p, w.t, w.idx, static_cast<long long>(blockIdx.x) - w.idx) * PART;
          // up to 64 columns per tensor-memory round trip
          constexpr int PW = BN < 64 ? BN : 64;
#pragma unroll 1
          for (int cc = 0; cc < BN; cc += PW) {
            uint32_t v[PW];
            tsrc.get<PW>(cc, v);
#pragma unroll
            for (int h = 0; h < PW; h += 16)
              put_partial16(part, row_local, cc + h, *reinterpret_cast<uint32_t(*)[16]>(&v[h]));
          }
          tc_fence_before();
          mbar_arrive(smem_u32(&acce_bar[a]));  // the accumulator is free again
          __threadfence();
          epilogue_bar();
          if (row_local == 0) atomicAdd(&p.counters[w.t], 0x10000u);
        } else {
          bool gave_up = false;
          if (row_local == 0) {
            // every other piece has arrived, so each is writing its partial
            // and will signal without waiting on anything: a bounded wait
            const unsigned need = static_cast<unsigned>(w.count - 1);
            const volatile unsigned* cnt = p.counters + w.t;
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
      if (finish) {
        const PieceSumSrc psrc{tsrc,    &p,      w.t,   static_cast<long long>(blockIdx.x) - w.idx,
                               PART,    w.count, w.idx, row_local};
        if constexpr (!SWAP) {
          const InT* bias_g = bias_t;
          if (TMA_EPI && p.tma_store) {
            if (w.count > 1 && bias_g != nullptr)
              store_tile_from<BN, InT, OutT, true>(psrc, c.p0 + quad * 32, q0, c.group, p, br,
                                                   relu, stage, stores, &tmC);
            else if (w.count > 1)
              store_tile_from<BN, InT, OutT, false>(psrc, c.p0 + quad * 32, q0, c.group, p, br,
                                                    relu, stage, stores, &tmC);
            else if (bias_g != nullptr)
              store_tile_from<BN, InT, OutT, true>(tsrc, c.p0 + quad * 32, q0, c.group, p, br,
                                                   relu, stage, stores, &tmC);
            else
              store_tile_from<BN, InT, OutT, false>(tsrc, c.p0 + quad * 32, q0, c.group, p, br,
                                                    relu, stage, stores, &tmC);
          } else {
            // accumulator row = output row prow, columns q0 .. q0+BN
            if (w.count > 1)
              store_rows_from<BN, InT, OutT>(psrc, prow, c.row_end, q0, p, bias_g, relu, C);
            else
              store_rows_from<BN, InT, OutT>(tsrc, prow, c.row_end, q0, p, bias_g, relu, C);
          }
        } else {
          // accumulator row = output column prow (an N index); accumulator
          // columns are output rows q0 .. q0+BN
          const bool col_ok = prow < p.N;
          const float b = (has_bias && col_ok) ? to_f32<InT>(bias_t[prow]) : 0.0f;
#pragma unroll 1
          for (int cc = 0; cc < BN; cc += 16) {
            const int row0 = q0 + cc;
            if (row0 >= p.M) break;  // warp-uniform
            uint32_t v[16];
            if (w.count > 1)
              psrc.get<16>(cc, v);
            else
              tsrc.get<16>(cc, v);
            if (col_ok) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                if (row0 + j < p.M) {
                  float x = __uint_as_float(v[j]) + b;
                  if (relu) x = fmaxf(x, 0.0f);
                  C[static_cast<long long>(row0 + j) * p.ldc + prow] = from_f32<OutT>(x);
                }
              }
            }
          }
        }
        if (w.count > 1 && row_local == 0) p.counters[w.t] = 0u;  // ready for the next launch
        tc_fence_before();
        mbar_arrive(smem_u32(&acce_bar[a]));  // this block's accumulator has been read
      }
    }
    // every TMA store has finished reading shared memory before the block
    // retires; the writes themselves complete before the grid does
    if (TMA_EPI && lane == 0) tma_store_wait_read<0>();
    if (warp == 2 && lane == 0) trace_mark(p, kTrEpiDone);
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

// Shared memory a kernel instance needs (bytes, including alignment slack).
template <int BN, int STAGES, bool GROUPED, bool SWAP = false>
constexpr int gemm_smem_bytes() {
  return 1024 + STAGES * (kBM * 128 + BN * 128) +
         ((!GROUPED && !SWAP) ? static_cast<int>(kEpiStageBytes) : 0) + (2 * STAGES + 5) * 8 +
         static_cast<int>(sizeof(SharedCtl)) + (GROUPED ? static_cast<int>(sizeof(GroupTable)) : 0);
}

// C = act(bias) (or zeros) for K == 0: the definition with an empty sum,
// for `batch` outputs stride_c elements apart (bias stride_bias apart).
template <typename InT, typename OutT>
__global__ void fill_bias_kernel(int batch, int M, int N, OutT* C, long long ldc,
                                 long long stride_c, const InT* bias, long long stride_bias,
                                 int epi) {
  const long long per = static_cast<long long>(M) * N;
  const long long total = per * batch;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long b = i / per, rc = i - b * per;
    const int r = static_cast<int>(rc / N), c = static_cast<int>(rc % N);
    float x = (epi & 1) ? to_f32<InT>(bias[b * stride_bias + c]) : 0.0f;
    if (epi & 2) x = fmaxf(x, 0.0f);
    C[b * stride_c + static_cast<long long>(r) * ldc + c] = from_f32<OutT>(x);
  }
}

// Grouped K == 0: every stored row gets act(bias_g).
template <typename InT, typename OutT>
__global__ void fill_bias_grouped_kernel(int num_groups, const int* group_rows, int total_rows,
                                         int N, OutT* C, long long ldc, const InT* bias, int epi) {
  int row0 = 0;
  for (int g = 0; g < num_groups; ++g) {
    const int m = max(0, min(group_rows[g], total_rows - row0));
    const long long total = static_cast<long long>(m) * N;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
      const int r = row0 + static_cast<int>(i / N), c = static_cast<int>(i % N);
      float x = (epi & 1) ? to_f32<InT>(bias[static_cast<long long>(g) * N + c]) : 0.0f;
      if (epi & 2) x = fmaxf(x, 0.0f);
      C[static_cast<long long>(r) * ldc + c] = from_f32<OutT>(x);
    }
    row0 += m;
  }
}

}  // namespace dg16
