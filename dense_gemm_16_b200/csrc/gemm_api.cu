// gemm_api.cu -- the C ABI (include/dense_gemm.h): argument checks, tensor
// maps, config choice and launches.  All compute runs in the kernels of
// gemm_kernel.cuh; nothing here touches matrix data.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <algorithm>
#include <unordered_set>
#include <vector>

#include "../../include/dense_gemm.h"
#include "config_table.h"
#include "dispatch.h"
#include "gemm_kernel.cuh"
#include "gemm_kernel_gswap.cuh"
#include "raster.h"

namespace dg16 {

__device__ unsigned g_status_word;  // watchdog / argument status (first error wins)

// One block waits on a barrier nothing completes; the bounded wait must give
// up and record a time-out.
__global__ void watchdog_selftest_kernel(unsigned* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ SharedCtl ctl;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    KParams p{};
    p.status = status;
    p.timeout_ns = timeout_ns;
    wait_phase(smem_u32(&bar), 0, &ctl, p, kStatusTimeoutSelftest);
  }
  __syncthreads();
}


namespace {

constexpr unsigned kEpiMask = GEMM_EPI_BIAS | GEMM_EPI_RELU | GEMM_B_COL_MAJOR;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
constexpr int kMaxDevices = 64;

std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};
// gemm_set_trace: the caller's trace buffer and how many blocks it holds
std::atomic<unsigned long long*> g_trace{nullptr};
std::atomic<int> g_trace_blocks{0};

// Stamp the current trace setting into a launch's parameters.
void set_trace(KParams& kp) {
  kp.trace = g_trace.load();
  kp.trace_blocks = kp.trace ? g_trace_blocks.load() : 0;
}
std::atomic<int> g_forced_config{-1};

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  unsigned* status = nullptr;
  std::unordered_set<const void*> attr_set;  // kernels whose smem limit is raised
};
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

int cuda_fail(cudaError_t e) {
  (void)cudaGetLastError();  // clear a non-sticky error so later calls are unaffected
  (void)e;
  return GEMM_ERR_CUDA;
}

// Split-K scratch, one buffer per (device, stream): calls on one stream run
// in order, so they can share it; calls on different streams never do.
// Layout: [kCounterSlots tile counters][kSchedSlots tile-queue counters]
// [partial tiles]; the counters are zeroed once and every kernel leaves
// them at 0.
constexpr size_t kCounterSlots = 65536;
constexpr size_t kSchedSlots = 64;  // slot 0: the grouped-swap tile queue
constexpr size_t kCounterBytes = (kCounterSlots + kSchedSlots) * sizeof(unsigned);
struct Workspace {
  int device;
  cudaStream_t stream;
  int slot;  // 0: split/stream-K pieces (counters + partials); 1: im2col matrix
  void* ptr;
  size_t bytes;
};
std::mutex g_ws_mu;
std::vector<Workspace> g_ws;

// Plain per-(device, stream, slot) scratch of at least `bytes` (slot 1 and
// up; contents undefined).  Same growth rule as stream_workspace.
int stream_buffer(int device, cudaStream_t stream, int slot, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace* w = nullptr;
  for (auto& e : g_ws)
    if (e.device == device && e.stream == stream && e.slot == slot) w = &e;
  if (!w || w->bytes < bytes) {
    if (w) {
      cudaError_t e = cudaStreamSynchronize(stream);
      if (e != cudaSuccess) return cuda_fail(e);
      cudaFree(w->ptr);
      w->ptr = nullptr;
      w->bytes = 0;
    } else {
      g_ws.push_back({device, stream, slot, nullptr, 0});
      w = &g_ws.back();
    }
    const size_t sz = std::max(bytes, static_cast<size_t>(16) << 20);
    void* ptr = nullptr;
    cudaError_t e = cudaMalloc(&ptr, sz);
    if (e != cudaSuccess) return cuda_fail(e);
    w->ptr = ptr;
    w->bytes = sz;
  }
  *out = w->ptr;
  return GEMM_OK;
}

// Scratch of at least `partial_bytes` after the counters for (device, stream).
// The first call per stream allocates (cudaMalloc) and zeroes the counters;
// a larger request waits for the stream, frees the old buffer and allocates
// anew.  Kernels leave every counter at 0, so no per-call reset is needed.
int stream_workspace(int device, cudaStream_t stream, size_t partial_bytes, float** ws,
                     unsigned** counters) {
  std::lock_guard<std::mutex> lk(g_ws_mu);
  const size_t need = kCounterBytes + partial_bytes;
  Workspace* w = nullptr;
  for (auto& e : g_ws)
    if (e.device == device && e.stream == stream && e.slot == 0) w = &e;
  if (!w || w->bytes < need) {
    if (w) {
      cudaError_t e = cudaStreamSynchronize(stream);
      if (e != cudaSuccess) return cuda_fail(e);
      cudaFree(w->ptr);
      w->ptr = nullptr;
      w->bytes = 0;
    } else {
      g_ws.push_back({device, stream, 0, nullptr, 0});
      w = &g_ws.back();
    }
    const size_t bytes = std::max(need, static_cast<size_t>(16) << 20);
    void* ptr = nullptr;
    cudaError_t e = cudaMalloc(&ptr, bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemsetAsync(ptr, 0, kCounterBytes, stream);
    if (e != cudaSuccess) {
      cudaFree(ptr);
      return cuda_fail(e);
    }
    w->ptr = ptr;
    w->bytes = bytes;
  }
  *counters = static_cast<unsigned*>(w->ptr);
  *ws = reinterpret_cast<float*>(static_cast<char*>(w->ptr) + kCounterBytes);
  return GEMM_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;


// Device state for the current device, initialised once.
int device_state(DeviceState** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (major != 10) return GEMM_ERR_UNSUPPORTED;  // built for sm_100a only
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e);
    s.num_sms = sms;
    s.status = static_cast<unsigned*>(p);
    s.ready = true;
  }
  *out = &s;
  return GEMM_OK;
}

int ensure_smem_attr(DeviceState* s, const KernelEntry& k) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (s->attr_set.count(k.fn)) return GEMM_OK;
  cudaError_t e =
      cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, k.smem);
  if (e != cudaSuccess) return cuda_fail(e);
  s->attr_set.insert(k.fn);
  return GEMM_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else
      (void)cudaGetLastError();
  });
  return g_encode;
}

// A 2- or 3-D tensor map with 128-byte swizzle and zero fill outside the
// tensor.  dims[0] is the contiguous dimension; strides in bytes.
int make_map_t(CUtensorMap* m, const void* base, CUtensorMapDataType type, int rank,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto enc = encoder();
  if (!enc) return GEMM_ERR_CUDA;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = enc(m, type, rank, const_cast<void*>(base), gd, gs, bx, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GEMM_OK : GEMM_ERR_CUDA;
}

// 16-bit operand map (A or B).
int make_map(CUtensorMap* m, const void* base, bool bf16, int rank, const uint64_t* dims,
             const uint64_t* strides_bytes, const uint32_t* box) {
  return make_map_t(m, base, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                    rank, dims, strides_bytes, box);
}

// Output map for the TMA-store epilogue: M x N with leading dimension ldc,
// boxes of 32 rows x 128 bytes (64 16-bit or 32 fp32 outputs).  TMA stores
// clip at M and N.
int make_c_map(CUtensorMap* m, void* C, int M, int N, int64_t ldc, int dtype) {
  const int ob = (dtype == GEMM_F16_OUT_F32 || dtype == GEMM_BF16_OUT_F32) ? 4 : 2;
  const CUtensorMapDataType t = ob == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : (dtype == GEMM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  const uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
  const uint64_t stride = static_cast<uint64_t>(ldc) * ob;
  const uint32_t box[2] = {static_cast<uint32_t>(128 / ob), 32u};
  return make_map_t(m, C, t, 2, dims, &stride, box);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int out_bytes(int dtype) {
  return (dtype == GEMM_F16_OUT_F32 || dtype == GEMM_BF16_OUT_F32 || dtype == GEMM_F32_TF32) ? 4
                                                                                             : 2;
}
bool in_bf16(int dtype) { return dtype == GEMM_BF16 || dtype == GEMM_BF16_OUT_F32; }
bool in_tf32(int dtype) { return dtype == GEMM_F32_TF32; }
int in_bytes(int dtype) { return in_tf32(dtype) ? 4 : 2; }
// K elements per ring stage: one 128-byte swizzle row
int kb_elems(int dtype) { return 128 / in_bytes(dtype); }
CUtensorMapDataType in_map_type(int dtype) {
  return in_tf32(dtype) ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                        : (in_bf16(dtype) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

// Checks shared by gemm() and grouped_gemm() once sizes are known.
int check_common(int N, int K, const void* A, int64_t lda, const void* B, int64_t ldb, void* C,
                 int64_t ldc, const void* bias, unsigned epi, int dtype) {
  if (!C) return GEMM_ERR_INVALID_ARG;
  if ((epi & GEMM_EPI_BIAS) && !bias) return GEMM_ERR_INVALID_ARG;
  if (ldc < N) return GEMM_ERR_INVALID_ARG;
  if (!aligned16(C) || (ldc * out_bytes(dtype)) % 16 != 0) return GEMM_ERR_MISALIGNED;
  if ((epi & GEMM_EPI_BIAS) &&
      (reinterpret_cast<uintptr_t>(bias) & static_cast<uintptr_t>(in_bytes(dtype) - 1)))
    return GEMM_ERR_MISALIGNED;
  if (K > 0) {
    if (!A || !B) return GEMM_ERR_INVALID_ARG;
    const bool bcol = (epi & GEMM_B_COL_MAJOR) != 0;
    if (lda < K || ldb < (bcol ? K : N)) return GEMM_ERR_INVALID_ARG;
    const int per16 = 16 / in_bytes(dtype);  // elements per 16 bytes
    if (!aligned16(A) || !aligned16(B) || lda % per16 != 0 || ldb % per16 != 0)
      return GEMM_ERR_MISALIGNED;
  }
  return GEMM_OK;
}

int check_dtype_epi(unsigned epi, int dtype) {
  if (dtype < GEMM_F16 || dtype > GEMM_F32_TF32) return GEMM_ERR_UNSUPPORTED;
  if (epi & ~kEpiMask) return GEMM_ERR_UNSUPPORTED;
  return GEMM_OK;
}

// The kernel instance for a config and problem variant.
KernelEntry kernel_for(const Config& c, bool q_mn, bool bf16, bool f32, bool grouped,
                       bool tf32 = false) {
  if (tf32) {  // fp32 inputs: single-CTA dense tiles only
    if (c.kind != kKindSingle || grouped) return {nullptr, 0};
    return kernels_tf32(c.bn, q_mn);
  }
  if (c.kind == kKindSwap) {
    if (q_mn || grouped) return {nullptr, 0};  // needs column-major B
    return kernels_swap(c.bn, bf16, f32);
  }
  if (c.kind == kKindClusterSplitK) {
    if (grouped) return {nullptr, 0};
    return kernels_csk(c.bn, q_mn, bf16, f32);
  }
  if (c.kind == kKindClusterSplitKSwap) {
    if (q_mn || grouped) return {nullptr, 0};  // needs column-major B
    return kernels_csk_swap(c.bn, bf16, f32);
  }
  if (c.kind == kKindGroupedSwap || c.kind == kKindGroupedSwapPair) {
    if (!grouped) return {nullptr, 0};
    return c.kind == kKindGroupedSwap ? kernels_gswap(c.bn, q_mn, bf16, f32)
                                      : kernels_gswap2(c.bn, q_mn, bf16, f32);
  }
  if (c.kind == kKindPair) {
    if (grouped) return kernels_pair_grouped(c.bn, q_mn, bf16, f32);
    return kernels_pair(c.bn, c.stages, q_mn, bf16, f32);
  }
  if (c.bn == 256) return kernels_bn256(q_mn, bf16, f32, grouped);
  if (c.bn == 128) return kernels_bn128(q_mn, bf16, f32, grouped);
  if (c.bn == 64) return kernels_bn64(q_mn, bf16, f32, grouped);
  return {nullptr, 0};
}

int launch(const KernelEntry& k, int grid, cudaStream_t stream, const CUtensorMap& tp,
           const CUtensorMap& tq, const CUtensorMap& tc, const KParams& kp, int cluster = 1) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = k.smem;
  cfg.stream = stream;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  if (cluster > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  KParams kpt = kp;
  set_trace(kpt);
  void* args[4] = {const_cast<CUtensorMap*>(&tp), const_cast<CUtensorMap*>(&tq),
                   const_cast<CUtensorMap*>(&tc), &kpt};
  cudaError_t e = cudaLaunchKernelExC(&cfg, k.fn, args);
  return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

int select_config(int M, int N, int K, unsigned epi, bool grouped) {
  const int forced = g_forced_config.load();
  if (forced >= 0) return forced;
  return table_lookup(M, N, K, (epi & GEMM_B_COL_MAJOR) != 0, grouped);
}

// The config a dense call runs: the table's (or the forced) choice, with two
// substitutions when the choice came from the table: fp32 inputs run on the
// single-CTA tf32 kernels only, and the CTA-pair split-K kernel, which needs
// one SM pair per tile and two K blocks, gives way to 128 x 128 tiles when a
// (batched) problem has more tiles than that.
int dense_config(int batch, int M, int N, int K, unsigned epi, int dtype, const DeviceState* ds) {
  int cid = select_config(M, N, K, epi, false);
  if (cid < 0 || cid >= kNumConfigs || g_forced_config.load() >= 0) return cid;
  if (in_tf32(dtype) && kConfigs[cid].kind != kKindSingle) {
    const long long tiles256 = static_cast<long long>((M + 127) / 128) * ((N + 255) / 256);
    return (N <= 128 || tiles256 < 96) ? 1 : 0;
  }
  const int kind = kConfigs[cid].kind;
  if (kind == kKindClusterSplitK || kind == kKindClusterSplitKSwap) {
    const bool sw = kind == kKindClusterSplitKSwap;
    const int rows = sw ? N : M, cols = sw ? M : N;  // MMA rows / MMA-N of the tiles
    const long long tiles = static_cast<long long>(batch) * ((rows + kBM - 1) / kBM) *
                            ((cols + kConfigs[cid].bn - 1) / kConfigs[cid].bn);
    if (tiles > ds->num_sms / 2 || (K + kBK - 1) / kBK < 2) return sw ? 21 : 1;
  }
  return cid;
}

// One dense (optionally strided-batched) problem as the entry points take it.
struct DenseProblem {
  int batch, M, N, K;
  const void* A;
  int64_t lda, stride_a;
  const void* B;
  int64_t ldb, stride_b;
  void* C;
  int64_t ldc, stride_c;
  const void* bias;
  int64_t stride_bias;
  unsigned epi;
  int dtype;
};

// Batch strides: an operand is either shared by every batch (stride 0) or
// its batches do not overlap; outputs never overlap; every stride a TMA map
// uses is a multiple of 16 bytes.
int check_batch(const DenseProblem& d) {
  if (d.stride_a < 0 || d.stride_b < 0 || d.stride_c < 0 || d.stride_bias < 0)
    return GEMM_ERR_INVALID_ARG;
  if (d.batch <= 1) return GEMM_OK;
  const bool bcol = (d.epi & GEMM_B_COL_MAJOR) != 0;
  const int64_t ext_a = d.lda * d.M;
  const int64_t ext_b = bcol ? d.ldb * d.N : d.ldb * d.K;
  if (d.K > 0) {
    if (d.stride_a != 0 && d.stride_a < ext_a) return GEMM_ERR_INVALID_ARG;
    if (d.stride_b != 0 && d.stride_b < ext_b) return GEMM_ERR_INVALID_ARG;
    const int ib = in_bytes(d.dtype);
    if ((d.stride_a * ib) % 16 != 0 || (d.stride_b * ib) % 16 != 0) return GEMM_ERR_MISALIGNED;
  }
  if (d.stride_c < d.ldc * d.M) return GEMM_ERR_INVALID_ARG;
  if ((d.stride_c * out_bytes(d.dtype)) % 16 != 0) return GEMM_ERR_MISALIGNED;
  return GEMM_OK;
}

template <typename InT, typename OutT>
int launch_fill(const DenseProblem& d, cudaStream_t stream) {
  const long long total = static_cast<long long>(d.M) * d.N * d.batch;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 4096));
  fill_bias_kernel<InT, OutT><<<blocks, 256, 0, stream>>>(
      d.batch, d.M, d.N, static_cast<OutT*>(d.C), d.ldc, d.batch > 1 ? d.stride_c : 0,
      static_cast<const InT*>(d.bias), d.batch > 1 ? d.stride_bias : 0,
      static_cast<int>(d.epi & 3));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

int fill_dispatch(const DenseProblem& d, cudaStream_t stream) {
  switch (d.dtype) {
    case GEMM_F32_TF32: return launch_fill<float, float>(d, stream);
    case GEMM_F16: return launch_fill<__half, __half>(d, stream);
    case GEMM_BF16: return launch_fill<__nv_bfloat16, __nv_bfloat16>(d, stream);
    case GEMM_F16_OUT_F32: return launch_fill<__half, float>(d, stream);
    default: return launch_fill<__nv_bfloat16, float>(d, stream);
  }
}

// Fixed scratch for callers that must not allocate (gemm_splitk_noalloc).
struct FixedScratch {
  unsigned* counters;
  size_t counter_slots;
  float* ws;
  size_t partial_bytes;
};

// Plan and launch one dense problem with config `cfg`; `splits` overrides
// the config's split factor (1 whole tiles, > 1 split-K, -1 stream-K).  The
// pieces' scratch comes from the per-stream workspace, or from `fixed`.
int run_dense(DeviceState* ds, const DenseProblem& d, const Config& cfg, int splits,
              const FixedScratch* fixed, cudaStream_t stream) {
  const int M = d.M, N = d.N, K = d.K;
  const bool bcol = (d.epi & GEMM_B_COL_MAJOR) != 0;
  const bool bf16 = in_bf16(d.dtype);
  const bool tf32 = in_tf32(d.dtype);
  const bool f32 = out_bytes(d.dtype) == 4;
  const bool swap = cfg.kind == kKindSwap || cfg.kind == kKindClusterSplitKSwap;
  const bool pair = cfg.kind == kKindPair;
  const bool csk = cfg.kind == kKindClusterSplitK || cfg.kind == kKindClusterSplitKSwap;
  const KernelEntry k = kernel_for(cfg, swap ? false : !bcol, bf16, f32, false, tf32);
  const int ib = in_bytes(d.dtype);
  const uint32_t kbe = static_cast<uint32_t>(kb_elems(d.dtype));  // K per stage
  const CUtensorMapDataType it = in_map_type(d.dtype);
  if (!k.fn || (swap && !bcol)) return GEMM_ERR_UNSUPPORTED;

  // batch extents of the 3-D maps: a shared operand has one batch
  const bool bat = d.batch > 1;
  const uint64_t nb_a = (bat && d.stride_a) ? d.batch : 1, nb_b = (bat && d.stride_b) ? d.batch : 1;
  const uint64_t sa = (bat && d.stride_a) ? d.stride_a : d.lda * M;
  const uint64_t sb = (bat && d.stride_b) ? d.stride_b : (bcol ? d.ldb * N : d.ldb * K);
  const uint64_t str_a[2] = {static_cast<uint64_t>(d.lda) * ib, sa * ib};
  const uint64_t str_b[2] = {static_cast<uint64_t>(d.ldb) * ib, sb * ib};

  CUtensorMap tp, tq, tc;
  std::memset(&tc, 0, sizeof(tc));  // swapped tiles store from registers
  const int ob = out_bytes(d.dtype);
  const bool tma_store = !swap && (static_cast<int64_t>(N) * ob) % 16 == 0;
  int rc;
  if (tma_store) {
    const CUtensorMapDataType t = ob == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : (bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    const uint64_t sc = bat ? d.stride_c : d.ldc * M;
    const uint64_t dims[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                              static_cast<uint64_t>(d.batch)};
    const uint64_t str[2] = {static_cast<uint64_t>(d.ldc) * ob, sc * ob};
    const uint32_t box[3] = {static_cast<uint32_t>(128 / ob), 32u, 1u};
    rc = make_map_t(&tc, d.C, t, 3, dims, str, box);
    if (rc) return rc;
  }
  KParams kp = {};
  kp.tma_store = tma_store ? 1 : 0;
  kp.M = M;
  kp.N = N;
  kp.K = K;
  kp.num_kb = static_cast<int>((K + kbe - 1) / kbe);
  kp.group_m = cfg.group_m;
  kp.C = d.C;
  kp.ldc = d.ldc;
  kp.bias = d.bias;
  kp.epi = static_cast<int>(d.epi & 3);
  kp.status = ds->status;
  kp.timeout_ns = g_timeout_ns.load();
  kp.stride_c = bat ? d.stride_c : 0;
  kp.stride_bias = bat ? d.stride_bias : 0;
  if (!swap) {
    const uint64_t dA[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M), nb_a};
    const uint32_t bA[3] = {kbe, static_cast<uint32_t>(kBM), 1u};
    rc = make_map_t(&tp, d.A, it, 3, dA, str_a, bA);
    if (rc) return rc;
    if (bcol) {
      // the pair kernel's CTAs each load half of the tile's B columns
      // (pair tiles wider than 256 are several N=256 MMAs, each split in two)
      const uint64_t dB[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), nb_b};
      const uint32_t rows_b = pair ? static_cast<uint32_t>(std::min(cfg.bn, 256) / 2)
                                   : static_cast<uint32_t>(cfg.bn);
      const uint32_t bB[3] = {kbe, rows_b, 1u};
      rc = make_map_t(&tq, d.B, it, 3, dB, str_b, bB);
    } else {
      // MN-major B: boxes one 128-byte row of N wide, one stage of K deep
      // (MN-major tf32 must use the 128-byte swizzle with 32-byte atoms)
      const uint64_t dB[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(K), nb_b};
      const uint32_t bB[3] = {static_cast<uint32_t>(128 / ib), kbe, 1u};
      rc = make_map_t(&tq, d.B, it, 3, dB, str_b, bB,
                      tf32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (rc) return rc;
    const int rows_per_tile = pair ? 2 * kBM : kBM;
    kp.num_p = (M + rows_per_tile - 1) / rows_per_tile;
    kp.num_q = (N + cfg.bn - 1) / cfg.bn;
    kp.z_p = nb_a > 1 ? 1 : 0;
    kp.z_q = nb_b > 1 ? 1 : 0;
  } else {
    // P = B stored N x K, Q = A (M x K); the accumulator is C^T
    const uint64_t dB[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), nb_b};
    const uint32_t bB[3] = {kbe, static_cast<uint32_t>(kBM), 1u};
    rc = make_map_t(&tp, d.B, it, 3, dB, str_b, bB);
    if (rc) return rc;
    const uint64_t dA[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M), nb_a};
    const uint32_t bA[3] = {kbe, static_cast<uint32_t>(cfg.bn), 1u};
    rc = make_map_t(&tq, d.A, it, 3, dA, str_a, bA);
    if (rc) return rc;
    kp.num_p = (N + kBM - 1) / kBM;
    kp.num_q = (M + cfg.bn - 1) / cfg.bn;
    kp.z_p = nb_b > 1 ? 1 : 0;
    kp.z_q = nb_a > 1 ? 1 : 0;
  }
  kp.tiles_per_batch = static_cast<long long>(kp.num_p) * kp.num_q;
  kp.num_tiles = kp.tiles_per_batch * d.batch;
  kp.pol_p = cfg.pol_p;
  kp.pol_q = cfg.pol_q;
  kp.work_mode = 0;
  kp.splits = 1;
  kp.kb_per_split = kp.num_kb;
  kp.slot_stride = 1;
  // workers: blocks, or CTA pairs for the pair kernel, whose two CTAs keep
  // their own counters and partial slots for their 128-row halves
  const int ranks = pair ? 2 : 1;
  const int workers = ds->num_sms / ranks;
  int grid_units = static_cast<int>(std::min<long long>(kp.num_tiles, workers));
  const size_t counter_cap = fixed ? fixed->counter_slots : kCounterSlots;
  if (!csk && splits != 1 && kp.num_kb >= 2 &&
      kp.num_tiles * ranks <= static_cast<long long>(counter_cap)) {
    if (splits > 1) {
      // split-K: every tile's K range in `splits` equal pieces
      const int per = (kp.num_kb + splits - 1) / splits;
      kp.work_mode = 1;
      kp.kb_per_split = per;
      kp.splits = (kp.num_kb + per - 1) / per;  // no empty K range
      kp.slot_stride = kp.splits;
      grid_units = static_cast<int>(std::min<long long>(kp.num_tiles * kp.splits, workers));
    } else if (splits == -2) {
      // hybrid: stream-K over the last waves' tiles, whole tiles before
      // them; the kernel derives the split from the tile count and grid
      kp.work_mode = 3;
      kp.sk_width = 1;
      grid_units = static_cast<int>(std::min<long long>(kp.num_tiles, workers));
    } else {
      // stream-K: every block gets an equal share of the (tile, K block)
      // iterations, cut at tile edges
      const long long total = kp.num_tiles * kp.num_kb;
      kp.work_mode = 2;
      kp.sk_width = (total + workers - 1) / workers;
      grid_units = static_cast<int>((total + kp.sk_width - 1) / kp.sk_width);
      kp.slot_stride = static_cast<int>((kp.num_kb + kp.sk_width - 1) / kp.sk_width) + 1;
    }
    if (kp.work_mode == 1 && kp.splits == 1) kp.work_mode = 0;
  }
  if (kp.work_mode != 0) {
    // split-K: slot_stride slots per tile; stream-K: two per block
    const size_t slots = (kp.work_mode >= 2 ? 2 * static_cast<size_t>(grid_units)
                                            : static_cast<size_t>(kp.num_tiles) * kp.slot_stride) *
                         ranks;
    const size_t partial = slots * kBM * cfg.bn * 4;
    if (fixed) {
      if (partial > fixed->partial_bytes) return GEMM_ERR_UNSUPPORTED;  // beyond the scratch
      kp.ws = fixed->ws;
      kp.counters = fixed->counters;
      // counters left by an earlier call that gave up early must not leak in
      cudaError_t e = cudaMemsetAsync(
          kp.counters, 0, static_cast<size_t>(kp.num_tiles) * ranks * sizeof(unsigned), stream);
      if (e != cudaSuccess) return cuda_fail(e);
    } else {
      int dev = 0;
      cudaError_t e = cudaGetDevice(&dev);
      if (e != cudaSuccess) return cuda_fail(e);
      rc = stream_workspace(dev, stream, partial, &kp.ws, &kp.counters);
      if (rc) return rc;
    }
  } else if (fixed && splits > 1 && kp.num_tiles * ranks > static_cast<long long>(counter_cap)) {
    return GEMM_ERR_UNSUPPORTED;  // beyond the scratch's tile counters
  }
  rc = ensure_smem_attr(ds, k);
  if (rc) return rc;
  if (pair) return launch(k, 2 * grid_units, stream, tp, tq, tc, kp, 2);
  if (csk) {
    // one CTA pair per tile, each CTA one half of the K blocks
    if (kp.num_tiles > ds->num_sms / 2 || kp.num_kb < 2) return GEMM_ERR_UNSUPPORTED;
    return launch(k, static_cast<int>(2 * kp.num_tiles), stream, tp, tq, tc, kp, 2);
  }
  return launch(k, grid_units, stream, tp, tq, tc, kp);
}

template <typename InT, typename OutT>
int launch_fill_grouped(int G, const int32_t* rows, int total, int N, void* C, int64_t ldc,
                        const void* bias, unsigned epi, cudaStream_t stream) {
  fill_bias_grouped_kernel<InT, OutT><<<512, 256, 0, stream>>>(
      G, rows, total, N, static_cast<OutT*>(C), ldc, static_cast<const InT*>(bias),
      static_cast<int>(epi & 3));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

}  // namespace
}  // namespace dg16

using namespace dg16;

extern "C" {

const char* gemm_version(void) { return "dense_gemm_16_b200 0.1 (sm_100a, tcgen05)"; }

const char* gemm_status_string(int status) {
  switch (status) {
    case GEMM_OK: return "GEMM_OK";
    case GEMM_ERR_INVALID_ARG: return "GEMM_ERR_INVALID_ARG: invalid argument";
    case GEMM_ERR_UNSUPPORTED: return "GEMM_ERR_UNSUPPORTED: unsupported dtype, flag or config";
    case GEMM_ERR_MISALIGNED:
      return "GEMM_ERR_MISALIGNED: pointers must be 16-byte aligned and leading dimensions "
             "16-byte multiples";
    case GEMM_ERR_CUDA: return "GEMM_ERR_CUDA: a CUDA call failed (or no usable device)";
    case GEMM_ERR_DEVICE_TIMEOUT: return "GEMM_ERR_DEVICE_TIMEOUT: a kernel's bounded wait ran out";
    default: return "unknown gemm_status";
  }
}

int gemm(int M, int N, int K, const void* A, int64_t lda, const void* B, int64_t ldb, void* C,
         int64_t ldc, const void* bias, unsigned epilogue, int dtype, void* stream_) {
  return gemm_strided_batched(1, M, N, K, A, lda, 0, B, ldb, 0, C, ldc, 0, bias, 0, epilogue, dtype,
                              stream_);
}

int gemm_strided_batched(int batch, int M, int N, int K, const void* A, int64_t lda,
                         int64_t stride_a, const void* B, int64_t ldb, int64_t stride_b, void* C,
                         int64_t ldc, int64_t stride_c, const void* bias, int64_t stride_bias,
                         unsigned epilogue, int dtype, void* stream_) {
  int rc = check_dtype_epi(epilogue, dtype);
  if (rc) return rc;
  if (batch < 0 || M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_ARG;
  if (batch == 0 || M == 0 || N == 0) return GEMM_OK;
  rc = check_common(N, K, A, lda, B, ldb, C, ldc, bias, epilogue, dtype);
  if (rc) return rc;
  DenseProblem d{batch, M, N, K, A, lda, stride_a, B, ldb, stride_b, C, ldc, stride_c, bias,
                 stride_bias, epilogue, dtype};
  rc = check_batch(d);
  if (rc) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc) return rc;
  if (K == 0) return fill_dispatch(d, stream);
  const int cid = dense_config(batch, M, N, K, epilogue, dtype, ds);
  if (cid < 0 || cid >= kNumConfigs) return GEMM_ERR_UNSUPPORTED;
  return run_dense(ds, d, kConfigs[cid], kConfigs[cid].splits, nullptr, stream);
}

int conv2d_im2col(int batch, int H, int W, int cin, int cout, int KH, int KW, int stride_h,
                  int stride_w, int pad_h, int pad_w, int dil_h, int dil_w, const void* x,
                  const void* w, void* y, const void* bias, unsigned epilogue, int dtype,
                  void* stream_) {
  int rc = check_dtype_epi(epilogue, dtype);
  if (rc) return rc;
  if (epilogue & GEMM_B_COL_MAJOR) return GEMM_ERR_UNSUPPORTED;  // the filter layout is fixed
  if (in_tf32(dtype)) return GEMM_ERR_UNSUPPORTED;               // 16-bit activations only
  if (batch < 0 || H < 1 || W < 1 || cin < 1 || cout < 1 || KH < 1 || KW < 1 || stride_h < 1 ||
      stride_w < 1 || pad_h < 0 || pad_w < 0 || dil_h < 1 || dil_w < 1)
    return GEMM_ERR_INVALID_ARG;
  const int OH = (H + 2 * pad_h - dil_h * (KH - 1) - 1) / stride_h + 1;
  const int OW = (W + 2 * pad_w - dil_w * (KW - 1) - 1) / stride_w + 1;
  if (OH < 1 || OW < 1) return GEMM_ERR_INVALID_ARG;
  if (batch == 0) return GEMM_OK;
  if (!x || !w || !y || ((epilogue & GEMM_EPI_BIAS) && !bias)) return GEMM_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) ||
      (static_cast<int64_t>(cout) * out_bytes(dtype)) % 16 != 0 || cout % 8 != 0)
    return GEMM_ERR_MISALIGNED;
  const long long M = static_cast<long long>(batch) * OH * OW;
  const long long K = static_cast<long long>(KH) * KW * cin;
  if (M > INT32_MAX || K > INT32_MAX) return GEMM_ERR_UNSUPPORTED;
  const long long lda = (K + 7) / 8 * 8;  // 16-byte rows for the TMA
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  void* A = nullptr;
  rc = stream_buffer(dev, stream, 1, static_cast<size_t>(M) * lda * 2, &A);
  if (rc) return rc;
  e = launch_im2col(x, A, lda, batch, H, W, cin, KH, KW, stride_h, stride_w, pad_h, pad_w, dil_h,
                    dil_w, OH, OW, ds->num_sms, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  const DenseProblem d{1,     static_cast<int>(M), cout, static_cast<int>(K), A, lda, 0, w, cout,
                       0,     y, cout, 0, bias, 0, epilogue, dtype};
  const int cid = dense_config(1, d.M, d.N, d.K, epilogue, dtype, ds);
  if (cid < 0 || cid >= kNumConfigs) return GEMM_ERR_UNSUPPORTED;
  return run_dense(ds, d, kConfigs[cid], kConfigs[cid].splits, nullptr, stream);
}

// Grouped GEMM with swapped operands (gemm_gswap_kernel, or the CTA-pair
// gemm_gswap2_kernel): W_g is the 128-row (pair: 256-row) MMA operand, X's
// rows the MMA's N; tiles come from a counter in the stream's scratch, which
// every launch leaves at 0.
int launch_grouped_swap(DeviceState* ds, const KernelEntry& k, const Config& cfg, int num_groups,
                        const int32_t* group_rows, int total_rows, int N, int K, const void* A,
                        int64_t lda, const void* B, int64_t ldb, int64_t stride_b, void* C,
                        int64_t ldc, const void* bias, unsigned epilogue, bool bf16,
                        cudaStream_t stream) {
  const bool bcol = (epilogue & GEMM_B_COL_MAJOR) != 0;
  CUtensorMap tw;
  const uint64_t sW[2] = {static_cast<uint64_t>(ldb) * 2,
                          num_groups > 1 ? static_cast<uint64_t>(stride_b) * 2
                                         : static_cast<uint64_t>(bcol ? N : K) * ldb * 2};
  int rc;
  if (bcol) {  // W_g stored N x K: K-major boxes of 64 K x 128 columns
    const uint64_t d[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                           static_cast<uint64_t>(num_groups)};
    const uint32_t b[3] = {static_cast<uint32_t>(kBK), static_cast<uint32_t>(kBM), 1u};
    rc = make_map(&tw, B, bf16, 3, d, sW, b);
  } else {  // W_g stored K x N: MN-major boxes of 64 columns x 64 K
    const uint64_t d[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                           static_cast<uint64_t>(num_groups)};
    const uint32_t b[3] = {64u, static_cast<uint32_t>(kBK), 1u};
    rc = make_map(&tw, B, bf16, 3, d, sW, b);
  }
  if (rc) return rc;
  RowMaps tx;
  const uint64_t dX[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(total_rows)};
  const uint64_t sX = static_cast<uint64_t>(lda) * 2;
  for (int i = 0; i < 5; ++i) {
    const uint32_t b[2] = {static_cast<uint32_t>(kBK), static_cast<uint32_t>(128 >> i)};
    rc = make_map(&tx.m[i], A, bf16, 2, dX, &sX, b);
    if (rc) return rc;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  float* ws = nullptr;
  unsigned* counters = nullptr;
  rc = stream_workspace(dev, stream, 0, &ws, &counters);
  if (rc) return rc;

  KParams kp = {};
  kp.M = total_rows;
  kp.N = N;
  kp.K = K;
  kp.num_kb = (K + kBK - 1) / kBK;
  kp.group_m = 1;
  kp.C = C;
  kp.ldc = ldc;
  kp.bias = bias;
  kp.epi = static_cast<int>(epilogue & 3);
  kp.group_rows = group_rows;
  kp.num_groups = num_groups;
  kp.status = ds->status;
  kp.timeout_ns = g_timeout_ns.load();
  kp.pol_p = cfg.pol_p;
  kp.pol_q = cfg.pol_q;
  kp.counters = counters + kCounterSlots;  // the tile-queue counter
  set_trace(kp);
  const bool pair = cfg.kind == kKindGroupedSwapPair;
  const long long cols = pair ? 2 * kBM : kBM;
  const long long nb = (N + cols - 1) / cols;
  const long long max_tiles = (static_cast<long long>(total_rows) / cfg.bn + num_groups) * nb;
  const int grid = pair ? 2 * static_cast<int>(std::min<long long>(max_tiles, ds->num_sms / 2))
                        : static_cast<int>(std::min<long long>(max_tiles, ds->num_sms));
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  lc.gridDim = dim3(grid, 1, 1);
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = k.smem;
  lc.stream = stream;
  if (pair) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
  }
  void* args[3] = {&tw, &tx, &kp};
  e = cudaLaunchKernelExC(&lc, k.fn, args);
  return e == cudaSuccess ? GEMM_OK : cuda_fail(e);
}

int grouped_gemm(int num_groups, const int32_t* group_rows, int total_rows, int N, int K,
                 const void* A, int64_t lda, const void* B, int64_t ldb, int64_t stride_b,
                 void* C, int64_t ldc, const void* bias, unsigned epilogue, int dtype,
                 void* stream_) {
  int rc = check_dtype_epi(epilogue, dtype);
  if (rc) return rc;
  if (num_groups < 1 || num_groups > kMaxGroups || !group_rows) return GEMM_ERR_INVALID_ARG;
  if (total_rows < 0 || N < 0 || K < 0 || stride_b < 0) return GEMM_ERR_INVALID_ARG;
  if (total_rows == 0 || N == 0) return GEMM_OK;
  rc = check_common(N, K, A, lda, B, ldb, C, ldc, bias, epilogue, dtype);
  if (rc) return rc;
  if ((reinterpret_cast<uintptr_t>(group_rows) & 3u) != 0) return GEMM_ERR_MISALIGNED;
  const bool bcol = (epilogue & GEMM_B_COL_MAJOR) != 0;
  if (K > 0) {
    // each group's B must fit before the next one starts
    const int64_t one = bcol ? static_cast<int64_t>(N) * ldb : static_cast<int64_t>(K) * ldb;
    if (num_groups > 1 && stride_b < one) return GEMM_ERR_INVALID_ARG;
    if ((stride_b * 2) % 16 != 0) return GEMM_ERR_MISALIGNED;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc) return rc;
  if (in_tf32(dtype)) return GEMM_ERR_UNSUPPORTED;  // grouped runs 16-bit inputs only
  const bool bf16 = in_bf16(dtype);
  const bool f32 = out_bytes(dtype) == 4;
  if (K == 0) {
    switch (dtype) {
      case GEMM_F16:
        return launch_fill_grouped<__half, __half>(num_groups, group_rows, total_rows, N, C, ldc,
                                                   bias, epilogue, stream);
      case GEMM_BF16:
        return launch_fill_grouped<__nv_bfloat16, __nv_bfloat16>(
            num_groups, group_rows, total_rows, N, C, ldc, bias, epilogue, stream);
      case GEMM_F16_OUT_F32:
        return launch_fill_grouped<__half, float>(num_groups, group_rows, total_rows, N, C, ldc,
                                                  bias, epilogue, stream);
      default:
        return launch_fill_grouped<__nv_bfloat16, float>(num_groups, group_rows, total_rows, N,
                                                         C, ldc, bias, epilogue, stream);
    }
  }
  const int cid = select_config(total_rows, N, K, epilogue, true);
  if (cid < 0 || cid >= kNumConfigs) return GEMM_ERR_UNSUPPORTED;
  const Config& cfg = kConfigs[cid];
  const KernelEntry k = kernel_for(cfg, !bcol, bf16, f32, true);
  if (!k.fn) return GEMM_ERR_UNSUPPORTED;
  rc = ensure_smem_attr(ds, k);
  if (rc) return rc;
  if (cfg.kind == kKindGroupedSwap || cfg.kind == kKindGroupedSwapPair)
    return launch_grouped_swap(ds, k, cfg, num_groups, group_rows, total_rows, N, K, A, lda, B,
                               ldb, stride_b, C, ldc, bias, epilogue, bf16, stream);

  CUtensorMap tp, tq;
  const bool pair = cfg.kind == kKindPair;
  const uint64_t lda_b = static_cast<uint64_t>(lda) * 2;
  if (pair) {  // the pair kernel copies A with 3-D boxes (one batch)
    const uint64_t dA[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(total_rows), 1};
    const uint64_t sA[2] = {lda_b, lda_b * static_cast<uint64_t>(total_rows)};
    const uint32_t bA[3] = {static_cast<uint32_t>(kBK), static_cast<uint32_t>(kBM), 1u};
    rc = make_map(&tp, A, bf16, 3, dA, sA, bA);
  } else {
    const uint64_t dA[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(total_rows)};
    const uint32_t bA[2] = {static_cast<uint32_t>(kBK), static_cast<uint32_t>(kBM)};
    rc = make_map(&tp, A, bf16, 2, dA, &lda_b, bA);
  }
  if (rc) return rc;
  const uint64_t sB[2] = {static_cast<uint64_t>(ldb) * 2, static_cast<uint64_t>(stride_b) * 2};
  // a single group may pass stride_b = 0; give the map a valid stride
  uint64_t sB_fix[2] = {sB[0], num_groups > 1 ? sB[1] : (bcol ? N : K) * sB[0]};
  if (bcol) {
    const uint64_t dB[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(num_groups)};
    // each CTA of a pair loads half of every N=256 MMA's B rows
    const uint32_t rows_b = pair ? static_cast<uint32_t>(std::min(cfg.bn, 256) / 2)
                                 : static_cast<uint32_t>(cfg.bn);
    const uint32_t bB[3] = {static_cast<uint32_t>(kBK), rows_b, 1u};
    rc = make_map(&tq, B, bf16, 3, dB, sB_fix, bB);
  } else {
    const uint64_t dB[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                            static_cast<uint64_t>(num_groups)};
    const uint32_t bB[3] = {64u, static_cast<uint32_t>(kBK), 1u};
    rc = make_map(&tq, B, bf16, 3, dB, sB_fix, bB);
  }
  if (rc) return rc;

  KParams kp = {};
  kp.M = total_rows;
  kp.N = N;
  kp.K = K;
  kp.num_kb = (K + kBK - 1) / kBK;
  kp.group_m = cfg.group_m;
  kp.C = C;
  kp.ldc = ldc;
  kp.bias = bias;
  kp.epi = static_cast<int>(epilogue & 3);
  kp.group_rows = group_rows;
  kp.num_groups = num_groups;
  kp.status = ds->status;
  kp.timeout_ns = g_timeout_ns.load();
  kp.pol_p = cfg.pol_p;
  kp.pol_q = cfg.pol_q;
  kp.work_mode = 0;
  kp.splits = 1;
  kp.kb_per_split = kp.num_kb;
  kp.slot_stride = 1;
  kp.sk_width = 1;
  // upper bound on tiles: each group adds at most one partial row block
  const long long nq = (N + cfg.bn - 1) / cfg.bn;
  const long long max_tiles = (static_cast<long long>(total_rows) / kBM + num_groups) * nq;
  CUtensorMap tc;
  std::memset(&tc, 0, sizeof(tc));  // grouped tiles store from registers
  if (pair) {
    // 256-row pair tiles; one cluster of two CTAs per pair.  Rows whose N
    // columns are whole 16-byte vectors leave by vector stores of staged
    // row segments (flag reused from the dense TMA store)
    kp.tma_store = (static_cast<int64_t>(N) * (f32 ? 4 : 2)) % 16 == 0 ? 1 : 0;
    const long long max_pair_tiles =
        (static_cast<long long>(total_rows) / (2 * kBM) + num_groups) * nq;
    const int pairs = static_cast<int>(std::min<long long>(max_pair_tiles, ds->num_sms / 2));
    return launch(k, 2 * pairs, stream, tp, tq, tc, kp, 2);
  }
  const int grid = static_cast<int>(std::min<long long>(max_tiles, ds->num_sms));
  if (cfg.splits < 0 && kp.num_kb >= 2 && max_tiles <= static_cast<long long>(kCounterSlots)) {
    // stream-K (-1) or the hybrid (-2) over the (tile, K block) space; the
    // kernel derives the width from the tile count it computes from the
    // group sizes
    kp.work_mode = cfg.splits == -2 ? 3 : 2;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    rc = stream_workspace(dev, stream, 2 * static_cast<size_t>(grid) * kBM * cfg.bn * 4, &kp.ws,
                          &kp.counters);
    if (rc) return rc;
  }
  return launch(k, grid, stream, tp, tq, tc, kp);
}

int gemm_device_status(void* stream_, int clear) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned w = 0;
  e = cudaMemcpy(&w, ds->status, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    const unsigned zero = 0;
    e = cudaMemcpy(ds->status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (w == kStatusOk) return GEMM_OK;
  if (w == kStatusBadGroups) return GEMM_ERR_INVALID_ARG;
  return GEMM_ERR_DEVICE_TIMEOUT;
}

int gemm_free_scratch(void* stream_, int all_streams) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  std::lock_guard<std::mutex> lk(g_ws_mu);
  int rc = GEMM_OK;
  for (auto it = g_ws.begin(); it != g_ws.end();) {
    if (it->device != dev || (!all_streams && it->stream != stream)) {
      ++it;
      continue;
    }
    e = cudaStreamSynchronize(it->stream);
    if (e != cudaSuccess) {
      rc = cuda_fail(e);
      ++it;
      continue;
    }
    cudaFree(it->ptr);
    it = g_ws.erase(it);
  }
  return rc;
}

int gemm_set_trace(void* buffer, int64_t bytes) {
  if (buffer && (reinterpret_cast<uintptr_t>(buffer) & 7u) != 0) return GEMM_ERR_MISALIGNED;
  const int64_t blocks = buffer ? bytes / static_cast<int64_t>(8 * kTraceEvents) : 0;
  if (blocks <= 0) {
    g_trace.store(nullptr);
    g_trace_blocks.store(0);
    return GEMM_OK;
  }
  g_trace_blocks.store(static_cast<int>(std::min<int64_t>(blocks, INT32_MAX)));
  g_trace.store(static_cast<unsigned long long*>(buffer));
  return GEMM_OK;
}

uint64_t gemm_set_timeout_ns(uint64_t ns) {
  return g_timeout_ns.exchange(ns ? ns : kDefaultTimeoutNs);
}

int gemm_watchdog_selftest(uint64_t timeout_ns, void* stream_) {
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc) return rc;
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return GEMM_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(ds->status, timeout_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return gemm_device_status(stream_, 1);
}

int gemm_num_configs(void) { return kNumConfigs; }

int gemm_config_name(int id, char* buf, int buflen) {
  if (id < 0 || id >= kNumConfigs) return GEMM_ERR_UNSUPPORTED;
  if (!buf || buflen <= 0) return GEMM_ERR_INVALID_ARG;
  std::snprintf(buf, static_cast<size_t>(buflen), "%s", kConfigs[id].name);
  return GEMM_OK;
}

int gemm_select_config(int M, int N, int K, int dtype, unsigned epilogue) {
  int rc = check_dtype_epi(epilogue, dtype);
  if (rc) return rc;
  if (M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_ARG;
  return select_config(M, N, K, epilogue, false);
}

int gemm_force_config(int id) {
  if (id < -1 || id >= kNumConfigs) return GEMM_ERR_UNSUPPORTED;
  g_forced_config.store(id);
  return GEMM_OK;
}

int64_t gemm_smem_ring_bytes(int bm, int bn, int bk, int stages, int elem_bytes) {
  if (bm < 0 || bn < 0 || bk < 0 || stages < 0 || elem_bytes < 0) return -1;
  return (static_cast<int64_t>(bm) * bk + static_cast<int64_t>(bk) * bn) * elem_bytes * stages;
}

int gemm_k_iterations(int K, int bk) {
  if (K < 0 || bk <= 0) return -1;
  return (K + bk - 1) / bk;
}

int gemm_tile_coord(int64_t tile, int grid_m, int grid_n, int group_m, int* m_block,
                    int* n_block) {
  if (tile < 0 || grid_m <= 0 || grid_n <= 0 || group_m <= 0 || !m_block || !n_block)
    return GEMM_ERR_INVALID_ARG;
  if (tile >= static_cast<int64_t>(grid_m) * grid_n) return GEMM_ERR_INVALID_ARG;
  int m = 0, n = 0;
  raster_tile(tile, grid_m, grid_n, group_m, m, n);
  *m_block = m;
  *n_block = n;
  return GEMM_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Split-K with library-owned scratch (gemm_splitk_noalloc).  The scratch is a
// fixed array inside this module, so the entry point never allocates.

// One array per device that loads the library: 16 KiB of tile counters, then
// fp32 partial tiles.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GEMM_NOALLOC_SCRATCH_BYTES];

namespace dg16 {
namespace {

constexpr size_t kNoAllocCounterSlots = 4096;
constexpr size_t kNoAllocCounterBytes = kNoAllocCounterSlots * sizeof(unsigned);
constexpr int kNoAllocTileConfig = 1;  // tc1_128x128_s6_g8
constexpr int kNoAllocSwapConfig = 2;  // swap_128x16_s8
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// `g_noalloc_scratch` names a host-side stand-in, not device memory, so its
// address is looked up once per device (with that device current).
int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GEMM_OK;
}

}  // namespace
}  // namespace dg16

extern "C" int gemm_splitk_noalloc(int M, int N, int K, const void* A, int64_t lda,
                                   const void* B, int64_t ldb, void* C, int64_t ldc,
                                   const void* bias, unsigned epilogue, int dtype, int splits,
                                   void* stream_) {
  int rc = check_dtype_epi(epilogue, dtype);
  if (rc) return rc;
  if (M < 0 || N < 0 || K < 0 || splits < 1 || splits > 64) return GEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return GEMM_OK;
  rc = check_common(N, K, A, lda, B, ldb, C, ldc, bias, epilogue, dtype);
  if (rc) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc) return rc;
  const DenseProblem d{1, M, N, K, A, lda, 0, B, ldb, 0, C, ldc, 0, bias, 0, epilogue, dtype};
  if (K == 0) return fill_dispatch(d, stream);
  const bool swap = (epilogue & GEMM_B_COL_MAJOR) != 0 && M <= 32;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  FixedScratch fs;
  fs.counters = static_cast<unsigned*>(scratch);
  fs.counter_slots = kNoAllocCounterSlots;
  fs.ws = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kNoAllocCounterBytes);
  fs.partial_bytes = GEMM_NOALLOC_SCRATCH_BYTES - kNoAllocCounterBytes;
  return run_dense(ds, d, kConfigs[swap ? kNoAllocSwapConfig : kNoAllocTileConfig], splits, &fs,
                   stream);
}
