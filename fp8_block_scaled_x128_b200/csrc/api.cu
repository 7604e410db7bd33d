// api.cu -- host side of the C ABI declared in include/fp8gemm.h: argument
// validation, per-device capability cache, TMA tensor-map encoding, kernel
// variant table and selection, launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8gemm.h"
#include "fp8gemm_testing.h"
#include "kernel.cuh"
#include "kernel_pair.cuh"
#include "kernel_bf16.cuh"
#include "kernel_ue8m0.cuh"

using namespace fp8g;

namespace {

// ---------------------------------------------------------------- variants
using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, Params);

struct Variant {
  const char* name;
  int kind;
  bool swap;
  int bnc, stages, split;
  bool reg_split;  // setmaxnreg variant: needs exactly launch_regs at launch
  KernelFn fn;
  int smem;
  bool pair;        // CTA pairs (clusters of two) sharing a 256 x bnc tile
  int threads;      // threads per CTA
  int launch_regs;  // register-split variants: registers per thread at launch
  bool tma_store = false;  // m-lanes TMA-store epilogue: the third tensor map is D
};

template <bool kSwap, int BNC, int STAGES, int KIND, int SPLIT, int OPT = 0>
Variant make_variant(const char* name) {
  constexpr bool kStore = (OPT & kOptTmaStore) != 0;
  using L = Layout<kSwap, BNC, STAGES, SPLIT, kStore>;
  return Variant{name,     KIND, kSwap, BNC, STAGES, SPLIT, L::kRegSplit,
                 &fp8_gemm_kernel<kSwap, BNC, STAGES, KIND, SPLIT, OPT>, L::kSmemAlloc, false,
                 kThreads, kLaunchRegs, kStore};
}

template <int STAGES, bool kTmaStore>
Variant make_bf16_variant(const char* name) {
  return Variant{name, kBf16Dense, false, 256, STAGES, 1, false, &bf16_gemm_pair_kernel<STAGES, kTmaStore>,
                 Bf16Layout<STAGES, kTmaStore>::kSmemAlloc, true, kBf16Threads, 0};
}

template <int STAGES>
Variant make_ue8m0_variant(const char* name) {
  return Variant{name, kUe8m0Dense, false, 256, STAGES, 1, false, &fp8_gemm_ue8m0_kernel<STAGES>,
                 Ue8Layout<STAGES>::kSmemAlloc, false, kUe8Threads, 0};
}

template <int KIND, int STAGES, int BN, int OPT = 0, int NWG = default_nwg(BN)>
Variant make_pair_variant(const char* name) {
  using S = PairShape<BN, NWG>;
  return Variant{name, KIND, false, BN, STAGES, 1, S::kRegSplit, &fp8_gemm_pair_kernel<KIND, STAGES, BN, OPT, NWG>,
                 PairLayout<STAGES, BN>::kSmemAlloc, true, S::kThreads, S::kLaunchRegs};
}

// "nlanes": TMEM lanes are rows of B (small M); "mlanes": lanes are rows of A.
// Every entry is reachable: select_variant picks it for some call, or it is
// the fallback of one (cluster split-K without a workspace, single-CTA tiles
// when too few pair tiles fill the GPU), or fp8_gemm_nt_no_alloc runs it.
const Variant kVariants[] = {
    make_variant<true, 64, 6, kDense, 8>("dense_nlanes_bn64_st6_splitk8"),
    make_variant<true, 64, 6, kDense, 4>("dense_nlanes_bn64_st6_splitk4"),
    make_variant<true, 64, 6, kDense, 2>("dense_nlanes_bn64_st6_splitk2"),
    make_variant<true, 64, 8, kDense, 1>("dense_nlanes_bn64_st8"),
    make_variant<true, 64, 8, kDense, kGlobalSplit>("dense_nlanes_bn64_st8_gsplit"),
    make_variant<true, 64, 8, kDense, kGlobalSplitPartials>("dense_nlanes_bn64_st8_gsplit_2k"),
    make_variant<false, 128, 6, kDense, 1>("dense_mlanes_bn128_st6"),
    make_variant<false, 256, 4, kDense, 1>("dense_mlanes_bn256_st4"),
    make_pair_variant<kDense, 6, 192, kOptFma2>("dense_mlanes_pair_bn192_st6_f"),
    make_variant<false, 128, 6, kContiguous, 1>("contiguous_mlanes_bn128_st6"),
    make_variant<false, 256, 4, kContiguous, 1>("contiguous_mlanes_bn256_st4"),
    make_variant<false, 256, 4, kContiguous, 1, kOptTmaStore>("contiguous_mlanes_bn256_st4_tmastore"),
    make_variant<false, 128, 6, kMasked, 1>("masked_mlanes_bn128_st6"),
    make_variant<false, 256, 4, kMasked, 1>("masked_mlanes_bn256_st4"),
    make_pair_variant<kMasked, 6, 192, kOptFma2>("masked_mlanes_pair_bn192_st6_f"),
    make_bf16_variant<6, false>("bf16_pair_bn256_st6"),
    make_bf16_variant<6, true>("bf16_pair_bn256_st6_tmastore"),
    make_ue8m0_variant<4>("ue8m0_mlanes_bn256_st4"),
};
constexpr int kNumVariants = static_cast<int>(sizeof(kVariants) / sizeof(kVariants[0]));
enum : int {
  V_DENSE_SPLIT = 0,
  V_DENSE_SPLIT4,
  V_DENSE_SPLIT2,
  V_DENSE_N64,
  V_DENSE_GSPLIT,
  V_DENSE_GSPLIT2K,
  V_DENSE_M128,
  V_DENSE_M256,
  V_DENSE_PAIR192,
  V_CONTIG_M128,
  V_CONTIG_M256,
  V_CONTIG_M256_TMASTORE,
  V_MASKED_M128,
  V_MASKED_M256,
  V_MASKED_PAIR192,
  V_BF16,
  V_BF16_TMASTORE,
  V_UE8M0,
  V_COUNT
};
static_assert(V_COUNT == kNumVariants, "variant table and names");

std::atomic<int> g_override{-1};

// test hook (fp8g_testing_withhold_stage): -1 = off
std::atomic<int> g_test_withhold{-1};
std::atomic<uint32_t> g_test_wait_limit_us{kWaitLimitUs};

// Programmatic dependent launch is on unless FP8G_DISABLE_PDL is set to a
// nonzero value in the environment (read once).
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("FP8G_DISABLE_PDL");
    return !(e && *e && std::strcmp(e, "0") != 0);
  }();
  return on;
}
thread_local int t_last_variant = -1;

// ---------------------------------------------------------------- devices
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sms = 0;
  int max_smem_optin = 0;
  bool attr_set[kNumVariants] = {};
  int max_clusters[kNumVariants] = {};  // split and pair variants: co-resident clusters
  // global split-K workspace: sms slots of 64 x 128 floats, 2 counters per tile
  float* ws = nullptr;
  uint32_t* sync = nullptr;
  bool ws_failed = false;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8G_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return FP8G_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.probed = true;
  }
  *out = &d;
  return d.supported ? FP8G_OK : FP8G_ERR_UNSUPPORTED;
}

// Opt the variant into its shared-memory size on this device (once).
int prepare_variant(DeviceInfo* d, int v) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (d->attr_set[v]) return FP8G_OK;
  const Variant& V = kVariants[v];
  if (V.smem > d->max_smem_optin) return FP8G_ERR_UNSUPPORTED;
  if (V.reg_split) {
    // the setmaxnreg split is sized for exactly launch_regs per thread at
    // launch; any other count would leave the promotion warps waiting
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(V.fn)) != cudaSuccess) return FP8G_ERR_CUDA;
    if (fa.numRegs != V.launch_regs) return FP8G_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(reinterpret_cast<const void*>(V.fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           V.smem) != cudaSuccess)
    return FP8G_ERR_CUDA;
  if (V.split > 1 || V.pair) {
    const int cs = V.pair ? 2 : V.split;
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(V.fn), cudaFuncAttributeNonPortableClusterSizeAllowed,
                             cs > 8 ? 1 : 0) != cudaSuccess)
      return FP8G_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(cs * 64, 1, 1);
    cfg.blockDim = dim3(V.threads, 1, 1);
    cfg.dynamicSmemBytes = V.smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(V.fn), &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    d->max_clusters[v] = n;
  }
  d->attr_set[v] = true;
  return FP8G_OK;
}

// The global split-K workspace of this device (sms x 64 x 128 floats and two
// counters per tile, ~4.7 MB on B200): allocated on the first call that needs
// it, counters zeroed.  Allocation is not allowed while `stream` is being
// captured; the caller then uses a variant without a workspace.
int ensure_workspace(DeviceInfo* d, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (d->ws) return FP8G_OK;
  if (d->ws_failed) return FP8G_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    (void)cudaGetLastError();
    return FP8G_ERR_UNSUPPORTED;
  }
  const size_t ws_bytes = static_cast<size_t>(d->sms) * 64 * 128 * sizeof(float);
  const size_t sync_bytes = static_cast<size_t>(d->sms) * 2 * sizeof(uint32_t);
  void *ws = nullptr, *sync = nullptr;
  if (cudaMalloc(&ws, ws_bytes) != cudaSuccess || cudaMalloc(&sync, sync_bytes) != cudaSuccess ||
      cudaMemset(sync, 0, sync_bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    (void)cudaGetLastError();
    if (ws) (void)cudaFree(ws);
    if (sync) (void)cudaFree(sync);
    d->ws_failed = true;
    return FP8G_ERR_UNSUPPORTED;
  }
  d->ws = static_cast<float*>(ws);
  d->sync = static_cast<uint32_t*>(sync);
  return FP8G_OK;
}

// Split count of the global split-K variant for a decode shape: as many CTAs
// per tile as fit one per SM, each with at least 4 K-blocks.
int gsplit_for(const DeviceInfo* d, int tiles, int kb) {
  if (tiles <= 0 || tiles > d->sms) return 0;
  return std::max(1, std::min({d->sms / tiles, kb / 4, kMaxGSplit}));
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 3-D map (dim0 innermost).  strides are in bytes for dims 1 and 2.
int encode3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
             uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FP8G_ERR_CUDA;
  const cuuint64_t dims[3] = {d0, std::max<uint64_t>(d1, 1), std::max<uint64_t>(d2, 1)};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8G_OK : FP8G_ERR_CUDA;
}

// ---------------------------------------------------------------- validation
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_shapes(int rows, int N, int K, int ld_sa) {
  if (rows < 0 || N < 0 || K <= 0 || K % 128 != 0 || K > 128 * kKBMax) return FP8G_ERR_INVALID_ARG;
  if (ld_sa < rows || ld_sa < 1) return FP8G_ERR_INVALID_ARG;
  if (N % 8 != 0 || ld_sa % 4 != 0) return FP8G_ERR_MISALIGNED;
  return FP8G_OK;
}

int check_ptrs(const uint8_t* A, const float* sa, const uint8_t* B, const float* sb, const uint16_t* D) {
  if (!A || !sa || !B || !sb || !D) return FP8G_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(sa, 16) || !aligned(D, 16) || !aligned(sb, 4))
    return FP8G_ERR_MISALIGNED;
  return FP8G_OK;
}

struct Problem {
  int kind;
  const uint8_t* A;
  const float* sa;
  int ld_sa;
  const uint8_t* B;
  const float* sb;
  uint16_t* D;
  const int32_t* idx;  // m_indices or masked_m
  int M;               // rows (Mmax for masked)
  int N, K, G;
  int expected_m;
};

int launch(const Problem& P, int v, DeviceInfo* dev, cudaStream_t stream) {
  const Variant& V = kVariants[v];
  if (V.kind != P.kind) return FP8G_ERR_UNSUPPORTED;
  if (P.kind == kContiguous && V.swap && V.bnc != 128) return FP8G_ERR_UNSUPPORTED;
  int rc = prepare_variant(dev, v);
  if (rc) return rc;

  const int KB = P.K / 128, NB = (P.N + 127) / 128;
  // output tile: n-lanes BNC rows of A x 128 rows of B; m-lanes 128 x BNC;
  // pairs 256 x BNC (each CTA loads 128 rows of A and BNC / 2 rows of B)
  const int m_ext = V.pair ? 256 : V.swap ? V.bnc : 128;
  const int n_ext = V.pair ? V.bnc : V.swap ? 128 : V.bnc;
  const int G_a = P.kind == kMasked ? P.G : 1;
  const int G_b = P.kind == kDense ? 1 : P.G;

  Params p{};
  p.M = P.M;
  p.N = P.N;
  p.K = P.K;
  p.KB = KB;
  p.NB = NB;
  p.G = G_b;
  p.n_tiles = (P.N + n_ext - 1) / n_ext;
  // contiguous: 128-row expert blocks, two per pair tile
  p.m_tiles = P.kind != kContiguous ? (P.M + m_ext - 1) / m_ext : V.pair ? (P.M / 128 + 1) / 2 : P.M / 128;
  p.num_tiles = p.n_tiles * p.m_tiles * (P.kind == kMasked ? P.G : 1);
  p.m_indices = P.kind == kContiguous ? P.idx : nullptr;
  p.masked_m = P.kind == kMasked ? P.idx : nullptr;
  p.sa = P.sa;
  p.ld_sa = P.ld_sa;
  p.sb = P.sb;
  p.D = P.D;
  // the test hook applies to the single-CTA kernel only
  const int withhold = V.pair ? -1 : g_test_withhold.load(std::memory_order_relaxed);
  p.test_withhold_it = withhold;
  p.wait_limit_us = withhold >= 0 ? g_test_wait_limit_us.load(std::memory_order_relaxed) : kWaitLimitUs;
  if (p.num_tiles <= 0) return FP8G_OK;
  if (V.split < 0) {
    p.gsplit = gsplit_for(dev, p.num_tiles, KB);
    if (p.gsplit < 1 || p.num_tiles * p.gsplit > dev->sms) return FP8G_ERR_UNSUPPORTED;
    if ((rc = ensure_workspace(dev, stream))) return rc;
    p.ws = dev->ws;
    p.sync = dev->sync;
  }

  CUtensorMap tmA, tmB, tmSA;
  const uint32_t a_box_rows = V.swap ? V.bnc : 128;
  const uint32_t b_box_rows = V.pair ? V.bnc / 2 : V.swap ? 128 : V.bnc;
  rc = encode3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, P.A, P.K, P.M, G_a, (uint64_t)P.K,
                (uint64_t)P.K * std::max(P.M, 1), 128, a_box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, P.B, P.K, P.N, G_b, (uint64_t)P.K,
                  (uint64_t)P.K * P.N, 128, b_box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc && V.tma_store)
    // the third map is D: boxes of 32 rows x 32 columns (clipped at M and N)
    rc = encode3d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P.D, P.N, P.M, 1, (uint64_t)P.N * 2,
                  (uint64_t)P.N * 2 * P.M, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  else if (!rc)
    rc = encode3d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, P.sa, P.M, KB, G_a, (uint64_t)P.ld_sa * 4,
                  (uint64_t)P.ld_sa * 4 * KB, V.swap ? V.bnc : 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned nattr = 0;
  cfg.blockDim = dim3(V.threads, 1, 1);
  cfg.dynamicSmemBytes = V.smem;
  cfg.stream = stream;
  if (pdl_enabled()) {
    // the kernel may start its prologue while the previous kernel in the
    // stream finishes; it waits for that kernel before touching memory
    attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[nattr].val.programmaticStreamSerializationAllowed = 1;
    ++nattr;
  }
  if (V.split > 1) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = V.split;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = 1;
    ++nattr;
    cfg.gridDim = dim3(p.num_tiles * V.split, 1, 1);
  } else if (V.split < 0) {
    cfg.gridDim = dim3(p.gsplit, p.n_tiles, p.m_tiles);
  } else if (V.pair) {
    const int clusters = std::min(p.num_tiles, dev->max_clusters[v]);
    if (clusters < 1) return FP8G_ERR_UNSUPPORTED;
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = 2;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = 1;
    ++nattr;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
  } else {
    cfg.gridDim = dim3(std::min(p.num_tiles, dev->sms), 1, 1);
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  void* args[] = {&tmA, &tmB, &tmSA, &p};
  if (cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(V.fn), args) != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }
  if (V.split == kGlobalSplitPartials) {
    // the sum of the partials, one thread per output element
    cudaLaunchConfig_t rc_cfg = {};
    cudaLaunchAttribute rc_attr[1];
    const long outputs = static_cast<long>(p.num_tiles) * V.bnc * 128;
    rc_cfg.gridDim = dim3(static_cast<unsigned>(std::min<long>((outputs + 255) / 256, 4L * dev->sms)), 1, 1);
    rc_cfg.blockDim = dim3(256, 1, 1);
    rc_cfg.stream = stream;
    rc_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    rc_attr[0].val.programmaticStreamSerializationAllowed = 1;
    rc_cfg.attrs = rc_attr;
    rc_cfg.numAttrs = pdl_enabled() ? 1 : 0;
    void* rargs[] = {&p};
    if (cudaLaunchKernelExC(&rc_cfg, reinterpret_cast<const void*>(&splitk_reduce_kernel<64>), rargs) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return FP8G_ERR_CUDA;
    }
  }
  t_last_variant = v;
  return FP8G_OK;
}

int select_variant(const Problem& P, DeviceInfo* dev, cudaStream_t stream) {
  const int ov = g_override.load(std::memory_order_relaxed);
  if (ov >= 0) return ov;
  // m-lanes, 256 columns when there are enough such tiles to fill the GPU
  auto wide = [&](int v256, int v128, long tiles256) {
    return tiles256 >= dev->sms && prepare_variant(dev, v256) == FP8G_OK ? v256 : v128;
  };
  // CTA pairs, 256 x 192 tiles, when there are enough to give every
  // co-resident cluster one
  auto pair = [&](int v, long pair_tiles) {
    return prepare_variant(dev, v) == FP8G_OK && dev->max_clusters[v] > 0 && pair_tiles >= dev->max_clusters[v];
  };
  // contiguous: single-CTA 128 x 256 tiles with the TMA-store epilogue
  // (G=4, M=8192 per expert, N=4096, K=7168: 1212-1227 us against 1243-1245
  // us with direct stores; CTA pairs with 256 x 192 tiles 1317-1345 us, 256 x
  // 256 pair tiles 1401 us); direct stores if its shared memory cannot be had
  if (P.kind == kContiguous) {
    const long tiles256 = static_cast<long>(P.M / 128) * ((P.N + 255) / 256);
    if (tiles256 >= dev->sms && prepare_variant(dev, V_CONTIG_M256_TMASTORE) == FP8G_OK) return V_CONTIG_M256_TMASTORE;
    return wide(V_CONTIG_M256, V_CONTIG_M128, tiles256);
  }
  if (P.kind == kMasked) {
    // B streams once per 128 (or 256) rows of a group's A: m-lanes tiles read
    // it the fewest times; count the tiles the typical group fills
    // (G=16, N=4096, K=7168, masked_m <= 64: pair 140 us, m-lanes 128 148 us,
    // n-lanes 64 254 us)
    const long m_pairs = (std::max(P.expected_m, 1) + 255) / 256;
    if (pair(V_MASKED_PAIR192, static_cast<long>(P.G) * m_pairs * ((P.N + 191) / 192))) return V_MASKED_PAIR192;
    if (P.expected_m > 0 && P.expected_m <= 64) return V_MASKED_M128;
    const long m_blocks = (std::max(P.expected_m, 1) + 127) / 128;
    return wide(V_MASKED_M256, V_MASKED_M128, static_cast<long>(P.G) * m_blocks * ((P.N + 255) / 256));
  }
  if (P.M <= 64) {
    // decode shapes: few 128-row tiles of B, so K is split for many SMs to
    // stream B.  First choice: up to 16 CTAs per tile with partials in the
    // workspace and a reduce kernel.  Without the workspace (a capture before
    // the device's first call): a cluster split whose clusters are all
    // co-resident and that leaves each CTA at least 4 K-blocks.
    const int nt = (P.N + 127) / 128;
    const int kb = P.K / 128;
    if (gsplit_for(dev, nt, kb) >= 2 && prepare_variant(dev, V_DENSE_GSPLIT2K) == FP8G_OK &&
        ensure_workspace(dev, stream) == FP8G_OK)
      return V_DENSE_GSPLIT2K;
    for (int v : {V_DENSE_SPLIT, V_DENSE_SPLIT4, V_DENSE_SPLIT2}) {
      const int split = kVariants[v].split;
      if (kb < 4 * split || nt * split > dev->sms) continue;
      if (prepare_variant(dev, v) != FP8G_OK) continue;
      if (nt <= dev->max_clusters[v]) return v;
    }
    return V_DENSE_N64;
  }
  if (pair(V_DENSE_PAIR192, static_cast<long>((P.M + 255) / 256) * ((P.N + 191) / 192))) return V_DENSE_PAIR192;
  return wide(V_DENSE_M256, V_DENSE_M128, static_cast<long>((P.M + 127) / 128) * ((P.N + 255) / 256));
}

// BF16 NT GEMM on CTA pairs: 256 x 256 tiles, K-blocks of 64.
int launch_bf16(const uint16_t* A, const uint16_t* B, uint16_t* D, int M, int N, int K, int v, DeviceInfo* dev,
                cudaStream_t stream) {
  const Variant& V = kVariants[v];
  if (V.kind != kBf16Dense) return FP8G_ERR_UNSUPPORTED;
  int rc = prepare_variant(dev, v);
  if (rc) return rc;
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.KB = K / 64;
  p.NB = 1;
  p.G = 1;
  p.n_tiles = (N + 255) / 256;
  p.m_tiles = (M + 255) / 256;
  p.num_tiles = p.n_tiles * p.m_tiles;
  p.D = D;
  p.wait_limit_us = kWaitLimitUs;
  p.test_withhold_it = -1;
  CUtensorMap tmA, tmB, tmD;
  rc = encode3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, M, 1, (uint64_t)K * 2, (uint64_t)K * 2 * M, 64, 128,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, K, N, 1, (uint64_t)K * 2, (uint64_t)K * 2 * N, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D, N, M, 1, (uint64_t)N * 2, (uint64_t)N * 2 * M, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  const int clusters = std::min(p.num_tiles, dev->max_clusters[v]);
  if (clusters < 1) return FP8G_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned nattr = 0;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(V.threads, 1, 1);
  cfg.dynamicSmemBytes = V.smem;
  cfg.stream = stream;
  attr[nattr].id = cudaLaunchAttributeClusterDimension;
  attr[nattr].val.clusterDim.x = 2;
  attr[nattr].val.clusterDim.y = 1;
  attr[nattr].val.clusterDim.z = 1;
  ++nattr;
  if (pdl_enabled()) {
    attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[nattr].val.programmaticStreamSerializationAllowed = 1;
    ++nattr;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  void* args[] = {&tmA, &tmB, &tmD, &p};
  if (cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(V.fn), args) != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }
  t_last_variant = v;
  return FP8G_OK;
}

// FP8 GEMM with UE8M0 scales: one CTA per 128 x 256 tile, block-scaled MMA.
int launch_ue8m0(const uint8_t* A, const uint8_t* sfa, int ld_sf, const uint8_t* B, const uint8_t* sfb, uint16_t* D,
                 int M, int N, int K, int v, DeviceInfo* dev, cudaStream_t stream) {
  const Variant& V = kVariants[v];
  if (V.kind != kUe8m0Dense) return FP8G_ERR_UNSUPPORTED;
  int rc = prepare_variant(dev, v);
  if (rc) return rc;
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.KB = K / 128;
  p.NB = (N + 127) / 128;
  p.G = 1;
  p.n_tiles = (N + 255) / 256;
  p.m_tiles = (M + 127) / 128;
  p.num_tiles = p.n_tiles * p.m_tiles;
  p.D = D;
  p.ld_sa = ld_sf;
  p.sfa = sfa;
  p.sfb = sfb;
  p.wait_limit_us = kWaitLimitUs;
  p.test_withhold_it = -1;
  CUtensorMap tmA, tmB, tmD;
  rc = encode3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, 1, (uint64_t)K, (uint64_t)K * M, 128, 128,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, 1, (uint64_t)K, (uint64_t)K * N, 128, 256,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, D, N, M, 1, (uint64_t)N * 2, (uint64_t)N * 2 * M, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(std::min(p.num_tiles, dev->sms), 1, 1);
  cfg.blockDim = dim3(V.threads, 1, 1);
  cfg.dynamicSmemBytes = V.smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  void* args[] = {&tmA, &tmB, &tmD, &p};
  if (cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(V.fn), args) != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }
  t_last_variant = v;
  return FP8G_OK;
}

int run(const Problem& P, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int v = select_variant(P, dev, stream);
  if (v < 0 || v >= kNumVariants) return FP8G_ERR_UNSUPPORTED;
  return launch(P, v, dev, stream);
}

}  // namespace

namespace fp8g {
// Device address of this library's error word on the current device (looked
// up once per device), for kernels of other translation units.
uint32_t* device_error_word() {
  static std::mutex mu;
  static uint32_t* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fp8g_error_word) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}
}  // namespace fp8g

extern "C" {

int fp8_gemm_nt(const uint8_t* A, const float* sa, int ld_sa, const uint8_t* B, const float* sb, uint16_t* D,
                int M, int N, int K, cudaStream_t stream) {
  int rc = check_shapes(M, N, K, ld_sa);
  if (rc) return rc;
  if (M == 0 || N == 0) return FP8G_OK;
  if ((rc = check_ptrs(A, sa, B, sb, D))) return rc;
  return run(Problem{kDense, A, sa, ld_sa, B, sb, D, nullptr, M, N, K, 1, 0}, stream);
}

int m_grouped_fp8_gemm_nt_contiguous(const uint8_t* A, const float* sa, int ld_sa, const uint8_t* B,
                                     const float* sb, uint16_t* D, const int32_t* m_indices, int M, int N,
                                     int K, int G, cudaStream_t stream) {
  int rc = check_shapes(M, N, K, ld_sa);
  if (rc) return rc;
  if (G < 0 || M % 128 != 0) return FP8G_ERR_INVALID_ARG;
  if (M == 0 || N == 0 || G == 0) return FP8G_OK;
  if ((rc = check_ptrs(A, sa, B, sb, D))) return rc;
  if (!m_indices) return FP8G_ERR_INVALID_ARG;
  if (!aligned(m_indices, 4)) return FP8G_ERR_MISALIGNED;
  return run(Problem{kContiguous, A, sa, ld_sa, B, sb, D, m_indices, M, N, K, G, 0}, stream);
}

int m_grouped_fp8_gemm_nt_masked(const uint8_t* A, const float* sa, int ld_sa, const uint8_t* B, const float* sb,
                                 uint16_t* D, const int32_t* masked_m, int G, int Mmax, int N, int K,
                                 int expected_m, cudaStream_t stream) {
  int rc = check_shapes(Mmax, N, K, ld_sa);
  if (rc) return rc;
  if (G < 0 || expected_m < 0) return FP8G_ERR_INVALID_ARG;
  if (Mmax == 0 || N == 0 || G == 0) return FP8G_OK;
  if ((rc = check_ptrs(A, sa, B, sb, D))) return rc;
  if (!masked_m) return FP8G_ERR_INVALID_ARG;
  if (!aligned(masked_m, 4)) return FP8G_ERR_MISALIGNED;
  return run(Problem{kMasked, A, sa, ld_sa, B, sb, D, masked_m, Mmax, N, K, G, expected_m}, stream);
}

int fp8g_sa_to_mn_major(const float* src, float* dst, int G, int rows, int KB, int ld_sa) {
  if (!src || !dst || G < 1 || rows < 0 || KB < 1 || ld_sa < rows || ld_sa < 1) return FP8G_ERR_INVALID_ARG;
  if (ld_sa % 4 != 0) return FP8G_ERR_MISALIGNED;
  for (long g = 0; g < G; ++g) {
    const float* s = src + g * rows * static_cast<long>(KB);
    float* d = dst + g * KB * static_cast<long>(ld_sa);
    for (long kb = 0; kb < KB; ++kb) {
      float* drow = d + kb * ld_sa;
      for (long m = 0; m < rows; ++m) drow[m] = s[m * KB + kb];
      for (long m = rows; m < ld_sa; ++m) drow[m] = 0.f;
    }
  }
  return FP8G_OK;
}

int bf16_gemm_nt(const uint16_t* A, const uint16_t* B, uint16_t* D, int M, int N, int K, cudaStream_t stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || K > 65536) return FP8G_ERR_INVALID_ARG;
  if (N % 8 != 0) return FP8G_ERR_MISALIGNED;
  if (M == 0 || N == 0) return FP8G_OK;
  if (!A || !B || !D) return FP8G_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16)) return FP8G_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  int rc = device_info(&dev);
  if (rc) return rc;
  const int ov = g_override.load(std::memory_order_relaxed);
  // the TMA-store epilogue measured 1-3 % faster than direct stores (8192^3:
  // 861 vs 871 us; 4096 x 7168 x 16384: 766 vs 791 us)
  const int v = ov >= 0 ? ov : V_BF16_TMASTORE;
  return launch_bf16(A, B, D, M, N, K, v, dev, stream);
}

int fp8_gemm_nt_ue8m0(const uint8_t* A, const uint8_t* sfa, int ld_sf, const uint8_t* B, const uint8_t* sfb,
                      uint16_t* D, int M, int N, int K, cudaStream_t stream) {
  int rc = check_shapes(M, N, K, ld_sf);
  if (rc) return rc;
  if (M == 0 || N == 0) return FP8G_OK;
  if (!A || !sfa || !B || !sfb || !D) return FP8G_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16)) return FP8G_ERR_MISALIGNED;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev))) return rc;
  const int ov = g_override.load(std::memory_order_relaxed);
  return launch_ue8m0(A, sfa, ld_sf, B, sfb, D, M, N, K, ov >= 0 ? ov : V_UE8M0, dev, stream);
}

const char* fp8g_status_string(int status) {
  switch (status) {
    case FP8G_OK: return "ok";
    case FP8G_ERR_INVALID_ARG: return "invalid argument";
    case FP8G_ERR_MISALIGNED: return "misaligned pointer or pitch";
    case FP8G_ERR_UNSUPPORTED: return "unsupported device or no kernel variant for this call";
    case FP8G_ERR_CUDA: return "CUDA call failed";
    case FP8G_ERR_DEVICE: return "device-side error recorded";
    default: return "unknown status";
  }
}

int fp8g_get_device_error(int device, uint32_t* bits, int clear) {
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return FP8G_ERR_CUDA;
  if (device != prev && cudaSetDevice(device) != cudaSuccess) return FP8G_ERR_CUDA;
  uint32_t w = 0;
  int rc = FP8G_OK;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(&w, g_fp8g_error_word, sizeof(w), 0, cudaMemcpyDeviceToHost) != cudaSuccess) {
    rc = FP8G_ERR_CUDA;
  } else {
    if (clear) {
      const uint32_t z = 0;
      if (cudaMemcpyToSymbol(g_fp8g_error_word, &z, sizeof(z), 0, cudaMemcpyHostToDevice) != cudaSuccess)
        rc = FP8G_ERR_CUDA;
      // a call that gave up can leave split-K counters behind: zero them
      DeviceInfo* d = (device >= 0 && device < kMaxDevices) ? &g_dev[device] : nullptr;
      if (w && d && d->sync && cudaMemset(d->sync, 0, static_cast<size_t>(d->sms) * 2 * sizeof(uint32_t)) != cudaSuccess)
        rc = FP8G_ERR_CUDA;
    }
    if (!rc && w) rc = FP8G_ERR_DEVICE;
  }
  if (bits) *bits = w;
  if (device != prev) (void)cudaSetDevice(prev);
  return rc;
}

int fp8g_set_variant_override(int variant) {
  if (variant < -1 || variant >= kNumVariants) return FP8G_ERR_INVALID_ARG;
  g_override.store(variant, std::memory_order_relaxed);
  return FP8G_OK;
}

int fp8g_num_variants(void) { return kNumVariants; }

const char* fp8g_variant_name(int variant) {
  return variant >= 0 && variant < kNumVariants ? kVariants[variant].name : nullptr;
}

int fp8g_last_variant(void) { return t_last_variant; }

int fp8g_version(void) { return 200; }

int fp8g_testing_withhold_stage(int iteration, unsigned wait_limit_us) {
  if (iteration < 0) {
    g_test_withhold.store(-1, std::memory_order_relaxed);
    g_test_wait_limit_us.store(kWaitLimitUs, std::memory_order_relaxed);
    return FP8G_OK;
  }
  if (wait_limit_us < 100 || wait_limit_us > kWaitLimitUs) return FP8G_ERR_INVALID_ARG;
  g_test_wait_limit_us.store(wait_limit_us, std::memory_order_relaxed);
  g_test_withhold.store(iteration, std::memory_order_relaxed);
  return FP8G_OK;
}

}  // extern "C"

// ===========================================================================
// fp8_gemm_nt_no_alloc: the dense GEMM for callers that must not allocate
// device memory.
//
// Some callers cannot call cudaMalloc at the point where they run a GEMM: an
// engine that hands out all device memory from its own fixed pool, or a
// runtime that forbids allocations after start-up so that its memory
// footprint is known in advance.  The
// regular fp8_gemm_nt allocates its split-K workspace (about 4.7 MB) on the
// first decode-shaped call of a device.  This entry point runs the same
// split-K kernel with its scratch in a statically sized array that the
// library carries in its own device image instead.
// ===========================================================================
namespace {

// Scratch of the static variant: 160 tile slots of 64 x 128 FP32 partial sums,
// then 2 counters per tile.  Every GPU that loads the library holds it until
// the process exits.
constexpr int kNoAllocSlots = 160;
constexpr size_t kNoAllocPartialBytes = static_cast<size_t>(kNoAllocSlots) * 64 * 128 * sizeof(float);
constexpr size_t kNoAllocCounterBytes = static_cast<size_t>(kNoAllocSlots) * 2 * sizeof(uint32_t);

static __device__ __align__(256) unsigned char g_no_alloc_scratch[kNoAllocPartialBytes + kNoAllocCounterBytes];

std::mutex g_no_alloc_mu;
void* g_no_alloc_ptr[kMaxDevices] = {};  // device address of g_no_alloc_scratch, per device

// Device address of the static scratch on the current device.  The symbol's
// name in host code only stands for the array; the device address comes from
// cudaGetSymbolAddress, once per device, with that device current.
int no_alloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_no_alloc_mu);
  if (!g_no_alloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_no_alloc_scratch) != cudaSuccess || !ptr) {
      (void)cudaGetLastError();
      return FP8G_ERR_CUDA;
    }
    g_no_alloc_ptr[dev] = ptr;
  }
  *out = g_no_alloc_ptr[dev];
  return FP8G_OK;
}

}  // namespace

extern "C" int fp8_gemm_nt_no_alloc(const uint8_t* A, const float* sa, int ld_sa, const uint8_t* B,
                                    const float* sb, uint16_t* D, int M, int N, int K, cudaStream_t stream) {
  int rc = check_shapes(M, N, K, ld_sa);
  if (rc) return rc;
  if (M == 0 || N == 0) return FP8G_OK;
  if ((rc = check_ptrs(A, sa, B, sb, D))) return rc;
  DeviceInfo* dev = nullptr;
  if ((rc = device_info(&dev))) return rc;
  int dev_id = 0;
  if (cudaGetDevice(&dev_id) != cudaSuccess) return FP8G_ERR_CUDA;

  // tiles of 128 rows of B x 64 rows of A; K split over `gsplit` CTAs per tile
  const Variant& V = kVariants[V_DENSE_GSPLIT];
  const int KB = K / 128, NB = (N + 127) / 128;
  const int n_tiles = NB, m_tiles = (M + 63) / 64;
  const long tiles = static_cast<long>(n_tiles) * m_tiles;
  if (tiles > kNoAllocSlots || tiles > dev->sms) return FP8G_ERR_UNSUPPORTED;  // scratch or GPU too small
  const int gsplit = std::min(gsplit_for(dev, static_cast<int>(tiles), KB), kNoAllocSlots / static_cast<int>(tiles));
  if (gsplit < 1) return FP8G_ERR_UNSUPPORTED;
  if ((rc = prepare_variant(dev, V_DENSE_GSPLIT))) return rc;
  void* scratch = nullptr;
  if ((rc = no_alloc_scratch(dev_id, &scratch))) return rc;

  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.KB = KB;
  p.NB = NB;
  p.G = 1;
  p.n_tiles = n_tiles;
  p.m_tiles = m_tiles;
  p.num_tiles = static_cast<int>(tiles);
  p.sa = sa;
  p.ld_sa = ld_sa;
  p.sb = sb;
  p.D = D;
  p.gsplit = gsplit;
  p.wait_limit_us = kWaitLimitUs;
  p.test_withhold_it = -1;
  p.ws = static_cast<float*>(scratch);
  p.sync = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(scratch) + kNoAllocPartialBytes);
  // the counters of this call start at zero even if an earlier call gave up
  // half-way; the partial sums are always written before they are read
  if (cudaMemsetAsync(p.sync, 0, static_cast<size_t>(2) * p.num_tiles * sizeof(uint32_t), stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }

  CUtensorMap tmA, tmB, tmSA;
  rc = encode3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, 1, (uint64_t)K, (uint64_t)K * M, 128, V.bnc,
                CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, 1, (uint64_t)K, (uint64_t)K * N, 128, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (!rc)
    rc = encode3d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sa, M, KB, 1, (uint64_t)ld_sa * 4, (uint64_t)ld_sa * 4 * KB,
                  V.bnc, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(p.gsplit, p.n_tiles, p.m_tiles);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = V.smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  void* args[] = {&tmA, &tmB, &tmSA, &p};
  if (cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(V.fn), args) != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }
  t_last_variant = V_DENSE_GSPLIT;
  return FP8G_OK;
}
