// quant.cu -- FP8 (e4m3) quantisers for the GEMM's inputs, sm_100a.
//
// The pages leave quantisation to the caller (kakushin.no, "Hvorfor FP8 og
// FP4 er interessant": inputs are converted to FP8 by the user); the
// granularity is the GEMM's fine-grained scaling (GeekNews, "DeepSeek,
// DeepGEMM 오픈소스 공개", topic body, first bullet): one FP32 scale per 1x128
// row group of the activations A and per 128x128 block of the weights B.
//
//   scale = amax / 448 (FP32; 1 for an all-zero group),
//   code  = e4m3_rne_satfinite(x / scale)   (one IEEE FP32 division)
//
// Both kernels are HBM-bound streams: each input element is read once (2 or
// 4 bytes) and each code written once (1 byte).  The arithmetic (the
// correctly rounded quotient without a division) is in quant_impl.cuh.
//   quantize_1x128_kernel   a warp per row (quantize_row_1x128), 8 rows per
//                           CTA, scales staged in shared memory.
//   quantize_128x128_kernel one CTA per 128x128 block: a thread holds 8 rows x
//                           8 columns in registers, the amax is a CTA max, and
//                           the codes are stored from the same registers (the
//                           block is read from HBM once).
// The 1x128 quantiser (activations, run right before a GEMM) is a programmatic
// dependent launch: it waits for the previous kernel before it reads x and
// lets the next kernel (the GEMM) start its prologue, and the early B stream
// of a GEMM whose B is declared static, at once.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "fp8gemm.h"
#include "quant_impl.cuh"

namespace {

using namespace fp8g::quant;

// A CTA of 8 warps quantises 8 consecutive rows (warp w: row r0 + w), so the
// input is read in long contiguous runs.  The scales go through shared
// memory, so that the 8 rows' scales of a K-block leave as one 32-byte store
// into sa's MN-major layout.  CTAs stride over row blocks.
constexpr int kRowsPerCta = 8;
constexpr int kMaxKB = 512;  // K <= 65536

template <bool kF32>
__global__ void __launch_bounds__(256, 3) quantize_1x128_kernel(const void* __restrict__ x, int rows, int K,
                                                             uint8_t* __restrict__ q, float* __restrict__ sa,
                                                             int ld_sa) {
  __shared__ float s_scale[kMaxKB][kRowsPerCta];
  // x may be written by the previous kernel in the stream (a no-op without a
  // programmatic dependency); the next kernel may start its prologue now
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int w = threadIdx.x >> 5;
  const int KB = K / 128;
  const size_t esz = kF32 ? 4 : 2;
  for (long r0 = static_cast<long>(blockIdx.x) * kRowsPerCta; r0 < rows; r0 += static_cast<long>(gridDim.x) * kRowsPerCta) {
    const long row = r0 + w;
    if (row < rows)  // warp-uniform
      quantize_row_1x128<kF32>(static_cast<const uint8_t*>(x) + row * K * esz, K,
                               [&](long off, const auto& c) { store_code_words(q + row * K + off, c); },
                               [&](int kb, float s) { s_scale[kb][w] = s; });
    __syncthreads();
    // sa[kb][r0 .. r0 + 7]: consecutive threads write consecutive rows
    const int nrows = static_cast<int>(rows - r0 < kRowsPerCta ? rows - r0 : kRowsPerCta);
    for (int i = threadIdx.x; i < KB * kRowsPerCta; i += blockDim.x) {
      const int kb = i / kRowsPerCta, rr = i % kRowsPerCta;
      if (rr < nrows) sa[static_cast<long>(kb) * ld_sa + r0 + rr] = s_scale[kb][rr];
    }
    __syncthreads();
  }
}

// Block (nb, kb) = rows 128nb.. (fewer in the last block row), columns
// 128kb..+127.  Thread t covers rows r = t/16 + 16i (i = 0..7) and columns
// 8*(t%16)..+7 of the block; it keeps its 64 input values in registers in
// their input format (32 registers for bf16) across the CTA's amax.
template <bool kF32>
__global__ void __launch_bounds__(256) quantize_128x128_kernel(const void* __restrict__ x, int N, int K,
                                                               uint8_t* __restrict__ q, float* __restrict__ sb) {
  constexpr int kVec = kF32 ? 2 : 1;  // 16-byte loads per row chunk of 8 values
  __shared__ float warp_max[8];
  const int KB = K / 128;
  const int nb = blockIdx.x / KB, kb = blockIdx.x % KB;
  const int t = threadIdx.x;
  const int c0 = 128 * kb + 8 * (t & 15);
  const int r0 = 128 * nb + (t >> 4);
  uint4 raw[8][kVec];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + 16 * i;
    const long e = static_cast<long>(r) * K + c0;
#pragma unroll
    for (int h = 0; h < kVec; ++h)
      raw[i][h] = r < N ? __ldcs(kF32 ? reinterpret_cast<const uint4*>(static_cast<const float*>(x) + e) + h
                                      : reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + e))
                        : make_uint4(0u, 0u, 0u, 0u);
  }
  auto values = [&](int i, float (&v)[8]) {
    if constexpr (kF32) {
      v[0] = __uint_as_float(raw[i][0].x), v[1] = __uint_as_float(raw[i][0].y);
      v[2] = __uint_as_float(raw[i][0].z), v[3] = __uint_as_float(raw[i][0].w);
      v[4] = __uint_as_float(raw[i][kVec - 1].x), v[5] = __uint_as_float(raw[i][kVec - 1].y);
      v[6] = __uint_as_float(raw[i][kVec - 1].z), v[7] = __uint_as_float(raw[i][kVec - 1].w);
    } else {
      const uint32_t wd[4] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) v[2 * j] = __uint_as_float(wd[j] << 16), v[2 * j + 1] = __uint_as_float(wd[j] & 0xFFFF0000u);
    }
  };
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float v[8];
    values(i, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((t & 31) == 0) warp_max[t >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
  const float s = scale_of(amax);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + 16 * i;
    float v[8];
    values(i, v);
    uint32_t c[2];
    encode_group(v, s, c);
    if (r < N) __stcs(reinterpret_cast<uint2*>(q + static_cast<long>(r) * K + c0), make_uint2(c[0], c[1]));
  }
  if (t == 0) sb[static_cast<long>(nb) * KB + kb] = s;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// FP8G_DISABLE_PDL set (and not "0") turns programmatic dependent launch off,
// as for the GEMMs
bool pdl_on() {
  static const bool on = [] {
    const char* e = std::getenv("FP8G_DISABLE_PDL");
    return !(e && *e && std::strcmp(e, "0") != 0);
  }();
  return on;
}

template <bool kF32>
cudaError_t launch_1x128(unsigned blocks, cudaStream_t stream, const void* x, int rows, int K, uint8_t* q, float* sa,
                         int ld_sa) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  if (pdl_on()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, quantize_1x128_kernel<kF32>, x, rows, K, q, sa, ld_sa);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return -1;
  return n;
}

}  // namespace

extern "C" int fp8g_quantize_1x128(const void* x, int x_dtype, int rows, int K, uint8_t* q, float* sa, int ld_sa,
                                   cudaStream_t stream) {
  if (x_dtype != FP8G_IN_BF16 && x_dtype != FP8G_IN_F32) return FP8G_ERR_INVALID_ARG;
  if (rows < 0 || K <= 0 || K % 128 != 0 || ld_sa < rows || ld_sa < 1) return FP8G_ERR_INVALID_ARG;
  if (ld_sa % 4 != 0) return FP8G_ERR_MISALIGNED;
  if (rows == 0) return FP8G_OK;
  if (!x || !q || !sa) return FP8G_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sa, 16)) return FP8G_ERR_MISALIGNED;
  const int sms = sm_count();
  if (sms <= 0) return FP8G_ERR_CUDA;
  if (K / 128 > kMaxKB) return FP8G_ERR_INVALID_ARG;
  const long row_blocks = (static_cast<long>(rows) + kRowsPerCta - 1) / kRowsPerCta;
  const long blocks = std::min<long>(row_blocks, 16L * sms);
  const cudaError_t e = x_dtype == FP8G_IN_F32
                            ? launch_1x128<true>(static_cast<unsigned>(blocks), stream, x, rows, K, q, sa, ld_sa)
                            : launch_1x128<false>(static_cast<unsigned>(blocks), stream, x, rows, K, q, sa, ld_sa);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return FP8G_ERR_CUDA;
  }
  return FP8G_OK;
}

extern "C" int fp8g_quantize_128x128(const void* x, int x_dtype, int N, int K, uint8_t* q, float* sb,
                                     cudaStream_t stream) {
  if (x_dtype != FP8G_IN_BF16 && x_dtype != FP8G_IN_F32) return FP8G_ERR_INVALID_ARG;
  if (N < 0 || K <= 0 || K % 128 != 0) return FP8G_ERR_INVALID_ARG;
  if (N == 0) return FP8G_OK;
  if (!x || !q || !sb) return FP8G_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sb, 4)) return FP8G_ERR_MISALIGNED;
  const long blocks = static_cast<long>((N + 127) / 128) * (K / 128);
  if (blocks > 0x7FFFFFFFL) return FP8G_ERR_INVALID_ARG;
  if (x_dtype == FP8G_IN_F32)
    quantize_128x128_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, N, K, q, sb);
  else
    quantize_128x128_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, N, K, q, sb);
  if (cudaGetLastError() != cudaSuccess) return FP8G_ERR_CUDA;
  return FP8G_OK;
}
