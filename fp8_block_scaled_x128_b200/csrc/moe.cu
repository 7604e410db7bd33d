// moe.cu -- the expert pipeline on either side of the contiguous grouped
// GEMM, sm_100a.
//
// The contiguous layout (GeekNews, "MoE 모델을 위한 그룹화 GEMM 성능": rows of
// A grouped along M by expert, N and K shared, one expert per 128-row block)
// has to be built from the router's output before the GEMM, and the GEMM's
// rows have to go back to their tokens after it.  The pages describe only
// the layout; these kernels build it the plainest way:
//
//   dispatch  routed row r = t * topk + k (token t, slot k) goes to expert
//             e[r] (-1: dropped).  Expert g's rows keep their order r and
//             fill a segment padded to a multiple of 128 rows; segments
//             follow each other in expert order.  m_indices gets each block's
//             expert (-1 past the last segment).  Row pos[r] of A receives
//             token t quantised per 1x128 group (the GEMM's A scaling);
//             padding rows get zero codes and zero scales.
//   combine   out[t] = bf16(sum_k w[r] * D[pos[r]]), FP32, one fused
//             multiply-add per slot in slot order.
//
// Dispatch kernels, all on the caller's stream, no host synchronisation
// (the counts never reach the host, so a fixed capacity of blocks keeps the
// whole pipeline capturable in a CUDA graph):
//   1 moe_count_kernel   per chunk of 1024 routed rows, a histogram of
//                        experts (shared-memory atomics).
//   2 moe_scan_kernel    one CTA: per expert the exclusive prefix of the
//                        chunk histograms (the chunk's first slot in the
//                        expert's segment), the counts, the padded segment
//                        offsets, m_indices.
//   3 moe_rank_kernel    per chunk: each row's rank among the earlier rows
//                        of its expert in the chunk (__match_any_sync within
//                        a warp, per-warp counts across warps), hence pos[r].
//   4 moe_gather_kernel  one warp per token: the token's row read and
//                        quantised once, codes and scales stored into every
//                        row it was routed to (HBM-bound).
//   5 moe_pad_kernel     zero codes and scales of the padding rows.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "fp8gemm.h"
#include "quant_impl.cuh"

namespace fp8g {
uint32_t* device_error_word();  // api.cu: this device's FP8G_DEVERR_* word
}

namespace {

using namespace fp8g::quant;

constexpr int kChunk = 1024;       // routed rows per CTA in the count and rank kernels
constexpr int kMaxExperts = 256;   // per-warp expert counts live in shared memory
constexpr uint32_t kBadExpert = 0x8u;  // FP8G_DEVERR_BAD_EXPERT

// Expert of routed row r, or -1 (dropped, out of range, or past the end).
__device__ __forceinline__ int expert_of(const int32_t* e, int R, int G, long r, uint32_t* err) {
  if (r >= R) return -1;
  const int g = __ldg(e + r);
  if (g >= G || g < -1) {
    atomicOr(err, kBadExpert);
    return -1;
  }
  return g;
}

__global__ void __launch_bounds__(kChunk) moe_count_kernel(const int32_t* __restrict__ e, int R, int G,
                                                           int32_t* __restrict__ hist, uint32_t* err) {
  __shared__ int32_t h[kMaxExperts];
  for (int g = threadIdx.x; g < G; g += blockDim.x) h[g] = 0;
  __syncthreads();
  const int g = expert_of(e, R, G, static_cast<long>(blockIdx.x) * kChunk + threadIdx.x, err);
  if (g >= 0) atomicAdd(&h[g], 1);
  __syncthreads();
  for (int j = threadIdx.x; j < G; j += blockDim.x) hist[static_cast<long>(blockIdx.x) * G + j] = h[j];
}

// One CTA of kMaxExperts threads, thread g = expert g.  hist [C][G] becomes
// the exclusive prefix over chunks; off [G] = first row of g's segment;
// cnt [G] = g's rows; m_indices [blocks].
__global__ void __launch_bounds__(kMaxExperts) moe_scan_kernel(int32_t* __restrict__ hist, int C, int G,
                                                                int32_t* __restrict__ off, int32_t* __restrict__ cnt,
                                                                int32_t* __restrict__ m_indices, int blocks) {
  __shared__ int32_t s_blk[kMaxExperts];
  const int g = threadIdx.x;
  int32_t run = 0;
  if (g < G) {
    for (int c = 0; c < C; ++c) {
      const int32_t v = hist[static_cast<long>(c) * G + g];
      hist[static_cast<long>(c) * G + g] = run;
      run += v;
    }
  }
  const int32_t nblk = g < G ? (run + 127) / 128 : 0;
  // inclusive scan of the padded block counts over experts
  s_blk[g] = nblk;
  __syncthreads();
  for (int d = 1; d < kMaxExperts; d <<= 1) {
    const int32_t v = g >= d ? s_blk[g - d] : 0;
    __syncthreads();
    s_blk[g] += v;
    __syncthreads();
  }
  const int32_t first = s_blk[g] - nblk;  // exclusive
  const int32_t used = s_blk[kMaxExperts - 1];
  if (g < G) {
    off[g] = first * 128;
    cnt[g] = run;
    for (int b = first; b < first + nblk; ++b) m_indices[b] = g;
  }
  for (int b = used + g; b < blocks; b += blockDim.x) m_indices[b] = -1;
}

__global__ void __launch_bounds__(kChunk) moe_rank_kernel(const int32_t* __restrict__ e, int R, int G,
                                                          const int32_t* __restrict__ base,
                                                          const int32_t* __restrict__ off,
                                                          int32_t* __restrict__ pos, uint32_t* err) {
  __shared__ int32_t s_w[kChunk / 32][kMaxExperts];  // per warp and expert: rows, then the prefix over warps
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kChunk / 32) * G; i += blockDim.x) s_w[i / G][i % G] = 0;
  __syncthreads();
  const long r = static_cast<long>(blockIdx.x) * kChunk + threadIdx.x;
  const int g = expert_of(e, R, G, r, err);
  const uint32_t peers = __match_any_sync(0xffffffffu, g);
  const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
  if (g >= 0 && rank_in_warp == 0) s_w[w][g] = __popc(peers);
  __syncthreads();
  for (int j = threadIdx.x; j < G; j += blockDim.x) {
    int32_t run = 0;
    for (int ww = 0; ww < kChunk / 32; ++ww) {
      const int32_t v = s_w[ww][j];
      s_w[ww][j] = run;
      run += v;
    }
  }
  __syncthreads();
  if (r < R) pos[r] = g < 0 ? -1 : off[g] + base[static_cast<long>(blockIdx.x) * G + g] + s_w[w][g] + rank_in_warp;
}

// One warp per token: token t is read and quantised once, and its codes and
// scales are stored into every row pos[t*topk + k] it was routed to (k <
// topk <= kMaxTopk; dropped slots are skipped).
constexpr int kMaxTopk = 16;

// kCap: a compile-time bound on topk (4, 8 or 16, the smallest that holds
// it), so each store of a lane's codes tests only that many destinations
template <bool kF32, int kCap>
__global__ void __launch_bounds__(256, 3) moe_gather_kernel(const void* __restrict__ x, int K, int T, int topk,
                                                            const int32_t* __restrict__ pos, uint8_t* __restrict__ A,
                                                            float* __restrict__ sa, int ld_sa) {
  const int lane = threadIdx.x & 31;
  const size_t esz = kF32 ? 4 : 2;
  const long warp = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long t = warp; t < T; t += nwarps) {
    const int mine = lane < topk ? __ldg(pos + t * topk + lane) : -1;
    int dst[kCap];
    bool any = false;
#pragma unroll
    for (int k = 0; k < kCap; ++k) {
      dst[k] = __shfl_sync(0xffffffffu, mine, k);
      any = any || (k < topk && dst[k] >= 0);
    }
    if (!any) continue;  // warp-uniform
    quantize_row_1x128<kF32>(
        static_cast<const uint8_t*>(x) + t * K * esz, K,
        [&](long off, const auto& c) {
#pragma unroll
          for (int k = 0; k < kCap; ++k)
            if (k < topk && dst[k] >= 0) store_code_words(A + static_cast<long>(dst[k]) * K + off, c);
        },
        [&](int kb, float s) {
#pragma unroll
          for (int k = 0; k < kCap; ++k)
            if (k < topk && dst[k] >= 0) sa[static_cast<long>(kb) * ld_sa + dst[k]] = s;
        });
  }
}

// Padding rows of each segment: expert g owns rows off[g] + cnt[g] .. up to
// the next multiple of 128.  Work item (g, i), i < 128: one warp zeroes row
// off[g] + cnt[g] + i if it is padding.
__global__ void __launch_bounds__(256) moe_pad_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ cnt,
                                                      int G, int K, uint8_t* __restrict__ A, float* __restrict__ sa,
                                                      int ld_sa) {
  const int lane = threadIdx.x & 31;
  const long warp = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long item = warp; item < static_cast<long>(G) * 128; item += nwarps) {
    const int g = static_cast<int>(item / 128), i = static_cast<int>(item % 128);
    const int c = cnt[g];
    const int padded = (c + 127) / 128 * 128;
    if (c + i >= padded) continue;  // warp-uniform
    const long row = static_cast<long>(off[g]) + c + i;
    uint4* dst = reinterpret_cast<uint4*>(A + row * K);
    for (int j = lane; j < K / 16; j += 32) dst[j] = make_uint4(0u, 0u, 0u, 0u);
    for (int kb = lane; kb < K / 128; kb += 32) sa[static_cast<long>(kb) * ld_sa + row] = 0.f;
  }
}

// out[t, 8j .. 8j+7] from the topk rows pos[t*topk + k] of D: a CTA per
// token (grid-stride), its threads over the 16-byte column groups j.  The
// token's slots (positions and weights, kCap >= topk of them) are read once;
// all of a thread's row loads are issued before the first FMA, and the FMAs
// run in slot order, one rounding each, as the definition states.
template <int kCap>
__global__ void __launch_bounds__(256) moe_combine_kernel(const uint16_t* __restrict__ D, int N,
                                                          const int32_t* __restrict__ pos, const float* __restrict__ w,
                                                          int T, int topk, uint16_t* __restrict__ out) {
  const int per_row = N / 8;
  for (long t = blockIdx.x; t < T; t += gridDim.x) {
    int p[kCap];
    float wk[kCap];
#pragma unroll
    for (int k = 0; k < kCap; ++k) {
      p[k] = k < topk ? __ldg(pos + t * topk + k) : -1;
      wk[k] = k < topk && w ? __ldg(w + t * topk + k) : 1.f;
    }
    for (int j = threadIdx.x; j < per_row; j += blockDim.x) {
      uint4 v[kCap];
#pragma unroll
      for (int k = 0; k < kCap; ++k)
        v[k] = p[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(D + static_cast<long>(p[k]) * N) + j)
                         : make_uint4(0u, 0u, 0u, 0u);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < kCap; ++k) {
        if (p[k] < 0) continue;
        const uint32_t wd[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(wk[k], __uint_as_float(wd[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(wk[k], __uint_as_float(wd[i] & 0xFFFF0000u), acc[2 * i + 1]);
        }
      }
      uint4 o;
      uint32_t* ow = &o.x;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t packed;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(packed) : "f"(acc[2 * i + 1]), "f"(acc[2 * i]));
        ow[i] = packed;
      }
      reinterpret_cast<uint4*>(out + t * N)[j] = o;
    }
  }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

long chunks_of(long R) { return (R + kChunk - 1) / kChunk; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return -1;
  return n;
}

}  // namespace

extern "C" size_t fp8g_moe_dispatch_workspace_bytes(int R, int G) {
  if (R < 0 || G < 1 || G > kMaxExperts) return 0;
  return static_cast<size_t>(chunks_of(R) * G + 2L * G) * sizeof(int32_t);
}

extern "C" int fp8g_moe_dispatch(const void* x, int x_dtype, int T, int K, const int32_t* expert, int topk, int G,
                                 int blocks, uint8_t* A, float* sa, int ld_sa, int32_t* pos, int32_t* m_indices,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (x_dtype != FP8G_IN_BF16 && x_dtype != FP8G_IN_F32) return FP8G_ERR_INVALID_ARG;
  if (T < 0 || topk < 1 || topk > kMaxTopk || K <= 0 || K % 128 != 0 || K > 65536 || G < 1 || G > kMaxExperts)
    return FP8G_ERR_INVALID_ARG;
  const long R = static_cast<long>(T) * topk;
  if (R > 0x7FFFFFFFL) return FP8G_ERR_INVALID_ARG;
  // capacity for every possible routing: each expert wastes < 128 rows
  const long need_blocks = (R + 127) / 128 + G;
  if (blocks < need_blocks || ld_sa < blocks * 128L) return FP8G_ERR_INVALID_ARG;
  if (ld_sa % 4 != 0) return FP8G_ERR_MISALIGNED;
  if (workspace_bytes < fp8g_moe_dispatch_workspace_bytes(static_cast<int>(R), G)) return FP8G_ERR_INVALID_ARG;
  if (!A || !sa || !m_indices || !workspace || (R > 0 && (!x || !expert || !pos))) return FP8G_ERR_INVALID_ARG;
  if ((R > 0 && !aligned(x, 16)) || !aligned(A, 16) || !aligned(sa, 16) || !aligned(workspace, 4) ||
      !aligned(m_indices, 4) || (R > 0 && (!aligned(pos, 4) || !aligned(expert, 4))))
    return FP8G_ERR_MISALIGNED;
  const int sms = sm_count();
  uint32_t* err = fp8g::device_error_word();
  if (sms <= 0 || !err) return FP8G_ERR_CUDA;
  const int C = static_cast<int>(chunks_of(R));
  int32_t* hist = static_cast<int32_t*>(workspace);
  int32_t* off = hist + static_cast<long>(C) * G;
  int32_t* cnt = off + G;
  if (C > 0) moe_count_kernel<<<C, kChunk, 0, stream>>>(expert, static_cast<int>(R), G, hist, err);
  moe_scan_kernel<<<1, kMaxExperts, 0, stream>>>(hist, C, G, off, cnt, m_indices, blocks);
  if (C > 0) {
    moe_rank_kernel<<<C, kChunk, 0, stream>>>(expert, static_cast<int>(R), G, hist, off, pos, err);
    const long gblocks = std::min<long>((static_cast<long>(T) + 7) / 8, 6L * sms);
    const unsigned gb = static_cast<unsigned>(gblocks);
    const bool f32 = x_dtype == FP8G_IN_F32;
    if (topk <= 4) {
      if (f32) moe_gather_kernel<true, 4><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
      else moe_gather_kernel<false, 4><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
    } else if (topk <= 8) {
      if (f32) moe_gather_kernel<true, 8><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
      else moe_gather_kernel<false, 8><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
    } else {
      if (f32) moe_gather_kernel<true, kMaxTopk><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
      else moe_gather_kernel<false, kMaxTopk><<<gb, 256, 0, stream>>>(x, K, T, topk, pos, A, sa, ld_sa);
    }
  }
  const long pblocks = std::min<long>((static_cast<long>(G) * 128 + 7) / 8, 4L * sms);
  moe_pad_kernel<<<static_cast<unsigned>(pblocks), 256, 0, stream>>>(off, cnt, G, K, A, sa, ld_sa);
  if (cudaGetLastError() != cudaSuccess) return FP8G_ERR_CUDA;
  return FP8G_OK;
}

extern "C" int fp8g_moe_combine(const uint16_t* D, int N, const int32_t* pos, const float* w, int T, int topk,
                                uint16_t* out, cudaStream_t stream) {
  if (T < 0 || topk < 1 || topk > kMaxTopk || N < 0) return FP8G_ERR_INVALID_ARG;
  if (N % 8 != 0) return FP8G_ERR_MISALIGNED;
  if (T == 0 || N == 0) return FP8G_OK;
  if (!D || !pos || !out) return FP8G_ERR_INVALID_ARG;
  if (!aligned(D, 16) || !aligned(out, 16) || !aligned(pos, 4) || (w && !aligned(w, 4))) return FP8G_ERR_MISALIGNED;
  const int sms = sm_count();
  if (sms <= 0) return FP8G_ERR_CUDA;
  // a CTA per token: 256 threads, or fewer for narrow rows
  const int threads = std::min(256, std::max(32, (N / 8 + 31) / 32 * 32));
  const unsigned blocks = static_cast<unsigned>(std::min<long>(T, 16L * sms));
  if (topk <= 4)
    moe_combine_kernel<4><<<blocks, threads, 0, stream>>>(D, N, pos, w, T, topk, out);
  else if (topk <= 8)
    moe_combine_kernel<8><<<blocks, threads, 0, stream>>>(D, N, pos, w, T, topk, out);
  else
    moe_combine_kernel<kMaxTopk><<<blocks, threads, 0, stream>>>(D, N, pos, w, T, topk, out);
  if (cudaGetLastError() != cudaSuccess) return FP8G_ERR_CUDA;
  return FP8G_OK;
}
