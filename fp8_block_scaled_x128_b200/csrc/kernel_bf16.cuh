// kernel_bf16.cuh -- BF16 NT GEMM on the same TMA + tcgen05 pipeline, sm_100a.
//
//   D[m,n] = bf16( sum_k A[m,k] * B[n,k] ),  A [M,K], B [N,K], D [M,N] bf16,
//
// the other input format the pages list next to FP8 (kakushin.no, "Hva gjør
// DeepGEMM?").  Without per-K-block scales nothing has to leave the tensor
// core between K-blocks: the FP32 accumulator stays in tensor memory for the
// whole K loop and is read once per tile.
//
// CTA pairs (tcgen05 cta_group::2), 256 x 256 tiles, persistent, the grouped
// raster of the FP8 pair kernel:
//   warps 0, 3    TMA producers (lanes 0..3), as in the FP8 pair kernel: each
//                 CTA loads its 128 rows of A and 128 rows of B per 64-wide
//                 K-block (128 bytes per row, 128-byte swizzle); rank 1's
//                 bytes complete on rank 0's full barrier.
//   warp 1        rank 0, lane 0: four tcgen05.mma.cta_group::2.kind::f16
//                 (M = 256, N = 256, K = 16, bf16 x bf16 -> FP32) per K-block
//                 into one of two 256-column TMEM accumulators; after the
//                 tile's last K-block one commit (multicast to both CTAs)
//                 hands the accumulator to the epilogue.  Two accumulators
//                 let the MMA run the next tile while the epilogue drains.
//   warps 4..7    epilogue, both CTAs: tcgen05.ld 32 columns at a time, round
//                 to bf16 and store D; then release the accumulator (rank 1
//                 on rank 0's barrier).  kTmaStore: each warp writes its 32 x
//                 32 chunk to shared memory (double-buffered) and one lane
//                 issues a TMA tensor store (clipped at M and N by the
//                 tensor map); otherwise 16-byte stores straight from
//                 registers, predicated on M and N.
// Every wait is bounded as in the FP8 kernels.
#pragma once

#include "kernel_pair.cuh"

namespace fp8g {

constexpr int kBf16Threads = 256;

template <int STAGES, bool kTmaStore>
struct Bf16Layout {
  static constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16 (one K-block) of A or of B per CTA
  static constexpr int kOffA = 0;
  static constexpr int kOffB = STAGES * kTileBytes;
  static constexpr int kStageBytes = 32 * 32 * 2;                  // one warp's 32 x 32 bf16 chunk
  static constexpr int kOffStage = kOffB + STAGES * kTileBytes;    // 4 warps x 2 buffers
  static constexpr int kStageAll = kTmaStore ? 4 * 2 * kStageBytes : 0;
  static constexpr int kOffBar = kOffStage + kStageAll;
  static constexpr int kNumBars = 2 * STAGES + 2 * 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory");
};

// Instruction descriptor for kind::f16: D = F32 (bits 4-5 = 1), A and B =
// BF16 (bits 7-9 and 10-12 = 1; both operands of one MMA must have the same
// type), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

template <int STAGES, bool kTmaStore>
__global__ void __launch_bounds__(kBf16Threads, 1)
    bf16_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmD, const Params p) {
  using L = Bf16Layout<STAGES, kTmaStore>;
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();

  const uint32_t bar0 = sbase + L::kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto afull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto aempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile uint32_t* abort_flag = tmem_slot + 1;  // [0] abort flag, [1] wait limit (us)
  auto a_tile = [&](int s) { return sbase + L::kOffA + s * L::kTileBytes; };
  auto b_tile = [&](int s) { return sbase + L::kOffB + s * L::kTileBytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(afull_bar(b), 1);
      mbar_init(aempty_bar(b), 2 * 4);  // the epilogue warps of both CTAs
    }
    mbar_init(drain_bar, 1);
    abort_flag[0] = 0u;
    abort_flag[1] = p.wait_limit_us;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if constexpr (kTmaStore) prefetch_tmap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int t_first = static_cast<int>(blockIdx.x / 2);
  const int t_step = static_cast<int>(gridDim.x / 2);
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr uint32_t kPairStageTx = 2u * (2u * L::kTileBytes);  // A and B of both CTAs

  if (warp < 4) {
    if (warp == 0 || warp == 3) {
      // ------------------------------------------------------------ producers (both CTAs)
      if (lane < kIssuersPerWarp) {
        const uint32_t me = static_cast<uint32_t>((warp == 3 ? kIssuersPerWarp : 0) + lane);
        uint32_t it = 0;
        bool ok = true;
        for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
          const PairTile T = get_pair_tile<kDense, BN>(p, t, 0, rank, false);
          const int arow = T.m0 + 128 * static_cast<int>(rank);
          const int brow = T.n0 + 128 * static_cast<int>(rank);
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            if ((it % STAGES) % kIssuers != me) continue;
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            const uint32_t fb = rank == 0 ? full_bar(s) : mapa(full_bar(s), 0);
            if (rank == 0) mbar_arrive_expect_tx(full_bar(s), kPairStageTx);
            tma_load_3d_pair(a_tile(s), &tmA, fb, kb * 64, arow, 0);
            tma_load_3d_pair(b_tile(s), &tmB, fb, kb * 64, brow, 0);
          }
        }
        if (rank == 0) {
          const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
          for (uint32_t i = first; i < it; ++i)
            if ((i % STAGES) % kIssuers == me) drain_phase(full_bar(i % STAGES), (i / STAGES) & 1u);
        }
      }
    } else if (warp == 1 && rank == 0 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer (rank 0)
      constexpr uint32_t kIdesc = idesc_bf16_f32(256, BN);
      uint32_t it = 0, tile_it = 0;
      bool ok = true;
      for (int t = t_first; ok && t < p.num_tiles; t += t_step, ++tile_it) {
        const int buf = tile_it & 1;
        if (!wait_phase(aempty_bar(buf), ((tile_it >> 1) & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase(full_bar(s), ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_k128_sw128(a_tile(s));
          const uint64_t bdesc = sdesc_k128_sw128(b_tile(s));
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K = 16 bf16 (32 bytes) = one 64-wide K-block
            mma_bf16_pair(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k), kIdesc,
                          (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(empty_bar(s), 0x3);
        }
        if (ok) mma_commit_pair(afull_bar(buf), 0x3);
      }
      mma_commit_pair(drain_bar, 0x1);
      drain_phase(drain_bar, 0u);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const uint32_t aempty_remote = mapa(aempty_bar(0), 0);
    const int q = warp % 4;
    const int row = 32 * q + lane;  // TMEM lane = row of this CTA's half of the tile
    uint32_t tile_it = 0, chunk_it = 0;
    const uint32_t stage0 = sbase + L::kOffStage + static_cast<uint32_t>(q) * 2u * L::kStageBytes;
    for (int t = t_first; t < p.num_tiles; t += t_step, ++tile_it) {
      const PairTile T = get_pair_tile<kDense, BN>(p, t, 0, rank, false);
      const int buf = tile_it & 1;
      if (!__all_sync(0xffffffffu, wait_phase(afull_bar(buf), (tile_it >> 1) & 1u, abort_flag))) break;
      tc_fence_after();
      const int m = T.m0 + 128 * static_cast<int>(rank) + row;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * BN);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c0, r);
        tmem_ld_wait_bind(r);
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[j].x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
          v[j].y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
          v[j].z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
          v[j].w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
        }
        const int n = T.n0 + c0;
        if constexpr (kTmaStore) {
          // this warp's 32 rows x 32 columns through shared memory, if any of
          // them is inside D (warp-uniform): every buffer write is followed
          // by a store, so waiting until at most one store group is pending
          // (the other buffer's) frees this buffer
          const int r0 = T.m0 + 128 * static_cast<int>(rank) + 32 * q;
          if (n < p.N && r0 < p.M) {
            const uint32_t buf_addr = stage0 + (chunk_it & 1u) * L::kStageBytes;
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j) st_shared_v4(buf_addr + static_cast<uint32_t>(lane * 64 + j * 16), v[j]);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmD, buf_addr, n, r0, 0);
              bulk_commit_group();
            }
            ++chunk_it;
          }
        } else {
          if (m < p.M) {
            uint16_t* drow = p.D + static_cast<long>(m) * p.N + n;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (n + 8 * j < p.N) *reinterpret_cast<uint4*>(drow + 8 * j) = v[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive_relaxed(aempty_bar(buf));
        else mbar_arrive_remote_relaxed(aempty_remote + 8u * buf);
      }
    }
    if constexpr (kTmaStore) {
      if (lane == 0) bulk_wait_group<0>();  // every store of this warp has completed
      __syncwarp();
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace fp8g
