// kernel_ue8m0.cuh -- FP8 NT GEMM with power-of-two (UE8M0) scales on the
// block-scaled tensor-core MMA, sm_100a.
//
//   D[m,n] = bf16( sum_kb ( sum_{k in kb} A[m,k] * B[n,k] )
//                          * 2^(ea[kb][m] - 127) * 2^(eb[n/128][kb] - 127) )
//
// The same fine-grained granularity as the FP32-scale GEMM (one scale per 1x128
// group of A, per 128x128 block of B), but the scales are powers of two, which
// the block-scaled MMA (tcgen05.mma kind::mxf8f6f4.block_scale, E8M0 scale
// factors per 32 elements of K) applies inside the tensor core.  Nothing
// leaves the tensor core between K-blocks: the FP32 accumulator stays in
// tensor memory for the whole K loop (the SM100 generation the pages list,
// kakushin.no requirements list; the numerics are those of the tensor core's
// FP32 accumulation, not the per-K-block promotion of the FP32-scale GEMM).
//
// One CTA per 128 x 256 tile (persistent):
//   warps 0, 3    TMA producers (lanes 0..3): A 128 x 128 and B 256 x 128
//                 bytes per K-block into a ring of stages.
//   warp 1        lane 0: per K-block four block-scaled MMAs (M = 128,
//                 N = 256, K = 32) into the accumulator at TMEM columns
//                 0..255, with the K-block's scale factors from a ring slot
//                 of TMEM (sf_id k selects the byte of K-chunk k); commits
//                 free the stage and the scale slot; after the tile's last
//                 K-block a commit hands the accumulator to the epilogue.
//   warps 4..7    scale writers: per K-block they write the scale factors
//                 into a TMEM ring slot with tcgen05.st, in the layout the
//                 broadcasting 32x128b.warpx4 copy produces from a 128-row
//                 scale atom: lane L, column j holds the scale bytes of row
//                 32j + L % 32 (4 columns per 128 rows; B's 256 rows take 8).
//                 All four bytes of a word are equal (one scale per 128 of K).
//   warps 8..11   epilogue: tcgen05.ld, bf16, shared memory + TMA store.
// Every wait is bounded as in the other kernels.
#pragma once

#include "kernel_pair.cuh"

namespace fp8g {

constexpr int kUe8Threads = 384;
constexpr int kSfSlots = 8;      // scale-factor ring slots in TMEM
constexpr int kSfSlotCols = 16;  // per slot: A at +0 (4 columns), B at +4 (8 columns)
constexpr int kSfBase = 256;     // TMEM column of slot 0 (the accumulator takes 0..255)

template <int STAGES>
struct Ue8Layout {
  static constexpr int kATile = 128 * 128;  // 128 rows x one K-block of e4m3
  static constexpr int kBTile = 256 * 128;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = STAGES * kATile;
  static constexpr int kStageBytes = 32 * 32 * 2;  // one epilogue warp's 32 x 32 bf16 chunk
  static constexpr int kOffStage = kOffB + STAGES * kBTile;
  static constexpr int kOffBar = kOffStage + 4 * 2 * kStageBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 * kSfSlots + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory");
};

// Instruction descriptor of kind::mxf8f6f4.block_scale: B scale-factor id in
// bits 4-5, A and B = E4M3 (bits 7-9, 10-12 = 0), K-major, N >> 3 in bits
// 17-22, scale format E8M0 (bit 23 = 1), M >> 4 in bits 24-28, A scale-factor
// id in bits 29-30, K = 32 (bit 31 = 0).
__host__ __device__ constexpr uint32_t idesc_mxf8_e8m0(uint32_t M, uint32_t N, uint32_t sf_id) {
  return (sf_id << 4) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) | (sf_id << 29);
}

template <int STAGES>
__global__ void __launch_bounds__(kUe8Threads, 1)
    fp8_gemm_ue8m0_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmD, const Params p) {
  using L = Ue8Layout<STAGES>;
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  const uint32_t bar0 = sbase + L::kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto sffull_bar = [&](int j) { return bar0 + 8u * (2 * STAGES + j); };
  auto sfempty_bar = [&](int j) { return bar0 + 8u * (2 * STAGES + kSfSlots + j); };
  const uint32_t afull_bar = bar0 + 8u * (2 * STAGES + 2 * kSfSlots);
  const uint32_t aempty_bar = afull_bar + 8u;
  const uint32_t drain_bar = afull_bar + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile uint32_t* abort_flag = tmem_slot + 1;  // [0] abort flag, [1] wait limit (us)
  auto a_tile = [&](int s) { return sbase + L::kOffA + s * L::kATile; };
  auto b_tile = [&](int s) { return sbase + L::kOffB + s * L::kBTile; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int j = 0; j < kSfSlots; ++j) {
      mbar_init(sffull_bar(j), 4);  // the four scale-writer warps
      mbar_init(sfempty_bar(j), 1);
    }
    mbar_init(afull_bar, 1);
    mbar_init(aempty_bar, 4);  // the four epilogue warps
    mbar_init(drain_bar, 1);
    abort_flag[0] = 0u;
    abort_flag[1] = p.wait_limit_us;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int t_first = static_cast<int>(blockIdx.x);
  const int t_step = static_cast<int>(gridDim.x);
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  auto tile_of = [&](int t, int& m0, int& n0) {
    m0 = (t / p.n_tiles) * 128;
    n0 = (t % p.n_tiles) * BN;
  };

  if (warp < 4) {
    if (warp == 0 || warp == 3) {
      // ------------------------------------------------------------ producers
      if (lane < kIssuersPerWarp) {
        const uint32_t me = static_cast<uint32_t>((warp == 3 ? kIssuersPerWarp : 0) + lane);
        uint32_t it = 0;
        bool ok = true;
        for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
          int m0, n0;
          tile_of(t, m0, n0);
          for (int kb = 0; kb < p.KB; ++kb, ++it) {
            if ((it % STAGES) % kIssuers != me) continue;
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full_bar(s), L::kATile + L::kBTile);
            tma_load_3d(a_tile(s), &tmA, full_bar(s), kb * 128, m0, 0);
            tma_load_3d(b_tile(s), &tmB, full_bar(s), kb * 128, n0, 0);
          }
        }
        const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i)
          if ((i % STAGES) % kIssuers == me) drain_phase(full_bar(i % STAGES), (i / STAGES) & 1u);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t it = 0, sit = 0, tile_it = 0;
      bool ok = true;
      for (int t = t_first; ok && t < p.num_tiles; t += t_step, ++tile_it) {
        if (!wait_phase(aempty_bar, (tile_it & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.KB; ++kb, ++it, ++sit) {
          const int s = it % STAGES;
          const int j = sit % kSfSlots;
          if (!wait_phase(full_bar(s), (it / STAGES) & 1u, abort_flag) ||
              !wait_phase(sffull_bar(j), (sit / kSfSlots) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_k128_sw128(a_tile(s));
          const uint64_t bdesc = sdesc_k128_sw128(b_tile(s));
          const uint32_t sfa = tmem_base + static_cast<uint32_t>(kSfBase + kSfSlotCols * j);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 4 x K = 32 = one 128-wide K-block; scale byte k
            mma_mxf8_block_scale(tmem_base, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                                 idesc_mxf8_e8m0(128, BN, static_cast<uint32_t>(k)), sfa, sfa + 4u,
                                 (kb | k) != 0 ? 1u : 0u);
          mma_commit(empty_bar(s));
          mma_commit(sfempty_bar(j));
        }
        if (ok) mma_commit(afull_bar);
      }
      mma_commit(drain_bar);
      drain_phase(drain_bar, 0u);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ scale writers
    const int q = warp % 4;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    uint32_t sit = 0;
    bool ok = true;
    for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
      int m0, n0;
      tile_of(t, m0, n0);
      const int nb0 = n0 / 128;
      for (int kb = 0; kb < p.KB; ++kb, ++sit) {
        const int j = sit % kSfSlots;
        // A: rows m0 + lane + 32 c (c = 0..3); B: the tile's two 128-row blocks
        uint32_t wa[4], wb[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = m0 + lane + 32 * c;
          const uint32_t e = row < p.M ? __ldg(p.sfa + static_cast<long>(kb) * p.ld_sa + row) : 127u;
          wa[c] = e * 0x01010101u;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t e = nb0 + h < p.NB ? __ldg(p.sfb + static_cast<long>(nb0 + h) * p.KB + kb) : 127u;
#pragma unroll
          for (int c = 0; c < 4; ++c) wb[4 * h + c] = e * 0x01010101u;
        }
        if (!__all_sync(0xffffffffu, wait_phase(sfempty_bar(j), ((sit / kSfSlots) & 1u) ^ 1u, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = tmem_base + lane_addr + static_cast<uint32_t>(kSfBase + kSfSlotCols * j);
        tmem_st_32x32b_x4(col, wa);
        tmem_st_32x32b_x8(col + 4u, wb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(sffull_bar(j));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp % 4;
    uint32_t tile_it = 0, chunk_it = 0;
    const uint32_t stage0 = sbase + L::kOffStage + static_cast<uint32_t>(q) * 2u * L::kStageBytes;
    for (int t = t_first; t < p.num_tiles; t += t_step, ++tile_it) {
      int m0, n0;
      tile_of(t, m0, n0);
      if (!__all_sync(0xffffffffu, wait_phase(afull_bar, tile_it & 1u, abort_flag))) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32, ++chunk_it) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c0, r);
        tmem_ld_wait_bind(r);
        uint4 v[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          v[jj].x = pack_bf16x2(__uint_as_float(r[8 * jj + 0]), __uint_as_float(r[8 * jj + 1]));
          v[jj].y = pack_bf16x2(__uint_as_float(r[8 * jj + 2]), __uint_as_float(r[8 * jj + 3]));
          v[jj].z = pack_bf16x2(__uint_as_float(r[8 * jj + 4]), __uint_as_float(r[8 * jj + 5]));
          v[jj].w = pack_bf16x2(__uint_as_float(r[8 * jj + 6]), __uint_as_float(r[8 * jj + 7]));
        }
        const uint32_t buf_addr = stage0 + (chunk_it & 1u) * L::kStageBytes;
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) st_shared_v4(buf_addr + static_cast<uint32_t>(lane * 64 + jj * 16), v[jj]);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0 && n0 + c0 < p.N && m0 + 32 * q < p.M) {
          tma_store_3d(&tmD, buf_addr, n0 + c0, m0 + 32 * q, 0);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(aempty_bar);
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace fp8g
