// kernel_pair.cuh -- the m-lanes GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same arithmetic as fp8_gemm_kernel with kSwap = false (D rows on TMEM
// lanes, one scale sa[m,kb] * sb[n/128,kb] per thread and K-block, FP32
// promotion on the CUDA cores), but a cluster of two CTAs computes a
// 256 x BN output tile (BN = 256 or 192) with one MMA stream:
//
//   rank r (0, 1)  holds rows m0 + 128 r .. +127 of A and rows n0 + BN/2 r ..
//                  + BN/2 - 1 of B for each K-block, in its own shared memory at the
//                  same offsets as its peer, and the 128 values sa[kb][m0 + 128 r ..]
//                  of its rows (a TMA load of its own, so the promotion reads its
//                  scales from shared memory: a global load per K-block would wait
//                  behind the operand stream in the L2-to-SM path);
//   rank 0         issues tcgen05.mma.cta_group::2 (M = 256, N = BN), which
//                  reads both CTAs' operands and writes D rows m0 + 128 r of
//                  all BN columns into CTA r's TMEM;
//   both           promote and store their own 128 rows.
//
// With BN = 256 each CTA loads 32 KB per K-block instead of the 48 KB a 128 x
// 256 tile on one CTA needs: a third less data from L2 per FLOP.
//
// Barriers (all in each CTA; the ones marked "rank 0" are used there only):
//   full[s]    rank 0: both CTAs' TMA bytes of stage s (rank 0 posts the
//              expected count for both)
//   sfull[s]   this CTA's sa slice of stage s
//   empty[s]   stage s consumed: one tcgen05.commit multicast to both CTAs,
//              plus one arrival per promotion warp of this CTA (sa slice read)
//   tfull[b]   partial b ready: one commit multicast to both CTAs
//   tempty[b]  rank 0: partial b read by every promotion warp of both CTAs
//              (the peer's arrive remotely)
// Every wait is bounded as in fp8_gemm_kernel; the CTAs of a pair leave
// through one cluster barrier after all their work (and aborts) have drained.
#pragma once

#include "kernel.cuh"

namespace fp8g {

// BN: columns of the pair tile (the MMA's N); NWG: promotion warpgroups,
// each owning BN / NWG columns.  256 / 2: 128 columns per thread (384
// threads); 192 / 3: 64 columns (512 threads), which spreads the FP32
// promotion over more warps at the cost of a narrower tile; 128 / 2: 64
// columns and four TMEM buffers instead of two, so the MMA may run up to
// three K-blocks ahead of the promotion.
constexpr int default_nwg(int BN) { return BN == 192 ? 3 : 2; }

template <int BN, int NWG = default_nwg(BN)>
struct PairShape {
  static_assert(BN == 256 || BN == 192 || BN == 128, "pair tile width");
  static_assert(NWG == default_nwg(BN), "promotion warpgroups");
  static constexpr int kNWG = NWG;                        // promotion warpgroups
  static constexpr int kCW = BN / kNWG;                   // columns per promotion thread
  static constexpr int kThreads = 128 * (1 + kNWG);
  // registers per thread at launch (the compiler's cap for kThreads per SM)
  // and after the setmaxnreg split between the control and promotion roles
  static constexpr int kLaunchRegs = kNWG == 2 ? 168 : 128;
  static constexpr bool kRegSplit = kCW > 64 || kNWG >= 3;
  static constexpr int kControlRegs = 56;
  static constexpr int kPromoRegs = kNWG == 2 ? 224 : 152;
  static constexpr int kGroup = kCW >= 128 ? 2 : 1;       // 32-column TMEM loads per wait
  static_assert(128 * kControlRegs + 128 * kNWG * kPromoRegs <= kThreads * kLaunchRegs, "register split");
  static_assert(kThreads * kLaunchRegs <= 65536, "register file");
};

template <int STAGES, int BN = 256>
struct PairLayout {
  static constexpr int kTileBytes = 128 * 128;       // A: 128 rows x one K-block of e4m3
  static constexpr int kBTileBytes = (BN / 2) * 128;  // B: this CTA's BN / 2 rows
  static constexpr int kSaBytes = 128 * 4;            // sa of this CTA's 128 rows
  static constexpr int kNBuf = 512 / BN >= 4 ? 4 : 2;  // TMEM partial buffers of BN columns
  static constexpr int kOffA = 0;
  static constexpr int kOffB = STAGES * kTileBytes;
  static constexpr int kOffSa = kOffB + STAGES * kBTileBytes;
  static constexpr int kOffBar = kOffSa + STAGES * kSaBytes;
  static constexpr int kNumBars = 3 * STAGES + 2 * kNBuf + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(STAGES % 2 == 0, "stages alternate between the two MMA issuers");
  static_assert(kBTileBytes % 1024 == 0, "swizzle-128B tiles need 1024 alignment");
  static_assert(kSmemAlloc <= 232448, "shared memory");
};

struct PairTile {
  int g, m0, n0;  // g: group of B (and of A, masked); m0: first row of the pair tile, this CTA's rows start at m0 + 128 * rank
  int mvalid;     // rows of this CTA's half to store (may be <= 0)
  bool valid;     // the pair has work on this (tile, pass)
  bool active;    // this CTA accumulates and stores in this pass
};

// Tile t, pass ps -> work of this CTA.  Dense and masked tiles have one
// pass.  A contiguous pair tile covers two 128-row blocks of A; when they
// belong to one expert it has one pass, otherwise one pass per expert block
// (the MMA runs over the whole pair each time and only the CTA whose block
// belongs to that expert keeps the result).  Every role calls this with the
// same (t, ps) and gets the same answer.
template <int KIND, int BN>
__device__ __forceinline__ PairTile get_pair_tile(const Params& p, int t, int ps, uint32_t rank, bool report) {
  PairTile T;
  T.g = 0;
  T.valid = ps == 0;
  T.active = true;
  if constexpr (KIND == kContiguous) {
    const int nt = t % p.n_tiles, mt = t / p.n_tiles;
    const int mb = p.M / 128;  // 128-row blocks of A
    int e[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int blk = 2 * mt + h;
      e[h] = blk < mb ? __ldg(p.m_indices + blk) : -1;
      if (e[h] >= p.G) {
        if (report && ps == 0) atomicOr(&g_fp8g_error_word, FP8G_DEVERR_BAD_M_INDEX);
        e[h] = -1;
      }
    }
    T.m0 = mt * 256;
    T.n0 = nt * BN;
    if (e[0] == e[1]) {
      T.valid = ps == 0 && e[0] >= 0;
      T.g = e[0];
    } else {
      // passes: block 0's expert (if any), then block 1's (if any)
      const int first = e[0] >= 0 ? 0 : 1;
      const int owner = ps == 0 ? first : 1;
      T.valid = (ps == 0 && e[first] >= 0) || (ps == 1 && first == 0 && e[1] >= 0);
      T.g = e[owner];
      T.active = static_cast<uint32_t>(owner) == rank;
    }
    T.mvalid = T.active ? min(128, p.M - (T.m0 + 128 * static_cast<int>(rank))) : 0;
  } else if constexpr (KIND == kDense) {
    // grouped raster: runs of kGroupM pair rows, N fastest within a run's
    // columns, so that the tiles in flight share few A and B tiles in L2
    constexpr int kGroupM = 8;
    const int per_group = kGroupM * p.n_tiles;
    const int grp = t / per_group, r = t % per_group;
    const int gm = min(kGroupM, p.m_tiles - grp * kGroupM);
    const int mt = grp * kGroupM + r % gm, nt = r / gm;
    T.m0 = mt * 256;
    T.n0 = nt * BN;
    T.mvalid = min(128, p.M - (T.m0 + 128 * static_cast<int>(rank)));
  } else {
    static_assert(KIND == kMasked, "pair tiles: dense, contiguous and masked");
    const int per_g = p.n_tiles * p.m_tiles;
    const int g = t / per_g, r = t % per_g;
    const int nt = r / p.m_tiles, mt = r % p.m_tiles;
    int mg = __ldg(p.masked_m + g);
    if (mg > p.M) {
      if (report) atomicOr(&g_fp8g_error_word, FP8G_DEVERR_MASKED_OVER);
      mg = p.M;
    }
    mg = max(mg, 0);
    T.g = g;
    T.m0 = mt * 256;
    T.n0 = nt * BN;
    T.mvalid = min(128, mg - (T.m0 + 128 * static_cast<int>(rank)));
    T.valid = ps == 0 && T.m0 < mg;
  }
  return T;
}

// OPT: promotion options (kOptFma2; kernel.cuh).
template <int KIND, int STAGES, int BN = 256, int OPT = 0, int NWG = default_nwg(BN)>
__global__ void __launch_bounds__(PairShape<BN, NWG>::kThreads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSA, const Params p) {
  using L = PairLayout<STAGES, BN>;
  using S = PairShape<BN, NWG>;
  constexpr int BNC = BN;
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
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + L::kNBuf + b); };
  auto drain_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 * L::kNBuf + i); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + 2 * L::kNBuf + 2 + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile uint32_t* abort_flag = tmem_slot + 1;  // [0] abort flag, [1] wait limit (us)
  auto a_tile = [&](int s) { return sbase + L::kOffA + s * L::kTileBytes; };
  auto b_tile = [&](int s) { return sbase + L::kOffB + s * L::kBTileBytes; };
  auto sa_slot = [&](int s) { return sbase + L::kOffSa + s * L::kSaBytes; };
  const float* sa_f = reinterpret_cast<const float*>(smem + L::kOffSa);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1 + 4 * S::kNWG);
      mbar_init(sfull_bar(s), 1);
    }
    for (int b = 0; b < L::kNBuf; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * 4 * S::kNWG);  // every promotion warp of both CTAs
    }
    mbar_init(drain_bar(0), 1);
    mbar_init(drain_bar(1), 1);
    abort_flag[0] = 0u;
    abort_flag[1] = p.wait_limit_us;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised before either CTA signals the other
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int t_first = static_cast<int>(blockIdx.x / 2);
  const int t_step = static_cast<int>(gridDim.x / 2);

  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr uint32_t kPairStageTx = 2u * (L::kTileBytes + L::kBTileBytes);  // A and B parts of both CTAs
  constexpr int kPasses = KIND == kContiguous ? 2 : 1;

  if (warp < 4) {
    if constexpr (S::kRegSplit) setmaxnreg_dec<S::kControlRegs>();
    if (warp == 0 || warp == 3) {
      // ------------------------------------------------------------ producers (both CTAs)
      if (lane < kIssuersPerWarp) {
        const uint32_t me = static_cast<uint32_t>((warp == 3 ? kIssuersPerWarp : 0) + lane);
        uint32_t it = 0;
        bool ok = true;
        for (int t = t_first; ok && t < p.num_tiles; t += t_step)
        for (int ps = 0; ok && ps < kPasses; ++ps) {
          const PairTile T = get_pair_tile<KIND, BN>(p, t, ps, rank, false);
          if (!T.valid) continue;
          const int ga = KIND == kMasked ? T.g : 0;
          const int gb = KIND == kDense ? 0 : T.g;
          const int arow = T.m0 + 128 * static_cast<int>(rank);
          const int brow = T.n0 + (BN / 2) * static_cast<int>(rank);
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
            tma_load_3d_pair(a_tile(s), &tmA, fb, kb * 128, arow, ga);
            tma_load_3d_pair(b_tile(s), &tmB, fb, kb * 128, brow, gb);
            // this CTA's row scales of the K-block (rows past M read as zero)
            mbar_arrive_expect_tx(sfull_bar(s), L::kSaBytes);
            tma_load_3d(sa_slot(s), &tmSA, sfull_bar(s), arow, kb, ga);
          }
        }
        // drain: rank 0's full barriers count both CTAs' operand bytes, and
        // each CTA's sfull barriers its own scale loads, so every load of the
        // pair has landed once they complete
        {
          const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
          for (uint32_t i = first; i < it; ++i) {
            if ((i % STAGES) % kIssuers != me) continue;
            if (rank == 0) drain_phase(full_bar(i % STAGES), (i / STAGES) & 1u);
            drain_phase(sfull_bar(i % STAGES), (i / STAGES) & 1u);
          }
        }
      }
    } else if (rank == 0 && lane == 0) {
      // ------------------------------------------------------------ MMA issuers (rank 0, warps 1 and 2)
      const uint32_t me = static_cast<uint32_t>(warp - 1);
      constexpr uint32_t kIdesc = idesc_e4m3_f32(256, BNC);
      uint32_t it = 0;
      bool ok = true;
      for (int t = t_first; ok && t < p.num_tiles; t += t_step)
      for (int ps = 0; ok && ps < kPasses; ++ps) {
        const PairTile T = get_pair_tile<KIND, BN>(p, t, ps, rank, false);
        if (!T.valid) continue;
        for (int kb = 0; kb < p.KB; ++kb, ++it) {
          if ((it % STAGES) % 2 != me) continue;
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const int b = it % L::kNBuf;
          const uint32_t tph = (it / L::kNBuf) & 1u;
          if (!wait_phase(full_bar(s), ph, abort_flag) ||
              !wait_phase(tempty_bar(b), tph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BNC);
          const uint64_t adesc = sdesc_k128_sw128(a_tile(s));
          const uint64_t bdesc = sdesc_k128_sw128(b_tile(s));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f8f6f4_pair(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                            kIdesc, k > 0 ? 1u : 0u);
          mma_commit_pair(empty_bar(s), 0x3);
          mma_commit_pair(tfull_bar(b), 0x3);
        }
      }
      // drain: every MMA of this thread completes before TMEM is freed
      mma_commit_pair(drain_bar(me), 0x1);
      drain_phase(drain_bar(me), 0u);
    }
  } else {
    // ------------------------------------------------------------ promotion + epilogue (both CTAs)
    if constexpr (S::kRegSplit) setmaxnreg_inc<S::kPromoRegs>();
    // rank 1 releases TMEM buffers on rank 0's barriers (consecutive offsets
    // in rank 0's shared memory window)
    const uint32_t tempty_remote = mapa(tempty_bar(0), 0);
    constexpr int kCW = S::kCW;  // columns per promotion warpgroup
    const int wg = (warp - 4) / 4;
    const int q = warp % 4;
    const int row = 32 * q + lane;
    float acc[kCW];
    uint32_t it = 0;
    bool ok = true;
    for (int t = t_first; ok && t < p.num_tiles; t += t_step)
    for (int ps = 0; ok && ps < kPasses; ++ps) {
      const PairTile T = get_pair_tile<KIND, BN>(p, t, ps, rank, warp == 4 && lane == 0 && rank == 0);
      if (!T.valid) continue;
#pragma unroll
      for (int c = 0; c < kCW; ++c) acc[c] = 0.f;
      const int m_row = T.m0 + 128 * static_cast<int>(rank) + row;  // this thread's row of A and D
      const int nb = min((T.n0 + wg * kCW) / 128, p.NB - 1);
      const float* sbp = p.sb + (static_cast<long>(T.g) * p.NB + nb) * p.KB;
      const bool row_in = m_row < p.M;
      // sb of this warpgroup's columns, 32 K-blocks per register: lane i
      // holds K-block 32 j + i; the next 32 are loaded one chunk ahead and
      // each K-block's value is broadcast with a shuffle
      float sb_cur = lane < p.KB ? __ldg(sbp + lane) : 0.f;
      float sb_nxt = 32 + lane < p.KB ? __ldg(sbp + 32 + lane) : 0.f;
      for (int kb = 0; ok && kb < p.KB; ++kb, ++it) {
        if ((kb & 31) == 0 && kb != 0) {
          sb_cur = sb_nxt;
          sb_nxt = kb + 32 + lane < p.KB ? __ldg(sbp + kb + 32 + lane) : 0.f;
        }
        const float s_b = __shfl_sync(0xffffffffu, sb_cur, kb & 31);
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        const int b = it % L::kNBuf;
        const uint32_t tph = (it / L::kNBuf) & 1u;
        bool w = wait_phase(tfull_bar(b), tph, abort_flag);
        w = w && wait_phase(sfull_bar(s), ph, abort_flag);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the row's scale for this K-block; the stage's sa slot is free once
        // every lane has read it (release arrive, after the warp's reads)
        const float sc = row_in ? sa_f[s * 128 + row] * s_b : 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                               static_cast<uint32_t>(b * BNC + wg * kCW);
        constexpr int kG = S::kGroup;
        // a CTA whose block belongs to the other expert of this pass only
        // hands the buffer back
        if (T.active) {
#pragma unroll
          for (int j0 = 0; j0 < kCW / 32; j0 += kG) {
            uint32_t r[kG][32];
#pragma unroll
            for (int j = 0; j < kG; ++j) tmem_ld_32x32b_x32(taddr + 32 * (j0 + j), r[j]);
            tmem_ld_wait_bind(r[0]);
#pragma unroll
            for (int j = 1; j < kG; ++j) bind_after_wait(r[j]);
#pragma unroll
            for (int j = 0; j < kG; ++j) {
              float* a = acc + 32 * (j0 + j);
              if constexpr ((OPT & kOptFma2) != 0) {
#pragma unroll
                for (int c = 0; c < 32; c += 2) ffma2(a[c], a[c + 1], r[j][c], r[j][c + 1], sc);
              } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) a[c] = fmaf(__uint_as_float(r[j][c]), sc, a[c]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive_relaxed(tempty_bar(b));
          else mbar_arrive_remote_relaxed(tempty_remote + 8u * b);
        }
      }
      if (!ok) break;

      // epilogue: a thread holds kCW consecutive columns of its row
      if (row < T.mvalid) {
        const long drow0 = KIND == kMasked ? static_cast<long>(T.g) * p.M : 0;
        uint16_t* drow = p.D + (drow0 + m_row) * p.N + T.n0 + wg * kCW;
#pragma unroll
        for (int c = 0; c < kCW; c += 8) {
          if (T.n0 + wg * kCW + c < p.N) {
            uint4 v;
            v.x = pack_bf16x2(acc[c + 0], acc[c + 1]);
            v.y = pack_bf16x2(acc[c + 2], acc[c + 3]);
            v.z = pack_bf16x2(acc[c + 4], acc[c + 5]);
            v.w = pack_bf16x2(acc[c + 6], acc[c + 7]);
            *reinterpret_cast<uint4*>(drow + c) = v;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // rank 0's MMAs into rank 1's TMEM, rank 1's loads counted on rank 0's
  // barriers and rank 1's remote arrivals are all finished past this point
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace fp8g
