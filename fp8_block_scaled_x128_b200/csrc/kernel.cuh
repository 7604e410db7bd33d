// kernel.cuh -- the fine-grained-scaled FP8 GEMM kernel for sm_100a.
//
//   D[m,n] = bf16( sum_kb P_kb[m,n] * sa[m,kb] * sb[n/128,kb] ),
//   P_kb[m,n] = sum_{k in kb} A[m,k] * B[n,k]     (one 128-wide K-block)
//
// Fine-grained scaling of DeepSeek-V3 with the per-K-block partial promoted
// out of the tensor-core accumulator onto the CUDA cores (GeekNews, "DeepSeek,
// DeepGEMM 오픈소스 공개", topic body, first and fifth bullets).  The pages'
// own design is a Hopper one (wgmma, register accumulators); this is a
// Blackwell design:
//
//   warps 0, 3    TMA producers: for every (tile, K-block) one stage of a
//                 shared-memory ring receives the 128-row "lane" operand
//                 tile, the "column" operand tile and (n-lanes only) the
//                 tile's slice of sa.
//                 Lanes 0..3 of both warps issue; stage s belongs to issuer
//                 s % 8 for every round (one thread issues only about one
//                 TMA operation per 150 ns, which would cap a CTA near
//                 50 GB/s).
//   warps 1, 2    MMA issuers (lane 0 of each; stage s belongs to issuer
//                 s % 2): four tcgen05.mma kind::f8f6f4 (K = 32 each) write
//                 the K-block partial P_kb, FP32, into one of several
//                 tensor-memory (TMEM) buffers; tcgen05.commit frees the
//                 stage and signals the partial.  A single thread spends
//                 several hundred cycles per K-block on waits, MMA issue
//                 and commits, more than an N <= 128 MMA takes to execute;
//                 two issuers overlap that work.
//   warps 4..11   two promotion warpgroups, each owning half the tile's
//                 columns: tcgen05.ld the finished partial, acc += P * scale
//                 in FP32 registers (CUDA cores), release the TMEM buffer so
//                 the MMA of a later K-block overlaps; after the tile's last
//                 K-block, round to bf16 and store D.  m-lanes: the thread's
//                 scale sa[kb][m] * sb[g][nb][kb] is loaded from global
//                 memory two K-blocks ahead; n-lanes: the per-column sa comes
//                 with the stage and sb is prefetched 32 K-blocks at a time
//                 into a register per lane and broadcast with a shuffle.
//                 TMEM buffers are released with relaxed arrives.
//
// Orientation.  The MMA's M side (TMEM lanes) is always 128 rows.
//   kSwap = true : lanes are 128 rows of B (n), columns are BNC rows of A
//                  (m).  Used when M is small (decode), so that the large
//                  operand fills the MMA's M; the B scale is one scalar per
//                  (tile, K-block) and the A scale varies per column.
//   kSwap = false: lanes are 128 rows of A (m), columns are BNC rows of B.
//                  The A scale is one scalar per thread, the B scale one per
//                  128 columns.  With BNC = 256 each promotion thread holds
//                  128 accumulators, so the warpgroups trade registers with
//                  setmaxnreg (control 56, promotion 224 per thread).
// Scheduling kinds: dense; contiguous (128-row blocks of A map to experts via
// m_indices, -1 = skip); masked (tiles at or past masked_m[g] are skipped).
// SPLIT > 1 (dense, kSwap only): a cluster of SPLIT CTAs shares one output
// tile, each over K/SPLIT.  Each CTA stores its partial sums into the shared
// memory of the CTA that owns those columns; after one cluster barrier every
// CTA adds the SPLIT partials of its columns in rank order (deterministic).
// SPLIT < 0 (global split-K): gsplit CTAs per tile store FP32 partials to a
// workspace; either the CTAs of the tile reduce them after an arrival count
// (kGlobalSplit) or splitk_reduce_kernel, launched next, does
// (kGlobalSplitPartials).
// The CTA-pair kernel (tcgen05 cta_group::2) is in kernel_pair.cuh.
//
// Programmatic dependent launch: the prologue (barrier init, TMEM
// allocation, tensor-map prefetch) runs before griddepcontrol.wait, so it can
// overlap the previous kernel in the stream; no global memory is touched
// before that wait.
//
// Every wait is bounded: after kWaitTimeoutNs the waiter records
// FP8G_DEVERR_TIMEOUT, raises a CTA-wide abort flag, and every role leaves
// its loop; the teardown drains in-flight TMA and MMA work (again with a
// bound) and frees TMEM before the CTA exits.
#pragma once

#include <cstdint>

#include "ptx.cuh"

#ifndef FP8G_DEVERR_TIMEOUT
#define FP8G_DEVERR_TIMEOUT 0x1u
#define FP8G_DEVERR_BAD_M_INDEX 0x2u
#define FP8G_DEVERR_MASKED_OVER 0x4u
#endif

namespace fp8g {

enum Kind : int { kDense = 0, kContiguous = 1, kMasked = 2, kBf16Dense = 3, kUe8m0Dense = 4 };

constexpr int kThreads = 384;
constexpr int kIssuersPerWarp = 4;                  // TMA-issuing lanes in each producer warp
constexpr int kIssuers = 2 * kIssuersPerWarp;       // warps 0 and 3
constexpr int kKBMax = 512;                         // K <= 65536
constexpr uint32_t kWaitLimitUs = 1000000u;         // 1 s: the default wait limit
constexpr uint64_t kDrainTimeoutNs = 100000000ull;  // 0.1 s

// Per-device error word (FP8G_DEVERR_* bits); read by fp8g_get_device_error.
__device__ uint32_t g_fp8g_error_word;

struct Params {
  int M;        // dense/contiguous: rows of A; masked: Mmax
  int N, K, KB, NB, G;
  int n_tiles;  // tiles along N
  int m_tiles;  // tiles along M (per group for masked)
  int num_tiles;
  const int32_t* m_indices;
  const int32_t* masked_m;
  const float* sa;  // [G][KB][ld_sa] (masked) or [KB][ld_sa]
  int ld_sa;
  const float* sb;  // [G][NB][KB]
  uint16_t* D;
  // global split-K (SPLIT == kGlobalSplit): K is split over `gsplit` CTAs per
  // tile; partials go to ws[tile][rank][BNC][128] and sync[2*tile + {0,1}]
  // counts arrivals and departures (zero between calls: the last CTA of a
  // tile to leave resets them)
  int gsplit;
  float* ws;
  uint32_t* sync;
  // every pipeline wait gives up after wait_limit_us microseconds; a test
  // hook may also make the TMA producers of the single-CTA kernel skip the
  // loads of pipeline iteration test_withhold_it (-1: none), so that a wait
  // runs out without any fault
  uint32_t wait_limit_us;
  int test_withhold_it;
  // power-of-two scale bytes of the UE8M0 GEMM: sfa [KB][ld_sa], sfb [NB][KB]
  const uint8_t* sfa;
  const uint8_t* sfb;
};

// SPLIT template values selecting the global-memory split-K (count at run
// time): kGlobalSplit reduces inside the kernel after a per-tile arrival
// count; kGlobalSplitPartials only stores the partials and leaves the sum to
// splitk_reduce_kernel, launched next on the same stream.
constexpr int kGlobalSplit = -1;
constexpr int kGlobalSplitPartials = -2;

constexpr int kMaxGSplit = 16;  // the host never picks more

// OPT bits of the promotion (template parameter of both kernels):
//   kOptFma2: packed FP32x2 fused multiply-adds (fma.rn.f32x2; each half
//             rounds like fmaf, so results are unchanged).  Measured: 5-11 %
//             fewer cycles on the dense CTA-pair kernel, 4-5 % less time on
//             the masked one; slower on the single-CTA 256-wide kernel, whose
//             promotion threads then spill.
constexpr int kOptFma2 = 2;
//   kOptTmaStore (m-lanes, single CTA, no split): the epilogue stages each
//             warp's 32 rows x 32 columns of bf16 in shared memory (two
//             buffers per warp) and one lane stores them with a TMA tensor
//             store; the D tensor map takes the third map slot (tmSA, which
//             the m-lanes kernels do not use otherwise).  Every row of a
//             valid tile is written (contiguous and dense tiles, whose rows
//             past M the map clips), so masked tiles keep direct stores.
constexpr int kOptTmaStore = 4;

constexpr int pow2_at_least(int x, int lo) {
  int p = lo;
  while (p < x) p *= 2;
  return p;
}

template <bool kSwap, int BNC, int STAGES, int SPLIT, bool kTmaStore = false>
struct Layout {
  static constexpr int kLaneBytes = 128 * 128;   // 128 rows x 128 e4m3 (one K-block)
  static constexpr int kColBytes = BNC * 128;
  static constexpr int kSaFloats = kSwap ? BNC : 0;  // sa slice (n-lanes only): the tile's m-extent
  static constexpr int kNBuf = 512 / BNC < 8 ? 512 / BNC : 8;  // TMEM partial buffers
  static constexpr int kTmemCols = pow2_at_least(kNBuf * BNC, 32);
  static constexpr int kCW = BNC / 2;                  // columns per promotion warpgroup
  static constexpr bool kRegSplit = kCW > 64;          // 128 accumulators per thread
  static constexpr int kCPD = SPLIT > 1 ? BNC / SPLIT : BNC;  // cluster split-K: columns reduced per CTA
  static constexpr int kOffLane = 0;
  static constexpr int kOffCol = kOffLane + STAGES * kLaneBytes;
  static constexpr int kOffSa = kOffCol + STAGES * kColBytes;
  static constexpr int kOffRecv = kOffSa + STAGES * kSaFloats * 4;
  static constexpr int kRecvBytes = SPLIT > 1 ? SPLIT * 128 * kCPD * 4 : 0;
  static constexpr int kStoreChunk = 32 * 32 * 2;                       // one warp's 32 x 32 bf16
  static constexpr int kOffStore = kOffRecv + kRecvBytes;
  static constexpr int kStoreBytes = kTmaStore ? 8 * 2 * kStoreChunk : 0;  // 8 promotion warps x 2 buffers
  static constexpr int kOffBar = kOffStore + kStoreBytes;
  static constexpr int kNumBars = 2 * STAGES + 2 * kNBuf + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;  // + slack to align the base to 1024

  static_assert(BNC % 32 == 0 && BNC >= 32 && BNC <= 256, "column tile");
  static_assert(kCW % 32 == 0, "promotion chunking");
  static_assert(kTmemCols <= 512, "TMEM");
  static_assert(STAGES % 2 == 0 && kNBuf % 2 == 0, "stages and TMEM buffers alternate between the two MMA issuers");
  static_assert(kOffCol % 1024 == 0 && kOffSa % 1024 == 0, "swizzle-128B tiles need 1024 alignment");
  static_assert(kColBytes % 1024 == 0, "column tile rows must be a multiple of 8");
  static_assert(SPLIT <= 1 || (kSwap && BNC % SPLIT == 0 && kCW % kCPD == 0 && kCPD % 4 == 0),
                "cluster split-K layout");
  static_assert(SPLIT >= 1 || kSwap, "global split-K is for the n-lanes orientation");
  static_assert(!kRegSplit || !kSwap, "the register split is for the m-lanes orientation");
  static_assert(kSmemAlloc <= 232448, "shared memory");
  static_assert(kNBuf >= 2, "TMEM buffers");
  static_assert(!kTmaStore || (!kSwap && SPLIT == 1), "TMA-store epilogue: m-lanes tiles without split-K");
};

// Register budget of the BNC = 256 variants: 384 threads launch with 168
// registers each (the compiler's cap for 384 threads per SM); the control
// warpgroup gives back 112 per thread and the two promotion warpgroups take
// 56 more each: 128 * (168 - 56) == 256 * (224 - 168).
constexpr int kLaunchRegs = 168, kControlRegs = 56, kPromoRegs = 224;
static_assert(128 * (kLaunchRegs - kControlRegs) == 256 * (kPromoRegs - kLaunchRegs), "register split");

struct Tile {
  int g, m0, n0, mvalid, kb0, kb1;
  bool valid;
};

// Tile t -> (group, rows, columns, valid row count, K-block range).  Every
// role calls this with the same t and gets the same answer.
template <bool kSwap, int BNC, int KIND, int SPLIT>
__device__ __forceinline__ Tile get_tile(const Params& p, int t, uint32_t rank, bool report) {
  constexpr int kMExt = kSwap ? BNC : 128;
  constexpr int kNExt = kSwap ? 128 : BNC;
  Tile T;
  T.valid = true;
  T.g = 0;
  T.kb0 = 0;
  T.kb1 = p.KB;
  if constexpr (SPLIT != 1) {
    const long ns = SPLIT > 1 ? SPLIT : p.gsplit;
    T.kb0 = static_cast<int>((static_cast<long>(p.KB) * rank) / ns);
    T.kb1 = static_cast<int>((static_cast<long>(p.KB) * (rank + 1)) / ns);
  }
  if constexpr (KIND == kDense) {
    // global split-K: the grid carries the tile coordinates (t == mt*n_tiles + nt)
    const int nt = SPLIT < 0 ? static_cast<int>(blockIdx.y) : t % p.n_tiles;
    const int mt = SPLIT < 0 ? static_cast<int>(blockIdx.z) : t / p.n_tiles;
    T.m0 = mt * kMExt;
    T.n0 = nt * kNExt;
    T.mvalid = min(kMExt, p.M - T.m0);
  } else if constexpr (KIND == kContiguous) {
    const int nt = t % p.n_tiles, mt = t / p.n_tiles;
    T.m0 = mt * 128;
    T.n0 = nt * kNExt;
    T.mvalid = 128;
    const int g = __ldg(p.m_indices + mt);
    if (g < 0 || g >= p.G) {
      if (g >= p.G && report) atomicOr(&g_fp8g_error_word, FP8G_DEVERR_BAD_M_INDEX);
      T.valid = false;
    }
    T.g = g;
  } else {
    const int per_g = p.n_tiles * p.m_tiles;
    const int g = t / per_g, r = t % per_g;
    const int nt = r / p.m_tiles, mt = r % p.m_tiles;  // tiles sharing a B tile are adjacent
    int mg = __ldg(p.masked_m + g);
    if (mg > p.M) {
      if (report) atomicOr(&g_fp8g_error_word, FP8G_DEVERR_MASKED_OVER);
      mg = p.M;
    }
    mg = max(mg, 0);
    T.g = g;
    T.m0 = mt * kMExt;
    T.n0 = nt * kNExt;
    T.mvalid = min(kMExt, mg - T.m0);
    T.valid = T.m0 < mg;
  }
  return T;
}

// Bounded wait on a local mbarrier phase.  Returns false on timeout (after
// recording it) or when another role has already aborted.  ctl[0] is the
// CTA's abort flag, ctl[1] the wait limit in microseconds (both in shared
// memory, set up by thread 0 from Params::wait_limit_us).
template <bool kClusterScope = false>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity,
                                           volatile uint32_t* abort_flag) {
  auto poll = [&]() {
    return kClusterScope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (poll()) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (poll()) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      // the limit is read only here, off the path of a wait that completes
      if (globaltimer_ns() - t0 > 1000ull * abort_flag[1]) {
        *abort_flag = 1u;
        atomicOr(&g_fp8g_error_word, FP8G_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Teardown drain: like wait_phase, but ignores the abort flag and gives up
// silently after kDrainTimeoutNs.
__device__ __forceinline__ void drain_phase(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainTimeoutNs) return;
  }
}

// Global split-K reduction, run by the 256 promotion threads of every CTA of
// a tile after they stored their partial: publish (fence + arrival count),
// wait until all p.gsplit CTAs of the tile have published, then add the
// partials of this CTA's columns (rows of D) in rank order and store bf16.
// The CTAs of a tile must be resident together: the grid never exceeds the
// SM count and the wait is bounded.
template <int BNC, int KIND>
__device__ __forceinline__ void global_split_reduce(const Params& p, int tile, uint32_t rank,
                                                    volatile uint32_t* abort_flag) {
  const int tid = threadIdx.x - 128;  // 0..255
  uint32_t* arrive = p.sync + 2 * tile;
  uint32_t* depart = arrive + 1;
  named_barrier_sync(1, 256);  // every partial of this CTA is written
  if (tid == 0) {
    __threadfence();
    atomicAdd(arrive, 1u);
  }
  // wait for the other CTAs of the tile (one poller, then the barrier)
  if (tid == 0) {
    const uint32_t need = static_cast<uint32_t>(p.gsplit);
    if (ld_acquire_gpu(arrive) < need && !*abort_flag) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_gpu(arrive) < need) {
        if (*abort_flag) break;
        if (globaltimer_ns() - t0 > 1000ull * abort_flag[1]) {
          *abort_flag = 1u;
          atomicOr(&g_fp8g_error_word, FP8G_DEVERR_TIMEOUT);
          break;
        }
      }
    }
  }
  named_barrier_sync(1, 256);
  if (!*abort_flag) {
    // columns [c0, c1) of the tile: rows m0 + c of D; thread -> (row, column parity)
    const int cpd = (BNC + p.gsplit - 1) / p.gsplit;
    const int c0 = static_cast<int>(rank) * cpd, c1 = min(BNC, c0 + cpd);
    const int row = tid & 127;
    const int tile_n = tile % p.n_tiles, tile_m = tile / p.n_tiles;
    const int n = tile_n * 128 + row;
    const int m0 = tile_m * BNC;
    const long base = static_cast<long>(tile) * p.gsplit * (BNC * 128);
    for (int c = c0 + (tid >> 7); c < c1; c += 2) {
      // all partials of this element are loaded before the rank-order sum
      float v[kMaxGSplit];
#pragma unroll
      for (int src = 0; src < kMaxGSplit; ++src)
        v[src] = src < p.gsplit ? __ldcg(p.ws + base + (src * BNC + c) * 128 + row) : 0.f;
      float sum = 0.f;
#pragma unroll
      for (int src = 0; src < kMaxGSplit; ++src) sum += v[src];
      if (n < p.N && m0 + c < p.M)
        p.D[static_cast<long>(m0 + c) * p.N + n] = static_cast<uint16_t>(pack_bf16x2(sum, 0.f) & 0xFFFFu);
    }
  }
  named_barrier_sync(1, 256);  // this CTA's reads of the workspace are done
  if (tid == 0 && atomicAdd(depart, 1u) == static_cast<uint32_t>(p.gsplit) - 1) {
    // the last CTA of the tile to leave resets the counters for the next call
    *arrive = 0u;
    *depart = 0u;
  }
}

template <bool kSwap, int BNC, int STAGES, int KIND, int SPLIT, int OPT = 0>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSA, const Params p) {
  constexpr bool kTmaStore = (OPT & kOptTmaStore) != 0;
  using L = Layout<kSwap, BNC, STAGES, SPLIT, kTmaStore>;
  static_assert(!kTmaStore || KIND != kMasked, "masked tiles store only their valid rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // barriers
  const uint32_t bar0 = sbase + L::kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + L::kNBuf + b); };
  auto drain_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 * L::kNBuf + i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
  volatile uint32_t* abort_flag = tmem_slot + 1;  // [0] abort flag, [1] wait limit (us)

  // stage buffers
  auto lane_tile = [&](int s) { return sbase + L::kOffLane + s * L::kLaneBytes; };
  auto col_tile = [&](int s) { return sbase + L::kOffCol + s * L::kColBytes; };
  auto sa_slice = [&](int s) { return sbase + L::kOffSa + s * L::kSaFloats * 4; };
  const float* sa_f = reinterpret_cast<const float*>(smem + L::kOffSa);

  constexpr int kPromoWarps = 8;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      // MMA commit, plus the promotion warps where they read the stage's sa slice
      mbar_init(empty_bar(s), kSwap ? 1 + kPromoWarps : 1);
    }
    for (int b = 0; b < L::kNBuf; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kPromoWarps);
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
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (SPLIT > 1) cluster_sync_all();
  const uint32_t tmem_base = *tmem_slot;

  // split-K: one tile per CTA (t_step ends the tile loop after it).  The
  // global split-K grid is (rank, N-tile, M-tile), so no division is needed.
  const uint32_t rank = SPLIT > 1 ? cluster_ctarank() : SPLIT < 0 ? blockIdx.x : 0u;
  const int t_first = SPLIT > 1 ? static_cast<int>(blockIdx.x) / SPLIT
                      : SPLIT < 0 ? static_cast<int>(blockIdx.z * gridDim.y + blockIdx.y)
                                  : static_cast<int>(blockIdx.x);
  const int t_step = SPLIT != 1 ? p.num_tiles : static_cast<int>(gridDim.x);

  // inputs may be written by the previous kernel in the stream: wait for it
  // (a no-op without a programmatic dependency), then let the next one start
  // its own prologue
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr uint32_t kStageTx = L::kLaneBytes + L::kColBytes + L::kSaFloats * 4;

  if (warp < 4) {
  if constexpr (L::kRegSplit) setmaxnreg_dec<kControlRegs>();
  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    if (lane < kIssuersPerWarp) {
      const uint32_t me = static_cast<uint32_t>((warp == 3 ? kIssuersPerWarp : 0) + lane);
      uint32_t it = 0;
      bool ok = true;
      for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
        const Tile T = get_tile<kSwap, BNC, KIND, SPLIT>(p, t, rank, false);
        if (!T.valid) continue;
        const int ga = KIND == kMasked ? T.g : 0;
        const int gb = KIND == kDense ? 0 : T.g;
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          // a stage always has the same issuer, which walks its rounds in
          // order; the parity wait below is only unambiguous under that rule
          if ((it % STAGES) % kIssuers != me) continue;
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (static_cast<int>(it) == p.test_withhold_it) continue;  // test hook: this stage never fills
          mbar_arrive_expect_tx(full_bar(s), kStageTx);
          if constexpr (kSwap) {
            tma_load_3d(lane_tile(s), &tmB, full_bar(s), kb * 128, T.n0, gb);
            tma_load_3d(col_tile(s), &tmA, full_bar(s), kb * 128, T.m0, ga);
          } else {
            tma_load_3d(lane_tile(s), &tmA, full_bar(s), kb * 128, T.m0, ga);
            tma_load_3d(col_tile(s), &tmB, full_bar(s), kb * 128, T.n0, gb);
          }
          if constexpr (kSwap) tma_load_3d(sa_slice(s), &tmSA, full_bar(s), T.m0, kb, ga);
        }
      }
      // drain: every load this thread issued must land before the CTA exits
      // (the last STAGES iterations use distinct stages)
      const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
      for (uint32_t i = first; i < it; ++i)
        if ((i % STAGES) % kIssuers == me) drain_phase(full_bar(i % STAGES), (i / STAGES) & 1u);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const uint32_t me = static_cast<uint32_t>(warp - 1);
      uint32_t it = 0;
      bool ok = true;
      for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
        const Tile T = get_tile<kSwap, BNC, KIND, SPLIT>(p, t, rank, false);
        if (!T.valid) continue;
        // n-lanes: the MMA's N is the tile's rows of A; a masked tail tile
        // multiplies only its valid rows (rounded up to 16, the MMA's N step)
        const uint32_t n_mma = kSwap ? static_cast<uint32_t>(min(BNC, (T.mvalid + 15) / 16 * 16)) : BNC;
        const uint32_t kIdesc = idesc_e4m3_f32(128, n_mma);
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          // stage s and TMEM buffer it % kNBuf (both even counts) belong to
          // issuer s % 2 in every round
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
          const uint64_t adesc = sdesc_k128_sw128(lane_tile(s));
          const uint64_t bdesc = sdesc_k128_sw128(col_tile(s));
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 x K=32 bytes = one 128-wide K-block
            mma_f8f6f4(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                       kIdesc, k > 0 ? 1u : 0u);
          }
          mma_commit(empty_bar(s));
          mma_commit(tfull_bar(b));
        }
      }
      // drain: all MMAs this thread issued complete before TMEM is freed
      mma_commit(drain_bar(me));
      drain_phase(drain_bar(me), 0u);
    }
  }
  } else {
    // ------------------------------------------------------------ promotion + epilogue
    if constexpr (L::kRegSplit) setmaxnreg_inc<kPromoRegs>();
    constexpr int kCW = L::kCW;
    const int wg = (warp - 4) / 4;  // column half
    const int q = warp % 4;         // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;  // tile row = TMEM lane
    float acc[kCW];
    uint32_t it = 0;
    [[maybe_unused]] uint32_t store_it = 0;  // TMA-store epilogue: chunks stored by this warp
    bool ok = true;
    for (int t = t_first; ok && t < p.num_tiles; t += t_step) {
      // one thread records bad m_indices / masked_m entries in the error word
      const Tile T = get_tile<kSwap, BNC, KIND, SPLIT>(p, t, rank, warp == 4 && lane == 0);
      if (!T.valid) continue;
#pragma unroll
      for (int c = 0; c < kCW; ++c) acc[c] = 0.f;
      // column chunks of 32 that hold valid output (kSwap: columns are rows of A)
      const int live = kSwap ? min(kCW, max(0, T.mvalid - wg * kCW)) : kCW;
      // the sb row of this thread's columns (n-lanes: 32 K-blocks per
      // register, lane i holding K-block kb0 + 32j + i, the next 32 loaded
      // one chunk ahead and broadcast with a shuffle)
      const int nb = min((kSwap ? T.n0 : T.n0 + wg * kCW) / 128, p.NB - 1);
      const float* sbp = p.sb + (static_cast<long>(T.g) * p.NB + nb) * p.KB;
      // chunks of 32 columns, loaded two at a time (64 staging registers)
      constexpr int kChunks = kCW / 32;
      constexpr int kGroup = kChunks < 2 ? kChunks : 2;
      if constexpr (!kSwap) {
        // m-lanes: one scale per thread and K-block, sa[kb][m0 + row] *
        // sb[g][nb][kb], read from global memory two K-blocks ahead, so the
        // loop waits on nothing but the partial in TMEM
        const bool row_in = T.m0 + row < p.M;
        const float* sap = p.sa + (KIND == kMasked ? static_cast<long>(T.g) * p.KB * p.ld_sa : 0L) + T.m0 + row;
        auto sa_at = [&](int kb) { return row_in && kb < T.kb1 ? __ldg(sap + static_cast<long>(kb) * p.ld_sa) : 0.f; };
        auto sb_at = [&](int kb) { return kb < T.kb1 ? __ldg(sbp + kb) : 0.f; };
        float sa0 = sa_at(T.kb0), sa1 = sa_at(T.kb0 + 1);
        float sb0 = sb_at(T.kb0), sb1 = sb_at(T.kb0 + 1);
        for (int kb = T.kb0; ok && kb < T.kb1; kb += 2) {
          const float sc2[2] = {sa0 * sb0, sa1 * sb1};
          sa0 = sa_at(kb + 2);
          sa1 = sa_at(kb + 3);
          sb0 = sb_at(kb + 2);
          sb1 = sb_at(kb + 3);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (kb + u >= T.kb1) break;
            const int b = it % L::kNBuf;
            const uint32_t tph = (it / L::kNBuf) & 1u;
            if (!__all_sync(0xffffffffu, wait_phase(tfull_bar(b), tph, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                   static_cast<uint32_t>(b * BNC + wg * kCW);
#pragma unroll
            for (int j0 = 0; j0 < kChunks; j0 += kGroup) {
              uint32_t r[kGroup][32];
#pragma unroll
              for (int j = 0; j < kGroup; ++j) tmem_ld_32x32b_x32(taddr + 32 * (j0 + j), r[j]);
              tmem_ld_wait_bind(r[0]);
#pragma unroll
              for (int j = 1; j < kGroup; ++j) bind_after_wait(r[j]);
#pragma unroll
              for (int j = 0; j < kGroup; ++j) {
                float* a = acc + 32 * (j0 + j);
                if constexpr ((OPT & kOptFma2) != 0) {
#pragma unroll
                  for (int c = 0; c < 32; c += 2) ffma2(a[c], a[c + 1], r[j][c], r[j][c + 1], sc2[u]);
                } else {
#pragma unroll
                  for (int c = 0; c < 32; ++c) a[c] = fmaf(__uint_as_float(r[j][c]), sc2[u], a[c]);
                }
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(tempty_bar(b));
            ++it;
          }
        }
      } else {
        // n-lanes: the scale varies per column (sa slice of the stage) and
        // is uniform over the lanes for sb (broadcast from a register)
        float sb_cur = T.kb0 + lane < T.kb1 ? __ldg(sbp + T.kb0 + lane) : 0.f;
        float sb_nxt = T.kb0 + 32 + lane < T.kb1 ? __ldg(sbp + T.kb0 + 32 + lane) : 0.f;
        for (int kb = T.kb0; kb < T.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const int b = it % L::kNBuf;
          const uint32_t tph = (it / L::kNBuf) & 1u;
          const int i32 = (kb - T.kb0) & 31;
          if (i32 == 0 && kb != T.kb0) {
            sb_cur = sb_nxt;
            sb_nxt = kb + 32 + lane < T.kb1 ? __ldg(sbp + kb + 32 + lane) : 0.f;
          }
          const float s_b = __shfl_sync(0xffffffffu, sb_cur, i32);
          // the stage's sa slice is read below: wait for its TMA as well
          bool w = wait_phase(tfull_bar(b), tph, abort_flag);
          w = w && wait_phase(full_bar(s), ph, abort_flag);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                 static_cast<uint32_t>(b * BNC + wg * kCW);
#pragma unroll
          for (int j0 = 0; j0 < kChunks; j0 += kGroup) {
            if (32 * j0 >= live) break;
            uint32_t r[kGroup][32];
#pragma unroll
            for (int j = 0; j < kGroup; ++j)
              if (32 * (j0 + j) < live) tmem_ld_32x32b_x32(taddr + 32 * (j0 + j), r[j]);
            tmem_ld_wait_bind(r[0]);
#pragma unroll
            for (int j = 1; j < kGroup; ++j) bind_after_wait(r[j]);
#pragma unroll
            for (int j = 0; j < kGroup; ++j) {
              if (32 * (j0 + j) >= live) continue;
              float* a = acc + 32 * (j0 + j);
              // per column: sa[m0 + c, kb] * sb[nb, kb]
              const float4* f4 = reinterpret_cast<const float4*>(sa_f + s * L::kSaFloats + wg * kCW + 32 * (j0 + j));
#pragma unroll
              for (int c4 = 0; c4 < 8; ++c4) {
                const float4 f = f4[c4];
                a[4 * c4 + 0] = fmaf(__uint_as_float(r[j][4 * c4 + 0]), f.x * s_b, a[4 * c4 + 0]);
                a[4 * c4 + 1] = fmaf(__uint_as_float(r[j][4 * c4 + 1]), f.y * s_b, a[4 * c4 + 1]);
                a[4 * c4 + 2] = fmaf(__uint_as_float(r[j][4 * c4 + 2]), f.z * s_b, a[4 * c4 + 2]);
                a[4 * c4 + 3] = fmaf(__uint_as_float(r[j][4 * c4 + 3]), f.w * s_b, a[4 * c4 + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(tempty_bar(b));
            mbar_arrive(empty_bar(s));
          }
        }
      }
      if (!ok) break;

      const long drow0 = KIND == kMasked ? static_cast<long>(T.g) * p.M : 0;
      if constexpr (SPLIT < 0) {
        // partial sums to the workspace, column-major per tile slot so that a
        // warp's 32 rows of one column are 128 contiguous bytes
        float* slot = p.ws + (static_cast<long>(t) * p.gsplit + rank) * (BNC * 128);
#pragma unroll
        for (int c = 0; c < kCW; ++c) slot[(wg * kCW + c) * 128 + row] = acc[c];
      } else if constexpr (SPLIT > 1) {
        // store this CTA's partial columns into the shared memory of the CTA
        // that reduces them (slot = this CTA's rank); the reduction follows
        // the cluster barrier after the role loops
        constexpr int kCPD = L::kCPD;
        const uint32_t recv_local = sbase + L::kOffRecv + (rank * 128u + row) * (kCPD * 4u);
#pragma unroll
        for (int d0 = 0; d0 < kCW; d0 += kCPD) {
          const uint32_t dst = static_cast<uint32_t>((wg * kCW + d0) / kCPD);
          const uint32_t raddr = mapa(recv_local, dst);
#pragma unroll
          for (int c = 0; c < kCPD; c += 4)
            st_cluster_v4(raddr + 4u * c, acc[d0 + c], acc[d0 + c + 1], acc[d0 + c + 2], acc[d0 + c + 3]);
        }
      } else if constexpr (kSwap) {
        // lanes hold consecutive n: each column store is 64 contiguous bytes per warp
        const int n = T.n0 + row;
        if (n < p.N) {
          uint16_t* dcol = p.D + (drow0 + T.m0 + wg * kCW) * p.N + n;
#pragma unroll
          for (int c = 0; c < kCW; ++c)
            if (c < live) dcol[static_cast<long>(c) * p.N] = static_cast<uint16_t>(pack_bf16x2(acc[c], 0.f) & 0xFFFFu);
        }
      } else if constexpr (kTmaStore) {
        // a warp's 32 rows x 32 columns at a time through shared memory, for
        // the chunks inside D (warp-uniform): every buffer write is followed
        // by a store, so waiting until at most one store group is pending
        // (the other buffer's) frees the buffer about to be written
        const CUtensorMap* tmD = &tmSA;
        const uint32_t stage0 = sbase + L::kOffStore + static_cast<uint32_t>((warp - 4) * 2 * L::kStoreChunk);
#pragma unroll
        for (int c0 = 0; c0 < kCW; c0 += 32) {
          const int n = T.n0 + wg * kCW + c0;
          if (n >= p.N) continue;
          const uint32_t buf = stage0 + (store_it & 1u) * L::kStoreChunk;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 v;
            v.x = pack_bf16x2(acc[c0 + 8 * j + 0], acc[c0 + 8 * j + 1]);
            v.y = pack_bf16x2(acc[c0 + 8 * j + 2], acc[c0 + 8 * j + 3]);
            v.z = pack_bf16x2(acc[c0 + 8 * j + 4], acc[c0 + 8 * j + 5]);
            v.w = pack_bf16x2(acc[c0 + 8 * j + 6], acc[c0 + 8 * j + 7]);
            st_shared_v4(buf + static_cast<uint32_t>(lane * 64 + j * 16), v);
          }
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(tmD, buf, n, T.m0 + 32 * q, 0);
            bulk_commit_group();
          }
          ++store_it;
        }
      } else {
        // a thread holds kCW consecutive columns of its row: 16-byte stores
        if (row < T.mvalid) {
          uint16_t* drow = p.D + (drow0 + T.m0 + row) * p.N + T.n0 + wg * kCW;
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
    if constexpr (kTmaStore) {
      // every store of this warp has finished (its shared memory may go)
      if (lane == 0) bulk_wait_group<0>();
      __syncwarp();
    }
  }

  __syncwarp();
  if constexpr (SPLIT == kGlobalSplit) {
    if (warp >= 4) global_split_reduce<BNC, KIND>(p, t_first, rank, abort_flag);
  }

  if constexpr (SPLIT > 1) {
    // all partials of this cluster's tile are in place after the barrier;
    // the warpgroup whose columns this CTA owns adds them in rank order
    cluster_sync_all();
    constexpr int kCPD = L::kCPD;
    const int wg = (warp - 4) / 4;
    if (warp >= 4 && !*abort_flag && wg == static_cast<int>((rank * kCPD) / L::kCW)) {
      const Tile T = get_tile<kSwap, BNC, KIND, SPLIT>(p, t_first, rank, false);
      const int row = 32 * (warp % 4) + lane;
      float sum[kCPD];
#pragma unroll
      for (int c = 0; c < kCPD; ++c) sum[c] = 0.f;
      const float* rv = reinterpret_cast<const float*>(smem + L::kOffRecv);
      for (int src = 0; src < SPLIT; ++src) {
        const float4* v = reinterpret_cast<const float4*>(rv + (src * 128 + row) * kCPD);
#pragma unroll
        for (int c4 = 0; c4 < kCPD / 4; ++c4) {
          const float4 f = v[c4];
          sum[4 * c4 + 0] += f.x;
          sum[4 * c4 + 1] += f.y;
          sum[4 * c4 + 2] += f.z;
          sum[4 * c4 + 3] += f.w;
        }
      }
      const int n = T.n0 + row;
      if (T.valid && n < p.N) {
#pragma unroll
        for (int c = 0; c < kCPD; ++c) {
          const int mc = static_cast<int>(rank) * kCPD + c;
          if (mc < T.mvalid)
            p.D[static_cast<long>(T.m0 + mc) * p.N + n] = static_cast<uint16_t>(pack_bf16x2(sum[c], 0.f) & 0xFFFFu);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// Second kernel of the two-kernel split-K: D[m0 + c, n0 + r] = bf16(sum over
// ranks, in rank order, of the partials ws[tile][rank][c][r]).  Launched after
// the GEMM kernel on the same stream (programmatic dependent launch: it waits
// for the GEMM kernel's partials, and lets the next kernel start its
// prologue early).  One thread per output element, grid-stride.
template <int BNC>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const Params p) {
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const long total = static_cast<long>(p.num_tiles) * BNC * 128;
  const long stride = static_cast<long>(gridDim.x) * blockDim.x;
  for (long e = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int tile = static_cast<int>(e / (BNC * 128));
    const int c = static_cast<int>((e / 128) % BNC);
    const int r = static_cast<int>(e % 128);
    const int m = (tile / p.n_tiles) * BNC + c;
    const int n = (tile % p.n_tiles) * 128 + r;
    if (m >= p.M || n >= p.N) continue;
    const float* src = p.ws + static_cast<long>(tile) * p.gsplit * (BNC * 128) + c * 128 + r;
    float v[kMaxGSplit];
#pragma unroll
    for (int i = 0; i < kMaxGSplit; ++i) v[i] = i < p.gsplit ? __ldcg(src + static_cast<long>(i) * (BNC * 128)) : 0.f;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxGSplit; ++i) sum += v[i];
    p.D[static_cast<long>(m) * p.N + n] = static_cast<uint16_t>(pack_bf16x2(sum, 0.f) & 0xFFFFu);
  }
}

}  // namespace fp8g
