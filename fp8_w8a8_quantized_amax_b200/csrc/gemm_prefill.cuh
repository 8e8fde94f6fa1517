// gemm_prefill.cuh -- persistent, warp-specialised tcgen05 FP8 GEMM for M > 64.
//
//   Y[m, n] = bf16( sum_k E4M3(Xq[m,k]) E4M3(Wq[n,k]) * x_scale[m] * w_scale[n] )   (channel mode)
//   Y[m, n] = bf16( sum_kb x_scale[m,kb] w_scale[n/128,kb] sum_{k in kb} ... )        (block mode)
//
// Roles inside one CTA (one CTA per SM, tiles handed out round-robin):
//   warp 0      TMA producer: Xq and Wq tiles of 128 K-bytes into a ring of
//               shared-memory stages (128-byte swizzle), one mbarrier per stage.
//   warp 1      allocates tensor memory, then one thread issues tcgen05.mma
//               (E4M3 x E4M3 -> fp32 in TMEM) and tcgen05.commit to release
//               stages and to publish finished accumulators.
//   warps 2..   epilogue: tcgen05.ld the fp32 accumulator, apply the scales,
//               round to bf16 (RNE) and store.  Channel mode stages each
//               32 x 32 output chunk in shared memory (64-byte swizzle,
//               double-buffered per warp) and writes it with a TMA store.
// Channel mode: tile 128 x 256, two TMEM accumulators of 256 columns, so the
// epilogue of one tile overlaps the main loop of the next.
// Block mode: tile 128 x 128 (one weight block wide).  Every 128-wide K slice
// is accumulated into its own TMEM slot (4 slots of 128 columns); 8 epilogue
// warps fold each slot into fp32 registers with that slice's scale product.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "sched.cuh"

namespace fp8q {
namespace prefill {

constexpr int BM = 128;       // rows of X per tile (UMMA M)
constexpr int BK = 128;       // K bytes per stage: one 128-byte swizzle row
constexpr int UMMA_K = 32;    // K of one tcgen05.mma for 8-bit operands

struct Params {
  const float* xs;
  const float* ws;
  __nv_bfloat16* y;
  int M, N, K;
  int64_t ldy;
  int KB;          // ceil(K / 128)
  int num_m, num_n, num_tiles, group_m;
  // Channel kernel work list: tiles [0, full) are whole (tile t goes to CTA
  // t % gridDim.x); the remaining tiles are cut along N into `split` pieces
  // (256 / split columns each) handed out round-robin after them.
  int full, split;
};

// Tile order: groups of `group_m` row-blocks, column-blocks within a group,
// so that the tiles in flight at one time share operands in L2.
__host__ __device__ __forceinline__ void tile_coords(const Params& p, int t, int& mb, int& nb) {
  const int per_group = p.group_m * p.num_n;
  const int g = t / per_group;
  const int first_m = g * p.group_m;
  const int gm = min(p.group_m, p.num_m - first_m);
  const int r = t - g * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Work list of G persistent workers (CTAs or CTA pairs): tiles [0, full)
// whole, tile t to worker t % G; then the remaining tiles cut along N into
// `split` pieces, handed out round-robin.  work_items: the number of items of
// worker c.  work_item: item i of worker c -- tile coordinates, the first
// column inside the tile (`tile_cols` wide) and the column count.
__host__ __device__ __forceinline__ int work_items(const Params& p, int c, int G) {
  const int tail = (p.num_tiles - p.full) * p.split;
  return p.full / G + (c < tail ? (tail - 1 - c) / G + 1 : 0);
}

__host__ __device__ __forceinline__ void work_item(const Params& p, int c, int G, int i, int tile_cols, int& mb,
                                                   int& nb, int& off, int& cols) {
  const int nfull = p.full / G;
  if (i < nfull) {
    tile_coords(p, c + i * G, mb, nb);
    off = 0;
    cols = tile_cols;
  } else {
    const int j = c + (i - nfull) * G;
    tile_coords(p, p.full + j / p.split, mb, nb);
    cols = tile_cols / p.split;
    off = (j % p.split) * cols;
  }
}

// Whole rounds of `per_round` tiles stay whole; the partial last round is cut
// along N into two halves when that shortens it.  Returns the split (1 or 2)
// and the number of whole tiles.
inline void tail_split(int num_tiles, int per_round, int* full, int* split) {
  *full = num_tiles >= per_round ? num_tiles / per_round * per_round : 0;
  const int rest = num_tiles - *full;
  *split = 1;
  if (rest) {
    const double whole = 1.0 * ((rest + per_round - 1) / per_round);
    const double halves = 0.5 * ((2 * rest + per_round - 1) / per_round);
    if (halves < whole - 1e-9) *split = 2;
  }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

template <int BN, int STAGES>
struct ChannelLayout {
  static constexpr int kA = BM * BK;
  static constexpr int kB = BN * BK;
  static constexpr int kOutChunk = 32 * 32 * 2;                  // 32 rows x 32 bf16 columns
  static constexpr int kOutOff = STAGES * (kA + kB);             // 4 warps x 2 staging buffers
  static constexpr int kWsOff = kOutOff + 4 * 2 * kOutChunk;     // 4 warps x BN w_scale values
  static constexpr int kBarOff = kWsOff + 4 * BN * 4;
  static constexpr int kBarBytes = (2 * STAGES + 4) * 8 + 8;    // mbarriers, TMEM address, abort flag
  static constexpr int kBytes = kBarOff + 1024 + 1024;           // + barrier area + alignment slack
  static_assert(kBarBytes <= 1024, "barrier area");
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// ------------------------------------------------------------- channel ---
template <int BN, int STAGES>
__global__ void __launch_bounds__(192, 1)
    gemm_channel_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB128, const __grid_constant__ CUtensorMap tmB64,
                        const __grid_constant__ CUtensorMap tmY, const Params p) {
  static_assert(BN == 256, "the work list assumes 256-column tiles");
  using L = ChannelLayout<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = 2 * BN;   // 512

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);                  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB128);
    tma_prefetch_desc(&tmB64);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();   // global memory only from here on

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const int nitems = work_items(p, blockIdx.x, gridDim.x);
      for (int i = 0; ok && i < nitems; ++i) {
        int mb, nb, n_off, n_cols;
        work_item(p, blockIdx.x, gridDim.x, i, 256, mb, nb, n_off, n_cols);
        const CUtensorMap* tb = n_cols == 256 ? &tmB : (n_cols == 128 ? &tmB128 : &tmB64);
        const uint32_t bytes = static_cast<uint32_t>(L::kA + n_cols * BK);
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(sA + stage * L::kA, &tmA, &full[stage], kb * BK, mb * BM, pol);
          tma_load_2d(sB + stage * L::kB, tb, &full[stage], kb * BK, nb * BN + n_off, pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      griddep_launch_dependents();
      // Tail: wait until the MMA has released every stage, so that no
      // tcgen05.commit arrival is still in flight when the CTA exits.
      for (int i = 0; ok && i < STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) break;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const int nitems = work_items(p, blockIdx.x, gridDim.x);
      for (int it = 0; ok && it < nitems; ++it) {
        int mb, nb, n_off, n_cols;
        work_item(p, blockIdx.x, gridDim.x, it, 256, mb, nb, n_off, n_cols);
        const uint32_t idesc = idesc_e4m3_f32(BM, n_cols);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, kErrWaitTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kA);
          const uint32_t b0 = smem_u32(sB + stage * L::kB);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            mma_e4m3(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc,
                     (kb | k) != 0);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit(&tfull[acc]);
      }
    }
  } else {
    // Epilogue: warp w may read TMEM lanes 32*(w%4) .. +31, i.e. tile rows
    // 32*(w%4) .. +31; each thread owns one row.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float* ws_s = reinterpret_cast<float*>(smem + L::kWsOff) + ew * BN;
    uint8_t* out_s = smem + L::kOutOff + ew * 2 * L::kOutChunk;
    const int swz = (lane >> 1) & 3;         // 64-byte swizzle of this thread's staging row
    int buf = 0;
    const int nitems = work_items(p, blockIdx.x, gridDim.x);
    for (int it = 0; it < nitems; ++it) {
      int mb, nb, n_off, n_cols;
      work_item(p, blockIdx.x, gridDim.x, it, 256, mb, nb, n_off, n_cols);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // Scales of this tile, fetched while the main loop still runs.
      const int m = mb * BM + quarter * 32 + lane;
      const float xsm = m < p.M ? __ldg(p.xs + m) : 0.0f;
      float wv[BN / 32];
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        const int n = nb * BN + n_off + i * 32 + lane;
        wv[i] = (i * 32 < n_cols && n < p.N) ? __ldg(p.ws + n) : 0.0f;
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrWaitTmemFull))) break;
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) ws_s[i * 32 + lane] = wv[i];
      __syncwarp();
#pragma unroll 1
      for (int c = 0; c < n_cols; c += 32) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + lane_addr + acc * BN + c, r);
        tmem_ld_wait();
        if (c + 32 == n_cols) {          // accumulator fully read: hand it back to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_relaxed(&tempty[acc]);
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 w = *reinterpret_cast<const float2*>(ws_s + c + 2 * j);
          pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * xsm * w.x, __uint_as_float(r[2 * j + 1]) * xsm * w.y);
        }
        // The staging buffer written two chunks ago must have been read by its store.
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        uint8_t* sb = out_s + buf * L::kOutChunk;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(sb + lane * 64 + ((q ^ swz) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        const int row0 = mb * BM + quarter * 32, col0 = nb * BN + n_off + c;
        if (lane == 0 && row0 < p.M && col0 < p.N) {   // the store clips the rest of the box
          tma_store_2d(&tmY, sb, col0, row0);
          bulk_commit();
        }
        buf ^= 1;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------ channel, CTA pair ---
// The same GEMM with 256 x 256 tiles computed by a cluster of two CTAs with
// tcgen05 pair instructions.  CTA r of the pair loads rows [128 r, 128 r + 128)
// of the A tile and of the B tile (B's N split the same way) into its own
// shared memory; the leader (r = 0) issues one M=256 MMA over both; each CTA's
// tensor memory receives its own 128 rows of the accumulator.  Per CTA this
// moves 32 KB per 128-wide K block instead of 48 KB for the same 128 x 256
// share of the work, and 6 stages fit.
//   full[s]    leader only: the leader's producer expects both CTAs' bytes;
//              both CTAs' TMA loads complete on it.
//   empty[s]   both CTAs: the leader's commit arrives on both.
//   tfull[a]   both CTAs: the leader's commit arrives on both.
//   tempty[a]  leader only: lane 0 of each of the pair's 16 epilogue warps arrives.
template <int STAGES, int NACC = 2>
struct PairLayout {
  static constexpr int kA = 128 * BK;                           // this CTA's 128 rows of A
  static constexpr int kB = 128 * BK;                           // this CTA's (up to) 128 rows of B
  static constexpr int kEpiWarps = 8;                           // two per TMEM lane quarter
  static constexpr int kOutChunk = 32 * 32 * 2;
  static constexpr int kOutOff = STAGES * (kA + kB);           // 2 staging tiles per epilogue warp
  static constexpr int kBarOff = kOutOff + kEpiWarps * 2 * kOutChunk;
  static constexpr int kBarBytes = (2 * STAGES + 2 * NACC) * 8 + 8;   // + TMEM address, abort flag
  static constexpr int kBytes = kBarOff + 256 + 1024;           // + barrier area + alignment slack
  static_assert(kBarBytes <= 256, "barrier area");
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

// Stream-K schedule (SK = true), for problems whose 256 x 256 tiles fill the
// pairs unevenly (a few tiles more than a whole number of rounds): the
// (tile, K block) steps are cut into equal contiguous ranges, one per pair
// (sched.cuh), as the decode kernel does.  A tile cut between pairs is
// accumulated by each in its own segment; every epilogue warp stores its
// 32 x 128 fp32 share of a partial segment to a workspace slot, counts itself
// in on a per-(tile, CTA, warp) counter, and the warp that arrives last adds
// the tile's slots in pair order (deterministic), applies the scales and
// writes bf16 through the usual staging path, and sets the counter back to 0.
// A pair's partial segments can only lie in the first or the last tile of its
// range: slot 2c holds pair c's share of its first tile, slot 2c + 1 of its
// last.  Nothing waits on another pair.
struct SkParams {
  unsigned int* count;  // [num_tiles][2 CTAs][8 warps] arrival counters, left zero
  float* part;          // [2 * pairs][2 CTAs][8 warps][128 columns][32 rows] fp32 partial tiles
};

constexpr int kSkSlotFloats = 256 * 256;

template <int STAGES, bool SK = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    gemm_channel2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmB64, const __grid_constant__ CUtensorMap tmY,
                         const Params p, const SkParams sk) {
  using L = PairLayout<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  constexpr uint32_t kTmemCols = 512;                           // 2 accumulators x 256 columns
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * L::kEpiWarps);                  // every epilogue warp of the pair
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB64);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                 // barriers of both CTAs initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();                 // global memory only from here on

  // Work items are per pair: use the pair index and the number of pairs.
  const int G2 = gridDim.x >> 1;
  auto coords = [&](int i, int& mb, int& nb, int& n_off, int& n_cols) {
    work_item(p, pair, G2, i, 256, mb, nb, n_off, n_cols);
  };
  const int nitems = SK ? 0 : work_items(p, pair, G2);
  // Stream-K: this pair's steps [ub, ue) of the num_tiles * KB list.
  const sched::Split sp = sched::split_of(SK ? p.num_tiles * p.KB : G2, G2);
  const int ub = SK ? sched::range_begin(pair, sp) : 0;
  const int ue = SK ? sched::range_begin(pair + 1, sp) : 0;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto load = [&](int mb, int nb, int n_off, int half, int kb) -> bool {
        const CUtensorMap* tb = half == 128 ? &tmB : &tmB64;
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) return false;
        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2u * static_cast<uint32_t>(L::kA + half * BK));
        const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
        tma_load_2d_pair(sA + stage * L::kA, &tmA, bar0, kb * BK, mb * 256 + static_cast<int>(rank) * 128, pol);
        tma_load_2d_pair(sB + stage * L::kB, tb, bar0, kb * BK, nb * 256 + n_off + static_cast<int>(rank) * half,
                         pol);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        return true;
      };
      if constexpr (SK) {
        for (sched::StepIter it(ub, ue, p.KB); ok && it.valid(); it.next()) {
          int mb, nb;
          tile_coords(p, it.t, mb, nb);
          ok = load(mb, nb, 0, 128, it.kb);
        }
      } else {
        for (int i = 0; ok && i < nitems; ++i) {
          int mb, nb, n_off, n_cols;
          coords(i, mb, nb, n_off, n_cols);
          for (int kb = 0; ok && kb < p.KB; ++kb) ok = load(mb, nb, n_off, n_cols / 2, kb);
        }
      }
      griddep_launch_dependents();
      for (int i = 0; ok && i < STAGES; ++i) {   // every stage released by the leader's commits
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) break;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // one K block into accumulator d (accumulate unless it is the first of the segment)
      auto mma_step = [&](uint32_t d, uint32_t idesc, bool first) -> bool {
        if (!mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) return false;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + stage * L::kA);
        const uint32_t b0 = smem_u32(sB + stage * L::kB);
#pragma unroll
        for (int k = 0; k < BK / UMMA_K; ++k)
          mma_e4m3_pair(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc,
                        (!first || k != 0) ? 1u : 0u);
        mma_commit_pair(&empty[stage], kBoth);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        return true;
      };
      if constexpr (SK) {
        constexpr uint32_t idesc = idesc_e4m3_f32(256, 256);
        int seg = 0;
        for (sched::StepIter it(ub, ue, p.KB); it.valid(); it.next()) {
          const int acc = seg & 1;
          if (it.seg_first()) {
            if (!mbar_wait_cluster(&tempty[acc], ((seg >> 1) & 1) ^ 1u, abort_flag, kErrWaitTmemEmpty)) break;
            tc_fence_after();
          }
          if (!mma_step(tmem_base + acc * 256, idesc, it.seg_first())) break;
          if (it.seg_last()) {
            mma_commit_pair(&tfull[acc], kBoth);
            ++seg;
          }
        }
      } else {
        for (int it = 0; ok && it < nitems; ++it) {
          int mb, nb, n_off, n_cols;
          coords(it, mb, nb, n_off, n_cols);
          const uint32_t idesc = idesc_e4m3_f32(256, n_cols);
          const int acc = it & 1;
          const uint32_t acc_phase = (it >> 1) & 1;
          if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag, kErrWaitTmemEmpty)) break;
          tc_fence_after();
          const uint32_t d = tmem_base + acc * 256;
          for (int kb = 0; ok && kb < p.KB; ++kb) ok = mma_step(d, idesc, kb == 0);
          if (ok) mma_commit_pair(&tfull[acc], kBoth);
        }
      }
    }
  } else {
    // 8 epilogue warps: warp w reads TMEM lanes 32*(w%4)..+31 (its 32 rows)
    // and takes one half of the item's columns (4 or 2 chunks of 32).  The
    // TMEM load of the next chunk is issued before the current one is scaled,
    // staged and stored, so its latency overlaps that work.  w_scale of the
    // chunk's columns is held one value per lane and broadcast by shuffles.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* out_s = smem + L::kOutOff + ew * 2 * L::kOutChunk;
    const int swz = (lane >> 1) & 3;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int buf = 0;
    // One output segment: tile (mb, nb), columns [n_off, n_off + n_cols), in
    // accumulator `acc`.  This warp takes rows row0.. of its lane quarter and
    // half of the columns.
    float xsm = 0.0f, wv[4];
    int row0 = 0, col_base = 0;
    auto setup = [&](int mb, int nb, int n_off, int n_cols) {
      const int my_cols = n_cols / 2;                           // 128 or 64
      const int c_begin = half * my_cols;
      row0 = mb * 256 + static_cast<int>(rank) * 128 + quarter * 32;
      const int m = row0 + lane;
      xsm = m < p.M ? __ldg(p.xs + m) : 0.0f;
      col_base = nb * 256 + n_off + c_begin;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = col_base + i * 32 + lane;
        wv[i] = (i < my_cols / 32 && n < p.N) ? __ldg(p.ws + n) : 0.0f;
      }
      return c_begin;
    };
    // Scale, stage and store one 32-column chunk held in registers.
    auto emit = [&](const uint32_t (&cur)[32], float w_lane, int c) {
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float w0 = __shfl_sync(0xFFFFFFFFu, w_lane, 2 * j);
        const float w1 = __shfl_sync(0xFFFFFFFFu, w_lane, 2 * j + 1);
        pk[j] = pack_bf16x2(__uint_as_float(cur[2 * j]) * xsm * w0, __uint_as_float(cur[2 * j + 1]) * xsm * w1);
      }
      if (lane == 0) bulk_wait_read<1>();   // the tile written two chunks ago has been read
      __syncwarp();
      uint8_t* sb = out_s + buf * L::kOutChunk;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(sb + lane * 64 + ((q ^ swz) << 4)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      const int col0 = col_base + c;
      if (lane == 0 && row0 < p.M && col0 < p.N) {
        tma_store_2d(&tmY, sb, col0, row0);
        bulk_commit();
      }
      buf ^= 1;
    };
    // The whole segment from TMEM: the load of the next chunk is issued before
    // the current one is scaled, staged and stored, so its latency overlaps
    // that work; the accumulator is released once all chunks are in registers.
    auto emit_from_tmem = [&](uint32_t tcol, int nchunks, int acc) {
      uint32_t ra[32], rb[32];
      __syncwarp();
      tmem_ld_32x32b_x32(tcol, ra);
#pragma unroll
      for (int ci = 0; ci < 4; ci += 2) {
        if (ci < nchunks) {
          tmem_ld_wait_regs(ra);
          __syncwarp();
          tmem_ld_32x32b_x32(tcol + (ci + 1) * 32, rb);
          emit(ra, wv[ci], ci * 32);
          tmem_ld_wait_regs(rb);
          if (ci + 2 < nchunks) {
            __syncwarp();
            tmem_ld_32x32b_x32(tcol + (ci + 2) * 32, ra);
          } else {                      // all of this warp's columns read: release the accumulator
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + acc * 8);
          }
          emit(rb, wv[ci + 1], (ci + 1) * 32);
        }
      }
    };
    if constexpr (SK) {
      int seg = 0, seg_len = 0;
      for (sched::StepIter st(ub, ue, p.KB); st.valid(); st.next()) {
        seg_len = st.seg_first() ? 1 : seg_len + 1;
        if (!st.seg_last()) continue;
        const int t = st.t;
        int mb, nb;
        tile_coords(p, t, mb, nb);
        const int acc = seg & 1;
        const uint32_t acc_phase = (seg >> 1) & 1;
        ++seg;
        const int c_begin = setup(mb, nb, 0, 256);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrWaitTmemFull))) break;
        tc_fence_after();
        const uint32_t tcol = tmem_base + lane_addr + acc * 256 + c_begin;
        if (seg_len == p.KB) {          // the whole tile in this pair
          emit_from_tmem(tcol, 4, acc);
          continue;
        }
        // A part of the tile: this warp's 32 x 128 fp32 share to the pair's
        // slot (column-major in 32-row strips: each store is 128 contiguous
        // bytes), then count in.
        auto share = [&](int c) -> int64_t {
          const int slot = (sched::range_begin(c, sp) / p.KB == t) ? 2 * c : 2 * c + 1;
          return (static_cast<int64_t>(slot) * 16 + static_cast<int>(rank) * 8 + ew) * (128 * 32) + lane;
        };
        float* dst = sk.part + share(pair);
        uint32_t ra[32];
#pragma unroll 1
        for (int ci = 0; ci < 4; ++ci) {
          __syncwarp();
          tmem_ld_32x32b_x32(tcol + ci * 32, ra);
          tmem_ld_wait_regs(ra);
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(ci * 32 + j) * 32] = __uint_as_float(ra[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + acc * 8);
        __threadfence();
        __syncwarp();
        const int c0 = sched::cta_of_step(t * p.KB, sp);
        const int c1 = sched::cta_of_step(t * p.KB + p.KB - 1, sp);
        unsigned int* cnt = sk.count + (static_cast<int64_t>(t) * 2 + rank) * 8 + ew;
        unsigned int prev = 0;
        if (lane == 0) prev = atomicAdd(cnt, 1u);
        prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
        if (prev != static_cast<unsigned int>(c1 - c0)) continue;
        // Every other part is in: sum the shares in pair order, then scale and store.
        __threadfence();
#pragma unroll 1
        for (int ci = 0; ci < 4; ++ci) {
          float sum[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) sum[j] = 0.0f;
          for (int cc = c0; cc <= c1; ++cc) {
            const float* src = sk.part + share(cc) + ci * 32 * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) sum[j] += __ldcg(src + j * 32);
          }
          uint32_t bits[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) bits[j] = __float_as_uint(sum[j]);
          emit(bits, wv[ci], ci * 32);
        }
        if (lane == 0) *cnt = 0u;
      }
    } else {
      for (int it = 0; it < nitems; ++it) {
        int mb, nb, n_off, n_cols;
        coords(it, mb, nb, n_off, n_cols);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        const int c_begin = setup(mb, nb, n_off, n_cols);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrWaitTmemFull))) break;
        tc_fence_after();
        emit_from_tmem(tmem_base + lane_addr + acc * 256 + c_begin, n_cols / 64, acc);
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();                 // no CTA leaves while its pair may still signal it or read its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// --------------------------------------------- gate/up with SiLU*up, pair ---
// The Llama MLP's gate and up projections share their input and are combined
// as silu(gate) * up.  Here one CTA pair computes, for 256 tokens and 128
// output channels, both linears in one M=256, N=256 MMA per K step: the
// leader loads the 128 gate rows and its peer the same 128 up rows as their B
// halves, so TMEM columns [0, 128) hold gate and [128, 256) hold up for the
// same channels.  The epilogue scales both (x_scale * w_scale, channel mode),
// rounds them to bf16 as the separate linears would, and writes only
//   act = bf16( bf16(silu(gate)) * up ),
// half the output of the two linears and no separate SiLU * up pass.  Tail
// items of 64 channels use N=128 MMAs.  Schedule, barriers and pipeline are
// those of gemm_channel2_kernel.
template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    gemm_swiglu2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmG64, const __grid_constant__ CUtensorMap tmU,
                        const __grid_constant__ CUtensorMap tmU64, const __grid_constant__ CUtensorMap tmY,
                        const Params p, const float* __restrict__ ws_up) {
  using L = PairLayout<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * L::kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(rank == 0 ? &tmG : &tmU);
    tma_prefetch_desc(rank == 0 ? &tmG64 : &tmU64);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();

  const int G2 = gridDim.x >> 1;
  // Item i: tile (mb, nb) of 256 tokens x 128 channels, channel offset c_off
  // inside it and its channel count (128, or 64 for a tail half).
  auto coords = [&](int i, int& mb, int& nb, int& c_off, int& n_ch) {
    work_item(p, pair, G2, i, 128, mb, nb, c_off, n_ch);
  };
  const int nitems = work_items(p, pair, G2);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; ok && i < nitems; ++i) {
        int mb, nb, c_off, n_ch;
        coords(i, mb, nb, c_off, n_ch);
        // B rows of this CTA: gate (leader) or up (peer), the item's channels
        const CUtensorMap* tb = rank == 0 ? (n_ch == 128 ? &tmG : &tmG64) : (n_ch == 128 ? &tmU : &tmU64);
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2u * static_cast<uint32_t>(L::kA + n_ch * BK));
          const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_2d_pair(sA + stage * L::kA, &tmA, bar0, kb * BK, mb * 256 + static_cast<int>(rank) * 128, pol);
          tma_load_2d_pair(sB + stage * L::kB, tb, bar0, kb * BK, nb * 128 + c_off, pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      griddep_launch_dependents();
      for (int i = 0; ok && i < STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) break;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok && it < nitems; ++it) {
        int mb, nb, c_off, n_ch;
        coords(it, mb, nb, c_off, n_ch);
        const uint32_t idesc = idesc_e4m3_f32(256, 2 * n_ch);   // gate and up columns
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, abort_flag, kErrWaitTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * 256;
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kA);
          const uint32_t b0 = smem_u32(sB + stage * L::kB);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            mma_e4m3_pair(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc,
                          (kb | k) != 0);
          mma_commit_pair(&empty[stage], kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit_pair(&tfull[acc], kBoth);
      }
    }
  } else {
    // 8 epilogue warps: warp w reads TMEM lanes 32*(w%4)..+31 (its 32 rows)
    // and half of the item's channels, h = (w - 2) / 4: gate
    // columns [h wc, +wc) and the matching up columns [n_ch + h wc, +wc),
    // wc = n_ch / 2, in chunks of 32.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int h = ew >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* out_s = smem + L::kOutOff + ew * 2 * L::kOutChunk;
    const int swz = (lane >> 1) & 3;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const int N = p.N;                                       // output channels (intermediate size)
    int buf = 0;
    for (int it = 0; it < nitems; ++it) {
      int mb, nb, c_off, n_ch;
      coords(it, mb, nb, c_off, n_ch);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int wc = n_ch / 2;                               // this warp's channels: 64 or 32
      const int nchunks = wc / 32;
      const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quarter * 32;
      const int m = row0 + lane;
      const float xsm = m < p.M ? __ldg(p.xs + m) : 0.0f;
      const int ch0 = nb * 128 + c_off + h * wc;             // first output channel of this warp
      float wg[2], wu[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int n = ch0 + i * 32 + lane;
        const bool live = i < nchunks && n < N;
        wg[i] = live ? __ldg(p.ws + n) : 0.0f;
        wu[i] = live ? __ldg(ws_up + n) : 0.0f;
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[acc], acc_phase, abort_flag, kErrWaitTmemFull))) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + lane_addr + acc * 256;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c < nchunks) {
          uint32_t rg[32], ru[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tbase + h * wc + c * 32, rg);
          tmem_ld_32x32b_x32(tbase + n_ch + h * wc + c * 32, ru);
          tmem_ld_wait_regs(rg);
          tmem_ld_wait_regs(ru);
          if (c + 1 == nchunks) {                           // all of this warp's columns read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + acc * 8);
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float a[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = 2 * j + e;
              const float gsc = __shfl_sync(0xFFFFFFFFu, wg[c], col);
              const float usc = __shfl_sync(0xFFFFFFFFu, wu[c], col);
              // the two linears' bf16 outputs
              const float g = __bfloat162float(__float2bfloat16_rn(__uint_as_float(rg[col]) * xsm * gsc));
              const float u = __bfloat162float(__float2bfloat16_rn(__uint_as_float(ru[col]) * xsm * usc));
              const float sl = __bfloat162float(__float2bfloat16_rn(g / (1.0f + __expf(-g))));
              a[e] = sl * u;                                 // exact in fp32; rounded once below
            }
            pk[j] = pack_bf16x2(a[0], a[1]);
          }
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          uint8_t* sb = out_s + buf * L::kOutChunk;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(sb + lane * 64 + ((q ^ swz) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          const int col0 = ch0 + c * 32;
          if (lane == 0 && row0 < p.M && col0 < N) {
            tma_store_2d(&tmY, sb, col0, row0);
            bulk_commit();
          }
          buf ^= 1;
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------- block, CTA pair ---
// Block-scaled GEMM on 256 x 256 tiles computed by a CTA pair, with the same
// operand split as the channel pair kernel (32 KB per CTA per 128-wide K
// block) and the same M=256, N=256 MMAs.  The scale x_scale[m, kb] *
// w_scale[n / 128, kb] changes with every K block, so each K block's MMAs
// write a fresh partial product into one of two 256-column TMEM slots, which
// the epilogue folds into fp32 registers and hands back; the MMAs of the next
// K block run meanwhile in the other slot.  Accumulator columns [0, 128) are
// the first weight block of the tile (the leader's B rows), [128, 256) the
// second (the peer's), so each epilogue warp meets one scale per K block.
//   tfull[s]   both CTAs: the leader's commit arrives on both.
//   tempty[s]  leader only: one arrival per epilogue warp of the pair (16),
//              by lane 0 once the whole warp has read the slot.
// A tail item of 128 columns (one weight block) uses N=128 MMAs over 64 B
// rows per CTA.
// Three warpgroups: warp 0 loads, warp 1 issues the MMAs (warps 2-3 idle),
// warpgroups 1 and 2 are the epilogue.  The epilogue keeps 128 fp32
// accumulators per thread, so registers are moved from the first warpgroup
// to the other two: 128 x kCtlRegs + 256 x kEpiRegs = 384 x kLaunchRegs.
constexpr int kBlock2Threads = 384;
constexpr int kBlock2LaunchRegs = 168;
constexpr int kBlock2CtlRegs = 56;
constexpr int kBlock2EpiRegs = 224;
static_assert(128 * kBlock2CtlRegs + 256 * kBlock2EpiRegs <= kBlock2Threads * kBlock2LaunchRegs, "register split");
static_assert(kBlock2CtlRegs + 2 * kBlock2EpiRegs <= 512, "registers of one SM sub-partition");
static_assert(kBlock2CtlRegs % 8 == 0 && kBlock2EpiRegs % 8 == 0, "setmaxnreg takes multiples of 8");

template <int STAGES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kBlock2Threads, 1)
    gemm_block2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmB64, const __grid_constant__ CUtensorMap tmY,
                       const Params p) {
  constexpr int kSlots = 2;
  using L = PairLayout<STAGES, kSlots>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + kSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  constexpr uint32_t kTmemCols = kSlots * 256;
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kSlots; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * L::kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmB64);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();

  const int G2 = gridDim.x >> 1;
  auto coords = [&](int i, int& mb, int& nb, int& n_off, int& n_cols) {
    work_item(p, pair, G2, i, 256, mb, nb, n_off, n_cols);
  };
  const int nitems = work_items(p, pair, G2);

  if (warp < 4) regs_shrink<kBlock2CtlRegs>();
  if (warp == 0) {
    // The whole warp runs the loop; one elected lane issues the copies.
    const uint64_t pol = policy_evict_last();
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int i = 0; ok && i < nitems; ++i) {
      int mb, nb, n_off, n_cols;
      coords(i, mb, nb, n_off, n_cols);
      const int half = n_cols / 2;
      const CUtensorMap* tb = half == 128 ? &tmB : &tmB64;
      for (int kb = 0; kb < p.KB; ++kb) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2u * static_cast<uint32_t>(L::kA + half * BK));
          const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_2d_pair(sA + stage * L::kA, &tmA, bar0, kb * BK, mb * 256 + static_cast<int>(rank) * 128, pol);
          tma_load_2d_pair(sB + stage * L::kB, tb, bar0, kb * BK, nb * 256 + n_off + static_cast<int>(rank) * half,
                           pol);
        }
        __syncwarp();
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (elect_one()) griddep_launch_dependents();
    __syncwarp();
    for (int i = 0; ok && i < STAGES; ++i) {
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty))) break;
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
  } else if (warp == 1) {
    // The leader's whole warp runs the loop; one elected lane issues the MMAs
    // and commits (always the same lane: a commit tracks that thread's MMAs).
    if (rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t slot_count = 0;
      bool ok = true;
      for (int it = 0; ok && it < nitems; ++it) {
        int mb, nb, n_off, n_cols;
        coords(it, mb, nb, n_off, n_cols);
        const uint32_t idesc = idesc_e4m3_f32(256, n_cols);
        for (int kb = 0; ok && kb < p.KB; ++kb) {
          const int slot = static_cast<int>(slot_count & (kSlots - 1));
          const uint32_t sphase = (slot_count / kSlots) & 1u;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) ||
              !__all_sync(0xFFFFFFFFu,
                          mbar_wait_cluster(&tempty[slot], sphase ^ 1u, abort_flag, kErrWaitTmemEmpty))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * L::kA);
          const uint32_t b0 = smem_u32(sB + stage * L::kB);
          const uint32_t d = tmem_base + slot * 256;
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              mma_e4m3_pair(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc, k != 0);
            mma_commit_pair(&tfull[slot], kBoth);
            mma_commit_pair(&empty[stage], kBoth);
          }
          __syncwarp();
          ++slot_count;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp >= 4) {
    regs_grow<kBlock2EpiRegs>();
    // 8 epilogue warps: warp w reads TMEM lanes 32*(w%4)..+31 (its 32 rows)
    // and columns [h hb, h hb + hb) of every slot, h = (w - 4) / 4, hb = half
    // the item's columns (128, or 64 for a tail half): one weight block's
    // part.  acc[c] holds its columns [32 c, +32).
    // Each slot is read 64 columns at a time as four 16-column loads in
    // flight; a slot is handed back once all of its columns are in registers.
    // The scale products are fetched two K blocks ahead.
    const int ew = warp - 4;
    const int quarter = warp & 3;
    const int h = ew >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* out_s = smem + L::kOutOff + ew * 2 * L::kOutChunk;
    const int swz = (lane >> 1) & 3;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const int NB = (p.N + 127) / 128;
    uint32_t slot_count = 0;
    int buf = 0;
    bool ok = true;

    auto wait_full = [&](uint32_t u) -> bool {
      const bool done = __all_sync(0xFFFFFFFFu, mbar_wait(&tfull[u & (kSlots - 1)], (u / kSlots) & 1u, abort_flag,
                                                          kErrWaitTmemFull));
      tc_fence_after();
      return done;
    };
    auto release = [&](uint32_t u) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + (u & (kSlots - 1)) * 8);
    };

    for (int it = 0; ok && it < nitems; ++it) {
      int mb, nb, n_off, n_cols;
      coords(it, mb, nb, n_off, n_cols);
      const int hb = n_cols / 2;                                // columns of this warp: 128 or 64
      const int col_base = h * hb;                              // first accumulator column of this warp
      const int n_first = nb * 256 + n_off + col_base;          // its first output column
      const int blk = n_first / 128;
      const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quarter * 32;
      const int m = row0 + lane;
      const bool live = m < p.M && blk < NB;
      const float* xsrow = p.xs + static_cast<int64_t>(live ? m : 0) * p.KB;
      const float* wsrow = p.ws + static_cast<int64_t>(live ? blk : 0) * p.KB;
      uint64_t acc[4][16];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[c][i] = 0ull;
      float xa = live ? __ldg(xsrow) : 0.0f, wa = live ? __ldg(wsrow) : 0.0f;
      float xb = live && p.KB > 1 ? __ldg(xsrow + 1) : 0.0f, wb = live && p.KB > 1 ? __ldg(wsrow + 1) : 0.0f;

      uint32_t r[64];
      uint32_t u = slot_count;                                  // slot of the current K block
      const int nh = hb / 64;                                   // 64-column loads: 2, or 1 for a tail half
      // Per K block: nh loads of 64 columns, each waited for and folded in;
      // the slot is handed back after its last load.
      for (int kb = 0; kb < p.KB; ++kb) {
        const uint64_t f2 = f32x2_pack(xa * wa, xa * wa);
        xa = xb;
        wa = wb;
        if (live && kb + 2 < p.KB) {
          xb = __ldg(xsrow + kb + 2);
          wb = __ldg(wsrow + kb + 2);
        }
        if (!wait_full(u)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c < nh) {
            __syncwarp();
            tmem_ld_32x32b_x16x4(tmem_base + lane_addr + (u & (kSlots - 1)) * 256 + col_base + c * 64, r);
            tmem_ld_wait_regs64(r);
            if (c + 1 == nh) release(u);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[2 * c + (i >> 4)][i & 15] =
                  fma_f32x2(f32x2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), f2,
                            acc[2 * c + (i >> 4)][i & 15]);
          }
        }
        ++u;
      }
      slot_count = u;
      if (!ok) break;
      // Round to bf16 and store: columns [32 c, +32) of this warp's part.
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c * 32 < hb) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float lo, hi;
            f32x2_unpack(acc[c][i], lo, hi);
            pk[i] = pack_bf16x2(lo, hi);
          }
          if (lane == 0) bulk_wait_read<1>();     // the staging tile written two chunks ago has been read
          __syncwarp();
          uint8_t* sb = out_s + buf * L::kOutChunk;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(sb + lane * 64 + ((q ^ swz) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          const int col0 = n_first + 32 * c;
          if (lane == 0 && row0 < p.M && col0 < p.N) {
            tma_store_2d(&tmY, sb, col0, row0);
            bulk_commit();
          }
          buf ^= 1;
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// --------------------------------------------------------------- block ---
template <int STAGES>
struct BlockLayout {
  static constexpr int BN = 128;
  static constexpr int kA = BM * BK;
  static constexpr int kB = BN * BK;
  static constexpr int kSlots = 4;
  static constexpr int kEpiWarps = 16;                          // 4 per TMEM lane quarter, 32 columns each
  static constexpr int kOutChunk = 32 * 32 * 2;                 // one 32 x 32 bf16 staging tile per warp
  static constexpr int kOutOff = STAGES * (kA + kB);
  static constexpr int kBarOff = kOutOff + kEpiWarps * kOutChunk;
  static constexpr int kBarBytes = (2 * STAGES + 2 * kSlots) * 8 + 8;
  static constexpr int kBytes = kBarOff + 1024 + 1024;
  static_assert(kBarBytes <= 1024, "barrier area");
  static_assert(kBytes <= 232448, "shared memory per CTA");
};

template <int STAGES>
__global__ void __launch_bounds__(576, 1)
    gemm_block_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmY, const Params p) {
  using L = BlockLayout<STAGES>;
  constexpr int BN = L::BN;
  constexpr int kSlots = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * L::kA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* sfull = empty + STAGES;
  uint64_t* sempty = sfull + kSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sempty + kSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr uint32_t kTmemCols = kSlots * BN;   // 512

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kSlots; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], L::kEpiWarps);      // one arrival per epilogue warp
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();   // global memory only from here on

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        int mb, nb;
        tile_coords(p, t, mb, nb);
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], L::kA + L::kB);
          tma_load_2d(sA + stage * L::kA, &tmA, &full[stage], kb * BK, mb * BM, pol);
          tma_load_2d(sB + stage * L::kB, &tmB, &full[stage], kb * BK, nb * BN, pol);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      griddep_launch_dependents();
      for (int i = 0; ok && i < STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) break;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
      int stage = 0, slot = 0;
      uint32_t phase = 0, sphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        for (int kb = 0; kb < p.KB; ++kb) {
          if (!mbar_wait(&sempty[slot], sphase ^ 1u, abort_flag, kErrWaitTmemEmpty)) { ok = false; break; }
          if (!mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + slot * BN;
          const uint32_t a0 = smem_u32(sA + stage * L::kA);
          const uint32_t b0 = smem_u32(sB + stage * L::kB);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            mma_e4m3(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc, k != 0);
          mma_commit(&empty[stage]);
          mma_commit(&sfull[slot]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
        }
      }
    }
  } else {
    // 16 epilogue warps: four per TMEM lane quarter, each owning 32 columns.
    // Each 128-wide K slice is folded in with that slice's scale product
    // (packed fp32x2 FMAs); the finished 32 x 32 bf16 chunk goes out through
    // a 64-byte-swizzled staging tile and a TMA store.
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int cg = ew >> 2;                                   // column group 0..3
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* out_s = smem + L::kOutOff + ew * L::kOutChunk;
    const int swz = (lane >> 1) & 3;
    int slot = 0;
    uint32_t sphase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(p, t, mb, nb);
      const int m = mb * BM + row;
      const bool row_ok = m < p.M;
      const float* xsrow = p.xs + static_cast<int64_t>(m) * p.KB;
      const float* wsrow = p.ws + static_cast<int64_t>(nb) * p.KB;
      uint64_t acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = 0ull;
      float f_next = row_ok ? __ldg(xsrow) * __ldg(wsrow) : 0.0f;
      for (int kb = 0; kb < p.KB; ++kb) {
        const float f = f_next;
        if (kb + 1 < p.KB) f_next = row_ok ? __ldg(xsrow + kb + 1) * __ldg(wsrow + kb + 1) : 0.0f;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sfull[slot], sphase, abort_flag, kErrWaitTmemFull))) { ok = false; break; }
        tc_fence_after();
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem_base + lane_addr + slot * BN + cg * 32, r);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&sempty[slot]);
        const uint64_t f2 = f32x2_pack(f, f);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          acc[j] = fma_f32x2(f32x2_pack(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), f2, acc[j]);
        if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
      }
      if (!ok) break;
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float lo, hi;
        f32x2_unpack(acc[j], lo, hi);
        pk[j] = pack_bf16x2(lo, hi);
      }
      // The staging tile of the previous tile's store must have been read.
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(out_s + lane * 64 + ((q ^ swz) << 4)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      const int row0 = mb * BM + quarter * 32, col0 = nb * BN + cg * 32;
      if (lane == 0 && row0 < p.M && col0 < p.N) {   // the store clips the rest of the box
        tma_store_2d(&tmY, out_s, col0, row0);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace prefill
}  // namespace fp8q
