// gemm_decode.cuh -- FP8 linear for small M (decode, M <= 64): HBM-bound weight stream.
//
// Swap-AB: a 128-row slice of Wq is the tcgen05 "A" operand (UMMA M = 128)
// and the M tokens, padded with zero rows to NX in {16, 32, 64}, are "B"
// (UMMA N = NX), so the accumulator D[n, m] sits in TMEM with lane = output
// channel and column = token.
//
// Stream-K: the (weight tile t, K block kb) pairs, t-major, form one list of
// T = n_tiles * KB steps that is cut into G equal contiguous ranges, one per
// CTA (G <= #SMs, every range non-empty).  Each run of a CTA's steps inside
// one weight tile is a "segment".  A segment that is a whole tile is scaled
// and written as bf16 at once.  A partial segment's fp32 sums D[n, m]
// (already multiplied by the block scales in block mode) go to workspace
// slot (t + c) -- unique because a CTA's tiles increase with c -- and each
// epilogue warp counts its 32 channels in with an atomic on a per-(tile,
// warp) counter.  The warp that arrives last adds the tile's segments for its
// channels in CTA order (deterministic: the same sum whichever CTA finishes
// last), applies the channel scales in channel mode, writes bf16, and sets
// the counter and the partial sums it read back to zero: the workspace is all
// zero between calls, whatever their shapes.  Nothing waits on another CTA.
// A CTA takes its steps in the order: the partial segment at the end of its
// range (the start of a tile it shares with the next CTA), the segment at the
// start of its range, then the whole tiles between them, so that the
// reductions happen under the rest of the weight stream.  Where that does
// not pay (SUMS = kSumsSeparate; the host decides per shape) the partial segments
// are summed by decode_reduce_kernel after the GEMM kernel, which clears them
// likewise.  Partial traffic is at most (n_tiles + G) * NX * 512 bytes, small
// next to the N * K weight bytes.
//
// Cluster split-K (SUMS = kSumsCluster; the host picks it for small block-mode
// problems, n_tiles * C CTAs filling most SMs): CTA rank r of cluster t (C
// CTAs) takes K blocks [r KB / C, (r + 1) KB / C) of weight tile t, a single
// partial segment.  Its sums stay in its own shared memory; after a cluster
// barrier rank 0 adds the C partial tiles in rank order through distributed
// shared memory and writes the bf16 tile, and a second barrier keeps every
// CTA resident until then.  No workspace, no atomics, no second kernel.
//
// Roles: warp 0 TMA (W tile 128 x 128 B evict-first + X tile NX x 128 B),
// warp 1 TMEM allocation + MMA issue, warps 2..5 drain TMEM and write
// segments.  TMEM holds 8 slots of NX columns.  Channel mode accumulates a
// whole segment in one slot (drained once per segment); block mode gives
// every K block its own slot, folded into registers with that block's
// x_scale * w_scale.  Block mode's scales reach each epilogue warp through a
// small shared-memory ring, filled by asynchronous 4-byte copies several
// steps ahead, so that no scale load sits on the fold's critical path.
//
// Weight-only variant (WIDEN > 0 warps, bf16 activations, channel scales):
// the same schedule with the activation tile loaded as bf16 (two 64-value
// atoms per K block), WIDEN extra warps that widen each staged E4M3 weight
// tile into a bf16 tile in the same swizzled layout (exactly: every E4M3
// value is a bf16 value), and bf16 MMAs (kind::f16, K = 16) on that tile.
// No x_scale: the epilogue applies w_scale alone.
#pragma once

#include "ptx.cuh"
#include "sched.cuh"

namespace fp8q {
namespace decode {

using sched::Split;
using sched::StepIter;
using sched::cta_of_step;
using sched::range_begin;
using sched::split_of;

constexpr int BK = 128;
constexpr int UMMA_K = 32;
constexpr int kSlots = 8;

// Where a weight tile's partial segments are added: decode_reduce_kernel after
// the GEMM kernel, the last CTA to finish one (through the workspace), or rank 0
// of the tile's cluster (through distributed shared memory).
constexpr int kSumsSeparate = 0, kSumsKernel = 1, kSumsCluster = 2;

struct Params {
  const float* xs;
  const float* ws;
  unsigned int* count;  // workspace: [n_tiles][4] arrival counters
  float* part;          // workspace: [(n_tiles + G - 1)][NX][128] fp32 partial sums
  __nv_bfloat16* y;
  int64_t ldy;
  int M, N, K, KB;
  int n_tiles;
  int total;            // n_tiles * KB (the host refuses 2^31 or more)
  int G;                // CTAs (cluster split-K: n_tiles * cluster size)
  int early;            // in-kernel sums: a known last contributor loads its partners' sums early
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// WIDEN > 0: the weight-only variant (bf16 activations).  Each stage then also
// holds the bf16 activation tile (NX rows x 128 values, two 128-byte-swizzle
// atoms of 64 values) and the widened bf16 weight tile (128 rows x 128 values,
// two atoms of 16 KB), and WIDEN extra warps (4: a thread widens one weight
// row; 8: half a row) write the latter from the E4M3 tile the TMA brought in.
template <int NX, int STAGES, int WIDEN = 0>
struct Layout {
  static constexpr bool W16 = WIDEN > 0;
  static constexpr int kW = 128 * BK;
  static constexpr int kX = NX * BK * (W16 ? 2 : 1);
  static constexpr int kWide = W16 ? 128 * BK * 2 : 0;
  static constexpr int kBarOff = STAGES * (kW + kX + kWide);
  static constexpr int kThreads = 192 + 32 * WIDEN;
  static constexpr int kBarBytes = (2 * STAGES + 2 * kSlots + (W16 ? STAGES : 0) + 1) * 8 + 8;   // mbarriers, TMEM address, abort flag
  static constexpr int kBytes = kBarOff + 1024 + 1024;                  // + barrier area + alignment slack
  static_assert(kBarBytes <= 1024, "barrier area");
  static_assert(kBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = (kSlots * NX) < 32 ? 32 : (kSlots * NX);
};

// MINB = 2: built to fit two CTAs per SM (registers; the caller picks stages
// that fit two in shared memory), so that the next kernel's CTAs can start
// beside this one's while it finishes.
template <int NX, int STAGES, bool BLOCK, int SUMS, int WIDEN = 0, int MINB = 1>
__global__ void __launch_bounds__(Layout<NX, STAGES, WIDEN>::kThreads, MINB)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const Params p) {
  using L = Layout<NX, STAGES, WIDEN>;
  constexpr bool W16 = WIDEN > 0;
  static_assert(WIDEN == 0 || WIDEN == 4 || WIDEN == 8, "widen warps");
  static_assert(NX % 16 == 0 && NX >= 16 && NX <= 64, "token tile");
  static_assert(!(W16 && (BLOCK || SUMS != kSumsKernel)),
                "the weight-only variant has channel scales and sums its own splits");
  static_assert(SUMS == kSumsSeparate || SUMS == kSumsKernel || SUMS == kSumsCluster, "sums");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sW = smem;
  uint8_t* sX = smem + STAGES * L::kW;
  uint8_t* sWide = sX + STAGES * L::kX;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* sfull = empty + STAGES;
  uint64_t* sempty = sfull + kSlots;
  uint64_t* wfull = sempty + kSlots;                       // W16: widened tile ready (STAGES of them)
  uint64_t* drain = wfull + (W16 ? STAGES : 0);            // abort path: the MMAs issued have completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const Split sp = split_of(p.total, p.G);
  int b, e;
  if constexpr (SUMS == kSumsCluster) {
    const int C = static_cast<int>(cluster_nctarank());
    sched::cluster_range(c / C, static_cast<int>(cluster_ctarank()), C, p.KB, &b, &e);
  } else {
    b = range_begin(c, sp);
    e = range_begin(c + 1, sp);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kSlots; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], 4);                  // one arrival per epilogue warp
    }
    if constexpr (W16)
      for (int s = 0; s < STAGES; ++s) mbar_init(&wfull[s], WIDEN);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The first weight tiles of this CTA's range are prefetched into L2 before
  // the wait for the previous kernel: the weights are not what that kernel
  // writes (and L2 is coherent if they were), so their DRAM latency overlaps
  // its tail.  The epilogue warps issue them (every fourth step each; they
  // have nothing to do until the first accumulator is ready), so that the
  // producer's first load is not queued behind them.  Only where the range
  // is longer than the stages: where the producer issues every load of the
  // range at once, the doubled requests measured slower (3B FP8-Block shapes,
  // ~1 us), while longer ranges gain (70B gate/qkv, 0.5-1 us back to back).
  // Prefetching twice the stages measured 1-3% slower on every 70B shape,
  // and prefetching a whole range of up to twice the stages slower on the 3B
  // FP8-Block decode (M=1: 10.4 against 10.1 us back to back).
  if (warp >= 2 && warp < 6 && lane == 0 && e - b > STAGES) {
    int i = 0;
    for (StepIter it(b, e, p.KB); it.valid() && i < STAGES; it.next(), ++i)
      if ((i & 3) == warp - 2) tma_prefetch_l2_2d(&tmW, it.kb * BK, it.t * 128);
  }
  griddep_wait();   // global memory only from here on (reads of the prefetched tiles included)

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (StepIter it(b, e, p.KB); it.valid(); it.next()) {
        const int t = it.t, kb = it.kb;
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) { ok = false; break; }
        ++issued;
        mbar_arrive_expect_tx(&full[stage], L::kW + L::kX);
        tma_load_2d(sW + stage * L::kW, &tmW, &full[stage], kb * BK, t * 128, pol_w);
        tma_load_2d(sX + stage * L::kX, &tmX, &full[stage], kb * BK, 0, pol_x);
        if constexpr (W16)   // bf16 activations: the second 64-value atom of the K block
          tma_load_2d(sX + stage * L::kX + NX * 128, &tmX, &full[stage], kb * BK + 64, 0, pol_x);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      griddep_launch_dependents();
      for (int i = 0; ok && i < STAGES; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, kErrWaitEmpty)) { ok = false; break; }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        // Aborted: the last load of each stage may still be in flight.  Each
        // completes on its own; wait for all of them before the CTA's shared
        // memory is released.  Walk back from the stage that was not issued.
        const int n = issued < STAGES ? issued : STAGES;
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < n; ++i) {
          if (--s < 0) { s = STAGES - 1; ph ^= 1u; }
          mbar_wait_drain(&full[s], ph, kErrWaitDrain);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = W16 ? idesc_bf16_f32(128, NX) : idesc_e4m3_f32(128, NX);
      int stage = 0, slot = 0;
      uint32_t phase = 0, sphase = 0;
      bool ok = true;
#ifdef FP8Q_TEST_HOOKS
      bool withheld = false;
#endif
      for (StepIter it(b, e, p.KB); it.valid(); it.next()) {
        const bool seg_first = it.seg_first();
        const bool seg_last = it.seg_last();
        // Block mode: one TMEM slot per K block (its scales differ).  Channel
        // mode: one slot per segment, accumulated across its K blocks.
        const bool open_slot = BLOCK || seg_first;
        const bool close_slot = BLOCK || seg_last;
        if (open_slot && !mbar_wait(&sempty[slot], sphase ^ 1u, abort_flag, kErrWaitTmemEmpty)) { ok = false; break; }
        if (!mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull)) { ok = false; break; }
        if (W16 && !mbar_wait(&wfull[stage], phase, abort_flag, kErrWaitFull)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + slot * NX;
        const uint32_t b0 = smem_u32(sX + stage * L::kX);
        if constexpr (W16) {
          // 8 MMAs of K = 16 bf16 values (32 bytes): 4 per 64-value atom
          const uint32_t a0 = smem_u32(sWide + stage * L::kWide);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d, umma_desc_sw128(a0 + (k >> 2) * (128 * 128) + (k & 3) * 32),
                     umma_desc_sw128(b0 + (k >> 2) * (NX * 128) + (k & 3) * 32), idesc,
                     (!open_slot || k != 0) ? 1u : 0u);
        } else {
          const uint32_t a0 = smem_u32(sW + stage * L::kW);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            mma_e4m3(d, umma_desc_sw128(a0 + k * UMMA_K), umma_desc_sw128(b0 + k * UMMA_K), idesc,
                     (!open_slot || k != 0) ? 1u : 0u);
        }
        mma_commit(&empty[stage]);
        if (close_slot) {
#ifdef FP8Q_TEST_HOOKS
          // Test build, switch 2: CTA 0 withholds its first accumulator commit.
          const bool withhold = c == 0 && !withheld && g_test_withhold == 2;
          withheld = withheld || withhold;
          if (!withhold) mma_commit(&sfull[slot]);
#else
          mma_commit(&sfull[slot]);
#endif
          if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
        }
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      // Every MMA issued must finish before the tensor memory is released.
      // Normally the epilogue's waits already imply it; after an abort they
      // do not, so one more commit tracks all of them, always.
      mma_commit(drain);
      if (!mbar_wait_drain(drain, 0, kErrWaitDrain)) ok = false;
    }
  } else if (W16 && warp >= 6) {
    // Widen: a thread takes one weight row of the tile (8 warps: half of it).
    // Its chunks of 16 codes (128-byte swizzle: chunk c sits at c ^ (row & 7))
    // become chunks of 8 bf16 values in the two 64-value atoms, swizzled the
    // same way.
    constexpr int kChunks = WIDEN == 8 ? 4 : 8;
    const int row = ((warp - 6) & 3) * 32 + lane;
    const int ch0 = ((warp - 6) >> 2) * kChunks;
    const int sw = row & 7;
    int stage = 0;
    uint32_t phase = 0;
    for (StepIter it(b, e, p.KB); it.valid(); it.next()) {
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[stage], phase, abort_flag, kErrWaitFull))) break;
      const uint8_t* src = sW + stage * L::kW + row * 128;
      uint8_t* dst = sWide + stage * L::kWide + row * 128;
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int ch = ch0 + i;
        const uint4 q = *reinterpret_cast<const uint4*>(src + ((ch ^ sw) << 4));
        uint4 lo, hi;
        widen16_bf16(q, lo, hi);
        uint8_t* atom = dst + (ch >> 2) * (128 * 128);
        const int c2 = 2 * (ch & 3);
        *reinterpret_cast<uint4*>(atom + ((c2 ^ sw) << 4)) = lo;
        *reinterpret_cast<uint4*>(atom + (((c2 + 1) ^ sw) << 4)) = hi;
      }
      fence_proxy_async_smem();   // generic-proxy writes, read by the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&wfull[stage]);
      if (++stage == STAGES) { stage = 0; phase ^= 1u; }
    }
  } else {
    const int quarter = warp & 3;
    const int nl = quarter * 32 + lane;          // output channel within the tile
    // Channel mode: this warp's copy of x_scale in shared memory, read by the
    // output loop (global loads there would queue behind the output stores).
    __shared__ float s_xs[4][NX];
    if constexpr (!BLOCK) {
      for (int j = lane; j < NX; j += 32) s_xs[quarter][j] = j < p.M ? (W16 ? 1.0f : __ldg(p.xs + j)) : 0.0f;
      __syncwarp();
    }
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float acc[NX];
#pragma unroll
    for (int j = 0; j < NX; ++j) acc[j] = 0.0f;
    int slot = 0;
    uint32_t sphase = 0;
    // Block mode: the x_scale column and w_scale of each step go into this
    // warp's ring slot (step index % kRing) kAhead steps before the step is
    // folded, by cp.async copies of one float per lane; one commit group per
    // step, so wait_group<kAhead - 1> means the current step's scales are in.
    constexpr int kRing = 8, kAhead = 6;
    __shared__ float s_ring[BLOCK ? 4 : 1][BLOCK ? kRing : 1][NX + 1];
    float* ring = &s_ring[BLOCK ? quarter : 0][0][0];
    StepIter pf(b, e, p.KB);                        // the step whose scales are fetched next
    int pf_i = 0;
    auto prefetch = [&]() {
      if constexpr (BLOCK) {
        if (pf.valid()) {
          float* dst = ring + (pf_i % kRing) * (NX + 1);
          for (int j = lane; j < NX; j += 32)
            if (j < p.M) cp_async_f32(dst + j, p.xs + static_cast<int64_t>(j) * p.KB + pf.kb);
          if (lane == 0) cp_async_f32(dst + NX, p.ws + static_cast<int64_t>(pf.t) * p.KB + pf.kb);
          pf.next();
        }
        ++pf_i;
        cp_async_commit();
      }
    };
    if constexpr (BLOCK) {
      for (int i = lane; i < kRing * NX; i += 32)   // padded tokens (never copied into) stay 0
        if (i % NX >= p.M) ring[(i / NX) * (NX + 1) + i % NX] = 0.0f;
      __syncwarp();
      for (int i = 0; i < kAhead; ++i) prefetch();
    }
    StepIter it(b, e, p.KB);
    int step_i = 0;
    int seg_len = 0;
#ifdef FP8Q_TEST_HOOKS
    bool withheld = false;
#endif
    for (; it.valid(); it.next(), ++step_i) {
      const int t = it.t;
      seg_len = it.seg_first() ? 1 : seg_len + 1;
      const bool seg_last = it.seg_last();
      if (!BLOCK && !seg_last) continue;           // channel mode: one drain per segment
      // channel mode: the channel's w_scale is loaded before the wait for the
      // accumulator, so that scaling the output never waits on a DRAM load
      float wn_pre = 1.0f;
      if constexpr (!BLOCK) {
        const int n0 = t * 128 + nl;
        if (n0 < p.N) wn_pre = __ldg(p.ws + n0);
      }
      // In-kernel sums, a partial segment's last step: if every other CTA of
      // the tile has already published its part (an acquire load of the
      // counter), this warp is the tile's last contributor for certain.  It
      // then loads their partial sums now, while its own MMAs finish, and
      // later adds them to its own in CTA order without publishing anything:
      // the same sums in the same order as the last arriver's, off the end
      // of the kernel's critical path.
      // (at most 168 registers when built for two CTAs per SM: up to two
      // partners, channel scales)
      constexpr int kPre = SUMS != kSumsKernel ? 0
                           : MINB == 1 ? (NX == 16 ? 3 : (NX == 32 ? 1 : 0))
                                       : ((NX == 16 && !BLOCK) ? 2 : 0);
      bool known_last = false;
      float pre[kPre > 0 ? kPre + 1 : 1][NX];      // by position in c0..c0+kPre (own and absent: 0)
      if constexpr (kPre > 0) {
        if (p.early && seg_last && seg_len != p.KB) {
          const int c0 = cta_of_step(t * p.KB, sp);
          const int c1 = cta_of_step(t * p.KB + p.KB - 1, sp);
          if (c1 - c0 <= kPre) {
            unsigned int cnt = 0;
            if (lane == 0) cnt = ld_acquire_gpu(p.count + t * 4 + quarter);
            cnt = __shfl_sync(0xFFFFFFFFu, cnt, 0);
            __syncwarp();                          // the other lanes' loads come after the acquire
            known_last = cnt == static_cast<unsigned int>(c1 - c0);
            if (known_last) {
#pragma unroll
              for (int u = 0; u <= kPre; ++u) {
                const int cc = c0 + u;
                const float* src = p.part + (static_cast<int64_t>(t) + cc) * NX * 128 + nl;
#pragma unroll
                for (int j = 0; j < NX; ++j)
                  pre[u][j] = (cc != c && cc <= c1 && j < p.M) ? __ldcg(src + j * 128) : 0.0f;
              }
            }
          }
        }
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sfull[slot], sphase, abort_flag, kErrWaitTmemFull))) break;
      tc_fence_after();
      uint32_t r[NX];
      __syncwarp();
#pragma unroll
      for (int j = 0; j < NX; j += 16) tmem_ld_32x32b_x16(tmem_base + lane_addr + slot * NX + j,
                                                           *reinterpret_cast<uint32_t(*)[16]>(&r[j]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
#ifdef FP8Q_TEST_HOOKS
      // Test build, switch 1: CTA 0's warp 2 withholds its first slot release.
      const bool withhold = c == 0 && warp == 2 && !withheld && g_test_withhold == 1;
      withheld = withheld || withhold;
      if (lane == 0 && !withhold) mbar_arrive_relaxed(&sempty[slot]);
#else
      if (lane == 0) mbar_arrive_relaxed(&sempty[slot]);
#endif
      if (++slot == kSlots) { slot = 0; sphase ^= 1u; }
      if constexpr (BLOCK) {
        cp_async_wait<kAhead - 1>();               // this step's scales are in the ring
        __syncwarp();
        const float* sc = ring + (step_i % kRing) * (NX + 1);
        const float wsf = sc[NX];
#pragma unroll
        for (int j = 0; j < NX; ++j) acc[j] = fmaf(__uint_as_float(r[j]), sc[j] * wsf, acc[j]);
        __syncwarp();                              // every lane has read the slot before it is refilled
        prefetch();
      } else {
#pragma unroll
        for (int j = 0; j < NX; ++j) acc[j] = __uint_as_float(r[j]);
      }
      if (seg_last) {                              // segment ends
        const int tile_first = t * p.KB;
        const int n = t * 128 + nl;
        // bf16 output of channel n for the token sums v[j]
        auto emit = [&](const float (&v)[NX]) {
          if (n < p.N) {
            const float wn = wn_pre;
#pragma unroll
            for (int j = 0; j < NX; ++j) {
              if (j < p.M) {
                const float o = BLOCK ? v[j] : v[j] * s_xs[quarter][j] * wn;
                p.y[static_cast<int64_t>(j) * p.ldy + n] = __float2bfloat16_rn(o);
              }
            }
          }
        };
        if (seg_len == p.KB) {                     // the whole tile: no partial sums
          emit(acc);
        } else if (kPre > 0 && known_last) {
          // every other part is in (loaded above): add the parts in CTA order,
          // clear what was read, write the tile, reset the counter
          const int c0 = cta_of_step(tile_first, sp);
          const int c1 = cta_of_step(tile_first + p.KB - 1, sp);
          float sum[NX];
#pragma unroll
          for (int j = 0; j < NX; ++j) sum[j] = 0.0f;
#pragma unroll
          for (int u = 0; u <= kPre; ++u) {            // position u of c0..c1 (the +0 of an absent one changes no sum)
            const bool own = c0 + u == c;
#pragma unroll
            for (int j = 0; j < NX; ++j) sum[j] += own ? acc[j] : pre[u][j];
          }
          for (int cc = c0; cc <= c1; ++cc) {
            if (cc == c) continue;
            float* src = p.part + (static_cast<int64_t>(t) + cc) * NX * 128 + nl;
#pragma unroll
            for (int j = 0; j < NX; ++j)
              if (j < p.M) src[j * 128] = 0.0f;
          }
          emit(sum);
          __syncwarp();
          if (lane == 0) p.count[t * 4 + quarter] = 0u;
        } else if constexpr (SUMS == kSumsCluster) {
          // the CTA's one segment: every MMA has completed (this slot was the
          // last one committed) and every stage has been consumed, so the
          // stage area holds the partial tile [NX][128] for rank 0 to read
          float* part_s = reinterpret_cast<float*>(sW);
#pragma unroll
          for (int j = 0; j < NX; ++j) part_s[j * 128 + nl] = acc[j];
        } else {
          float* dst = p.part + (static_cast<int64_t>(t) + c) * NX * 128 + nl;
#pragma unroll
          for (int j = 0; j < NX; ++j)
            if (j < p.M) dst[j * 128] = acc[j];
          if constexpr (SUMS == kSumsSeparate) {
#pragma unroll
            for (int j = 0; j < NX; ++j) acc[j] = 0.0f;
            continue;                              // summed by decode_reduce_kernel
          }
          // publish: the warp's partial stores, then one acquire-release
          // increment (a release of the stores the __syncwarp ordered before
          // it, and for the last arriver an acquire of everyone else's)
          __syncwarp();
          const int c0 = cta_of_step(tile_first, sp);
          const int c1 = cta_of_step(tile_first + p.KB - 1, sp);
          unsigned int prev = 0;
          if (lane == 0) prev = atom_add_acq_rel_gpu(p.count + t * 4 + quarter, 1u);
          prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
          __syncwarp();                            // the other lanes' loads come after the acquire
          if (prev == static_cast<unsigned int>(c1 - c0)) {   // every other segment is in
            // acc is published; it now collects the tile's sum in CTA order,
            // the partial sums of kBatch CTAs loaded at once (one L2 round
            // trip per batch; the +0 of an absent CTA changes no sum, which
            // starts at +0 and so is never -0)
            constexpr int kBatch = NX <= 16 ? 4 : (NX <= 32 ? 2 : 1);
#pragma unroll
            for (int j = 0; j < NX; ++j) acc[j] = 0.0f;
            for (int cc0 = c0; cc0 <= c1; cc0 += kBatch) {
              if constexpr (kBatch == 1) {           // 64 tokens: no registers for a batch
                const float* src = p.part + (static_cast<int64_t>(t) + cc0) * NX * 128 + nl;
#pragma unroll
                for (int j = 0; j < NX; ++j)
                  if (j < p.M) acc[j] += __ldcg(src + j * 128);
              } else {
                float v[kBatch][NX];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                  const float* src = p.part + (static_cast<int64_t>(t) + cc0 + u) * NX * 128 + nl;
#pragma unroll
                  for (int j = 0; j < NX; ++j)
                    v[u][j] = (cc0 + u <= c1 && j < p.M) ? __ldcg(src + j * 128) : 0.0f;
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
#pragma unroll
                  for (int j = 0; j < NX; ++j) acc[j] += v[u][j];
              }
            }
            for (int cc = c0; cc <= c1; ++cc) {   // the workspace is left all zero
              float* src = p.part + (static_cast<int64_t>(t) + cc) * NX * 128 + nl;
#pragma unroll
              for (int j = 0; j < NX; ++j)
                if (j < p.M) src[j * 128] = 0.0f;
            }
            emit(acc);
            if (lane == 0) p.count[t * 4 + quarter] = 0u;
          }
        }
#pragma unroll
        for (int j = 0; j < NX; ++j) acc[j] = 0.0f;
      }
    }
    if constexpr (BLOCK) cp_async_wait<0>();     // no copy into the ring outlives the CTA
  }

  if constexpr (SUMS == kSumsCluster) {
    cluster_sync();   // every CTA of the cluster has its partial tile in shared memory
    const int C = static_cast<int>(cluster_nctarank());
    if (C > 1 && cluster_ctarank() == 0 && warp >= 2 && warp < 6) {
      // rank 0's epilogue threads: channel nl of the tile, the C partial sums
      // of each token added in rank order
      const int nl = (warp & 3) * 32 + lane;
      const int n = (c / C) * 128 + nl;
      const uint32_t part_s = smem_u32(sW);
      float sum[NX];
#pragma unroll
      for (int j = 0; j < NX; ++j) sum[j] = 0.0f;
      for (int r = 0; r < C; ++r) {
        const uint32_t src = mapa_shared(part_s, static_cast<uint32_t>(r)) + static_cast<uint32_t>(nl) * 4u;
#pragma unroll
        for (int j = 0; j < NX; ++j)
          if (j < p.M) sum[j] += ld_shared_cluster_f32(src + static_cast<uint32_t>(j) * 512u);
      }
      if (n < p.N) {
        const float wn = BLOCK ? 1.0f : __ldg(p.ws + n);
#pragma unroll
        for (int j = 0; j < NX; ++j)
          if (j < p.M) {
            const float o = BLOCK ? sum[j] : sum[j] * __ldg(p.xs + j) * wn;
            p.y[static_cast<int64_t>(j) * p.ldy + n] = __float2bfloat16_rn(o);
          }
      }
    }
    cluster_sync_relaxed();   // rank 0 has read every partial tile before any CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// Sum the partial segments of every weight tile that more than one CTA
// worked on, in CTA order, write bf16 output and clear the partial sums read.
// grid (n_tiles, M), 128 threads: thread = output channel within the tile.
// Tiles one CTA covered whole were written by the GEMM kernel.
template <bool BLOCK>
__global__ void __launch_bounds__(128) decode_reduce_kernel(const Params p, int nx) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x;
  const int m = blockIdx.y;
  const int nl = threadIdx.x;
  const int n = t * 128 + nl;
  const Split sp = split_of(p.total, p.G);
  const int c0 = cta_of_step(t * p.KB, sp);
  const int c1 = cta_of_step((t + 1) * p.KB - 1, sp);
  if (c0 == c1) return;
  float sum = 0.0f;
  for (int c = c0; c <= c1; ++c) sum += __ldcg(p.part + ((static_cast<int64_t>(t) + c) * nx + m) * 128 + nl);
  for (int c = c0; c <= c1; ++c) p.part[((static_cast<int64_t>(t) + c) * nx + m) * 128 + nl] = 0.0f;
  if (n < p.N) {
    const float v = BLOCK ? sum : sum * __ldg(p.xs + m) * __ldg(p.ws + n);
    p.y[static_cast<int64_t>(m) * p.ldy + n] = __float2bfloat16_rn(v);
  }
}

}  // namespace decode
}  // namespace fp8q
