// sched.cuh -- stream-K work split shared by the decode and prefill GEMMs.
//
// A GEMM's work is a list of T = n_tiles * KB steps (output tile t, K block
// kb), tile-major.  G workers (CTAs, or CTA pairs) take contiguous ranges of
// it; each run of a worker's steps inside one tile is a "segment", and a tile
// cut between workers is summed by the last of them to finish.
#pragma once

#include <stdint.h>

namespace fp8q {
namespace sched {

// The steps are cut into G contiguous ranges with q = total / G, r = total % G:
// CTA c takes q + 1 steps when c < r, else q.  32-bit arithmetic throughout
// (64-bit divisions are long instruction sequences on the critical path of
// the first load).
struct Split {
  int q, r;
};

__host__ __device__ __forceinline__ Split split_of(int total, int G) { return {total / G, total % G}; }

__host__ __device__ __forceinline__ int range_begin(int c, const Split& sp) { return c * sp.q + min(c, sp.r); }

// The CTA whose range holds step x.
__host__ __device__ __forceinline__ int cta_of_step(int x, const Split& sp) {
  const int big = sp.r * (sp.q + 1);
  return x < big ? x / (sp.q + 1) : sp.r + (x - big) / sp.q;
}

// Walks the steps [b, e) of a CTA's range in the order: the partial segment
// that ends the range ([last_begin, e), empty when e ends a tile), then the
// segment that starts it ([b, first_end)), then the whole tiles between them
// ([first_end, last_begin)).  The tile t and K block kb are kept
// incrementally: divisions only where a run starts.
struct StepIter {
  int first_end, last_begin, b0, e0;
  int s, cur_b, cur_e;   // the current run [cur_b, cur_e)
  int run, t, kb, KB;
  __host__ __device__ StepIter(int b, int e, int kblocks) : b0(b), e0(e), KB(kblocks) {
    first_end = min(e, (b / KB + 1) * KB);
    last_begin = (e % KB == 0) ? e : max(first_end, ((e - 1) / KB) * KB);
    run = -1;
    next_run();
  }
  __host__ __device__ void next_run() {
    for (;;) {
      ++run;
      if (run == 0) { cur_b = last_begin; cur_e = e0; }
      else if (run == 1) { cur_b = b0; cur_e = first_end; }
      else if (run == 2) { cur_b = first_end; cur_e = last_begin; }
      else return;
      if (cur_b < cur_e) break;
    }
    s = cur_b;
    t = s / KB;
    kb = s - t * KB;
  }
  __host__ __device__ bool valid() const { return run < 3; }
  // Whether this step starts / ends a segment (a run of steps in one tile).
  __host__ __device__ bool seg_first() const { return s == cur_b || kb == 0; }
  __host__ __device__ bool seg_last() const { return s + 1 == cur_e || kb + 1 == KB; }
  __host__ __device__ void next() {
    if (++s == cur_e) {
      next_run();
    } else if (++kb == KB) {
      kb = 0;
      ++t;
    }
  }
};

// Cluster split-K (decode): rank r of the C CTAs that share weight tile t
// takes its K blocks [r KB / C, (r + 1) KB / C), the steps [b, e) of the
// list: one segment, non-empty when C <= KB.
__host__ __device__ __forceinline__ void cluster_range(int t, int r, int C, int KB, int* b, int* e) {
  *b = t * KB + r * KB / C;
  *e = t * KB + (r + 1) * KB / C;
}

}  // namespace sched
}  // namespace fp8q
