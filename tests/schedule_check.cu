// Host-side check of the GEMM kernels' work schedules (compiled by nvcc for
// the host only and run by tests/test_schedule.py; no GPU).
//
// Decode (stream-K): for many (tiles, K blocks, CTAs) it checks, with the
// kernel's own StepIter, range_begin and cta_of_step:
//   - the CTA ranges partition the T = n_tiles * KB steps, none empty;
//   - a CTA visits each step of its range exactly once, in the order partial
//     last segment, first segment, whole tiles, with the right (t, kb) and
//     segment flags;
//   - cta_of_step(s) is the CTA owning step s;
//   - the workspace slots (t + c) of partial segments are unique and below
//     n_tiles + G - 1, the slot count the host allocates;
//   - for every split tile, CTAs c0..c1 (as the last-arriver sums them) are
//     exactly the CTAs holding a partial segment of it.
//
// Cluster split-K (decode): for every K-block count and cluster size C <= KB,
// with the kernel's own cluster_range and StepIter, the C ranks' ranges
// partition the tile's K blocks in rank order, each is one non-empty segment
// of that tile (first and last step flagged), and none is the whole tile.
//
// Prefill (persistent CTAs or CTA pairs): for many (row blocks, column
// blocks, workers), with the kernels' own tail_split, work_items, work_item
// and tile_coords, every column of every tile is computed by exactly one
// item, for 256- and 128-column tiles.
#include <cstdio>
#include <cstdlib>
#include <set>
#include <vector>

#include "../fp8_w8a8_quantized_amax_b200/csrc/gemm_decode.cuh"
#include "../fp8_w8a8_quantized_amax_b200/csrc/gemm_prefill.cuh"

using namespace fp8q::sched;

static int fail(const char* what, int n_tiles, int KB, int G) {
  std::printf("FAIL %s (n_tiles=%d KB=%d G=%d)\n", what, n_tiles, KB, G);
  return 1;
}

static int check(int n_tiles, int KB, int G) {
  const int total = n_tiles * KB;
  const Split sp = split_of(total, G);
  std::vector<int> owner(total, -1), seen(total, 0);
  std::set<int64_t> slots;
  std::vector<std::set<int>> partial_ctas(n_tiles);
  // sizes: every range q or q + 1 steps
  for (int c = 0; c < G; ++c) {
    const int len = range_begin(c + 1, sp) - range_begin(c, sp);
    if (len != total / G && len != total / G + 1) return fail("range size", n_tiles, KB, G);
  }
  if (range_begin(0, sp) != 0 || range_begin(G, sp) != total) return fail("ranges cover", n_tiles, KB, G);
  for (int c = 0; c < G; ++c) {
    const int b = range_begin(c, sp), e = range_begin(c + 1, sp);
    if (b >= e) return fail("empty range", n_tiles, KB, G);
    for (int s = b; s < e; ++s) owner[s] = c;
    // expected order
    const int first_end = std::min(e, (b / KB + 1) * KB);
    const int last_begin = (e % KB == 0) ? e : std::max(first_end, ((e - 1) / KB) * KB);
    std::vector<int> want;
    for (int s = last_begin; s < e; ++s) want.push_back(s);
    for (int s = b; s < first_end; ++s) want.push_back(s);
    for (int s = first_end; s < last_begin; ++s) want.push_back(s);
    size_t i = 0;
    int seg_len = 0;
    for (StepIter it(b, e, KB); it.valid(); it.next(), ++i) {
      if (i >= want.size() || it.s != want[i]) return fail("step order", n_tiles, KB, G);
      if (it.t != it.s / KB || it.kb != it.s % KB) return fail("tile / K block", n_tiles, KB, G);
      ++seen[it.s];
      const bool first = (i == 0) || it.kb == 0 || want[i - 1] + 1 != it.s;
      const bool last = (i + 1 == want.size()) || it.kb + 1 == KB || want[i + 1] != it.s + 1;
      if (it.seg_first() != first || it.seg_last() != last) return fail("segment flags", n_tiles, KB, G);
      seg_len = first ? 1 : seg_len + 1;
      if (last && seg_len != KB) {                       // a partial segment of tile t
        if (!slots.insert(it.t + c).second) return fail("workspace slot reused", n_tiles, KB, G);
        if (it.t + c >= n_tiles + G - 1) return fail("workspace slot out of range", n_tiles, KB, G);
        partial_ctas[it.t].insert(c);
      }
    }
    if (i != want.size()) return fail("steps missing", n_tiles, KB, G);
  }
  for (int s = 0; s < total; ++s) {
    if (seen[s] != 1) return fail("step not visited once", n_tiles, KB, G);
    if (cta_of_step(s, sp) != owner[s]) return fail("cta_of_step", n_tiles, KB, G);
  }
  for (int t = 0; t < n_tiles; ++t) {
    const int c0 = cta_of_step(t * KB, sp);
    const int c1 = cta_of_step(t * KB + KB - 1, sp);
    std::set<int> want;
    if (c0 != c1)
      for (int c = c0; c <= c1; ++c) want.insert(c);
    if (want != partial_ctas[t]) return fail("split tile's CTAs", n_tiles, KB, G);
  }
  return 0;
}

static int check_cluster(int n_tiles, int KB, int C) {
  for (int t = 0; t < n_tiles; ++t) {
    int next = t * KB;
    for (int r = 0; r < C; ++r) {
      int b, e;
      cluster_range(t, r, C, KB, &b, &e);
      if (b != next || e <= b || e > (t + 1) * KB) return fail("cluster ranges", n_tiles, KB, C);
      next = e;
      int n = 0;
      for (StepIter it(b, e, KB); it.valid(); it.next(), ++n) {
        if (it.s != b + n || it.t != t || it.kb != it.s - t * KB) return fail("cluster steps", n_tiles, KB, C);
        if (it.seg_first() != (n == 0) || it.seg_last() != (it.s + 1 == e))
          return fail("cluster segment flags", n_tiles, KB, C);
      }
      if (n != e - b || n == KB) return fail("cluster segment length", n_tiles, KB, C);
    }
    if (next != (t + 1) * KB) return fail("cluster ranges cover the tile", n_tiles, KB, C);
  }
  return 0;
}

static int check_prefill(int num_m, int num_n, int G, int tile_cols) {
  fp8q::prefill::Params p{};
  p.num_m = num_m;
  p.num_n = num_n;
  p.num_tiles = num_m * num_n;
  p.group_m = num_m < 8 ? num_m : 8;
  fp8q::prefill::tail_split(p.num_tiles, G, &p.full, &p.split);
  std::vector<int> cov(static_cast<size_t>(p.num_tiles) * tile_cols, 0);
  for (int c = 0; c < G; ++c) {
    const int n = fp8q::prefill::work_items(p, c, G);
    for (int i = 0; i < n; ++i) {
      int mb, nb, off, cols;
      fp8q::prefill::work_item(p, c, G, i, tile_cols, mb, nb, off, cols);
      if (mb < 0 || mb >= num_m || nb < 0 || nb >= num_n || off < 0 || cols <= 0 || off + cols > tile_cols) {
        std::printf("FAIL prefill item out of range (m=%d n=%d G=%d)\n", num_m, num_n, G);
        return 1;
      }
      for (int x = off; x < off + cols; ++x) ++cov[(static_cast<size_t>(mb) * num_n + nb) * tile_cols + x];
    }
  }
  for (int v : cov)
    if (v != 1) {
      std::printf("FAIL prefill coverage (m=%d n=%d G=%d cols=%d)\n", num_m, num_n, G, tile_cols);
      return 1;
    }
  return 0;
}

int main() {
  int bad = 0, cases = 0;
  for (int num_m = 1; num_m <= 12; ++num_m)
    for (int num_n = 1; num_n <= 12; ++num_n)
      for (int G : {1, 2, 3, 5, 7, 8, 16, 37, 74, 148})
        for (int cols : {256, 128}) {
          bad |= check_prefill(num_m, num_n, G, cols);
          ++cases;
        }
  // the Llama prefill shapes on 74 CTA pairs / 148 CTAs
  const int pshapes[][2] = {{8, 32}, {32, 56}, {32, 16}, {32, 4}, {2, 112}, {2, 40}, {16, 32}, {32, 112}};
  for (auto& sh : pshapes)
    for (int G : {74, 148})
      for (int cols : {256, 128}) {
        bad |= check_prefill(sh[0], sh[1], G, cols);
        ++cases;
      }
  // every small case, then the Llama decode shapes on 148 SMs
  for (int n_tiles = 1; n_tiles <= 24; ++n_tiles)
    for (int KB = 1; KB <= 12; ++KB)
      for (int G = 1; G <= n_tiles * KB && G <= 40; ++G, ++cases) bad |= check(n_tiles, KB, G);
  const int shapes[][2] = {{224, 64}, {64, 224}, {80, 64}, {64, 24}, {32, 32}, {8, 24}, {448, 64}, {1, 1}};
  for (auto& sh : shapes)
    for (int G : {1, 2, 7, 74, 147, 148}) {
      if (G > sh[0] * sh[1]) continue;
      bad |= check(sh[0], sh[1], G);
      ++cases;
    }
  // cluster split-K: every cluster size on small K-block counts and the
  // FP8-Block decode shapes (K = 3072 and 8192: 24 and 64 K blocks)
  for (int KB = 2; KB <= 70; ++KB)
    for (int C = 2; C <= 8 && C <= KB; ++C, ++cases) bad |= check_cluster(3, KB, C);
  std::printf("%s: %d schedules\n", bad ? "FAIL" : "ok", cases);
  return bad;
}
