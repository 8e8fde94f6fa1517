// Host-side check of the decode kernel's stream-K schedule (compiled by nvcc
// for the host only and run by tests/test_schedule.py; no GPU).  For many
// (tiles, K blocks, CTAs) it checks, with the kernel's own StepIter,
// range_begin and cta_of_step:
//   - the CTA ranges partition the T = n_tiles * KB steps, none empty;
//   - a CTA visits each step of its range exactly once, in the order partial
//     last segment, first segment, whole tiles, with the right (t, kb) and
//     segment flags;
//   - cta_of_step(s) is the CTA owning step s;
//   - the workspace slots (t + c) of partial segments are unique and below
//     n_tiles + G - 1, the slot count the host allocates;
//   - for every split tile, CTAs c0..c1 (as the last-arriver sums them) are
//     exactly the CTAs holding a partial segment of it.
#include <cstdio>
#include <cstdlib>
#include <set>
#include <vector>

#include "../fp8_w8a8_quantized_amax_b200/csrc/gemm_decode.cuh"

using namespace fp8q::decode;

static int fail(const char* what, int n_tiles, int KB, int G) {
  std::printf("FAIL %s (n_tiles=%d KB=%d G=%d)\n", what, n_tiles, KB, G);
  return 1;
}

static int check(int n_tiles, int KB, int G) {
  const int64_t total = static_cast<int64_t>(n_tiles) * KB;
  std::vector<int> owner(total, -1), seen(total, 0);
  std::set<int64_t> slots;
  std::vector<std::set<int>> partial_ctas(n_tiles);
  for (int c = 0; c < G; ++c) {
    const int64_t b = range_begin(c, total, G), e = range_begin(c + 1, total, G);
    if (b >= e) return fail("empty range", n_tiles, KB, G);
    for (int64_t s = b; s < e; ++s) owner[s] = c;
    // expected order
    const int64_t first_end = std::min(e, (b / KB + 1) * KB);
    const int64_t last_begin = (e % KB == 0) ? e : std::max(first_end, ((e - 1) / KB) * KB);
    std::vector<int64_t> want;
    for (int64_t s = last_begin; s < e; ++s) want.push_back(s);
    for (int64_t s = b; s < first_end; ++s) want.push_back(s);
    for (int64_t s = first_end; s < last_begin; ++s) want.push_back(s);
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
  for (int64_t s = 0; s < total; ++s) {
    if (seen[s] != 1) return fail("step not visited once", n_tiles, KB, G);
    if (cta_of_step(s, total, G) != owner[s]) return fail("cta_of_step", n_tiles, KB, G);
  }
  for (int t = 0; t < n_tiles; ++t) {
    const int c0 = cta_of_step(static_cast<int64_t>(t) * KB, total, G);
    const int c1 = cta_of_step(static_cast<int64_t>(t) * KB + KB - 1, total, G);
    std::set<int> want;
    if (c0 != c1)
      for (int c = c0; c <= c1; ++c) want.insert(c);
    if (want != partial_ctas[t]) return fail("split tile's CTAs", n_tiles, KB, G);
  }
  return 0;
}

int main() {
  int bad = 0, cases = 0;
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
  std::printf("%s: %d schedules\n", bad ? "FAIL" : "ok", cases);
  return bad;
}
