// Host-only check of the kernels' per-row mask forms (no kernel launched):
// row_span / span_visible (a query row's keys) and key_span (a key's query
// tokens) select exactly the pairs visible_elem selects,
// and a tile that sink_only_tile marks has no visible column outside the
// sink prefix for any of its query rows.  Prints "ok N" or the first failure.
#include <cstdio>

#include "../../learnable_sink_b200/csrc/plan.cuh"

int main() {
  long long checked = 0;
  const int lens[] = {1, 5, 64, 130, 300};
  for (int L : lens)
    for (int causal = 0; causal <= 1; ++causal)
      for (int window = 0; window <= 70; window += (window < 8 ? 1 : 31))
        for (int n_sink = 0; n_sink <= 20; n_sink += 3) {
          if (window > 0 && !causal) continue;
          for (int qi = 0; qi < L; qi += (L > 64 ? 7 : 1))
            for (int k0 = 0; k0 < L; k0 += 16) {
              const sk::RowSpan s = sk::row_span(qi, k0, L, causal, n_sink, window);
              for (int c = 0; c < 128; ++c) {
                const bool a = sk::visible_elem(qi, k0 + c, L, causal, n_sink, window);
                const bool b = sk::span_visible(s, c);
                // the same pair from the key's side: query token qi - q0 of a
                // query tile starting at q0 = k0 (any start works)
                const sk::KeySpan ks = sk::key_span(k0 + c, k0, L, causal, n_sink, window);
                const bool d = (qi - k0) >= ks.lo && (qi - k0) <= ks.hi;
                if (a != b || a != d) {
                  std::printf("span mismatch L=%d causal=%d window=%d n_sink=%d qi=%d k0=%d c=%d\n",
                              L, causal, window, n_sink, qi, k0, c);
                  return 1;
                }
                ++checked;
              }
            }
        }
  // sink-only tiles (128-key tiles, rows [q0, q0 + 128))
  for (int window = 1; window <= 600; window += 37)
    for (int n_sink = 0; n_sink <= 20; ++n_sink)
      for (int q0 = 0; q0 < 2000; q0 += 128) {
        if (!sk::sink_only_tile(0, q0, 128, n_sink, window)) continue;
        for (int qi = q0; qi < q0 + 128; ++qi)
          for (int kj = 0; kj < 128; ++kj)
            if (sk::visible_elem(qi, kj, 4096, 1, n_sink, window) != (kj < n_sink)) {
              std::printf("sink-only tile q0=%d window=%d n_sink=%d qi=%d kj=%d\n", q0, window,
                          n_sink, qi, kj);
              return 1;
            }
        ++checked;
      }
  std::printf("ok %lld\n", checked);
  return 0;
}
