// Host-only check of the streaming decode's static schedule (no kernel is
// launched): for many problem shapes, every warp run stays within the
// launched warps and no (sequence, KV head) pair is cut into more runs than
// the partial slots the workspace holds, which is what keeps the kernel's
// partial writes inside the workspace.  Prints "ok" or the first failure.
#include <cstdio>

#include "../../learnable_sink_b200/csrc/internal.h"

int main() {
  const long long Bs[] = {1, 2, 5, 32, 100, 1100, 4096};
  const long long Hkvs[] = {1, 2, 8};
  const long long Ss[] = {1, 15, 16, 17, 64, 1024, 3000, 100004};
  const int Ns[] = {1, 2, 3, 6, 7, 40, 97, 128};
  const long long Ws[] = {8, 1184, 2048};
  long long checked = 0;
  for (long long B : Bs)
    for (long long Hkv : Hkvs)
      for (long long S : Ss)
        for (int N0 : Ns)
          for (long long Wmax : Ws) {
            const int N = sk::decode_clamp_splits(N0, 0, (int)S);
            const sk::DecSchedule d = sk::decode_schedule(B, Hkv, S, N, Wmax);
            if (d.n_warps > Wmax || d.ppw < 1) {
              std::printf("too many warps B=%lld Hkv=%lld S=%lld N=%d W=%lld: %lld\n", B, Hkv, S,
                          N, Wmax, d.n_warps);
              return 1;
            }
            for (long long pair = 0; pair < B * Hkv; pair += (B * Hkv > 64 ? 37 : 1)) {
              const long long F = pair * d.np_max;
              const long long runs = (F + d.np_max - 1) / d.ppw - F / d.ppw + 1;
              if (runs > N) {
                std::printf("pair %lld cut into %lld runs > %d (B=%lld Hkv=%lld S=%lld W=%lld)\n",
                            pair, runs, N, B, Hkv, S, Wmax);
                return 1;
              }
              ++checked;
            }
          }
  std::printf("ok %lld\n", checked);
  return 0;
}
