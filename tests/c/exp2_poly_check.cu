// Error of the FMA-pipe exp2 (exp2_poly) against the exact 2^y, on the
// host (the same fp32 operations the kernels run per element): relative
// error over y in [-126, 8], exact zero for live = 0.  Prints "ok <max rel
// err>" or the first failure.
#include <cmath>
#include <cstdio>

#include "../../learnable_sink_b200/csrc/common.cuh"

int main() {
  double worst = 0.0;
  for (long i = 0; i <= 2000000; ++i) {
    const float y = -126.0f + 134.0f * float(i) / 2000000.0f;
    const double ref = std::exp2(double(y));
    const double got = double(sk::exp2_poly(y, 1.0f));
    const double rel = std::fabs(got - ref) / ref;
    if (!(rel <= 1e-4)) {
      std::printf("y=%.9g got %.9g ref %.9g rel %.3g\n", y, got, ref, rel);
      return 1;
    }
    if (rel > worst) worst = rel;
  }
  // far below the clamp: a tiny positive value, never a wrapped exponent
  const float tiny = sk::exp2_poly(-1000.0f, 1.0f);
  if (!(tiny > 0.0f && tiny < 1e-37f)) { std::printf("clamp %g\n", tiny); return 1; }
  if (sk::exp2_poly(-INFINITY, 1.0f) > 1e-37f) { std::printf("-inf\n"); return 1; }
  if (sk::exp2_poly(3.0f, 0.0f) != 0.0f || sk::exp2_poly(-INFINITY, 0.0f) != 0.0f) {
    std::printf("live = 0\n");
    return 1;
  }
  std::printf("ok %.3g\n", worst);
  return 0;
}
