// Page scoring over E4M3 caches: the instances of the plain-load scoring
// kernel that read one byte per cached column (the latent and residual
// caches stored as FP8 E4M3, as in Table 13 of the BasisKV pages).
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "route_mma.cuh"

namespace basiskv {

// Routers with an E4M3 instance: the full-width shapes of the bf16 kernel
// and the narrow ones (widths 16 or 32 each), with (G, S) in {(4, 16),
// (8, 32)} for the narrow ones.
#define BKV_RM8_LIST(X)                                                                   \
  X(4, 64, 32, 64, 32, 16) X(4, 96, 32, 96, 32, 16) X(4, 128, 32, 128, 32, 16)            \
  X(4, 64, 32, 64, 32, 32) X(4, 96, 32, 96, 32, 32) X(8, 64, 32, 64, 32, 16)              \
  X(8, 96, 32, 96, 32, 16) X(8, 128, 32, 128, 32, 16) X(8, 64, 32, 64, 32, 32)            \
  X(8, 96, 32, 96, 32, 32) X(8, 128, 32, 128, 32, 32)                                     \
  X(4, 64, 32, 16, 16, 16) X(4, 64, 32, 16, 32, 16) X(4, 64, 32, 32, 16, 16)              \
  X(4, 64, 32, 32, 32, 16) X(4, 96, 32, 16, 16, 16) X(4, 96, 32, 16, 32, 16)              \
  X(4, 96, 32, 32, 16, 16) X(4, 96, 32, 32, 32, 16) X(8, 64, 32, 16, 16, 32)              \
  X(8, 64, 32, 16, 32, 32) X(8, 64, 32, 32, 16, 32) X(8, 64, 32, 32, 32, 32)              \
  X(8, 96, 32, 16, 16, 32) X(8, 96, 32, 16, 32, 32) X(8, 96, 32, 32, 16, 32)              \
  X(8, 96, 32, 32, 32, 32)

bool route_fp8_supported(int G, int r_v, int r_k, int rb, int rq, int S) {
#define BKV_RM8Q(GG, V, K, RB_, RQ_, SS) \
  if (G == GG && r_v == V && r_k == K && rb == RB_ && rq == RQ_ && S == SS) return true;
  BKV_RM8_LIST(BKV_RM8Q)
#undef BKV_RM8Q
  return false;
}

cudaError_t launch_route_scores_fp8(const RouteArgs& a, cudaStream_t st, bool pdl) {
  if (!(a.Z && a.E)) return cudaErrorNotSupported;
#define BKV_RM8(GG, V, K, RB_, RQ_, SS)                                                   \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.rb == RB_ && a.rq == RQ_ && a.S == SS) \
    return launch_route_mma<GG, V, K, RB_, RQ_, SS, true>(a, st, pdl);
  BKV_RM8_LIST(BKV_RM8)
#undef BKV_RM8
  return cudaErrorNotSupported;
}

}  // namespace basiskv
