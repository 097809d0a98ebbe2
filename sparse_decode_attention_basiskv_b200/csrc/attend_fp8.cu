// Attention over E4M3 caches: the instances of the plain-load attention
// kernel that read one byte per cached Key and latent column (the caches
// stored as FP8 E4M3, as in Table 13 of the BasisKV pages).
#include "attend_mma.cuh"
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

bool attend_mma_fp8_supported(int G, int d, int r_v, int S) {
  return (G == 4 || G == 8) && attend_mma_supported(G, d, r_v, S);
}

cudaError_t launch_attend_mma_fp8(const AttendArgs& a, cudaStream_t st, bool pdl) {
  if (!attend_mma_fp8_supported(a.G, a.d, a.r_v, a.S) || !a.cnt) return cudaErrorNotSupported;
#define BKV_AM8_RV(GG, DD)                                                 \
  switch (a.r_v) {                                                         \
    case 32: return launch_attend_mma_t<GG, DD, 32, true>(a, st, pdl);     \
    case 64: return launch_attend_mma_t<GG, DD, 64, true>(a, st, pdl);     \
    case 96: return launch_attend_mma_t<GG, DD, 96, true>(a, st, pdl);     \
    default: return launch_attend_mma_t<GG, DD, 128, true>(a, st, pdl);    \
  }
  if (a.G == 4) {
    if (a.d == 64) {
      BKV_AM8_RV(4, 64)
    } else {
      BKV_AM8_RV(4, 128)
    }
  } else {
    if (a.d == 64) {
      BKV_AM8_RV(8, 64)
    } else {
      BKV_AM8_RV(8, 128)
    }
  }
#undef BKV_AM8_RV
}

}  // namespace basiskv
