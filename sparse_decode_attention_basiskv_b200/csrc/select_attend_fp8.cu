// E4M3-cache instances of the fused selection + attention kernel
// (select_attend.cuh): Keys and latents stored as FP8 E4M3 (Table 13 of
// the BasisKV pages), widened to f16 for the tensor cores.
#include "select_attend.cuh"

namespace basiskv {

cudaError_t launch_select_attend_fp8(const SelectArgs& s, const AttendArgs& a, cudaStream_t st,
                                     bool pdl) {
  if (!attend_mma_fp8_supported(a.G, a.d, a.r_v, a.S)) return cudaErrorNotSupported;
#define BKV_SA8_RV(GG, DD)                                                    \
  switch (a.r_v) {                                                            \
    case 32: return launch_select_attend_t<GG, DD, 32, true>(s, a, st, pdl);  \
    case 64: return launch_select_attend_t<GG, DD, 64, true>(s, a, st, pdl);  \
    case 96: return launch_select_attend_t<GG, DD, 96, true>(s, a, st, pdl);  \
    default: return launch_select_attend_t<GG, DD, 128, true>(s, a, st, pdl); \
  }
  if (a.G == 4) {
    if (a.d == 64) {
      BKV_SA8_RV(4, 64)
    } else {
      BKV_SA8_RV(4, 128)
    }
  } else {
    if (a.d == 64) {
      BKV_SA8_RV(8, 64)
    } else {
      BKV_SA8_RV(8, 128)
    }
  }
#undef BKV_SA8_RV
}

}  // namespace basiskv
