// bf16-cache instances of the fused selection + attention kernel
// (select_attend.cuh) and the host-side choice of its cluster size.
#include "select_attend.cuh"

namespace basiskv {

int select_attend_cluster_size(int G, int d, int r_v, int S, int rp, int fp8, int B, int Hkv,
                               int max_seq_len, int top_k) {
  if (fp8 ? !attend_mma_fp8_supported(G, d, r_v, S) : !attend_mma_supported(G, d, r_v, S))
    return 0;
  const int P_max = (max_seq_len + rp - 1) / rp;  // routing pages
  return select_attend_cluster(G, d, r_v, fp8 != 0, B, Hkv, P_max, top_k, num_sms());
}

cudaError_t launch_select_attend(const SelectArgs& s, const AttendArgs& a, cudaStream_t st,
                                 bool pdl) {
  if (a.fp8) return launch_select_attend_fp8(s, a, st, pdl);
  if (!attend_mma_supported(a.G, a.d, a.r_v, a.S)) return cudaErrorNotSupported;
#define BKV_SA_RV(GG, DD)                                                   \
  switch (a.r_v) {                                                          \
    case 32: return launch_select_attend_t<GG, DD, 32>(s, a, st, pdl);      \
    case 64: return launch_select_attend_t<GG, DD, 64>(s, a, st, pdl);      \
    case 96: return launch_select_attend_t<GG, DD, 96>(s, a, st, pdl);      \
    default: return launch_select_attend_t<GG, DD, 128>(s, a, st, pdl);     \
  }
#define BKV_SA(GG)                 \
  case GG:                         \
    if (a.d == 64) {               \
      BKV_SA_RV(GG, 64)            \
    } else {                       \
      BKV_SA_RV(GG, 128)           \
    }
  switch (a.G) {
    BKV_SA(1)
    BKV_SA(2)
    BKV_SA(4)
    BKV_SA(8)
    default: return cudaErrorNotSupported;
  }
#undef BKV_SA
#undef BKV_SA_RV
}

}  // namespace basiskv
