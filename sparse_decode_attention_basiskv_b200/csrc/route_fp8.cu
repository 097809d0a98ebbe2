// Page scoring over E4M3 caches (the latent and residual caches stored as
// FP8 E4M3, the KV format of Table 13 of the BasisKV pages).
//
// Same scores as the bf16 plain-load kernel (route_mma.cuh), laid out for
// one byte per cached column:
// - Lane (r = lane/4, c = lane%4) loads, per 8-token tile of a page and per
//   32-column chunk of a token row, the 8 bytes at columns 32k + 8c of token
//   r (a 16-column chunk: 4 bytes at 4c); the bytes are widened to f16
//   exactly.
// - Tokens are the M index of mma.m16n8k16 (f16 operands, fp32 accumulate):
//   tiles 2m and 2m + 1 of the page are rows r and r + 8 of M-tile m, the
//   columns taken in the order the lanes hold them.  B holds the group's
//   folded queries, column n of N-tile j = head 4j + n/2, part n%2: each
//   fp32 value split into f16 hi + lo after scaling the group by a power of
//   two that brings its largest magnitude into [2^14, 2^15) (both parts stay
//   in the f16 normal range; the scale is divided out of the page maximum,
//   exactly).  A lane's accumulators (columns 2c, 2c + 1) are the hi and lo
//   parts of one head for tokens r and r + 8, so the score is their sum.
// - Each warp keeps two batches of pages in flight: the next batch is
//   requested (into registers) before the current one is scored.  (A ring
//   of pages in shared memory filled by 8-byte cp.async copies measured
//   slower: 100 vs 81 us at the 32K-context, B = 16 Llama-8B shape.)
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "route_mma.cuh"

namespace basiskv {

namespace {

constexpr int kR8Threads = 256;
constexpr int kR8Warps = kR8Threads / 32;

// Load registers of one page per lane: 2 per 32-column chunk and 1 per
// 16-column chunk, per 8-token tile.
template <int RB, int RQ, int S>
constexpr int r8_page_regs() {
  return (S / 8) * (2 * (RB / 32 + RQ / 32) + (RB % 32) / 16 + (RQ % 32) / 16);
}
// Pages per batch: one, or two while a batch stays within 16 load
// registers (two batches are in flight).
template <int RB, int RQ, int S>
constexpr int r8_pages_per_batch() {
  return r8_page_regs<RB, RQ, S>() <= 8 ? 2 : 1;
}
// CTAs per SM from the registers a lane holds for two batches and its
// accumulators: four (64 registers a thread) up to 28 for the full-width
// routers, three up to 40.  Measured at the 32K-context, B = 16 Llama-8B
// shape (28): four CTAs 77.9 us, three 81.1 us; the narrow routers' batch
// bookkeeping spills at 64 registers.
template <int RB, int RQ, int S, int G>
constexpr int r8_live_regs() {
  return 2 * r8_pages_per_batch<RB, RQ, S>() * r8_page_regs<RB, RQ, S>() + (S / 16) * (G / 4) * 4;
}
template <int G, int RB, int RQ, int S>
constexpr int r8_ctas_per_sm() {
  return (RB >= 64 && r8_live_regs<RB, RQ, S, G>() <= 28)
             ? 4
             : (r8_live_regs<RB, RQ, S, G>() <= 40 ? 3 : 2);
}

// RP: the routing page (RP = S: one score per cache page; RP = 4 or 8: a
// score for every RP tokens of a cache page, the scores row of a group
// holding max_pages * S / RP entries).
template <int G, int RV, int RK, int RB, int RQ, int S, int PW, int RP = S>
__global__ void __launch_bounds__(kR8Threads, (r8_ctas_per_sm<G, RB, RQ, S>()))
    route_f8_kernel(RouteArgs a) {
  static_assert((G == 4 || G == 8) && S % 16 == 0, "E4M3 scoring shapes");
  static_assert(RP == S || RP == 4 || RP == 8, "routing pages of 4 or 8 tokens, or the page");
  constexpr int NR = S / RP;  // routing pages per cache page
  extern __shared__ uint2 r8_frags[];
  constexpr int NZF = RB / 32, NZH = (RB % 32) / 16, NEF = RQ / 32, NEH = (RQ % 32) / 16;
  constexpr int NCZ = NZF + NZH, NC = NCZ + NEF + NEH, NT = S / 8, NM = S / 16, NJ = G / 4;
  constexpr int RQ_ = RV + RK, ZP = RB, EP = RQ;
  const int lane = threadIdx.x & 31, lr = lane >> 2, lc = lane & 3, warp = threadIdx.x >> 5;
  const long wid = (long)blockIdx.x * kR8Warps + warp;
  const long nw = (long)gridDim.x * kR8Warps;

  // Work: pages (sequence, KV head, logical page) in that order; warp wid
  // takes a contiguous range; pages past a sequence's length are skipped.
  // The lengths, block table and caches are not written by the launch this
  // kernel follows; the grid-dependency wait comes before the folded
  // queries are read.
  PageWalk<S> w(a, wid, nw, lane);
  if (!w.more()) return;

  // B fragments of the current group, per warp in shared memory:
  // [chunk][k-step][N-tile][lane] -> (b0, b1); each lane writes and reads
  // only its own entries.
  uint2* qb = r8_frags + (size_t)warp * (NC * 2 * NJ * 32) + lane;
  int frag_bg = -1;
  float qscale_inv = 1.f;
  auto load_frags = [&](int gbg) {  // group (sequence, KV head) gbg
    pdl_wait();
    const float* qs = a.qt + (size_t)gbg * G * RQ_;
    // four consecutive values of head 4j + r/2 at this lane's columns
    auto qv = [&](int c, int k, int j) -> float4 {
      const bool zc = c < NCZ;
      const int cc = zc ? c : c - NCZ;
      const bool half = zc ? (NZH && cc == NZF) : (NEH && cc == NEF);
      if (half && k == 1) return make_float4(0.f, 0.f, 0.f, 0.f);
      const int col = (zc ? 0 : RV) + 32 * cc + (half ? 4 * lc : 8 * lc + 4 * k);
      return *reinterpret_cast<const float4*>(qs + (4 * j + (lr >> 1)) * RQ_ + col);
    };
    float m = 0.f;  // the lanes cover every read column of every head
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float4 v = qv(c, k, j);
          m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
    m = warp_max(m);
    // m = f 2^ex with f in [1/2, 1): scale 2^(15 - ex), within the normal
    // fp32 powers of two
    const int ex = m > 0.f ? (int)((__float_as_uint(m) >> 23) & 0xffu) - 126 : 15;
    const int sh = max(-126, min(126, 15 - ex));
    const float sc = __uint_as_float((uint32_t)(127 + sh) << 23);
    qscale_inv = __uint_as_float((uint32_t)(127 - sh) << 23);
#pragma unroll 1
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float4 v = qv(c, k, j);
          uint32_t h01, l01, h23, l23;
          split_f16x2(v.x * sc, v.y * sc, h01, l01);
          split_f16x2(v.z * sc, v.w * sc, h23, l23);
          qb[((c * 2 + k) * NJ + j) * 32] = (lr & 1) ? make_uint2(l01, l23) : make_uint2(h01, h23);
        }
  };

  struct Batch {  // per page: group, logical page, live tokens (0: no page)
    int bg[PW], lp[PW], nv[PW];
  };
  // Requests every load of the next PW pages into x.
  auto issue = [&](Batch& bt, uint2 (&x)[PW][NT][NC]) {
#pragma unroll
    for (int k = 0; k < PW; ++k) {
      bt.bg[k] = w.bg;
      bt.lp[k] = w.lp;
      bt.nv[k] = w.more() ? min(S, w.T - w.lp * S) : 0;
      if (bt.nv[k] > 0) {
        int pp = w.page_of(w.b, w.lp);
        if (pp < 0 || pp >= a.num_phys) {
          if (lane == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
          pp = 0;  // the page's score is flagged garbage
        }
        // a narrow router's columns lead each tile: [S][RB] then the rest
        const size_t tile = (size_t)pp * a.Hkv + w.g;
        const uint8_t* zr =
            reinterpret_cast<const uint8_t*>(a.Z) + tile * S * RV + lr * ZP + 8 * lc;
        const uint8_t* er =
            reinterpret_cast<const uint8_t*>(a.E) + tile * S * RK + lr * EP + 8 * lc;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
#pragma unroll
          for (int c = 0; c < NCZ; ++c) {
            if (NZH && c == NZF)
              ldg_stream4(x[k][t][c], zr - 4 * lc + t * 8 * ZP + 32 * c);
            else
              ldg_stream8(x[k][t][c], zr + t * 8 * ZP + 32 * c);
          }
#pragma unroll
          for (int c = NCZ; c < NC; ++c) {
            if (NEH && c - NCZ == NEF)
              ldg_stream4(x[k][t][c], er - 4 * lc + t * 8 * EP + 32 * (c - NCZ));
            else
              ldg_stream8(x[k][t][c], er + t * 8 * EP + 32 * (c - NCZ));
          }
        }
        w.advance();
        w.skip();
      }
    }
  };
  // This lane's maximum over page k's live tokens and the group's heads;
  // tbest[m][h] keeps it per token (16 m + r + 8 h) for routing pages.
  float tbest[NM][2];
  auto page_best = [&](const Batch& bt, uint2 (&x)[PW][NT][NC], int k) -> float {
    float acc[NM][NJ][4];
#pragma unroll
    for (int mt = 0; mt < NM; ++mt)
#pragma unroll
      for (int j = 0; j < NJ; ++j) acc[mt][j][0] = acc[mt][j][1] = acc[mt][j][2] = acc[mt][j][3] = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const bool half = c < NCZ ? (NZH && c == NZF) : (NEH && c - NCZ == NEF);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        if (half && ks == 1) continue;
        uint2 bq[NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) bq[j] = qb[((c * 2 + ks) * NJ + j) * 32];
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) {
          uint32_t a0, a2, a1, a3;  // tile 2mt (rows r), tile 2mt + 1 (rows r + 8)
          e4m3x4_to_f16(ks ? x[k][2 * mt][c].y : x[k][2 * mt][c].x, a0, a2);
          e4m3x4_to_f16(ks ? x[k][2 * mt + 1][c].y : x[k][2 * mt + 1][c].x, a1, a3);
#pragma unroll
          for (int j = 0; j < NJ; ++j) mma_f16_16816(acc[mt][j], a0, a1, a2, a3, bq[j].x, bq[j].y);
        }
      }
    }
    float best = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < NM; ++mt) {
      const int tok = 16 * mt + lr;  // within the page
      float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (tok < bt.nv[k]) t0 = fmaxf(t0, acc[mt][j][0] + acc[mt][j][1]);
        if (tok + 8 < bt.nv[k]) t1 = fmaxf(t1, acc[mt][j][2] + acc[mt][j][3]);
      }
      tbest[mt][0] = t0;
      tbest[mt][1] = t1;
      best = fmaxf(best, fmaxf(t0, t1));
    }
    return best * qscale_inv;
  };
  // The scores of page k's routing pages (RP < S): token 16 m + r + 8 h
  // lies in routing page (16 m + 8 h + r) / RP, held by the lanes that
  // share r / 4 (RP = 4: lane bit 4) or by the whole warp (RP = 8); one
  // lane per routing page writes it.
  auto routing_scores = [&](const Batch& bt, int k) {
#pragma unroll
    for (int mt = 0; mt < NM; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v = tbest[mt][h];
#pragma unroll
        for (int o = 1; o < (RP == 8 ? 32 : 16); o <<= 1)
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        const int sub = RP == 8 ? 2 * mt + h : 4 * mt + 2 * h + (lane >> 4);
        if (RP == 8 ? lane == 0 : (lane & 15) == 0)
          a.scores[((size_t)bt.bg[k] * a.max_pages + bt.lp[k]) * NR + sub] = v * qscale_inv;
      }
  };
  auto score = [&](const Batch& bt, uint2 (&x)[PW][NT][NC]) {
    bool one_group = true;
#pragma unroll
    for (int k = 1; k < PW; ++k) one_group = one_group && (bt.nv[k] == 0 || bt.bg[k] == bt.bg[0]);
    if (NR > 1) {  // routing pages smaller than the cache page: one page at a time
#pragma unroll
      for (int k = 0; k < PW; ++k) {
        if (bt.nv[k] == 0) continue;
        if (bt.bg[k] != frag_bg) {
          load_frags(bt.bg[k]);
          frag_bg = bt.bg[k];
        }
        (void)page_best(bt, x, k);
        routing_scores(bt, k);
      }
    } else if (one_group) {  // the common case: the batch's pages are scored side by side
      if (bt.bg[0] != frag_bg) {
        load_frags(bt.bg[0]);
        frag_bg = bt.bg[0];
      }
      float best[PW];
#pragma unroll
      for (int k = 0; k < PW; ++k) best[k] = bt.nv[k] > 0 ? page_best(bt, x, k) : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < PW; ++k)
          best[k] = fmaxf(best[k], __shfl_xor_sync(0xffffffffu, best[k], o));
      if (lane == 0)
#pragma unroll
        for (int k = 0; k < PW; ++k)
          if (bt.nv[k] > 0) a.scores[(size_t)bt.bg[k] * a.max_pages + bt.lp[k]] = best[k];
    } else {  // the batch crosses a group boundary
#pragma unroll
      for (int k = 0; k < PW; ++k) {
        if (bt.nv[k] == 0) continue;
        if (bt.bg[k] != frag_bg) {
          load_frags(bt.bg[k]);
          frag_bg = bt.bg[k];
        }
        const float best = warp_max(page_best(bt, x, k));
        if (lane == 0) a.scores[(size_t)bt.bg[k] * a.max_pages + bt.lp[k]] = best;
      }
    }
  };

  w.skip();
  Batch b0, b1;
  uint2 x0[PW][NT][NC], x1[PW][NT][NC];
  issue(b0, x0);
  while (b0.nv[0] > 0) {
    issue(b1, x1);  // in flight while batch 0 is scored
    score(b0, x0);
    if (b1.nv[0] == 0) break;
    issue(b0, x0);
    score(b1, x1);
  }
}

template <int G, int RV, int RK, int RB, int RQ, int S, int RP = S>
cudaError_t launch_route_f8(const RouteArgs& a, cudaStream_t st, bool pdl) {
  constexpr int PW = r8_pages_per_batch<RB, RQ, S>();
  const int P_max = (a.max_seq_len + S - 1) / S;
  const long pages = (long)a.B * a.Hkv * P_max;
  long grid = (long)num_sms() * r8_ctas_per_sm<G, RB, RQ, S>();
  const long need = (pages + kR8Warps - 1) / kR8Warps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  const size_t smem = (size_t)kR8Warps * ((RB + 31) / 32 + (RQ + 31) / 32) * 2 * (G / 4) * 32 * 8;
  return launch_k(route_f8_kernel<G, RV, RK, RB, RQ, S, PW, RP>, dim3((unsigned)grid),
                  dim3(kR8Threads), smem, st, pdl, a);
}

}  // namespace

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

// E4M3 instances with routing pages smaller than the cache page: the
// routers of the bf16 list that have an E4M3 instance.
#define BKV_RM8_SUBPAGE(X)                                                            \
  X(4, 64, 32, 16, 16, 16, 4) X(4, 64, 32, 16, 16, 16, 8) X(4, 96, 32, 16, 16, 16, 4) \
  X(4, 64, 32, 64, 32, 16, 4) X(4, 96, 32, 96, 32, 16, 4) X(8, 96, 32, 16, 16, 32, 4) \
  X(8, 96, 32, 96, 32, 32, 4)

bool route_fp8_subpage_supported(int G, int r_v, int r_k, int rb, int rq, int S, int rp) {
#define BKV_RM8P(GG, V, K, RB_, RQ_, SS, RP_) \
  if (G == GG && r_v == V && r_k == K && rb == RB_ && rq == RQ_ && S == SS && rp == RP_) return true;
  BKV_RM8_SUBPAGE(BKV_RM8P)
#undef BKV_RM8P
  return false;
}

cudaError_t launch_route_scores_fp8(const RouteArgs& a, cudaStream_t st, bool pdl) {
  if (!(a.Z && a.E)) return cudaErrorNotSupported;
  if (a.rp && a.rp != a.S) {  // routing pages smaller than the cache page
#define BKV_RM8P(GG, V, K, RB_, RQ_, SS, RP_)                                               \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.rb == RB_ && a.rq == RQ_ && a.S == SS && \
      a.rp == RP_)                                                                          \
    return launch_route_f8<GG, V, K, RB_, RQ_, SS, RP_>(a, st, pdl);
    BKV_RM8_SUBPAGE(BKV_RM8P)
#undef BKV_RM8P
    return cudaErrorNotSupported;
  }
#define BKV_RM8(GG, V, K, RB_, RQ_, SS)                                                   \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.rb == RB_ && a.rq == RQ_ && a.S == SS) \
    return launch_route_f8<GG, V, K, RB_, RQ_, SS>(a, st, pdl);
  BKV_RM8_LIST(BKV_RM8)
#undef BKV_RM8
  return cudaErrorNotSupported;
}

}  // namespace basiskv
