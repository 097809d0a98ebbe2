// Page scoring from plain loads on the warp-level tensor cores: the bf16
// scoring kernel (instantiated in route.cu) and the page walk that the E4M3
// scoring kernel (route_fp8.cu) shares with it.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {
namespace {

__device__ __forceinline__ int clamp_len(int T, int max_seq_len, unsigned int* status,
                                         bool report) {
  if (T < 0 || T > max_seq_len) {
    if (report) raise_status(status, BASISKV_DEV_BAD_LENGTH);
    T = T < 0 ? 0 : max_seq_len;
  }
  return T;
}

// A warp's contiguous range of pages in (sequence, KV head, logical page)
// order, skipping pages past each sequence's length, with a 32-entry window
// of the block table per lane: the next window is requested as soon as one
// opens, so walking a sequence's pages never waits on the table.
template <int S>
struct PageWalk {
  const int32_t* seq_lens;
  const int32_t* block_table;
  unsigned int* status;
  int Hkv, max_pages, max_seq_len, len_offset, lane, P_max;
  long u, u_end;
  int bg, lp, b, g, T, P;
  int win_b, win_base, tb_cur, tb_nxt;

  __device__ __forceinline__ PageWalk(const RouteArgs& a, long wid, long nw, int lane_)
      : seq_lens(a.seq_lens), block_table(a.block_table), status(a.status), Hkv(a.Hkv),
        max_pages(a.max_pages), max_seq_len(a.max_seq_len), len_offset(a.len_offset),
        lane(lane_), bg(0), lp(0), b(0), g(0), T(0), P(0), win_b(-1), win_base(0), tb_cur(0),
        tb_nxt(0) {
    P_max = (max_seq_len + S - 1) / S;
    const long total = (long)a.B * Hkv * P_max;
    u = total * wid / nw;
    u_end = total * (wid + 1) / nw;
    if (u < u_end) {
      bg = (int)(u / P_max);
      lp = (int)(u - (long)bg * P_max);
      b = bg / Hkv;
      g = bg - b * Hkv;
      T = clamp_len(seq_lens[b] + len_offset, max_seq_len, status, lane == 0 && lp == 0);
      P = (T + S - 1) / S;
    }
  }
  __device__ __forceinline__ bool more() const { return u < u_end; }
  __device__ __forceinline__ void advance() {
    ++u;
    if (++lp == P_max) {
      lp = 0;
      ++bg;
      if (++g == Hkv) {
        g = 0;
        ++b;
        if (u < u_end) {
          T = clamp_len(seq_lens[b] + len_offset, max_seq_len, status, lane == 0);
          P = (T + S - 1) / S;
        }
      }
    }
  }
  // to the next page inside its sequence's length
  __device__ __forceinline__ void skip() {
    while (u < u_end && lp >= P) {
      u += P_max - 1 - lp;
      lp = P_max - 1;
      advance();
    }
  }
  __device__ __forceinline__ int tbl(int bb, int i) const {
    return i < max_pages ? __ldg(block_table + (size_t)bb * max_pages + i) : 0;
  }
  // Physical page of logical page l of sequence bb (warp-uniform arguments).
  __device__ __forceinline__ int page_of(int bb, int l) {
    if (bb != win_b || l < win_base || l >= win_base + 32) {
      if (bb == win_b && l >= win_base + 32 && l < win_base + 64) {
        tb_cur = tb_nxt;
        win_base += 32;
      } else {
        win_b = bb;
        win_base = l;
        tb_cur = tbl(bb, l + lane);
      }
      tb_nxt = tbl(bb, win_base + 32 + lane);
    }
    return __shfl_sync(0xffffffffu, tb_cur, l - win_base);
  }
};

// -------------------------------------- page scoring, plain loads + MMA
// The same scores without TMA or a staging ring: one warp scores one page
// at a time straight from plain 16-byte global loads (PW pages per batch,
// all loads of a batch in flight before any math).  Lane (r = lane/4,
// c = lane%4) loads, for each 8-token tile of the page and each 32-column
// chunk of a token row ([z | e]), the 8 bf16 at columns 32k + 8c of token r:
// whole 32-byte sectors, 8 rows x 64 contiguous bytes per instruction.
//
// Those 16 bytes are the B operand (two k-steps) of mma.m16n8k16, with the
// token as the N index and the row's columns taken in the order the lanes
// hold them (a contraction does not care about the order of its index; the A
// operand uses the same order).  A holds the folded queries of the group,
// each fp32 value split into three bf16 parts (hi, mid, lo: about 24
// significant bits) on separate rows, so the fp32 accumulators hold every
// (part, head) x token dot product of exact bf16 x bf16 products; the parts
// are added in fp32 and the page maximum is a warp reduction.  A token past
// the length only reaches its own accumulator column, which is masked.
constexpr int kRmThreads = 256;
constexpr int kRmWarps = kRmThreads / 32;

// CTAs per SM: three (at most 85 registers a thread) when one page's loads
// and accumulators fit, else two.  Measured at the 32K-context, B = 16
// Llama-8B shape: one page in flight per warp with 24 warps per SM beats two
// pages per warp with 16 warps (136 vs 153 us for fold + scoring + select),
// and four CTAs per SM at 64 registers (fold + scoring 130.4 vs 135.7 us).
template <int G, int RB, int RQ, int S>
__host__ __device__ constexpr int rm_ctas_per_sm() {
  return (S / 8) * ((RB + 31) / 32 + (RQ + 31) / 32) * 4 + (S / 8) * (G == 8 ? 2 : 1) * 4 <= 40
             ? 3
             : 2;
}

// A-operand row r of row set `set`: the head it holds (-1: a zero row) and
// the part (0 hi, 1 mid, 2 lo).  G = 8: set 0 = hi rows 0-7 and mid rows
// 8-15, set 1 = lo rows 0-7.  G <= 4: hi rows [0, G), lo rows [G, 2G), mid
// rows [8, 8 + G), so a lane holds hi and mid of one head and reads lo from
// the lane 4G above it.
template <int G>
__device__ __forceinline__ void rm_row(int set, int r, int& head, int& part) {
  head = -1;
  part = 0;
  if (G == 8) {
    if (set == 0) {
      head = r & 7;
      part = r >> 3;
    } else if (r < 8) {
      head = r;
      part = 2;
    }
  } else if (r < G) {
    head = r;
  } else if (r < 2 * G) {
    head = r - G;
    part = 2;
  } else if (r >= 8 && r < 8 + G) {
    head = r - 8;
    part = 1;
  }
}

// Part `part` of x in the three-way bf16 split x = hi + mid + lo (each step's
// remainder is exact in fp32).
__device__ __forceinline__ float bf16_part(float x, int part) {
  const float h = __bfloat162float(__float2bfloat16_rn(x));
  if (part == 0) return h;
  const float m = __bfloat162float(__float2bfloat16_rn(x - h));
  return part == 1 ? m : (x - h) - m;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f_to_bf16(lo) | ((uint32_t)f_to_bf16(hi) << 16);
}

// RV, RK: the cache rows' widths (pitches); RB <= RV, RQ <= RK: the columns
// the router reads (multiples of 16).  A row's read columns form chunks of 32
// (lane c loads columns 8c .. 8c+7, 16 bytes: two k-steps of the MMA) and at
// most one 16-column tail chunk (lane c loads columns 4c .. 4c+3, 8 bytes:
// one k-step), so every lane loads and every loaded byte is used.
// RP: the routing page (RP = S: one score per cache page; RP = 4 or 8: the
// router scores every RP tokens of a cache page, S / RP scores a page, the
// scores row of a group holding max_pages * S / RP entries).
template <int G, int RV, int RK, int RB, int RQ, int S, int PW, int RP = S>
__global__ void __launch_bounds__(kRmThreads, (rm_ctas_per_sm<G, RB, RQ, S>()))
    route_mma_kernel(RouteArgs a) {
  static_assert(RP == S || RP == 4 || RP == 8, "routing pages of 4 or 8 tokens, or the page");
  constexpr int NR = S / RP;  // routing pages per cache page
  extern __shared__ uint4 rm_frags[];
  constexpr int NZF = RB / 32, NZH = (RB % 32) / 16, NEF = RQ / 32, NEH = (RQ % 32) / 16;
  constexpr int NCZ = NZF + NZH, NC = NCZ + NEF + NEH, NT = S / 8, RQ_ = RV + RK;
  constexpr int ZP = RB, EP = RQ;  // row pitch of the columns read (== RV, RK when full)
  constexpr int SETS = G == 8 ? 2 : 1;
  const int lane = threadIdx.x & 31, lr = lane >> 2, lc = lane & 3;
  const long wid = (long)blockIdx.x * kRmWarps + (threadIdx.x >> 5);
  const long nw = (long)gridDim.x * kRmWarps;
  // The grid-dependency wait comes only before the folded queries are read:
  // the lengths, the block table and the caches are not written by the fold
  // launch this kernel follows, so the first pages are requested while it
  // finishes.

  // Work: pages (sequence, KV head, logical page) in that order; warp wid
  // takes a contiguous range.  Pages past a sequence's length are skipped.
  PageWalk<S> w(a, wid, nw, lane);
  if (!w.more()) return;

  // A fragments of the current group, per warp in shared memory:
  // [set][chunk][k-step][lane] -> (a0, a1, a2, a3).  Each lane writes and
  // reads only its own entries.
  uint4* qa = rm_frags + (size_t)(threadIdx.x >> 5) * (SETS * NC * 2 * 32) + lane;
  int frag_bg = -1;
  auto load_frags = [&](int bb, int gg) {
    pdl_wait();
    const float* qs = a.qt + ((size_t)bb * a.Hkv + gg) * G * RQ_;
#pragma unroll
    for (int set = 0; set < SETS; ++set) {
      int h0, p0, h1, p1;
      rm_row<G>(set, lr, h0, p0);
      rm_row<G>(set, lr + 8, h1, p1);
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const bool zc = c < NCZ;  // latent chunk, else residual chunk
          const int cc = zc ? c : c - NCZ;
          const bool half = zc ? (NZH && cc == NZF) : (NEH && cc == NEF);
          const bool live = !(half && k == 1);  // a 16-column chunk has one k-step
          const int col = (zc ? 0 : RV) + 32 * cc + (half ? 4 * lc : 8 * lc + 4 * k);
          const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 v0 =
              (h0 >= 0 && live) ? *reinterpret_cast<const float4*>(qs + h0 * RQ_ + col) : z4;
          const float4 v1 =
              (h1 >= 0 && live) ? *reinterpret_cast<const float4*>(qs + h1 * RQ_ + col) : z4;
          qa[((set * NC + c) * 2 + k) * 32] =
              make_uint4(pack_bf16x2(bf16_part(v0.x, p0), bf16_part(v0.y, p0)),
                         pack_bf16x2(bf16_part(v1.x, p1), bf16_part(v1.y, p1)),
                         pack_bf16x2(bf16_part(v0.z, p0), bf16_part(v0.w, p0)),
                         pack_bf16x2(bf16_part(v1.z, p1), bf16_part(v1.w, p1)));
        }
    }
  };

  w.skip();
  while (w.more()) {
    uint4 x[PW][NT][NC];
    int ubg[PW], ub[PW], ug[PW], ulp[PW], uT[PW];
    bool uok[PW];
#pragma unroll
    for (int k = 0; k < PW; ++k) {  // issue every load of the batch
      uok[k] = w.more();
      ubg[k] = w.bg;
      ub[k] = w.b;
      ug[k] = w.g;
      ulp[k] = w.lp;
      uT[k] = w.T;
      if (uok[k]) {
        int pp = w.page_of(w.b, w.lp);
        if (pp < 0 || pp >= a.num_phys) {
          if (lane == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
          pp = 0;  // the page's score is flagged garbage
        }
        // a narrow router's columns lead each tile: [S][RB] then the rest
        const size_t tile = (size_t)pp * a.Hkv + w.g;
        const uint16_t* zr = a.Z + tile * S * RV + lr * ZP + 8 * lc;
        const uint16_t* er = a.E + tile * S * RK + lr * EP + 8 * lc;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
#pragma unroll
          for (int c = 0; c < NCZ; ++c) {
            if (NZH && c == NZF) {
              ldg_stream8(x[k][t][c], zr - 4 * lc + t * 8 * ZP + 32 * c);
            } else {
              x[k][t][c] = ldg_stream(zr + t * 8 * ZP + 32 * c);
            }
          }
#pragma unroll
          for (int c = NCZ; c < NC; ++c) {
            if (NEH && c - NCZ == NEF) {
              ldg_stream8(x[k][t][c], er - 4 * lc + t * 8 * EP + 32 * (c - NCZ));
            } else {
              x[k][t][c] = ldg_stream(er + t * 8 * EP + 32 * (c - NCZ));
            }
          }
        }
        w.advance();
        w.skip();
      }
    }
    // This lane's maximum over page k's live tokens and the group's heads
    // (the warp reduction follows); with routing pages smaller than 8
    // tokens, per 8-token tile instead (tbest[t]).
    float tbest[NT];
    auto page_best = [&](int k) -> float {
      float acc[NT][SETS][4];
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int set = 0; set < SETS; ++set)
          acc[t][set][0] = acc[t][set][1] = acc[t][set][2] = acc[t][set][3] = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int set = 0; set < SETS; ++set) {
          const uint4 f0 = qa[((set * NC + c) * 2 + 0) * 32];
          const uint4 f1 = qa[((set * NC + c) * 2 + 1) * 32];
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            mma_bf16_16816(acc[t][set], f0.x, f0.y, f0.z, f0.w, x[k][t][c].x, x[k][t][c].y);
            const bool half = c < NCZ ? (NZH && c == NZF) : (NEH && c - NCZ == NEF);
            if (!half)
              mma_bf16_16816(acc[t][set], f1.x, f1.y, f1.z, f1.w, x[k][t][c].z, x[k][t][c].w);
          }
        }
      float best = -INFINITY;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float s0, s1;  // tokens 2c and 2c + 1 of the tile, head r
        if (G == 8) {
          s0 = acc[t][0][0] + (acc[t][0][2] + acc[t][SETS - 1][0]);
          s1 = acc[t][0][1] + (acc[t][0][3] + acc[t][SETS - 1][1]);
        } else {
          const float lo0 = __shfl_down_sync(0xffffffffu, acc[t][0][0], 4 * G);
          const float lo1 = __shfl_down_sync(0xffffffffu, acc[t][0][1], 4 * G);
          s0 = lr < G ? acc[t][0][0] + (acc[t][0][2] + lo0) : -INFINITY;
          s1 = lr < G ? acc[t][0][1] + (acc[t][0][3] + lo1) : -INFINITY;
        }
        const int tok = ulp[k] * S + t * 8 + 2 * lc;
        float tb = -INFINITY;
        if (tok < uT[k]) tb = s0;
        if (tok + 1 < uT[k]) tb = fmaxf(tb, s1);
        tbest[t] = tb;
        best = fmaxf(best, tb);
      }
      return best;
    };
    // The scores of the routing pages of page k (RP < S): tile t's maximum
    // over the lanes that hold tokens of the same routing page (RP = 4:
    // lanes with equal c >> 1; RP = 8: the whole warp), written by one lane
    // per routing page.
    auto routing_scores = [&](int k) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float v = tbest[t];
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
        if (RP == 8) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        const int sub = RP == 8 ? t : 2 * t + (lc >> 1);
        if (lr == 0 && (RP == 8 ? lc == 0 : (lc & 1) == 0))
          a.scores[(size_t)ubg[k] * a.max_pages * NR + (size_t)ulp[k] * NR + sub] = v;
      }
    };
    bool one_group = true;
#pragma unroll
    for (int k = 1; k < PW; ++k) one_group = one_group && (!uok[k] || ubg[k] == ubg[0]);
    if (NR > 1) {  // routing pages smaller than the cache page: scored one page at a time
#pragma unroll
      for (int k = 0; k < PW; ++k) {
        if (!uok[k]) continue;
        if (ubg[k] != frag_bg) {
          load_frags(ub[k], ug[k]);
          frag_bg = ubg[k];
        }
        (void)page_best(k);
        routing_scores(k);
      }
    } else if (one_group) {  // the common case: the batch's pages are scored side by side
      if (ubg[0] != frag_bg) {
        load_frags(ub[0], ug[0]);
        frag_bg = ubg[0];
      }
      float best[PW];
#pragma unroll
      for (int k = 0; k < PW; ++k) best[k] = uok[k] ? page_best(k) : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < PW; ++k)
          best[k] = fmaxf(best[k], __shfl_xor_sync(0xffffffffu, best[k], o));
      if (lane == 0)
#pragma unroll
        for (int k = 0; k < PW; ++k)
          if (uok[k]) a.scores[(size_t)ubg[k] * a.max_pages + ulp[k]] = best[k];
    } else {  // the batch crosses a group boundary
#pragma unroll
      for (int k = 0; k < PW; ++k) {
        if (!uok[k]) continue;
        if (ubg[k] != frag_bg) {
          load_frags(ub[k], ug[k]);
          frag_bg = ubg[k];
        }
        const float best = warp_max(page_best(k));
        if (lane == 0) a.scores[(size_t)ubg[k] * a.max_pages + ulp[k]] = best;
      }
    }
  }
}

// Pages a warp loads before scoring them: the full-width router keeps one
// page (24 load registers at r_v 64) in flight with 24 warps per SM; a narrow
// router's pages are a few registers each, so a warp batches more of them to
// keep about as many bytes in flight.
template <int RB, int RQ, int S>
constexpr int rm_pages_per_batch() {
  return (S / 8) * (4 * (RB / 32 + RQ / 32) + 2 * ((RB % 32) / 16 + (RQ % 32) / 16)) <= 8
             ? 3
             : ((S / 8) * (4 * (RB / 32 + RQ / 32) + 2 * ((RB % 32) / 16 + (RQ % 32) / 16)) <= 12
                    ? 2
                    : 1);
}

template <int G, int RV, int RK, int RB, int RQ, int S, int RP = S>
cudaError_t launch_route_mma(const RouteArgs& a, cudaStream_t st, bool pdl) {
  constexpr int PW = rm_pages_per_batch<RB, RQ, S>();
  constexpr int NC = (RB + 31) / 32 + (RQ + 31) / 32;
  const int P_max = (a.max_seq_len + S - 1) / S;
  const long pages = (long)a.B * a.Hkv * P_max;
  long grid = (long)num_sms() * rm_ctas_per_sm<G, RB, RQ, S>();
  const long need = (pages + kRmWarps - 1) / kRmWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  const size_t smem = (size_t)kRmWarps * (G == 8 ? 2 : 1) * NC * 2 * 32 * 16;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_mma_kernel<G, RV, RK, RB, RQ, S, PW, RP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(route_mma_kernel<G, RV, RK, RB, RQ, S, PW, RP>, dim3((unsigned)grid),
                  dim3(kRmThreads), smem, st, pdl, a);
}

}  // namespace
}  // namespace basiskv
