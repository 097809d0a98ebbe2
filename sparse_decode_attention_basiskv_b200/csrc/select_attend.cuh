// Page selection and exact attention of a decode step in one launch, one
// thread-block cluster per (sequence, KV head) group (instantiated for bf16
// caches in select_attend.cu and for E4M3 caches in select_attend_fp8.cu).
//
// BasisKV ranks pages with the routing scores and attends exactly over the
// chosen pages only (abstract; Table 4: selected attention reads the exact
// Key and the Value latent).  Each of the C CTAs of a group's cluster:
//   1. reads the length, the group's queries and its block-table row (no
//      earlier launch of the step writes them), then waits for the scores;
//   2. selects the group's pages itself (the exact radix selection of
//      select_block.cuh, into shared memory: the ascending page list is the
//      same in every CTA of the cluster);
//   3. attends over its contiguous share of the selected 16-token units
//      with the warp-level tensor-core loop of the plain-load attention
//      (Keys straight into MMA fragments, latents through a per-warp
//      cp.async ring, online softmax per warp);
//   4. merges its warps into one partial (max, sum, unnormalised latent per
//      head) in its own shared memory;
// and after a cluster barrier every CTA merges one slice of the output
// columns over all C partials, read through distributed shared memory, and
// writes the latent output a.  A second cluster barrier keeps each CTA's
// partial alive until the others have read it.
//
// Compared with a selection launch followed by the attention launch, this
// drops one launch boundary, the round trip of the page ids through global
// memory, and the global arrival count and merge of split partials.  It
// covers steps whose groups fit one wave of CTAs (groups * C <= resident
// CTAs); larger batches keep the two-launch path.
#pragma once

#include <climits>
#include <cooperative_groups.h>

#include "attend_mma.cuh"
#include "select_block.cuh"

namespace basiskv {
namespace {

namespace cg = cooperative_groups;

constexpr int kSaMaxCluster = 8;  // CTAs per group at most (portable cluster size)

__host__ __device__ constexpr size_t sa_align16(size_t x) { return (x + 15) & ~size_t(15); }

// Dynamic shared memory of one CTA.  Region A is used first by the
// selection (keys, radix state) and then by the attention (per-warp latent
// sums and maxima, latent rings); qs, list, tbl and part live throughout.
struct SaLayout {
  size_t sel_state, qs, list, tbl, part, total;
};

__host__ __device__ inline SaLayout sa_layout(int G, int D, int RV, bool F8, int P_max,
                                              int top_k) {
  SaLayout L{};
  const size_t keys = sa_align16((size_t)P_max * 4);
  const size_t sel = keys + sa_align16(sizeof(SelShared));
  const size_t ring = (size_t)2 * (RV / 32) * 2 * 32 * (F8 ? 8 : 16);  // am_ring_bytes
  const size_t att = (size_t)kAmWarps * (G * RV + 16) * 4 + (size_t)kAmWarps * ring;
  L.sel_state = keys;
  size_t off = sa_align16(sel > att ? sel : att);
  L.qs = off;
  off += (size_t)(D / 32) * 32 * 16;
  L.list = off;
  off += sa_align16((size_t)top_k * 4);
  L.tbl = off;
  off += sa_align16((size_t)P_max * 4);
  L.part = off;
  off += sa_align16((size_t)G * (RV + 2) * 4);
  L.total = off;
  return L;
}

// CTAs per group (the cluster size): the largest power of two up to 8 that
// keeps every group's CTAs in one wave of resident CTAs; 0 when the step
// does not fit (one CTA per group is more than a wave, or the shared
// memory of a CTA is too large): the two-launch path then runs.
inline int select_attend_cluster(int G, int D, int RV, bool F8, int B, int Hkv, int P_max,
                                 int top_k, int sms) {
  const SaLayout L = sa_layout(G, D, RV, F8, P_max, top_k);
  if (L.total > 200 * 1024) return 0;
  const int resident = sms * (L.total * kAmCtasPerSm <= 220 * 1024 ? kAmCtasPerSm : 1);
  const int groups = B * Hkv;
  if (groups > resident) return 0;
  int C = 1;
  while (C < kSaMaxCluster && groups * C * 2 <= resident) C *= 2;
  return C;
}

template <int G, int D, int RV, bool F8>
__global__ void __launch_bounds__(kAmThreads, kAmCtasPerSm)
    select_attend_kernel(SelectArgs s, AttendArgs a, int C) {
  constexpr int NKC = D / 32, NZC = RV / 32, RS = RV + 2;
  extern __shared__ __align__(16) uint8_t sa_smem[];
  const int P_max = (s.max_seq_len + s.S - 1) / s.S;
  const SaLayout Ly = sa_layout(G, D, RV, F8, P_max, s.top_k);
  // region A, attention view
  float* wacc = reinterpret_cast<float*>(sa_smem);  // [warp][G][RV]
  float* wml = wacc + kAmWarps * G * RV;             // [warp][16]: m of heads 0-7, then l
  uint8_t* zring_b = reinterpret_cast<uint8_t*>(wml + kAmWarps * 16) +
                     (size_t)(threadIdx.x >> 5) * am_ring_bytes<RV, F8>();
  uint4* zring = reinterpret_cast<uint4*>(zring_b);
  uint2* zring8 = reinterpret_cast<uint2*>(zring_b);
  // region A, selection view
  uint32_t* keys = reinterpret_cast<uint32_t*>(sa_smem);
  SelShared& ss = *reinterpret_cast<SelShared*>(sa_smem + Ly.sel_state);
  uint4* qs = reinterpret_cast<uint4*>(sa_smem + Ly.qs);  // [NKC][lane] query fragments
  int32_t* list = reinterpret_cast<int32_t*>(sa_smem + Ly.list);
  int32_t* tbl = reinterpret_cast<int32_t*>(sa_smem + Ly.tbl);
  float* part = reinterpret_cast<float*>(sa_smem + Ly.part);  // [G][RV + 2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, lr = lane >> 2, lc = lane & 3;
  const int rank = C > 1 ? (int)cg::this_cluster().block_rank() : 0;
  const int bg = blockIdx.x / C, b = bg / a.Hkv, g = bg - b * a.Hkv;
  const int S = a.S, TP = S >> 4, logS = 31 - __clz(S);
  // Routing pages of RPG tokens (the selection's unit); NR per cache page.
  // A 16-token unit is 1 / TP of a routing page of S tokens, or QP routing
  // pages of 4 or 8 tokens.
  const int RPG = a.rp ? a.rp : S, NR = S / RPG, QP = RPG < 16 ? 16 / RPG : 0;
  // every one of these is a power of two: the unit addressing below shifts
  // and masks (TP is 1 or 2 wherever it is used)
  const int logTP = TP >> 1, logNR = 31 - __clz(NR), logRPG = 31 - __clz(RPG);
  const int P_phys = (s.max_seq_len + S - 1) / S;  // block-table entries read

  // The out-projection may take SMs as this grid's CTAs retire; it requests
  // only its weight tiles before its own wait.
  pdl_launch_dependents();
  // No earlier launch of the step writes the length, the queries or the
  // block table: all three are requested before the wait, the queries and
  // the block-table row as asynchronous copies into shared memory (nothing
  // waits for them until the selection is done).
  int T = a.seq_lens[b] + a.len_offset;
  for (int i = tid; i < NKC * 32; i += kAmThreads) {
    const int k = i >> 5, r = (i & 31) >> 2, cc = i & 3;
    if (r < G)
      cp_async16(qs + i, a.q + ((size_t)b * a.Hq + g * G + r) * D + 32 * k + 8 * cc);
    else
      qs[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  {
    const int32_t* row = a.block_table + (size_t)b * a.max_pages;
    for (int i = tid; i < P_phys; i += kAmThreads) cp_async4(tbl + i, row + i);
  }
  cp_async_commit();
  pdl_wait();  // the page scores are the previous launch's output
  select_group<kAmThreads>(s, bg, keys, nullptr, ss, list, nullptr);
  cp_async_wait_all();
  __syncthreads();  // the page list, queries and block-table row are in; region A is free
  T = T < 0 ? 0 : (T > s.max_seq_len ? s.max_seq_len : T);
  const int nsel = min(a.top_k, (T + RPG - 1) / RPG);
  const int U = QP ? (nsel + QP - 1) / QP : nsel * TP;  // units with a page
  const int u0 = (int)((long)U * rank / C), u1 = (int)((long)U * (rank + 1) / C);
  const int count = u0 + warp < u1 ? (u1 - u0 - warp + kAmWarps - 1) / kAmWarps : 0;

  // E4M3: this lane's query fragments as f16 (head lr, scaled) and the
  // score factors of heads 2c, 2c + 1 (log2(e)/sqrt(d) over their scales)
  uint4 qh[F8 ? NKC : 1];
  float sl0 = a.scale_log2, sl1 = a.scale_log2;
  if constexpr (F8) {
    float m = 0.f;
#pragma unroll
    for (int c = 0; c < NKC; ++c) {
      const uint4 r = qs[c * 32 + lane];
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_f2(w[i]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    const int ex = m > 0.f ? (int)((__float_as_uint(m) >> 23) & 0xffu) - 126 : 15;
    const int sh = max(-126, min(126, 15 - ex));
    const float sc = __uint_as_float((uint32_t)(127 + sh) << 23);
#pragma unroll
    for (int c = 0; c < NKC; ++c) {
      const uint4 r = qs[c * 32 + lane];
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_f2(w[i]);
        const __half2 h = __floats2half2_rn(f.x * sc, f.y * sc);
        o[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      qh[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    const int sh0 = __shfl_sync(0xffffffffu, sh, 8 * lc);
    const int sh1 = __shfl_sync(0xffffffffu, sh, 8 * lc + 4);
    sl0 = a.scale_log2 * __uint_as_float((uint32_t)(127 - sh0) << 23);
    sl1 = a.scale_log2 * __uint_as_float((uint32_t)(127 - sh1) << 23);
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2c, 2c + 1
  float acc[NZC][2][4];
#pragma unroll
  for (int c = 0; c < NZC; ++c)
#pragma unroll
    for (int e = 0; e < 2; ++e) acc[c][e][0] = acc[c][e][1] = acc[c][e][2] = acc[c][e][3] = 0.f;

  // Unit nn of this warp is unit u0 + warp + 8 nn of the group.  This lane
  // holds tokens lr and lr + 8 of it: their cache rows (global row index in
  // the [page][KV head][S] row space) and their positions in the sequence
  // (past the length when there is no page).  Routing pages of S tokens:
  // the unit is part idx % TP of list entry idx / TP.  Smaller routing
  // pages: token x is row x % RPG of list entry idx * QP + x / RPG, which
  // sits at row (page % NR) * RPG of cache page page / NR.  A bad
  // block-table entry is flagged and read as page 0.
  struct Rows {
    size_t r0, r1;
    int p0, p1;
  };
  auto cache_page = [&](int lp) -> int {
    const int cp = lp >> logNR;
    int pp = lp >= 0 && cp < P_phys ? tbl[cp] : -1;
    if (lp < 0) {
      pp = 0;
    } else if (pp < 0 || pp >= a.num_phys) {
      if (lane == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
      pp = 0;
    }
    return pp;
  };
  auto unit_rows = [&](int nn) -> Rows {
    const int idx = u0 + warp + kAmWarps * nn;
    Rows u;
    if (QP == 0) {
      const int lp = list[idx >> logTP], tau = idx & (TP - 1);
      u.r0 = ((size_t)cache_page(lp) * a.Hkv + g) * S + 16 * tau + lr;
      u.r1 = u.r0 + 8;
      u.p0 = lp >= 0 ? lp * S + 16 * tau + lr : INT_MAX;
      u.p1 = lp >= 0 ? u.p0 + 8 : INT_MAX;
    } else {
      const int x0 = lr, x1 = lr + 8, m = RPG - 1;
      const int s0 = idx * QP + (x0 >> logRPG), s1 = idx * QP + (x1 >> logRPG);
      const int lp0 = s0 < nsel ? list[s0] : -1, lp1 = s1 < nsel ? list[s1] : -1;
      u.r0 = ((size_t)cache_page(lp0) * a.Hkv + g) * S +
             (lp0 >= 0 ? (lp0 & (NR - 1)) << logRPG : 0) + (x0 & m);
      u.r1 = ((size_t)cache_page(lp1) * a.Hkv + g) * S +
             (lp1 >= 0 ? (lp1 & (NR - 1)) << logRPG : 0) + (x1 & m);
      u.p0 = lp0 >= 0 ? (lp0 << logRPG) + (x0 & m) : INT_MAX;
      u.p1 = lp1 >= 0 ? (lp1 << logRPG) + (x1 & m) : INT_MAX;
    }
    return u;
  };
  uint4 kx[NKC][2], zx[NZC][2];
  auto load_k = [&](const Rows& u) {
    if constexpr (F8) {
      const uint8_t* K8 = reinterpret_cast<const uint8_t*>(a.K);
#pragma unroll
      for (int c = 0; c < NKC; ++c) {
        ldg_stream8(kx[c][0], K8 + u.r0 * D + 32 * c + 8 * lc);
        ldg_stream8(kx[c][1], K8 + u.r1 * D + 32 * c + 8 * lc);
      }
    } else {
#pragma unroll
      for (int c = 0; c < NKC; ++c) {
        kx[c][0] = ldg_stream(a.K + u.r0 * D + 32 * c + 8 * lc);
        kx[c][1] = ldg_stream(a.K + u.r1 * D + 32 * c + 8 * lc);
      }
    }
  };
  auto load_z = [&](const Rows& u, int slot) {  // asynchronous, into the warp's ring
    // rows r0 and r1 = r0 + 8 share one tile unless routing pages split the unit
    const size_t tile0 = u.r0 >> logS, tile1 = QP == 0 ? tile0 : u.r1 >> logS;
    const int trow0 = (int)(u.r0 & (S - 1)), trow1 = QP == 0 ? trow0 + 8 : (int)(u.r1 & (S - 1));
    const size_t zt0 = tile0 * S * RV, zt1 = QP == 0 ? zt0 : tile1 * S * RV;
    if constexpr (F8) {
      const uint8_t* z8 = reinterpret_cast<const uint8_t*>(a.Z);
#pragma unroll
      for (int c = 0; c < NZC; ++c) {
        const int col = 32 * c + 8 * lc;
        cp_async8(zring8 + ((slot * NZC + c) * 2 + 0) * 32 + lane,
                  z8 + zt0 + split_off(trow0, col, S, RV, a.zsplit));
        cp_async8(zring8 + ((slot * NZC + c) * 2 + 1) * 32 + lane,
                  z8 + zt1 + split_off(trow1, col, S, RV, a.zsplit));
      }
      return;
    }
#pragma unroll
    for (int c = 0; c < NZC; ++c) {
      const int col = 32 * c + 8 * lc;
      cp_async16(zring + ((slot * NZC + c) * 2 + 0) * 32 + lane,
                 a.Z + zt0 + split_off(trow0, col, S, RV, a.zsplit));
      cp_async16(zring + ((slot * NZC + c) * 2 + 1) * 32 + lane,
                 a.Z + zt1 + split_off(trow1, col, S, RV, a.zsplit));
    }
  };
  Rows cur{0, 8, INT_MAX, INT_MAX};
  if (count > 0) {
    cur = unit_rows(0);
    load_k(cur);
    load_z(cur, 0);
  }
  cp_async_commit();
  // Unit n computes while unit n + 1 loads: its latents are requested (into
  // shared memory) before unit n starts, its Keys (into registers) as soon
  // as QK has consumed the current ones.
  for (int n = 0; n < count; ++n) {
    const bool more = n + 1 < count;
    Rows nxt{0, 8, INT_MAX, INT_MAX};
    if (more) {
      nxt = unit_rows(n + 1);
      load_z(nxt, (n + 1) & 1);
    }
    cp_async_commit();
    float sc4[4] = {0.f, 0.f, 0.f, 0.f};  // [tokens r, r + 8] x [heads 2c, 2c + 1]
#pragma unroll
    for (int c = 0; c < NKC; ++c) {
      if constexpr (F8) {
        uint32_t t0[4], t1[4];  // tokens r, r + 8: columns 8c .. 8c + 7 as f16 pairs
        e4m3x4_to_f16(kx[c][0].x, t0[0], t0[1]);
        e4m3x4_to_f16(kx[c][0].y, t0[2], t0[3]);
        e4m3x4_to_f16(kx[c][1].x, t1[0], t1[1]);
        e4m3x4_to_f16(kx[c][1].y, t1[2], t1[3]);
        mma_f16_16816(sc4, t0[0], t1[0], t0[1], t1[1], qh[c].x, qh[c].y);
        mma_f16_16816(sc4, t0[2], t1[2], t0[3], t1[3], qh[c].z, qh[c].w);
      } else {
        const uint4 qf = qs[c * 32 + lane];
        mma_bf16_16816(sc4, kx[c][0].x, kx[c][1].x, kx[c][0].y, kx[c][1].y, qf.x, qf.y);
        mma_bf16_16816(sc4, kx[c][0].z, kx[c][1].z, kx[c][0].w, kx[c][1].w, qf.z, qf.w);
      }
    }
    if (more) load_k(nxt);
    const bool v0 = cur.p0 < T, v1 = cur.p1 < T;
    const float x00 = v0 ? sc4[0] * sl0 : -INFINITY;
    const float x01 = v0 ? sc4[1] * sl1 : -INFINITY;
    const float x10 = v1 ? sc4[2] * sl0 : -INFINITY;
    const float x11 = v1 ? sc4[3] * sl1 : -INFINITY;
    float mx0 = fmaxf(x00, x10), mx1 = fmaxf(x01, x11);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float sc0 = exp2f(m0 - base0), sc1 = exp2f(m1 - base1);
    m0 = mn0;
    m1 = mn1;
    const float p00 = exp2f(x00 - base0), p01 = exp2f(x01 - base1);
    const float p10 = exp2f(x10 - base0), p11 = exp2f(x11 - base1);
    l0 = fmaf(l0, sc0, p00 + p10);
    l1 = fmaf(l1, sc1, p01 + p11);
#pragma unroll
    for (int c = 0; c < NZC; ++c)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        acc[c][e][0] *= sc0;
        acc[c][e][1] *= sc1;
        acc[c][e][2] *= sc0;
        acc[c][e][3] *= sc1;
      }
    // weights as the B operand of PV: transposes of the [token][head] tiles
    uint32_t wh0, wl0, wh1, wl1;
    if constexpr (F8) {
      split_f16x2(p00, p01, wh0, wl0);
      split_f16x2(p10, p11, wh1, wl1);
    } else {
      split_bf16x2(p00, p01, wh0, wl0);
      split_bf16x2(p10, p11, wh1, wl1);
    }
    const uint32_t bh0 = movmatrix_trans(wh0), bh1 = movmatrix_trans(wh1);
    const uint32_t bl0 = movmatrix_trans(wl0), bl1 = movmatrix_trans(wl1);
    cp_async_wait_prior();  // unit n's latents have landed
#pragma unroll
    for (int c = 0; c < NZC; ++c) {
      if constexpr (F8) {  // widened to the bf16 path's register layout
        const uint2 z0 = zring8[(((n & 1) * NZC + c) * 2 + 0) * 32 + lane];
        const uint2 z1 = zring8[(((n & 1) * NZC + c) * 2 + 1) * 32 + lane];
        e4m3x4_to_f16(z0.x, zx[c][0].x, zx[c][0].y);
        e4m3x4_to_f16(z0.y, zx[c][0].z, zx[c][0].w);
        e4m3x4_to_f16(z1.x, zx[c][1].x, zx[c][1].y);
        e4m3x4_to_f16(z1.y, zx[c][1].z, zx[c][1].w);
      } else {
        zx[c][0] = zring[(((n & 1) * NZC + c) * 2 + 0) * 32 + lane];
        zx[c][1] = zring[(((n & 1) * NZC + c) * 2 + 1) * 32 + lane];
      }
    }
    // latent rows past the length hold stale data (0 * NaN would poison the sum)
    if (!v0)
#pragma unroll
      for (int c = 0; c < NZC; ++c) zx[c][0] = make_uint4(0u, 0u, 0u, 0u);
    if (!v1)
#pragma unroll
      for (int c = 0; c < NZC; ++c) zx[c][1] = make_uint4(0u, 0u, 0u, 0u);
    // PV: 8x8 tile m of a 32-column chunk = columns 8c' + 2m, +1 (c' = 0..3)
#pragma unroll
    for (int c = 0; c < NZC; ++c) {
      const uint32_t t0[4] = {movmatrix_trans(zx[c][0].x), movmatrix_trans(zx[c][0].y),
                              movmatrix_trans(zx[c][0].z), movmatrix_trans(zx[c][0].w)};
      const uint32_t t1[4] = {movmatrix_trans(zx[c][1].x), movmatrix_trans(zx[c][1].y),
                              movmatrix_trans(zx[c][1].z), movmatrix_trans(zx[c][1].w)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if constexpr (F8) {
          mma_f16_16816(acc[c][e], t0[2 * e], t0[2 * e + 1], t1[2 * e], t1[2 * e + 1], bh0, bh1);
          mma_f16_16816(acc[c][e], t0[2 * e], t0[2 * e + 1], t1[2 * e], t1[2 * e + 1], bl0, bl1);
        } else {
          mma_bf16_16816(acc[c][e], t0[2 * e], t0[2 * e + 1], t1[2 * e], t1[2 * e + 1], bh0, bh1);
          mma_bf16_16816(acc[c][e], t0[2 * e], t0[2 * e + 1], t1[2 * e], t1[2 * e + 1], bl0, bl1);
        }
      }
    }
    cur = nxt;
  }
  cp_async_wait_all();

  // ---- the CTA's warps meet: per-warp state to shared memory, one partial
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int h0 = 2 * lc, h1 = 2 * lc + 1;
  if (lr == 0) {
    if (h0 < G) {
      wml[warp * 16 + h0] = m0;
      wml[warp * 16 + 8 + h0] = l0;
    }
    if (h1 < G) {
      wml[warp * 16 + h1] = m1;
      wml[warp * 16 + 8 + h1] = l1;
    }
  }
#pragma unroll
  for (int c = 0; c < NZC; ++c)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      // accumulator rows r and r + 8 = column r of tiles 2e and 2e + 1
      const int j0 = 32 * c + 8 * (lr >> 1) + 4 * e + (lr & 1), j1 = j0 + 2;
      if (h0 < G) {
        wacc[(warp * G + h0) * RV + j0] = acc[c][e][0];
        wacc[(warp * G + h0) * RV + j1] = acc[c][e][2];
      }
      if (h1 < G) {
        wacc[(warp * G + h1) * RV + j0] = acc[c][e][1];
        wacc[(warp * G + h1) * RV + j1] = acc[c][e][3];
      }
    }
  __syncthreads();
  for (int o = tid; o < G * RV; o += kAmThreads) {
    const int h = o / RV, j = o - h * RV;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAmWarps; ++w) M = fmaxf(M, wml[w * 16 + h]);
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kAmWarps; ++w) {
      const float mw = wml[w * 16 + h];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
      L = fmaf(wml[w * 16 + 8 + h], f, L);
      A = fmaf(wacc[(w * G + h) * RV + j], f, A);
    }
    part[h * RS + 2 + j] = A;
    if (j == 0) {
      part[h * RS] = M;
      part[h * RS + 1] = L;
    }
  }
  // ---- the cluster's partials: every CTA merges a slice of the outputs
  if (C > 1)
    cg::this_cluster().sync();
  else
    __syncthreads();
  const int o0 = G * RV * rank / C, o1 = G * RV * (rank + 1) / C;
  for (int o = o0 + tid; o < o1; o += kAmThreads) {
    const int h = o / RV, j = o - h * RV;
    // every partial requested before any is used (independent remote loads)
    float pm[kSaMaxCluster], pl[kSaMaxCluster], pa[kSaMaxCluster];
#pragma unroll
    for (int r = 0; r < kSaMaxCluster; ++r) {
      if (r < C) {
        const float* src = C > 1 ? cg::this_cluster().map_shared_rank(part, r) : part;
        pm[r] = src[h * RS];
        pl[r] = src[h * RS + 1];
        pa[r] = src[h * RS + 2 + j];
      }
    }
    float M = -INFINITY, L = 0.f, A = 0.f;
#pragma unroll
    for (int r = 0; r < kSaMaxCluster; ++r) {
      if (r >= C) break;
      const float mc = pm[r], lcv = pl[r], ac = pa[r];
      if (mc == -INFINITY) continue;
      if (mc > M) {
        const float rr = exp2f(M - mc);  // 0 while M is -inf
        L *= rr;
        A *= rr;
        M = mc;
      }
      const float f = exp2f(mc - M);
      L = fmaf(lcv, f, L);
      A = fmaf(ac, f, A);
    }
    const float v = L > 0.f ? A / L : 0.f;  // an empty sequence has no token: zero
    const size_t oi = ((size_t)b * a.Hq + g * G + h) * RV + j;
    if (a.a_lat) a.a_lat[oi] = v;
    if (a.a_bf16) a.a_bf16[oi] = f_to_bf16(v);
  }
  if (rank == 0 && s.sel)  // the selection, when the caller asked for it
    for (int i = tid; i < a.top_k; i += kAmThreads) s.sel[(size_t)bg * a.top_k + i] = list[i];
  if (C > 1) cg::this_cluster().sync();  // the other CTAs have read this CTA's partial
}

template <int G, int D, int RV, bool F8 = false>
cudaError_t launch_select_attend_t(const SelectArgs& s, const AttendArgs& a, cudaStream_t st,
                                   bool pdl) {
  const int P_max = (s.max_seq_len + s.S - 1) / s.S;
  const SaLayout L = sa_layout(G, D, RV, F8, P_max, s.top_k);
  const int C = select_attend_cluster(G, D, RV, F8, a.B, a.Hkv, P_max, s.top_k, num_sms());
  if (C == 0) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(select_attend_kernel<G, D, RV, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  return launch_kc(select_attend_kernel<G, D, RV, F8>, dim3((unsigned)(a.B * a.Hkv * C)),
                   dim3(kAmThreads), L.total, st, pdl, dim3((unsigned)C, 1, 1), s, a, C);
}

}  // namespace
}  // namespace basiskv
