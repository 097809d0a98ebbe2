// Attention over the selected pages from plain loads on the warp-level
// tensor cores (shared by the bf16 instances in attend.cu and the E4M3
// instances in attend_fp8.cu, so the two sets compile in parallel).
#pragma once

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {
namespace {

// ------------------------------------------- attention, plain loads + MMA
// The same attention without TMA, a staging ring or CTA barriers per item.
// Work unit = 16 tokens of one selected page (one page when S = 16, half a
// page when S = 32).  CTA c takes a contiguous range of units in
// (sequence, KV head, selection slot) order; its 8 warps take every 8th unit
// of each run of one (sequence, KV head) and keep an online softmax.
//
// Per unit a warp issues 16-byte loads: lane (r = lane/4, c = lane%4) reads
// tokens r and r + 8 of the unit, columns 32k + 8c, of the exact Keys and of
// the Value latents (whole 32-byte sectors).  QK is mma.m16n8k16 with the
// Keys as the A operand straight from those registers (tokens = M, the head
// dimension taken in the order the lanes hold it) and the group's queries as
// B (heads = N, same column order); the scores land as [token][head].  The
// softmax weights, split into bf16 hi + lo, are transposed in registers
// (movmatrix) into the B operand of PV, and the latent tile, transposed the
// same way, is the A operand: a[latent][head] += z^T p, fp32 accumulation.
//
// A run's warps meet in shared memory and write one partial (max, sum,
// unnormalised latent per head, log2 domain) to slot (CTA + sequence * Hkv
// + KV head), unique because both grow along the unit order; the CTA whose
// arrival completes the group's count merges the partials.
//
// E4M3 caches (F8): the same lanes load the same columns as 8-byte rows of
// bytes, widened to f16 (exact) for f16 MMAs.  Each warp scales every
// head's query by a power of two that brings its largest magnitude into
// [2^14, 2^15) before rounding it to f16 (exact for bf16 values in range),
// and divides the scale out of the scores; the weights are split into f16
// hi + lo.
constexpr int kAmThreads = 256;
constexpr int kAmWarps = kAmThreads / 32;
constexpr int kAmCtasPerSm = 2;
constexpr int kAmMaxCtas = 1024;

// Bytes of one warp's latent ring: two units x chunks x two token halves x
// 32 lanes x 8 columns.
template <int RV, bool F8>
constexpr int am_ring_bytes() {
  return 2 * (RV / 32) * 2 * 32 * (F8 ? 8 : 16);
}

template <int G, int D, int RV, bool F8>
__global__ void __launch_bounds__(kAmThreads, kAmCtasPerSm) attend_mma_kernel(AttendArgs a) {
  constexpr int NKC = D / 32, NZC = RV / 32, RS = RV + 2;
  extern __shared__ float am_smem[];
  float* wacc = am_smem;                        // [warp][G][RV] latent sums of the run
  float* wml = am_smem + kAmWarps * G * RV;     // [warp][16]: m of heads 0-7, then l
  uint4* qs = reinterpret_cast<uint4*>(wml + kAmWarps * 16);  // [NKC][lane] query fragments
  // per-warp ring of two units' Value-latent chunks, [slot][chunk][half][lane]:
  // each lane copies (cp.async) and later reads only its own 16-byte (E4M3:
  // 8-byte) entries
  uint8_t* zring_b = reinterpret_cast<uint8_t*>(qs + NKC * 32) +
                     (size_t)(threadIdx.x >> 5) * am_ring_bytes<RV, F8>();
  uint4* zring = reinterpret_cast<uint4*>(zring_b);
  uint2* zring8 = reinterpret_cast<uint2*>(zring_b);
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, lr = lane >> 2, lc = lane & 3;
  const int S = a.S, TP = S >> 4, logS = 31 - __clz(S);
  const int upb = a.top_k * TP;  // units per (sequence, KV head)
  const long total = (long)a.B * a.Hkv * upb;
  const int C = gridDim.x;
  const long c_end = total * (blockIdx.x + 1) / C;
  // CTA holding unit x (every CTA holds at least one unit: grid <= units)
  auto cta_of = [&](long x) -> int {
    const long c = ((x + 1) * C - 1) / total;
    return (int)(c < C - 1 ? c : C - 1);
  };
  // The next launch (the out-projection) may take SMs as this grid's CTAs
  // retire; it requests only its weight tiles before its own wait (measured:
  // about 1 us per fused step).
  pdl_launch_dependents();
  if (!a.early_inputs) pdl_wait();

  long seg = total * blockIdx.x / C;
  while (seg < c_end) {
    const int bg = (int)(seg / upb);
    const long bg0 = (long)bg * upb;
    const long seg_end = c_end < bg0 + upb ? c_end : bg0 + upb;
    const int b = bg / a.Hkv, g = bg - b * a.Hkv;
    const long u_first = seg + warp;
    // Page ids of the warp's units in this run, fetched 32 at a time (lane i:
    // unit seg + warp + 8 (n0 + i)) with the physical page from the
    // selection's companion list when there is one, else through the block
    // table.  The first batch goes out with the length and the queries (one
    // round trip); entries past the selection are fetched but never used.
    int lp_l = -1, pp_l = -1, n0 = 0;
    auto fetch_ids = [&](int base) {
      const long uu = u_first + (long)kAmWarps * (base + lane);
      lp_l = -1;
      pp_l = -1;
      if (uu < seg_end) {
        const size_t si = (size_t)bg * a.top_k + (int)(uu - bg0) / TP;
        lp_l = __ldg(a.sel + si);
        if (a.sel_phys)
          pp_l = __ldg(a.sel_phys + si);
        else if (lp_l >= 0 && lp_l < a.max_pages)
          pp_l = __ldg(a.block_table + (size_t)b * a.max_pages + lp_l);
      }
    };
    int T = a.seq_lens[b] + a.len_offset;
    // the group's queries as B fragments, shared by the CTA's warps: entry
    // [k][lane (r, c)] holds head r, columns 32k + 8c .. +7 (zero past G)
    for (int i = tid; i < NKC * 32; i += kAmThreads) {
      const int k = i >> 5, r = (i & 31) >> 2, cc = i & 3;
      qs[i] = r < G ? __ldg(reinterpret_cast<const uint4*>(
                          a.q + ((size_t)b * a.Hq + g * G + r) * D + 32 * k + 8 * cc))
                    : make_uint4(0u, 0u, 0u, 0u);
    }
    pdl_wait();  // the selection is the previous launch's output
    fetch_ids(0);
    T = T < 0 ? 0 : T;
    const int nsel = min(a.top_k, (T + S - 1) / S);
    const long valid_end = bg0 + (long)nsel * TP;  // units past it have no page
    __syncthreads();
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

    const long u_stop = seg_end < valid_end ? seg_end : valid_end;
    const int count =
        u_first < u_stop ? (int)((u_stop - u_first + kAmWarps - 1) / kAmWarps) : 0;
    // ids of unit nn (warp-uniform); a missing entry becomes a fully masked
    // unit on page 0, a bad page is flagged and read as page 0
    auto unit_ids = [&](int nn, int& lp, int& pp) {
      if (nn - n0 >= 32) {
        n0 = nn;
        fetch_ids(n0);
      }
      lp = __shfl_sync(0xffffffffu, lp_l, nn - n0);
      pp = __shfl_sync(0xffffffffu, pp_l, nn - n0);
      if (lp < 0) {
        pp = 0;
      } else if (pp < 0 || pp >= a.num_phys) {
        if (lane == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
        pp = 0;
      }
    };
    auto unit_row = [&](int nn, int pp) -> size_t {
      const int tau = (int)(u_first + (long)kAmWarps * nn - bg0) % TP;
      return ((size_t)pp * a.Hkv + g) * S + 16 * tau + lr;
    };
    uint4 kx[NKC][2], zx[NZC][2];
    auto load_k = [&](size_t row) {
      if constexpr (F8) {
        const uint8_t* K8 = reinterpret_cast<const uint8_t*>(a.K);
#pragma unroll
        for (int c = 0; c < NKC; ++c) {
          ldg_stream8(kx[c][0], K8 + row * D + 32 * c + 8 * lc);
          ldg_stream8(kx[c][1], K8 + (row + 8) * D + 32 * c + 8 * lc);
        }
      } else {
#pragma unroll
        for (int c = 0; c < NKC; ++c) {
          kx[c][0] = ldg_stream(a.K + row * D + 32 * c + 8 * lc);
          kx[c][1] = ldg_stream(a.K + (row + 8) * D + 32 * c + 8 * lc);
        }
      }
    };
    auto load_z = [&](size_t row, int slot) {  // asynchronous, into the warp's ring
      // tiles may store their first zsplit columns first (a narrow router's)
      const size_t tile = row >> logS;
      const int trow = (int)(row & (S - 1));
      if constexpr (F8) {
        const uint8_t* zt8 = reinterpret_cast<const uint8_t*>(a.Z) + tile * S * RV;
#pragma unroll
        for (int c = 0; c < NZC; ++c) {
          const int col = 32 * c + 8 * lc;
          cp_async8(zring8 + ((slot * NZC + c) * 2 + 0) * 32 + lane,
                    zt8 + split_off(trow, col, S, RV, a.zsplit));
          cp_async8(zring8 + ((slot * NZC + c) * 2 + 1) * 32 + lane,
                    zt8 + split_off(trow + 8, col, S, RV, a.zsplit));
        }
        return;
      }
      const uint16_t* zt = a.Z + tile * S * RV;
#pragma unroll
      for (int c = 0; c < NZC; ++c) {
        const int col = 32 * c + 8 * lc;
        cp_async16(zring + ((slot * NZC + c) * 2 + 0) * 32 + lane,
                   zt + split_off(trow, col, S, RV, a.zsplit));
        cp_async16(zring + ((slot * NZC + c) * 2 + 1) * 32 + lane,
                   zt + split_off(trow + 8, col, S, RV, a.zsplit));
      }
    };
    int lp_c = -1, pp_c = 0;
    if (count > 0) {
      unit_ids(0, lp_c, pp_c);
      const size_t row0 = unit_row(0, pp_c);
      load_k(row0);
      load_z(row0, 0);
    }
    cp_async_commit();
    // Unit n computes while unit n + 1 loads: its latents are requested
    // (into shared memory) before unit n starts, its Keys (into registers) as
    // soon as QK has consumed the current ones.
    for (int n = 0; n < count; ++n) {
      const int tau = (int)(u_first + (long)kAmWarps * n - bg0) % TP;
      const bool more = n + 1 < count;
      int lp_n = -1, pp_n = 0;
      if (more) unit_ids(n + 1, lp_n, pp_n);
      const size_t row_n = more ? unit_row(n + 1, pp_n) : 0;
      if (more) load_z(row_n, (n + 1) & 1);
      cp_async_commit();
      // s = [tokens r, r + 8] x [heads 2c, 2c + 1]
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < NKC; ++c) {
        if constexpr (F8) {
          uint32_t t0[4], t1[4];  // tokens r, r + 8: columns 8c .. 8c + 7 as f16 pairs
          e4m3x4_to_f16(kx[c][0].x, t0[0], t0[1]);
          e4m3x4_to_f16(kx[c][0].y, t0[2], t0[3]);
          e4m3x4_to_f16(kx[c][1].x, t1[0], t1[1]);
          e4m3x4_to_f16(kx[c][1].y, t1[2], t1[3]);
          mma_f16_16816(s, t0[0], t1[0], t0[1], t1[1], qh[c].x, qh[c].y);
          mma_f16_16816(s, t0[2], t1[2], t0[3], t1[3], qh[c].z, qh[c].w);
        } else {
          const uint4 qf = qs[c * 32 + lane];
          mma_bf16_16816(s, kx[c][0].x, kx[c][1].x, kx[c][0].y, kx[c][1].y, qf.x, qf.y);
          mma_bf16_16816(s, kx[c][0].z, kx[c][1].z, kx[c][0].w, kx[c][1].w, qf.z, qf.w);
        }
      }
      if (more) load_k(row_n);
      const int pos = lp_c * S + 16 * tau + lr;
      const bool v0 = lp_c >= 0 && pos < T, v1 = lp_c >= 0 && pos + 8 < T;
      const float x00 = v0 ? s[0] * sl0 : -INFINITY;
      const float x01 = v0 ? s[1] * sl1 : -INFINITY;
      const float x10 = v1 ? s[2] * sl0 : -INFINITY;
      const float x11 = v1 ? s[3] * sl1 : -INFINITY;
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
      lp_c = lp_n;
      pp_c = pp_n;
    }
    cp_async_wait_all();  // the ring is refilled by the next run
    (void)pp_c;

    // ---- the run's warps meet: per-warp state to shared memory
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
    const bool has = seg < valid_end;  // the run holds units with pages
    if (has) {
      float* slot = a.partial + (size_t)(blockIdx.x + bg) * G * RS;
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
        slot[h * RS + 2 + j] = A;
        if (j == 0) {
          slot[h * RS] = M;
          slot[h * RS + 1] = L;
        }
      }
    } else if (seg == bg0) {  // an empty sequence: its output is zero
      const size_t o0 = ((size_t)b * a.Hq + g * G) * RV;
      for (int o = tid; o < G * RV; o += kAmThreads) {
        if (a.a_lat) a.a_lat[o0 + o] = 0.f;
        if (a.a_bf16) a.a_bf16[o0 + o] = 0;
      }
    }
    __syncthreads();  // slot written; the shared state is free again
    if (has) {
      const int c0 = cta_of(bg0), c1 = cta_of(valid_end - 1);
      if (tid == 0) s_last = arrive_acq_rel(&a.cnt[bg], 1) + 1 == c1 - c0 + 1;
      __syncthreads();
      if (s_last) {  // every run of the group is written: merge them
        for (int o = tid; o < G * RV; o += kAmThreads) {
          const int h = o / RV, j = o - h * RV;
          // one pass with a running maximum: every slot's loads are independent
          float M = -INFINITY, L = 0.f, A = 0.f;
#pragma unroll 8
          for (int c = c0; c <= c1; ++c) {
            const float* sl = a.partial + (size_t)(c + bg) * G * RS + h * RS;
            const float mc = __ldcg(sl), lcv = __ldcg(sl + 1), ac = __ldcg(sl + 2 + j);
            if (mc == -INFINITY) continue;
            if (mc > M) {
              const float r = exp2f(M - mc);  // 0 while M is -inf
              L *= r;
              A *= r;
              M = mc;
            }
            const float f = exp2f(mc - M);
            L = fmaf(lcv, f, L);
            A = fmaf(ac, f, A);
          }
          const float v = L > 0.f ? A / L : 0.f;
          const size_t oi = ((size_t)b * a.Hq + g * G + h) * RV + j;
          if (a.a_lat) a.a_lat[oi] = v;
          if (a.a_bf16) a.a_bf16[oi] = f_to_bf16(v);
        }
        if (tid == 0) a.cnt[bg] = 0;  // ready for the next call
      }
    }
    seg = seg_end;
  }
}

template <int G, int D, int RV, bool F8 = false>
cudaError_t launch_attend_mma_t(const AttendArgs& a, cudaStream_t st, bool pdl) {
  const long units = (long)a.B * a.Hkv * a.top_k * (a.S / 16);
  if (units <= 0) return cudaSuccess;  // nothing to attend: no launch
  long grid = (long)num_sms() * kAmCtasPerSm;
  if (grid > kAmMaxCtas) grid = kAmMaxCtas;
  // At least 16 units a CTA (every CTA gets at least one): at small batches
  // fewer, longer runs beat many one-unit CTAs whose partials the last CTA
  // of a group must merge one by one.  Measured per fused step at the
  // Llama-8B layer (G 4, page 16, top_k 128, 32K context): B = 1 40.8 vs
  // 50.1 us, B = 4 66.7 vs 70.7 us, B = 16 unchanged (the grid is the same
  // there).
  if (grid > units / 16) grid = units / 16 > 0 ? units / 16 : 1;
  const size_t smem = (size_t)kAmWarps * (G * RV + 16) * sizeof(float) + (D / 32) * 32 * 16 +
                      (size_t)kAmWarps * am_ring_bytes<RV, F8>();
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attend_mma_kernel<G, D, RV, F8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(attend_mma_kernel<G, D, RV, F8>, dim3((unsigned)grid), dim3(kAmThreads), smem,
                  st, pdl, a);
}

}  // namespace
}  // namespace basiskv
