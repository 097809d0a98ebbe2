// Block-level bodies of the two latency-bound kernels of a decode step: the
// token append (csrc/append.cu) and the query fold (csrc/route.cu).  Kept as
// device functions so the fused decode can also run both in one launch.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace basiskv {

constexpr int kAppendThreads = 128;  // >= max(d, r_v, r_k) of every supported shape
constexpr int kFoldThreads = 128;    // 32 outputs x 4 quarters of the head dim

// Starts copying n bf16 values (n % 8 == 0, both pointers 16-byte aligned)
// into shared memory with asynchronous 16-byte copies spread over the block:
// every copy is in flight at once (one memory round trip in all).  Complete
// after cp_async_wait_all() and a barrier.
__device__ __forceinline__ void stage_bf16_async(uint16_t* dst, const uint16_t* src, int n,
                                                 int tid, int nthreads) {
  for (int i = tid; i < n / 8; i += nthreads) cp_async16(dst + 8 * i, src + 8 * i);
}

// Appends token j of sequence b for KV head g:
//   z = v A_V,g;  e = (k - z P_K,g) U_K,g (z unrounded);  K <- k.
// The head's three factors (at most 128x128 + 128x128 + 128x64 bf16 = 80 KB)
// are first staged in `fac` (shared) with asynchronous 16-byte copies, so the
// dot products read shared memory instead of waiting on one global load per
// step.  vs, ks, zs, rs: shared scratch of kAppendThreads floats each.  Run
// by kAppendThreads threads (tid = 0..kAppendThreads-1) that synchronise on
// named barrier bar (0 when they are the whole block).
__device__ __forceinline__ void append_block(const AppendArgs& a, int g, int j, int b,
                                             uint16_t* fac, float* vs, float* ks, float* zs,
                                             float* rs, int tid, int bar) {
  const int d = a.d, r_v = a.r_v, r_k = a.r_k;
  uint16_t* A = fac;
  uint16_t* Pk = fac + d * r_v;
  uint16_t* U = Pk + r_v * d;
  // Every input is read after the wait (a kernel just before this one may
  // have written any of them), but all first reads go out together: the
  // factor copies, the length, and the token itself, whose position in the
  // cache is not needed until the final stores.
  pdl_wait();
  stage_bf16_async(A, a.A_V + (size_t)g * d * r_v, d * r_v, tid, kAppendThreads);
  stage_bf16_async(Pk, a.P_K + (size_t)g * r_v * d, r_v * d, tid, kAppendThreads);
  stage_bf16_async(U, a.U_K + (size_t)g * d * r_k, d * r_k, tid, kAppendThreads);
  cp_async_commit();
  const size_t tok = (((size_t)b * a.n_new + j) * a.Hkv + g) * d;
  uint16_t kb = 0;
  if (tid < d) {
    kb = a.k_new[tok + tid];
    ks[tid] = bf16_to_f(kb);
    vs[tid] = bf16_to_f(a.v_new[tok + tid]);
  }
  const int len = a.seq_lens[b];
  const int cap = a.max_pages * a.S;
  const bool fits = len >= 0 && len + a.n_new <= cap;
  const int pos = len + j;
  // block-table entry requested now, used at the end
  const int pp = fits ? a.block_table[(size_t)b * a.max_pages + pos / a.S] : -1;
  cp_async_wait_all();
  named_bar_sync(bar, kAppendThreads);
  float zv = 0.f, ev = 0.f;
  // Each dot product keeps four independent partial sums (d and r_v are
  // multiples of 32), so its chain of dependent FMAs is a quarter as long.
  if (tid < r_v) {  // z_j = sum_i v_i A_V[i][j]
    float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll 4
    for (int i = 0; i < d; i += 4) {
      c0 = fmaf(vs[i], bf16_to_f(A[i * r_v + tid]), c0);
      c1 = fmaf(vs[i + 1], bf16_to_f(A[(i + 1) * r_v + tid]), c1);
      c2 = fmaf(vs[i + 2], bf16_to_f(A[(i + 2) * r_v + tid]), c2);
      c3 = fmaf(vs[i + 3], bf16_to_f(A[(i + 3) * r_v + tid]), c3);
    }
    zv = (c0 + c1) + (c2 + c3);
    zs[tid] = zv;
  }
  named_bar_sync(bar, kAppendThreads);
  if (tid < d) {  // residual_i = k_i - sum_j z_j P_K[j][i]   (z unrounded)
    float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll 4
    for (int jj = 0; jj < r_v; jj += 4) {
      c0 = fmaf(zs[jj], bf16_to_f(Pk[jj * d + tid]), c0);
      c1 = fmaf(zs[jj + 1], bf16_to_f(Pk[(jj + 1) * d + tid]), c1);
      c2 = fmaf(zs[jj + 2], bf16_to_f(Pk[(jj + 2) * d + tid]), c2);
      c3 = fmaf(zs[jj + 3], bf16_to_f(Pk[(jj + 3) * d + tid]), c3);
    }
    rs[tid] = ks[tid] - ((c0 + c1) + (c2 + c3));
  }
  named_bar_sync(bar, kAppendThreads);
  if (tid < r_k) {  // e_c = sum_i residual_i U_K[i][c]
    float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll 4
    for (int i = 0; i < d; i += 4) {
      c0 = fmaf(rs[i], bf16_to_f(U[i * r_k + tid]), c0);
      c1 = fmaf(rs[i + 1], bf16_to_f(U[(i + 1) * r_k + tid]), c1);
      c2 = fmaf(rs[i + 2], bf16_to_f(U[(i + 2) * r_k + tid]), c2);
      c3 = fmaf(rs[i + 3], bf16_to_f(U[(i + 3) * r_k + tid]), c3);
    }
    ev = (c0 + c1) + (c2 + c3);
  }
  if (!fits) {
    if (tid == 0 && g == 0 && j == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
    return;
  }
  if (pp < 0 || pp >= a.num_phys) {
    if (tid == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
    return;
  }
  const size_t tile = (size_t)pp * a.Hkv + g;
  const int row = pos % a.S;
  if (a.fp8) {  // E4M3 caches: one byte per value, rounded to nearest even, saturated
    if (tid < d)
      reinterpret_cast<uint8_t*>(a.K_cache)[(tile * a.S + row) * d + tid] =
          (uint8_t)f_to_e4m3x2(bf16_to_f(kb), 0.f);
    if (tid < r_v)
      reinterpret_cast<uint8_t*>(a.Z_cache)[tile * a.S * r_v +
                                            split_off(row, tid, a.S, r_v, a.zsplit)] =
          (uint8_t)f_to_e4m3x2(zv, 0.f);
    if (tid < r_k)
      reinterpret_cast<uint8_t*>(a.E_cache)[tile * a.S * r_k +
                                            split_off(row, tid, a.S, r_k, a.esplit)] =
          (uint8_t)f_to_e4m3x2(ev, 0.f);
    return;
  }
  if (tid < d) a.K_cache[(tile * a.S + row) * d + tid] = kb;
  if (tid < r_v)
    a.Z_cache[tile * a.S * r_v + split_off(row, tid, a.S, r_v, a.zsplit)] = f_to_bf16(zv);
  if (tid < r_k)
    a.E_cache[tile * a.S * r_k + split_off(row, tid, a.S, r_k, a.esplit)] = f_to_bf16(ev);
}

// The same append without staging the factors in shared memory, for a block
// that runs beside the query fold and the early page loads of the scoring
// grid (a few KB of shared memory, like the fold's blocks, so the scoring
// CTAs still fit beside it).  Each of the three products is split into
// tasks of 8 outputs x 8 rows of the factor: a task's 8 16-byte row loads
// are independent, so a product costs about one memory round trip; the
// per-row-block partial sums meet in shared memory (red: at least
// max(d/8 * r_v, r_v/8 * d, d/8 * r_k) floats).  Run by kAppendThreads
// threads on named barrier bar.
__device__ __forceinline__ void append_block_direct(const AppendArgs& a, int g, int b,
                                                    float* vs, float* ks, float* zs, float* rs,
                                                    float* red, int tid, int bar) {
  const int d = a.d, r_v = a.r_v, r_k = a.r_k;
  pdl_wait();
  const size_t tok = ((size_t)b * a.n_new * a.Hkv + g) * d;  // token 0 of sequence b
  uint16_t kb = 0;
  if (tid < d) {
    kb = a.k_new[tok + tid];
    ks[tid] = bf16_to_f(kb);
    vs[tid] = bf16_to_f(a.v_new[tok + tid]);
  }
  const int len = a.seq_lens[b];
  const int cap = a.max_pages * a.S;
  const bool fits = len >= 0 && len + 1 <= cap;
  const int pp = fits ? a.block_table[(size_t)b * a.max_pages + len / a.S] : -1;
  named_bar_sync(bar, kAppendThreads);
  // y[o] = sum_i x[i] F[i][o] for a factor F [rows][outs] (row-major, bf16):
  // task (row block rb, output group og) adds rows 8rb .. 8rb+7 for outputs
  // 8og .. 8og+7 into red[rb][8og ..]; then y[o] = sum over row blocks.
  auto product = [&](const uint16_t* F, const float* x, int rows, int outs, float* y) {
    const int ngr = outs / 8, nrb = rows / 8;
    for (int t = tid; t < ngr * nrb; t += kAppendThreads) {
      const int og = t % ngr, rb = t / ngr;
      uint4 w[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        w[r] = __ldg(reinterpret_cast<const uint4*>(F + (size_t)(8 * rb + r) * outs + 8 * og));
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float xv = x[8 * rb + r];
        const uint32_t u[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] = fmaf(xv, bf16lo(u[e]), acc[2 * e]);
          acc[2 * e + 1] = fmaf(xv, bf16hi(u[e]), acc[2 * e + 1]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) red[rb * outs + 8 * og + e] = acc[e];
    }
    named_bar_sync(bar, kAppendThreads);
    for (int o = tid; o < outs; o += kAppendThreads) {
      float v = 0.f;
      for (int rb = 0; rb < nrb; ++rb) v += red[rb * outs + o];
      y[o] = v;
    }
    named_bar_sync(bar, kAppendThreads);
  };
  // z = v A_V (A_V [d][r_v]); the residual k - z P_K (P_K [r_v][d]), with
  // the unrounded z; e = residual U_K (U_K [d][r_k])
  product(a.A_V + (size_t)g * d * r_v, vs, d, r_v, zs);
  product(a.P_K + (size_t)g * r_v * d, zs, r_v, d, rs);
  if (tid < d) rs[tid] = ks[tid] - rs[tid];
  named_bar_sync(bar, kAppendThreads);
  product(a.U_K + (size_t)g * d * r_k, rs, d, r_k, red + d / 8 * r_k);
  const float* es = red + d / 8 * r_k;
  if (!fits) {
    if (tid == 0 && g == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
    return;
  }
  if (pp < 0 || pp >= a.num_phys) {
    if (tid == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
    return;
  }
  const size_t tile = (size_t)pp * a.Hkv + g;
  const int row = len % a.S;
  if (a.fp8) {  // E4M3 caches: one byte per value, rounded to nearest even, saturated
    if (tid < d)
      reinterpret_cast<uint8_t*>(a.K_cache)[(tile * a.S + row) * d + tid] =
          (uint8_t)f_to_e4m3x2(bf16_to_f(kb), 0.f);
    if (tid < r_v)
      reinterpret_cast<uint8_t*>(a.Z_cache)[tile * a.S * r_v +
                                            split_off(row, tid, a.S, r_v, a.zsplit)] =
          (uint8_t)f_to_e4m3x2(zs[tid], 0.f);
    if (tid < r_k)
      reinterpret_cast<uint8_t*>(a.E_cache)[tile * a.S * r_k +
                                            split_off(row, tid, a.S, r_k, a.esplit)] =
          (uint8_t)f_to_e4m3x2(es[tid], 0.f);
    return;
  }
  if (tid < d) a.K_cache[(tile * a.S + row) * d + tid] = kb;
  if (tid < r_v)
    a.Z_cache[tile * a.S * r_v + split_off(row, tid, a.S, r_v, a.zsplit)] = f_to_bf16(zs[tid]);
  if (tid < r_k)
    a.E_cache[tile * a.S * r_k + split_off(row, tid, a.S, r_k, a.esplit)] = f_to_bf16(es[tid]);
}

// Shared memory of append_block_direct's partial sums (floats).
__host__ __device__ inline int append_direct_red_floats(int d, int r_v, int r_k) {
  int n = d / 8 * r_v;
  if (r_v / 8 * d > n) n = r_v / 8 * d;
  if (d / 8 * r_k > n) n = d / 8 * r_k;
  return n + d / 8 * r_k;  // + the residual code e, kept past the partials
}

// Folds the queries of (sequence, KV head) bg for outputs 32*yblk .. +31:
//   qt[b][h][j]       = sum_i P_K[g][j][i] q[b][h][i]          j < r_v
//   qt[b][h][r_v + c] = sum_i q[b][h][i] U_K[g][i][c]           c < r_k
// Latent outputs (P_K, whose rows hold the head dimension contiguously):
// warp w sums the products over the w-th quarter of the head dimension for
// every head of the group, from 16-byte loads of its P_K rows; the four
// partial sums meet in shared memory.  Residual-code outputs (U_K, whose
// columns are strided): thread (row block rb, output group og) loads rows
// 8rb .. 8rb+7 of U_K at columns 8og .. 8og+7 as one 16-byte load each and
// sums them against every head; the row blocks' partial sums meet in shared
// memory (fsm: G*d + max(4, d/8)*G*32 floats).  All loads of a thread are
// independent, so the block costs about one memory round trip.  Run by
// kFoldThreads threads (tid = 0..kFoldThreads-1, whole warps) on named
// barrier bar.
__device__ __forceinline__ void fold_query_block(const FoldQArgs& a, int bg, int yblk,
                                                 float* fsm, int tid, int bar) {
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int lane = tid & 31, quarter = tid >> 5;
  const int G = a.Hq / a.Hkv, rq = a.r_v + a.r_k, d = a.d;
  const int j = yblk * 32 + lane;
  const int i0 = quarter * (d / 4), n = d / 4;
  float* qs = fsm;            // [G][d]
  float* part = fsm + G * d;  // [4][G][32], or [d/8][G][32] for residual outputs
  pdl_wait();
  if (yblk * 32 >= a.r_v) {  // residual-code outputs: U_K columns cs .. cs + nout - 1
    const int cs = yblk * 32 - a.r_v, nout = min(32, a.r_k - cs), ngr = nout / 8;
    const int rb = tid / max(ngr, 1), og = tid - rb * max(ngr, 1);
    const bool act = ngr > 0 && rb < d / 8;
    uint4 w[8];
    if (act) {
      const uint16_t* src = a.U_K + ((size_t)g * d + 8 * rb) * a.r_k + cs + 8 * og;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        w[r] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * a.r_k));
    }
    const uint4* q8 = reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + g * G) * d);
    for (int i = tid; i < G * d / 8; i += kFoldThreads) {
      const uint4 x = q8[i];
      float4* dst = reinterpret_cast<float4*>(qs + 8 * i);
      dst[0] = make_float4(bf16lo(x.x), bf16hi(x.x), bf16lo(x.y), bf16hi(x.y));
      dst[1] = make_float4(bf16lo(x.z), bf16hi(x.z), bf16lo(x.w), bf16hi(x.w));
    }
    named_bar_sync(bar, kFoldThreads);
    if (act) {
      for (int h = 0; h < G; ++h) {
        float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float qv = qs[h * d + 8 * rb + r];
          const uint32_t u[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc8[2 * e] = fmaf(qv, bf16lo(u[e]), acc8[2 * e]);
            acc8[2 * e + 1] = fmaf(qv, bf16hi(u[e]), acc8[2 * e + 1]);
          }
        }
        float4* dst = reinterpret_cast<float4*>(part + (rb * G + h) * 32 + 8 * og);
        dst[0] = make_float4(acc8[0], acc8[1], acc8[2], acc8[3]);
        dst[1] = make_float4(acc8[4], acc8[5], acc8[6], acc8[7]);
      }
    }
    named_bar_sync(bar, kFoldThreads);
    for (int o = tid; o < G * nout; o += kFoldThreads) {
      const int h = o / nout, c = o - h * nout;
      float v = 0.f;
      for (int r8 = 0; r8 < d / 8; ++r8) v += part[(r8 * G + h) * 32 + c];
      a.qt[((size_t)b * a.Hq + g * G + h) * rq + a.r_v + cs + c] = v;
    }
    return;
  }
  // Latent outputs.  This thread's factor values go out first, all at once
  // (they do not depend on the queries): a row quarter of P_K (n/8 <= 4
  // chunks of 16 bytes).
  uint4 prow[4];
  {
    const uint4* row = reinterpret_cast<const uint4*>(a.P_K + ((size_t)g * a.r_v + j) * d + i0);
#pragma unroll
    for (int c = 0; c < 4; ++c) prow[c] = c < n / 8 ? row[c] : make_uint4(0u, 0u, 0u, 0u);
  }
  {  // the group's queries: 16-byte loads, all in flight together (G*d/8 <= 128)
    const uint4* q8 = reinterpret_cast<const uint4*>(a.q + ((size_t)b * a.Hq + g * G) * d);
    for (int i = tid; i < G * d / 8; i += kFoldThreads) {
      const uint4 w = q8[i];
      float4* dst = reinterpret_cast<float4*>(qs + 8 * i);
      dst[0] = make_float4(bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y));
      dst[1] = make_float4(bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w));
    }
  }
  named_bar_sync(bar, kFoldThreads);
  float acc[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) acc[h] = 0.f;
  {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c >= n / 8) break;
      const uint32_t ws[4] = {prow[c].x, prow[c].y, prow[c].z, prow[c].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p0 = bf16lo(ws[e]), p1 = bf16hi(ws[e]);
        const int ii = i0 + c * 8 + 2 * e;
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (h < G) {
            const float2 qv = *reinterpret_cast<const float2*>(qs + h * d + ii);
            acc[h] = fmaf(p1, qv.y, fmaf(p0, qv.x, acc[h]));
          }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h)
    if (h < G) part[(quarter * G + h) * 32 + lane] = acc[h];
  named_bar_sync(bar, kFoldThreads);
  for (int o = tid; o < G * 32; o += kFoldThreads) {
    const int h = o / 32, jj = yblk * 32 + (o % 32);
    if (jj < rq) {
      const float v = part[(0 * G + h) * 32 + o % 32] + part[(1 * G + h) * 32 + o % 32] +
                      part[(2 * G + h) * 32 + o % 32] + part[(3 * G + h) * 32 + o % 32];
      a.qt[((size_t)b * a.Hq + g * G + h) * rq + jj] = v;
    }
  }
}

__host__ __device__ inline size_t append_block_smem(int d, int r_v, int r_k) {
  return (size_t)(2 * d * r_v + d * r_k) * sizeof(uint16_t);
}
__host__ __device__ inline size_t fold_block_smem(int G, int d) {
  return (size_t)(G * d + (d / 8 > 4 ? d / 8 : 4) * G * 32) * sizeof(float);
}
static_assert(kAppendThreads == kFoldThreads, "the prologue's groups share one size");

}  // namespace basiskv
