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
// are first staged in `fac` (shared) with independent 16-byte loads, so the
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
  // Factors are inputs no predecessor writes: their copies start before the
  // wait and land while the length and the page are looked up.
  stage_bf16_async(A, a.A_V + (size_t)g * d * r_v, d * r_v, tid, kAppendThreads);
  stage_bf16_async(Pk, a.P_K + (size_t)g * r_v * d, r_v * d, tid, kAppendThreads);
  stage_bf16_async(U, a.U_K + (size_t)g * d * r_k, d * r_k, tid, kAppendThreads);
  cp_async_commit();
  pdl_wait();
  const int len = a.seq_lens[b];
  const int cap = a.max_pages * a.S;
  if (len < 0 || len + a.n_new > cap) {
    if (tid == 0 && g == 0 && j == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
    cp_async_wait_all();  // no copy outlives the block
    return;
  }
  const int pos = len + j;
  const int pp = a.block_table[(size_t)b * a.max_pages + pos / a.S];
  if (pp < 0 || pp >= a.num_phys) {
    if (tid == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
    cp_async_wait_all();
    return;
  }
  const size_t slot = ((size_t)pp * a.Hkv + g) * a.S + pos % a.S;
  const size_t tok = (((size_t)b * a.n_new + j) * a.Hkv + g) * d;
  if (tid < d) {
    const uint16_t kb = a.k_new[tok + tid];
    ks[tid] = bf16_to_f(kb);
    vs[tid] = bf16_to_f(a.v_new[tok + tid]);
    a.K_cache[slot * d + tid] = kb;
  }
  cp_async_wait_all();
  named_bar_sync(bar, kAppendThreads);
  if (tid < r_v) {  // z_j = sum_i v_i A_V[i][j]
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < d; ++i) acc = fmaf(vs[i], bf16_to_f(A[i * r_v + tid]), acc);
    zs[tid] = acc;
    a.Z_cache[slot * r_v + tid] = f_to_bf16(acc);
  }
  named_bar_sync(bar, kAppendThreads);
  if (tid < d) {  // residual_i = k_i - sum_j z_j P_K[j][i]   (z unrounded)
    float acc = ks[tid];
#pragma unroll 8
    for (int jj = 0; jj < r_v; ++jj) acc = fmaf(-zs[jj], bf16_to_f(Pk[jj * d + tid]), acc);
    rs[tid] = acc;
  }
  named_bar_sync(bar, kAppendThreads);
  if (tid < r_k) {  // e_c = sum_i residual_i U_K[i][c]
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < d; ++i) acc = fmaf(rs[i], bf16_to_f(U[i * r_k + tid]), acc);
    a.E_cache[slot * r_k + tid] = f_to_bf16(acc);
  }
}

// Folds the queries of (sequence, KV head) bg for outputs 32*yblk .. +31:
//   qt[b][h][j]       = sum_i P_K[g][j][i] q[b][h][i]          j < r_v
//   qt[b][h][r_v + c] = sum_i q[b][h][i] U_K[g][i][c]           c < r_k
// Warp w sums the products over the w-th quarter of the head dimension for
// every head of the group; the four partial sums meet in shared memory
// (fsm: G*d + 4*G*32 floats).  All loads of a thread are independent, so the
// block costs about one memory round trip.  Run by kFoldThreads threads
// (tid = 0..kFoldThreads-1, whole warps) on named barrier bar.
__device__ __forceinline__ void fold_query_block(const FoldQArgs& a, int bg, int yblk,
                                                 float* fsm, int tid, int bar) {
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int lane = tid & 31, quarter = tid >> 5;
  const int G = a.Hq / a.Hkv, rq = a.r_v + a.r_k, d = a.d;
  const int j = yblk * 32 + lane;
  const int i0 = quarter * (d / 4), n = d / 4;
  float* qs = fsm;            // [G][d]
  float* part = fsm + G * d;  // [4][G][32]
  pdl_wait();
  for (int i = tid; i < G * d; i += kFoldThreads)
    qs[i] = bf16_to_f(a.q[((size_t)b * a.Hq + g * G) * d + i]);
  named_bar_sync(bar, kFoldThreads);
  float acc[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) acc[h] = 0.f;
  if (j < a.r_v) {  // row j of P_K, this quarter: n contiguous bf16 (16-byte aligned)
    const uint4* row = reinterpret_cast<const uint4*>(a.P_K + ((size_t)g * a.r_v + j) * d + i0);
#pragma unroll 4
    for (int c = 0; c < n / 8; ++c) {
      const uint4 w = row[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p0 = bf16lo(ws[e]), p1 = bf16hi(ws[e]);
        const int ii = i0 + c * 8 + 2 * e;
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (h < G) acc[h] = fmaf(p1, qs[h * d + ii + 1], fmaf(p0, qs[h * d + ii], acc[h]));
      }
    }
  } else if (j < rq) {  // column j - r_v of U_K, this quarter (coalesced across lanes)
    const uint16_t* col = a.U_K + (size_t)g * d * a.r_k + (j - a.r_v);
#pragma unroll 8
    for (int i = i0; i < i0 + n; ++i) {
      const float u = bf16_to_f(col[(size_t)i * a.r_k]);
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G) acc[h] = fmaf(u, qs[h * d + i], acc[h]);
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
  return (size_t)(G * d + 4 * G * 32) * sizeof(float);
}
static_assert(kAppendThreads == kFoldThreads, "the prologue's groups share one size");

}  // namespace basiskv
