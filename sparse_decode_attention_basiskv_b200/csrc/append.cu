// Cache append for a few tokens (decode): BasisKV's Value latent and Key
// residual (abstract; Table 4, compressed-Value and residual-code rows).
//
//   z = v A_V,g        e = (k - z P_K,g) U_K,g       K <- k
//
// One CTA per (KV head, token, sequence); each output element is one
// thread's fp32 dot product over the head's factors, staged in shared memory.
// The work is a few hundred thousand FMAs per decode step, so the kernel is
// bounded by latency (factor staging from L2, launch), not by any pipe.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

constexpr int kAppendThreads = 128;  // >= max(d, r_v, r_k) of every supported shape

// Copies n bf16 values (n % 8 == 0, both pointers 16-byte aligned) with
// independent 16-byte loads spread over the block.
__device__ __forceinline__ void stage_bf16(uint16_t* dst, const uint16_t* src, int n) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int i = threadIdx.x; i < n / 8; i += blockDim.x) d4[i] = s4[i];
}

// One CTA per (KV head, token, sequence).  The head's three factors (at most
// 128x128 + 128x128 + 128x64 bf16 = 80 KB) are first staged in shared memory
// with independent 16-byte loads, so the dot products below read shared
// memory instead of waiting on one global load per step.
__global__ void __launch_bounds__(kAppendThreads) append_small_kernel(AppendArgs a) {
  extern __shared__ __align__(16) uint16_t fac[];  // A_V | P_K | U_K of head g
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
  const int g = blockIdx.x, j = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int d = a.d, r_v = a.r_v, r_k = a.r_k;
  uint16_t* A = fac;
  uint16_t* Pk = fac + d * r_v;
  uint16_t* U = Pk + r_v * d;
  // Factors are inputs no predecessor writes: stage them before the wait.
  stage_bf16(A, a.A_V + (size_t)g * d * r_v, d * r_v);
  stage_bf16(Pk, a.P_K + (size_t)g * r_v * d, r_v * d);
  stage_bf16(U, a.U_K + (size_t)g * d * r_k, d * r_k);
  pdl_wait();
  const int len = a.seq_lens[b];
  const int cap = a.max_pages * a.S;
  if (len < 0 || len + a.n_new > cap) {
    if (tid == 0 && g == 0 && j == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
    return;
  }
  const int pos = len + j;
  const int pp = a.block_table[(size_t)b * a.max_pages + pos / a.S];
  if (pp < 0 || pp >= a.num_phys) {
    if (tid == 0) raise_status(a.status, BASISKV_DEV_BAD_PAGE);
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
  __syncthreads();
  if (tid < r_v) {  // z_j = sum_i v_i A_V[i][j]
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < d; ++i) acc = fmaf(vs[i], bf16_to_f(A[i * r_v + tid]), acc);
    zs[tid] = acc;
    a.Z_cache[slot * r_v + tid] = f_to_bf16(acc);
  }
  __syncthreads();
  if (tid < d) {  // residual_i = k_i - sum_j z_j P_K[j][i]   (z unrounded)
    float acc = ks[tid];
#pragma unroll 8
    for (int jj = 0; jj < r_v; ++jj) acc = fmaf(-zs[jj], bf16_to_f(Pk[jj * d + tid]), acc);
    rs[tid] = acc;
  }
  __syncthreads();
  if (tid < r_k) {  // e_c = sum_i residual_i U_K[i][c]
    float acc = 0.f;
#pragma unroll 8
    for (int i = 0; i < d; ++i) acc = fmaf(rs[i], bf16_to_f(U[i * r_k + tid]), acc);
    a.E_cache[slot * r_k + tid] = f_to_bf16(acc);
  }
}

// seq_lens[b] += n_new, skipped (with the overflow bit) when the append
// kernel skipped the sequence for the same reason.
__global__ void bump_lengths_kernel(const int32_t* seq_lens, int32_t* out, int B, int n_new,
                                    int cap, unsigned int* status) {
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int len = seq_lens[b];
  if (len < 0 || len + n_new > cap) {
    raise_status(status, BASISKV_DEV_OVERFLOW);
    return;
  }
  out[b] = len + n_new;
}

}  // namespace

cudaError_t launch_append_small(const AppendArgs& a, cudaStream_t st, bool pdl) {
  dim3 grid(a.Hkv, a.n_new, a.B);
  const size_t smem = (size_t)(2 * a.d * a.r_v + a.d * a.r_k) * sizeof(uint16_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(append_small_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(append_small_kernel, grid, dim3(kAppendThreads), smem, st, pdl, a);
}

cudaError_t launch_bump_lengths(const AppendArgs& a, cudaStream_t st, bool pdl) {
  const int threads = 128;
  return launch_k(bump_lengths_kernel, dim3((a.B + threads - 1) / threads), dim3(threads), 0,
                  st, pdl, a.seq_lens, a.seq_lens_out, a.B, a.n_new, a.max_pages * a.S,
                  a.status);
}

}  // namespace basiskv
