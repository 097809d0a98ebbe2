// Cache append for a few tokens (decode): BasisKV's Value latent and Key
// residual (abstract; Table 4, compressed-Value and residual-code rows).
//
//   z = v A_V,g        e = (k - z P_K,g) U_K,g       K <- k
//
// One CTA per (KV head, token, sequence); each output element is one
// thread's fp32 dot product over factor rows that stay resident in L2.  The
// work is a few hundred thousand FMAs per decode step, so the kernel is
// bounded by launch latency, not by any pipe.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

constexpr int kAppendThreads = 128;  // >= max(d, r_v, r_k) of every supported shape

__global__ void __launch_bounds__(kAppendThreads) append_small_kernel(AppendArgs a) {
  pdl_wait();
  const int g = blockIdx.x, j = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
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
  const size_t tok = (((size_t)b * a.n_new + j) * a.Hkv + g) * a.d;
  if (tid < a.d) {
    const uint16_t kb = a.k_new[tok + tid];
    ks[tid] = bf16_to_f(kb);
    vs[tid] = bf16_to_f(a.v_new[tok + tid]);
    a.K_cache[slot * a.d + tid] = kb;
  }
  __syncthreads();
  if (tid < a.r_v) {  // z_j = sum_i v_i A_V[i][j]
    const uint16_t* A = a.A_V + (size_t)g * a.d * a.r_v + tid;
    float acc = 0.f;
    for (int i = 0; i < a.d; ++i) acc = fmaf(vs[i], bf16_to_f(A[(size_t)i * a.r_v]), acc);
    zs[tid] = acc;
    a.Z_cache[slot * a.r_v + tid] = f_to_bf16(acc);
  }
  __syncthreads();
  if (tid < a.d) {  // residual_i = k_i - sum_j z_j P_K[j][i]   (z unrounded)
    const uint16_t* P = a.P_K + (size_t)g * a.r_v * a.d + tid;
    float acc = ks[tid];
    for (int jj = 0; jj < a.r_v; ++jj) acc = fmaf(-zs[jj], bf16_to_f(P[(size_t)jj * a.d]), acc);
    rs[tid] = acc;
  }
  __syncthreads();
  if (tid < a.r_k) {  // e_c = sum_i residual_i U_K[i][c]
    const uint16_t* U = a.U_K + (size_t)g * a.d * a.r_k + tid;
    float acc = 0.f;
    for (int i = 0; i < a.d; ++i) acc = fmaf(rs[i], bf16_to_f(U[(size_t)i * a.r_k]), acc);
    a.E_cache[slot * a.r_k + tid] = f_to_bf16(acc);
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
  return launch_k(append_small_kernel, grid, dim3(kAppendThreads), 0, st, pdl, a);
}

cudaError_t launch_bump_lengths(const AppendArgs& a, cudaStream_t st, bool pdl) {
  const int threads = 128;
  return launch_k(bump_lengths_kernel, dim3((a.B + threads - 1) / threads), dim3(threads), 0,
                  st, pdl, a.seq_lens, a.seq_lens_out, a.B, a.n_new, a.max_pages * a.S,
                  a.status);
}

}  // namespace basiskv
