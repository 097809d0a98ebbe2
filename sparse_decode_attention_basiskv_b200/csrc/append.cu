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
#include "step_blocks.cuh"

namespace basiskv {

namespace {

// One CTA per (KV head, token, sequence).
__global__ void __launch_bounds__(kAppendThreads) append_small_kernel(AppendArgs a) {
  extern __shared__ __align__(16) uint16_t fac[];  // A_V | P_K | U_K of head g
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
  append_block(a, blockIdx.x, blockIdx.y, blockIdx.z, fac, vs, ks, zs, rs);
}

// The first launch of a fused decode step: blocks [0, n_fold) fold the
// queries, the next B*Hkv blocks append the step's token (one per sequence
// and KV head), and block 0 also zeroes the step's arrival counters.  The
// two jobs are independent, so one launch runs them side by side.
__global__ void __launch_bounds__(kAppendThreads)
    decode_prologue_kernel(FoldQArgs f, AppendArgs a, int n_fold, int fold_ny, int* counters,
                           int n_counters) {
  extern __shared__ __align__(16) uint16_t dyn[];
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
  const int bid = blockIdx.x;
  if (bid == 0 && counters) {
    pdl_wait();
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  }
  if (bid < n_fold) {
    fold_query_block(f, bid / fold_ny, bid % fold_ny, reinterpret_cast<float*>(dyn));
  } else {
    const int r = bid - n_fold;  // (sequence, KV head)
    append_block(a, r % a.Hkv, 0, r / a.Hkv, dyn, vs, ks, zs, rs);
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
  const size_t smem = append_block_smem(a.d, a.r_v, a.r_k);
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

cudaError_t launch_decode_prologue(const FoldQArgs& f, const AppendArgs& a, int* counters,
                                   int n_counters, cudaStream_t st, bool pdl) {
  const int G = f.Hq / f.Hkv;
  const int fold_ny = (f.r_v + f.r_k + 31) / 32;
  const int n_fold = f.B * f.Hkv * fold_ny;
  const int n_app = a.k_new ? a.B * a.Hkv : 0;
  size_t smem = fold_block_smem(G, f.d);
  if (n_app) {
    const size_t s2 = append_block_smem(a.d, a.r_v, a.r_k);
    if (s2 > smem) smem = s2;
  }
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_prologue_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(decode_prologue_kernel, dim3(n_fold + n_app), dim3(kAppendThreads), smem, st,
                  pdl, f, a, n_fold, fold_ny, counters, n_counters);
}

}  // namespace basiskv
