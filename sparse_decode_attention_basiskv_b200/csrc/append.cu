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
  append_block(a, blockIdx.x, blockIdx.y, blockIdx.z, fac, vs, ks, zs, rs, threadIdx.x, 0);
}

// The first launch of a fused decode step: block (bg, i < n_fold) folds the
// queries of (sequence, KV head) bg for outputs 32i .. 32i + 31 (one
// 128-thread group each, so a small batch still spreads the fold over many
// SMs); when the step appends, block (bg, n_fold) appends the step's token of
// bg without staging the factors; block (0, 0) also zeroes the step's
// arrival counters.  Every block needs only a few KB of shared memory, so
// the scoring grid, let in once the wait below has returned, takes the rest
// of the SMs and starts on its page loads while this grid finishes.  The
// scoring may read the newest page before the token lands: that only
// changes that page's score, and the newest page is selected whatever its
// score.
__global__ void __launch_bounds__(kFoldThreads)
    decode_prologue_kernel(FoldQArgs f, AppendArgs a, int n_fold, int* counters,
                           int n_counters) {
  extern __shared__ __align__(16) float fsm[];
  // The next launches read the step's inputs before their own waits: they
  // are let in only once this wait has seen the caller's work complete.
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0 && blockIdx.y == 0 && counters)
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  if ((int)blockIdx.y < n_fold) {
    fold_query_block(f, blockIdx.x, blockIdx.y, fsm, threadIdx.x, 0);
  } else if (a.k_new) {
    float* vs = fsm;
    append_block_direct(a, blockIdx.x % a.Hkv, blockIdx.x / a.Hkv, vs, vs + kAppendThreads,
                        vs + 2 * kAppendThreads, vs + 3 * kAppendThreads,
                        vs + 4 * kAppendThreads, threadIdx.x, 0);
  }
}

// seq_lens[b] += n_new, skipped (with the overflow bit) when the append
// kernel skipped the sequence for the same reason.
__global__ void bump_lengths_kernel(const int32_t* seq_lens, int32_t* out, int B, int n_new,
                                    int cap, unsigned int* status) {
  // the next launch may be scheduled at once: it waits for this grid to
  // complete before it touches the lengths
  pdl_launch_dependents();
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
  const int n_fold = (f.r_v + f.r_k + 31) / 32;
  const bool app = a.k_new != nullptr;
  size_t smem = fold_block_smem(f.Hq / f.Hkv, f.d);
  const size_t app_smem =
      (size_t)(4 * kAppendThreads + append_direct_red_floats(a.d, a.r_v, a.r_k)) * sizeof(float);
  if (app && app_smem > smem) smem = app_smem;
  return launch_k(decode_prologue_kernel, dim3(f.B * f.Hkv, n_fold + (app ? 1 : 0)),
                  dim3(kFoldThreads), smem, st, pdl, f, a, n_fold, counters, n_counters);
}

}  // namespace basiskv
