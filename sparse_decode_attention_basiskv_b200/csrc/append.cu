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

// The first launch of a fused decode step, one block per (sequence, KV
// head): 128-thread group i < n_fold folds the group's queries for outputs
// 32i .. 32i + 31, and (when the step appends) the last group appends the
// step's token; each group synchronises on its own named barrier, so the
// fold and the append run side by side in one wave.  Block 0 also zeroes
// the step's arrival counters.
constexpr int kPrologueMaxThreads = 7 * 128;  // up to 6 fold groups + the append group

__global__ void __launch_bounds__(kPrologueMaxThreads)
    decode_prologue_kernel(FoldQArgs f, AppendArgs a, int n_fold, int* counters,
                           int n_counters) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
  const int bg = blockIdx.x, grp = threadIdx.x / kFoldThreads, gtid = threadIdx.x % kFoldThreads;
  // One wave of blocks: the scoring grid may take the rest of the SMs and
  // start on its page loads while the fold finishes.
  pdl_launch_dependents();
  if (bg == 0 && counters) {
    pdl_wait();
    for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0;
  }
  const size_t fold_bytes = fold_block_smem(f.Hq / f.Hkv, f.d);
  if (grp < n_fold) {
    fold_query_block(f, bg, grp, reinterpret_cast<float*>(dyn + grp * fold_bytes), gtid,
                     1 + grp);
  } else {
    append_block(a, bg % a.Hkv, 0, bg / a.Hkv,
                 reinterpret_cast<uint16_t*>(dyn + n_fold * fold_bytes), vs, ks, zs, rs, gtid,
                 1 + grp);
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
  const int n_fold = (f.r_v + f.r_k + 31) / 32;
  const bool app = a.k_new != nullptr;
  const int threads = (n_fold + (app ? 1 : 0)) * kFoldThreads;
  if (threads > kPrologueMaxThreads) return cudaErrorInvalidConfiguration;
  size_t smem = (size_t)n_fold * fold_block_smem(f.Hq / f.Hkv, f.d);
  if (app) smem += append_block_smem(a.d, a.r_v, a.r_k);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_prologue_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(decode_prologue_kernel, dim3(f.B * f.Hkv), dim3(threads), smem, st, pdl, f, a,
                  n_fold, counters, n_counters);
}

}  // namespace basiskv
