// basiskv_decode_noalloc: the fused decode step for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run a decode step: an embedding runtime that owns all device memory
// through its own pool and forbids side allocations, a plug-in invoked from
// a host callback where allocation is not allowed, or a program that must
// keep its memory footprint fixed after start-up.  They still own and pass
// every input and output; only the scratch that basiskv_decode needs comes
// from a fixed array compiled into this library instead of a caller-supplied
// workspace.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits.  Host
// code must not hand the array's symbol to a kernel (on the host it is only
// a stand-in, not a device address): its device address is looked up once
// per device with cudaGetSymbolAddress, with that device current, the first
// time the entry point runs there.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/basiskv.h"

namespace {

constexpr size_t kNoallocScratchBytes = BASISKV_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr if the lookup fails.
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

int basiskv_decode_noalloc(const basiskv_dims* dims, const basiskv_bf16* q,
                           const basiskv_bf16* k_new, const basiskv_bf16* v_new,
                           int32_t* seq_lens, int max_seq_len, const int32_t* block_table,
                           const basiskv_bf16* A_V, const basiskv_bf16* P_K,
                           const basiskv_bf16* U_K, const basiskv_bf16* W_fold,
                           basiskv_bf16* K_cache, basiskv_bf16* Z_cache, basiskv_bf16* E_cache,
                           int top_k, int32_t* sel, basiskv_bf16* y, void* stream) {
  const size_t need = basiskv_workspace_size(dims, top_k, max_seq_len);
  if (need == 0)  // dims, top_k or length rejected: let the decode report which
    return basiskv_decode(dims, q, k_new, v_new, seq_lens, max_seq_len, block_table, A_V, P_K,
                          U_K, W_fold, K_cache, Z_cache, E_cache, top_k, sel, y, nullptr, 0,
                          stream);
  if (need > kNoallocScratchBytes) return BASISKV_ERR_SCRATCH_LIMIT;
  void* scratch = scratch_for_current_device();
  if (!scratch) return BASISKV_ERR_CUDA;
  return basiskv_decode(dims, q, k_new, v_new, seq_lens, max_seq_len, block_table, A_V, P_K, U_K,
                        W_fold, K_cache, Z_cache, E_cache, top_k, sel, y, scratch,
                        kNoallocScratchBytes, stream);
}

}  // extern "C"
