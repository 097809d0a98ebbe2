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
// a stand-in, not a device address): its device address is looked up with
// cudaGetSymbolAddress in the caller's current context, on every call made
// outside stream capture.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/basiskv.h"
#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = BASISKV_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// The array's address belongs to one CUDA context (the module is loaded per
// context), so it is cached per context, not per device number: after a
// cudaDeviceReset, or under another context on the same device, the old
// address is stale.  Outside stream capture every call looks the address up
// again (a cheap table lookup once the module is loaded) and refreshes the
// cache; during capture, where a lookup that loads the module is not
// allowed, the cached address of the current context is used.
constexpr int kMaxContexts = 64;
std::mutex g_mu;
CUcontext g_ctx[kMaxContexts];
void* g_ptr[kMaxContexts];
int g_n;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array in the current context, or nullptr.
void* scratch_for_current_context(cudaStream_t st) {
  // (a runtime call first: it makes the device's primary context current
  // when the caller has none yet)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return nullptr;
  const CUcontext ctx = current_context();
  if (!ctx) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  int slot = -1;
  for (int i = 0; i < g_n; ++i)
    if (g_ctx[i] == ctx) slot = i;
  if (cap != cudaStreamCaptureStatusNone) return slot >= 0 ? g_ptr[slot] : nullptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  if (slot < 0) {
    slot = g_n < kMaxContexts ? g_n++ : (int)(reinterpret_cast<uintptr_t>(ctx) % kMaxContexts);
    g_ctx[slot] = ctx;
  }
  g_ptr[slot] = p;
  return p;
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
  const int rc = basiskv::validate_decode_shape(dims, top_k, max_seq_len);
  if (rc) return rc;
  if (basiskv_workspace_size(dims, top_k, max_seq_len) > kNoallocScratchBytes)
    return BASISKV_ERR_SCRATCH_LIMIT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = scratch_for_current_context(st);
  if (!scratch) return BASISKV_ERR_CUDA;
  return basiskv_decode(dims, q, k_new, v_new, seq_lens, max_seq_len, block_table, A_V, P_K, U_K,
                        W_fold, K_cache, Z_cache, E_cache, top_k, sel, y, scratch,
                        kNoallocScratchBytes, stream);
}

}  // extern "C"
