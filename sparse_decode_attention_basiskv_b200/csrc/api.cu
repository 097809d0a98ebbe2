// C-ABI of the BasisKV decode-attention block: argument validation,
// workspace layout, tensor-map encoding and the launch sequences.
//
// Validation is pure host arithmetic and runs before any CUDA call, so an
// invalid call neither launches nor changes state (and can be exercised on a
// machine without a GPU).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/basiskv.h"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

__device__ unsigned int g_status;  // BASISKV_DEV_* bits, cleared by read_device_status
std::atomic<unsigned long long> g_launches{0};

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices];
int g_sms[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

unsigned int* device_status_ptr() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_status_ptr[dev];
}

int num_sms() {
  const int dev = current_device();
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

bool make_tmap_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                  uint64_t row_bytes, uint32_t box_rows, uint32_t box_cols,
                  CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* out, const void* base, const uint64_t dims[3],
                  const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t gd[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t gs[2] = {strides[0], strides[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gd, gs, bx, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace basiskv

using namespace basiskv;

namespace {

constexpr int kMaxKsplit = 16;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("BASISKV_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

// Effective router widths and kept pages (zero fields select the defaults).
int route_rv(const basiskv_dims* d) { return d->route_r_v ? d->route_r_v : d->r_v; }
int route_rk(const basiskv_dims* d) { return d->route_r_k ? d->route_r_k : d->r_k; }
int sink_pages(const basiskv_dims* d) { return d->sink_pages == 0 ? 1 : (d->sink_pages < 0 ? 0 : d->sink_pages); }
int recent_pages(const basiskv_dims* d) { return d->recent_pages == 0 ? 1 : d->recent_pages; }
// Routing page: tokens per score and per selected page (the cache page by default).
int route_page(const basiskv_dims* d) { return d->route_page ? d->route_page : d->page_size; }
// Scores per cache page.
int route_spp(const basiskv_dims* d) { return d->page_size / route_page(d); }

int check_dims(const basiskv_dims* d) {
  if (!d) return BASISKV_ERR_INVALID_ARG;
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->max_pages_per_seq < 1 ||
      d->num_phys_pages < 1 || d->hidden < 1)
    return BASISKV_ERR_INVALID_ARG;
  if (d->Hq % d->Hkv) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  const int G = d->Hq / d->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->d != 64 && d->d != 128) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->r_v != 32 && d->r_v != 64 && d->r_v != 96 && d->r_v != 128)
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->r_k != 16 && d->r_k != 32 && d->r_k != 64) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->page_size != 8 && d->page_size != 16 && d->page_size != 32)
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->hidden % 128) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (((long)d->Hq * d->r_v) % 64) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if (d->B > 256) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  // Tensor-map row coordinates are 32-bit.
  if ((long long)d->num_phys_pages * d->Hkv * d->page_size >= (1ll << 31))
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  if ((long long)d->max_pages_per_seq * d->page_size >= (1ll << 30))
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  // router widths and kept pages
  if (d->route_r_v < 0 || d->route_r_v > d->r_v || d->route_r_v % 16) return BASISKV_ERR_INVALID_ARG;
  if (d->route_r_k < 0 || d->route_r_k > d->r_k || d->route_r_k % 16) return BASISKV_ERR_INVALID_ARG;
  if (d->recent_pages < 0) return BASISKV_ERR_INVALID_ARG;
  if ((route_rv(d) < d->r_v || route_rk(d) < d->r_k) &&
      !route_narrow_supported(G, d->r_v, d->r_k, route_rv(d), route_rk(d), d->page_size))
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  // routing page
  if (d->route_page != 0 && d->route_page != d->page_size) {
    if (d->route_page != 4 && d->route_page != 8) return BASISKV_ERR_INVALID_ARG;
    if (d->route_page > d->page_size ||
        !(d->cache_fp8 ? route_fp8_subpage_supported(G, d->r_v, d->r_k, route_rv(d),
                                                     route_rk(d), d->page_size, d->route_page)
                       : route_subpage_supported(G, d->r_v, d->r_k, route_rv(d), route_rk(d),
                                                 d->page_size, d->route_page)))
      return BASISKV_ERR_UNSUPPORTED_SHAPE;
  }
  // cache element type
  if (d->cache_fp8 != 0 && d->cache_fp8 != 1) return BASISKV_ERR_INVALID_ARG;
  if (d->cache_fp8 &&
      !(route_fp8_supported(G, d->r_v, d->r_k, route_rv(d), route_rk(d), d->page_size) &&
        attend_mma_fp8_supported(G, d->d, d->r_v, d->page_size)))
    return BASISKV_ERR_UNSUPPORTED_SHAPE;
  return BASISKV_OK;
}

int check_len_topk(const basiskv_dims* d, int top_k, int max_seq_len) {
  if (top_k < 2 || top_k < sink_pages(d) + recent_pages(d)) return BASISKV_ERR_INVALID_ARG;
  if (max_seq_len < 1 || (long long)max_seq_len > (long long)d->max_pages_per_seq * d->page_size)
    return BASISKV_ERR_INVALID_ARG;
  // Page selection keeps a 32-bit key and a block-table entry per page in
  // shared memory.
  const long long P = (max_seq_len + route_page(d) - 1) / route_page(d);
  if (P * 8 > 200 * 1024) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  return BASISKV_OK;
}

}  // namespace

// Shape, length and top_k checks of the decode entry points (host only).
int basiskv::validate_decode_shape(const basiskv_dims* d, int top_k, int max_seq_len) {
  const int rc = check_dims(d);
  return rc ? rc : check_len_topk(d, top_k, max_seq_len);
}

namespace {

struct WsLayout {
  size_t qt, scores, sel, selp, partial, a_f32, a_bf16, op_part, w_app, counters, total;
  int n_att_cnt, n_op_cnt;
  int nsplit, ppi;
};

WsLayout ws_layout(const basiskv_dims* d, int top_k) {
  WsLayout w{};
  const int G = d->Hq / d->Hkv;
  size_t off = 0;
  w.qt = off;
  off += align256((size_t)d->B * d->Hq * (d->r_v + d->r_k) * 4);
  w.scores = off;
  off += align256((size_t)d->B * d->Hkv * d->max_pages_per_seq * route_spp(d) * 4);
  w.sel = off;
  off += align256((size_t)d->B * d->Hkv * top_k * 4);
  w.selp = off;  // physical pages of the selection
  off += align256((size_t)d->B * d->Hkv * top_k * 4);
  w.ppi = attend_pages_per_split(d->page_size);
  w.nsplit = (top_k + w.ppi - 1) / w.ppi;
  w.partial = off;
  size_t slots = (size_t)d->B * d->Hkv * w.nsplit;
  if (attend_mma_supported(G, d->d, d->r_v, d->page_size))
    slots = (size_t)attend_mma_slots(d->B, d->Hkv);
  off += align256(slots * G * (d->r_v + 2) * 4);
  w.a_f32 = off;
  off += align256((size_t)d->B * d->Hq * d->r_v * 4);
  w.a_bf16 = off;
  off += align256((size_t)d->B * d->Hq * d->r_v * 2);
  w.op_part = off;
  off += align256((size_t)kMaxKsplit * d->B * d->hidden * 4);
  w.w_app = off;
  off += align256(append_factor_bytes(d->Hkv, d->d, d->r_v, d->r_k));
  // arrival counters of the fused decode: one per (sequence, KV head) for the
  // attention merge, then one per 128-row tile of the out-projection
  w.n_att_cnt = d->B * d->Hkv;
  w.n_op_cnt = (d->hidden + 127) / 128;
  w.counters = off;
  off += align256((size_t)(w.n_att_cnt + w.n_op_cnt) * 4);
  w.total = off;
  return w;
}

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BASISKV_OK : BASISKV_ERR_LAUNCH_FAILED;
}

CUtensorMapSwizzle swizzle_for_cols(int cols) {
  return cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                    : (cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// Tensor map over a paged cache viewed as [num_phys*Hkv*S rows][width].
bool cache_map(CUtensorMap* m, const void* base, const basiskv_dims* d, int width, int box_cols) {
  const uint64_t rows = (uint64_t)d->num_phys_pages * d->Hkv * d->page_size;
  return make_tmap_2d(m, base, rows, width, (uint64_t)width * 2, d->page_size, box_cols,
                      swizzle_for_cols(box_cols));
}

// z boxes: full 128-byte rows when r_v allows (fewer, larger TMA requests).
int z_box_cols(int r_v) { return r_v % 64 == 0 ? 64 : (r_v % 32 == 0 ? 32 : 16); }
int e_box_cols(int r_k) { return r_k % 32 == 0 ? 32 : 16; }

// ---------------------------------------------------------------- stages
AppendArgs make_append_args(const basiskv_dims* d, const basiskv_bf16* k_new,
                            const basiskv_bf16* v_new, int n_new, int32_t* seq_lens,
                            const int32_t* block_table, const basiskv_bf16* A_V,
                            const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                            basiskv_bf16* K_cache, basiskv_bf16* Z_cache, basiskv_bf16* E_cache) {
  AppendArgs a{};
  a.k_new = k_new;
  a.v_new = v_new;
  a.n_new = n_new;
  a.seq_lens = seq_lens;
  a.seq_lens_out = seq_lens;
  a.block_table = block_table;
  a.A_V = A_V;
  a.P_K = P_K;
  a.U_K = U_K;
  a.K_cache = K_cache;
  a.Z_cache = Z_cache;
  a.E_cache = E_cache;
  a.B = d->B;
  a.Hkv = d->Hkv;
  a.d = d->d;
  a.r_v = d->r_v;
  a.r_k = d->r_k;
  a.S = d->page_size;
  a.max_pages = d->max_pages_per_seq;
  a.num_phys = d->num_phys_pages;
  a.status = device_status_ptr();
  a.zsplit = route_rv(d);
  a.esplit = route_rk(d);
  a.fp8 = d->cache_fp8;
  return a;
}

int run_append(const basiskv_dims* d, const basiskv_bf16* k_new, const basiskv_bf16* v_new,
               int n_new, int32_t* seq_lens, const int32_t* block_table, const basiskv_bf16* A_V,
               const basiskv_bf16* P_K, const basiskv_bf16* U_K, basiskv_bf16* K_cache,
               basiskv_bf16* Z_cache, basiskv_bf16* E_cache, cudaStream_t st, bool pdl,
               bool bump = true, uint16_t* w_app = nullptr, bool fold_first = false) {
  AppendArgs a = make_append_args(d, k_new, v_new, n_new, seq_lens, block_table, A_V, P_K, U_K,
                                  K_cache, Z_cache, E_cache);
  if (!a.status) return BASISKV_ERR_CUDA;
  int rc;
  if (w_app) {  // prefill chunk: one tensor-core product per KV head
    if (fold_first) {
      FoldAppArgs f{A_V, P_K, U_K, w_app, d->Hkv, d->d, d->r_v, d->r_k};
      // no programmatic early start: this kernel reads its inputs without a
      // grid-dependency wait
      rc = launch_status(launch_fold_append(f, st, false));
      if (rc) return rc;
    }
    const int N = d->r_v + d->r_k;
    const uint64_t rows = (uint64_t)d->B * n_new;
    // The five tensor maps depend only on these addresses and sizes; a
    // caller that appends chunk after chunk from the same buffers (a prefill
    // loop) reuses the previous call's maps instead of encoding them again.
    struct MapKey {
      const void *v, *k, *w, *kc;
      uint64_t rows;
      int d, Hkv, N, r_k, slots_rows, fp8;
      bool operator==(const MapKey& o) const {
        return v == o.v && k == o.k && w == o.w && kc == o.kc && rows == o.rows && d == o.d &&
               Hkv == o.Hkv && N == o.N && r_k == o.r_k && slots_rows == o.slots_rows &&
               fp8 == o.fp8;
      }
    };
    struct MapSet {
      bool valid = false;
      MapKey key;
      CUtensorMap v, k, w, wk, kc;
    };
    thread_local MapSet cache;
    const MapKey key{v_new, k_new, w_app, K_cache, rows, d->d, d->Hkv, N, d->r_k,
                     d->num_phys_pages * d->Hkv * d->page_size, d->cache_fp8};
    if (!(cache.valid && cache.key == key)) {
      cache.valid = false;
      const uint64_t dims3[3] = {(uint64_t)d->d, (uint64_t)d->Hkv, rows};
      const uint64_t str3[2] = {(uint64_t)d->d * 2, (uint64_t)d->Hkv * d->d * 2};
      const uint32_t box3[3] = {64, 1, 128};
      if (!make_tmap_3d(&cache.v, v_new, dims3, str3, box3, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !make_tmap_3d(&cache.k, k_new, dims3, str3, box3, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !make_tmap_2d(&cache.w, w_app, (uint64_t)d->Hkv * N, 2 * d->d, (uint64_t)4 * d->d, N,
                        64, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !make_tmap_2d(&cache.wk, w_app, (uint64_t)d->Hkv * N, 2 * d->d, (uint64_t)4 * d->d,
                        d->r_k, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return BASISKV_ERR_CUDA;
      if (d->cache_fp8) {
        cache.kc = cache.k;  // not read: E4M3 Key rows are rounded lane by lane
      } else if (!make_tmap_2d(&cache.kc, K_cache,
                               (uint64_t)d->num_phys_pages * d->Hkv * d->page_size, d->d,
                               (uint64_t)d->d * 2, 8, 64, CU_TENSOR_MAP_SWIZZLE_128B)) {
        return BASISKV_ERR_CUDA;
      }
      cache.key = key;
      cache.valid = true;
    }
    // the tensor-core kernel advances the lengths itself
    return launch_status(
        launch_append_tc(a, cache.v, cache.k, cache.w, cache.wk, cache.kc, bump, st, pdl));
  } else {
    rc = launch_status(launch_append_small(a, st, pdl));
  }
  if (rc || !bump) return rc;
  return launch_status(launch_bump_lengths(a, st, pdl));
}

int run_route(const basiskv_dims* d, const basiskv_bf16* q, const int32_t* seq_lens,
              int max_seq_len, const int32_t* block_table, const basiskv_bf16* P_K,
              const basiskv_bf16* U_K, const basiskv_bf16* Z_cache, const basiskv_bf16* E_cache,
              int top_k, float* scores, int32_t* sel, uint8_t* ws, const WsLayout& L,
              cudaStream_t st, bool pdl, int len_offset = 0, bool do_fold = true,
              const AppendArgs* with_append = nullptr) {
  unsigned int* status = device_status_ptr();
  if (!status) return BASISKV_ERR_CUDA;
  const int wz = z_box_cols(d->r_v), we = e_box_cols(d->r_k);
  CUtensorMap tmZ{}, tmE{};  // bf16 caches only: the E4M3 kernels use plain loads
  if (!d->cache_fp8 &&
      (!cache_map(&tmZ, Z_cache, d, d->r_v, wz) || !cache_map(&tmE, E_cache, d, d->r_k, we)))
    return BASISKV_ERR_CUDA;
  float* qt = reinterpret_cast<float*>(ws + L.qt);
  int rc = BASISKV_OK;
  if (do_fold) {
    FoldQArgs f{q, P_K, U_K, qt, d->B, d->Hq, d->Hkv, d->d, d->r_v, d->r_k};
    rc = launch_status(launch_fold_query(f, st, pdl));
    if (rc) return rc;
  }
  RouteArgs r{};
  r.qt = qt;
  r.Z = Z_cache;
  r.E = E_cache;
  r.seq_lens = seq_lens;
  r.block_table = block_table;
  r.scores = scores;
  r.B = d->B;
  r.Hkv = d->Hkv;
  r.G = d->Hq / d->Hkv;
  r.r_v = d->r_v;
  r.r_k = d->r_k;
  r.S = d->page_size;
  r.max_pages = d->max_pages_per_seq;
  r.num_phys = d->num_phys_pages;
  r.max_seq_len = max_seq_len;
  r.len_offset = len_offset;
  r.status = status;
  r.rb = route_rv(d);
  r.rq = route_rk(d);
  r.fp8 = d->cache_fp8;
  r.rp = route_page(d);
  rc = launch_status(launch_route_scores(r, tmZ, tmE, wz, we, st, pdl));
  if (rc || !sel) return rc;  // no selection requested: scores only
  SelectArgs s{scores, seq_lens, sel, d->B, d->Hkv, route_page(d), d->max_pages_per_seq, top_k,
               max_seq_len, len_offset, block_table,
               route_spp(d) > 1 ? nullptr : reinterpret_cast<int32_t*>(ws + L.selp),
               sink_pages(d), recent_pages(d), route_spp(d)};
  if (with_append) return launch_status(launch_select_append(s, *with_append, st, pdl));
  return launch_status(launch_select(s, st, pdl));
}

AttendArgs make_attend_args(const basiskv_dims* d, const basiskv_bf16* q, const int32_t* seq_lens,
                            const int32_t* block_table, const basiskv_bf16* K_cache,
                            const basiskv_bf16* Z_cache, const int32_t* sel,
                            const int32_t* sel_phys, int top_k, uint8_t* ws, const WsLayout& L,
                            int len_offset, unsigned int* status) {
  AttendArgs a{};
  a.q = q;
  a.K = K_cache;
  a.Z = Z_cache;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.sel = sel;
  a.sel_phys = sel_phys;
  a.zsplit = route_rv(d);
  a.fp8 = d->cache_fp8;
  a.partial = reinterpret_cast<float*>(ws + L.partial);
  a.B = d->B;
  a.Hq = d->Hq;
  a.Hkv = d->Hkv;
  a.G = d->Hq / d->Hkv;
  a.d = d->d;
  a.r_v = d->r_v;
  a.S = d->page_size;
  a.max_pages = d->max_pages_per_seq;
  a.num_phys = d->num_phys_pages;
  a.top_k = top_k;
  a.nsplit = L.nsplit;
  a.pages_per_split = L.ppi;
  a.len_offset = len_offset;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d->d));
  a.status = status;
  return a;
}

// The cluster size of the fused selection + attention launch for this step
// (0: the step takes the separate selection and attention launches).
int fused_cluster(const basiskv_dims* d, int top_k, int max_seq_len) {
  return select_attend_cluster_size(d->Hq / d->Hkv, d->d, d->r_v, d->page_size, route_page(d),
                                    d->cache_fp8, d->B, d->Hkv, max_seq_len, top_k);
}

// Selection and attention of a fused step in one launch (after the scores):
// the bf16 latents to a_bf16, the selection to sel when it is set.
int run_select_attend(const basiskv_dims* d, const basiskv_bf16* q, const int32_t* seq_lens,
                      int max_seq_len, const int32_t* block_table, const basiskv_bf16* K_cache,
                      const basiskv_bf16* Z_cache, int top_k, int32_t* sel, uint16_t* a_bf16,
                      uint8_t* ws, const WsLayout& L, cudaStream_t st, bool pdl, int len_offset) {
  unsigned int* status = device_status_ptr();
  if (!status) return BASISKV_ERR_CUDA;
  SelectArgs s{reinterpret_cast<float*>(ws + L.scores), seq_lens, sel, d->B, d->Hkv,
               route_page(d), d->max_pages_per_seq, top_k, max_seq_len, len_offset,
               block_table, nullptr, sink_pages(d), recent_pages(d), route_spp(d)};
  AttendArgs a = make_attend_args(d, q, seq_lens, block_table, K_cache, Z_cache, nullptr, nullptr,
                                  top_k, ws, L, len_offset, status);
  a.early_inputs = 1;
  a.rp = route_page(d);
  a.a_bf16 = a_bf16;
  return launch_status(launch_select_attend(s, a, st, pdl));
}

int run_attend(const basiskv_dims* d, const basiskv_bf16* q, const int32_t* seq_lens,
               const int32_t* block_table, const basiskv_bf16* K_cache,
               const basiskv_bf16* Z_cache, const int32_t* sel, int top_k, float* a_lat,
               uint16_t* a_bf16, uint8_t* ws, const WsLayout& L, cudaStream_t st, bool pdl,
               int len_offset = 0, int* cnt = nullptr, const int32_t* sel_phys = nullptr) {
  unsigned int* status = device_status_ptr();
  if (!status) return BASISKV_ERR_CUDA;
  const int wz = z_box_cols(d->r_v);
  CUtensorMap tmK{}, tmZ{};  // bf16 caches only: the E4M3 kernel uses plain loads
  if (!d->cache_fp8 &&
      (!cache_map(&tmK, K_cache, d, d->d, 64) || !cache_map(&tmZ, Z_cache, d, d->r_v, wz)))
    return BASISKV_ERR_CUDA;
  AttendArgs a = make_attend_args(d, q, seq_lens, block_table, K_cache, Z_cache, sel, sel_phys,
                                  top_k, ws, L, len_offset, status);
  if (attend_mma_supported(a.G, a.d, a.r_v, a.S)) {
    a.early_inputs = cnt != nullptr;  // inside the fused step: follows the selection launch
    if (!cnt) {  // a standalone call: the arrival counters start from zero here
      cnt = reinterpret_cast<int*>(ws + L.counters);
      if (cudaMemsetAsync(cnt, 0, (size_t)L.n_att_cnt * 4, st) != cudaSuccess)
        return BASISKV_ERR_LAUNCH_FAILED;
    }
    a.cnt = cnt;
    a.a_lat = a_lat;
    a.a_bf16 = a_bf16;
    return launch_status(launch_attend_mma(a, st, pdl));
  }
  // Fused merge of the splits when its shared-memory scratch stays small.
  if (cnt && (size_t)2 * L.nsplit * a.G * 4 <= 4096) {
    a.cnt = cnt;
    a.a_lat = a_lat;
    a.a_bf16 = a_bf16;
    return launch_status(launch_attend(a, tmK, tmZ, wz, st, pdl));
  }
  int rc = launch_status(launch_attend(a, tmK, tmZ, wz, st, pdl));
  if (rc) return rc;
  CombineArgs c{a.partial, seq_lens, a_lat, a_bf16, d->B, d->Hq, d->Hkv, a.G, d->r_v,
                d->page_size, top_k, L.nsplit, L.ppi, len_offset};
  return launch_status(launch_combine(c, st, pdl));
}

// n_src > 1: the latents are stored source-major, [n_src][B][K / n_src].
int run_outproj(const basiskv_dims* d, const uint16_t* a_bf16, const basiskv_bf16* W_fold,
                basiskv_bf16* y, uint8_t* ws, const WsLayout& L, cudaStream_t st, bool pdl,
                int32_t* bump_lens = nullptr, int* cnt = nullptr, int n_src = 1) {
  unsigned int* status = device_status_ptr();
  if (!status) return BASISKV_ERR_CUDA;
  const int K = d->Hq * d->r_v, K_src = K / n_src;
  const int bn = outproj_bn(d->B);
  CUtensorMap tmW, tmA;
  if (!make_tmap_2d(&tmW, W_fold, d->hidden, K, (uint64_t)K * 2, 128, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tmA, a_bf16, (uint64_t)n_src * d->B, K_src, (uint64_t)K_src * 2, bn, 64,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return BASISKV_ERR_CUDA;
  OutprojArgs o{};
  o.partial = reinterpret_cast<float*>(ws + L.op_part);
  o.y = y;
  o.B = d->B;
  o.H = d->hidden;
  o.K = K;
  o.ksplit = outproj_ksplit(d->hidden, K, d->B);
  if (o.ksplit > kMaxKsplit) o.ksplit = kMaxKsplit;
  o.bn = bn;
  o.status = status;
  o.bump_lens = bump_lens;
  o.bump_n = 1;
  o.bump_cap = d->max_pages_per_seq * d->page_size;
  o.cnt = cnt;
  o.k_src = K_src;
  return launch_status(launch_outproj(o, tmW, tmA, st, pdl));
}

int check_ws(const basiskv_dims* d, int top_k, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = ws_layout(d, top_k);
  if (!ws) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return BASISKV_ERR_INVALID_ARG;
  if (ws_bytes < L->total) return BASISKV_ERR_WORKSPACE_TOO_SMALL;
  return BASISKV_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// bf16 tensors: non-null and 16-byte aligned (TMA and vector loads).
#define BKV_REQUIRE(p)                                         \
  do {                                                         \
    if (!(p) || !aligned16(p)) return BASISKV_ERR_INVALID_ARG; \
  } while (0)
// int32 / fp32 arrays: non-null and 4-byte aligned.
#define BKV_REQUIRE4(p)                                       \
  do {                                                        \
    if (!(p) || !aligned4(p)) return BASISKV_ERR_INVALID_ARG; \
  } while (0)

}  // namespace

extern "C" {

size_t basiskv_workspace_size(const basiskv_dims* dims, int top_k, int max_seq_len) {
  if (check_dims(dims) != BASISKV_OK || check_len_topk(dims, top_k, max_seq_len) != BASISKV_OK)
    return 0;
  return ws_layout(dims, top_k).total;
}

int basiskv_fold_outproj(const basiskv_dims* dims, const basiskv_bf16* B_V,
                         const basiskv_bf16* W_O, basiskv_bf16* W_fold, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  BKV_REQUIRE(B_V);
  BKV_REQUIRE(W_O);
  BKV_REQUIRE(W_fold);
  FoldOutArgs a{B_V, W_O, W_fold, dims->Hq, dims->Hkv, dims->d, dims->r_v, dims->hidden};
  return launch_status(launch_fold_outproj(a, static_cast<cudaStream_t>(stream)));
}

int basiskv_fold_append(const basiskv_dims* dims, const basiskv_bf16* A_V,
                        const basiskv_bf16* P_K, const basiskv_bf16* U_K, basiskv_bf16* W_app,
                        void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  BKV_REQUIRE(A_V);
  BKV_REQUIRE(P_K);
  BKV_REQUIRE(U_K);
  BKV_REQUIRE(W_app);
  FoldAppArgs f{A_V, P_K, U_K, W_app, dims->Hkv, dims->d, dims->r_v, dims->r_k};
  return launch_status(launch_fold_append(f, static_cast<cudaStream_t>(stream), false));
}

int basiskv_append(const basiskv_dims* dims, const basiskv_bf16* k_new, const basiskv_bf16* v_new,
                   int n_new, int32_t* seq_lens, const int32_t* block_table,
                   const basiskv_bf16* A_V, const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                   const basiskv_bf16* W_app, basiskv_bf16* K_cache, basiskv_bf16* Z_cache, basiskv_bf16* E_cache,
                   void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n_new < 1 || (long long)n_new > (long long)dims->max_pages_per_seq * dims->page_size)
    return BASISKV_ERR_INVALID_ARG;
  BKV_REQUIRE(k_new);
  BKV_REQUIRE(v_new);
  BKV_REQUIRE4(seq_lens);
  BKV_REQUIRE4(block_table);
  BKV_REQUIRE(A_V);
  BKV_REQUIRE(P_K);
  BKV_REQUIRE(U_K);
  BKV_REQUIRE(K_cache);
  BKV_REQUIRE(Z_cache);
  BKV_REQUIRE(E_cache);
  // Chunks of at least 128 token rows take the tensor-core path; without a
  // caller-folded W_app the fold goes to the workspace first.
  uint16_t* w_ws = nullptr;
  const bool tc = (long long)dims->B * n_new >= 128;
  if (tc && W_app && !aligned16(W_app)) return BASISKV_ERR_INVALID_ARG;
  if (tc && !W_app) {
    WsLayout L;
    rc = check_ws(dims, 2, workspace, workspace_bytes, &L);
    if (rc) return rc;
    w_ws = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + L.w_app);
  }
  return run_append(dims, k_new, v_new, n_new, seq_lens, block_table, A_V, P_K, U_K, K_cache,
                    Z_cache, E_cache, static_cast<cudaStream_t>(stream), pdl_enabled(), true,
                    tc ? (W_app ? const_cast<uint16_t*>(W_app) : w_ws) : nullptr,
                    tc && !W_app);
}

int basiskv_route(const basiskv_dims* dims, const basiskv_bf16* q, const int32_t* seq_lens,
                  int max_seq_len, const int32_t* block_table, const basiskv_bf16* P_K,
                  const basiskv_bf16* U_K, const basiskv_bf16* Z_cache,
                  const basiskv_bf16* E_cache, int top_k, float* page_scores, int32_t* sel,
                  void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_len_topk(dims, top_k, max_seq_len);
  if (rc) return rc;
  BKV_REQUIRE(q);
  BKV_REQUIRE4(seq_lens);
  BKV_REQUIRE4(block_table);
  BKV_REQUIRE(P_K);
  BKV_REQUIRE(U_K);
  BKV_REQUIRE(Z_cache);
  BKV_REQUIRE(E_cache);
  if (!sel && !page_scores) return BASISKV_ERR_INVALID_ARG;  // nothing to write
  if (sel && !aligned4(sel)) return BASISKV_ERR_INVALID_ARG;
  if (page_scores && !aligned4(page_scores)) return BASISKV_ERR_INVALID_ARG;
  WsLayout L;
  rc = check_ws(dims, top_k, workspace, workspace_bytes, &L);
  if (rc) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scores = page_scores ? page_scores : reinterpret_cast<float*>(ws + L.scores);
  return run_route(dims, q, seq_lens, max_seq_len, block_table, P_K, U_K, Z_cache, E_cache, top_k,
                   scores, sel, ws, L, static_cast<cudaStream_t>(stream), pdl_enabled());
}

int basiskv_attend(const basiskv_dims* dims, const basiskv_bf16* q, const int32_t* seq_lens,
                   int max_seq_len, const int32_t* block_table, const basiskv_bf16* K_cache,
                   const basiskv_bf16* Z_cache, const int32_t* sel, int top_k, float* a_lat,
                   void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_len_topk(dims, top_k, max_seq_len);
  if (rc) return rc;
  if (route_spp(dims) > 1) return BASISKV_ERR_UNSUPPORTED_SHAPE;  // takes cache pages only
  BKV_REQUIRE(q);
  BKV_REQUIRE4(seq_lens);
  BKV_REQUIRE4(block_table);
  BKV_REQUIRE(K_cache);
  BKV_REQUIRE(Z_cache);
  BKV_REQUIRE4(sel);
  BKV_REQUIRE4(a_lat);
  WsLayout L;
  rc = check_ws(dims, top_k, workspace, workspace_bytes, &L);
  if (rc) return rc;
  return run_attend(dims, q, seq_lens, block_table, K_cache, Z_cache, sel, top_k, a_lat, nullptr,
                    static_cast<uint8_t*>(workspace), L, static_cast<cudaStream_t>(stream),
                    pdl_enabled());
}

int basiskv_outproj(const basiskv_dims* dims, const float* a_lat, const basiskv_bf16* W_fold,
                    basiskv_bf16* y, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  BKV_REQUIRE4(a_lat);
  BKV_REQUIRE(W_fold);
  BKV_REQUIRE(y);
  WsLayout L;
  rc = check_ws(dims, 2, workspace, workspace_bytes, &L);
  if (rc) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* a16 = reinterpret_cast<uint16_t*>(ws + L.a_bf16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pdl = pdl_enabled();
  rc = launch_status(launch_cast_bf16(a_lat, a16, (size_t)dims->B * dims->Hq * dims->r_v, st, pdl));
  if (rc) return rc;
  return run_outproj(dims, a16, W_fold, y, ws, L, st, pdl);
}

int basiskv_decode(const basiskv_dims* dims, const basiskv_bf16* q, const basiskv_bf16* k_new,
                   const basiskv_bf16* v_new, int32_t* seq_lens, int max_seq_len,
                   const int32_t* block_table, const basiskv_bf16* A_V, const basiskv_bf16* P_K,
                   const basiskv_bf16* U_K, const basiskv_bf16* W_fold, basiskv_bf16* K_cache,
                   basiskv_bf16* Z_cache, basiskv_bf16* E_cache, int top_k, int32_t* sel,
                   basiskv_bf16* y, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_len_topk(dims, top_k, max_seq_len);
  if (rc) return rc;
  const bool append = k_new || v_new;
  if (append) {
    BKV_REQUIRE(k_new);
    BKV_REQUIRE(v_new);
    BKV_REQUIRE(A_V);
    BKV_REQUIRE(K_cache);
    BKV_REQUIRE(E_cache);
  }
  BKV_REQUIRE(q);
  BKV_REQUIRE4(seq_lens);
  BKV_REQUIRE4(block_table);
  BKV_REQUIRE(P_K);
  BKV_REQUIRE(U_K);
  BKV_REQUIRE(W_fold);
  BKV_REQUIRE(K_cache);
  BKV_REQUIRE(Z_cache);
  BKV_REQUIRE(E_cache);
  BKV_REQUIRE(y);
  if (sel && !aligned4(sel)) return BASISKV_ERR_INVALID_ARG;
  WsLayout L;
  rc = check_ws(dims, top_k, workspace, workspace_bytes, &L);
  if (rc) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pdl = pdl_enabled();
  int32_t* sel_buf = sel ? sel : reinterpret_cast<int32_t*>(ws + L.sel);
  // With an append, the new token is written first; the lengths are bumped
  // only at the end of the step (by the out-projection launch), and the
  // stages in between read seq_lens[b] + 1.
  const int off = append ? 1 : 0;
  // Launch 1: the query fold; it also zeroes the arrival counters of the
  // fused merges and reduction below.  When the selection and the attention
  // share one launch (groups that fit one wave of CTA clusters), launch 1
  // also appends the token, and the scoring (launch 2) may start before the
  // token lands: it reads the newest page either way, which only changes
  // that page's score, and the newest page is selected whatever its score
  // (its score is not an output of this call).  Otherwise the append runs in
  // the selection launch, after the scoring.
  int* cnt = reinterpret_cast<int*>(ws + L.counters);
  AppendArgs app = make_append_args(dims, append ? k_new : nullptr, v_new, 1, seq_lens,
                                    block_table, A_V, P_K, U_K, K_cache, Z_cache, E_cache);
  if (!app.status) return BASISKV_ERR_CUDA;
  const bool fused = fused_cluster(dims, top_k, max_seq_len) > 0;
  if (route_spp(dims) > 1 && !fused) return BASISKV_ERR_UNSUPPORTED_SHAPE;  // routing pages
  {
    FoldQArgs f{q, P_K, U_K, reinterpret_cast<float*>(ws + L.qt), dims->B, dims->Hq, dims->Hkv,
                dims->d, dims->r_v, dims->r_k};
    AppendArgs first = app;
    if (!fused) first.k_new = nullptr;  // the append then runs in the selection launch
    rc = launch_status(
        launch_decode_prologue(f, first, cnt, L.n_att_cnt + L.n_op_cnt, st, pdl));
    if (rc) return rc;
  }
  uint16_t* a16 = reinterpret_cast<uint16_t*>(ws + L.a_bf16);
  if (fused) {
    rc = run_route(dims, q, seq_lens, max_seq_len, block_table, P_K, U_K, Z_cache, E_cache, top_k,
                   reinterpret_cast<float*>(ws + L.scores), nullptr, ws, L, st, pdl, off,
                   /*do_fold=*/false);
    if (rc) return rc;
    rc = run_select_attend(dims, q, seq_lens, max_seq_len, block_table, K_cache, Z_cache, top_k,
                           sel, a16, ws, L, st, pdl, off);
  } else {
    rc = run_route(dims, q, seq_lens, max_seq_len, block_table, P_K, U_K, Z_cache, E_cache,
                   top_k, reinterpret_cast<float*>(ws + L.scores), sel_buf, ws, L, st, pdl, off,
                   /*do_fold=*/false, append ? &app : nullptr);
    if (rc) return rc;
    rc = run_attend(dims, q, seq_lens, block_table, K_cache, Z_cache, sel_buf, top_k, nullptr,
                    a16, ws, L, st, pdl, off, cnt,
                    reinterpret_cast<const int32_t*>(ws + L.selp));
  }
  if (rc) return rc;
  return run_outproj(dims, a16, W_fold, y, ws, L, st, pdl, append ? seq_lens : nullptr,
                     cnt + L.n_att_cnt);
}

int basiskv_decode_latents(const basiskv_dims* dims, const basiskv_bf16* q,
                           const basiskv_bf16* k_new, const basiskv_bf16* v_new,
                           int32_t* seq_lens, int max_seq_len, const int32_t* block_table,
                           const basiskv_bf16* A_V, const basiskv_bf16* P_K,
                           const basiskv_bf16* U_K, basiskv_bf16* K_cache, basiskv_bf16* Z_cache,
                           basiskv_bf16* E_cache, int top_k, int32_t* sel, basiskv_bf16* a_out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_len_topk(dims, top_k, max_seq_len);
  if (rc) return rc;
  const bool append = k_new || v_new;
  if (append) {
    BKV_REQUIRE(k_new);
    BKV_REQUIRE(v_new);
    BKV_REQUIRE(A_V);
  }
  BKV_REQUIRE(q);
  BKV_REQUIRE4(seq_lens);
  BKV_REQUIRE4(block_table);
  BKV_REQUIRE(P_K);
  BKV_REQUIRE(U_K);
  BKV_REQUIRE(K_cache);
  BKV_REQUIRE(Z_cache);
  BKV_REQUIRE(E_cache);
  BKV_REQUIRE(a_out);
  if (sel && !aligned4(sel)) return BASISKV_ERR_INVALID_ARG;
  WsLayout L;
  rc = check_ws(dims, top_k, workspace, workspace_bytes, &L);
  if (rc) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool pdl = pdl_enabled();
  int32_t* sel_buf = sel ? sel : reinterpret_cast<int32_t*>(ws + L.sel);
  const int off = append ? 1 : 0;
  int* cnt = reinterpret_cast<int*>(ws + L.counters);
  AppendArgs app = make_append_args(dims, append ? k_new : nullptr, v_new, 1, seq_lens,
                                    block_table, A_V, P_K, U_K, K_cache, Z_cache, E_cache);
  if (!app.status) return BASISKV_ERR_CUDA;
  const bool fused = fused_cluster(dims, top_k, max_seq_len) > 0;  // as in basiskv_decode
  if (route_spp(dims) > 1 && !fused) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  {
    FoldQArgs f{q, P_K, U_K, reinterpret_cast<float*>(ws + L.qt), dims->B, dims->Hq, dims->Hkv,
                dims->d, dims->r_v, dims->r_k};
    AppendArgs first = app;
    if (!fused) first.k_new = nullptr;
    rc = launch_status(launch_decode_prologue(f, first, cnt, L.n_att_cnt, st, pdl));
    if (rc) return rc;
  }
  if (fused) {
    rc = run_route(dims, q, seq_lens, max_seq_len, block_table, P_K, U_K, Z_cache, E_cache, top_k,
                   reinterpret_cast<float*>(ws + L.scores), nullptr, ws, L, st, pdl, off,
                   /*do_fold=*/false);
    if (rc) return rc;
    rc = run_select_attend(dims, q, seq_lens, max_seq_len, block_table, K_cache, Z_cache, top_k,
                           sel, a_out, ws, L, st, pdl, off);
  } else {
    rc = run_route(dims, q, seq_lens, max_seq_len, block_table, P_K, U_K, Z_cache, E_cache,
                   top_k, reinterpret_cast<float*>(ws + L.scores), sel_buf, ws, L, st, pdl, off,
                   /*do_fold=*/false, append ? &app : nullptr);
    if (rc) return rc;
    rc = run_attend(dims, q, seq_lens, block_table, K_cache, Z_cache, sel_buf, top_k, nullptr,
                    a_out, ws, L, st, pdl, off, cnt,
                    reinterpret_cast<const int32_t*>(ws + L.selp));
  }
  if (rc || !append) return rc;
  return launch_status(launch_bump_lengths(app, st, pdl));  // after every reader
}

int basiskv_outproj_sources(const basiskv_dims* dims, const basiskv_bf16* a_src, int n_src,
                            const basiskv_bf16* W_fold, basiskv_bf16* y, void* workspace,
                            size_t workspace_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n_src < 1 || dims->Hq % n_src) return BASISKV_ERR_INVALID_ARG;
  if ((dims->Hq / n_src * dims->r_v) % 64) return BASISKV_ERR_UNSUPPORTED_SHAPE;
  BKV_REQUIRE(a_src);
  BKV_REQUIRE(W_fold);
  BKV_REQUIRE(y);
  WsLayout L;
  rc = check_ws(dims, 2, workspace, workspace_bytes, &L);
  if (rc) return rc;
  return run_outproj(dims, a_src, W_fold, y, static_cast<uint8_t*>(workspace), L,
                     static_cast<cudaStream_t>(stream), pdl_enabled(), nullptr, nullptr, n_src);
}

int basiskv_read_device_status(void* stream, uint32_t* flags) {
  if (!flags) return BASISKV_ERR_INVALID_ARG;
  *flags = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return BASISKV_ERR_CUDA;
  unsigned int* p = device_status_ptr();
  if (!p) return BASISKV_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return BASISKV_ERR_CUDA;
  if (v && cudaMemset(p, 0, sizeof(v)) != cudaSuccess) return BASISKV_ERR_CUDA;
  *flags = v;
  return v ? BASISKV_ERR_DEVICE : BASISKV_OK;
}

uint64_t basiskv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* basiskv_strerror(int status) {
  switch (status) {
    case BASISKV_OK: return "ok";
    case BASISKV_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer or bad count)";
    case BASISKV_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BASISKV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case BASISKV_ERR_LAUNCH_FAILED: return "kernel launch failed";
    case BASISKV_ERR_DEVICE: return "device reported an error (see device status bits)";
    case BASISKV_ERR_CUDA: return "CUDA runtime call failed";
    case BASISKV_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the static no-alloc buffer holds";
    default: return "unknown status";
  }
}

}  // extern "C"
