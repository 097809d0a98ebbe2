// Host-side interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/basiskv.h"

namespace basiskv {

// Encodes a 2-D bf16 tensor map: `rows` rows of `cols` elements with a row
// pitch of `row_bytes`, boxes of box_rows x box_cols, the given swizzle.
// Returns false when the driver rejects the description.
bool make_tmap_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                  uint64_t row_bytes, uint32_t box_rows, uint32_t box_cols,
                  CUtensorMapSwizzle swizzle);
// 3-D bf16 tensor map, dims innermost first, byte strides of dims 1 and 2.
bool make_tmap_3d(CUtensorMap* out, const void* base, const uint64_t dims[3],
                  const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle);

// Address of this library's device status word on the current device.
unsigned int* device_status_ptr();
// BASISKV_OK, or the status basiskv_decode returns for these dims, top_k and
// max_seq_len (host arithmetic only, before any CUDA call).
int validate_decode_shape(const basiskv_dims* d, int top_k, int max_seq_len);

int num_sms();

// ------------------------------------------------------------------ append
struct AppendArgs {
  const uint16_t* k_new;  // [B][n_new][Hkv][d]
  const uint16_t* v_new;
  int n_new;
  const int32_t* seq_lens;
  int32_t* seq_lens_out;
  const int32_t* block_table;
  const uint16_t* A_V;
  const uint16_t* P_K;
  const uint16_t* U_K;
  uint16_t* K_cache;
  uint16_t* Z_cache;
  uint16_t* E_cache;
  int B, Hkv, d, r_v, r_k, S, max_pages, num_phys;
  unsigned int* status;
  int zsplit, esplit;  // Z / E tiles store their first zsplit / esplit columns first
  int fp8;  // the three caches hold E4M3 bytes (pointers reinterpreted)
};
cudaError_t launch_append_small(const AppendArgs& a, cudaStream_t st, bool pdl);

// Prefill path (tensor cores): W_app = [[A_V^T, 0], [-(A_V P_K U_K)^T, U_K^T]]
// per KV head, [Hkv][r_v + r_k][2d] bf16, then [z | e] = [v | k] W_app^T.
struct FoldAppArgs {
  const uint16_t* A_V;
  const uint16_t* P_K;
  const uint16_t* U_K;
  uint16_t* W_app;
  int Hkv, d, r_v, r_k;
};
size_t append_factor_bytes(int Hkv, int d, int r_v, int r_k);
cudaError_t launch_fold_append(const FoldAppArgs& a, cudaStream_t st, bool pdl);
// tmV, tmK: 3-D maps over [rows][Hkv][d] (box 64 x 1 x 128); tmW: 2-D map over
// [Hkv*(r_v+r_k)][2d] (box (r_v+r_k) x 64); all with 128-byte swizzle.
// tmWk: the same W_app map with a box of r_k rows (the residual rows of the
// k k-blocks).  tmKc: the bf16 Key cache as [num_phys * Hkv * S][d] (box
// 8 x 64, 128-byte swizzle), the target of the Key's TMA stores (unused for
// E4M3 caches).
// bump: the kernel also advances seq_lens by n_new (its last CTA to read
// them does it); calls whose launches overlap on the device (other streams)
// use different arrival slots, up to 64 at once.
cudaError_t launch_append_tc(const AppendArgs& a, const CUtensorMap& tmV, const CUtensorMap& tmK,
                             const CUtensorMap& tmW, const CUtensorMap& tmWk,
                             const CUtensorMap& tmKc, bool bump, cudaStream_t st, bool pdl);
cudaError_t launch_bump_lengths(const AppendArgs& a, cudaStream_t st, bool pdl);

// ------------------------------------------------------------------- route
struct FoldQArgs {
  const uint16_t* q;    // [B][Hq][d]
  const uint16_t* P_K;  // [Hkv][r_v][d]
  const uint16_t* U_K;  // [Hkv][d][r_k]
  float* qt;            // [B][Hq][r_v + r_k]
  int B, Hq, Hkv, d, r_v, r_k;
};
cudaError_t launch_fold_query(const FoldQArgs& a, cudaStream_t st, bool pdl);
// First launch of a fused decode step: the query fold, one block per 32
// outputs of each (sequence, KV head), and (when a.k_new is set) the
// one-token append, one more block per (sequence, KV head); n_counters ints
// at `counters` are zeroed.
cudaError_t launch_decode_prologue(const FoldQArgs& f, const AppendArgs& a, int* counters,
                                   int n_counters, cudaStream_t st, bool pdl);

struct RouteArgs {
  const float* qt;  // [B][Hq][r_v + r_k]
  const uint16_t* Z;  // Z cache [num_phys][Hkv][S][r_v] (plain-load kernel)
  const uint16_t* E;  // E cache [num_phys][Hkv][S][r_k]
  const int32_t* seq_lens;
  const int32_t* block_table;
  float* scores;  // [B][Hkv][max_pages]
  int B, Hkv, G, r_v, r_k, S, max_pages, num_phys, max_seq_len;
  int len_offset;  // added to seq_lens[b] (tokens appended in this step, not yet counted)
  unsigned int* status;
  int rb, rq;  // widths the router reads: z[:, :rb], e[:, :rq]
  int fp8;     // Z and E hold E4M3 bytes
  int rp;      // routing page (tokens per score); S: one score per cache page
};
// Whether the plain-load scoring kernel has an instance for routing pages
// of rp < S tokens with this router.
bool route_subpage_supported(int G, int r_v, int r_k, int rb, int rq, int S, int rp);
// Whether the plain-load scoring kernel has an instance for a router
// narrower than the cached widths.
bool route_narrow_supported(int G, int r_v, int r_k, int rb, int rq, int S);
// Whether it has an instance over E4M3 caches for this router.
bool route_fp8_supported(int G, int r_v, int r_k, int rb, int rq, int S);
bool route_fp8_subpage_supported(int G, int r_v, int r_k, int rb, int rq, int S, int rp);
cudaError_t launch_route_scores_fp8(const RouteArgs& a, cudaStream_t st, bool pdl);
cudaError_t launch_route_scores(const RouteArgs& a, const CUtensorMap& tmZ,
                                const CUtensorMap& tmE, int wz, int we, cudaStream_t st,
                                bool pdl);

struct SelectArgs {
  const float* scores;  // [B][Hkv][max_pages * spp]
  const int32_t* seq_lens;
  int32_t* sel;  // [B][Hkv][top_k]
  int B, Hkv, S, max_pages, top_k, max_seq_len;
  int len_offset;
  // Optional: the physical page of each selected entry (block-table lookup
  // done here, so the attention kernel reads page ids in one round trip).
  const int32_t* block_table;
  int32_t* sel_phys;  // [B][Hkv][top_k] or null
  int n_sink, n_recent;  // leading / trailing pages always kept
  // Scores per cache page (routing pages of S tokens each, S above being
  // the routing page): 1, or page_size / route_page (sel_phys then null).
  int spp;
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl);
// The selection together with a one-token append (a.n_new == 1), whose
// result no stage before the attention reads.
cudaError_t launch_select_append(const SelectArgs& s, const AppendArgs& a, cudaStream_t st,
                                 bool pdl);

// ------------------------------------------------------------------ attend
struct AttendArgs {
  const uint16_t* q;
  const uint16_t* K;  // exact-Key cache [num_phys][Hkv][S][d] (plain-load kernel)
  const uint16_t* Z;  // Value-latent cache [num_phys][Hkv][S][r_v]
  const int32_t* seq_lens;
  const int32_t* block_table;
  const int32_t* sel;
  const int32_t* sel_phys;  // physical pages of sel (null: look them up)
  float* partial;  // [B*Hkv][nsplit][G][r_v + 2]
  int B, Hq, Hkv, G, d, r_v, S, max_pages, num_phys, top_k, nsplit, pages_per_split;
  int len_offset;
  float scale_log2;  // log2(e) / sqrt(d)
  unsigned int* status;
  // Fused merge of the splits (when cnt is set): per (sequence, KV head) an
  // arrival counter, zeroed before the launch; the CTA that writes a group's
  // last split merges them into a_lat / a_bf16.
  int* cnt;
  float* a_lat;
  uint16_t* a_bf16;
  // Set when this launch follows another kernel of the same call (never a
  // caller's kernel): the queries and lengths are then read before the
  // grid-dependency wait.
  int early_inputs;
  int zsplit;  // Z tiles store their first zsplit columns first
  int fp8;     // K and Z hold E4M3 bytes
  int rp;      // routing page: sel holds routing pages of rp tokens (rp <= S)
};
int attend_pages_per_split(int S);
// Plain-load tensor-core attention with its own merge (needs a.cnt zeroed,
// a.partial of attend_mma_slots(B, Hkv) * G * (r_v + 2) floats); returns
// cudaErrorNotSupported for shapes it does not cover.
bool attend_mma_supported(int G, int d, int r_v, int S);
// Its E4M3 form (a subset of the shapes above).
bool attend_mma_fp8_supported(int G, int d, int r_v, int S);
cudaError_t launch_attend_mma_fp8(const AttendArgs& a, cudaStream_t st, bool pdl);
int attend_mma_slots(int B, int Hkv);
cudaError_t launch_attend_mma(const AttendArgs& a, cudaStream_t st, bool pdl);
// Selection and attention of a fused decode step in one launch, one cluster
// of CTAs per (sequence, KV head) (select_attend.cuh).  The cluster size for
// a step, or 0 when the step does not fit one wave (then the selection and
// the attention launch separately).  s.sel, when set, receives the selection.
int select_attend_cluster_size(int G, int d, int r_v, int S, int rp, int fp8, int B, int Hkv,
                               int max_seq_len, int top_k);
cudaError_t launch_select_attend(const SelectArgs& s, const AttendArgs& a, cudaStream_t st,
                                 bool pdl);
cudaError_t launch_select_attend_fp8(const SelectArgs& s, const AttendArgs& a, cudaStream_t st,
                                     bool pdl);
cudaError_t launch_attend(const AttendArgs& a, const CUtensorMap& tmK, const CUtensorMap& tmZ,
                          int wz, cudaStream_t st, bool pdl);

struct CombineArgs {
  const float* partial;
  const int32_t* seq_lens;
  float* a_lat;        // [B][Hq][r_v] fp32 (may be null)
  uint16_t* a_bf16;    // [B][Hq][r_v] bf16 (may be null)
  int B, Hq, Hkv, G, r_v, S, top_k, nsplit, pages_per_split;
  int len_offset;  // added to seq_lens[b] (tokens appended in this step, not yet counted)
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, bool pdl);

// ----------------------------------------------------------------- outproj
struct OutprojArgs {
  float* partial;  // [ksplit][B][H] fp32 (ksplit > 1)
  uint16_t* y;     // [B][H] bf16
  int B, H, K, ksplit, bn;
  unsigned int* status;
  // Deferred length update of a fused decode step: when bump_lens is set,
  // seq_lens[b] += bump_n (unless that passes bump_cap), done once every
  // earlier kernel of the step has finished reading the lengths.
  int32_t* bump_lens;
  int bump_n, bump_cap;
  // Fused K-split reduction (when cnt is set and ksplit > 1): per M tile an
  // arrival counter, zeroed before the launch; the tile's last CTA sums the
  // partials and writes y.
  int* cnt;
  // Latents stored source-major, [K / k_src sources][src_rows = B][k_src]:
  // column k of row b is element (k % k_src) of row (k / k_src) * B + b.
  // k_src = K for the plain [B][K] layout.
  int k_src;
};
// Chooses the K split for a given problem.
int outproj_ksplit(int H, int K, int B);
int outproj_bn(int B);
cudaError_t launch_outproj(const OutprojArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmA,
                           cudaStream_t st, bool pdl);
cudaError_t launch_cast_bf16(const float* x, uint16_t* y, size_t n, cudaStream_t st, bool pdl);

struct FoldOutArgs {
  const uint16_t* B_V;  // [Hkv][r_v][d]
  const uint16_t* W_O;  // [Hq*d][H]
  uint16_t* W_fold;     // [H][Hq*r_v]
  int Hq, Hkv, d, r_v, H;
};
cudaError_t launch_fold_outproj(const FoldOutArgs& a, cudaStream_t st);

}  // namespace basiskv
