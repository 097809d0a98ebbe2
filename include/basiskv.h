/*
 * basiskv.h — C-ABI of the BasisKV decode-attention block on NVIDIA B200.
 *
 * Method: BasisKV, "Value Latents for Communication and Key Routing" (arXiv
 * 2611.02583).  Its abstract states the method: the Value is cached only as
 * a low-rank latent (width r_v) that is also associated with the output
 * projection; the latent predicts part of each Key for routing while a
 * Key-specific residual (rank r_k) stores what the Value cannot recover; the
 * exact Keys are fetched only for the selected pages.  Figure 1's caption
 * says the same latent is kept in the cache and reused for Key routing.
 * Table 4 lists the per-token state (compressed Value r_V, residual code
 * r_q, exact Key d_h) and which phase reads which state.
 *
 * Notation: B sequences, Hq query heads, Hkv KV heads, G = Hq/Hkv query heads
 * per KV head, d head dim, H = hidden width, S = page_size tokens per page,
 * T_b = seq_lens[b] tokens of sequence b, P_b = ceil(T_b/S) pages,
 * g(h) = h / G the KV head of query head h.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers are raw DEVICE pointers unless a parameter says otherwise.  The
 *   caller allocates and owns every buffer; the library keeps no pointer
 *   after a call returns and allocates nothing.
 * - "bf16" buffers hold IEEE bfloat16 bit patterns (basiskv_bf16); each
 *   bf16 pointer must be 16-byte aligned (every bf16 row width below is a
 *   multiple of 16 bytes for the supported shapes).  int32 and fp32 arrays
 *   need 4-byte alignment, so a row of a block table or an offset into
 *   seq_lens may be passed directly.  The workspace must be 256-byte
 *   aligned.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *   compute call only enqueues work on it and returns; nothing synchronises
 *   the host, so results are valid once the stream has reached that point.
 * - The arguments are validated on the host before anything is enqueued.  A
 *   call that returns an error has launched nothing and changed no buffer.
 * - Conditions only the device can see (a block-table entry outside
 *   [0, num_phys_pages), a sequence that would outgrow its block-table row,
 *   a bounded wait that timed out) skip the offending work and set a bit in
 *   a device status word; basiskv_read_device_status() returns and clears it.
 * - Calls are not thread-safe with respect to one workspace: two calls that
 *   may overlap on the GPU need two workspaces.
 *
 * Cache layouts (paged; one page of one KV head is a contiguous tile):
 *   K_cache [num_phys_pages][Hkv][S][d]    exact Keys        (Table 4 "Exact Key")
 *   Z_cache [num_phys_pages][Hkv][S][r_v]  Value latents z   (Table 4 "Compressed Value")
 *   E_cache [num_phys_pages][Hkv][S][r_k]  Key residuals e   (Table 4 "Residual code")
 *   With a narrow router (route_r_v < r_v or route_r_k < r_k, below), each
 *   Z (E) tile stores its rows' first route_r_v (route_r_k) columns first,
 *   [S][route_r_v] then [S][r_v - route_r_v], so the router reads one
 *   contiguous block per tile (HBM fetches whole lines: a strided subset of
 *   each row would cost the full row).
 *   block_table int32 [B][max_pages_per_seq]: logical page -> physical page.
 *   Token t of sequence b lives in physical page block_table[b][t / S], row
 *   t % S.
 *
 * Factor layouts (per KV head g, row-major):
 *   A_V [Hkv][d][r_v]   z = v A_V
 *   P_K [Hkv][r_v][d]   Key prediction from the latent
 *   U_K [Hkv][d][r_k]   orthonormal columns; e = (k - z P_K) U_K
 *   B_V [Hkv][r_v][d]   Value reconstruction
 *   W_O [Hq*d][H]       output projection; rows h*d..h*d+d-1 are W_O,h
 *   W_fold [H][Hq*r_v]  folded out-projection: W_fold[o][h*r_v + j] =
 *                       (B_V,g(h) W_O,h)[j][o]  (built by basiskv_fold_outproj)
 *
 * Supported shapes: d in {64, 128}; r_v in {32, 64, 96, 128}; r_k in
 * {16, 32, 64}; G in {1, 2, 4, 8}; S in {8, 16, 32}; H a multiple of 128;
 * top_k >= 2.  A router narrower than (r_v, r_k) is supported for G in
 * {4, 8}, r_k = 32 and S in {16, 32} (widths 16 or 32 each).  Other shapes
 * return BASISKV_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef BASISKV_H_
#define BASISKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BASISKV_API __attribute__((visibility("default")))
#else
#define BASISKV_API
#endif

typedef uint16_t basiskv_bf16; /* bfloat16 bit pattern */

typedef struct basiskv_dims {
  int32_t B;                 /* sequences in the batch */
  int32_t Hq;                /* query heads */
  int32_t Hkv;               /* KV heads; Hq % Hkv == 0 */
  int32_t d;                 /* head dimension */
  int32_t hidden;            /* H, width of the out-projection output */
  int32_t r_v;               /* Value latent width */
  int32_t r_k;               /* Key residual rank */
  int32_t page_size;         /* S, tokens per page */
  int32_t max_pages_per_seq; /* length of one block-table row */
  int32_t num_phys_pages;    /* pages held by each physical cache */
  /* Router and budget (zero-initialised = the default router):
   *   route_r_v     latent dims the router reads, z[:, :route_r_v] with
   *                 P_K[:route_r_v] (Table 4: routing reads r_b of r_V);
   *                 0 = all r_v, else a multiple of 16 <= r_v
   *   route_r_k     residual dims the router reads, e[:, :route_r_k] with
   *                 U_K[:, :route_r_k]; 0 = all r_k, else a multiple of 16
   *                 <= r_k
   *   sink_pages    leading pages always selected; 0 = 1 (the sink page),
   *                 negative = none
   *   recent_pages  trailing pages always selected (a recent window, Table
   *                 9's budget); 0 = 1 (the newest page), else >= 1
   * top_k counts the forced pages; top_k >= sink + recent. */
  int32_t route_r_v;
  int32_t route_r_k;
  int32_t sink_pages;
  int32_t recent_pages;
  /* Cache element type (Table 13 stores the caches as FP8 E4M3):
   *   0  K_cache, Z_cache and E_cache hold bf16 (the layouts above)
   *   1  they hold FP8 E4M3 bytes (1 sign, 4 exponent bits with bias 7, 3
   *      mantissa bits; largest finite value 448) in the same layouts, one
   *      byte per element; pass the byte buffers through the bf16 pointer
   *      parameters.  Every write rounds to nearest even and saturates to
   *      +-448.  Supported when the router has an E4M3 instance (G in {4,
   *      8}, r_k = 32, r_v in {64, 96, 128} at full width for S in {16, 32};
   *      the narrow routers listed below) and the attention has one (G in
   *      {4, 8}, S in {16, 32}); otherwise BASISKV_ERR_UNSUPPORTED_SHAPE.
   *      The routing and attention kernels widen the bytes to f16 exactly
   *      and multiply them by f16 copies of the queries, each query group
   *      (routing) or head (attention) first scaled by a power of two that
   *      is divided out of the scores, so queries of any fp32 magnitude
   *      keep about 22 (routing) or all 8 (attention) significant bits. */
  int32_t cache_fp8;
  /* Routing page (Table 10's adopted Page4: pages of 4 tokens are scored and
   * selected; Table 9's budget counts tokens):
   *   0 = page_size (a routing page is a cache page)
   *   4 or 8 with page_size 16 or 32: the cache keeps its page_size pages
   *     (one block-table entry per page_size tokens), while the router
   *     scores every route_page tokens, and top_k, sink_pages,
   *     recent_pages, the selection and page_scores count routing pages.
   *     Needs a router with a routing-page instance: the B16R16 and
   *     full-width routers at G 4, r_v 64 or 96, page 16 (route_page 4;
   *     also 8 for B16R16 at r_v 64) and at G 8, r_v 96, page 32
   *     (route_page 4), over bf16 or E4M3 caches; and, for basiskv_decode /
   *     basiskv_decode_latents, a batch whose (sequence, KV head) groups
   *     fit one wave of the fused selection + attention launch
   *     (basiskv_workspace_size returns 0 otherwise); basiskv_attend does
   *     not take it (BASISKV_ERR_UNSUPPORTED_SHAPE). */
  int32_t route_page;
} basiskv_dims;

enum basiskv_status {
  BASISKV_OK = 0,
  BASISKV_ERR_INVALID_ARG = -1,       /* null / misaligned pointer, bad count */
  BASISKV_ERR_UNSUPPORTED_SHAPE = -2, /* dims outside the supported set */
  BASISKV_ERR_WORKSPACE_TOO_SMALL = -3,
  BASISKV_ERR_LAUNCH_FAILED = -4,     /* a kernel launch was rejected */
  BASISKV_ERR_DEVICE = -5,            /* the device status word was non-zero */
  BASISKV_ERR_CUDA = -6,              /* another CUDA runtime call failed */
  BASISKV_ERR_SCRATCH_LIMIT = -7      /* needs more than the static scratch holds */
};

/* Device status bits (basiskv_read_device_status). */
#define BASISKV_DEV_BAD_PAGE 0x1u     /* block-table entry out of range */
#define BASISKV_DEV_OVERFLOW 0x2u     /* append past the block-table row */
#define BASISKV_DEV_TIMEOUT 0x4u      /* a bounded wait gave up */
#define BASISKV_DEV_BAD_LENGTH 0x8u   /* seq_lens[b] outside [0, max_seq_len] */

/* Bytes of workspace every call below needs for these dims, a selection of
 * top_k pages and contexts of at most max_seq_len tokens.  Returns 0 when
 * the dims are invalid.  One workspace serves every entry point. */
BASISKV_API size_t basiskv_workspace_size(const basiskv_dims* dims, int top_k,
                              int max_seq_len);

/* Offline fold of the out-projection.  The abstract ties the Value factor to
 * the output projection, so the two are multiplied once, offline (Table 1
 * caption compares the resulting W_O traffic):
 *   W_fold[o][h*r_v + j] = sum_i B_V[g(h)][j][i] * W_O[h*d + i][o]
 * accumulated in fp32, stored as bf16.  Uses no workspace. */
BASISKV_API int basiskv_fold_outproj(const basiskv_dims* dims, const basiskv_bf16* B_V,
                         const basiskv_bf16* W_O, basiskv_bf16* W_fold,
                         void* stream);

/* Offline fold of the append factors for the tensor-core prefill path.
 * Per KV head g, with M_g = A_V,g P_K,g U_K,g (d x r_k, fp32):
 *   W_app[g][n][i]     = A_V[g][i][n]      n < r_v, i < d     (z = v A_V)
 *   W_app[g][n][d + i] = 0                 n < r_v
 *   W_app[g][r_v+c][i]     = -M_g[i][c]    c < r_k, i < d
 *   W_app[g][r_v+c][d + i] = U_K[g][i][c]               (e = k U_K - v M_g)
 * so that [z | e] = [v | k] W_app^T.  W_app: bf16 [Hkv][r_v + r_k][2d].
 * Uses no workspace. */
BASISKV_API int basiskv_fold_append(const basiskv_dims* dims, const basiskv_bf16* A_V,
                                    const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                                    basiskv_bf16* W_app, void* stream);

/* Cache append: the Value is kept only as its latent and the Key as a
 * residual code beside the exact Key (abstract; Table 4 rows).  For each sequence b and its n_new new tokens j:
 *   position t = seq_lens[b] + j, KV head g:
 *     z = v A_V,g ;  e = (k - z P_K,g) U_K,g   (fp32, z unrounded in e)
 *     Z_cache <- bf16(z), E_cache <- bf16(e), K_cache <- k
 * then seq_lens[b] += n_new (device-side).
 *   k_new, v_new  bf16 [B][n_new][Hkv][d]
 *   seq_lens      int32 [B], read and updated on the device
 * Tokens that would land past max_pages_per_seq*S are dropped and
 * BASISKV_DEV_OVERFLOW is raised; seq_lens[b] is then left unchanged.
 * A prefill chunk is an append with n_new > 1; to fill one sequence only,
 * pass dims->B = 1 and seq_lens / block_table offset to that sequence.
 * n_new*B >= 128 runs the tensor-core (tcgen05) path: [z | e] = [v | k]
 * W_app^T with W_app as built by basiskv_fold_append (W_app may be NULL:
 * the call then folds it into the workspace first); the residual then uses
 * the bf16-rounded fold instead of the unrounded z.  Smaller appends run
 * the two-step CUDA-core form and ignore W_app.  The tensor-core path is
 * one launch that also advances seq_lens (its last CTA to read them does);
 * up to 64 such calls may be in flight at once on different streams (each
 * takes one of 64 device arrival counters in turn; more would share one). */
BASISKV_API int basiskv_append(const basiskv_dims* dims, const basiskv_bf16* k_new,
                   const basiskv_bf16* v_new, int n_new, int32_t* seq_lens,
                   const int32_t* block_table, const basiskv_bf16* A_V,
                   const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                   const basiskv_bf16* W_app, basiskv_bf16* K_cache, basiskv_bf16* Z_cache,
                   basiskv_bf16* E_cache, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Routing and page selection: the cached Value latent, completed by the Key
 * residual, predicts each Key well enough to rank pages over the whole
 * context (abstract; Table 4, full-context routing column).
 * For every (b, KV head g) and page p < P_b:
 *   score[b][g][p] = max over live tokens t of page p and heads h of group g
 *                    of  q_h . (z_t P_K,g + e_t U_K,g^T)       (fp32)
 * computed as z_t.(P_K,g q_h) + e_t.(U_K,g^T q_h).  Then per (b, g): keep the
 * sink page 0 and the newest page P_b-1, fill the remaining top_k-2 slots
 * with the best other pages by (score desc, page index asc; -0 == +0), and
 * write them ascending to sel[b][g][0..top_k), padded with -1.  If
 * top_k >= P_b every page is selected.
 *   q            bf16 [B][Hq][d]
 *   seq_lens     int32 [B]; max_seq_len: host bound >= every seq_lens[b]
 *                (used to size the grid; <= max_pages_per_seq*S)
 *   page_scores  fp32 [B][Hkv][max_pages_per_seq * page_size / route_page]
 *                (one per routing page) or NULL; entries p >= P_b are not
 *                written
 *   sel          int32 [B][Hkv][top_k], or NULL to compute the page scores
 *                only (page_scores must then be given)
 * Both outputs NULL is BASISKV_ERR_INVALID_ARG. */
BASISKV_API int basiskv_route(const basiskv_dims* dims, const basiskv_bf16* q,
                  const int32_t* seq_lens, int max_seq_len,
                  const int32_t* block_table, const basiskv_bf16* P_K,
                  const basiskv_bf16* U_K, const basiskv_bf16* Z_cache,
                  const basiskv_bf16* E_cache, int top_k, float* page_scores,
                  int32_t* sel, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Exact attention on the selected pages: only the chosen pages' exact Keys
 * are read, and the softmax weights combine Value latents (abstract; Table
 * 4, selected-attention column: exact Key and Value latent).
 * For every query head h (group g) over the live tokens t of the pages in
 * sel[b][g] (entries < 0 ignored):
 *   s_t = (q_h . K_t) / sqrt(d);  p = softmax(s);  a_h = sum_t p_t z_t
 * with fp32 accumulation.
 *   sel    int32 [B][Hkv][top_k] (as written by basiskv_route)
 *   a_lat  fp32 [B][Hq][r_v] */
BASISKV_API int basiskv_attend(const basiskv_dims* dims, const basiskv_bf16* q,
                   const int32_t* seq_lens, int max_seq_len,
                   const int32_t* block_table, const basiskv_bf16* K_cache,
                   const basiskv_bf16* Z_cache, const int32_t* sel, int top_k,
                   float* a_lat, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Latent out-projection: the full output is rebuilt from the per-head Value
 * latents through the folded projection (abstract; Figure 1 caption):
 *   y[b][o] = sum_h sum_j a_lat[b][h][j] * W_fold[o][h*r_v + j]
 * on the tcgen05 tensor cores (a_lat rounded to bf16, fp32 accumulation).
 *   a_lat  fp32 [B][Hq][r_v];  W_fold bf16 [H][Hq*r_v];  y bf16 [B][H] */
BASISKV_API int basiskv_outproj(const basiskv_dims* dims, const float* a_lat,
                    const basiskv_bf16* W_fold, basiskv_bf16* y,
                    void* workspace, size_t workspace_bytes, void* stream);

/* One fused decode step: append (when k_new and v_new are both non-NULL,
 * one token per sequence, layout [B][Hkv][d]), then route + select, attend
 * and out-project over the lengthened context.  max_seq_len bounds the
 * lengths AFTER the append.  sel may be NULL (kept in the workspace). */
BASISKV_API int basiskv_decode(const basiskv_dims* dims, const basiskv_bf16* q,
                   const basiskv_bf16* k_new, const basiskv_bf16* v_new,
                   int32_t* seq_lens, int max_seq_len,
                   const int32_t* block_table, const basiskv_bf16* A_V,
                   const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                   const basiskv_bf16* W_fold, basiskv_bf16* K_cache,
                   basiskv_bf16* Z_cache, basiskv_bf16* E_cache, int top_k,
                   int32_t* sel, basiskv_bf16* y, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Tensor parallelism (Figure 1): each GPU holds some KV heads (with their
 * query heads) of a layer, compresses its local attention output into the
 * heads' Value latents, the GPUs exchange those latents with an AllGather,
 * and each rebuilds the complete output from all of them.  The two calls
 * below are the per-GPU compute on either side of that AllGather (which
 * the caller issues, e.g. NCCL over NVLink).
 *
 * basiskv_decode_latents: basiskv_decode without the out-projection, for
 * the heads described by dims (a rank's share: its Hq and Hkv).  Writes the
 * Value latents a_out bf16 [B][Hq][r_v] (fp32 softmax accumulation, one
 * bf16 rounding) and, with an append, advances seq_lens after every reader.
 * Uses no W_fold. */
BASISKV_API int basiskv_decode_latents(const basiskv_dims* dims, const basiskv_bf16* q,
                                       const basiskv_bf16* k_new, const basiskv_bf16* v_new,
                                       int32_t* seq_lens, int max_seq_len,
                                       const int32_t* block_table, const basiskv_bf16* A_V,
                                       const basiskv_bf16* P_K, const basiskv_bf16* U_K,
                                       basiskv_bf16* K_cache, basiskv_bf16* Z_cache,
                                       basiskv_bf16* E_cache, int top_k, int32_t* sel,
                                       basiskv_bf16* a_out, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* basiskv_outproj_sources: the complete output from the latents of n_src
 * sources, stored source-major as an AllGather leaves them:
 *   a_src bf16 [n_src][B][Hq / n_src][r_v]   (source s holds query heads
 *                                             s*Hq/n_src .. (s+1)*Hq/n_src-1)
 *   y[b][o] = sum_h sum_j a[b][h][j] * W_fold[o][h*r_v + j]
 * on the tcgen05 tensor cores (fp32 accumulation).  dims describes the whole
 * layer (all Hq heads; W_fold [H][Hq*r_v] as built by basiskv_fold_outproj).
 * Hq % n_src != 0 is BASISKV_ERR_INVALID_ARG; (Hq / n_src) * r_v must be a
 * multiple of 64 (else BASISKV_ERR_UNSUPPORTED_SHAPE).  n_src = 1 is the
 * out-projection of bf16 latents [B][Hq][r_v]. */
BASISKV_API int basiskv_outproj_sources(const basiskv_dims* dims, const basiskv_bf16* a_src,
                                        int n_src, const basiskv_bf16* W_fold,
                                        basiskv_bf16* y, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Size of the static device scratch array behind basiskv_decode_noalloc. */
#define BASISKV_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* basiskv_decode for callers that cannot allocate device memory.  The method
 * has no counterpart: this is a deployment variant of the fused decode step.
 *
 * Some callers cannot call cudaMalloc when they run a step: a runtime that
 * owns all device memory through its own pool and forbids side allocations,
 * a plug-in invoked where allocation is not allowed, or a service that must
 * keep its footprint fixed after start-up.  This entry point takes the same
 * arguments as basiskv_decode minus the workspace; the scratch comes from a
 * static __device__ array of BASISKV_NOALLOC_SCRATCH_BYTES (32 MiB) compiled
 * into the library, which every GPU that loads the library holds until the
 * process exits.  It allocates nothing itself.
 *   - Shapes whose basiskv_workspace_size exceeds the array return
 *     BASISKV_ERR_SCRATCH_LIMIT and launch nothing.
 *   - The array's device address belongs to the current CUDA context; each
 *     call made outside stream capture looks it up (cudaGetSymbolAddress in
 *     that context), and a call inside a capture uses the address its
 *     context's last call found.  Make the first call in each context
 *     before any stream capture.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents (nothing in it needs to start at zero).  Calls that may
 *     overlap on the GPU (two streams, two host threads) race on it: order
 *     them on one stream, or use basiskv_decode with separate workspaces. */
BASISKV_API int basiskv_decode_noalloc(const basiskv_dims* dims, const basiskv_bf16* q,
                                       const basiskv_bf16* k_new,
                                       const basiskv_bf16* v_new, int32_t* seq_lens,
                                       int max_seq_len, const int32_t* block_table,
                                       const basiskv_bf16* A_V, const basiskv_bf16* P_K,
                                       const basiskv_bf16* U_K, const basiskv_bf16* W_fold,
                                       basiskv_bf16* K_cache, basiskv_bf16* Z_cache,
                                       basiskv_bf16* E_cache, int top_k, int32_t* sel,
                                       basiskv_bf16* y, void* stream);

/* Waits for `stream`, then returns the device status word in *flags (a
 * HOST pointer; BASISKV_DEV_* bits, 0 = clean) and clears it.  Returns
 * BASISKV_ERR_DEVICE when it was non-zero, BASISKV_ERR_CUDA when the stream
 * itself reported an error. */
BASISKV_API int basiskv_read_device_status(void* stream, uint32_t* flags);

/* Self-test of the library's bounded waits.  The method has no counterpart:
 * this checks the failure path every kernel relies on.  Every wait of a
 * kernel here on an mbarrier gives up after a time limit, records
 * BASISKV_DEV_TIMEOUT in the device status word and lets the kernel return,
 * so a wait that can never complete (a logic error, a copy that never
 * lands) ends with a status the host can read instead of a hung GPU.  This
 * call launches one CTA on `stream` that waits, through that same bounded
 * wait, on an mbarrier nothing arrives on, with a limit of limit_ns
 * nanoseconds (1 .. 1e9; anything else is BASISKV_ERR_INVALID_ARG before
 * any CUDA call).  Afterwards basiskv_read_device_status reports
 * BASISKV_DEV_TIMEOUT (and clears it); the context stays usable. */
BASISKV_API int basiskv_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* Kernels this library has launched in this process so far (a host-side
 * counter; lets a caller count the launches inside a timed region). */
BASISKV_API uint64_t basiskv_launch_count(void);

/* Static description of a status code; never NULL. */
BASISKV_API const char* basiskv_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* BASISKV_H_ */
