// Cache append for a prefill chunk on the 5th-generation tensor cores.
//
// BasisKV stores each token's Value as its latent and its Key as a residual
// code beside the exact Key (abstract; Table 4 rows):
//   z = v A_V,g ;   e = (k - z P_K,g) U_K,g = k U_K,g - v (A_V,g P_K,g U_K,g)
// For a chunk of M tokens both are one product per KV head g:
//   [z | e] = [v | k] . W_app,g^T,   W_app,g = [[A_V^T, 0], [-(A_V P_K U_K)^T, U_K^T]]
// with W_app,g of shape (r_v + r_k) x 2d.  fold_append_kernel builds W_app
// (fp32 products, stored bf16) and append_tc_kernel runs the product:
// 128-token M tiles, N = r_v + r_k, K = 2d, operands staged by TMA in
// 128-byte-swizzled K-major tiles, a single thread issuing tcgen05.mma
// (kind::f16, bf16 inputs, fp32 accumulator in tensor memory), four
// epilogue warps that read the accumulator with tcgen05.ld and write the
// z / e rows into the paged caches, and four warps that copy the exact Key
// there; the same launch advances the sequence lengths.  The folded factor
// is rounded to bf16 once; the decode-time append (append.cu) keeps the
// two-step form with an unrounded z.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

// ------------------------------------------------------------------- fold
// CTA = (KV head g, quarter p of the 2d columns of W_app).  P_K and U_K of
// the head are staged in shared memory; PU = P_K U_K (r_v x r_k) is formed
// there, then the CTA's rows of M = A_V PU (only quarters covering columns
// < d need them) and its columns of W_app are written.  All fp32.
constexpr int kFoldAppThreads = 256;
constexpr int kFoldAppParts = 4;

__global__ void __launch_bounds__(kFoldAppThreads) fold_append_kernel(FoldAppArgs a) {
  extern __shared__ __align__(16) float fa[];
  const int g = blockIdx.x, part = blockIdx.y, tid = threadIdx.x;
  const int d = a.d, r_v = a.r_v, r_k = a.r_k, N = r_v + r_k;
  const int kw = 2 * d / kFoldAppParts, kk0 = part * kw;  // this CTA's W columns
  float* PU = fa;                                  // [r_v][r_k]
  float* Mt = PU + r_v * r_k;                      // [kw][r_k] rows kk0.. of M
  uint16_t* Ps = reinterpret_cast<uint16_t*>(Mt + kw * r_k);  // [r_v][d]
  uint16_t* Us = Ps + r_v * d;                                  // [d][r_k]
  uint16_t* A = Us + d * r_k;                                   // [d][r_v]
  {
    const uint4* s1 = reinterpret_cast<const uint4*>(a.P_K + (size_t)g * r_v * d);
    const uint4* s2 = reinterpret_cast<const uint4*>(a.U_K + (size_t)g * d * r_k);
    const uint4* s3 = reinterpret_cast<const uint4*>(a.A_V + (size_t)g * d * r_v);
    uint4* d1 = reinterpret_cast<uint4*>(Ps);
    uint4* d2 = reinterpret_cast<uint4*>(Us);
    uint4* d3 = reinterpret_cast<uint4*>(A);
    for (int i = tid; i < r_v * d / 8; i += kFoldAppThreads) d1[i] = s1[i];
    for (int i = tid; i < d * r_k / 8; i += kFoldAppThreads) d2[i] = s2[i];
    for (int i = tid; i < d * r_v / 8; i += kFoldAppThreads) d3[i] = s3[i];
  }
  __syncthreads();
  const bool need_m = kk0 < d;
  if (need_m) {
    // four outputs per thread (columns c..c+3): independent accumulation chains
    for (int o = tid; o < r_v * r_k / 4; o += kFoldAppThreads) {
      const int jj = o / (r_k / 4), c = (o % (r_k / 4)) * 4;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
      for (int i = 0; i < d; ++i) {
        const float p = bf16_to_f(Ps[jj * d + i]);
        const uint2 u = *reinterpret_cast<const uint2*>(Us + i * r_k + c);
        a0 = fmaf(p, bf16lo(u.x), a0);
        a1 = fmaf(p, bf16hi(u.x), a1);
        a2 = fmaf(p, bf16lo(u.y), a2);
        a3 = fmaf(p, bf16hi(u.y), a3);
      }
      PU[jj * r_k + c] = a0;
      PU[jj * r_k + c + 1] = a1;
      PU[jj * r_k + c + 2] = a2;
      PU[jj * r_k + c + 3] = a3;
    }
    __syncthreads();
    for (int o = tid; o < kw * r_k / 4; o += kFoldAppThreads) {
      const int i = o / (r_k / 4), c = (o % (r_k / 4)) * 4;
      const uint16_t* arow = A + (kk0 + i) * r_v;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
      for (int jj = 0; jj < r_v; ++jj) {
        const float av = bf16_to_f(arow[jj]);
        const float4 pu = *reinterpret_cast<const float4*>(PU + jj * r_k + c);
        a0 = fmaf(av, pu.x, a0);
        a1 = fmaf(av, pu.y, a1);
        a2 = fmaf(av, pu.z, a2);
        a3 = fmaf(av, pu.w, a3);
      }
      Mt[i * r_k + c] = a0;
      Mt[i * r_k + c + 1] = a1;
      Mt[i * r_k + c + 2] = a2;
      Mt[i * r_k + c + 3] = a3;
    }
    __syncthreads();
  }
  uint16_t* W = a.W_app + (size_t)g * N * 2 * d;  // [N][2d]
  for (int o = tid; o < N * kw; o += kFoldAppThreads) {
    const int n = o / kw, kk = kk0 + o % kw;
    float w;
    if (n < r_v)
      w = kk < d ? bf16_to_f(A[kk * r_v + n]) : 0.f;
    else
      w = kk < d ? -Mt[(kk - kk0) * r_k + (n - r_v)] : bf16_to_f(Us[(kk - d) * r_k + (n - r_v)]);
    W[(size_t)n * 2 * d + kk] = f_to_bf16(w);
  }
}

// ------------------------------------------------------------------- GEMM
// One persistent CTA per SM walks a contiguous range of work items (KV head
// g, 128-row M tile), head-major, so W_app,g is staged once per head and
// stays resident while the v/k tiles stream through a ring of 16 KB slots.
// Only W_app's nonzero blocks are staged: the v k-blocks multiply all N
// rows, the k k-blocks only the r_k residual rows (N = r_k, into the
// accumulator's e columns).  The accumulator is double-buffered in tensor
// memory: the MMA of tile i+1 runs while the epilogue drains tile i.  The
// epilogue converts each lane's row into dense per-part staging blocks and
// hands every run of consecutive cache rows to the copy engine as one bulk
// copy per cache part.  Four more warps copy the exact Key out of each k
// slot as soon as it lands: 8-row TMA tensor stores wherever 8 rows land on
// 8 consecutive cache rows (every group of an aligned chunk; a ragged group,
// and E4M3 rounding, fall back to plain stores), so a slot returns to the
// producer once its MMAs are done and the copy engine has read it, and the
// ring keeps streaming while the epilogue works.
// warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue, warps 6-9 Key copy
constexpr int kTcEpiWarps = 4, kTcKeyWarps = 4;
constexpr int kTcKeyWarp0 = 2 + kTcEpiWarps;
constexpr int kTcThreads = 32 * (kTcKeyWarp0 + kTcKeyWarps);
constexpr int kTcBM = 128, kTcBK = 64;
constexpr int kTcABytes = kTcBM * kTcBK * 2;  // one ring slot: 128 rows x 128 bytes
constexpr int kTcMaxSlots = 12;
constexpr unsigned long long kTcDrainNs = 10000000ull;  // waits for copies in flight at exit

// Arrival counts for the in-kernel length update, one slot per call in
// flight (the host hands slots out round-robin): zero when the library
// loads, and reset by the CTA that completes a call's count.
constexpr int kTcArriveSlots = 64;
__device__ unsigned int g_tc_arrive[kTcArriveSlots];

__host__ __device__ constexpr uint32_t tc_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Shared memory: W_app's v k-blocks (d/64 tiles of N x 128 bytes), its k
// k-blocks (d/64 tiles of r_k x 128 bytes), the ring, the epilogue's
// staging (per warp: 32 dense rows of each cache part, z | e in the cache
// element type), then the barriers.
struct TcSmem {
  size_t wk, ring, stage, kstage, bars, lens, total;
};

__host__ __device__ inline TcSmem tc_smem(int r_v, int r_k, int d, int fp8, int slots) {
  const int N = r_v + r_k;
  TcSmem L;
  L.wk = (size_t)(d / 64) * N * 128;                 // multiples of 2 KB
  L.ring = L.wk + (size_t)(d / 64) * r_k * 128;
  L.stage = L.ring + (size_t)slots * kTcABytes;
  L.kstage = L.stage + (size_t)kTcEpiWarps * 32 * N * (fp8 ? 1 : 2);
  // E4M3 caches: each Key warp's 32 rounded Key rows (d bytes each)
  L.bars = L.kstage + (fp8 ? (size_t)kTcKeyWarps * 32 * d : 0);
  L.lens = L.bars + (2 * (size_t)slots + 7) * 8 + 16;
  L.total = L.lens + 256 * 4;  // the sequences' lengths (B <= 256)
  return L;
}

// Cache position of token row r of the chunk (pos = -1: no such row, or its
// sequence would overflow) and the block-table entry of that position's
// page, loaded here and checked where it is used, a tile later.
struct RowRef {
  int pos, pp;
};

__device__ __forceinline__ RowRef row_ref(const AppendArgs& a, const int* lens, int rows, int r,
                                          int g, bool report) {
  RowRef x{-1, -1};
  if (r >= rows) return x;
  const int b = r / a.n_new, j = r - b * a.n_new;
  const int len = lens[b];
  if (len < 0 || len + a.n_new > a.max_pages * a.S) {
    if (report && j == 0 && g == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
    return x;
  }
  x.pos = len + j;
  x.pp = a.block_table[(size_t)b * a.max_pages + x.pos / a.S];
  return x;
}

__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0], %1; }" ::"r"(
                   smem_u32(bar)),
               "r"(n)
               : "memory");
}

// shared -> global bulk copy (16-byte aligned ends, size % 16 == 0)
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

// 2-D tiled store of one box from shared memory (bulk group)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int32_t x,
                                             int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// this thread's bulk copies have read their shared-memory sources
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// this thread's bulk copies are complete
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kTcThreads, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmWk,
                     const __grid_constant__ CUtensorMap tmKc, AppendArgs a, int N, int tmem_cols,
                     int slots, int n_mt, int bump_slot) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int d = a.d, nkb = 2 * d / kTcBK;  // k-blocks: first d/64 from v, then from k
  const int cb = a.fp8 ? 1 : 2;            // cache bytes per element
  const TcSmem L = tc_smem(a.r_v, a.r_k, d, a.fp8, slots);
  uint8_t* w_tiles = smem;            // v k-blocks: N rows each
  uint8_t* wk_tiles = smem + L.wk;    // k k-blocks: the r_k residual rows
  uint8_t* ring = smem + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + slots;
  uint64_t* tfull = empty + slots;  // [2] accumulator buffer written
  uint64_t* tempty = tfull + 2;     // [2] accumulator buffer drained
  uint64_t* wfull = tempty + 2;
  uint64_t* wempty = wfull + 1;
  uint64_t* drain = wempty + 1;  // the MMA thread's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rows = a.B * a.n_new;
  const int n_items = n_mt * a.Hkv;
  const int i0 = (int)((long long)blockIdx.x * n_items / gridDim.x);
  const int i1 = (int)((long long)(blockIdx.x + 1) * n_items / gridDim.x);
  const int acc_cols = tmem_cols / 2;

  if (tid == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      // the MMAs' commit + the Key warps' releases (v slots: a stand-in)
      mbar_init(&empty[s], 1 + kTcKeyWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kTcEpiWarps);
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  // The next launch may be scheduled now: it waits for this grid to
  // complete before it reads or writes anything.
  pdl_launch_dependents();
  // the epilogue and Key warps read the lengths from shared memory
  int* lens = reinterpret_cast<int*>(smem + L.lens);
  if (warp >= 2) {
    for (int i = tid - 64; i < a.B; i += kTcThreads - 64) lens[i] = a.seq_lens[i];
    asm volatile("bar.sync 1, %0;" ::"r"(kTcThreads - 64) : "memory");
    // The lengths advance once every CTA holds its copy: each CTA arrives
    // after reading them, and the last to arrive advances them (skipping,
    // with the overflow bit, a sequence whose chunk does not fit its
    // block-table row) and resets the count.  Nothing waits here.
    if (bump_slot >= 0 && tid == 64) {
      __threadfence();
      if (atomicAdd(&g_tc_arrive[bump_slot], 1u) == gridDim.x - 1) {
        __threadfence();
        const int cap = a.max_pages * a.S;
        for (int b = 0; b < a.B; ++b) {
          const int len = lens[b];
          if (len < 0 || len + a.n_new > cap)
            raise_status(a.status, BASISKV_DEV_OVERFLOW);
          else
            a.seq_lens_out[b] = len + a.n_new;
        }
        g_tc_arrive[bump_slot] = 0;
      }
    }
  }

  if (warp == 0 && lane == 0) {  // ------------------------------------- TMA
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmWk);
    if (!a.fp8) prefetch_tmap(&tmKc);
    int it = 0, wl = 0, cur_g = -1;
    bool ok = true;
    for (int item = i0; item < i1 && ok; ++item) {
      const int g = item / n_mt, m0 = (item % n_mt) * kTcBM;
      if (item == i0) {  // the first head's factor goes first: every MMA needs it
        mbar_arrive_expect_tx(wfull, (uint32_t)(N + a.r_k) * d * 2);
        for (int kb = 0; kb < nkb / 2; ++kb) {
          tma_load_2d(w_tiles + kb * N * 128, &tmW, kb * kTcBK, g * N, wfull);
          tma_load_2d(wk_tiles + kb * a.r_k * 128, &tmWk, d + kb * kTcBK, g * N + a.r_v, wfull);
        }
        wl = 1;
        cur_g = g;
      }
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % slots;
        // the slot is free once its previous k-block has been consumed
        if (it >= slots && !(ok = mbar_wait_or_abort(&empty[s], ((it / slots) - 1) & 1,
                                                     a.status, abort_flag)))
          break;
        mbar_arrive_expect_tx(&full[s], kTcABytes);
        const bool from_v = kb < nkb / 2;
        const int col = (from_v ? kb : kb - nkb / 2) * kTcBK;
        // 3-D maps over [rows][Hkv][d]: coordinates (column, head, row)
        tma_load_3d(ring + s * kTcABytes, from_v ? &tmV : &tmK, col, g, m0, &full[s]);
      }
      if (ok && g != cur_g) {  // a new head: its factor, once the last MMA on the old one is done
        if (wl > 0 && !(ok = mbar_wait_or_abort(wempty, (wl - 1) & 1, a.status, abort_flag)))
          break;
        mbar_arrive_expect_tx(wfull, (uint32_t)(N + a.r_k) * d * 2);
        for (int kb = 0; kb < nkb / 2; ++kb) {
          tma_load_2d(w_tiles + kb * N * 128, &tmW, kb * kTcBK, g * N, wfull);
          tma_load_2d(wk_tiles + kb * a.r_k * 128, &tmWk, d + kb * kTcBK, g * N + a.r_v, wfull);
        }
        ++wl;
        cur_g = g;
      }
    }
    // drain: every copy issued must have landed before the CTA exits
    for (int u = it - 1; u >= 0 && u >= it - slots; --u)
      mbar_wait(&full[u % slots], (u / slots) & 1, a.status, kTcDrainNs);
    if (wl > 0) mbar_wait(wfull, (wl - 1) & 1, a.status, kTcDrainNs);
  } else if (warp == 1 && lane == 0) {  // ------------------------------ MMA
    const uint32_t idesc = tc_idesc(kTcBM, N), idesc_e = tc_idesc(kTcBM, a.r_k);
    int it = 0, wl = 0, cur_g = -1, lt = 0;
    bool ok = true;
    for (int item = i0; item < i1 && ok; ++item, ++lt) {
      const int g = item / n_mt;
      if (g != cur_g) {
        if (!(ok = mbar_wait_or_abort(wfull, wl & 1, a.status, abort_flag))) break;
        ++wl;
        cur_g = g;
      }
      const int buf = lt & 1;
      if (lt >= 2 && !(ok = mbar_wait_or_abort(&tempty[buf], ((lt >> 1) - 1) & 1, a.status,
                                               abort_flag)))
        break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t dt = tmem + (uint32_t)(buf * acc_cols);
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % slots;
        if (!(ok = mbar_wait_or_abort(&full[s], (it / slots) & 1, a.status, abort_flag))) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // a v k-block feeds all N columns; a k k-block only the e columns
        const bool from_v = kb < nkb / 2;
        const uint64_t da = tc_sdesc(smem_u32(ring + s * kTcABytes));
        const uint64_t db = tc_sdesc(smem_u32(
            from_v ? w_tiles + kb * N * 128 : wk_tiles + (kb - nkb / 2) * a.r_k * 128));
        const uint32_t dk = from_v ? dt : dt + (uint32_t)a.r_v;
        const uint32_t ik = from_v ? idesc : idesc_e;
#pragma unroll
        for (int k = 0; k < kTcBK / 16; ++k) {
          const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
          asm volatile(
              "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
              " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(dk),
              "l"(da + 2 * k), "l"(db + 2 * k), "r"(ik), "r"(acc)
              : "memory");
        }
        // slot s is released when these MMAs complete (and, for a k slot,
        // once the Key warps have copied it out)
        tc_commit(&empty[s]);
        if (from_v) mbar_arrive_n(&empty[s], kTcKeyWarps);
      }
      if (!ok) break;
      tc_commit(&tfull[buf]);
      if (item + 1 < i1 && (item + 1) / n_mt != g) tc_commit(wempty);
    }
    // drain: one more commit tracks every MMA this thread issued
    tc_commit(drain);
    mbar_wait(drain, 0, a.status, kTcDrainNs);
  } else if (warp >= 2 && warp < kTcKeyWarp0) {  // ----------------------- epilogue
    const int quarter = warp & 3;  // this warp's 32 TMEM lanes = tile rows
    const int zs = a.zsplit, es = a.esplit;
    // this warp's staging: 32 dense rows of each part (Z's first zs
    // columns, the rest of Z, E's first es columns, the rest of E)
    uint8_t* const zA = smem + L.stage + (size_t)(warp - 2) * 32 * N * cb;
    uint8_t* const zB = zA + 32 * zs * cb;
    uint8_t* const eA = zA + 32 * a.r_v * cb;
    uint8_t* const eB = eA + 32 * es * cb;
    uint8_t* const zc = reinterpret_cast<uint8_t*>(a.Z_cache);
    uint8_t* const ec = reinterpret_cast<uint8_t*>(a.E_cache);
    int lt = 0;
    RowRef cur = i0 < i1 ? row_ref(a, lens, rows, (i0 % n_mt) * kTcBM + quarter * 32 + lane,
                                   i0 / n_mt, true)
                         : RowRef{-1, -1};
    for (int item = i0; item < i1; ++item, ++lt) {
      const int g = item / n_mt;
      // the next tile's block-table entry is in flight while this tile drains
      const RowRef nxt =
          item + 1 < i1 ? row_ref(a, lens, rows, ((item + 1) % n_mt) * kTcBM + quarter * 32 + lane,
                                  (item + 1) / n_mt, true)
                        : RowRef{-1, -1};
      // this lane's row: its cache tile (physical page x KV head) and row
      // within the tile, or dead
      long long tile = 0;
      int trow = 0, live = 0;
      if (cur.pos >= 0) {
        if (cur.pp < 0 || cur.pp >= a.num_phys) {
          raise_status(a.status, BASISKV_DEV_BAD_PAGE);
        } else {
          tile = (long long)cur.pp * a.Hkv + g;
          trow = cur.pos % a.S;
          live = 1;
        }
      }
      cur = nxt;
      // runs: consecutive live lanes on consecutive rows of one cache tile
      const long long ptile = __shfl_up_sync(0xffffffffu, tile, 1);
      const int ptrow = __shfl_up_sync(0xffffffffu, trow, 1);
      const int plive = __shfl_up_sync(0xffffffffu, live, 1);
      const bool lead =
          live && (lane == 0 || !plive || ptile != tile || ptrow + 1 != trow);
      const unsigned stops = __ballot_sync(0xffffffffu, lead || !live);
      const unsigned after = stops & ~((2u << lane) - 1u);  // stops above this lane
      const int run = (after ? __ffs(after) - 1 : 32) - lane;
      const int buf = lt & 1;
      bool ok = mbar_wait_or_abort(&tfull[buf], (lt >> 1) & 1, a.status, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      // accumulator -> cache element type -> this lane's rows of the parts
      const uint32_t ta = tmem + (uint32_t)(buf * acc_cols) + ((uint32_t)(quarter * 32) << 16);
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t rr[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]),
              "=r"(rr[6]), "=r"(rr[7]), "=r"(rr[8]), "=r"(rr[9]), "=r"(rr[10]), "=r"(rr[11]),
              "=r"(rr[12]), "=r"(rr[13]), "=r"(rr[14]), "=r"(rr[15])
            : "r"(ta + (uint32_t)c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        // the part holding columns c0 .. c0 + 15 (zs, es are multiples of 16)
        uint8_t* dst;
        if (c0 < zs)
          dst = zA + (lane * zs + c0) * cb;
        else if (c0 < a.r_v)
          dst = zB + (lane * (a.r_v - zs) + c0 - zs) * cb;
        else if (c0 < a.r_v + es)
          dst = eA + (lane * es + c0 - a.r_v) * cb;
        else
          dst = eB + (lane * (a.r_k - es) + c0 - a.r_v - es) * cb;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(rr[i]);
        if (a.fp8) {  // E4M3: 16 columns are one 16-byte chunk
          uint32_t pb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            pb[i] = f_to_e4m3x2(v[4 * i], v[4 * i + 1]) |
                    (f_to_e4m3x2(v[4 * i + 2], v[4 * i + 3]) << 16);
          *reinterpret_cast<uint4*>(dst) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
        } else {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = (uint32_t)f_to_bf16(v[2 * i]) | ((uint32_t)f_to_bf16(v[2 * i + 1]) << 16);
          reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      // the accumulator buffer is free for the MMA two tiles on
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      // the staged rows are visible to the copy engine once every lane is here
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (lead) {
        // one bulk copy per part for the run's rows (Z and E tiles store the
        // first zs / es columns of every row first)
        const size_t zt = (size_t)tile * a.S * a.r_v * cb, et = (size_t)tile * a.S * a.r_k * cb;
        bulk_store(zc + zt + (size_t)trow * zs * cb, zA + lane * zs * cb, run * zs * cb);
        if (zs < a.r_v)
          bulk_store(zc + zt + ((size_t)a.S * zs + (size_t)trow * (a.r_v - zs)) * cb,
                     zB + lane * (a.r_v - zs) * cb, run * (a.r_v - zs) * cb);
        bulk_store(ec + et + (size_t)trow * es * cb, eA + lane * es * cb, run * es * cb);
        if (es < a.r_k)
          bulk_store(ec + et + ((size_t)a.S * es + (size_t)trow * (a.r_k - es)) * cb,
                     eB + lane * (a.r_k - es) * cb, run * (a.r_k - es) * cb);
      }
      // the staging is rewritten next tile, once the copy engine has read it
      bulk_commit();
      bulk_wait_read();
      __syncwarp();
    }
    bulk_wait_all();
  } else if (warp >= kTcKeyWarp0) {  // ---------------------------------- Key copy
    // The exact Key of tile rows 32w .. 32w + 31 (w = this Key warp), straight
    // from each k slot (16-byte chunk j of tile row t sits at chunk
    // j ^ (t & 7) of its 128-byte row).  E4M3 caches: each lane rounds its
    // row into the warp's staging rows, and every run of consecutive cache
    // rows leaves as one bulk copy.
    const int t = (warp - kTcKeyWarp0) * 32 + lane;  // this lane's tile row
    uint8_t* const kc = reinterpret_cast<uint8_t*>(a.K_cache);
    uint8_t* const k8 = smem + L.kstage + (size_t)(warp - kTcKeyWarp0) * 32 * d;  // [32][d]
    // Lane-dependent chunk order for the rounding: chunk c = ch ^ A(l) of
    // row l in step ch, A(l) = 2l over GF(8) (x^3 + x + 1).  A and A + 1 are
    // both one-to-one, so in every step eight consecutive lanes read eight
    // different 16-byte chunk positions of the swizzled slot (c ^ l) and
    // write eight different 8-byte columns of their staging rows (c).
    const int gl = lane & 7, gfa = ((gl << 1) ^ ((gl >> 2) * 3)) & 7;
    int lt = 0;
    bool ok = true;
    RowRef cur = i0 < i1 ? row_ref(a, lens, rows, (i0 % n_mt) * kTcBM + t, i0 / n_mt, false)
                         : RowRef{-1, -1};
    for (int item = i0; item < i1 && ok; ++item, ++lt) {
      const int g = item / n_mt;
      // the next tile's block-table entry is in flight while this tile's slots drain
      const RowRef nxt = item + 1 < i1 ? row_ref(a, lens, rows, ((item + 1) % n_mt) * kTcBM + t,
                                                 (item + 1) / n_mt, false)
                                       : RowRef{-1, -1};
      long long sl = -1;  // this row's Key cache row, or -1 (dead)
      if (cur.pos >= 0 && cur.pp >= 0 && cur.pp < a.num_phys)
        sl = ((long long)cur.pp * a.Hkv + g) * a.S + cur.pos % a.S;
      cur = nxt;
      // do the 8 rows of this lane's group land on 8 consecutive cache rows?
      const long long s0 = __shfl_sync(0xffffffffu, sl, lane & ~7);
      const unsigned seq = __ballot_sync(0xffffffffu, sl >= 0 && sl == s0 + (lane & 7));
      const bool boxed = !a.fp8 && ((seq >> (lane & ~7)) & 0xffu) == 0xffu;
      for (int kb = 0; kb < nkb / 2; ++kb) {
        const int u = lt * nkb + nkb / 2 + kb, s = u % slots;
        ok = __all_sync(0xffffffffu,
                        mbar_wait_or_abort(&full[s], (u / slots) & 1, a.status, abort_flag));
        if (!ok) break;
        const uint8_t* row = ring + (size_t)s * kTcABytes + t * 128;
        if (a.fp8) {
          if (sl >= 0)
            for (int ch = 0; ch < 8; ++ch) {
              const int c = ch ^ gfa;
              const uint4 x = *reinterpret_cast<const uint4*>(row + ((c ^ (t & 7)) << 4));
              const float2 f0 = bf16x2_to_f2(x.x), f1 = bf16x2_to_f2(x.y),
                           f2 = bf16x2_to_f2(x.z), f3 = bf16x2_to_f2(x.w);
              *reinterpret_cast<uint2*>(k8 + lane * d + kb * kTcBK + c * 8) =
                  make_uint2(f_to_e4m3x2(f0.x, f0.y) | (f_to_e4m3x2(f1.x, f1.y) << 16),
                             f_to_e4m3x2(f2.x, f2.y) | (f_to_e4m3x2(f3.x, f3.y) << 16));
            }
        } else if (boxed) {
          if ((lane & 7) == 0) tma_store_2d(&tmKc, row, kb * kTcBK, (int32_t)sl);
        } else if (sl >= 0) {
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(kc + (sl * d + kb * kTcBK + ch * 8) * 2) =
                *reinterpret_cast<const uint4*>(row + ((ch ^ (t & 7)) << 4));
        }
        // the slot goes back to the producer once the copy engine has read it
        bulk_commit();
        bulk_wait_read();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (a.fp8 && ok) {
        // runs: consecutive lanes on consecutive Key cache rows
        const long long psl = __shfl_up_sync(0xffffffffu, sl, 1);
        const bool lead = sl >= 0 && (lane == 0 || psl < 0 || psl + 1 != sl);
        const unsigned stops = __ballot_sync(0xffffffffu, lead || sl < 0);
        const unsigned after = stops & ~((2u << lane) - 1u);
        const int run = (after ? __ffs(after) - 1 : 32) - lane;
        fence_proxy_async();  // the rounded rows are visible to the copy engine
        __syncwarp();
        if (lead) bulk_store(kc + sl * d, k8 + lane * d, (uint32_t)(run * d));
        bulk_commit();
        bulk_wait_read();  // the staging rows are rewritten next tile
        __syncwarp();
      }
    }
    bulk_wait_all();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(tmem_cols)
                 : "memory");
  }
}

}  // namespace

size_t append_factor_bytes(int Hkv, int d, int r_v, int r_k) {
  return (size_t)Hkv * (r_v + r_k) * 2 * d * 2;
}

cudaError_t launch_fold_append(const FoldAppArgs& a, cudaStream_t st, bool pdl) {
  const int kw = 2 * a.d / kFoldAppParts;
  const size_t smem = (size_t)(a.r_v * a.r_k + kw * a.r_k) * sizeof(float) +
                      (size_t)(2 * a.r_v * a.d + a.d * a.r_k) * sizeof(uint16_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fold_append_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(fold_append_kernel, dim3(a.Hkv, kFoldAppParts), dim3(kFoldAppThreads), smem, st,
                  pdl, a);
}

cudaError_t launch_append_tc(const AppendArgs& a, const CUtensorMap& tmV, const CUtensorMap& tmK,
                             const CUtensorMap& tmW, const CUtensorMap& tmWk,
                             const CUtensorMap& tmKc, bool bump, cudaStream_t st, bool pdl) {
  const int N = a.r_v + a.r_k;
  const int acc = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
  const int tmem_cols = 2 * acc;  // two accumulator buffers
  const int nkb = 2 * a.d / kTcBK;
  const size_t cap = 227 * 1024 - 1024;  // the 1 KB alignment pad comes off the top
  const size_t fixed = tc_smem(a.r_v, a.r_k, a.d, a.fp8, 0).total;
  if (fixed + (size_t)nkb * kTcABytes > cap) return cudaErrorInvalidConfiguration;
  const int slots = (int)std::min<size_t>(kTcMaxSlots, (cap - fixed) / kTcABytes);
  const size_t smem = tc_smem(a.r_v, a.r_k, a.d, a.fp8, slots).total + 1024;
  // the kernel's shared-memory limit, raised once per device to the largest
  // size asked for so far
  static std::atomic<int> raised[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || raised[dev].load(std::memory_order_relaxed) < (int)smem) {
    e = cudaFuncSetAttribute(append_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
      int cur = raised[dev].load();
      while (cur < (int)smem && !raised[dev].compare_exchange_weak(cur, (int)smem)) {
      }
    }
  }
  const int rows = a.B * a.n_new;
  const int n_mt = (rows + kTcBM - 1) / kTcBM;
  const int grid = std::min(n_mt * a.Hkv, num_sms());
  static std::atomic<unsigned> next_slot{0};
  const int bump_slot = bump ? (int)(next_slot.fetch_add(1) % kTcArriveSlots) : -1;
  return launch_k(append_tc_kernel, dim3(grid), dim3(kTcThreads), smem, st, pdl, tmV, tmK, tmW,
                  tmWk, tmKc, a, N, tmem_cols, slots, n_mt, bump_slot);
}

}  // namespace basiskv
