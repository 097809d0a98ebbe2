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
// 128-byte-swizzled K-major tiles through a two-slot ring (so two or three
// CTAs share an SM and one CTA's loads overlap another's epilogue), a
// single thread issuing tcgen05.mma
// (kind::f16, bf16 inputs, fp32 accumulator in tensor memory), and four
// epilogue warps that read the accumulator with tcgen05.ld and scatter the
// bf16 z / e rows, and the exact Key, into the paged caches.  The folded
// factor is rounded to bf16 once; the decode-time append (append.cu) keeps
// the two-step form with an unrounded z.
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
constexpr int kTcThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kTcBM = 128, kTcBK = 64;
constexpr int kTcSlots = 2;  // k-block ring

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

__global__ void __launch_bounds__(kTcThreads, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmW, AppendArgs a, int N, int tmem_cols) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const int d = a.d, nkb = 2 * d / kTcBK;  // k-blocks: first d/64 from v, then from k
  const int a_bytes = kTcBM * kTcBK * 2, b_bytes = N * kTcBK * 2;
  uint8_t* a_tiles = smem;                           // kTcSlots x 16 KB
  uint8_t* b_tiles = smem + kTcSlots * a_bytes;      // kTcSlots x N*128 B
  uint64_t* full = reinterpret_cast<uint64_t*>(b_tiles + kTcSlots * b_bytes);
  uint64_t* empty = full + kTcSlots;
  uint64_t* accum = empty + kTcSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y, m0 = blockIdx.x * kTcBM;
  const int rows = a.B * a.n_new;

  if (tid == 0) {
    for (int s = 0; s < kTcSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
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

  if (warp == 0 && lane == 0) {  // ------------------------------------- TMA
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmW);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kTcSlots;
      // the slot is free once the MMAs that read its previous k-block are done
      if (kb >= kTcSlots && !mbar_wait(&empty[s], ((kb / kTcSlots) - 1) & 1, a.status)) break;
      mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
      const bool from_v = kb < nkb / 2;
      const int col = (from_v ? kb : kb - nkb / 2) * kTcBK;
      // 3-D maps over [rows][Hkv][d]: coordinates (column, head, row)
      tma_load_3d(a_tiles + s * a_bytes, from_v ? &tmV : &tmK, col, g, m0, &full[s]);
      tma_load_2d(b_tiles + s * b_bytes, &tmW, kb * kTcBK, g * N, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {  // ------------------------------ MMA
    const uint32_t idesc = tc_idesc(kTcBM, N);
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int s = kb % kTcSlots;
      ok = mbar_wait(&full[s], (kb / kTcSlots) & 1, a.status);
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint64_t da = tc_sdesc(smem_u32(a_tiles + s * a_bytes));
      const uint64_t db = tc_sdesc(smem_u32(b_tiles + s * b_bytes));
#pragma unroll
      for (int k = 0; k < kTcBK / 16; ++k) {
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        asm volatile(
            "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
            " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem),
            "l"(da + 2 * k), "l"(db + 2 * k), "r"(idesc), "r"(acc)
            : "memory");
      }
      // slot s is released when these MMAs complete
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(&empty[s]))
          : "memory");
    }
    if (ok)
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              smem_u32(accum))
          : "memory");
  } else if (warp >= 2) {  // ---------------------------------------- epilogue
    const int quarter = warp & 3;
    const int r = m0 + quarter * 32 + lane;  // token row of the chunk
    bool ok = mbar_wait(accum, 0, a.status);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    size_t slot = 0;
    bool live = false;
    if (r < rows) {
      const int b = r / a.n_new, j = r % a.n_new;
      const int len = a.seq_lens[b];
      const int cap = a.max_pages * a.S;
      if (len < 0 || len + a.n_new > cap) {
        if (j == 0 && g == 0) raise_status(a.status, BASISKV_DEV_OVERFLOW);
      } else {
        const int pos = len + j;
        const int pp = a.block_table[(size_t)b * a.max_pages + pos / a.S];
        if (pp < 0 || pp >= a.num_phys) {
          raise_status(a.status, BASISKV_DEV_BAD_PAGE);
        } else {
          slot = ((size_t)pp * a.Hkv + g) * a.S + pos % a.S;
          live = true;
        }
      }
    }
    // every lane of the warp joins the tcgen05.ld; only live rows store
    for (int c0 = 0; c0 < N; c0 += 16) {
      float v[16];
      uint32_t rr[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
          "%11, %12, %13, %14, %15}, [%16];"
          : "=r"(rr[0]), "=r"(rr[1]), "=r"(rr[2]), "=r"(rr[3]), "=r"(rr[4]), "=r"(rr[5]),
            "=r"(rr[6]), "=r"(rr[7]), "=r"(rr[8]), "=r"(rr[9]), "=r"(rr[10]), "=r"(rr[11]),
            "=r"(rr[12]), "=r"(rr[13]), "=r"(rr[14]), "=r"(rr[15])
          : "r"(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c0));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (!(ok && live)) continue;
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(rr[i]);
      const size_t tile = slot / a.S;
      const int trow = (int)(slot - tile * a.S);
      if (a.fp8) {  // E4M3 caches: 16 bytes per 16 columns
        uint32_t pb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          pb[i] = f_to_e4m3x2(v[4 * i], v[4 * i + 1]) |
                  (f_to_e4m3x2(v[4 * i + 2], v[4 * i + 3]) << 16);
        uint8_t* dst8 =
            c0 < a.r_v
                ? reinterpret_cast<uint8_t*>(a.Z_cache) + tile * a.S * a.r_v +
                      split_off(trow, c0, a.S, a.r_v, a.zsplit)
                : reinterpret_cast<uint8_t*>(a.E_cache) + tile * a.S * a.r_k +
                      split_off(trow, c0 - a.r_v, a.S, a.r_k, a.esplit);
        *reinterpret_cast<uint4*>(dst8) = make_uint4(pb[0], pb[1], pb[2], pb[3]);
        continue;
      }
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pk[i] = (uint32_t)f_to_bf16(v[2 * i]) | ((uint32_t)f_to_bf16(v[2 * i + 1]) << 16);
      // columns c0..c0+15 are z (c < r_v) or e (c >= r_v); r_v, r_k are multiples of 16
      uint16_t* dst =
          c0 < a.r_v
              ? a.Z_cache + tile * a.S * a.r_v + split_off(trow, c0, a.S, a.r_v, a.zsplit)
              : a.E_cache + tile * a.S * a.r_k +
                    split_off(trow, c0 - a.r_v, a.S, a.r_k, a.esplit);
      uint4* d4 = reinterpret_cast<uint4*>(dst);
      d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    if (ok && live) {  // the exact Key, copied as is (E4M3: rounded)
      // The row is still in shared memory: the last d/64 k-blocks staged for
      // the product are the Key's columns (128-byte rows, 16-byte chunk j of
      // row t stored at chunk j ^ (t & 7)).
      const int t = quarter * 32 + lane;
      // acquire the staged tiles' TMA writes (their last phases are complete)
      bool kok = true;
      for (int kb = nkb / 2; kb < nkb; ++kb)
        kok = kok && mbar_wait(&full[kb % kTcSlots], (kb / kTcSlots) & 1, a.status);
      uint4 kr[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < d / 8) {
          const int kb = nkb / 2 + i / 8;  // the k-block of columns 8i .. 8i + 7
          const uint8_t* tile = a_tiles + (kb % kTcSlots) * a_bytes;
          kr[i] = *reinterpret_cast<const uint4*>(tile + t * 128 + (((i & 7) ^ (t & 7)) << 4));
        }
      }
      if (!kok) {
      } else if (a.fp8) {
        uint2* dstk = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(a.K_cache) + slot * d);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i < d / 8) {
            const uint4 x = kr[i];
            const float2 f0 = bf16x2_to_f2(x.x), f1 = bf16x2_to_f2(x.y), f2 = bf16x2_to_f2(x.z),
                         f3 = bf16x2_to_f2(x.w);
            dstk[i] = make_uint2(f_to_e4m3x2(f0.x, f0.y) | (f_to_e4m3x2(f1.x, f1.y) << 16),
                                 f_to_e4m3x2(f2.x, f2.y) | (f_to_e4m3x2(f3.x, f3.y) << 16));
          }
        }
      } else {
        uint4* dstk = reinterpret_cast<uint4*>(a.K_cache + slot * d);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < d / 8) dstk[i] = kr[i];
      }
    }
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
                             const CUtensorMap& tmW, cudaStream_t st, bool pdl) {
  const int N = a.r_v + a.r_k;
  const int tmem_cols = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
  size_t smem = (size_t)kTcSlots * (kTcBM * kTcBK * 2 + N * kTcBK * 2) + 64 + 1024;
  // At most 512 / tmem_cols CTAs per SM may hold tensor memory at once: with
  // 256 columns keep it to two by shared memory (three would need <= 75 KB).
  if (tmem_cols > 128 && smem < 76 * 1024) smem = 76 * 1024;
  cudaError_t e = cudaFuncSetAttribute(append_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = a.B * a.n_new;
  dim3 grid((rows + kTcBM - 1) / kTcBM, a.Hkv);
  return launch_k(append_tc_kernel, grid, dim3(kTcThreads), smem, st, pdl, tmV, tmK, tmW, a, N,
                  tmem_cols);
}

}  // namespace basiskv
