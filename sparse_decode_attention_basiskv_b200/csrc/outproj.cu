// Latent out-projection on the 5th-generation tensor cores.
//
// BasisKV associates the Value factor with the output projection (abstract;
// Figure 1 caption: the complete output is reconstructed from the Value
// latents), so the decode output is
//   y[b][o] = sum_h a_h[b] . W'_h[:, o],   W'_h = B_V,g(h) W_O,h
// i.e. one [B x Hq*r_v] x [Hq*r_v x H] product per step.  The batch is small,
// so the product is computed transposed ("swap AB"):
//   D[o][b] = sum_k W_fold[o][k] * a[b][k]      M = H, N = B (padded), K = Hq*r_v
// with both operands K-major.  Each CTA owns a 128-row M tile and a slice of
// K; a TMA producer warp streams 128x64 W tiles and Nx64 a tiles (128-byte
// swizzle) into a ring of stages, one thread issues tcgen05.mma (kind::f16,
// bf16 inputs, fp32 accumulator in tensor memory), and four epilogue warps
// read the accumulator back with tcgen05.ld.  K slices are summed by a
// second small kernel when the K dimension is split.  The kernel is bound by
// streaming W_fold from HBM.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

constexpr int kOpThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kOpBM = 128, kOpBK = 64;
// Ring depth: as many stages of (16 KB + BN*128 B) as fit in 200 KB, at most
// 8 (a decode-size K slice is 8 stages deep, so the whole slice of W' can be
// in flight before the latents are ready).
template <int BN>
constexpr int op_stages() {
  return (200 * 1024) / (kOpBM * kOpBK * 2 + BN * kOpBK * 2) < 8
             ? (200 * 1024) / (kOpBM * kOpBK * 2 + BN * kOpBK * 2)
             : 8;
}
constexpr int kOpATile = kOpBM * kOpBK * 2;  // 16 KB

// tcgen05 instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B,
// both K-major, N>>3 at bit 17, M>>4 at bit 24.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major tile with 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);  // start address
  d |= (uint64_t)1 << 16;                   // leading byte offset (unused here)
  d |= (uint64_t)(1024 >> 4) << 32;         // stride byte offset
  d |= (uint64_t)1 << 46;                   // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                   // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <int BN>
__global__ void __launch_bounds__(kOpThreads, 1)
    outproj_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                   OutprojArgs a) {
  constexpr int kBTile = BN * kOpBK * 2;
  constexpr int kOpStages = op_stages<BN>();
  constexpr int kTmemCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint8_t* a_tiles = smem;                              // kOpStages x 16 KB
  uint8_t* b_tiles = smem + kOpStages * kOpATile;       // kOpStages x kBTile
  uint64_t* full = reinterpret_cast<uint64_t*>(b_tiles + kOpStages * kBTile);
  uint64_t* empty = full + kOpStages;
  uint64_t* accum = empty + kOpStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kOpBM;
  const int nkb_total = a.K / kOpBK;
  const int kb0 = nkb_total * blockIdx.y / a.ksplit;
  const int kb1 = nkb_total * (blockIdx.y + 1) / a.ksplit;

  if (tid == 0) {
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmA);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Only the producer (before the latent tiles) and the length update wait
  // for the earlier kernels: W' is a weight no kernel of the step writes, so
  // the first stages of it are requested while the attention finishes.
  if (a.bump_lens && blockIdx.x == 0 && blockIdx.y == 0 && warp == 2) {
    pdl_wait();
    for (int b = lane; b < a.B; b += 32) {
      const int len = a.bump_lens[b];
      if (len >= 0 && len + a.bump_n <= a.bump_cap) a.bump_lens[b] = len + a.bump_n;
    }
  }

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------- TMA producer
      const int pre = kb1 - kb0 < kOpStages ? kb1 - kb0 : kOpStages;
      for (int it = 0; it < pre; ++it) {  // stages start empty
        mbar_arrive_expect_tx(&full[it], kOpATile + kBTile);
        tma_load_2d(a_tiles + it * kOpATile, &tmW, (kb0 + it) * kOpBK, m0, &full[it]);
      }
      pdl_wait();
      // latent column k = source k / k_src, column k % k_src of its B rows
      auto load_a = [&](uint8_t* dst, int kb, uint64_t* bar) {
        const int kc = kb * kOpBK;
        tma_load_2d(dst, &tmA, kc % a.k_src, (kc / a.k_src) * a.B, bar);
      };
      for (int it = 0; it < pre; ++it) load_a(b_tiles + it * kBTile, kb0 + it, &full[it]);
      for (int kb = kb0 + pre, it = pre; kb < kb1; ++kb, ++it) {
        const int s = it % kOpStages;
        if (!mbar_wait(&empty[s], ((it / kOpStages) & 1) ^ 1, a.status)) break;
        mbar_arrive_expect_tx(&full[s], kOpATile + kBTile);
        tma_load_2d(a_tiles + s * kOpATile, &tmW, kb * kOpBK, m0, &full[s]);
        load_a(b_tiles + s * kBTile, kb, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ------------------------------------------ MMA issue
      const uint32_t idesc = make_idesc(kOpBM, BN);
      bool ok = true;
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s = it % kOpStages;
        if (!mbar_wait(&full[s], (it / kOpStages) & 1, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = make_sdesc(smem_u32(a_tiles + s * kOpATile));
        const uint64_t db = make_sdesc(smem_u32(b_tiles + s * kBTile));
#pragma unroll
        for (int k = 0; k < kOpBK / 16; ++k)  // 32 bytes of K per instruction
          tc_mma(tmem, da + 2 * k, db + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (ok) tc_commit(accum);
    }
  } else {  // ------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    if (mbar_wait(accum, 0, a.status)) {
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n < a.B) {
            if (a.ksplit == 1)
              a.y[(size_t)n * a.H + m0 + row] = f_to_bf16(v[j]);
            else
              a.partial[((size_t)blockIdx.y * a.B + n) * a.H + m0 + row] = v[j];
          }
        }
      }
    }
  }
  if (a.ksplit > 1 && a.cnt) {
    // arrival: the last CTA of this M tile sums the K-split partials into y
    __shared__ int last;
    __syncthreads();  // this CTA's partials are written
    if (tid == 0) last = arrive_acq_rel(&a.cnt[blockIdx.x], 1) == a.ksplit - 1;
    __syncthreads();
    if (last) {
      // four rows of one batch column per float4; up to three groups per
      // thread, every load of a split issued before any sum needs it
      const int ngrp = kOpBM / 4 * a.B;
      const size_t kstride = (size_t)a.B * a.H;
      for (int i0 = tid; i0 < ngrp; i0 += 3 * kOpThreads) {
        float4 acc[3];
        const float* src[3];
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          const int i = min(i0 + u * kOpThreads, ngrp - 1);
          const int n = i / (kOpBM / 4), r4 = (i - n * (kOpBM / 4)) * 4;
          src[u] = a.partial + (size_t)n * a.H + m0 + r4;
          acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll 4
        for (int k = 0; k < a.ksplit; ++k) {  // splits summed in order, as the reduce kernel does
          float4 v[3];
#pragma unroll
          for (int u = 0; u < 3; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(src[u] + k * kstride));
#pragma unroll
          for (int u = 0; u < 3; ++u) {
            acc[u].x += v[u].x;
            acc[u].y += v[u].y;
            acc[u].z += v[u].z;
            acc[u].w += v[u].w;
          }
        }
#pragma unroll
        for (int u = 0; u < 3; ++u) {
          if (i0 + u * kOpThreads >= ngrp) break;
          uint16_t* dst = a.y + (src[u] - a.partial);
          *reinterpret_cast<uint2*>(dst) =
              make_uint2((uint32_t)f_to_bf16(acc[u].x) | ((uint32_t)f_to_bf16(acc[u].y) << 16),
                         (uint32_t)f_to_bf16(acc[u].z) | ((uint32_t)f_to_bf16(acc[u].w) << 16));
        }
      }
      if (tid == 0) a.cnt[blockIdx.x] = 0;  // ready for the next call
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

__global__ void ksplit_reduce_kernel(const float* part, uint16_t* y, int ksplit, size_t n) {
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int k = 0; k < ksplit; ++k) v += part[k * n + i];
    y[i] = f_to_bf16(v);
  }
}

__global__ void cast_bf16_kernel(const float* x, uint16_t* y, size_t n) {
  pdl_wait();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    y[i] = f_to_bf16(x[i]);
}

// W_fold[o][h*r_v + j] = sum_i B_V[g(h)][j][i] * W_O[h*d + i][o]   (fp32 -> bf16)
// One-time setup: thread = output column o, CTA = (128 columns, head h,
// 32-wide slice of j).
__global__ void __launch_bounds__(128) fold_outproj_kernel(FoldOutArgs a) {
  const int o = blockIdx.x * 128 + threadIdx.x;
  const int h = blockIdx.y, j0 = blockIdx.z * 32;
  const int g = h / (a.Hq / a.Hkv);
  __shared__ float bv[32][129];
  const int nj = min(32, a.r_v - j0);
  for (int i = threadIdx.x; i < nj * a.d; i += 128) {
    const int jj = i / a.d, ii = i % a.d;
    bv[jj][ii] = bf16_to_f(a.B_V[((size_t)g * a.r_v + j0 + jj) * a.d + ii]);
  }
  __syncthreads();
  if (o >= a.H) return;
  float acc[32];
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) acc[jj] = 0.f;
  for (int i = 0; i < a.d; ++i) {
    const float w = bf16_to_f(a.W_O[((size_t)h * a.d + i) * a.H + o]);
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) acc[jj] = fmaf(bv[jj][i], w, acc[jj]);
  }
  const size_t K = (size_t)a.Hq * a.r_v;
  for (int jj = 0; jj < nj; ++jj) a.W_fold[(size_t)o * K + h * a.r_v + j0 + jj] = f_to_bf16(acc[jj]);
}

template <int BN>
cudaError_t launch_outproj_bn(const OutprojArgs& a, const CUtensorMap& tmW,
                              const CUtensorMap& tmA, cudaStream_t st, bool pdl) {
  constexpr int kOpStages = op_stages<BN>();
  const size_t smem = kOpStages * (kOpATile + BN * kOpBK * 2) + (2 * kOpStages + 1) * 8 + 16 + 1024;
  cudaError_t e = cudaFuncSetAttribute(outproj_kernel<BN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.H / kOpBM, a.ksplit);
  e = launch_k(outproj_kernel<BN>, grid, dim3(kOpThreads), smem, st, pdl, tmW, tmA, a);
  if (e != cudaSuccess || a.ksplit == 1 || a.cnt) return e;
  const size_t n = (size_t)a.B * a.H;
  return launch_k(ksplit_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, pdl,
                  (const float*)a.partial, a.y, a.ksplit, n);
}

}  // namespace

int outproj_bn(int B) {
  if (B <= 16) return 16;
  if (B <= 32) return 32;
  if (B <= 64) return 64;
  if (B <= 128) return 128;
  return 256;
}

int outproj_ksplit(int H, int K, int B) {
  (void)B;
  const int mtiles = H / kOpBM, nkb = K / kOpBK;
  int ks = num_sms() / mtiles;
  if (ks < 1) ks = 1;
  if (ks > nkb) ks = nkb;
  if (ks > 16) ks = 16;
  return ks;
}

cudaError_t launch_outproj(const OutprojArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmA,
                           cudaStream_t st, bool pdl) {
  switch (a.bn) {
    case 16: return launch_outproj_bn<16>(a, tmW, tmA, st, pdl);
    case 32: return launch_outproj_bn<32>(a, tmW, tmA, st, pdl);
    case 64: return launch_outproj_bn<64>(a, tmW, tmA, st, pdl);
    case 128: return launch_outproj_bn<128>(a, tmW, tmA, st, pdl);
    case 256: return launch_outproj_bn<256>(a, tmW, tmA, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_cast_bf16(const float* x, uint16_t* y, size_t n, cudaStream_t st, bool pdl) {
  const unsigned blocks = (unsigned)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  return launch_k(cast_bf16_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, pdl, x, y, n);
}

cudaError_t launch_fold_outproj(const FoldOutArgs& a, cudaStream_t st) {
  dim3 grid((a.H + 127) / 128, a.Hq, (a.r_v + 31) / 32);
  return launch_k(fold_outproj_kernel, grid, dim3(128), 0, st, false, a);
}

}  // namespace basiskv
