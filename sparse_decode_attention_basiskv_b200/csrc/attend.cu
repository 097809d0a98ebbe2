// Exact attention on the selected pages: BasisKV fetches the original Keys
// only for the pages the router chose (abstract; Table 4's selected-attention
// column reads the exact Key and the Value latent), and the softmax
// weights combine Value LATENTS, so each head's output is a_h in R^{r_v}.
//
//   s_t = q_h . K_t / sqrt(d);  p = softmax(s);  a_h = sum_t p_t z_t
//
// Work item = (sequence, KV head, split of the selection list) holding up to
// 128 tokens.  A persistent grid walks the items; a producer warp gathers the
// selected K and z page tiles with 2-D TMA loads (K in 128-byte swizzled
// boxes, z in 64-byte ones) through the block table into a ring of stages;
// four consumer warps compute QK with one token per thread, the item's
// softmax statistics per head, and the latent sum p.z.  Each item writes
// (max, sum, unnormalised latent) per head in the log2 domain; the combine
// kernel merges the splits.  All accumulation is fp32.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

constexpr int kAttTokens = 128;  // tokens per item = consumer threads
constexpr int kAttConsumerWarps = kAttTokens / 32;
constexpr int kAttThreads = kAttTokens + 32;

struct AttendGeom {
  int ppi;            // pages per item
  int nkb, kbox;      // K boxes per page (64 columns each) and their bytes
  int nzb, zbox, wz;  // z boxes per page, bytes, columns
  uint32_t zmask;
  int k_off, z_off;   // region offsets inside a stage
  int stage_bytes;
  int stages;
  int q_off, p_off, red_off, acc_off;  // single-buffered scratch after the ring
  int smem_bytes;
};

template <int G>
__global__ void __launch_bounds__(kAttThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmZ,
                  AttendArgs a, AttendGeom geo) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.smem_bytes);
  uint64_t* empty = full + geo.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + geo.stages);
  float* qs = reinterpret_cast<float*>(smem + geo.q_off);     // [G][d], pre-scaled
  float* ps = reinterpret_cast<float*>(smem + geo.p_off);     // [128][G]
  float* red = reinterpret_cast<float*>(smem + geo.red_off);  // [2][warps][G]
  float* accs = reinterpret_cast<float*>(smem + geo.acc_off); // [groups][G*r_v]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < geo.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kAttConsumerWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kAttConsumerWarps && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmZ);
  }
  __syncthreads();
  pdl_wait();

  const int S = a.S, d = a.d, r_v = a.r_v;
  const long total = (long)a.B * a.Hkv * a.nsplit;
  const long i_begin = total * blockIdx.x / gridDim.x;
  const long i_end = total * (blockIdx.x + 1) / gridDim.x;

  if (warp == kAttConsumerWarps) {
    if (lane == 0) {  // ------------------------------------------ producer
      int it = 0;
      for (long item = i_begin; item < i_end; ++item) {
        const int bg = (int)(item / a.nsplit), j = (int)(item % a.nsplit);
        const int b = bg / a.Hkv, g = bg % a.Hkv;
        const int32_t* sel = a.sel + (size_t)bg * a.top_k + j * geo.ppi;
        int npg = 0;
        for (int k = 0; k < geo.ppi && j * geo.ppi + k < a.top_k; ++k) npg += sel[k] >= 0;
        if (npg == 0) continue;
        const int s = it % geo.stages;
        ++it;
        if (!mbar_wait_or_abort(&empty[s], (((it - 1) / geo.stages) & 1) ^ 1, a.status,
                                abort_flag))
          continue;  // aborted: issue nothing more
        uint8_t* st = smem + (size_t)s * geo.stage_bytes;
        mbar_arrive_expect_tx(&full[s], npg * S * (d + r_v) * 2);
        for (int k = 0; k < geo.ppi && j * geo.ppi + k < a.top_k; ++k) {
          const int lp = sel[k];
          if (lp < 0) continue;
          int pp = (lp < a.max_pages) ? a.block_table[(size_t)b * a.max_pages + lp] : -1;
          if (pp < 0 || pp >= a.num_phys) {
            raise_status(a.status, BASISKV_DEV_BAD_PAGE);
            pp = 0;
          }
          const int row = (pp * a.Hkv + g) * S;
          for (int kb = 0; kb < geo.nkb; ++kb)
            tma_load_2d(st + geo.k_off + (k * geo.nkb + kb) * geo.kbox, &tmK, kb * 64, row,
                        &full[s]);
          for (int zb = 0; zb < geo.nzb; ++zb)
            tma_load_2d(st + geo.z_off + (k * geo.nzb + zb) * geo.zbox, &tmZ, zb * geo.wz, row,
                        &full[s]);
        }
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int page_local = tid / S, row = tid % S;
  const int zc_per_box = geo.wz / 8;
  const int nslot = G * r_v / 8;                 // (head, 8-wide latent chunk) slots
  const int ngrp = kAttTokens / nslot > 0 ? kAttTokens / nslot : 1;
  const int nact = nslot < kAttTokens ? nslot * ngrp : kAttTokens;
  int it = 0;
  for (long item = i_begin; item < i_end; ++item) {
    const int bg = (int)(item / a.nsplit), j = (int)(item % a.nsplit);
    const int b = bg / a.Hkv, g = bg % a.Hkv;
    const int32_t* sel = a.sel + (size_t)bg * a.top_k + j * geo.ppi;
    const int nk = min(geo.ppi, a.top_k - j * geo.ppi);
    int npg = 0;
    for (int k = 0; k < nk; ++k) npg += sel[k] >= 0;
    if (npg == 0) continue;
    int T = a.seq_lens[b];
    T = T < 0 ? 0 : T;
    const int s = it % geo.stages;
    // On a timeout every later wait fails at once; the item is skipped but
    // the barrier sequence below is kept, so all consumer warps stay in step.
    const bool ready = mbar_wait_or_abort(&full[s], (it / geo.stages) & 1, a.status, abort_flag);
    const uint32_t st = smem_u32(smem + (size_t)s * geo.stage_bytes);

    // Query of the group, scaled so that exp2 gives the softmax.
    for (int i = tid; i < G * d; i += kAttTokens)
      qs[i] = bf16_to_f(a.q[((size_t)b * a.Hq + g * G) * d + i]) * a.scale_log2;
    named_bar_sync(1, kAttTokens);

    const int lp = page_local < nk ? sel[page_local] : -1;
    const bool valid = ready && lp >= 0 && lp * S + row < T;
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sc[h] = -INFINITY;
    if (valid) {
      float acc[G][2];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = 0.f;
      const uint32_t kb0 = st + geo.k_off + page_local * geo.nkb * geo.kbox + row * 128;
      const uint32_t qb = smem_u32(qs);
#pragma unroll 4
      for (int c = 0; c < d / 8; ++c) {
        const uint32_t xa = swz(kb0 + (c >> 3) * geo.kbox + (c & 7) * 16, 7u);
        const uint4 w = lds128(xa);
        const float x0 = bf16lo(w.x), x1 = bf16hi(w.x), x2 = bf16lo(w.y), x3 = bf16hi(w.y);
        const float x4 = bf16lo(w.z), x5 = bf16hi(w.z), x6 = bf16lo(w.w), x7 = bf16hi(w.w);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 q0 = lds128f(qb + (h * d + c * 8) * 4);
          const float4 q1 = lds128f(qb + (h * d + c * 8 + 4) * 4);
          acc[h][0] = fmaf(x0, q0.x, acc[h][0]);
          acc[h][1] = fmaf(x1, q0.y, acc[h][1]);
          acc[h][0] = fmaf(x2, q0.z, acc[h][0]);
          acc[h][1] = fmaf(x3, q0.w, acc[h][1]);
          acc[h][0] = fmaf(x4, q1.x, acc[h][0]);
          acc[h][1] = fmaf(x5, q1.y, acc[h][1]);
          acc[h][0] = fmaf(x6, q1.z, acc[h][0]);
          acc[h][1] = fmaf(x7, q1.w, acc[h][1]);
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) sc[h] = acc[h][0] + acc[h][1];
    }
    // Item maximum per head.
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = warp_max(sc[h]);
      if (lane == 0) red[warp * G + h] = m;
    }
    named_bar_sync(1, kAttTokens);
    float mh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = red[h];
      for (int w = 1; w < kAttConsumerWarps; ++w) m = fmaxf(m, red[w * G + h]);
      mh[h] = m;
    }
    // Weights and their sum per head.
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float p = valid ? exp2f(sc[h] - mh[h]) : 0.f;
      ps[tid * G + h] = p;
      const float l = warp_sum(p);
      if (lane == 0) red[(kAttConsumerWarps + warp) * G + h] = l;
    }
    named_bar_sync(1, kAttTokens);
    // Latent accumulation: thread = (head, 8-wide chunk) slot x token group.
    if (ready && tid < nact) {
      const int slot = tid % nslot, grp = tid / nslot;
      const int h = slot / (r_v / 8), c = slot % (r_v / 8);
      const int box = c / zc_per_box, cc = c - box * zc_per_box;
      float acc8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc8[i] = 0.f;
      const uint32_t zb0 = st + geo.z_off + box * geo.zbox + cc * 16;
      for (int t = grp; t < kAttTokens; t += ngrp) {
        const float p = ps[t * G + h];
        if (p > 0.f) {  // skips tokens never loaded (their slots hold stale data)
          const int pl = t / S, rw = t % S;
          const uint4 w = lds128(swz(zb0 + pl * geo.nzb * geo.zbox + rw * geo.wz * 2, geo.zmask));
          acc8[0] = fmaf(p, bf16lo(w.x), acc8[0]);
          acc8[1] = fmaf(p, bf16hi(w.x), acc8[1]);
          acc8[2] = fmaf(p, bf16lo(w.y), acc8[2]);
          acc8[3] = fmaf(p, bf16hi(w.y), acc8[3]);
          acc8[4] = fmaf(p, bf16lo(w.z), acc8[4]);
          acc8[5] = fmaf(p, bf16hi(w.z), acc8[5]);
          acc8[6] = fmaf(p, bf16lo(w.w), acc8[6]);
          acc8[7] = fmaf(p, bf16hi(w.w), acc8[7]);
        }
      }
      float* dst = accs + (size_t)grp * G * r_v + h * r_v + c * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = acc8[i];
    }
    named_bar_sync(1, kAttTokens);
    // All reads of the stage are done: release it to the producer.
    if (lane == 0) mbar_arrive(&empty[s]);
    float* out = a.partial + ((size_t)bg * a.nsplit + j) * G * (r_v + 2);
    for (int i = tid; ready && i < G * r_v; i += kAttTokens) {
      const int h = i / r_v, jj = i % r_v;
      float v = 0.f;
      for (int gi = 0; gi < ngrp; ++gi) v += accs[(size_t)gi * G * r_v + i];
      out[h * (r_v + 2) + 2 + jj] = v;
    }
    if (ready && tid < G) {
      float l = 0.f;
      for (int w = 0; w < kAttConsumerWarps; ++w) l += red[(kAttConsumerWarps + w) * G + tid];
      out[tid * (r_v + 2)] = mh[tid];
      out[tid * (r_v + 2) + 1] = l;
    }
    named_bar_sync(1, kAttTokens);  // scratch is reused by the next item
    ++it;
  }
}

// Merges the splits of one head: a = sum_j acc_j 2^(m_j - M) / sum_j l_j 2^(m_j - M).
__global__ void combine_kernel(CombineArgs a) {
  pdl_wait();
  const int bh = blockIdx.x, b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / a.G, hh = h % a.G;
  const int bg = b * a.Hkv + g;
  int T = a.seq_lens[b];
  T = T < 0 ? 0 : T;
  const int P = (T + a.S - 1) / a.S;
  const int nsel = min(a.top_k, P);
  const int nitems = (nsel + a.pages_per_split - 1) / a.pages_per_split;
  const float* base = a.partial + (size_t)bg * a.nsplit * a.G * (a.r_v + 2) + hh * (a.r_v + 2);
  const size_t item_stride = (size_t)a.G * (a.r_v + 2);
  float M = -INFINITY;
  for (int j = 0; j < nitems; ++j) M = fmaxf(M, base[j * item_stride]);
  float L = 0.f;
  for (int j = 0; j < nitems; ++j) L += base[j * item_stride + 1] * exp2f(base[j * item_stride] - M);
  const float invL = L > 0.f ? 1.f / L : 0.f;
  for (int c = threadIdx.x; c < a.r_v; c += blockDim.x) {
    float v = 0.f;
    for (int j = 0; j < nitems; ++j)
      v += base[j * item_stride + 2 + c] * exp2f(base[j * item_stride] - M);
    v *= invL;
    const size_t o = ((size_t)b * a.Hq + h) * a.r_v + c;
    if (a.a_lat) a.a_lat[o] = v;
    if (a.a_bf16) a.a_bf16[o] = f_to_bf16(v);
  }
}

AttendGeom attend_geometry(int G, int d, int r_v, int S, int wz) {
  AttendGeom g{};
  g.ppi = kAttTokens / S;
  g.nkb = d / 64;
  g.kbox = S * 128;
  g.wz = wz;
  g.nzb = r_v / wz;
  g.zbox = S * wz * 2;
  g.zmask = wz == 32 ? 3u : 1u;
  g.k_off = 0;
  g.z_off = g.ppi * g.nkb * g.kbox;
  g.stage_bytes = (g.z_off + g.ppi * g.nzb * g.zbox + 1023) / 1024 * 1024;
  const int nslot = G * r_v / 8;
  const int ngrp = kAttTokens / nslot > 0 ? kAttTokens / nslot : 1;
  const int scratch = G * d * 4 + kAttTokens * G * 4 + 2 * kAttConsumerWarps * G * 4 +
                      ngrp * G * r_v * 4 + 4096;
  const int budget = 220 * 1024 - scratch;
  g.stages = budget / g.stage_bytes;
  if (g.stages > 6) g.stages = 6;
  g.q_off = g.stages * g.stage_bytes;
  g.p_off = g.q_off + G * d * 4;
  g.red_off = g.p_off + kAttTokens * G * 4;
  g.acc_off = g.red_off + 2 * kAttConsumerWarps * G * 4;
  g.smem_bytes = (g.acc_off + ngrp * G * r_v * 4 + 15) / 16 * 16;
  return g;
}

template <int G>
cudaError_t launch_attend_g(const AttendArgs& a, const CUtensorMap& tmK, const CUtensorMap& tmZ,
                            const AttendGeom& geo, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)geo.smem_bytes + 2 * geo.stages * 8 + 16 + 1024;
  cudaError_t e = cudaFuncSetAttribute(attend_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long items = (long)a.B * a.Hkv * a.nsplit;
  long grid = num_sms();
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  return launch_k(attend_kernel<G>, dim3((unsigned)grid), dim3(kAttThreads), smem, st, pdl, tmK,
                  tmZ, a, geo);
}

}  // namespace

int attend_pages_per_split(int S) { return kAttTokens / S; }

cudaError_t launch_attend(const AttendArgs& a, const CUtensorMap& tmK, const CUtensorMap& tmZ,
                          int wz, cudaStream_t st, bool pdl) {
  const AttendGeom geo = attend_geometry(a.G, a.d, a.r_v, a.S, wz);
  if (geo.stages < 2) return cudaErrorInvalidConfiguration;
  switch (a.G) {
    case 1: return launch_attend_g<1>(a, tmK, tmZ, geo, st, pdl);
    case 2: return launch_attend_g<2>(a, tmK, tmZ, geo, st, pdl);
    case 4: return launch_attend_g<4>(a, tmK, tmZ, geo, st, pdl);
    case 8: return launch_attend_g<8>(a, tmK, tmZ, geo, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, bool pdl) {
  const int threads = a.r_v < 32 ? 32 : a.r_v;
  return launch_k(combine_kernel, dim3(a.B * a.Hq), dim3(threads), 0, st, pdl, a);
}

}  // namespace basiskv
