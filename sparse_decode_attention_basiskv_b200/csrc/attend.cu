// Exact attention on the selected pages: BasisKV fetches the original Keys
// only for the pages the router chose (abstract; Table 4's selected-attention
// column reads the exact Key and the Value latent), and the softmax
// weights combine Value LATENTS, so each head's output is a_h in R^{r_v}.
//
//   s_t = q_h . K_t / sqrt(d);  p = softmax(s);  a_h = sum_t p_t z_t
//
// Work item = (sequence, KV head, split of the selection list) holding up to
// 64 tokens.  A persistent grid walks the items.  The producer warp fetches
// the item's page ids (selection list, then block table) a few items ahead,
// and per item issues, one lane per page, 2-D TMA loads of the exact-Key and
// Value-latent page tiles (K in 128-byte swizzled boxes, z in 64-byte ones);
// it also copies the group's queries and a small record (page ids, length)
// into the stage, so consumers never wait on global memory.  Four consumer
// warps handle an item: two threads per token split the head dimension for
// QK (packed fp32x2 FMAs), the item's softmax statistics come from warp
// shuffles and one shared-memory exchange, and the latent sum p.z is spread
// over (head, 8-wide chunk, token group).  Each item writes (max, sum,
// unnormalised latent) per head in the log2 domain; the combine kernel
// merges the splits.  All accumulation is fp32.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace basiskv {

namespace {

// Three small independent rings per SM (3 CTAs of 64-token items) stream
// faster than one large ring: a single producer/consumer ring per CTA caps
// well below the HBM bandwidth on B200 (measured on the routing stream).
constexpr int kAttTokens = 64;                        // tokens per item
constexpr int kAttConsumers = 2 * kAttTokens;         // two threads per token
constexpr int kAttConsumerWarps = kAttConsumers / 32;
constexpr int kAttThreads = kAttConsumers + 32;       // + producer warp
constexpr int kAttCtasPerSm = 3;
constexpr int kAttAhead = 4;                          // items of page ids fetched ahead
constexpr int kMetaInts = 32;                         // page ids [ppi] | T at [31]

struct AttendGeom {
  int ppi;            // pages per item
  int nkb, kbox;      // K boxes per page (64 columns each) and their bytes
  int nzb, zbox, wz;  // z boxes per page, bytes, columns
  uint32_t zmask;
  int k_off, z_off, q_off, meta_off;  // regions inside a stage
  int stage_bytes;
  int stages;
  int qs_off, ps_off, red_off, acc_off;  // single-buffered scratch after the ring
  int qs_stride;                          // floats per head in qs (d + 8)
  int smem_bytes;
};

// Walks a contiguous range of (sequence, KV head, split) items with one
// division at the start and increments afterwards.
struct ItemCursor {
  int bg, j, b, g;
  __device__ void init(long item, int nsplit, int Hkv) {
    bg = (int)(item / nsplit);
    j = (int)(item - (long)bg * nsplit);
    b = bg / Hkv;
    g = bg - b * Hkv;
  }
  __device__ void next(int nsplit, int Hkv) {
    if (++j == nsplit) {
      j = 0;
      ++bg;
      if (++g == Hkv) {
        g = 0;
        ++b;
      }
    }
  }
};

template <int G>
__global__ void __launch_bounds__(kAttThreads, kAttCtasPerSm)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmZ,
                  AttendArgs a, AttendGeom geo) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.smem_bytes);
  uint64_t* empty = full + geo.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + geo.stages);
  float* qs = reinterpret_cast<float*>(smem + geo.qs_off);     // [G][d + 8], pre-scaled
  float* ps = reinterpret_cast<float*>(smem + geo.ps_off);     // [128][G]
  float* red = reinterpret_cast<float*>(smem + geo.red_off);   // [2][warps][G]
  float* accs = reinterpret_cast<float*>(smem + geo.acc_off);  // [groups][G*r_v]
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
    // ------------------------------------------------------------ producer
    // lane k < ppi owns page k of each item; the rings hold the physical and
    // logical page (or -1) of the next kAttAhead items.
    const int count = (int)(i_end - i_begin);
    ItemCursor pre, cur;
    pre.init(i_begin, a.nsplit, a.Hkv);
    cur = pre;
    auto fetch = [&](int n, int& lp) -> int {  // pages of item i_begin + n, then advance
      lp = -1;
      int pp = -1;
      if (n < count) {
        const int k = pre.j * geo.ppi + lane;
        if (lane < geo.ppi && k < a.top_k) {
          lp = a.sel[(size_t)pre.bg * a.top_k + k];
          if (lp >= 0) {
            pp = lp < a.max_pages ? a.block_table[(size_t)pre.b * a.max_pages + lp] : -1;
            if (pp < 0 || pp >= a.num_phys) {
              raise_status(a.status, BASISKV_DEV_BAD_PAGE);
              pp = 0;  // keep the byte count; this page's tokens are flagged garbage
            }
          }
        }
        pre.next(a.nsplit, a.Hkv);
      }
      return pp;
    };
    int ring_pp[kAttAhead], ring_lp[kAttAhead];
#pragma unroll
    for (int k = 0; k < kAttAhead; ++k) ring_pp[k] = fetch(k, ring_lp[k]);
    int it = 0;
    for (int n = 0; n < count; ++n, cur.next(a.nsplit, a.Hkv)) {
      const int pp = ring_pp[0], lp = ring_lp[0];
#pragma unroll
      for (int k = 0; k + 1 < kAttAhead; ++k) {
        ring_pp[k] = ring_pp[k + 1];
        ring_lp[k] = ring_lp[k + 1];
      }
      ring_pp[kAttAhead - 1] = fetch(n + kAttAhead, ring_lp[kAttAhead - 1]);
      // Every item gets a stage; an empty split (its first selection entry is
      // -1: the list is ascending with the padding at the end) carries only
      // its record, so the consumers never read the selection list.
      const int npg = __popc(__ballot_sync(0xffffffffu, lp >= 0));
      const int b = cur.b, g = cur.g;
      const int s = it % geo.stages;
      ++it;
      uint8_t* st = smem + (size_t)s * geo.stage_bytes;
      bool go = true;
      if (lane == 0)
        go = mbar_wait_or_abort(&empty[s], (((it - 1) / geo.stages) & 1) ^ 1, a.status,
                                abort_flag);
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) continue;  // aborted: issue nothing more
      // record: page ids and the sequence length, published by the arrive below
      int* meta = reinterpret_cast<int*>(st + geo.meta_off);
      if (lane < geo.ppi) meta[lane] = lp;
      if (lane == 31) meta[31] = a.seq_lens[b] + a.len_offset;
      __syncwarp();
      if (lane == 0) {
        if (npg > 0) {
          mbar_arrive_expect_tx(&full[s], npg * S * (d + r_v) * 2 + G * d * 2);
          bulk_load(st + geo.q_off, a.q + ((size_t)b * a.Hq + g * G) * d, G * d * 2, &full[s]);
        } else {
          mbar_arrive(&full[s]);
        }
      }
      __syncwarp();
      if (lp >= 0) {
        const int row = (pp * a.Hkv + g) * S;
        for (int kb = 0; kb < geo.nkb; ++kb)
          tma_load_2d(st + geo.k_off + (lane * geo.nkb + kb) * geo.kbox, &tmK, kb * 64, row,
                      &full[s]);
        for (int zb = 0; zb < geo.nzb; ++zb)
          tma_load_2d(st + geo.z_off + (lane * geo.nzb + zb) * geo.zbox, &tmZ, zb * geo.wz,
                      row, &full[s]);
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int tok = tid >> 1, half = tid & 1;
  const int page_local = tok / S, row = tok % S;
  const int zc_per_box = geo.wz / 8;
  const int nslot = G * r_v / 8;  // (head, 8-wide latent chunk) slots
  const int ngrp = kAttConsumers / nslot > 0 ? kAttConsumers / nslot : 1;
  const int nact = nslot < kAttConsumers ? nslot * ngrp : kAttConsumers;
  const int QS = geo.qs_stride;
  const int nch = d / 16;  // 16-byte chunks per half of a K row
  int it = 0;
  const int count = (int)(i_end - i_begin);
  ItemCursor cur;
  cur.init(i_begin, a.nsplit, a.Hkv);
  for (int n = 0; n < count; ++n, cur.next(a.nsplit, a.Hkv)) {
    const int bg = cur.bg, j = cur.j;
    const int s = it % geo.stages;
    const int my = it++;
    // On a timeout every later wait fails at once; the item is skipped but
    // the barrier sequence below is kept, so all consumer warps stay in step.
    bool ready = mbar_wait_or_abort(&full[s], (my / geo.stages) & 1, a.status, abort_flag);
    const uint8_t* st = smem + (size_t)s * geo.stage_bytes;
    const int* meta = reinterpret_cast<const int*>(st + geo.meta_off);
    if (ready && meta[0] < 0) {  // empty split: nothing to attend, nothing to write
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      continue;
    }

    // Queries of the group, fp32 and scaled so that exp2 gives the softmax;
    // the second half of each head is shifted by 4 floats (bank spread).
    if (ready) {
      const uint16_t* qb = reinterpret_cast<const uint16_t*>(st + geo.q_off);
      for (int i = tid; i < G * d; i += kAttConsumers) {
        const int h = i / d, c = i % d;
        qs[h * QS + c + (c >= d / 2 ? 4 : 0)] = bf16_to_f(qb[i]) * a.scale_log2;
      }
    }
    named_bar_sync(1, kAttConsumers);

    const int T = ready ? meta[31] : 0;
    const int lp = (ready && page_local < geo.ppi) ? meta[page_local] : -1;
    const bool valid = lp >= 0 && lp * S + row < T;
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) sc[h] = 0.f;
    if (valid) {
      float2 acc[G][2];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = make_float2(0.f, 0.f);
      const uint8_t* kb0 = st + geo.k_off + page_local * geo.nkb * geo.kbox;
      for (int i = 0; i < nch; ++i) {
        // half 1 walks its chunks in a rotated order so that the two halves of
        // neighbouring tokens hit different banks
        const int c = half ? nch + ((i + nch / 2) % nch) : i;
        const uint32_t off = (c >> 3) * geo.kbox + swz(row * 128 + (c & 7) * 16, 7u);
        const uint4 w = *reinterpret_cast<const uint4*>(kb0 + off);
        const float2 x0 = bf16x2_to_f2(w.x), x1 = bf16x2_to_f2(w.y);
        const float2 x2 = bf16x2_to_f2(w.z), x3 = bf16x2_to_f2(w.w);
        const int qo = c * 8 + (half ? 4 : 0);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 q0 = *reinterpret_cast<const float4*>(qs + h * QS + qo);
          const float4 q1 = *reinterpret_cast<const float4*>(qs + h * QS + qo + 4);
          ffma2(acc[h][0], x0, make_float2(q0.x, q0.y));
          ffma2(acc[h][1], x1, make_float2(q0.z, q0.w));
          ffma2(acc[h][0], x2, make_float2(q1.x, q1.y));
          ffma2(acc[h][1], x3, make_float2(q1.z, q1.w));
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
        sc[h] = (acc[h][0].x + acc[h][1].x) + (acc[h][0].y + acc[h][1].y);
    }
    // The two halves of a token sum their partial dot products.
#pragma unroll
    for (int h = 0; h < G; ++h) {
      sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], 1);
      if (!valid) sc[h] = -INFINITY;
    }
    // Item maximum per head.
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m = warp_max(sc[h]);
      if (lane == 0) red[warp * G + h] = m;
    }
    named_bar_sync(1, kAttConsumers);
    float mh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = red[h];
      for (int w = 1; w < kAttConsumerWarps; ++w) m = fmaxf(m, red[w * G + h]);
      mh[h] = m;
    }
    // Weights and their sum per head (one thread of each token pair counts).
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float p = valid ? exp2f(sc[h] - mh[h]) : 0.f;
      if (half == 0) ps[tok * G + h] = p;
      const float l = warp_sum(half == 0 ? p : 0.f);
      if (lane == 0) red[(kAttConsumerWarps + warp) * G + h] = l;
    }
    named_bar_sync(1, kAttConsumers);
    // Latent accumulation: thread = (head, 8-wide chunk) slot x token group.
    if (ready && tid < nact) {
      const int slot = tid % nslot, grp = tid / nslot;
      const int h = slot / (r_v / 8), c = slot % (r_v / 8);
      const int box = c / zc_per_box, cc = c - box * zc_per_box;
      float2 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
      const uint8_t* zb0 = st + geo.z_off + box * geo.zbox;
      for (int t = grp; t < kAttTokens; t += ngrp) {
        const float p = ps[t * G + h];
        if (p > 0.f) {  // skips tokens never loaded (their slots hold stale data)
          const int pl = t / S, rw = t % S;
          const uint4 w = *reinterpret_cast<const uint4*>(
              zb0 + pl * geo.nzb * geo.zbox + swz(rw * geo.wz * 2 + cc * 16, geo.zmask));
          const float2 pp = make_float2(p, p);
          ffma2(acc[0], pp, bf16x2_to_f2(w.x));
          ffma2(acc[1], pp, bf16x2_to_f2(w.y));
          ffma2(acc[2], pp, bf16x2_to_f2(w.z));
          ffma2(acc[3], pp, bf16x2_to_f2(w.w));
        }
      }
      float* dst = accs + (size_t)grp * G * r_v + h * r_v + c * 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dst[2 * i] = acc[i].x;
        dst[2 * i + 1] = acc[i].y;
      }
    }
    named_bar_sync(1, kAttConsumers);
    // All reads of the stage are done: release it to the producer.
    if (lane == 0) mbar_arrive(&empty[s]);
    float* out = a.partial + ((size_t)bg * a.nsplit + j) * G * (r_v + 2);
    for (int i = tid; ready && i < G * r_v; i += kAttConsumers) {
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
    named_bar_sync(1, kAttConsumers);  // scratch is reused by the next item
  }
}

// Merges the splits of one head: a = sum_j acc_j 2^(m_j - M) / sum_j l_j 2^(m_j - M).
// The split statistics are read in parallel (one thread per split), the
// weights formed once in shared memory, and the latent channels then
// accumulate with independent loads.
constexpr int kCombineMaxSplits = 1024;

__global__ void combine_kernel(CombineArgs a) {
  __shared__ float wsh[kCombineMaxSplits];
  __shared__ float red[32];
  pdl_wait();
  const int bh = blockIdx.x, b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / a.G, hh = h % a.G;
  const int bg = b * a.Hkv + g;
  const int tid = threadIdx.x, nth = blockDim.x;
  int T = a.seq_lens[b] + a.len_offset;
  T = T < 0 ? 0 : T;
  const int P = (T + a.S - 1) / a.S;
  const int nsel = min(a.top_k, P);
  const int nitems = (nsel + a.pages_per_split - 1) / a.pages_per_split;
  const size_t item_stride = (size_t)a.G * (a.r_v + 2);
  const float* base = a.partial + (size_t)bg * a.nsplit * item_stride + hh * (a.r_v + 2);
  // maximum of the split maxima
  float m = -INFINITY;
  for (int j = tid; j < nitems; j += nth) {
    const float mj = base[j * item_stride];
    wsh[j] = mj;
    m = fmaxf(m, mj);
  }
  m = warp_max(m);
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  float M = red[0];
  for (int w = 1; w < (nth + 31) / 32; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  // weights 2^(m_j - M) and the total mass
  float l = 0.f;
  for (int j = tid; j < nitems; j += nth) {
    const float w = exp2f(wsh[j] - M);
    wsh[j] = w;
    l += base[j * item_stride + 1] * w;
  }
  l = warp_sum(l);
  if ((tid & 31) == 0) red[tid >> 5] = l;
  __syncthreads();
  float L = 0.f;
  for (int w = 0; w < (nth + 31) / 32; ++w) L += red[w];
  const float invL = L > 0.f ? 1.f / L : 0.f;
  for (int c = tid; c < a.r_v; c += nth) {
    float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
    int j = 0;
    for (; j + 4 <= nitems; j += 4) {
      v0 = fmaf(base[(j + 0) * item_stride + 2 + c], wsh[j + 0], v0);
      v1 = fmaf(base[(j + 1) * item_stride + 2 + c], wsh[j + 1], v1);
      v2 = fmaf(base[(j + 2) * item_stride + 2 + c], wsh[j + 2], v2);
      v3 = fmaf(base[(j + 3) * item_stride + 2 + c], wsh[j + 3], v3);
    }
    for (; j < nitems; ++j) v0 = fmaf(base[j * item_stride + 2 + c], wsh[j], v0);
    const float v = ((v0 + v1) + (v2 + v3)) * invL;
    const size_t o = ((size_t)b * a.Hq + h) * a.r_v + c;
    if (a.a_lat) a.a_lat[o] = v;
    if (a.a_bf16) a.a_bf16[o] = f_to_bf16(v);
  }
}

int round1k(int x) { return (x + 1023) / 1024 * 1024; }

AttendGeom attend_geometry(int G, int d, int r_v, int S, int wz) {
  AttendGeom g{};
  g.ppi = kAttTokens / S;
  g.nkb = d / 64;
  g.kbox = S * 128;
  g.wz = wz;
  g.nzb = r_v / wz;
  g.zbox = S * wz * 2;
  g.zmask = wz == 64 ? 7u : (wz == 32 ? 3u : 1u);
  g.k_off = 0;
  g.z_off = round1k(g.ppi * g.nkb * g.kbox);
  g.q_off = g.z_off + round1k(g.ppi * g.nzb * g.zbox);
  g.meta_off = g.q_off + G * d * 2;
  g.stage_bytes = round1k(g.meta_off + kMetaInts * 4);
  g.qs_stride = d + 8;
  const int nslot = G * r_v / 8;
  const int ngrp = kAttConsumers / nslot > 0 ? kAttConsumers / nslot : 1;
  const int scratch = G * g.qs_stride * 4 + kAttTokens * G * 4 +
                      2 * kAttConsumerWarps * G * 4 + ngrp * G * r_v * 4 + 2048;
  // 228 KB of shared memory per SM, 1 KB reserved per CTA, 1 KB of slack for
  // the 1024-byte alignment of the base.
  const int budget = 228 * 1024 / kAttCtasPerSm - 2048 - 64 - scratch;
  g.stages = budget / g.stage_bytes;
  if (g.stages > 6) g.stages = 6;
  g.qs_off = g.stages * g.stage_bytes;
  g.ps_off = g.qs_off + G * g.qs_stride * 4;
  g.red_off = g.ps_off + kAttTokens * G * 4;
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
  long grid = (long)num_sms() * kAttCtasPerSm;
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
  if (geo.stages < 2 || geo.ppi > 31) return cudaErrorInvalidConfiguration;
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
