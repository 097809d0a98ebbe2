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
#include "attend_mma.cuh"

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
  int ps_off, red_off;  // scratch after the ring, double-buffered by item parity
  int comb_off;         // fused merge: split weights and masses [2][nsplit][G] + a flag
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

template <int G, int D>
__global__ void __launch_bounds__(kAttThreads, kAttCtasPerSm)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmZ,
                  AttendArgs a, AttendGeom geo) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.smem_bytes +
                                               (a.cnt ? ((2 * a.nsplit * G * 4 + 15) & ~15) : 0));
  uint64_t* empty = full + geo.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + geo.stages);
  float* psb = reinterpret_cast<float*>(smem + geo.ps_off);    // [2][G][64] weights
  float* redb = reinterpret_cast<float*>(smem + geo.red_off);  // [2][2][warps][G]
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

  constexpr int d = D;
  const int S = a.S, r_v = a.r_v;
  const int logS = 31 - __clz(S);  // S is a power of two
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
  // Warp w owns item tokens [16w, 16w + 16) for QK and latent tiles w, w+4,
  // ... (16 latent dims each) for PV, both as warp-level tensor-core MMAs
  // (mma.m16n8k16, bf16 operands, fp32 accumulation; heads are the N = 8
  // columns).  Fragment layout: lane l holds accumulator rows l/4 and
  // l/4 + 8, columns 2(l%4) and 2(l%4)+1.  QK multiplies the exact bf16
  // products; PV splits each softmax weight into bf16 hi + lo parts (two
  // MMAs), which keeps ~16 mantissa bits of the weights.
  const int lq = lane >> 2, lr = lane & 3;
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix index, row in it
  const int zc_per_box = geo.wz / 8;
  const uint32_t zmask = geo.zmask;
  int it = 0;
  const int count = (int)(i_end - i_begin);
  // Fused merge (a.cnt set): at the end of each run of consecutive items of
  // one group, the CTA adds how many of the group's splits it wrote to the
  // group's arrival counter; the CTA that completes the count merges the
  // splits into a_lat / a_bf16.  One atomic per run instead of per item.
  float* wsp = reinterpret_cast<float*>(smem + geo.comb_off);  // [nitems][G] weights
  float* lsp = wsp + a.nsplit * G;                             // [nitems][G] masses
  volatile int* flag = reinterpret_cast<volatile int*>(lsp + a.nsplit * G);
  int seg_first = 0;  // first split of the current run
  int n = 0, bg = 0, j = 0;
  bool ready = false;
  auto arrive = [&](int T) {
    if (!a.cnt || (n + 1 < count && j + 1 < a.nsplit)) return;  // not the end of a run
    const int Pb = T > 0 ? (T + S - 1) >> logS : 0;
    const int nitems = (min(a.top_k, Pb) + geo.ppi - 1) / geo.ppi;
    const int mine = min(j + 1, nitems) - seg_first;
    named_bar_sync(1, kAttConsumers);  // the run's partial results are written
    if (tid == 0) {
      int last = 0;
      if (ready && mine > 0) last = arrive_acq_rel(&a.cnt[bg], mine) + mine == nitems;
      *flag = last;
    }
    named_bar_sync(1, kAttConsumers);
    if (!*flag) return;
    const float* part = a.partial + (size_t)bg * a.nsplit * G * (r_v + 2);
    // split statistics, all (split, head) pairs at once
    for (int i = tid; i < nitems * G; i += kAttConsumers) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(part + (size_t)i * (r_v + 2)));
      wsp[i] = ml.x;
      lsp[i] = ml.y;
    }
    named_bar_sync(1, kAttConsumers);
    // weights 2^(m_j - M) / L: warp w merges heads w, w + 4, ...
    for (int h = warp; h < G; h += kAttConsumerWarps) {
      float M = -INFINITY;
      for (int it2 = lane; it2 < nitems; it2 += 32) M = fmaxf(M, wsp[it2 * G + h]);
      M = warp_max(M);
      float L = 0.f;
      for (int it2 = lane; it2 < nitems; it2 += 32) {
        const float w = exp2f(wsp[it2 * G + h] - M);
        wsp[it2 * G + h] = w;
        L += lsp[it2 * G + h] * w;
      }
      L = warp_sum(L);
      const float invL = L > 0.f ? 1.f / L : 0.f;
      for (int it2 = lane; it2 < nitems; it2 += 32) wsp[it2 * G + h] *= invL;
    }
    named_bar_sync(1, kAttConsumers);
    // outputs, two latent channels per thread, sixteen splits in flight
    const int b = bg / a.Hkv, g = bg - b * a.Hkv;
    const size_t istride = (size_t)G * (r_v + 2);
    for (int o2 = tid; o2 < G * r_v / 2; o2 += kAttConsumers) {
      const int h = (2 * o2) / r_v, c = 2 * o2 - h * r_v;
      const float* pc = part + (size_t)h * (r_v + 2) + 2 + c;
      float vx = 0.f, vy = 0.f;
      for (int i0 = 0; i0 < nitems; i0 += 16) {
        float2 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          v[u] = i0 + u < nitems ? __ldcg(reinterpret_cast<const float2*>(pc + (i0 + u) * istride))
                                 : make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float w = i0 + u < nitems ? wsp[(i0 + u) * G + h] : 0.f;
          vx = fmaf(v[u].x, w, vx);
          vy = fmaf(v[u].y, w, vy);
        }
      }
      const size_t oi = ((size_t)b * a.Hq + g * G + h) * r_v + c;
      if (a.a_lat) {
        a.a_lat[oi] = vx;
        a.a_lat[oi + 1] = vy;
      }
      if (a.a_bf16)
        *reinterpret_cast<uint32_t*>(a.a_bf16 + oi) =
            (uint32_t)f_to_bf16(vx) | ((uint32_t)f_to_bf16(vy) << 16);
    }
    if (tid == 0) a.cnt[bg] = 0;  // ready for the next call
    named_bar_sync(1, kAttConsumers);  // wsp is reused by the next merge
  };
  ItemCursor cur;
  cur.init(i_begin, a.nsplit, a.Hkv);
  for (n = 0; n < count; ++n, cur.next(a.nsplit, a.Hkv)) {
    bg = cur.bg;
    j = cur.j;
    if (n == 0 || j == 0) seg_first = j;
    const int s = it % geo.stages;
    const int my = it++;
    // On a timeout every later wait fails at once; the item is skipped but
    // the barrier sequence below is kept, so all consumer warps stay in step.
    ready = mbar_wait_or_abort(&full[s], (my / geo.stages) & 1, a.status, abort_flag);
    const uint8_t* st = smem + (size_t)s * geo.stage_bytes;
    const int* meta = reinterpret_cast<const int*>(st + geo.meta_off);
    if (ready && meta[0] < 0) {  // empty split: nothing to attend, nothing to write
      const int T_empty = meta[31];  // read before the stage is handed back
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (a.cnt && j == 0) {  // an empty sequence: its fused merge output is zero
        const size_t o0 = ((size_t)(bg / a.Hkv) * a.Hq + (bg % a.Hkv) * G) * r_v;
        for (int o = tid; o < G * r_v; o += kAttConsumers) {
          if (a.a_lat) a.a_lat[o0 + o] = 0.f;
          if (a.a_bf16) a.a_bf16[o0 + o] = 0;
        }
      }
      arrive(T_empty);
      continue;
    }
    float* red = redb + (my & 1) * 2 * kAttConsumerWarps * G;  // scratch by item parity
    float* ps = psb + (my & 1) * G * kAttTokens;
    const int T = ready ? meta[31] : 0;
    auto tok_ok = [&](int t) -> bool {
      const int lp = ready ? meta[t >> logS] : -1;
      return lp >= 0 && (lp << logS) + (t & (S - 1)) < T;
    };

    // ---- QK: scores of the warp's 16 tokens for all heads
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    if (ready) {
      const uint16_t* qb = reinterpret_cast<const uint16_t*>(st + geo.q_off);  // [G][D] bf16
      const int t_ld = warp * 16 + (mi & 1) * 8 + mr;
      const uint8_t* krow = st + geo.k_off + (t_ld >> logS) * geo.nkb * geo.kbox;
      const int r_ld = t_ld & (S - 1);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int cc = 2 * ks + (mi >> 1);  // 16-byte chunk of the K row
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(smem_u32(krow + (cc >> 3) * geo.kbox + swz(r_ld * 128 + (cc & 7) * 16, 7u)),
                    a0, a1, a2, a3);
        uint32_t b0 = 0u, b1 = 0u;
        if (lq < G) {
          b0 = *reinterpret_cast<const uint32_t*>(qb + lq * D + ks * 16 + 2 * lr);
          b1 = *reinterpret_cast<const uint32_t*>(qb + lq * D + ks * 16 + 8 + 2 * lr);
        }
        mma_bf16_16816(c, a0, a1, a2, a3, b0, b1);
      }
    }
    const int t0 = warp * 16 + lq, t1 = t0 + 8;
    const bool v0 = tok_ok(t0), v1 = tok_ok(t1);
    const int h0 = 2 * lr, h1 = 2 * lr + 1;
    float sc[2][2];  // [token 0/1][head h0/h1], log2-scaled
    sc[0][0] = (v0 && h0 < G) ? c[0] * a.scale_log2 : -INFINITY;
    sc[0][1] = (v0 && h1 < G) ? c[1] * a.scale_log2 : -INFINITY;
    sc[1][0] = (v1 && h0 < G) ? c[2] * a.scale_log2 : -INFINITY;
    sc[1][1] = (v1 && h1 < G) ? c[3] * a.scale_log2 : -INFINITY;
    // item maximum per head: over the warp's tokens (lanes with equal l%4),
    // then over the warps
    float mx0 = fmaxf(sc[0][0], sc[1][0]), mx1 = fmaxf(sc[0][1], sc[1][1]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (lq == 0) {
      if (h0 < G) red[warp * G + h0] = mx0;
      if (h1 < G) red[warp * G + h1] = mx1;
    }
    named_bar_sync(1, kAttConsumers);
    float m0 = -INFINITY, m1 = -INFINITY;
    for (int w = 0; w < kAttConsumerWarps; ++w) {
      if (h0 < G) m0 = fmaxf(m0, red[w * G + h0]);
      if (h1 < G) m1 = fmaxf(m1, red[w * G + h1]);
    }
    // weights, their sums, and the weights for PV (ps[h][t])
    const float p00 = sc[0][0] > -INFINITY ? exp2f(sc[0][0] - m0) : 0.f;
    const float p01 = sc[0][1] > -INFINITY ? exp2f(sc[0][1] - m1) : 0.f;
    const float p10 = sc[1][0] > -INFINITY ? exp2f(sc[1][0] - m0) : 0.f;
    const float p11 = sc[1][1] > -INFINITY ? exp2f(sc[1][1] - m1) : 0.f;
    if (h0 < G) {
      ps[h0 * kAttTokens + t0] = p00;
      ps[h0 * kAttTokens + t1] = p10;
    }
    if (h1 < G) {
      ps[h1 * kAttTokens + t0] = p01;
      ps[h1 * kAttTokens + t1] = p11;
    }
    float l0 = p00 + p10, l1 = p01 + p11;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (lq == 0) {
      if (h0 < G) red[(kAttConsumerWarps + warp) * G + h0] = l0;
      if (h1 < G) red[(kAttConsumerWarps + warp) * G + h1] = l1;
    }
    // Latent rows of tokens that do not exist (past the length, or pages the
    // split does not have) hold whatever the stage held before: zero them so
    // a zero weight never meets a NaN.
    if (ready && lane < 16) {
      const int t = warp * 16 + lane;
      if (!tok_ok(t)) {
        const int pl = t >> logS, rw = t & (S - 1);
        uint8_t* zb = const_cast<uint8_t*>(st) + geo.z_off + pl * geo.nzb * geo.zbox;
        for (int cz = 0; cz < r_v / 8; ++cz)
          *reinterpret_cast<uint4*>(zb + (cz / zc_per_box) * geo.zbox +
                                    swz(rw * geo.wz * 2 + (cz % zc_per_box) * 16, zmask)) =
              make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async();  // the stage is refilled by TMA (async proxy) later
      }
    }
    named_bar_sync(1, kAttConsumers);

    // ---- PV: a[h][j] = sum_t p[h][t] z[t][j], warp = 16-row latent tiles
    float* out = a.partial + ((size_t)bg * a.nsplit + j) * G * (r_v + 2);
    for (int mt = warp; ready && mt < r_v / 16; mt += kAttConsumerWarps) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < kAttTokens / 16; ++ks) {
        const int t_ld = ks * 16 + (mi >> 1) * 8 + mr;
        const int jc = mt * 2 + (mi & 1);  // 16-byte chunk of the z row
        const uint8_t* zrow = st + geo.z_off + (t_ld >> logS) * geo.nzb * geo.zbox;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(smem_u32(zrow + (jc / zc_per_box) * geo.zbox +
                                   swz((t_ld & (S - 1)) * geo.wz * 2 + (jc % zc_per_box) * 16,
                                       zmask)),
                          a0, a1, a2, a3);
        float q00 = 0.f, q01 = 0.f, q10 = 0.f, q11 = 0.f;
        if (lq < G) {
          const float* pr = ps + lq * kAttTokens + ks * 16 + 2 * lr;
          q00 = pr[0];
          q01 = pr[1];
          q10 = pr[8];
          q11 = pr[9];
        }
        uint32_t bh0, bh1, bl0, bl1;
        split_bf16x2(q00, q01, bh0, bl0);
        split_bf16x2(q10, q11, bh1, bl1);
        mma_bf16_16816(acc, a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(acc, a0, a1, a2, a3, bl0, bl1);
      }
      const int jr = mt * 16 + lq;
      if (h0 < G) {
        out[h0 * (r_v + 2) + 2 + jr] = acc[0];
        out[h0 * (r_v + 2) + 2 + jr + 8] = acc[2];
      }
      if (h1 < G) {
        out[h1 * (r_v + 2) + 2 + jr] = acc[1];
        out[h1 * (r_v + 2) + 2 + jr + 8] = acc[3];
      }
    }
    // this warp has finished reading the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (ready && tid < G) {
      float l = 0.f, m = -INFINITY;
      for (int w = 0; w < kAttConsumerWarps; ++w) {
        l += red[(kAttConsumerWarps + w) * G + tid];
        m = fmaxf(m, red[w * G + tid]);
      }
      out[tid * (r_v + 2)] = m;
      out[tid * (r_v + 2) + 1] = l;
    }
    arrive(T);
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

// Shared-memory bytes of the fused merge (0 when it is off).
size_t attend_merge_bytes(const AttendArgs& a) {
  return a.cnt ? ((size_t)2 * a.nsplit * a.G * 4 + 15) / 16 * 16 : 0;
}

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
  // weights [2][G][64] and reductions [2][2][warps][G]
  const int scratch = 2 * G * kAttTokens * 4 + 2 * 2 * kAttConsumerWarps * G * 4 + 64;
  // 228 KB of shared memory per SM, 1 KB reserved per CTA, 1 KB of slack for
  // the 1024-byte alignment of the base.
  const int budget = 228 * 1024 / kAttCtasPerSm - 2048 - 64 - scratch;
  g.stages = budget / g.stage_bytes;
  if (g.stages > 6) g.stages = 6;
  g.ps_off = g.stages * g.stage_bytes;
  g.red_off = g.ps_off + 2 * G * kAttTokens * 4;
  g.comb_off = g.red_off + 2 * 2 * kAttConsumerWarps * G * 4;
  g.smem_bytes = (g.comb_off + 16 + 15) / 16 * 16;  // + merge scratch, added at launch
  return g;
}

template <int G, int D>
cudaError_t launch_attend_g(const AttendArgs& a, const CUtensorMap& tmK, const CUtensorMap& tmZ,
                            const AttendGeom& geo, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)geo.smem_bytes + attend_merge_bytes(a) + 2 * geo.stages * 8 + 16 +
                      1024;
  cudaError_t e = cudaFuncSetAttribute(attend_kernel<G, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long items = (long)a.B * a.Hkv * a.nsplit;
  long grid = (long)num_sms() * kAttCtasPerSm;
  if (grid > items) grid = items;
  if (grid < 1) grid = 1;
  return launch_k(attend_kernel<G, D>, dim3((unsigned)grid), dim3(kAttThreads), smem, st, pdl, tmK,
                  tmZ, a, geo);
}

}  // namespace

int attend_pages_per_split(int S) { return kAttTokens / S; }

cudaError_t launch_attend(const AttendArgs& a, const CUtensorMap& tmK, const CUtensorMap& tmZ,
                          int wz, cudaStream_t st, bool pdl) {
  const AttendGeom geo = attend_geometry(a.G, a.d, a.r_v, a.S, wz);
  if (geo.stages < 2 || geo.ppi > 31) return cudaErrorInvalidConfiguration;
  switch (a.G) {
#define BKV_ATT(GG)                                                        \
  case GG:                                                                 \
    return a.d == 64 ? launch_attend_g<GG, 64>(a, tmK, tmZ, geo, st, pdl) \
                     : launch_attend_g<GG, 128>(a, tmK, tmZ, geo, st, pdl);
    BKV_ATT(1)
    BKV_ATT(2)
    BKV_ATT(4)
    BKV_ATT(8)
#undef BKV_ATT
    default: return cudaErrorInvalidValue;
  }
}

bool attend_mma_supported(int G, int d, int r_v, int S) {
  return (G == 1 || G == 2 || G == 4 || G == 8) && (d == 64 || d == 128) && r_v % 32 == 0 &&
         r_v >= 32 && r_v <= 128 && (S == 16 || S == 32);
}

int attend_mma_slots(int B, int Hkv) { return kAmMaxCtas + B * Hkv; }

cudaError_t launch_attend_mma(const AttendArgs& a, cudaStream_t st, bool pdl) {
  if (a.fp8) return launch_attend_mma_fp8(a, st, pdl);
  if (!attend_mma_supported(a.G, a.d, a.r_v, a.S) || !a.cnt) return cudaErrorNotSupported;
#define BKV_AM_RV(GG, DD)                                                   \
  switch (a.r_v) {                                                          \
    case 32: return launch_attend_mma_t<GG, DD, 32>(a, st, pdl);            \
    case 64: return launch_attend_mma_t<GG, DD, 64>(a, st, pdl);            \
    case 96: return launch_attend_mma_t<GG, DD, 96>(a, st, pdl);            \
    default: return launch_attend_mma_t<GG, DD, 128>(a, st, pdl);           \
  }
#define BKV_AM(GG)                 \
  case GG:                         \
    if (a.d == 64) {               \
      BKV_AM_RV(GG, 64)            \
    } else {                       \
      BKV_AM_RV(GG, 128)           \
    }
  switch (a.G) {
    BKV_AM(1)
    BKV_AM(2)
    BKV_AM(4)
    BKV_AM(8)
    default: return cudaErrorNotSupported;
  }
#undef BKV_AM
#undef BKV_AM_RV
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st, bool pdl) {
  const int threads = a.r_v < 32 ? 32 : a.r_v;
  return launch_k(combine_kernel, dim3(a.B * a.Hq), dim3(threads), 0, st, pdl, a);
}

}  // namespace basiskv
