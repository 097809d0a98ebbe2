// Routing: BasisKV scores every page of the full context from the narrow
// per-token state (Value latent z and Key residual e) instead of the exact
// Keys (abstract: the cached latent stands in for part of each Key when
// pages are ranked; Table 4, full-context routing column).
//
// The predicted key of token t is khat_t = z_t P_K + e_t U_K^T, and
//   q_h . khat_t = z_t . (P_K q_h) + e_t . (U_K^T q_h),
// so the query is folded once per step (fold_query_kernel) and the hot loop
// streams only z and e: (r_v + r_k) * 2 bytes per token and KV head.
//
// route_kernel is HBM-bound.  A persistent grid of one CTA per SM walks a
// contiguous range of (sequence, KV head, page-tile) work; a producer warp
// gathers each tile's pages through the block table with 2-D TMA loads
// (swizzled boxes, so the consumers' row-per-thread reads are free of bank
// conflicts) into a ring of shared-memory stages; eight consumer warps own
// one token each per stage, do the G head dot products in fp32, and reduce
// the page maximum with warp shuffles.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "route_mma.cuh"
#include "select_block.cuh"
#include "step_blocks.cuh"

namespace basiskv {

namespace {

// ----------------------------------------------------------- query folding
// qt[b][h][j]       = sum_i P_K[g][j][i] q[b][h][i]          j < r_v
// qt[b][h][r_v + c] = sum_i q[b][h][i] U_K[g][i][c]           c < r_k
__global__ void __launch_bounds__(kFoldThreads) fold_query_kernel(FoldQArgs a) {
  extern __shared__ float fsm[];
  fold_query_block(a, blockIdx.x, blockIdx.y, fsm, threadIdx.x, 0);
}

// ------------------------------------------------------------ page scoring
constexpr int kRouteConsumers = 256;  // one token per consumer thread per stage
constexpr int kRouteThreads = kRouteConsumers + 32;
constexpr int kRouteConsumerWarps = kRouteConsumers / 32;

struct RouteGeom {
  int np;           // pages per stage (kRouteConsumers / S)
  int page_bytes;   // shared-memory bytes of one page slot (1 KB multiple)
  int q_off;        // offset of the folded-query slot in a stage
  int q_bytes;      // G * (r_v + r_k) * 4
  int stage_bytes;  // 1 KB multiple
  int stages;
  int wz, we;       // box widths (columns) of the z and e tensor maps
  int nzb, neb;     // boxes per page
  int zbox, ebox;   // bytes per box
  uint32_t zmask, emask;  // swizzle masks
};

__device__ __forceinline__ void decode_tile(long tile, int tiles_per_bg, int Hkv, int& bg,
                                            int& b, int& g, int& ti) {
  bg = (int)(tile / tiles_per_bg);
  ti = (int)(tile % tiles_per_bg);
  b = bg / Hkv;
  g = bg % Hkv;
}

// Walks a contiguous range of (sequence, KV head, page-tile) work without a
// division per tile: one division at the start, then increments.  The
// length of the current sequence is cached and reloaded only when the
// sequence changes.
struct TileCursor {
  int bg, b, g, ti;  // flat (sequence, KV head), sequence, KV head, tile in it
  int T, P;          // length (clamped) and pages of sequence b
  __device__ void init(long tile, int tiles_per_bg, int Hkv) {
    bg = (int)(tile / tiles_per_bg);
    ti = (int)(tile - (long)bg * tiles_per_bg);
    b = bg / Hkv;
    g = bg - b * Hkv;
    T = -1;
  }
  __device__ void next(int tiles_per_bg, int Hkv) {
    if (++ti == tiles_per_bg) {
      ti = 0;
      ++bg;
      if (++g == Hkv) {
        g = 0;
        ++b;
        T = -1;
      }
    }
  }
  // Loads the length when the sequence changed since the last call.
  __device__ void length(const int32_t* seq_lens, int len_offset, int max_seq_len, int S,
                         unsigned int* status, bool report) {
    if (T < 0) {
      T = clamp_len(seq_lens[b] + len_offset, max_seq_len, status, report);
      P = (T + S - 1) / S;
    }
  }
};

// Adds the contribution of one 8-wide chunk of a token row to the G head
// accumulators.  `xa` is the swizzled shared address of the row chunk, `qa`
// the address of the chunk in head 0's folded query; heads are rq floats
// apart.
template <int G>
__device__ __forceinline__ void chunk_fma(uint32_t xa, uint32_t qa, uint32_t qstride,
                                          float (&acc)[G][2]) {
  const uint4 w = lds128(xa);
  const float x0 = bf16lo(w.x), x1 = bf16hi(w.x), x2 = bf16lo(w.y), x3 = bf16hi(w.y);
  const float x4 = bf16lo(w.z), x5 = bf16hi(w.z), x6 = bf16lo(w.w), x7 = bf16hi(w.w);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float4 q0 = lds128f(qa + h * qstride);
    const float4 q1 = lds128f(qa + h * qstride + 16);
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

template <int G>
__global__ void __launch_bounds__(kRouteThreads, 1)
    route_kernel(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmE,
                 RouteArgs a, RouteGeom geo) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)geo.stages * geo.stage_bytes);
  uint64_t* empty = full + geo.stages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < geo.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kRouteConsumerWarps);
    }
    fence_barrier_init();
  }
  if (warp == kRouteConsumerWarps && lane == 0) {
    prefetch_tmap(&tmZ);
    prefetch_tmap(&tmE);
  }
  __syncthreads();
  pdl_wait();

  const int S = a.S, rq = a.r_v + a.r_k;
  const int P_max = (a.max_seq_len + S - 1) / S;
  const int tiles_per_bg = (P_max + geo.np - 1) / geo.np;
  const long total = (long)a.B * a.Hkv * tiles_per_bg;
  const long t_begin = total * blockIdx.x / gridDim.x;
  const long t_end = total * (blockIdx.x + 1) / gridDim.x;

  if (warp == kRouteConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      for (long tile = t_begin; tile < t_end; ++tile) {
        int bg, b, g, ti;
        decode_tile(tile, tiles_per_bg, a.Hkv, bg, b, g, ti);
        const int T = clamp_len(a.seq_lens[b] + a.len_offset, a.max_seq_len, a.status, false);
        const int P = (T + S - 1) / S, p0 = ti * geo.np;
        if (p0 >= P) continue;
        const int npg = min(geo.np, P - p0);
        const int s = it % geo.stages;
        if (!mbar_wait(&empty[s], ((it / geo.stages) & 1) ^ 1, a.status)) break;
        uint8_t* st = smem + (size_t)s * geo.stage_bytes;
        mbar_arrive_expect_tx(&full[s], geo.q_bytes + npg * S * rq * 2);
        bulk_load(st + geo.q_off, a.qt + ((size_t)b * a.Hkv * G + (size_t)g * G) * rq,
                  geo.q_bytes, &full[s]);
        const int32_t* bt = a.block_table + (size_t)b * a.max_pages + p0;
        for (int j = 0; j < npg; ++j) {
          int pp = bt[j];
          if (pp < 0 || pp >= a.num_phys) {
            raise_status(a.status, BASISKV_DEV_BAD_PAGE);
            pp = 0;  // keep the byte count; the page's score is flagged garbage
          }
          const int row = (pp * a.Hkv + g) * S;
          uint8_t* pg = st + j * geo.page_bytes;
          for (int k = 0; k < geo.nzb; ++k)
            tma_load_2d(pg + k * geo.zbox, &tmZ, k * geo.wz, row, &full[s]);
          uint8_t* pe = pg + geo.nzb * geo.zbox;
          for (int k = 0; k < geo.neb; ++k)
            tma_load_2d(pe + k * geo.ebox, &tmE, k * geo.we, row, &full[s]);
        }
        ++it;
      }
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  const int page_local = tid / S, row = tid % S;
  const uint32_t qstride = rq * 4;
  const int zc_per_box = geo.wz / 8, ec_per_box = geo.we / 8;
  const int nzc = a.r_v / 8, nec = a.r_k / 8;
  int it = 0;
  for (long tile = t_begin; tile < t_end; ++tile) {
    int bg, b, g, ti;
    decode_tile(tile, tiles_per_bg, a.Hkv, bg, b, g, ti);
    const int T = clamp_len(a.seq_lens[b] + a.len_offset, a.max_seq_len, a.status, tid == 0 && ti == 0);
    const int P = (T + S - 1) / S, p0 = ti * geo.np;
    if (p0 >= P) continue;
    const int npg = min(geo.np, P - p0);
    const int s = it % geo.stages;
    if (!mbar_wait(&full[s], (it / geo.stages) & 1, a.status)) break;
    const uint32_t st = smem_u32(smem + (size_t)s * geo.stage_bytes);
    float best = -INFINITY;
    const int p = p0 + page_local;
    if (page_local < npg && p * S + row < T) {
      float acc[G][2];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = 0.f;
      const uint32_t pgb = st + page_local * geo.page_bytes;
      const uint32_t qb = st + geo.q_off;
#pragma unroll 4
      for (int c = 0; c < nzc; ++c) {
        const int box = c / zc_per_box, cc = c - box * zc_per_box;
        const uint32_t xa = swz(pgb + box * geo.zbox + row * geo.wz * 2 + cc * 16, geo.zmask);
        chunk_fma<G>(xa, qb + c * 32, qstride, acc);
      }
      const uint32_t peb = pgb + geo.nzb * geo.zbox;
#pragma unroll 4
      for (int c = 0; c < nec; ++c) {
        const int box = c / ec_per_box, cc = c - box * ec_per_box;
        const uint32_t xa = swz(peb + box * geo.ebox + row * geo.we * 2 + cc * 16, geo.emask);
        chunk_fma<G>(xa, qb + (a.r_v + c * 8) * 4, qstride, acc);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) best = fmaxf(best, acc[h][0] + acc[h][1]);
    }
    for (int o = S >> 1; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (row == 0 && page_local < npg) a.scores[(size_t)bg * a.max_pages + p] = best;
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    ++it;
  }
}


// ----------------------------------------------- page scoring, specialised
// The same stream with the head count and the state widths fixed at compile
// time.  Each consumer thread copies its token's whole row (r_v + r_k bf16)
// from the stage into registers and releases the stage at once, so shared
// memory holds data in flight rather than data being computed on; the folded
// queries live in a per-CTA buffer that is refreshed when the (sequence, KV
// head) changes.  The G dot products use packed fp32x2 FMAs.
//
// Pipeline shape (measured on B200 at the 32K-context, B = 16 workload): one
// producer/consumer ring per CTA caps at about 29 GB/s per SM however deep
// it is, so the kernel runs three small independent rings per SM (3 CTAs of
// 4 consumer warps, 128 tokens per stage) rather than one large one; z
// boxes are 64 columns (full 128-byte rows) whenever r_v allows.
constexpr int kRsGroupThreads = 128;  // tokens per stage (4 consumer warps)
constexpr int kRsGroups = 1;
constexpr int kRsCtasPerSm = 3;
constexpr int kRsThreads = kRsGroups * kRsGroupThreads + 32;
constexpr int kRsProducerWarp = kRsGroups * kRsGroupThreads / 32;

// Box width of the z tensor map the specialised kernel expects.
__host__ __device__ constexpr int rs_z_box_cols(int r_v) { return r_v % 64 == 0 ? 64 : 32; }

struct RsGeom {
  int np;           // pages per stage
  int page_bytes;   // 1 KB multiple
  int stage_bytes;  // 1 KB multiple
  int stages;
  int q_off;        // per-group folded-query buffers, after the ring
  int bar_off;
};

template <int G, int RV, int RK>
__global__ void __launch_bounds__(kRsThreads, kRsCtasPerSm)
    route_rs_kernel(const __grid_constant__ CUtensorMap tmZ,
                    const __grid_constant__ CUtensorMap tmE, RouteArgs a, RsGeom geo) {
  constexpr int WZ = rs_z_box_cols(RV), WE = (RK % 32 == 0) ? 32 : 16;
  constexpr int NZB = RV / WZ, NEB = RK / WE;
  constexpr int NZC = RV / 8, NEC = RK / 8, NCH = NZC + NEC, RQ = RV + RK;
  constexpr uint32_t ZM = (WZ == 64) ? 7u : 3u, EM = (WE == 32) ? 3u : 1u;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.bar_off);
  uint64_t* empty = full + geo.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + geo.stages);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.S;
  const int zbox = S * WZ * 2, ebox = S * WE * 2;
  if (tid == 0) {
    for (int s = 0; s < geo.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kRsGroupThreads / 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kRsProducerWarp && lane == 0) {
    prefetch_tmap(&tmZ);
    prefetch_tmap(&tmE);
  }
  __syncthreads();
  pdl_wait();

  const int P_max = (a.max_seq_len + S - 1) / S;
  const int tiles_per_bg = (P_max + geo.np - 1) / geo.np;
  const long total = (long)a.B * a.Hkv * tiles_per_bg;
  const long t_begin = total * blockIdx.x / gridDim.x;
  const long t_end = total * (blockIdx.x + 1) / gridDim.x;

  if (warp == kRsProducerWarp) {
    // ------------------------------------------------------------ producer
    // The whole warp: lane j fetches page j's block-table entry and issues
    // that page's boxes, so a tile's gathers go out in parallel.  Entries are
    // fetched kBtAhead tiles ahead into a per-lane register ring: the table is
    // evicted from L2 by the cache stream, and one dependent round trip per
    // tile would otherwise pace the whole pipeline.
    constexpr int kBtAhead = 8;
    const int count = (int)(t_end - t_begin);
    TileCursor pre, cur;
    pre.init(t_begin, tiles_per_bg, a.Hkv);
    cur = pre;
    auto fetch = [&](int n) -> int {  // entry of tile t_begin + n, then advance
      int v = 0;
      if (n < count) {
        pre.length(a.seq_lens, a.len_offset, a.max_seq_len, S, a.status, false);
        const int p0_ = pre.ti * geo.np;
        if (lane < min(geo.np, pre.P - p0_))
          v = a.block_table[(size_t)pre.b * a.max_pages + p0_ + lane];
        pre.next(tiles_per_bg, a.Hkv);
      }
      return v;
    };
    int ring[kBtAhead];
#pragma unroll
    for (int k = 0; k < kBtAhead; ++k) ring[k] = fetch(k);
    int it = 0;
    for (int n = 0; n < count; ++n, cur.next(tiles_per_bg, a.Hkv)) {
      int pp = ring[0];
#pragma unroll
      for (int k = 0; k + 1 < kBtAhead; ++k) ring[k] = ring[k + 1];
      ring[kBtAhead - 1] = fetch(n + kBtAhead);
      cur.length(a.seq_lens, a.len_offset, a.max_seq_len, S, a.status, false);
      const int b = cur.b, g = cur.g, P = cur.P, p0 = cur.ti * geo.np;
      if (p0 >= P) continue;
      const int npg = min(geo.np, P - p0);
      const int s = it % geo.stages;
      ++it;
      bool go = true;
      if (lane == 0) {
        go = mbar_wait_or_abort(&empty[s], (((it - 1) / geo.stages) & 1) ^ 1, a.status,
                                abort_flag);
        if (go) mbar_arrive_expect_tx(&full[s], npg * S * RQ * 2);
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (!go) continue;  // aborted: issue nothing more
      if (lane < npg) {
        if (pp < 0 || pp >= a.num_phys) {
          raise_status(a.status, BASISKV_DEV_BAD_PAGE);
          pp = 0;  // keep the byte count; the page's score is flagged garbage
        }
        const int row = (pp * a.Hkv + g) * S;
        uint8_t* pg = smem + (size_t)s * geo.stage_bytes + lane * geo.page_bytes;
#pragma unroll
        for (int k = 0; k < NZB; ++k) tma_load_2d(pg + k * zbox, &tmZ, k * WZ, row, &full[s]);
#pragma unroll
        for (int k = 0; k < NEB; ++k)
          tma_load_2d(pg + NZB * zbox + k * ebox, &tmE, k * WE, row, &full[s]);
      }
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  const int group = tid / kRsGroupThreads, gtid = tid % kRsGroupThreads;
  const int page_local = gtid / S, row = gtid % S;
  float* qbuf = reinterpret_cast<float*>(smem + geo.q_off) + group * G * RQ;
  int cur_bg = -1;
  int it = 0;
  const int count = (int)(t_end - t_begin);
  TileCursor cur;
  cur.init(t_begin, tiles_per_bg, a.Hkv);
  for (int n = 0; n < count; ++n, cur.next(tiles_per_bg, a.Hkv)) {
    cur.length(a.seq_lens, a.len_offset, a.max_seq_len, S, a.status, tid == 0);
    const int bg = cur.bg, b = cur.b, g = cur.g, T = cur.T, P = cur.P;
    const int p0 = cur.ti * geo.np;
    if (p0 >= P) continue;
    const int my = it++;
    if ((my % kRsGroups) != group) continue;
    const int npg = min(geo.np, P - p0);
    if (bg != cur_bg) {  // refresh the group's folded queries (uniform control flow)
      named_bar_sync(1 + group, kRsGroupThreads);
      const float* src = a.qt + ((size_t)b * a.Hkv * G + (size_t)g * G) * RQ;
      for (int i = gtid; i < G * RQ; i += kRsGroupThreads) qbuf[i] = src[i];
      named_bar_sync(1 + group, kRsGroupThreads);
      cur_bg = bg;
    }
    const int s = my % geo.stages;
    const bool ready = mbar_wait_or_abort(&full[s], (my / geo.stages) & 1, a.status, abort_flag);
    const int p = p0 + page_local;
    const bool valid = ready && page_local < npg && p * S + row < T;
    uint4 x[NCH];
    if (valid) {
      const uint8_t* pg = smem + (size_t)s * geo.stage_bytes + page_local * geo.page_bytes;
#pragma unroll
      for (int c = 0; c < NZC; ++c) {
        const uint32_t off = (c / (WZ / 8)) * zbox + row * (WZ * 2) + (c % (WZ / 8)) * 16;
        x[c] = *reinterpret_cast<const uint4*>(pg + swz(off, ZM));
      }
#pragma unroll
      for (int c = 0; c < NEC; ++c) {
        const uint32_t off =
            NZB * zbox + (c / (WE / 8)) * ebox + row * (WE * 2) + (c % (WE / 8)) * 16;
        x[NZC + c] = *reinterpret_cast<const uint4*>(pg + swz(off, EM));
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // the rows are in registers now
    float best = -INFINITY;
    if (valid) {
      float2 acc[G][2];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const float2 p0v = bf16x2_to_f2(x[c].x), p1v = bf16x2_to_f2(x[c].y);
        const float2 p2v = bf16x2_to_f2(x[c].z), p3v = bf16x2_to_f2(x[c].w);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 qa = *reinterpret_cast<const float4*>(qbuf + h * RQ + c * 8);
          const float4 qb = *reinterpret_cast<const float4*>(qbuf + h * RQ + c * 8 + 4);
          ffma2(acc[h][0], p0v, make_float2(qa.x, qa.y));
          ffma2(acc[h][1], p1v, make_float2(qa.z, qa.w));
          ffma2(acc[h][0], p2v, make_float2(qb.x, qb.y));
          ffma2(acc[h][1], p3v, make_float2(qb.z, qb.w));
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
        best = fmaxf(best, (acc[h][0].x + acc[h][1].x) + (acc[h][0].y + acc[h][1].y));
    }
    for (int o = S >> 1; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (ready && row == 0 && page_local < npg) a.scores[(size_t)bg * a.max_pages + p] = best;
  }
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelShared ss;
  pdl_wait();
  int* tbl = reinterpret_cast<int*>(keys + (a.max_seq_len + a.S - 1) / a.S);
  select_group<kSelThreads>(a, blockIdx.x, keys, tbl, ss, a.sel + (size_t)blockIdx.x * a.top_k,
                            a.sel_phys ? a.sel_phys + (size_t)blockIdx.x * a.top_k : nullptr);
}

RouteGeom route_geometry(int G, int r_v, int r_k, int S, int wz, int we) {
  RouteGeom g{};
  g.np = kRouteConsumers / S;
  g.wz = wz;
  g.we = we;
  g.nzb = r_v / wz;
  g.neb = r_k / we;
  g.zbox = S * wz * 2;
  g.ebox = S * we * 2;
  g.zmask = wz == 64 ? 7u : (wz == 32 ? 3u : 1u);
  g.emask = we == 64 ? 7u : (we == 32 ? 3u : 1u);
  g.page_bytes = ((S * (r_v + r_k) * 2) + 1023) / 1024 * 1024;
  g.q_off = g.np * g.page_bytes;
  g.q_bytes = G * (r_v + r_k) * 4;
  g.stage_bytes = (g.q_off + g.q_bytes + 1023) / 1024 * 1024;
  const int budget = 220 * 1024;
  g.stages = budget / g.stage_bytes;
  if (g.stages > 8) g.stages = 8;
  return g;
}

template <int G>
cudaError_t launch_route_g(const RouteArgs& a, const CUtensorMap& tmZ, const CUtensorMap& tmE,
                           const RouteGeom& geo, cudaStream_t st, bool pdl) {
  const size_t smem = (size_t)geo.stages * geo.stage_bytes + 2 * geo.stages * 8 + 1024;
  cudaError_t e = cudaFuncSetAttribute(route_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int P_max = (a.max_seq_len + a.S - 1) / a.S;
  const long tiles = (long)a.B * a.Hkv * ((P_max + geo.np - 1) / geo.np);
  long grid = num_sms();
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  return launch_k(route_kernel<G>, dim3((unsigned)grid), dim3(kRouteThreads), smem, st, pdl,
                  tmZ, tmE, a, geo);
}

template <int G, int RV, int RK>
cudaError_t launch_route_rs(const RouteArgs& a, const CUtensorMap& tmZ, const CUtensorMap& tmE,
                            cudaStream_t st, bool pdl) {
  RsGeom geo{};
  geo.np = kRsGroupThreads / a.S;
  geo.page_bytes = (a.S * (RV + RK) * 2 + 1023) / 1024 * 1024;
  geo.stage_bytes = geo.np * geo.page_bytes;
  const int qbytes = kRsGroups * G * (RV + RK) * 4;
  // 228 KB of shared memory per SM, 1 KB of it reserved per CTA; 1 KB of
  // slack for the 1024-byte alignment of the base.
  const int budget = 228 * 1024 / kRsCtasPerSm - 1024 - 1024 - qbytes - 256;
  geo.stages = budget / geo.stage_bytes;
  if (geo.stages > 8) geo.stages = 8;
  if (geo.stages < 2) return cudaErrorInvalidConfiguration;
  geo.q_off = geo.stages * geo.stage_bytes;
  geo.bar_off = geo.q_off + qbytes;
  const size_t smem = (size_t)geo.bar_off + 2 * geo.stages * 8 + 16 + 1024;
  cudaError_t e = cudaFuncSetAttribute(route_rs_kernel<G, RV, RK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int P_max = (a.max_seq_len + a.S - 1) / a.S;
  const long tiles = (long)a.B * a.Hkv * ((P_max + geo.np - 1) / geo.np);
  long grid = (long)num_sms() * kRsCtasPerSm;
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  return launch_k(route_rs_kernel<G, RV, RK>, dim3((unsigned)grid), dim3(kRsThreads), smem, st,
                  pdl, tmZ, tmE, a, geo);
}

// Narrow routers with an instance: (G, S) in {(4, 16), (8, 32)}, r_k 32,
// r_v in {64, 96}, widths 16 or 32 each.
// The full-width routers with a plain-load scoring instance (G, r_v, r_k, S).
#define BKV_RM_FULL(X) \
  X(4, 32, 32, 16)     \
  X(4, 32, 32, 32)     \
  X(8, 32, 32, 16)     \
  X(8, 32, 32, 32)     \
  X(4, 64, 32, 16)     \
  X(4, 96, 32, 16)     \
  X(4, 128, 32, 16)    \
  X(4, 64, 32, 32)     \
  X(4, 96, 32, 32)     \
  X(8, 64, 32, 16)     \
  X(8, 96, 32, 16)     \
  X(8, 128, 32, 16)    \
  X(8, 64, 32, 32)     \
  X(8, 96, 32, 32)     \
  X(8, 128, 32, 32)

#define BKV_RM_NARROW(X)                                                            \
  X(4, 64, 32, 16, 16, 16) X(4, 64, 32, 16, 32, 16) X(4, 64, 32, 32, 16, 16)        \
  X(4, 64, 32, 32, 32, 16) X(4, 96, 32, 16, 16, 16) X(4, 96, 32, 16, 32, 16)        \
  X(4, 96, 32, 32, 16, 16) X(4, 96, 32, 32, 32, 16) X(8, 64, 32, 16, 16, 32)        \
  X(8, 64, 32, 16, 32, 32) X(8, 64, 32, 32, 16, 32) X(8, 64, 32, 32, 32, 32)        \
  X(8, 96, 32, 16, 16, 32) X(8, 96, 32, 16, 32, 32) X(8, 96, 32, 32, 16, 32)        \
  X(8, 96, 32, 32, 32, 32)

}  // namespace

bool route_narrow_supported(int G, int r_v, int r_k, int rb, int rq, int S) {
#define BKV_RMQ(GG, V, K, RB_, RQ_, SS) \
  if (G == GG && r_v == V && r_k == K && rb == RB_ && rq == RQ_ && S == SS) return true;
  BKV_RM_NARROW(BKV_RMQ)
#undef BKV_RMQ
  return false;
}

cudaError_t launch_fold_query(const FoldQArgs& a, cudaStream_t st, bool pdl) {
  const int G = a.Hq / a.Hkv;
  const size_t smem = fold_block_smem(G, a.d);
  dim3 grid(a.B * a.Hkv, (a.r_v + a.r_k + 31) / 32);
  return launch_k(fold_query_kernel, grid, dim3(kFoldThreads), smem, st, pdl, a);
}

// Routers with routing pages smaller than the cache page (G, r_v, r_k, rb,
// rq, S, rp): the pages' B16R16 router and the full-width router at the
// Llama-3.1-8B (page 16) and Qwen3-32B (page 32) shapes.
#define BKV_RM_SUBPAGE(X)                                                             \
  X(4, 64, 32, 16, 16, 16, 4) X(4, 64, 32, 16, 16, 16, 8) X(4, 96, 32, 16, 16, 16, 4) \
  X(4, 64, 32, 64, 32, 16, 4) X(4, 96, 32, 96, 32, 16, 4) X(8, 96, 32, 16, 16, 32, 4) \
  X(8, 96, 32, 96, 32, 32, 4)

bool route_subpage_supported(int G, int r_v, int r_k, int rb, int rq, int S, int rp) {
#define BKV_RMP(GG, V, K, RB_, RQ_, SS, RP_) \
  if (G == GG && r_v == V && r_k == K && rb == RB_ && rq == RQ_ && S == SS && rp == RP_) return true;
  BKV_RM_SUBPAGE(BKV_RMP)
#undef BKV_RMP
  return false;
}

cudaError_t launch_route_scores(const RouteArgs& a, const CUtensorMap& tmZ,
                                const CUtensorMap& tmE, int wz, int we, cudaStream_t st,
                                bool pdl) {
  if (a.rp && a.rp != a.S) {  // routing pages smaller than the cache page
    if (a.fp8) return launch_route_scores_fp8(a, st, pdl);
    if (!(a.Z && a.E)) return cudaErrorNotSupported;
#define BKV_RMP(GG, V, K, RB_, RQ_, SS, RP_)                                              \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.rb == RB_ && a.rq == RQ_ && a.S == SS && \
      a.rp == RP_)                                                                       \
    return launch_route_mma<GG, V, K, RB_, RQ_, SS, RP_>(a, st, pdl);
    BKV_RM_SUBPAGE(BKV_RMP)
#undef BKV_RMP
    return cudaErrorNotSupported;
  }
  if (a.fp8) return launch_route_scores_fp8(a, st, pdl);
  if ((a.rb != a.r_v || a.rq != a.r_k) && !(a.Z && a.E)) return cudaErrorNotSupported;
  if (a.Z && a.E) {
    if (a.rb != a.r_v || a.rq != a.r_k) {  // a narrow router
#define BKV_RMN(GG, V, K, RB_, RQ_, SS)                                                    \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.rb == RB_ && a.rq == RQ_ && a.S == SS) \
    return launch_route_mma<GG, V, K, RB_, RQ_, SS>(a, st, pdl);
      BKV_RM_NARROW(BKV_RMN)
#undef BKV_RMN
      return cudaErrorNotSupported;
    }
#define BKV_RM(GG, V, K, SS)                                     \
  if (a.G == GG && a.r_v == V && a.r_k == K && a.S == SS) \
    return launch_route_mma<GG, V, K, V, K, SS>(a, st, pdl);
    BKV_RM_FULL(BKV_RM)
#undef BKV_RM
  }
  if (wz == rs_z_box_cols(a.r_v) && we == (a.r_k % 32 == 0 ? 32 : 16)) {
#define BKV_RS(GG, V, K) \
  if (a.G == GG && a.r_v == V && a.r_k == K) return launch_route_rs<GG, V, K>(a, tmZ, tmE, st, pdl);
    BKV_RS(4, 32, 16)
    BKV_RS(4, 64, 32)
    BKV_RS(4, 96, 32)
    BKV_RS(4, 128, 32)
    BKV_RS(8, 64, 32)
    BKV_RS(8, 96, 32)
    BKV_RS(8, 128, 32)
#undef BKV_RS
  }
  const RouteGeom geo = route_geometry(a.G, a.r_v, a.r_k, a.S, wz, we);
  if (geo.stages < 2) return cudaErrorInvalidConfiguration;
  switch (a.G) {
    case 1: return launch_route_g<1>(a, tmZ, tmE, geo, st, pdl);
    case 2: return launch_route_g<2>(a, tmZ, tmE, geo, st, pdl);
    case 4: return launch_route_g<4>(a, tmZ, tmE, geo, st, pdl);
    case 8: return launch_route_g<8>(a, tmZ, tmE, geo, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

namespace {
// Selection blocks [0, B*Hkv) and, after them, one block per (sequence, KV
// head) that appends the step's token (its first 128 threads; the append's
// result is first read by the attention kernel, so it runs in the shadow of
// the selection instead of before the scoring).
__global__ void __launch_bounds__(kSelThreads)
    select_append_kernel(SelectArgs s, AppendArgs a) {
  extern __shared__ __align__(16) uint8_t sa_dyn[];
  __shared__ SelShared ss;
  __shared__ float vs[kAppendThreads], ks[kAppendThreads], zs[kAppendThreads],
      rs[kAppendThreads];
  const int nsel = s.B * s.Hkv;
  pdl_launch_dependents();  // one wave: the attention CTAs may take the free SMs
  if ((int)blockIdx.x < nsel) {
    pdl_wait();
    uint32_t* keys = reinterpret_cast<uint32_t*>(sa_dyn);
    select_group<kSelThreads>(s, blockIdx.x, keys,
                              reinterpret_cast<int*>(keys + (s.max_seq_len + s.S - 1) / s.S), ss,
                              s.sel + (size_t)blockIdx.x * s.top_k,
                              s.sel_phys ? s.sel_phys + (size_t)blockIdx.x * s.top_k : nullptr);
  } else if (threadIdx.x < kAppendThreads) {
    const int r = blockIdx.x - nsel;  // (sequence, KV head)
    append_block(a, r % a.Hkv, 0, r / a.Hkv, reinterpret_cast<uint16_t*>(sa_dyn), vs, ks, zs, rs,
                 threadIdx.x, 1);
  }
}
}  // namespace

cudaError_t launch_select_append(const SelectArgs& s, const AppendArgs& a, cudaStream_t st,
                                 bool pdl) {
  const int P_max = (s.max_seq_len + s.S - 1) / s.S;
  size_t smem = (size_t)(P_max > 2 ? P_max : 2) * sizeof(uint32_t) * (s.sel_phys ? 2 : 1);
  const size_t app = append_block_smem(a.d, a.r_v, a.r_k);
  if (app > smem) smem = app;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_append_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(select_append_kernel, dim3(2 * s.B * s.Hkv), dim3(kSelThreads), smem, st, pdl,
                  s, a);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t st, bool pdl) {
  const int P_max = (a.max_seq_len + a.S - 1) / a.S;
  const size_t smem = (size_t)(P_max > 2 ? P_max : 2) * sizeof(uint32_t) * (a.sel_phys ? 2 : 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_k(select_kernel, dim3(a.B * a.Hkv), dim3(kSelThreads), smem, st, pdl, a);
}

}  // namespace basiskv
