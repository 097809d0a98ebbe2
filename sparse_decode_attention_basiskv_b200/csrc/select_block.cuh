// Exact top-k page selection of one (sequence, KV head) by a block of
// threads (the separate selection launch in route.cu and the fused
// selection + attention kernel in select_attend.cuh share it).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace basiskv {
namespace {

// -------------------------------------------------------- page selection
// Per (sequence, KV head): the first n_sink and the last n_recent pages
// always (by default the sink page 0 and the newest page P-1); the other
// slots go to the best remaining pages by (score desc, index asc),
// found exactly with an MSB-first radix select over order-preserving 32-bit
// keys; ties at the threshold are taken in index order.  Output ascending.
constexpr int kSelThreads = 512;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;  // -0 ranks as +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Bins of the value histogram and members of the threshold bin that are
// ranked one by one (more members: the radix select decides).
constexpr int kSelBins = 2048;
constexpr int kSelMembers = 256;

struct SelShared {
  int hist[2][256];  // radix histograms, alternating between passes
  int sh[32];        // scan scratch
  uint32_t digit;
  int rem;
  int done;  // the chosen bucket is taken whole: later digits are not needed
  int bins[kSelBins];       // value histogram
  uint32_t wmin[32], wmax[32];  // per-warp key extremes
  int memb[kSelMembers];    // candidates in the threshold bin
  int nmemb, tb, above, radix;
  uint32_t thr;
};

// The float whose order_key is k (-0 never occurs: it was mapped to +0).
__device__ __forceinline__ float key_value(uint32_t k) {
  return (k & 0x80000000u) ? __uint_as_float(k & 0x7fffffffu) : __uint_as_float(~k);
}

// Histogram bin of key k: the score's position between the extremes,
// scaled to [0, kSelBins) (monotone in the score, so a higher bin holds only
// higher scores).
__device__ __forceinline__ int value_bin(uint32_t k, float vmin, float scale) {
  // explicit roundings: both uses of a key give the same bin
  const int b = (int)__fmul_rn(__fsub_rn(key_value(k), vmin), scale);
  return b < 0 ? 0 : (b >= kSelBins ? kSelBins - 1 : b);
}

// Exclusive prefix sum over a block of NT threads; *total receives the sum.
// One barrier: each thread adds up the warp totals before its own warp
// itself (at most 15 shared reads).  sh must not be written again until the
// block has met at another barrier.
template <int NT>
__device__ int block_excl_scan(int v, int* sh, int* total) {
  constexpr int W = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const int t = sh[w];
    before += w < warp ? t : 0;
    all += t;
  }
  *total = all;
  return before + x - v;
}

// Selection of one (sequence, KV head) by a block of NT threads.  keys and
// tbl: shared arrays of at least ceil(max_seq_len / S) entries.
// The ascending selection goes to out[0, top_k) (global or shared memory)
// and, when outp is set, the physical page of each entry to outp (tbl then
// holds the block-table row; unused otherwise).
template <int NT>
__device__ __forceinline__ void select_group(const SelectArgs& a, int bg, uint32_t* keys, int* tbl,
                                          SelShared& ss, int32_t* out, int32_t* outp) {
  const int b = bg / a.Hkv, tid = threadIdx.x;
  const int P_max = (a.max_seq_len + a.S - 1) / a.S;
  const int32_t* bt = a.block_table + (size_t)b * a.max_pages;
  const int ns = a.n_sink, nr = a.n_recent;  // forced leading / trailing pages
  // candidate i = page ns + i (routing pages when spp > 1)
  const float* sc = a.scores + (size_t)bg * a.max_pages * (a.spp > 1 ? a.spp : 1) + ns;
  // The length, the first batch of scores and the block-table row are
  // requested together (up to the longest possible context; what lies past
  // this sequence's pages is dropped): one memory round trip, not two.
  int T = a.seq_lens[b] + a.len_offset;
  float v[8];
  int t[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = u * NT + tid;
    v[u] = i < P_max - ns ? __ldcg(sc + i) : 0.f;
    t[u] = (outp && i < P_max) ? bt[i] : 0;
  }
  T = T < 0 ? 0 : (T > a.max_seq_len ? a.max_seq_len : T);
  const int P = (T + a.S - 1) / a.S;
  if (a.top_k >= P) {
    for (int i = tid; i < a.top_k; i += NT) {
      out[i] = i < P ? i : -1;
      if (outp) outp[i] = i < P ? bt[i] : -1;
    }
    return;
  }
  const int n = P - ns - nr, need = a.top_k - ns - nr;  // n >= 1: P > top_k >= ns + nr
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int base = 0; base < P; base += 8 * NT) {  // batches of eight loads a thread
    if (base > 0) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * NT + tid;
        v[u] = i < n ? __ldcg(sc + i) : 0.f;
        t[u] = (outp && i < P) ? bt[i] : 0;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * NT + tid;
      if (i < n) {
        const uint32_t k = order_key(v[u]);
        keys[i] = k;
        kmin = k < kmin ? k : kmin;
        kmax = k > kmax ? k : kmax;
      }
      if (outp && i < P) tbl[i] = t[u];
    }
  }
  for (int i = tid; i < 512; i += NT) (&ss.hist[0][0])[i] = 0;
  for (int i = tid; i < kSelBins; i += NT) ss.bins[i] = 0;
  {
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t a0 = __shfl_xor_sync(0xffffffffu, kmin, o);
      const uint32_t a1 = __shfl_xor_sync(0xffffffffu, kmax, o);
      kmin = a0 < kmin ? a0 : kmin;
      kmax = a1 > kmax ? a1 : kmax;
    }
    if (lane == 0) {
      ss.wmin[warp] = kmin;
      ss.wmax[warp] = kmax;
    }
    if (tid == 0) ss.nmemb = 0;
  }
  __syncthreads();

  // The threshold (the need-th largest key) from a histogram of the scores'
  // values: 2048 bins between the extremes spread the keys thinly (few
  // atomics on one address), the bin holding the threshold is found by one
  // scan, and its few members are ranked one by one.  When that bin holds
  // more than kSelMembers keys (many equal or nearly equal scores) or the
  // extremes give no usable scale, the MSB-first radix select below decides.
  uint32_t thr = 0;
  int rem = need;
  if (need > 0) {
    for (int w = 0; w < NT / 32; ++w) {
      kmin = ss.wmin[w] < kmin ? ss.wmin[w] : kmin;
      kmax = ss.wmax[w] > kmax ? ss.wmax[w] : kmax;
    }
    const float vmin = key_value(kmin), span = key_value(kmax) - vmin;
    const float scale = (float)kSelBins / span;
    const bool usable = span > 0.f && span < INFINITY && scale < INFINITY;
    if (usable) {
      for (int i = tid; i < n; i += NT) atomicAdd(&ss.bins[value_bin(keys[i], vmin, scale)], 1);
    }
    __syncthreads();
    if (usable) {
      // thread t holds bins kSelBins - BPT (t + 1) .. kSelBins - BPT t - 1, high to low
      constexpr int BPT = kSelBins / NT;
      int local = 0;
#pragma unroll
      for (int j = 0; j < BPT; ++j) local += ss.bins[kSelBins - 1 - BPT * tid - j];
      int total;
      const int before = block_excl_scan<NT>(local, ss.sh, &total);
      if (before < need && before + local >= need) {  // the threshold's bin is here
        int acc = before;
        for (int j = 0; j < BPT; ++j) {
          const int bin = kSelBins - 1 - BPT * tid - j;
          const int c = ss.bins[bin];
          if (acc + c >= need) {
            ss.tb = bin;
            ss.above = acc;
            break;
          }
          acc += c;
        }
      }
      __syncthreads();
      const int tb = ss.tb;
      for (int i = tid; i < n; i += NT)
        if (value_bin(keys[i], vmin, scale) == tb) {
          const int slot = atomicAdd(&ss.nmemb, 1);
          if (slot < kSelMembers) ss.memb[slot] = i;
        }
      __syncthreads();
      const int m = ss.nmemb;
      if (m <= kSelMembers) {
        // rank of member j by (score desc, page asc); the one at rank
        // need - above - 1 is the threshold key
        const int r_need = need - ss.above - 1;
        for (int j = tid; j < m; j += NT) {
          const int ij = ss.memb[j];
          const uint32_t kj = keys[ij];
          int gt = 0, eq_before = 0;
          for (int q = 0; q < m; ++q) {
            const uint32_t kq = keys[ss.memb[q]];
            gt += kq > kj;
            eq_before += kq == kj && ss.memb[q] < ij;
          }
          if (gt + eq_before == r_need) {
            ss.thr = kj;
            ss.rem = need - ss.above - gt;  // keys equal to the threshold to take
          }
        }
      }
      if (tid == 0) ss.radix = m > kSelMembers;
    } else if (tid == 0) {
      ss.radix = 1;
    }
    __syncthreads();
  }
  const bool radix = need > 0 && ss.radix;
  if (!radix && need > 0) {
    thr = ss.thr;
    rem = ss.rem;
  }

  // MSB-first radix select of the need-th largest key: two barriers a pass
  // (the scanning warp clears the other histogram for the next pass).
  uint32_t prefix = 0, pmask = 0;
  if (radix) {
    int cur = 0;
    for (int shift = 24; shift >= 0; shift -= 8, cur ^= 1) {
      int* hist = ss.hist[cur];
      // The leading digits of one context's scores are mostly the same (sign
      // and exponent): lanes sharing lane 0's digit add through one atomic,
      // the others individually, so same-address atomics do not serialise.
      for (int base = 0; base < n; base += NT) {
        const int i = base + tid;
        int bin = -1;
        if (i < n) {
          const uint32_t k = keys[i];
          if ((k & pmask) == prefix) bin = (int)((k >> shift) & 255);
        }
        const int b0 = __shfl_sync(0xffffffffu, bin, 0);
        const unsigned same = __ballot_sync(0xffffffffu, bin == b0);
        if (bin >= 0) {
          if (bin != b0)
            atomicAdd(&hist[bin], 1);
          else if ((tid & 31) == __ffs(same) - 1)
            atomicAdd(&hist[bin], __popc(same));
        }
      }
      __syncthreads();
      if (tid < 32) {  // lane l covers digits 255-8l .. 248-8l, high to low
        int local = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) local += hist[255 - 8 * tid - j];
        int cum = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, cum, o);
          if (tid >= o) cum += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, cum >= rem);
        const int L = __ffs(hit) - 1;
        if (tid == L) {
          int start = cum - local;
          for (int j = 0; j < 8; ++j) {
            const int dg = 255 - 8 * L - j;
            if (start + hist[dg] >= rem) {
              ss.digit = (uint32_t)dg;
              ss.rem = rem - start;
              ss.done = hist[dg] == rem - start;
              break;
            }
            start += hist[dg];
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) ss.hist[cur ^ 1][8 * tid + j] = 0;
      }
      __syncthreads();
      prefix |= ss.digit << shift;
      pmask |= 0xffu << shift;
      rem = ss.rem;
      // Every key of the bucket is taken: with the remaining digits zero the
      // threshold is at or below all of them, so the keys above it plus all
      // keys equal to it are exactly the bucket and everything above.
      if (ss.done) {
        rem = n;
        break;
      }
    }
  }
  if (radix) thr = prefix;
  // Contiguous candidate chunk per thread, so prefix sums follow index order.
  // One scan of packed counts (keys above the threshold << 16 | keys equal to
  // it): the first `rem` equal keys in index order are taken.
  const int E = (n + NT - 1) / NT;
  const int i0 = min(tid * E, n), i1 = min(i0 + E, n);
  int n_gt = 0, n_eq = 0;
  if (need > 0)
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = keys[i];
      n_gt += k > thr;
      n_eq += k == thr;
    }
  int total;
  const int before = block_excl_scan<NT>((n_gt << 16) | n_eq, ss.sh, &total);
  if (need > 0) {
    int r = before & 0xffff;
    int pos = ns + (before >> 16) + min(r, rem);
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = keys[i];
      if ((k > thr) || (k == thr && r < rem)) {
        if (outp) outp[pos] = tbl[i + ns];
        out[pos++] = i + ns;
      }
      r += k == thr;
    }
  }
  for (int i = tid; i < ns + nr; i += NT) {  // the forced pages, first and last
    const int slot = i < ns ? i : a.top_k - nr + (i - ns);
    const int page = i < ns ? i : P - nr + (i - ns);
    out[slot] = page;
    if (outp) outp[slot] = tbl[page];
  }
}

}  // namespace
}  // namespace basiskv
