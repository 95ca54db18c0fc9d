// Top-k over long score rows (decode: one query against every visible
// compressed entry, up to 786,432 of them), spread over many CTAs.
// ("Paper Breakdown: DeepSeek-V4", section 4, DSA on Compressed KV: the top-k
// entries by I_{t,s}; "How DeepSeek-V4 architecture and training work
// together": 1,024 entries per query.)
//
//   1. histogram:   a 2048-bin histogram per row of the top 11 bits of the
//                   order-preserving key, either built by the tensor-core
//                   decode indexer while it writes the scores, or by
//                   topk_hist_kernel (each CTA a slice, merged by atomics).
//   2. topk_select: every CTA finds the row's threshold bin T (fewer than k
//                   keys above it, at least k from it up) and routes its slice:
//                   bins above T are taken, bin T keys become candidates.  The
//                   last CTA of a row to finish (atomic count after a fence)
//                   then selects exactly: radix select of the remaining count
//                   among the candidates (21 low bits), then the selected set
//                   in a bitmap of the row, read out in ascending index order
//                   (one block prefix sum over per-thread word ranges); when
//                   more keys tie at the threshold than are still to take, the
//                   lowest-index ones through a bitmap scan in index order.
#pragma once
#include <limits.h>
#include "topk.cuh"

namespace csahca {

constexpr int kHistBins = 2048;            // top 11 bits of the key
// per-row counters of the multi-CTA top-k scratch
constexpr int kTopkCounters = 8;
constexpr int kCntAbove = 0;               // keys routed to the taken list
constexpr int kCntCand = 1;                // keys routed to the candidate list
constexpr int kCntSlices = 2;              // select CTAs done with the row
constexpr int kCntItems = 3;               // indexer work items done with the row
constexpr int kCntT = 4;                   // threshold bin (set by the indexer's last item; unrouted rows)
constexpr int kCntAboveT = 5;              // keys in bins above it
constexpr int kHistShift = 21;
constexpr int kTopkLargeMaxN = 786432;     // two bitmaps of N bits in shared memory

struct TopkLargeParams {
  const float* scores; int64_t row_stride;
  const int* q_pos;
  int* idx;
  int rows, N, m, k;
  int entry_base;                          // local row j is global entry entry_base + j
  int slices;                              // CTAs per row in passes 1 and 2
  // workspace (per row)
  uint32_t* hist;                          // [rows][kHistBins]
  uint32_t* counters;                      // [rows][kTopkCounters]: see kCnt* below
  int thresh_ready;                        // the indexer stored T and n_above_T in the counters
  int sorted;                              // 1: each row's indices in ascending order; 0: any order
  int* above;                              // [rows][k]
  uint2* cand;                             // [rows][N]: (key, index)
  // optional: row j of sequence `row` of a [rows][N] table of prefetch_row_bytes
  // rows is prefetched into L2 for every selected j (decode: the KV rows the
  // attention kernel gathers next)
  const char* prefetch_base;
  int64_t prefetch_row_bytes;
};

__device__ __forceinline__ int topk_visible(const TopkLargeParams& p, int row) {
  return visible_count(p.q_pos[row], p.m, p.N, p.entry_base);
}

// Zeroes n16 16-byte words of top-k scratch (histograms and counters).  A
// kernel rather than a memset node, so that the stream's chain of
// programmatic dependent launches is not broken; it writes only after the
// previous kernel has completed.
__global__ void __launch_bounds__(256) zero16_kernel(uint4* p, int64_t n16) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(512) topk_hist_kernel(TopkLargeParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ uint32_t h[kHistBins];
  const int row = blockIdx.x / p.slices, slice = blockIdx.x % p.slices;
  const int v = topk_visible(p, row);
  if (v <= p.k) return;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int per = (v + p.slices - 1) / p.slices;
  const int j0 = slice * per, j1 = min(v, j0 + per);
  const float* s = p.scores + (int64_t)row * p.row_stride;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) atomicAdd(&h[order_key(s[j]) >> kHistShift], 1u);
  __syncthreads();
  uint32_t* g = p.hist + (int64_t)row * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

// Threshold bin of a row from its histogram (block-wide, 512 threads):
// returns T and writes the number of keys in bins above T to *above.
__device__ __forceinline__ int threshold_bin(const uint32_t* g, int k, uint32_t* sh, uint32_t* above) {
  // sh[0..kHistBins): suffix sums from the top, computed per 4-bin group then scanned
  const int tid = threadIdx.x;                 // 512 threads, 4 bins each
  uint32_t c[4], tot = 0;
#pragma unroll
  for (int e = 3; e >= 0; --e) { c[e] = g[tid * 4 + e]; tot += c[e]; }
  sh[tid] = tot;
  __syncthreads();
  // inclusive suffix scan of the 512 group totals (Hillis-Steele, in place with a second buffer)
  uint32_t* a = sh;
  uint32_t* b = sh + 512;
  for (int off = 1; off < 512; off <<= 1) {
    const uint32_t x = a[tid] + (tid + off < 512 ? a[tid + off] : 0u);
    b[tid] = x;
    __syncthreads();
    uint32_t* t = a; a = b; b = t;
  }
  // a[tid] = keys in groups tid .. 511 ; keys strictly above group tid = a[tid] - tot
  __shared__ int sh_T;
  __shared__ uint32_t sh_above;
  uint32_t run = a[tid] - tot;                 // keys above this group's top bin
  if (run < (uint32_t)k && run + tot >= (uint32_t)k) {
#pragma unroll
    for (int e = 3; e >= 0; --e) {
      if (run + c[e] >= (uint32_t)k) { sh_T = tid * 4 + e; sh_above = run; break; }
      run += c[e];
    }
  }
  __syncthreads();
  *above = sh_above;
  return sh_T;
}

// Index-ordered scan of a bitmap of `words` 32-bit words: calls out(i) for the
// set bits in ascending order, at most `limit` of them; returns how many.
// blockDim.x a multiple of 32 (<= 1024); warp_buf holds at least 65 ints.
template <typename F>
__device__ __forceinline__ int bitmap_scan(const uint32_t* bm, int words, int limit, int* warp_buf, F out) {
  int done = 0;
  for (int base = 0; base < words; base += blockDim.x) {
    const int wi = base + threadIdx.x;
    const uint32_t wv = wi < words ? bm[wi] : 0u;
    // exclusive prefix of popcounts over the block
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int c = __popc(wv), incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_buf[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int x = lane < (int)(blockDim.x >> 5) ? warp_buf[lane] : 0;
      int wincl = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wincl, o);
        if (lane >= o) wincl += y;
      }
      warp_buf[32 + lane] = wincl - x;
      if (lane == 31) warp_buf[64] = wincl;
    }
    __syncthreads();
    int pos = done + warp_buf[32 + wid] + incl - c;
    const int total = warp_buf[64];
    uint32_t bits = wv;
    while (bits && pos < limit) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      out(pos, wi * 32 + b);
      ++pos;
    }
    done += total;
    __syncthreads();
    if (done >= limit) break;
  }
  return done < limit ? done : limit;
}

constexpr int kTopkSelectThreads = 512;
constexpr int kTopkCandCache = 4096;       // candidates staged in shared memory (8 bytes each)
constexpr int kTopkFinishBins = 2048;      // first radix digit of the finish: bits 20..10
constexpr int kTopkSortMax = 1024;         // k up to this: the selection is sorted, not bitmapped

// Dynamic shared memory of topk_select_kernel: the candidate cache, the
// finish histogram and a region for the sorted selection or the v-bit
// bitmap; the tie path reuses all of it as two bitmaps.
__host__ __device__ __forceinline__ int topk_select_smem_bytes(int N) {
  const int words = (N + 31) / 32;
  const int ties = 2 * words * 4;
  const int common = kTopkCandCache * 8 + kTopkFinishBins * 4 + (words > kTopkSortMax ? words : kTopkSortMax) * 4;
  return ties > common ? ties : common;
}

// Largest digit d of an nb-bin histogram (nb = 2 or 4 x blockDim) with
// count(digits > d) < need <= count(digits >= d); one thread writes d and
// need - count(digits > d).  Thread t sums bins [nb - per (t + 1), nb - per t),
// and one block prefix sum places the crossing.  Every thread calls it.
__device__ __forceinline__ void find_digit_block(const uint32_t* hist, int nb, uint32_t need, int* warp_buf,
                                                 uint32_t* out_digit, uint32_t* out_need) {
  const int per = nb / (int)blockDim.x;
  const int hi = nb - (int)threadIdx.x * per;
  uint32_t local = 0;
  for (int e = 0; e < per; ++e) local += hist[hi - 1 - e];
  int tot;
  const uint32_t above = (uint32_t)block_excl_count((int)local, warp_buf, &tot);
  if (above < need && above + local >= need) {
    uint32_t cum = above;
    for (int e = 0; e < per; ++e) {
      const int b = hi - 1 - e;
      if (cum + hist[b] >= need) { *out_digit = (uint32_t)b; *out_need = need - cum; break; }
      cum += hist[b];
    }
  }
}

// Ascending bitonic sort of a[0, 1024) by a block of 512 threads.  Thread
// (warp w, lane l) holds elements p0 = 64 w + l and p1 = p0 + 32 in
// registers: strides below 32 are warp shuffles, stride 32 pairs a thread's
// own two elements, and only the ten steps with stride >= 64 go through
// shared memory.
__device__ __forceinline__ int bitonic_cmpx(int mine, int other, int p, int s, int size) {
  const bool lower = (p & s) == 0, asc = (p & size) == 0;
  return lower == asc ? min(mine, other) : max(mine, other);
}
__device__ __forceinline__ void sort1024_block(int* a) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int p0 = 64 * w + lane, p1 = p0 + 32;
  int e0 = a[p0], e1 = a[p1];
  for (int size = 2; size <= 1024; size <<= 1) {
    for (int s = size >> 1; s > 0; s >>= 1) {
      if (s >= 64) {
        __syncthreads();
        a[p0] = e0;
        a[p1] = e1;
        __syncthreads();
        const int o0 = a[p0 ^ s], o1 = a[p1 ^ s];
        e0 = bitonic_cmpx(e0, o0, p0, s, size);
        e1 = bitonic_cmpx(e1, o1, p1, s, size);
      } else if (s == 32) {
        const bool asc = (p0 & size) == 0;
        const int lo = min(e0, e1), hi = max(e0, e1);
        e0 = asc ? lo : hi;
        e1 = asc ? hi : lo;
      } else {
        const int o0 = __shfl_xor_sync(0xffffffffu, e0, s), o1 = __shfl_xor_sync(0xffffffffu, e1, s);
        e0 = bitonic_cmpx(e0, o0, p0, s, size);
        e1 = bitonic_cmpx(e1, o1, p1, s, size);
      }
    }
  }
  __syncthreads();
  a[p0] = e0;
  a[p1] = e1;
  __syncthreads();
}

// Exact finish of one row (one CTA, every thread): the taken list holds the
// keys above the threshold bin T, the candidate list those in T; selects the
// remaining count among the candidates (radix select of their 21 low bits)
// and writes the row's k indices (ascending when p.sorted).  The shared
// arrays are the caller's: bm_sel of topk_select_smem_bytes(N) bytes.
__device__ __forceinline__ void topk_finish_row(const TopkLargeParams& p, int row, int v, int* out, uint32_t* cnt,
                                             const int* above, const uint2* cand, uint32_t* bm_sel, int* warp_buf,
                                             uint32_t* sh_digit_p, uint32_t* sh_need_p) {
  uint32_t& sh_digit = *sh_digit_p;
  uint32_t& sh_need = *sh_need_p;
  __threadfence();

  const uint32_t n_above = min(__ldcg(&cnt[kCntAbove]), (uint32_t)p.k);
  const uint32_t n_cand = min(__ldcg(&cnt[kCntCand]), (uint32_t)p.N);
  const int words = (v + 31) / 32;
  constexpr uint32_t kLowMask = (1u << kHistShift) - 1u;
  uint2* cand_s = reinterpret_cast<uint2*>(bm_sel);                // candidate cache
  uint32_t* hist = bm_sel + 2 * kTopkCandCache;                     // finish histogram
  uint32_t* R = hist + kTopkFinishBins;                             // selection or bitmap
  // the taken list's loads go out first; the candidates are staged in shared
  // memory (when they fit, the usual case) while the first digit is counted
  int abv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t i = threadIdx.x + u * blockDim.x;
    abv[u] = i < n_above ? __ldcg(above + i) : -1;
  }
  for (int i = threadIdx.x; i < kTopkFinishBins; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  const bool cand_local = n_cand <= (uint32_t)kTopkCandCache;
  for (uint32_t i0 = 0; i0 < n_cand; i0 += 8 * blockDim.x) {
    uint2 cc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t i = i0 + u * blockDim.x + threadIdx.x;
      cc[u] = i < n_cand ? __ldcg(cand + i) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t i = i0 + u * blockDim.x + threadIdx.x;
      if (i < n_cand) {
        if (cand_local) cand_s[i] = cc[u];
        atomicAdd(&hist[(cc[u].x & kLowMask) >> 10], 1u);
      }
    }
  }
  const uint2* C = cand_local ? cand_s : cand;
  __syncthreads();
  // radix select of the need-th largest key among the candidates: digit
  // bits 20..10, then bits 9..0 among the keys of that digit
  uint32_t need = (uint32_t)p.k - n_above;
  find_digit_block(hist, kTopkFinishBins, need, warp_buf, &sh_digit, &sh_need);
  __syncthreads();
  const uint32_t d1 = sh_digit;
  need = sh_need;
  for (int i = threadIdx.x; i < 1024; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
    const uint32_t key = (cand_local ? C[i].x : __ldcg(&cand[i].x)) & kLowMask;
    if ((key >> 10) == d1) atomicAdd(&hist[key & 1023u], 1u);
  }
  __syncthreads();
  find_digit_block(hist, 1024, need, warp_buf, &sh_digit, &sh_need);
  __syncthreads();
  const uint32_t prefix = (d1 << 10) | sh_digit;   // low 21 bits of the threshold key
  need = sh_need;                                   // keys equal to the threshold still to take
  const uint32_t n_eq = hist[sh_digit];             // keys equal to the threshold
  if (n_eq == need && !p.sorted) {
    // ---- common path, any order: the taken list, then the candidates at or
    // above the threshold (a block prefix sum places them)
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (abv[u] >= 0) out[threadIdx.x + u * blockDim.x] = abv[u];
    for (uint32_t i = threadIdx.x + 4 * blockDim.x; i < n_above; i += blockDim.x) out[i] = __ldcg(above + i);
    int mine = 0;
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) mine += ((C[i].x & kLowMask) >= prefix);
    int tot;
    int q = (int)n_above + block_excl_count(mine, warp_buf, &tot);
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
      const uint2 c = cand_local ? C[i] : __ldcg(cand + i);
      if ((c.x & kLowMask) >= prefix) {
        if (q < p.k) out[q] = (int)c.y;
        ++q;
      }
    }
    for (int i = (int)n_above + tot + (int)threadIdx.x; i < p.k; i += blockDim.x) out[i] = -1;
    return;
  }
  if (n_eq == need && p.k <= kTopkSortMax) {
    // ---- common path: every key equal to the threshold is taken.  The
    // selection (the taken list, then the candidates at or above the
    // threshold) is sorted ascending in shared memory: the output is in
    // index order.
    int* sel = reinterpret_cast<int*>(R);
    constexpr int kp = kTopkSortMax;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (abv[u] >= 0) sel[threadIdx.x + u * blockDim.x] = abv[u];
    for (uint32_t i = threadIdx.x + 4 * blockDim.x; i < n_above; i += blockDim.x) sel[i] = __ldcg(above + i);
    int mine = 0;
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) mine += ((C[i].x & kLowMask) >= prefix);
    int tot;
    int q = (int)n_above + block_excl_count(mine, warp_buf, &tot);
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
      const uint2 c = cand_local ? C[i] : __ldcg(cand + i);
      if ((c.x & kLowMask) >= prefix) {
        if (q < kp) sel[q] = (int)c.y;
        ++q;
      }
    }
    for (int i = (int)n_above + tot + (int)threadIdx.x; i < kp; i += blockDim.x) sel[i] = INT_MAX;
    __syncthreads();
    sort1024_block(sel);
    for (int i = threadIdx.x; i < p.k; i += blockDim.x) {
      const int j = sel[i];
      out[i] = j == INT_MAX ? -1 : j;
      if (p.prefetch_base && j != INT_MAX)
        bulk_prefetch_l2(p.prefetch_base + ((int64_t)row * p.N + j) * p.prefetch_row_bytes,
                         (uint32_t)p.prefetch_row_bytes);
    }
    return;
  }
  if (n_eq == need) {
    // ---- common path, k above the sort limit: the selection goes into a
    // v-bit bitmap; each warp owns a contiguous range of words, read
    // lane-interleaved (conflict-free); one block prefix sum of the warps'
    // popcounts and a warp scan per 32 words place the indices in order.
    uint32_t* bm = R;
    for (int i = threadIdx.x; i < words; i += blockDim.x) bm[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (abv[u] >= 0 && abv[u] < v) atomicOr(&bm[abv[u] >> 5], 1u << (abv[u] & 31));
    for (uint32_t i = threadIdx.x + 4 * blockDim.x; i < n_above; i += blockDim.x) {
      const int j = __ldcg(above + i);
      if (j >= 0 && j < v) atomicOr(&bm[j >> 5], 1u << (j & 31));
    }
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
      const uint2 c = cand_local ? C[i] : __ldcg(cand + i);
      if ((c.x & kLowMask) >= prefix && c.y < (uint32_t)v) atomicOr(&bm[c.y >> 5], 1u << (c.y & 31));
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    // rounds of 512 words per warp: lane l reads words 32 i + l (conflict
    // free); the 16 warp scans are independent, so they run interleaved
    int done = 0;
    for (int r0 = 0; r0 < words; r0 += nwarps * 512) {
      const int wb = r0 + warp * 512;
      uint32_t bits[16];
      int c[16], incl[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int w = wb + 32 * i + lane;
        bits[i] = w < words ? bm[w] : 0u;
        c[i] = __popc(bits[i]);
        incl[i] = c[i];
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int y = __shfl_up_sync(0xffffffffu, incl[i], o);
          if (lane >= o) incl[i] += y;
        }
      }
      int goff[16], wtot = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        goff[i] = wtot;
        wtot += __shfl_sync(0xffffffffu, incl[i], 31);
      }
      int tot;
      const int wbase = block_excl_count(lane == 0 ? wtot : 0, warp_buf, &tot);
      const int pos0 = done + __shfl_sync(0xffffffffu, wbase, 0);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        uint32_t b = bits[i];
        int q = pos0 + goff[i] + incl[i] - c[i];
        const int w = wb + 32 * i + lane;
        while (b) {
          const int j = w * 32 + __ffs(b) - 1;
          b &= b - 1u;
          if (q < p.k) {
            out[q] = j;
            if (p.prefetch_base)
              bulk_prefetch_l2(p.prefetch_base + ((int64_t)row * p.N + j) * p.prefetch_row_bytes,
                               (uint32_t)p.prefetch_row_bytes);
          }
          ++q;
        }
      }
      done += tot;
    }
    return;
  }
  // ---- tie path (more keys equal to the threshold than still to take):
  // the lowest-index ties through a bitmap scan in index order
  __syncthreads();
  uint32_t* bm_eq = bm_sel + words;
  for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bm_sel[i] = 0;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_above; i += blockDim.x) {
    const int j = __ldcg(above + i);
    if (j >= 0 && j < v) atomicOr(&bm_sel[j >> 5], 1u << (j & 31));
  }
  for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
    const uint2 c = __ldcg(cand + i);
    const uint32_t low = c.x & ((1u << kHistShift) - 1u);
    if (c.y >= (uint32_t)v) continue;              // (the lists hold indices < v; a bitmap has v bits)
    if (low > prefix) atomicOr(&bm_sel[c.y >> 5], 1u << (c.y & 31));
    else if (low == prefix) atomicOr(&bm_eq[c.y >> 5], 1u << (c.y & 31));
  }
  __syncthreads();
  // ties to the lower index: the first `need` set bits of bm_eq
  bitmap_scan(bm_eq, words, (int)need, warp_buf,
              [&](int, int j) { atomicOr(&bm_sel[j >> 5], 1u << (j & 31)); });
  __syncthreads();
  bitmap_scan(bm_sel, words, p.k, warp_buf, [&](int pos, int j) {
    out[pos] = j;
    if (p.prefetch_base) bulk_prefetch_l2(p.prefetch_base + ((int64_t)row * p.N + j) * p.prefetch_row_bytes,
                                          (uint32_t)p.prefetch_row_bytes);
  });
}

__global__ void __launch_bounds__(kTopkSelectThreads, 2) topk_select_kernel(TopkLargeParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t bm_sel[];               // [words] taken, then [words] ties
  __shared__ uint32_t sh[1024];
  __shared__ int warp_buf[72];
  __shared__ uint32_t sh_digit, sh_need, sh_base_t, sh_base_c;
  __shared__ int sh_last;
  const int row = blockIdx.x / p.slices, slice = blockIdx.x % p.slices;
  const int v = topk_visible(p, row);
  int* out = p.idx + (int64_t)row * p.k;
  if (v <= p.k) {
    if (slice == 0)
      for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  uint32_t* cnt = p.counters + (int64_t)row * kTopkCounters;
  int* above = p.above + (int64_t)row * p.k;
  uint2* cand = p.cand + (int64_t)row * p.N;
  {
    uint32_t n_above_T;
    int T;
    if (p.thresh_ready) {
      T = (int)__ldcg(&cnt[kCntT]);
      n_above_T = __ldcg(&cnt[kCntAboveT]);
    } else {
      T = threshold_bin(p.hist + (int64_t)row * kHistBins, p.k, sh, &n_above_T);
    }
    const int per = (v + p.slices - 1) / p.slices;
    const int j0 = slice * per, j1 = min(v, j0 + per);
    const float* s = p.scores + (int64_t)row * p.row_stride;
    // 8 keys per thread per round; the CTA reserves its ranges of the row's
    // taken / candidate lists with one atomic each (a block prefix sum places
    // every thread's entries), so the row counters see one atomic per CTA
    constexpr int kPer = 8;
    for (int base = j0; base < j1; base += kPer * (int)blockDim.x) {
      uint32_t key[kPer];
      int nt = 0, nc = 0;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int j = base + u * (int)blockDim.x + (int)threadIdx.x;
        key[u] = j < j1 ? order_key(__ldcg(s + j)) : 0u;
        const int bin = (int)(key[u] >> kHistShift);
        nt += (j < j1 && bin > T);
        nc += (j < j1 && bin == T);
      }
      int tot;
      const int off = block_excl_count(nt | (nc << 16), warp_buf, &tot);
      if (threadIdx.x == 0) {
        sh_base_t = atomicAdd(&cnt[kCntAbove], (uint32_t)(tot & 0xFFFF));
        sh_base_c = atomicAdd(&cnt[kCntCand], (uint32_t)(tot >> 16));
      }
      __syncthreads();
      uint32_t pt = sh_base_t + (uint32_t)(off & 0xFFFF), pc = sh_base_c + (uint32_t)(off >> 16);
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int j = base + u * (int)blockDim.x + (int)threadIdx.x;
        const int bin = (int)(key[u] >> kHistShift);
        if (j < j1 && bin > T) {
          if (pt < (uint32_t)p.k) above[pt] = j;
          ++pt;
        } else if (j < j1 && bin == T) {
          if (pc < (uint32_t)p.N) cand[pc] = make_uint2(key[u], (uint32_t)j);
          ++pc;
        }
      }
      __syncthreads();
    }
  }
  // publish this slice, then let the last CTA of the row finish it
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sh_last = atomicAdd(&cnt[kCntSlices], 1u) == (uint32_t)(p.slices - 1);
  __syncthreads();
  if (!sh_last) return;
  topk_finish_row(p, row, v, out, cnt, above, cand, bm_sel, warp_buf, &sh_digit, &sh_need);
}

// The finish alone, one CTA per row, after a kernel that has routed every
// key of the row into its taken and candidate lists (the FP8 decode indexer
// does so in its epilogue, with the scores still on chip).
__global__ void __launch_bounds__(kTopkSelectThreads) topk_finish_kernel(TopkLargeParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t bm_sel[];
  __shared__ int warp_buf[72];
  __shared__ uint32_t sh_digit, sh_need;
  const int row = blockIdx.x;
  const int v = topk_visible(p, row);
  int* out = p.idx + (int64_t)row * p.k;
  if (v <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  uint32_t* cnt = p.counters + (int64_t)row * kTopkCounters;
  topk_finish_row(p, row, v, out, cnt, p.above + (int64_t)row * p.k, p.cand + (int64_t)row * p.N, bm_sel,
                  warp_buf, &sh_digit, &sh_need);
}

}  // namespace csahca
