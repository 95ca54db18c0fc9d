// Top-k over long score rows (decode: one query against every visible
// compressed entry, up to 2^20 of them), spread over many CTAs.
// ("Paper Breakdown: DeepSeek-V4", section 4, DSA on Compressed KV: the top-k
// entries by I_{t,s}; "How DeepSeek-V4 architecture and training work
// together": 1,024 entries per query.)
//
//   1. topk_hist:   each CTA histograms its slice of the row on the top 11
//                   bits of the order-preserving key; global atomics merge.
//   2. topk_split:  every CTA finds the row's threshold bin T (fewer than k
//                   keys above it, at least k from it up) and routes its keys:
//                   bins above T are taken, bin T keys become candidates.
//   3. topk_finish: one CTA per row: exact radix select of the remaining
//                   count among the candidates (21 low bits), ties to the
//                   lower index through a bitmap scan in index order, and the
//                   taken set is written in ascending index order through a
//                   second bitmap scan.
#pragma once
#include "topk.cuh"

namespace csahca {

constexpr int kHistBins = 2048;            // top 11 bits of the key
constexpr int kHistShift = 21;
constexpr int kTopkLargeMaxN = 786432;     // two bitmaps of N bits in shared memory

struct TopkLargeParams {
  const float* scores; int64_t row_stride;
  const int* q_pos;
  int* idx;
  int rows, N, m, k;
  int slices;                              // CTAs per row in passes 1 and 2
  // workspace (per row)
  uint32_t* hist;                          // [rows][kHistBins]
  uint32_t* counters;                      // [rows][4]: n_above, n_cand
  int* above;                              // [rows][k]
  uint2* cand;                             // [rows][N]: (key, index)
};

__device__ __forceinline__ int topk_visible(const TopkLargeParams& p, int row) {
  const int t = p.q_pos[row];
  if (t < 0) return 0;
  const int64_t v = ((int64_t)t + 1) / p.m;
  return (int)(v < p.N ? v : p.N);
}

__global__ void __launch_bounds__(512) topk_hist_kernel(TopkLargeParams p) {
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

__global__ void __launch_bounds__(512) topk_split_kernel(TopkLargeParams p) {
  __shared__ uint32_t sh[1024];
  const int row = blockIdx.x / p.slices, slice = blockIdx.x % p.slices;
  const int v = topk_visible(p, row);
  if (v <= p.k) return;
  uint32_t n_above;
  const int T = threshold_bin(p.hist + (int64_t)row * kHistBins, p.k, sh, &n_above);
  const int per = (v + p.slices - 1) / p.slices;
  const int j0 = slice * per, j1 = min(v, j0 + per);
  const float* s = p.scores + (int64_t)row * p.row_stride;
  uint32_t* cnt = p.counters + (int64_t)row * 4;
  int* above = p.above + (int64_t)row * p.k;
  uint2* cand = p.cand + (int64_t)row * p.N;
  const int lane = threadIdx.x & 31;
  for (int base = j0; base < j1; base += blockDim.x) {
    const int j = base + threadIdx.x;
    const uint32_t key = j < j1 ? order_key(s[j]) : 0u;
    const int bin = (int)(key >> kHistShift);
    const bool take = j < j1 && bin > T;
    const bool cnd = j < j1 && bin == T;
    // warp-aggregated appends
    const unsigned mt = __ballot_sync(0xffffffffu, take);
    if (mt) {
      uint32_t basei = 0;
      if (lane == 0) basei = atomicAdd(&cnt[0], (uint32_t)__popc(mt));
      basei = __shfl_sync(0xffffffffu, basei, 0);
      if (take) {
        const uint32_t pos = basei + __popc(mt & ((1u << lane) - 1u));
        if (pos < (uint32_t)p.k) above[pos] = j;
      }
    }
    const unsigned mc = __ballot_sync(0xffffffffu, cnd);
    if (mc) {
      uint32_t basei = 0;
      if (lane == 0) basei = atomicAdd(&cnt[1], (uint32_t)__popc(mc));
      basei = __shfl_sync(0xffffffffu, basei, 0);
      if (cnd) {
        const uint32_t pos = basei + __popc(mc & ((1u << lane) - 1u));
        if (pos < (uint32_t)p.N) cand[pos] = make_uint2(key, (uint32_t)j);
      }
    }
  }
}

// Index-ordered scan of a bitmap of `words` 32-bit words: calls out(i) for the
// set bits in ascending order, at most `limit` of them; returns how many.
// blockDim.x == 1024; warp_buf as for block_excl_scan.
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
      const int x = warp_buf[lane];
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

__global__ void __launch_bounds__(1024) topk_finish_kernel(TopkLargeParams p) {
  extern __shared__ uint32_t bm_sel[];               // [words] taken, then [words] ties
  __shared__ uint32_t hist8[256];
  __shared__ int warp_buf[72];
  __shared__ uint32_t sh_digit, sh_need;
  const int row = blockIdx.x;
  const int v = topk_visible(p, row);
  int* out = p.idx + (int64_t)row * p.k;
  if (v <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  const int words = (v + 31) / 32;
  uint32_t* bm_eq = bm_sel + words;
  for (int i = threadIdx.x; i < 2 * words; i += blockDim.x) bm_sel[i] = 0;
  const uint32_t* cnt = p.counters + (int64_t)row * 4;
  const uint32_t n_above = min(cnt[0], (uint32_t)p.k);
  const uint32_t n_cand = min(cnt[1], (uint32_t)p.N);
  const uint2* cand = p.cand + (int64_t)row * p.N;
  const int* above = p.above + (int64_t)row * p.k;
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < n_above; i += blockDim.x) {
    const int j = above[i];
    atomicOr(&bm_sel[j >> 5], 1u << (j & 31));
  }
  // radix select of the need-th largest key among the candidates (bits 20..0)
  uint32_t need = (uint32_t)p.k - n_above;
  uint32_t prefix = 0, mask = 0;
  if (threadIdx.x == 0) sh_need = need;
  const int shifts[3] = {13, 5, 0};
  const int widths[3] = {8, 8, 5};
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const uint32_t dm = (1u << widths[pass]) - 1u;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist8[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
      const uint32_t key = cand[i].x & ((1u << kHistShift) - 1u);
      if ((key & mask) == prefix) atomicAdd(&hist8[(key >> sh) & dm], 1u);
    }
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) {
      const uint32_t nd = sh_need;
      __syncwarp();
      find_digit_warp(hist8, (int)dm + 1 >= 32 ? (int)dm + 1 : 32, nd, &sh_digit, &sh_need);
    }
    __syncthreads();
    prefix |= sh_digit << sh;
    mask |= dm << sh;
    __syncthreads();
  }
  need = sh_need;                              // keys equal to the threshold still to take
  for (uint32_t i = threadIdx.x; i < n_cand; i += blockDim.x) {
    const uint2 c = cand[i];
    const uint32_t low = c.x & ((1u << kHistShift) - 1u);
    if (low > prefix) atomicOr(&bm_sel[c.y >> 5], 1u << (c.y & 31));
    else if (low == prefix) atomicOr(&bm_eq[c.y >> 5], 1u << (c.y & 31));
  }
  __syncthreads();
  // ties to the lower index: the first `need` set bits of bm_eq
  bitmap_scan(bm_eq, words, (int)need, warp_buf,
              [&](int, int j) { atomicOr(&bm_sel[j >> 5], 1u << (j & 31)); });
  __syncthreads();
  bitmap_scan(bm_sel, words, p.k, warp_buf, [&](int pos, int j) { out[pos] = j; });
}

}  // namespace csahca
