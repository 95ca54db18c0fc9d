// Per-query top-k over indexer scores ("Paper Breakdown: DeepSeek-V4",
// section 4, DSA on Compressed KV: the top-k entries by I_{t,s}).
//
// Radix select on order-preserving 32-bit keys gives the exact key T of the
// k-th largest score and how many keys equal to T are taken; a pass in index
// order then takes every key > T and the lowest-index keys == T (ties to the
// lower index), placed by prefix counts, so the output comes out sorted
// ascending with no sort.  This file holds the shared pieces (order key,
// block prefix counts) and the kernel for rows up to kTopkSmemMaxN keys;
// longer rows use topk_large.cuh.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kTopkSmemMaxN = 32768;        // rows up to this length: topk_rows_sample_kernel
                                            // (16-bit candidate indices)

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.0f) f = 0.0f;                    // -0 and +0 are one value
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block prefix sum of per-thread counts (blockDim.x a multiple of
// 32, <= 1024).
__device__ __forceinline__ int block_excl_count(int c, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_buf[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int x = lane < (int)(blockDim.x >> 5) ? warp_buf[lane] : 0;
    int wi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_buf[32 + lane] = wi - x;
    if (lane == 31) warp_buf[64] = wi;
  }
  __syncthreads();
  const int res = warp_buf[32 + wid] + incl - c;
  *total = warp_buf[64];
  __syncthreads();
  return res;
}

struct TopkParams {
  const float* scores; int64_t row_stride;     // row r of the chunk
  const int* q_pos;                            // [B, nq]
  int* idx;                                    // [B, nq, k]
  int B, nq, N, m, k;
  int q_begin, q_count;
  int entry_base;                              // local row j is global entry entry_base + j
};

// ---- rows up to kTopkSmemMaxN: three passes over the row ---------------------
// The fallback of topk_rows_sample_kernel (below), one CTA of 256 threads per
// row, the row itself not held in shared memory:
//   pass 1 (the row from HBM): histogram of the order keys' bits 31..21 ->
//     the bin B of the k-th largest key;
//   pass 2 (from L2): each warp walks its own contiguous range of the row,
//     counting the keys in bins above B and appending the keys in B (with
//     their indices) to a candidate list in shared memory;
//   the exact key T of the k-th largest and the number of keys equal to T to
//     take follow from two histograms over the candidates (bits 20..10, then
//     9..0), and so do each warp's counts of keys > T and == T;
//   output pass (from L2): the same walk places every key > T and the
//     lowest-index keys == T by warp ballots, so the output is in index order.
// When bin B holds more keys than the list, the two digits come from passes
// over the row instead and a counting pass precedes the output pass.
constexpr int kTopkStreamThreads = 256;
constexpr int kTopkStreamWarps = kTopkStreamThreads / 32;
constexpr int kTopkStreamCand = 2048;
static_assert(kTopkSmemMaxN <= 65536, "candidate indices are 16-bit");

// One digit of the radix select over `nb` bins (nb = 8 or 4 per thread): the
// largest digit d with sum_{e >= d} hist[e] >= need; stores d and
// need - sum_{e > d} hist[e].  All threads call it.
__device__ __forceinline__ void find_digit_stream(const uint32_t* hist, int nb, uint32_t need, uint32_t* wsum,
                                                  uint32_t* out_digit, uint32_t* out_need) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int per = nb / kTopkStreamThreads;           // bins per thread (8 or 4)
  const int hi = nb - threadIdx.x * per;              // this thread's bins [hi - per, hi), top bins first
  uint32_t local = 0;
  for (int e = 0; e < per; ++e) local += hist[hi - 1 - e];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int w = 0; w < kTopkStreamWarps; ++w) before += w < wid ? wsum[w] : 0u;
  const uint32_t above = before + incl - local;        // keys in the bins above this thread's
  if (above < need && above + local >= need) {
    uint32_t cum = above;
    for (int e = 0; e < per; ++e) {
      const int b = hi - 1 - e;
      if (cum + hist[b] >= need) { *out_digit = (uint32_t)b; *out_need = need - cum; break; }
      cum += hist[b];
    }
  }
  __syncthreads();
}

// Histogram pass over the row: bins (u >> shift) & (nb - 1) of the keys u
// whose bits above hshift equal `prefix` (every key for hshift = 32).
__device__ __forceinline__ void stream_hist_pass(const float* s, int v, bool vec, uint32_t* hist, int nb, int shift,
                                                 int hshift, uint32_t prefix) {
  for (int x = threadIdx.x; x < nb; x += blockDim.x) hist[x] = 0u;
  __syncthreads();
  const uint32_t dmask = (uint32_t)nb - 1u;
  const int v4 = vec ? (v >> 2) : 0;
  const float4* s4 = reinterpret_cast<const float4*>(s);
  auto count = [&](float f) {
    const uint32_t u = order_key(f);
    if (hshift == 32 || (u >> hshift) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
  };
  for (int base = 0; base < v4; base += 4 * blockDim.x) {
    float4 f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j4 = base + u * blockDim.x + threadIdx.x;
      f[u] = j4 < v4 ? __ldg(s4 + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j4 = base + u * blockDim.x + threadIdx.x;
      if (j4 < v4) { count(f[u].x); count(f[u].y); count(f[u].z); count(f[u].w); }
    }
  }
  for (int j = 4 * v4 + threadIdx.x; j < v; j += blockDim.x) count(__ldg(s + j));
  __syncthreads();
}

// Shared memory of one row's selection (both kernels below).
struct TopkRowSmem {
  uint32_t hist[2048];
  uint32_t wsum[kTopkStreamWarps];
  uint32_t sh_digit, sh_need;
  int n_cand;
  int wcnt[kTopkStreamWarps][2];                     // per warp: keys > T, keys == T
};

// The three-pass selection of one row of v > k keys (every thread of the
// CTA): see the comment above kTopkStreamThreads.
__device__ __forceinline__ void topk_row_passes(const TopkParams& p, const float* s, int v, int* out,
                                                TopkRowSmem& sm, uint32_t* cand_key, uint16_t* cand_idx) {
  uint32_t* hist = sm.hist;
  uint32_t* wsum = sm.wsum;
  uint32_t& sh_digit = sm.sh_digit;
  uint32_t& sh_need = sm.sh_need;
  int& n_cand = sm.n_cand;
  auto& wcnt = sm.wcnt;
  const bool vec = (p.row_stride & 3) == 0;          // 16-byte aligned rows (the base is)
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  // warp w walks [j0, j1), 32 keys at a time, in the candidate and output passes
  const int L = ((v + kTopkStreamWarps * 32 - 1) / (kTopkStreamWarps * 32)) * 32;
  const int j0 = wid * L, j1 = min(v, j0 + L);

  // pass 1: bin of the k-th largest key
  if (threadIdx.x == 0) n_cand = 0;
  if (threadIdx.x < kTopkStreamWarps) { wcnt[threadIdx.x][0] = 0; wcnt[threadIdx.x][1] = 0; }
  stream_hist_pass(s, v, vec, hist, 2048, 21, 32, 0u);
  find_digit_stream(hist, 2048, (uint32_t)p.k, wsum, &sh_digit, &sh_need);
  const uint32_t B1 = sh_digit;
  uint32_t need = sh_need;

  // pass 2: keys above the bin per warp; the bin's keys to the candidate list
  int n_above = 0;
  for (int j = j0 + lane; j - lane < j1; j += 32) {
    const bool in = j < j1;
    const uint32_t u = in ? order_key(__ldg(s + j)) : 0u;
    const uint32_t bin = u >> 21;
    n_above += __popc(__ballot_sync(0xffffffffu, in && bin > B1));
    if (in && bin == B1) {
      const int slot = atomicAdd(&n_cand, 1);
      if (slot < kTopkStreamCand) { cand_key[slot] = u; cand_idx[slot] = (uint16_t)j; }
    }
  }
  __syncthreads();
  const int nc = n_cand;
  uint32_t T;
  if (nc <= kTopkStreamCand) {
    // the two lower digits from the candidates
    for (int x = threadIdx.x; x < 2048; x += blockDim.x) hist[x] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < nc; i += blockDim.x) atomicAdd(&hist[(cand_key[i] >> 10) & 2047u], 1u);
    __syncthreads();
    find_digit_stream(hist, 2048, need, wsum, &sh_digit, &sh_need);
    const uint32_t pre22 = (B1 << 11) | sh_digit;
    need = sh_need;
    for (int x = threadIdx.x; x < 1024; x += blockDim.x) hist[x] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < nc; i += blockDim.x)
      if ((cand_key[i] >> 10) == pre22) atomicAdd(&hist[cand_key[i] & 1023u], 1u);
    __syncthreads();
    find_digit_stream(hist, 1024, need, wsum, &sh_digit, &sh_need);
    T = (pre22 << 10) | sh_digit;
    need = sh_need;
    // per-warp counts: keys above the bin (pass 2) plus the candidates > T, == T
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      const uint32_t u = cand_key[i];
      const int w = (int)cand_idx[i] / L;
      if (u > T) atomicAdd(&wcnt[w][0], 1);
      else if (u == T) atomicAdd(&wcnt[w][1], 1);
    }
    if (lane == 0) atomicAdd(&wcnt[wid][0], n_above);
  } else {
    // more keys in the bin than the list holds: the digits by passes over the row
    stream_hist_pass(s, v, vec, hist, 2048, 10, 21, B1);
    find_digit_stream(hist, 2048, need, wsum, &sh_digit, &sh_need);
    const uint32_t pre22 = (B1 << 11) | sh_digit;
    need = sh_need;
    stream_hist_pass(s, v, vec, hist, 1024, 0, 10, pre22);
    find_digit_stream(hist, 1024, need, wsum, &sh_digit, &sh_need);
    T = (pre22 << 10) | sh_digit;
    need = sh_need;
    int n_gt = 0, n_eq = 0;
    for (int j = j0 + lane; j - lane < j1; j += 32) {
      const bool in = j < j1;
      const uint32_t u = in ? order_key(__ldg(s + j)) : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, in && u > T));
      n_eq += __popc(__ballot_sync(0xffffffffu, in && u == T));
    }
    if (lane == 0) { wcnt[wid][0] = n_gt; wcnt[wid][1] = n_eq; }
  }
  __syncthreads();
  const int n_eq = wcnt[wid][1];
  int eq_before = 0, out_before = 0;
  for (int w = 0; w < wid; ++w) {
    const int eb = eq_before;
    eq_before += wcnt[w][1];
    int et = (int)need - eb;
    et = et < 0 ? 0 : (et > wcnt[w][1] ? wcnt[w][1] : et);
    out_before += wcnt[w][0] + et;
  }
  int eq_take = (int)need - eq_before;               // ties this warp takes (lowest indices first)
  eq_take = eq_take < 0 ? 0 : (eq_take > n_eq ? n_eq : eq_take);
  // output pass: keys > T and the first eq_take keys == T of this warp's range
  int pos = out_before, eq_seen = 0;
  for (int j = j0 + lane; j - lane < j1; j += 32) {
    const bool in = j < j1;
    const uint32_t u = in ? order_key(__ldg(s + j)) : 0u;
    const uint32_t eqb = __ballot_sync(0xffffffffu, in && u == T);
    const bool take = in && (u > T || (u == T && eq_seen + __popc(eqb & lt) < eq_take));
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = pos + __popc(tb & lt);
      if (o < p.k) out[o] = j;
    }
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

// Row r of the chunk: its position, visible count, output and scores.
struct TopkRow { int v; int* out; const float* s; };
__device__ __forceinline__ TopkRow topk_row(const TopkParams& p) {
  const int rloc = blockIdx.x;                       // row within the chunk
  const int b = rloc / p.q_count, qi = p.q_begin + rloc % p.q_count;
  const int t = p.q_pos[(int64_t)b * p.nq + qi];
  TopkRow r;
  r.v = visible_count(t, p.m, p.N, p.entry_base);
  r.out = p.idx + ((int64_t)b * p.nq + qi) * p.k;
  r.s = p.scores + (int64_t)rloc * p.row_stride;
  return r;
}

// ---- rows up to kTopkSmemMaxN, one pass over the row --------------------------
// topk_rows_sample_kernel (256 threads, ~33 KB of shared memory):
//   bound: a row whose warp ranges fit the warps' candidate lists keeps
//     every key; otherwise a histogram of one 32-key segment in 8 gives the
//     bin of the sample's k_s-th largest key, k_s = the sample's share of k
//     plus a margin, and every key in that bin or above is kept (the k-th
//     largest of the row is in a bin at least as high unless the sample
//     misleads, which the count below detects);
//   collect (the row from HBM, once): each warp walks its contiguous range of
//     the row in index order and appends the kept keys with their indices to
//     its own list in shared memory (warp ballots place them);
//   when the lists hold at least k keys and none overflowed, the exact key T
//     of the k-th largest and the ties to take come from three histograms
//     over the lists (bits 31..21, 20..10, 9..0), and each warp writes its
//     list's keys > T and its share of the lowest-index keys == T, in index
//     order; otherwise the row takes the three passes of topk_row_passes.
constexpr int kTopkSampPerWarp = 512;
constexpr int kTopkSampCand = kTopkSampPerWarp * kTopkStreamWarps;
static_assert(kTopkSampCand >= kTopkStreamCand, "the fallback's candidate list fits the sample lists");

__global__ void __launch_bounds__(kTopkStreamThreads) topk_rows_sample_kernel(TopkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ TopkRowSmem sm;
  __shared__ uint32_t ck[kTopkSampCand];
  __shared__ uint16_t ci[kTopkSampCand];
  __shared__ int wn[kTopkStreamWarps];
  const TopkRow r = topk_row(p);
  const int v = r.v;
  int* out = r.out;
  const float* s = r.s;
  if (v <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int L = ((v + kTopkStreamWarps * 32 - 1) / (kTopkStreamWarps * 32)) * 32;
  const int j0 = wid * L, j1 = min(v, j0 + L);
  const uint32_t k = (uint32_t)p.k;

  // ---- the bin from which keys are kept
  uint32_t Blo = 0;
  if (L > kTopkSampPerWarp) {
    for (int x = threadIdx.x; x < 2048; x += blockDim.x) sm.hist[x] = 0u;
    __syncthreads();
    const int nseg = (v + 31) / 32;                  // 32-key segments; segment 8 g is sampled
    // warp w takes sampled segments 8 g, g = w + 8 i; eight loads go out
    // before any is used (the row comes from HBM)
    for (int g0 = wid; 8 * g0 < nseg; g0 += 8 * kTopkStreamWarps) {
      float f[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int j = 8 * (g0 + x * kTopkStreamWarps) * 32 + lane;
        f[x] = j < v ? __ldg(s + j) : 0.f;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int j = 8 * (g0 + x * kTopkStreamWarps) * 32 + lane;
        if (j < v) atomicAdd(&sm.hist[order_key(f[x]) >> 21], 1u);
      }
    }
    __syncthreads();
    // the sample size, then its k_s-th largest bin
    const int nfull = nseg / 8 + (nseg % 8 != 0 ? 1 : 0);
    const int last = 8 * (nfull - 1);                // the last sampled segment may be short
    const int ns = (nfull - 1) * 32 + min(32, v - 32 * last);
    const int ks0 = (int)(((int64_t)p.k * ns + v - 1) / v);
    const int ks = min(ns, ks0 + max(64, ks0 / 4));
    find_digit_stream(sm.hist, 2048, (uint32_t)ks, sm.wsum, &sm.sh_digit, &sm.sh_need);
    Blo = sm.sh_digit;
  }

  // ---- collect: each warp's kept keys, in index order, into its list.  A key
  // is kept when its order key is at least Blo << 21, i.e. when its score is
  // at least the score fb whose order key that is (order keys are monotone in
  // the score), so the walk compares scores and forms order keys for kept
  // keys only
  // (bins below 4 hold no finite score: every key is kept from there)
  const uint32_t klo = Blo << 21;
  const float fb = Blo < 4 ? -INFINITY : __uint_as_float((klo & 0x80000000u) ? (klo & 0x7fffffffu) : ~klo);
  uint32_t* lk = ck + wid * kTopkSampPerWarp;
  uint16_t* li = ci + wid * kTopkSampPerWarp;
  int cnt = 0;
  // eight 32-key steps per round: their loads go out before any is used
  for (int base = j0; base < j1; base += 8 * 32) {
    float f[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int j = base + 32 * x + lane;
      f[x] = j < j1 ? __ldg(s + j) : 0.f;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const int j = base + 32 * x + lane;
      const bool keep = j < j1 && f[x] >= fb;
      const uint32_t kb = __ballot_sync(0xffffffffu, keep);
      if (keep) {
        const int o = cnt + __popc(kb & lt);
        if (o < kTopkSampPerWarp) { lk[o] = order_key(f[x]); li[o] = (uint16_t)j; }
      }
      cnt += __popc(kb);
    }
  }
  if (lane == 0) wn[wid] = cnt;
  __syncthreads();
  int total = 0;
  bool over = false;
#pragma unroll
  for (int w = 0; w < kTopkStreamWarps; ++w) {
    total += wn[w];
    over = over || wn[w] > kTopkSampPerWarp;
  }
  if (over || total < (int)k) {
    // the sample misled or one bin holds too many keys: the three passes
    // (every thread takes this branch together: total and over are uniform)
    if (threadIdx.x == 0) sm.n_cand = 0;
    if (threadIdx.x < kTopkStreamWarps) { sm.wcnt[threadIdx.x][0] = 0; sm.wcnt[threadIdx.x][1] = 0; }
    __syncthreads();
    topk_row_passes(p, s, v, out, sm, ck, ci);
    return;
  }

  // ---- the exact threshold over the lists: three digits of 11, 11, 10 bits
  uint32_t need = k, prefix = 0;
  const int shifts[3] = {21, 10, 0};
  const int bins[3] = {2048, 2048, 1024};
#pragma unroll 1
  for (int dgt = 0; dgt < 3; ++dgt) {
    const int sh = shifts[dgt], nb = bins[dgt], hs = dgt == 0 ? 32 : shifts[dgt - 1];
    for (int x = threadIdx.x; x < 2048; x += blockDim.x) sm.hist[x] = 0u;
    __syncthreads();
    for (int x = threadIdx.x; x < kTopkSampCand; x += blockDim.x) {
      const int w = x / kTopkSampPerWarp, o = x % kTopkSampPerWarp;
      if (o < wn[w]) {
        const uint32_t u = ck[x];
        if (hs == 32 || (u >> hs) == prefix) atomicAdd(&sm.hist[(u >> sh) & (uint32_t)(nb - 1)], 1u);
      }
    }
    __syncthreads();
    find_digit_stream(sm.hist, nb, need, sm.wsum, &sm.sh_digit, &sm.sh_need);
    prefix = dgt == 0 ? sm.sh_digit : ((prefix << (dgt == 1 ? 11 : 10)) | sm.sh_digit);
    need = sm.sh_need;
  }
  const uint32_t T = prefix;                         // the k-th largest key; `need` ties at T to take

  // ---- per-warp counts, then each warp writes its list's selection in order
  int n_gt = 0, n_eq = 0;
  for (int o = lane; o - lane < wn[wid]; o += 32) {
    const bool in = o < wn[wid];
    const uint32_t u = in ? lk[o] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, in && u > T));
    n_eq += __popc(__ballot_sync(0xffffffffu, in && u == T));
  }
  if (lane == 0) { sm.wcnt[wid][0] = n_gt; sm.wcnt[wid][1] = n_eq; }
  __syncthreads();
  int eq_before = 0, out_before = 0;
  for (int w = 0; w < wid; ++w) {
    const int eb = eq_before;
    eq_before += sm.wcnt[w][1];
    int et = (int)need - eb;
    et = et < 0 ? 0 : (et > sm.wcnt[w][1] ? sm.wcnt[w][1] : et);
    out_before += sm.wcnt[w][0] + et;
  }
  int eq_take = (int)need - eq_before;               // ties this warp takes (lowest indices first)
  eq_take = eq_take < 0 ? 0 : (eq_take > n_eq ? n_eq : eq_take);
  int pos = out_before, eq_seen = 0;
  for (int o = lane; o - lane < wn[wid]; o += 32) {
    const bool in = o < wn[wid];
    const uint32_t u = in ? lk[o] : 0u;
    const uint32_t eqb = __ballot_sync(0xffffffffu, in && u == T);
    const bool take = in && (u > T || (u == T && eq_seen + __popc(eqb & lt) < eq_take));
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int q = pos + __popc(tb & lt);
      if (q < p.k) out[q] = (int)li[o];
    }
    pos += __popc(tb);
    eq_seen += __popc(eqb);
  }
}

}  // namespace csahca
