// Per-query top-k over indexer scores ("Paper Breakdown: DeepSeek-V4",
// section 4, DSA on Compressed KV: the top-k entries by I_{t,s}).
//
// Radix select on order-preserving 32-bit keys: four 8-bit digit passes find
// the exact key T of the k-th largest score and how many keys equal to T are
// taken; a last pass in index order takes every key > T and the lowest-index
// keys == T (ties to the lower index), and block prefix sums place each taken
// index, so the output comes out sorted ascending with no sort.
//
// Rows up to kTopkSmemMaxN long: one CTA per row, the row's keys read from
// HBM once into shared memory; histograms are spread over 8 sub-histograms
// (warp % 8) to cut atomic contention; the digit that crosses k is found by
// one warp with a shuffle scan.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemMaxN = 32768;        // keys held in shared memory (128 KB)
constexpr int kTopkSubHist = 8;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.0f) f = 0.0f;                    // -0 and +0 are one value
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of 0/1 flags (blockDim.x a multiple of 32, <= 1024);
// returns the exclusive prefix of this thread and writes the block total to
// *total.
__device__ __forceinline__ int block_excl_scan(int flag, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned ballot = __ballot_sync(0xffffffffu, flag);
  int in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) warp_buf[wid] = __popc(ballot);
  __syncthreads();
  if (wid == 0) {
    int x = lane < (int)(blockDim.x >> 5) ? warp_buf[lane] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    warp_buf[32 + lane] = incl - x;
    if (lane == 31) warp_buf[64] = incl;
  }
  __syncthreads();
  int res = warp_buf[32 + wid] + in_warp;
  *total = warp_buf[64];
  __syncthreads();
  return res;
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

// Executed by one full warp: hist[0, nb) with nb a multiple of 32 (<= 256).
// Finds the largest digit d with sum_{e >= d} hist[e] >= need and stores d and
// need - sum_{e > d} hist[e] (the count still to take inside bin d).
__device__ __forceinline__ void find_digit_warp(const uint32_t* hist, int nb, uint32_t need,
                                                uint32_t* out_digit, uint32_t* out_need) {
  const int lane = threadIdx.x & 31;
  const int per = nb / 32;
  const int hi = nb - lane * per;              // this lane's bins: [hi - per, hi), top bins at lane 0
  uint32_t local = 0;
  for (int e = 0; e < per; ++e) local += hist[hi - 1 - e];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t above = incl - local;
  if (above < need && incl >= need) {
    uint32_t cum = above;
    for (int e = 0; e < per; ++e) {
      const int b = hi - 1 - e;
      if (cum + hist[b] >= need) { *out_digit = (uint32_t)b; *out_need = need - cum; break; }
      cum += hist[b];
    }
  }
}

struct TopkParams {
  const float* scores; int64_t row_stride;     // row r of the chunk
  const int* q_pos;                            // [B, nq]
  int* idx;                                    // [B, nq, k]
  int B, nq, N, m, k;
  int q_begin, q_count;
  int entry_base;                              // local row j is global entry entry_base + j
};

// Shared-memory slot of key j: one pad word per 32 keys keeps both the
// strided (histogram) and the per-thread-segment (output) reads conflict-free.
__host__ __device__ __forceinline__ int kslot(int j) { return j + (j >> 5); }
__host__ __device__ __forceinline__ int topk_rows_smem_bytes(int n) { return (kslot(n) + 1) * 4; }

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(TopkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t keys[];           // order keys of the row at kslot(j)
  __shared__ uint32_t hist[kTopkSubHist * 256];
  __shared__ int warp_buf[72];
  __shared__ uint32_t sh_digit, sh_need;
  const int rloc = blockIdx.x;                 // row within the chunk
  const int b = rloc / p.q_count, qi = p.q_begin + rloc % p.q_count;
  const int t = p.q_pos[(int64_t)b * p.nq + qi];
  const int v = visible_count(t, p.m, p.N, p.entry_base);
  int* out = p.idx + ((int64_t)b * p.nq + qi) * p.k;
  const float* s = p.scores + (int64_t)rloc * p.row_stride;
  if (v <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  // row -> shared keys: 16-byte loads, four in flight per thread (rows are
  // 16-byte aligned when the row stride is a multiple of 4; else scalar)
  if ((p.row_stride & 3) == 0) {
    const int v4 = v >> 2;
    const float4* s4 = reinterpret_cast<const float4*>(s);
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
        if (j4 < v4) {
          keys[kslot(4 * j4 + 0)] = order_key(f[u].x); keys[kslot(4 * j4 + 1)] = order_key(f[u].y);
          keys[kslot(4 * j4 + 2)] = order_key(f[u].z); keys[kslot(4 * j4 + 3)] = order_key(f[u].w);
        }
      }
    }
    for (int j = 4 * v4 + threadIdx.x; j < v; j += blockDim.x) keys[kslot(j)] = order_key(__ldg(s + j));
  } else {
    for (int j = threadIdx.x; j < v; j += blockDim.x) keys[kslot(j)] = order_key(__ldg(s + j));
  }
  const int wid = threadIdx.x >> 5;
  uint32_t* myhist = hist + (wid % kTopkSubHist) * 256;
  uint32_t prefix = 0, mask = 0, need = (uint32_t)p.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int x = threadIdx.x; x < kTopkSubHist * 256; x += blockDim.x) hist[x] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < v; j += blockDim.x) {
      const uint32_t u = keys[kslot(j)];
      if ((u & mask) == prefix) atomicAdd(&myhist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      uint32_t tot = 0;
#pragma unroll
      for (int h = 0; h < kTopkSubHist; ++h) tot += hist[h * 256 + threadIdx.x];
      hist[threadIdx.x] = tot;                  // sub-histogram 0 <- total (own column only)
    }
    __syncthreads();
    if (wid == 0) find_digit_warp(hist, 256, need, &sh_digit, &sh_need);
    __syncthreads();
    prefix |= sh_digit << shift;
    mask |= 255u << shift;
    need = sh_need;
    __syncthreads();
  }
  // prefix = key of the k-th largest; take all keys > prefix and the first
  // `need` keys == prefix in index order.  Thread i owns the contiguous
  // segment [i*seg, (i+1)*seg): one block scan of its count of equal keys
  // ranks the ties, one of its count of taken keys places its output.
  __syncthreads();
  const int seg = (v + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * seg, j1 = min(v, j0 + seg);
  int n_eq = 0, n_gt = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = keys[kslot(j)];
    n_eq += (u == prefix);
    n_gt += (u > prefix);
  }
  int tot;
  const int eq_before = block_excl_count(n_eq, warp_buf, &tot);
  int eq_take = (int)need - eq_before;                  // ties this thread may still take
  eq_take = eq_take < 0 ? 0 : (eq_take > n_eq ? n_eq : eq_take);
  const int pos0 = block_excl_count(n_gt + eq_take, warp_buf, &tot);
  int pos = pos0, eq_used = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = keys[kslot(j)];
    bool take = u > prefix;
    if (u == prefix && eq_used < eq_take) { take = true; ++eq_used; }
    if (take) {
      if (pos < p.k) out[pos] = j;
      ++pos;
    }
  }
}

}  // namespace csahca
