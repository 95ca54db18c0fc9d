// Per-query top-k over indexer scores ("Paper Breakdown: DeepSeek-V4",
// section 4, DSA on Compressed KV: the top-k entries by I_{t,s}).
//
// Radix select on order-preserving 32-bit keys: four 8-bit digit passes find
// the exact key T of the k-th largest score and how many keys equal to T are
// taken; a last pass in index order takes every key > T and the lowest-index
// keys == T (ties to the lower index), and block prefix sums place each taken
// index, so the output comes out sorted ascending with no sort.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.0f) f = 0.0f;                    // -0 and +0 are one value
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of 0/1 flags (blockDim.x == kTopkThreads); returns the
// exclusive prefix of this thread and writes the block total to *total.
__device__ __forceinline__ int block_excl_scan(int flag, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned ballot = __ballot_sync(0xffffffffu, flag);
  int in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) warp_buf[wid] = __popc(ballot);
  __syncthreads();
  if (wid == 0) {
    int x = warp_buf[lane];
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

struct TopkParams {
  const float* scores; int64_t row_stride;     // row r of the chunk
  const int* q_pos;                            // [B, nq]
  int* idx;                                    // [B, nq, k]
  int B, nq, N, m, k;
  int q_begin, q_count;
};

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(TopkParams p) {
  __shared__ uint32_t hist[256];
  __shared__ int warp_buf[72];
  __shared__ uint32_t sh_digit, sh_krem;
  const int rloc = blockIdx.x;                 // row within the chunk
  const int b = rloc / p.q_count, qi = p.q_begin + rloc % p.q_count;
  const int t = p.q_pos[(int64_t)b * p.nq + qi];
  int v = 0;
  if (t >= 0) { int64_t vv = ((int64_t)t + 1) / p.m; v = (int)(vv < p.N ? vv : p.N); }
  int* out = p.idx + ((int64_t)b * p.nq + qi) * p.k;
  const float* s = p.scores + (int64_t)rloc * p.row_stride;
  if (v <= p.k) {
    for (int j = threadIdx.x; j < p.k; j += blockDim.x) out[j] = j < v ? j : -1;
    return;
  }
  uint32_t prefix = 0, mask = 0, krem = (uint32_t)p.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int x = threadIdx.x; x < 256; x += blockDim.x) hist[x] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < v; j += blockDim.x) {
      uint32_t u = order_key(s[j]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t cum = 0, digit = 0;
      for (int dgt = 255; dgt >= 0; --dgt) {
        if (cum + hist[dgt] >= krem) { digit = (uint32_t)dgt; break; }
        cum += hist[dgt];
      }
      sh_digit = digit;
      sh_krem = krem - cum;
    }
    __syncthreads();
    prefix |= sh_digit << shift;
    mask |= 255u << shift;
    krem = sh_krem;
    __syncthreads();
  }
  // prefix = key of the k-th largest; take all keys > prefix and the first
  // krem keys == prefix in index order.
  int taken = 0, eq_seen = 0;
  for (int base = 0; base < v; base += blockDim.x) {
    const int j = base + threadIdx.x;
    uint32_t u = j < v ? order_key(s[j]) : 0u;
    int gt = (j < v) && (u > prefix);
    int eq = (j < v) && (u == prefix);
    int eq_tot;
    int eq_rank = block_excl_scan(eq, warp_buf, &eq_tot) + eq_seen;
    int take = gt || (eq && eq_rank < (int)krem);
    int take_tot;
    int pos = block_excl_scan(take, warp_buf, &take_tot) + taken;
    if (take && pos < p.k) out[pos] = j;
    taken += take_tot;
    eq_seen += eq_tot;
  }
}

}  // namespace csahca
