// Lightning-indexer scores on CUDA cores ("Paper Breakdown: DeepSeek-V4",
// section 4, DSA on Compressed KV):  I_{t,i} = sum_j w_{t,j} ReLU(qI_{t,j} . kI_i).
//
// The fp32 path (CUDA cores are the only exact-fp32 units).  One CTA scores
// up to 256 keys of one query; the query's HI x dI block and head weights sit
// in shared memory and are read as broadcasts, each thread streams one key
// row in 16-byte pieces and accumulates all heads' dot products at once.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kIdxSimtMaxHeads = 64;

struct IndexerParams {
  const void* qI; const float* w; const void* kI; const float* kI_scale;
  const int* q_pos;
  float* scores; int64_t score_row_stride;   // row r = b * nq + q (within the chunk)
  int B, nq, HI, dI, N, m;
  int q_begin, q_count;                       // query chunk [q_begin, q_begin + q_count)
  int entry_base;                             // local row j is global entry entry_base + j
};

// Local rows of a cache shard (global entries base .. base + N - 1) visible
// to the query at position t: entry i is visible iff (i + 1) m - 1 <= t.
__device__ __forceinline__ int visible_count(int t, int m, int N, int base = 0) {
  if (t < 0) return 0;
  const int64_t v = ((int64_t)t + 1) / m - base;
  return v <= 0 ? 0 : (v < N ? (int)v : N);
}

template <typename TQ, typename TK, bool kFP8>
__global__ void __launch_bounds__(256) indexer_scores_simt(IndexerParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float smem_idx[];
  float* qs = smem_idx;                       // [HI * dI]
  float* ws = qs + p.HI * p.dI;               // [HI]
  const int qi = p.q_begin + blockIdx.y;
  const int b = blockIdx.z;
  const int t = p.q_pos[(int64_t)b * p.nq + qi];
  const int v = visible_count(t, p.m, p.N, p.entry_base);
  const int key0 = blockIdx.x * 256;
  if (key0 >= v) return;
  const TQ* Q = static_cast<const TQ*>(p.qI) + ((int64_t)b * p.nq + qi) * p.HI * p.dI;
  for (int x = threadIdx.x; x < p.HI * p.dI; x += blockDim.x) qs[x] = to_f32(Q[x]);
  for (int x = threadIdx.x; x < p.HI; x += blockDim.x) ws[x] = p.w[((int64_t)b * p.nq + qi) * p.HI + x];
  __syncthreads();
  const int key = key0 + threadIdx.x;
  if (key >= v) return;
  float dots[kIdxSimtMaxHeads];
#pragma unroll
  for (int h = 0; h < kIdxSimtMaxHeads; ++h) dots[h] = 0.f;
  const int64_t row = (int64_t)b * p.N + key;
  for (int d0 = 0; d0 < p.dI; d0 += 8) {
    float kv[8];
    if constexpr (kFP8) {
      const uint8_t* K = static_cast<const uint8_t*>(p.kI) + row * p.dI + d0;
      uint2 raw = __ldg(reinterpret_cast<const uint2*>(K));
      const uint8_t* bytes = reinterpret_cast<const uint8_t*>(&raw);
      float sc = __ldg(p.kI_scale + row * (p.dI / 128) + d0 / 128);
#pragma unroll
      for (int e = 0; e < 8; ++e) kv[e] = e4m3_to_f32(bytes[e]) * sc;
    } else {
      const TK* K = static_cast<const TK*>(p.kI) + row * p.dI + d0;
      load16(K, kv);
      if constexpr (sizeof(TK) == 4) load16(K + 4, kv + 4);
    }
#pragma unroll
    for (int h = 0; h < kIdxSimtMaxHeads; ++h) {
      if (h < p.HI) {
        const float* qh = qs + h * p.dI + d0;
#pragma unroll
        for (int e = 0; e < 8; ++e) dots[h] = fmaf(qh[e], kv[e], dots[h]);
      }
    }
  }
  float score = 0.f;
#pragma unroll
  for (int h = 0; h < kIdxSimtMaxHeads; ++h)
    if (h < p.HI) score = fmaf(ws[h], fmaxf(dots[h], 0.f), score);
  p.scores[((int64_t)b * p.q_count + blockIdx.y) * p.score_row_stride + key] = score;
}

}  // namespace csahca
