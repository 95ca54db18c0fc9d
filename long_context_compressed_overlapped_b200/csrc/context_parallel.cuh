// Context parallelism for compressed attention: the two exchange steps.
//
// "Paper Breakdown: DeepSeek-V4", infrastructure table ("2-Stage Context
// Parallel" for compressed attention).  A layer's compressed cache is split
// by entry range over R ranks.  Stage 1 merges every rank's top-k candidates
// into the global top-k (cp_topk_merge_kernel); stage 2 merges every rank's
// unnormalised attention share with the sink and de-rotates the output
// (cp_merge_kernel).  Both are small (a few KB per row) and one CTA handles
// one row (or one row and head).
#pragma once

#include "common.cuh"
#include "topk.cuh"

namespace csahca {

constexpr int kCpMaxRanks = 64;
constexpr int kCpMaxK = 4096;
constexpr int kCpMaxCand = 16384;
constexpr int kCpMergeThreads = 512;

// sel[row][j] = scores[row][idx[row][j]] (-inf where idx = -1): the scores of
// a row's selection, which the ranks exchange with the selection itself.
__global__ void __launch_bounds__(256) select_scores_kernel(const float* __restrict__ scores, int64_t stride,
                                                            const int* __restrict__ idx, float* __restrict__ sel,
                                                            int k) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t row = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int e = idx[row * k + j];
    sel[row * k + j] = e >= 0 ? scores[row * stride + e] : -INFINITY;
  }
}

struct CpTopkMergeParams {
  const int* cand_idx;        // [R][rows][k] local rows of each rank, -1 = none
  const float* cand_scores;   // [R][rows][k]
  int* idx_global;            // [rows][k] or null
  int* idx_local;             // [rows][k] or null
  int R, rows, k, rank;
  int kpow2;                  // smallest power of two >= k
  int bases[kCpMaxRanks];
};

__host__ __device__ inline int cp_topk_merge_smem_bytes(int R, int k, int kpow2) {
  return R * k * 8 + kpow2 * 8;
}

// One CTA per row.  Candidate (r, j) gets the 64-bit key
// (order_key(score) << 32) | (2^32 - 1 - global entry): keys are unique, and
// larger keys are higher scores, then lower entries (the top-k tie rule).
// The k-th largest key comes from a radix select over 8-bit digits; the keys
// at or above it are the selection, which a bitonic sort puts in entry order.
__global__ void __launch_bounds__(kCpMergeThreads) cp_topk_merge_kernel(const __grid_constant__ CpTopkMergeParams p) {
  extern __shared__ __align__(16) uint64_t cp_smem[];
  __shared__ uint32_t hist[256];
  __shared__ int n_valid, n_sel;
  __shared__ uint64_t sh_prefix;
  __shared__ int sh_need;
  uint64_t* keys = cp_smem;                       // [R * k]
  uint64_t* sel = cp_smem + (int64_t)p.R * p.k;   // [kpow2]: (entry << 32) | slot
  const int row = blockIdx.x, tid = threadIdx.x;
  const int n = p.R * p.k;
  if (tid == 0) { n_valid = 0; n_sel = 0; }
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();
  int mine = 0;
  for (int i = tid; i < n; i += blockDim.x) {
    const int r = i / p.k, j = i - r * p.k;
    const int64_t o = ((int64_t)r * p.rows + row) * p.k + j;
    const int loc = p.cand_idx[o];
    uint64_t key = 0;
    if (loc >= 0) {
      const uint32_t g = (uint32_t)(p.bases[r] + loc);
      key = ((uint64_t)order_key(p.cand_scores[o]) << 32) | (uint64_t)(0xFFFFFFFFu - g);
      ++mine;
    }
    keys[i] = key;
  }
  if (mine) atomicAdd(&n_valid, mine);
  __syncthreads();
  uint64_t thresh = 1;                             // every valid key (valid keys are > 0)
  if (n_valid > p.k) {
    uint64_t prefix = 0;
    int need = p.k;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
      __syncthreads();
      for (int i = tid; i < n; i += blockDim.x) {
        const uint64_t key = keys[i];
        const bool match = shift == 56 || ((key ^ prefix) >> (shift + 8)) == 0;
        if (match) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0, digit = 0;
        for (int dg = 255; dg >= 0; --dg) {
          if (cum + (int)hist[dg] >= need) { digit = dg; break; }
          cum += (int)hist[dg];
        }
        sh_need = need - cum;
        sh_prefix = prefix | ((uint64_t)digit << shift);
      }
      __syncthreads();
      need = sh_need;
      prefix = sh_prefix;
    }
    thresh = prefix;                               // the k-th largest key
  }
  for (int i = tid; i < n; i += blockDim.x) {
    const uint64_t key = keys[i];
    if (key != 0 && key >= thresh) {
      const int at = atomicAdd(&n_sel, 1);
      const uint32_t g = 0xFFFFFFFFu - (uint32_t)key;
      if (at < p.k) sel[at] = ((uint64_t)g << 32) | (uint32_t)i;
    }
  }
  __syncthreads();
  const int cnt = n_sel < p.k ? n_sel : p.k;
  for (int i = cnt + tid; i < p.kpow2; i += blockDim.x) sel[i] = ~0ull;
  __syncthreads();
  // bitonic sort of kpow2 entries, ascending
  for (int size = 2; size <= p.kpow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < p.kpow2 / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint64_t a = sel[lo], b = sel[hi];
        if ((a > b) == asc) { sel[lo] = b; sel[hi] = a; }
      }
      __syncthreads();
    }
  }
  for (int j = tid; j < p.k; j += blockDim.x) {
    int g = -1, l = -1;
    if (j < cnt) {
      const uint64_t e = sel[j];
      const int slot = (int)(uint32_t)e;
      const int r = slot / p.k;
      g = (int)(e >> 32);
      if (r == p.rank) l = p.cand_idx[((int64_t)r * p.rows + row) * p.k + (slot - r * p.k)];
    }
    if (p.idx_global) p.idx_global[(int64_t)row * p.k + j] = g;
    if (p.idx_local) p.idx_local[(int64_t)row * p.k + j] = l;
  }
}

struct CpMergeParams {
  const float* partials;      // [R][rows][2H + H*d]
  const float* sinks;         // [H]
  const int* pos;             // [rows]
  void* out;                  // [rows][H][d]
  int R, rows, H, d, rope_dims, out_bf16;
  double theta[64];           // base^(-2j/r) per rope pair j, from the host
};

// One CTA per (row, head), d / 4 threads of four dims each: the ranks'
// shares weighted by l_r 2^(mx_r - M) over the denominator with the sink,
// then the rope dims rotated back by -pos.
__global__ void __launch_bounds__(256) cp_merge_kernel(const __grid_constant__ CpMergeParams p) {
  __shared__ float c_s[kCpMaxRanks];
  __shared__ float inv_den;
  const int row = blockIdx.x / p.H, h = blockIdx.x - row * p.H;
  const int tid = threadIdx.x;
  const int64_t blk = 2 * (int64_t)p.H + (int64_t)p.H * p.d;
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) {
    const float z2 = p.sinks[h] * 1.4426950408889634f;
    float M = z2;
    for (int r = 0; r < p.R; ++r) M = fmaxf(M, p.partials[((int64_t)r * p.rows + row) * blk + h]);
    float den = exp2f(z2 - M);
    for (int r = 0; r < p.R; ++r) {
      const float* hd = p.partials + ((int64_t)r * p.rows + row) * blk;
      const float mx = hd[h];
      const float c = mx == -INFINITY ? 0.f : hd[p.H + h] * exp2f(mx - M);
      c_s[r] = c;
      den += c;
    }
    inv_den = 1.f / den;
  }
  __syncthreads();
  const int d0 = 4 * tid;
  if (d0 >= p.d) return;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < p.R; ++r) {
    const float c = c_s[r];
    if (c == 0.f) continue;
    const float4 o = *reinterpret_cast<const float4*>(p.partials + ((int64_t)r * p.rows + row) * blk + 2 * p.H +
                                                      (int64_t)h * p.d + d0);
    acc[0] = fmaf(c, o.x, acc[0]); acc[1] = fmaf(c, o.y, acc[1]);
    acc[2] = fmaf(c, o.z, acc[2]); acc[3] = fmaf(c, o.w, acc[3]);
  }
  const float inv = inv_den;
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] *= inv;
  const int r0 = p.d - p.rope_dims;
#pragma unroll
  for (int e = 0; e < 4; e += 2) {
    const int dim = d0 + e;
    if (dim >= r0) {
      float cs, sn;
      rope_sincos(-(double)p.pos[row], p.theta[(dim - r0) >> 1], &cs, &sn);
      const float x = acc[e], y = acc[e + 1];
      acc[e] = x * cs - y * sn;
      acc[e + 1] = x * sn + y * cs;
    }
  }
  const int64_t o = ((int64_t)row * p.H + h) * p.d + d0;
  if (p.out_bf16) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + o;
    __nv_bfloat162 v0 = __floats2bfloat162_rn(acc[0], acc[1]);
    __nv_bfloat162 v1 = __floats2bfloat162_rn(acc[2], acc[3]);
    reinterpret_cast<__nv_bfloat162*>(out)[0] = v0;
    reinterpret_cast<__nv_bfloat162*>(out)[1] = v1;
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

}  // namespace csahca
