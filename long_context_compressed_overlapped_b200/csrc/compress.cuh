// Compressors and row finishing ("Paper Breakdown: DeepSeek-V4", section 4:
// CSA KV compression, HCA, Additional Techniques).
//
// One warp produces one output row.  Each lane owns 16-byte channel chunks
// (lane, lane+32, ...), streams the token rows of its chunks with 128-bit
// loads, and keeps a per-channel online softmax (running max, sum, weighted
// sum) over the pooled tokens, so every input element is read exactly once
// and each costs one exp.  RMSNorm is a warp reduction; RoPE pairs are
// adjacent channels inside one lane's chunk.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kMaxChunksPerLane = 4;   // c <= 128 * (16 / sizeof(T))

struct CompressParams {
  const void* a; const void* b; const void* za; const void* zb;
  const float* bias_a; const float* bias_b; const float* gain;
  void* out;
  int B, n, c, m, first_block, num_blocks, rms_norm, rope_dims;
  double rope_base;
  float eps;
};

// Online softmax accumulation of one token into one channel state.
__device__ __forceinline__ void pool_update(float l, float v, float& mx, float& s, float& acc) {
  if (l > mx) {
    float sc = expf(mx - l);        // 0 on the first token (mx = -inf)
    acc = fmaf(acc, sc, v);
    s = fmaf(s, sc, 1.0f);
    mx = l;
  } else {
    float e = expf(l - mx);
    acc = fmaf(e, v, acc);
    s += e;
  }
}

// RMSNorm over the whole row (all lanes' chunks) then RoPE at `pos` on the
// last r channels.  vals[q][e] is channel (lane + 32 q) * VEC + e.
template <int VEC>
__device__ __forceinline__ void finish_row(float (&vals)[kMaxChunksPerLane][VEC], int lane,
                                           int nchunks, int c, bool rms, const float* gain,
                                           float eps, int r, double pos, double base) {
  if (rms) {
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxChunksPerLane; ++q) {
      int ch = lane + 32 * q;
      if (ch < nchunks) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) ss = fmaf(vals[q][e], vals[q][e], ss);
      }
    }
    ss = warp_sum(ss);
    float inv = rsqrtf(ss / (float)c + eps);
#pragma unroll
    for (int q = 0; q < kMaxChunksPerLane; ++q) {
      int ch = lane + 32 * q;
      if (ch < nchunks) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          float g = gain ? __ldg(gain + ch * VEC + e) : 1.0f;
          vals[q][e] = vals[q][e] * inv * g;
        }
      }
    }
  }
  if (r > 0) {
    const int r0 = c - r;
#pragma unroll
    for (int q = 0; q < kMaxChunksPerLane; ++q) {
      int ch = lane + 32 * q;
      if (ch < nchunks) {
#pragma unroll
        for (int e = 0; e < VEC; e += 2) {
          int cc = ch * VEC + e;
          if (cc >= r0) {
            float cs, sn;
            rope_cos_sin(pos, (cc - r0) >> 1, r, base, &cs, &sn);
            float x0 = vals[q][e], x1 = vals[q][e + 1];
            vals[q][e] = x0 * cs - x1 * sn;
            vals[q][e + 1] = x0 * sn + x1 * cs;
          }
        }
      }
    }
  }
}

template <typename T, bool kCSA>
__global__ void __launch_bounds__(256) compress_kernel(CompressParams p) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int VEC = Vec16<T>::N;
  const int warp = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= p.B * p.num_blocks) return;
  const int bb = warp / p.num_blocks;
  const int i = p.first_block + warp % p.num_blocks;
  const int c = p.c, m = p.m;
  const int nchunks = c / VEC;
  const T* A = static_cast<const T*>(p.a) + (int64_t)bb * p.n * c;
  const T* ZA = static_cast<const T*>(p.za) + (int64_t)bb * p.n * c;
  const T* Bs = kCSA ? static_cast<const T*>(p.b) + (int64_t)bb * p.n * c : nullptr;
  const T* ZB = kCSA ? static_cast<const T*>(p.zb) + (int64_t)bb * p.n * c : nullptr;

  float vals[kMaxChunksPerLane][VEC];
#pragma unroll
  for (int q = 0; q < kMaxChunksPerLane; ++q) {
    const int ch = lane + 32 * q;
    if (ch >= nchunks) break;
    const int c0 = ch * VEC;
    float mx[VEC], s[VEC], acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) { mx[e] = -INFINITY; s[e] = 0.f; acc[e] = 0.f; }
    // stream a: the current block (tokens i*m .. i*m+m-1)
    for (int rr = 0; rr < m; ++rr) {
      const int64_t tok = (int64_t)i * m + rr;
      float z[VEC], v[VEC], bz[VEC];
      load16(ZA + tok * c + c0, z);
      load16(A + tok * c + c0, v);
#pragma unroll
      for (int e = 0; e < VEC; e += 4) load16(p.bias_a + (int64_t)rr * c + c0 + e, bz + e);
#pragma unroll
      for (int e = 0; e < VEC; ++e) pool_update(z[e] + bz[e], v[e], mx[e], s[e], acc[e]);
    }
    // stream b: the preceding block (absent for entry 0)
    if (kCSA && i > 0) {
      for (int rr = 0; rr < m; ++rr) {
        const int64_t tok = (int64_t)(i - 1) * m + rr;
        float z[VEC], v[VEC], bz[VEC];
        load16(ZB + tok * c + c0, z);
        load16(Bs + tok * c + c0, v);
#pragma unroll
        for (int e = 0; e < VEC; e += 4) load16(p.bias_b + (int64_t)rr * c + c0 + e, bz + e);
#pragma unroll
        for (int e = 0; e < VEC; ++e) pool_update(z[e] + bz[e], v[e], mx[e], s[e], acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) vals[q][e] = acc[e] / s[e];
  }
  finish_row<VEC>(vals, lane, nchunks, c, p.rms_norm != 0, p.gain, p.eps, p.rope_dims,
                  (double)i * (double)m, p.rope_base);
  T* O = static_cast<T*>(p.out) + ((int64_t)bb * p.num_blocks + (i - p.first_block)) * c;
#pragma unroll
  for (int q = 0; q < kMaxChunksPerLane; ++q) {
    const int ch = lane + 32 * q;
    if (ch < nchunks) store16(O + ch * VEC, vals[q]);
  }
}

// Finishing of per-token rows (RMSNorm * gain, RoPE at the row's position):
// row rho of x [rows, c] sits at position (rho / group) % npos.
struct FinishParams {
  const void* x; void* out; const float* gain;
  int64_t rows; int c, group, npos, rms_norm, rope_dims;
  double rope_base;
  float eps;
};

template <typename T>
__global__ void __launch_bounds__(256) finish_rows_kernel(FinishParams p) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int VEC = Vec16<T>::N;
  const int64_t row = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const int nchunks = p.c / VEC;
  const T* X = static_cast<const T*>(p.x) + row * p.c;
  float vals[kMaxChunksPerLane][VEC];
#pragma unroll
  for (int q = 0; q < kMaxChunksPerLane; ++q) {
    const int ch = lane + 32 * q;
    if (ch < nchunks) load16(X + ch * VEC, vals[q]);
  }
  const int64_t pos = (row / p.group) % p.npos;
  finish_row<VEC>(vals, lane, nchunks, p.c, p.rms_norm != 0, p.gain, p.eps, p.rope_dims,
                  (double)pos, p.rope_base);
  T* O = static_cast<T*>(p.out) + row * p.c;
#pragma unroll
  for (int q = 0; q < kMaxChunksPerLane; ++q) {
    const int ch = lane + 32 * q;
    if (ch < nchunks) store16(O + ch * VEC, vals[q]);
  }
}

}  // namespace csahca
