// Sink attention over a key list on CUDA cores ("Paper Breakdown:
// DeepSeek-V4", section 4: MQA core attention over the selected compressed
// entries (CSA) or every visible entry (HCA), plus the uncompressed sliding
// window, a learnable sink logit per head; query/KV RMSNorm and partial RoPE).
//
// The fp32 path.  One CTA = one query x one group of HG heads x one split of
// the key list; warp h owns head h.  Keys arrive 32 at a time into padded
// shared memory (one row per lane for QK, conflict-free), the warp keeps an
// online softmax (max, sum) and each lane owns d/32 output dims, interleaved
// so that the P.V reads are conflict-free too.  A split either writes the
// final output (one split) or a partial (max, sum, acc) for the combine.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kSimtHG = 4;           // heads per CTA (one warp each)
constexpr int kSimtKeys = 32;        // keys per shared-memory chunk
constexpr int kSimtMaxDPL = 16;      // d <= 512
constexpr int kCombineMaxSplits = 1024;

struct SimtAttnParams {
  // query side
  const void* q; const float* q_gain; const float* sinks;
  const int* pos;                    // decode: [B]; prefill: NULL (pos = t)
  int q_norm; float eps; float scale; int rope_dims; double rope_base;
  int B, nq, H, d;                   // q is [B, nq, H, d]
  // keys
  const void* kv_comp; int N;        // [B, N, d]
  const int* idx; int k;             // CSA selection [B, nq, k] or NULL (HCA: dense)
  int m;                             // ratio (HCA visibility)
  const void* win; int w;            // window rows: prefill [B, nq, d] finished, decode ring [B, w, d]
  int decode;
  // split-KV
  int splits, keys_per_split;
  // outputs: partial == NULL -> final rows in out (one split); else partials
  void* out;                         // final [B, nq, H, d]
  float* partial;                    // [B, nq, H, splits, d + 4]: m, l, -, -, acc[d]
};

template <typename T>
__device__ __forceinline__ const T* key_row(const SimtAttnParams& p, int b, int qi, int t,
                                            int j, int ncomp, int wlo) {
  if (j < ncomp) {
    int e = p.idx ? p.idx[((int64_t)b * p.nq + qi) * p.k + j] : j;
    if (e < 0) return nullptr;
    if (e >= p.N) { raise_device_error(DEVERR_BAD_INDEX); return nullptr; }
    return static_cast<const T*>(p.kv_comp) + ((int64_t)b * p.N + e) * p.d;
  }
  const int s = wlo + (j - ncomp);            // token position in the window
  if (p.decode) return static_cast<const T*>(p.win) + ((int64_t)b * p.w + (s % p.w)) * p.d;
  return static_cast<const T*>(p.win) + ((int64_t)b * p.nq + s) * p.d;
}

template <typename T>
__global__ void __launch_bounds__(32 * kSimtHG) attn_simt_kernel(SimtAttnParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float smem_at[];
  const int d = p.d, ld = d + 1;
  float* qs = smem_at;                              // [HG][d]
  float* ks = qs + kSimtHG * d;                     // [32][d + 1]
  __shared__ const T* rows[kSimtKeys];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int qi = blockIdx.x % p.nq, b = blockIdx.x / p.nq;
  const int h = blockIdx.y * kSimtHG + wid;
  const int split = blockIdx.z;
  const int t = p.decode ? p.pos[b] : qi;
  const int dpl = d / 32;

  // ---- query prologue: RMSNorm * gain, RoPE at t (lane owns dims lane + 32 e)
  float qv[kSimtMaxDPL];
  if (h < p.H) {
    const T* Q = static_cast<const T*>(p.q) + (((int64_t)b * p.nq + qi) * p.H + h) * d;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < kSimtMaxDPL; ++e)
      if (e < dpl) { qv[e] = to_f32(Q[lane + 32 * e]); ss = fmaf(qv[e], qv[e], ss); }
    if (p.q_norm) {
      float inv = rsqrtf(warp_sum(ss) / (float)d + p.eps);
#pragma unroll
      for (int e = 0; e < kSimtMaxDPL; ++e)
        if (e < dpl) qv[e] *= inv * (p.q_gain ? p.q_gain[lane + 32 * e] : 1.f);
    }
    const int r0 = d - p.rope_dims;
#pragma unroll
    for (int e = 0; e < kSimtMaxDPL; ++e) {
      if (e < dpl) {
        const int dim = lane + 32 * e;
        float partner = __shfl_xor_sync(0xffffffffu, qv[e], 1);
        if (dim >= r0) {
          float cs, sn;
          rope_cos_sin((double)t, (dim - r0) >> 1, p.rope_dims, p.rope_base, &cs, &sn);
          qv[e] = (dim & 1) ? fmaf(partner, sn, qv[e] * cs) : fmaf(-partner, sn, qv[e] * cs);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kSimtMaxDPL; ++e)
      if (e < dpl) qs[wid * d + lane + 32 * e] = qv[e];
  }

  // ---- key list: compressed part then window part
  int ncomp;
  if (p.idx) ncomp = p.k;
  else {
    int v = t < 0 ? 0 : (int)(((int64_t)t + 1) / p.m);
    ncomp = v < p.N ? v : p.N;
  }
  const int wlo = t - p.w + 1 > 0 ? t - p.w + 1 : 0;
  const int nwin = p.w > 0 ? t - wlo + 1 : 0;
  const int J = ncomp + nwin;
  const int j0 = split * p.keys_per_split;
  const int j1 = min(J, j0 + p.keys_per_split);

  float mx = -INFINITY, lsum = 0.f;
  float acc[kSimtMaxDPL];
#pragma unroll
  for (int e = 0; e < kSimtMaxDPL; ++e) acc[e] = 0.f;
  __syncthreads();

  for (int c0 = j0; c0 < j1; c0 += kSimtKeys) {
    const int nk = min(kSimtKeys, j1 - c0);
    if (threadIdx.x < kSimtKeys)
      rows[threadIdx.x] = threadIdx.x < nk ? key_row<T>(p, b, qi, t, c0 + threadIdx.x, ncomp, wlo) : nullptr;
    __syncthreads();
    for (int x = threadIdx.x; x < kSimtKeys * d; x += blockDim.x) {
      const int kk = x / d, dim = x % d;
      const T* rp = rows[kk];
      ks[kk * ld + dim] = rp ? to_f32(rp[dim]) : 0.f;
    }
    __syncthreads();
    if (h < p.H) {
      float s = -INFINITY;
      if (rows[lane]) {
        float dot = 0.f;
        const float* kr = ks + lane * ld;
        const float* qh = qs + wid * d;
        for (int x = 0; x < d; ++x) dot = fmaf(qh[x], kr[x], dot);
        s = dot * p.scale;
      }
      const float cmax = warp_max(s);
      const float mnew = fmaxf(mx, cmax);
      if (mnew != -INFINITY) {
        const float pr = (s == -INFINITY) ? 0.f : expf(s - mnew);
        const float corr = (mx == -INFINITY) ? 0.f : expf(mx - mnew);
        lsum = lsum * corr + warp_sum(pr);
#pragma unroll
        for (int e = 0; e < kSimtMaxDPL; ++e) acc[e] *= corr;
        for (int kk = 0; kk < nk; ++kk) {
          const float pk = __shfl_sync(0xffffffffu, pr, kk);
          const float* kr = ks + kk * ld;
#pragma unroll
          for (int e = 0; e < kSimtMaxDPL; ++e)
            if (e < dpl) acc[e] = fmaf(pk, kr[lane + 32 * e], acc[e]);
        }
        mx = mnew;
      }
    }
    __syncthreads();
  }
  if (h >= p.H) return;

  if (p.partial == nullptr) {
    // final: o = acc / (e^{z} + lsum) in the max-shifted frame, rope dims back by -t
    const float z = p.sinks[h];
    const float M = fmaxf(mx, z);
    const float sc = (mx == -INFINITY) ? 0.f : expf(mx - M);
    const float den = expf(z - M) + lsum * sc;
    const int r0 = d - p.rope_dims;
    T* O = static_cast<T*>(p.out) + (((int64_t)b * p.nq + qi) * p.H + h) * d;
#pragma unroll
    for (int e = 0; e < kSimtMaxDPL; ++e) {
      if (e < dpl) {
        const int dim = lane + 32 * e;
        float o = acc[e] * sc / den;
        float partner = __shfl_xor_sync(0xffffffffu, o, 1);
        if (dim >= r0) {
          float cs, sn;
          rope_cos_sin(-(double)t, (dim - r0) >> 1, p.rope_dims, p.rope_base, &cs, &sn);
          o = (dim & 1) ? fmaf(partner, sn, o * cs) : fmaf(-partner, sn, o * cs);
        }
        O[dim] = from_f32<T>(o);
      }
    }
  } else {
    float* P = p.partial + ((((int64_t)b * p.nq + qi) * p.H + h) * p.splits + split) * (d + 4);
#pragma unroll
    for (int e = 0; e < kSimtMaxDPL; ++e)
      if (e < dpl) P[4 + lane + 32 * e] = acc[e];
    if (lane == 0) { P[0] = mx; P[1] = lsum; }
  }
}

// Merge split partials: M = max(max_s mx_s, z); o = sum_s acc_s e^{mx_s - M} /
// (e^{z - M} + sum_s l_s e^{mx_s - M}); then the rope dims rotated by -t.
struct CombineParams {
  const float* partial; const float* sinks; const int* pos;
  void* out;
  int B, nq, H, d, splits, rope_dims, decode;
  double rope_base;
};

template <typename T>
__global__ void __launch_bounds__(128) attn_combine_kernel(CombineParams p) {
  griddep_wait();
  griddep_launch_dependents();
  // one CTA per (b, q, h); the split weights f_s = e^{m_s - M} / den are
  // computed once into shared memory, then each thread sums 4 dims
  __shared__ float wsplit[kCombineMaxSplits];
  const int64_t bqh = blockIdx.x;                   // (b * nq + qi) * H + h
  const int h = (int)(bqh % p.H);
  const int64_t bq = bqh / p.H;
  const int qi = (int)(bq % p.nq), b = (int)(bq / p.nq);
  const int t = p.decode ? p.pos[b] : qi;
  const int64_t ps = p.d + 4;                       // partial row: m, l, -, -, acc[d]
  const float* P = p.partial + bqh * p.splits * ps;
  const float z = p.sinks[h];
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float M = z;
    for (int s = lane; s < p.splits; s += 32) M = fmaxf(M, P[(int64_t)s * ps]);
    M = warp_max(M);
    float den = 0.f;
    for (int s = lane; s < p.splits; s += 32) {
      const float ms = P[(int64_t)s * ps];
      const float f = (ms == -INFINITY) ? 0.f : expf(ms - M);
      wsplit[s] = f;
      den += P[(int64_t)s * ps + 1] * f;
    }
    den = warp_sum(den) + expf(z - M);
    const float inv = 1.f / den;
    for (int s = lane; s < p.splits; s += 32) wsplit[s] *= inv;
  }
  __syncthreads();
  const int r0 = p.d - p.rope_dims;
  T* O = static_cast<T*>(p.out) + bqh * p.d;
  for (int dim4 = threadIdx.x * 4; dim4 < p.d; dim4 += blockDim.x * 4) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 4 <= p.splits; s += 4) {
      float4 a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = *reinterpret_cast<const float4*>(P + (int64_t)(s + u) * ps + 4 + dim4);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float f = wsplit[s + u];
        o.x = fmaf(a[u].x, f, o.x); o.y = fmaf(a[u].y, f, o.y);
        o.z = fmaf(a[u].z, f, o.z); o.w = fmaf(a[u].w, f, o.w);
      }
    }
    for (; s < p.splits; ++s) {
      const float4 a = *reinterpret_cast<const float4*>(P + (int64_t)s * ps + 4 + dim4);
      const float f = wsplit[s];
      o.x = fmaf(a.x, f, o.x); o.y = fmaf(a.y, f, o.y); o.z = fmaf(a.z, f, o.z); o.w = fmaf(a.w, f, o.w);
    }
    float v[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int dim = dim4 + e;
      if (dim >= r0) {
        float cs, sn;
        rope_cos_sin(-(double)t, (dim - r0) >> 1, p.rope_dims, p.rope_base, &cs, &sn);
        const float x0 = v[e], x1 = v[e + 1];
        v[e] = x0 * cs - x1 * sn;
        v[e + 1] = x0 * sn + x1 * cs;
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) O[dim4 + e] = from_f32<T>(v[e]);
  }
}

}  // namespace csahca
