// One decode step of the compressors ("Paper Breakdown: DeepSeek-V4",
// section 4: CSA KV Compression, HCA, Sliding window KV, Additional
// Techniques).
//
// For each sequence b, with its new token at t = pos[b], one cluster of eight
// CTAs:
//  * stores the token's raw compressor streams in ring slot t % R (R = 2m for
//    CSA, m' for HCA): the only compressor state kept between steps;
//  * finishes the token's own window row (RMSNorm * gain, RoPE at t) into
//    slot t % w of the window ring;
//  * when t completes block i = (t+1)/m - 1: pools entry i over the ring
//    (token t straight from the inputs), finishes it (RMSNorm * gain, RoPE at
//    i*m) into kv_cache[b, i], and for CSA pools the indexer key of entry i
//    the same way (no norm, no RoPE) and stores it as bf16/f32, or as e4m3
//    codes with one fp32 scale per 128 elements (scale = amax / 448, 1 for an
//    all-zero block; codes round to nearest even and saturate).
//
// CTA q of a cluster owns channel slice q of every row (d/8 KV channels, dI/8
// indexer channels).  The window row is small enough for every CTA to read it
// whole and take its norm itself, so a step that completes no block needs no
// exchange between the CTAs.  The pooling of a slice is split over token
// groups, each keeping a per-channel online softmax (running max, sum,
// weighted sum) that is merged in shared memory; the entry's row-wide
// reductions -- its sum of squares and the amax of each 128-element key block
// -- are exchanged between the eight CTAs through distributed shared memory.
#pragma once
#include "common.cuh"

namespace csahca {

constexpr int kDcCluster = 8;          // CTAs per sequence (one channel slice each)
constexpr int kDcThreads = 256;
constexpr int kDcMaxVecs = 16;         // 16-byte vectors per slice and row kind
constexpr int kDcMaxRopePairs = 64;    // rope_dims <= 128

struct DecodeCompressParams {
  const int32_t* pos;
  const void* kv_raw;                         // [B, d] or null (no window row)
  const void* nw[4];                          // new token's streams [B, d]: a, b, za, zb (HCA: a, za)
  const float* bias_a; const float* bias_b;   // [m, d]
  const float* gain;                          // [d] or null
  void* ring;                                 // [B, R, S, d], S = 4 (CSA) or 2 (HCA)
  void* kv_cache;                             // [B, N_cap, d]
  void* win;                                  // [B, w, d]
  const void* inw[4];                         // indexer streams [B, dI]: a, b, za, zb
  const float* ibias_a; const float* ibias_b; // [m, dI]
  void* iring;                                // [B, 2m, 4, dI]
  void* kI;                                   // [B, N_cap, dI] (T, or e4m3 codes)
  float* kI_scale;                            // [B, N_cap, dI/128] (e4m3)
  int B, d, dI, m, N_cap, w, rope_dims, kv_norm, ki_e4m3;
  int kv_f8;                                  // kv_cache holds FP8 KV rows (one 64-dim block per CTA)
  int64_t kv_row_bytes;
  int entry_base;                             // local cache row j holds global entry entry_base + j
  float eps;
  // RoPE angle per unit of position of pair j, base^(-2j/r), computed in
  // double on the host: the kernel then carries no pow() of its own
  double theta[kDcMaxRopePairs];
};

__device__ __forceinline__ uint32_t dc_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ float dc_ld_remote(const float* local, uint32_t rank) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}
__device__ __forceinline__ void dc_cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void dc_cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// RMSNorm scale and gain, then RoPE at `pos` on the pairs of one vector whose
// channels fall in the last r; split in two so that the per-channel factors
// (gain, cos / sin of the angle) can be formed before the row's norm is known.
template <int VEC>
__device__ __forceinline__ void dc_finish_coef(int ch0, const DecodeCompressParams& p, double pos, float (&g)[VEC],
                                               float (&cs)[VEC / 2], float (&sn)[VEC / 2]) {
#pragma unroll
  for (int e = 0; e < VEC; ++e) g[e] = (p.kv_norm && p.gain) ? __ldg(p.gain + ch0 + e) : 1.f;
  const int r = p.rope_dims, r0 = p.d - r;
#pragma unroll
  for (int e = 0; e < VEC; e += 2) {
    cs[e / 2] = 1.f;
    sn[e / 2] = 0.f;
    if (r > 0 && ch0 + e >= r0) rope_sincos(pos, p.theta[(ch0 + e - r0) >> 1], &cs[e / 2], &sn[e / 2]);
  }
}
template <int VEC>
__device__ __forceinline__ void dc_finish_apply(float (&v)[VEC], int ch0, const DecodeCompressParams& p, float inv,
                                                const float (&g)[VEC], const float (&cs)[VEC / 2],
                                                const float (&sn)[VEC / 2]) {
  if (p.kv_norm) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) v[e] = v[e] * inv * g[e];
  }
  const int r = p.rope_dims, r0 = p.d - r;
#pragma unroll
  for (int e = 0; e < VEC; e += 2) {
    if (r > 0 && ch0 + e >= r0) {
      const float x0 = v[e], x1 = v[e + 1];
      v[e] = x0 * cs[e / 2] - x1 * sn[e / 2];
      v[e + 1] = x0 * sn[e / 2] + x1 * cs[e / 2];
    }
  }
}
template <int VEC>
__device__ __forceinline__ void dc_finish(float (&v)[VEC], int ch0, const DecodeCompressParams& p, float inv,
                                          double pos) {
  float g[VEC], cs[VEC / 2], sn[VEC / 2];
  dc_finish_coef<VEC>(ch0, p, pos, g, cs, sn);
  dc_finish_apply<VEC>(v, ch0, p, inv, g, cs, sn);
}

template <typename T, bool kCSA>
__global__ void __cluster_dims__(kDcCluster, 1, 1) __launch_bounds__(kDcThreads)
decode_compress_kernel(const __grid_constant__ DecodeCompressParams p) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int S = kCSA ? 4 : 2;             // streams per token
  // online-softmax state of each (token group, unit) pair, then the pooled slice
  __shared__ float st_mx[kDcThreads * VEC], st_s[kDcThreads * VEC], st_acc[kDcThreads * VEC];
  __shared__ float pooled[2 * kDcMaxVecs * VEC];
  __shared__ float wss[kDcThreads / 32];      // window row: sum of squares per warp
  __shared__ float red[2];                    // this CTA's: ss(entry), amax(key slice)
  __shared__ float tot[2];                    // the row's

  griddep_wait();
  griddep_launch_dependents();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = (int)dc_cluster_rank();
  const int b = blockIdx.x / kDcCluster;
  const int d = p.d, m = p.m;
  const int sc = d / kDcCluster, nvk = sc / VEC, nvr = d / VEC;
  const int dI = kCSA ? p.dI : 0;
  const int si = dI / kDcCluster, nvi = si / VEC;
  const int U = nvk + nvi;
  const int R = kCSA ? 2 * m : m;

  // ---- loads that need no position, issued together with the position's:
  // this CTA's slice of the new token's streams, and the whole raw window row
  // (each CTA normalises the row itself, so the common step needs no
  // exchange between the CTAs)
  uint4 nv = make_uint4(0, 0, 0, 0);
  int n_s = -1, n_ch = 0;
  bool n_idx = false;
  if (tid >= 96 && tid < 96 + S * nvk) {
    n_s = (tid - 96) / nvk;
    n_ch = q * sc + ((tid - 96) % nvk) * VEC;
    nv = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.nw[n_s]) + (int64_t)b * d + n_ch));
  } else if (tid >= 160 && tid < 160 + 4 * nvi) {
    if constexpr (kCSA) {
      n_s = (tid - 160) / nvi;
      n_ch = q * si + ((tid - 160) % nvi) * VEC;
      n_idx = true;
      nv = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.inw[n_s]) + (int64_t)b * dI + n_ch));
    }
  }
  const bool has_win = p.kv_raw != nullptr && p.w > 0;
  float wv[VEC];
  if (has_win && tid < nvr) load16(static_cast<const T*>(p.kv_raw) + (int64_t)b * d + tid * VEC, wv);
  const int t = p.pos[b];
  const int64_t t1 = (int64_t)t + 1;          // (no overflow for any position)
  // global entry i completes; it is stored in local row i - entry_base
  const bool emit = t >= 0 && t1 % m == 0 && t1 / m - 1 >= p.entry_base && t1 / m - 1 - p.entry_base < p.N_cap;
  const int i = emit ? (int)(t1 / m - 1) : 0;
  const int64_t lrow = emit ? (int64_t)i - p.entry_base : 0;
  const bool do_win = has_win && t >= 0;
  // this CTA's slice of the window row: its per-channel factors are formed
  // now, while the row's sum of squares is gathered, so that only the
  // scaling is left after the barrier
  const bool fin_win = do_win && tid >= q * nvk && tid < (q + 1) * nvk;
  float wg[VEC], wcs[VEC / 2], wsn[VEC / 2];
  if (fin_win) dc_finish_coef<VEC>(tid * VEC, p, (double)t, wg, wcs, wsn);

  // ---- the new token into ring slot t % R
  if (t >= 0 && n_s >= 0) {
    T* dst = n_idx ? static_cast<T*>(p.iring) + (((int64_t)b * R + t % R) * 4 + n_s) * dI + n_ch
                   : static_cast<T*>(p.ring) + (((int64_t)b * R + t % R) * S + n_s) * d + n_ch;
    *reinterpret_cast<uint4*>(dst) = nv;
  }

  // ---- window row: sum of squares over the whole row
  {
    float ss = 0.f;
    if (do_win && tid < nvr) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) ss = fmaf(wv[e], wv[e], ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) wss[warp] = ss;
  }

  // ---- pooling of entry i: unit u (a 16-byte vector of the KV or indexer
  // slice) x token group g; token j of the entry's list is taken by group j % G
  const T* ring = static_cast<const T*>(p.ring) + (int64_t)b * R * S * d;
  const T* iring = kCSA && dI ? static_cast<const T*>(p.iring) + (int64_t)b * R * 4 * dI : nullptr;
  const int J = kCSA ? 2 * m : m;
  const int G = min(kDcThreads / max(U, 1), J);
  if (emit) {
    const int u = tid % U, g = tid / U;
    if (g < G) {
      const bool idx = u >= nvk;
      const int c = idx ? dI : d;
      const int ch = idx ? q * si + (u - nvk) * VEC : q * sc + u * VEC;
      const T* rg = idx ? iring : ring;
      const int rs = idx ? 4 : S;
      float mx[VEC], sm[VEC], acc[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) { mx[e] = -INFINITY; sm[e] = 0.f; acc[e] = 0.f; }
#pragma unroll 2
      for (int j = g; j < J; j += G) {
        // stream a: block i, offset j; stream b: block i - 1, offset j - m (none for i = 0)
        const bool sb = kCSA && j >= m;
        const int off = sb ? j - m : j;
        if (sb && i == 0) continue;
        const int tok = (sb ? i - 1 : i) * m + off;
        const int sv = sb ? 1 : 0;                          // value stream
        const int sz = kCSA ? (sb ? 3 : 2) : 1;             // logit stream
        const T *pv, *pz;
        if (tok == t) {
          const void* const* nw = idx ? p.inw : p.nw;
          pv = static_cast<const T*>(nw[sv]) + (int64_t)b * c + ch;
          pz = static_cast<const T*>(nw[sz]) + (int64_t)b * c + ch;
        } else {
          const T* row = rg + (int64_t)(tok % R) * rs * c;
          pv = row + (int64_t)sv * c + ch;
          pz = row + (int64_t)sz * c + ch;
        }
        const float* bias = idx ? (sb ? p.ibias_b : p.ibias_a) : (sb ? p.bias_b : p.bias_a);
        float v[VEC], z[VEC], bz[VEC];
        load16(pv, v);
        load16(pz, z);
#pragma unroll
        for (int e = 0; e < VEC; e += 4) load16(bias + (int64_t)off * c + ch + e, bz + e);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float l = z[e] + bz[e];
          if (l > mx[e]) {
            const float f = expf(mx[e] - l);               // 0 on the first token (mx = -inf)
            acc[e] = fmaf(acc[e], f, v[e]);
            sm[e] = fmaf(sm[e], f, 1.0f);
            mx[e] = l;
          } else {
            const float f = expf(l - mx[e]);
            acc[e] = fmaf(f, v[e], acc[e]);
            sm[e] += f;
          }
        }
      }
      const int o = (g * U + u) * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) { st_mx[o + e] = mx[e]; st_s[o + e] = sm[e]; st_acc[o + e] = acc[e]; }
    }
  }
  __syncthreads();

  // ---- window row: this CTA's slice, normalised and rotated to position t
  if (fin_win) {
    float tw = 0.f;
    for (int k = 0; k < (nvr + 31) / 32; ++k) tw += wss[k];
    dc_finish_apply<VEC>(wv, tid * VEC, p, rsqrtf(tw / (float)d + p.eps), wg, wcs, wsn);
    store16(static_cast<T*>(p.win) + ((int64_t)b * p.w + t % p.w) * d + tid * VEC, wv);
  }
  if (!emit) return;                          // uniform over the cluster: one position per sequence

  if (tid < U * VEC) {
    // merge the groups' states of one channel
    const int u = tid / VEC, e = tid % VEC;
    float M = -INFINITY;
    for (int g = 0; g < G; ++g) M = fmaxf(M, st_mx[(g * U + u) * VEC + e]);
    float sum = 0.f, acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const int o = (g * U + u) * VEC + e;
      const float mg = st_mx[o];
      if (mg == -INFINITY) continue;                        // a group with no token
      const float f = expf(mg - M);
      sum = fmaf(st_s[o], f, sum);
      acc = fmaf(st_acc[o], f, acc);
    }
    pooled[tid] = acc / sum;
  }
  __syncthreads();

  // ---- the entry's row-wide reductions, exchanged between the cluster's CTAs
  if (warp == 0) {
    float ss = 0.f;
    for (int c = lane; c < sc; c += 32) ss = fmaf(pooled[c], pooled[c], ss);
    ss = warp_sum(ss);
    if (lane == 0) red[0] = ss;
  } else if (warp == 1) {
    float am = 0.f;
    for (int c = lane; c < si; c += 32) am = fmaxf(am, fabsf(pooled[nvk * VEC + c]));
    am = warp_max(am);
    if (lane == 0) red[1] = am;
  }
  dc_cluster_arrive();                        // red[] of every CTA written
  dc_cluster_wait();
  if (tid < 2) {
    float v = 0.f;
    // key block of this CTA's indexer slice: the ranks whose slices fall in it
    const int blk = si ? (q * si) / 128 : 0;
    for (int r = 0; r < kDcCluster; ++r) {
      if (tid == 1) {
        if (si && (r * si) / 128 == blk) v = fmaxf(v, dc_ld_remote(&red[1], (uint32_t)r));
      } else {
        v += dc_ld_remote(&red[0], (uint32_t)r);
      }
    }
    tot[tid] = v;
  }
  dc_cluster_arrive();                        // done reading the other CTAs' red[]
  __syncthreads();

  if (tid < nvk) {
    const int ch = q * sc + tid * VEC;
    float v[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) v[e] = pooled[tid * VEC + e];
    dc_finish<VEC>(v, ch, p, rsqrtf(tot[0] / (float)d + p.eps), (double)i * (double)m);
    if (p.kv_f8) {
      // FP8 KV row: this CTA's slice is one 64-dim block, of codes (with its
      // scale = amax / 448, codes = nearest e4m3 of x / scale) or of RoPE dims (bf16)
      uint8_t* row = static_cast<uint8_t*>(p.kv_cache) + ((int64_t)b * p.N_cap + lrow) * p.kv_row_bytes;
      const int r0 = d - p.rope_dims;
      if constexpr (VEC == 8) {
        if (q * sc >= r0) {
          store16(reinterpret_cast<__nv_bfloat16*>(row + r0 + 2 * (ch - r0)), v);
        } else {
          float am = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) am = fmaxf(am, fabsf(v[e]));
          const unsigned lanes = (1u << nvk) - 1u;            // the slice's threads: lanes 0 .. nvk-1
          for (int o = 1; o < nvk; o <<= 1) am = fmaxf(am, __shfl_xor_sync(lanes, am, o));
          const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
          uint32_t w8[2] = {0u, 0u};
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            w8[e / 4] |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v[e], scale), __NV_SATFINITE, __NV_E4M3)
                         << (8 * (e % 4));
          *reinterpret_cast<uint2*>(row + ch) = make_uint2(w8[0], w8[1]);
          if (tid == 0) *reinterpret_cast<float*>(row + d + p.rope_dims + 4 * (ch / 64)) = scale;
        }
      }
    } else {
      store16(static_cast<T*>(p.kv_cache) + ((int64_t)b * p.N_cap + lrow) * d + ch, v);
    }
  } else if (kCSA && tid >= 32 && tid < 32 + nvi) {
    const int u = tid - 32, ch = q * si + u * VEC;
    const float* x = pooled + (nvk + u) * VEC;
    const int64_t row = (int64_t)b * p.N_cap + lrow;
    float v[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) v[e] = x[e];
    bool stored = false;
    if constexpr (VEC % 8 == 0) {
      if (p.ki_e4m3) {                        // bf16 rows only (checked on the host)
        const float amax = tot[1];
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint32_t w8[VEC / 4];
#pragma unroll
        for (int e = 0; e < VEC / 4; ++e) w8[e] = 0;
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          w8[e / 4] |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v[e], scale), __NV_SATFINITE, __NV_E4M3)
                       << (8 * (e % 4));
        uint8_t* dst = static_cast<uint8_t*>(p.kI) + row * dI + ch;
#pragma unroll
        for (int e = 0; e < VEC / 8; ++e) *reinterpret_cast<uint2*>(dst + 8 * e) = make_uint2(w8[2 * e], w8[2 * e + 1]);
        if (u == 0 && ch % 128 == 0) p.kI_scale[row * (dI / 128) + ch / 128] = scale;
        stored = true;
      }
    }
    if (!stored) store16(static_cast<T*>(p.kI) + row * dI + ch, v);
  }
  dc_cluster_wait();                          // no CTA leaves while another still reads its red[]
}

}  // namespace csahca
