// Sink attention on the tensor cores for narrow heads: 16 query heads of 128
// dims, dense over every visible compressed entry (the HCA layer of "Paper
// Breakdown: DeepSeek-V4", section 4 "HCA": one shared KV head, no top-k),
// plus the uncompressed sliding window and a per-head sink ("Additional
// Techniques"; "Inside DeepSeek V4", "Local window"), with the query RMSNorm,
// the partial RoPE and the output de-rotation of the wide kernel
// (attention_tc.cuh).
//
// One work item is four consecutive queries t0 .. t0+3 of a sequence.  Their
// 4 x 16 (query, head) rows form the N = 64 columns of both products, written
// transposed as in the wide kernel (S^T = K Q^T, O^T += V^T P^T, K = V, M = 128
// keys or dims), because the four queries share their keys: they see the same
// compressed entries (at most the last one differs, masked per column) and
// their windows lie in the 131 positions t0-w+1 .. t0+3.  A key tile is 128
// rows x 128 dims (two 64-dim SW128 chunks, one TMA box); two tile buffers and
// two S accumulators let the score MMAs of tile t+1 run during the softmax of
// tile t.  Every column keeps its own running max (raised lazily, by more
// than 2^8 at a time) and sum; a column whose query lies past the sequence
// end, or whose query cannot see a key, gets p = 0 there.
//
// Roles (192 threads, two CTAs per SM): warps 0-3 query prologue, softmax and
// epilogue (thread i = key slot i of S^T and dim i of O^T); warp 4 loads the
// query block and the key tiles by TMA; warp 5 issues the MMAs (the score
// MMAs of tile t, then the P.V of tile t-1) and owns TMEM.  Each tile costs
// two tcgen05.commit (scores ready, P.V done), the minimum for this pipeline.
#pragma once
#include "attention_tc.cuh"

namespace csahca {

constexpr int kSmH = 16;             // query heads
constexpr int kSmD = 128;            // head dim
constexpr int kSmQ = 4;              // queries per work item
constexpr int kSmN = kSmQ * kSmH;    // MMA N: (query, head) columns
constexpr int kSmThreads = 192;

struct AttnSmallParams {
  const __nv_bfloat16* q; const float* q_gain; const float* sinks;
  int q_norm; float eps; float scale_log2; int rope_dims;
  int B, n, N, m, w;
  int n_items;                       // B * ceil(n / kSmQ)
  int first_kernel;                  // 1: the call's first kernel (inputs are read only after the wait)
  __nv_bfloat16* out;                // [B, n, kSmH, kSmD]
  double theta[64];                  // base^(-2j/r) per rope pair j, filled on the host
};

struct SmSmem {
  static constexpr int Q_CHUNK = kSmN * 128;         // 64 rows x 64 dims bf16
  static constexpr int Q_BYTES = 2 * Q_CHUNK;
  static constexpr int K_CHUNK = 128 * 128;          // 128 keys x 64 dims bf16
  static constexpr int K_BYTES = 2 * K_CHUNK;
  static constexpr int P_BYTES = 128 * 128;          // P^T: 128 keys x 64 columns bf16
  static constexpr int TOTAL = 1024 + Q_BYTES + 2 * K_BYTES + P_BYTES;
};

struct SmItem {
  int b, t0, tl, nq;                 // queries t0 .. tl (nq of them)
  int nc;                            // tiles of compressed entries (the last query's visible ones)
  int wlo, nw;                       // window positions wlo .. tl, in nw tiles
};

__device__ __forceinline__ int sm_visible(const AttnSmallParams& p, int t) {
  const int64_t v = ((int64_t)t + 1) / p.m;
  return (int)(v < p.N ? v : p.N);
}

// Latest query blocks first (they see the most entries).
__device__ __forceinline__ SmItem sm_item(const AttnSmallParams& p, int id) {
  SmItem it;
  const int groups = (p.n + kSmQ - 1) / kSmQ;
  it.b = id % p.B;
  it.t0 = (groups - 1 - id / p.B) * kSmQ;
  it.tl = min(it.t0 + kSmQ - 1, p.n - 1);
  it.nq = it.tl - it.t0 + 1;
  it.nc = (sm_visible(p, it.tl) + 127) / 128;
  it.wlo = max(0, it.t0 - p.w + 1);
  it.nw = p.w > 0 ? (it.tl - it.wlo + 1 + 127) / 128 : 0;
  return it;
}

// 32 per-thread values (one per column of a 32-column half) -> the per-column
// max or sum over the 128 key slots of warps 0-3 (a warp transpose-reduction,
// then the four warps through shared memory); out[c] for c < 32.
template <bool kMax>
__device__ __forceinline__ void sm_reduce32(float (&v)[32], float* red, float* out) {
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16, n = 16; o >= 1; o >>= 1, n >>= 1) {
#pragma unroll
    for (int j = 0; j < n; ++j) {
      const bool hi = lane & o;
      const float keep = hi ? v[n + j] : v[j];
      const float send = hi ? v[j] : v[n + j];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[j] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  red[wq * 32 + lane] = v[0];
  named_sync128();
  if (threadIdx.x < 32) {
    float r = red[lane];
#pragma unroll
    for (int w = 1; w < 4; ++w) r = kMax ? fmaxf(r, red[w * 32 + lane]) : r + red[w * 32 + lane];
    out[lane] = r;
  }
  named_sync128();
}

__global__ void __launch_bounds__(kSmThreads, 2)
attn_small_tc_kernel(const __grid_constant__ CUtensorMap comp_map, const __grid_constant__ CUtensorMap win_map,
                     const __grid_constant__ CUtensorMap q_map, const __grid_constant__ AttnSmallParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + SmSmem::Q_BYTES;              // two tile buffers
  uint8_t* sP = sK + 2 * SmSmem::K_BYTES;
  __shared__ uint64_t bar_kfull[2], bar_kfree[2], bar_sfull[2], bar_sfree[2];
  __shared__ uint64_t bar_pfull, bar_qraw, bar_qfull, bar_qfree, bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ float red[4 * 32];
  __shared__ __align__(16) float colv[kSmN];       // per-column scratch: tile max, tile sum, output factor
  __shared__ __align__(16) float m_use[kSmN];      // running max (log2 units)
  __shared__ __align__(16) float l_run[kSmN];      // running sum
  __shared__ __align__(16) float sc_c[kSmN];       // softmax scale of each column (log2 units, times 1/rms)
  __shared__ __align__(16) float alpha[kSmN];
  __shared__ float cs_s[kSmQ][64], sn_s[kSmQ][64]; // RoPE angle of each query, per pair
  __shared__ double theta_s[64];
  __shared__ __align__(16) float gain_s[kSmD];
  __shared__ int need_rescale;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_kfull[i], 1);
      mbar_init(&bar_kfree[i], 1);
      mbar_init(&bar_sfull[i], 1);
      mbar_init(&bar_sfree[i], 128);
    }
    mbar_init(&bar_pfull, 128);
    mbar_init(&bar_qraw, 1);
    mbar_init(&bar_qfull, 128);
    mbar_init(&bar_qfree, 1);
    mbar_init(&bar_done, 1);
    mbar_fence_init();
  }
  if (warp == 5) tmem_alloc(&tmem_base_sh, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tO = tmem + 128;                  // O^T: 64 columns after the two S buffers
  if (p.first_kernel) {
    griddep_wait();
    griddep_launch_dependents();
  }

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&comp_map);
      tma_prefetch_desc(&win_map);
      tma_prefetch_desc(&q_map);
      uint32_t tc = 0, ic = 0;
      bool waited = false;
      for (int id = blockIdx.x; id < p.n_items && !abort_flag; id += gridDim.x) {
        const SmItem it = sm_item(p, id);
        const int ntile = it.nc + it.nw;
        if (ntile == 0) continue;
        // the query block once the previous item's score MMAs have read it
        if (!mbar_wait(&bar_qfree, (ic & 1) ^ 1, &abort_flag)) break;
        mbar_expect_tx(&bar_qraw, SmSmem::Q_BYTES);
        tma_load_3d(sQ, &q_map, 0, (it.b * p.n + it.t0) * kSmH, 0, &bar_qraw);
        ++ic;
        if (!waited) {
          // the window rows come from an earlier kernel of this call
          griddep_wait();
          griddep_launch_dependents();
          waited = true;
        }
        bool ok = true;
        for (int tile = 0; tile < ntile; ++tile, ++tc) {
          const int bb = tc & 1;
          if (!mbar_wait(&bar_kfree[bb], ((tc >> 1) & 1) ^ 1, &abort_flag)) { ok = false; break; }
          mbar_expect_tx(&bar_kfull[bb], SmSmem::K_BYTES);
          if (tile < it.nc)
            tma_load_3d(sK + bb * SmSmem::K_BYTES, &comp_map, 0, it.b * p.N + tile * 128, 0, &bar_kfull[bb]);
          else
            tma_load_3d(sK + bb * SmSmem::K_BYTES, &win_map, 0, it.b * p.n + it.wlo + (tile - it.nc) * 128, 0,
                        &bar_kfull[bb]);
        }
        if (!ok) break;
      }
      // drain: the last fills have landed before the CTA may exit
      for (uint32_t i = (tc > 2 ? tc - 2 : 0); i < tc; ++i) mbar_wait(&bar_kfull[i & 1], (i >> 1) & 1, &abort_flag);
      if (ic) mbar_wait(&bar_qraw, (ic - 1) & 1, &abort_flag);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kSmN, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, kSmN, 1, 1);
      const uint64_t kdesc = umma_desc_kmajor(smem_u32(sK)), qdesc = umma_desc_kmajor(smem_u32(sQ));
      const uint64_t vdesc = umma_desc_mnmajor(smem_u32(sK), SmSmem::K_CHUNK);
      const uint64_t pdesc = umma_desc_mnmajor(smem_u32(sP), SmSmem::P_BYTES);
      uint32_t tc = 0, ic = 0;
      bool stop = false;
      for (int id = blockIdx.x; id < p.n_items && !stop && !abort_flag; id += gridDim.x) {
        const SmItem it = sm_item(p, id);
        const int ntile = it.nc + it.nw;
        if (ntile == 0) continue;
        if (!mbar_wait(&bar_qfull, ic & 1, &abort_flag)) break;
        ++ic;
        for (int tile = 0; tile <= ntile && !stop; ++tile) {
          if (tile < ntile) {
            // scores of this tile into S buffer tc & 1
            const int bb = tc & 1;
            const uint32_t ph = (tc >> 1) & 1;
            if (!mbar_wait(&bar_kfull[bb], ph, &abort_flag) || !mbar_wait(&bar_sfree[bb], ph ^ 1, &abort_flag)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint64_t kd = kdesc + (uint64_t)((bb * SmSmem::K_BYTES) >> 4);
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + bb * kSmN, kd + (uint64_t)(c * (SmSmem::K_CHUNK >> 4)) + 2 * ks,
                          qdesc + (uint64_t)(c * (SmSmem::Q_CHUNK >> 4)) + 2 * ks, idesc_s, (c | ks) != 0);
            umma_commit(&bar_sfull[bb]);
            if (tile == ntile - 1) umma_commit(&bar_qfree);
          }
          if (tile > 0) {
            // P.V of the previous tile, once its P^T is written
            const uint32_t pt = tc - 1;                              // that tile's global index
            if (!mbar_wait(&bar_pfull, pt & 1, &abort_flag)) { stop = true; break; }
            tc_fence_after();
            const uint64_t vd = vdesc + (uint64_t)(((pt & 1) * SmSmem::K_BYTES) >> 4);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              umma_bf16(tO, vd + 128 * ks, pdesc + 128 * ks, idesc_pv, !(tile == 1 && ks == 0));
            umma_commit(&bar_kfree[pt & 1]);
          }
          if (tile < ntile) ++tc;
        }
      }
      umma_commit(&bar_done);
      mbar_wait(&bar_done, 0, &abort_flag);
    }
  } else {
    // ------------------------------------------------------------ prologue / softmax / epilogue
    const int tid = threadIdx.x;                   // key slot of S^T, dim of O^T
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int r0 = kSmD - p.rope_dims;
    for (int x = tid; x < kSmD; x += 128) gain_s[x] = (p.q_norm && p.q_gain) ? __ldg(p.q_gain + x) : 1.f;
    if (tid < 64) theta_s[tid] = p.theta[tid];
    named_sync128();
    uint32_t tc = 0, qc = 0;
    bool waited = p.first_kernel != 0;
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
      const SmItem it = sm_item(p, id);
      const int ntile = it.nc + it.nw;
      if (!waited) {
        griddep_wait();                            // outputs are written below
        waited = true;
      }
      if (ntile == 0) {
        // no key at all: only the sink in the denominator, o = 0
        for (int x = tid; x < it.nq * kSmH * kSmD; x += 128)
          p.out[((int64_t)it.b * p.n + it.t0) * kSmH * kSmD + x] = __float2bfloat16_rn(0.f);
        continue;
      }
      // RoPE angles of the four queries; running max and sum per column
      for (int x = tid; x < kSmQ * (p.rope_dims / 2); x += 128) {
        const int qi = x / (p.rope_dims / 2), j = x % (p.rope_dims / 2);
        rope_sincos((double)(it.t0 + qi), theta_s[j], &cs_s[qi][j], &sn_s[qi][j]);
      }
      if (tid < kSmN) { m_use[tid] = -INFINITY; l_run[tid] = 0.f; }
      bool bad = !group128_all(mbar_wait(&bar_qraw, qc & 1, &abort_flag));
      ++qc;
      if (!bad) {
        // ---- query prologue: thread (row r = tid / 2, chunk tid % 2) rewrites
        // 64 dims of row r (query r / 16, head r % 16) as RoPE_t(q * g) and
        // takes the row's RMS over both halves
        const int r = tid >> 1, hc = tid & 1, qi = r / kSmH;
        uint8_t* row = sQ + hc * SmSmem::Q_CHUNK;
        float ss = 0.f;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          uint4* a = reinterpret_cast<uint4*>(row + sw128_offset(r, pc * 16));
          float x[8];
          {
            const uint4 raw = *a;
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(h2[i]);
              x[2 * i] = f.x; x[2 * i + 1] = f.y;
            }
          }
          const int d0 = hc * 64 + pc * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) { ss = fmaf(x[e], x[e], ss); x[e] *= gain_s[d0 + e]; }
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            if (d0 + e >= r0) {
              const int j = (d0 + e - r0) >> 1;
              const float x0 = x[e], x1 = x[e + 1];
              x[e] = x0 * cs_s[qi][j] - x1 * sn_s[qi][j];
              x[e + 1] = x0 * sn_s[qi][j] + x1 * cs_s[qi][j];
            }
          }
          uint4 o;
          store16(reinterpret_cast<__nv_bfloat16*>(&o), x);
          *a = o;
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (hc == 0) sc_c[r] = p.q_norm ? p.scale_log2 * rsqrtf(ss / (float)kSmD + p.eps) : p.scale_log2;
        fence_proxy_async_smem();
      }
      mbar_arrive(&bar_qfull);
      named_sync128();                             // sc_c complete
      int vis[kSmQ];
#pragma unroll
      for (int qi = 0; qi < kSmQ; ++qi) vis[qi] = qi < it.nq ? sm_visible(p, it.t0 + qi) : 0;
      for (int tile = 0; tile < ntile; ++tile, ++tc) {
        if (bad) continue;
        const int bb = tc & 1;
        const uint32_t ph = (tc >> 1) & 1;
        // which of the four queries may use this key slot
        bool vq[kSmQ];
        if (tile < it.nc) {
          const int e = tile * 128 + tid;
#pragma unroll
          for (int qi = 0; qi < kSmQ; ++qi) vq[qi] = e < vis[qi];
        } else {
          const int s = it.wlo + (tile - it.nc) * 128 + tid;
#pragma unroll
          for (int qi = 0; qi < kSmQ; ++qi) {
            const int t = it.t0 + qi;
            vq[qi] = qi < it.nq && s <= t && s > t - p.w;
          }
        }
        if (!mbar_wait128(&bar_sfull[bb], ph, &abort_flag)) { bad = true; continue; }
        tc_fence_after();
        float x[kSmN];
        {
          float v0[32], v1[32];
          tmem_ld32(tmem + lane_base + bb * kSmN, v0);
          tmem_ld32(tmem + lane_base + bb * kSmN + 32, v1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) { x[c] = v0[c]; x[32 + c] = v1[c]; }
        }
        tc_fence_before();
        mbar_arrive(&bar_sfree[bb]);
#pragma unroll
        for (int c = 0; c < kSmN; ++c) x[c] = vq[c / kSmH] ? x[c] * sc_c[c] : -INFINITY;
        // the running max is raised only when a score of this tile exceeds it
        // by more than 2^8 (or on the item's first tile)
        bool exceed = tile == 0;
#pragma unroll
        for (int c = 0; c < kSmN; ++c) exceed |= x[c] > m_use[c] + kRescaleThreshold;
        exceed = group128_any(exceed);
        bool rescale = false;
        if (exceed) {
          {
            float t0[32], t1[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) { t0[c] = x[c]; t1[c] = x[32 + c]; }
            sm_reduce32<true>(t0, red, colv);
            sm_reduce32<true>(t1, red, colv + 32);
          }
          if (tid == 0) need_rescale = 0;
          named_sync128();
          if (tid < kSmN) {
            const float mt = colv[tid], mo = m_use[tid];
            float a = 1.f;
            if (mt > mo + kRescaleThreshold || (mo == -INFINITY && mt != -INFINITY)) {
              a = mo == -INFINITY ? 0.f : exp2f(mo - mt);
              m_use[tid] = mt;
              if (tile > 0) need_rescale = 1;
            }
            alpha[tid] = a;
          }
          named_sync128();
          rescale = need_rescale != 0;
        }
        // the previous tile's P.V has finished: P^T may be rewritten and O^T rescaled
        if (tile > 0) {
          if (!mbar_wait128(&bar_kfree[(tc - 1) & 1], ((tc - 1) >> 1) & 1, &abort_flag)) { bad = true; continue; }
          tc_fence_after();
        }
        if (rescale) {
          float o0[32], o1[32];
          tmem_ld32(tO + lane_base, o0);
          tmem_ld32(tO + lane_base + 32, o1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) { o0[c] *= alpha[c]; o1[c] *= alpha[32 + c]; }
          tmem_st32(tO + lane_base, o0);
          tmem_st32(tO + lane_base + 32, o1);
          tmem_wait_st();
          if (tid < kSmN) l_run[tid] *= alpha[tid];
        }
        // p = 2^(s - m) (0 for keys the column's query cannot use): row tid of P^T
#pragma unroll
        for (int c = 0; c < kSmN; ++c) x[c] = vq[c / kSmH] ? fast_exp2(x[c] - m_use[c]) : 0.f;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          uint4 o;
          store16(reinterpret_cast<__nv_bfloat16*>(&o), x + 8 * pc);
          *reinterpret_cast<uint4*>(sP + sw128_offset(tid, pc * 16)) = o;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar_pfull);
        {
          float t0[32], t1[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) { t0[c] = x[c]; t1[c] = x[32 + c]; }
          sm_reduce32<false>(t0, red, colv);
          sm_reduce32<false>(t1, red, colv + 32);
        }
        if (tid < kSmN) l_run[tid] += colv[tid];
      }
      // ---- epilogue: wait for the last P.V; o = O / (l + e^{z - m}), rope dims rotated back by -t
      if (!bad) {
        bad = !mbar_wait128(&bar_kfree[(tc - 1) & 1], ((tc - 1) >> 1) & 1, &abort_flag);
        tc_fence_after();
      }
      bad = group128_any(bad);
      if (bad) break;
      named_sync128();                             // l_run complete
      if (tid < kSmN) {
        const float z2 = p.sinks[tid % kSmH] * kLog2e;
        const float mu = m_use[tid];
        const float M = fmaxf(mu, z2);
        const float den = exp2f(z2 - M) + (mu == -INFINITY ? 0.f : l_run[tid] * exp2f(mu - M));
        colv[tid] = mu == -INFINITY ? 0.f : exp2f(mu - M) / den;
      }
      named_sync128();
      float o[kSmN];
      {
        float o0[32], o1[32];
        tmem_ld32(tO + lane_base, o0);
        tmem_ld32(tO + lane_base + 32, o1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) { o[c] = o0[c] * colv[c]; o[32 + c] = o1[c] * colv[32 + c]; }
      }
      tc_fence_before();
      const int dim = tid;
      if (warp * 32 + 31 >= r0) {                  // uniform over the warp (the shuffles)
        // pair (dim & ~1, dim | 1) sits in lanes (l & ~1, l | 1) of this warp
        const int j = dim >= r0 ? (dim - r0) >> 1 : 0;
#pragma unroll
        for (int c = 0; c < kSmN; ++c) {
          const float partner = __shfl_xor_sync(0xffffffffu, o[c], 1);
          if (dim >= r0) {
            const float cs = cs_s[c / kSmH][j], sn = sn_s[c / kSmH][j];
            o[c] = (dim & 1) ? fmaf(-partner, sn, o[c] * cs) : fmaf(partner, sn, o[c] * cs);
          }
        }
      }
      __nv_bfloat16* O = p.out + ((int64_t)it.b * p.n + it.t0) * kSmH * kSmD + dim;
#pragma unroll
      for (int c = 0; c < kSmN; ++c)
        if (c / kSmH < it.nq) O[(int64_t)c * kSmD] = __float2bfloat16_rn(o[c]);
      named_sync128();                             // shared tables are rewritten by the next item
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

}  // namespace csahca
