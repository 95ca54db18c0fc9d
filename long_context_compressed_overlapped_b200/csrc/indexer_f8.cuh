// Lightning-indexer scores for e4m3 indexer keys on the FP8 tensor cores
// ("Paper Breakdown: DeepSeek-V4", section 4, DSA on Compressed KV:
// I_{t,i} = sum_j w_{t,j} ReLU(qI_{t,j} . kI_i); the keys are stored as e4m3
// with one fp32 scale per 128-element row).
//
// The keys stream from HBM by TMA straight into the A operand of
// tcgen05.mma.kind::f8f6f4 (128 keys x 128 e4m3 bytes, SW128), with no
// conversion.  The bf16 indexer query is made an exact e4m3 operand: with a
// per-head power of two s_h = 2^(E_h - 8), E_h the exponent of the head's
// largest |q| (so |q / s_h| < 256), every bf16 value x = q / s_h is the sum
// t0 + t1 of two e4m3 values, t0 = RNE_e4m3(x) and t1 = x - t0.  (x has 8
// significant bits; t0 keeps the top 4 after rounding, so t1 is an integer
// multiple of x's last-bit weight of magnitude <= 8 of them, which e4m3
// holds exactly whenever that weight is >= 2^-9, i.e. for every element of
// magnitude >= 2^-9 of the head's largest; smaller elements are rounded to
// within 2^-10 s_h.)  The B operand holds the two terms as 2 x HI rows (term
// t of head h in row t*HI + h), so one MMA chain of N = 2*HI over K = 128
// against the key tile gives D[i, t*HI + h] = kI_i . t_{t,h}, and
// kI_i . q_h / s_h = D[i, h] + D[i, HI + h] exactly in fp32.  Since s_h > 0 and
// the key row scale c_i > 0 commute with ReLU,
// I_{t,i} = c_i sum_h (w_h s_h) ReLU(D[i, h] + D[i, HI + h]).
// Heads whose largest |q| is below 2^-118 (s_h would leave the normal fp32
// range) contribute nothing.
//
// Roles (384 threads): two epilogue groups of 4 warps (warps 0-3, 4-7) take
// alternate key tiles, so the ReLU / weighted-sum epilogue of one tile
// overlaps the next; group 0 also writes the split query of each work item.
// Warps 8 and 11 issue the TMA key loads (and copy the keys' row scales) of
// alternate tiles into a 10-stage ring; warps 9 and 10 issue the MMAs of
// alternate tiles (N = 2*HI,
// 4 MMAs of K = 32 per tile, descriptors precomputed so that each issue is one
// add) into 4 TMEM accumulators; warp 9 owns TMEM.
// Work items as in indexer_tc.cuh: decode = (sequence, range of key tiles),
// prefill = (sequence, one query, every visible key tile).
//
// With p.hist set, the epilogue also counts each written score into a
// 2048-bin shared histogram of its order key's top 11 bits and adds it to the
// row's global histogram at the end of each work item: pass 1 of the
// multi-CTA top-k (topk_large.cuh), done while the scores are in registers.
// Unrouted, the last item of a row then finds the row's threshold bin for the
// select kernel; routed (p.route, scores kept in shared memory), every item
// waits for the row's histogram to be complete, finds the threshold bin
// itself and routes its own keys (idx_route).
#pragma once
#include "indexer_tc.cuh"
#include "topk_large.cuh"

namespace csahca {

constexpr int kIdxF8Threads = 384;
constexpr int kIdxF8Stages = 10;
constexpr int kIdxF8Acc = 4;

template <int HI>
struct IdxF8Cfg {
  static constexpr int B_TERM = HI * 128;           // one e4m3 term: HI rows x 128 bytes
  static constexpr int B_BYTES = 2 * B_TERM;
  static constexpr int A_BYTES = 128 * 128;         // 128 keys x 128 e4m3
  static constexpr int SMEM = 1024 + B_BYTES + kIdxF8Stages * A_BYTES;   // plus the fused route's score buffer
  static constexpr int NCOL = 2 * HI;               // MMA N: both terms of every head
  static constexpr int TMEM_COLS = kIdxF8Acc * NCOL <= 256 ? 256 : 512;
  static_assert(kIdxF8Acc * NCOL <= 512, "accumulators fit in TMEM");
  static_assert(kIdxF8Stages % 2 == 0 && kIdxF8Acc % 2 == 0, "tile parity picks issuer, stage and accumulator");
  static_assert(HI == 64, "two threads per head of a 128-thread group build the split query");
  static_assert(B_TERM % 1024 == 0, "SW128 operands start on 1024-byte boundaries");
};

// kind::f8f6f4 instruction descriptor: e4m3 x e4m3 -> fp32, both K-major.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 4-byte global -> shared copy; src_bytes = 0 fills zero without reading.
__device__ __forceinline__ void cp_async4_zfill(void* dst_smem, const void* src_gmem, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem), "r"(src_bytes)
               : "memory");
}

// Unrouted rows: the last work item of a top-k row (counted after a fence)
// sees the row's histogram complete, so the 256 epilogue threads find its
// threshold bin T (fewer than k keys in bins above T, at least k from T up)
// and store T and the count above it for the select kernel.  All 256
// threads call this.
__device__ __forceinline__ void idx_row_done(const IdxTcParams& p, int row, uint32_t* scan, int* sh_flag) {
  const int ept = threadIdx.x;
  uint32_t* cnt = p.counters + (int64_t)row * kTopkCounters;
  __threadfence();                                   // this item's histogram adds
  epi_sync256();
  if (ept == 0) *sh_flag = atomicAdd(&cnt[kCntItems], 1u) == (uint32_t)(p.items_per_row - 1);
  epi_sync256();
  if (!*sh_flag) return;
  __threadfence();
  const uint32_t* g = p.hist + (int64_t)row * kHistBins;
  uint32_t c[8], tot = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) { c[e] = __ldcg(g + ept * 8 + e); tot += c[e]; }
  uint32_t* a = scan;
  uint32_t* b = scan + 256;
  a[ept] = tot;
  epi_sync256();
  for (int off = 1; off < 256; off <<= 1) {          // inclusive suffix sums of the group totals
    b[ept] = a[ept] + (ept + off < 256 ? a[ept + off] : 0u);
    epi_sync256();
    uint32_t* t = a; a = b; b = t;
  }
  uint32_t run = a[ept] - tot;                        // keys in groups above this one
  const uint32_t k = (uint32_t)p.k;
  if (run < k && run + tot >= k) {
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      if (run + c[e] >= k) {
        cnt[kCntT] = (uint32_t)(ept * 8 + e);
        cnt[kCntAboveT] = run;
        break;
      }
      run += c[e];
    }
  }
  epi_sync256();
}

template <int HI>
__global__ void __launch_bounds__(kIdxF8Threads, 1)
indexer_f8_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16* __restrict__ qI, IdxTcParams p) {
  using Cfg = IdxF8Cfg<HI>;
  constexpr int NS = kIdxF8Stages, NACC = kIdxF8Acc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = base;
  uint8_t* sA = sB + Cfg::B_BYTES;
  __shared__ uint64_t bar_a_full[NS], bar_a_empty[NS];
  __shared__ uint64_t bar_acc_full[NACC], bar_acc_empty[NACC];
  __shared__ uint64_t bar_b_full, bar_b_empty, bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ float sW[2][HI];                     // per group: w_h * s_h of its current item
  __shared__ uint32_t hist_s[kHistBins];          // this item's score histogram (p.hist set)
  __shared__ float sScale[NS][128];               // key row scales of each stage
  __shared__ uint32_t scan_s[512];                // threshold search of a finished row
  __shared__ int row_flag;
  __shared__ int route_buf[9];
  __shared__ uint32_t route_T, route_base[2];
  __shared__ int route_ok;
  float* sc_s = reinterpret_cast<float*>(sA + NS * Cfg::A_BYTES);   // fused route: this item's scores

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    // a stage is full once its key tile (TMA bytes, lane 0's arrive) and its
    // scales (one cp.async arrive per producer lane) have landed; it is empty
    // once the owning epilogue group has seen the tile's accumulator (so the
    // MMAs have read the keys) and read the scales: a tcgen05.commit costs the
    // tensor pipe a few hundred cycles, so the MMA issuers commit once per tile
    for (int s = 0; s < NS; ++s) { mbar_init(&bar_a_full[s], 1 + 32); mbar_init(&bar_a_empty[s], 128); }
    // (the producer of tile i is warp 8 + (i & 1); its stage has that parity too)
    for (int j = 0; j < NACC; ++j) { mbar_init(&bar_acc_full[j], 1); mbar_init(&bar_acc_empty[j], 128); }
    mbar_init(&bar_b_full, 128);
    mbar_init(&bar_b_empty, 2);                    // both MMA issuers, once per item
    mbar_init(&bar_done, 2);
    mbar_fence_init();
  }
  if (warp == 9) tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // As a call's first kernel, nothing is read before the wait (the keys may
  // come from a compress kernel queued just before).  After the scratch
  // zeroing kernel of the same call, the key loads and MMAs start at once;
  // the epilogue waits (before the histograms) and then signals.
  if (p.first_kernel) {
    griddep_wait();
    griddep_launch_dependents();
  }

  if (warp == 8 || warp == 11) {
    // ------------------------------------------------------------ producers
    // warps 8 and 11 take alternate tiles; lane 0: the key tile by TMA; all
    // lanes: the tile's 128 row scales by cp.async (4 each, zero past the
    // row's end)
    const uint32_t pe = warp == 8 ? 0u : 1u;
    if (lane == 0) tma_prefetch_desc(&kmap);
    uint32_t a_iter = 0;
    bool stop = false;                               // warp-uniform
    for (int id = blockIdx.x; id < p.n_items && !stop; id += gridDim.x) {
      const IdxItem it = idx_item<1>(p, id);
      const float* srow = p.kI_scale + (int64_t)it.b * p.N;
      for (int kt = it.kt0; kt < it.kt1; ++kt, ++a_iter) {
        if ((a_iter & 1u) != pe) continue;
        const int s = a_iter % NS;
        const uint32_t ph = (a_iter / NS) & 1;
        int ok = 1;
        if (lane == 0) {
          ok = mbar_wait(&bar_a_empty[s], ph ^ 1, &abort_flag);
          if (ok) {
            mbar_expect_tx(&bar_a_full[s], Cfg::A_BYTES);
            tma_load_2d(sA + s * Cfg::A_BYTES, &kmap, 0, it.b * p.N + kt * 128, &bar_a_full[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { stop = true; break; }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kt * 128 + lane + 32 * e;
          const bool in = key < p.N;
          cp_async4_zfill(&sScale[s][lane + 32 * e], srow + (in ? key : 0), in ? 4u : 0u);
        }
        cp_async_arrive_noinc(&bar_a_full[s]);
      }
    }
    // drain: every fill this warp issued has landed before the CTA may exit
    // (the stage barriers complete only once the lanes' copies have; the
    // group wait orders nothing, the copies being uncommitted)
    cp_async_wait<0>();
    if (lane == 0)
      for (uint32_t i = (a_iter > NS ? a_iter - NS : 0); i < a_iter; ++i)
        if ((i & 1u) == pe) mbar_wait(&bar_a_full[i % NS], (i / NS) & 1, &abort_flag);
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // issuer e takes the tiles of parity e (their stages and accumulators have
    // that parity too), so two threads keep the tensor pipe fed
    if (lane == 0) {
      const uint32_t e = (uint32_t)(warp - 9);
      constexpr uint32_t idesc = umma_idesc_e4m3(128, Cfg::NCOL);
      uint32_t a_iter = 0, b_iter = 0, acc_iter = 0;
      // the start address is the descriptor's low field (in 16-byte units):
      // stage / K-step offsets are plain adds to the base descriptors
      const uint64_t adesc0 = umma_desc_kmajor(smem_u32(sA));
      const uint64_t bdesc0 = umma_desc_kmajor(smem_u32(sB));
      for (int id = blockIdx.x; id < p.n_items && !abort_flag; id += gridDim.x) {
        const IdxItem it = idx_item<1>(p, id);
        if (it.kt1 <= it.kt0) continue;
        if (!mbar_wait(&bar_b_full, b_iter & 1, &abort_flag)) break;
        ++b_iter;
        bool ok = true;
        for (int kt = it.kt0; kt < it.kt1; ++kt, ++a_iter, ++acc_iter) {
          if ((a_iter & 1u) != e) continue;
          const int s = a_iter % NS;
          const uint32_t ph = (a_iter / NS) & 1;
          const int j = acc_iter % NACC;
          const uint32_t aph = (acc_iter / NACC) & 1;
          if (!mbar_wait(&bar_a_full[s], ph, &abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bar_acc_empty[j], aph ^ 1, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = adesc0 + (uint64_t)((s * Cfg::A_BYTES) >> 4);
          const uint32_t d = tmem + j * Cfg::NCOL;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) umma_e4m3(d, ad + 2 * ks, bdesc0 + 2 * ks, idesc, ks != 0);
          umma_commit(&bar_acc_full[j]);
        }
        if (!ok) break;
        umma_commit(&bar_b_empty);
      }
      umma_commit(&bar_done);
      mbar_wait(&bar_done, 0, &abort_flag);
    }
  } else {
    // ------------------------------------------------------------ split query + epilogue (2 groups)
    const int g = warp >> 2;                         // group 0: warps 0-3, group 1: warps 4-7
    const int bar_id = 1 + g;
    const int et = threadIdx.x & 127;                // key lane within a tile
    const int ept = threadIdx.x;                     // 0..255 over both groups
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const bool do_hist = p.hist != nullptr;
    if (do_hist)
      for (int i = ept; i < kHistBins; i += 256) hist_s[i] = 0;
    epi_sync256();
    uint32_t acc_iter = 0, b_iter = 0;
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
      const IdxItem it = idx_item<1>(p, id);
      const int row = it.b * p.q_count + (it.q0 - p.q_begin);
      if (it.kt1 <= it.kt0) {
        if (!p.first_kernel) griddep_wait();
        // an empty item still counts
        if (do_hist) {
          if (p.route) idx_route(p, threadIdx.x, row, 0, 0, 0, sc_s, route_buf, &route_T, &route_ok, route_base, &abort_flag);
          else idx_row_done(p, row, scan_s, &row_flag);
        }
        continue;
      }
      // `bad` is uniform over a group; a group that gives up skips the rest of
      // the item and both groups leave together at its end
      bool bad = false;
      // group 0 rewrites B once the previous item's MMAs have read it
      if (g == 0 && !mbar_wait_group(bar_id, &bar_b_empty, (b_iter & 1) ^ 1, &abort_flag)) bad = true;
      ++b_iter;
      if (!bad) {
        // thread (h = et / 2, half = et % 2) owns 64 dims of head h
        const int h = et >> 1, half = et & 1;
        const int64_t qrow = ((int64_t)it.b * p.nq + it.q0) * HI + h;
        const __nv_bfloat16* src = qI + qrow * 128 + half * 64;
        float r[64];
#pragma unroll
        for (int i = 0; i < 8; ++i) load16(src + 8 * i, r + 8 * i);
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) mx = fmaxf(mx, fabsf(r[e]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        int E = 0;
        frexpf(mx, &E);                              // mx = f * 2^E, f in [0.5, 1)
        const bool live = mx >= 0x1p-118f;
        const float s_h = live ? ldexpf(1.f, E - 8) : 0.f;
        const float inv = live ? ldexpf(1.f, 8 - E) : 0.f;
        if (g == 0) {
#pragma unroll
          for (int pc = 0; pc < 4; ++pc) {           // 16 dims -> 16 bytes of each term
            uint32_t w0[4], w1[4];                   // packed explicitly: element e in byte e % 4
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t lo0 = 0, lo1 = 0;
#pragma unroll
              for (int pr = 0; pr < 2; ++pr) {
                const int e = pc * 16 + wd * 4 + pr * 2;
                const float x0 = r[e] * inv, x1 = r[e + 1] * inv;
                const __nv_fp8x2_storage_t c0 =
                    __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
                const float2 back = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(c0, __NV_E4M3)));
                const __nv_fp8x2_storage_t c1 =
                    __nv_cvt_float2_to_fp8x2(make_float2(x0 - back.x, x1 - back.y), __NV_SATFINITE, __NV_E4M3);
                lo0 |= (uint32_t)c0 << (16 * pr);
                lo1 |= (uint32_t)c1 << (16 * pr);
              }
              w0[wd] = lo0;
              w1[wd] = lo1;
            }
            *reinterpret_cast<uint4*>(sB + sw128_offset(h, half * 64 + pc * 16)) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
            *reinterpret_cast<uint4*>(sB + Cfg::B_TERM + sw128_offset(h, half * 64 + pc * 16)) =
                make_uint4(w1[0], w1[1], w1[2], w1[3]);
          }
        }
        if (half == 0) sW[g][h] = p.w[((int64_t)it.b * p.nq + it.q0) * HI + h] * s_h;
        if (g == 0) {
          fence_proxy_async_smem();
          mbar_arrive(&bar_b_full);
        }
      }
      group_sync(bar_id);                            // sW[g] complete
      if (!p.first_kernel) {
        griddep_wait();                              // the histograms and counters are zeroed
        griddep_launch_dependents();
      }
      const int v = idx_visible(p, it.b, it.q0);
      float* srow = p.scores + ((int64_t)it.b * p.q_count + (it.q0 - p.q_begin)) * p.score_row_stride;
      for (int kt = it.kt0; kt < it.kt1; ++kt, ++acc_iter) {
        if ((int)(acc_iter & 1) != g || bad) continue;   // the other group's tile, or giving up
        const int j = acc_iter % NACC;
        const uint32_t aph = (acc_iter / NACC) & 1;
        if (!mbar_wait_group(bar_id, &bar_acc_full[j], aph, &abort_flag)) { bad = true; continue; }
        tc_fence_after();
        const int key = kt * 128 + et;
        const int st = acc_iter % NS;                // this tile's stage (one stage per tile)
        const float kscale = sScale[st][et];
        mbar_arrive(&bar_a_empty[st]);
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < HI / 32; ++c) {
          float d0[32], d1[32];
          tmem_ld32(tmem + lane_base + j * Cfg::NCOL + c * 32, d0);
          tmem_ld32(tmem + lane_base + j * Cfg::NCOL + HI + c * 32, d1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) a4[e & 3] = fmaf(sW[g][c * 32 + e], fmaxf(d0[e] + d1[e], 0.f), a4[e & 3]);
        }
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        tc_fence_before();
        mbar_arrive(&bar_acc_empty[j]);
        if (key < v) {
          const float score = acc * kscale;
          if (p.route) sc_s[(kt - it.kt0) * 128 + et] = score;
          else srow[key] = score;
          if (do_hist) atomicAdd(&hist_s[order_key(score) >> kHistShift], 1u);
        }
      }
      if (epi_any256(bad)) break;                    // also: both groups are done with the item
      if (do_hist) {
        uint32_t* gh = p.hist + (int64_t)row * kHistBins;
        for (int i = ept; i < kHistBins; i += 256) {
          const uint32_t c = hist_s[i];
          if (c) { atomicAdd(gh + i, c); hist_s[i] = 0; }
        }
        if (p.route)
          idx_route(p, threadIdx.x, row, it.kt0 * 128, (it.kt1 - it.kt0) * 128, v, sc_s, route_buf, &route_T, &route_ok,
                    route_base, &abort_flag);
        else
          idx_row_done(p, row, scan_s, &row_flag);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

}  // namespace csahca
