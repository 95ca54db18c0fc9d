// Lightning-indexer scores on the tensor cores ("Paper Breakdown: DeepSeek-V4",
// section 4, DSA on Compressed KV):  I_{t,i} = sum_j w_{t,j} ReLU(qI_{t,j} . kI_i).
//
// One 128-key tile of compressed indexer keys is the M = 128 operand (A,
// K-major, SW128); the QT queries x HI heads of a work item are the N operand
// (B, QT*HI <= 256 rows); K = dI = 128.  The fp32 accumulator sits in TMEM
// with one key per lane, so the ReLU and the weighted sum over heads are
// thread-local in the epilogue: thread i of the 4 epilogue warps reads the
// QT*HI columns of lane i and writes QT scores of key i.
//
// Roles (320 threads): warps 0-3 epilogue, warp 4 TMA producer, warp 5 MMA
// issuer (and TMEM owner), warps 6-9 convert e4m3 key tiles to bf16 (exact)
// when the keys are stored in e4m3 (the per-row fp32 scale is applied to the
// score: a positive per-row factor commutes with ReLU), and with bf16 keys
// form a second epilogue group: the two groups take alternate tiles (and
// accumulators), since one group's TMEM reads and weighted sums took longer
// than the tile's MMAs.
//
// Work items: prefill = (sequence, tile of QT queries, every key tile any of
// its queries can see), longest first; decode = (sequence, contiguous range of
// key tiles).  CTAs stride over the item list.
#pragma once
#include "tc_common.cuh"
#include "topk_large.cuh"

namespace csahca {

constexpr int kIdxTcThreads = 320;
constexpr int kIdxTcDim = 128;       // dI handled by the tensor-core path

struct IdxTcParams {
  const float* w; const float* kI_scale; const int* q_pos;
  float* scores; int64_t score_row_stride;
  int B, nq, HI, N, m;
  int entry_base;             // local row j is global entry entry_base + j
  int q_begin, q_count;
  int n_items;
  int splits;                 // > 0: decode items (b, split); 0: prefill items (b, query tile)
  int tiles_per_split;
  uint32_t* hist;             // optional [rows][2048] score histograms (decode, e4m3 keys)
  uint32_t* counters;         // with hist: [rows][8] top-k counters (threshold bin stored here)
  int items_per_row;          // with hist: work items per row
  int k;                      // with hist: the top-k size
  int first_kernel;           // 0: an earlier kernel of the call precedes (the FP8 decode scan may
                              // then load keys before its wait; the keys are call inputs)
  // fused routing (FP8 decode scan, one work item per CTA): scores stay in
  // shared memory, and once the row's threshold bin is known every CTA routes
  // its own keys into the row's taken list `above` [rows][k] and candidate
  // list `cand` [rows][N]; topk_finish_kernel then selects exactly
  int route;
  int* above;
  uint2* cand;
};

// ---- fused top-k routing (decode; the histogram and counters of
// topk_large.cuh).  The 256 threads of two epilogue groups take part, each
// with its index ept (0..255) among them; named barrier 3.
// Named barrier 3 over the 256 threads of both epilogue groups.
__device__ __forceinline__ void epi_sync256() { asm volatile("bar.sync 3, 256;" ::: "memory"); }
__device__ __forceinline__ bool epi_any256(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 3, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Exclusive prefix of c over the 256 epilogue threads (named barrier 3);
// *total receives the sum.  buf: 9 ints.
__device__ __forceinline__ int epi_excl_count(int ept, int c, int* buf, int* total) {
  const int lane = ept & 31, wid = ept >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) buf[wid] = incl;
  epi_sync256();
  int base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const int x = buf[w];
    base += w < wid ? x : 0;
    tot += x;
  }
  *total = tot;
  epi_sync256();
  return base + incl - c;
}

// Fused routing of one work item (all 256 epilogue threads), run by every
// item of a top-k row once its scores and histogram adds are done: count the
// item as done, wait (bounded) until every item of the row has counted, find
// the row's threshold bin T from the row's histogram (fewer than k keys in
// bins above T, at least k from T up), and send this item's keys above T to
// the row's taken list and those in T to its candidate list, reserving each
// list range with one atomic per CTA.  Every item finds T itself, so no item
// waits for another to publish it.  Requires every item of the row to be
// resident at once (one CTA per item), and nkeys <= 32 * 256.  An item
// with no keys passes v = 0: it only counts.
__device__ __forceinline__ void idx_route(const IdxTcParams& p, int ept, int row, int key0, int nkeys, int v,
                                          const float* sc, int* buf, uint32_t* sh_T, int* sh_ok,
                                          uint32_t* sh_base, volatile int* abort_flag) {
  const int lane = ept & 31, wid = ept >> 5;
  uint32_t* cnt = p.counters + (int64_t)row * kTopkCounters;
  __threadfence();                                   // this item's histogram adds
  epi_sync256();
  if (v <= p.k) {                                    // the row takes every visible key: count only
    if (ept == 0) atomicAdd(&cnt[kCntItems], 1u);
    return;
  }
  if (ept == 0) {
    atomicAdd(&cnt[kCntItems], 1u);
    int ok = 0;
    for (uint32_t it = 0; it < kMbarSpinLimit; ++it) {
      uint32_t r;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(r) : "l"(cnt + kCntItems) : "memory");
      if (r >= (uint32_t)p.items_per_row) { ok = 1; break; }
      if ((it & 1023u) == 1023u && *abort_flag) break;
      __nanosleep(32);
    }
    if (!ok) { raise_device_error(DEVERR_MBAR_TIMEOUT); *abort_flag = 1; }
    *sh_ok = ok;
  }
  epi_sync256();
  if (!*sh_ok) return;
  // the row's histogram: thread ept holds bins [8 ept, 8 ept + 8); a suffix
  // sum over the threads gives the keys in bins above each thread's group
  const uint4* g4 = reinterpret_cast<const uint4*>(p.hist + (int64_t)row * kHistBins) + 2 * ept;
  const uint4 h0 = __ldcg(g4), h1 = __ldcg(g4 + 1);
  const uint32_t c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  uint32_t tot = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) tot += c[e];
  uint32_t suf = tot;                                // inclusive suffix sum within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  if (lane == 0) buf[wid] = (int)suf;                // the warp's total
  epi_sync256();
  uint32_t run = suf - tot;                          // keys in bins above this thread's group
#pragma unroll
  for (int w = 0; w < 8; ++w) run += w > wid ? (uint32_t)buf[w] : 0u;
  const uint32_t k = (uint32_t)p.k;
  if (run < k && run + tot >= k) {
#pragma unroll
    for (int e = 7; e >= 0; --e) {
      if (run + c[e] >= k) { *sh_T = (uint32_t)(ept * 8 + e); break; }
      run += c[e];
    }
  }
  epi_sync256();
  const uint32_t T = *sh_T;
  // one pass over this item's scores: bit j of ma / me marks key ept + 256 j
  // above T / in T
  uint32_t ma = 0u, me = 0u;
  const int lim = min(nkeys, v - key0);
#pragma unroll 4
  for (int j = 0; j < 32; ++j) {
    const int i = ept + 256 * j;
    if (i < lim) {
      const uint32_t b = order_key(sc[i]) >> kHistShift;
      ma |= (uint32_t)(b > T) << j;
      me |= (uint32_t)(b == T) << j;
    }
  }
  int tot2;
  const int off = epi_excl_count(ept, __popc(ma) | (__popc(me) << 16), buf, &tot2);
  if (ept == 0) {
    sh_base[0] = tot2 & 0xFFFF ? atomicAdd(&cnt[kCntAbove], (uint32_t)(tot2 & 0xFFFF)) : 0u;
    sh_base[1] = tot2 >> 16 ? atomicAdd(&cnt[kCntCand], (uint32_t)(tot2 >> 16)) : 0u;
  }
  epi_sync256();
  int* above = p.above + (int64_t)row * p.k;
  uint2* cand = p.cand + (int64_t)row * p.N;
  uint32_t pt = sh_base[0] + (uint32_t)(off & 0xFFFF), pc = sh_base[1] + (uint32_t)(off >> 16);
  for (; ma; ma &= ma - 1u, ++pt)
    if (pt < (uint32_t)p.k) above[pt] = key0 + ept + 256 * (__ffs(ma) - 1);
  for (; me; me &= me - 1u, ++pc) {
    const int i = ept + 256 * (__ffs(me) - 1);
    if (pc < (uint32_t)p.N) cand[pc] = make_uint2(order_key(sc[i]), (uint32_t)(key0 + i));
  }
}

// Route bound: the scores of a routed work item stay in shared memory, and
// the routing marks each thread's keys in one 32-bit mask.
constexpr int kRouteMaxTiles = 64;
static_assert(kRouteMaxTiles * 128 <= 32 * 256, "a routed item's keys fit the per-thread masks");

template <int QT, int HI, bool kFP8>
struct IdxTcCfg {
  static constexpr int NCOL = QT * HI;                          // MMA N
  static constexpr int NSTAGE = kFP8 ? 4 : 4;
  static constexpr int NACC = (512 / NCOL) > 4 ? 4 : (512 / NCOL);
  static constexpr int TMEM_COLS = NCOL * NACC <= 32 ? 32 : (NCOL * NACC <= 64 ? 64 : (NCOL * NACC <= 128 ? 128 : (NCOL * NACC <= 256 ? 256 : 512)));
  static constexpr int B_CHUNK = NCOL * 128;                    // bytes per 64-dim chunk of B
  static constexpr int B_BYTES = 2 * B_CHUNK;
  static constexpr int A_BYTES = 2 * 128 * 128;                 // 128 keys x 128 dims bf16
  static constexpr int RAW_BYTES = kFP8 ? 128 * 128 : 0;        // 128 keys x 128 e4m3
  static constexpr int SMEM = 1024 + B_BYTES + NSTAGE * (A_BYTES + RAW_BYTES) + 2 * QT * HI * 4 + 1024;
  static_assert(NCOL % 16 == 0 && NCOL <= 256, "MMA N");
  static_assert(HI % 32 == 0, "heads per query must be a multiple of 32");
};

struct IdxItem { int b, q0, qn, kt0, kt1; };

__device__ __forceinline__ int idx_visible(const IdxTcParams& p, int b, int q) {
  return visible_count(p.q_pos[(int64_t)b * p.nq + q], p.m, p.N, p.entry_base);
}

template <int QT>
__device__ __forceinline__ IdxItem idx_item(const IdxTcParams& p, int id) {
  IdxItem it;
  if (p.splits > 0) {
    it.b = id / p.splits;
    const int sp = id % p.splits;
    it.q0 = p.q_begin; it.qn = 1;
    const int v = idx_visible(p, it.b, it.q0);
    const int nt = (v + 127) / 128;
    it.kt0 = sp * p.tiles_per_split;
    it.kt1 = min(nt, it.kt0 + p.tiles_per_split);
  } else {
    const int nqt = (p.q_count + QT - 1) / QT;
    const int r = id / p.B;
    it.b = id % p.B;
    const int qt = nqt - 1 - r;                       // longest (latest) query tiles first
    it.q0 = p.q_begin + qt * QT;
    it.qn = min(QT, p.q_begin + p.q_count - it.q0);
    int vmax = 0;
    for (int q = 0; q < it.qn; ++q) vmax = max(vmax, idx_visible(p, it.b, it.q0 + q));
    it.kt0 = 0;
    it.kt1 = (vmax + 127) / 128;
  }
  return it;
}

template <int QT, int HI, bool kFP8>
__global__ void __launch_bounds__(kIdxTcThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                  IdxTcParams p) {
  using Cfg = IdxTcCfg<QT, HI, kFP8>;
  constexpr int NS = Cfg::NSTAGE, NACC = Cfg::NACC, NCOL = Cfg::NCOL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = base;
  uint8_t* sA = sB + Cfg::B_BYTES;
  uint8_t* sRaw = sA + NS * Cfg::A_BYTES;
  float* sW = reinterpret_cast<float*>(sRaw + NS * Cfg::RAW_BYTES);
  float* sc_s = sW + 2 * QT * HI;                  // routed decode: this item's scores
  __shared__ uint64_t bar_a_full[NS], bar_a_empty[NS], bar_raw_full[NS], bar_raw_empty[NS];
  __shared__ uint64_t bar_acc_full[NACC], bar_acc_empty[NACC];
  __shared__ uint64_t bar_b_full, bar_b_empty, bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  // routed decode (bf16 keys, one query per item): the item's score
  // histogram and the routing's scratch
  constexpr bool kRoute = !kFP8 && QT == 1;
  __shared__ uint32_t hist_s[kRoute ? kHistBins : 1];
  __shared__ int route_buf[9];
  __shared__ uint32_t route_T, route_base[2];
  __shared__ int route_ok;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_a_full[s], kFP8 ? 128 : 1);
      // empty once the epilogue has seen the tile's accumulator (the MMAs
      // have read the keys): one tcgen05.commit per tile, not two
      mbar_init(&bar_a_empty[s], 128);
      mbar_init(&bar_raw_full[s], 1);
      mbar_init(&bar_raw_empty[s], 128);
    }
    for (int j = 0; j < NACC; ++j) { mbar_init(&bar_acc_full[j], 1); mbar_init(&bar_acc_empty[j], 128); }
    mbar_init(&bar_b_full, 1);
    mbar_init(&bar_b_empty, 1);
    mbar_init(&bar_done, 1);
    mbar_fence_init();
  }
  if (warp == 5) tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  griddep_wait();                                  // keys may come from this stream's compress kernel
  griddep_launch_dependents();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&qmap);
      uint32_t a_iter = 0, b_iter = 0;
      for (int id = blockIdx.x; id < p.n_items && !abort_flag; id += gridDim.x) {
        const IdxItem it = idx_item<QT>(p, id);
        if (it.kt1 <= it.kt0) continue;
        if (!mbar_wait(&bar_b_empty, (b_iter & 1) ^ 1, &abort_flag)) break;
        mbar_expect_tx(&bar_b_full, Cfg::B_BYTES);
        const int qrow = (it.b * p.nq + it.q0) * HI;
        tma_load_2d(sB, &qmap, 0, qrow, &bar_b_full);
        tma_load_2d(sB + Cfg::B_CHUNK, &qmap, 64, qrow, &bar_b_full);
        ++b_iter;
        for (int kt = it.kt0; kt < it.kt1; ++kt, ++a_iter) {
          const int s = a_iter % NS;
          const uint32_t ph = (a_iter / NS) & 1;
          const int krow = it.b * p.N + kt * 128;
          if (kFP8) {
            if (!mbar_wait(&bar_raw_empty[s], ph ^ 1, &abort_flag)) break;
            mbar_expect_tx(&bar_raw_full[s], Cfg::RAW_BYTES);
            tma_load_2d(sRaw + s * Cfg::RAW_BYTES, &kmap, 0, krow, &bar_raw_full[s]);
          } else {
            if (!mbar_wait(&bar_a_empty[s], ph ^ 1, &abort_flag)) break;
            mbar_expect_tx(&bar_a_full[s], Cfg::A_BYTES);
            tma_load_2d(sA + s * Cfg::A_BYTES, &kmap, 0, krow, &bar_a_full[s]);
            tma_load_2d(sA + s * Cfg::A_BYTES + 16384, &kmap, 64, krow, &bar_a_full[s]);
          }
        }
      }
      // drain: every issued fill has landed before the CTA may exit
      for (uint32_t i = (a_iter > NS ? a_iter - NS : 0); i < a_iter; ++i) {
        const int s = i % NS;
        const uint32_t ph = (i / NS) & 1;
        if (kFP8) mbar_wait(&bar_raw_full[s], ph, &abort_flag);
        else mbar_wait(&bar_a_full[s], ph, &abort_flag);
      }
      if (b_iter) mbar_wait(&bar_b_full, (b_iter - 1) & 1, &abort_flag);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, NCOL, 0, 0);
      uint32_t a_iter = 0, b_iter = 0, acc_iter = 0;
      const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
      for (int id = blockIdx.x; id < p.n_items && !abort_flag; id += gridDim.x) {
        const IdxItem it = idx_item<QT>(p, id);
        if (it.kt1 <= it.kt0) continue;
        if (!mbar_wait(&bar_b_full, b_iter & 1, &abort_flag)) break;
        ++b_iter;
        for (int kt = it.kt0; kt < it.kt1; ++kt, ++a_iter, ++acc_iter) {
          const int s = a_iter % NS;
          const uint32_t ph = (a_iter / NS) & 1;
          const int j = acc_iter % NACC;
          const uint32_t aph = (acc_iter / NACC) & 1;
          if (!mbar_wait(&bar_a_full[s], ph, &abort_flag)) break;
          if (!mbar_wait(&bar_acc_empty[j], aph ^ 1, &abort_flag)) break;
          tc_fence_after();
          const uint32_t d = tmem + j * NCOL;
#pragma unroll
          for (int kc = 0; kc < 2; ++kc)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_bf16(d, umma_desc_kmajor(sA0 + s * Cfg::A_BYTES + kc * 16384 + ks * 32),
                        umma_desc_kmajor(sB0 + kc * Cfg::B_CHUNK + ks * 32), idesc, (kc | ks) != 0);
          umma_commit(&bar_acc_full[j]);
        }
        umma_commit(&bar_b_empty);
      }
      umma_commit(&bar_done);
      mbar_wait(&bar_done, 0, &abort_flag);
    }
  } else if (kFP8 && warp >= 6) {
    // ------------------------------------------------------------ e4m3 -> bf16
    {
      const int ct = threadIdx.x - 192;                 // 0..127
      uint32_t a_iter = 0;
      for (int id = blockIdx.x; id < p.n_items && !abort_flag; id += gridDim.x) {
        const IdxItem it = idx_item<QT>(p, id);
        for (int kt = it.kt0; kt < it.kt1; ++kt, ++a_iter) {
          const int s = a_iter % NS;
          const uint32_t ph = (a_iter / NS) & 1;
          if (!mbar_wait(&bar_raw_full[s], ph, &abort_flag)) break;
          if (!mbar_wait(&bar_a_empty[s], ph ^ 1, &abort_flag)) break;
          const uint8_t* raw = sRaw + s * Cfg::RAW_BYTES;
          uint8_t* dst = sA + s * Cfg::A_BYTES;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int piece = ct + 128 * i;             // 16-byte piece of the raw tile
            const int row = piece >> 3, pin = piece & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(raw + piece * 16);
            const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
            uint4 o0, o1;
            o0.x = e4m3x2_to_bf16x2(h[0]); o0.y = e4m3x2_to_bf16x2(h[1]);
            o0.z = e4m3x2_to_bf16x2(h[2]); o0.w = e4m3x2_to_bf16x2(h[3]);
            o1.x = e4m3x2_to_bf16x2(h[4]); o1.y = e4m3x2_to_bf16x2(h[5]);
            o1.z = e4m3x2_to_bf16x2(h[6]); o1.w = e4m3x2_to_bf16x2(h[7]);
            // elements pin*16 .. pin*16+15 of the row: chunk pin/4, bytes (pin%4)*32 ..
            uint8_t* chunk = dst + (pin >> 2) * 16384;
            const int byte = (pin & 3) * 32;
            *reinterpret_cast<uint4*>(chunk + sw128_offset(row, byte)) = o0;
            *reinterpret_cast<uint4*>(chunk + sw128_offset(row, byte + 16)) = o1;
          }
          fence_proxy_async_smem();
          mbar_arrive(&bar_a_full[s]);
          mbar_arrive(&bar_raw_empty[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: warps 0-3 (and 6-9)
    // group eg (bf16 keys: eg = 1 for warps 6-9) takes the tiles of parity eg
    // (one group takes every tile when the keys are e4m3)
    constexpr int kGroups = kFP8 ? 1 : 2;
    const int eg = warp >= 6 ? 1 : 0;
    const int quad = warp & 3;                          // TMEM lane quarter of this warp
    const int et = quad * 32 + lane;                    // key lane 0..127
    const int ept = eg * 128 + et;                      // 0..255 over both groups (bf16 keys)
    float* sWg = sW + eg * QT * HI;
    uint32_t acc_iter = 0;
    bool stop = false;                                  // uniform over the group's 128 threads
    const bool route = kRoute && p.route;               // (then both groups: 256 threads)
    if (route) {
      for (int i = ept; i < kHistBins; i += 256) hist_s[i] = 0u;
      epi_sync256();
    }
    for (int id = blockIdx.x; id < p.n_items && !stop; id += gridDim.x) {
      const IdxItem it = idx_item<QT>(p, id);
      if (it.kt1 <= it.kt0) {
        // an empty item still counts for its row
        if (route) idx_route(p, ept, it.b * p.q_count + (it.q0 - p.q_begin), 0, 0, 0, sc_s, route_buf, &route_T,
                             &route_ok, route_base, &abort_flag);
        continue;
      }
      group_sync(1 + eg);
      for (int x = et; x < QT * HI; x += 128) {
        const int q = x / HI;
        sWg[x] = q < it.qn ? p.w[((int64_t)it.b * p.nq + it.q0 + q) * HI + (x % HI)] : 0.f;
      }
      group_sync(1 + eg);
      int vq[QT];
#pragma unroll
      for (int q = 0; q < QT; ++q) vq[q] = q < it.qn ? idx_visible(p, it.b, it.q0 + q) : 0;
      for (int kt = it.kt0; kt < it.kt1; ++kt, ++acc_iter) {
        if (kGroups == 2 && (int)(acc_iter & 1u) != eg) continue;
        const int j = acc_iter % NACC;
        const uint32_t aph = (acc_iter / NACC) & 1;
        if (!mbar_wait_group(1 + eg, &bar_acc_full[j], aph, &abort_flag)) { stop = true; break; }
        mbar_arrive(&bar_a_empty[acc_iter % NS]);       // the tile's key stage is free
        tc_fence_after();
        const int key = kt * 128 + et;
        float scale = 1.f;
        if (kFP8 && key < p.N) scale = __ldg(p.kI_scale + (int64_t)it.b * p.N + key);
        const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + j * NCOL;
#pragma unroll
        for (int q = 0; q < QT; ++q) {
          // the query's HI columns in flight together, one wait
          float v[HI / 32][32];
#pragma unroll
          for (int c = 0; c < HI / 32; ++c) tmem_ld32(tbase + q * HI + c * 32, v[c]);
          tmem_wait_ld();
          float acc = 0.f;
          const float* wq = sWg + q * HI;
#pragma unroll
          for (int c = 0; c < HI / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) acc = fmaf(wq[c * 32 + e], fmaxf(v[c][e], 0.f), acc);
          if (key < vq[q]) {
            if (route) {
              sc_s[(kt - it.kt0) * 128 + et] = acc;
              atomicAdd(&hist_s[order_key(acc) >> kHistShift], 1u);
            } else {
              p.scores[((int64_t)it.b * p.q_count + (it.q0 + q - p.q_begin)) * p.score_row_stride + key] =
                  acc * scale;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar_acc_empty[j]);
      }
      if (route) {
        // both groups are done with the item: its histogram into the row's,
        // then every item of the row routes its own keys
        if (epi_any256(stop)) break;
        uint32_t* gh = p.hist + (int64_t)(it.b * p.q_count + (it.q0 - p.q_begin)) * kHistBins;
        for (int i = ept; i < kHistBins; i += 256) {
          const uint32_t c = hist_s[i];
          if (c) { atomicAdd(gh + i, c); hist_s[i] = 0; }
        }
        idx_route(p, ept, it.b * p.q_count + (it.q0 - p.q_begin), it.kt0 * 128, (it.kt1 - it.kt0) * 128, vq[0], sc_s,
                  route_buf, &route_T, &route_ok, route_base, &abort_flag);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}


}  // namespace csahca
