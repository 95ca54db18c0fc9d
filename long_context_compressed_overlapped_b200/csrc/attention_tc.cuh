// Sink attention on the tensor cores ("Paper Breakdown: DeepSeek-V4", section
// 4: MQA core attention over selected compressed entries (CSA) or every
// visible entry (HCA), plus the uncompressed sliding window and a per-head
// sink; query RMSNorm and partial RoPE; "Inside DeepSeek V4", "Local window").
//
// MQA: all H heads of a query share the key rows, and K = V.  Both products
// are written transposed so that every MMA has M = 128 and one operand copy
// serves both:
//   S^T [128 keys x H]  = K [128 keys x D]  . Q^T      (A = key tile, K-major)
//   O^T [D x H]        += V^T [D x 128 keys] . P^T     (A = the SAME key tile
//                                                       read MN-major; B = P^T)
// S^T lives in TMEM (H columns); O^T in TMEM as D/128 M-tiles of H columns.
// Thread i of the 4 softmax warps owns key slot i of S^T and dim slot i of
// each O^T M-tile.  Per-head max and sum over the 128 keys are warp
// transpose-reductions (62 shuffles) plus a 4-way shared-memory step; the
// running max is raised lazily (only when a head's tile max exceeds it by
// more than 2^8), so O^T is rescaled in TMEM rarely.
//
// Roles (384 threads): warps 0-7 query prologue, softmax and epilogue in two
// groups of four warps, group g owning heads [32g, 32g + 32); warps 8 and 9
// load key tiles (cp.async gathers of selected rows, 2D TMA tiles of
// contiguous rows); warp 10 issues the S MMAs and owns TMEM, warp 11 the P.V
// MMAs.  Key tiles arrive in 8 chunks of
// 64 dims with their own barriers, so the score MMAs of a chunk start as soon
// as it lands; the whole tile is released by the one commit that ends its
// P.V (a tcgen05.commit costs the tensor pipe a few hundred cycles, so each
// MMA issuer commits once per tile).
//
// Work items: prefill = one query (all its tiles, final output); decode = one
// query x a range of its tiles (partial max / sum / O for the combine).
#pragma once
#include "tc_common.cuh"

namespace csahca {

// Warps 0-7 softmax (two head groups), then the producer warps, then the S
// and P.V MMA issuers.  Decode: 2 producers (384 threads).  Prefill: 16
// producers (896 threads, the last two warps idle): a gather of selected rows
// from L2 runs at a few B/cycle per issuing warp and the prefill attention is
// bound by it.  Its registers are split per warpgroup (setmaxnreg, one role per
// warpgroup, launched at 72 a thread): softmax warpgroups 0-1, producer
// warpgroups 2-5, and warpgroup 6 (the two MMA issuers and two idle warps).
template <bool kDecode> __host__ __device__ constexpr int attn_producers() { return kDecode ? 2 : 16; }
template <bool kDecode> __host__ __device__ constexpr int attn_threads() { return kDecode ? 32 * 12 : 32 * 28; }
constexpr int kAttnRegsSoftmax = 128;   // prefill: warps 0-7
constexpr int kAttnRegsProducer = 48;   // prefill: warps 8-23
constexpr int kAttnRegsMma = 56;        // prefill: warps 24-27
__host__ __device__ constexpr int attn_prefill_regs_needed() {
  return 256 * kAttnRegsSoftmax + 512 * kAttnRegsProducer + 128 * kAttnRegsMma;
}
static_assert(attn_prefill_regs_needed() <= 72 * 896, "the prefill register split fits a 72-register launch");
constexpr int kAttnH = 64;          // heads (MMA N of both products)
constexpr int kAttnD = 512;         // head dim
constexpr int kAttnChunks = kAttnD / 64;
constexpr int kAttnMT = kAttnD / 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct AttnTcParams {
  const __nv_bfloat16* q; const float* q_gain; const float* sinks; const int* pos;
  const __nv_bfloat16* kv_comp_ptr;  // [B * N, D] compressed rows (gather source)
  const __nv_bfloat16* win_ptr;      // window rows (the window tensor map's memory)
  int64_t comp_rows_total, win_rows_total;   // rows behind kv_comp_ptr / win_ptr
  int q_norm; float eps; float scale_log2; int rope_dims; double rope_base;
  int B, nq, N, m, k, w;
  int csa;                      // 1: keys = idx rows; 0: every visible entry
  const int* idx;               // [B, nq, k]
  int decode;                   // window = ring [B, w, d] (decode) or finished rows [B, nq, d]
  int n_items, splits, tiles_per_split;
  int gtile;                    // CSA: selected rows per tile (128, 64 or 32); rows gtile..127 stay zero
  int first_kernel;             // 1: the call's first kernel (inputs are read only after the wait)
  __nv_bfloat16* out;           // final [B, nq, H, D]
  float* partial;               // [B, nq, H, splits, D + 4]
  double theta[64];             // base^(-2j/r) per rope pair j (r <= 128), filled on the host
  // FP8 KV rows (decode): codes of the non-RoPE dims, RoPE dims bf16, one fp32
  // scale per 64 dims (the header's layout), kv_row_bytes per row
  const uint8_t* kv_f8;
  int64_t kv_row_bytes;
  int f8_nope_chunks;           // (D - rope_dims) / 64 chunks of e4m3 codes
  // context parallelism (decode): the cache holds global entries entry_base ..
  // entry_base + N - 1; skip_window leaves the window to another rank
  int entry_base;
  int skip_window;
};

struct AttnItem { int b, qi, t, tile0, tile1, split, ncomp_tiles, nwin_tiles; };
struct AttnTile { int src; int row0; int lo, hi; int list_off; };   // src 0 gather, 1 comp rows, 2 window rows

__device__ __forceinline__ int attn_visible(const AttnTcParams& p, int t) {
  return visible_count(t, p.m, p.N, p.entry_base);
}

template <bool kDecode>
__device__ __forceinline__ AttnItem attn_item(const AttnTcParams& p, int id) {
  AttnItem it;
  int qid;
  if (kDecode) { qid = id / p.splits; it.split = id % p.splits; }
  else {
    // HCA prefill: latest queries (most tiles) first; CSA: all alike.
    qid = p.csa ? id : (p.n_items - 1 - id);
    it.split = 0;
  }
  it.b = qid / p.nq;
  it.qi = qid % p.nq;
  it.t = kDecode ? p.pos[it.b] : it.qi;
  it.ncomp_tiles = p.csa ? (p.k + p.gtile - 1) / p.gtile : (attn_visible(p, it.t) + 127) / 128;
  it.nwin_tiles = p.skip_window ? 0 : (p.w + 127) / 128;
  const int total = it.ncomp_tiles + it.nwin_tiles;
  if (kDecode) {
    it.tile0 = it.split * p.tiles_per_split;
    it.tile1 = min(total, it.tile0 + p.tiles_per_split);
  } else {
    it.tile0 = 0;
    it.tile1 = total;
  }
  return it;
}

template <bool kDecode>
__device__ __forceinline__ AttnTile attn_tile(const AttnTcParams& p, const AttnItem& it, int tile) {
  AttnTile T;
  if (tile < it.ncomp_tiles) {
    if (p.csa) {
      T.src = 0;
      T.list_off = tile * p.gtile;
      T.row0 = 0;
      T.lo = 0;
      T.hi = min(p.gtile, p.k - T.list_off);
    } else {
      T.src = 1;
      T.row0 = it.b * p.N + tile * 128;
      T.lo = 0;
      T.hi = min(128, attn_visible(p, it.t) - tile * 128);
      T.list_off = 0;
    }
  } else {
    const int wt = tile - it.ncomp_tiles;
    T.src = 2;
    T.list_off = 0;
    if (kDecode) {
      // ring slots [wt*128, wt*128 + 128); slot s is valid iff it holds a
      // position in [pos - w + 1, pos] that is >= 0
      T.row0 = it.b * p.w + wt * 128;
      T.lo = 0;
      const int nslot = min(128, p.w - wt * 128);
      T.hi = (it.t >= p.w - 1) ? nslot : max(0, min(nslot, it.t + 1 - wt * 128));
    } else {
      // positions [t - w + 1 + wt*128, ...] clipped to [0, t]
      const int p0 = it.t - p.w + 1 + wt * 128;
      T.row0 = it.b * p.nq + p0;
      T.lo = p0 < 0 ? -p0 : 0;
      T.hi = min(128, min(p.w - wt * 128, it.t - p0 + 1));
    }
  }
  return T;
}

// Named barrier 3 over the 256 softmax threads (both head groups).
__device__ __forceinline__ void softmax_sync256() { asm volatile("bar.sync 3, 256;" ::: "memory"); }
__device__ __forceinline__ bool softmax_any256(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 3, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool softmax_all256(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 3, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
// OR of v over the 128 threads of named barrier `id`.
__device__ __forceinline__ bool group_any(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

// 32 per-thread values (one per head of the group) -> per-head reduction over
// the group's 128 key slots: a warp transpose-reduction (31 shuffles) leaves
// head `lane` in lane `lane`, then the 4 warps combine through shared memory.
// red: 4 x 32 floats of this group; out: the group's 32 heads.  kMax: max,
// else sum.  Ends with a group barrier.
template <bool kMax>
__device__ __forceinline__ void reduce_group32(float (&v)[32], float* red, float* out, int gid) {
  const int lane = threadIdx.x & 31, wq = (threadIdx.x >> 5) & 3;
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
  group_sync(gid);
  if ((threadIdx.x & 127) < 32) {
    const int h = threadIdx.x & 31;
    float r = red[h];
#pragma unroll
    for (int w = 1; w < 4; ++w) r = kMax ? fmaxf(r, red[w * 32 + h]) : r + red[w * 32 + h];
    out[h] = r;
  }
  group_sync(gid);
}

struct AttnSmem {
  static constexpr int Q_CHUNK = kAttnH * 128;               // 8 KB
  static constexpr int Q_BYTES = kAttnChunks * Q_CHUNK;      // 64 KB
  static constexpr int K_CHUNK = 128 * 128;                  // 16 KB
  static constexpr int K_BYTES = kAttnChunks * K_CHUNK;      // 128 KB
  static constexpr int P_BYTES = 128 * 128;                  // 16 KB
  static constexpr int TOTAL = 1024 + Q_BYTES + K_BYTES + P_BYTES;
  static constexpr int F8_SCALES = 128 * 32;                 // FP8 rows: 8 scale slots per key row
};

// Decode partial of one (query, split): m[H], l[H] fp32, then O / l bf16 [D][H].
// O / l is a convex combination of bf16 value rows, so bf16 (fp32's exponent
// range) holds it whatever the rows' magnitude; the combine's output is
// rounded to bf16 as well, so the partial adds one rounding of the same size.
constexpr int kTcHdrFloats = 2 * kAttnH;
constexpr int kTcPartialHeader = kTcHdrFloats * 4;
constexpr int kTcPartialBytes = kTcPartialHeader + kAttnD * kAttnH * 2;
// The same blocks seen as 128-byte rows (64 bf16), as the TMA store writes them.
constexpr int kTcPartialRows = kTcPartialBytes / 128;
constexpr int kTcPartialHeaderRows = kTcPartialHeader / 128;
static_assert(kTcPartialBytes % 128 == 0 && kTcPartialHeader % 128 == 0, "partial blocks are whole 128-byte rows");

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 16 e4m3 codes (codes[i] in byte i) times the block scale -> 16 bf16 at
// dims 16q .. 16q+15 of row `row` of a 64-dim SW128 chunk.
__device__ __forceinline__ void f8_piece_to_bf16(uint8_t* chunk, int row, int q, uint4 codes, float scale) {
  const uint16_t* h = reinterpret_cast<const uint16_t*>(&codes);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(h[i]),
                                                                      __NV_E4M3)));
    w[i] = pack_bf16x2(f.x * scale, f.y * scale);
  }
  *reinterpret_cast<uint4*>(chunk + sw128_offset(row, 32 * q)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(chunk + sw128_offset(row, 32 * q + 16)) = make_uint4(w[4], w[5], w[6], w[7]);
}

// kF8 (decode only): the compressed rows are FP8 KV rows.  The producers
// bring each 64-dim chunk's e4m3 codes (64 bytes per row) into the upper half
// of the chunk's slot, the RoPE chunks (bf16) straight into their slots, and
// the rows' block scales into a staging area; the softmax warps, idle until
// the tile's scores, convert the codes in place to the bf16 SW128 rows the
// MMAs read (every code is read into registers before any row is written).
// comp_rows then maps the rows' bytes with a 64 x 128 box; f8_rope (128 x 128,
// 128-byte swizzle) and f8_scale (32 x 128) map the same bytes.
template <bool kDecode, bool kF8 = false>
__global__ void __launch_bounds__(attn_threads<kDecode>(), 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap comp_rows, const __grid_constant__ CUtensorMap win_rows,
               const __grid_constant__ CUtensorMap q_rows, const __grid_constant__ CUtensorMap part_rows,
               const __grid_constant__ CUtensorMap f8_rope, const __grid_constant__ CUtensorMap f8_scale,
               const __grid_constant__ AttnTcParams p) {
  static_assert(kDecode || !kF8, "FP8 KV rows are a decode cache format");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + AttnSmem::Q_BYTES;
  uint8_t* sP = sK + AttnSmem::K_BYTES;
  float* sScale = reinterpret_cast<float*>(sP + AttnSmem::P_BYTES);   // kF8: [128 rows][8]
  __shared__ uint64_t bar_kfull[kAttnChunks];
  __shared__ uint64_t bar_raw[kF8 ? kAttnChunks : 1], bar_raw_s;    // kF8: codes / scales landed
  // bar_pv: the tile's P.V MMAs have completed (its key buffer is free, O^T
  // and P^T may be touched again)
  __shared__ uint64_t bar_q_raw, bar_q_empty, bar_q_full, bar_s_full, bar_s_empty, bar_p_full, bar_pv, bar_done;
  // prefill: bar_pvm[j], the tile's P.V MMAs of O^T M-tiles 0..j have completed
  // (key chunks 2j, 2j + 1 are free), j < 3; M-tile 3 completes bar_pv
  __shared__ uint64_t bar_pvm[kAttnMT - 1];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ float red[2][4 * 32];
  __shared__ __align__(16) float stat_a[kAttnH];
  __shared__ __align__(16) float m_use[kAttnH];
  __shared__ __align__(16) float sc_h[kAttnH];     // softmax scale of head h (log2 units, times inv_rms_h)
  __shared__ __align__(16) float alpha[kAttnH];
  __shared__ float l_run[kAttnH];
  __shared__ float rope_cs[64], rope_sn[64];
  __shared__ double theta_s[64];                   // RoPE frequency of pair j
  __shared__ __align__(16) float gain_s[kAttnD];
  __shared__ int rows_s[kDecode ? attn_producers<kDecode>() : 1][128];   // decode: each producer's rows
  __shared__ int need_rescale[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kNP = attn_producers<kDecode>();
  constexpr int kWarpS = 8 + kNP, kWarpPV = 9 + kNP;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    // a chunk is full once its producer warp has arrived (TMA bytes or
    // cp.async completions) and, for FP8 rows, the 256 softmax threads that
    // convert it (they arrive on every chunk of every tile)
    for (int c = 0; c < kAttnChunks; ++c) mbar_init(&bar_kfull[c], kF8 ? 32 + 256 : (kNP == 2 ? 32 : 32 * kNP));
    if constexpr (kF8) {
      for (int c = 0; c < kAttnChunks; ++c) mbar_init(&bar_raw[c], 32);
      mbar_init(&bar_raw_s, 32);
    }
    mbar_init(&bar_q_raw, 1);
    mbar_init(&bar_q_empty, 1);
    mbar_init(&bar_q_full, 256);
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_s_empty, 256);
    mbar_init(&bar_p_full, 256);
    mbar_init(&bar_pv, 1);
    if constexpr (!kDecode)
      for (int j = 0; j < kAttnMT - 1; ++j) mbar_init(&bar_pvm[j], 1);
    mbar_init(&bar_done, 2);                       // both MMA issuers
    mbar_fence_init();
  }
  if (warp == kWarpS) tmem_alloc(&tmem_base_sh, 512);
  if (p.gtile < 128) {
    // rows [gtile, 128) of the key buffer are never written by a gathered
    // tile; zeros there keep the score and P.V MMAs finite (P = 0 there)
    const int per_chunk = (128 - p.gtile) * 8;     // 16-byte pieces
    for (int x = threadIdx.x; x < kAttnChunks * per_chunk; x += blockDim.x) {
      const int c = x / per_chunk, o = x - c * per_chunk;
      *reinterpret_cast<uint4*>(sK + c * AttnSmem::K_CHUNK + p.gtile * 128 + o * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tS = tmem;                 // S^T: columns [0, H)
  const uint32_t tO = tmem + 128;           // O^T M-tile j: columns [128 + j*H, ...)
  const uint32_t tL = tmem + 128 + kAttnMT * kAttnH;   // per-key-slot partial sums of p: H columns
  // Programmatic dependent launch: every kernel of the library signals its
  // dependents only after its own wait, so when a kernel starts, all work
  // queued before its predecessor has completed and the call's inputs may be
  // read before the wait.  As the call's first kernel this one waits before
  // reading anything (query, positions, gain).
  if (p.first_kernel) {
    griddep_wait();
    griddep_launch_dependents();
  }
  static_assert(kDecode || (kNP % 4 == 0 && kWarpPV < attn_threads<kDecode>() / 32 &&
                            attn_threads<kDecode>() == 32 * (8 + kNP + 4)),
                "prefill: whole warpgroups per role (softmax, producers, MMA issuers)");

  // (the decode instance keeps this exact form of the role test: its code
  // runs once per CTA, fetched cold, and an equivalent range test compiled
  // to a layout measured 4 us slower per launch)
  if (kDecode ? (warp == 8 || warp == 9) : (warp >= 8 && warp < 8 + kNP)) {
    if constexpr (!kDecode) setmaxnreg_dec<kAttnRegsProducer>();
    // ------------------------------------------------------------ producers
    // decode, two producers: warp 8 loads chunks 0,1,4,5 (and the raw Q),
    // warp 9 chunks 2,3,6,7, and a chunk barrier expects 32 arrivals.
    // Prefill, eighteen: every producer loads its share of every chunk
    // (gathered rows: copy instruction j, rows 4j..4j+3, goes to warp j mod
    // 18, which looks its rows up once per tile into registers; contiguous
    // rows: chunk c's box is issued by warp c mod 18), and a chunk barrier
    // expects 32 x 18 arrivals; warp 8 also loads the raw Q
    const int pw = warp - 8;
    tma_prefetch_desc(&comp_rows);
    tma_prefetch_desc(&win_rows);
    tma_prefetch_desc(&q_rows);
    if constexpr (kF8) {
      tma_prefetch_desc(&f8_rope);
      tma_prefetch_desc(&f8_scale);
    }
    uint32_t tcount = 0, icount = 0;
    bool stop = false;                       // warp-uniform
    constexpr int kRowGroups = (32 + kNP - 1) / kNP;   // prefill: 4-row copy groups per warp
    int rowreg[kRowGroups];
#pragma unroll
    for (int jj = 0; jj < kRowGroups; ++jj) rowreg[jj] = 0;
    for (int id = blockIdx.x; id < p.n_items && !stop; id += gridDim.x) {
      const AttnItem it = attn_item<kDecode>(p, id);
      if (it.tile1 <= it.tile0) continue;
      if (pw == 0) {
        // raw Q of this item into the Q buffer once the previous item's
        // score MMAs have read it; roped there by the softmax warps
        int ok = 1;
        if (lane == 0) {
          ok = mbar_wait(&bar_q_empty, (icount & 1) ^ 1, &abort_flag);
          if (ok) {
            mbar_expect_tx(&bar_q_raw, AttnSmem::Q_BYTES);
            tma_load_3d(sQ, &q_rows, 0, (it.b * p.nq + it.qi) * kAttnH, 0, &bar_q_raw);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { stop = true; break; }
        ++icount;
      }
      // key rows and selections may come from earlier kernels of this stream
      griddep_wait();
      if (lane == 0 && pw == 0) griddep_launch_dependents();
      for (int tile = it.tile0; tile < it.tile1 && !stop; ++tile, ++tcount) {
        const AttnTile T = attn_tile<kDecode>(p, it, tile);
        const uint32_t ph = tcount & 1;
        if (T.src == 0) {
          // selected rows of this tile (clamped; masked later by the softmax)
          const int* L = p.idx + ((int64_t)it.b * p.nq + it.qi) * p.k + T.list_off;
          if constexpr (kNP == 2) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = lane + 32 * e;
              int v = (j < T.hi) ? __ldg(L + j) : 0;
              v = (v < 0 || v >= p.N) ? 0 : v;
              rows_s[pw][j] = it.b * p.N + v;
            }
            __syncwarp();
          } else {
            // prefill: this lane's rows, 4j + (lane >> 3) of instructions j = pw + jj * kNP
#pragma unroll
            for (int jj = 0; jj < kRowGroups; ++jj) {
              const int r = 4 * (pw + jj * kNP) + (lane >> 3);
              int v = (r < T.hi) ? __ldg(L + r) : 0;
              v = (v < 0 || v >= p.N) ? 0 : v;
              rowreg[jj] = it.b * p.N + v;
            }
          }
        }
        if constexpr (kF8) {
          // FP8 rows: the tile's block scales (32 bytes per row) by warp 8
          if (T.src != 2 && pw == 0) {
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&bar_pv, ph ^ 1, &abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { stop = true; break; }
            const int sofs = kAttnD + p.rope_dims;
            if (T.src == 0) {
              const int piece = lane & 1, rg = lane >> 1;       // 16 rows per instruction
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int r = 16 * j + rg;
                cp_async16(reinterpret_cast<uint8_t*>(sScale) + r * 32 + piece * 16,
                           p.kv_f8 + (int64_t)rows_s[pw][r] * p.kv_row_bytes + sofs + piece * 16);
              }
              cp_async_arrive_noinc(&bar_raw_s);
            } else if (lane == 0) {
              mbar_expect_tx(&bar_raw_s, AttnSmem::F8_SCALES);
              tma_load_2d(sScale, &f8_scale, sofs, T.row0, &bar_raw_s);
            } else {
              mbar_arrive(&bar_raw_s);
            }
          }
        }
        // two producers (decode): warp pw owns chunks {0,1,4,5} or {2,3,6,7};
        // more (prefill): every producer takes a share of every chunk
        constexpr int kChunksPerWarp = kNP == 2 ? kAttnChunks / 2 : kAttnChunks;
        for (int cc = 0; cc < kChunksPerWarp; ++cc) {
          const int c = kNP == 2 ? 4 * (cc >> 1) + 2 * pw + (cc & 1) : cc;
          int ok = 1;
          // prefill: a chunk pair is free once the P.V of its O^T M-tile has
          // completed, so the next tile's rows start landing during the P.V
          uint64_t* freed = (!kDecode && c / 2 < kAttnMT - 1) ? &bar_pvm[c / 2] : &bar_pv;
          if (lane == 0) ok = mbar_wait(freed, ph ^ 1, &abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) { stop = true; break; }
          uint8_t* dst = sK + c * AttnSmem::K_CHUNK;
          if constexpr (kF8) {
            if (T.src != 2) {
              if (c < p.f8_nope_chunks) {
                // e4m3 codes of chunk c, 64 bytes per row, into the slot's upper half
                uint8_t* raw = dst + AttnSmem::K_CHUNK / 2;
                if (T.src == 0) {
                  const int piece = lane & 3, rg = lane >> 2;   // 8 rows per instruction
                  const uint8_t* src = p.kv_f8 + c * 64 + piece * 16;
#pragma unroll 8
                  for (int j = 0; j < 16; ++j) {
                    const int r = 8 * j + rg;
                    cp_async16(raw + r * 64 + piece * 16, src + (int64_t)rows_s[pw][r] * p.kv_row_bytes);
                  }
                  cp_async_arrive_noinc(&bar_raw[c]);
                } else if (lane == 0) {
                  mbar_expect_tx(&bar_raw[c], AttnSmem::K_CHUNK / 2);
                  tma_load_2d(raw, &comp_rows, c * 64, T.row0, &bar_raw[c]);
                } else {
                  mbar_arrive(&bar_raw[c]);
                }
                mbar_arrive(&bar_kfull[c]);          // the bf16 rows come from the softmax warps
              } else {
                // a RoPE chunk: bf16 bytes at (D - r) + 128 (c - nope) of each row
                const int rofs = (kAttnD - p.rope_dims) + 128 * (c - p.f8_nope_chunks);
                if (T.src == 0) {
                  const int piece = lane & 7, rg = lane >> 3;
                  const uint8_t* src = p.kv_f8 + rofs + piece * 16;
#pragma unroll 8
                  for (int j = 0; j < 32; ++j) {
                    const int r = 4 * j + rg;
                    cp_async16(dst + sw128_offset(r, piece * 16), src + (int64_t)rows_s[pw][r] * p.kv_row_bytes);
                  }
                  cp_async_arrive_noinc(&bar_kfull[c]);
                } else if (lane == 0) {
                  mbar_expect_tx(&bar_kfull[c], AttnSmem::K_CHUNK);
                  tma_load_2d(dst, &f8_rope, rofs, T.row0, &bar_kfull[c]);
                } else {
                  mbar_arrive(&bar_kfull[c]);
                }
              }
              continue;
            }
          }
          if (T.src == 0) {
            // gathered rows: 8 lanes per 128-byte row segment (coalesced,
            // conflict-free), 4 rows per instruction, gtile / 4 instructions
            // per chunk; each lane arrives on the chunk's barrier when its
            // copies have landed, without waiting for them
            const int piece = lane & 7, rg = lane >> 3;
            const __nv_bfloat16* src = p.kv_comp_ptr + c * 64 + piece * 8;
            const int nj = p.gtile >> 2;
            if constexpr (kNP == 2) {
#pragma unroll 8
              for (int j = 0; j < nj; ++j) {
                const int r = 4 * j + rg;
                cp_async16(dst + sw128_offset(r, piece * 16), src + (int64_t)rows_s[pw][r] * kAttnD);
              }
            } else {
#pragma unroll
              for (int jj = 0; jj < kRowGroups; ++jj) {
                const int j = pw + jj * kNP;
                if (j < nj) {
                  const int r = 4 * j + rg;
                  cp_async16(dst + sw128_offset(r, piece * 16), src + (int64_t)rowreg[jj] * kAttnD);
                }
              }
            }
            cp_async_arrive_noinc(&bar_kfull[c]);
          } else {
            // contiguous rows: one 16 KB box per chunk, so the score MMAs of
            // a chunk start as soon as it lands
            if (lane == 0 && (kNP == 2 || c % kNP == pw)) {
              mbar_expect_tx(&bar_kfull[c], AttnSmem::K_CHUNK);
              tma_load_3d(dst, T.src == 1 ? &comp_rows : &win_rows, 0, T.row0, c, &bar_kfull[c]);
            } else {
              mbar_arrive(&bar_kfull[c]);
            }
          }
        }
        // L2 prefetch of the next tile's rows, queued after this tile's
        // loads: HBM streams while this tile is processed, and the next
        // tile's loads hit L2.  Contiguous rows: one bulk prefetch (an SM
        // completes about one TMA op per 580 cycles, so not one per chunk);
        // gathered rows: line prefetches from the lanes (no TMA op per row)
        if (!stop && pw == 0 && tile + 1 < it.tile1) {
          const AttnTile Tn = attn_tile<kDecode>(p, it, tile + 1);
          if (Tn.src == 0) {
            const int* L = p.idx + ((int64_t)it.b * p.nq + it.qi) * p.k + Tn.list_off;
            for (int j = lane >> 3; j < Tn.hi; j += 4) {
              const int v = __ldg(L + j);
              if (v >= 0 && v < p.N) {
                if constexpr (kF8) {
                  if ((lane & 7) * 128 < p.kv_row_bytes)
                    prefetch_l2_line(p.kv_f8 + ((int64_t)it.b * p.N + v) * p.kv_row_bytes + (lane & 7) * 128);
                } else {
                  prefetch_l2_line(p.kv_comp_ptr + ((int64_t)it.b * p.N + v) * kAttnD + (lane & 7) * 64);
                }
              }
            }
          } else if (lane == 0 && Tn.row0 >= 0) {
            const int64_t total = Tn.src == 1 ? p.comp_rows_total : p.win_rows_total;
            const int64_t rows = min((int64_t)128, total - Tn.row0);
            if (rows > 0) {
              if (kF8 && Tn.src == 1)
                bulk_prefetch_l2(p.kv_f8 + Tn.row0 * p.kv_row_bytes, (uint32_t)(rows * p.kv_row_bytes));
              else
                bulk_prefetch_l2((Tn.src == 1 ? p.kv_comp_ptr : p.win_ptr) + (int64_t)Tn.row0 * kAttnD,
                                 (uint32_t)(rows * kAttnD * 2));
            }
          }
        }
      }
    }
    // drain the last loads before the CTA may exit: the last tile's chunk
    // barriers complete only once every producer lane's copies have landed
    // (the gathers are not committed to cp.async groups, so the group wait
    // orders nothing; this form of the drain measured fastest in decode)
    cp_async_wait<0>();
    if (lane == 0 && tcount > 0)
      for (int c = 0; c < kAttnChunks; ++c) mbar_wait(&bar_kfull[c], (tcount - 1) & 1, &abort_flag);
    if (pw == 0 && lane == 0 && icount > 0) mbar_wait(&bar_q_raw, (icount - 1) & 1, &abort_flag);
  } else if (warp >= kWarpS) {
    if constexpr (!kDecode) setmaxnreg_dec<kAttnRegsMma>();
    if (warp == kWarpS) {
    // ------------------------------------------------------------ S MMA issuer
    // (a separate thread issues the P.V MMAs, so the S MMAs of tile t+1 go out
    // while those of P.V(t) still do)
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, kAttnH, 0, 0);
      // base descriptors; chunk / K-step offsets are adds in 16-byte units
      const uint64_t kdesc = umma_desc_kmajor(smem_u32(sK)), qdesc = umma_desc_kmajor(smem_u32(sQ));
      uint32_t tcount = 0, icount = 0;
      bool stop = false;
      for (int id = blockIdx.x; id < p.n_items && !stop && !abort_flag; id += gridDim.x) {
        const AttnItem it = attn_item<kDecode>(p, id);
        if (it.tile1 <= it.tile0) continue;
        if (!mbar_wait(&bar_q_full, icount & 1, &abort_flag)) break;
        ++icount;
        for (int tile = it.tile0; tile < it.tile1 && !stop; ++tile, ++tcount) {
          const uint32_t ph = tcount & 1;
          if (!mbar_wait(&bar_s_empty, ph ^ 1, &abort_flag)) { stop = true; break; }
          tc_fence_after();
          for (int c = 0; c < kAttnChunks; ++c) {
            if (!mbar_wait(&bar_kfull[c], ph, &abort_flag)) { stop = true; break; }
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t kd = kdesc + (uint64_t)(c * (AttnSmem::K_CHUNK >> 4));
            const uint64_t qd = qdesc + (uint64_t)(c * (AttnSmem::Q_CHUNK >> 4));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) umma_bf16(tS, kd + 2 * ks, qd + 2 * ks, idesc_s, (c | ks) != 0);
          }
          if (stop) break;
          umma_commit(&bar_s_full);
          if (tile == it.tile1 - 1) umma_commit(&bar_q_empty);
        }
      }
      umma_commit(&bar_done);
      mbar_wait(&bar_done, 0, &abort_flag);
    }
    } else if (warp == kWarpPV) {
    // ------------------------------------------------------------ P.V MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, kAttnH, 1, 1);
      const uint64_t vdesc = umma_desc_mnmajor(smem_u32(sK), AttnSmem::K_CHUNK);
      const uint64_t pdesc = umma_desc_mnmajor(smem_u32(sP), AttnSmem::P_BYTES);
      uint32_t tcount = 0;
      bool stop = false;
      for (int id = blockIdx.x; id < p.n_items && !stop && !abort_flag; id += gridDim.x) {
        const AttnItem it = attn_item<kDecode>(p, id);
        for (int tile = it.tile0; tile < it.tile1; ++tile, ++tcount) {
          const uint32_t ph = tcount & 1;
          if (!mbar_wait(&bar_p_full, ph, &abort_flag)) { stop = true; break; }
          tc_fence_after();
          const bool first = tile == it.tile0;
          // key steps past the tile's last valid row hold P = 0 and are skipped
          const int hi = attn_tile<kDecode>(p, it, tile).hi;
          const int nks = hi <= 16 ? 1 : min(8, (hi + 15) >> 4);
          if (nks == 8) {
#pragma unroll
            for (int mt = 0; mt < kAttnMT; ++mt) {
              const uint64_t vd = vdesc + (uint64_t)((2 * mt) * (AttnSmem::K_CHUNK >> 4));
#pragma unroll
              for (int ks = 0; ks < 8; ++ks)
                umma_bf16(tO + mt * kAttnH, vd + 128 * ks, pdesc + 128 * ks, idesc_pv, !(first && ks == 0));
              if (!kDecode && mt < kAttnMT - 1) umma_commit(&bar_pvm[mt]);
            }
          } else {
#pragma unroll
            for (int mt = 0; mt < kAttnMT; ++mt) {
              const uint64_t vd = vdesc + (uint64_t)((2 * mt) * (AttnSmem::K_CHUNK >> 4));
              for (int ks = 0; ks < nks; ++ks)
                umma_bf16(tO + mt * kAttnH, vd + 128 * ks, pdesc + 128 * ks, idesc_pv, !(first && ks == 0));
              if (!kDecode && mt < kAttnMT - 1) umma_commit(&bar_pvm[mt]);
            }
          }
          umma_commit(&bar_pv);
        }
      }
      umma_commit(&bar_done);
      mbar_wait(&bar_done, 0, &abort_flag);
    }
    }
  } else if (warp < 8) {
    if constexpr (!kDecode) setmaxnreg_inc<kAttnRegsSoftmax>();
    // ------------------------------------------------------------ softmax / epilogue
    // Two groups of 4 warps; group g owns heads [32g, 32g + 32): its columns
    // of S^T, O^T and the row sums in TMEM, and its 64 bytes of each P^T row.
    // Thread tid of a group is key slot tid of a tile and dim slot tid of
    // each O^T M-tile (TMEM lane).
    const int g = warp >> 2;
    const int gid = 1 + g;                   // the group's named barrier
    const int tid = threadIdx.x & 127;
    const int st = threadIdx.x;              // 0..255 over both groups
    const int h0 = 32 * g;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t tcount = 0, qcount = 0, f8count = 0;
    const int r0 = kAttnD - p.rope_dims;
    // q gain (same for every head and query) staged once in shared memory;
    // an all-ones gain (or none) leaves the non-rope dims of q untouched
    bool ones = true;
    for (int x = st; x < kAttnD; x += 256) {
      const float gv = (p.q_norm && p.q_gain) ? __ldg(p.q_gain + x) : 1.f;
      gain_s[x] = gv;
      ones = ones && gv == 1.f;
    }
    if (st < p.rope_dims / 2) theta_s[st] = p.theta[st];
    const bool gain_ones = softmax_all256(ones);
    for (int id = blockIdx.x; id < p.n_items; id += gridDim.x) {
      const AttnItem it = attn_item<kDecode>(p, id);
      const bool empty = it.tile1 <= it.tile0;
      bool bad = false;                      // uniform over the group; both groups leave together
      // ---- query prologue.  RoPE is linear and the RMSNorm factor is one
      // scalar per head, so RoPE_t(RMSNorm(q) * g) = inv_rms_h * RoPE_t(q * g):
      // the MMA operand is RoPE_t(q * g) (with an all-ones gain only the rope
      // dims are rewritten), and inv_rms_h joins the softmax scale of head h.
      if (!empty) {
        if (st < p.rope_dims / 2) {
          float cs, sn;
          rope_sincos((double)it.t, theta_s[st], &cs, &sn);
          rope_cs[st] = cs;
          rope_sn[st] = sn;
        }
        if (st < kAttnH) m_use[st] = -INFINITY;
        // (the 256-thread reduction also publishes rope_cs / rope_sn)
        bad = !softmax_all256(mbar_wait(&bar_q_raw, qcount & 1, &abort_flag));
        ++qcount;
        if (!bad) {
          // thread (head h, quarter qq) owns dims [128 qq, 128 qq + 128) of row h
          const int h = st >> 2, qq = st & 3;
          float ss = 0.f;
          if (!gain_ones) {
            // q * g on every dim (sum of squares from the raw values), RoPE on the rope dims
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              const int chunk = 2 * qq + c;
              uint8_t* row = sQ + chunk * AttnSmem::Q_CHUNK;
#pragma unroll
              for (int pc = 0; pc < 8; ++pc) {
                uint4* a = reinterpret_cast<uint4*>(row + sw128_offset(h, pc * 16));
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
                const int d0 = chunk * 64 + pc * 8;
#pragma unroll
                for (int e = 0; e < 8; ++e) { ss = fmaf(x[e], x[e], ss); x[e] *= gain_s[d0 + e]; }
                if (d0 + 7 >= r0) {
#pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    if (d0 + e >= r0) {
                      const int j = (d0 + e - r0) >> 1;
                      const float x0 = x[e], x1 = x[e + 1];
                      x[e] = x0 * rope_cs[j] - x1 * rope_sn[j];
                      x[e + 1] = x0 * rope_sn[j] + x1 * rope_cs[j];
                    }
                  }
                }
                uint4 o;
                store16(reinterpret_cast<__nv_bfloat16*>(&o), x);
                *a = o;
              }
            }
          } else {
            // RoPE on the rope dims only: pairs (r0 + 2j, r0 + 2j + 1), this
            // thread taking j = qq, qq + 4, ...
            for (int j = qq; j < p.rope_dims / 2; j += 4) {
              const int dim = r0 + 2 * j;
              __nv_bfloat162* a = reinterpret_cast<__nv_bfloat162*>(sQ + (dim >> 6) * AttnSmem::Q_CHUNK +
                                                                     sw128_offset(h, (dim & 63) * 2));
              const float2 f = __bfloat1622float2(*a);
              *a = __floats2bfloat162_rn(f.x * rope_cs[j] - f.y * rope_sn[j], f.x * rope_sn[j] + f.y * rope_cs[j]);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&bar_q_full);
          if (p.q_norm) {
            if (gain_ones) {
              // the rotation keeps every pair's norm: sum the squares of the
              // operand once every pair is rotated (the MMAs already run)
              softmax_sync256();
#pragma unroll 1
              for (int c = 0; c < 2; ++c) {
                const uint8_t* row = sQ + (2 * qq + c) * AttnSmem::Q_CHUNK;
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                  const uint4 raw = *reinterpret_cast<const uint4*>(row + sw128_offset(h, pc * 16));
                  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h2[i]);
                    ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                  }
                }
              }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            if (qq == 0) sc_h[h] = p.scale_log2 * rsqrtf(ss / (float)kAttnD + p.eps);
          } else if (qq == 0) {
            sc_h[h] = p.scale_log2;
          }
        }
      }
      softmax_sync256();                     // sc_h, m_use complete
      griddep_wait();                        // selections read, outputs written below

      const float4* sc4 = reinterpret_cast<const float4*>(sc_h + h0);
      const float4* mu4 = reinterpret_cast<const float4*>(m_use + h0);
      for (int tile = it.tile0; tile < it.tile1; ++tile, ++tcount) {
        if constexpr (kF8) {
          // FP8 rows: both groups convert the tile's e4m3 chunks to bf16 in
          // place (a give-up seen by either group ends it for both), and
          // arrive on every chunk of every tile
          const AttnTile Tc = attn_tile<kDecode>(p, it, tile);
          const bool f8 = Tc.src != 2;
          bool cbad = softmax_any256(bad);
          if (!cbad && f8) cbad = !softmax_all256(mbar_wait(&bar_raw_s, f8count & 1, &abort_flag));
          for (int c = 0; c < kAttnChunks; ++c) {
            if (!cbad && f8 && c < p.f8_nope_chunks) {
              cbad = !softmax_all256(mbar_wait(&bar_raw[c], f8count & 1, &abort_flag));
              if (!cbad) {
                uint8_t* slot = sK + c * AttnSmem::K_CHUNK;
                const uint8_t* raw = slot + AttnSmem::K_CHUNK / 2;
                // piece pc = 16 codes: row pc / 4, quarter pc % 4 (raw + 64 row + 16 quarter)
                const int pc0 = st, pc1 = st + 256;
                const uint4 in0 = *reinterpret_cast<const uint4*>(raw + pc0 * 16);
                const uint4 in1 = *reinterpret_cast<const uint4*>(raw + pc1 * 16);
                const float s0 = sScale[(pc0 >> 2) * 8 + c], s1 = sScale[(pc1 >> 2) * 8 + c];
                softmax_sync256();                   // every code read before any row is written
                f8_piece_to_bf16(slot, pc0 >> 2, pc0 & 3, in0, s0);
                f8_piece_to_bf16(slot, pc1 >> 2, pc1 & 3, in1, s1);
                fence_proxy_async_smem();
              }
            }
            mbar_arrive(&bar_kfull[c]);
          }
          if (f8) ++f8count;
          bad = bad || cbad;
        }
        if (bad) continue;
        const uint32_t ph = tcount & 1;
        const bool first = tile == it.tile0;
        const AttnTile T = attn_tile<kDecode>(p, it, tile);
        bool valid = tid >= T.lo && tid < T.hi;
        if (valid && T.src == 0) {
          const int e = __ldg(p.idx + ((int64_t)it.b * p.nq + it.qi) * p.k + T.list_off + tid);
          valid = e >= 0 && e < p.N;
        }
        if (!mbar_wait_group(gid, &bar_s_full, ph, &abort_flag)) { bad = true; continue; }
        tc_fence_after();
        // this key's scores for the group's heads, scaled to log2 units
        float v[32];
        tmem_ld32(tS + lane_base + h0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 sc = sc4[e4];
          v[4 * e4 + 0] = valid ? v[4 * e4 + 0] * sc.x : -INFINITY;
          v[4 * e4 + 1] = valid ? v[4 * e4 + 1] * sc.y : -INFINITY;
          v[4 * e4 + 2] = valid ? v[4 * e4 + 2] * sc.z : -INFINITY;
          v[4 * e4 + 3] = valid ? v[4 * e4 + 3] * sc.w : -INFINITY;
        }
        // The running max m_use is raised only when some score of this tile
        // exceeds it by more than 2^8 (or on the item's first tile).
        bool exceed = first;
        if (!first) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 mu = mu4[e4];
            exceed |= (v[4 * e4 + 0] > mu.x + kRescaleThreshold) | (v[4 * e4 + 1] > mu.y + kRescaleThreshold) |
                      (v[4 * e4 + 2] > mu.z + kRescaleThreshold) | (v[4 * e4 + 3] > mu.w + kRescaleThreshold);
          }
        }
        exceed = group_any(gid, exceed);
        bool rescale = false;
        if (exceed) {
          {
            float t[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) t[e] = v[e];
            reduce_group32<true>(t, red[g], stat_a + h0, gid);      // stat_a = tile max per head
          }
          if (tid == 0) need_rescale[g] = 0;
          group_sync(gid);
          if (tid < 32) {
            const int h = h0 + tid;
            const float mt = stat_a[h], mo = m_use[h];
            float a = 1.f;
            if (mt > mo + kRescaleThreshold || (mo == -INFINITY && mt != -INFINITY)) {
              a = (mo == -INFINITY) ? 0.f : exp2f(mo - mt);
              m_use[h] = mt;
              if (!first) need_rescale[g] = 1;
            }
            alpha[h] = a;
          }
          group_sync(gid);
          rescale = need_rescale[g] != 0;
        }
        // the previous tile's P.V has finished: P^T may be overwritten and
        // O^T / the partial sums rescaled
        if (!first) {
          if (!mbar_wait_group(gid, &bar_pv, ph ^ 1, &abort_flag)) { bad = true; continue; }
          tc_fence_after();
        }
        if (rescale) {
          const float4* al4 = reinterpret_cast<const float4*>(alpha + h0);
#pragma unroll 1
          for (int mt = 0; mt <= kAttnMT; ++mt) {            // O^T M-tiles, then the partial sums
            float o[32];
            const uint32_t a = (mt < kAttnMT ? tO + mt * kAttnH : tL) + lane_base + h0;
            tmem_ld32(a, o);
            tmem_wait_ld();
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 al = al4[e4];
              o[4 * e4 + 0] *= al.x; o[4 * e4 + 1] *= al.y; o[4 * e4 + 2] *= al.z; o[4 * e4 + 3] *= al.w;
            }
            tmem_st32(a, o);
          }
          tmem_wait_st();
        }
        // p = 2^(s - m) (masked keys give 0): P^T row tid, bytes [64g, 64g + 64),
        // and this key slot's running sums per head in TMEM
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 mu = mu4[e4];
          v[4 * e4 + 0] = valid ? fast_exp2(v[4 * e4 + 0] - mu.x) : 0.f;
          v[4 * e4 + 1] = valid ? fast_exp2(v[4 * e4 + 1] - mu.y) : 0.f;
          v[4 * e4 + 2] = valid ? fast_exp2(v[4 * e4 + 2] - mu.z) : 0.f;
          v[4 * e4 + 3] = valid ? fast_exp2(v[4 * e4 + 3] - mu.w) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 o;
          store16(reinterpret_cast<__nv_bfloat16*>(&o), v + 8 * j);
          *reinterpret_cast<uint4*>(sP + sw128_offset(tid, (4 * g + j) * 16)) = o;
        }
        {
          const uint32_t la = tL + lane_base + h0;
          if (!first) {
            float l[32];
            tmem_ld32(la, l);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] += l[e];
          }
          tmem_st32(la, v);
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar_s_empty);
        mbar_arrive(&bar_p_full);
      }
      // ---- epilogue: wait for the last P.V, reduce the sums, write out
      if (!empty && !bad) {
        if (!mbar_wait_group(gid, &bar_pv, (tcount - 1) & 1, &abort_flag)) bad = true;
        else tc_fence_after();
      }
      if (!empty && !bad) {
        float v[32];
        tmem_ld32(tL + lane_base + h0, v);
        tmem_wait_ld();
        reduce_group32<false>(v, red[g], l_run + h0, gid);     // l_run = sum of p per head
      }
      bad = softmax_any256(bad);             // the output stage is entered by both groups or neither
      if (!bad) {
        if (kDecode) {
          // partial block of (query, split): m[H] (log2 units) and l[H] in
          // fp32, then O / l as bf16 [D][H] (a thread writes its dim's 32
          // heads, 64 contiguous bytes, straight from TMEM); an empty split
          // writes only its header, m = -inf, which the combine skips
          char* P = reinterpret_cast<char*>(p.partial) +
                    (((int64_t)it.b * p.nq + it.qi) * p.splits + it.split) * kTcPartialBytes;
          float* hdr = reinterpret_cast<float*>(P);
          if (tid < 32) {
            const int h = h0 + tid;
            const float l = empty ? 0.f : l_run[h];
            hdr[h] = empty ? -INFINITY : m_use[h];
            hdr[kAttnH + h] = l;
            stat_a[h] = l > 0.f ? 1.f / l : 0.f;
          }
          group_sync(gid);
          if (!empty) {
            // O / l of M-tile mt: 128 dims x 64 heads bf16 = 128-byte rows,
            // staged in P's buffer with the 128-byte swizzle (group g writes
            // pieces 4g..4g+3 of row tid) and stored by one TMA box
            const float4* f4 = reinterpret_cast<const float4*>(stat_a + h0);
            const int blk = ((it.b * p.nq + it.qi) * p.splits + it.split);
            // a CTA with a single item stages all four M-tiles in the key
            // buffer (its last P.V has completed and no further keys come),
            // so the four stores go out back to back
            const bool own_k = p.n_items <= (int)gridDim.x;
#pragma unroll 1
            for (int mt = 0; mt < kAttnMT; ++mt) {
              uint8_t* stg = own_k ? sK + mt * AttnSmem::K_CHUNK : sP;
              float o[32];
              tmem_ld32(tO + lane_base + mt * kAttnH + h0, o);
              tmem_wait_ld();
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const float4 f = f4[e4];
                o[4 * e4 + 0] *= f.x; o[4 * e4 + 1] *= f.y; o[4 * e4 + 2] *= f.z; o[4 * e4 + 3] *= f.w;
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
                w.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
                w.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
                w.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
                *reinterpret_cast<uint4*>(stg + sw128_offset(tid, (4 * g + q) * 16)) = w;
              }
              fence_proxy_async_smem();
              softmax_sync256();
              if (st == 0) {
                tma_store_2d(&part_rows, stg, 0, blk * kTcPartialRows + kTcPartialHeaderRows + mt * 128);
                bulk_commit();
                if (!own_k) bulk_wait_read<0>();     // sP may be rewritten
              }
              if (!own_k) softmax_sync256();
            }
            if (st == 0) bulk_wait_read<0>();       // the stores complete before the grid does
          }
        } else {
          // final rows: o = O / (l + e^{z - m}), rope dims rotated back by -t
          __nv_bfloat16* O = p.out + ((int64_t)it.b * p.nq + it.qi) * kAttnH * kAttnD;
          if (empty) {
            // no key at all: only the sink is in the denominator, o = 0
            for (int x = tid; x < 32 * kAttnD; x += 128) O[(int64_t)h0 * kAttnD + x] = __float2bfloat16_rn(0.f);
          } else {
            if (tid < 32) {
              const int h = h0 + tid;
              const float z2 = p.sinks[h] * kLog2e;
              const float mu = m_use[h];
              const float M = fmaxf(mu, z2);
              const float den = exp2f(z2 - M) + (mu == -INFINITY ? 0.f : l_run[h] * exp2f(mu - M));
              stat_a[h] = (mu == -INFINITY) ? 0.f : exp2f(mu - M) / den;   // factor on O
            }
            group_sync(gid);
            __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sP) + g * 32 * 128;   // [32 heads][128 dims]
            const float4* fac4 = reinterpret_cast<const float4*>(stat_a + h0);
#pragma unroll 1
            for (int mt = 0; mt < kAttnMT; ++mt) {
              const int dim = mt * 128 + tid;
              const bool mt_rope = mt * 128 + 127 >= r0;     // uniform over the group
              const bool rot = dim >= r0;
              float cs = 1.f, sn = 0.f;
              if (rot) rope_sincos(-(double)it.t, theta_s[(dim - r0) >> 1], &cs, &sn);
              float o[32];
              tmem_ld32(tO + lane_base + mt * kAttnH + h0, o);
              tmem_wait_ld();
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const float4 f = fac4[e4];
                o[e4 * 4 + 0] *= f.x; o[e4 * 4 + 1] *= f.y; o[e4 * 4 + 2] *= f.z; o[e4 * 4 + 3] *= f.w;
              }
              if (mt_rope) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const float partner = __shfl_xor_sync(0xffffffffu, o[e], 1);
                  if (rot) o[e] = (dim & 1) ? fmaf(partner, sn, o[e] * cs) : fmaf(-partner, sn, o[e] * cs);
                }
              }
#pragma unroll
              for (int e = 0; e < 32; ++e) stage[e * 128 + tid] = __float2bfloat16_rn(o[e]);
              group_sync(gid);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int piece = tid + 128 * i;             // 16-byte piece: head = piece / 16
                const int h = piece >> 4, off = (piece & 15) * 8;
                const uint4 val = *reinterpret_cast<const uint4*>(stage + h * 128 + off);
                *reinterpret_cast<uint4*>(O + (int64_t)(h0 + h) * kAttnD + mt * 128 + off) = val;
              }
              group_sync(gid);
            }
          }
        }
      }
      tc_fence_before();
      if (softmax_any256(bad)) break;        // also: both groups are done with the item
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpS) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Split-KV combine of the tensor-core decode partials, with the sink and the
// output de-rotation: o = sum_s f_s (O_s / l_s), f_s = l_s 2^(m_s - M) / den,
// den = 2^(z_h log2 e - M) + sum_s l_s 2^(m_s - M), M the largest of them; the
// rope dims of o are then rotated by -t.  One CTA per (query, 16 dims).  The
// m, l headers of every split and the 16-dim slices (16 x 64 bf16 per split)
// reach shared memory by two TMA boxes, so the kernel pays about one memory
// latency, not one per split.  With more splits than slice slots the slices
// go in rounds.
constexpr int kTcCombineMaxSplits = 160;
constexpr int kTcCombineSlots = 48;
constexpr int kTcCombineThreads = 512;        // four threads per (dim, 8 heads): every fourth split each
constexpr int kTcCombineDims = 16;
constexpr int kTcCombineSlice = kTcCombineDims * kAttnH * 2;

struct TcCombineParams {
  const char* partial;        // [B * nq][splits] blocks of kTcPartialBytes
  const float* sinks;         // [H]
  const int* pos;             // [B] query positions (decode)
  __nv_bfloat16* out;         // [B * nq, H, D]
  // context parallelism: instead of out, the rows' unnormalised shares
  // [rows][mx[H], l[H], o[H][D]] f32, without the sink and not de-rotated
  float* partial_out;
  int rows, splits, rope_dims;
  double theta[64];           // base^(-2j/r) per rope pair j (r <= 128), from the host
};

// dynamic shared memory of the combine: headers of all splits + slice slots
__host__ __device__ inline int tc_combine_smem_bytes(int splits) {
  const int slots = splits < kTcCombineSlots ? splits : kTcCombineSlots;
  return splits * kTcPartialHeader + slots * kTcCombineSlice;
}

// hdr_map: the partials as [blocks][516 rows][64 bf16], box [splits][4][64]
// (the m, l headers of all splits of one query); slc_map: the same tensor,
// box [min(splits, 64)][16][64] (16 dims of up to 64 splits).  A bulk copy per
// split was measured to complete one copy at a time; a box covering every
// split goes out as one transfer.
__global__ void __launch_bounds__(kTcCombineThreads) attn_combine_tc_kernel(
    const __grid_constant__ CUtensorMap hdr_map, const __grid_constant__ CUtensorMap slc_map,
    const __grid_constant__ TcCombineParams p) {
  extern __shared__ __align__(128) uint8_t cmb_smem[];
  __shared__ uint64_t bar_hdr, bar_slc;
  __shared__ float red[8][kAttnH];
  __shared__ float inv_s[kAttnH];
  __shared__ __align__(16) float acc_s[3][128][8];
  __shared__ __align__(16) __nv_bfloat16 ostage[kAttnH][kTcCombineDims];
  __shared__ volatile int abort_flag;
  constexpr int kChunks = kAttnD / kTcCombineDims;
  float* hdr = reinterpret_cast<float*>(cmb_smem);              // [splits][m[H], l[H]]; m slots -> weights
  uint8_t* slots = cmb_smem + p.splits * kTcPartialHeader;        // [slots][16 dims][H] bf16
  const int nslots = p.splits < kTcCombineSlots ? p.splits : kTcCombineSlots;
  const int row = blockIdx.x / kChunks, dc = blockIdx.x % kChunks;
  const int blk0 = row * p.splits, srow = kTcPartialHeaderRows + dc * kTcCombineDims;
  const int tid = threadIdx.x;
  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&bar_hdr, 1);
    mbar_init(&bar_slc, 1);
    mbar_fence_init();
    tma_prefetch_desc(&hdr_map);
    tma_prefetch_desc(&slc_map);
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) {
    mbar_expect_tx(&bar_hdr, (uint32_t)(p.splits * kTcPartialHeader));
    tma_load_3d(hdr, &hdr_map, 0, 0, blk0, &bar_hdr);
    // a last round shorter than the box reads past this query's splits (or
    // zero fill past the tensor); those slots are not used
    mbar_expect_tx(&bar_slc, (uint32_t)(nslots * kTcCombineSlice));
    tma_load_3d(slots, &slc_map, 0, srow, blk0, &bar_slc);
  }
  // split weights: thread (head h, part) takes the splits s = part mod 8
  const int h = tid & (kAttnH - 1), part = tid >> 6;
  bool ok = mbar_wait(&bar_hdr, 0, &abort_flag);
  const bool share = p.partial_out != nullptr;
  const float z2 = share ? -INFINITY : p.sinks[h] * kLog2e;
  float mx = -INFINITY;
  if (ok) {
#pragma unroll 4
    for (int s = part; s < p.splits; s += 8) mx = fmaxf(mx, hdr[s * kTcHdrFloats + h]);
  }
  red[part][h] = mx;
  __syncthreads();
  float M = z2;
#pragma unroll
  for (int i = 0; i < 8; ++i) M = fmaxf(M, red[i][h]);
  float den = 0.f;
  if (ok)
#pragma unroll 4
    for (int s = part; s < p.splits; s += 8) {
      const float ms = hdr[s * kTcHdrFloats + h];
      const float f = ms == -INFINITY ? 0.f : hdr[s * kTcHdrFloats + kAttnH + h] * exp2f(ms - M);
      hdr[s * kTcHdrFloats + h] = f;
      den += f;
    }
  __syncthreads();                                 // every read of red[] (M) is done
  red[part][h] = den;
  __syncthreads();
  if (part == 0) {
    float d = share ? 0.f : exp2f(z2 - M);
#pragma unroll
    for (int i = 0; i < 8; ++i) d += red[i][h];
    inv_s[h] = share ? (d > 0.f ? 1.f / d : 0.f) : 1.f / d;
    if (share && dc == 0) {
      float* hdr_out = p.partial_out + (int64_t)row * (2 * kAttnH + kAttnH * kAttnD);
      hdr_out[h] = M;
      hdr_out[kAttnH + h] = d;
    }
  }
  // weighted sum over the splits: thread (quarter qt, dim dl, heads 8 hg ..)
  // takes the splits s = qt mod 4
  const int qt = tid >> 7, lt = tid & 127;
  const int dl = lt >> 3, hg = lt & 7;
  const int dim = dc * kTcCombineDims + dl;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int s0 = 0, round = 0; s0 < p.splits; s0 += nslots, ++round) {
    if (round > 0) {
      __syncthreads();                             // every slot of the last round is consumed
      if (tid == 0) {
        mbar_expect_tx(&bar_slc, (uint32_t)(nslots * kTcCombineSlice));
        tma_load_3d(slots, &slc_map, 0, srow, blk0 + s0, &bar_slc);
      }
    }
    // a timed-out wait leaves ok false; the loop still runs to the end so
    // that every thread reaches the same barriers
    ok = mbar_wait(&bar_slc, round & 1, &abort_flag) && ok;
    if (ok) {
      const int n = min(p.splits, s0 + nslots) - s0;
      const float* wb = hdr + s0 * kTcHdrFloats + hg * 8;
      const uint8_t* sb = slots + dl * (kAttnH * 2) + hg * 16;
#pragma unroll 2
      for (int i = qt; i < n; i += 4) {
        const float4 w0 = *reinterpret_cast<const float4*>(wb + i * kTcHdrFloats);
        const float4 w1 = *reinterpret_cast<const float4*>(wb + i * kTcHdrFloats + 4);
        uint4 raw = *reinterpret_cast<const uint4*>(sb + i * kTcCombineSlice);
        // an empty split (all weights 0) has a header but no written slice
        const bool live = (w0.x != 0.f) | (w0.y != 0.f) | (w0.z != 0.f) | (w0.w != 0.f) | (w1.x != 0.f) |
                          (w1.y != 0.f) | (w1.z != 0.f) | (w1.w != 0.f);
        raw.x = live ? raw.x : 0u; raw.y = live ? raw.y : 0u; raw.z = live ? raw.z : 0u; raw.w = live ? raw.w : 0u;
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.z));
        const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.w));
        acc[0] = fmaf(w0.x, f0.x, acc[0]); acc[1] = fmaf(w0.y, f0.y, acc[1]);
        acc[2] = fmaf(w0.z, f1.x, acc[2]); acc[3] = fmaf(w0.w, f1.y, acc[3]);
        acc[4] = fmaf(w1.x, f2.x, acc[4]); acc[5] = fmaf(w1.y, f2.y, acc[5]);
        acc[6] = fmaf(w1.z, f3.x, acc[6]); acc[7] = fmaf(w1.w, f3.y, acc[7]);
      }
    }
  }
  if (qt > 0) {
    *reinterpret_cast<float4*>(&acc_s[qt - 1][lt][0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(&acc_s[qt - 1][lt][4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  ok = __syncthreads_and(ok);
  if (qt == 0) {
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += acc_s[j][lt][i];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= inv_s[hg * 8 + i];
    if (share) {
      // this rank's share: o[h][dim] as fp32 (ok is the block's AND here); the
      // merge adds the sink and de-rotates
      float* o = p.partial_out + (int64_t)row * (2 * kAttnH + kAttnH * kAttnD) + 2 * kAttnH;
      if (ok)
#pragma unroll
        for (int i = 0; i < 8; ++i) o[(hg * 8 + i) * kAttnD + dim] = acc[i];
    } else {
      // rope dims: the pair partner (dim ^ 1) is thread tid ^ 8
      const int r0 = kAttnD - p.rope_dims;
      float partner[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) partner[i] = __shfl_xor_sync(0xffffffffu, acc[i], 8);
      if (dim >= r0) {
        float cs, sn;
        rope_sincos(-(double)p.pos[row], p.theta[(dim - r0) >> 1], &cs, &sn);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[i] = (dim & 1) ? fmaf(partner[i], sn, acc[i] * cs) : fmaf(-partner[i], sn, acc[i] * cs);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ostage[hg * 8 + i][dl] = __float2bfloat16_rn(acc[i]);
    }
  }
  __syncthreads();
  if (!ok || share) return;
  if (tid < 128) {
    const int hh = tid >> 1, piece = tid & 1;
    *reinterpret_cast<uint4*>(p.out + ((int64_t)row * kAttnH + hh) * kAttnD + dc * kTcCombineDims + piece * 8) =
        *reinterpret_cast<const uint4*>(&ostage[hh][piece * 8]);
  }
}

}  // namespace csahca
