/*
 * csahca.h -- C ABI of the B200 (sm_100a) compressed-attention library
 * (libcsahca.so): the forward hot path of DeepSeek-V4's hybrid attention,
 * CSA (compressed sparse attention) and HCA (heavily compressed attention).
 *
 * Sources, cited by page title and section:
 *   [P2] "Paper Breakdown: DeepSeek-V4", section 4 "Hybrid Attention: CSA + HCA":
 *        CSA KV compression (two streams C^a, C^b, logits Z^a, Z^b, 2m entries
 *        per block, softmax with positional biases B^a, B^b), DSA on compressed
 *        KV (indexer keys compressed the same way, top-k, MQA core attention),
 *        sliding window KV, HCA (single stream, ratio 1/m', no overlap, dense),
 *        Additional Techniques (query/KV RMSNorm, partial RoPE on the last 64
 *        dims, attention sink logit per head).
 *   [P4] "How DeepSeek-V4 architecture and training work together", section
 *        "Two compressed views of one history": 1,024 selected entries per
 *        query, 128-token local window.
 *   [P5] "Inside DeepSeek V4": "Two compression regimes" (overlapping 4x,
 *        non-overlapping 128x) and "Local window" (128 uncompressed entries in
 *        every CSA and HCA layer).
 *
 * Conventions (all entry points):
 *   - Every tensor argument is a DEVICE pointer owned by the caller, row-major
 *     and contiguous in the layout stated, 16-byte aligned.  The library keeps
 *     no pointer after the call returns and allocates no device memory: where
 *     a call needs scratch it takes `workspace` / `workspace_bytes`, sized by
 *     the matching *_workspace_size() query (NULL / 0 is fine when that query
 *     returns 0).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  A return of CSAHCA_OK means the work was
 *     enqueued; errors found on the device surface through
 *     csahca_device_error().
 *   - Shapes are validated on the host before any launch; a bad argument
 *     returns a negative status and launches nothing.  There is no fallback
 *     path: a shape the kernels do not cover returns CSAHCA_ERR_UNSUPPORTED.
 *   - dtypes: F32 (float), BF16 (bfloat16), E4M3 (float8 e4m3 "fn" bytes, with
 *     one fp32 scale per 128 contiguous elements).  Arithmetic is fp32.
 *   - Fixed readings of the pages (stated once here, used by every call):
 *       entry i of ratio m covers tokens i*m .. (i+1)*m-1 and is visible to
 *       query t iff (i+1)*m-1 <= t; an incomplete trailing block forms no
 *       entry; RoPE rotates interleaved pairs (2j, 2j+1) of the last r dims by
 *       pos * base^(-2j/r); compressed entry i sits at position i*m; RMSNorm is
 *       x / sqrt(mean(x^2) + eps) * gain; softmax scale defaults to 1/sqrt(d);
 *       K = V = the compressed (or window) row; the sink adds e^{z_h} to the
 *       softmax denominator only; the rope dims of each output row are rotated
 *       back by -t (t = query position).
 */
#ifndef CSAHCA_H_
#define CSAHCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSAHCA_ABI_VERSION 4

/* ---- status codes ------------------------------------------------------- */
enum {
  CSAHCA_OK = 0,
  CSAHCA_ERR_INVALID_ARG = -1,   /* NULL pointer, negative size, bad enum      */
  CSAHCA_ERR_UNSUPPORTED = -2,   /* valid but not covered by the kernels       */
  CSAHCA_ERR_ALIGNMENT = -3,     /* a pointer is not 16-byte aligned           */
  CSAHCA_ERR_WORKSPACE = -4,     /* workspace NULL or smaller than required    */
  CSAHCA_ERR_LAUNCH = -5,        /* a CUDA launch or driver call failed        */
  CSAHCA_ERR_DEVICE_TIMEOUT = -6,/* a bounded device wait gave up (see below)  */
  CSAHCA_ERR_NO_DEVICE = -7      /* no usable sm_100 device                    */
};

/* ---- enums ---------------------------------------------------------------- */
enum { CSAHCA_F32 = 0, CSAHCA_BF16 = 1, CSAHCA_E4M3 = 2 };
enum { CSAHCA_CSA = 0, CSAHCA_HCA = 1 };

/* ---- csa_compress / hca_compress ----------------------------------------
 * [P2] CSA KV compression; HCA; Additional Techniques (RMSNorm, RoPE).
 *
 * CSA (overlapped, ratio 1/m, 2m tokens per entry), for entry i, channel c:
 *   la_r = za[i*m + r, c] + bias_a[r, c],  lb_r = zb[(i-1)*m + r, c] + bias_b[r, c]
 *   (lb = -inf for i = 0), S = softmax over the 2m logits jointly,
 *   C_i[c] = sum_r Sa_r a[i*m + r, c] + sum_r Sb_r b[(i-1)*m + r, c].
 * HCA (non-overlapped, ratio 1/m'): C_i[c] = sum_r softmax_r(za + bias_a) a.
 *   (b, zb, bias_b are ignored.)
 * Then, if rms_norm != 0: C_i <- C_i / sqrt(mean(C_i^2) + eps) * gain (gain
 * NULL = ones); if rope_dims > 0: RoPE at position i*m on the last rope_dims.
 * Indexer keys use the same pooling with rms_norm = 0 and rope_dims = 0.
 *
 * Layout: a, b, za, zb [B, n, c] (dtype); bias_a, bias_b [m, c] f32;
 * gain [c] f32; out [B, num_blocks, c] (dtype) holding entries
 * first_block .. first_block + num_blocks - 1, each of which must be complete
 * (first_block + num_blocks <= n / m).  num_blocks = -1 means all n / m
 * entries from first_block.  Constraints: dtype F32 (c % 4 == 0) or BF16
 * (c % 8 == 0); rope_dims even, <= c, (c - rope_dims) even; m >= 1.
 */
typedef struct {
  int32_t dtype;
  int32_t B, n, c;
  int32_t m;
  int32_t first_block, num_blocks;
  int32_t rms_norm;
  int32_t rope_dims;
  float rope_base;     /* 0 -> 10000 */
  float eps;           /* 0 -> 1e-6  */
  int32_t reserved0;
  const void* a;
  const void* b;
  const void* za;
  const void* zb;
  const float* bias_a;
  const float* bias_b;
  const float* gain;
  void* out;
} csahca_compress_args;

int csa_compress(const csahca_compress_args* args, void* stream);
int hca_compress(const csahca_compress_args* args, void* stream);

/* ---- indexer_topk ---------------------------------------------------------
 * [P2] DSA on Compressed KV (lightning indexer, top-k); [P4] 1,024 entries.
 * For query q of sequence b at absolute position t = q_pos[b, q]:
 *   I_{t,i} = sum_j w[b,q,j] * max(0, qI[b,q,j,:] . kI[b,i,:])  for the
 *   visible entries i < v = min(N, (t+1)/m);  kI row i = decode(codes) * scale
 *   per 128-element block when k_dtype = E4M3.
 *   idx[b,q,:] = the k entries with the largest I (ties to the lower index),
 *   sorted ascending, padded with -1 when v < k.
 * Layout: qI [B, nq, HI, dI] (q_dtype F32/BF16); w [B, nq, HI] f32;
 *   kI [B, N, dI] (k_dtype F32/BF16/E4M3); kI_scale [B, N, dI/128] f32 (E4M3
 *   only, else NULL); q_pos [B, nq] int32 on the device; idx [B, nq, k] int32.
 *   scores_out: optional [B, nq, N] f32; entries i < v of each row receive
 *   I_{t,i}, the rest is left untouched.  q_pos values < 0 give v = 0.
 *   sel_scores: optional [B, nq, k] f32; receives I_{t,idx} for each entry
 *   of idx (-inf where idx = -1): the candidates context parallelism
 *   exchanges (cp_topk_merge below).
 *   entry_base (>= 0; 0 for a whole cache): kI holds the global entries
 *   entry_base .. entry_base + N - 1 of a longer cache (one rank's shard under
 *   context parallelism).  Local row j is global entry entry_base + j, visible
 *   iff entry_base + j < (t+1)/m, so v = clamp((t+1)/m - entry_base, 0, N);
 *   idx, scores_out and sel_scores address LOCAL rows.
 * Constraints: k >= 1; dI % 8 == 0; E4M3 needs dI % 128 == 0 and the same
 *   q_dtype rules; q_dtype == k_dtype unless k_dtype is E4M3 (queries BF16).
 * Workspace: csahca_indexer_workspace_size().
 */
typedef struct {
  int32_t q_dtype, k_dtype;
  int32_t B, nq, HI, dI;
  int32_t N;
  int32_t m;
  int32_t k;
  int32_t entry_base;
  const void* qI;
  const float* w;
  const void* kI;
  const float* kI_scale;
  const int32_t* q_pos;
  int32_t* idx;
  float* scores_out;
  float* sel_scores;
  void* workspace;
  size_t workspace_bytes;
} csahca_indexer_args;

int indexer_topk(const csahca_indexer_args* args, void* stream);
size_t csahca_indexer_workspace_size(const csahca_indexer_args* args);

/* ---- indexer_topk_noalloc --------------------------------------------------
 * No counterpart on the pages: an addition of this library for callers that
 * cannot allocate device memory when they call it (for example code running
 * inside a pre-planned memory pool, or a host thread that must not touch the
 * allocator).  Computes exactly what indexer_topk computes, with the same
 * arguments and results, but allocates nothing and takes no workspace: the
 * score rows and top-k buffers live in one fixed __device__ array of
 * CSAHCA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  args->workspace and
 * args->workspace_bytes are ignored.
 *   - A problem whose scratch (csahca_indexer_workspace_size of the same
 *     args) exceeds CSAHCA_NOALLOC_SCRATCH_BYTES is rejected with
 *     CSAHCA_ERR_WORKSPACE before any launch.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and caches it with the
 *     id of the current context; make that first call outside any stream
 *     capture.  After a device reset (cudaDeviceReset, or any teardown of the
 *     primary context) the next call sees a new context id and looks the
 *     address up again, so make that call outside capture too.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (the parts that must start at zero are cleared by each call).
 *     Calls whose work overlaps on the GPU (other streams, or other host
 *     threads) race on it: serialise them.
 *   - Calls no cudaMalloc / cudaFree and no allocating library routine. */
#define CSAHCA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

int indexer_topk_noalloc(const csahca_indexer_args* args, void* stream);

/* ---- compressed_attn_prefill ----------------------------------------------
 * [P2] MQA core attention, sliding window, HCA dense attention, Additional
 * Techniques; [P5] Local window.  For sequence b, query t (position t), head h:
 *   q = RoPE_t(RMSNorm(q_raw[b,t,h,:]) * q_gain)     (norm only if q_norm)
 *   keys J_t = { kv_comp[b, idx[b,t,j]] : idx >= 0 }           (kind CSA)
 *            = { kv_comp[b, i] : i < min(N, (t+1)/m) }          (kind HCA)
 *     plus window rows s = max(0, t-w+1) .. t, each
 *     RoPE_s(RMSNorm(kv_win[b,s,:]) * kv_gain)        (norm only if kv_norm)
 *   o = sum_j e^{s_j} row_j / (e^{sinks[h]} + sum_j e^{s_j}),
 *   s_j = scale * q . row_j, then the last rope_dims of o rotated by -t.
 * Layout: q [B, n, H, d]; kv_comp [B, N, d] (final rows from csa/hca_compress);
 *   kv_win [B, n, d] raw per-token rows; q_gain, kv_gain [d] f32 or NULL
 *   (ones); idx [B, n, k] int32 (CSA; entries < 0 are skipped, entries must be
 *   < N); sinks [H] f32; out [B, n, H, d].  q, kv_comp, kv_win, out share
 *   `dtype` (F32 or BF16).
 * Constraints: d % 8 == 0, rope_dims even and <= d, w >= 0, H >= 1.
 * Workspace: csahca_prefill_workspace_size().
 */
typedef struct {
  int32_t kind;
  int32_t dtype;
  int32_t B, n, H, d;
  int32_t N;
  int32_t m;
  int32_t k;
  int32_t w;
  int32_t rope_dims;
  float rope_base;     /* 0 -> 10000 */
  float eps;           /* 0 -> 1e-6 */
  float scale;         /* 0 -> 1/sqrt(d) */
  int32_t q_norm, kv_norm;
  const void* q;
  const void* kv_comp;
  const void* kv_win;
  const float* q_gain;
  const float* kv_gain;
  const int32_t* idx;
  const float* sinks;
  void* out;
  void* workspace;
  size_t workspace_bytes;
} csahca_attn_args;

int compressed_attn_prefill(const csahca_attn_args* args, void* stream);
size_t csahca_prefill_workspace_size(const csahca_attn_args* args);

/* ---- FP8 KV cache rows ------------------------------------------------------
 * [P2] infrastructure table: KV cache storage FP8 for the non-RoPE dims, BF16
 * for the RoPE dims.  A row of kv_dtype CSAHCA_E4M3 (d and r = rope_dims with
 * d - r and r multiples of 64) is csahca_kv_row_bytes() bytes:
 *   bytes [0, d - r)                 e4m3 codes of dims 0 .. d - r - 1
 *   bytes [d - r, d + r)             the r RoPE dims as bf16
 *   bytes [d + r, d + r + 4 nb)      fp32 scale of each of the nb = (d - r) / 64
 *                                    64-dim blocks: amax / 448 (1 for an
 *                                    all-zero block); codes = nearest e4m3 of
 *                                    x / scale, ties to even, saturating
 *   then padding to a multiple of 128 bytes (never read).
 * Dim j < d - r of the row stands for decode(code_j) * scale_{j / 64}.  The
 * window ring stays bf16.  d = 512, r = 64: 448 + 128 + 28 -> 640 bytes. */

/* Bytes of one cache row: d times the element size for F32 / BF16, the FP8
 * layout above for E4M3; 0 for an invalid combination. */
int64_t csahca_kv_row_bytes(int32_t kv_dtype, int32_t d, int32_t rope_dims);

/* ---- compressed_attn_decode -----------------------------------------------
 * One decode step of one layer (CSA or HCA) for B sequences, one new query
 * token each at position pos[b] (device int32).  Caches hold final rows
 * (already normed and roped): kv_cache [B, N_cap, d] with entry i valid iff
 * i < min(N_cap, (pos+1)/m); win [B, w, d] ring buffer, slot p % w holding
 * the row of position p, for p = max(0, pos-w+1) .. pos (the new token's own
 * row included).  q [B, H, d] raw, normed (q_norm) and roped at pos here.
 * CSA: the selection is the lightning-indexer top-k over the visible entries
 *   (qI [B, HI, dI], wI [B, HI] f32, kI [B, N_cap, dI], kI_scale as in
 *   indexer_topk) unless idx_in [B, k] is given, which is then used as is.
 *   idx_out [B, k] (optional) receives the selection used.
 * HCA: dense over every visible entry.  Output and sink exactly as in
 * compressed_attn_prefill; out [B, H, d] (dtype).
 * kv_dtype CSAHCA_E4M3: kv_cache holds FP8 KV rows (layout above,
 *   [B, N_cap, csahca_kv_row_bytes] bytes), read as the rows they stand for;
 *   dtype BF16, H = 64, d = 512, rope_dims 64 or 128, else
 *   CSAHCA_ERR_UNSUPPORTED.  Any other kv_dtype: rows of `dtype`.
 * Context parallelism (one rank's share of a layer whose compressed cache is
 *   split by entry range across ranks; tensor-core shapes only: BF16, H = 64,
 *   d = 512, rope_dims <= 128, B * N_cap >= 128 and (unless skip_window)
 *   B * w >= 128, else CSAHCA_ERR_UNSUPPORTED):
 *   entry_base: kv_cache (and kI) hold the global entries entry_base ..
 *     entry_base + N_cap - 1; visibility as in indexer_topk's entry_base.
 *     CSA with entry_base > 0 needs idx_in (LOCAL rows, -1 to skip; as
 *     cp_topk_merge writes them).
 *   skip_window != 0: the window is left out (another rank attends it); win
 *     is not read and may be NULL.
 *   partial_out != NULL: instead of `out` (which may then be NULL), each row's
 *     unnormalised share of the softmax is written as one block of
 *     2H + H*d floats: mx[H], the largest scaled logit of the head in base-2
 *     units (s * scale * log2(e)), -inf if the rank attends no key; l[H] =
 *     sum over the keys of 2^(logit2 - mx) (0 if none); o[H][d] = the
 *     weighted mean of the keys' rows (0 if none).  The sink is left out and
 *     the output is not de-rotated: cp_attn_merge does both once.
 * Workspace: csahca_decode_workspace_size().
 */
typedef struct {
  int32_t kind;
  int32_t dtype;
  int32_t B, H, d;
  int32_t N_cap;
  int32_t m;
  int32_t w;
  int32_t rope_dims;
  float rope_base;
  float eps;
  float scale;
  int32_t q_norm;
  int32_t k;
  int32_t HI, dI;
  int32_t qI_dtype, kI_dtype;
  int32_t kv_dtype;    /* CSAHCA_E4M3: FP8 KV rows; else rows of dtype */
  int32_t entry_base;  /* context parallelism: first global entry of kv_cache */
  const void* q;
  const int32_t* pos;
  const float* q_gain;
  const void* kv_cache;
  const void* win;
  const float* sinks;
  const void* qI;
  const float* wI;
  const void* kI;
  const float* kI_scale;
  const int32_t* idx_in;
  int32_t* idx_out;
  void* out;
  float* partial_out;  /* context parallelism: [B, 2H + H*d] f32 instead of out */
  int32_t skip_window; /* context parallelism: leave the window out */
  int32_t reserved2;
  void* workspace;
  size_t workspace_bytes;
} csahca_decode_args;

int compressed_attn_decode(const csahca_decode_args* args, void* stream);
size_t csahca_decode_workspace_size(const csahca_decode_args* args);

/* ---- decode_compress --------------------------------------------------------
 * [P2] CSA KV compression, HCA, sliding window KV, Additional Techniques.
 * One decode step of one layer's compressors for B sequences, the new token
 * of sequence b at position t = pos[b] (device int32):
 *   1. its raw streams go into slot t % R of `ring` (R = 2m for CSA, m for
 *      HCA; ring [B, R, S, d] with S = 4 streams a, b, za, zb for CSA, 2
 *      streams a, za for HCA; the indexer streams likewise into `iring`
 *      [B, 2m, 4, dI]).  The rings are the compressor state between steps:
 *      slot p % R holds token p for the R tokens before t.
 *   2. if kv_raw != NULL and w > 0: win[b, t % w] = RoPE_t(RMSNorm(kv_raw[b])
 *      * kv_gain) (norm only if kv_norm).
 *   3. if t completes block i = (t+1)/m - 1 and i < N_cap: entry i is pooled
 *      exactly as csa_compress / hca_compress define it over the ring's tokens
 *      (token t from the inputs; the slots of other tokens must hold them) and
 *      kv_cache[b, i] = RoPE_{i*m}(RMSNorm(C_i) * kv_gain); for CSA with
 *      dI > 0 the indexer key of entry i is pooled from the indexer streams
 *      (no norm, no RoPE) and stored in kI[b, i] (kI_dtype = dtype), or, for
 *      kI_dtype E4M3, as e4m3 codes with kI_scale[b, i, j] = amax_j / 448 over
 *      each 128-element block j (1 for an all-zero block) and codes the
 *      nearest e4m3 of x / scale (ties to even, saturating at 448), all in
 *      fp32.  Entries with i >= N_cap are not stored.  A sequence with
 *      pos[b] < 0 is left untouched.  With kv_dtype CSAHCA_E4M3 the entry is
 *      stored as an FP8 KV row (layout above: the finished row's non-RoPE
 *      dims quantised in fp32 against their 64-dim block scales, the RoPE
 *      dims as bf16); dtype BF16, d = 512, rope_dims 64 or 128 only.
 *   entry_base (>= 0): kv_cache and kI hold the global entries entry_base ..
 *      entry_base + N_cap - 1 (context parallelism); entry i is stored in local
 *      row i - entry_base when entry_base <= i < entry_base + N_cap, else not
 *      at all.  The rings and the window are kept whatever entry_base is.
 * Layout: pos [B]; kv_raw, a, b, za, zb [B, d] (dtype; b, zb CSA only);
 *   bias_a, bias_b [m, d] f32; kv_gain [d] f32 or NULL (ones); kv_cache
 *   [B, N_cap, d]; win [B, w, d]; ia, ib, iza, izb [B, dI] (dtype); ibias_a,
 *   ibias_b [m, dI] f32; kI [B, N_cap, dI]; kI_scale [B, N_cap, dI/128] f32.
 * Constraints: dtype F32 (d % 32 == 0) or BF16 (d % 64 == 0), d <= 128 * 16 /
 *   (element bytes); rope_dims even, <= d and <= 128 (the RoPE angles are
 *   computed on the host, one per pair); dI = 0 or (CSA) dI % 8 == 0
 *   with dI / 8 a multiple of the 16-byte vector and dividing 128 (BF16:
 *   64, 128, 256, 512, 1024; F32: 32, 64, 128, 256, 512); E4M3 keys need
 *   BF16 and dI % 128 == 0.  No workspace.  Rows of one sequence are written
 *   by one cluster of eight CTAs, so calls for different layers may overlap.
 */
typedef struct {
  int32_t kind;
  int32_t dtype;
  int32_t B, d;
  int32_t m;
  int32_t N_cap;
  int32_t w;
  int32_t rope_dims;
  float rope_base;     /* 0 -> 10000 */
  float eps;           /* 0 -> 1e-6 */
  int32_t kv_norm;
  int32_t dI;
  int32_t kI_dtype;
  int32_t kv_dtype;    /* CSAHCA_E4M3: kv_cache holds FP8 KV rows; else rows of dtype */
  int32_t entry_base;  /* context parallelism: first global entry of kv_cache / kI */
  int32_t reserved1;
  const int32_t* pos;
  const void* kv_raw;
  const void* a;
  const void* b;
  const void* za;
  const void* zb;
  const float* bias_a;
  const float* bias_b;
  const float* kv_gain;
  void* ring;
  void* kv_cache;
  void* win;
  const void* ia;
  const void* ib;
  const void* iza;
  const void* izb;
  const float* ibias_a;
  const float* ibias_b;
  void* iring;
  void* kI;
  float* kI_scale;
} csahca_decode_compress_args;

int decode_compress(const csahca_decode_compress_args* args, void* stream);

/* ---- context parallelism: the two exchange steps ------------------------------
 * [P2] infrastructure table, "2-Stage Context Parallel" for compressed
 * attention (the pages name it and give no steps; the reading taken here):
 * a layer's compressed cache is split by entry range over R ranks, rank r
 * holding the global entries bases[r] .. bases[r] + N_r - 1 (ranges
 * disjoint), and the window and sink are attended once.  A decode step is
 *   stage 1 (CSA only): each rank runs indexer_topk over its shard
 *     (entry_base = bases[r], sel_scores), the ranks exchange their k
 *     candidates (local rows and scores; an all-gather), and every rank
 *     merges them with cp_topk_merge into the global top-k, which equals the
 *     top-k over the whole cache (every entry of it is in the top-k of its
 *     own shard);
 *   stage 2: each rank runs compressed_attn_decode over its shard (entry_base,
 *     partial_out; CSA with the merge's local rows as idx_in; skip_window on
 *     every rank but one), the ranks exchange the partials (an all-gather),
 *     and cp_attn_merge combines them with the sink and de-rotates the output.
 * The collectives themselves belong to the caller (NCCL, or anything that
 * lays the ranks' buffers out rank-major as stated below). */
#define CSAHCA_CP_MAX_RANKS 64

/* cp_topk_merge: the global top-k of one step from every rank's candidates.
 * cand_idx [R, rows, k] int32 (rank r's LOCAL rows, -1 = none) and
 * cand_scores [R, rows, k] f32, as indexer_topk writes idx / sel_scores;
 * bases[R] on the HOST (copied at the call).  Candidate (r, j) is global
 * entry bases[r] + cand_idx[r, row, j]; the k of largest score are kept, ties
 * to the lower global entry, exactly as indexer_topk ranks one cache.
 * Outputs [rows, k] int32, both optional, in the same order (ascending global
 * entry, -1 padded when fewer than k candidates exist): idx_global (global
 * entries) and idx_local (the entry's local row if it belongs to rank
 * `rank`, else -1: compressed_attn_decode's idx_in for that rank).
 * Constraints: 1 <= R <= CSAHCA_CP_MAX_RANKS; 1 <= k <= 4096; R * k <= 16384;
 * bases[r] >= 0 and every global entry < 2^31.  No workspace. */
typedef struct {
  int32_t R, rows, k;
  int32_t rank;
  const int32_t* bases;
  const int32_t* cand_idx;
  const float* cand_scores;
  int32_t* idx_global;
  int32_t* idx_local;
} csahca_cp_topk_merge_args;

int cp_topk_merge(const csahca_cp_topk_merge_args* args, void* stream);

/* cp_attn_merge: the layer's output from every rank's partial (the
 * partial_out blocks of compressed_attn_decode, laid out [R, rows, 2H + H*d]
 * f32): per row and head, M = max(z_h log2(e), mx_r), weights
 * c_r = l_r 2^(mx_r - M), D = sum_r c_r + 2^(z_h log2(e) - M), and
 * out = sum_r (c_r / D) o_r, whose last rope_dims dims are then rotated back
 * by -pos[row] (RoPE pairs as above, base rope_base).
 * Layout: partials [R, rows, 2H + H*d] f32; sinks [H] f32; pos [rows] int32;
 * out [rows, H, d] (dtype F32 or BF16).  Constraints: 1 <= R <=
 * CSAHCA_CP_MAX_RANKS; H even; d % 4 == 0, d <= 1024; rope_dims even, <= d
 * and <= 128.
 * No workspace. */
typedef struct {
  int32_t dtype;
  int32_t R, rows, H, d;
  int32_t rope_dims;
  float rope_base;     /* 0 -> 10000 */
  int32_t reserved0;
  const float* partials;
  const float* sinks;
  const int32_t* pos;
  void* out;
} csahca_cp_merge_args;

int cp_attn_merge(const csahca_cp_merge_args* args, void* stream);

/* ---- utilities ------------------------------------------------------------ */

/* Human-readable name of a status code (static string). */
const char* csahca_status_string(int status);

/* CSAHCA_ABI_VERSION of the loaded library. */
int csahca_abi_version(void);

/* sizeof() of the argument structs, for bindings to check their mirrors:
 * which = 0 compress, 1 indexer, 2 prefill, 3 decode, 4 decode_compress,
 * 5 cp_topk_merge, 6 cp_attn_merge; -1 for an unknown id. */
int64_t csahca_struct_size(int which);

/* Device-side error word of the current device: every bounded wait in the
 * kernels that gives up ORs a code into it and the kernel returns early
 * instead of hanging (1: a barrier wait reached its iteration limit; 2: a
 * selection index outside [0, N) was skipped).  Synchronises `stream`, stores
 * the word in *code (0 = no error) and clears it.  Returns CSAHCA_OK, or
 * CSAHCA_ERR_LAUNCH if the stream itself reports a CUDA error. */
int csahca_device_error(void* stream, int32_t* code);

/* Self-test of that failure path: launches one kernel on `stream` whose
 * bounded wait on a barrier that nothing completes gives up (well under a
 * second), so that csahca_device_error() on the same stream then reports
 * code 1 and the device stays usable for the calls that follow.  Returns
 * CSAHCA_OK, CSAHCA_ERR_NO_DEVICE without a B200, or CSAHCA_ERR_LAUNCH. */
int csahca_selftest_bounded_wait(void* stream);

/* ---- tracing ---------------------------------------------------------------
 * Optional per-kernel timing.  While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on its stream (events are
 * created once and reused; at most 65536 launches are held between collects,
 * later ones are not traced).  csahca_trace_collect() synchronises those
 * events, adds the elapsed times up per kernel name, writes at most
 * max_entries entries, stores how many it wrote in *n_entries and forgets
 * the recorded launches.  Not thread-safe: trace from one host thread. */
typedef struct {
  char name[48];
  int64_t launches;
  double total_ms;
} csahca_trace_entry;

int csahca_trace_enable(int enable);
int csahca_trace_collect(csahca_trace_entry* out, int max_entries, int* n_entries);

#ifdef __cplusplus
}
#endif

#endif /* CSAHCA_H_ */
