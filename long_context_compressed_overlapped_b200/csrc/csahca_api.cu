// C ABI of libcsahca.so (declared in include/csahca.h).  Host-side argument
// validation, workspace sizing and kernel dispatch; every step of the path
// runs in the kernels included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <utility>
#include <vector>

#include "../../include/csahca.h"
#include "common.cuh"
#include "compress.cuh"
#include "decode_compress.cuh"
#include "indexer_simt.cuh"
#include "topk.cuh"
#include "topk_large.cuh"
#include "attention_simt.cuh"
#include "indexer_tc.cuh"
#include "indexer_f8.cuh"
#include "attention_tc.cuh"
#include "context_parallel.cuh"
#include "attention_small_tc.cuh"

using namespace csahca;

namespace {

// ---------------------------------------------------------------- tracing --
namespace trace {
constexpr size_t kMaxRecords = 65536;
struct Record { cudaEvent_t begin, end; const char* name; };
bool g_enabled = false;
std::vector<cudaEvent_t> g_pool;      // free events
std::vector<Record> g_records;

cudaEvent_t take_event() {
  if (!g_pool.empty()) { cudaEvent_t e = g_pool.back(); g_pool.pop_back(); return e; }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) { (void)cudaGetLastError(); return nullptr; }
  return e;
}

// Bracket one launch: begin() before it, end() after it, on the same stream.
struct Scope {
  cudaEvent_t b = nullptr;
  const char* name;
  cudaStream_t s;
  Scope(const char* n, cudaStream_t st) : name(n), s(st) {
    if (!g_enabled || g_records.size() >= kMaxRecords) return;
    b = take_event();
    if (b) cudaEventRecord(b, s);
  }
  ~Scope() {
    if (!b) return;
    cudaEvent_t e = take_event();
    if (!e) { g_pool.push_back(b); return; }
    cudaEventRecord(e, s);
    g_records.push_back({b, e, name});
  }
};
}  // namespace trace

#define CSAHCA_TRACE(name, stream) trace::Scope trace_scope_##__LINE__(name, stream)

constexpr double kDefaultRopeBase = 10000.0;
constexpr float kDefaultEps = 1e-6f;

// theta[j] = base^(-2j/r), the RoPE angle per unit of position of pair j, in
// double, for the r/2 pairs (at most 64) of kernels that take it as a parameter.
void rope_theta_table(double* theta, int r, double base) {
  for (int j = 0; j < 64; ++j) theta[j] = j < r / 2 ? pow(base, -2.0 * j / r) : 0.0;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Every launch goes through launch_k: programmatic dependent launch lets a
// kernel start (barrier set-up, TMEM allocation, loads of caller inputs)
// while the previous kernel in the stream finishes; each kernel waits
// (griddep_wait) before touching what earlier kernels write.  CSAHCA_PDL=0 in
// the environment launches plainly instead.
bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* e = getenv("CSAHCA_PDL");
    on = (e && e[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

template <typename... KArgs, typename... Args>
void launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define CSAHCA_CHECK_LAUNCH()                                  \
  do {                                                         \
    if (cudaPeekAtLastError() != cudaSuccess) {                \
      (void)cudaGetLastError();                                \
      return CSAHCA_ERR_LAUNCH;                                \
    }                                                          \
  } while (0)

// ---- device facts and TMA descriptors -------------------------------------
int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    return n;
  (void)cudaGetLastError();
  return 148;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2D row-major tensor [rows, inner] of `dt`, box [box_rows, box_inner].
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* ptr, uint64_t inner,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(inner * elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D tensor [d2][d1][d0] of `dt` with byte strides s1 (between d1 rows) and
// s2 (between d2 blocks), box [b2][b1][b0], no swizzle.
bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
               CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t strides[2] = {(cuuint64_t)s1, (cuuint64_t)s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int dtype_size(int dt) {
  switch (dt) {
    case CSAHCA_F32: return 4;
    case CSAHCA_BF16: return 2;
    case CSAHCA_E4M3: return 1;
    default: return 0;
  }
}

int device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return CSAHCA_ERR_NO_DEVICE; }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return CSAHCA_ERR_NO_DEVICE;
  }
  return major == 10 ? CSAHCA_OK : CSAHCA_ERR_NO_DEVICE;
}

// ---------------------------------------------------------------- compress --

int validate_compress(const csahca_compress_args* a, bool csa, int* nblocks) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->dtype != CSAHCA_F32 && a->dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->B < 0 || a->n < 0 || a->c <= 0 || a->m < 1 || a->first_block < 0) return CSAHCA_ERR_INVALID_ARG;
  const int vec = 16 / dtype_size(a->dtype);
  if (a->c % vec) return CSAHCA_ERR_UNSUPPORTED;
  if (a->c > 128 * vec) return CSAHCA_ERR_UNSUPPORTED;
  if (a->rope_dims < 0 || a->rope_dims > a->c || (a->rope_dims & 1) || ((a->c - a->rope_dims) & 1))
    return CSAHCA_ERR_INVALID_ARG;
  const int total = a->n / a->m;
  int nb = a->num_blocks < 0 ? total - a->first_block : a->num_blocks;
  if (nb < 0 || a->first_block + nb > total) return CSAHCA_ERR_INVALID_ARG;
  *nblocks = nb;
  if (nb == 0 || a->B == 0) return CSAHCA_OK;
  if (!a->a || !a->za || !a->bias_a || !a->out) return CSAHCA_ERR_INVALID_ARG;
  if (csa && (!a->b || !a->zb || !a->bias_b)) return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->a, a->za, a->bias_a, a->out, a->gain, csa ? a->b : nullptr,
                        csa ? a->zb : nullptr, csa ? a->bias_b : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  return CSAHCA_OK;
}

int run_compress(const csahca_compress_args* a, void* stream, bool csa) {
  int nb = 0;
  int st = validate_compress(a, csa, &nb);
  if (st != CSAHCA_OK) return st;
  if (nb == 0 || a->B == 0) return CSAHCA_OK;
  if ((st = device_ok()) != CSAHCA_OK) return st;
  CompressParams p;
  p.a = a->a; p.b = a->b; p.za = a->za; p.zb = a->zb;
  p.bias_a = a->bias_a; p.bias_b = a->bias_b; p.gain = a->gain; p.out = a->out;
  p.B = a->B; p.n = a->n; p.c = a->c; p.m = a->m; p.first_block = a->first_block;
  p.num_blocks = nb; p.rms_norm = a->rms_norm; p.rope_dims = a->rope_dims;
  p.rope_base = a->rope_base > 0 ? a->rope_base : kDefaultRopeBase;
  p.eps = a->eps > 0 ? a->eps : kDefaultEps;
  const int64_t warps = (int64_t)a->B * nb;
  const int threads = 256;
  const int64_t blocks = ceil_div64(warps * 32, threads);
  if (blocks > INT32_MAX) return CSAHCA_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  CSAHCA_TRACE(csa ? "csa_compress" : "hca_compress", s);
  if (a->dtype == CSAHCA_F32) {
    if (csa) launch_k(compress_kernel<float, true>, dim3((unsigned)blocks), dim3(threads), 0, s, p);
    else launch_k(compress_kernel<float, false>, dim3((unsigned)blocks), dim3(threads), 0, s, p);
  } else {
    if (csa) launch_k(compress_kernel<__nv_bfloat16, true>, dim3((unsigned)blocks), dim3(threads), 0, s, p);
    else launch_k(compress_kernel<__nv_bfloat16, false>, dim3((unsigned)blocks), dim3(threads), 0, s, p);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// ------------------------------------------------------------------ indexer --

int validate_indexer(const csahca_indexer_args* a, bool shapes_only = false) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->q_dtype != CSAHCA_F32 && a->q_dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->k_dtype != CSAHCA_F32 && a->k_dtype != CSAHCA_BF16 && a->k_dtype != CSAHCA_E4M3)
    return CSAHCA_ERR_INVALID_ARG;
  if (a->B < 0 || a->nq < 0 || a->HI < 1 || a->dI < 1 || a->N < 0 || a->m < 1 || a->k < 1 ||
      a->entry_base < 0)
    return CSAHCA_ERR_INVALID_ARG;
  if (a->dI % 8) return CSAHCA_ERR_UNSUPPORTED;
  if (a->k_dtype == CSAHCA_E4M3) {
    if (a->dI % 128) return CSAHCA_ERR_UNSUPPORTED;
    if (a->q_dtype != CSAHCA_BF16 && a->q_dtype != CSAHCA_F32) return CSAHCA_ERR_UNSUPPORTED;
  } else if (a->k_dtype != a->q_dtype) {
    return CSAHCA_ERR_UNSUPPORTED;
  }
  if (a->HI > kIdxSimtMaxHeads) return CSAHCA_ERR_UNSUPPORTED;
  if (shapes_only || a->B == 0 || a->nq == 0) return CSAHCA_OK;
  if (!a->qI || !a->w || !a->q_pos || !a->idx) return CSAHCA_ERR_INVALID_ARG;
  if (a->N > 0 && !a->kI) return CSAHCA_ERR_INVALID_ARG;
  if (a->k_dtype == CSAHCA_E4M3 && a->N > 0 && !a->kI_scale) return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->qI, a->w, a->kI, a->kI_scale, a->q_pos, a->idx, a->scores_out, a->sel_scores,
                        a->workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  return CSAHCA_OK;
}

// Query chunk so that a chunk of scores stays below ~2 GiB of workspace.
int indexer_chunk_rows(const csahca_indexer_args* a) {
  const int64_t per_q = (int64_t)a->B * (a->N > 0 ? a->N : 1) * 4;
  int64_t rows = ((int64_t)2 << 30) / (per_q > 0 ? per_q : 1);
  if (rows < 1) rows = 1;
  if (rows > a->nq) rows = a->nq;
  if (rows > 65535) rows = 65535;
  return (int)rows;
}

constexpr int kTopkSmallMaxN = kTopkSmemMaxN;   // rows up to this length: one CTA per row

bool topk_uses_large(const csahca_indexer_args* a) { return a->N > kTopkSmallMaxN; }

// Scratch of the multi-CTA top-k for `rows` rows of length N.
struct TopkLargeLayout { size_t hist, counters, above, cand, total; };
TopkLargeLayout topk_large_layout(int64_t rows, int N, int k) {
  TopkLargeLayout L;
  size_t off = 0;
  L.hist = off; off += align_up((size_t)rows * kHistBins * 4, 256);
  L.counters = off; off += align_up((size_t)rows * kTopkCounters * 4, 256);
  L.above = off; off += align_up((size_t)rows * k * 4, 256);
  L.cand = off; off += align_up((size_t)rows * N * 8, 256);
  L.total = off;
  return L;
}

size_t indexer_scores_bytes(const csahca_indexer_args* a) {
  if (a->scores_out || a->B == 0 || a->nq == 0) return 0;
  return align_up((size_t)a->B * indexer_chunk_rows(a) * (size_t)(a->N > 0 ? a->N : 1) * 4, 256);
}

size_t indexer_workspace(const csahca_indexer_args* a) {
  if (a->B == 0 || a->nq == 0) return 0;
  size_t w = indexer_scores_bytes(a);
  if (topk_uses_large(a)) {
    const int64_t rows = a->scores_out ? (a->nq < 65535 ? a->nq : 65535) : (int64_t)a->B * indexer_chunk_rows(a);
    w += topk_large_layout(rows, a->N, a->k).total;
  }
  return w;
}

// Zeroes `bytes` (a multiple of 16, 16-byte aligned) of scratch in the stream.
int launch_zero(char* ptr, size_t bytes, cudaStream_t s) {
  const int64_t n16 = (int64_t)(bytes / 16);
  if (n16 == 0) return CSAHCA_OK;
  int64_t blocks = ceil_div64(n16, 256);
  if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
  {
    CSAHCA_TRACE("zero_scratch", s);
    launch_k(zero16_kernel, dim3((unsigned)blocks), dim3(256), 0, s, reinterpret_cast<uint4*>(ptr), n16);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// Top-k of `rows` score rows (row r at scores + r * stride, position q_pos[r]).
// Long rows use the multi-CTA path; hist_ready means the indexer has already
// zeroed the scratch and built the row histograms (pass 1) while scoring.
int launch_topk(const csahca_indexer_args* a, const float* scores, int64_t stride, const int* q_pos, int* idx,
                int rows, char* scratch, cudaStream_t s, bool hist_ready = false,
                const void* prefetch_base = nullptr, int64_t prefetch_row_bytes = 0, bool sorted = true,
                bool routed = false) {
  if (!topk_uses_large(a)) {
    TopkParams tp;
    tp.scores = scores; tp.row_stride = stride; tp.q_pos = q_pos; tp.idx = idx;
    tp.B = 1; tp.nq = rows; tp.N = a->N; tp.m = a->m; tp.k = a->k;
    tp.q_begin = 0; tp.q_count = rows; tp.entry_base = a->entry_base;
    CSAHCA_TRACE("topk_rows", s);
    launch_k(topk_rows_sample_kernel, dim3(rows), dim3(kTopkStreamThreads), 0, s, tp);
    CSAHCA_CHECK_LAUNCH();
    return CSAHCA_OK;
  }
  if (a->N > kTopkLargeMaxN) return CSAHCA_ERR_UNSUPPORTED;
  const TopkLargeLayout L = topk_large_layout(rows, a->N, a->k);
  TopkLargeParams tp;
  tp.scores = scores; tp.row_stride = stride; tp.q_pos = q_pos; tp.idx = idx;
  tp.rows = rows; tp.N = a->N; tp.m = a->m; tp.k = a->k; tp.entry_base = a->entry_base;
  int slices = (int)ceil_div64(2 * num_sms(), rows);
  const int max_slices = (int)ceil_div64(a->N, 2048);
  if (slices > max_slices) slices = max_slices;
  if (slices < 1) slices = 1;
  tp.slices = slices;
  tp.hist = reinterpret_cast<uint32_t*>(scratch + L.hist);
  tp.counters = reinterpret_cast<uint32_t*>(scratch + L.counters);
  tp.above = reinterpret_cast<int*>(scratch + L.above);
  tp.cand = reinterpret_cast<uint2*>(scratch + L.cand);
  tp.thresh_ready = hist_ready ? 1 : 0;
  tp.sorted = sorted ? 1 : 0;
  tp.prefetch_base = static_cast<const char*>(prefetch_base);
  tp.prefetch_row_bytes = prefetch_row_bytes;
  if (routed) {
    // the indexer has routed every key into the taken / candidate lists
    const int smem = topk_select_smem_bytes(a->N);
    cudaFuncSetAttribute(topk_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    {
      CSAHCA_TRACE("topk_finish", s);
      launch_k(topk_finish_kernel, dim3(rows), dim3(kTopkSelectThreads), smem, s, tp);
    }
    CSAHCA_CHECK_LAUNCH();
    return CSAHCA_OK;
  }
  if (!hist_ready) {
    {
      const int st = launch_zero(scratch + L.hist, L.above - L.hist, s);
      if (st != CSAHCA_OK) return st;
    }
    {
      CSAHCA_TRACE("topk_hist", s);
      launch_k(topk_hist_kernel, dim3(rows * slices), dim3(512), 0, s, tp);
    }
    CSAHCA_CHECK_LAUNCH();
  }
  const int smem = topk_select_smem_bytes(a->N);
  cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  {
    CSAHCA_TRACE("topk_select", s);
    launch_k(topk_select_kernel, dim3(rows * slices), dim3(kTopkSelectThreads), smem, s, tp);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

template <typename TQ, typename TK, bool kFP8>
void launch_indexer_simt(const IndexerParams& p, cudaStream_t s) {
  const size_t smem = ((size_t)p.HI * p.dI + p.HI) * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(indexer_scores_simt<TQ, TK, kFP8>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((unsigned)ceil_div64(p.N, 256), (unsigned)p.q_count, (unsigned)p.B);
  CSAHCA_TRACE("indexer_scores_simt", s);
  launch_k(indexer_scores_simt<TQ, TK, kFP8>, dim3(grid), dim3(256), smem, s, p);
}

bool indexer_tc_eligible(const csahca_indexer_args* a) {
  return a->q_dtype == CSAHCA_BF16 && (a->k_dtype == CSAHCA_BF16 || a->k_dtype == CSAHCA_E4M3) &&
         a->HI == 64 && a->dI == kIdxTcDim && a->N > 0;
}

template <int QT, bool kFP8>
int launch_indexer_tc_t(const csahca_indexer_args* a, IdxTcParams p, cudaStream_t s) {
  using Cfg = IdxTcCfg<QT, 64, kFP8>;
  CUtensorMap kmap, qmap;
  bool ok;
  if (kFP8)
    ok = encode_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a->kI, (uint64_t)a->dI, (uint64_t)a->B * a->N, 128, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    ok = encode_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->kI, (uint64_t)a->dI, (uint64_t)a->B * a->N, 64,
                   128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && encode_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->qI, (uint64_t)a->dI,
                       (uint64_t)a->B * a->nq * a->HI, 64, (uint32_t)Cfg::NCOL, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return CSAHCA_ERR_LAUNCH;
  auto kern = indexer_tc_kernel<QT, 64, kFP8>;
  // a routed decode scan keeps its item's scores beside the key stages
  const int smem = Cfg::SMEM + (p.route ? p.tiles_per_split * 128 * 4 : 0);
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  if (grid <= 0) return CSAHCA_OK;
  CSAHCA_TRACE(QT == 1 ? "indexer_scores_tc_decode" : "indexer_scores_tc_prefill", s);
  launch_k(kern, dim3(grid), dim3(kIdxTcThreads), smem, s, kmap, qmap, p);
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// Tensor-core scores for queries [q0, q0 + qc) into scores (row stride N).
// Decode split of a routed scan: each sequence's key tiles over about one CTA
// per SM, one work item per CTA.
void decode_split(const csahca_indexer_args* a, int* tiles_per_split, int* splits) {
  const int tiles = (int)ceil_div64(a->N, 128);
  int sp = num_sms() / (a->B > 0 ? a->B : 1);
  if (sp > tiles) sp = tiles;
  if (sp < 1) sp = 1;
  *tiles_per_split = (int)ceil_div64(tiles, sp);
  *splits = (int)ceil_div64(tiles, *tiles_per_split);
}

// A decode scan (e4m3 or bf16 keys) can route the top-k in its epilogue when
// every work item has a CTA of its own (a CTA waits for its row's other
// items) and the item's scores fit in shared memory beside the key stages.
bool decode_route_ok(const csahca_indexer_args* a) {
  int tps = 0, sp = 0;
  decode_split(a, &tps, &sp);
  return a->B * sp <= num_sms() && tps <= kRouteMaxTiles;
}

int launch_indexer_tc(const csahca_indexer_args* a, int q0, int qc, float* scores, int64_t stride,
                      cudaStream_t s, uint32_t* hist = nullptr, uint32_t* counters = nullptr, int* above = nullptr,
                      uint2* cand = nullptr) {
  IdxTcParams p;
  memset(&p, 0, sizeof(p));
  p.hist = hist;
  p.first_kernel = hist ? 0 : 1;           // with histograms, the zeroing kernel runs first
  p.counters = counters;
  p.k = a->k;
  p.w = a->w; p.kI_scale = a->kI_scale; p.q_pos = a->q_pos;
  p.scores = scores; p.score_row_stride = stride;
  p.B = a->B; p.nq = a->nq; p.HI = a->HI; p.N = a->N; p.m = a->m; p.entry_base = a->entry_base;
  p.q_begin = q0; p.q_count = qc;
  if (a->k_dtype == CSAHCA_E4M3) {
    // e4m3 keys straight into the FP8 tensor cores, one query per work item;
    // decode spreads each sequence's key tiles over about one CTA per SM
    if (qc == 1) {
      decode_split(a, &p.tiles_per_split, &p.splits);
      p.n_items = a->B * p.splits;
    } else {
      p.splits = 0;
      p.n_items = a->B * qc;
    }
    p.items_per_row = p.splits > 0 ? p.splits : 1;
    p.route = above != nullptr ? 1 : 0;
    p.above = above;
    p.cand = cand;
    using Cfg = IdxF8Cfg<64>;
    CUtensorMap kmap;
    if (!encode_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a->kI, (uint64_t)a->dI, (uint64_t)a->B * a->N, 128, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return CSAHCA_ERR_LAUNCH;
    const int smem = Cfg::SMEM + (p.route ? p.tiles_per_split * 128 * 4 : 0);
    cudaFuncSetAttribute(indexer_f8_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
    if (grid <= 0) return CSAHCA_OK;
    CSAHCA_TRACE("indexer_scores_f8", s);
    launch_k(indexer_f8_kernel<64>, dim3(grid), dim3(kIdxF8Threads), smem, s, kmap, static_cast<const __nv_bfloat16*>(a->qI), p);
    CSAHCA_CHECK_LAUNCH();
    return CSAHCA_OK;
  }
  if (qc == 1) {
    if (above != nullptr) {
      // routed: one work item per CTA; the epilogue keeps the item's scores
      // and histogram and routes its keys (indexer_tc.cuh)
      decode_split(a, &p.tiles_per_split, &p.splits);
      p.route = 1;
      p.above = above;
      p.cand = cand;
    } else {
      const int tiles = (int)ceil_div64(a->N, 128);
      int splits = (int)ceil_div64(2 * num_sms(), a->B);
      if (splits > tiles) splits = tiles;
      if (splits < 1) splits = 1;
      p.tiles_per_split = (int)ceil_div64(tiles, splits);
      p.splits = (int)ceil_div64(tiles, p.tiles_per_split);
    }
    p.n_items = a->B * p.splits;
    p.items_per_row = p.splits;
    return launch_indexer_tc_t<1, false>(a, p, s);
  }
  p.splits = 0;
  p.n_items = a->B * (int)ceil_div64(qc, 4);
  return launch_indexer_tc_t<4, false>(a, p, s);
}

// sel[r][j] = scores[r][idx[r][j]] for `rows` consecutive rows.
int launch_select_scores(const float* scores, int64_t stride, const int* idx, float* sel, int rows, int k,
                         cudaStream_t s) {
  if (rows <= 0) return CSAHCA_OK;
  {
    CSAHCA_TRACE("select_scores", s);
    launch_k(select_scores_kernel, dim3((unsigned)rows), dim3(256), 0, s, scores, stride, idx, sel, k);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// prefetch_base / prefetch_row_bytes (internal, decode only): every selected
// row of a long row's top-k is prefetched into L2 from that [B][N] table.
int run_indexer(const csahca_indexer_args* a, void* stream, const void* prefetch_base = nullptr,
                int64_t prefetch_row_bytes = 0, bool sorted = true) {
  int st = validate_indexer(a);
  if (st != CSAHCA_OK) return st;
  if (a->B == 0 || a->nq == 0) return CSAHCA_OK;
  if ((st = device_ok()) != CSAHCA_OK) return st;
  const size_t need = indexer_workspace(a);
  if (need && (!a->workspace || a->workspace_bytes < need)) return CSAHCA_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const int chunk = a->scores_out ? (a->nq < 65535 ? a->nq : 65535) : indexer_chunk_rows(a);
  for (int q0 = 0; q0 < a->nq; q0 += chunk) {
    const int qc = (a->nq - q0) < chunk ? (a->nq - q0) : chunk;
    IndexerParams p;
    p.qI = a->qI; p.w = a->w; p.kI = a->kI; p.kI_scale = a->kI_scale; p.q_pos = a->q_pos;
    p.B = a->B; p.nq = a->nq; p.HI = a->HI; p.dI = a->dI; p.N = a->N; p.m = a->m;
    p.q_begin = q0; p.q_count = qc; p.entry_base = a->entry_base;
    // scores rows of this chunk: row (b, q) -> b * qc + (q - q0); with
    // scores_out the full [B, nq, N] layout is addressed through the stride.
    float* base;
    int64_t stride = a->N > 0 ? a->N : 1;
    if (a->scores_out) {
      // one launch per batch entry keeps the [B, nq, N] layout
      for (int b = 0; b < a->B; ++b) {
        IndexerParams pb = p;
        pb.B = 1;
        pb.qI = static_cast<const char*>(a->qI) + (int64_t)b * a->nq * a->HI * a->dI * dtype_size(a->q_dtype);
        pb.w = a->w + (int64_t)b * a->nq * a->HI;
        pb.kI = a->kI ? static_cast<const char*>(a->kI) + (int64_t)b * a->N * a->dI * dtype_size(a->k_dtype) : nullptr;
        pb.kI_scale = a->kI_scale ? a->kI_scale + (int64_t)b * a->N * (a->dI / 128) : nullptr;
        pb.q_pos = a->q_pos + (int64_t)b * a->nq;
        pb.scores = a->scores_out + ((int64_t)b * a->nq + q0) * stride;
        pb.score_row_stride = stride;
        if (indexer_tc_eligible(a)) {
          csahca_indexer_args ab = *a;
          ab.B = 1; ab.qI = pb.qI; ab.w = pb.w; ab.kI = pb.kI; ab.kI_scale = pb.kI_scale; ab.q_pos = pb.q_pos;
          int st2 = launch_indexer_tc(&ab, q0, qc, pb.scores, stride, s);
          if (st2 != CSAHCA_OK) return st2;
        } else if (a->N > 0) {
          if (a->k_dtype == CSAHCA_E4M3) {
            if (a->q_dtype == CSAHCA_BF16) launch_indexer_simt<__nv_bfloat16, uint8_t, true>(pb, s);
            else launch_indexer_simt<float, uint8_t, true>(pb, s);
          } else if (a->q_dtype == CSAHCA_BF16) {
            launch_indexer_simt<__nv_bfloat16, __nv_bfloat16, false>(pb, s);
          } else {
            launch_indexer_simt<float, float, false>(pb, s);
          }
          CSAHCA_CHECK_LAUNCH();
        }
        int st3 = launch_topk(a, pb.scores, stride, pb.q_pos + q0, a->idx + ((int64_t)b * a->nq + q0) * a->k, qc,
                              static_cast<char*>(a->workspace), s);
        if (st3 != CSAHCA_OK) return st3;
        if (a->sel_scores) {
          const int64_t r0 = (int64_t)b * a->nq + q0;
          st3 = launch_select_scores(pb.scores, stride, a->idx + r0 * a->k, a->sel_scores + r0 * a->k, qc, a->k, s);
          if (st3 != CSAHCA_OK) return st3;
        }
      }
      continue;
    }
    base = static_cast<float*>(a->workspace);
    p.scores = base;
    p.score_row_stride = stride;
    char* scratch = static_cast<char*>(a->workspace) + indexer_scores_bytes(a);
    // decode with e4m3 keys: the FP8 indexer builds the top-k row histograms
    // while it writes the scores (the scratch it adds into is zeroed first)
    // (with bf16 keys only when the scan also routes: its epilogue has no
    // last-item threshold for the select kernel)
    const bool fuse_hist = qc == a->nq && topk_uses_large(a) && indexer_tc_eligible(a) && a->N <= kTopkLargeMaxN &&
                           (a->k_dtype == CSAHCA_E4M3 ||
                            (a->k_dtype == CSAHCA_BF16 && a->nq == 1 && decode_route_ok(a) && !a->sel_scores));
    uint32_t* hist = nullptr;
    uint32_t* counters = nullptr;
    int* above = nullptr;
    uint2* cand = nullptr;
    // decode with e4m3 keys and one CTA per work item: the indexer also
    // routes the keys into the top-k lists from shared memory, and one CTA
    // per row finishes
    // (sel_scores reads the scores back: they must reach the workspace)
    const bool route = fuse_hist && a->nq == 1 && decode_route_ok(a) && !a->sel_scores;
    if (fuse_hist) {
      const TopkLargeLayout L = topk_large_layout((int64_t)a->B * qc, a->N, a->k);
      const int zst = launch_zero(scratch + L.hist, L.above - L.hist, s);
      if (zst != CSAHCA_OK) return zst;
      hist = reinterpret_cast<uint32_t*>(scratch + L.hist);
      counters = reinterpret_cast<uint32_t*>(scratch + L.counters);
      if (route) {
        above = reinterpret_cast<int*>(scratch + L.above);
        cand = reinterpret_cast<uint2*>(scratch + L.cand);
      }
    }
    if (indexer_tc_eligible(a)) {
      int st2 = launch_indexer_tc(a, q0, qc, base, stride, s, hist, counters, above, cand);
      if (st2 != CSAHCA_OK) return st2;
    } else if (a->N > 0) {
      if (a->k_dtype == CSAHCA_E4M3) {
        if (a->q_dtype == CSAHCA_BF16) launch_indexer_simt<__nv_bfloat16, uint8_t, true>(p, s);
        else launch_indexer_simt<float, uint8_t, true>(p, s);
      } else if (a->q_dtype == CSAHCA_BF16) {
        launch_indexer_simt<__nv_bfloat16, __nv_bfloat16, false>(p, s);
      } else {
        launch_indexer_simt<float, float, false>(p, s);
      }
      CSAHCA_CHECK_LAUNCH();
    }
    // rows of this chunk: (b, q) -> b * qc + (q - q0); positions and outputs are
    // addressed per batch entry, so launch per b unless the chunk is the whole nq
    if (qc == a->nq) {
      int st3 = launch_topk(a, base, stride, a->q_pos, a->idx, a->B * qc, scratch, s, fuse_hist,
                            a->nq == 1 ? prefetch_base : nullptr, prefetch_row_bytes, sorted, route);
      if (st3 != CSAHCA_OK) return st3;
      if (a->sel_scores) {
        st3 = launch_select_scores(base, stride, a->idx, a->sel_scores, a->B * qc, a->k, s);
        if (st3 != CSAHCA_OK) return st3;
      }
    } else {
      for (int b = 0; b < a->B; ++b) {
        const int64_t r0 = (int64_t)b * a->nq + q0;
        int st3 = launch_topk(a, base + (int64_t)b * qc * stride, stride, a->q_pos + (int64_t)b * a->nq + q0,
                              a->idx + r0 * a->k, qc, scratch, s);
        if (st3 != CSAHCA_OK) return st3;
        if (a->sel_scores) {
          st3 = launch_select_scores(base + (int64_t)b * qc * stride, stride, a->idx + r0 * a->k,
                                     a->sel_scores + r0 * a->k, qc, a->k, s);
          if (st3 != CSAHCA_OK) return st3;
        }
      }
    }
  }
  return CSAHCA_OK;
}

// ----------------------------------------------------------------- prefill --

int validate_attn(const csahca_attn_args* a, bool shapes_only = false) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->kind != CSAHCA_CSA && a->kind != CSAHCA_HCA) return CSAHCA_ERR_INVALID_ARG;
  if (a->dtype != CSAHCA_F32 && a->dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->B < 0 || a->n < 0 || a->H < 1 || a->d < 1 || a->N < 0 || a->m < 1 || a->w < 0)
    return CSAHCA_ERR_INVALID_ARG;
  if (a->kind == CSAHCA_CSA && a->k < 1) return CSAHCA_ERR_INVALID_ARG;
  if (a->rope_dims < 0 || a->rope_dims > a->d || (a->rope_dims & 1)) return CSAHCA_ERR_INVALID_ARG;
  if (a->d % 32 || a->d > 32 * kSimtMaxDPL) return CSAHCA_ERR_UNSUPPORTED;
  if (shapes_only || a->B == 0 || a->n == 0) return CSAHCA_OK;
  if (!a->q || !a->sinks || !a->out) return CSAHCA_ERR_INVALID_ARG;
  if (a->N > 0 && !a->kv_comp) return CSAHCA_ERR_INVALID_ARG;
  if (a->w > 0 && !a->kv_win) return CSAHCA_ERR_INVALID_ARG;
  if (a->kind == CSAHCA_CSA && !a->idx) return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->q, a->kv_comp, a->kv_win, a->q_gain, a->kv_gain, a->idx, a->sinks,
                        a->out, a->workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  return CSAHCA_OK;
}

size_t prefill_workspace(const csahca_attn_args* a) {
  if (a->B == 0 || a->n == 0 || a->w == 0) return 0;
  return align_up((size_t)a->B * a->n * a->d * dtype_size(a->dtype), 256);
}

template <typename T>
int launch_finish(const void* x, void* out, const float* gain, int64_t rows, int c, int group,
                  int npos, int rms, int r, double base, float eps, cudaStream_t s) {
  FinishParams f;
  f.x = x; f.out = out; f.gain = gain; f.rows = rows; f.c = c; f.group = group; f.npos = npos;
  f.rms_norm = rms; f.rope_dims = r; f.rope_base = base; f.eps = eps;
  const int64_t blocks = ceil_div64(rows * 32, 256);
  CSAHCA_TRACE("finish_rows", s);
  launch_k(finish_rows_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, s, f);
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

template <typename T>
int launch_simt_attn(const SimtAttnParams& p, int nq_total, cudaStream_t s, const char* name) {
  const size_t smem = ((size_t)kSimtHG * p.d + (size_t)kSimtKeys * (p.d + 1)) * sizeof(float);
  cudaFuncSetAttribute(attn_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((unsigned)nq_total, (unsigned)ceil_div64(p.H, kSimtHG), (unsigned)p.splits);
  CSAHCA_TRACE(name, s);
  launch_k(attn_simt_kernel<T>, dim3(grid), dim3(32 * kSimtHG), smem, s, p);
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// ---- tensor-core attention (H = 64, d = 512, bf16) ---------------------------

bool attn_tc_shape_ok(int dtype, int H, int d, int rope_dims, int64_t comp_rows, int64_t win_rows) {
  return dtype == CSAHCA_BF16 && H == kAttnH && d == kAttnD && rope_dims <= 128 && comp_rows >= 128 &&
         win_rows >= 128;
}

// FP8 KV rows (the header's layout): bytes per row, 0 for an invalid combination.
int64_t kv_f8_row_bytes(int d, int r) {
  if (d <= 0 || r < 0 || r > d || (d - r) % 64 || r % 64) return 0;
  const int64_t raw = (int64_t)(d - r) + 2 * (int64_t)r + 4 * (int64_t)((d - r) / 64);
  return (raw + 127) / 128 * 128;
}

int launch_attn_tc(const AttnTcParams& p_in, const void* kv_comp, int64_t comp_rows, const void* win,
                   int64_t win_rows, cudaStream_t s, const char* name, bool f8 = false) {
  AttnTcParams p = p_in;
  rope_theta_table(p.theta, p.rope_dims, p.rope_base);
  if (f8) {
    p.kv_f8 = static_cast<const uint8_t*>(kv_comp);
    p.kv_row_bytes = kv_f8_row_bytes(kAttnD, p.rope_dims);
    p.f8_nope_chunks = (kAttnD - p.rope_dims) / 64;
  }
  p.win_ptr = static_cast<const __nv_bfloat16*>(win ? win : kv_comp);
  p.comp_rows_total = comp_rows;
  p.win_rows_total = win ? win_rows : comp_rows;
  // rows of d = 512 bf16 seen as [chunk 8][row][64]: a key box is one chunk
  // of 128 rows (16 KB); the query box is all 8 chunks x 64 heads (64 KB),
  // landing chunk-major with the 128-byte swizzle as the MMA operand wants it
  CUtensorMap m_rows, m_win, m_q, m_rope, m_scale;
  const uint64_t rs = kAttnD * 2;
  bool ok;
  if (f8) {
    // FP8 rows as bytes: 64-byte code boxes, the 128-byte RoPE chunks with the
    // MMA's swizzle, 32-byte scale boxes (all 128 rows)
    const uint64_t rb = (uint64_t)p.kv_row_bytes;
    ok = encode_2d(&m_rows, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kv_comp, rb, (uint64_t)comp_rows, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE) &&
         encode_2d(&m_rope, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kv_comp, rb, (uint64_t)comp_rows, 128, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_2d(&m_scale, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kv_comp, rb, (uint64_t)comp_rows, 32, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    ok = encode_3d(&m_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv_comp, 64, (uint64_t)comp_rows, kAttnChunks, rs,
                   128, 64, 128, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (win) ok = ok && encode_3d(&m_win, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, win, 64, (uint64_t)win_rows, kAttnChunks,
                                rs, 128, 64, 128, 1, CU_TENSOR_MAP_SWIZZLE_128B);
  else m_win = m_rows;
  ok = ok && encode_3d(&m_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, 64, (uint64_t)p.B * p.nq * kAttnH, kAttnChunks,
                       rs, 128, 64, kAttnH, kAttnChunks, CU_TENSOR_MAP_SWIZZLE_128B);
  // decode partials as 128-byte bf16 rows, stored 128 rows (one O^T M-tile) per box
  CUtensorMap m_part = m_rows;
  if (p.decode)
    ok = ok && encode_2d(&m_part, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.partial, kAttnH,
                         (uint64_t)p.B * p.nq * p.splits * kTcPartialRows, kAttnH, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return CSAHCA_ERR_LAUNCH;
  if (!f8) m_rope = m_scale = m_rows;                  // not read
  const int smem = AttnSmem::TOTAL + (f8 ? AttnSmem::F8_SCALES : 0);
  // decode and prefill are separate instances: each carries only its own
  // epilogue (a smaller kernel stalls less on instruction fetch)
  auto kern = p.decode ? (f8 ? attn_tc_kernel<true, true> : attn_tc_kernel<true, false>) : attn_tc_kernel<false, false>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (!p.decode) {
    // the prefill instance moves registers between warpgroups: the counts after
    // the move must fit the launch allocation, else an increase would wait
    static int launch_regs = -1;
    if (launch_regs < 0) {
      cudaFuncAttributes fa;
      launch_regs = cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : 0;
    }
    if ((int64_t)launch_regs * attn_threads<false>() < attn_prefill_regs_needed()) return CSAHCA_ERR_UNSUPPORTED;
  }
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  if (grid <= 0) return CSAHCA_OK;
  CSAHCA_TRACE(name, s);
  launch_k(kern, dim3(grid), dim3(p.decode ? attn_threads<true>() : attn_threads<false>()), smem, s, m_rows,
           m_win, m_q, m_part, m_rope, m_scale, p);
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// ---- tensor-core attention for 16 heads of 128 dims (HCA prefill, bf16) ------

bool attn_small_tc_ok(const csahca_attn_args* a) {
  return a->dtype == CSAHCA_BF16 && a->kind == CSAHCA_HCA && a->H == kSmH && a->d == kSmD &&
         a->rope_dims <= 128;
}

int launch_attn_small(const csahca_attn_args* a, const void* win_final, double base, float eps, float scale,
                      cudaStream_t s) {
  AttnSmallParams t;
  memset(&t, 0, sizeof(t));
  t.q = static_cast<const __nv_bfloat16*>(a->q); t.q_gain = a->q_gain; t.sinks = a->sinks;
  t.q_norm = a->q_norm; t.eps = eps; t.scale_log2 = scale * kLog2e; t.rope_dims = a->rope_dims;
  t.B = a->B; t.n = a->n; t.N = a->N; t.m = a->m; t.w = a->w;
  t.n_items = a->B * (int)ceil_div64(a->n, kSmQ);
  t.first_kernel = a->w > 0 ? 0 : 1;
  t.out = static_cast<__nv_bfloat16*>(a->out);
  rope_theta_table(t.theta, a->rope_dims, base);
  // rows of 128 bf16 seen as [chunk 2][row][64]: one box = 128 key rows x both
  // chunks (32 KB), the query box = 64 rows x both chunks (16 KB)
  const uint64_t rs = kSmD * 2;
  CUtensorMap m_q, m_comp, m_win;
  bool ok = encode_3d(&m_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a->q, 64, (uint64_t)a->B * a->n * kSmH, 2, rs, 128, 64,
                      kSmN, 2, CU_TENSOR_MAP_SWIZZLE_128B);
  m_comp = m_q;
  m_win = m_q;
  if ((int64_t)a->B * a->N > 0)
    ok = ok && encode_3d(&m_comp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a->kv_comp, 64, (uint64_t)a->B * a->N, 2, rs,
                         128, 64, 128, 2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (a->w > 0)
    ok = ok && encode_3d(&m_win, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, win_final, 64, (uint64_t)a->B * a->n, 2, rs, 128,
                         64, 128, 2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return CSAHCA_ERR_LAUNCH;
  cudaFuncSetAttribute(attn_small_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SmSmem::TOTAL);
  int grid = 2 * num_sms();
  if (grid > t.n_items) grid = t.n_items;
  if (grid <= 0) return CSAHCA_OK;
  CSAHCA_TRACE("attn_prefill_hca_small_tc", s);
  launch_k(attn_small_tc_kernel, dim3(grid), dim3(kSmThreads), SmSmem::TOTAL, s, m_comp, m_win, m_q, t);
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

template <typename T>
int run_prefill_t(const csahca_attn_args* a, cudaStream_t s) {
  const double base = a->rope_base > 0 ? a->rope_base : kDefaultRopeBase;
  const float eps = a->eps > 0 ? a->eps : kDefaultEps;
  void* win_final = nullptr;
  if (a->w > 0) {
    win_final = a->workspace;
    int st = launch_finish<T>(a->kv_win, win_final, a->kv_gain, (int64_t)a->B * a->n, a->d, 1,
                              a->n, a->kv_norm, a->rope_dims, base, eps, s);
    if (st != CSAHCA_OK) return st;
  }
  const float scale = a->scale > 0 ? a->scale : 1.0f / sqrtf((float)a->d);
  if (attn_small_tc_ok(a)) return launch_attn_small(a, win_final, base, eps, scale, s);
  if (attn_tc_shape_ok(a->dtype, a->H, a->d, a->rope_dims, (int64_t)a->B * a->N, (int64_t)a->B * a->n)) {
    AttnTcParams t;
    memset(&t, 0, sizeof(t));
    t.q = static_cast<const __nv_bfloat16*>(a->q); t.q_gain = a->q_gain; t.sinks = a->sinks; t.pos = nullptr;
    t.kv_comp_ptr = static_cast<const __nv_bfloat16*>(a->kv_comp);
    t.q_norm = a->q_norm; t.eps = eps; t.scale_log2 = scale * kLog2e; t.rope_dims = a->rope_dims;
    t.rope_base = base; t.B = a->B; t.nq = a->n; t.N = a->N; t.m = a->m; t.k = a->k; t.w = a->w;
    t.csa = a->kind == CSAHCA_CSA; t.idx = a->idx; t.decode = 0;
    t.n_items = a->B * a->n; t.splits = 1; t.tiles_per_split = 0; t.gtile = 128; t.first_kernel = a->w > 0 ? 0 : 1;
    t.out = static_cast<__nv_bfloat16*>(a->out); t.partial = nullptr;
    return launch_attn_tc(t, a->kv_comp, (int64_t)a->B * a->N, win_final, (int64_t)a->B * a->n, s,
                          a->kind == CSAHCA_CSA ? "attn_prefill_csa_tc" : "attn_prefill_hca_tc");
  }
  SimtAttnParams p;
  memset(&p, 0, sizeof(p));
  p.q = a->q; p.q_gain = a->q_gain; p.sinks = a->sinks; p.pos = nullptr;
  p.q_norm = a->q_norm; p.eps = eps; p.scale = scale;
  p.rope_dims = a->rope_dims; p.rope_base = base;
  p.B = a->B; p.nq = a->n; p.H = a->H; p.d = a->d;
  p.kv_comp = a->kv_comp; p.N = a->N;
  p.idx = a->kind == CSAHCA_CSA ? a->idx : nullptr; p.k = a->k; p.m = a->m;
  p.win = win_final; p.w = a->w; p.decode = 0;
  p.splits = 1; p.keys_per_split = INT32_MAX / 2;
  p.out = a->out; p.partial = nullptr;
  return launch_simt_attn<T>(p, a->B * a->n, s,
                             a->kind == CSAHCA_CSA ? "attn_prefill_csa_simt" : "attn_prefill_hca_simt");
}

int run_prefill(const csahca_attn_args* a, void* stream) {
  int st = validate_attn(a);
  if (st != CSAHCA_OK) return st;
  if (a->B == 0 || a->n == 0) return CSAHCA_OK;
  if ((st = device_ok()) != CSAHCA_OK) return st;
  const size_t need = prefill_workspace(a);
  if (need && (!a->workspace || a->workspace_bytes < need)) return CSAHCA_ERR_WORKSPACE;
  if ((int64_t)a->B * a->n > INT32_MAX) return CSAHCA_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  return a->dtype == CSAHCA_F32 ? run_prefill_t<float>(a, s) : run_prefill_t<__nv_bfloat16>(a, s);
}

// ------------------------------------------------------------------ decode --

constexpr int kDecodeKeysPerSplit = 256;

bool decode_tc(const csahca_decode_args* a);

int validate_decode(const csahca_decode_args* a, bool shapes_only = false) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->kind != CSAHCA_CSA && a->kind != CSAHCA_HCA) return CSAHCA_ERR_INVALID_ARG;
  if (a->dtype != CSAHCA_F32 && a->dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 1 || a->d < 1 || a->N_cap < 0 || a->m < 1 || a->w < 0 || a->entry_base < 0)
    return CSAHCA_ERR_INVALID_ARG;
  if (a->rope_dims < 0 || a->rope_dims > a->d || (a->rope_dims & 1)) return CSAHCA_ERR_INVALID_ARG;
  if (a->d % 32 || a->d > 32 * kSimtMaxDPL) return CSAHCA_ERR_UNSUPPORTED;
  // context parallelism: the tensor-core path only; a CSA shard past the
  // first takes its selection from cp_topk_merge
  const bool cp = a->entry_base > 0 || a->partial_out || a->skip_window;
  if (cp && !decode_tc(a)) return CSAHCA_ERR_UNSUPPORTED;
  if (a->kind == CSAHCA_CSA && a->entry_base > 0 && !a->idx_in) return CSAHCA_ERR_INVALID_ARG;
  if (a->kv_dtype == CSAHCA_E4M3 &&
      (a->dtype != CSAHCA_BF16 || !decode_tc(a) || kv_f8_row_bytes(a->d, a->rope_dims) == 0))
    return CSAHCA_ERR_UNSUPPORTED;
  if (a->kind == CSAHCA_CSA) {
    if (a->k < 1) return CSAHCA_ERR_INVALID_ARG;
    if (!a->idx_in) {
      csahca_indexer_args ia;
      memset(&ia, 0, sizeof(ia));
      ia.q_dtype = a->qI_dtype; ia.k_dtype = a->kI_dtype; ia.B = a->B; ia.nq = 1; ia.HI = a->HI;
      ia.dI = a->dI; ia.N = a->N_cap; ia.m = a->m; ia.k = a->k;
      ia.qI = a->qI; ia.w = a->wI; ia.kI = a->kI; ia.kI_scale = a->kI_scale;
      int st = validate_indexer(&ia, /*shapes_only=*/true);
      if (st != CSAHCA_OK) return st;
    }
  }
  if (shapes_only || a->B == 0) return CSAHCA_OK;
  if (!a->q || !a->pos || !a->sinks || (!a->out && !a->partial_out)) return CSAHCA_ERR_INVALID_ARG;
  if (a->kind == CSAHCA_CSA && !a->idx_in && (!a->qI || !a->wI || (a->N_cap > 0 && !a->kI) ||
                                              (a->kI_dtype == CSAHCA_E4M3 && a->N_cap > 0 && !a->kI_scale)))
    return CSAHCA_ERR_INVALID_ARG;
  if (a->N_cap > 0 && !a->kv_cache) return CSAHCA_ERR_INVALID_ARG;
  if (a->w > 0 && !a->win && !a->skip_window) return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->q, a->pos, a->q_gain, a->kv_cache, a->win, a->sinks, a->qI, a->wI,
                        a->kI, a->kI_scale, a->idx_in, a->idx_out, a->out, a->partial_out, a->workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  return CSAHCA_OK;
}

struct DecodeLayout {
  size_t scores_off, idx_off, partial_off, total;
  int splits;
  bool tc;
  int tiles_per_split;
  int gtile;                    // gathered rows per CSA tile
};

bool decode_tc(const csahca_decode_args* a) {
  // (a skipped window is never read: its tensor map falls back to the cache)
  return attn_tc_shape_ok(a->dtype, a->H, a->d, a->rope_dims, (int64_t)a->B * a->N_cap,
                          a->skip_window ? 128 : (int64_t)a->B * a->w);
}

DecodeLayout decode_layout(const csahca_decode_args* a) {
  DecodeLayout L;
  const bool csa = a->kind == CSAHCA_CSA;
  const bool run_indexer = csa && !a->idx_in;
  const int64_t jmax = (csa ? (int64_t)a->k : (int64_t)a->N_cap) + a->w;
  L.tc = decode_tc(a);
  L.tiles_per_split = 0;
  L.gtile = 128;
  if (L.tc) {
    // tensor-core path: split each query's tiles so that B x splits ~ one
    // wave (gathered CSA tiles of 128 rows: smaller ones, 64 or 32 rows,
    // measured slower at decode_1m, the per-tile fixed costs dominating)
    const int B = a->B > 0 ? a->B : 1;
    const int64_t wt = a->skip_window ? 0 : ceil_div64(a->w, 128);
    const int tiles = (int)(ceil_div64(csa ? a->k : a->N_cap, csa ? L.gtile : 128) + wt);
    int want = (int)ceil_div64(num_sms(), B);
    if (want > kTcCombineMaxSplits) want = kTcCombineMaxSplits;
    if (want < 1) want = 1;
    L.tiles_per_split = (int)ceil_div64(tiles > 0 ? tiles : 1, want);
    L.splits = (int)ceil_div64(tiles > 0 ? tiles : 1, L.tiles_per_split);
  } else {
    L.splits = (int)(jmax > 0 ? ceil_div64(jmax, kDecodeKeysPerSplit) : 1);
  }
  size_t off = 0;
  L.scores_off = off;
  if (run_indexer) {
    csahca_indexer_args ia;
    memset(&ia, 0, sizeof(ia));
    ia.q_dtype = a->qI_dtype; ia.k_dtype = a->kI_dtype; ia.B = a->B; ia.nq = 1; ia.HI = a->HI;
    ia.dI = a->dI; ia.N = a->N_cap; ia.m = a->m; ia.k = a->k;
    off += align_up(indexer_workspace(&ia), 256);
  }
  L.idx_off = off;
  if (csa && !a->idx_out) off += align_up((size_t)a->B * a->k * 4, 256);
  L.partial_off = off;
  if (L.tc) off += align_up((size_t)a->B * L.splits * kTcPartialBytes, 256);
  else off += align_up((size_t)a->B * a->H * L.splits * (a->d + 4) * 4, 256);
  L.total = off;
  return L;
}

template <typename T>
int run_decode_t(const csahca_decode_args* a, cudaStream_t s, char* ws) {
  const DecodeLayout L = decode_layout(a);
  const double base = a->rope_base > 0 ? a->rope_base : kDefaultRopeBase;
  const float eps = a->eps > 0 ? a->eps : kDefaultEps;
  const int32_t* sel = nullptr;
  if (a->kind == CSAHCA_CSA) {
    if (a->idx_in) {
      sel = a->idx_in;
      if (a->idx_out)
        cudaMemcpyAsync(a->idx_out, a->idx_in, (size_t)a->B * a->k * 4, cudaMemcpyDeviceToDevice, s);
    } else {
      int32_t* idx = a->idx_out ? a->idx_out : reinterpret_cast<int32_t*>(ws + L.idx_off);
      csahca_indexer_args ia;
      memset(&ia, 0, sizeof(ia));
      ia.q_dtype = a->qI_dtype; ia.k_dtype = a->kI_dtype; ia.B = a->B; ia.nq = 1; ia.HI = a->HI;
      ia.dI = a->dI; ia.N = a->N_cap; ia.m = a->m; ia.k = a->k;
      ia.qI = a->qI; ia.w = a->wI; ia.kI = a->kI; ia.kI_scale = a->kI_scale;
      ia.q_pos = a->pos; ia.idx = idx;
      ia.workspace = ws + L.scores_off;
      ia.workspace_bytes = L.idx_off - L.scores_off;
      // the attention needs the selected set only: index order is kept
      // when the caller asked for the selection
      int st = run_indexer(&ia, s, nullptr, 0, a->idx_out != nullptr);
      if (st != CSAHCA_OK) return st;
      sel = idx;
    }
  }
  const float scale = a->scale > 0 ? a->scale : 1.0f / sqrtf((float)a->d);
  float* partial = reinterpret_cast<float*>(ws + L.partial_off);
  int st;
  if (L.tc) {
    AttnTcParams t;
    memset(&t, 0, sizeof(t));
    t.q = static_cast<const __nv_bfloat16*>(a->q); t.q_gain = a->q_gain; t.sinks = a->sinks; t.pos = a->pos;
    t.kv_comp_ptr = static_cast<const __nv_bfloat16*>(a->kv_cache);
    t.q_norm = a->q_norm; t.eps = eps; t.scale_log2 = scale * kLog2e; t.rope_dims = a->rope_dims;
    t.rope_base = base; t.B = a->B; t.nq = 1; t.N = a->N_cap; t.m = a->m; t.k = a->k; t.w = a->w;
    t.csa = a->kind == CSAHCA_CSA; t.idx = sel; t.decode = 1;
    t.entry_base = a->entry_base; t.skip_window = a->skip_window ? 1 : 0;
    t.splits = L.splits; t.tiles_per_split = L.tiles_per_split; t.n_items = a->B * L.splits; t.gtile = L.gtile;
    t.first_kernel = (a->kind != CSAHCA_CSA || a->idx_in) ? 1 : 0;
    t.out = nullptr; t.partial = partial;
    const bool f8 = a->kv_dtype == CSAHCA_E4M3;
    st = launch_attn_tc(t, a->kv_cache, (int64_t)a->B * a->N_cap, (a->w > 0 && !a->skip_window) ? a->win : nullptr,
                        (int64_t)a->B * a->w, s,
                        a->kind == CSAHCA_CSA ? (f8 ? "attn_decode_csa_tc_f8kv" : "attn_decode_csa_tc")
                                              : (f8 ? "attn_decode_hca_tc_f8kv" : "attn_decode_hca_tc"),
                        f8);
  } else {
    SimtAttnParams p;
    memset(&p, 0, sizeof(p));
    p.q = a->q; p.q_gain = a->q_gain; p.sinks = a->sinks; p.pos = a->pos;
    p.q_norm = a->q_norm; p.eps = eps; p.scale = scale;
    p.rope_dims = a->rope_dims; p.rope_base = base;
    p.B = a->B; p.nq = 1; p.H = a->H; p.d = a->d;
    p.kv_comp = a->kv_cache; p.N = a->N_cap;
    p.idx = sel; p.k = a->k; p.m = a->m;
    p.win = a->win; p.w = a->w; p.decode = 1;
    p.splits = L.splits; p.keys_per_split = kDecodeKeysPerSplit;
    p.out = nullptr; p.partial = partial;
    st = launch_simt_attn<T>(p, a->B, s, a->kind == CSAHCA_CSA ? "attn_decode_csa_simt" : "attn_decode_hca_simt");
  }
  if (st != CSAHCA_OK) return st;
  if (L.tc) {
    TcCombineParams c;
    c.partial = reinterpret_cast<const char*>(partial); c.sinks = a->sinks; c.pos = a->pos;
    c.out = static_cast<__nv_bfloat16*>(a->out);
    c.partial_out = a->partial_out;
    c.rows = a->B; c.splits = L.splits; c.rope_dims = a->rope_dims;
    rope_theta_table(c.theta, a->rope_dims, base);              // rope_dims <= 128 on this path
    const int smem = tc_combine_smem_bytes(L.splits);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(attn_combine_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // the partials as [B * splits blocks][516 rows][64 bf16]: one box takes
    // the m, l headers of every split of a query, one the 16-dim slices
    CUtensorMap hdr_map, slc_map;
    const uint64_t blocks = (uint64_t)a->B * L.splits;
    const uint32_t slc_box = (uint32_t)(L.splits < kTcCombineSlots ? L.splits : kTcCombineSlots);
    if (!encode_3d(&hdr_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, partial, kAttnH, kTcPartialRows, blocks, kAttnH * 2,
                   kTcPartialBytes, kAttnH, kTcPartialHeaderRows, (uint32_t)L.splits) ||
        !encode_3d(&slc_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, partial, kAttnH, kTcPartialRows, blocks, kAttnH * 2,
                   kTcPartialBytes, kAttnH, kTcCombineDims, slc_box))
      return CSAHCA_ERR_LAUNCH;
    {
      CSAHCA_TRACE("attn_combine", s);
      launch_k(attn_combine_tc_kernel, dim3((unsigned)(a->B * (kAttnD / kTcCombineDims))), dim3(kTcCombineThreads),
               smem, s, hdr_map, slc_map, c);
    }
    CSAHCA_CHECK_LAUNCH();
    return CSAHCA_OK;
  }
  CombineParams c;
  c.partial = partial; c.sinks = a->sinks; c.pos = a->pos; c.out = a->out;
  c.B = a->B; c.nq = 1; c.H = a->H; c.d = a->d; c.splits = L.splits;
  c.rope_dims = a->rope_dims; c.decode = 1; c.rope_base = base;
  {
    CSAHCA_TRACE("attn_combine", s);
    launch_k(attn_combine_kernel<T>, dim3((unsigned)(a->B * a->H)), dim3(128), 0, s, c);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

int run_decode(const csahca_decode_args* a, void* stream, char* ws, size_t ws_bytes) {
  int st = validate_decode(a);
  if (st != CSAHCA_OK) return st;
  if (a->B == 0) return CSAHCA_OK;
  if ((st = device_ok()) != CSAHCA_OK) return st;
  const DecodeLayout L = decode_layout(a);
  if (L.splits > kCombineMaxSplits) return CSAHCA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < L.total) return CSAHCA_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  return a->dtype == CSAHCA_F32 ? run_decode_t<float>(a, s, ws) : run_decode_t<__nv_bfloat16>(a, s, ws);
}

// --------------------------------------------------------- decode_compress --

int run_decode_compress(const csahca_decode_compress_args* a, void* stream) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->kind != CSAHCA_CSA && a->kind != CSAHCA_HCA) return CSAHCA_ERR_INVALID_ARG;
  if (a->dtype != CSAHCA_F32 && a->dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->B < 0 || a->d <= 0 || a->m < 1 || a->N_cap < 0 || a->w < 0 || a->dI < 0 || a->entry_base < 0)
    return CSAHCA_ERR_INVALID_ARG;
  if (a->rope_dims < 0 || a->rope_dims > a->d || (a->rope_dims & 1)) return CSAHCA_ERR_INVALID_ARG;
  if (a->rope_dims > 2 * kDcMaxRopePairs) return CSAHCA_ERR_UNSUPPORTED;
  const bool csa = a->kind == CSAHCA_CSA;
  const int vec = 16 / dtype_size(a->dtype);
  if (a->d % (kDcCluster * vec) || a->d / (kDcCluster * vec) > kDcMaxVecs) return CSAHCA_ERR_UNSUPPORTED;
  const int dI = csa ? a->dI : 0;
  if (dI) {
    const int si = dI / kDcCluster;
    if (dI % kDcCluster || si % vec || 128 % si || si / vec > kDcMaxVecs) return CSAHCA_ERR_UNSUPPORTED;
    if (a->kI_dtype == CSAHCA_E4M3) {
      if (a->dtype != CSAHCA_BF16 || dI % 128) return CSAHCA_ERR_UNSUPPORTED;
    } else if (a->kI_dtype != a->dtype) {
      return CSAHCA_ERR_UNSUPPORTED;
    }
  }
  if (a->B == 0) return CSAHCA_OK;
  if (!a->pos || !a->a || !a->za || !a->bias_a || !a->ring || !a->kv_cache) return CSAHCA_ERR_INVALID_ARG;
  if (csa && (!a->b || !a->zb || !a->bias_b)) return CSAHCA_ERR_INVALID_ARG;
  if (a->kv_raw && a->w > 0 && !a->win) return CSAHCA_ERR_INVALID_ARG;
  if (dI && (!a->ia || !a->ib || !a->iza || !a->izb || !a->ibias_a || !a->ibias_b || !a->iring || !a->kI))
    return CSAHCA_ERR_INVALID_ARG;
  if (dI && a->kI_dtype == CSAHCA_E4M3 && !a->kI_scale) return CSAHCA_ERR_INVALID_ARG;
  // FP8 KV rows: each CTA of a cluster owns one 64-dim block of the row
  const bool kv_f8 = a->kv_dtype == CSAHCA_E4M3;
  if (kv_f8 && (a->dtype != CSAHCA_BF16 || a->d != 64 * kDcCluster || kv_f8_row_bytes(a->d, a->rope_dims) == 0))
    return CSAHCA_ERR_UNSUPPORTED;
  const void* ptrs[] = {a->pos, a->kv_raw, a->a, a->b, a->za, a->zb, a->bias_a, a->bias_b, a->kv_gain,
                        a->ring, a->kv_cache, a->win, a->ia, a->ib, a->iza, a->izb, a->ibias_a,
                        a->ibias_b, a->iring, a->kI, a->kI_scale};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  if ((int64_t)a->B * kDcCluster > INT32_MAX) return CSAHCA_ERR_UNSUPPORTED;
  int st = device_ok();
  if (st != CSAHCA_OK) return st;
  DecodeCompressParams p;
  memset(&p, 0, sizeof(p));
  p.pos = a->pos; p.kv_raw = a->kv_raw;
  p.nw[0] = a->a; p.nw[1] = csa ? a->b : a->za; p.nw[2] = csa ? a->za : nullptr; p.nw[3] = csa ? a->zb : nullptr;
  p.bias_a = a->bias_a; p.bias_b = a->bias_b; p.gain = a->kv_gain;
  p.ring = a->ring; p.kv_cache = a->kv_cache; p.win = a->win;
  if (dI) {
    p.inw[0] = a->ia; p.inw[1] = a->ib; p.inw[2] = a->iza; p.inw[3] = a->izb;
    p.ibias_a = a->ibias_a; p.ibias_b = a->ibias_b; p.iring = a->iring; p.kI = a->kI; p.kI_scale = a->kI_scale;
  }
  p.B = a->B; p.d = a->d; p.dI = dI; p.m = a->m; p.N_cap = a->N_cap; p.w = a->w;
  p.rope_dims = a->rope_dims; p.kv_norm = a->kv_norm; p.ki_e4m3 = dI && a->kI_dtype == CSAHCA_E4M3;
  p.kv_f8 = kv_f8 ? 1 : 0;
  p.kv_row_bytes = kv_f8 ? kv_f8_row_bytes(a->d, a->rope_dims) : 0;
  p.entry_base = a->entry_base;
  p.eps = a->eps > 0 ? a->eps : kDefaultEps;
  rope_theta_table(p.theta, a->rope_dims, a->rope_base > 0 ? a->rope_base : kDefaultRopeBase);
  cudaStream_t s = as_stream(stream);
  const dim3 grid((unsigned)(a->B * kDcCluster)), block(kDcThreads);
  CSAHCA_TRACE("decode_compress", s);
  if (a->dtype == CSAHCA_F32) {
    if (csa) launch_k(decode_compress_kernel<float, true>, grid, block, 0, s, p);
    else launch_k(decode_compress_kernel<float, false>, grid, block, 0, s, p);
  } else {
    if (csa) launch_k(decode_compress_kernel<__nv_bfloat16, true>, grid, block, 0, s, p);
    else launch_k(decode_compress_kernel<__nv_bfloat16, false>, grid, block, 0, s, p);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

// ------------------------------------------------------ context parallelism --

int run_cp_topk_merge(const csahca_cp_topk_merge_args* a, void* stream) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->R < 1 || a->rows < 0 || a->k < 1 || a->rank < 0 || a->rank >= a->R) return CSAHCA_ERR_INVALID_ARG;
  if (a->R > kCpMaxRanks || a->k > kCpMaxK || (int64_t)a->R * a->k > kCpMaxCand) return CSAHCA_ERR_UNSUPPORTED;
  if (a->rows == 0) return CSAHCA_OK;
  if (!a->bases || !a->cand_idx || !a->cand_scores || (!a->idx_global && !a->idx_local))
    return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->cand_idx, a->cand_scores, a->idx_global, a->idx_local};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  CpTopkMergeParams p;
  memset(&p, 0, sizeof(p));
  for (int r = 0; r < a->R; ++r) {
    if (a->bases[r] < 0) return CSAHCA_ERR_INVALID_ARG;
    p.bases[r] = a->bases[r];
  }
  int st = device_ok();
  if (st != CSAHCA_OK) return st;
  p.cand_idx = a->cand_idx; p.cand_scores = a->cand_scores;
  p.idx_global = a->idx_global; p.idx_local = a->idx_local;
  p.R = a->R; p.rows = a->rows; p.k = a->k; p.rank = a->rank;
  p.kpow2 = 1;
  while (p.kpow2 < a->k) p.kpow2 <<= 1;
  const int smem = cp_topk_merge_smem_bytes(a->R, a->k, p.kpow2);
  cudaFuncSetAttribute(cp_topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  cudaStream_t s = as_stream(stream);
  {
    CSAHCA_TRACE("cp_topk_merge", s);
    launch_k(cp_topk_merge_kernel, dim3((unsigned)a->rows), dim3(kCpMergeThreads), smem, s, p);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

int run_cp_attn_merge(const csahca_cp_merge_args* a, void* stream) {
  if (!a) return CSAHCA_ERR_INVALID_ARG;
  if (a->dtype != CSAHCA_F32 && a->dtype != CSAHCA_BF16) return CSAHCA_ERR_INVALID_ARG;
  if (a->R < 1 || a->rows < 0 || a->H < 1 || a->d < 1) return CSAHCA_ERR_INVALID_ARG;
  if (a->rope_dims < 0 || a->rope_dims > a->d || (a->rope_dims & 1)) return CSAHCA_ERR_INVALID_ARG;
  // (H even and d % 4 == 0 keep every row's o[h] 16-byte aligned for float4 loads)
  if (a->R > kCpMaxRanks || a->H % 2 || a->d % 4 || a->d > 1024 || a->rope_dims > 128)
    return CSAHCA_ERR_UNSUPPORTED;
  if ((int64_t)a->rows * a->H > INT32_MAX) return CSAHCA_ERR_UNSUPPORTED;
  if (a->rows == 0) return CSAHCA_OK;
  if (!a->partials || !a->sinks || !a->pos || !a->out) return CSAHCA_ERR_INVALID_ARG;
  const void* ptrs[] = {a->partials, a->sinks, a->pos, a->out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return CSAHCA_ERR_ALIGNMENT;
  int st = device_ok();
  if (st != CSAHCA_OK) return st;
  CpMergeParams p;
  memset(&p, 0, sizeof(p));
  p.partials = a->partials; p.sinks = a->sinks; p.pos = a->pos; p.out = a->out;
  p.R = a->R; p.rows = a->rows; p.H = a->H; p.d = a->d; p.rope_dims = a->rope_dims;
  p.out_bf16 = a->dtype == CSAHCA_BF16 ? 1 : 0;
  rope_theta_table(p.theta, a->rope_dims, a->rope_base > 0 ? a->rope_base : kDefaultRopeBase);
  cudaStream_t s = as_stream(stream);
  {
    CSAHCA_TRACE("cp_attn_merge", s);
    launch_k(cp_merge_kernel, dim3((unsigned)(a->rows * a->H)), dim3((unsigned)(a->d / 4)), 0, s, p);
  }
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

}  // namespace

// ============================================================== C ABI ======

// Self-test of the failure detection: one thread waits on an mbarrier that
// nothing arrives at; the bounded wait gives up after its iteration limit,
// ORs DEVERR_MBAR_TIMEOUT into the device error word and the kernel returns.
__global__ void selftest_bounded_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag);
}

extern "C" {

int csa_compress(const csahca_compress_args* args, void* stream) { return run_compress(args, stream, true); }
int hca_compress(const csahca_compress_args* args, void* stream) { return run_compress(args, stream, false); }

int indexer_topk(const csahca_indexer_args* args, void* stream) { return run_indexer(args, stream); }

size_t csahca_indexer_workspace_size(const csahca_indexer_args* args) {
  if (validate_indexer(args, true) != CSAHCA_OK) return 0;
  return indexer_workspace(args);
}

int compressed_attn_prefill(const csahca_attn_args* args, void* stream) { return run_prefill(args, stream); }

size_t csahca_prefill_workspace_size(const csahca_attn_args* args) {
  if (validate_attn(args, true) != CSAHCA_OK) return 0;
  return prefill_workspace(args);
}

int compressed_attn_decode(const csahca_decode_args* args, void* stream) {
  if (!args) return CSAHCA_ERR_INVALID_ARG;
  return run_decode(args, stream, static_cast<char*>(args->workspace), args->workspace_bytes);
}

int decode_compress(const csahca_decode_compress_args* args, void* stream) {
  return run_decode_compress(args, stream);
}

int cp_topk_merge(const csahca_cp_topk_merge_args* args, void* stream) { return run_cp_topk_merge(args, stream); }

int cp_attn_merge(const csahca_cp_merge_args* args, void* stream) { return run_cp_attn_merge(args, stream); }

size_t csahca_decode_workspace_size(const csahca_decode_args* args) {
  if (validate_decode(args, true) != CSAHCA_OK) return 0;
  if (args->B == 0) return 0;
  return decode_layout(args).total;
}

const char* csahca_status_string(int status) {
  switch (status) {
    case CSAHCA_OK: return "ok";
    case CSAHCA_ERR_INVALID_ARG: return "invalid argument";
    case CSAHCA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case CSAHCA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case CSAHCA_ERR_WORKSPACE: return "workspace missing or too small";
    case CSAHCA_ERR_LAUNCH: return "CUDA launch or driver error";
    case CSAHCA_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case CSAHCA_ERR_NO_DEVICE: return "no sm_100 CUDA device";
    default: return "unknown status";
  }
}

int csahca_abi_version(void) { return CSAHCA_ABI_VERSION; }

int64_t csahca_kv_row_bytes(int32_t kv_dtype, int32_t d, int32_t rope_dims) {
  if (d <= 0) return 0;
  switch (kv_dtype) {
    case CSAHCA_F32: return (int64_t)d * 4;
    case CSAHCA_BF16: return (int64_t)d * 2;
    case CSAHCA_E4M3: return kv_f8_row_bytes(d, rope_dims);
    default: return 0;
  }
}

int64_t csahca_struct_size(int which) {
  switch (which) {
    case 0: return (int64_t)sizeof(csahca_compress_args);
    case 1: return (int64_t)sizeof(csahca_indexer_args);
    case 2: return (int64_t)sizeof(csahca_attn_args);
    case 3: return (int64_t)sizeof(csahca_decode_args);
    case 4: return (int64_t)sizeof(csahca_decode_compress_args);
    case 5: return (int64_t)sizeof(csahca_cp_topk_merge_args);
    case 6: return (int64_t)sizeof(csahca_cp_merge_args);
    default: return -1;
  }
}

int csahca_trace_enable(int enable) {
  trace::g_enabled = enable != 0;
  return CSAHCA_OK;
}

int csahca_trace_collect(csahca_trace_entry* out, int max_entries, int* n_entries) {
  if (!n_entries || (max_entries > 0 && !out) || max_entries < 0) return CSAHCA_ERR_INVALID_ARG;
  *n_entries = 0;
  std::vector<csahca_trace_entry> acc;
  int status = CSAHCA_OK;
  for (const auto& r : trace::g_records) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.end) != cudaSuccess || cudaEventElapsedTime(&ms, r.begin, r.end) != cudaSuccess) {
      (void)cudaGetLastError();
      status = CSAHCA_ERR_LAUNCH;
    }
    size_t i = 0;
    for (; i < acc.size(); ++i)
      if (strncmp(acc[i].name, r.name, sizeof(acc[i].name)) == 0) break;
    if (i == acc.size()) {
      csahca_trace_entry e;
      memset(&e, 0, sizeof(e));
      strncpy(e.name, r.name, sizeof(e.name) - 1);
      acc.push_back(e);
    }
    acc[i].launches += 1;
    acc[i].total_ms += ms;
    trace::g_pool.push_back(r.begin);
    trace::g_pool.push_back(r.end);
  }
  trace::g_records.clear();
  int n = 0;
  for (; n < (int)acc.size() && n < max_entries; ++n) out[n] = acc[n];
  *n_entries = n;
  return status;
}

int csahca_selftest_bounded_wait(void* stream) {
  const int st = device_ok();
  if (st != CSAHCA_OK) return st;
  selftest_bounded_wait_kernel<<<1, 32, 0, as_stream(stream)>>>();
  CSAHCA_CHECK_LAUNCH();
  return CSAHCA_OK;
}

int csahca_device_error(void* stream, int32_t* code) {
  if (!code) return CSAHCA_ERR_INVALID_ARG;
  *code = 0;
  cudaStream_t s = as_stream(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) { (void)cudaGetLastError(); return CSAHCA_ERR_LAUNCH; }
  int32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) {
    (void)cudaGetLastError();
    return CSAHCA_ERR_LAUNCH;
  }
  *code = v;
  return CSAHCA_OK;
}

}  // extern "C"

// ======================================================= allocation-free ======
// indexer_topk_noalloc: indexer_topk with its scratch (score rows and the
// multi-CTA top-k buffers) in a fixed device array of this library instead of
// a caller-provided workspace.  It exists for callers that cannot allocate
// device memory at the point of the call.  The array is a file-scope
// __device__ object, so every GPU that loads the library holds it until the
// process exits.

namespace {

constexpr size_t kNoAllocScratchBytes = CSAHCA_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocMaxDevices = 64;

// Host code must not pass the array's name to a kernel: on the host it is only
// a stand-in symbol.  Its device address comes from cudaGetSymbolAddress with
// the device current, and is cached per device together with the id of the
// context it was looked up in: after a device reset (a new primary context)
// the next call looks the address up again instead of using a stale one.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_noalloc_mu;
struct NoAllocSlot { unsigned long long ctx_id; void* ptr; };
NoAllocSlot g_noalloc_slot[kNoAllocMaxDevices];

// Unique id of the calling thread's current context (0 if none or unknown).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  if (!get_cur || !get_id) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) { (void)cudaGetLastError(); return 0; }
    get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) { (void)cudaGetLastError(); return 0; }
    get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return CSAHCA_ERR_NO_DEVICE; }
  if (dev < 0 || dev >= kNoAllocMaxDevices) return CSAHCA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocSlot& slot = g_noalloc_slot[dev];
  const unsigned long long id = current_context_id();
  if (!slot.ptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return CSAHCA_ERR_LAUNCH;
    }
    // (cudaGetSymbolAddress made the primary context current if none was)
    slot.ptr = p;
    slot.ctx_id = id != 0 ? id : current_context_id();
  }
  *out = slot.ptr;
  return CSAHCA_OK;
}

}  // namespace

extern "C" int indexer_topk_noalloc(const csahca_indexer_args* args, void* stream) {
  int st = validate_indexer(args);
  if (st != CSAHCA_OK) return st;
  if (args->B == 0 || args->nq == 0) return CSAHCA_OK;
  if (indexer_workspace(args) > kNoAllocScratchBytes) return CSAHCA_ERR_WORKSPACE;
  if ((st = device_ok()) != CSAHCA_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != CSAHCA_OK) return st;
  csahca_indexer_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = kNoAllocScratchBytes;
  return run_indexer(&a, stream);
}
