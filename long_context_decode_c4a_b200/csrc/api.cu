// api.cu -- the C ABI of libcsa.so (declared in include/csa.h): argument checks, workspace
// layout, TMA descriptor encoding and the launch sequence of every entry point.
//
// The library never allocates device memory. Scratch space (the indexer's score rows and the
// top-k merge lists) lives in the caller's workspace; its first 256 bytes are the device
// status word that kernels set instead of trapping.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "csa.h"
#include "kernels.cuh"

namespace csa {

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

#define CSA_CHECK_ARG(cond, ...)                                   \
  do {                                                             \
    if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__);    \
  } while (0)
#define CSA_CHECK_SUP(cond, ...)                                   \
  do {                                                             \
    if (!(cond)) return fail(CSA_ERR_UNSUPPORTED, __VA_ARGS__);    \
  } while (0)
#define CSA_CUDA(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- TMA descriptors through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (fn == nullptr) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *out = fn;
  return CSA_OK;
}

// 2D bf16 tensor [rows, cols] with row pitch `pitch_elems`, box {box_cols, box_rows}, 128B swizzle.
int make_map_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch_elems,
                uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc;
  if (int rc = get_encoder(&enc)) return rc;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_elems * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CSA_OK;
}

struct DeviceInfo {
  int sms = 0;
  int max_smem = 0;
  bool attrs_set = false;
};

// Launch with programmatic stream serialization: the kernel may begin launching while the
// previous kernel on the stream runs; it calls pdl_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int device_info(DeviceInfo** out) {
  static DeviceInfo info[64];
  static std::mutex mu;
  int dev = 0;
  CSA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(CSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  DeviceInfo& d = info[dev];
  if (!d.attrs_set) {
    CSA_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    CSA_CUDA(cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    int cc_major = 0, cc_minor = 0;
    CSA_CUDA(cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, dev));
    CSA_CUDA(cudaDeviceGetAttribute(&cc_minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (cc_major != 10 || cc_minor != 0)
      return fail(CSA_ERR_UNSUPPORTED, "libcsa is built for sm_100a; device is sm_%d%d", cc_major, cc_minor);
    const int ms = d.max_smem;
    CSA_CUDA(cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    CSA_CUDA(cudaFuncSetAttribute(indexer_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, ms));
    d.attrs_set = true;
  }
  *out = &d;
  return CSA_OK;
}

// ---- workspace layout
struct IdxWs {
  size_t scores_off, cand_key_off, cand_idx_off, cand_cnt_off, flags_off, total;
  int max_chunks;
};

IdxWs indexer_ws_layout(long long queries, int max_entries, int topk, bool with_flags = false) {
  IdxWs w{};
  size_t off = kStatusBytes;
  w.scores_off = off;
  off = round_up(off + (size_t)queries * (size_t)max_entries * 4, 256);
  w.max_chunks = max_entries > kTopkChunk ? (max_entries + kTopkChunk - 1) / kTopkChunk : 0;
  w.cand_key_off = off;
  off = round_up(off + (size_t)queries * w.max_chunks * topk * 4, 256);
  w.cand_idx_off = off;
  off = round_up(off + (size_t)queries * w.max_chunks * topk * 4, 256);
  w.cand_cnt_off = off;
  off = round_up(off + (size_t)queries * w.max_chunks * 4, 256);
  w.flags_off = off;                       // fused decode step: per-request index-entry flags
  if (with_flags) off = round_up(off + (size_t)queries * 4, 256);
  w.total = off;
  return w;
}

int check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned(ws, 256)) return fail(CSA_ERR_WORKSPACE, "workspace null or not 256-byte aligned");
  if (ws_bytes < need) return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
  return CSA_OK;
}

int check_cfg(const csa_compressor_cfg* c) {
  CSA_CHECK_ARG(c != nullptr, "cfg is null");
  CSA_CHECK_SUP((c->ratio == 4 && c->overlap == 1) || (c->ratio == 128 && c->overlap == 0),
                "(ratio, overlap) must be (4,1) or (128,0)");
  CSA_CHECK_SUP(c->d == 128 || c->d == 512, "d must be 128 or 512");
  CSA_CHECK_SUP(c->rope_dim >= 8 && c->rope_dim % 8 == 0 && c->rope_dim <= c->d && c->rope_dim / 2 <= kMaxRopePairs,
                "rope_dim must be a multiple of 8 in [8, min(d, 128)]");
  CSA_CHECK_ARG(std::isfinite(c->rope_base) && c->rope_base > 0.f, "rope_base must be positive");
  CSA_CHECK_ARG(std::isfinite(c->eps) && c->eps >= 0.f, "eps must be >= 0");
  return CSA_OK;
}

CompressParams compress_params(const csa_compressor_cfg* c, int B, int S, const int32_t* start_pos, const uint16_t* kv,
                               const uint16_t* score, const uint16_t* gamma, uint16_t* skv, uint16_t* ssc,
                               uint16_t* cache, int64_t cache_bstride, int max_entries, float* cache_f32,
                               uint32_t* status) {
  CompressParams p{};
  p.ratio = c->ratio;
  p.overlap = c->overlap;
  p.d = c->d;
  p.rope_dim = c->rope_dim;
  p.rope_base = c->rope_base;
  p.eps = c->eps;
  for (int i = 0; i < c->rope_dim / 2; ++i) p.inv_freq[i] = std::pow((double)c->rope_base, -2.0 * i / c->rope_dim);
  p.B = B;
  p.S = S;
  p.start_pos = start_pos;
  p.kv = kv;
  p.score = score;
  p.gamma = gamma;
  p.state_kv = skv;
  p.state_score = ssc;
  p.cache = cache;
  p.cache_bstride = cache_bstride;
  p.max_entries = max_entries;
  p.cache_f32 = cache_f32;
  p.status = status;
  return p;
}

int check_compress_args(const csa_compressor_cfg* cfg, int B, int S, const int32_t* start_pos, const uint16_t* kv,
                        const uint16_t* score, const uint16_t* gamma, const uint16_t* skv, const uint16_t* ssc,
                        const uint16_t* cache, int64_t cache_bstride, int max_entries, const float* cache_f32) {
  if (int rc = check_cfg(cfg)) return rc;
  CSA_CHECK_ARG(B > 0 && S > 0, "B and S must be positive");
  CSA_CHECK_ARG(start_pos && kv && score && gamma && skv && ssc && cache, "null pointer argument");
  CSA_CHECK_ARG(aligned(kv, 16) && aligned(score, 16) && aligned(gamma, 16) && aligned(skv, 16) &&
                    aligned(ssc, 16) && aligned(cache, 16) && aligned(start_pos, 4),
                "pointers must be 16-byte aligned");
  CSA_CHECK_ARG(cache_f32 == nullptr || aligned(cache_f32, 16), "cache_f32 must be 16-byte aligned");
  CSA_CHECK_ARG(max_entries > 0, "max_entries must be positive");
  CSA_CHECK_ARG(cache_bstride >= (int64_t)max_entries * cfg->d && cache_bstride % 8 == 0,
                "cache_bstride must be >= max_entries*d and a multiple of 8");
  return CSA_OK;
}

int launch_compress(const CompressLaunch& L, int nstreams, int B, int S, int ratio, cudaStream_t st) {
  if (S == 1) {
    if (ratio == 128 && nstreams == 1 && L.p[0].d == 512 && L.p[0].overlap == 0) {
      // C128A with d = 512: a cluster of channel-block CTAs per request.
      CSA_CUDA(launch_pdl(compress_decode_c128_kernel, dim3(kC128Split, (unsigned)B), dim3(kCompressThreads), 0, st, L));
      return CSA_OK;
    }
    CSA_CUDA(launch_pdl(compress_decode_kernel, dim3((unsigned)B, (unsigned)nstreams), dim3(kCompressThreads), 0, st, L));
    return CSA_OK;
  }
  const dim3 grid((unsigned)((S + ratio - 1) / ratio), (unsigned)B, (unsigned)nstreams);
  CSA_CUDA(launch_pdl(compress_kernel, grid, dim3(kCompressThreads), 0, st, L));
  if (S > 1) {
    CSA_CUDA(launch_pdl(compress_state_kernel, dim3((unsigned)B, 1, (unsigned)nstreams), dim3(kCompressThreads), 0, st, L));
  }
  return CSA_OK;
}

// ---- indexer + top-k
struct IndexerArgs {
  int B, S, H_I, d_I, ratio, topk;
  const int32_t* q_pos;
  const uint16_t* q_idx;
  const float* w;
  const uint16_t* idx_cache;
  int64_t idx_bstride;
  int max_entries;
  int32_t* topk_idx;
  float* scores_opt;
  void* ws;
  size_t ws_bytes;
};

int check_indexer_args(const IndexerArgs& a, bool scores = true, bool select = true) {
  CSA_CHECK_ARG(a.B > 0 && a.S > 0, "B and S must be positive");
  if (!scores) {  // selection over caller-provided scores
    CSA_CHECK_ARG(a.ratio > 0, "ratio must be positive");
    CSA_CHECK_SUP(a.topk >= 1 && a.topk <= kAttnMaxTopk, "topk must be in [1, %d]", kAttnMaxTopk);
    CSA_CHECK_SUP(a.max_entries >= 1 && a.max_entries <= (1 << 24), "max_entries must be in [1, 2^24]");
    CSA_CHECK_ARG(a.q_pos && a.scores_opt && a.topk_idx, "null pointer argument");
    CSA_CHECK_ARG(aligned(a.scores_opt, 16) && aligned(a.topk_idx, 4) && aligned(a.q_pos, 4), "misaligned pointer");
    return CSA_OK;
  }
  if (!select) CSA_CHECK_ARG(a.scores_opt != nullptr, "scores is null");
  CSA_CHECK_SUP(a.d_I == 128, "d_I must be 128");
  CSA_CHECK_SUP(a.H_I == 4 || a.H_I == 8 || a.H_I == 16 || a.H_I == 32 || a.H_I == 64 || a.H_I == 128,
                "H_I must be a power of two in [4, 128]");
  CSA_CHECK_ARG(a.ratio > 0, "ratio must be positive");
  CSA_CHECK_SUP(a.topk >= 1 && a.topk <= kAttnMaxTopk, "topk must be in [1, %d]", kAttnMaxTopk);
  CSA_CHECK_SUP(a.max_entries >= 1 && a.max_entries <= (1 << 24), "max_entries must be in [1, 2^24]");
  CSA_CHECK_ARG(a.q_pos && a.q_idx && a.w && a.idx_cache && (a.topk_idx || !select), "null pointer argument");
  CSA_CHECK_ARG(aligned(a.q_idx, 16) && aligned(a.idx_cache, 16) && aligned(a.w, 4) && aligned(a.topk_idx, 4) &&
                    aligned(a.q_pos, 4),
                "misaligned pointer");
  CSA_CHECK_ARG(a.idx_bstride >= (int64_t)a.max_entries * a.d_I && a.idx_bstride % a.d_I == 0,
                "idx_bstride must be >= max_entries*d_I and a multiple of d_I");
  CSA_CHECK_ARG(a.scores_opt == nullptr || aligned(a.scores_opt, 4), "scores_opt misaligned");
  const long long rows = (long long)a.B * (a.idx_bstride / a.d_I);
  CSA_CHECK_SUP(rows < (1ll << 31), "index cache too large for 32-bit row coordinates");
  const long long qrows = (long long)a.B * a.S * a.H_I;
  CSA_CHECK_SUP(qrows < (1ll << 31), "too many query rows");
  return CSA_OK;
}

// The indexer (scores) and / or the top-k selection over them. Scores-only and selection-only calls
// serve the tensor-parallel indexer: partial scores per head shard, a sum across ranks, then the
// selection.
int run_indexer_topk(const IndexerArgs& a, cudaStream_t st, cudaEvent_t const* ev = nullptr, bool run_scores = true,
                     bool run_select = true, const CompressLaunch* fuse = nullptr) {
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  const long long queries = (long long)a.B * a.S;
  const IdxWs L = indexer_ws_layout(queries, a.max_entries, run_select ? a.topk : 1, fuse != nullptr);
  const size_t need = run_select ? (a.scores_opt ? L.total - (L.cand_key_off - L.scores_off) : L.total) : kStatusBytes;
  if (int rc = check_ws(a.ws, a.ws_bytes, need)) return rc;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  // With caller-provided scores the workspace's score region is not needed: the candidate lists
  // move down to start right after the status word.
  const size_t shift = a.scores_opt ? (L.cand_key_off - L.scores_off) : 0;
  float* scores = a.scores_opt ? a.scores_opt : reinterpret_cast<float*>(ws + L.scores_off);
  if (run_scores) {
    IndexerParams P{};
    P.B = a.B;
    P.S = a.S;
    P.QG = a.S == 1 ? 1 : std::min(a.S, 256 / a.H_I);
    P.N = (int)round_up((size_t)P.QG * a.H_I, 16);
    P.ratio = a.ratio;
    P.max_entries = a.max_entries;
    P.groups_per_req = (a.S + P.QG - 1) / P.QG;
    P.tiles_per_group = (a.max_entries + 127) / 128;
    P.total_items = (long long)a.B * P.groups_per_req * P.tiles_per_group;
    P.rows_per_req = a.idx_bstride / a.d_I;
    const bool fused = fuse != nullptr;
    int stages = kIdxMaxStages;
    while (stages > 2 && indexer_smem_bytes(stages, P.N, fused) > (size_t)dev->max_smem) --stages;
    CSA_CHECK_SUP(indexer_smem_bytes(stages, P.N, fused) <= (size_t)dev->max_smem,
                  "shared memory too small for the indexer");
    P.stages = stages;
    P.n_acc = (4 * P.N <= 512) ? 4 : 2;
    int cols = 32;
    while (cols < P.n_acc * P.N) cols <<= 1;
    P.tmem_cols = cols;
    P.q_pos = a.q_pos;
    P.w = a.w;
    P.scores = scores;
    P.scores_stride = a.max_entries;
    P.status = status;

    CUtensorMap map_k, map_q;
    if (int rc = make_map_2d(&map_k, a.idx_cache, 128, (uint64_t)a.B * P.rows_per_req, 128, 64, 128)) return rc;
    if (int rc = make_map_2d(&map_q, a.q_idx, 128, (uint64_t)queries * a.H_I, 128, 64, (uint32_t)P.N)) return rc;
    const size_t smem = indexer_smem_bytes(stages, P.N, fused);
    const dim3 grid((unsigned)std::min<long long>(P.total_items, dev->sms));
    IndexerFuse F{};
    if (fused) {
      F.njobs = 2 * a.B;
      F.B = a.B;
      F.flags = reinterpret_cast<uint32_t*>(ws + L.flags_off - shift);
      F.L = *fuse;
    }
    cudaError_t e = cudaSuccess;
    switch (a.H_I) {
      case 4: e = launch_pdl(indexer_kernel<4>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
      case 8: e = launch_pdl(indexer_kernel<8>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
      case 16: e = launch_pdl(indexer_kernel<16>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
      case 32: e = launch_pdl(indexer_kernel<32>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
      case 64: e = launch_pdl(indexer_kernel<64>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
      default: e = launch_pdl(indexer_kernel<128>, grid, dim3(kIdxThreads), smem, st, map_k, map_q, P, F); break;
    }
    CSA_CUDA(e);
  }
  if (ev) CSA_CUDA(cudaEventRecord(ev[0], st));
  if (!run_select) return CSA_OK;

  TopkParams T{};
  T.topk = a.topk;
  T.ratio = a.ratio;
  T.max_entries = a.max_entries;
  T.chunk = kTopkChunk;
  T.max_chunks = L.max_chunks;
  T.q_pos = a.q_pos;
  T.scores = scores;
  T.scores_stride = a.max_entries;
  T.out = a.topk_idx;
  T.cand_key = reinterpret_cast<uint32_t*>(ws + L.cand_key_off - shift);
  T.cand_idx = reinterpret_cast<int32_t*>(ws + L.cand_idx_off - shift);
  T.cand_cnt = reinterpret_cast<int*>(ws + L.cand_cnt_off - shift);
  T.status = status;
  const int nchunks = std::max(1, L.max_chunks);
  const int tk_threads = a.max_entries <= kTopkShortRow ? kTopkShortThreads : kTopkThreads;
  CSA_CUDA(launch_pdl(topk_chunk_kernel, dim3((unsigned)nchunks, (unsigned)queries), dim3(tk_threads), 0, st, T));
  if (L.max_chunks > 1) {
    CSA_CHECK_SUP(L.max_chunks <= kTopkMaxChunks, "max_entries too large for the top-k merge");
    CSA_CUDA(launch_pdl(topk_merge_kernel, dim3((unsigned)queries), dim3(kTopkThreads), 0, st, T));
  }
  if (ev) CSA_CUDA(cudaEventRecord(ev[1], st));
  return CSA_OK;
}

// ---- attention
struct AttnArgs {
  int B, S, H, d, rope_dim;
  float rope_base, scale;
  int ratio;
  const int32_t* q_pos;
  const uint16_t* q;
  const uint16_t* ring;
  int64_t ring_bstride;
  int ring_cap, window;
  const uint16_t* cache;
  int64_t cache_bstride;
  int max_entries;
  const int32_t* topk_idx;
  int topk;
  const float* sink;
  void* out;
  int out_is_f32;
  void* ws;
  size_t ws_bytes;
  size_t part_off = kStatusBytes;  // workspace offset of the split-candidate partials
  bool early_window = false;       // q and the ring are final before the dependency wait (AttnParams)
};

// Split-candidate attention: a query's candidate tiles are spread over `splits` CTA pairs when the
// queries alone would leave most SMs idle. The workspace is sized for kAttnSplitPairs pairs (the
// B200's 148 SMs); a launch uses no more splits than its device's pairs and its workspace allow.
constexpr int kAttnSplitPairs = 74;

int attn_ws_splits(long long queries) {
  if (queries <= 0) return 1;
  return (int)std::max<long long>(1, std::min<long long>(kAttnMaxSplits, kAttnSplitPairs / queries));
}

size_t attn_part_bytes(long long queries, int splits) {
  if (splits <= 1) return 0;
  return (size_t)queries * splits * (128 * 512 + 2 * 128) * sizeof(float);
}

int check_attn_args(const AttnArgs& a, bool csa_mode) {
  CSA_CHECK_ARG(a.B > 0 && a.S > 0, "B and S must be positive");
  CSA_CHECK_SUP(a.d == 512, "d must be 512");
  CSA_CHECK_SUP(a.H >= 1 && a.H <= 128, "H must be in [1, 128]");
  CSA_CHECK_SUP(a.rope_dim >= 2 && a.rope_dim % 2 == 0 && a.rope_dim <= 256 && a.rope_dim / 2 <= kMaxRopePairs,
                "rope_dim must be even and <= 128");
  CSA_CHECK_ARG(std::isfinite(a.rope_base) && a.rope_base > 0.f, "rope_base must be positive");
  CSA_CHECK_ARG(std::isfinite(a.scale), "scale must be finite");
  CSA_CHECK_ARG(a.ratio > 0, "ratio must be positive");
  CSA_CHECK_SUP(a.window >= 1 && a.window <= kAttnMaxWindow, "window must be in [1, %d]", kAttnMaxWindow);
  CSA_CHECK_ARG(a.ring_cap >= a.window, "ring_cap must be >= window");
  CSA_CHECK_ARG(a.max_entries >= 1, "max_entries must be positive");
  CSA_CHECK_ARG(a.q_pos && a.q && a.ring && a.cache && a.sink && a.out, "null pointer argument");
  CSA_CHECK_ARG(aligned(a.q, 16) && aligned(a.ring, 16) && aligned(a.cache, 16) && aligned(a.out, 16) &&
                    aligned(a.sink, 4) && aligned(a.q_pos, 4),
                "misaligned pointer");
  CSA_CHECK_ARG(a.ring_bstride % a.d == 0 && a.ring_bstride >= (int64_t)a.ring_cap * a.d,
                "ring_bstride must be a multiple of d and >= ring_cap*d");
  CSA_CHECK_ARG(a.cache_bstride % a.d == 0 && a.cache_bstride >= (int64_t)a.max_entries * a.d,
                "cache_bstride must be a multiple of d and >= max_entries*d");
  CSA_CHECK_SUP((long long)a.B * (a.ring_bstride / a.d) < (1ll << 30) &&
                    (long long)a.B * (a.cache_bstride / a.d) < (1ll << 30),
                "ring or cache too large for 30-bit row coordinates");
  CSA_CHECK_SUP((long long)a.B * a.S * a.H < (1ll << 31), "too many query rows");
  if (csa_mode) {
    CSA_CHECK_ARG(a.topk_idx != nullptr && aligned(a.topk_idx, 4), "topk_idx null or misaligned");
    CSA_CHECK_SUP(a.topk >= 1 && a.topk <= kAttnMaxTopk, "topk must be in [1, %d]", kAttnMaxTopk);
  }
  return check_ws(a.ws, a.ws_bytes, kStatusBytes);
}

int run_attn(const AttnArgs& a, bool csa_mode, cudaStream_t st) {
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  AttnParams P{};
  P.B = a.B;
  P.S = a.S;
  P.H = a.H;
  P.d = a.d;
  P.rope_dim = a.rope_dim;
  for (int i = 0; i < a.rope_dim / 2; ++i) P.inv_freq[i] = std::pow((double)a.rope_base, -2.0 * i / a.rope_dim);
  P.scale_log2 = a.scale * 1.4426950408889634f;
  P.window = a.window;
  P.ring_cap = a.ring_cap;
  P.ring_rows = a.ring_bstride / a.d;
  P.cache_rows = a.cache_bstride / a.d;
  P.max_entries = a.max_entries;
  P.ratio = a.ratio;
  P.q_pos = a.q_pos;
  P.topk_idx = csa_mode ? a.topk_idx : nullptr;
  P.topk = csa_mode ? a.topk : 0;
  P.sink = a.sink;
  P.out = a.out;
  P.out_is_f32 = a.out_is_f32 ? 1 : 0;
  P.status = reinterpret_cast<uint32_t*>(a.ws);
  P.ring = a.ring;
  P.cache = a.cache;
  P.early_window = a.early_window ? 1 : 0;
  CUtensorMap map_q;
  const long long queries = (long long)a.B * a.S;
  if (int rc = make_map_2d(&map_q, a.q, 512, (uint64_t)queries * a.H, 512, 64, 128)) return rc;
  const size_t smem = attn_smem_bytes();
  CSA_CHECK_SUP(smem <= (size_t)dev->max_smem, "shared memory too small for the attention kernel");
  CSA_CHECK_SUP(queries <= 65535, "at most 65535 queries per call");
  // Splits: as many as the device's CTA pairs allow per query (and the workspace was sized for),
  // with at least two tiles of the longest candidate list per split.
  const long long max_cands = (long long)a.window + (csa_mode ? a.topk : std::min(a.max_entries, kAttnMaxCompressed));
  const int max_tiles = (int)((max_cands + 31) / 32);
  int splits = std::min<long long>(attn_ws_splits(queries), std::max<long long>(1, (dev->sms / 2) / queries));
  splits = std::max(1, std::min(splits, max_tiles / 2));
  const size_t part_off = round_up(a.part_off, 256);
  if (splits > 1 && a.ws_bytes < part_off + attn_part_bytes(queries, splits)) splits = 1;
  P.splits = splits;
  if (splits > 1) {
    P.part_o = reinterpret_cast<float*>(static_cast<char*>(a.ws) + part_off);
    P.part_ml = P.part_o + (size_t)queries * splits * 128 * 512;
  }
  CSA_CHECK_SUP(queries * splits <= 65535, "at most 65535 (query, split) items per call");
  CSA_CUDA(launch_pdl(attn_kernel, dim3(2, (unsigned)(queries * splits)), dim3(kAttnThreads), smem, st, map_q, P));
  if (splits > 1) {
    AttnCombineParams C{};
    C.splits = splits;
    C.H = a.H;
    C.d = a.d;
    C.rope_dim = a.rope_dim;
    for (int i = 0; i < a.rope_dim / 2; ++i) C.inv_freq[i] = P.inv_freq[i];
    C.q_pos = a.q_pos;
    C.part_o = P.part_o;
    C.part_ml = P.part_ml;
    C.out = a.out;
    C.out_is_f32 = P.out_is_f32;
    C.status = P.status;
    CSA_CUDA(launch_pdl(attn_combine_kernel, dim3((unsigned)a.H, (unsigned)queries), dim3(kAttnCombineThreads), 0, st,
                        C));
  }
  return CSA_OK;
}

// K splits for a product whose output tiles alone would leave SMs idle: the largest power of two
// (at most 8) that keeps every CTA in one wave and divides the K blocks.
int gemm_splits(long long tiles, int kblocks, int sms) {
  int splits = 1;
  while (splits < 8 && tiles * splits * 2 <= sms && kblocks % (splits * 2) == 0) splits *= 2;
  return splits;
}

// C = A . B^T on the tensor cores (gemm_kernel). A [a_rows, a_cols] and B [b_rows, b_cols] are
// row-major bf16 with pitches lda / ldb; `groups` independent products along blockIdx.z.
int run_gemm(const void* A, uint64_t a_cols, uint64_t a_rows, uint64_t lda, const void* Bm, uint64_t b_cols,
             uint64_t b_rows, uint64_t ldb, GemmParams P, int groups, int sms, cudaStream_t st) {
  CUtensorMap map_a, map_b;
  if (int rc = make_map_2d(&map_a, A, a_cols, a_rows, lda, 64, 128)) return rc;
  if (int rc = make_map_2d(&map_b, Bm, b_cols, b_rows, ldb, 64, 128)) return rc;
  const unsigned mt = (unsigned)((P.M + 127) / 128);
  CSA_CHECK_SUP(mt <= 65535u, "too many rows");
  const dim3 grid((unsigned)(P.N / 128), mt, (unsigned)(groups * P.splits));
  if (P.c_mode == kGemmOutF32Add) {
    const long long n4 = (long long)P.M * P.ldc / 4;
    const int blocks = (int)std::min<long long>((n4 + 255) / 256, 4LL * sms);
    CSA_CUDA(launch_pdl(zero_f32_kernel, dim3(blocks), dim3(256), 0, st, static_cast<float*>(P.c), n4));
  }
  CSA_CUDA(launch_pdl(gemm_kernel, grid, dim3(kGemmThreads), gemm_smem_bytes(), st, map_a, map_b, P));
  return CSA_OK;
}

}  // namespace

int check_indexer_topk_args(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                            const uint16_t* q_idx, const float* w, const uint16_t* idx_cache, int64_t idx_bstride,
                            int max_entries, const int32_t* topk_idx) {
  IndexerArgs a{B, S, H_I, d_I, ratio, topk, q_pos, q_idx, w, idx_cache, idx_bstride, max_entries,
                const_cast<int32_t*>(topk_idx), nullptr, nullptr, 0};
  return check_indexer_args(a);
}

}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported shape";
    case CSA_ERR_CUDA: return "CUDA error";
    case CSA_ERR_TIMEOUT: return "device wait timed out";
    case CSA_ERR_WORKSPACE: return "workspace missing or too small";
    case CSA_ERR_BOUNDS: return "index out of range";
    default: return "unknown status";
  }
}

const char* csa_last_error(void) { return g_err; }

int csa_version(void) { return 1; }

int csa_workspace_size(int kind, int B, int S, int max_entries, int topk, size_t* bytes) {
  CSA_CHECK_ARG(bytes != nullptr, "bytes is null");
  CSA_CHECK_ARG(B > 0 && S > 0 && max_entries > 0, "B, S and max_entries must be positive");
  switch (kind) {
    case CSA_WS_INDEXER_TOPK:
      CSA_CHECK_ARG(topk > 0, "topk must be positive");
      *bytes = indexer_ws_layout((long long)B * S, max_entries, topk).total;
      return CSA_OK;
    case CSA_WS_DECODE_FUSED: {
      CSA_CHECK_ARG(topk > 0, "topk must be positive");
      const long long q = (long long)B * S;
      *bytes = indexer_ws_layout(q, max_entries, topk, true).total + attn_part_bytes(q, attn_ws_splits(q));
      return CSA_OK;
    }
    case CSA_WS_SPARSE_ATTN:
    case CSA_WS_HCA_ATTN:
    case CSA_WS_HCA_DECODE_FUSED: {
      const long long q = (long long)B * S;
      *bytes = kStatusBytes + attn_part_bytes(q, attn_ws_splits(q));
      return CSA_OK;
    }
    case CSA_WS_OUTPUT_PROJ:
    case CSA_WS_Q_PROJ:
      *bytes = kStatusBytes;
      return CSA_OK;
    default:
      return fail(CSA_ERR_INVALID_ARG, "unknown workspace kind %d", kind);
  }
}

int csa_state_reset(const csa_compressor_cfg* cfg, int B, uint16_t* state_kv, uint16_t* state_score, void* stream) {
  if (int rc = check_cfg(cfg)) return rc;
  CSA_CHECK_ARG(B > 0 && state_kv && state_score, "bad arguments");
  const long long n = (long long)B * (1 + cfg->overlap) * cfg->ratio * (1 + cfg->overlap) * cfg->d;
  const int blocks = (int)std::min<long long>((n + 255) / 256, 4096);
  state_reset_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(state_kv, state_score, n);
  CSA_CUDA(cudaGetLastError());
  return CSA_OK;
}

int csa_compress(const csa_compressor_cfg* cfg, int B, int S, const int32_t* start_pos, const uint16_t* kv,
                 const uint16_t* score, const uint16_t* gamma, uint16_t* state_kv, uint16_t* state_score,
                 uint16_t* cache, int64_t cache_bstride, int max_entries, float* cache_f32, void* stream) {
  if (int rc = check_compress_args(cfg, B, S, start_pos, kv, score, gamma, state_kv, state_score, cache,
                                   cache_bstride, max_entries, cache_f32))
    return rc;
  CompressLaunch L{};
  L.p[0] = compress_params(cfg, B, S, start_pos, kv, score, gamma, state_kv, state_score, cache, cache_bstride,
                           max_entries, cache_f32, nullptr);
  L.p[1] = L.p[0];
  return launch_compress(L, 1, B, S, cfg->ratio, static_cast<cudaStream_t>(stream));
}

int csa_indexer_scores(int B, int S, int H_I, int d_I, int ratio, const int32_t* q_pos, const uint16_t* q_idx,
                       const float* w, const uint16_t* idx_cache, int64_t idx_bstride, int max_entries, float* scores,
                       void* ws, size_t ws_bytes, void* stream) {
  IndexerArgs a{B, S, H_I, d_I, ratio, 1, q_pos, q_idx, w, idx_cache, idx_bstride, max_entries, nullptr, scores,
                ws, ws_bytes};
  if (int rc = check_indexer_args(a, true, false)) return rc;
  return run_indexer_topk(a, static_cast<cudaStream_t>(stream), nullptr, true, false);
}

int csa_topk(int B, int S, int ratio, int topk, const int32_t* q_pos, const float* scores, int max_entries,
             int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream) {
  IndexerArgs a{B, S, 0, 0, ratio, topk, q_pos, nullptr, nullptr, nullptr, 0, max_entries, topk_idx,
                const_cast<float*>(scores), ws, ws_bytes};
  if (int rc = check_indexer_args(a, false, true)) return rc;
  return run_indexer_topk(a, static_cast<cudaStream_t>(stream), nullptr, false, true);
}

int csa_indexer_topk(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                     const uint16_t* q_idx, const float* w, const uint16_t* idx_cache, int64_t idx_bstride,
                     int max_entries, int32_t* topk_idx, float* scores_opt, void* ws, size_t ws_bytes,
                     void* stream) {
  IndexerArgs a{B, S, H_I, d_I, ratio, topk, q_pos, q_idx, w, idx_cache, idx_bstride, max_entries, topk_idx,
                scores_opt, ws, ws_bytes};
  if (int rc = check_indexer_args(a)) return rc;
  return run_indexer_topk(a, static_cast<cudaStream_t>(stream));
}

int csa_sparse_attn(int B, int S, int H, int d, int rope_dim, float rope_base, float scale, const int32_t* q_pos,
                    const uint16_t* q, const uint16_t* ring, int64_t ring_bstride, int ring_cap, int window,
                    const uint16_t* cache, int64_t cache_bstride, int max_entries, const int32_t* topk_idx, int topk,
                    const float* sink, void* out, int out_is_f32, void* ws, size_t ws_bytes, void* stream) {
  AttnArgs a{B, S, H, d, rope_dim, rope_base, scale, 4, q_pos, q, ring, ring_bstride, ring_cap, window, cache,
             cache_bstride, max_entries, topk_idx, topk, sink, out, out_is_f32, ws, ws_bytes};
  if (int rc = check_attn_args(a, true)) return rc;
  return run_attn(a, true, static_cast<cudaStream_t>(stream));
}

int hca_attn(int B, int S, int H, int d, int rope_dim, float rope_base, float scale, int ratio, const int32_t* q_pos,
             const uint16_t* q, const uint16_t* ring, int64_t ring_bstride, int ring_cap, int window,
             const uint16_t* cache, int64_t cache_bstride, int max_entries, const float* sink, void* out,
             int out_is_f32, void* ws, size_t ws_bytes, void* stream) {
  AttnArgs a{B, S, H, d, rope_dim, rope_base, scale, ratio, q_pos, q, ring, ring_bstride, ring_cap, window, cache,
             cache_bstride, max_entries, nullptr, 0, sink, out, out_is_f32, ws, ws_bytes};
  if (int rc = check_attn_args(a, false)) return rc;
  return run_attn(a, false, static_cast<cudaStream_t>(stream));
}

int csa_output_projection(int M, int G, int Kg, int R, int D, const uint16_t* o, const uint16_t* wo_a,
                          const uint16_t* wo_b, uint16_t* r, float* y, void* ws, size_t ws_bytes, void* stream) {
  CSA_CHECK_ARG(M > 0 && G > 0 && Kg > 0 && R > 0 && D > 0, "sizes must be positive");
  CSA_CHECK_ARG(o && wo_a && wo_b && r && y, "null pointer");
  CSA_CHECK_ARG(aligned(o, 16) && aligned(wo_a, 16) && aligned(wo_b, 16) && aligned(r, 16) && aligned(y, 16),
                "pointers must be 16-byte aligned");
  CSA_CHECK_SUP(Kg % 64 == 0 && (G * R) % 64 == 0, "Kg and G*R must be multiples of 64");
  CSA_CHECK_SUP(R % 128 == 0 && D % 128 == 0, "R and D must be multiples of 128");
  CSA_CHECK_SUP((long long)G * Kg <= (1LL << 31) && (long long)G * R <= (1LL << 31), "too wide");
  if (int rc = check_ws(ws, ws_bytes, kStatusBytes)) return rc;
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  CSA_CHECK_SUP(gemm_smem_bytes() <= (size_t)dev->max_smem, "shared memory too small for the GEMM kernel");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  // r = o . Wo_a^T per group (bf16 out).
  GemmParams P1{};
  P1.M = M;
  P1.N = R;
  P1.K = Kg;
  P1.splits = 1;
  P1.a_group_cols = Kg;
  P1.b_group_rows = R;
  P1.c_group_cols = R;
  P1.ldc = (long long)G * R;
  P1.c = r;
  P1.c_mode = kGemmOutBf16;
  P1.status = status;
  if (int rc = run_gemm(o, (uint64_t)G * Kg, (uint64_t)M, (uint64_t)G * Kg, wo_a, (uint64_t)Kg, (uint64_t)G * R,
                        (uint64_t)Kg, P1, G, dev->sms, st))
    return rc;
  // y = r . Wo_b^T; when the output tiles alone would leave SMs idle, K is split (fp32 reduction).
  const int splits = gemm_splits((long long)(D / 128) * ((M + 127) / 128), G * R / 64, dev->sms);
  GemmParams P2{};
  P2.M = M;
  P2.N = D;
  P2.K = G * R;
  P2.splits = splits;
  P2.ldc = D;
  P2.c = y;
  P2.c_mode = splits > 1 ? kGemmOutF32Add : kGemmOutF32;
  P2.status = status;
  return run_gemm(r, (uint64_t)G * R, (uint64_t)M, (uint64_t)G * R, wo_b, (uint64_t)G * R, (uint64_t)D,
                  (uint64_t)G * R, P2, 1, dev->sms, st);
}

int csa_linear(int M, int N, int K, const uint16_t* x, const uint16_t* w, void* y, int y_is_f32, void* ws,
               size_t ws_bytes, void* stream) {
  CSA_CHECK_ARG(M > 0 && N > 0 && K > 0, "sizes must be positive");
  CSA_CHECK_ARG(x && w && y, "null pointer");
  CSA_CHECK_ARG(aligned(x, 16) && aligned(w, 16) && aligned(y, 16), "pointers must be 16-byte aligned");
  CSA_CHECK_SUP(N % 128 == 0 && K % 64 == 0, "N must be a multiple of 128 and K of 64");
  if (int rc = check_ws(ws, ws_bytes, kStatusBytes)) return rc;
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  GemmParams P{};
  P.M = M;
  P.N = N;
  P.K = K;
  // fp32 output may be split over K (fp32 reductions); bf16 output is stored by one CTA per tile.
  P.splits = y_is_f32 ? gemm_splits((long long)(N / 128) * ((M + 127) / 128), K / 64, dev->sms) : 1;
  P.ldc = N;
  P.c = y;
  P.c_mode = !y_is_f32 ? kGemmOutBf16 : (P.splits > 1 ? kGemmOutF32Add : kGemmOutF32);
  P.status = reinterpret_cast<uint32_t*>(ws);
  return run_gemm(x, (uint64_t)K, (uint64_t)M, (uint64_t)K, w, (uint64_t)K, (uint64_t)N, (uint64_t)K, P, 1, dev->sms,
                  static_cast<cudaStream_t>(stream));
}

int csa_q_projection(int M, int hidden, int q_rank, int H, int d, int rope_dim, float rope_base, float eps,
                     const int32_t* pos, const uint16_t* x, const uint16_t* wq_a, const uint16_t* gamma,
                     const uint16_t* wq_b, float* qa, uint16_t* qr, uint16_t* q, void* ws, size_t ws_bytes,
                     void* stream) {
  CSA_CHECK_ARG(M > 0 && hidden > 0 && q_rank > 0 && H > 0, "sizes must be positive");
  CSA_CHECK_ARG(pos && x && wq_a && gamma && wq_b && qa && qr && q, "null pointer");
  CSA_CHECK_ARG(aligned(x, 16) && aligned(wq_a, 16) && aligned(gamma, 16) && aligned(wq_b, 16) && aligned(qa, 16) &&
                    aligned(qr, 16) && aligned(q, 16) && aligned(pos, 4),
                "pointers must be 16-byte aligned");
  CSA_CHECK_SUP(d == 512, "d must be 512");
  CSA_CHECK_SUP(rope_dim > 0 && rope_dim % 2 == 0 && rope_dim / 2 <= kMaxRopePairs, "rope_dim must be even, <= 128");
  CSA_CHECK_SUP(hidden % 64 == 0 && q_rank % 128 == 0 && (H * d) % 128 == 0,
                "hidden must be a multiple of 64, q_rank and H*d of 128");
  CSA_CHECK_SUP((long long)M * H <= (1LL << 31) - 1, "too many rows");
  if (int rc = check_ws(ws, ws_bytes, kStatusBytes)) return rc;
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  // qa = x . wq_a^T (fp32; split over K when the 128-column tiles alone leave SMs idle).
  GemmParams P1{};
  P1.M = M;
  P1.N = q_rank;
  P1.K = hidden;
  P1.splits = gemm_splits((long long)(q_rank / 128) * ((M + 127) / 128), hidden / 64, dev->sms);
  P1.ldc = q_rank;
  P1.c = qa;
  P1.c_mode = P1.splits > 1 ? kGemmOutF32Add : kGemmOutF32;
  P1.status = status;
  if (int rc = run_gemm(x, (uint64_t)hidden, (uint64_t)M, (uint64_t)hidden, wq_a, (uint64_t)hidden, (uint64_t)q_rank,
                        (uint64_t)hidden, P1, 1, dev->sms, st))
    return rc;
  CSA_CUDA(launch_pdl(rmsnorm_rows_kernel, dim3((unsigned)M), dim3(kRowNormThreads), 0, st,
                      static_cast<const float*>(qa), gamma, qr, q_rank, eps));
  // q = qr . wq_b^T (bf16), then the per-head norm and RoPE in place.
  GemmParams P2{};
  P2.M = M;
  P2.N = H * d;
  P2.K = q_rank;
  P2.splits = 1;
  P2.ldc = (long long)H * d;
  P2.c = q;
  P2.c_mode = kGemmOutBf16;
  P2.status = status;
  if (int rc = run_gemm(qr, (uint64_t)q_rank, (uint64_t)M, (uint64_t)q_rank, wq_b, (uint64_t)q_rank,
                        (uint64_t)H * d, (uint64_t)q_rank, P2, 1, dev->sms, st))
    return rc;
  HeadNormParams N{};
  N.M = M;
  N.H = H;
  N.rope_dim = rope_dim;
  N.normalize = 1;
  N.eps = eps;
  for (int i = 0; i < rope_dim / 2; ++i) N.inv_freq[i] = std::pow((double)rope_base, -2.0 * i / rope_dim);
  N.pos = pos;
  N.q = q;
  const long long items = (long long)M * H;
  const int per = kHeadNormThreads / 32;
  CSA_CUDA(launch_pdl(head_norm_rope_kernel, dim3((unsigned)((items + per - 1) / per)), dim3(kHeadNormThreads), 0,
                      st, N));
  return CSA_OK;
}

int csa_window_projection(int M, int hidden, int d, int rope_dim, float rope_base, const int32_t* pos,
                          const uint16_t* x, const uint16_t* wkv, uint16_t* win, void* ws, size_t ws_bytes,
                          void* stream) {
  CSA_CHECK_ARG(M > 0 && hidden > 0, "sizes must be positive");
  CSA_CHECK_ARG(pos && x && wkv && win, "null pointer");
  CSA_CHECK_ARG(aligned(x, 16) && aligned(wkv, 16) && aligned(win, 16) && aligned(pos, 4),
                "pointers must be 16-byte aligned");
  CSA_CHECK_SUP(d == 512, "d must be 512");
  CSA_CHECK_SUP(rope_dim > 0 && rope_dim % 2 == 0 && rope_dim / 2 <= kMaxRopePairs, "rope_dim must be even, <= 128");
  CSA_CHECK_SUP(hidden % 64 == 0, "hidden must be a multiple of 64");
  if (int rc = check_ws(ws, ws_bytes, kStatusBytes)) return rc;
  DeviceInfo* dev;
  if (int rc = device_info(&dev)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmParams P{};
  P.M = M;
  P.N = d;
  P.K = hidden;
  P.splits = 1;
  P.ldc = d;
  P.c = win;
  P.c_mode = kGemmOutBf16;
  P.status = reinterpret_cast<uint32_t*>(ws);
  if (int rc = run_gemm(x, (uint64_t)hidden, (uint64_t)M, (uint64_t)hidden, wkv, (uint64_t)hidden, (uint64_t)d,
                        (uint64_t)hidden, P, 1, dev->sms, st))
    return rc;
  HeadNormParams N{};
  N.M = M;
  N.H = 1;
  N.rope_dim = rope_dim;
  N.normalize = 0;
  N.eps = 0.f;
  for (int i = 0; i < rope_dim / 2; ++i) N.inv_freq[i] = std::pow((double)rope_base, -2.0 * i / rope_dim);
  N.pos = pos;
  N.q = win;
  const int per = kHeadNormThreads / 32;
  CSA_CUDA(launch_pdl(head_norm_rope_kernel, dim3((unsigned)((M + per - 1) / per)), dim3(kHeadNormThreads), 0, st, N));
  return CSA_OK;
}

int csa_decode_fused(const csa_decode_args* a, void* stream) {
  CSA_CHECK_ARG(a != nullptr, "args is null");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const csa_compressor_cfg main_cfg{a->ratio, 1, a->d, a->rope_dim, a->rope_base, a->eps};
  const csa_compressor_cfg idx_cfg{a->ratio, 1, a->d_I, a->rope_dim, a->rope_base, a->eps};
  CSA_CHECK_SUP(a->ratio == 4, "CSA decode uses ratio 4");
  if (int rc = check_compress_args(&main_cfg, a->B, 1, a->pos, a->kv, a->score, a->gamma, a->state_kv,
                                   a->state_score, a->cache, a->cache_bstride, a->max_entries, a->cache_f32))
    return rc;
  if (int rc = check_compress_args(&idx_cfg, a->B, 1, a->pos, a->idx_kv, a->idx_score, a->idx_gamma,
                                   a->idx_state_kv, a->idx_state_score, a->idx_cache, a->idx_bstride,
                                   a->max_entries, nullptr))
    return rc;
  CSA_CHECK_ARG(a->win_kv && aligned(a->win_kv, 16), "win_kv null or misaligned");
  IndexerArgs ia{a->B, 1, a->H_I, a->d_I, a->ratio, a->topk, a->pos, a->q_idx, a->w, a->idx_cache, a->idx_bstride,
                 a->max_entries, a->topk_idx, nullptr, a->ws, a->ws_bytes};
  if (int rc = check_indexer_args(ia)) return rc;
  AttnArgs aa{a->B, 1, a->H, a->d, a->rope_dim, a->rope_base, a->scale, a->ratio, a->pos, a->q, a->ring,
              a->ring_bstride, a->ring_cap, a->window, a->cache, a->cache_bstride, a->max_entries, a->topk_idx,
              a->topk, a->sink, a->out, a->out_is_f32, a->ws, a->ws_bytes};
  if (int rc = check_attn_args(aa, true)) return rc;
  const IdxWs L = indexer_ws_layout(a->B, a->max_entries, a->topk, true);
  if (int rc = check_ws(a->ws, a->ws_bytes, L.total)) return rc;
  aa.part_off = L.total;  // the attention's split partials follow the indexer's buffers
  // The ring row of token t is written by the indexer launch; the top-k launch between it and the
  // attention waits for it to complete before it triggers the attention's launch.
  aa.early_window = true;

  uint32_t* status = static_cast<uint32_t*>(a->ws);
  CompressLaunch CL{};
  CL.p[0] = compress_params(&main_cfg, a->B, 1, a->pos, a->kv, a->score, a->gamma, a->state_kv, a->state_score,
                            a->cache, a->cache_bstride, a->max_entries, a->cache_f32, status);
  CL.p[0].win_src = a->win_kv;
  CL.p[0].ring = a->ring;
  CL.p[0].ring_bstride = a->ring_bstride;
  CL.p[0].ring_cap = a->ring_cap;
  CL.p[1] = compress_params(&idx_cfg, a->B, 1, a->pos, a->idx_kv, a->idx_score, a->idx_gamma, a->idx_state_kv,
                            a->idx_state_score, a->idx_cache, a->idx_bstride, a->max_entries, nullptr, status);
  cudaEvent_t const* ev = reinterpret_cast<cudaEvent_t const*>(a->stage_events);
  // The compressor step of both streams runs inside the indexer launch (its epilogue warps, before
  // their first tile); the "compress" stage interval is therefore empty.
  if (ev) CSA_CUDA(cudaEventRecord(ev[0], st));
  if (ev) CSA_CUDA(cudaEventRecord(ev[1], st));
  if (int rc = run_indexer_topk(ia, st, ev ? ev + 2 : nullptr, true, true, &CL)) return rc;
  if (int rc = run_attn(aa, true, st)) return rc;
  if (ev) CSA_CUDA(cudaEventRecord(ev[4], st));
  return CSA_OK;
}

int hca_decode_fused(const hca_decode_args* a, void* stream) {
  CSA_CHECK_ARG(a != nullptr, "args is null");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const csa_compressor_cfg cfg{a->ratio, 0, a->d, a->rope_dim, a->rope_base, a->eps};
  CSA_CHECK_SUP(a->ratio == 128, "HCA decode uses ratio 128");
  if (int rc = check_compress_args(&cfg, a->B, 1, a->pos, a->kv, a->score, a->gamma, a->state_kv, a->state_score,
                                   a->cache, a->cache_bstride, a->max_entries, a->cache_f32))
    return rc;
  CSA_CHECK_ARG(a->win_kv && aligned(a->win_kv, 16), "win_kv null or misaligned");
  AttnArgs aa{a->B, 1, a->H, a->d, a->rope_dim, a->rope_base, a->scale, a->ratio, a->pos, a->q, a->ring,
              a->ring_bstride, a->ring_cap, a->window, a->cache, a->cache_bstride, a->max_entries, nullptr, 0,
              a->sink, a->out, a->out_is_f32, a->ws, a->ws_bytes};
  if (int rc = check_attn_args(aa, false)) return rc;
  uint32_t* status = static_cast<uint32_t*>(a->ws);
  CompressLaunch CL{};
  CL.p[0] = compress_params(&cfg, a->B, 1, a->pos, a->kv, a->score, a->gamma, a->state_kv, a->state_score, a->cache,
                            a->cache_bstride, a->max_entries, a->cache_f32, status);
  CL.p[0].win_src = a->win_kv;
  CL.p[0].ring = a->ring;
  CL.p[0].ring_bstride = a->ring_bstride;
  CL.p[0].ring_cap = a->ring_cap;
  CL.p[1] = CL.p[0];
  cudaEvent_t const* ev = reinterpret_cast<cudaEvent_t const*>(a->stage_events);
  if (ev) CSA_CUDA(cudaEventRecord(ev[0], st));
  if (int rc = launch_compress(CL, 1, a->B, 1, a->ratio, st)) return rc;
  if (ev) CSA_CUDA(cudaEventRecord(ev[1], st));
  if (int rc = run_attn(aa, false, st)) return rc;
  if (ev) CSA_CUDA(cudaEventRecord(ev[2], st));
  return CSA_OK;
}

int csa_get_device_status(void* ws, void* stream, int* status) {
  CSA_CHECK_ARG(ws != nullptr && status != nullptr && aligned(ws, 256), "bad arguments");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  CSA_CUDA(cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st));
  CSA_CUDA(cudaStreamSynchronize(st));
  const uint32_t zero = 0;
  CSA_CUDA(cudaMemcpyAsync(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice, st));
  CSA_CUDA(cudaStreamSynchronize(st));
  *status = (int)v;
  return CSA_OK;
}

}  // extern "C"
