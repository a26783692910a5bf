// kernels.cuh -- parameter blocks and launch constants shared by the kernels and the C ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "status.cuh"

namespace csa {

// ------------------------------------------------------------------------------ compressor (K1)

constexpr int kCompressThreads = 256;
constexpr int kMaxRopePairs = 64;
// Per-thread stash of C4A cur rows that become pre rows (update_state, phase A). The host checks
// ratio * width / 8 <= kMaxKeepChunks * kCompressThreads.
constexpr int kMaxKeepChunks = 4;

struct CompressParams {
  int ratio, overlap, d, rope_dim;
  float rope_base, eps;
  double inv_freq[kMaxRopePairs];   // rope_base^(-2i/rope_dim), formed on the host in double
  int B, S;
  const int32_t* start_pos;   // [B]
  const uint16_t* kv;         // [B, S, width]
  const uint16_t* score;      // [B, S, width]
  const uint16_t* gamma;      // [d]
  uint16_t* state_kv;         // [B, rows, width]
  uint16_t* state_score;
  uint16_t* cache;            // entry g of request b at cache + b*cache_bstride + g*d
  long long cache_bstride;
  int max_entries;
  float* cache_f32;           // nullable, same layout as cache
  // Window-ring write of the fused decode step (nullable win_src disables it; S == 1 only).
  const uint16_t* win_src;    // [B, d]
  uint16_t* ring;
  long long ring_bstride;
  int ring_cap;
  uint32_t* status;
};

struct CompressLaunch {
  CompressParams p[2];        // blockIdx.z selects the stream (main / index)
};

__global__ void compress_kernel(CompressLaunch L);
__global__ void compress_decode_kernel(CompressLaunch L);
constexpr int kC128Split = 8;             // CTAs (channel blocks) per request of the C128A decode step
__global__ void compress_decode_c128_kernel(CompressLaunch L);
__global__ void compress_state_kernel(CompressLaunch L);
__global__ void state_reset_kernel(uint16_t* kv, uint16_t* score, long long n);


// ------------------------------------------------------------------------------ indexer (K2)

constexpr int kIdxThreads = 320;          // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue (2 groups)
constexpr int kIdxMaxStages = 8;

struct IndexerParams {
  int B, S;
  int QG;                                 // queries per group (N = QG*H_I columns, padded to 16)
  int N;
  int ratio, max_entries;
  int groups_per_req, tiles_per_group;
  long long total_items;                  // B * groups_per_req * tiles_per_group
  long long rows_per_req;                 // index-cache rows per request (idx_bstride / d_I)
  int stages, tmem_cols, n_acc;
  const int32_t* q_pos;                   // [B*S]
  const float* w;                         // [B*S, H_I]
  float* scores;                          // [B*S, scores_stride]
  long long scores_stride;
  uint32_t* status;
};

// The decode step's compression, run by the indexer (csa_decode_fused): the epilogue warps of CTA c
// take jobs c, c + gridDim.x, ... before their first tile. Job j < B compresses request j's index
// stream (L.p[1]) and then raises flags[j]; job B + j request j's main stream (L.p[0]). The producer
// waits for flags[b] before it loads the tile holding request b's last visible entry (the one the
// step may complete) and clears it. njobs = 0: no compression.
struct IndexerFuse {
  int njobs, B;
  uint32_t* flags;                        // [B]; zero between calls
  CompressLaunch L;
};

template <int HI>
__global__ void indexer_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                               IndexerParams P, IndexerFuse F);

// ------------------------------------------------------------------------------ top-k (K3)

constexpr int kTopkThreads = 1024;
constexpr int kTopkShortThreads = 1024;   // rows of <= kTopkShortRow entries: 1024 threads x 8 keys
constexpr int kTopkShortRow = 8192;
constexpr int kTopkChunk = 16384;         // entries per chunk (staged in 64 KB of smem)
constexpr int kTopkMaxChunks = 1024;

struct TopkParams {
  int topk, ratio, max_entries;
  int chunk, max_chunks;
  const int32_t* q_pos;                   // [queries]
  const float* scores;                    // [queries, scores_stride]
  long long scores_stride;
  int32_t* out;                           // [queries, topk]
  uint32_t* cand_key;                     // [queries, max_chunks, topk]
  int32_t* cand_idx;
  int* cand_cnt;                          // [queries, max_chunks]
  uint32_t* status;
};

__global__ void topk_chunk_kernel(TopkParams P);
__global__ void topk_merge_kernel(TopkParams P);

// ------------------------------------------------------------------------------ attention (K4/K5)

constexpr int kAttnThreads = 608;         // warps 0..3 gathers, 4-5 score MMAs, 6 PV MMAs, 7..10 senders, 11..18 softmax
constexpr int kAttnMaxWindow = 1024;
constexpr int kAttnMaxTopk = 2048;
constexpr int kAttnMaxCompressed = 2048;  // HCA: visible entries read per query
constexpr int kAttnMaxCands = 3200;       // window + entries + padding
constexpr int kAttnMaxTiles = kAttnMaxCands / 64;

struct AttnParams {
  int B, S, H, d, rope_dim;
  float scale_log2;                       // scale * log2(e)
  double inv_freq[kMaxRopePairs];         // rope_base^(-2i/rope_dim), formed on the host in double
  int window, ring_cap;
  long long ring_rows;                    // ring rows per request (ring_bstride / d)
  long long cache_rows;                   // cache rows per request (cache_bstride / d)
  int max_entries, ratio;
  const int32_t* q_pos;                   // [B*S]
  const uint16_t* ring;                   // row r (of B*ring_rows) at ring + r*d
  const uint16_t* cache;                  // row r (of B*cache_rows) at cache + r*d
  const int32_t* topk_idx;                // [B*S, topk]; null: HCA (every visible entry)
  int topk;
  const float* sink;                      // [H]
  void* out;                              // [B*S, H, d]
  int out_is_f32;
  uint32_t* status;
  // Split-candidate mode (splits > 1): the CTA pair of work item (query qi, split s) takes the s-th
  // of `splits` contiguous runs of the query's candidate tiles and leaves its unnormalised partial
  // in part_o [item, H, d] (fp32, O relative to the partial's max) and part_ml [item, 2, H] (the max
  // in log2 units, then the denominator), item = qi * splits + s; attn_combine_kernel merges them.
  int splits;
  float* part_o;
  float* part_ml;
  // Nonzero when q, q_pos and the ring rows are final before the kernel's dependency wait: the
  // launch before this one waits for the launch that writes them before it lets this one start
  // (the fused CSA decode step: compressor step and ring write in the indexer launch, then top-k,
  // then this kernel). The producers then load Q and gather the window tiles first.
  int early_window;
};

__global__ void attn_kernel(const __grid_constant__ CUtensorMap map_q, AttnParams P);

constexpr int kAttnMaxSplits = 16;
constexpr int kAttnCombineThreads = 128;  // one (query, head) row of 512 dims per CTA, 4 per thread

struct AttnCombineParams {
  int splits, H, d, rope_dim;
  double inv_freq[kMaxRopePairs];
  const int32_t* q_pos;
  const float* part_o;
  const float* part_ml;
  void* out;
  int out_is_f32;
  uint32_t* status;
};

__global__ void attn_combine_kernel(AttnCombineParams P);

// ------------------------------------------------------------------------------ output projection

constexpr int kGemmThreads = 128;
constexpr int kGemmStages = 6;
constexpr int kGemmOutBf16 = 0;           // C stored as bf16
constexpr int kGemmOutF32 = 1;            // C stored as fp32
constexpr int kGemmOutF32Add = 2;         // C += tile (fp32 reduction; C zeroed first), for split K

// C[m, g*c_group_cols + n] = sum_k A[m, g*a_group_cols + k] * B[g*b_group_rows + n, k] over this CTA's
// K split; A, B through the tensor maps (bf16, 128B swizzle, boxes of 64 x 128).
struct GemmParams {
  int M, N, K;                            // rows of C, columns of C per group, K per group
  int splits;                             // K splits (blockIdx.z = group * splits + split)
  int a_group_cols, b_group_rows, c_group_cols;
  long long ldc;                          // row pitch of C (elements)
  void* c;
  int c_mode;
  uint32_t* status;
};

__global__ void gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                            GemmParams P);
__global__ void zero_f32_kernel(float* p, long long n4);

// ------------------------------------------------------------------------------ query path

constexpr int kRowNormThreads = 256;
constexpr int kHeadNormThreads = 256;     // 8 warps: one (row, head) each

struct HeadNormParams {
  int M, H, rope_dim;
  int normalize;                          // 1: divide each head by its RMS first (query path)
  float eps;
  double inv_freq[kMaxRopePairs];         // rope_base^(-2i/rope_dim), formed on the host in double
  const int32_t* pos;                     // [M] token positions
  uint16_t* q;                            // [M, H, 512] bf16, normalised and rotated in place
};

__global__ void rmsnorm_rows_kernel(const float* x, const uint16_t* gamma, uint16_t* y, int n, float eps);
__global__ void head_norm_rope_kernel(HeadNormParams P);

// Host-side checks of csa_indexer_topk's arguments, the workspace aside (api.cu): the
// workspace-free entry point runs them before it touches its fixed scratch array.
int check_indexer_topk_args(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                            const uint16_t* q_idx, const float* w, const uint16_t* idx_cache, int64_t idx_bstride,
                            int max_entries, const int32_t* topk_idx);

size_t attn_smem_bytes();
size_t gemm_smem_bytes();
size_t indexer_smem_bytes(int stages, int N, bool fuse);

}  // namespace csa
