/*
 * csa.h -- C ABI of libcsa.so: the DeepSeek-V4-Pro compressed-sparse-attention (CSA)
 * layer and its heavily-compressed (HCA) variant on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [P1] "DeepSeek-V4-Pro 架构：一个 token 的旅程" (hs-black.github.io/posts/deepseek-v4-pro)
 *   [P5] "图解DeepSeek V4：详细计算流程解析" (jsqmd.com)
 *
 * Conventions for every entry point:
 *   - Pointers marked "dev" are device pointers owned by the caller. The library never
 *     allocates or frees memory; scratch space is the caller's workspace `ws`.
 *   - bf16 values are passed as uint16_t (IEEE bfloat16 bit patterns).
 *   - `stream` is a cudaStream_t passed as void*. Every call only enqueues work on it; no
 *     call synchronises the host except csa_get_device_status.
 *   - Every call returns a csa_status. Arguments are checked on the host before any launch:
 *     on CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED / CSA_ERR_WORKSPACE nothing was enqueued.
 *     CSA_ERR_CUDA reports a launch error; csa_last_error() gives its text.
 *   - Device-side faults never trap: a kernel that gives up a bounded wait, or that meets an
 *     out-of-range index, records a code in the workspace status word and returns.
 *     csa_get_device_status reads it.
 *   - Positions t are absolute token positions (0-based). Batch strides are in elements.
 *   - Every size that counts work (B, S, M, the widths) must be at least 1: a call with no work
 *     (B = 0, S = 0, M = 0) is refused with CSA_ERR_INVALID_ARG and enqueues nothing, so a
 *     caller with an empty batch skips the call.
 *   - Thread safety: the library keeps no state except a thread-local error string.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer or stride */
  CSA_ERR_UNSUPPORTED = 2,   /* a shape outside what the kernels implement */
  CSA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  CSA_ERR_TIMEOUT = 4,       /* (device status) a bounded wait inside a kernel gave up */
  CSA_ERR_WORKSPACE = 5,     /* ws is null, misaligned or smaller than csa_workspace_size */
  CSA_ERR_BOUNDS = 6         /* (device status) an index read from memory was out of range */
} csa_status;

/* Text of a status code (static string). */
CSA_API const char* csa_status_string(int status);
/* Text of the last CSA_ERR_CUDA / argument error seen on the calling thread. */
CSA_API const char* csa_last_error(void);
/* ABI version: 1. */
CSA_API int csa_version(void);

/*
 * Compressor configuration.
 *   ratio 4,  overlap 1: C4A. Each token carries kv and score streams of width 2d; compressed
 *             entry g pools channels [:d] of group g-1's 4 tokens and channels [d:] of group
 *             g's 4 tokens (8 slots per channel) ([P5] §2.1, the torch.cat of pre/cur state).
 *   ratio 128, overlap 0: C128A. Streams of width d; entry g pools tokens 128g..128g+127
 *             ([P5] §3.1, "state is concatenated directly").
 * Pooling is a per-channel softmax over the slots times kv, summed over slots; then
 * RMSNorm (gamma, eps) over the d dims, then RoPE on the last rope_dim dims at position
 * g*ratio ([P1] "压缩是逐通道的 learned pooling"). RoPE rotates adjacent pairs (2i, 2i+1) by
 * pos * rope_base^(-2i/rope_dim).
 * Supported: (ratio, overlap) in {(4,1), (128,0)}; d in {128, 512}; rope_dim 64 (even, <= d,
 * multiple of 8).
 */
typedef struct {
  int ratio;
  int overlap;
  int d;
  int rope_dim;
  float rope_base;
  float eps;
} csa_compressor_cfg;

/* Workspace kinds for csa_workspace_size. */
enum {
  CSA_WS_INDEXER_TOPK = 1,
  CSA_WS_SPARSE_ATTN = 2,
  CSA_WS_HCA_ATTN = 3,
  CSA_WS_DECODE_FUSED = 4,
  CSA_WS_HCA_DECODE_FUSED = 5,
  CSA_WS_OUTPUT_PROJ = 6,
  CSA_WS_Q_PROJ = 7
};

/*
 * Bytes of workspace the call of `kind` needs for B requests x S queries, with up to
 * max_entries compressed entries per request and top-k `topk` (ignored for HCA kinds).
 * The workspace must be 256-byte aligned. Its first 256 bytes hold the device status word;
 * the caller zeroes the whole workspace once before first use (later calls keep the status
 * word sticky until csa_get_device_status clears it).
 * The attention kinds (and CSA_WS_DECODE_FUSED) also hold, for small batches (B*S <= 37), the
 * partial results of split-candidate attention: a query's candidates are then spread over
 * min(16, 74 / (B*S)) CTA pairs, each leaving 128 x 512 + 2 x 128 floats that a second kernel
 * merges. A smaller workspace (down to the 256-byte status word) is accepted by the attention
 * entry points: they then run one CTA pair per query (same results up to rounding, slower).
 */
CSA_API int csa_workspace_size(int kind, int B, int S, int max_entries, int topk, size_t* bytes);

/*
 * Put a compressor state into its initial value: kv rows 0, score rows -inf, so that the
 * previous-group slots of group 0 carry gate -inf and weight 0 ([P1] "一个通道，逐项算出压缩结果").
 *   state_kv, state_score: dev bf16 [B, rows, width], rows = (1+overlap)*ratio,
 *                          width = (1+overlap)*d.
 */
CSA_API int csa_state_reset(const csa_compressor_cfg* cfg, int B, uint16_t* state_kv, uint16_t* state_score,
                    void* stream);

/*
 * csa_compress -- run the compressor over a segment of S new tokens per request
 * ([P5] §2.1 and §3.1; [P1] "压缩条目必须等整组完成后才可见": entry t//ratio is written when
 * (t+1) % ratio == 0; prefill computes every completed entry of the segment in parallel).
 *   start_pos   dev int32 [B]: position of each request's first new token.
 *   kv, score   dev bf16 [B, S, width] (width = (1+overlap)*d), contiguous.
 *   gamma       dev bf16 [d]: RMSNorm weight.
 *   state_kv, state_score  dev bf16 [B, rows, width], in/out. On entry: the state after token
 *               start_pos-1 (or csa_state_reset). On exit: the state after token start_pos+S-1,
 *               exactly as the token-by-token rolling state would leave it: token p lives in row
 *               ratio + p%ratio (C4A) or p%ratio (C128A); after each completed group the C4A cur
 *               rows are copied over the pre rows.
 *   cache       dev bf16, entry g of request b at cache + b*cache_bstride + g*d. Only entries that
 *               complete inside the segment are written. g must be < max_entries.
 *   cache_f32   optional dev float with the same layout (nullable): the same entries before the
 *               bf16 rounding.
 * Alignment: all pointers 16-byte aligned; cache_bstride a multiple of 8.
 * Errors: CSA_ERR_INVALID_ARG on a null or misaligned pointer, B<=0, S<=0.
 */
CSA_API int csa_compress(const csa_compressor_cfg* cfg, int B, int S, const int32_t* start_pos,
                 const uint16_t* kv, const uint16_t* score, const uint16_t* gamma,
                 uint16_t* state_kv, uint16_t* state_score,
                 uint16_t* cache, int64_t cache_bstride, int max_entries, float* cache_f32,
                 void* stream);

/*
 * csa_indexer_topk -- lightning indexer and top-k selection ([P1] "少读 KV 之前，Indexer 仍要给历史打分";
 * [P5] §2.2). For query i of request b at position t = q_pos[b*S+i], with E = (t+1)//ratio visible
 * entries:
 *     score[s] = sum_h w[h] * ReLU(q_idx[h,:] . idx_cache[s,:])      for s < E
 * then the indices of the min(topk, E) largest scores (ties to the lower index), written in
 * ascending order and padded with -1.
 *   q_pos     dev int32 [B, S].
 *   q_idx     dev bf16 [B, S, H_I, d_I].   w: dev float [B, S, H_I] (may be negative).
 *   idx_cache dev bf16, entry s of request b at idx_cache + b*idx_bstride + s*d_I.
 *   topk_idx  dev int32 [B, S, topk], out.
 *   scores_opt optional dev float [B, S, max_entries], out (nullable): the scores, s < E only.
 *   ws/ws_bytes: workspace of at least csa_workspace_size(CSA_WS_INDEXER_TOPK, ...).
 * Supported: d_I = 128; H_I a power of two in [4, 128]; topk in [1, 2048]; E <= max_entries <= 2^24.
 * A query with E > max_entries records CSA_ERR_BOUNDS in the status word and uses max_entries.
 */
CSA_API int csa_indexer_topk(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                     const uint16_t* q_idx, const float* w, const uint16_t* idx_cache,
                     int64_t idx_bstride, int max_entries, int32_t* topk_idx, float* scores_opt,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * csa_sparse_attn -- sparse MQA over one candidate set with a learned sink, then inverse RoPE
 * ([P1] "局部和压缩记忆，共用一次归一化" and "输出投影也分组"; [P5] §2 and §2.3).
 * For query i of request b at position t:
 *   candidates C = window rows ring[p % ring_cap] for p = max(0, t-window+1) .. t
 *                  plus cache rows s for every topk_idx[b,i,j] >= 0 (entries < max_entries);
 *   one cached row serves as key and value (MQA). For each head h:
 *     l_j = scale * q[h] . c_j;  m = max(max_j l_j, sink[h]);
 *     o[h] = sum_j e^(l_j-m) c_j / (sum_j e^(l_j-m) + e^(sink[h]-m));
 *   then the last rope_dim dims of o[h] are rotated by -t (inverse RoPE).
 *   q      dev bf16 [B, S, H, d].   sink: dev float [H].
 *   ring   dev bf16, slot j of request b at ring + b*ring_bstride + j*d; window <= ring_cap.
 *   cache  dev bf16, entry s at cache + b*cache_bstride + s*d.
 *   topk_idx dev int32 [B, S, topk].
 *   out    dev [B, S, H, d]: bf16 if out_is_f32 == 0, float otherwise.
 * Supported: d = 512, rope_dim 64, 1 <= H <= 128, window <= 1024, topk <= 2048.
 * Alignment: pointers 16 bytes; ring_bstride and cache_bstride multiples of d.
 * A selected index s >= min((t+1)//ratio, max_entries) (an entry not visible at t) is skipped and
 * records CSA_ERR_BOUNDS in the workspace's status word (csa_get_device_status).
 */
CSA_API int csa_sparse_attn(int B, int S, int H, int d, int rope_dim, float rope_base, float scale,
                    const int32_t* q_pos, const uint16_t* q, const uint16_t* ring,
                    int64_t ring_bstride, int ring_cap, int window, const uint16_t* cache,
                    int64_t cache_bstride, int max_entries, const int32_t* topk_idx, int topk,
                    const float* sink, void* out, int out_is_f32, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * hca_attn -- HCA attention ([P5] §3: no index module): as csa_sparse_attn, but the compressed
 * candidates are every visible entry s < (t+1)//ratio (capped at max_entries), read in order.
 * Supported: as csa_sparse_attn, with at most 2048 visible entries per query; a query with more
 * attends to the first 2048 and records CSA_ERR_BOUNDS in the workspace's status word.
 */
CSA_API int hca_attn(int B, int S, int H, int d, int rope_dim, float rope_base, float scale, int ratio,
             const int32_t* q_pos, const uint16_t* q, const uint16_t* ring, int64_t ring_bstride,
             int ring_cap, int window, const uint16_t* cache, int64_t cache_bstride,
             int max_entries, const float* sink, void* out, int out_is_f32, void* ws,
             size_t ws_bytes, void* stream);

/*
 * Arguments of one CSA decode step for B requests (S = 1), each at its own position pos[b].
 * Shapes follow [P5] §2: per token the main compressor streams are [2d], the index compressor
 * streams [2 d_I], the window row [d] (already rotated by RoPE upstream), q [H, d], q_idx
 * [H_I, d_I], w [H_I].
 */
typedef struct {
  int B;
  int H, d, rope_dim;          /* 128, 512, 64 */
  int H_I, d_I;                /* 64, 128 */
  int ratio;                   /* 4 */
  int window;                  /* 128 */
  int topk;                    /* 1024 */
  float rope_base, eps, scale; /* 1e4, 1e-6, 1/sqrt(d) */
  const int32_t* pos;          /* dev [B] */
  const uint16_t* kv;          /* dev [B, 2d]   main compressor kv stream of token pos[b] */
  const uint16_t* score;       /* dev [B, 2d] */
  const uint16_t* idx_kv;      /* dev [B, 2d_I] index compressor streams */
  const uint16_t* idx_score;   /* dev [B, 2d_I] */
  const uint16_t* win_kv;      /* dev [B, d] window row of token pos[b] */
  const uint16_t* q;           /* dev [B, H, d] */
  const uint16_t* q_idx;       /* dev [B, H_I, d_I] */
  const float* w;              /* dev [B, H_I] */
  const float* sink;           /* dev [H] */
  const uint16_t* gamma;       /* dev [d] */
  const uint16_t* idx_gamma;   /* dev [d_I] */
  uint16_t* state_kv;          /* dev [B, 2ratio, 2d] in/out */
  uint16_t* state_score;
  uint16_t* idx_state_kv;      /* dev [B, 2ratio, 2d_I] in/out */
  uint16_t* idx_state_score;
  uint16_t* cache;             /* dev, entry g at cache + b*cache_bstride + g*d */
  int64_t cache_bstride;
  uint16_t* idx_cache;         /* dev, entry g at idx_cache + b*idx_bstride + g*d_I */
  int64_t idx_bstride;
  int max_entries;
  uint16_t* ring;              /* dev, slot j at ring + b*ring_bstride + j*d */
  int64_t ring_bstride;
  int ring_cap;
  int32_t* topk_idx;           /* dev [B, topk] out: the selection used */
  float* cache_f32;            /* nullable dev, as cache: the new main entry before rounding */
  void* out;                   /* dev [B, H, d] */
  int out_is_f32;
  void* ws;
  size_t ws_bytes;             /* >= csa_workspace_size(CSA_WS_DECODE_FUSED, B, 1, max_entries, topk) */
  void* const* stage_events;   /* nullable: 5 cudaEvent_t recorded on the stream before the compressor
                                  step, after it, after the indexer, after top-k and after attention */
} csa_decode_args;

/*
 * csa_decode_fused -- one CSA decode step ([P5] §2 order): the C4A step of the main and index
 * streams (writing entry pos//ratio of both caches when (pos+1)%ratio == 0, then rolling the
 * state), the window-ring write of slot pos % ring_cap, the indexer over the (pos+1)//ratio
 * visible entries, top-k, sparse MQA with the sink and inverse RoPE. Stream-ordered; no host
 * synchronisation, so it can be captured in a CUDA graph.
 */
CSA_API int csa_decode_fused(const csa_decode_args* a, void* stream);

/* Arguments of one HCA decode step (C128A, no index module). */
typedef struct {
  int B;
  int H, d, rope_dim;          /* 128, 512, 64 */
  int ratio;                   /* 128 */
  int window;                  /* 128 */
  float rope_base, eps, scale;
  const int32_t* pos;          /* dev [B] */
  const uint16_t* kv;          /* dev [B, d] */
  const uint16_t* score;       /* dev [B, d] */
  const uint16_t* win_kv;      /* dev [B, d] */
  const uint16_t* q;           /* dev [B, H, d] */
  const float* sink;           /* dev [H] */
  const uint16_t* gamma;       /* dev [d] */
  uint16_t* state_kv;          /* dev [B, ratio, d] in/out */
  uint16_t* state_score;
  uint16_t* cache;
  int64_t cache_bstride;
  int max_entries;
  uint16_t* ring;
  int64_t ring_bstride;
  int ring_cap;
  float* cache_f32;            /* nullable */
  void* out;
  int out_is_f32;
  void* ws;
  size_t ws_bytes;
  void* const* stage_events;   /* nullable: 3 cudaEvent_t recorded before the C128A step, after it and
                                  after attention */
} hca_decode_args;

/* hca_decode_fused -- one HCA decode step ([P5] §3): C128A step, window write, hca_attn. */
CSA_API int hca_decode_fused(const hca_decode_args* a, void* stream);

/*
 * csa_indexer_scores / csa_topk -- the two halves of csa_indexer_topk, for the tensor-parallel
 * indexer ([P1] "少读 KV 之前，Indexer 仍要给历史打分": with the indexer heads split over ranks, the
 * partial scores are summed across ranks before the selection). csa_indexer_scores writes
 * scores[b, i, s] = sum over this call's H_I heads of w[h] * ReLU(q_idx[h,:] . idx_cache[s,:]) for the
 * visible s < E (entries s >= E are not written); its workspace holds only the status word
 * (csa_workspace_size(CSA_WS_SPARSE_ATTN, ...) suffices). csa_topk selects, from caller-provided
 * scores [B, S, max_entries], exactly as csa_indexer_topk does; its workspace:
 * csa_workspace_size(CSA_WS_INDEXER_TOPK, ...) (an upper bound). Arguments, layouts and limits as
 * in csa_indexer_topk; scores must be 16-byte aligned.
 */
CSA_API int csa_indexer_scores(int B, int S, int H_I, int d_I, int ratio, const int32_t* q_pos, const uint16_t* q_idx,
                               const float* w, const uint16_t* idx_cache, int64_t idx_bstride, int max_entries,
                               float* scores, void* ws, size_t ws_bytes, void* stream);
CSA_API int csa_topk(int B, int S, int ratio, int topk, const int32_t* q_pos, const float* scores, int max_entries,
                     int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream);

/*
 * csa_indexer_topk_noalloc -- csa_indexer_topk for callers that cannot allocate device memory (no
 * counterpart in the pages; it is a deployment convenience). Such callers include code running
 * inside another framework's memory pool without access to its allocator, plugins that are handed
 * only the tensors they read and write, and paths that must never call cudaMalloc. Instead of a
 * workspace it uses one fixed scratch array (4 MiB + 256 bytes) that the library defines in device
 * memory; every GPU that loads the library holds it until the process exits. Arguments and
 * results are those of csa_indexer_topk, without scores_opt and ws.
 * Limits: max_entries <= 16384 and B*S*max_entries <= 1,048,576; larger calls return
 * CSA_ERR_UNSUPPORTED without launching. Every argument is checked as csa_indexer_topk checks it
 * before the array is touched, so a refused call writes nothing to the device.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress), so
 * make that first call before any stream capture on that device. Every call shares the array:
 * calls that overlap on the GPU (unordered streams) race. Device-side status (timeouts, bounds) is
 * cleared at the start of each call and is not reported by this entry point.
 */
CSA_API int csa_indexer_topk_noalloc(int B, int S, int H_I, int d_I, int ratio, int topk, const int32_t* q_pos,
                                     const uint16_t* q_idx, const float* w, const uint16_t* idx_cache,
                                     int64_t idx_bstride, int max_entries, int32_t* topk_idx, void* stream);

/*
 * csa_output_projection -- the grouped output projection after the inverse RoPE ([P1] section
 * "输出投影也分组，并且降低中间维度"): the M = B*S output rows o [M, G*Kg] (G groups of 8 heads, Kg = 8*d)
 * are projected per group, r[m, g*R + i] = sum_k o[m, g*Kg + k] * wo_a[g*R + i, k], then
 * y[m, j] = sum_c r[m, c] * wo_b[j, c]. Pro: G = 16, Kg = 4096, R = 1024, D = 7168.
 *   o      dev bf16 [M, G*Kg] (the attention output [B, S, H, d] read as rows of H*d).
 *   wo_a   dev bf16 [G*R, Kg] (Wo_a [G, R, Kg]).   wo_b: dev bf16 [D, G*R].
 *   r      dev bf16 [M, G*R], written (r is rounded to bf16 before the second product).
 *   y      dev float [M, D], written.
 *   ws/ws_bytes: workspace of at least csa_workspace_size(CSA_WS_OUTPUT_PROJ, ...) (status word).
 * Supported: Kg and G*R multiples of 64, R and D multiples of 128, M <= 8,388,480 (65535 tiles of
 * 128 rows). Alignment: every pointer 16 bytes. Contractions run on the tensor cores with fp32
 * accumulation; the order of the fp32 additions differs from a sequential sum.
 * Returns CSA_ERR_INVALID_ARG / CSA_ERR_UNSUPPORTED without launching on bad arguments.
 */
CSA_API int csa_output_projection(int M, int G, int Kg, int R, int D, const uint16_t* o, const uint16_t* wo_a,
                                  const uint16_t* wo_b, uint16_t* r, float* y, void* ws, size_t ws_bytes,
                                  void* stream);

/*
 * csa_linear -- y = x . w^T on the tensor cores (the kernel of the projections around the layer),
 * e.g. the compressor's streams ([P5] §2.1: each token's hidden state [hidden] -> the kv and score
 * states [2*head_dim] of the main stream and [2*d_I] of the index stream).
 *   x dev bf16 [M, K]; w dev bf16 [N, K]; y dev [M, N]: bf16 (y_is_f32 == 0, rounded from the fp32
 *   accumulation) or float.
 *   ws/ws_bytes: workspace of at least csa_workspace_size(CSA_WS_Q_PROJ, ...) (status word).
 * Supported: N a multiple of 128, K a multiple of 64. Alignment: 16 bytes.
 */
CSA_API int csa_linear(int M, int N, int K, const uint16_t* x, const uint16_t* w, void* y, int y_is_f32, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * csa_q_projection -- the low-rank query path in front of the layer ([P1] section "低秩 Q：两次
 * 矩阵乘法接起来"), for M = B*S tokens:
 *   qa = x . wq_a^T                        (fp32, written to the caller's scratch qa)
 *   qr = gamma * qa / sqrt(mean(qa^2) + eps)   (bf16, written)
 *   q  = qr . wq_b^T as [M, H, d], rounded to bf16, then each head divided by
 *        sqrt(mean(q_h^2) + eps) and its last rope_dim dims rotated by pos[m]
 *        (adjacent pairs, theta_i = rope_base^(-2i/rope_dim)); written as bf16.
 *   x      dev bf16 [M, hidden].  wq_a: dev bf16 [q_rank, hidden].  gamma: dev bf16 [q_rank].
 *   wq_b   dev bf16 [H*d, q_rank].  pos: dev int32 [M].
 *   qa     dev float [M, q_rank] scratch.  qr: dev bf16 [M, q_rank].  q: dev bf16 [M, H, d].
 *   ws/ws_bytes: workspace of at least csa_workspace_size(CSA_WS_Q_PROJ, ...) (status word).
 * Supported: d = 512, rope_dim even and <= 128, hidden a multiple of 64, q_rank and H*d multiples
 * of 128. Pro: hidden 7168, q_rank 1536, H 128. Alignment: pointers 16 bytes.
 */
CSA_API int csa_q_projection(int M, int hidden, int q_rank, int H, int d, int rope_dim, float rope_base, float eps,
                             const int32_t* pos, const uint16_t* x, const uint16_t* wq_a, const uint16_t* gamma,
                             const uint16_t* wq_b, float* qa, uint16_t* qr, uint16_t* q, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * csa_window_projection -- the window row of each token ([P5] §2: the KV down-projection
 * [hidden] -> [head_dim], then RoPE on the last rope_dim dims; the pages' quantisation of the
 * other dims is not applied): win[m] = RoPE_pos[m](x[m] . wkv^T), rounded to bf16 before the
 * rotation and stored as bf16.
 *   x dev bf16 [M, hidden]; wkv dev bf16 [d, hidden]; pos dev int32 [M]; win dev bf16 [M, d].
 *   ws/ws_bytes: workspace of at least csa_workspace_size(CSA_WS_Q_PROJ, ...) (status word).
 * Supported: d = 512, rope_dim even and <= 128, hidden a multiple of 64. Alignment: 16 bytes.
 */
CSA_API int csa_window_projection(int M, int hidden, int d, int rope_dim, float rope_base, const int32_t* pos,
                                  const uint16_t* x, const uint16_t* wkv, uint16_t* win, void* ws, size_t ws_bytes,
                                  void* stream);

/*
 * csa_get_device_status -- synchronise `stream`, read the status word in `ws` into *status
 * (CSA_OK, CSA_ERR_TIMEOUT or CSA_ERR_BOUNDS) and clear it. Returns CSA_ERR_CUDA if the
 * stream itself reports an error.
 */
CSA_API int csa_get_device_status(void* ws, void* stream, int* status);

/*
 * csa_watchdog_selftest -- check the failure path of the kernels' bounded waits (no counterpart in
 * the pages; failure detection of the library). Every mbarrier wait inside the kernels gives up after
 * a bounded number of SM cycles (2^30, about half a second), records CSA_ERR_TIMEOUT and the site of
 * the wait in the status word of `ws` and lets its CTA unwind, instead of hanging the GPU. This call
 * enqueues one tiny kernel that runs that same wait on a barrier phase nothing completes, giving up
 * after `limit_cycles` (1 .. 2^30): afterwards csa_get_device_status reports CSA_ERR_TIMEOUT (site
 * 900 in status word 1) and the context stays usable. Only the status word is written.
 *   ws/ws_bytes: any workspace of at least 256 bytes, 256-byte aligned (its status word).
 * Returns CSA_ERR_WORKSPACE / CSA_ERR_INVALID_ARG without launching on bad arguments.
 */
CSA_API int csa_watchdog_selftest(void* ws, size_t ws_bytes, long long limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
