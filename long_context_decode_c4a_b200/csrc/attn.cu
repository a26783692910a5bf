// attn.cu -- sparse MQA with a learned sink and inverse RoPE on the tcgen05 tensor cores (K4, K5).
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", sections "局部和压缩记忆，共用一次归一化" (window rows and the
// selected compressed entries form ONE candidate set with one normalisation; a learned per-head
// sink adds to the denominator and has no value) and "输出投影也分组" (o = inverse_RoPE(o));
// "图解DeepSeek V4：详细计算流程解析" §2 (window KV concatenated with the top-k compressed KV), §2.3 (sink,
// MQA, inverse rotation after MQA), §3 (HCA: no index module, every visible entry).
//
// For query t of request b and head h (one 512-dim row c_j serves as key and value):
//   l_j = scale * q_h . c_j,  m = max(max_j l_j, sink_h),
//   o_h = sum_j e^(l_j - m) c_j / (sum_j e^(l_j - m) + e^(sink_h - m)),  then rotate o_h[448:] by -t.
//
// Layout of the work: a cluster of two CTAs per query; CTA c owns dims [256c, 256c+256). Each CTA
// gathers only its half of every candidate row (an SM gathers scattered rows at a fixed rate, so
// halving the bytes each CTA gathers halves the time this kernel is bound by), computes the
// partial scores S_c = Q[:, half] K[:, half]^T (M = 128 heads, N = 32 candidates per tile,
// K = 256) and sends them to the other CTA through distributed shared memory; both add
// S_0 + S_1 (the same sum in both, fp addition being commutative), run the same online softmax,
// and accumulate O[:, half] += P V[:, half].
//   TMEM (512 columns): [0,128) Q[:, half] as bf16 pairs (A operand of the score TS-MMAs);
//     [128,192) two 32-column partial-score tiles, rewritten once the senders have loaded them;
//     [192,256) two 32-column P tiles (P_hi in columns [0,16), P_lo in [16,32)), the A operand of
//     the PV TS-MMAs; [256,512) O[:, half].
//   SMEM: eight 16 KB stages of 32 half-rows (4 blocks of 64 dims in the 128B-swizzled layout that
//     serves S as a K-major B operand and PV as an MN-major B operand); two 16 KB outgoing and two
//     16 KB incoming exchange buffers (together they first stage Q[:, half] on its way into TMEM);
//     the candidate list. At the end the stages stage the bf16 output rows.
//   Warps: 0..3 build the candidate list and gather half-rows with coalesced 16-byte cp.async,
//     announcing each tile as soon as it lands; 4 and 5 issue the score MMAs of even and odd tiles
//     (one thread issues a tcgen05.mma only every ~50 cycles); 6 issues the PV MMAs in tile order
//     (and owns TMEM); 7..10 load the partial scores of their 32 heads, free the score tile, stage
//     the 4 KB in the outgoing buffer and bulk-copy it into the same quadrant's rows of the other
//     CTA's incoming buffer; 11..14 (even tiles) and 15..18 (odd tiles) add this CTA's staged
//     partial scores and the other CTA's, run the softmax (the running max passes from one group to
//     the other after every tile) and store P. A sender and the softmax warps of the same TMEM lane
//     quadrant trade with the warps of that quadrant in the other CTA, with barriers of their own,
//     so the four quadrants run independently. Warps 7..14 own one head (TMEM lane) per thread and
//     share the epilogue.
// Split-candidate mode (few queries): the pair of work item (query, split) takes one contiguous run
// of the query's tiles and leaves its unnormalised O, max and denominator in the workspace;
// attn_combine_kernel (end of this file) merges the splits.
// Precision: P = P_hi + P_lo with both parts in bf16 (about 16 significant bits), accumulated by two
// PV MMAs; a single bf16 P (8 bits) leaves errors near 1% of the output RMS on short candidate sets.
// Online softmax in the log2 domain; the running max starts at the sink; O is rescaled only when a
// tile raises a row's max by more than 2^8.

#include <math_constants.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace csa {

namespace {

constexpr uint32_t kInvalid = 0x80000000u;    // list entry flag: padding slot (masked)
constexpr uint32_t kFromCache = 0x40000000u;  // list entry flag: row of the compressed cache
constexpr uint32_t kRowMask = 0x3FFFFFFFu;
constexpr int kProducers = 128;               // warps 0..3
constexpr int kQkWarp0 = 4;                   // warps 4, 5: score MMAs of even / odd tiles
constexpr int kPvWarp = 6;                    // PV MMAs; owns TMEM
constexpr int kSendWarp0 = 7;                 // warps 7..10: send partial scores
constexpr int kSoftWarp0 = 11;                // warps 11..14: softmax of even tiles, 15..18 of odd tiles
constexpr int kRoleThreads = 128;
constexpr int kTile = 32;                     // candidates per tile
// Gather stages and exchange buffers (build-time tuning knobs; attn_smem_bytes() reports the shared
// memory they take, which the launch checks).
#ifndef CSA_ATTN_STAGES
#define CSA_ATTN_STAGES 8
#endif
#ifndef CSA_ATTN_XBUFS
#define CSA_ATTN_XBUFS 2
#endif
constexpr int kStages = CSA_ATTN_STAGES;
constexpr int kSBufs = 2;                     // partial-score tiles in TMEM
constexpr uint32_t kStageBytes = 16 * 1024;   // 32 rows x 256 dims of bf16
constexpr uint32_t kBlockBytes = 4096;        // one 64-dim block of a stage: [32 rows][128 B]
constexpr uint32_t kXBytes = 16 * 1024;       // 128 heads x 32 fp32 partial scores
constexpr uint32_t kOutRow = 512 + 16;        // bf16 output staging: 256 dims per head row, padded
constexpr int kXBufs = CSA_ATTN_XBUFS;        // exchange buffers each way
constexpr int kPBufs = 2;                     // P tiles in TMEM

static_assert(kAttnThreads == 32 * (kSoftWarp0 + 8), "warp roles");
static_assert(kAttnMaxCands % kTile == 0, "candidate capacity");
static_assert(kXBufs >= 2, "exchange buffers");
static_assert(kXBufs * 2 * kXBytes >= 64 * 1024, "Q[:, half] is staged over the exchange buffers");

struct AttnSmem {
  uint64_t q_full, q_done, list_ready;
  uint64_t kv_full[kStages], buf_free[kStages];  // buf_free: PV(j) completed, stage j % kStages free
  uint64_t s_full[kSBufs];            // score MMAs of tile j done (score tile j % kSBufs)
  uint64_t s_rd[kSBufs];              // the senders read the partial scores of tile j
  uint64_t p_full[kPBufs];            // P of tile j stored (P tile j % kPBufs)
  uint64_t p_free[kPBufs];            // PV(j) completed: P tile j % kPBufs is free, O holds PV(0..j)
  // Per TMEM lane quadrant q (32 heads): the sender warp of quadrant q stages its 4 KB of each
  // tile in the outgoing buffer and copies it to the same rows of the other CTA's incoming buffer;
  // the softmax warp of quadrant q reads its own 4 KB from the outgoing buffer and the other CTA's
  // from the incoming buffer.
  uint64_t x_full[kXBufs][4];         // incoming 4 KB landed (bulk copy from the other CTA)
  uint64_t x_empty[kXBufs][4];        // the other CTA consumed the 4 KB this warp sent last
  uint64_t x_staged[kXBufs][4];       // this CTA's 4 KB is staged in the outgoing buffer
  uint64_t x_own[kXBufs][4];          // this CTA's softmax warp read its staged 4 KB
  uint64_t hand[2][4];                // softmax group g published the running max after its tile (quadrant q)
  uint64_t b_done;                    // softmax group 1 left its part of the denominator in l_b / m_b
  uint64_t epi;                       // the softmax warps published 1/l
  uint64_t drain[3];
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles;                        // tiles this CTA pair processes
  int tile0;                          // the first of them in the query's candidate list
  int bad;
  int epi_bad;                        // some epilogue warp lacks a complete O
  uint32_t scan[kProducers / 32];
  float rope_cs[kMaxRopePairs][2];
  float inv_l[128];
  float m_hand[4][32];                // running max handed from one softmax group to the other
  float l_b[128], m_b[128];           // softmax group 1's part of the denominator and its max
  uint32_t mask[kAttnMaxCands / kTile];
  uint32_t list[kAttnMaxCands];
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

// 2^x by the MUFU.EX2 unit (ex2.approx: about 2 ulp, 2^-inf = 0); its error is far below the
// ~2^-16 relative precision that the P_hi + P_lo pair keeps.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


// Byte offset of 16-byte chunk k (0..7) of head row h in a 16 KB exchange buffer (rows of 128
// bytes); the XOR spreads a quarter-warp's accesses over all banks.
__device__ __forceinline__ uint32_t xoff(uint32_t h, uint32_t k) { return h * 128u + ((k ^ (h & 7u)) << 4); }

// Exclusive prefix sum over the 128 producer threads (named barrier 2).
__device__ __forceinline__ uint32_t producer_scan(uint32_t v, uint32_t* scan, uint32_t& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) scan[w] = inc;
  named_bar_sync(2, kProducers);
  uint32_t off = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kProducers / 32; ++i) {
    const uint32_t x = scan[i];
    off += (i < w) ? x : 0u;
    tot += x;
  }
  named_bar_sync(2, kProducers);
  total = tot;
  return off + inc - v;
}

// Fine-grained timeline of tile j (debugging builds only): slot 0..15 of word 2000 + 16 j.
__device__ __forceinline__ void trace_tile(uint32_t* status, int j, int slot) {
  if (j < 40) trace_time(status, 2000 + 16 * j + slot);
}

// O[:, half] / l for columns [c0, c0 + 32 nchunks) of this CTA's 256 dims of row h (the global dims
// [256 half + c0, ...)), with the inverse RoPE on the rotated dims. fp32 output is stored to global
// memory directly; bf16 output goes to the staging row `srow` (this CTA's 512 bytes of the output
// row) for one bulk store per row. Warp-collective (TMEM loads).
__device__ __forceinline__ void finish_rows(const AttnParams& P, const AttnSmem& sm, uint32_t o_taddr, int c0, int nchunks,
                                            int half, long long orow, int h, float inv, uint8_t* srow) {
  const int rope0 = P.d - P.rope_dim;  // first rotated dim
#pragma unroll 1
  for (int cc = 0; cc < nchunks; ++cc) {
    const int lc = c0 + 32 * cc;
    uint32_t o[32];
    tmem_ld32(o_taddr + lc, o);
    tmem_wait_ld();
    float y[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) y[c] = __uint_as_float(o[c]) * inv;
    const int col0 = 256 * half + lc;  // global dim of y[0]
    if (col0 + 32 > rope0) {
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const int dim = col0 + c;
        if (dim >= rope0) {
          const int pi = (dim - rope0) >> 1;
          const float cs = sm.rope_cs[pi][0], sn = sm.rope_cs[pi][1];
          const float e = y[c], od = y[c + 1];
          y[c] = e * cs - od * sn;
          y[c + 1] = e * sn + od * cs;
        }
      }
    }
    if (P.out_is_f32) {
      if (h < P.H) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.out) + orow * P.d + col0);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
      }
    } else {
      uint4* dst = reinterpret_cast<uint4*>(srow + 2 * lc);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        dst[c] = make_uint4(pack_bf16(y[8 * c], y[8 * c + 1]), pack_bf16(y[8 * c + 2], y[8 * c + 3]),
                            pack_bf16(y[8 * c + 4], y[8 * c + 5]), pack_bf16(y[8 * c + 6], y[8 * c + 7]));
    }
  }
}

// Split-candidate mode: this CTA's O[:, half] columns [c0, c0 + 32 nchunks) of row h, unnormalised,
// to the partial buffer row `prow` (fp32). Warp-collective (TMEM loads).
__device__ __forceinline__ void store_partial_rows(const AttnParams& P, uint32_t o_taddr, int c0, int nchunks,
                                                   int half, long long prow, int h) {
#pragma unroll 1
  for (int cc = 0; cc < nchunks; ++cc) {
    const int lc = c0 + 32 * cc;
    uint32_t o[32];
    tmem_ld32(o_taddr + lc, o);
    tmem_wait_ld();
    if (h < P.H) {
      float4* dst = reinterpret_cast<float4*>(P.part_o + prow * P.d + 256 * half + lc);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[c] = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]), __uint_as_float(o[4 * c + 2]),
                             __uint_as_float(o[4 * c + 3]));
    }
  }
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage0 = base;                        // stage s at stage0 + s * 16 KB: 4 x [32 rows][128 B]
  uint8_t* xin = base + kStages * kStageBytes;   // kXBufs x 16 KB incoming partial scores
  uint8_t* xout = xin + kXBufs * kXBytes;        // kXBufs x 16 KB outgoing partial scores
  uint8_t* qbuf = xin;                           // first Q[:, half]: 4 x [128 rows][128 B]
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(xout + kXBufs * kXBytes);

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t half = cluster_ctarank();    // which 256 dims this CTA owns
  const uint32_t peer = half ^ 1u;
  const int nq = P.B * P.S;
  const int item = nq * P.splits - 1 - (int)blockIdx.y;  // later queries (more candidates) first
  const int qi = item / P.splits;
  const int sp = item % P.splits;             // which run of the query's tiles (split-candidate mode)
  const int b = qi / P.S;
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t* status = P.status;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_done, 2 * kRoleThreads);
    mbar_init(&sm.list_ready, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.kv_full[i], kProducers);
      mbar_init(&sm.buf_free[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_rd[i], kRoleThreads);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&sm.p_full[i], kRoleThreads);
      mbar_init(&sm.p_free[i], 1);
    }
    for (int i = 0; i < kXBufs; ++i) {
      for (int q = 0; q < 4; ++q) {
        mbar_init(&sm.x_full[i][q], 1);
        mbar_init(&sm.x_empty[i][q], 1);
        mbar_init(&sm.x_staged[i][q], 1);
        mbar_init(&sm.x_own[i][q], 1);
      }
    }
    mbar_init(&sm.epi, kRoleThreads);
    for (int gg = 0; gg < 2; ++gg)
      for (int q = 0; q < 4; ++q) mbar_init(&sm.hand[gg][q], 32);
    mbar_init(&sm.b_done, kRoleThreads);
    for (int i = 0; i < 3; ++i) mbar_init(&sm.drain[i], 1);
    sm.abort_flag = 0;
    sm.bad = 0;
    sm.epi_bad = 0;
    fence_mbar_init();
  }
  if (warp == kPvWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();   // the barriers of both CTAs are initialised before any remote access
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  timeline_mark(P.status, kTlAttn, kTlEntry);
  // With early_window the producers wait for the previous launch only before they read the
  // selection (below); every other warp waits here.
  const bool early = P.early_window != 0;
  if (!early || warp >= kProducers / 32) {
    pdl_wait();
    pdl_trigger();
  }
  if (!early) timeline_mark(P.status, kTlAttn, kTlReady);
  const int t = P.q_pos[qi];
  if (threadIdx.x == 0) trace_time(status, 0);

  if (warp < kProducers / 32) {
    // ------------------------------------------------------------ Q load, candidate list, gathers
    const int pt = threadIdx.x;  // 0..127
    if (pt == 0) {
      const int row0 = qi * P.H;
      mbar_arrive_expect_tx(&sm.q_full, 4u * 16384u);
      for (int k = 0; k < 4; ++k) tma_load_2d(qbuf + k * 16384, &map_q, 256 * (int)half + 64 * k, row0, &sm.q_full);
    }
    // Candidate list: window rows, then the compressed entries, padded to tiles of 32.
    const long long ring_row0 = (long long)b * P.ring_rows;
    const long long cache_row0 = (long long)b * P.cache_rows;
    const int p0 = max(0, t - P.window + 1);
    const int nwin = t - p0 + 1;
    const uint32_t self_slot = (uint32_t)(ring_row0 + (t % P.ring_cap)) & kRowMask;
    for (int k = pt; k < nwin; k += kProducers)
      sm.list[k] = (uint32_t)(ring_row0 + (long long)((p0 + k) % P.ring_cap)) & kRowMask;
    // Gather of tile `tile` into stage tile % kStages: this CTA's 512 bytes of each of its 32 rows.
    // Thread pt copies the 16-byte chunks pt, pt+128, ... of the tile (32 rows x 32 chunks): a warp
    // covers the 512 contiguous bytes of one row per instruction.
    const char* ring_base = reinterpret_cast<const char*>(P.ring) + 512 * half;
    const char* cache_base = reinterpret_cast<const char*>(P.cache) + 512 * half;
    int tile0 = 0;  // local tile `tile` is tile tile0 + tile of the query's list
    auto issue = [&](int tile) {
      const uint32_t st = smem_u32(stage0 + (size_t)(tile % kStages) * kStageBytes);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = pt + kProducers * i;  // chunk of the tile
        const int r = c >> 5;               // candidate row 0..31
        const int w = c & 31;               // chunk within the half-row
        const uint32_t e = sm.list[(tile0 + tile) * kTile + r];
        const char* src = ((e & kFromCache) ? cache_base : ring_base) + (size_t)(e & kRowMask) * 1024 + w * 16;
        cp_async_16(st + (w >> 3) * kBlockBytes + sw128_offset(r, w & 7), src);
      }
      cp_async_arrive_noinc(&sm.kv_full[tile % kStages]);
    };
    // Tiles made only of window rows are known now: their gathers start before the compressed
    // entries are read (one pair per query: its tiles start at the window).
    named_bar_sync(2, kProducers);
    const int w_tiles = P.splits == 1 ? min(nwin / kTile, kStages) : 0;
    for (int tile = 0; tile < w_tiles; ++tile) issue(tile);
    if (early) {
      pdl_wait();   // the selection comes from the previous launch
      pdl_trigger();
      timeline_mark(P.status, kTlAttn, kTlReady);
    }
    const int ecap = min((t + 1) / P.ratio, P.max_entries);
    int n = nwin;
    bool bad = false;
    if (P.topk_idx != nullptr) {
      // Each thread takes a contiguous run of the (ascending) selection; runs are compacted in order.
      const int32_t* sel = P.topk_idx + (long long)qi * P.topk;
      const int per = (P.topk + kProducers - 1) / kProducers;
      const int lo = min(P.topk, pt * per), hi = min(P.topk, lo + per);
      int vals[kAttnMaxTopk / kProducers];
      uint32_t cnt = 0;
#pragma unroll
      for (int u = 0; u < kAttnMaxTopk / kProducers; ++u) {
        const int j = lo + u;
        const int s = (u < per && j < hi) ? sel[j] : -1;
        vals[u] = s;
        const bool ok = s >= 0 && s < ecap;
        bad |= s >= ecap;
        cnt += ok ? 1u : 0u;
      }
      uint32_t total;
      uint32_t pos = (uint32_t)n + producer_scan(cnt, sm.scan, total);
#pragma unroll
      for (int u = 0; u < kAttnMaxTopk / kProducers; ++u) {
        const int s = vals[u];
        if (s >= 0 && s < ecap) sm.list[pos++] = ((uint32_t)(cache_row0 + s) & kRowMask) | kFromCache;
      }
      n += (int)total;
    } else {
      int cnt = ecap;
      if (cnt > kAttnMaxCompressed) {
        bad = true;
        cnt = kAttnMaxCompressed;
      }
      for (int k = pt; k < cnt; k += kProducers) sm.list[n + k] = ((uint32_t)(cache_row0 + k) & kRowMask) | kFromCache;
      n += cnt;
    }
    if (bad) sm.bad = 1;
    const int nt = (n + kTile - 1) & ~(kTile - 1);
    for (int k = n + pt; k < nt; k += kProducers) sm.list[k] = self_slot | kInvalid;
    const int Jq = nt / kTile;  // the query's tiles
    // Entries [0, n) are valid, [n, nt) padding.
    for (int j = pt; j < Jq; j += kProducers) {
      const int rem = n - j * kTile;
      sm.mask[j] = rem >= kTile ? 0xFFFFFFFFu : (rem > 0 ? (1u << rem) - 1u : 0u);
    }
    // This pair's run of them: tiles [Jq*sp/splits, Jq*(sp+1)/splits).
    tile0 = (int)(((long long)Jq * sp) / P.splits);
    const int J = (int)(((long long)Jq * (sp + 1)) / P.splits) - tile0;
    if (pt == 0) {
      sm.n_tiles = J;
      sm.tile0 = tile0;
    }
    named_bar_sync(2, kProducers);
    if (pt == 0) {
      if (sm.bad && half == 0) record_status(status, CSA_DEV_BOUNDS);
      mbar_arrive(&sm.list_ready);
      trace_time(status, 1);
    }

    // Gathers: tile j -> stage j % kStages, issued in order as soon as the stage is free (PV of tile
    // j - kStages completed). Each thread's copies arrive on kv_full by themselves when they land
    // (cp.async.mbarrier.arrive), so issuing never waits for a tile in flight; the consumers order
    // the landed bytes before their tensor-core reads with a proxy fence.
    for (int next = w_tiles; next < J; ++next) {
      if (next >= kStages &&
          !mbar_wait(&sm.buf_free[next % kStages], (uint32_t)((next / kStages - 1) & 1), abort_flag, status, 102))
        break;
      issue(next);
      if (pt == 0 && next < 60) trace_time(status, 2 + next);
    }
    cp_async_wait_all();  // after an abort: let the copies land before teardown
  } else if (warp < kPvWarp) {
    // ------------------------------------------------------------ score MMAs: tiles j = w, w+2, ...
    if (lane == 0) {
      const int w = warp - kQkWarp0;  // 0: even tiles, 1: odd tiles
      bool ok = mbar_wait(&sm.q_done, 0, abort_flag, status, 112) &&
                mbar_wait(&sm.list_ready, 0, abort_flag, status, 113);
      const int J = ok ? sm.n_tiles : 0;
      const uint32_t idesc_qk = idesc_bf16_f32(128, kTile, 0, 0);
      for (int j = w; j < J; j += 2) {
        const int s = j % kStages, sb = j % kSBufs;
        // Score tile sb is rewritten only once the senders have loaded tile j - kSBufs.
        if (j >= kSBufs && !mbar_wait(&sm.s_rd[sb], (uint32_t)((j / kSBufs - 1) & 1), abort_flag, status, 117))
          break;
        trace_tile(status, j, 0);
        if (!mbar_wait(&sm.kv_full[s], (uint32_t)((j / kStages) & 1), abort_flag, status, 114)) break;
        fence_proxy_async_smem();  // the gathered rows (written by cp.async) before the MMAs read them
        tc_fence_after();
        if (j < 60) trace_time(status, 64 + j);
        const uint32_t kbase = smem_u32(stage0 + (size_t)s * kStageBytes);
        const uint32_t d_s = tmem + 128 + kTile * sb;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {  // this CTA's 256 dims: A = Q[:, half] from TMEM
          const uint64_t bdesc = smem_desc_sw128(kbase + (ks >> 2) * kBlockBytes + (ks & 3) * 32, 16, 1024);
          mma_ts(d_s, tmem + 8 * ks, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[sb]);
        trace_tile(status, j, 2);
      }
      // Every MMA issued above completes on its own; wait for them before TMEM is released.
      mma_commit(&sm.drain[w]);
      mbar_wait_drain(&sm.drain[w], 0, status, 116);
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ PV MMAs, in tile order
    if (lane == 0) {
      bool ok = mbar_wait(&sm.list_ready, 0, abort_flag, status, 118);
      const int J = ok ? sm.n_tiles : 0;
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      for (int j = 0; j < J; ++j) {
        const int pb = j % kPBufs;
        if (!mbar_wait(&sm.p_full[pb], (uint32_t)((j / kPBufs) & 1), abort_flag, status, 115)) break;
        trace_tile(status, j, 3);
        fence_proxy_async_smem();  // the gathered rows of the tile before the MMAs read them
        tc_fence_after();
        const uint32_t vbase = smem_u32(stage0 + (size_t)(j % kStages) * kStageBytes);
        const uint32_t pcol = tmem + 128 + kTile * (kSBufs + pb);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // P_hi (columns 0..15 of the P tile), then P_lo (16..31)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t bdesc = smem_desc_sw128(vbase + ks * 2048, kBlockBytes, 1024);
            mma_ts(tmem + 256, pcol + 16 * part + 8 * ks, bdesc, idesc_pv, (j > 0 || part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&sm.buf_free[j % kStages]);
        mma_commit(&sm.p_free[pb]);
        if (j < 60) trace_time(status, 192 + j);
      }
      mma_commit(&sm.drain[2]);
      mbar_wait_drain(&sm.drain[2], 0, status, 119);
    }
  } else {
    // ------------------------------------------------------------ senders (7..10), softmax (11..14)
    const bool sender = warp < kSoftWarp0;
    const bool softB = warp >= kSoftWarp0 + 4;  // second softmax group (odd tiles)
    const int quad = warp & 3;             // TMEM lane quadrant
    const int h = quad * 32 + lane;        // head = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int rt = threadIdx.x - (sender ? kSendWarp0 : (softB ? kSoftWarp0 + 4 : kSoftWarp0)) * 32;  // 0..127 within the role
    // Q[:, half] -> TMEM columns [0, 128): blocks 0-1 by the senders, 2-3 by the softmax warps.
    bool ok = softB || __all_sync(0xffffffffu, mbar_wait(&sm.q_full, 0, abort_flag, status, 121));
    if (ok && !softB) {
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = (sender ? 0 : 2) + kk;
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(qbuf + kb * 16384 + sw128_offset(h, ch));
          r[4 * ch + 0] = v.x;
          r[4 * ch + 1] = v.y;
          r[4 * ch + 2] = v.z;
          r[4 * ch + 3] = v.w;
        }
        tmem_st32(tmem + lane_addr + 32 * kb, r);
      }
      tmem_wait_st();
    }
    if (!softB) {
      tc_fence_before();
      mbar_arrive(&sm.q_done);
    }
    // Inverse-RoPE table for position t.
    const int npairs = P.rope_dim / 2;
    if (!sender && !softB && rt < npairs) {
      float cs, sn;
      rope_cos_sin(t, P.inv_freq[rt], &cs, &sn);
      sm.rope_cs[rt][0] = cs;
      sm.rope_cs[rt][1] = -sn;
    }
    if (!softB) named_bar_sync(1, 2 * kRoleThreads);   // the Q staging area is no longer read
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&sm.list_ready, 0, abort_flag, status, 122));
    const int J = ok ? sm.n_tiles : 0;
    // Tile j travels through exchange buffer c = j % kXBufs; phase (j / kXBufs) & 1 of x_full /
    // x_empty [c][quad] belongs to it. The sender and softmax warps of quadrant quad own the 4 KB
    // of its 32 heads (rows [32 quad, 32 quad + 32) of every exchange buffer) and trade them with
    // the warps of the same quadrant in the other CTA.
    const uint32_t qoff = (uint32_t)quad * (kXBytes / 4);
    const uint32_t xempty_peer = mapa_shared(smem_u32(&sm.x_empty[0][quad]), peer);
    int j = 0;
    if (sender) {
      const uint32_t xin_peer = mapa_shared(smem_u32(xin), peer) + qoff;
      const uint32_t xfull_peer = mapa_shared(smem_u32(&sm.x_full[0][quad]), peer);
      for (; j < J; ++j) {
        const int c = j % kXBufs, sb = j % kSBufs;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (uint32_t)((j / kSBufs) & 1), abort_flag, status, 123)))
          break;
        if (rt == 0) trace_tile(status, j, 5);
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(tmem + lane_addr + 128 + kTile * sb, v);
        tmem_wait_ld();
        if (rt == 0) trace_tile(status, j, 6);
        // The partial scores are read: the score MMAs of tile j + kSBufs may overwrite them.
        tc_fence_before();
        mbar_arrive(&sm.s_rd[sb]);
        // The other CTA consumed tile j - kXBufs (its incoming buffer c and this CTA's outgoing
        // buffer c, read by that copy, are free), and this CTA's softmax warp read it too.
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(&sm.x_empty[c][quad], (uint32_t)((j / kXBufs) & 1), abort_flag,
                                                        status, 126)))
          break;
        if (rt == 0) trace_tile(status, j, 7);
        if (j >= kXBufs &&
            !__all_sync(0xffffffffu, mbar_wait(&sm.x_own[c][quad], (uint32_t)((j / kXBufs - 1) & 1), abort_flag, status, 130)))
          break;
        uint8_t* xo = xout + c * kXBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(xo + xoff(h, i)) = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.x_staged[c][quad]);
          bulk_copy_to_cluster(xin_peer + c * kXBytes, smem_u32(xo) + qoff, kXBytes / 4, xfull_peer + 32 * c);
          if (rt == 0 && j < 60) trace_time(status, 300 + j);
        }
      }
    } else {
      // Softmax warps: group 0 (warps 11..14) takes the even tiles, group 1 (warps 15..18) the odd
      // ones; each owns the 32 heads of its quadrant. The running max passes from the group that
      // finished tile j - 1 to the one taking tile j through hand[group][quad] (one mbarrier phase
      // per tile, 32 arrivals: the publishing warp's lanes).
      const int g = softB ? 1 : 0;
      if (!softB && lane == 0)
        for (int c = 0; c < kXBufs; ++c) {  // every incoming buffer is free: arm them, let the other CTA send
          mbar_arrive_expect_tx(&sm.x_full[c][quad], kXBytes / 4);
          mbar_arrive_remote_relaxed(xempty_peer + 32 * c);
        }
      const float sl = (h < P.H) ? P.sink[h] * 1.4426950408889634f : 0.f;
      float m_used = sl;         // running max in log2 units (starts at the sink), as this group last saw it
      float l = (softB || sp > 0) ? 0.f : 1.f;  // this group's part of the denominator, relative to m_used;
                                 // group 0 of the first (or only) split holds the sink's exp2(sl - m_used) = 1
      const int tile0 = sm.tile0;
      // p_free[i % 2] completes once per PV(i): p_free[g] counts the PVs of group g's tiles. A parity
      // wait for PV(i) is unambiguous while the barrier's previous phase (PV(i - 2)) has completed and
      // its next one (PV(i + 2)) cannot have. Each group therefore waits only for: PV(j - 2) of its
      // own previous tile before storing P of tile j (it waited for PV(j - 4) before storing P(j - 2);
      // PV(j) is not issued yet); before a rescale, that one and then PV(j - 1) of the other group
      // (PV completions are in issue order, so PV(j - 3) is done once PV(j - 2) is, and PV(j + 1)
      // waits for the running max this group has not published yet); group 0 waits for the last PVs
      // before the epilogue the same way.
      static_assert(kPBufs == 2, "P tile j is stored once PV(j - 2) completed");
      auto wait_pv = [&](int i) -> bool {
        return i < 0 || __all_sync(0xffffffffu, mbar_wait(&sm.p_free[i % kPBufs], (uint32_t)((i / kPBufs) & 1),
                                                           abort_flag, status, 124));
      };
      bool done = true;
      for (j = g; j < J; j += 2) {
        const int c = j % kXBufs;
        // This CTA's partial scores of the tile (staged by the sender) and the other CTA's.
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.x_staged[c][quad], (uint32_t)((j / kXBufs) & 1), abort_flag, status, 128))) {
          done = false;
          break;
        }
        if (rt == 0) trace_tile(status, j, 10);
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.x_full[c][quad], (uint32_t)((j / kXBufs) & 1), abort_flag, status, 127))) {
          done = false;
          break;
        }
        if (rt == 0 && j < 60) trace_time(status, 400 + j);
        // S = S_0 + S_1 (the same sum in both CTAs), scaled to log2 units; padding -> -inf.
        const uint8_t* xi = xin + c * kXBytes;
        const uint8_t* xm = xout + c * kXBytes;
        const uint32_t mk = sm.mask[tile0 + j];
        float x[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 o = *reinterpret_cast<const uint4*>(xi + xoff(h, i));
          const uint4 m = *reinterpret_cast<const uint4*>(xm + xoff(h, i));
          const float ov[4] = {__uint_as_float(o.x), __uint_as_float(o.y), __uint_as_float(o.z), __uint_as_float(o.w)};
          const float mv[4] = {__uint_as_float(m.x), __uint_as_float(m.y), __uint_as_float(m.z), __uint_as_float(m.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int cc = 4 * i + e;
            const float sc = (mv[e] + ov[e]) * P.scale_log2;
            x[cc] = ((mk >> cc) & 1u) ? sc : -CUDART_INF_F;
          }
        }
        float mt;
        {
          float r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = fmaxf(x[e], x[e + 16]);
#pragma unroll
          for (int w = 8; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) r[e] = fmaxf(r[e], r[e + w]);
          mt = r[0];
        }
        // mt depends on every value the warp loaded from the buffers (and a warp's loads complete
        // together), so once it is formed the incoming buffer can be armed for tile j + kXBufs and
        // released to the other CTA, and the outgoing one to the sender.
        asm volatile("" ::"f"(mt) : "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.x_full[c][quad], kXBytes / 4);
          mbar_arrive_remote_relaxed(xempty_peer + 32 * c);
          mbar_arrive(&sm.x_own[c][quad]);
        }
        if (rt == 0 && j < 60) trace_time(status, 500 + j);
        // The running max after tile j - 1, from the other group (it only grows: this group's part
        // of the denominator follows it).
        if (j > 0) {
          const int pj = j - 1;  // published by group 1 - g as its (pj / 2)-th tile
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.hand[1 - g][quad], (uint32_t)((pj / 2) & 1), abort_flag, status,
                                                 131))) {
            done = false;
            break;
          }
          const float mp = sm.m_hand[quad][lane];
          if (mp != m_used) {
            l *= exp2f(m_used - mp);
            m_used = mp;
          }
        }
        // Lazy rescale: only when this tile raises the row max by more than 2^8. The TMEM accesses
        // are warp-collective, so the whole warp takes the branch if any lane needs it (lanes that do
        // not need it scale by 1).
        if (rt == 0) trace_tile(status, j, 12);
        const bool need = mt > m_used + 8.f;
        const float alpha = need ? exp2f(m_used - mt) : 1.f;
        if (__any_sync(0xffffffffu, need)) {
          if (j > 0) {
            // O holds PV(0..j-1): wait for PV(j-1), then scale the rows of this warp.
            if (!wait_pv(j - 2) || !wait_pv(j - 1)) {
              done = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
              uint32_t o[32];
              const uint32_t oa = tmem + lane_addr + 256 + 32 * cc;
              tmem_ld32(oa, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(oa, o);
            }
            tmem_wait_st();
            tc_fence_before();
          }
          if (need) {
            l *= alpha;
            m_used = mt;
          }
        }
        // Publish the running max for tile j + 1 (taken by the other group).
        if (j + 1 < J) {
          sm.m_hand[quad][lane] = m_used;
          mbar_arrive(&sm.hand[g][quad]);
        }
        // P = P_hi + P_lo, both bf16, in P tile j % kPBufs: P_hi in columns [0,16), P_lo in
        // [16,32). P_hi is p truncated to bf16 (the high half of its bits); P_lo = p - P_hi is exact
        // in fp32 and is rounded to bf16, so P_hi + P_lo is within 2^-16 of p relative.
        uint32_t phi[16], plo[16];
        float ps[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float p0 = ex2_approx(x[2 * q] - m_used);
          const float p1 = ex2_approx(x[2 * q + 1] - m_used);
          const uint32_t u0 = __float_as_uint(p0), u1 = __float_as_uint(p1);
          phi[q] = __byte_perm(u0, u1, 0x7632);
          plo[q] = pack_bf16(p0 - __uint_as_float(u0 & 0xFFFF0000u), p1 - __uint_as_float(u1 & 0xFFFF0000u));
          ps[q] = p0 + p1;
        }
#pragma unroll
        for (int w = 8; w > 0; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) ps[e] += ps[e + w];
        l += ps[0];
        // P tile j % kPBufs was read by PV(j - kPBufs).
        if (rt == 0) trace_tile(status, j, 13);
        if (!wait_pv(j - 2)) {
          done = false;
          break;
        }
        if (rt == 0) trace_tile(status, j, 14);
        tc_fence_after();
        const uint32_t pa = tmem + lane_addr + 128 + kTile * (kSBufs + j % kPBufs);
        tmem_st16(pa, phi);
        tmem_st16(pa + 16, plo);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[j % kPBufs]);
        if (lane == 0 && j < 40) trace_time(status, 3000 + 4 * j + quad);
        if (rt == 0 && j < 60) trace_time(status, 128 + j);
      }
      if (softB) {
        // Group 1 hands its part of the denominator (and the max it is relative to) to group 0.
        sm.l_b[h] = l;
        sm.m_b[h] = m_used;
        mbar_arrive(&sm.b_done);
        j = done ? J : -1;
      } else {
        // Every PV completed: this group's last one, then (when the last tile was group 1's) PV(J - 1).
        const int last0 = ((J - 1) & ~1);
        if (done && J > 0 && (!wait_pv(last0) || !wait_pv(J - 1))) done = false;
        if (done && !__all_sync(0xffffffffu, mbar_wait(&sm.b_done, 0, abort_flag, status, 132))) done = false;
        float m_fin = m_used;
        if (done) {
          const float lb = sm.l_b[h], mb = sm.m_b[h];
          const float mf = fmaxf(m_used, mb);  // the last published max (it only grows): O's reference
          l = (l != 0.f ? l * exp2f(m_used - mf) : 0.f) + (lb != 0.f ? lb * exp2f(mb - mf) : 0.f);
          m_fin = mf;
        }
        sm.inv_l[h] = 1.f / l;
        if (P.splits > 1 && half == 0 && h < P.H) {
          const long long r = (long long)item * 2 * P.H + h;
          P.part_ml[r] = m_fin;
          P.part_ml[r + P.H] = l;
        }
        j = done ? J : -1;
      }
    }
    // Epilogue: O / l, inverse RoPE on the rotated dims, store. The softmax warps of group 0 take O
    // columns [0, 128) of their rows, the senders [128, 256); group 1 has finished.
    if (!softB) {
    bool fin;
    if (sender) {
      fin = __all_sync(0xffffffffu, j == J && J > 0 && mbar_wait(&sm.epi, 0, abort_flag, status, 125));
    } else {
      fin = __all_sync(0xffffffffu, j == J && J > 0);  // every PV observed complete
      mbar_arrive(&sm.epi);
    }
    if (!fin && lane == 0) sm.epi_bad = 1;
    uint8_t* srow = stage0 + (size_t)h * kOutRow;  // every gather and MMA reading the stages completed
    if (fin) {
      tc_fence_after();
      if (P.splits > 1)
        store_partial_rows(P, tmem + lane_addr + 256, sender ? 128 : 0, 4, (int)half, (long long)item * P.H + h, h);
      else
        finish_rows(P, sm, tmem + lane_addr + 256, sender ? 128 : 0, 4, (int)half, (long long)qi * P.H + h, h,
                    sm.inv_l[h], srow);
    } else if (P.splits > 1 && J == 0 && j == 0 && h < P.H) {
      // A split whose run of tiles is empty (the query has fewer tiles than splits): O = 0; its max
      // and denominator (the sink's term for split 0, nothing otherwise) were stored above.
      float4* dst = reinterpret_cast<float4*>(P.part_o + ((long long)item * P.H + h) * P.d + 256 * half + (sender ? 128 : 0));
#pragma unroll 4
      for (int c = 0; c < 32; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (!P.out_is_f32 && P.splits == 1) {
      // bf16: each head row's 512 bytes leave in one bulk store, once both roles staged their halves.
      fence_proxy_async_smem();
      named_bar_sync(1, kRoleThreads + kRoleThreads);
      if (!sender && h < P.H && !sm.epi_bad) {
        bulk_store_global(static_cast<uint16_t*>(P.out) + ((long long)qi * P.H + h) * P.d + 256 * half, smem_u32(srow), 512);
        bulk_commit();
        bulk_wait_read_all();
      }
    }
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();   // no remote access into this CTA's shared memory after this point
  tc_fence_after();
  if (threadIdx.x == 0) trace_time(status, 255);
  if (warp == kPvWarp) tmem_dealloc(tmem, 512);
  timeline_mark(P.status, kTlAttn, kTlExit);
}

// Merge of the split-candidate partials of one (query, head) row: with M = max_s m_s and
// w_s = 2^(m_s - M), o = sum_s w_s O_s / sum_s w_s l_s (the sink is in l_0), then the inverse RoPE
// of the last rope_dim dims at position t. grid (H, queries); thread i owns dims [4i, 4i + 4).
__global__ void __launch_bounds__(kAttnCombineThreads) attn_combine_kernel(AttnCombineParams P) {
  timeline_mark(P.status, kTlCombine, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlCombine, kTlReady);
  const int h = blockIdx.x, qi = blockIdx.y, dim = 4 * threadIdx.x;
  const int ns = P.splits;
  const long long item0 = (long long)qi * ns;
  // Every split's max and denominator first (independent loads), then the partials four at a time,
  // so the loads of a thread are in flight together rather than one latency each.
  float ms[kAttnMaxSplits], ls[kAttnMaxSplits];
  float M = -CUDART_INF_F;
#pragma unroll
  for (int s = 0; s < kAttnMaxSplits; ++s) {
    if (s < ns) {
      const long long r = (item0 + s) * 2 * P.H + h;
      ms[s] = P.part_ml[r];
      ls[s] = P.part_ml[r + P.H];
      M = fmaxf(M, ms[s]);
    }
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* po = P.part_o + (item0 * P.H + h) * P.d + dim;
  const long long stride = (long long)P.H * P.d;  // from one split's row to the next's
#pragma unroll
  for (int s0 = 0; s0 < kAttnMaxSplits; s0 += 4) {
    if (s0 >= ns) break;
    float4 o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < ns) o[u] = *reinterpret_cast<const float4*>(po + (s0 + u) * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + u;
      if (s < ns) {
        const float w = ms[s] == -CUDART_INF_F ? 0.f : exp2f(ms[s] - M);
        L += w * ls[s];
        acc.x += w * o[u].x;
        acc.y += w * o[u].y;
        acc.z += w * o[u].z;
        acc.w += w * o[u].w;
      }
    }
  }
  const float inv = 1.f / L;
  float y[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  const int rope0 = P.d - P.rope_dim;
  if (dim >= rope0) {
    const int t = P.q_pos[qi];
#pragma unroll
    for (int c = 0; c < 4; c += 2) {
      float cs, sn;
      rope_cos_sin(t, P.inv_freq[(dim + c - rope0) >> 1], &cs, &sn);
      const float e = y[c], od = y[c + 1];
      y[c] = e * cs + od * sn;   // rotation by -t
      y[c + 1] = od * cs - e * sn;
    }
  }
  const long long orow = (long long)qi * P.H + h;
  if (P.out_is_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(P.out) + orow * P.d + dim) = make_float4(y[0], y[1], y[2], y[3]);
  } else {
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(P.out) + orow * P.d + dim) =
        make_uint2(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]));
  }
  timeline_mark(P.status, kTlCombine, kTlExit);
}

size_t attn_smem_bytes() { return 1024 + kStages * kStageBytes + 2 * kXBufs * (size_t)kXBytes + sizeof(AttnSmem); }

}  // namespace csa
