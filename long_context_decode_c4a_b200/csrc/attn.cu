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
// Layout of the work: two CTAs per query; CTA c accumulates dims [256c, 256c+256) of O. Both
// gather the full candidate rows (the second read of a row is served by L2) and compute the full
// scores S = Q K^T (M = 128 heads, N = 32 candidates per tile, K = 512), so they need no
// communication: each runs the same online softmax on its own copy of S. TMEM's 512 columns hold
// Q[:, 0:256] as bf16 pairs (the A operand of the TS-MMA for dims 0..255; dims 256..511 come from
// shared memory), four 32-column score tiles, and O[:, half] (256 columns). With four score
// tiles the MMA warp runs up to four tiles ahead of the softmax.
//   SMEM: Q[:, 256:512] (64 KB, 128B-swizzled K-major, TMA); four 32 KB stages of 32 candidate
//     rows (8 blocks of 64 dims in the 128B-swizzled layout that serves S as a K-major B operand
//     and PV as an MN-major B operand; Q[:, 0:256] passes through stages 2-3 on its way into
//     TMEM); the candidate list.
//   Warps: 0..3 build the candidate list and gather rows with coalesced 16-byte cp.async (then
//     share the epilogue); 4 and 5 issue the score MMAs of even and odd tiles (one thread issues a
//     tcgen05.mma only every ~50 cycles, so two issuers keep the tensor pipe fed); 6 issues the PV
//     MMAs in tile order (and owns TMEM); 7..10 run the softmax (thread = head = TMEM lane) and the
//     epilogue.
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
constexpr int kSoftWarp0 = 7;                 // warps 7..10
constexpr int kSoftThreads = 128;
constexpr int kTile = 32;                     // candidates per tile
constexpr int kStages = 4;
constexpr int kSBufs = 4;                     // score tiles in TMEM
constexpr size_t kQhiBytes = 64 * 1024;       // Q[:, 256:512]
constexpr size_t kStageBytes = 32 * 1024;     // 32 rows x 512 dims of bf16
constexpr uint32_t kBlockBytes = 4096;        // one 64-dim block of a stage: [32 rows][128 B]

static_assert(kAttnThreads == 32 * (kSoftWarp0 + 4), "warp roles");
static_assert(kAttnMaxCands % kTile == 0, "candidate capacity");

static_assert(kStages == kSBufs, "tile j uses stage and score tile j % kStages");

struct AttnSmem {
  uint64_t q_full, q_done, list_ready;
  uint64_t kv_full[kStages];
  uint64_t buf_free[kStages];         // PV(j) completed: stage and score tile j % kStages are free
  uint64_t s_full[kSBufs], p_full[kSBufs], o_done[2];
  uint64_t epi;                       // the softmax warps published 1/l
  uint64_t drain[3];
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles;
  int bad;
  uint32_t scan[kProducers / 32];
  float rope_cs[kMaxRopePairs][2];
  float inv_l[128];
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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

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

// O[:, half] / l for 128 of this CTA's 256 dims of row h (columns [c0, c0+128) of its O), the
// inverse RoPE on the rotated dims, and the store. Warp-collective (TMEM loads).
__device__ __forceinline__ void store_rows(const AttnParams& P, const AttnSmem& sm, uint32_t o_taddr, int c0,
                                           int half, long long orow, int h, float inv) {
  const int rope0 = P.d - P.rope_dim;  // first rotated dim
#pragma unroll 1
  for (int cc = 0; cc < 4; ++cc) {
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
    if (h < P.H) {
      if (P.out_is_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.out) + orow * P.d + col0);
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.out) + orow * P.d + col0);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          dst[c] = make_uint4(pack_bf16(y[8 * c], y[8 * c + 1]), pack_bf16(y[8 * c + 2], y[8 * c + 3]),
                              pack_bf16(y[8 * c + 4], y[8 * c + 5]), pack_bf16(y[8 * c + 6], y[8 * c + 7]));
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_hi = base;                       // 4 x [128 rows][128 B]
  uint8_t* stage0 = base + kQhiBytes;         // stage s at stage0 + s * 32 KB: 8 x [32 rows][128 B]
  uint8_t* q_lo = stage0 + 2 * kStageBytes;   // Q[:, 0:256] staging over stages 2-3: 4 x [128 rows][128 B]
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(stage0 + kStages * kStageBytes);

  const int warp = warp_id();
  const int lane = lane_id();
  const int half = blockIdx.x;                // which 256 dims of O this CTA owns
  const int nq = P.B * P.S;
  const int qi = nq - 1 - (int)blockIdx.y;    // later queries (more candidates) first
  const int b = qi / P.S;
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t* status = P.status;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_done, kSoftThreads);
    mbar_init(&sm.list_ready, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.kv_full[i], kProducers);
      mbar_init(&sm.buf_free[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], kSoftThreads);
    }
    mbar_init(&sm.o_done[0], 1);
    mbar_init(&sm.o_done[1], 1);
    mbar_init(&sm.epi, kSoftThreads);
    for (int i = 0; i < 3; ++i) mbar_init(&sm.drain[i], 1);
    sm.abort_flag = 0;
    sm.bad = 0;
    fence_mbar_init();
  }
  if (warp == kPvWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  pdl_trigger();
  const int t = P.q_pos[qi];
  if (threadIdx.x == 0) trace_time(status, 0);

  if (warp < kProducers / 32) {
    // ------------------------------------------------------------ Q loads, candidate list, gathers
    const int pt = threadIdx.x;  // 0..127
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    if (pt == 0) {
      const int row0 = qi * P.H;
      mbar_arrive_expect_tx(&sm.q_full, 8u * 16384u);
      for (int k = 0; k < 4; ++k) tma_load_2d(q_hi + k * 16384, &map_q, 256 + 64 * k, row0, &sm.q_full);
      for (int k = 0; k < 4; ++k) tma_load_2d(q_lo + k * 16384, &map_q, 64 * k, row0, &sm.q_full);
    }
    // Candidate list: window rows, then the compressed entries, padded to tiles of 32.
    const long long ring_row0 = (long long)b * P.ring_rows;
    const long long cache_row0 = (long long)b * P.cache_rows;
    const int p0 = max(0, t - P.window + 1);
    const int nwin = t - p0 + 1;
    const uint32_t self_slot = (uint32_t)(ring_row0 + (t % P.ring_cap)) & kRowMask;
    for (int k = pt; k < nwin; k += kProducers)
      sm.list[k] = (uint32_t)(ring_row0 + (long long)((p0 + k) % P.ring_cap)) & kRowMask;
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
    const int J = nt / kTile;
    named_bar_sync(2, kProducers);
    for (int j = pt; j < J; j += kProducers) {
      uint32_t mk = 0;
      for (int c = 0; c < kTile; ++c)
        if (!(sm.list[j * kTile + c] & kInvalid)) mk |= 1u << c;
      sm.mask[j] = mk;
    }
    if (pt == 0) sm.n_tiles = J;
    named_bar_sync(2, kProducers);
    if (pt == 0) {
      if (sm.bad && half == 0) record_status(status, CSA_DEV_BOUNDS);
      mbar_arrive(&sm.list_ready);
      trace_time(status, 1);
    }

    // Gathers: tile j -> stage j % kStages. Thread pt copies the 16-byte chunks pt, pt+128, ... of
    // the tile (32 rows x 64 chunks): a warp covers 512 contiguous bytes of one row per
    // instruction. The loop issues the next tile whenever its stage is free and otherwise waits
    // for its oldest tile in flight and announces it (kv_full), so tiles are announced as soon as
    // they land while up to kStages tiles are in flight. Each thread runs the loop on its own
    // (its decisions may differ from other threads'); every thread arrives once per tile. Stages
    // 2 and 3 first hold Q[:, 0:256] until the softmax warps moved it into TMEM (q_done).
    const char* ring_base = reinterpret_cast<const char*>(P.ring);
    const char* cache_base = reinterpret_cast<const char*>(P.cache);
    int next = 0, ann = 0;
    bool ok = true;
    while (ann < J) {
      bool issue = next < J;
      if (issue && next >= 2 && next < kStages) {
        if (next > ann) {
          issue = mbar_test(smem_u32(&sm.q_done), 0);
        } else if (!mbar_wait(&sm.q_done, 0, abort_flag, status, 101)) {
          ok = false;
          break;
        }
      } else if (issue && next >= kStages) {
        uint64_t* empty = &sm.buf_free[next % kStages];
        const uint32_t par = (uint32_t)((next / kStages - 1) & 1);
        if (next > ann) {
          issue = mbar_test(smem_u32(empty), par);
        } else if (!mbar_wait(empty, par, abort_flag, status, 102)) {
          ok = false;
          break;
        }
      }
      if (issue) {
        const uint32_t st = smem_u32(stage0 + (size_t)(next % kStages) * kStageBytes);
#pragma unroll 8
        for (int i = 0; i < 16; ++i) {
          const int c = pt + kProducers * i;  // chunk of the tile
          const int r = c >> 6;               // candidate row 0..31
          const int w = c & 63;               // chunk within the row
          const uint32_t e = sm.list[next * kTile + r];
          const char* src = ((e & kFromCache) ? cache_base : ring_base) + (size_t)(e & kRowMask) * 1024 + w * 16;
          cp_async_16(st + (w >> 3) * kBlockBytes + sw128_offset(r, w & 7), src);
        }
        cp_async_commit();
        ++next;
        continue;
      }
      switch (next - ann) {  // groups committed after the oldest tile in flight
        case 1: cp_async_wait<0>(); break;
        case 2: cp_async_wait<1>(); break;
        case 3: cp_async_wait<2>(); break;
        default: cp_async_wait<3>(); break;
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.kv_full[ann % kStages]);
      if (pt == 0 && ann < 60) trace_time(status, 2 + ann);
      ++ann;
    }
    cp_async_wait<0>();  // after an abort: let the copies land before teardown
    // Epilogue share: O columns [128, 256) of this warp's rows, once the softmax published 1/l.
    const bool fin =
        __all_sync(0xffffffffu, ok && ann == J && J > 0 && mbar_wait(&sm.epi, 0, abort_flag, status, 103));
    if (fin) {
      tc_fence_after();
      store_rows(P, sm, tmem + ((uint32_t)(quad * 32) << 16) + 256, 128, half, (long long)qi * P.H + h, h,
                 sm.inv_l[h]);
    }
  } else if (warp < kPvWarp) {
    // ------------------------------------------------------------ score MMAs: tiles j = w, w+2, ...
    if (lane == 0) {
      const int w = warp - kQkWarp0;  // 0: even tiles, 1: odd tiles
      bool ok = mbar_wait(&sm.q_full, 0, abort_flag, status, 111) &&
                mbar_wait(&sm.q_done, 0, abort_flag, status, 112) &&
                mbar_wait(&sm.list_ready, 0, abort_flag, status, 113);
      const int J = ok ? sm.n_tiles : 0;
      const uint32_t idesc_qk = idesc_bf16_f32(128, kTile, 0, 0);
      const uint32_t qhi = smem_u32(q_hi);
      for (int j = w; j < J; j += 2) {
        const int s = j % kStages;
        // Score tile s is rewritten only once PV(j - kStages), which read its P, has completed.
        if (j >= kStages && !mbar_wait(&sm.buf_free[s], (uint32_t)((j / kStages - 1) & 1), abort_flag, status, 117))
          break;
        if (!mbar_wait(&sm.kv_full[s], (uint32_t)((j / kStages) & 1), abort_flag, status, 114)) break;
        tc_fence_after();
        if (j < 60) trace_time(status, 64 + j);
        const uint32_t kbase = smem_u32(stage0 + (size_t)s * kStageBytes);
        const uint32_t d_s = tmem + 128 + kTile * s;
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {  // dims 0..255: A = Q from TMEM
          const uint64_t bdesc = smem_desc_sw128(kbase + (ks >> 2) * kBlockBytes + (ks & 3) * 32, 16, 1024);
          mma_ts(d_s, tmem + 8 * ks, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 16; ks < 32; ++ks) {  // dims 256..511: A = Q from smem
          const uint64_t adesc = smem_desc_sw128(qhi + ((ks - 16) >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(kbase + (ks >> 2) * kBlockBytes + (ks & 3) * 32, 16, 1024);
          mma_ss(d_s, adesc, bdesc, idesc_qk, 1u);
        }
        mma_commit(&sm.s_full[s]);
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
        const int sb = j % kSBufs;
        if (!mbar_wait(&sm.p_full[sb], (uint32_t)((j / kSBufs) & 1), abort_flag, status, 115)) break;
        tc_fence_after();
        const uint32_t vbase =
            smem_u32(stage0 + (size_t)(j % kStages) * kStageBytes) + (uint32_t)(4 * half) * kBlockBytes;
        const uint32_t pcol = tmem + 128 + kTile * sb;
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // P_hi, then P_lo
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t bdesc = smem_desc_sw128(vbase + ks * 2048, kBlockBytes, 1024);
            mma_ts(tmem + 256, pcol + 16 * part + 8 * ks, bdesc, idesc_pv, (j > 0 || part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&sm.o_done[j & 1]);
        mma_commit(&sm.buf_free[j % kStages]);
        if (j < 60) trace_time(status, 192 + j);
      }
      mma_commit(&sm.drain[2]);
      mbar_wait_drain(&sm.drain[2], 0, status, 119);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 5..8), epilogue
    const int quad = warp & 3;             // TMEM lane quadrant
    const int h = quad * 32 + lane;        // head = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int et = threadIdx.x - kSoftWarp0 * 32;
    // Q[:, 0:256] -> TMEM columns [0, 128).
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full, 0, abort_flag, status, 121));
    if (ok) {
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(q_lo + kb * 16384 + sw128_offset(h, ch));
          r[4 * ch + 0] = v.x;
          r[4 * ch + 1] = v.y;
          r[4 * ch + 2] = v.z;
          r[4 * ch + 3] = v.w;
        }
        tmem_st32(tmem + lane_addr + 32 * kb, r);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&sm.q_done);
    // Inverse-RoPE table for position t.
    const int npairs = P.rope_dim / 2;
    if (et < npairs) {
      float cs, sn;
      rope_cos_sin(t, P.inv_freq[et], &cs, &sn);
      sm.rope_cs[et][0] = cs;
      sm.rope_cs[et][1] = -sn;
    }
    named_bar_sync(1, kSoftThreads);
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&sm.list_ready, 0, abort_flag, status, 122));
    const int J = ok ? sm.n_tiles : 0;
    const float sl = (h < P.H) ? P.sink[h] * 1.4426950408889634f : 0.f;
    float m_used = sl;  // running max in log2 units (starts at the sink)
    float l = 1.f;      // running denominator; the sink contributes exp2(sl - m_used) = 1
    int j = 0;
    for (; j < J; ++j) {
      const int sb = j % kSBufs;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (uint32_t)((j / kSBufs) & 1), abort_flag, status, 123)))
        break;
      if (et == 0 && j < 60) trace_time(status, 500 + j);
      tc_fence_after();
      const uint32_t sa = tmem + lane_addr + 128 + kTile * sb;
      uint32_t v[32];
      tmem_ld32(sa, v);
      tmem_wait_ld();
      const uint32_t mk = sm.mask[j];
      float x[32];
      float mt = -CUDART_INF_F;
      if (mk == 0xFFFFFFFFu) {  // a full tile (the common case): no padding to mask
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(v[c]) * P.scale_log2;
          mt = fmaxf(mt, x[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = ((mk >> c) & 1u) ? __uint_as_float(v[c]) * P.scale_log2 : -CUDART_INF_F;
          mt = fmaxf(mt, x[c]);
        }
      }
      // Lazy rescale: only when this tile raises the row max by more than 2^8. The TMEM accesses
      // are warp-collective, so the whole warp takes the branch if any lane needs it (lanes that do
      // not need it scale by 1).
      const bool need = mt > m_used + 8.f;
      const float alpha = need ? exp2f(m_used - mt) : 1.f;
      if (__any_sync(0xffffffffu, need)) {
        if (j > 0) {
          // O holds PV(0..j-1): wait for PV(j-1), then scale the rows of this warp.
          const bool okw = mbar_wait(&sm.o_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort_flag, status, 124);
          if (!__all_sync(0xffffffffu, okw)) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t o[32];
            const uint32_t oa = tmem + lane_addr + 256 + 32 * cc;
            tmem_ld32(oa, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(oa, o);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= alpha;
          m_used = mt;
        }
      }
      // P = P_hi + P_lo, both bf16: P_hi in columns [0,16) of the tile, P_lo in [16,32).
      uint32_t phi[16], plo[16];
      float rs = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float p0 = ex2_approx(x[2 * q] - m_used);
        const float p1 = ex2_approx(x[2 * q + 1] - m_used);
        phi[q] = pack_bf16(p0, p1);
        plo[q] = pack_bf16(p0 - bf16_lo(phi[q]), p1 - bf16_hi(phi[q]));
        rs += p0 + p1;
      }
      l += rs;
      tmem_st16(sa, phi);
      tmem_st16(sa + 16, plo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[sb]);
      if (et == 0 && j < 60) trace_time(status, 128 + j);
    }
    // Epilogue: this warp's rows, O columns [0, 128); the producer warps take [128, 256).
    const bool fin = __all_sync(0xffffffffu, j == J && J > 0 &&
                                                 mbar_wait(&sm.o_done[(J - 1) & 1], (uint32_t)(((J - 1) >> 1) & 1),
                                                           abort_flag, status, 125));
    const float inv = 1.f / l;
    sm.inv_l[h] = inv;
    mbar_arrive(&sm.epi);
    if (fin) {
      tc_fence_after();
      store_rows(P, sm, tmem + lane_addr + 256, 0, half, (long long)qi * P.H + h, h, inv);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) trace_time(status, 255);
  if (warp == kPvWarp) tmem_dealloc(tmem, 512);
}

size_t attn_smem_bytes() { return 1024 + kQhiBytes + kStages * kStageBytes + sizeof(AttnSmem); }

}  // namespace csa
