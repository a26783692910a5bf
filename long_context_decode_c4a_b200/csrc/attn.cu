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
// Layout of the work: a cluster of two CTAs per query; CTA c owns dims [256c, 256c+256) of the
// head dim. Each CTA gathers only its half of every candidate row, so a row crosses HBM once.
// Per tile of 64 candidates each CTA computes the partial scores S_c = Q[:, half] K[:, half]^T
// (M = 128 heads, N = 64, K = 256) and sends them to the other CTA through distributed shared
// memory; both add S_0 + S_1 (the same sum in both, fp addition being commutative), run the same
// online softmax, and accumulate O[:, half] += P V[:, half]. Per CTA:
//   TMEM (512 columns): [0,128) Q[:, half] as bf16 pairs (A operand of the TS-MMA for S);
//     [128,192) and [192,256) the S tiles (double buffer) -- after the softmax reads a tile, its
//     first 32 columns hold P_hi and the next 32 P_lo (bf16 pairs); [256,512) O[:, half].
//   SMEM: four 32 KB stages of 64 half-rows (4 blocks of 64 dims in the 128B-swizzled layout that
//     serves S as a K-major B operand and PV as an MN-major B operand); two 32 KB exchange
//     buffers that receive the other CTA's partial S tiles (they first stage Q[:, half] on its
//     way into TMEM); the candidate list.
//   Warps: 0..3 build the candidate list and gather half-rows with coalesced 16-byte cp.async,
//     up to three tiles in flight; 4 issues the MMAs (and owns TMEM); 5..12 run the exchange and
//     the softmax, two warps per TMEM lane quadrant (thread = head = TMEM lane, each warp of the
//     pair owning 32 of the tile's 64 columns), then the epilogue.
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
constexpr int kMmaWarp = 4;
constexpr int kSoftmaxWarp0 = 5;              // warps 5..12
constexpr int kSoftmaxThreads = 256;
constexpr int kStages = 4;
constexpr int kGatherDepth = 2;               // committed gather groups left in flight per producer
constexpr size_t kStageBytes = 32 * 1024;     // 64 rows x 256 dims of bf16
constexpr size_t kXBytes = 32 * 1024;         // 128 heads x 64 fp32 partial scores

static_assert(kAttnThreads == 32 * (kSoftmaxWarp0 + 8), "warp roles");

struct AttnSmem {
  uint64_t q_full, q_done, list_ready;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t x_full[2], x_empty[2];     // arrived on by the other CTA of the cluster
  uint64_t pair[4][2], pair_end[4];   // the two softmax warps of a TMEM lane quadrant
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int n_tiles;
  int bad;
  uint32_t scan[kProducers / 32];
  float rope_cs[kMaxRopePairs][2];
  float red_max[2][2][128];           // [tile parity][column half][head]
  float red_l[2][128];
  unsigned long long mask[kAttnMaxTiles];
  uint32_t list[kAttnMaxCands];
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of 16-byte chunk k (0..15) of head row h in an exchange buffer; the XOR spreads a
// quarter-warp's accesses over all banks.
__device__ __forceinline__ uint32_t xoff(uint32_t h, uint32_t k) { return h * 256u + ((k ^ (h & 15u)) << 4); }

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

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage0 = base;                        // stage s at stage0 + s * 32 KB: 4 x [64 rows][128 B]
  uint8_t* xbuf = base + kStages * kStageBytes;  // 2 x 32 KB; first Q[:, half] as 4 x [128 rows][128 B]
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(xbuf + 2 * kXBytes);

  const int warp = warp_id();
  const int lane = lane_id();
  const uint32_t half = cluster_ctarank();    // which 256 dims this CTA owns
  const uint32_t peer = half ^ 1u;
  const int nq = P.B * P.S;
  const int qi = nq - 1 - (int)blockIdx.y;    // later queries (more candidates) first
  const int b = qi / P.S;
  const int t = P.q_pos[qi];
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t* status = P.status;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_done, kSoftmaxThreads);
    mbar_init(&sm.list_ready, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.kv_full[i], kProducers);
      mbar_init(&sm.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], kSoftmaxThreads);
      mbar_init(&sm.o_done[i], 1);
      mbar_init(&sm.x_full[i], kSoftmaxThreads);
      mbar_init(&sm.x_empty[i], kSoftmaxThreads);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sm.pair[q][0], 64);
      mbar_init(&sm.pair[q][1], 64);
      mbar_init(&sm.pair_end[q], 64);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    sm.bad = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();   // the barriers of both CTAs are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) trace_time(status, 0);

  if (warp < kProducers / 32) {
    // ------------------------------------------------------------ Q load, candidate list, gathers
    const int pt = threadIdx.x;  // 0..127
    if (pt == 0) {
      const int row0 = qi * P.H;
      mbar_arrive_expect_tx(&sm.q_full, 4u * 16384u);
      for (int k = 0; k < 4; ++k) tma_load_2d(xbuf + k * 16384, &map_q, 256 * (int)half + 64 * k, row0, &sm.q_full);
    }
    // Candidate list: window rows, then the compressed entries, padded to tiles of 64.
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
    const int n64 = (n + 63) & ~63;
    for (int k = n + pt; k < n64; k += kProducers) sm.list[k] = self_slot | kInvalid;
    const int J = n64 / 64;
    named_bar_sync(2, kProducers);
    for (int j = pt; j < J; j += kProducers) {
      unsigned long long mk = 0;
      for (int c = 0; c < 64; ++c)
        if (!(sm.list[j * 64 + c] & kInvalid)) mk |= 1ull << c;
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
    // the tile (64 half-rows x 32 chunks): a warp covers one contiguous 512-byte half-row per
    // instruction. A tile is announced (kv_full) once kGatherDepth later tiles have been issued,
    // so up to kGatherDepth + 1 tiles are in flight.
    const char* ring_base = reinterpret_cast<const char*>(P.ring) + 512 * half;
    const char* cache_base = reinterpret_cast<const char*>(P.cache) + 512 * half;
    int issued = 0;
    for (int j = 0; j < J; ++j) {
      const int s = j % kStages;
      if (j >= kStages && !mbar_wait(&sm.kv_empty[s], (uint32_t)((j / kStages - 1) & 1), abort_flag, status, 102))
        break;
      const uint32_t st = smem_u32(stage0 + (size_t)s * kStageBytes);
#pragma unroll 8
      for (int i = 0; i < 16; ++i) {
        const int c = pt + kProducers * i;  // chunk of the tile
        const int r = c >> 5;               // candidate row 0..63
        const int w = c & 31;               // chunk within the half-row
        const uint32_t e = sm.list[j * 64 + r];
        const char* src = ((e & kFromCache) ? cache_base : ring_base) + (size_t)(e & kRowMask) * 1024 + w * 16;
        cp_async_16(st + (w >> 3) * 8192 + sw128_offset(r, w & 7), src);
      }
      cp_async_commit();
      issued = j + 1;
      if (j >= kGatherDepth) {
        cp_async_wait<kGatherDepth>();
        fence_proxy_async_smem();
        mbar_arrive(&sm.kv_full[(j - kGatherDepth) % kStages]);
        if (pt == 0) trace_time(status, 2 + j - kGatherDepth);
      }
    }
    // Announce the last tiles (or, after an abort, just let the copies land before teardown).
    if (issued >= 2) {
      cp_async_wait<1>();
      fence_proxy_async_smem();
      mbar_arrive(&sm.kv_full[(issued - 2) % kStages]);
    }
    if (issued >= 1) {
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&sm.kv_full[(issued - 1) % kStages]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.q_done, 0, abort_flag, status, 112) &&
                mbar_wait(&sm.list_ready, 0, abort_flag, status, 113);
      const int J = ok ? sm.n_tiles : 0;
      const uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      auto issue_pv = [&](int jj) -> bool {
        const int x = jj & 1;
        const int s = jj % kStages;
        if (!mbar_wait(&sm.p_full[x], (uint32_t)((jj >> 1) & 1), abort_flag, status, 115)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(stage0 + (size_t)s * kStageBytes);
        const uint32_t pcol = tmem + 128 + 64 * x;
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // P_hi, then P_lo
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bdesc = smem_desc_sw128(vbase + ks * 2048, 8192, 1024);
            mma_ts(tmem + 256, pcol + 32 * part + 8 * ks, bdesc, idesc_pv, (jj > 0 || part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        mma_commit(&sm.o_done[x]);
        mma_commit(&sm.kv_empty[s]);
        trace_time(status, 192 + jj);
        return true;
      };
      int j = 0;
      for (; j < J; ++j) {
        const int s = j % kStages;
        if (!mbar_wait(&sm.kv_full[s], (uint32_t)((j / kStages) & 1), abort_flag, status, 114)) break;
        tc_fence_after();
        trace_time(status, 64 + j);
        const uint32_t kbase = smem_u32(stage0 + (size_t)s * kStageBytes);
        const uint32_t d_s = tmem + 128 + 64 * (j & 1);
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {  // the CTA's 256 dims: A = Q from TMEM
          const uint64_t bdesc = smem_desc_sw128(kbase + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
          mma_ts(d_s, tmem + 8 * ks, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[j & 1]);
        if (j >= 1 && !issue_pv(j - 1)) break;
      }
      if (j == J && J > 0) issue_pv(J - 1);
      // Every MMA issued above completes on its own; wait for them before TMEM is released.
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, status, 116);
    }
  } else {
    // ------------------------------------------------------------ exchange, softmax, epilogue
    const int sw = warp - kSoftmaxWarp0;   // 0..7
    const int quad = warp & 3;             // TMEM lane quadrant
    const int cb = sw >> 2;                // which 32 columns of each tile this warp owns
    const int h = quad * 32 + lane;        // head = TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int et = threadIdx.x - kSoftmaxWarp0 * 32;
    const uint32_t xpeer = mapa_shared(smem_u32(xbuf), peer);
    // Q[:, half] -> TMEM columns [0, 128); this warp moves blocks 2cb and 2cb+1.
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.q_full, 0, abort_flag, status, 121));
    if (ok) {
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = 2 * cb + kk;
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(xbuf + kb * 16384 + sw128_offset(h, ch));
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
    // The staging area is free: the other CTA may send its first two partial tiles.
    mbar_arrive_remote(mapa_shared(smem_u32(&sm.x_empty[0]), peer));
    mbar_arrive_remote(mapa_shared(smem_u32(&sm.x_empty[1]), peer));
    // Inverse-RoPE table for position t.
    const int npairs = P.rope_dim / 2;
    if (et < npairs) {
      float cs, sn;
      rope_cos_sin(t, P.inv_freq[et], &cs, &sn);
      sm.rope_cs[et][0] = cs;
      sm.rope_cs[et][1] = -sn;
    }
    named_bar_sync(1, kSoftmaxThreads);
    ok = __all_sync(0xffffffffu, ok && mbar_wait(&sm.list_ready, 0, abort_flag, status, 122));
    const int J = ok ? sm.n_tiles : 0;
    const float sl = (h < P.H) ? P.sink[h] * 1.4426950408889634f : 0.f;
    float m_used = sl;              // running max in log2 units (starts at the sink)
    float l = cb == 0 ? 1.f : 0.f;  // this warp's part of the denominator; the sink counts once
    int j = 0;
    for (; j < J; ++j) {
      const int x = j & 1;
      const uint32_t par = (uint32_t)((j >> 1) & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[x], par, abort_flag, status, 123))) break;
      if (et == 0 && j < 40) trace_time(status, 300 + j);
      tc_fence_after();
      uint32_t v[32];
      const uint32_t sa = tmem + lane_addr + 128 + 64 * x;
      tmem_ld32(sa + 32 * cb, v);
      tmem_wait_ld();
      // Send this CTA's partial scores to the other CTA, then add the other CTA's.
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(&sm.x_empty[x], par, abort_flag, status, 126))) break;
      if (et == 0 && j < 40) trace_time(status, 340 + j);
      const uint32_t xo = (uint32_t)x * (uint32_t)kXBytes;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_cluster_v4(xpeer + xo + xoff(h, 8 * cb + i), v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      mbar_arrive_remote(mapa_shared(smem_u32(&sm.x_full[x]), peer));
      if (et == 0 && j < 40) trace_time(status, 380 + j);
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(&sm.x_full[x], par, abort_flag, status, 127))) break;
      if (et == 0 && j < 40) trace_time(status, 420 + j);
      float sc[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 o = *reinterpret_cast<const uint4*>(xbuf + xo + xoff(h, 8 * cb + i));
        sc[4 * i + 0] = __uint_as_float(v[4 * i + 0]) + __uint_as_float(o.x);
        sc[4 * i + 1] = __uint_as_float(v[4 * i + 1]) + __uint_as_float(o.y);
        sc[4 * i + 2] = __uint_as_float(v[4 * i + 2]) + __uint_as_float(o.z);
        sc[4 * i + 3] = __uint_as_float(v[4 * i + 3]) + __uint_as_float(o.w);
      }
      mbar_arrive_remote(mapa_shared(smem_u32(&sm.x_empty[x]), peer));
      const uint32_t mk = (uint32_t)(sm.mask[j] >> (32 * cb));
      float mt = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        sc[c] = ((mk >> c) & 1u) ? sc[c] * P.scale_log2 : -CUDART_INF_F;
        mt = fmaxf(mt, sc[c]);
      }
      // Row max over the tile's 64 columns: combine with the other warp of the quadrant.
      sm.red_max[x][cb][h] = mt;
      mbar_arrive(&sm.pair[quad][x]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.pair[quad][x], par, abort_flag, status, 128))) break;
      if (et == 0 && j < 40) trace_time(status, 460 + j);
      mt = fmaxf(mt, sm.red_max[x][cb ^ 1][h]);
      // Lazy rescale: only when this tile raises the row max by more than 2^8. The TMEM accesses
      // are warp-collective, so the whole warp takes the branch if any lane needs it (lanes that do
      // not need it scale by 1). Both warps of a quadrant take the same decisions.
      const bool need = mt > m_used + 8.f;
      const float alpha = need ? exp2f(m_used - mt) : 1.f;
      if (__any_sync(0xffffffffu, need)) {
        if (j > 0) {
          // O holds PV(0..j-1): wait for PV(j-1), then scale this warp's 128 columns of its rows.
          const bool okw = mbar_wait(&sm.o_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort_flag, status, 124);
          if (!__all_sync(0xffffffffu, okw)) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            const uint32_t oa = tmem + lane_addr + 256 + 128 * cb + 32 * cc;
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
      // P = P_hi + P_lo, both bf16: P_hi in columns [0,32) of the tile, P_lo in [32,64); this warp
      // writes the 16 packed columns of its 32 candidates in each. The other warp of the quadrant
      // finished reading its scores before the pair barrier above.
      uint32_t phi[16], plo[16];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float p0 = exp2f(sc[2 * c] - m_used);
        const float p1 = exp2f(sc[2 * c + 1] - m_used);
        phi[c] = pack_bf16(p0, p1);
        const float r0 = p0 - bf16_lo(phi[c]);
        const float r1 = p1 - bf16_hi(phi[c]);
        plo[c] = pack_bf16(r0, r1);
        rs += p0 + p1;
      }
      l += rs;
      tmem_st16(sa + 16 * cb, phi);
      tmem_st16(sa + 32 + 16 * cb, plo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[x]);
      if (et == 0) trace_time(status, 128 + j);
    }
    // Epilogue: O / l, inverse RoPE on the rotated dims, store. Each warp of a quadrant stores
    // 128 of the CTA's 256 dims of its rows.
    bool fin = __all_sync(0xffffffffu, j == J && J > 0 &&
                                           mbar_wait(&sm.o_done[(J - 1) & 1], (uint32_t)(((J - 1) >> 1) & 1),
                                                     abort_flag, status, 125));
    if (fin) {
      sm.red_l[cb][h] = l;
      mbar_arrive(&sm.pair_end[quad]);
      fin = __all_sync(0xffffffffu, mbar_wait(&sm.pair_end[quad], 0, abort_flag, status, 129));
    }
    if (fin) {
      tc_fence_after();
      const float inv = 1.f / (l + sm.red_l[cb ^ 1][h]);
      const int rope0 = P.d - P.rope_dim;  // first rotated dim
      const long long orow = (long long)qi * P.H + h;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + 256 + 128 * cb + 32 * cc, o);
        tmem_wait_ld();
        float y[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) y[c] = __uint_as_float(o[c]) * inv;
        const int col0 = 256 * (int)half + 128 * cb + 32 * cc;  // global dim of y[0]
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
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();   // no remote access into this CTA's smem after this point
  tc_fence_after();
  if (threadIdx.x == 0) trace_time(status, 255);
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

size_t attn_smem_bytes() { return 1024 + kStages * kStageBytes + 2 * kXBytes + sizeof(AttnSmem); }

}  // namespace csa
