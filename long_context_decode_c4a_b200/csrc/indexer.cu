// indexer.cu -- lightning-indexer scores on the tcgen05 tensor cores (K2).
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", section "少读 KV 之前，Indexer 仍要给历史打分": 64 heads of
// 128 dims score every visible entry of one shared 128-dim compressed index cache,
//     score(t, s) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[s,:]),   s < (t+1)//ratio,
// with w free in sign (not a softmax). "图解DeepSeek V4：详细计算流程解析" §2.2: the index keys come from
// the same 4:1 C4A compressor.
//
// Contraction: per work item, D[128 entries x N] = K_tile[128 x 128] . Q_group^T, where the N
// columns are (query, head) pairs of QG consecutive queries of one request (N = QG*H_I <= 256;
// decode: QG = 1, N = 64). A = index-cache tile (K-major, TMA, 128B swizzle), B = the group's
// q_idx rows (K-major, TMA), D in TMEM (fp32, double-buffered). The epilogue (thread = entry =
// TMEM lane) applies ReLU, weights by w and sums over heads, and writes one fp32 score per
// (query, entry) with coalesced stores.
//
// Persistent kernel, one CTA per SM, warp roles: warp 0 = TMA producer, warp 1 = MMA issuer
// (and TMEM owner), warps 2..5 = epilogue. Work items (request, query group, 128-entry tile) are
// split into contiguous ranges per CTA so the Q tile of a group is loaded once per CTA. Tiles
// past the group's last visible entry are skipped by every role alike.

#include "compress_decode.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace csa {

namespace {

// ReLU that keeps NaN (a NaN dot product stays NaN, as max(x, 0) does in IEEE propagation).
__device__ __forceinline__ float relu_nan(float x) {
  float r;
  asm("max.NaN.f32 %0, %1, 0f00000000;" : "=f"(r) : "f"(x));
  return r;
}

struct ItemCoord {
  int b, qg, et;
};

// Visible entries of query (b, i): (t+1)//ratio, capped at max_entries.
__device__ __forceinline__ int visible_of(const IndexerParams& P, int b, int i) {
  const int t = P.q_pos[(long long)b * P.S + i];
  int E = (t + 1) / P.ratio;
  E = E < 0 ? 0 : E;
  return E > P.max_entries ? P.max_entries : E;
}

// Walks the work items [it, it1) that hold at least one visible entry, in order, and numbers
// the query groups met (gi). Every role runs its own copy over the same range. The coordinates
// advance incrementally (one division, at construction); the tiles of a group past its last
// visible entry are skipped in one step.
struct ItemIter {
  long long it, it1;
  int et, qg, b;  // coordinates of item `it`
  int cur_b, cur_qg, gv, gi;
  bool started;

  __device__ ItemIter(const IndexerParams& P, long long a, long long e)
      : it(a), it1(e), cur_b(-1), cur_qg(-1), gv(0), gi(-1), started(false) {
    const long long gq = a / P.tiles_per_group;
    et = (int)(a - gq * P.tiles_per_group);
    b = (int)(gq / P.groups_per_req);
    qg = (int)(gq - (long long)b * P.groups_per_req);
  }

  __device__ void next_group(const IndexerParams& P) {
    et = 0;
    if (++qg == P.groups_per_req) {
      qg = 0;
      ++b;
    }
  }

  __device__ bool next(const IndexerParams& P, ItemCoord& c, bool& new_group) {
    while (it < it1) {
      c.et = et;
      c.qg = qg;
      c.b = b;
      if (c.b != cur_b || c.qg != cur_qg) {
        cur_b = c.b;
        cur_qg = c.qg;
        started = false;
        gv = 0;
        const int i0 = c.qg * P.QG, i1 = min(P.S, i0 + P.QG);
        for (int i = i0; i < i1; ++i) gv = max(gv, visible_of(P, c.b, i));
      }
      if (c.et * 128 >= gv) {  // nothing visible in the rest of this group
        it += P.tiles_per_group - c.et;
        next_group(P);
        continue;
      }
      ++it;
      if (++et == P.tiles_per_group) next_group(P);
      new_group = !started;
      if (new_group) {
        ++gi;
        started = true;
      }
      return true;
    }
    return false;
  }
};

// Wait (bounded) until another CTA raises *flag, then clear it for the next call and order the
// loads that follow through the tensor-memory-access (async) proxy after what the flag published.
__device__ __forceinline__ bool wait_flag_and_clear(uint32_t* flag, volatile int* abort_flag, uint32_t* status,
                                                    uint32_t site) {
  const long long t0 = clock64();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0u) break;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      record_status(status, CSA_DEV_TIMEOUT);
      record_site(status, site);
      *abort_flag = 1;
      return false;
    }
  }
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(0u) : "memory");
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

struct IdxSmem {
  uint64_t k_full[kIdxMaxStages], k_empty[kIdxMaxStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t acc_full[4], acc_empty[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int HI>
__device__ __forceinline__ void epilogue_tile(const IndexerParams& P, const float* w_s, const int* vis_s,
                                              uint32_t tmem_acc, int b, int qg, int et, int row) {
  constexpr int kQPerChunk = HI >= 32 ? 1 : 32 / HI;
  constexpr int kChunksPerQ = HI >= 32 ? HI / 32 : 1;
  constexpr int kColsPerQ = HI >= 32 ? 32 : HI;
  const int nq = min(P.QG, P.S - qg * P.QG);
  const int s = et * 128 + row;
  const int ncols = nq * HI;
  for (int col0 = 0; col0 < ncols; col0 += 32 * kChunksPerQ) {
    // Four independent partial sums per query keep the FMA chains short.
    float part[kQPerChunk][4];
#pragma unroll
    for (int j = 0; j < kQPerChunk; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u) part[j][u] = 0.f;
#pragma unroll
    for (int c = 0; c < kChunksPerQ; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem_acc + col0 + 32 * c, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = __uint_as_float(v[j]);
        float& acc = part[j / kColsPerQ][j & 3];
        acc = fmaf(w_s[col0 + 32 * c + j], relu_nan(x), acc);
      }
    }
#pragma unroll
    for (int j = 0; j < kQPerChunk; ++j) {
      const int qi = col0 / HI + j;
      if (qi < nq && s < vis_s[qi]) {
        const long long qrow = (long long)b * P.S + (long long)qg * P.QG + qi;
        P.scores[qrow * P.scores_stride + s] = (part[j][0] + part[j][1]) + (part[j][2] + part[j][3]);
      }
    }
  }
}

}  // namespace

template <int HI>
__global__ void __launch_bounds__(kIdxThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                   IndexerParams P, IndexerFuse F) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NS = P.stages;
  const int N = P.N;
  const uint32_t q_bytes = (uint32_t)N * 256u;   // N rows x 128 dims x 2 bytes (two 64-dim blocks)
  uint8_t* k_tiles = base;                       // NS x 32 KB: [2 d-blocks][128 rows][128 B]
  uint8_t* q_tiles = base + (size_t)NS * 32768;  // 2 x q_bytes: [2 d-blocks][N rows][128 B]
  IdxSmem& sm = *reinterpret_cast<IdxSmem*>(q_tiles + 2 * (size_t)q_bytes);
  // Per epilogue group: w of the group's current queries (N floats) and their visible entries.
  float* w_arr = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(&sm) + sizeof(IdxSmem));
  int* vis_arr = reinterpret_cast<int*>(w_arr + 2 * N);
  // Fused decode compression: the body's partials and reduction scratch.
  DecodePartial* part = reinterpret_cast<DecodePartial*>(
      (reinterpret_cast<uintptr_t>(vis_arr + 2 * N) + 15) & ~uintptr_t(15));
  float* red = reinterpret_cast<float*>(part + kCompressThreads);

  const int warp = warp_id();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], 128);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_q);
  }
  const uint32_t acc_cols = (uint32_t)P.tmem_cols;  // power of two >= n_acc * N
  const int n_acc = P.n_acc;                         // 2 or 4 accumulators (even: one parity per group)
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, acc_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  timeline_mark(P.status, kTlIndexer, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlIndexer, kTlReady);
  if (threadIdx.x == 0) trace_time(P.status, 599);

  const long long total = P.total_items;
  const long long per = (total + gridDim.x - 1) / gridDim.x;
  const long long it0 = min(total, (long long)blockIdx.x * per);
  const long long it1 = min(total, it0 + per);
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t* status = P.status;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      ItemIter iter(P, it0, it1);
      ItemCoord c;
      bool ng;
      long long n = 0;
      while (iter.next(P, c, ng)) {
        if (ng) {
          const int slot = iter.gi & 1;
          if (!mbar_wait(&sm.q_empty[slot], ((iter.gi >> 1) & 1) ^ 1, abort_flag, status, 201)) break;
          mbar_arrive_expect_tx(&sm.q_full[slot], q_bytes);
          const int row0 = (int)(((long long)c.b * P.S + (long long)c.qg * P.QG) * HI);
          uint8_t* dst = q_tiles + (size_t)slot * q_bytes;
          tma_load_2d(dst, &map_q, 0, row0, &sm.q_full[slot]);
          tma_load_2d(dst + (size_t)N * 128, &map_q, 64, row0, &sm.q_full[slot]);
        }
        const int st = (int)(n % NS);
        const uint32_t ph = (uint32_t)((n / NS) & 1);
        if (!mbar_wait(&sm.k_empty[st], ph ^ 1, abort_flag, status, 202)) break;
        if (F.njobs > 0) {
          // The tile holding the request's last visible entry waits for this step's index entry.
          const int vis = visible_of(P, c.b, c.qg * P.QG);
          if (vis > 0 && c.et == (vis - 1) / 128 && !wait_flag_and_clear(&F.flags[c.b], abort_flag, status, 204)) break;
        }
        mbar_arrive_expect_tx(&sm.k_full[st], 32768);
        const int krow = (int)((long long)c.b * P.rows_per_req + (long long)c.et * 128);
        uint8_t* dst = k_tiles + (size_t)st * 32768;
        tma_load_2d(dst, &map_k, 0, krow, &sm.k_full[st]);
        tma_load_2d(dst + 16384, &map_k, 64, krow, &sm.k_full[st]);
        trace_mark(status, 0, (uint32_t)(100 + n));
        if (n < 100) trace_time(status, 600 + (int)n);
        ++n;
      }
      // After an abort the loads issued last may still be landing in the stages: wait for them
      // (they complete by themselves) before the CTA can exit. Each of the last min(n, NS) stages
      // has one load outstanding at most, so its phase parity is unambiguous.
      for (long long i = n > NS ? n - NS : 0; i < n; ++i)
        mbar_wait_drain(&sm.k_full[(int)(i % NS)], (uint32_t)((i / NS) & 1), status, 203);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, N, 0, 0);
      ItemIter iter(P, it0, it1);
      ItemCoord c;
      bool ng;
      long long n = 0;
      int slot = 0;
      while (iter.next(P, c, ng)) {
        if (ng) {
          if (iter.gi > 0) mma_commit(&sm.q_empty[(iter.gi - 1) & 1]);  // previous group's Q is free
          slot = iter.gi & 1;
          if (!mbar_wait(&sm.q_full[slot], (iter.gi >> 1) & 1, abort_flag, status, 211)) break;
        }
        const int st = (int)(n % NS);
        if (!mbar_wait(&sm.k_full[st], (uint32_t)((n / NS) & 1), abort_flag, status, 212)) break;
        const int a = (int)(n % n_acc);
        if (!mbar_wait(&sm.acc_empty[a], (uint32_t)(((n / n_acc) & 1) ^ 1), abort_flag, status, 213)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(a * N);
        const uint32_t ka = smem_u32(k_tiles + (size_t)st * 32768);
        const uint32_t qa = smem_u32(q_tiles + (size_t)slot * q_bytes);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t kb = ks >> 2, off = (ks & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(ka + kb * 16384 + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(qa + kb * (uint32_t)N * 128 + off, 16, 1024);
          mma_ss(d_tmem, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&sm.k_empty[st]);
        mma_commit(&sm.acc_full[a]);
        trace_mark(status, 1, (uint32_t)(100 + n));
        if (n < 100) trace_time(status, 700 + (int)n);
        ++n;
      }
      // Every MMA issued by this thread completes before TMEM is released.
      mma_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, status, 214);
      trace_mark(status, 1, 9);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..9)
    // Two groups of four warps take alternate work items (group g: items n with n % 2 == g), each
    // group covering the four TMEM lane quadrants.
    if (F.njobs > 0) {
      // The step's compression jobs first (index streams before main streams); named barriers 5-7.
      const int et = threadIdx.x - 64;                // 0..255
      for (int job = blockIdx.x; job < F.njobs; job += gridDim.x) {
        const bool idx_stream = job < F.B;
        const int b = idx_stream ? job : job - F.B;
        const CompressParams& CP = F.L.p[idx_stream ? 1 : 0];
        if (CP.d == 512) compress_decode_body<4, 512>(CP, b, part, red, et, 5, 6);
        else compress_decode_body<4, 128>(CP, b, part, red, et, 5, 6);
        named_bar_sync(7, 256);   // the job's writes are issued and its shared partials read
        if (idx_stream && et == 0) {
          __threadfence();
          atomicExch(&F.flags[b], 1u);
        }
      }
    }
    const int grp = (warp - 2) >> 2;
    const int gt = threadIdx.x - 64 - 128 * grp;      // 0..127 within the group
    const int quad = warp & 3;                        // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    float* w_s = w_arr + grp * N;
    int* vis_s = vis_arr + grp * N;
    ItemIter iter(P, it0, it1);
    ItemCoord c;
    bool ng;
    long long n = 0;
    int cur_b = -1, cur_qg = -1;
    while (iter.next(P, c, ng)) {
      const long long my = n++;
      if ((my & 1) != grp) continue;
      if (c.b != cur_b || c.qg != cur_qg) {
        named_bar_sync(1 + 2 * grp, 128);
        const int nq = min(P.QG, P.S - c.qg * P.QG);
        const long long q0 = (long long)c.b * P.S + (long long)c.qg * P.QG;
        for (int j = gt; j < nq * HI; j += 128) w_s[j] = P.w[q0 * HI + j];
        for (int j = gt; j < nq; j += 128) vis_s[j] = visible_of(P, c.b, c.qg * P.QG + j);
        named_bar_sync(1 + 2 * grp, 128);
        cur_b = c.b;
        cur_qg = c.qg;
      }
      const int a = (int)(my % n_acc);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[a], (uint32_t)((my / n_acc) & 1), abort_flag, status, 221))) break;
      if (gt == 0) trace_mark(status, 2, (uint32_t)(100 + my));
      if (gt == 0 && my < 100) trace_time(status, 800 + (int)my);
      tc_fence_after();
      epilogue_tile<HI>(P, w_s, vis_s, tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * N), c.b, c.qg, c.et, row);
      tc_fence_before();
      mbar_arrive(&sm.acc_empty[a]);
      if (gt == 0 && my < 100) trace_time(status, 900 + (int)my);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) trace_mark(status, 3, 2);
  if (warp == 1) tmem_dealloc(tmem, acc_cols);
  if (threadIdx.x == 32) trace_mark(status, 3, 3);
  timeline_mark(status, kTlIndexer, kTlExit);
}

size_t indexer_smem_bytes(int stages, int N, bool fuse) {
  const size_t base = 1024 + (size_t)stages * 32768 + 2 * (size_t)N * 256 + sizeof(IdxSmem) + 2 * 2 * (size_t)N * 4;
  return fuse ? base + 16 + kCompressThreads * sizeof(DecodePartial) + kCompressThreads / 32 * sizeof(float) : base;
}

template __global__ void indexer_kernel<4>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);
template __global__ void indexer_kernel<8>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);
template __global__ void indexer_kernel<16>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);
template __global__ void indexer_kernel<32>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);
template __global__ void indexer_kernel<64>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);
template __global__ void indexer_kernel<128>(const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap, IndexerParams, IndexerFuse);

}  // namespace csa
