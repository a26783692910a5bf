// topk.cu -- top-k selection of the lightning indexer's scores (K3).
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", section "少读 KV 之前，Indexer 仍要给历史打分": top-k fixes
// the main attention reads; "图解DeepSeek V4：详细计算流程解析" §2.2: the index module outputs the
// indices of <= topK compressed entries. Ties go to the lower index; the output lists the chosen
// indices in ascending order, padded with -1.
//
// Method: block-level radix select on order-preserving 32-bit keys finds the k-th largest key T
// and how many keys equal to T to keep; a compaction pass in index order then keeps every key > T
// and the first `need` keys == T. Each radix pass bins the keys of the current key range into at
// most 2048 equal bins (the first range is [min, max] of the keys, so the bins follow the data's
// own spread and the shared-memory counters see little contention); three passes always suffice.
// A chunk of up to 16384 scores is held in registers (16 per thread); longer score rows are cut
// into chunks whose local top-k lists (in index order) are merged by a second launch with the
// same routine. The global order (score desc, index asc) restricted to a chunk is the chunk's own
// order, so the global top-k is contained in the union of the chunks' top-k lists.

#include "kernels.cuh"
#include "ptx.cuh"

namespace csa {

namespace {

// Order-preserving key, offset by one so that 0 can mark an empty position: larger score ->
// larger key; -0 == +0; NaN (key 1) below every number; +inf -> 0xFF800001.
__device__ __forceinline__ uint32_t score_key(float f) {
  if (f != f) return 1u;
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) + 1u;
}

constexpr int kSelBits = 11;
constexpr int kSelBins = 1 << kSelBits;   // histogram bins per pass (2 per thread at 1024 threads)

struct SelectShared {
  uint32_t hist[kSelBins];
  uint32_t wred[32][3];
  uint32_t bin, above;
};

// The k-th largest key T among the nonzero keys of the block, and how many keys equal to T the
// top k holds (need = k - #keys > T). take_all: at most k nonzero keys, all of them are chosen.
struct Threshold {
  uint32_t T, need;
  bool take_all;
};

// Radix select over an adaptive key range. The range starts as [min, max] of the keys; each pass
// splits the current range into at most kSelBins equal power-of-two bins, counts the keys of the
// range per bin, and narrows the range to the bin that holds the krem-th largest key. A range of
// up to 2^32 keys needs at most three passes (bin widths <= 2^21, <= 2^10, 1). `each(f)` calls
// f(key) for every key the calling thread owns; all threads of the block call these together.

// Count, minimum and maximum of the nonzero keys of the block.
template <class ForEach>
__device__ __forceinline__ void select_stats(ForEach each, SelectShared& sh, uint32_t& total, uint32_t& lo,
                                             uint32_t& hi) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  uint32_t c = 0, mn = 0xFFFFFFFFu, mx = 0u;
  each([&](uint32_t key) {
    if (key != 0u) {
      ++c;
      mn = min(mn, key);
      mx = max(mx, key);
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sh.wred[w][0] = c;
    sh.wred[w][1] = mn;
    sh.wred[w][2] = mx;
  }
  __syncthreads();
  // Every warp reduces the per-warp partials with shuffles (lane i reads warp i's).
  total = lane < nw ? sh.wred[lane][0] : 0u;
  lo = lane < nw ? sh.wred[lane][1] : 0xFFFFFFFFu;
  hi = lane < nw ? sh.wred[lane][2] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    total += __shfl_xor_sync(0xffffffffu, total, o);
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  __syncthreads();  // wred is reused by the first pass
}

// Exclusive prefix (in thread order) and total of one count per thread; wred[*][0] is scratch.
// All threads of the block call it; it ends with a barrier so wred can be reused.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, SelectShared& sh, uint32_t& total) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.wred[w][0] = incl;
  __syncthreads();
  uint32_t wv = lane < nw ? sh.wred[lane][0] : 0u;  // inclusive scan of the warp totals
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wv, o);
    if (lane >= o) wv += y;
  }
  total = __shfl_sync(0xffffffffu, wv, 31);
  const uint32_t before = w == 0 ? 0u : __shfl_sync(0xffffffffu, wv, w - 1);
  __syncthreads();
  return before + incl - v;
}

// One pass: narrow [lo, hi] (lo < hi) to the bin holding the krem-th largest key of the range.
// NT = threads of the block (each owns kSelBins / NT consecutive bins, in descending order).
template <int NT, class ForEach>
__device__ __forceinline__ void select_pass(ForEach each, SelectShared& sh, uint32_t& lo, uint32_t& hi,
                                            uint32_t& krem) {
  constexpr int BPT = kSelBins / NT;
  static_assert(BPT * NT == kSelBins, "bins per thread");
  const int tid = threadIdx.x;
  const uint32_t range = hi - lo;
  const int shift = range < (uint32_t)kSelBins ? 0 : (32 - __clz((int)range)) - kSelBits;
  const int nb = (int)(range >> shift) + 1;
  const uint32_t l0 = lo, h0r = hi;
  for (int i = tid; i < nb; i += NT) sh.hist[i] = 0u;
  __syncthreads();
  each([&](uint32_t key) {
    if (key >= l0 && key <= h0r) atomicAdd(&sh.hist[(key - l0) >> shift], 1u);
  });
  __syncthreads();
  // Thread t owns bins nb-1-t*BPT down to nb-(t+1)*BPT: a scan in thread order runs over
  // descending bins.
  uint32_t hb[BPT];
  uint32_t cnt = 0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    const int bin = nb - 1 - tid * BPT - k;
    hb[k] = bin >= 0 ? sh.hist[bin] : 0u;
    cnt += hb[k];
  }
  uint32_t tot;
  uint32_t run = block_excl_scan(cnt, sh, tot);
  if (run < krem && run + cnt >= krem) {
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      if (run + hb[k] >= krem) {
        sh.bin = (uint32_t)(nb - 1 - tid * BPT - k);
        sh.above = run;
        break;
      }
      run += hb[k];
    }
  }
  __syncthreads();
  krem -= sh.above;
  const uint32_t nlo = lo + (sh.bin << shift);
  hi = min(hi, nlo + ((1u << shift) - 1u));
  lo = nlo;
  __syncthreads();  // sh.bin / sh.above are rewritten by the next pass
}

template <class ForEach>
__device__ Threshold select_threshold(int k, ForEach each, SelectShared& sh) {
  uint32_t total, lo, hi;
  select_stats(each, sh, total, lo, hi);
  Threshold r;
  if (total <= (uint32_t)k) {
    r.take_all = true;
    r.T = 1u;
    r.need = 0u;
    return r;
  }
  uint32_t krem = (uint32_t)k;  // rank of T counted from the top of [lo, hi]
  while (lo != hi) select_pass<1024>(each, sh, lo, hi, krem);
  r.take_all = false;
  r.T = lo;
  r.need = krem;
  return r;
}

struct TopkShared {
  SelectShared sel;
  uint32_t warp_tot[32][2];
};

// Exclusive prefix of two per-thread counts across the block (thread order), and the totals.
__device__ __forceinline__ void block_scan2(uint32_t a, uint32_t b, TopkShared& sh, uint32_t& pre_a, uint32_t& pre_b,
                                            uint32_t& tot_a, uint32_t& tot_b) {
  pre_a = block_excl_scan(a, sh.sel, tot_a);
  pre_b = block_excl_scan(b, sh.sel, tot_b);
}

// Select the top k of the n keys key_of(i) (0 = empty position) with ties to the lower position,
// and call emit(pos, i) for the chosen positions in increasing i (pos = 0, 1, ...). Returns the
// count. Each thread owns the contiguous positions [tid*per, tid*per + per); keys are re-read on
// every pass, so key_of should read memory that stays in cache.
template <class KeyFn, class EmitFn>
__device__ uint32_t block_topk(int n, int k, KeyFn key_of, EmitFn emit, TopkShared& sh) {
  const int tid = threadIdx.x;
  const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  const Threshold th = select_threshold(k, [&](auto&& f) {
    for (int i = lo; i < hi; ++i) f(key_of(i));
  }, sh.sel);
  // Compaction in index order: keep every key > T and the first `need` keys == T.
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = lo; i < hi; ++i) {
    const uint32_t key = key_of(i);
    if (key == 0u) continue;
    if (th.take_all || key > th.T) ++n_gt;
    else if (key == th.T) ++n_eq;
  }
  uint32_t pre_gt, pre_eq, tot_gt, tot_eq;
  block_scan2(n_gt, n_eq, sh, pre_gt, pre_eq, tot_gt, tot_eq);
  uint32_t eq_seen = pre_eq;                            // keys == T before this thread's range
  uint32_t pos = pre_gt + min(pre_eq, th.need);         // output slot of the next selected key
  for (int i = lo; i < hi; ++i) {
    const uint32_t key = key_of(i);
    if (key == 0u) continue;
    if (th.take_all || key > th.T) {
      emit(pos++, i);
    } else if (key == th.T) {
      if (eq_seen < th.need) emit(pos++, i);
      ++eq_seen;
    }
  }
  return tot_gt + min(tot_eq, th.need);
}

constexpr int kCandCap = 4096;   // keys of the threshold bin after the first pass, kept in smem
constexpr int kRankMax = 128;    // at most this many: the threshold is found by ranking them directly

struct TopkRegShared {
  TopkShared t;
  uint32_t cand[kCandCap];
  uint32_t ncand;
  uint32_t T, need;                // threshold found by ranking the candidates
};

// Exclusive prefix (in thread order) and totals of two per-thread counts below 2^16 each, with
// one block scan of the packed pair (the totals stay below 2^16: no carry between the halves).
__device__ __forceinline__ void block_scan2_packed(uint32_t a, uint32_t b, SelectShared& sh, uint32_t& pre_a,
                                                   uint32_t& pre_b, uint32_t& tot_a, uint32_t& tot_b) {
  uint32_t tot;
  const uint32_t pre = block_excl_scan((a << 16) | b, sh, tot);
  pre_a = pre >> 16;
  pre_b = pre & 0xFFFFu;
  tot_a = tot >> 16;
  tot_b = tot & 0xFFFFu;
}

// Top-k of up to KPT * blockDim keys held in registers (0 = empty position); thread t holds the
// keys of positions t*KPT .. t*KPT+KPT-1. The first radix pass runs over the registers; the keys
// left in the threshold bin (usually a few dozen) are then gathered into shared memory and the
// remaining passes run over that list. Chosen positions are passed to emit(pos, r) (r = slot in
// the thread's registers) with pos = 0, 1, ... in increasing position. Returns the count.
template <int NT, int KPT, class EmitFn>
__device__ uint32_t block_topk_regs(const uint32_t (&key)[KPT], int k, EmitFn emit, TopkRegShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31;
  auto regs = [&](auto&& f) {
#pragma unroll
    for (int r = 0; r < KPT; ++r) f(key[r]);
  };
  uint32_t total, lo, hi;
  select_stats(regs, sh.t.sel, total, lo, hi);
  const bool take_all = total <= (uint32_t)k;
  uint32_t krem = (uint32_t)k;
  if (!take_all && lo != hi) {
    select_pass<NT>(regs, sh.t.sel, lo, hi, krem);
    if (lo != hi) {
      if (tid == 0) sh.ncand = 0;
      __syncthreads();
      // The keys left in [lo, hi] go to shared memory: one counter update per warp.
      const uint32_t lt = (1u << lane) - 1u;
      uint32_t bal[KPT];
      uint32_t wcnt = 0;
#pragma unroll
      for (int r = 0; r < KPT; ++r) {
        bal[r] = __ballot_sync(0xffffffffu, key[r] >= lo && key[r] <= hi);
        wcnt += (uint32_t)__popc(bal[r]);
      }
      uint32_t base = 0;
      if (lane == 0 && wcnt != 0u) base = atomicAdd(&sh.ncand, wcnt);
      base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
      for (int r = 0; r < KPT; ++r) {
        const uint32_t pos = base + (uint32_t)__popc(bal[r] & lt);
        if (((bal[r] >> lane) & 1u) && pos < (uint32_t)kCandCap) sh.cand[pos] = key[r];
        base += (uint32_t)__popc(bal[r]);
      }
      __syncthreads();
      const uint32_t nc = sh.ncand;
      if (nc <= (uint32_t)kRankMax) {
        // Few candidates: the krem-th largest of them is the key c with g < krem <= g + e, where g
        // (e) counts the candidates greater than (equal to) c; need = krem - g. (Each candidate's
        // thread reads all nc: worth it only while nc is small.)
        if (tid < (int)nc) {
          const uint32_t c = sh.cand[tid];
          uint32_t g = 0, e = 0;
          for (uint32_t j = 0; j < nc; ++j) {
            const uint32_t x = sh.cand[j];
            g += x > c ? 1u : 0u;
            e += x == c ? 1u : 0u;
          }
          if (g < krem && krem <= g + e) {  // every thread holding T writes the same values
            sh.T = c;
            sh.need = krem - g;
          }
        }
        __syncthreads();
        lo = hi = sh.T;
        krem = sh.need;
      } else if (nc <= (uint32_t)kCandCap) {
        auto list = [&](auto&& f) {
          for (uint32_t i = tid; i < nc; i += NT) f(sh.cand[i]);
        };
        while (lo != hi) select_pass<NT>(list, sh.t.sel, lo, hi, krem);
      } else {
        while (lo != hi) select_pass<NT>(regs, sh.t.sel, lo, hi, krem);
      }
    }
  }
  // Compaction in position order: keep every key > T and the first `need` keys == T.
  const uint32_t T = take_all ? 1u : lo;
  const uint32_t need = take_all ? 0u : krem;
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int r = 0; r < KPT; ++r) {
    if (key[r] == 0u) continue;
    if (take_all || key[r] > T) ++n_gt;
    else if (key[r] == T) ++n_eq;
  }
  static_assert(KPT * NT < 65536, "packed counts");
  uint32_t pre_gt, pre_eq, tot_gt, tot_eq;
  block_scan2_packed(n_gt, n_eq, sh.t.sel, pre_gt, pre_eq, tot_gt, tot_eq);
  uint32_t eq_seen = pre_eq;                       // keys == T before this thread's range
  uint32_t pos = pre_gt + min(pre_eq, need);       // output slot of the next chosen key
#pragma unroll
  for (int r = 0; r < KPT; ++r) {
    if (key[r] == 0u) continue;
    if (take_all || key[r] > T) {
      emit(pos++, r);
    } else if (key[r] == T) {
      if (eq_seen < need) emit(pos++, r);
      ++eq_seen;
    }
  }
  return tot_gt + min(tot_eq, need);
}

// Loads the keys of positions [t*KPT, t*KPT+KPT) of a score row of n entries (0 past the end).
template <int KPT>
__device__ __forceinline__ void load_keys(const float* row, int n, bool vec, uint32_t (&key)[KPT]) {
  const int p0 = (int)threadIdx.x * KPT;
  if (vec && p0 + KPT <= n) {
#pragma unroll
    for (int v = 0; v < KPT / 4; ++v) {
      const float4 f = reinterpret_cast<const float4*>(row + p0)[v];
      key[4 * v + 0] = score_key(f.x);
      key[4 * v + 1] = score_key(f.y);
      key[4 * v + 2] = score_key(f.z);
      key[4 * v + 3] = score_key(f.w);
    }
  } else {
#pragma unroll
    for (int r = 0; r < KPT; ++r) key[r] = p0 + r < n ? score_key(row[p0 + r]) : 0u;
  }
}

template <int NT, int KPT>
__device__ void topk_chunk(const TopkParams& P, TopkRegShared& sh) {
  const int q = blockIdx.y;
  const int c = blockIdx.x;
  const int t = P.q_pos[q];
  int E = (t + 1) / P.ratio;
  if (E > P.max_entries) {
    if (threadIdx.x == 0 && c == 0) record_status(P.status, CSA_DEV_BOUNDS);
    E = P.max_entries;
  }
  if (E < 0) E = 0;
  const int nchunks = (E + P.chunk - 1) / P.chunk;
  const int lo = c * P.chunk;
  const int n = max(0, min(E - lo, P.chunk));
  int32_t* out = P.out + (long long)q * P.topk;
  if (nchunks <= 1) {
    if (c != 0) return;
  } else if (c >= nchunks) {
    // No entries here: mark the slot empty for the merge.
    if (threadIdx.x == 0) P.cand_cnt[(long long)q * P.max_chunks + c] = 0;
    return;
  }
  const float* row = P.scores + (long long)q * P.scores_stride + lo;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
  uint32_t key[KPT];
  load_keys<KPT>(row, n, vec, key);
  const int p0 = lo + (int)threadIdx.x * KPT;
  if (nchunks <= 1) {
    const uint32_t cnt = block_topk_regs<NT, KPT>(key, P.topk, [&](uint32_t pos, int r) { out[pos] = p0 + r; }, sh);
    for (int j = cnt + threadIdx.x; j < P.topk; j += blockDim.x) out[j] = -1;
  } else {
    const long long cb = ((long long)q * P.max_chunks + c) * P.topk;
    uint32_t* ck = P.cand_key + cb;
    int32_t* ci = P.cand_idx + cb;
    const uint32_t cnt = block_topk_regs<NT, KPT>(key, P.topk, [&](uint32_t pos, int r) {
      ck[pos] = key[r];
      ci[pos] = p0 + r;
    }, sh);
    if (threadIdx.x == 0) P.cand_cnt[(long long)q * P.max_chunks + c] = (int)cnt;
  }
}

}  // namespace

// One CTA per (query, chunk). Chunk c of query q covers entries [c*chunk, min(E, (c+1)*chunk)).
// Single-chunk queries write the final list; otherwise the chunk's top-k (key, index) pairs go to
// the candidate buffers for topk_merge_kernel.
__global__ void __launch_bounds__(kTopkThreads) topk_chunk_kernel(TopkParams P) {
  __shared__ TopkRegShared sh;
  timeline_mark(P.status, kTlTopk, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlTopk, kTlReady);
  // Rows of <= kTopkShortRow entries hold 8 keys per thread, chunks of kTopkChunk entries 16.
  if (P.max_entries <= kTopkShortRow) topk_chunk<kTopkShortThreads, kTopkShortRow / kTopkShortThreads>(P, sh);
  else topk_chunk<kTopkThreads, kTopkChunk / kTopkThreads>(P, sh);
  timeline_mark(P.status, kTlTopk, kTlExit);
}

// One CTA per query with more than one chunk: top-k over the union of the chunks' lists. The
// lists are in ascending index order and chunk order is index order, so position order in the
// concatenation is index order (unused slots are marked invalid).
__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(TopkParams P) {
  __shared__ TopkRegShared sh;
  __shared__ int cnts[kTopkMaxChunks];
  timeline_mark(P.status, kTlTopkMerge, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlTopkMerge, kTlReady);
  const int q = blockIdx.x;
  const int t = P.q_pos[q];
  int E = (t + 1) / P.ratio;
  if (E > P.max_entries) E = P.max_entries;
  if (E < 0) E = 0;
  const int nchunks = (E + P.chunk - 1) / P.chunk;
  if (nchunks <= 1) return;
  for (int c = threadIdx.x; c < nchunks; c += blockDim.x) cnts[c] = P.cand_cnt[(long long)q * P.max_chunks + c];
  __syncthreads();
  const long long cb = (long long)q * P.max_chunks * P.topk;
  const uint32_t* ck = P.cand_key + cb;
  const int32_t* ci = P.cand_idx + cb;
  const int n = nchunks * P.topk;
  const int K = P.topk;
  auto key_of = [&](int i) -> uint32_t { return (i % K) < cnts[i / K] ? ck[i] : 0u; };
  int32_t* out = P.out + (long long)q * P.topk;
  uint32_t cnt;
  constexpr int KPT = kTopkChunk / kTopkThreads;
  if (n <= KPT * kTopkThreads) {
    // The union fits the registers (16 per thread): the same register-resident select as a chunk.
    // Thread t holds positions [t*KPT, t*KPT + KPT) of the concatenation.
    uint32_t key[KPT];
    int32_t idx[KPT];
    const int p0 = (int)threadIdx.x * KPT;
    if (K % KPT == 0 && p0 + KPT <= n) {
      // The thread's positions lie in one chunk's list: one count check, vector loads of the keys
      // and of their indices.
      const int c = p0 / K, s0 = p0 % K;
      const uint4* src = reinterpret_cast<const uint4*>(ck + p0);
      const int4* isrc = reinterpret_cast<const int4*>(ci + p0);
#pragma unroll
      for (int v = 0; v < KPT / 4; ++v) {
        const uint4 u = src[v];
        const int4 iv = isrc[v];
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        const int32_t i4[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          key[4 * v + e] = (s0 + 4 * v + e) < cnts[c] ? w4[e] : 0u;
          idx[4 * v + e] = i4[e];
        }
      }
    } else {
#pragma unroll
      for (int r = 0; r < KPT; ++r) {
        key[r] = p0 + r < n ? key_of(p0 + r) : 0u;
        idx[r] = key[r] != 0u ? ci[p0 + r] : -1;
      }
    }
    cnt = block_topk_regs<kTopkThreads, KPT>(key, P.topk, [&](uint32_t pos, int r) { out[pos] = idx[r]; }, sh);
  } else {
    cnt = block_topk(n, P.topk, key_of, [&](uint32_t pos, int i) { out[pos] = ci[i]; }, sh.t);
  }
  for (int j = cnt + threadIdx.x; j < P.topk; j += blockDim.x) out[j] = -1;
  timeline_mark(P.status, kTlTopkMerge, kTlExit);
}

}  // namespace csa
