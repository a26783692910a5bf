// compress.cu -- the C4A / C128A token compressor (K1).
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", sections "压缩是逐通道的 learned pooling" and
// "压缩条目必须等整组完成后才可见"; "图解DeepSeek V4：详细计算流程解析" §2.1 (C4A rolling state) and
// §3.1 (C128A).
//
// Entry g pools, per channel c, a softmax over slots of the score stream times the kv stream:
//   C4A  (ratio 4, overlap): 8 slots = channels [:d] of tokens 4(g-1)..4g-1 and channels [d:] of
//        tokens 4g..4g+3; the previous-group slots of g = 0 are missing (weight 0).
//   C128A (ratio 128): the 128 tokens of group g, one width-d stream.
// then RMSNorm over the d channels and RoPE on the last rope_dim channels at position g*ratio.
//
// Decode (one token per request): compress_decode_kernel, one CTA per (request, stream), feeds the
// token to the rolling state and pools the group it completes (the fused CSA decode step runs the
// same body inside the indexer launch); for C128A with d = 512, compress_decode_c128_kernel spreads
// a request's 128 rows x 512 channels over a cluster of 8 channel-block CTAs. Segments (prefill):
// compress_kernel, one CTA per (request, completed group), each thread owning 8 consecutive
// channels read with 16-byte loads, then compress_state_kernel for the final state. Memory-bound:
// no tensor-core work here.

#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "rope.cuh"
#include "compress_decode.cuh"

namespace csa {

namespace {

// Where token p's stream row comes from: the segment (element offset into the kv/score inputs,
// *from_state = false), a row of the input state (offset into the state arrays, *from_state =
// true), or nowhere (-1: a previous group before position 0).
__device__ __forceinline__ long long token_row(const CompressParams& P, int b, long long p, long long start,
                                               bool* from_state) {
  *from_state = false;
  if (p < 0) return -1;
  const int width = (1 + P.overlap) * P.d;
  if (p >= start) return ((long long)b * P.S + (p - start)) * width;
  *from_state = true;
  const long long g0 = start / P.ratio;  // group in progress at the segment start
  const int rows = (1 + P.overlap) * P.ratio;
  const long long st = (long long)b * rows * width;
  if (P.overlap) {
    if (p / P.ratio == g0) return st + (long long)(P.ratio + p % P.ratio) * width;  // cur rows
    if (p / P.ratio == g0 - 1) return st + (long long)(p % P.ratio) * width;        // pre rows
    return -1;
  }
  if (p / P.ratio == g0) return st + (long long)(p % P.ratio) * width;
  return -1;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int nw = (blockDim.x + 31) >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}

// Update request b's state to the state after token end-1, as the token-by-token rolling state
// leaves it. Called by one whole CTA. The only rows that feed other rows are the C4A cur rows
// that become pre rows when a group completes; those are read into registers before any row is
// written.
__device__ void update_state(const CompressParams& P, int b, long long start, long long end) {
  const int width = (1 + P.overlap) * P.d;
  const int rows = (1 + P.overlap) * P.ratio;
  uint16_t* skv = P.state_kv + (long long)b * rows * width;
  uint16_t* ssc = P.state_score + (long long)b * rows * width;
  const int cpr = width / 8;                    // 16-byte chunks per row
  const long long g0 = start / P.ratio;
  const long long g_end = end / P.ratio;        // groups 0..g_end-1 are complete after the segment
  const long long last = end - 1;
  const bool roll = P.overlap && g_end > g0;
  // Phase A: stash pre-row values that come from the input cur rows.
  uint4 keep_kv[kMaxKeepChunks], keep_sc[kMaxKeepChunks];
  if (roll) {
    int k = 0;
    for (int idx = threadIdx.x; idx < P.ratio * cpr && k < kMaxKeepChunks; idx += blockDim.x, ++k) {
      const int row = idx / cpr, ch = idx % cpr;
      const long long p = (g_end - 1) * P.ratio + row;
      if (p < start) {
        keep_kv[k] = *reinterpret_cast<const uint4*>(skv + (long long)(P.ratio + row) * width + ch * 8);
        keep_sc[k] = *reinterpret_cast<const uint4*>(ssc + (long long)(P.ratio + row) * width + ch * 8);
      }
    }
  }
  __syncthreads();
  // Phase B: every row whose newest token lies in the segment is copied from the segment.
  for (int idx = threadIdx.x; idx < rows * cpr; idx += blockDim.x) {
    const int row = idx / cpr, ch = idx % cpr;
    int j;
    if (P.overlap) {
      if (row < P.ratio) continue;  // pre rows: phase C
      j = row - P.ratio;
    } else {
      j = row;
    }
    const long long q = last - (((last - j) % P.ratio) + P.ratio) % P.ratio;  // newest token with q%ratio == j
    if (q < start) continue;                                                   // unchanged
    const long long off = ((long long)b * P.S + (q - start)) * width + ch * 8;
    *reinterpret_cast<uint4*>(skv + (long long)row * width + ch * 8) = *reinterpret_cast<const uint4*>(P.kv + off);
    *reinterpret_cast<uint4*>(ssc + (long long)row * width + ch * 8) = *reinterpret_cast<const uint4*>(P.score + off);
  }
  // Phase C: C4A pre rows <- the tokens of the last group completed in the segment.
  if (roll) {
    int k = 0;
    for (int idx = threadIdx.x; idx < P.ratio * cpr && k < kMaxKeepChunks; idx += blockDim.x, ++k) {
      const int row = idx / cpr, ch = idx % cpr;
      const long long p = (g_end - 1) * P.ratio + row;
      uint4 vk, vs;
      if (p >= start) {
        const long long off = ((long long)b * P.S + (p - start)) * width + ch * 8;
        vk = *reinterpret_cast<const uint4*>(P.kv + off);
        vs = *reinterpret_cast<const uint4*>(P.score + off);
      } else {
        vk = keep_kv[k];
        vs = keep_sc[k];
      }
      *reinterpret_cast<uint4*>(skv + (long long)row * width + ch * 8) = vk;
      *reinterpret_cast<uint4*>(ssc + (long long)row * width + ch * 8) = vs;
    }
  }
}

}  // namespace

// Segments of S > 1 tokens (prefill): grid (group slots, B, streams); block kCompressThreads.
// compress_state_kernel then brings the state to the end of the segment.
__global__ void __launch_bounds__(kCompressThreads) compress_kernel(CompressLaunch L) {
  pdl_wait();
  pdl_trigger();
  const CompressParams& P = L.p[blockIdx.z];
  const int b = blockIdx.y;
  if (b >= P.B) return;
  __shared__ float red[kCompressThreads / 32];
  __shared__ float rope_cs[2 * kMaxRopePairs];

  const long long start = P.start_pos[b];
  const long long end = start + P.S;
  const long long g_first = start / P.ratio;
  const long long g_last = end / P.ratio - 1;  // last group completed inside the segment
  const long long g = g_first + blockIdx.x;
  const int d = P.d;
  const int tid = threadIdx.x;
  const bool active = tid < d / 8;
  const int c0 = tid * 8;

  if (g <= g_last) {
    if (g >= P.max_entries) {
      if (tid == 0) record_status(P.status, CSA_DEV_BOUNDS);
    } else {
      // Per-channel online softmax over the slots, in the log2 domain. Slots are processed in
      // blocks of 8 whose 16-byte loads are all issued before any arithmetic.
      float m[8], s[8], acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        m[i] = -CUDART_INF_F;
        s[i] = 0.f;
        acc[i] = 0.f;
      }
      const int nslots = P.overlap ? 2 * P.ratio : P.ratio;
      if (active) {
        for (int j0 = 0; j0 < nslots; j0 += 8) {
          uint4 kraw[8], sraw[8];
          bool have[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + u;
            long long p;
            int coff;
            if (P.overlap) {
              const bool prev = j < P.ratio;
              p = prev ? (g - 1) * P.ratio + j : g * P.ratio + (j - P.ratio);
              coff = prev ? c0 : d + c0;
            } else {
              p = g * P.ratio + j;
              coff = c0;
            }
            bool from_state;
            const long long off = token_row(P, b, p, start, &from_state);
            have[u] = off >= 0;  // a missing slot has weight exactly 0 and is never read
            if (have[u]) {
              kraw[u] = *reinterpret_cast<const uint4*>((from_state ? P.state_kv : P.kv) + off + coff);
              sraw[u] = *reinterpret_cast<const uint4*>((from_state ? P.state_score : P.score) + off + coff);
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (!have[u]) continue;
            const uint32_t kw[4] = {kraw[u].x, kraw[u].y, kraw[u].z, kraw[u].w};
            const uint32_t sw[4] = {sraw[u].x, sraw[u].y, sraw[u].z, sraw[u].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float kvv = __uint_as_float((i & 1) ? (kw[i >> 1] & 0xFFFF0000u) : (kw[i >> 1] << 16));
              const float scv = __uint_as_float((i & 1) ? (sw[i >> 1] & 0xFFFF0000u) : (sw[i >> 1] << 16));
              const float x = scv * 1.4426950408889634f;  // log2(e)
              if (x > m[i]) {
                const float a = exp2f(m[i] - x);
                s[i] *= a;
                acc[i] *= a;
                m[i] = x;
              }
              const float e = exp2f(x - m[i]);
              s[i] += e;
              acc[i] += e * kvv;
            }
          }
        }
      }
          float x[8];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[i] = active ? acc[i] / s[i] : 0.f;
        ss += x[i] * x[i];
      }
      const float tot = block_sum(ss, red);
          const float r = rsqrtf(tot / (float)d + P.eps);
      // RoPE table for position g*ratio.
      const int npairs = P.rope_dim / 2;
      if (tid < npairs) {
        float cs, sn;
        rope_cos_sin(g * P.ratio, P.inv_freq[tid], &cs, &sn);
        rope_cs[2 * tid] = cs;
        rope_cs[2 * tid + 1] = sn;
      }
      __syncthreads();
          if (active) {
        const Vec8 gm = load8(P.gamma + c0);
        float y[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[i] * r * gm.v[i];
        const int rope0 = d - P.rope_dim;
        if (c0 >= rope0) {
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const int pi = (c0 + i - rope0) >> 1;
            const float cs = rope_cs[2 * pi], sn = rope_cs[2 * pi + 1];
            const float e = y[i], o = y[i + 1];
            y[i] = e * cs - o * sn;
            y[i + 1] = e * sn + o * cs;
          }
        }
        uint16_t* dst = P.cache + (long long)b * P.cache_bstride + g * d + c0;
        uint4 out;
        out.x = pack_bf16x2(y[0], y[1]);
        out.y = pack_bf16x2(y[2], y[3]);
        out.z = pack_bf16x2(y[4], y[5]);
        out.w = pack_bf16x2(y[6], y[7]);
        *reinterpret_cast<uint4*>(dst) = out;
        if (P.cache_f32 != nullptr) {
          float* df = P.cache_f32 + (long long)b * P.cache_bstride + g * d + c0;
          reinterpret_cast<float4*>(df)[0] = make_float4(y[0], y[1], y[2], y[3]);
          reinterpret_cast<float4*>(df)[1] = make_float4(y[4], y[5], y[6], y[7]);
        }
      }
    }
  }

}

// ---------------------------------------------------------------------------------- decode (S == 1)
//

// grid: (B, streams); block: kCompressThreads. Decode step (S == 1) with the state update fused.
__global__ void __launch_bounds__(kCompressThreads) compress_decode_kernel(CompressLaunch L) {
  __shared__ DecodePartial part[kCompressThreads];
  __shared__ float red[kCompressThreads / 32];
  const CompressParams& P = blockIdx.y != 0 ? L.p[1] : L.p[0];
  timeline_mark(P.status, kTlCompress, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlCompress, kTlReady);
  const int b = blockIdx.x;
  if (b >= P.B) return;
  if (P.ratio == 4) {
    if (P.d == 512) compress_decode_body<4, 512>(P, b, part, red, threadIdx.x, -1, 1);
    else compress_decode_body<4, 128>(P, b, part, red, threadIdx.x, -1, 1);
  } else {
    if (P.d == 512) compress_decode_body<128, 512>(P, b, part, red, threadIdx.x, -1, 1);
    else compress_decode_body<128, 128>(P, b, part, red, threadIdx.x, -1, 1);
  }
  timeline_mark(P.status, kTlCompress, kTlExit);
}

// C128A decode step over a cluster of kC128Split CTAs per request (grid: (kC128Split, B)); CTA r of
// the cluster owns channels [r*CH, r*CH + CH) of the d = 512 (CH = 64, 8 chunks of 8). Thread t
// takes chunk t % 8 of the slots (t / 8) + 32k, k = 0..3: a warp load covers 128 contiguous bytes
// of each of 4 slot rows, and the CTA reads its 32 KB of state in one round of loads. The softmax
// over the 128 slots of each channel: the max over a thread's slots, across the warp (lanes 8
// apart share the channels) and across the warps (shared memory); then the terms against that max,
// summed the same way. The RMS over all d channels adds the CTAs' partial sums of squares through
// distributed shared memory. Token t's row (and the window row) go out as 16-byte slices; when t
// completes its group the state rows read are rows 0..126 (row 127 is token t's own row, taken
// from the input), so no write aliases a read.
__global__ void __cluster_dims__(kC128Split, 1, 1) __launch_bounds__(kCompressThreads)
    compress_decode_c128_kernel(CompressLaunch L) {
  constexpr int D = 512, RATIO = 128, CH = D / kC128Split, NCH = CH / 8;
  constexpr int kGroups = kCompressThreads / NCH;   // slot groups (32)
  constexpr int kPer = RATIO / kGroups;             // slots per thread (4)
  constexpr int kWarps = kCompressThreads / 32;
  static_assert(NCH == 8 && kGroups == 32 && kPer == 4, "thread layout");
  __shared__ float red_m[kWarps][CH];   // per-warp partial max, then partial sums of the terms
  __shared__ float red_a[kWarps][CH];   // per-warp partial weighted sums
  __shared__ float ch_m[CH];            // the channels' max
  __shared__ float ss_w[CH / 8];
  __shared__ float ss_all[kC128Split];  // every CTA's partial sum of squares, written by that CTA
  const CompressParams& P = L.p[0];
  cluster_arrive_relaxed();  // waited for before the first store into another CTA's shared memory
  timeline_mark(P.status, kTlCompress, kTlEntry);
  pdl_wait();
  pdl_trigger();
  timeline_mark(P.status, kTlCompress, kTlReady);
  const int b = blockIdx.y;                      // the same for every CTA of the cluster
  const int rank = (int)cluster_ctarank();
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int t = P.start_pos[b];
  if (t < 0) {
    if (tid == 0) record_status(P.status, CSA_DEV_BOUNDS);
    return;                                      // uniform over the cluster: no cluster barrier is skipped alone
  }
  const int g = t / RATIO;
  const int cur = t % RATIO;
  const bool done = cur == RATIO - 1;
  uint16_t* skv = P.state_kv + (size_t)b * RATIO * D;
  uint16_t* ssc = P.state_score + (size_t)b * RATIO * D;
  const uint16_t* xkv = P.kv + (size_t)b * D;
  const uint16_t* xsc = P.score + (size_t)b * D;
  const int ch0 = rank * CH;
  // Token t's row into state row `cur`, the window row into the ring: 16-byte slices of this CTA's
  // channels (threads 0-7, 8-15 and 16-23).
  if (tid < 3 * NCH) {
    const int part = tid / NCH, k = ch0 + 8 * (tid % NCH);
    if (part == 0) {
      *reinterpret_cast<uint4*>(skv + (size_t)cur * D + k) = *reinterpret_cast<const uint4*>(xkv + k);
    } else if (part == 1) {
      *reinterpret_cast<uint4*>(ssc + (size_t)cur * D + k) = *reinterpret_cast<const uint4*>(xsc + k);
    } else if (P.win_src != nullptr) {
      uint16_t* dst = P.ring + (long long)b * P.ring_bstride + (long long)(t % P.ring_cap) * D;
      *reinterpret_cast<uint4*>(dst + k) = *reinterpret_cast<const uint4*>(P.win_src + (size_t)b * D + k);
    }
  }
  if (!done) return;                             // uniform over the cluster
  if (g >= P.max_entries) {
    if (tid == 0) record_status(P.status, CSA_DEV_BOUNDS);
    return;
  }
  const int chunk = tid % NCH, grp = tid / NCH;
  const int c0 = ch0 + 8 * chunk;                // this thread's 8 channels
  uint4 kr[kPer], sr[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int j = grp + kGroups * k;
    const uint16_t* rk = j == RATIO - 1 ? xkv : skv + (size_t)j * D;
    const uint16_t* rs = j == RATIO - 1 ? xsc : ssc + (size_t)j * D;
    kr[k] = *reinterpret_cast<const uint4*>(rk + c0);
    sr[k] = *reinterpret_cast<const uint4*>(rs + c0);
  }
  // Max over the thread's slots (log2 domain), then over the lanes with the same chunk (xor 8,
  // 16), then over the warps.
  Vec8 kv[kPer], sc[kPer];
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = -CUDART_INF_F;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    kv[k] = load8_regs(kr[k]);
    sc[k] = load8_regs(sr[k]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[k].v[i] *= 1.4426950408889634f;  // log2(e)
      m[i] = fmaxf(m[i], sc[k].v[i]);
    }
  }
#pragma unroll
  for (int o = NCH; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], o));
  if (lane < NCH) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red_m[w][8 * chunk + i] = m[i];
  }
  __syncthreads();
  if (tid < CH) {
    float v = red_m[0][tid];
#pragma unroll
    for (int q = 1; q < kWarps; ++q) v = fmaxf(v, red_m[q][tid]);
    ch_m[tid] = v;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = ch_m[8 * chunk + i];
  // Terms against the max: their sum s and the weighted sum a, reduced the same way.
  float s[8], a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s[i] = 0.f;
    a[i] = 0.f;
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float e = exp2f(sc[k].v[i] - m[i]);
      s[i] += e;
      a[i] += e * kv[k].v[i];
    }
#pragma unroll
  for (int o = NCH; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s[i] += __shfl_xor_sync(0xffffffffu, s[i], o);
      a[i] += __shfl_xor_sync(0xffffffffu, a[i], o);
    }
  if (lane < NCH) {  // (every read of the maxima in red_m preceded the last barrier)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      red_m[w][8 * chunk + i] = s[i];
      red_a[w][8 * chunk + i] = a[i];
    }
  }
  __syncthreads();
  // Thread c < CH finishes channel ch0 + c: x = a / s, and its square for the RMS.
  float x = 0.f;
  if (tid < CH) {
    float S = 0.f, A = 0.f;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) {
      S += red_m[q][tid];
      A += red_a[q][tid];
    }
    x = A / S;
    float sq = x * x;
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if ((tid & 7) == 0) ss_w[tid >> 3] = sq;
  }
  __syncthreads();
  cluster_wait();  // every CTA of the cluster has started: its shared memory may be written
  if (tid < kC128Split) {
    // Thread r stores this CTA's partial into slot `rank` of CTA r's ss_all.
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < CH / 8; ++i) v += ss_w[i];
    st_cluster_f32(mapa_shared(smem_u32(&ss_all[rank]), (uint32_t)tid), v);
  }
  // Every partial has landed in every CTA's shared memory; nothing crosses CTAs after this
  // barrier, so a CTA may leave as soon as it is done.
  cluster_sync();
  if (tid >= CH) return;
  float tot = 0.f;
#pragma unroll
  for (int r = 0; r < kC128Split; ++r) tot += ss_all[r];
  // Channel c = ch0 + tid: RMSNorm, gamma, RoPE on the rotated channels (pairs in adjacent threads).
  const int c = ch0 + tid;
  const float gm = __uint_as_float((uint32_t)P.gamma[c] << 16);
  float y = x * rsqrtf(tot / (float)D + P.eps) * gm;
  const int rope0 = D - P.rope_dim;
  const float yo = __shfl_xor_sync(0xffffffffu, y, 1);   // the other element of the pair
  if (c >= rope0) {
    float cs, sn;
    rope_cos_sin((long long)g * RATIO, P.inv_freq[(c - rope0) >> 1], &cs, &sn);
    y = (c & 1) ? yo * sn + y * cs : y * cs - yo * sn;
  }
  // Pack pairs of channels: even threads store 2 bf16 (and 2 fp32).
  const float y1 = __shfl_xor_sync(0xffffffffu, y, 1);
  if ((tid & 1) == 0) {
    uint16_t* dst = P.cache + (long long)b * P.cache_bstride + (long long)g * D + c;
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(y, y1);
    if (P.cache_f32 != nullptr) {
      float* df = P.cache_f32 + (long long)b * P.cache_bstride + (long long)g * D + c;
      *reinterpret_cast<float2*>(df) = make_float2(y, y1);
    }
  }
  timeline_mark(P.status, kTlCompress, kTlExit);
}

// Final state of a multi-token segment: one CTA per request, reads before writes.
__global__ void __launch_bounds__(kCompressThreads) compress_state_kernel(CompressLaunch L) {
  pdl_wait();
  pdl_trigger();
  const CompressParams& P = L.p[blockIdx.z];
  const int b = blockIdx.x;
  if (b >= P.B) return;
  const long long start = P.start_pos[b];
  update_state(P, b, start, start + P.S);
}

// state <- kv rows 0, score rows -inf.
__global__ void state_reset_kernel(uint16_t* kv, uint16_t* score, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    kv[i] = 0;
    score[i] = 0xFF80;  // bf16 -inf
  }
}

}  // namespace csa
