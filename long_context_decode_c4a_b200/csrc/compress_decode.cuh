// compress_decode.cuh -- the body of the decode-step compressor (K1), shared by the compressor's
// own kernel and by kernels that run it on a group of 256 of their threads.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace csa {

struct Vec8 {
  float v[8];
};

__device__ __forceinline__ Vec8 load8(const uint16_t* p) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  Vec8 r;
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[2 * i] = __uint_as_float(w[i] << 16);
    r.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  return r;
}

__device__ __forceinline__ Vec8 load8_regs(const uint4 u) {
  Vec8 r;
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.v[2 * i] = __uint_as_float(w[i] << 16);
    r.v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One CTA per (request, stream) feeds token t = start_pos[b] to the rolling state and, when t
// completes group g = t / ratio, writes entry g. Work split: a slot row of D channels is read by
// C = D/8 threads (16 bytes each); the 256 threads form G = 256/C groups that take the slots
// round-robin, each keeping a per-channel partial softmax (max, sum, weighted sum) that group 0
// merges. Every read of the state (slots and the C4A roll) is issued before the first barrier,
// every write after it, so the kernel costs about two dependent memory round trips.

struct DecodePartial {
  float m[8], s[8], a[8];
};

// tid: the calling thread's index among the kCompressThreads threads that run the body. bar_all: the
// named barrier those threads share (-1: they are the whole CTA, __syncthreads); bar_norm: a named
// barrier for the first kNormThreads of them (the RMS reduction). part: kCompressThreads partials
// in shared memory; red: kCompressThreads / 32 floats in shared memory.
template <int RATIO, int D>
__device__ __forceinline__ void compress_decode_body(const CompressParams& P, int b, DecodePartial* part,
                                                     float* red, int tid, int bar_all, int bar_norm) {
  constexpr bool kOverlap = RATIO == 4;
  constexpr int C = D / 8;                        // chunk threads per slot row
  constexpr int G = kCompressThreads / C;          // slot groups
  constexpr int kWidth = kOverlap ? 2 * D : D;     // channels per state row
  constexpr int kRows = kOverlap ? 2 * RATIO : RATIO;
  constexpr int kSlots = kOverlap ? 2 * RATIO : RATIO;
  constexpr int kRowChunks = kWidth / 8;
  constexpr int kRollChunks = kOverlap ? RATIO * kRowChunks : 0;
  constexpr int kRollPer = (kRollChunks + kCompressThreads - 1) / kCompressThreads;
  constexpr int kPer = (kSlots + G - 1) / G;      // slots per thread
  constexpr int kBatch = kPer < 8 ? kPer : 8;
  static_assert(kCompressThreads % C == 0, "C must divide the block");
  const int c = tid % C, grp = tid / C;
  const int c0 = c * 8;
  const int t = P.start_pos[b];
  uint16_t* skv = P.state_kv + (size_t)b * kRows * kWidth;
  uint16_t* ssc = P.state_score + (size_t)b * kRows * kWidth;
  const uint16_t* xkv = P.kv + (size_t)b * kWidth;  // token t's row (S == 1)
  const uint16_t* xsc = P.score + (size_t)b * kWidth;
  // C4A reads its state rows before t is known: if t completes a group, token t is the last cur
  // row (row 2*RATIO-1), so every slot and roll source is fixed; when t does not complete a group
  // the values read are not used. C128A reads its (many) rows only for completing tokens.
  constexpr int kLastRow = kRows - 1;
  // Token t's row, written to state row `cur` after the barrier.
  uint4 tok_kv = make_uint4(0, 0, 0, 0), tok_sc = make_uint4(0, 0, 0, 0);
  if (tid < kRowChunks) {
    tok_kv = *reinterpret_cast<const uint4*>(xkv + tid * 8);
    tok_sc = *reinterpret_cast<const uint4*>(xsc + tid * 8);
  }
  // C4A roll: after group g completes, pre rows <- cur rows (token t's row from the input).
  uint4 roll_kv[kRollPer > 0 ? kRollPer : 1], roll_sc[kRollPer > 0 ? kRollPer : 1];
  if (kOverlap) {
#pragma unroll
    for (int k = 0; k < kRollPer; ++k) {
      const int idx = tid + k * kCompressThreads;
      if (idx < kRollChunks) {
        const int row = RATIO + idx / kRowChunks, ch = idx % kRowChunks;
        const uint16_t* sk = row == kLastRow ? xkv : skv + (size_t)row * kWidth;
        const uint16_t* ss = row == kLastRow ? xsc : ssc + (size_t)row * kWidth;
        roll_kv[k] = *reinterpret_cast<const uint4*>(sk + ch * 8);
        roll_sc[k] = *reinterpret_cast<const uint4*>(ss + ch * 8);
      }
    }
  }
  if (t < 0) {
    if (tid == 0) record_status(P.status, CSA_DEV_BOUNDS);
    return;
  }
  const int g = t / RATIO;
  const int cur = kOverlap ? RATIO + t % RATIO : t % RATIO;  // state row of token t
  const bool done = (t + 1) % RATIO == 0;

  // Window-ring write of the fused decode step.
  if (P.win_src != nullptr && tid < D / 8) {
    uint16_t* dst = P.ring + (long long)b * P.ring_bstride + (long long)(t % P.ring_cap) * D;
    *reinterpret_cast<uint4*>(dst + c0) = *reinterpret_cast<const uint4*>(P.win_src + (size_t)b * D + c0);
  }
  // Partial softmax over this thread's slots, in the log2 domain.
  DecodePartial pt;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    pt.m[i] = -CUDART_INF_F;
    pt.s[i] = 0.f;
    pt.a[i] = 0.f;
  }
  if (kOverlap || done) {
#pragma unroll 1
    for (int k0 = 0; k0 < kPer; k0 += kBatch) {
      uint4 kraw[kBatch], sraw[kBatch];
      bool have[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = grp + (k0 + u) * G;       // slot index
        have[u] = j < kSlots && k0 + u < kPer;
        int row, coff;
        if (kOverlap) {
          row = j;                              // pre rows 0..RATIO-1 (channels [0, D)), cur rows after
          coff = j < RATIO ? c0 : D + c0;
        } else {
          row = j;
          coff = c0;
        }
        if (have[u]) {
          const uint16_t* sk = row == kLastRow ? xkv : skv + (size_t)row * kWidth;  // done: cur == kLastRow
          const uint16_t* ss = row == kLastRow ? xsc : ssc + (size_t)row * kWidth;
          kraw[u] = *reinterpret_cast<const uint4*>(sk + coff);
          sraw[u] = *reinterpret_cast<const uint4*>(ss + coff);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (!have[u]) continue;
        if (kOverlap && grp + (k0 + u) * G < RATIO && g == 0) continue;  // no group before group 0: weight 0
        const uint32_t kw[4] = {kraw[u].x, kraw[u].y, kraw[u].z, kraw[u].w};
        const uint32_t sw[4] = {sraw[u].x, sraw[u].y, sraw[u].z, sraw[u].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float kvv = __uint_as_float((i & 1) ? (kw[i >> 1] & 0xFFFF0000u) : (kw[i >> 1] << 16));
          const float x = __uint_as_float((i & 1) ? (sw[i >> 1] & 0xFFFF0000u) : (sw[i >> 1] << 16)) *
                          1.4426950408889634f;  // log2(e)
          if (x > pt.m[i]) {
            const float a = exp2f(pt.m[i] - x);
            pt.s[i] *= a;
            pt.a[i] *= a;
            pt.m[i] = x;
          }
          const float e = exp2f(x - pt.m[i]);
          pt.s[i] += e;
          pt.a[i] += e * kvv;
        }
      }
    }
    if (G > 1 && done) part[tid] = pt;
  }
  // Every state read above is complete before any state write below.
  if (bar_all < 0) __syncthreads();
  else named_bar_sync(bar_all, kCompressThreads);

  if (tid < kRowChunks) {
    *reinterpret_cast<uint4*>(skv + (size_t)cur * kWidth + tid * 8) = tok_kv;
    *reinterpret_cast<uint4*>(ssc + (size_t)cur * kWidth + tid * 8) = tok_sc;
  }
  if (kOverlap && done) {
#pragma unroll
    for (int k = 0; k < kRollPer; ++k) {
      const int idx = tid + k * kCompressThreads;
      if (idx < kRollChunks) {
        const int row = idx / kRowChunks, ch = idx % kRowChunks;
        *reinterpret_cast<uint4*>(skv + (size_t)row * kWidth + ch * 8) = roll_kv[k];
        *reinterpret_cast<uint4*>(ssc + (size_t)row * kWidth + ch * 8) = roll_sc[k];
      }
    }
  }
  if (!done) return;
  if (g >= P.max_entries) {
    if (tid == 0) record_status(P.status, CSA_DEV_BOUNDS);
    return;
  }
  // Group 0 merges the partials of its 8 channels; warps 0..(C-1)/32 then normalise and store.
  constexpr int kNormThreads = C < 32 ? 32 : C;
  if (tid >= kNormThreads) return;
  float x[8];
  float ss = 0.f;
  if (tid < C) {
    if (G > 1) {
      float M[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) M[i] = pt.m[i];
      for (int q = 1; q < G; ++q) {
        const DecodePartial& o = part[q * C + c];
#pragma unroll
        for (int i = 0; i < 8; ++i) M[i] = fmaxf(M[i], o.m[i]);
      }
      float S[8], A[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float f = pt.m[i] == -CUDART_INF_F ? 0.f : exp2f(pt.m[i] - M[i]);
        S[i] = pt.s[i] * f;
        A[i] = pt.a[i] * f;
      }
      for (int q = 1; q < G; ++q) {
        const DecodePartial& o = part[q * C + c];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float f = o.m[i] == -CUDART_INF_F ? 0.f : exp2f(o.m[i] - M[i]);
          S[i] += o.s[i] * f;
          A[i] += o.a[i] * f;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = A[i] / S[i];
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = pt.a[i] / pt.s[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += x[i] * x[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (kNormThreads > 32) {
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    named_bar_sync(bar_norm, kNormThreads);
    ss = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) ss += red[i];
  }
  if (tid >= C) return;
  const float rs = rsqrtf(ss / (float)D + P.eps);
  const Vec8 gm = load8(P.gamma + c0);
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = x[i] * rs * gm.v[i];
  const int rope0 = D - P.rope_dim;
  if (c0 >= rope0) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float cs, sn;
      rope_cos_sin((long long)g * RATIO, P.inv_freq[(c0 + i - rope0) >> 1], &cs, &sn);
      const float e = y[i], o = y[i + 1];
      y[i] = e * cs - o * sn;
      y[i + 1] = e * sn + o * cs;
    }
  }
  uint16_t* dst = P.cache + (long long)b * P.cache_bstride + (long long)g * D + c0;
  uint4 out;
  out.x = pack_bf16x2(y[0], y[1]);
  out.y = pack_bf16x2(y[2], y[3]);
  out.z = pack_bf16x2(y[4], y[5]);
  out.w = pack_bf16x2(y[6], y[7]);
  *reinterpret_cast<uint4*>(dst) = out;
  if (P.cache_f32 != nullptr) {
    float* df = P.cache_f32 + (long long)b * P.cache_bstride + (long long)g * D + c0;
    reinterpret_cast<float4*>(df)[0] = make_float4(y[0], y[1], y[2], y[3]);
    reinterpret_cast<float4*>(df)[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
}


}  // namespace csa
