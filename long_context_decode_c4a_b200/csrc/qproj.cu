// qproj.cu -- the low-rank query path in front of the layer (the contractions run in gemm_kernel).
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", section "低秩 Q：两次矩阵乘法接起来":
//   qr = rms_norm(X . Wq_a^T)                       X [M, hidden], Wq_a [q_rank, hidden]
//   q  = (qr . Wq_b^T).reshape(M, H, 512)           Wq_b [H*512, q_rank]
//   q  = q / sqrt(mean(q*q over each head) + eps)   (no weight)
//   q[..., -64:] = RoPE(q[..., -64:], position)
// rmsnorm_rows_kernel normalises the fp32 rows of X . Wq_a^T (weight gamma) into bf16 qr;
// head_norm_rope_kernel normalises each head of the bf16 product in place and rotates its last
// rope_dim dims by the token's position (adjacent pairs, theta_i = base^(-2i/rope_dim)). Without the
// normalisation it is the rotation of the window row after its down-projection ("图解DeepSeek V4：
// 详细计算流程解析" §2: the KV row [hidden] -> [head_dim], then RoPE on rope_dim dims).

#include "kernels.cuh"
#include "ptx.cuh"
#include "rope.cuh"

namespace csa {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

}  // namespace

// One CTA of kRowNormThreads per row: y = gamma * x / sqrt(mean(x^2) + eps), stored as bf16.
__global__ void __launch_bounds__(kRowNormThreads) rmsnorm_rows_kernel(const float* x, const uint16_t* gamma,
                                                                       uint16_t* y, int n, float eps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float part[kRowNormThreads / 32];
  const float* row = x + (long long)blockIdx.x * n;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n; i += kRowNormThreads) ss += row[i] * row[i];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kRowNormThreads / 32; ++w) tot += part[w];
  const float inv = rsqrtf(tot / (float)n + eps);
  uint16_t* out = y + (long long)blockIdx.x * n;
  for (int i = threadIdx.x; i < n; i += kRowNormThreads) {
    const float g = __uint_as_float((uint32_t)gamma[i] << 16);
    const uint32_t p = pack2(row[i] * inv * g, 0.f);
    out[i] = (uint16_t)(p & 0xFFFFu);
  }
}

// One warp per (row, head) of d = 512 bf16 values: lane l holds dims [16 l, 16 l + 16).
__global__ void __launch_bounds__(kHeadNormThreads) head_norm_rope_kernel(HeadNormParams P) {
  pdl_wait();
  pdl_trigger();
  const long long item = (long long)blockIdx.x * (kHeadNormThreads / 32) + (threadIdx.x >> 5);
  if (item >= (long long)P.M * P.H) return;
  const int lane = threadIdx.x & 31;
  const long long m = item / P.H;
  uint4* p = reinterpret_cast<uint4*>(P.q + item * 512) + 2 * lane;
  const uint4 a = p[0], b = p[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
  if (P.normalize) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) ss += v[i] * v[i];
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / 512.f + P.eps);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] *= inv;
  }
  const int dim0 = 16 * lane;
  const int rope0 = 512 - P.rope_dim;
  if (dim0 + 16 > rope0) {
    const long long t = P.pos[m];
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const int dim = dim0 + i;
      if (dim >= rope0) {
        float c, s;
        rope_cos_sin(t, P.inv_freq[(dim - rope0) >> 1], &c, &s);
        const float e = v[i], o = v[i + 1];
        v[i] = e * c - o * s;
        v[i + 1] = e * s + o * c;
      }
    }
  }
  p[0] = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
  p[1] = make_uint4(pack2(v[8], v[9]), pack2(v[10], v[11]), pack2(v[12], v[13]), pack2(v[14], v[15]));
}

}  // namespace csa
