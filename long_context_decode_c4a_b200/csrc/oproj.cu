// oproj.cu -- the grouped output projection on the tcgen05 tensor cores.
//
// "DeepSeek-V4-Pro 架构：一个 token 的旅程", section "输出投影也分组，并且降低中间维度": after the inverse
// RoPE, o [B, S, H, d] is viewed as [B*S, G, 8 d] (groups of 8 heads); each group is projected to
// R dims, r[:, g] = o[:, g] . Wo_a[g]^T with Wo_a [G, R, 8 d], and y = r.flatten(1) . Wo_b^T with
// Wo_b [D, G R] (Pro: G = 16, 8 d = 4096, R = 1024, D = 7168; 64 Mi + 112 Mi weights).
//
// gemm_kernel computes C = A . B^T for K-major bf16 A [M, K] and B [N, K], accumulating in fp32 in
// TMEM. A CTA owns a 128 x 128 tile of C and a range of K (split-K when the tiles alone would not
// cover the GPU); blockIdx.z selects the group and the K split. 4 warps: lane 0 of warp 0 streams
// 64-wide K blocks of A and B with TMA (128B swizzle) through kGemmStages stages, lane 0 of warp 1
// issues the 4 MMAs (M = 128, N = 128, K = 16) of each block and releases the stage when they
// complete, then all four warps read the accumulator (thread = TMEM lane = row of C) and store it:
// bf16, fp32, or an fp32 reduction into C when the K range is split. Rows past M (a partial last
// M tile) are read as zeros by TMA and not stored.

#include "kernels.cuh"
#include "ptx.cuh"

namespace csa {

namespace {

constexpr uint32_t kGemmTileBytes = 128 * 128;  // one operand block: 128 rows x 64 bf16 (128 B)
constexpr uint32_t kGemmStageBytes = 2 * kGemmTileBytes;

struct GemmSmem {
  uint64_t full[kGemmStages], empty[kGemmStages];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(base + kGemmStages * kGemmStageBytes);
  const int warp = warp_id();
  const int lane = lane_id();
  const int n0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * 128;
  const int g = blockIdx.z / P.splits;
  const int split = blockIdx.z % P.splits;
  const int kblocks = P.K / 64 / P.splits;          // K blocks of this CTA
  const int kb0 = split * kblocks;
  volatile int* abort_flag = &sm.abort_flag;
  uint32_t* status = P.status;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(&sm.done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  pdl_wait();
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    const int ax = g * P.a_group_cols, by = g * P.b_group_rows + n0;
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % kGemmStages;
      if (kb >= kGemmStages &&
          !mbar_wait(&sm.empty[s], (uint32_t)((kb / kGemmStages - 1) & 1), abort_flag, status, 301))
        break;
      uint8_t* st = base + (size_t)s * kGemmStageBytes;
      mbar_arrive_expect_tx(&sm.full[s], kGemmStageBytes);
      tma_load_2d(st, &map_a, ax + 64 * (kb0 + kb), m0, &sm.full[s]);
      tma_load_2d(st + kGemmTileBytes, &map_b, 64 * (kb0 + kb), by, &sm.full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
    int kb = 0;
    for (; kb < kblocks; ++kb) {
      const int s = kb % kGemmStages;
      if (!mbar_wait(&sm.full[s], (uint32_t)((kb / kGemmStages) & 1), abort_flag, status, 302)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(base + (size_t)s * kGemmStageBytes);
      const uint32_t b = a + kGemmTileBytes;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ss(tmem, smem_desc_sw128(a + 32 * ks, 16, 1024), smem_desc_sw128(b + 32 * ks, 16, 1024), idesc,
               (kb > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&sm.empty[s]);
    }
    if (kb < kblocks) *abort_flag = 1;
    // Every MMA issued above completes before `done` (also after an abort, before TMEM is freed).
    mma_commit(&sm.done);
  }
  __syncwarp();
  // -------------------------------------------------------------------- epilogue (all 4 warps)
  const bool ok = __all_sync(0xffffffffu, mbar_wait_drain(&sm.done, 0, status, 303)) && !*abort_flag;
  tc_fence_after();
  const int row = warp * 32 + lane;  // TMEM lane = row of the tile
  const int m = m0 + row;
  if (ok) {
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * cc, v);
      tmem_wait_ld();
      if (m < P.M) {
        const long long col = (long long)g * P.c_group_cols + n0 + 32 * cc;
        if (P.c_mode == kGemmOutBf16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.c) + (long long)m * P.ldc + col);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        } else {
          float* dst = static_cast<float*>(P.c) + (long long)m * P.ldc + col;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float a = __uint_as_float(v[4 * q]), b = __uint_as_float(v[4 * q + 1]);
            const float c = __uint_as_float(v[4 * q + 2]), d = __uint_as_float(v[4 * q + 3]);
            if (P.c_mode == kGemmOutF32)
              reinterpret_cast<float4*>(dst)[q] = make_float4(a, b, c, d);
            else
              red_add_v4(dst + 4 * q, a, b, c, d);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

__global__ void zero_f32_kernel(float* p, long long n4) {
  pdl_wait();
  pdl_trigger();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
    reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

size_t gemm_smem_bytes() { return 1024 + kGemmStages * (size_t)kGemmStageBytes + sizeof(GemmSmem); }

}  // namespace csa
