// pool_kernel.cuh -- block mean pooling of bf16 Q/K/V into fp32 block means.
//
// Step "mean-pooled query and key blocks" of Sol-Attn (paperlayer summary,
// §2 Preliminaries, Block-Sparse Attention: the block proxy is derived from the
// means of the query and key blocks) and the pooled values of the correction
// (§3 Methodology, Approximate correction: pooled keys and summed values).
//
// HBM-bound: every input byte is read once with 16-byte coalesced loads; the
// outputs are B*H*nB*d fp32 means and, for V, an fp16 copy that the attention
// kernel's P.V product reads (P is carried in fp16, whose 11-bit significand
// keeps the product's rounding error well inside the output tolerance; both MMA
// operands must share one type). One CTA of 128 threads reduces one block: D/8
// threads cover a row (8 bf16 each), 128/(D/8) rows are in flight per pass.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace solattn {

struct PoolJob {
  const __nv_bfloat16 *x;  // [BH][N][D]
  float *xbar;             // [BH][nB][D] block means, or null
  __half *x16;             // [BH][N][D] fp16 copy of x, or null
  int blk;                 // rows per block
  int nB;                  // ceil(N / blk)
};

struct PoolArgs {
  PoolJob job[3];
  int njobs;
  int N;
};

template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const PoolArgs args) {
  constexpr int TPR = D / 8;              // threads per row
  constexpr int RPP = 128 / TPR;          // rows per pass
  __shared__ float red[RPP][D + 4];

  const PoolJob &job = args.job[blockIdx.z];
  const int j = blockIdx.x;
  if (j >= job.nB) return;
  const int bh = blockIdx.y;
  const int N = args.N;
  const int start = j * job.blk;
  const int n = min(job.blk, N - start);
  const int c8 = threadIdx.x % TPR;
  const int r0 = threadIdx.x / TPR;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  const size_t off = (static_cast<size_t>(bh) * N + start) * D;
  const uint4 *src = reinterpret_cast<const uint4 *>(job.x + off) + c8;
  uint4 *dst16 = job.x16 ? reinterpret_cast<uint4 *>(job.x16 + off) + c8 : nullptr;
#pragma unroll 8
  for (int r = r0; r < n; r += RPP) {
    const uint4 w = __ldg(src + static_cast<size_t>(r) * (D / 8));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w);
    uint4 o16;
    __half2 *o = reinterpret_cast<__half2 *>(&o16);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
      o[e] = __floats2half2_rn(f.x, f.y);  // exact for |x| in [2^-14, 65504]
    }
    if (dst16) dst16[static_cast<size_t>(r) * (D / 8)] = o16;
  }
  if (!job.xbar) return;
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r0][c8 * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < RPP; ++g) s += red[g][threadIdx.x];
    job.xbar[(static_cast<size_t>(bh) * job.nB + j) * D + threadIdx.x] = s / static_cast<float>(n);
  }
}

// bf16 copy of the pooled keys and fp16 copy of the pooled values ([B*H][nKB][d], same
// layout as the fp32 arrays), the operands of the token-to-block correction tiles.
__global__ void __launch_bounds__(256) pooled_copy_kernel(const float *kbar, const float *vbar, __nv_bfloat16 *k16,
                                                          __half *v16, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    k16[i] = __float2bfloat16_rn(kbar[i]);
    v16[i] = __float2half_rn(vbar[i]);
  }
}

}  // namespace solattn
