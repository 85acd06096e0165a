// route_kernels.cuh -- the routing stage on its own, for the routing-overhead measurement
// ("Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification", paperlayer summary §4 Experiments, "Efficient On-the-Fly Sparsification":
// routing that consumes the proxy scores on chip against top-k and top-p routing, which
// materialise the proxy map and traverse whole rows of it; §2 Block-Sparse Attention).
//
//   plan_kernel       (plan_kernel.cuh) Sol-Attn's running-max rule, the forward's own
//                     routing pass with its correction and schedule steps off: proxies of
//                     a group of query blocks in shared memory, keep bits out. No proxy
//                     leaves the chip.
//   proxy_map_kernel  s_ij = q_i . k_j / sqrt(d) for every (query block, key block), to HBM.
//   select_kernel     one CTA per proxy row: a bitonic sort of the row in shared memory,
//                     then top-k (the k largest proxies) or top-p (the heaviest blocks,
//                     mass n_j e^{s_ij}, until their share of the row reaches p).
// All three write keep bits in the layout of the forward operator's keep mask.
#pragma once

#include <cstdint>

#include "plan_kernel.cuh"

namespace solattn {

// smap[bh][i][j] = qbar[bh][i] . kbar[bh][j] / sqrt(D) in fp32. Grid (ceil(nKB / 64),
// ceil(nQB / 64), B*H), 256 threads, each a 4 x 4 block of outputs; 64-row tiles of the
// pooled queries and keys are staged in shared memory 32 dimensions at a time.
template <int D>
__global__ void __launch_bounds__(256) proxy_map_kernel(const float *qbar, const float *kbar, float *smap, int nQB,
                                                        int nKB) {
  __shared__ float qs[32][64 + 4];  // [dimension][row]
  __shared__ float ks[32][64 + 4];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const float *qb = qbar + static_cast<size_t>(bh) * nQB * D;
  const float *kb = kbar + static_cast<size_t>(bh) * nKB * D;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int e0 = 0; e0 < D; e0 += 32) {
    for (int x = threadIdx.x; x < 64 * 32; x += 256) {
      const int rr = x >> 5, ee = x & 31;
      qs[ee][rr] = (i0 + rr < nQB) ? qb[static_cast<size_t>(i0 + rr) * D + e0 + ee] : 0.f;
      ks[ee][rr] = (j0 + rr < nKB) ? kb[static_cast<size_t>(j0 + rr) * D + e0 + ee] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int ee = 0; ee < 32; ++ee) {
      float a[4], b[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a[t] = qs[ee][ty * 4 + t];
        b[t] = ks[ee][tx * 4 + t];
      }
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[t][u] = fmaf(a[t], b[u], acc[t][u]);
    }
    __syncthreads();
  }
  const float sc = rsqrtf(static_cast<float>(D));
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int i = i0 + ty * 4 + t;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + tx * 4 + u;
      if (i < nQB && j < nKB) smap[(static_cast<size_t>(bh) * nQB + i) * nKB + j] = acc[t][u] * sc;
    }
  }
}

// "a before b" in the rank order: larger key first, lower block index first on ties.
__device__ __forceinline__ bool rank_before(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// One CTA (512 threads) per proxy row. P: power of two >= nKB (<= kMaxKeyBlocks).
// topp == 0: keep the min(k, nKB) blocks with the largest proxies.
// topp == 1: rank by mass n_j e^{s_ij} (key s_ij + ln n_j) and keep a block iff the mass
//            ranked before it is < p * (the row's total).
template <int P>
__global__ void __launch_bounds__(512) select_kernel(const float *smap, uint32_t *keep_mask, int nKB, int N, int Bk,
                                                     int topp, int k, float pmass) {
  __shared__ float key[P];
  __shared__ int idx[P];
  __shared__ float scan[P];
  __shared__ uint32_t words[P / 32];
  const int row = blockIdx.x;
  const float *s = smap + static_cast<size_t>(row) * nKB;
  const float ln_bk = logf(static_cast<float>(Bk));
  const float ln_last = logf(static_cast<float>(N - (nKB - 1) * Bk));
  for (int t = threadIdx.x; t < P; t += blockDim.x) {
    float kv = -CUDART_INF_F;
    if (t < nKB) kv = s[t] + (topp ? (t == nKB - 1 ? ln_last : ln_bk) : 0.f);
    key[t] = kv;
    idx[t] = t;  // padding (t >= nKB) sorts last: key -inf, index above every block's
  }
  for (int t = threadIdx.x; t < P / 32; t += blockDim.x) words[t] = 0u;
  // Bitonic sort into rank order.
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
        const int pos = 2 * stride * (t / stride) + (t % stride);
        const int oth = pos + stride;
        const bool first_half_desc = (pos & size) == 0;  // this subsequence sorts into rank order
        const float ka = key[pos], kb = key[oth];
        const int ia = idx[pos], ib = idx[oth];
        const bool ordered = rank_before(ka, ia, kb, ib);
        if (ordered != first_half_desc) {
          key[pos] = kb;
          key[oth] = ka;
          idx[pos] = ib;
          idx[oth] = ia;
        }
      }
    }
  }
  __syncthreads();
  if (!topp) {
    for (int t = threadIdx.x; t < nKB && t < k; t += blockDim.x) atomicOr(&words[idx[t] >> 5], 1u << (idx[t] & 31));
  } else {
    // Masses relative to the heaviest block, then an inclusive scan (Hillis-Steele).
    const float top = key[0];
    for (int t = threadIdx.x; t < P; t += blockDim.x) scan[t] = (t < nKB) ? __expf(key[t] - top) : 0.f;
    for (int off = 1; off < P; off <<= 1) {
      __syncthreads();
      float add[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = threadIdx.x + h * 512;
        add[h] = (t < P && t >= off) ? scan[t - off] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = threadIdx.x + h * 512;
        if (t < P) scan[t] += add[h];
      }
    }
    __syncthreads();
    const float limit = pmass * scan[P - 1];
    for (int t = threadIdx.x; t < nKB; t += blockDim.x) {
      const float before = (t == 0) ? 0.f : scan[t - 1];
      if (before < limit) atomicOr(&words[idx[t] >> 5], 1u << (idx[t] & 31));
    }
  }
  __syncthreads();
  const int nW = (nKB + 31) >> 5;
  for (int w = threadIdx.x; w < nW; w += blockDim.x) keep_mask[static_cast<size_t>(row) * nW + w] = words[w];
}

}  // namespace solattn
