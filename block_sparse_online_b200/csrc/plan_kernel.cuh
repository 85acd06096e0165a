// plan_kernel.cuh -- the routing pass: block proxies, keep decisions, block correction and
// the attention kernel's work order.
//
// ("Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification", paperlayer summary §3 Methodology: the block proxy from mean-pooled
// query and key blocks, keep decisions against the running maximum minus tau (or the
// query-dependent Gaussian threshold), and the zeroth-order correction that lets every
// dropped block re-enter through its pooled value; §4 "Efficient On-the-Fly
// Sparsification": the proxies are consumed on chip, never written out.)
//
// One CTA routes kPlanQG consecutive query blocks of one (b, h):
//   1. proxies s_ij = qbar_i . kbar_j / sqrt(d) of the group against every key block of
//      the head, into shared memory (each pooled key row is read once per group, not once
//      per query block);
//   2. one warp per query block visits the key blocks in the router's order (its own
//      diagonal block first, then on, wrapping) and keeps block j iff s_ij >= (running max
//      so far) - tau (or s_ij >= theta_i), sink blocks always; under the Gaussian threshold
//      a query block that keeps nothing keeps its top block. The keep bits go to memory;
//   3. keep_correct with the block correction: weights w_ij = n_j e^{s_ij - M_i} of the
//      dropped blocks (M_i the row's running max at the end of the visit, i.e. its maximum)
//      and the record {M_i, L_i = sum_j w_ij, C_i = sum_j w_ij vbar_j};
//   4. the kept count of every work item (the query tiles of the group) and, in the last
//      CTA to finish, the order in which the attention kernel takes the items.
// The same kernel without steps 3 and 4 is the routing-only entry point, so both take the
// same decisions bit for bit.
#pragma once

#include <cstdint>

#include "attn_kernel.cuh"

namespace solattn {

constexpr int kPlanQG = 12;       // query blocks per CTA
constexpr int kPlanWarps = 8;     // 256 threads
constexpr int kPlanBatch = 4;     // pooled-key float4 loads per batch (step 1; two batches in flight)
constexpr int kPlanOrderCap = 4096;  // most work items in one ordering group (host-enforced)

// Vector of the D/32 consecutive dimensions one lane holds (pooled value rows).
template <int VPL>
struct VecOf;
template <>
struct VecOf<4> {
  using T = float4;
  static __device__ __forceinline__ void axpy(float (&acc)[4], float w, const float4 &b) {
    acc[0] = fmaf(w, b.x, acc[0]);
    acc[1] = fmaf(w, b.y, acc[1]);
    acc[2] = fmaf(w, b.z, acc[2]);
    acc[3] = fmaf(w, b.w, acc[3]);
  }
  static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <>
struct VecOf<2> {
  using T = float2;
  static __device__ __forceinline__ void axpy(float (&acc)[2], float w, const float2 &b) {
    acc[0] = fmaf(w, b.x, acc[0]);
    acc[1] = fmaf(w, b.y, acc[1]);
  }
  static __device__ __forceinline__ float2 zero() { return make_float2(0.f, 0.f); }
};

// Dynamic shared memory of plan_kernel for nKB key blocks.
template <int D>
__host__ __device__ constexpr size_t plan_smem_bytes(int nKB) {
  return sizeof(float) * (static_cast<size_t>(kPlanQG) * D +                   // pooled query rows
                          static_cast<size_t>(kPlanQG) * ((nKB + 3) & ~3) +     // proxies, then weights
                          static_cast<size_t>(kPlanWarps) * kPlanQG * D) +      // per-warp sums of C
         sizeof(uint32_t) * kPlanQG * kMaskWords;                              // keep bits
}

// keep_out: keep bits [BH][nQB][ceil(nKB/32)]. cost == null: routing only (no correction
// record, no schedule). Grid (ceil(nQB / kPlanQG), B*H), 256 threads.
template <int D, int BQ, int BK, int SUBQ>
__global__ void __launch_bounds__(256, 2) plan_kernel(const FwdParams p, uint32_t *keep_out, int *cost, int *order,
                                                      unsigned int *done, int group_heads) {
  static_assert(kPlanQG % SUBQ == 0, "a work item's query blocks share one CTA");
  constexpr int C4 = D / 4;  // float4 columns of a pooled row
  extern __shared__ __align__(16) unsigned char plan_smem[];
  __shared__ float Mrow[kPlanQG], Lrow[kPlanQG];
  __shared__ int hist[kMaxKeyBlocks + 2];
  __shared__ int warp_tot[kPlanWarps];
  __shared__ int is_last;
  const int nKB = p.nKB, nQB = p.nQB, nW = (nKB + 31) >> 5;
  const int ldS = (nKB + 3) & ~3;
  float *qs = reinterpret_cast<float *>(plan_smem);                     // [QG][D]
  float *sm = qs + kPlanQG * D;                                         // [QG][ldS]
  float *red = sm + kPlanQG * ldS;                                      // [warps][QG][D]
  uint32_t *msk = reinterpret_cast<uint32_t *>(red + kPlanWarps * kPlanQG * D);  // [QG][kMaskWords]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qb0 = blockIdx.x * kPlanQG;
  const int nrows = min(kPlanQG, nQB - qb0);
  const bool correct = cost != nullptr && p.mode == 2 && !p.token_corr;

  // ---- 1. proxies of the group
  {
    const float4 *src = reinterpret_cast<const float4 *>(p.qbar + (static_cast<size_t>(bh) * nQB + qb0) * D);
    for (int x = threadIdx.x; x < kPlanQG * C4; x += blockDim.x)
      reinterpret_cast<float4 *>(qs)[x] = (x / C4 < nrows) ? __ldg(src + x) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int x = threadIdx.x; x < kPlanQG * kMaskWords; x += blockDim.x) msk[x] = 0u;
  }
  __syncthreads();
  const float inv_sqrt_d = rsqrtf(static_cast<float>(D));
  for (int j = threadIdx.x; j < nKB; j += blockDim.x) {
    // Thread = key block; every lane walks the columns in the same order, so each shared-
    // memory read of a pooled query row is one broadcast. Each dot product is one fp32 fma
    // chain over the dimensions in order.
    const float4 *kr = reinterpret_cast<const float4 *>(p.kbar + (static_cast<size_t>(bh) * nKB + j) * D);
    float acc[kPlanQG];
#pragma unroll
    for (int i = 0; i < kPlanQG; ++i) acc[i] = 0.f;
    // Batches of kPlanBatch float4 loads, the next batch in flight while this one is used.
    float4 kv[kPlanBatch], kn[kPlanBatch];
#pragma unroll
    for (int e = 0; e < kPlanBatch; ++e) kv[e] = __ldg(kr + e);
#pragma unroll 1
    for (int b0 = 0; b0 < C4; b0 += kPlanBatch) {
      if (b0 + kPlanBatch < C4) {
#pragma unroll
        for (int e = 0; e < kPlanBatch; ++e) kn[e] = __ldg(kr + b0 + kPlanBatch + e);
      }
#pragma unroll
      for (int e = 0; e < kPlanBatch; ++e) {
        const int c = b0 + e;
#pragma unroll
        for (int i = 0; i < kPlanQG; ++i) {
          const float4 qv = reinterpret_cast<const float4 *>(qs + i * D)[c];
          acc[i] = fmaf(qv.x, kv[e].x, acc[i]);
          acc[i] = fmaf(qv.y, kv[e].y, acc[i]);
          acc[i] = fmaf(qv.z, kv[e].z, acc[i]);
          acc[i] = fmaf(qv.w, kv[e].w, acc[i]);
        }
      }
#pragma unroll
      for (int e = 0; e < kPlanBatch; ++e) kv[e] = kn[e];
    }
#pragma unroll
    for (int i = 0; i < kPlanQG; ++i) sm[i * ldS + j] = acc[i] * inv_sqrt_d;
  }
  __syncthreads();

  // ---- 2. keep decisions (and 3a. correction weights), one warp per query block
  const bool gauss = p.theta != nullptr;
  const int nsb = p.n_sink_blocks;
  for (int i = warp; i < nrows; i += kPlanWarps) {
    const int qb = qb0 + i;
    const int j0 = min((qb * BQ) / BK, nKB - 1);
    const float th = gauss ? __ldg(p.theta + static_cast<size_t>(bh) * nQB + qb) : 0.f;
    const float *srow = sm + i * ldS;
    uint32_t *mrow = msk + i * kMaskWords;
    float M = -CUDART_INF_F;
    int kept = 0;
    float top_s = -CUDART_INF_F;
    int top_j = nKB;
    for (int t0 = 0; t0 < nKB; t0 += 32) {
      const int tt = t0 + lane;
      const bool valid = tt < nKB;
      int j = j0 + tt;
      if (j >= nKB) j -= nKB;
      if (!valid) j = 0;
      const float s = valid ? srow[j] : -CUDART_INF_F;
      // Running maximum in visit order: inclusive prefix max over the lanes.
      float m = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, m, off);
        if (lane >= off) m = fmaxf(m, y);
      }
      m = fmaxf(m, M);
      const float thr = gauss ? th : m - p.tau;
      const bool keep = valid && (s >= thr || j < nsb);
      M = __shfl_sync(0xffffffffu, m, 31);
      if (keep) atomicOr(&mrow[j >> 5], 1u << (j & 31));
      kept += __popc(__ballot_sync(0xffffffffu, keep));
      if (gauss) {  // the largest proxy, lowest index on ties
        float bs = s;
        int bj = valid ? j : nKB;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float os = __shfl_xor_sync(0xffffffffu, bs, off);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
          if (os > bs || (os == bs && oj < bj)) {
            bs = os;
            bj = oj;
          }
        }
        if (bs > top_s || (bs == top_s && bj < top_j)) {
          top_s = bs;
          top_j = bj;
        }
      }
    }
    __syncwarp();
    if (gauss && kept == 0 && lane == 0) atomicOr(&mrow[top_j >> 5], 1u << (top_j & 31));
    __syncwarp();
    uint32_t *kw = keep_out + (static_cast<size_t>(bh) * nQB + qb) * nW;
    // bits past nKB stay clear: the router turns every set bit into a key block index
    for (int w = lane; w < nW; w += 32)
      if (SOLATTN_DCHECK_STATUS(w < nW - 1 || (nKB & 31) == 0 || (mrow[w] >> (nKB & 31)) == 0u, p.status))
        kw[w] = mrow[w];
    if (correct) {
      float l = 0.f;
      for (int j = lane; j < nKB; j += 32) {
        const bool drop = !((mrow[j >> 5] >> (j & 31)) & 1u);
        const float nj = (j == nKB - 1) ? static_cast<float>(p.N - j * BK) : static_cast<float>(BK);
        const float w = drop ? nj * expf(srow[j] - M) : 0.f;
        sm[i * ldS + j] = w;
        l += w;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      if (lane == 0) {
        Mrow[i] = M;
        Lrow[i] = l;
      }
    }
  }
  __syncthreads();

  // ---- 3b. C_i = sum_j w_ij vbar_j: warp w takes key blocks w, w + 8, ...; lane l holds
  // dimensions l*D/32 .. of all the group's rows; the warps' sums are added in warp order.
  if (correct) {
    constexpr int VPL = D / 32;
    using V = VecOf<VPL>;
    using VecT = typename V::T;
    float acc[kPlanQG][VPL];
#pragma unroll
    for (int i = 0; i < kPlanQG; ++i)
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[i][e] = 0.f;
    const VecT *vb = reinterpret_cast<const VecT *>(p.vbar + static_cast<size_t>(bh) * nKB * D) + lane;
    for (int jb = warp; jb < nKB; jb += kPlanWarps * 8) {
      VecT vx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = jb + u * kPlanWarps;
        vx[u] = (j < nKB) ? __ldg(vb + static_cast<size_t>(j) * 32) : V::zero();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = jb + u * kPlanWarps;
        if (j < nKB) {
#pragma unroll
          for (int i = 0; i < kPlanQG; ++i) V::axpy(acc[i], sm[i * ldS + j], vx[u]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kPlanQG; ++i)
#pragma unroll
      for (int e = 0; e < VPL; ++e) red[(warp * kPlanQG + i) * D + lane * VPL + e] = acc[i][e];
    __syncthreads();
    for (int x = threadIdx.x; x < nrows * D; x += blockDim.x) {
      const int i = x / D, e = x - i * D;
      float c = 0.f;
#pragma unroll
      for (int w = 0; w < kPlanWarps; ++w) c += red[(w * kPlanQG + i) * D + e];
      float *rec = p.corr + (static_cast<size_t>(bh) * nQB + qb0 + i) * corr_stride<D>();
      rec[4 + e] = c;
      if (e == 0) {
        rec[0] = Mrow[i];
        rec[1] = Lrow[i];
      }
    }
  }
  if (cost == nullptr) return;  // routing only

  // ---- 4. kept count of each work item of the group (union over its query blocks)
  for (int it = warp; it * SUBQ < nrows; it += kPlanWarps) {
    int cnt = 0;
    for (int w = lane; w < nW; w += 32) {
      uint32_t u = 0;
#pragma unroll
      for (int sb = 0; sb < SUBQ; ++sb)
        if (it * SUBQ + sb < nrows) u |= msk[(it * SUBQ + sb) * kMaskWords + w];
      cnt += __popc(u);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    const int item = bh * p.items_per_head + qb0 / SUBQ + it;
    if (lane == 0 && SOLATTN_DCHECK_STATUS(item < p.n_items && cnt <= nKB, p.status)) cost[item] = cnt;
  }
  // The last CTA to finish orders the items: groups of `group_heads` consecutive heads in
  // head order (the group's K/V stays resident in L2), and within a group the costliest
  // items first, so the short items fill the end of the attention kernel.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int BH = p.n_items / p.items_per_head;
  const int nbins = nKB + 1;  // cost in [0, nKB]
  // The group's costs are copied to shared memory first (one round of independent loads
  // instead of a dependent global load per pass), into the dynamic shared memory this CTA
  // no longer needs: at least plan_smem_bytes<64>(1) / 4 = 7344 ints, while the host keeps
  // a group to max(items_per_head, kPlanOrderCap) <= 4096 items.
  int *cs = reinterpret_cast<int *>(plan_smem);
  for (int h0 = 0; h0 < BH; h0 += group_heads) {
    const int i0 = h0 * p.items_per_head;
    const int i1 = min(BH, h0 + group_heads) * p.items_per_head;
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) cs[i - i0] = cost[i];
    for (int c = threadIdx.x; c < nbins; c += blockDim.x) hist[c] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < i1 - i0; i += blockDim.x) atomicAdd(&hist[cs[i]], 1);
    __syncthreads();
    // Exclusive scan over descending cost: start[c] = number of items costlier than c.
    // Each thread owns a contiguous run of bins (from the costliest end).
    const int per = (nbins + blockDim.x - 1) / blockDim.x;
    const int c_hi = nbins - 1 - threadIdx.x * per;  // this thread's bins: c_hi, c_hi-1, ...
    int local = 0;
    for (int k = 0; k < per; ++k) {
      const int c = c_hi - k;
      if (c >= 0) local += hist[c];
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    int run = before + incl - local;
    for (int k = 0; k < per; ++k) {
      const int c = c_hi - k;
      if (c >= 0) {
        const int cnt_c = hist[c];
        hist[c] = run;
        run += cnt_c;
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < i1 - i0; i += blockDim.x) {
      const int pos = atomicAdd(&hist[cs[i]], 1);
      if (SOLATTN_DCHECK_STATUS(pos < i1 - i0, p.status)) order[i0 + pos] = i0 + i;
    }
    __syncthreads();
  }
}

}  // namespace solattn
