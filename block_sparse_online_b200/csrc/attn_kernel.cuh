// attn_kernel.cuh -- the fused Sol-Attn forward kernel for sm_100a.
//
// One persistent CTA per SM processes work items. An item is one 128-row query tile
// of one (batch, head) pair (the tile holds 128/Bq query blocks); its key stream is
// the list of key blocks kept by any of the tile's query blocks. Roles, by warp:
//   warp 0      TMA producer: the item's Q tile (double-buffered across items), then
//               K_j and V_j of every kept block into a ring of shared-memory slots.
//   warps 1, 3  MMA issuers (one thread each, for warpgroups A and B, taking turns):
//               S = Q K_j^T into tensor memory (TMEM, bf16 -> fp32), O += P V_j with P
//               read from TMEM (fp16 -> fp32).
//   warp 2      router: for the NEXT item (double-buffered), reads the keep bits and the
//               correction record the routing pass (plan_kernel) left for each query
//               block, and builds the item's kept list in shared memory.
//   warps 4..7  softmax warpgroup A, warps 8..11 softmax warpgroup B. The tile's kept
//               list is split between them (A takes entries 0, 2, 4, ..., B takes 1, 3,
//               5, ...); each keeps its own S, O, running max and sum for all 128 rows.
//               At the end of the item they exchange max and sum through shared memory
//               and each writes half of the output columns of the merged result.
// The MMA groups alternate A and B (ping-pong): while one warpgroup exponentiates its
// S tile, the tensor core runs the other's P V and next Q K^T. Every K/V block is
// loaded once.
//
// Method (paperlayer summary "Sol-Attn: Accelerating Video Generation Inference
// via On-the-Fly Attention Sparsification", §3 Methodology):
//  * routing (plan_kernel, before this kernel): block proxy s = mean(Q_i) . mean(K_j) /
//    sqrt(d) is compared, as it is produced, against the running maximum of the proxies
//    visited so far minus tau ("On-the-fly sparsification"); key blocks are visited from
//    query block i's diagonal block upward with wrap-around. The proxies stay in shared
//    memory; only one keep bit per (query block, key block) reaches HBM.
//  * exact attention on kept blocks with one online-softmax state per row
//    ("Unified execution": one online-softmax state, original K/V tiles loaded only
//    for routed indices).
//  * each dropped block re-enters as one pseudo-key of weight n_j e^{s} and value
//    mean(V_j) ("Approximate correction": zeroth-order proxy-score reuse with pooled
//    keys and summed values). Because s does not depend on the query row, the
//    correction is one d-vector and one scalar per query block, which the routing pass
//    folds with the whole GPU's parallelism.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <type_traits>

#include "ptx_sm100.cuh"

namespace solattn {

constexpr int kMaxKeyBlocks = 1024;
constexpr int kMaskWords = kMaxKeyBlocks / 32;
// Token-to-block correction: the item's key stream ends with ceil(nKB / BK) tiles of the
// head's pooled keys ("pseudo tiles"), flagged in the kept list.
constexpr int kPseudoFlag = 0x8000;
constexpr int kMaxPseudo = kMaxKeyBlocks / 64;
constexpr int kStatusTimeout = -4;
constexpr int kStatusBounds = -6;  // a debug-build bounds check failed
constexpr float kLog2e = 1.4426950408889634f;
// Lazy rescaling: a row's reference max moves only when the tile max exceeds it by
// more than this many log2 units, so O is rarely rescaled (P <= 2^8 on the tile that moves
// it; a lagging reference is kept while every row sum of a tile stays <= 2^15).
constexpr float kRescaleSlack = 8.0f;
// Largest row sum of a tile exponentiated against a reference max that may lag the row:
// every value is then <= 2^15, inside fp16's range.
constexpr float kSpecRowSumLimit = 32768.0f;
// Pairs of exponentials computed on the FMA pipe (polynomial) instead of the MUFU unit:
// bit e % 8 of this mask set -> pair e of a 16-pair chunk goes to the polynomial.
constexpr uint32_t kPolyMask = 0x80u;

struct FwdParams {
  int N;
  int nQB;
  int nKB;
  int mode;  // 0 dense, 1 keep_drop, 2 keep_correct
  float tau;
  int items_per_head;
  int n_items;
  const float *qbar;  // [BH][nQB][D]
  const float *kbar;  // [BH][nKB][D]
  const float *vbar;  // [BH][nKB][D] (keep_correct only)
  __nv_bfloat16 *out; // [BH][N][D]
  unsigned long long *kept_per_head;  // [BH]
  uint32_t *keep_mask;                // [BH][nQB][ceil(nKB/32)] or null
  unsigned int *counter;              // work-item counter, zero at launch
  const int *order;                   // fetch order of the work items, or null (item order)
  int *status;                        // device status word
  unsigned long long timeout_ns;      // limit of every device-side wait
  // Query-dependent Gaussian threshold per (b, h, query block), or null: with it a block
  // is kept iff its proxy is >= theta (and the row's top block always), in place of the
  // running-max rule with tau.
  const float *theta;
  // Key blocks 0 .. n_sink_blocks - 1 hold sink tokens: kept by every query block.
  int n_sink_blocks;
  // keep_correct with the token-to-block correction: each row meets every dropped block
  // as one pseudo-key (pooled key, logit q_r . k_j / sqrt(d), weight n_j, value v_j), fed
  // to the tensor cores as n_pseudo tiles of pooled keys at the end of every item.
  int token_corr;
  int n_pseudo;
  // keep_correct with the block correction: per (b, h, query block), {M, L, -, -, C[D]}
  // (corr_stride floats), written by plan_kernel and read by the router.
  float *corr;
  // Keep bits per (b, h, query block) ([BH][nQB][ceil(nKB/32)]), written by plan_kernel and
  // read by the router; null in dense mode (no routing).
  uint32_t *keep_bits;
};

// Floats per query block of the correction record: M (running proxy max, natural-log
// units), L = sum over dropped j of n_j e^{s_ij - M}, two pad words, then
// C = sum over dropped j of n_j e^{s_ij - M} mean(V_j) (16-byte aligned).
template <int D>
__host__ __device__ constexpr int corr_stride() { return D + 4; }

template <int D_, int BK_, int SUBQ_>
struct Cfg {
  static constexpr int D = D_;
  static constexpr int BK = BK_;
  static constexpr int SUBQ = SUBQ_;  // query blocks per 128-row tile
  static constexpr int TILE_M = 128;
  static constexpr int BQ = TILE_M / SUBQ;
  static constexpr int NSB = SUBQ;       // query blocks per work item
  static constexpr int PANELS = D / 64;  // 128-byte swizzle panels per row
  static constexpr int Q_TILE_BYTES = TILE_M * D * 2;
  static constexpr int NQBUF = 2;        // Q tiles in flight (current and next item)
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int NSLOT = (131072 / KV_BYTES) < 8 ? (131072 / KV_BYTES) : 8;
  static constexpr int NWG = 2;              // softmax warpgroups sharing one tile
  static constexpr int WG_COLS = BK + D;     // TMEM columns per warpgroup: S (aliased by P) + O
  static constexpr int TMEM_NEED = NWG * WG_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  // One control warpgroup (warp 0 producer, warps 1 and 3 MMA issuers, warp 2 router)
  // and two softmax warpgroups. A warp may only touch TMEM lanes 32*(warp%4)..+31, so
  // each softmax warpgroup covers the four lane quadrants once.
  static constexpr int CTRL_WARPS = 4;
  static constexpr int NUM_THREADS = 32 * CTRL_WARPS + 128 * NWG;
  // Register split: the control warpgroup hands registers to the softmax warpgroups.
  // The sum stays within the registers the block is launched with (384 threads x 168).
  // The softmax holds a whole row of S (BK fp32 values) in registers and needs about 190;
  // the router and MMA issuers fit in 120 (ptxas -v: no spill beyond the 12 bytes of the
  // kernel's stack in the headline instantiation).
  static constexpr int CTRL_REGS = 120;
  static constexpr int SOFTMAX_REGS = 192;
  static_assert(128 * CTRL_REGS + 256 * SOFTMAX_REGS <= 384 * 168, "register split");
  // S = Q K^T in bf16; O += P V in fp16 (P in [0, 2^15] under the lazy rescale; V is the
  // fp16 copy written by the pooling pass).
  static constexpr uint32_t IDESC_QK = idesc_16bit_f32(128, BK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_16bit_f32(128, D, true, true);
  static_assert(TMEM_NEED <= 512, "TMEM budget");
  static_assert(NSB <= 8, "member bits");
};

template <class C>
struct RouteSlot {
  int item;     // work item, or -1 when the CTA has no more work
  int n_union;  // number of key blocks kept by at least one query block of the item
  int pad[2];
  float M[C::NSB];        // running proxy max (natural log units), -inf if no correction
  float L[C::NSB];        // sum over dropped j of n_j e^{s_ij - M}
  float Cv[C::NSB][C::D]; // sum over dropped j of n_j e^{s_ij - M} mean(V_j)
  uint32_t kmask[C::NSB][kMaskWords];  // keep bits per query block (token-to-block correction)
  uint16_t jlist[kMaxKeyBlocks + kMaxPseudo];  // kept key blocks (union over the item), ascending,
                                               // then the pseudo tiles (kPseudoFlag | t)
  uint8_t member[kMaxKeyBlocks + kMaxPseudo];  // bit sb: query block sb of the item keeps jlist[u]
};

template <class C>
struct SmemCtl {
  RouteSlot<C> route[2];
  uint32_t mask[C::NSB][kMaskWords];  // router scratch: keep bits per query block
  float xm[C::NWG][C::TILE_M];        // merge exchange: row max (log2 units) per warpgroup
  float xl[C::NWG][C::TILE_M];        // merge exchange: row sum per warpgroup
  uint64_t full[C::NSLOT];
  uint64_t empty[C::NSLOT];
  uint64_t q_full[C::NQBUF], q_empty[C::NQBUF];
  uint64_t s_full[C::NWG], p_full[C::NWG], xchg[C::NWG];
  uint64_t o_full, o_empty;
  uint64_t route_full[2], route_empty[2];
  uint64_t mma_done[C::NWG];
  uint32_t mma_group;  // number of MMA groups issued so far (turn of the two MMA threads)
  uint32_t tmem_base;
  int abort_flag;
};

template <class C>
constexpr size_t fwd_smem_bytes() {
  return 1024 + static_cast<size_t>(C::NQBUF) * C::Q_TILE_BYTES +
         static_cast<size_t>(C::NSLOT) * C::KV_BYTES + sizeof(SmemCtl<C>);
}

// The first error of a launch is kept: a role that gave up on a wait records a timeout
// unless another role recorded an error first, then raises the block-wide abort flag.
__device__ __forceinline__ void raise_abort(int *abort_flag, int *status) {
  atomicCAS(status, 0, kStatusTimeout);
  *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

// Debug builds (-DSOLATTN_DEBUG) check the indices each role derives from shared state
// before it uses them for a copy, an MMA operand or a store. A failed check records
// kStatusBounds (if no error is recorded yet) and raises the abort flag; the role then
// leaves as it does after a timeout, and the other roles follow at their next wait.
// Release builds compile every check to `true`.
__device__ __forceinline__ bool debug_fail(int *abort_flag, int *status) {
  atomicCAS(status, 0, kStatusBounds);
  *reinterpret_cast<volatile int *>(abort_flag) = 1;
  return false;
}
// Kernels without an abort flag (the routing pass) record the status only; the routing-only
// entry point runs without a status word (null), and then a failed check only skips the access.
__device__ __forceinline__ bool debug_fail_status(int *status) {
  if (status) atomicCAS(status, 0, kStatusBounds);
  return false;
}
#ifdef SOLATTN_DEBUG
#define SOLATTN_DCHECK(cond, abort_flag, status) ((cond) ? true : debug_fail((abort_flag), (status)))
#define SOLATTN_DCHECK_STATUS(cond, status) ((cond) ? true : debug_fail_status(status))
#else
#define SOLATTN_DCHECK(cond, abort_flag, status) true
#define SOLATTN_DCHECK_STATUS(cond, status) true
#endif

__device__ __forceinline__ float u2f(uint32_t x) { return __uint_as_float(x); }

// ------------------------------------------------------------------ router

template <class C>
__device__ __forceinline__ void route_query_block(SmemCtl<C> &sc, RouteSlot<C> &rs, const FwdParams &p,
                                                  int bh, int sb, int qb, int lane) {
  constexpr int D = C::D;
  const bool correct = (p.mode == 2) && !p.token_corr;  // block-level correction sums
  // The routing pass (plan_kernel) left this query block's keep bits and, with the block
  // correction, its correction record: the router only reads them.
  const int nW = (p.nKB + 31) >> 5;
  const uint32_t *kw = p.keep_bits + (static_cast<size_t>(bh) * p.nQB + qb) * nW;
  for (int w = lane; w < nW; w += 32) sc.mask[sb][w] = kw[w];
  if (correct) {
    const float *rec = p.corr + (static_cast<size_t>(bh) * p.nQB + qb) * corr_stride<D>();
    for (int e = lane; e < D; e += 32) rs.Cv[sb][e] = __ldg(rec + 4 + e);
    if (lane == 0) {
      rs.M[sb] = __ldg(rec);
      rs.L[sb] = __ldg(rec + 1);
    }
  } else {
    for (int e = lane; e < D; e += 32) rs.Cv[sb][e] = 0.f;
    if (lane == 0) {
      rs.L[sb] = 0.f;
      rs.M[sb] = -CUDART_INF_F;
    }
  }
}

template <class C>
__device__ void run_router(SmemCtl<C> &sc, const FwdParams &p, int lane) {
  constexpr int D = C::D;
  const int nKB = p.nKB;
  const int nW = (nKB + 31) >> 5;
  const uint32_t last_word = (nKB & 31) ? ((1u << (nKB & 31)) - 1u) : 0xffffffffu;
  const volatile int *ab = &sc.abort_flag;
  bool ok = true;
  for (uint32_t r_it = 0;; ++r_it) {
    const int s = r_it & 1;
    bool w_ok = mbar_wait(&sc.route_empty[s], ((r_it >> 1) & 1) ^ 1, p.timeout_ns, ab);
    if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
    int item = 0;
    if (lane == 0) {
      item = static_cast<int>(atomicAdd(p.counter, 1u));
      if (p.order && item < p.n_items) item = p.order[item];  // planned order
    }
    item = __shfl_sync(0xffffffffu, item, 0);
    RouteSlot<C> &rs = sc.route[s];
    if (item >= p.n_items) {
      if (lane == 0) {
        rs.item = -1;
        rs.n_union = 0;
        mbar_arrive(&sc.route_full[s]);
      }
      break;
    }
    const int bh = item / p.items_per_head;
    const int pidx = item - bh * p.items_per_head;
    for (int sb = 0; sb < C::NSB; ++sb)
      for (int w = lane; w < nW; w += 32) sc.mask[sb][w] = 0u;
    __syncwarp();
    for (int sb = 0; sb < C::NSB; ++sb) {
      const int qb = pidx * C::NSB + sb;
      if (qb >= p.nQB || p.mode == 0) {
        if (qb < p.nQB)
          for (int w = lane; w < nW; w += 32) sc.mask[sb][w] = (w == nW - 1) ? last_word : 0xffffffffu;
        for (int e = lane; e < D; e += 32) rs.Cv[sb][e] = 0.f;
        if (lane == 0) {
          rs.L[sb] = 0.f;
          rs.M[sb] = -CUDART_INF_F;
        }
        continue;
      }
      route_query_block<C>(sc, rs, p, bh, sb, qb, lane);
      __syncwarp();
    }
    // Union of the item's keep sets, ascending, with per-query-block membership bits.
    int base = 0;
    for (int w0 = 0; w0 < nW; w0 += 32) {
      const int w = w0 + lane;
      uint32_t words[C::NSB];
      uint32_t u = 0;
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) {
        words[sb] = (w < nW) ? sc.mask[sb][w] : 0u;
        u |= words[sb];
      }
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = base + incl - cnt;
      while (u) {
        const int b = __ffs(u) - 1;
        u &= u - 1;
        uint32_t mem = 0;
#pragma unroll
        for (int sb = 0; sb < C::NSB; ++sb) mem |= ((words[sb] >> b) & 1u) << sb;
        if (!SOLATTN_DCHECK(w * 32 + b < nKB && pos < kMaxKeyBlocks, &sc.abort_flag, p.status)) break;
        rs.jlist[pos] = static_cast<uint16_t>(w * 32 + b);
        rs.member[pos] = static_cast<uint8_t>(mem);
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
#ifdef SOLATTN_DEBUG
    if (*ab) {  // a check above failed
      ok = false;
      break;
    }
#endif
    // Statistics: kept blocks per head, and the optional keep bit-mask.
    unsigned long long kept = 0;
    for (int sb = 0; sb < C::NSB; ++sb) {
      const int qb = pidx * C::NSB + sb;
      if (qb >= p.nQB) continue;
      for (int w = lane; w < nW; w += 32) {
        const uint32_t word = sc.mask[sb][w];
        kept += __popc(word);
        if (p.keep_mask && p.keep_mask != p.keep_bits)
          p.keep_mask[(static_cast<size_t>(bh) * p.nQB + qb) * nW + w] = word;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, off);
    __syncwarp();
    int n_list = base;
    if (p.mode == 2 && p.token_corr) {
      // The pseudo tiles of the head's pooled keys, and the keep bits that mask them.
      for (int sb = 0; sb < C::NSB; ++sb)
        for (int w = lane; w < nW; w += 32) rs.kmask[sb][w] = sc.mask[sb][w];
      for (int t = lane; t < p.n_pseudo; t += 32) {
        rs.jlist[base + t] = static_cast<uint16_t>(kPseudoFlag | t);
        rs.member[base + t] = static_cast<uint8_t>((1u << C::NSB) - 1u);
      }
      n_list += p.n_pseudo;
    }
    __syncwarp();
    if (lane == 0) {
      atomicAdd(p.kept_per_head + bh, kept);
      rs.item = item;
      rs.n_union = n_list;
      mbar_arrive(&sc.route_full[s]);
    }
    __syncwarp();
  }
  if (!ok && lane == 0) raise_abort(&sc.abort_flag, p.status);
}

// ------------------------------------------------------------------ producer

template <class C>
__device__ void run_producer(SmemCtl<C> &sc, const FwdParams &p, uint8_t *q_smem, uint8_t *ring,
                             const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                             const CUtensorMap *tm_kp, const CUtensorMap *tm_vp) {
  const volatile int *ab = &sc.abort_flag;
  uint32_t kv_it = 0, q_it = 0;
  bool ok = true;
  // L2 priorities: a Q tile is read by one item only; a K or V tile by every query tile of
  // its head that keeps the block, so it should still be in L2 when the next one needs it.
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_reuse = l2_policy_evict_last();
  // Loads one K or V tile of key block j into the next ring slot.
  auto load = [&](int j, bool is_v, int bh) {
    const int slot = kv_it % C::NSLOT;
    const uint32_t ph = (kv_it / C::NSLOT) & 1;
    if (!mbar_wait(&sc.empty[slot], ph ^ 1, p.timeout_ns, ab)) {
      ok = false;
      return;
    }
    // a pseudo tile is BK rows of the head's pooled keys / values (zero past nKB)
    const bool pseudo = (j & kPseudoFlag) != 0;
    if (!SOLATTN_DCHECK(pseudo ? (j & (kPseudoFlag - 1)) < p.n_pseudo : j < p.nKB, &sc.abort_flag, p.status)) {
      ok = false;
      return;
    }
    mbar_arrive_expect_tx(&sc.full[slot], C::KV_BYTES);
    uint8_t *dst = ring + slot * C::KV_BYTES;
    const CUtensorMap *map = pseudo ? (is_v ? tm_vp : tm_kp) : (is_v ? tm_v : tm_k);
    const int row = (j & (kPseudoFlag - 1)) * C::BK;
#pragma unroll
    for (int pn = 0; pn < C::PANELS; ++pn)
      tma_load_3d_hint(smem_u32(dst + pn * (C::BK * 128)), map, smem_u32(&sc.full[slot]), pn * 64, row, bh,
                       pol_reuse);
    ++kv_it;
  };
  for (uint32_t r_it = 0;; ++r_it) {
    const int s = r_it & 1;
    if (!mbar_wait(&sc.route_full[s], (r_it >> 1) & 1, p.timeout_ns, ab)) { ok = false; break; }
    const RouteSlot<C> &rs = sc.route[s];
    const int item = rs.item;
    if (item < 0) break;
    const int bh = item / p.items_per_head;
    const int row0 = (item - bh * p.items_per_head) * C::TILE_M;
    if (!SOLATTN_DCHECK(item < p.n_items && row0 < p.N, &sc.abort_flag, p.status)) {
      ok = false;
      break;
    }
    const int qb = q_it & 1;
    if (!mbar_wait(&sc.q_empty[qb], ((q_it >> 1) & 1) ^ 1, p.timeout_ns, ab)) { ok = false; break; }
    mbar_arrive_expect_tx(&sc.q_full[qb], C::Q_TILE_BYTES);
#pragma unroll
    for (int pn = 0; pn < C::PANELS; ++pn)
      tma_load_3d_hint(smem_u32(q_smem + qb * C::Q_TILE_BYTES + pn * (C::TILE_M * 128)), tm_q,
                       smem_u32(&sc.q_full[qb]), pn * 64, row0, bh, pol_stream);
    ++q_it;
    // Ring order = consumption order of the MMA warp: K_0, K_1, then V_u, K_{u+2}.
    const int n = rs.n_union;
    load(rs.jlist[0], false, bh);
    if (ok && n > 1) load(rs.jlist[1], false, bh);
    for (int u = 0; u < n && ok; ++u) {
      load(rs.jlist[u], true, bh);
      if (ok && u + 2 < n) load(rs.jlist[u + 2], false, bh);
    }
    if (!ok) break;
    mbar_arrive(&sc.route_empty[s]);
  }
  if (!ok) raise_abort(&sc.abort_flag, p.status);
  // No copy may outlive the block: wait (bounded, ignoring the abort flag) for the
  // last fill of every slot and of the Q buffers to land.
  const int zero = 0;
  for (uint32_t f = (kv_it > C::NSLOT ? kv_it - C::NSLOT : 0); f < kv_it; ++f)
    mbar_wait(&sc.full[f % C::NSLOT], (f / C::NSLOT) & 1, p.timeout_ns, &zero);
  for (uint32_t f = (q_it > C::NQBUF ? q_it - C::NQBUF : 0); f < q_it; ++f)
    mbar_wait(&sc.q_full[f & 1], (f >> 1) & 1, p.timeout_ns, &zero);
}

// ------------------------------------------------------------------ MMA issuer

// MMA issue takes prebuilt shared-memory descriptors of the operand tiles and adds only
// compile-time offsets per 16-wide k step (the start-address field counts 16-byte units
// and never carries, as shared memory ends below 256 KB): building descriptors per
// instruction starves the tensor core when the softmax warps keep the issue slots busy.
template <class C>
__device__ __forceinline__ void issue_qk(uint32_t tmem, int w, uint64_t q_desc, uint64_t k_desc) {
  const uint32_t d_tmem = tmem + w * C::WG_COLS;
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk) {
    const uint64_t off_q = static_cast<uint64_t>((kk >> 2) * (C::TILE_M * 128 / 16) + (kk & 3) * 2);
    const uint64_t off_k = static_cast<uint64_t>((kk >> 2) * (C::BK * 128 / 16) + (kk & 3) * 2);
    mma_bf16_ss(d_tmem, q_desc + off_q, k_desc + off_k, C::IDESC_QK, kk > 0 ? 1u : 0u);
  }
}
template <class C>
__device__ __forceinline__ void issue_pv(uint32_t tmem, int w, uint64_t v_desc, bool accumulate) {
  const uint32_t d_tmem = tmem + w * C::WG_COLS + C::BK;
  const uint32_t p_tmem = tmem + w * C::WG_COLS;
#pragma unroll
  for (int kk = 0; kk < C::BK / 16; ++kk) {
    mma_bf16_ts(d_tmem, p_tmem + kk * 8, v_desc + static_cast<uint64_t>(kk * (16 * 128 / 16)), C::IDESC_PV,
                (accumulate || kk > 0) ? 1u : 0u);
  }
}
__device__ __forceinline__ int ring_index_v(int u, int n) {
  return min(n, 2) + u + min(u, max(n - 2, 0));
}
__device__ __forceinline__ int ring_index_k(int u, int n) {
  return u < 2 ? u : ring_index_v(u - 2, n) + 1;
}

// Wait (bounded) until the shared MMA group counter reaches `target`.
__device__ __forceinline__ bool wait_turn(const volatile uint32_t *gidx, uint32_t target, uint64_t limit_ns,
                                          const volatile int *abort_flag) {
  if (*gidx == target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (*gidx == target) return true;
    if ((it & 255u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) return false;
    }
  }
}

// MMA issue, one thread per softmax warpgroup w. Thread w issues, for the positions u =
// w, w + 2, ... of each item's kept list, the group O_w += P_w V_u followed by
// S_w = Q K_{u+2}^T (and the first S_w of the item up front). The two threads take
// turns through a shared group counter, so the tensor core sees the groups in the
// order A, B, A, B, ... while each thread does its barrier waits (K/V landed, P ready)
// during the other's issue: tcgen05 issue advances only as fast as the tensor core
// drains, so waits between groups would otherwise leave it idle.
// Group numbering within an item of n kept blocks: S_A(0) = 0, S_B(1) = 1, step u =
// 2 + u (for n == 1: S_A(0) = 0, step 0 = 1); an item has n + 2 groups (2 if n == 1).
template <class C>
__device__ void run_mma(SmemCtl<C> &sc, const FwdParams &p, uint32_t tmem, uint8_t *q_smem, uint8_t *ring, int w) {
  const volatile int *ab = &sc.abort_flag;
  volatile uint32_t *gidx = &sc.mma_group;
  // Descriptors of Q buffer 0 and of ring slot 0 (as a K tile and as a V tile); other
  // buffers and slots are whole multiples of 16 bytes further on.
  const uint64_t q_desc0 = smem_desc_sw128(smem_u32(q_smem), 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem_u32(ring), 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(smem_u32(ring), C::BK * 128, 1024);
  constexpr uint32_t kSlotUnits = C::KV_BYTES / 16;
  uint32_t kv_base = 0, q_it = 0, o_it = 0, p_ph = 0, g_base = 0;
  bool ok = true;
  auto wait = [&](uint64_t *bar, uint32_t par) {
    if (!ok) return false;
    if (!mbar_wait(bar, par, p.timeout_ns, ab)) ok = false;
    else tc_fence_after_sync();
    return ok;
  };
  auto turn = [&](uint32_t g) {
    if (!ok) return false;
    if (!wait_turn(gidx, g_base + g, p.timeout_ns, ab)) ok = false;
    return ok;
  };
  auto pass_turn = [&](uint32_t g) { *gidx = g_base + g + 1; };
  // Ring slot of entry e of the current item, once its copy has landed (-1 on timeout).
  auto slot_of = [&](int e) {
    const uint32_t gg = kv_base + static_cast<uint32_t>(e);
    const int slot = gg % C::NSLOT;
    if (!wait(&sc.full[slot], (gg / C::NSLOT) & 1)) return -1;
    return slot;
  };
  for (uint32_t r_it = 0; ok; ++r_it) {
    const int s = r_it & 1;
    if (!wait(&sc.route_full[s], (r_it >> 1) & 1)) break;
    const RouteSlot<C> &rs = sc.route[s];
    const int item = rs.item;
    if (item < 0) break;
    const int n = rs.n_union;
    const int qb = q_it % C::NQBUF;
    if (!wait(&sc.q_full[qb], (q_it / C::NQBUF) & 1)) break;
    ++q_it;
    const uint64_t q_desc = q_desc0 + static_cast<uint64_t>(qb * (C::Q_TILE_BYTES / 16));
    if (w < n) {
      const int ks = slot_of(ring_index_k(w, n));
      if (ks < 0 || !turn(w)) break;
      issue_qk<C>(tmem, w, q_desc, k_desc0 + static_cast<uint64_t>(ks * kSlotUnits));
      tc_commit(&sc.s_full[w]);
      pass_turn(w);
    } else {
      mbar_arrive(&sc.q_empty[qb]);  // no S for this warpgroup in this item
    }
    bool first = true;
    for (int u = w; u < n && ok; u += 2) {
      // Everything the group needs except P is waited for first (V_u and K_{u+2} landed,
      // O free), so that once the softmax hands over P only the turn remains. K_{u+2}'s ring
      // slot is freed by S_w(u)'s completion and O by the previous item's epilogue, both
      // independent of P_w(u).
      const int vs = slot_of(ring_index_v(u, n));
      if (vs < 0) break;
      int ks = -1;
      if (u + 2 < n) {
        ks = slot_of(ring_index_k(u + 2, n));
        if (ks < 0) break;
      }
      // The first P V of the item overwrites O: the previous item's epilogue must be done.
      if (first && !wait(&sc.o_empty, (o_it & 1) ^ 1)) break;
      if (!wait(&sc.p_full[w], p_ph)) break;
      p_ph ^= 1;
      const uint32_t g = (n == 1) ? 1u : static_cast<uint32_t>(2 + u);
      if (!turn(g)) break;
      issue_pv<C>(tmem, w, v_desc0 + static_cast<uint64_t>(vs * kSlotUnits), !first);
      first = false;
      if (ks >= 0) {
        issue_qk<C>(tmem, w, q_desc, k_desc0 + static_cast<uint64_t>(ks * kSlotUnits));
        tc_commit(&sc.s_full[w]);
      }
      pass_turn(g);
    }
    if (!ok) break;
    if (first) {  // no P V for this warpgroup in this item (n == 1, w == 1)
      // Arrive only once the previous item's epilogue is done, as a first P V would: this
      // thread could otherwise run an item ahead of the other one and complete the previous
      // item's o_full phase with two arrivals of its own, before the other's last P V.
      if (!wait(&sc.o_empty, (o_it & 1) ^ 1)) break;
      mbar_arrive(&sc.o_full);
    } else {
      tc_commit(&sc.o_full);
    }
    ++o_it;
    kv_base += 2 * static_cast<uint32_t>(n);
    g_base += (n == 1) ? 2u : static_cast<uint32_t>(n + 2);
    mbar_arrive(&sc.route_empty[s]);
  }
  if (!ok) raise_abort(&sc.abort_flag, p.status);
  // Every tcgen05 operation issued here must finish before TMEM is released.
  const int zero = 0;
  tc_commit(&sc.mma_done[w]);
  mbar_wait(&sc.mma_done[w], 0, p.timeout_ns, &zero);
}

// ------------------------------------------------------------------ softmax / epilogue

// Softmax of one pseudo tile of the head's pooled keys (token-to-block correction):
// column c is key block jb = t * BK + c. It enters this row as one pseudo-key (logit
// q_r . k_jb / sqrt(d), weight n_jb, value mean(V_jb)) only if jb exists and this row's
// query block dropped it (bit clear in km). Kept out of line: it runs for a few tiles per
// item and would otherwise add to the register pressure of the exact-block path.
template <int BK>
__device__ __noinline__ void softmax_pseudo_tile(uint32_t s_addr, int t, const uint32_t *km, int N, int nKB,
                                                 float sc_log2, float &m_ref, float &alpha, float &lsum) {
  constexpr int NCH = BK / 32;
  const float lb = log2f(static_cast<float>(BK));
  const float lb_last = log2f(static_cast<float>(N - (nKB - 1) * BK));
  float mxs = -CUDART_INF_F;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    uint32_t xs[32];
    tmem_ld32(s_addr + c * 32, xs);
    tmem_wait_ld();
    reg_fence32(xs);
    const int jb0 = t * BK + c * 32;
    const uint32_t kw = (jb0 < nKB) ? km[jb0 >> 5] : 0xffffffffu;  // past nKB: masked
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int jb = jb0 + e;
      if (jb < nKB && !((kw >> e) & 1u)) mxs = fmaxf(mxs, fmaf(__uint_as_float(xs[e]), sc_log2, jb == nKB - 1 ? lb_last : lb));
    }
  }
  if (mxs > m_ref + kRescaleSlack) {
    if (m_ref != -CUDART_INF_F) alpha = ex2_approx(m_ref - mxs);
    m_ref = mxs;
  }
  const float neg_m = (m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    uint32_t xs[32];
    tmem_ld32(s_addr + c * 32, xs);
    tmem_wait_ld();
    reg_fence32(xs);
    const int jb0 = t * BK + c * 32;
    const uint32_t kw = (jb0 < nKB) ? km[jb0 >> 5] : 0xffffffffu;
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float pp[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int jb = jb0 + 2 * e + h;
        const bool ok_col = jb < nKB && !((kw >> (2 * e + h)) & 1u);
        const float bias = (jb == nKB - 1 ? lb_last : lb) + neg_m;
        pp[h] = ok_col ? ex2_approx(fmaf(__uint_as_float(xs[2 * e + h]), sc_log2, bias)) : 0.f;
      }
      lsum += pp[0] + pp[1];
      pk[e] = pack_f16x2(pp[0], pp[1]);
    }
    tmem_st16(s_addr + c * 16, pk);
  }
}

// TOKEN: this instantiation handles pseudo tiles (token-to-block correction); the other
// one has no such branch in its loop.
template <class C, bool TOKEN>
__device__ void run_softmax(SmemCtl<C> &sc, const FwdParams &p, uint32_t tmem, int w, int warp, int lane) {
  constexpr int BK = C::BK;
  constexpr int D = C::D;
  const volatile int *ab = &sc.abort_flag;
  const int wq = warp & 3;  // TMEM lane quadrant this warp may access
  const int row = wq * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t s_addr = lane_base + w * C::WG_COLS;
  const uint32_t o_addr = s_addr + BK;
  const float sc_log2 = kLog2e * rsqrtf(static_cast<float>(D));
  const int sb = (C::SUBQ == 2 ? (row >> 6) : 0);
  const uint32_t row_bit = 1u << sb;
  uint32_t s_ph = 0;
  uint32_t kv_base = 0;  // ring entries of earlier items (2 per kept block)
  const uint64_t pol_out = l2_policy_evict_first();
  // One thread per warpgroup returns the ring slots (and the Q buffer) the tensor core
  // has finished reading: the MMA issuers commit only the barrier this warpgroup waits on.
  const bool leader = (threadIdx.x & 127) == 0;
  auto release = [&](int entry) { mbar_arrive(&sc.empty[(kv_base + static_cast<uint32_t>(entry)) % C::NSLOT]); };
  bool ok = true;
  auto wait = [&](uint64_t *bar, uint32_t par) {
    bool wt = mbar_wait(bar, par, p.timeout_ns, ab);
    wt = __all_sync(0xffffffffu, wt);
    if (!wt) ok = false;
    else tc_fence_after_sync();
    return wt;
  };
  for (uint32_t r_it = 0; ok; ++r_it) {
    const int s = r_it & 1;
    if (!wait(&sc.route_full[s], (r_it >> 1) & 1)) break;
    const RouteSlot<C> &rs = sc.route[s];
    const int item = rs.item;
    if (item < 0) break;
    const int bh = item / p.items_per_head;
    const int tile = item - bh * p.items_per_head;
    const int grow = tile * C::TILE_M + row;
    const int n = rs.n_union;
    float m_ref = -CUDART_INF_F;  // reference max of this row, log2 units
    float l = 0.f;
    for (int u = w; u < n; u += 2) {
      const uint32_t mem = rs.member[u];
      const int j = rs.jlist[u];
      if (!SOLATTN_DCHECK((j & kPseudoFlag) ? (j & (kPseudoFlag - 1)) < p.n_pseudo : j < p.nKB, &sc.abort_flag,
                          p.status)) {
        ok = false;
        break;
      }
      if (!wait(&sc.s_full[w], s_ph)) break;
      s_ph ^= 1;
      // The group that produced this S (O += P V of position u - 2, then S of position u)
      // is complete: its K and V tiles and, after this warpgroup's last S, Q are free.
      if (leader) {
        release(ring_index_k(u, n));
        if (u >= w + 2) release(ring_index_v(u - 2, n));
        if (u + 2 >= n) mbar_arrive(&sc.q_empty[r_it % C::NQBUF]);
      }
      float alpha = 1.f;  // rescale of this row's O and l for this S tile
      float lsum = 0.f;
      if (!TOKEN || !(j & kPseudoFlag)) {
        // One pass over the row of S held in registers: all BK columns are loaded at once
        // (BK / 32 TMEM loads, one wait) and the exponentials go back to TMEM as fp16 pairs,
        // 16 columns per store. Once every row of the warp has a reference max, the tile is
        // first exponentiated against it without the row maximum: that is exact whatever the
        // reference, as long as no P value overflows fp16, and a row sum <= 2^15 bounds every
        // value by 2^15 < 65504. A warp where some row's sum is larger (or infinite) takes the
        // row maxima (a tree of three-input max instructions) and redoes the tile, as the
        // first tile of a row does: the reference moves when the maximum exceeds it by more
        // than the slack (O and l are then rescaled once, below), so P never needs rescaling.
        // A row sum above 2^15 implies a maximum more than log2(2^15 / BK) >= 8 above the
        // reference, so such a row's reference always moves.
        constexpr int NCH = BK / 32;
        const bool rk = (mem & row_bit) != 0;  // warp-uniform (a warp's rows share a query block)
        const int ncol = (j == p.nKB - 1) ? (p.N - j * BK) : BK;
        uint32_t x[BK];
        auto exp_all = [&](float neg_m) {
          const uint64_t scp = f2(sc_log2, sc_log2);
          const uint64_t nmp = f2(neg_m, neg_m);
          uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int col = c * 32 + 2 * e;
              const uint64_t xx = fma2(f2(u2f(x[col]), u2f(x[col + 1])), scp, nmp);
              float x0, x1, p0, p1;
              f2_split(xx, x0, x1);
              if ((kPolyMask >> (e % 8)) & 1u) {
                exp2_poly_x2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              acc[e & 3] = add2(acc[e & 3], f2(p0, p1));
              pk[e] = pack_f16x2(p0, p1);
            }
            tmem_st16(s_addr + c * 16, pk);
          }
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2_split(acc[0], s0, s1);
          f2_split(acc[1], s2, s3);
          f2_split(acc[2], s4, s5);
          f2_split(acc[3], s6, s7);
          return ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        };
        bool done = false;
        float mx = -CUDART_INF_F;
        if (rk) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(x + c * 32));
          tmem_wait_ld();
          reg_fence<BK>(x);
          if (ncol < BK) {  // ragged last key block: columns past N are not keys
#pragma unroll
            for (int e = 0; e < BK; ++e)
              if (e >= ncol) x[e] = __float_as_uint(-CUDART_INF_F);
          }
          if (__all_sync(0xffffffffu, m_ref != -CUDART_INF_F)) {
            lsum = exp_all(-m_ref);
            done = __all_sync(0xffffffffu, lsum <= kSpecRowSumLimit);
            if (!done) tmem_wait_st();
          }
          if (!done) mx = max_tree_bits<BK>(x);
        }
        if (!done) {
          const float mxs = mx * sc_log2;
          if (mxs > m_ref + kRescaleSlack) {
            if (m_ref != -CUDART_INF_F) alpha = ex2_approx(m_ref - mxs);
            m_ref = mxs;
          }
          const float neg_m = (m_ref == -CUDART_INF_F) ? 0.f : -m_ref;
          if (rk) {
            lsum = exp_all(neg_m);
          } else {
            // This row's query block does not keep the block (two query blocks per tile): P = 0.
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
#pragma unroll
            for (int c = 0; c < NCH; ++c) tmem_st16(s_addr + c * 16, pk);
          }
        }
      } else if constexpr (TOKEN) {
        softmax_pseudo_tile<BK>(s_addr, j & (kPseudoFlag - 1), rs.kmask[sb], p.N, p.nKB, sc_log2, m_ref, alpha, lsum);
      }
      l = l * alpha + lsum;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // The previous P V of this warpgroup has completed (the commit that signalled this
        // S tile was issued after it), so O can be rescaled in place before the next one.
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_addr + c * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(u2f(o[e]) * alpha);
          tmem_st32(o_addr + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&sc.p_full[w]);
    }
    if (!ok) break;
    // Epilogue: wait for the last P V of both warpgroups, exchange the row max and sum,
    // and write this warpgroup's half of the output columns of the merged rows.
    if (!wait(&sc.o_full, r_it & 1)) break;
    if (leader && w < n) release(ring_index_v(w + ((n - 1 - w) & ~1), n));  // V of the last P V
    kv_base += 2 * static_cast<uint32_t>(n);
    sc.xm[w][row] = m_ref;
    sc.xl[w][row] = l;
    mbar_arrive(&sc.xchg[w]);
    if (!wait(&sc.xchg[w ^ 1], r_it & 1)) break;
    const float mA = sc.xm[0][row], lA = sc.xl[0][row];
    const float mB = sc.xm[1][row], lB = sc.xl[1][row];
    const bool hasB = n >= 2;  // warpgroup B ran at least one P V (A always does)
    const int qb = tile * C::NSB + sb;
    const bool valid = (grow < p.N) && (qb < p.nQB);
    const float Lc = rs.L[sb];
    const float M2 = rs.M[sb] * kLog2e;
    float Ms = -CUDART_INF_F;
    if (lA > 0.f) Ms = mA;
    if (hasB && lB > 0.f) Ms = fmaxf(Ms, mB);
    if (Lc > 0.f) Ms = fmaxf(Ms, M2);
    const float aA = (lA > 0.f) ? ex2_approx(mA - Ms) : 0.f;
    const float aB = (hasB && lB > 0.f) ? ex2_approx(mB - Ms) : 0.f;
    const float b = (Lc > 0.f) ? ex2_approx(M2 - Ms) : 0.f;
    const float inv = 1.f / (aA * lA + aB * lB + b * Lc);
    const float *cv = rs.Cv[sb];
    const uint32_t oA = lane_base + C::BK;
    const uint32_t oB = lane_base + C::WG_COLS + C::BK;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(bh) * p.N + grow) * D);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const int col0 = w * (D / 2) + c * 16;
      uint32_t xa[16], xb[16];
      tmem_ld16(oA + col0, xa);
      if (hasB) tmem_ld16(oB + col0, xb);
      tmem_wait_ld();
      reg_fence16(xa);
      reg_fence16(xb);
      if (valid) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float y0 = fmaf(aA, u2f(xa[2 * e]), b * cv[col0 + 2 * e]);
          float y1 = fmaf(aA, u2f(xa[2 * e + 1]), b * cv[col0 + 2 * e + 1]);
          if (hasB) {
            y0 = fmaf(aB, u2f(xb[2 * e]), y0);
            y1 = fmaf(aB, u2f(xb[2 * e + 1]), y1);
          }
          pk[e] = pack_bf16x2(y0 * inv, y1 * inv);
        }
        // output rows are not read again by this kernel: they should not displace K and V in L2
        st_global_v4_hint(dst + (col0 >> 3), pk[0], pk[1], pk[2], pk[3], pol_out);
        st_global_v4_hint(dst + (col0 >> 3) + 1, pk[4], pk[5], pk[6], pk[7], pol_out);
      }
    }
    tc_fence_before_sync();
    mbar_arrive(&sc.o_empty);
    mbar_arrive(&sc.route_empty[s]);
  }
  if (!ok && lane == 0) raise_abort(&sc.abort_flag, p.status);
}

// ------------------------------------------------------------------ kernel

template <class C, bool TOKEN>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
    solattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                       const __grid_constant__ CUtensorMap tm_vp, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_smem = base;
  uint8_t *ring = base + C::NQBUF * C::Q_TILE_BYTES;
  SmemCtl<C> &sc = *reinterpret_cast<SmemCtl<C> *>(ring + C::NSLOT * C::KV_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&sc.full[i], 1);
      mbar_init(&sc.empty[i], 1);
    }
    for (int i = 0; i < C::NQBUF; ++i) {
      mbar_init(&sc.q_full[i], 1);
      mbar_init(&sc.q_empty[i], C::NWG);  // one arrival per softmax warpgroup (or its MMA thread)
    }
    for (int w = 0; w < C::NWG; ++w) {
      mbar_init(&sc.s_full[w], 1);
      mbar_init(&sc.p_full[w], 128);
      mbar_init(&sc.xchg[w], 128);
    }
    mbar_init(&sc.o_full, C::NWG);  // one commit (or arrive) per MMA thread
    mbar_init(&sc.o_empty, 128 * C::NWG);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sc.route_full[s], 1);
      mbar_init(&sc.route_empty[s], 1 + C::NWG + 128 * C::NWG);  // producer, MMA threads, softmax
    }
    for (int w = 0; w < C::NWG; ++w) mbar_init(&sc.mma_done[w], 1);
    sc.mma_group = 0;
    sc.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (p.token_corr) {
      tma_prefetch_desc(&tm_kp);
      tma_prefetch_desc(&tm_vp);
    }
  }
  if (warp == 1) {
    tmem_alloc(&sc.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sc.tmem_base;

  if (warp < C::CTRL_WARPS) {
    regs_dec<C::CTRL_REGS>();
    if (warp == 0) {
      if (lane == 0) run_producer<C>(sc, p, q_smem, ring, &tm_q, &tm_k, &tm_v, &tm_kp, &tm_vp);
    } else if (warp == 1 || warp == 3) {
      if (lane == 0) run_mma<C>(sc, p, tmem, q_smem, ring, warp == 1 ? 0 : 1);
    } else if (warp == 2) {
      run_router<C>(sc, p, lane);
    }
  } else {
    regs_inc<C::SOFTMAX_REGS>();
    run_softmax<C, TOKEN>(sc, p, tmem, (warp - C::CTRL_WARPS) >> 2, warp, lane);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ Gaussian threshold

// Pooled-key moments of one (b, h) over its key blocks (equal weight, 1/nKB): the mean
// m[D] and the covariance C[D][D] (diag = 0) or only its diagonal (diag = 1), written to
// kmom[bh] = {m, C or diag(C)}. One CTA per (b, h), 256 threads; the covariance is
// accumulated as 16 x 16 thread tiles of (D/16)^2 entries over 32-row chunks of the
// centred pooled keys staged in shared memory.
template <int D>
__global__ void __launch_bounds__(256) gauss_moments_kernel(const float *kbar, float *kmom, int nKB, int diag) {
  constexpr int T = D / 16;
  __shared__ float mean[D];
  __shared__ float rows[32][D];
  const int bh = blockIdx.x;
  const float *kb = kbar + static_cast<size_t>(bh) * nKB * D;
  float *out = kmom + static_cast<size_t>(bh) * (D + D * D);
  const float inv_n = 1.f / static_cast<float>(nKB);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float a = 0.f;
    for (int j = 0; j < nKB; ++j) a += kb[static_cast<size_t>(j) * D + e];
    mean[e] = a * inv_n;
    out[e] = a * inv_n;
  }
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[T][T];
#pragma unroll
  for (int a = 0; a < T; ++a)
#pragma unroll
    for (int b = 0; b < T; ++b) acc[a][b] = 0.f;
  for (int j0 = 0; j0 < nKB; j0 += 32) {
    for (int x = threadIdx.x; x < 32 * D; x += blockDim.x) {
      const int r = x / D, e = x - r * D;
      rows[r][e] = (j0 + r < nKB) ? kb[static_cast<size_t>(j0 + r) * D + e] - mean[e] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < 32; ++r) {
      float ra[T], rb[T];
#pragma unroll
      for (int a = 0; a < T; ++a) ra[a] = rows[r][ty * T + a];
#pragma unroll
      for (int b = 0; b < T; ++b) rb[b] = rows[r][tx * T + b];
      if (diag) {
        if (tx == ty) {
#pragma unroll
          for (int a = 0; a < T; ++a) acc[a][a] = fmaf(ra[a], ra[a], acc[a][a]);
        }
      } else {
#pragma unroll
        for (int a = 0; a < T; ++a)
#pragma unroll
          for (int b = 0; b < T; ++b) acc[a][b] = fmaf(ra[a], rb[b], acc[a][b]);
      }
    }
    __syncthreads();
  }
  float *c = out + D;
  if (diag) {
    if (tx == ty) {
#pragma unroll
      for (int a = 0; a < T; ++a) c[ty * T + a] = acc[a][a] * inv_n;
    }
  } else {
#pragma unroll
    for (int a = 0; a < T; ++a)
#pragma unroll
      for (int b = 0; b < T; ++b) c[(ty * T + a) * D + tx * T + b] = acc[a][b] * inv_n;
  }
}

// theta_i = mu_i + beta * sigma_i per query block: mu_i = q_i . m / sqrt(D) and
// sigma_i^2 = q_i^T C q_i / D (or sum_e q_ie^2 C_ee / D). Grid (ceil(nQB / 8), B*H), one
// warp per query block; C is staged in shared memory with a padded row stride.
template <int D>
__global__ void __launch_bounds__(256) gauss_theta_kernel(const float *qbar, const float *kmom, float *theta,
                                                          int nQB, float beta, int diag) {
  extern __shared__ float cs[];  // [D][D + 1] (exact) or [D] (diag), then q rows [8][D]
  const int bh = blockIdx.y;
  const float *mom = kmom + static_cast<size_t>(bh) * (D + D * D);
  const int ncov = diag ? D : D * D;
  float *cov = cs;
  float *qs = cs + (diag ? D : D * (D + 1));
  for (int x = threadIdx.x; x < ncov; x += blockDim.x) cov[diag ? x : (x / D) * (D + 1) + (x % D)] = mom[D + x];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  if (i >= nQB) return;
  const float *qr = qbar + (static_cast<size_t>(bh) * nQB + i) * D;
  float *q = qs + warp * D;
  for (int e = lane; e < D; e += 32) q[e] = qr[e];
  __syncwarp();
  float mu = 0.f, var = 0.f;
  for (int e = lane; e < D; e += 32) {
    mu = fmaf(q[e], mom[e], mu);
    if (diag) {
      var = fmaf(q[e] * q[e], cov[e], var);
    } else {
      float y = 0.f;
      const float *row = cov + e * (D + 1);
      for (int b = 0; b < D; ++b) y = fmaf(row[b], q[b], y);
      var = fmaf(q[e], y, var);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mu += __shfl_xor_sync(0xffffffffu, mu, off);
    var += __shfl_xor_sync(0xffffffffu, var, off);
  }
  if (lane == 0) {
    float t;
    if (beta == -CUDART_INF_F) t = -CUDART_INF_F;
    else if (beta == CUDART_INF_F) t = CUDART_INF_F;
    else t = mu * rsqrtf(static_cast<float>(D)) + beta * sqrtf(fmaxf(var / static_cast<float>(D), 0.f));
    theta[static_cast<size_t>(bh) * nQB + i] = t;
  }
}

// Evaluates the FMA-pipe exp2 used by the softmax on n inputs (self-test).
__global__ void exp2_selftest_kernel(const float *x, float *y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float y0, y1;
  exp2_poly_x2(x[i], x1, y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

// Device watchdog self-test: one thread waits on a barrier that nobody completes.
__global__ void watchdog_selftest_kernel(int *status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, limit_ns, &abort_flag);
    *status = ok ? 0 : kStatusTimeout;
  }
}

}  // namespace solattn
