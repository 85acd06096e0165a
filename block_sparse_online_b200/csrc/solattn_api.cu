// solattn_api.cu -- host side of libsolattn: argument checks, workspace layout,
// TMA descriptors and kernel launches behind the C ABI declared in solattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "attn_kernel.cuh"
#include "plan_kernel.cuh"
#include "pool_kernel.cuh"
#include "route_kernels.cuh"
#include "solattn.h"

namespace {

using namespace solattn;

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;  // [0]: work counter (u32), [4]: status word (i32), [8]: plan counter
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per device-side wait

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int nblocks(int N, int blk) { return (N + blk - 1) / blk; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// NVTX range around the host code that enqueues one stage ("solattn pool", "solattn route",
// "solattn attention", ...), for timeline tools; without a tool attached it costs a few ns.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

struct WsLayout {
  size_t qbar, kbar, vbar, v16, cost, order, kmom, theta, kbar16, vbar16, corr, keep, total;
};

int check_shape(int B, int H, int N, int d, int Bq, int Bk) {
  if (B < 1 || H < 1 || N < 1) return SOLATTN_EINVAL;
  if (d != 64 && d != 128) return SOLATTN_EUNSUPPORTED;
  if ((Bq != 64 && Bq != 128) || (Bk != 64 && Bk != 128)) return SOLATTN_EUNSUPPORTED;
  if (nblocks(N, Bk) > SOLATTN_MAX_KEY_BLOCKS) return SOLATTN_EUNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return SOLATTN_EUNSUPPORTED;  // pooling grid y
  return SOLATTN_OK;
}

WsLayout ws_layout(int B, int H, int N, int d, int Bq, int Bk) {
  const size_t bh = static_cast<size_t>(B) * H;
  WsLayout w;
  w.qbar = kHeaderBytes;
  w.kbar = w.qbar + align_up(bh * nblocks(N, Bq) * d * sizeof(float), kAlign);
  w.vbar = w.kbar + align_up(bh * nblocks(N, Bk) * d * sizeof(float), kAlign);
  w.v16 = w.vbar + align_up(bh * nblocks(N, Bk) * d * sizeof(float), kAlign);
  const size_t items = bh * static_cast<size_t>(nblocks(N, 128));  // one work item per 128-row tile
  w.cost = w.v16 + align_up(bh * N * d * 2, kAlign);
  w.order = w.cost + align_up(items * sizeof(int), kAlign);
  w.kmom = w.order + align_up(items * sizeof(int), kAlign);  // pooled-key moments (Gaussian threshold)
  w.theta = w.kmom + align_up(bh * (d + static_cast<size_t>(d) * d) * sizeof(float), kAlign);
  w.kbar16 = w.theta + align_up(bh * nblocks(N, Bq) * sizeof(float), kAlign);  // token-to-block correction
  w.vbar16 = w.kbar16 + align_up(bh * nblocks(N, Bk) * d * 2, kAlign);
  w.corr = w.vbar16 + align_up(bh * nblocks(N, Bk) * d * 2, kAlign);  // block correction per query block
  w.keep = w.corr + align_up(bh * nblocks(N, Bq) * (d + 4) * sizeof(float), kAlign);  // keep bits
  w.total = w.keep + align_up(bh * nblocks(N, Bq) * ((nblocks(N, Bk) + 31) / 32) * sizeof(uint32_t), kAlign);
  return w;
}

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool known = false;
};

std::mutex g_mu;
DeviceInfo g_dev[64];

int device_info(DeviceInfo *out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOLATTN_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev[dev].known) {
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SOLATTN_ECUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return SOLATTN_ECUDA;
    g_dev[dev].sms = sms;
    g_dev[dev].major = major;
    g_dev[dev].known = true;
  }
  *out = g_dev[dev];
  return SOLATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D view (d, N, B*H) of a contiguous bf16 [B][H][N][d] tensor; boxes of 64 x rows x 1
// with the 128-byte swizzle. Rows past N read as zeros.
int make_map(CUtensorMap *map, const void *ptr, int d, int N, int BH, int box_rows,
             CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return SOLATTN_ECUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dtype, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOLATTN_OK : SOLATTN_ECUDA;
}

int launch_pool(const PoolArgs &args, int BH, int d, int max_nb, cudaStream_t st) {
  dim3 grid(max_nb, BH, args.njobs);
  if (d == 128)
    pool_kernel<128><<<grid, 128, 0, st>>>(args);
  else
    pool_kernel<64><<<grid, 128, 0, st>>>(args);
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

template <class C, bool TOKEN>
int launch_fwd_v(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mkp,
                 const CUtensorMap &mvp, const FwdParams &p, int sms, cudaStream_t st) {
  constexpr size_t smem = fwd_smem_bytes<C>();
  static bool attr_set[64] = {};  // per device; guarded by g_mu (calls may come from several threads)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOLATTN_ECUDA;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(solattn_fwd_kernel<C, TOKEN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess)
        return SOLATTN_ECUDA;
      attr_set[dev] = true;
    }
  }
  const int grid = p.n_items < sms ? p.n_items : sms;
  solattn_fwd_kernel<C, TOKEN><<<grid, C::NUM_THREADS, smem, st>>>(mq, mk, mv, mkp, mvp, p);
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

// The kernel with pseudo-tile handling only when the token-to-block correction is on.
template <class C>
int launch_fwd(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mkp,
               const CUtensorMap &mvp, const FwdParams &p, int sms, cudaStream_t st) {
  return p.token_corr ? launch_fwd_v<C, true>(mq, mk, mv, mkp, mvp, p, sms, st)
                      : launch_fwd_v<C, false>(mq, mk, mv, mkp, mvp, p, sms, st);
}

template <int D, int BK, int SUBQ>
int dispatch_tiles(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mkp,
                   const CUtensorMap &mvp, FwdParams p, int sms,
                   cudaStream_t st) {
  using C = Cfg<D, BK, SUBQ>;
  return launch_fwd<C>(mq, mk, mv, mkp, mvp, p, sms, st);
}

// The routing pass over B*H heads. cost == null: keep bits only (the routing-only entry
// point); otherwise also the correction records (keep_correct) and the work order.
template <int D, int BK, int SUBQ>
int launch_plan(const FwdParams &p, int BH, uint32_t *keep_out, int *cost, int *order, unsigned int *done,
                int group_heads, cudaStream_t st) {
  auto kern = plan_kernel<D, 128 / SUBQ, BK, SUBQ>;
  static bool attr_set[64] = {};  // per device; guarded by g_mu
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOLATTN_ECUDA;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(plan_smem_bytes<D>(kMaxKeyBlocks))) != cudaSuccess)
        return SOLATTN_ECUDA;
      attr_set[dev] = true;
    }
  }
  const dim3 grid((p.nQB + kPlanQG - 1) / kPlanQG, BH);
  kern<<<grid, kPlanWarps * 32, plan_smem_bytes<D>(p.nKB), st>>>(p, keep_out, cost, order, done, group_heads);
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

int dispatch_plan(int d, int Bq, int Bk, const FwdParams &p, int BH, uint32_t *keep_out, int *cost, int *order,
                  unsigned int *done, int group_heads, cudaStream_t st) {
  const int subq = 128 / Bq;
  if (d == 128) {
    if (Bk == 128) return subq == 1 ? launch_plan<128, 128, 1>(p, BH, keep_out, cost, order, done, group_heads, st)
                                    : launch_plan<128, 128, 2>(p, BH, keep_out, cost, order, done, group_heads, st);
    return subq == 1 ? launch_plan<128, 64, 1>(p, BH, keep_out, cost, order, done, group_heads, st)
                     : launch_plan<128, 64, 2>(p, BH, keep_out, cost, order, done, group_heads, st);
  }
  if (Bk == 128) return subq == 1 ? launch_plan<64, 128, 1>(p, BH, keep_out, cost, order, done, group_heads, st)
                                  : launch_plan<64, 128, 2>(p, BH, keep_out, cost, order, done, group_heads, st);
  return subq == 1 ? launch_plan<64, 64, 1>(p, BH, keep_out, cost, order, done, group_heads, st)
                   : launch_plan<64, 64, 2>(p, BH, keep_out, cost, order, done, group_heads, st);
}

int dispatch(int d, int Bq, int Bk, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
             const CUtensorMap &mkp, const CUtensorMap &mvp, const FwdParams &p, int sms, cudaStream_t st) {
  const int subq = 128 / Bq;
  if (d == 128) {
    if (Bk == 128) return subq == 1 ? dispatch_tiles<128, 128, 1>(mq, mk, mv, mkp, mvp, p, sms, st)
                                    : dispatch_tiles<128, 128, 2>(mq, mk, mv, mkp, mvp, p, sms, st);
    return subq == 1 ? dispatch_tiles<128, 64, 1>(mq, mk, mv, mkp, mvp, p, sms, st)
                     : dispatch_tiles<128, 64, 2>(mq, mk, mv, mkp, mvp, p, sms, st);
  }
  if (Bk == 128) return subq == 1 ? dispatch_tiles<64, 128, 1>(mq, mk, mv, mkp, mvp, p, sms, st)
                                  : dispatch_tiles<64, 128, 2>(mq, mk, mv, mkp, mvp, p, sms, st);
  return subq == 1 ? dispatch_tiles<64, 64, 1>(mq, mk, mv, mkp, mvp, p, sms, st)
                   : dispatch_tiles<64, 64, 2>(mq, mk, mv, mkp, mvp, p, sms, st);
}

// ---- scratch for solattn_forward_noalloc
//
// A fixed device array, reserved when the library's module is loaded on a GPU and kept
// until the process exits, so that callers who cannot allocate device memory still get
// the operator's scratch (work counter, status word, pooled blocks, fp16 copy of V).
// In host code `g_noalloc_scratch` is only a stand-in symbol: its device address is
// looked up with cudaGetSymbolAddress, once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = SOLATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void *g_noalloc_addr[64] = {};

int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOLATTN_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_addr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SOLATTN_ECUDA;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return SOLATTN_OK;
}

// Pooled-key moments per (b, h), then the threshold of every query block.
template <int D>
int launch_threshold_d(const float *qbar, const float *kbar, float *kmom, float *theta, int BH, int nQB, int nKB,
                       float beta, bool diag, cudaStream_t st) {
  gauss_moments_kernel<D><<<BH, 256, 0, st>>>(kbar, kmom, nKB, diag ? 1 : 0);
  if (cudaGetLastError() != cudaSuccess) return SOLATTN_ECUDA;
  const size_t smem = sizeof(float) * ((diag ? D : D * (D + 1)) + 8 * D);
  if (cudaFuncSetAttribute(gauss_theta_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SOLATTN_ECUDA;
  gauss_theta_kernel<D><<<dim3((nQB + 7) / 8, BH), 256, smem, st>>>(qbar, kmom, theta, nQB, beta, diag ? 1 : 0);
  if (cudaGetLastError() != cudaSuccess) return SOLATTN_ECUDA;
  return SOLATTN_OK;
}
int launch_threshold(int d, const float *qbar, const float *kbar, float *kmom, float *theta, int BH, int nQB, int nKB,
                     float beta, bool diag, cudaStream_t st) {
  return d == 64 ? launch_threshold_d<64>(qbar, kbar, kmom, theta, BH, nQB, nKB, beta, diag, st)
                 : launch_threshold_d<128>(qbar, kbar, kmom, theta, BH, nQB, nKB, beta, diag, st);
}

// A device pointer that belongs to another GPU than the current one (the kernels would
// read or write it from the wrong device). Host, managed and unregistered pointers pass:
// the alignment and null checks above cover them, and managed memory is reachable.
bool foreign_device_pointer(const void *p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device != dev;
}

int items_total(int B, int H, int N) {
  // One work item per 128-row query tile.
  return B * H * ((N + 127) / 128);
}

// Routing rule of a forward call: the running maximum with tau, or the query-dependent
// Gaussian threshold with beta (exact covariance or its diagonal).
enum Rule { kRunningMax = 0, kGaussExact = 1, kGaussDiag = 2 };

int forward_impl(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int Bq, int Bk,
                 float tau, int mode, const solattn_stats *stats, void *workspace, size_t ws_bytes, void *stream,
                 void *ev_attn_begin, void *ev_attn_end, int rule = kRunningMax, float beta = 0.f,
                 int n_sink = 0, int token_corr = 0) {
  if (!q || !k || !v || !out || !stats || !stats->kept_per_head) return SOLATTN_EINVAL;
  const int rc = check_shape(B, H, N, d, Bq, Bk);
  if (rc != SOLATTN_OK) return rc;
  if (mode < SOLATTN_DENSE || mode > SOLATTN_KEEP_CORRECT) return SOLATTN_EINVAL;
  if (rule == kRunningMax) {
    if (!(tau >= 0.f)) return SOLATTN_EINVAL;  // negative or NaN
  } else if (beta != beta) {
    return SOLATTN_EINVAL;  // NaN
  }
  if (n_sink < 0 || n_sink > N) return SOLATTN_EINVAL;
  if (token_corr != 0 && token_corr != 1) return SOLATTN_EINVAL;
  const bool token = token_corr && mode == SOLATTN_KEEP_CORRECT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return SOLATTN_EINVAL;
  if (!aligned(stats->kept_per_head, 8) || (stats->keep_mask && !aligned(stats->keep_mask, 4)))
    return SOLATTN_EINVAL;
  const WsLayout wl = ws_layout(B, H, N, d, Bq, Bk);
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < wl.total) return SOLATTN_EWORKSPACE;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SOLATTN_ECUDA;
    const void *ptrs[] = {q, k, v, out, stats->kept_per_head, stats->keep_mask, workspace};
    for (const void *ptr : ptrs)
      if (ptr && foreign_device_pointer(ptr, dev)) return SOLATTN_EINVAL;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int BH = B * H;
  const int nQB = nblocks(N, Bq), nKB = nblocks(N, Bk);
  float *qbar = reinterpret_cast<float *>(ws + wl.qbar);
  float *kbar = reinterpret_cast<float *>(ws + wl.kbar);
  float *vbar = reinterpret_cast<float *>(ws + wl.vbar);
  __half *v16 = reinterpret_cast<__half *>(ws + wl.v16);

  CUtensorMap mq, mk, mv, mkp, mvp;
  if (make_map(&mq, q, d, N, BH, 128) != SOLATTN_OK || make_map(&mk, k, d, N, BH, Bk) != SOLATTN_OK ||
      make_map(&mv, v16, d, N, BH, Bk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != SOLATTN_OK)
    return SOLATTN_ECUDA;
  // Token-to-block correction: the pooled keys (bf16) and values (fp16) of every head, read
  // by the attention kernel as BK-row tiles; otherwise the K/V maps stand in (never read).
  __nv_bfloat16 *kbar16 = reinterpret_cast<__nv_bfloat16 *>(ws + wl.kbar16);
  __half *vbar16 = reinterpret_cast<__half *>(ws + wl.vbar16);
  if (token) {
    if (make_map(&mkp, kbar16, d, nKB, BH, Bk) != SOLATTN_OK ||
        make_map(&mvp, vbar16, d, nKB, BH, Bk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != SOLATTN_OK)
      return SOLATTN_ECUDA;
  } else {
    mkp = mk;
    mvp = mv;
  }

  if (cudaMemsetAsync(ws, 0, kHeaderBytes, st) != cudaSuccess) return SOLATTN_ECUDA;
  if (cudaMemsetAsync(stats->kept_per_head, 0, sizeof(int64_t) * BH, st) != cudaSuccess) return SOLATTN_ECUDA;

  {
    // One pass over the inputs: block means of Q and K (routing) and of V (correction),
    // and the fp16 copy of V for the P.V product. Dense mode needs only the copy.
    const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(v);
    PoolArgs a{};
    a.N = N;
    if (mode == SOLATTN_DENSE) {
      a.job[0] = PoolJob{vb, nullptr, v16, Bk, nKB};
      a.njobs = 1;
    } else {
      a.job[0] = PoolJob{vb, mode == SOLATTN_KEEP_CORRECT ? vbar : nullptr, v16, Bk, nKB};
      a.job[1] = PoolJob{static_cast<const __nv_bfloat16 *>(q), qbar, nullptr, Bq, nQB};
      a.job[2] = PoolJob{static_cast<const __nv_bfloat16 *>(k), kbar, nullptr, Bk, nKB};
      a.njobs = 3;
    }
    NvtxRange r("solattn pool");
    const int rcp = launch_pool(a, BH, d, nQB > nKB ? nQB : nKB, st);
    if (rcp != SOLATTN_OK) return rcp;
  }
  if (token) {
    const size_t n = static_cast<size_t>(BH) * nKB * d;
    const int blocks = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    pooled_copy_kernel<<<blocks, 256, 0, st>>>(kbar, vbar, kbar16, vbar16, n);
    if (cudaGetLastError() != cudaSuccess) return SOLATTN_ECUDA;
  }

  FwdParams p{};
  p.N = N;
  p.nQB = nQB;
  p.nKB = nKB;
  p.mode = mode;
  p.tau = tau;
  p.n_items = items_total(B, H, N);
  p.qbar = qbar;
  p.kbar = kbar;
  p.vbar = vbar;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.kept_per_head = reinterpret_cast<unsigned long long *>(stats->kept_per_head);
  p.keep_mask = stats->keep_mask;
  p.counter = reinterpret_cast<unsigned int *>(ws);
  p.status = reinterpret_cast<int *>(ws + 4);
  p.timeout_ns = kDefaultTimeoutNs;
  p.items_per_head = nblocks(N, 128);
  p.order = nullptr;
  p.theta = nullptr;
  p.n_sink_blocks = nblocks(n_sink, Bk);
  p.token_corr = token ? 1 : 0;
  p.n_pseudo = token ? nblocks(nKB, Bk) : 0;
  p.corr = reinterpret_cast<float *>(ws + wl.corr);
  // Keep bits: into the caller's keep mask when there is one (same layout), else scratch.
  p.keep_bits = mode == SOLATTN_DENSE ? nullptr
                                      : (stats->keep_mask ? stats->keep_mask : reinterpret_cast<uint32_t *>(ws + wl.keep));
  if (mode != SOLATTN_DENSE && rule != kRunningMax) {
    float *kmom = reinterpret_cast<float *>(ws + wl.kmom);
    float *theta = reinterpret_cast<float *>(ws + wl.theta);
    const int rt = launch_threshold(d, qbar, kbar, kmom, theta, BH, nQB, nKB, beta, rule == kGaussDiag, st);
    if (rt != SOLATTN_OK) return rt;
    p.theta = theta;
  }
  if (mode != SOLATTN_DENSE) {
    // Schedule: heads in groups whose K and V16 fit in ~64 MB of L2 together, costliest
    // tiles first within a group.
    const size_t head_kv = static_cast<size_t>(N) * d * 4;
    int group_heads = static_cast<int>((64ull << 20) / (head_kv ? head_kv : 1));
    group_heads = group_heads < 1 ? 1 : (group_heads > BH ? BH : group_heads);
    // The routing pass orders a group's items in shared memory: at most kPlanOrderCap of
    // them (or one head's, up to 1024).
    const int per_head = items_total(1, 1, N);
    if (group_heads > 1 && group_heads * per_head > kPlanOrderCap)
      group_heads = kPlanOrderCap / per_head > 1 ? kPlanOrderCap / per_head : 1;
    int *cost = reinterpret_cast<int *>(ws + wl.cost);
    int *order = reinterpret_cast<int *>(ws + wl.order);
    NvtxRange r("solattn route");
    const int rp = dispatch_plan(d, Bq, Bk, p, BH, p.keep_bits, cost, order, reinterpret_cast<unsigned int *>(ws + 8),
                                 group_heads, st);
    if (rp != SOLATTN_OK) return rp;
    p.order = order;
  }
  if (ev_attn_begin && cudaEventRecord(static_cast<cudaEvent_t>(ev_attn_begin), st) != cudaSuccess)
    return SOLATTN_ECUDA;
  {
    NvtxRange r("solattn attention");
    const int rl = dispatch(d, Bq, Bk, mq, mk, mv, mkp, mvp, p, di.sms, st);
    if (rl != SOLATTN_OK) return rl;
  }
  if (ev_attn_end && cudaEventRecord(static_cast<cudaEvent_t>(ev_attn_end), st) != cudaSuccess)
    return SOLATTN_ECUDA;
  return SOLATTN_OK;
}

// ---- routing on its own (routing-overhead measurement)

template <int P>
int launch_select_t(const float *smap, uint32_t *mask, int rows, int nKB, int N, int Bk, int topp, int k, float pm,
                    cudaStream_t st) {
  select_kernel<P><<<rows, 512, 0, st>>>(smap, mask, nKB, N, Bk, topp, k, pm);
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

// Materialise the proxy map, then select per row (top-k: topp = 0, k; top-p: topp = 1, pm).
int route_select(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk, int topp, int k,
                 float pm, float *proxy_map, size_t map_bytes, uint32_t *keep_mask, void *stream) {
  if (!qbar || !kbar || !proxy_map || !keep_mask) return SOLATTN_EINVAL;
  const int rc = check_shape(B, H, N, d, Bq, Bk);
  if (rc != SOLATTN_OK) return rc;
  if (!aligned(qbar, 16) || !aligned(kbar, 16) || !aligned(proxy_map, 4) || !aligned(keep_mask, 4)) return SOLATTN_EINVAL;
  const int BH = B * H, nQB = nblocks(N, Bq), nKB = nblocks(N, Bk);
  if (map_bytes < static_cast<size_t>(BH) * nQB * nKB * sizeof(float)) return SOLATTN_EWORKSPACE;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid((nKB + 63) / 64, (nQB + 63) / 64, BH);
  if (d == 128)
    proxy_map_kernel<128><<<grid, 256, 0, st>>>(qbar, kbar, proxy_map, nQB, nKB);
  else
    proxy_map_kernel<64><<<grid, 256, 0, st>>>(qbar, kbar, proxy_map, nQB, nKB);
  if (cudaGetLastError() != cudaSuccess) return SOLATTN_ECUDA;
  const int rows = BH * nQB;
  if (nKB <= 64) return launch_select_t<64>(proxy_map, keep_mask, rows, nKB, N, Bk, topp, k, pm, st);
  if (nKB <= 128) return launch_select_t<128>(proxy_map, keep_mask, rows, nKB, N, Bk, topp, k, pm, st);
  if (nKB <= 256) return launch_select_t<256>(proxy_map, keep_mask, rows, nKB, N, Bk, topp, k, pm, st);
  if (nKB <= 512) return launch_select_t<512>(proxy_map, keep_mask, rows, nKB, N, Bk, topp, k, pm, st);
  return launch_select_t<1024>(proxy_map, keep_mask, rows, nKB, N, Bk, topp, k, pm, st);
}

// ---- streams and events of solattn_forward_host, created once per device

constexpr int kHostChunks = 16;  // most chunks of heads one host call pipelines

struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev_start = nullptr, ev_end = nullptr;
  cudaEvent_t ev_up[kHostChunks] = {}, ev_done[kHostChunks] = {};
};
HostPipe g_pipe[64];

int host_pipe(HostPipe **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SOLATTN_ECUDA;
  HostPipe &hp = g_pipe[dev];
  std::lock_guard<std::mutex> lk(hp.mu);
  if (!hp.ready) {
    // Each handle is created once; after a failure the next call creates only the rest.
    auto stream = [](cudaStream_t *x) {
      return *x || cudaStreamCreateWithFlags(x, cudaStreamNonBlocking) == cudaSuccess;
    };
    auto event = [](cudaEvent_t *x) { return *x || cudaEventCreateWithFlags(x, cudaEventDisableTiming) == cudaSuccess; };
    bool ok = stream(&hp.up) && stream(&hp.down) && event(&hp.ev_start) && event(&hp.ev_end);
    for (int c = 0; ok && c < kHostChunks; ++c) ok = event(&hp.ev_up[c]) && event(&hp.ev_done[c]);
    if (!ok) return SOLATTN_ECUDA;
    hp.ready = true;
  }
  *out = &hp;
  return SOLATTN_OK;
}

}  // namespace

extern "C" {

size_t solattn_workspace_size(int B, int H, int N, int d, int Bq, int Bk) {
  if (check_shape(B, H, N, d, Bq, Bk) != SOLATTN_OK) return 0;
  return ws_layout(B, H, N, d, Bq, Bk).total;
}

int solattn_pool(const void *x, float *xbar, int B, int H, int N, int d, int blk, void *stream) {
  if (!x || !xbar) return SOLATTN_EINVAL;
  const int rc = check_shape(B, H, N, d, blk, blk);
  if (rc != SOLATTN_OK) return rc;
  if (!aligned(x, 16) || !aligned(xbar, 16)) return SOLATTN_EINVAL;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  PoolArgs a{};
  a.job[0] = PoolJob{static_cast<const __nv_bfloat16 *>(x), xbar, nullptr, blk, nblocks(N, blk)};
  a.njobs = 1;
  a.N = N;
  return launch_pool(a, B * H, d, nblocks(N, blk), static_cast<cudaStream_t>(stream));
}

int solattn_forward(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int Bq,
                    int Bk, float tau, int mode, const solattn_stats *stats, void *workspace, size_t ws_bytes,
                    void *stream) {
  return forward_impl(q, k, v, out, B, H, N, d, Bq, Bk, tau, mode, stats, workspace, ws_bytes, stream, nullptr,
                      nullptr);
}

int solattn_forward_events(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d,
                           int Bq, int Bk, float tau, int mode, const solattn_stats *stats, void *workspace,
                           size_t ws_bytes, void *stream, void *ev_attn_begin, void *ev_attn_end) {
  return forward_impl(q, k, v, out, B, H, N, d, Bq, Bk, tau, mode, stats, workspace, ws_bytes, stream,
                      ev_attn_begin, ev_attn_end);
}

int solattn_forward_noalloc(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d,
                            int Bq, int Bk, float tau, int mode, const solattn_stats *stats, void *stream) {
  const int rc = check_shape(B, H, N, d, Bq, Bk);
  if (rc != SOLATTN_OK) return rc;
  if (ws_layout(B, H, N, d, Bq, Bk).total > kNoAllocScratchBytes) return SOLATTN_EWORKSPACE;
  void *scratch = nullptr;
  const int rs = noalloc_scratch(&scratch);
  if (rs != SOLATTN_OK) return rs;
  // The forward path clears the scratch header (work counter, status word) on the
  // stream before its kernels run, and overwrites every pooled block it reads.
  return forward_impl(q, k, v, out, B, H, N, d, Bq, Bk, tau, mode, stats, scratch, kNoAllocScratchBytes, stream,
                      nullptr, nullptr);
}

int solattn_forward_gaussian(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d,
                             int Bq, int Bk, float beta, int variant, int mode, const solattn_stats *stats,
                             void *workspace, size_t ws_bytes, void *stream) {
  if (variant != SOLATTN_GAUSS_EXACT && variant != SOLATTN_GAUSS_DIAG) return SOLATTN_EINVAL;
  return forward_impl(q, k, v, out, B, H, N, d, Bq, Bk, 0.f, mode, stats, workspace, ws_bytes, stream, nullptr,
                      nullptr, variant == SOLATTN_GAUSS_EXACT ? kGaussExact : kGaussDiag, beta);
}

int solattn_forward_ex(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d, int Bq,
                       int Bk, const solattn_route *route, int mode, const solattn_stats *stats, void *workspace,
                       size_t ws_bytes, void *stream) {
  if (!route) return SOLATTN_EINVAL;
  int rule;
  switch (route->rule) {
    case SOLATTN_RULE_RUNNING_MAX: rule = kRunningMax; break;
    case SOLATTN_RULE_GAUSS_EXACT: rule = kGaussExact; break;
    case SOLATTN_RULE_GAUSS_DIAG: rule = kGaussDiag; break;
    default: return SOLATTN_EINVAL;
  }
  return forward_impl(q, k, v, out, B, H, N, d, Bq, Bk, route->tau, mode, stats, workspace, ws_bytes, stream, nullptr,
                      nullptr, rule, route->beta, route->n_sink, route->correction);
}

int solattn_get_status(const void *workspace, void *stream) {
  if (!workspace) return SOLATTN_EWORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int status = 0;
  if (cudaMemcpyAsync(&status, static_cast<const uint8_t *>(workspace) + 4, sizeof(int), cudaMemcpyDeviceToHost,
                      st) != cudaSuccess)
    return SOLATTN_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SOLATTN_ECUDA;
  return status;
}

size_t solattn_host_workspace_size(int B, int H, int N, int d, int Bq, int Bk) {
  if (check_shape(B, H, N, d, Bq, Bk) != SOLATTN_OK) return 0;
  const size_t elems = static_cast<size_t>(B) * H * N * d;
  const size_t t = align_up(elems * 2, kAlign);
  const size_t kp = align_up(sizeof(int64_t) * B * H, kAlign);
  const size_t sp = align_up(sizeof(int) * kHostChunks, kAlign);
  return 4 * t + kp + sp + ws_layout(B, H, N, d, Bq, Bk).total;
}

int solattn_forward_host(const void *q, const void *k, const void *v, void *out, int B, int H, int N, int d,
                         int Bq, int Bk, float tau, int mode, int64_t *kept_per_head, void *dev_scratch,
                         size_t scratch_bytes, void *stream) {
  if (!q || !k || !v || !out) return SOLATTN_EINVAL;
  const int rc = check_shape(B, H, N, d, Bq, Bk);
  if (rc != SOLATTN_OK) return rc;
  if (mode < SOLATTN_DENSE || mode > SOLATTN_KEEP_CORRECT || !(tau >= 0.f)) return SOLATTN_EINVAL;
  const size_t need = solattn_host_workspace_size(B, H, N, d, Bq, Bk);
  if (!dev_scratch || !aligned(dev_scratch, kAlign) || scratch_bytes < need) return SOLATTN_EWORKSPACE;
  HostPipe *hp = nullptr;
  const int rp = host_pipe(&hp);
  if (rp != SOLATTN_OK) return rp;
  std::lock_guard<std::mutex> lk(hp->mu);  // the pipe's streams and events serve one call at a time

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t head = static_cast<size_t>(N) * d * 2;  // bytes of one head of q, k, v or out
  const size_t t = align_up(head * BH, kAlign);
  uint8_t *base = static_cast<uint8_t *>(dev_scratch);
  uint8_t *dq = base, *dk = base + t, *dv = base + 2 * t, *dout = base + 3 * t;
  int64_t *dkept = reinterpret_cast<int64_t *>(base + 4 * t);
  int *dstatus = reinterpret_cast<int *>(base + 4 * t + align_up(sizeof(int64_t) * BH, kAlign));
  uint8_t *ws = reinterpret_cast<uint8_t *>(dstatus) + align_up(sizeof(int) * kHostChunks, kAlign);
  const size_t ws_bytes = scratch_bytes - (ws - base);

  // Heads are independent, so the call runs as a pipeline over chunks of heads: the upload
  // of chunk c+1 (stream `up`) and the download of chunk c-1 (stream `down`) overlap the
  // forward of chunk c on the caller's stream. Every result equals the one-call result.
  const int per = (BH + kHostChunks - 1) / kHostChunks;
  const int nch = (BH + per - 1) / per;
  const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k),
                *hv = static_cast<const uint8_t *>(v);
  uint8_t *hout = static_cast<uint8_t *>(out);
  int rf = SOLATTN_OK;
  bool enqueued = false;  // copies may be in flight on the pipe's streams
  auto fail = [&](int code) {
    if (enqueued) {  // the host buffers must outlive every copy that reads or writes them
      cudaStreamSynchronize(hp->up);
      cudaStreamSynchronize(hp->down);
      cudaStreamSynchronize(st);
    }
    return code;
  };
  if (cudaEventRecord(hp->ev_start, st) != cudaSuccess || cudaStreamWaitEvent(hp->up, hp->ev_start, 0) != cudaSuccess)
    return fail(SOLATTN_ECUDA);
  for (int c = 0; c < nch; ++c) {
    const int h0 = c * per, hn = (BH - h0 < per) ? BH - h0 : per;
    const size_t off = head * h0, bytes = head * hn;
    enqueued = true;
    if (cudaMemcpyAsync(dq + off, hq + off, bytes, cudaMemcpyHostToDevice, hp->up) != cudaSuccess ||
        cudaMemcpyAsync(dk + off, hk + off, bytes, cudaMemcpyHostToDevice, hp->up) != cudaSuccess ||
        cudaMemcpyAsync(dv + off, hv + off, bytes, cudaMemcpyHostToDevice, hp->up) != cudaSuccess ||
        cudaEventRecord(hp->ev_up[c], hp->up) != cudaSuccess || cudaStreamWaitEvent(st, hp->ev_up[c], 0) != cudaSuccess)
      return fail(SOLATTN_ECUDA);
    solattn_stats stats{dkept + h0, nullptr};
    rf = solattn_forward(dq + off, dk + off, dv + off, dout + off, 1, hn, N, d, Bq, Bk, tau, mode, &stats, ws, ws_bytes,
                         stream);
    if (rf != SOLATTN_OK) return fail(rf);
    // Each chunk clears the status word when it starts: keep this chunk's.
    if (cudaMemcpyAsync(dstatus + c, ws + 4, sizeof(int), cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaEventRecord(hp->ev_done[c], st) != cudaSuccess ||
        cudaStreamWaitEvent(hp->down, hp->ev_done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(hout + off, dout + off, bytes, cudaMemcpyDeviceToHost, hp->down) != cudaSuccess)
      return fail(SOLATTN_ECUDA);
  }
  int status[kHostChunks] = {};
  if (cudaEventRecord(hp->ev_end, hp->down) != cudaSuccess || cudaStreamWaitEvent(st, hp->ev_end, 0) != cudaSuccess ||
      (kept_per_head &&
       cudaMemcpyAsync(kept_per_head, dkept, sizeof(int64_t) * BH, cudaMemcpyDeviceToHost, st) != cudaSuccess) ||
      cudaMemcpyAsync(status, dstatus, sizeof(int) * nch, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return fail(SOLATTN_ECUDA);
  if (cudaStreamSynchronize(st) != cudaSuccess) return fail(SOLATTN_ECUDA);
  for (int c = 0; c < nch; ++c)
    if (status[c] != SOLATTN_OK) return status[c];
  return SOLATTN_OK;
}

int solattn_watchdog_selftest(void *workspace, size_t ws_bytes, uint64_t limit_ns, void *stream) {
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < kHeaderBytes) return SOLATTN_EWORKSPACE;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int *status = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + 4);
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, st) != cudaSuccess) return SOLATTN_ECUDA;
  watchdog_selftest_kernel<<<1, 32, 0, st>>>(status, static_cast<unsigned long long>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

int solattn_selftest_exp2(const float *x, float *y, int n, void *stream) {
  if (!x || !y || n < 0) return SOLATTN_EINVAL;
  if (n == 0) return SOLATTN_OK;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  const int pairs = (n + 1) / 2;
  exp2_selftest_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? SOLATTN_OK : SOLATTN_ECUDA;
}

int solattn_route_keep(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk, float tau,
                       uint32_t *keep_mask, void *stream) {
  if (!qbar || !kbar || !keep_mask) return SOLATTN_EINVAL;
  const int rc = check_shape(B, H, N, d, Bq, Bk);
  if (rc != SOLATTN_OK) return rc;
  if (!(tau >= 0.f)) return SOLATTN_EINVAL;
  if (!aligned(qbar, 16) || !aligned(kbar, 16) || !aligned(keep_mask, 4)) return SOLATTN_EINVAL;
  DeviceInfo di;
  if (device_info(&di) != SOLATTN_OK) return SOLATTN_ECUDA;
  if (di.major != 10) return SOLATTN_EUNSUPPORTED;
  FwdParams p{};
  p.N = N;
  p.nQB = nblocks(N, Bq);
  p.nKB = nblocks(N, Bk);
  p.mode = SOLATTN_KEEP_DROP;  // keep decisions only
  p.tau = tau;
  p.qbar = qbar;
  p.kbar = kbar;
  // The forward's routing pass with its correction and schedule steps off (cost = null).
  return dispatch_plan(d, Bq, Bk, p, B * H, keep_mask, nullptr, nullptr, nullptr, 1,
                       static_cast<cudaStream_t>(stream));
}

size_t solattn_proxy_map_bytes(int B, int H, int N, int Bq, int Bk) {
  if (check_shape(B, H, N, 128, Bq, Bk) != SOLATTN_OK) return 0;
  return static_cast<size_t>(B) * H * nblocks(N, Bq) * nblocks(N, Bk) * sizeof(float);
}

int solattn_route_topk(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk, int k,
                       float *proxy_map, size_t map_bytes, uint32_t *keep_mask, void *stream) {
  if (k < 1) return SOLATTN_EINVAL;
  return route_select(qbar, kbar, B, H, N, d, Bq, Bk, 0, k, 0.f, proxy_map, map_bytes, keep_mask, stream);
}

int solattn_route_topp(const float *qbar, const float *kbar, int B, int H, int N, int d, int Bq, int Bk, float p,
                       float *proxy_map, size_t map_bytes, uint32_t *keep_mask, void *stream) {
  if (!(p > 0.f && p <= 1.f)) return SOLATTN_EINVAL;
  return route_select(qbar, kbar, B, H, N, d, Bq, Bk, 1, 0, p, proxy_map, map_bytes, keep_mask, stream);
}

const char *solattn_strerror(int status) {
  switch (status) {
    case SOLATTN_OK: return "ok";
    case SOLATTN_EINVAL: return "invalid argument";
    case SOLATTN_EUNSUPPORTED: return "unsupported shape or device";
    case SOLATTN_ECUDA: return "CUDA error";
    case SOLATTN_ETIMEOUT: return "device-side wait timed out";
    case SOLATTN_EWORKSPACE: return "workspace missing, misaligned or too small";
    case SOLATTN_EBOUNDS: return "device-side bounds check failed (debug build)";
    default: return "unknown status";
  }
}

}  // extern "C"
