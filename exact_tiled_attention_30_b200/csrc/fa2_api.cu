// C ABI of the exact tiled attention library (declared in include/fa2.h).
//
// Host side only: argument checks, Tensor Memory Accelerator descriptors,
// kernel selection and launch on the caller's stream. Every kernel of the
// library is compiled into this one translation unit so that they share the
// device status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa2.h"
#include "sm100_ptx.cuh"
#include "fwd_sm100.cuh"
#include "bwd_sm100.cuh"

namespace {

using fa2::FwdCfg;

constexpr int kMaxDevices = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Driver entry points, resolved through the runtime (the library does not link
// libcuda directly, so it loads on machines without a GPU).
void* driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return p;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { fn = reinterpret_cast<EncodeTiledFn>(driver_entry("cuTensorMapEncodeTiled")); });
  return fn;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*MemsetD32AsyncFn)(CUdeviceptr, unsigned int, size_t, CUstream);

// The context current on this thread (nullptr if none or unknown).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { fn = reinterpret_cast<CtxGetCurrentFn>(driver_entry("cuCtxGetCurrent")); });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

MemsetD32AsyncFn memset_d32_fn() {
  static MemsetD32AsyncFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { fn = reinterpret_cast<MemsetD32AsyncFn>(driver_entry("cuMemsetD32Async")); });
  return fn;
}

// Device address of a __device__ symbol, cached per device together with the
// context it was looked up in, and looked up again when the current context
// differs (a cudaDeviceReset or a new primary context frees the old address).
// The caller holds the cache's mutex and has made `dev` current.
struct SymbolCache {
  CUcontext ctx[kMaxDevices] = {};
  void* addr[kMaxDevices] = {};
};

template <class T>
void* symbol_address(SymbolCache& cache, int dev, const T& symbol, fa2_status* st) {
  const CUcontext ctx = current_context();
  if (!cache.addr[dev] || cache.ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      *st = FA2_ERR_CUDA;
      return nullptr;
    }
    cache.addr[dev] = p;
    cache.ctx[dev] = ctx;
  }
  *st = FA2_OK;
  return cache.addr[dev];
}

// Tensor map over a contiguous bf16 [BH, N, d] array seen as 3-D (d, N, BH),
// box = 64 elements of d x box_rows rows x 1 head, 128-byte swizzle. Rows past
// N read as zeros.
bool make_map_bhnd(CUtensorMap* map, const void* base, int BH, int N, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the fp32 dQ accumulator [BH, Np, d] seen as 3-D (d, Np, BH),
// box = 32 elements of d (128 bytes) x 128 rows x 1 head, 128-byte swizzle: the
// backward kernel adds staged dQ tiles into it with TMA reductions.
bool make_map_acc(CUtensorMap* map, float* base, int BH, int Np, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Np),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(Np) * d * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Current device must be compute capability 10.0 (B200 class, sm_100a code).
fa2_status check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  static std::atomic<int> cc[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return FA2_ERR_UNSUPPORTED;
  if (cc[dev].load(std::memory_order_relaxed) == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA2_ERR_CUDA;
    }
    cc[dev].store(major * 10 + minor, std::memory_order_relaxed);
  }
  if (cc[dev].load(std::memory_order_relaxed) != 100) return FA2_ERR_UNSUPPORTED;
  *dev_out = dev;
  return FA2_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa2_status check_common(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1) return FA2_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return FA2_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA2_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return FA2_ERR_UNSUPPORTED;
  // the backward's work items (key tiles x heads) are counted in 32 bits
  if (static_cast<long long>(B) * H * ((N + 127) / 128) > 0x7FFFFFFFLL) return FA2_ERR_UNSUPPORTED;
  // every tensor index must fit the 32-bit TMA coordinates and our size_t math,
  // and the 128-row tiles a grid dimension (at most 65535)
  if (static_cast<long long>(N) > 65535LL * 128) return FA2_ERR_UNSUPPORTED;
  return FA2_OK;
}

template <class KernelT>
fa2_status ensure_smem(KernelT kernel, int bytes, int dev, bool* done) {
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
      cudaGetLastError();
      return FA2_ERR_CUDA;
    }
    done[dev] = true;
  }
  return FA2_OK;
}

int sm_count(int dev);

// Causal kernels walk their work in groups of heads, heaviest items first
// inside a group, so that the tiles every item of a group re-reads stay in L2
// while the group runs. The group is as many heads as fit a share of the
// 126 MB L2 (at most 16): per head the forward re-reads K and V (4 N d bytes)
// and the backward Q, dO and the fp32 dQ accumulator (8 N d bytes). Measured at
// B=1 H=16 N=16384 d=128: 4 heads instead of 16 cut the backward's DRAM
// traffic from 3.0 GB to 0.65 GB a launch (its algorithmic bytes: 0.67 GB) and
// its time by 3 %; at N <= 4096 the group stays 16 heads, the fastest there.
constexpr long long kL2GroupBudget = 64ll << 20;

int causal_head_group(long long bytes_per_head) {
  long long g = bytes_per_head > 0 ? kL2GroupBudget / bytes_per_head : 16;
  return static_cast<int>(g < 1 ? 1 : (g > 16 ? 16 : g));
}

// Work-item counters of the persistent forward kernel. Each launch takes the
// next slot of a ring (one per device) and a fresh nonzero 32-bit tag, and one
// 32-bit memset on the launch's stream writes the tag into both halves of the
// slot right before the kernel (the kernel counts items in the low half from
// the tag up and checks the high half on every item). Launches enqueued under
// stream capture take their slots from a second ring, so eager launches never
// reuse the slot that a captured graph replays with. When more than
// kFwdCounters launches of one ring are in flight at once, a launch can find its
// slot reset by a later one: it then stops taking items and records
// FA2_ERR_CONFLICT in the device status word instead of silently sharing items.
constexpr unsigned int kFwdCounters = 256;
__device__ unsigned long long g_fwd_counters[2 * kFwdCounters];

#ifdef FA2_TEST_HOOKS
std::atomic<int> g_tag_skew{0};  // added to the tag the kernel is given (test builds only)
#endif

unsigned long long* fwd_counter(int dev, cudaStream_t stream, unsigned int* tag, fa2_status* st) {
  static SymbolCache base;
  static unsigned int next[kMaxDevices] = {0}, next_captured[kMaxDevices] = {0}, next_tag[kMaxDevices] = {0};
  static std::mutex mu;
  MemsetD32AsyncFn memset_d32 = memset_d32_fn();
  if (!memset_d32) {
    *st = FA2_ERR_CUDA;
    return nullptr;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
    cudaGetLastError();
    cs = cudaStreamCaptureStatusNone;
  }
  unsigned long long* c = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    void* b = symbol_address(base, dev, g_fwd_counters, st);
    if (!b) return nullptr;
    const unsigned int idx = cs == cudaStreamCaptureStatusActive
                                 ? kFwdCounters + (next_captured[dev]++ % kFwdCounters)
                                 : next[dev]++ % kFwdCounters;
    c = static_cast<unsigned long long*>(b) + idx;
    if (++next_tag[dev] == 0) ++next_tag[dev];
    *tag = next_tag[dev];
  }
  if (memset_d32(reinterpret_cast<CUdeviceptr>(c), *tag, 2, reinterpret_cast<CUstream>(stream)) !=
      CUDA_SUCCESS) {
    *st = FA2_ERR_CUDA;
    return nullptr;
  }
#ifdef FA2_TEST_HOOKS
  *tag += static_cast<unsigned int>(g_tag_skew.load());
#endif
  *st = FA2_OK;
  return c;
}

template <int D>
fa2_status launch_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int Nq, int Nk, int causal, float scale, cudaStream_t stream,
                          int dev) {
  using C = FwdCfg<D>;
  // d = 128 without the causal mask: the instantiation that starts each item's
  // tile 0 while the previous item's tile 1 finishes (every item's two query
  // tiles then have the same number of key tiles)
  const bool early = (D == 128) && !causal;
  static bool smem_set[kMaxDevices] = {false};
  static bool smem_set_early[kMaxDevices] = {false};
  (void)smem_set_early;
  (void)early;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    fa2_status st;
    if constexpr (D == 128)
      st = early ? ensure_smem(fa2::fa2_fwd_kernel<D, true>, C::SMEM_ALLOC, dev, smem_set_early)
                 : ensure_smem(fa2::fa2_fwd_kernel<D, false>, C::SMEM_ALLOC, dev, smem_set);
    else
      st = ensure_smem(fa2::fa2_fwd_kernel<D, false>, C::SMEM_ALLOC, dev, smem_set);
    if (st != FA2_OK) return st;
  }
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (!make_map_bhnd(&tq, q, BH, Nq, D, 128) || !make_map_bhnd(&tk, k, BH, Nk, D, 128) ||
      !make_map_bhnd(&tv, v, BH, Nk, D, 128))
    return FA2_ERR_CUDA;
  fa2::FwdParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.Nq = Nq;
  p.Nk = Nk;
  p.kq_offset = Nk - Nq;
  p.n_qtiles = (Nq + C::BM - 1) / C::BM;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.BH = BH;
  p.head_group = causal_head_group(4ll * Nk * D);
  fa2_status st = FA2_OK;
  p.counter = fwd_counter(dev, stream, &p.tag, &st);
  if (st != FA2_OK) return st;
  // persistent: one CTA per SM (its shared memory and TMEM allow no second one)
  const long long items = static_cast<long long>(BH) * p.n_pairs;
  const int ctas = static_cast<int>(items < sm_count(dev) ? items : sm_count(dev));
  if constexpr (D == 128) {
    if (early)
      fa2::fa2_fwd_kernel<D, true><<<ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
    else
      fa2::fa2_fwd_kernel<D, false><<<ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  } else {
    fa2::fa2_fwd_kernel<D, false><<<ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  }
  if (cudaGetLastError() != cudaSuccess) return FA2_ERR_CUDA;
  return FA2_OK;
}

struct WsLayout {
  float* dq_acc;
  float* delta;
  float* lse2;
  unsigned int* counter;
  int Np;
};

WsLayout ws_layout(void* workspace, int BH, int N, int d) {
  WsLayout w;
  w.Np = (N + 127) / 128 * 128;
  w.dq_acc = reinterpret_cast<float*>(workspace);
  w.delta = w.dq_acc + static_cast<size_t>(BH) * w.Np * d;
  w.lse2 = w.delta + static_cast<size_t>(BH) * w.Np;
  w.counter = reinterpret_cast<unsigned int*>(w.lse2 + static_cast<size_t>(BH) * w.Np);
  return w;
}

int sm_count(int dev) {
  static std::atomic<int> count[kMaxDevices] = {};
  int c = count[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c < 1) {
      cudaGetLastError();
      c = 148;
    }
    count[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

// Grid (blocks per head, heads) of the streaming kernels: about 16 blocks per SM
// in total, each looping over its share of a head.
inline dim3 per_head_grid(long long want_per_head, int BH) {
  long long x = (148LL * 16 + BH - 1) / BH;
  if (x > want_per_head) x = want_per_head;
  if (x < 1) x = 1;
  return dim3(static_cast<unsigned int>(x), static_cast<unsigned int>(BH));
}

template <int D>
fa2_status launch_bwd_pre(const void* o, const float* lse, const void* dO, int BH, int N,
                          void* workspace, cudaStream_t stream) {
  const WsLayout w = ws_layout(workspace, BH, N, D);
  fa2::BwdPreParams pp;
  pp.o = reinterpret_cast<const __nv_bfloat16*>(o);
  pp.dout = reinterpret_cast<const __nv_bfloat16*>(dO);
  pp.lse = lse;
  pp.dq_acc = w.dq_acc;
  pp.delta = w.delta;
  pp.lse2 = w.lse2;
  pp.counter = w.counter;
  pp.N = N;
  pp.Np = w.Np;
  constexpr int rpb = 256 / (D / 8);
  fa2::fa2_bwd_pre_kernel<D><<<per_head_grid((w.Np + rpb - 1) / rpb, BH), 256, 0, stream>>>(pp);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}

template <int D, bool WITH_DQ = true>
fa2_status launch_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk,
                           void* dv, int BH, int Nq, int Nk, int causal, float scale,
                           void* workspace, cudaStream_t stream, int dev) {
  using C = fa2::BwdCfg<D>;
  static bool smem_set[kMaxDevices] = {false};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    fa2_status st = ensure_smem(fa2::fa2_bwd_kernel<D, WITH_DQ>, C::SMEM_ALLOC, dev, smem_set);
    if (st != FA2_OK) return st;
  }
  const WsLayout w = ws_layout(workspace, BH, Nq, D);
  CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
  if (!make_map_bhnd(&tq, q, BH, Nq, D, 128) || !make_map_bhnd(&tk, k, BH, Nk, D, 128) ||
      !make_map_bhnd(&tv, v, BH, Nk, D, 128) || !make_map_bhnd(&tdo, dO, BH, Nq, D, 128) ||
      !make_map_acc(&tdq, w.dq_acc, BH, w.Np, D) || !make_map_bhnd(&tdk, dk, BH, Nk, D, 128) ||
      !make_map_bhnd(&tdv, dv, BH, Nk, D, 128))
    return FA2_ERR_CUDA;
  fa2::BwdParams bp;
  bp.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  bp.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  bp.dq_acc = w.dq_acc;
  bp.lse2 = w.lse2;
  bp.delta = w.delta;
  bp.counter = w.counter;
  bp.Np = w.Np;
  bp.BH = BH;
  bp.n_ktiles = (Nk + 127) / 128;
  bp.n_qtiles = w.Np / 128;
  bp.kq_offset = Nk - Nq;
  bp.causal = causal ? 1 : 0;
  bp.head_group = causal_head_group(8ll * Nq * D);
  bp.scale = scale;
  bp.scale_log2 = scale * 1.4426950408889634f;
  // persistent: one CTA per SM (its shared memory allows no second one)
  const long long items = static_cast<long long>(bp.n_ktiles) * BH;
  const int ctas = static_cast<int>(items < sm_count(dev) ? items : sm_count(dev));
  fa2::fa2_bwd_kernel<D, WITH_DQ><<<ctas, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, tdo, tdq, tdk,
                                                                                    tdv, bp);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}

// dQ by the query-parallel kernel (reads D and LSE2 from the workspace, writes bf16 dq)
template <int D>
fa2_status launch_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dq,
                         int BH, int N, int causal, float scale, void* workspace,
                         cudaStream_t stream, int dev) {
  using C = fa2::BwdDqCfg<D>;
  static bool smem_set[kMaxDevices] = {false};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    fa2_status st = ensure_smem(fa2::fa2_bwd_dq_kernel<D>, C::SMEM_ALLOC, dev, smem_set);
    if (st != FA2_OK) return st;
  }
  const WsLayout w = ws_layout(workspace, BH, N, D);
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_bhnd(&tq, q, BH, N, D, 128) || !make_map_bhnd(&tk, k, BH, N, D, 128) ||
      !make_map_bhnd(&tv, v, BH, N, D, 128) || !make_map_bhnd(&tdo, dO, BH, N, D, 128))
    return FA2_ERR_CUDA;
  fa2::BwdDqParams dp;
  dp.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  dp.lse2 = w.lse2;
  dp.delta = w.delta;
  dp.N = N;
  dp.Np = w.Np;
  dp.BH = BH;
  dp.n_qtiles = w.Np / 128;
  dp.causal = causal ? 1 : 0;
  dp.scale = scale;
  dp.scale_log2 = scale * 1.4426950408889634f;
  const dim3 grid = dp.causal ? dim3(BH * dp.n_qtiles) : dim3(dp.n_qtiles, BH);
  fa2::fa2_bwd_dq_kernel<D><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, tdo, dp);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}

fa2_status launch_bwd_convert(void* dq, int BH, int N, int d, float scale, void* workspace,
                              cudaStream_t stream) {
  const WsLayout w = ws_layout(workspace, BH, N, d);
  fa2::BwdConvertParams cp;
  cp.dq_acc = w.dq_acc;
  cp.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  cp.N = N;
  cp.Np = w.Np;
  cp.d = d;
  cp.head8 = N * (d / 8);
  cp.scale = scale;
  fa2::fa2_bwd_dq_convert_kernel<<<per_head_grid((cp.head8 + 255) / 256, BH), 256, 0, stream>>>(cp);
  return cudaGetLastError() == cudaSuccess ? FA2_OK : FA2_ERR_CUDA;
}

// Query and key lengths of the _qk entry points: each within the limits of one
// sequence, and causal only with Nq <= Nk (bottom-right alignment leaves no
// query row without keys).
fa2_status check_qk(int B, int H, int Nq, int Nk, int d, int causal, float scale) {
  fa2_status st = check_common(B, H, Nq, d, scale);
  if (st == FA2_OK) st = check_common(B, H, Nk, d, scale);
  if (st != FA2_OK) return st;
  if (causal && Nq > Nk) return FA2_ERR_UNSUPPORTED;
  return FA2_OK;
}

fa2_status check_workspace(int B, int H, int N, int d, const void* workspace, size_t bytes) {
  if (!workspace) return FA2_ERR_INVALID_ARG;
  if (bytes < fa2_backward_workspace_size(B, H, N, d)) return FA2_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return FA2_ERR_MISALIGNED;
  return FA2_OK;
}

}  // namespace

extern "C" {

const char* fa2_status_string(int status) {
  switch (status) {
    case FA2_OK: return "FA2_OK";
    case FA2_ERR_INVALID_ARG: return "FA2_ERR_INVALID_ARG";
    case FA2_ERR_UNSUPPORTED: return "FA2_ERR_UNSUPPORTED";
    case FA2_ERR_MISALIGNED: return "FA2_ERR_MISALIGNED";
    case FA2_ERR_CUDA: return "FA2_ERR_CUDA";
    case FA2_ERR_TIMEOUT: return "FA2_ERR_TIMEOUT";
    case FA2_ERR_CONFLICT: return "FA2_ERR_CONFLICT";
    default: return "FA2_ERR_UNKNOWN";
  }
}

fa2_status fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int d, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) return launch_forward<64>(q, k, v, o, lse, B, H, N, N, causal, scale, s, dev);
  return launch_forward<128>(q, k, v, o, lse, B, H, N, N, causal, scale, s, dev);
}

fa2_status fa2_forward_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int Nq, int Nk, int d, int causal, float scale, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_qk(B, H, Nq, Nk, d, causal, scale);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) return launch_forward<64>(q, k, v, o, lse, B, H, Nq, Nk, causal, scale, s, dev);
  return launch_forward<128>(q, k, v, o, lse, B, H, Nq, Nk, causal, scale, s, dev);
}

fa2_status fa2_backward_qk(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                           int H, int Nq, int Nk, int d, int causal, float scale, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_qk(B, H, Nq, Nk, d, causal, scale);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, Nq, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (d == 64) {
    st = launch_bwd_pre<64>(o, lse, dO, BH, Nq, workspace, s);
    if (st == FA2_OK) st = launch_bwd_main<64>(q, k, v, dO, dk, dv, BH, Nq, Nk, causal, scale, workspace, s, dev);
  } else {
    st = launch_bwd_pre<128>(o, lse, dO, BH, Nq, workspace, s);
    if (st == FA2_OK) st = launch_bwd_main<128>(q, k, v, dO, dk, dv, BH, Nq, Nk, causal, scale, workspace, s, dev);
  }
  if (st == FA2_OK) st = launch_bwd_convert(dq, BH, Nq, d, scale, workspace, s);
  return st;
}

size_t fa2_backward_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  const size_t np = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t bh = static_cast<size_t>(B) * H;
  return bh * np * d * 4 + 2 * bh * np * 4 + 16;
}

fa2_status fa2_backward_preprocess(const void* o, const float* lse, const void* dO, int B, int H,
                                   int N, int d, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!o || !lse || !dO) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, 1.0f);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, N, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(o) || !aligned16(lse) || !aligned16(dO)) return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bwd_pre<64>(o, lse, dO, B * H, N, workspace, s)
                 : launch_bwd_pre<128>(o, lse, dO, B * H, N, workspace, s);
}

fa2_status fa2_backward_main(const void* q, const void* k, const void* v, const void* dO, void* dk,
                             void* dv, int B, int H, int N, int d, int causal, float scale,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, N, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bwd_main<64>(q, k, v, dO, dk, dv, B * H, N, N, causal, scale, workspace, s, dev)
                 : launch_bwd_main<128>(q, k, v, dO, dk, dv, B * H, N, N, causal, scale, workspace, s, dev);
}

fa2_status fa2_backward_dq_convert(void* dq, int B, int H, int N, int d, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!dq) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, N, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(dq)) return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  return launch_bwd_convert(dq, B * H, N, d, scale, workspace, reinterpret_cast<cudaStream_t>(stream));
}

fa2_status fa2_backward_main_dkdv(const void* q, const void* k, const void* v, const void* dO,
                                  void* dk, void* dv, int B, int H, int N, int d, int causal,
                                  float scale, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, N, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64
             ? launch_bwd_main<64, false>(q, k, v, dO, dk, dv, B * H, N, N, causal, scale, workspace, s, dev)
             : launch_bwd_main<128, false>(q, k, v, dO, dk, dv, B * H, N, N, causal, scale, workspace, s, dev);
}

fa2_status fa2_backward_dq(const void* q, const void* k, const void* v, const void* dO, void* dq,
                           int B, int H, int N, int d, int causal, float scale, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dq) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  st = check_workspace(B, H, N, d, workspace, workspace_bytes);
  if (st != FA2_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_bwd_dq<64>(q, k, v, dO, dq, B * H, N, causal, scale, workspace, s, dev)
                 : launch_bwd_dq<128>(q, k, v, dO, dq, B * H, N, causal, scale, workspace, s, dev);
}

fa2_status fa2_backward_ex(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                           int H, int N, int d, int causal, float scale, void* workspace,
                           size_t workspace_bytes, int dq_strategy, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace)
    return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  if (dq_strategy != FA2_DQ_AUTO && dq_strategy != FA2_DQ_REDUCE && dq_strategy != FA2_DQ_SEPARATE)
    return FA2_ERR_INVALID_ARG;
  if (workspace_bytes < fa2_backward_workspace_size(B, H, N, d)) return FA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const bool separate = dq_strategy == FA2_DQ_SEPARATE ||
                        (dq_strategy == FA2_DQ_AUTO && fa2_backward_dq_strategy(B, H, N, d, causal) == FA2_DQ_SEPARATE);
  if (d == 64) {
    st = launch_bwd_pre<64>(o, lse, dO, BH, N, workspace, s);
    if (st == FA2_OK)
      st = separate ? launch_bwd_main<64, false>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, workspace, s, dev)
                    : launch_bwd_main<64, true>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, workspace, s, dev);
    if (st == FA2_OK && separate)
      st = launch_bwd_dq<64>(q, k, v, dO, dq, BH, N, causal, scale, workspace, s, dev);
  } else {
    st = launch_bwd_pre<128>(o, lse, dO, BH, N, workspace, s);
    if (st == FA2_OK)
      st = separate ? launch_bwd_main<128, false>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, workspace, s, dev)
                    : launch_bwd_main<128, true>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, workspace, s, dev);
    if (st == FA2_OK && separate)
      st = launch_bwd_dq<128>(q, k, v, dO, dq, BH, N, causal, scale, workspace, s, dev);
  }
  if (st == FA2_OK && !separate) st = launch_bwd_convert(dq, BH, N, d, scale, workspace, s);
  return st;
}

// Measured on B200 for d in {64, 128}, N from 2048 to 16384, causal and not:
// the reductions beat the separate query-parallel kernel by 13-24% everywhere.
int fa2_backward_dq_strategy(int B, int H, int N, int d, int causal) {
  (void)B;
  (void)H;
  (void)N;
  (void)d;
  (void)causal;
  return FA2_DQ_REDUCE;
}

fa2_status fa2_backward(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                        int H, int N, int d, int causal, float scale, void* workspace,
                        size_t workspace_bytes, void* stream) {
  return fa2_backward_ex(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, workspace,
                         workspace_bytes, FA2_DQ_AUTO, stream);
}

fa2_status fa2_get_device_status(void* stream, int* info) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, fa2::g_status, sizeof(word)) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  if (info) *info = static_cast<int>(word & 0xFFFFu);
  if (word & fa2::kStatusTimeout) return FA2_ERR_TIMEOUT;
  if (word & fa2::kStatusConflict) return FA2_ERR_CONFLICT;
  return FA2_OK;
}

fa2_status fa2_clear_device_status(void) {
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(fa2::g_status, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without a caller-provided workspace.
//
// Some callers cannot allocate device memory when they run the backward pass:
// code that reserved all of its device memory up front and may not call
// cudaMalloc afterwards, plugins whose host forbids allocation (and the
// implicit device synchronisation cudaMalloc may cause) on its hot path, or
// plain C callers with no allocator of their own to size a workspace with.
// fa2_backward_noalloc serves them: its scratch (fp32 dQ accumulator, D and the
// log2-scaled LSE) lives in the fixed device array below instead of a
// workspace argument. Every GPU that loads this library keeps the array for
// the life of the process.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA2_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on device `dev` (which must be current).
// In host code the array's name only stands in for the symbol; the address a
// kernel may use comes from cudaGetSymbolAddress, looked up once per device and
// context (again after a cudaDeviceReset).
void* noalloc_scratch(int dev, fa2_status* st) {
  static SymbolCache cache;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  return symbol_address(cache, dev, g_noalloc_scratch, st);
}

}  // namespace

extern "C" {

fa2_status fa2_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                int B, int H, int N, int d, int causal, float scale,
                                void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  if (fa2_backward_workspace_size(B, H, N, d) > static_cast<size_t>(FA2_NOALLOC_SCRATCH_BYTES))
    return FA2_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;
  void* scratch = noalloc_scratch(dev, &st);
  if (st != FA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * H;
  // the preprocess kernel re-zeroes the dQ accumulator and rewrites D and LSE,
  // so whatever an earlier call left in the array does not matter
  if (d == 64) {
    st = launch_bwd_pre<64>(o, lse, dO, BH, N, scratch, s);
    if (st == FA2_OK) st = launch_bwd_main<64>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, scratch, s, dev);
  } else {
    st = launch_bwd_pre<128>(o, lse, dO, BH, N, scratch, s);
    if (st == FA2_OK) st = launch_bwd_main<128>(q, k, v, dO, dk, dv, BH, N, N, causal, scale, scratch, s, dev);
  }
  if (st == FA2_OK) st = launch_bwd_convert(dq, BH, N, d, scale, scratch, s);
  return st;
}

}  // extern "C"

// ------------------------------------------------------- host-buffer pipeline
namespace {

constexpr int kHostSlots = 3;  // chunks in flight

int host_chunk_heads(int BH, int heads_per_chunk) {
  int c = heads_per_chunk > 0 ? heads_per_chunk : (BH + 7) / 8;
  return c < 1 ? 1 : (c > BH ? BH : c);
}

inline size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device layout of one slot: q, k, v, dO, o, dq, dk, dv (bf16 [c, N, d] each),
// lse (fp32 [c, N]), then the backward workspace of c heads.
struct HostSlot {
  size_t tensor_bytes, lse_bytes, ws_bytes, bytes;
};

HostSlot host_slot(int c, int N, int d) {
  HostSlot h;
  h.tensor_bytes = round256(static_cast<size_t>(c) * N * d * 2);
  h.lse_bytes = round256(static_cast<size_t>(c) * N * 4);
  h.ws_bytes = round256(fa2_backward_workspace_size(1, c, N, d));
  h.bytes = 8 * h.tensor_bytes + h.lse_bytes + h.ws_bytes;
  return h;
}

// Three non-blocking streams (copy in, compute, copy out) and the events that
// chain a slot through them, created once per device and kept for the process.
struct HostPipe {
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t entry = nullptr, exit = nullptr;
  cudaEvent_t in_done[kHostSlots] = {}, comp_done[kHostSlots] = {}, out_done[kHostSlots] = {};
  bool used[kHostSlots] = {};
  bool ready = false;
};

HostPipe g_host_pipe[kMaxDevices];
std::mutex g_host_mu;  // serialises enqueueing on the shared streams

fa2_status host_pipe_init(HostPipe& hp) {
  if (hp.ready) return FA2_OK;
  bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.entry, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.exit, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; ok && i < kHostSlots; ++i)
    ok = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  hp.ready = true;
  return FA2_OK;
}

}  // namespace

extern "C" {

size_t fa2_forward_backward_host_workspace_size(int B, int H, int N, int d, int heads_per_chunk) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128) || heads_per_chunk < 0) return 0;
  const int c = host_chunk_heads(B * H, heads_per_chunk);
  return kHostSlots * host_slot(c, N, d).bytes;
}

fa2_status fa2_forward_backward_host(const void* q, const void* k, const void* v, const void* dO,
                                     void* o, float* lse, void* dq, void* dk, void* dv, int B,
                                     int H, int N, int d, int causal, float scale,
                                     int heads_per_chunk, void* device_workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !o || !lse || !dq || !dk || !dv || !device_workspace)
    return FA2_ERR_INVALID_ARG;
  if (heads_per_chunk < 0) return FA2_ERR_INVALID_ARG;
  fa2_status st = check_common(B, H, N, d, scale);
  if (st != FA2_OK) return st;
  if (workspace_bytes < fa2_forward_backward_host_workspace_size(B, H, N, d, heads_per_chunk))
    return FA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(device_workspace) & 255u) != 0) return FA2_ERR_MISALIGNED;
  int dev = 0;
  st = check_device(&dev);
  if (st != FA2_OK) return st;

  const int BH = B * H;
  const int c = host_chunk_heads(BH, heads_per_chunk);
  const HostSlot hs = host_slot(c, N, d);
  const size_t head_elems = static_cast<size_t>(N) * d;  // bf16 elements of one head

  std::lock_guard<std::mutex> lock(g_host_mu);
  HostPipe& hp = g_host_pipe[dev];
  st = host_pipe_init(hp);
  if (st != FA2_OK) return st;
  cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  bool ok = cudaEventRecord(hp.entry, user) == cudaSuccess &&
            cudaStreamWaitEvent(hp.in, hp.entry, 0) == cudaSuccess;
  const char* hq = static_cast<const char*>(q);
  const char* hk = static_cast<const char*>(k);
  const char* hv = static_cast<const char*>(v);
  const char* hdo = static_cast<const char*>(dO);
  char* ho = static_cast<char*>(o);
  char* hdq = static_cast<char*>(dq);
  char* hdk = static_cast<char*>(dk);
  char* hdv = static_cast<char*>(dv);
  for (int h0 = 0, chunk = 0; ok && h0 < BH; h0 += c, ++chunk) {
    const int slot = chunk % kHostSlots;
    const int nh = BH - h0 < c ? BH - h0 : c;
    const size_t tb = static_cast<size_t>(nh) * head_elems * 2;  // bytes of one tensor chunk
    const size_t off = static_cast<size_t>(h0) * head_elems * 2;
    char* base = static_cast<char*>(device_workspace) + slot * hs.bytes;
    char* dt[8];  // q, k, v, dO, o, dq, dk, dv
    for (int i = 0; i < 8; ++i) dt[i] = base + i * hs.tensor_bytes;
    float* dlse = reinterpret_cast<float*>(base + 8 * hs.tensor_bytes);
    void* dws = base + 8 * hs.tensor_bytes + hs.lse_bytes;
    // copy in, once the outputs of the chunk that used this slot are out
    if (hp.used[slot]) ok = ok && cudaStreamWaitEvent(hp.in, hp.out_done[slot], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dt[0], hq + off, tb, cudaMemcpyHostToDevice, hp.in) == cudaSuccess &&
         cudaMemcpyAsync(dt[1], hk + off, tb, cudaMemcpyHostToDevice, hp.in) == cudaSuccess &&
         cudaMemcpyAsync(dt[2], hv + off, tb, cudaMemcpyHostToDevice, hp.in) == cudaSuccess &&
         cudaMemcpyAsync(dt[3], hdo + off, tb, cudaMemcpyHostToDevice, hp.in) == cudaSuccess &&
         cudaEventRecord(hp.in_done[slot], hp.in) == cudaSuccess;
    // forward + backward of the chunk's heads (as B = 1, H = nh)
    ok = ok && cudaStreamWaitEvent(hp.comp, hp.in_done[slot], 0) == cudaSuccess;
    if (!ok) break;
    st = fa2_forward(dt[0], dt[1], dt[2], dt[4], dlse, 1, nh, N, d, causal, scale, hp.comp);
    if (st == FA2_OK)
      st = fa2_backward(dt[0], dt[1], dt[2], dt[4], dlse, dt[3], dt[5], dt[6], dt[7], 1, nh, N, d,
                        causal, scale, dws, hs.ws_bytes, hp.comp);
    if (st != FA2_OK) break;
    ok = cudaEventRecord(hp.comp_done[slot], hp.comp) == cudaSuccess &&
         cudaStreamWaitEvent(hp.out, hp.comp_done[slot], 0) == cudaSuccess;
    // copy out
    const size_t loff = static_cast<size_t>(h0) * N * 4;
    ok = ok && cudaMemcpyAsync(ho + off, dt[4], tb, cudaMemcpyDeviceToHost, hp.out) == cudaSuccess &&
         cudaMemcpyAsync(reinterpret_cast<char*>(lse) + loff, dlse, static_cast<size_t>(nh) * N * 4,
                         cudaMemcpyDeviceToHost, hp.out) == cudaSuccess &&
         cudaMemcpyAsync(hdq + off, dt[5], tb, cudaMemcpyDeviceToHost, hp.out) == cudaSuccess &&
         cudaMemcpyAsync(hdk + off, dt[6], tb, cudaMemcpyDeviceToHost, hp.out) == cudaSuccess &&
         cudaMemcpyAsync(hdv + off, dt[7], tb, cudaMemcpyDeviceToHost, hp.out) == cudaSuccess &&
         cudaEventRecord(hp.out_done[slot], hp.out) == cudaSuccess;
    hp.used[slot] = true;
  }
  // the caller's stream continues once the last copy out has completed (the
  // copy-out stream runs the chunks in order)
  const bool joined = cudaEventRecord(hp.exit, hp.out) == cudaSuccess &&
                      cudaStreamWaitEvent(user, hp.exit, 0) == cudaSuccess;
  if (st != FA2_OK) return st;
  if (!ok || !joined) {
    cudaGetLastError();
    return FA2_ERR_CUDA;
  }
  return FA2_OK;
}

}  // extern "C"

#ifdef FA2_TEST_HOOKS
// Test-hooks builds only: the forward kernels launched after this call are given
// their slot's tag plus `skew`, so that a nonzero skew makes every launch see a
// foreign tag in its work counter (the FA2_ERR_CONFLICT path). Returns 0.
extern "C" FA2_API int fa2_debug_forward_tag_skew(int skew) {
  g_tag_skew.store(skew);
  return 0;
}

// Test-hooks builds only: plants (key_tile > 0) or removes (0) the forward
// producer's skipped load described at g_test_stall_kv. Returns 0 on success.
extern "C" FA2_API int fa2_debug_set_stall(int key_tile) {
  return cudaMemcpyToSymbol(fa2::g_test_stall_kv, &key_tile, sizeof(key_tile)) == cudaSuccess ? 0 : 1;
}
#endif

#ifdef FA2_TRACE
// Debug builds only: copies the trace stamps of the last traced launch.
extern "C" FA2_API int fa2_debug_trace_read(unsigned long long* host, int n) {
  if (n > 64 * 64) n = 64 * 64;
  return cudaMemcpyFromSymbol(host, fa2::g_trace, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : 1;
}
#endif
