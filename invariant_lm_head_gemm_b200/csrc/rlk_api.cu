// rlk_api.cu -- the C ABI declared in include/rlk.h: argument checks,
// workspace layout, TMA tensor-map encoding and the launch sequences of the
// forward and backward passes.  No allocation, no host synchronisation
// (except rlk_read_device_error), no fallback path.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "rlk.h"
#include "rlk_decode.cuh"
#include "rlk_device.h"
#include "rlk_kernel.cuh"

namespace rlk {
namespace {

// Vocab tiles per forward unit: each (row, split of 2 x 256 vocab entries)
// yields one online triple.  Fixed, so partials never depend on T.
constexpr int kFwdGroup = 2;
// Vocab chunk of the backward: dlogits for kVChunk vocab entries at a time
// go through the workspace.  Fixed (for a given V), so dHidden rows never
// depend on T.
constexpr int64_t kVChunk = 8192;
constexpr size_t kHeader = 256;  // device error word + padding

std::atomic<uint64_t> g_calls[3];

constexpr int kMaxDevices = 64;
// Per-device facts looked up on first use.  Host threads may race to fill a
// slot (each writes the same value); the SM count is published before the
// state that says it is valid.
std::atomic<int> g_dev_state[kMaxDevices];  // 0 unknown, 1 supported, 2 unsupported
std::atomic<int> g_dev_sms[kMaxDevices];

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int64_t fwd_groups(int64_t V) { return ceil_div(ceil_div(V, kBN), kFwdGroup); }

// Vocab columns per backward chunk (a multiple of kBN, at most kVChunk).
int64_t vchunk(int64_t V) { return std::min<int64_t>(kVChunk, ceil_div(V, kBN) * kBN); }

// Plan of the fused backward for these sizes (see rlk_bwd.cuh).
BwdPlan bwd_plan(int64_t T, int64_t H, int64_t V) { return make_bwd_plan(T, H, V, vchunk(V)); }

size_t bwd_counter_words(const BwdPlan& p) {
  const size_t nc = static_cast<size_t>(p.NC);
  return nc * p.MT + nc * p.RT_full + nc * p.MT * p.NH + nc + 1;
}

struct Layout {
  size_t pm, ps, pb, yt, fwd_end;
  size_t dx[kDxBuffers], dh, cnt, bwd_end;
};

Layout layout(int64_t T, int64_t H, int64_t V) {
  Layout L;
  const size_t G = static_cast<size_t>(fwd_groups(V));
  const size_t t = static_cast<size_t>(T);
  L.pm = kHeader;
  L.ps = L.pm + align256(G * t * 4);
  L.pb = L.ps + align256(G * t * 4);
  L.yt = L.pb + align256(G * t * 4);
  L.fwd_end = L.yt + align256(t * 4);
  const size_t dx_bytes = align256(t * static_cast<size_t>(vchunk(V)) * 2);
  L.dx[0] = kHeader;
  for (int i = 1; i < kDxBuffers; ++i) L.dx[i] = L.dx[i - 1] + dx_bytes;
  L.dh = L.dx[kDxBuffers - 1] + dx_bytes;
  L.cnt = L.dh + align256(t * static_cast<size_t>(H) * 4);
  L.bwd_end = L.cnt + align256(bwd_counter_words(bwd_plan(T, H, V)) * 4);
  return L;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

rlk_status check_sizes(int64_t T, int64_t H, int64_t V, float temperature) {
  if (T < 0 || H <= 0 || V <= 0) return RLK_ERR_INVALID_ARG;
  if (!std::isfinite(temperature) || !(temperature > 0.f)) return RLK_ERR_INVALID_ARG;
  if (!std::isfinite(kLog2e / temperature)) return RLK_ERR_INVALID_ARG;
  if (H % 64 != 0 || H > (int64_t{1} << 20)) return RLK_ERR_UNSUPPORTED_SHAPE;
  if (V >= (int64_t{1} << 31) || T >= (int64_t{1} << 31)) return RLK_ERR_UNSUPPORTED_SHAPE;
  // unit indices of the backward travel as 32-bit integers
  if (make_bwd_plan(T, H, V, vchunk(V)).total >= (int64_t{1} << 31)) return RLK_ERR_UNSUPPORTED_SHAPE;
  return RLK_OK;
}

// Current device must be compute capability 10.0 (B200, sm_100a code).
rlk_status check_device(int* num_sms) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) {
    cudaGetLastError();
    return RLK_ERR_UNSUPPORTED_DEVICE;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return RLK_ERR_UNSUPPORTED_DEVICE;
  int state = g_dev_state[dev].load(std::memory_order_acquire);
  if (state == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return RLK_ERR_CUDA;
    }
    state = (major == 10 && minor == 0) ? 1 : 2;
    g_dev_sms[dev].store(sms, std::memory_order_relaxed);
    g_dev_state[dev].store(state, std::memory_order_release);
  }
  if (state != 1) return RLK_ERR_UNSUPPORTED_DEVICE;
  *num_sms = g_dev_sms[dev].load(std::memory_order_relaxed);
  return RLK_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// A driver entry point by name, or null.
void* driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return p;
  cudaGetLastError();
  return nullptr;
}

EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn =
      reinterpret_cast<EncodeTiledFn>(driver_fn("cuTensorMapEncodeTiled"));
  return fn;
}

// 2-D bf16 tensor map over a row-major matrix with `inner` contiguous
// elements per row, `outer` rows and a row pitch of `pitch_elems`; boxes of
// box_inner x box_outer, 128-byte swizzle, zero fill outside the matrix.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch_elems, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MN-major operand stored [K, MN] (MN contiguous, pitch elements per K row)
// mapped 3-D as (64 MN, K, MN / 64) with box 64 x 64 x 2: one copy lands the
// 128 MN columns of a stage as two 8 KB 64 x 64 swizzled blocks back to back,
// the same bytes and layout as two 2-D boxes.  Needs MN % 64 == 0; false if
// the driver declines the map.
bool map_mnmajor3(CUtensorMap* m, const void* base, int64_t MN, int64_t K, int64_t pitch) {
  if (MN % 64 != 0) return false;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(MN / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch) * 2, 128};
  cuuint32_t box[3] = {64, 64, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major operand [rows, K] (K contiguous, pitch elements per row) mapped 3-D
// as (64 K, rows, K / 64) with box 64 x 128 x 2: one copy lands two K blocks of
// 128 rows as two 16 KB swizzled blocks back to back, the same bytes and layout
// as two 2-D boxes.  Needs K % 64 == 0 (a 2-D box fills zeros past K, this map
// would read on into the next row); false if the driver declines the map.
bool map_kmajor3(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int64_t pitch) {
  if (K % 64 != 0) return false;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch) * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBM), 2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major operand [rows, K] (K contiguous): one 64 x box_rows box per K block.
bool map_kmajor(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int64_t pitch,
                uint32_t box_rows) {
  return make_map(m, base, K, rows, pitch, 64, box_rows);
}

// MN-major operand stored [K, MN] (MN contiguous): 64 x 64 boxes.
bool map_mnmajor(CUtensorMap* m, const void* base, int64_t MN, int64_t K, int64_t pitch) {
  return make_map(m, base, MN, K, pitch, 64, 64);
}

typedef CUresult (*StreamWaitValueFn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
typedef CUresult (*StreamWriteValueFn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);

// Sets n chunk-completion words to `seq` in stream order (no kernel).
rlk_status write_chunk_words(uint32_t* words, int64_t n, uint32_t seq, cudaStream_t st) {
  static const StreamWriteValueFn write =
      reinterpret_cast<StreamWriteValueFn>(driver_fn("cuStreamWriteValue32"));
  if (!write) return RLK_ERR_CUDA;
  for (int64_t c = 0; c < n; ++c)
    if (write(static_cast<CUstream>(st), reinterpret_cast<CUdeviceptr>(words + c), seq, 0) !=
        CUDA_SUCCESS)
      return RLK_ERR_CUDA;
  return RLK_OK;
}

std::atomic<int> g_max_clusters[3][kMaxDevices];

// Launches pair_kernel<Mode> on clusters of two CTAs: at most one cluster per
// unit and no more clusters than can be resident at once.  `cooperative`
// makes the launch fail rather than start with some CTAs not resident (the
// backward's units wait on each other).
template <int Mode>
rlk_status launch_pair(const typename ModeArgs<Mode>::type& args, long long total,
                       bool cooperative, cudaStream_t st) {
  if (total <= 0) return RLK_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  auto kern = pair_kernel<Mode>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(PipeCfg<Mode>::kSmemBytes)) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PipeCfg<Mode>::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int mc = g_max_clusters[Mode][dev].load(std::memory_order_relaxed);
  if (mc == 0) {
    cfg.gridDim = dim3(2);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return RLK_ERR_CUDA;
    }
    mc = n;
    g_max_clusters[Mode][dev].store(n, std::memory_order_relaxed);
  }
  cfg.numAttrs = cooperative ? 2 : 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * std::min<long long>(total, mc)));
  if (cudaLaunchKernelEx(&cfg, kern, args) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  return RLK_OK;
}

// Forward, first half: the pair-tile GEMM over the `Vloc` rows of W (global
// vocab rows v0 .. v0 + Vloc) with the online epilogue, writing one triple per
// (row, 512-column split) to part_* ([T][ceil(Vloc / 512)]) and, for rows whose
// target falls in these rows, the target's scaled logit to ytgt.
static_assert(kDecSplit == kBN * kFwdGroup, "both forward kernels must use the same splits");

std::atomic<int> g_dec_max_clusters[2][3][kDecMaxRows / 16][kMaxDevices];  // store, form, N/16-1

// The MMA width of the short-batch kernel for T rows: 16, or T rounded up to 32.
int dec_width(int64_t T) { return T <= 16 ? 16 : static_cast<int>(ceil_div(T, 32) * 32); }

// Launches the short-batch kernel (rlk_decode.cuh) on args whose maps, epilogue
// fields, KB and NG are set: the single-CTA MMA form below N = kDecPairMinN, the
// CTA-pair form from there (its hidden map's box must then hold N / 2 rows);
// `store` selects the plain GEMM epilogue instead of the online fold, and
// `half` (with `store`, N <= kDecHalfMaxN) the half-height single-CTA form,
// whose W map's box holds 64 rows and whose units cover 256 W rows.
rlk_status launch_short(DecArgs& a, bool store, cudaStream_t st, bool half = false) {
  if (half && (!store || a.N > kDecHalfMaxN)) return RLK_ERR_INVALID_ARG;
  const bool pair = !half && a.N >= kDecPairMinN;
  constexpr uint32_t kSmemLimit = 227u * 1024u;
  a.stages = dec_stages(a.N, pair, kSmemLimit, half);
  if (a.stages == 0) return RLK_ERR_CUDA;
  const uint32_t smem = dec_smem_bytes(a.N, a.stages, pair, half);
  void (*kern)(DecArgs) =
      half ? decode_fwd_kernel<false, true, true>
           : store ? (pair ? decode_fwd_kernel<true, true> : decode_fwd_kernel<false, true>)
                   : (pair ? decode_fwd_kernel<true, false> : decode_fwd_kernel<false, false>);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemLimit)) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kDecCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  std::atomic<int>& cache = g_dec_max_clusters[store ? 1 : 0][half ? 2 : pair ? 1 : 0][a.N / 16 - 1][dev];
  int mc = cache.load(std::memory_order_relaxed);
  if (mc == 0) {
    cfg.gridDim = dim3(kDecCluster);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return RLK_ERR_CUDA;
    }
    mc = n;
    cache.store(n, std::memory_order_relaxed);
  }
  cfg.gridDim = dim3(static_cast<unsigned>(kDecCluster * std::min<int>(a.NG, mc)));
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  return RLK_OK;
}

// Forward partials for T <= kDecMaxT (decode_fwd_kernel, rlk_decode.cuh).
rlk_status enqueue_fwd_partials_short(const rlk_bf16* hidden, const rlk_bf16* W,
                                      const int64_t* targets, int64_t T, int64_t H, int64_t Vloc,
                                      int64_t v0, float temperature, float* part_m, float* part_s,
                                      float* part_b, int64_t ldp, float* ytgt, uint32_t* err,
                                      cudaStream_t st, uint64_t wait_limit_ns = kWaitLimitNs,
                                      int stall = 0) {
  DecArgs a;
  a.wait_limit_ns = wait_limit_ns;
  a.stall = stall;
  a.N = dec_width(T);
  const bool pair = a.N >= kDecPairMinN;
  if (!map_kmajor(&a.w_k, W, H, Vloc, H, kBM) ||
      !map_kmajor(&a.hid_k, hidden, H, T, H, pair ? a.N / 2 : a.N))
    return RLK_ERR_CUDA;
  a.ep.targets = targets;
  a.ep.part_m = part_m;
  a.ep.part_s = part_s;
  a.ep.part_b = part_b;
  a.ep.ytgt = ytgt;
  a.ep.T = static_cast<int>(T);
  a.ep.V = static_cast<int>(Vloc);
  a.ep.ldp = static_cast<int>(ldp);
  a.ep.v0 = v0;
  a.ep.scale_log2 = kLog2e / temperature;
  a.err = err;
  a.KB = static_cast<int>(H / kBK);
  a.NG = static_cast<int>(fwd_groups(Vloc));
  return launch_short(a, false, st);
}

rlk_status enqueue_fwd_partials(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                                int64_t T, int64_t H, int64_t Vloc, int64_t v0, float temperature,
                                float* part_m, float* part_s, float* part_b, int64_t ldp,
                                float* ytgt, uint32_t* err, cudaStream_t st) {
  if (T <= kDecMaxT)
    return enqueue_fwd_partials_short(hidden, W, targets, T, H, Vloc, v0, temperature, part_m,
                                      part_s, part_b, ldp, ytgt, err, st);
  FwdArgs a;
  // 3-D maps (one copy per operand and stage) when the driver takes them
  a.k3 = map_kmajor3(&a.hid_k, hidden, H, T, H) && map_kmajor3(&a.w_k, W, H, Vloc, H) ? 1 : 0;
  if (!a.k3 &&
      (!map_kmajor(&a.hid_k, hidden, H, T, H, kBM) || !map_kmajor(&a.w_k, W, H, Vloc, H, kBM)))
    return RLK_ERR_CUDA;
  a.ep.targets = targets;
  a.ep.part_m = part_m;
  a.ep.part_s = part_s;
  a.ep.part_b = part_b;
  a.ep.ytgt = ytgt;
  a.ep.T = static_cast<int>(T);
  a.ep.V = static_cast<int>(Vloc);
  a.ep.ldp = static_cast<int>(ldp);
  a.ep.v0 = v0;
  a.ep.scale_log2 = kLog2e / temperature;
  a.err = err;
  a.MT = static_cast<int>(ceil_div(T, kPairM));
  a.NT = static_cast<int>(ceil_div(Vloc, kBN));
  a.group = kFwdGroup;
  a.NG = static_cast<int>(fwd_groups(Vloc));
  a.KB = static_cast<int>(H / kBK);
  a.total = static_cast<long long>(a.MT) * a.NG;
  return launch_pair<kModeFwd>(a, a.total, false, st);
}

// Forward, second half: merge the splits (layout [nshards][T][Gs]) in global
// split order.
rlk_status enqueue_combine(const float* pm, const float* ps, const float* pb, int64_t Gs,
                           const float* ytgt, const int64_t* targets, int64_t T, int64_t V,
                           float* logp, float* entropy, float* lse, uint32_t* err,
                           cudaStream_t st) {
  combine_kernel<<<static_cast<unsigned>(ceil_div(T, 8)), 256, 0, st>>>(
      pm, ps, pb, ytgt, targets, static_cast<int>(T), static_cast<int>(V),
      static_cast<int>(fwd_groups(V)), static_cast<int>(Gs), logp, entropy, lse, err);
  return cudaGetLastError() == cudaSuccess ? RLK_OK : RLK_ERR_CUDA;
}

rlk_status enqueue_fwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                       int64_t T, int64_t H, int64_t V, float temperature, float* logp,
                       float* entropy, float* lse, uint8_t* ws, const Layout& L,
                       cudaStream_t st) {
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  float* pm = reinterpret_cast<float*>(ws + L.pm);
  float* ps = reinterpret_cast<float*>(ws + L.ps);
  float* pb = reinterpret_cast<float*>(ws + L.pb);
  float* yt = reinterpret_cast<float*>(ws + L.yt);
  rlk_status s = enqueue_fwd_partials(hidden, W, targets, T, H, V, 0, temperature, pm, ps, pb,
                                      fwd_groups(V), yt, err, st);
  if (s != RLK_OK) return s;
  return enqueue_combine(pm, ps, pb, fwd_groups(V), yt, targets, T, V, logp, entropy, lse, err,
                         st);
}

// Backward over W rows [v0, v0 + Vloc) of a Vfull-row head (the whole head:
// v0 = 0, Vloc = Vfull), chunked as the full head is.  dh_parts null: dHidden
// accumulated over the chunks and written as bf16; else each chunk's fp32
// product goes to dh_parts (EpiDh::kPart layout).
rlk_status enqueue_bwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                       int64_t T, int64_t H, int64_t Vloc, int64_t v0, int64_t Vfull,
                       float temperature, const float* lse, const float* entropy,
                       const float* dlogp, const float* dentropy, rlk_bf16* dHidden,
                       float* dh_parts, int64_t part_rows, int64_t part_chunks, float* dW,
                       uint8_t* ws, const Layout& L, cudaStream_t st,
                       uint64_t wait_limit_ns = kWaitLimitNs, int stall_first_h = 0,
                       uint32_t* chunk_done = nullptr, uint32_t seq = 0) {
  BwdParams P;
  P.plan = make_bwd_plan(T, H, Vloc, vchunk(Vfull));
  const BwdPlan& pl = P.plan;
  void* dx[kDxBuffers];
  for (int i = 0; i < kDxBuffers; ++i) {
    dx[i] = ws + L.dx[i];
    if (!make_map(&P.maps.dx_st[i], dx[i], pl.ldx, T, pl.ldx, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return RLK_ERR_CUDA;
  }
  // K-major operands of the recompute and dHidden units: one 2-D box per K
  // block (the forward's one-copy 3-D stages made this kernel 1.7% slower)
  if (!map_kmajor(&P.maps.hid_k, hidden, H, T, H, kBM) ||
      !map_kmajor(&P.maps.w_k, W, H, Vloc, H, kBM))
    return RLK_ERR_CUDA;
  for (int i = 0; i < kDxBuffers; ++i)
    if (!map_kmajor(&P.maps.dx_k[i], dx[i], pl.ldx, T, pl.ldx, kBM)) return RLK_ERR_CUDA;
  // MN-major operands of the dHidden and dW units: 3-D maps (half the copies)
  // when the driver takes them, else 2-D maps; same shared-memory bytes.
  bool mn3 = map_mnmajor3(&P.maps.w_mn, W, H, Vloc, H) &&
             map_mnmajor3(&P.maps.hid_mn, hidden, H, T, H);
  for (int i = 0; mn3 && i < kDxBuffers; ++i)
    mn3 = map_mnmajor3(&P.maps.dx_mn[i], dx[i], pl.ldx, T, pl.ldx);
  if (!mn3) {
    if (!map_mnmajor(&P.maps.w_mn, W, H, Vloc, H) || !map_mnmajor(&P.maps.hid_mn, hidden, H, T, H))
      return RLK_ERR_CUDA;
    for (int i = 0; i < kDxBuffers; ++i)
      if (!map_mnmajor(&P.maps.dx_mn[i], dx[i], pl.ldx, T, pl.ldx)) return RLK_ERR_CUDA;
  }
  P.mn3 = mn3 ? 1 : 0;
  P.targets = targets;
  P.lse = lse;
  P.entropy = entropy;
  P.dlogp = dlogp;
  P.dentropy = dentropy;
  P.dh_acc = reinterpret_cast<float*>(ws + L.dh);
  P.dhidden = reinterpret_cast<__nv_bfloat16*>(dHidden);
  P.dh_parts = dh_parts;
  P.part_rows = static_cast<int>(part_rows);
  P.part_chunks = static_cast<int>(part_chunks);
  P.v0 = v0;
  P.Vfull = Vfull;
  P.dW = dW;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ws + L.cnt);
  const size_t nc = static_cast<size_t>(pl.NC);
  P.rdone_m = cnt;
  P.rdone_j = P.rdone_m + nc * pl.MT;
  P.hdone = P.rdone_j + nc * pl.RT_full;
  P.bufdone = P.hdone + nc * pl.MT * pl.NH;
  P.next_unit = P.bufdone + nc;
  P.err = reinterpret_cast<uint32_t*>(ws);
  P.scale_log2 = kLog2e / temperature;
  P.inv_tau = 1.0f / temperature;
  P.wait_limit_ns = wait_limit_ns;
  P.stall_first_h = stall_first_h;
  P.chunk_done = chunk_done;
  P.seq = seq;

  if (cudaMemsetAsync(cnt, 0, bwd_counter_words(pl) * 4, st) != cudaSuccess) return RLK_ERR_CUDA;
  // Units wait on units claimed earlier, and only running CTA pairs claim
  // units, so no pair ever waits on one that has not started: the launch needs
  // no co-residency guarantee.
  return launch_pair<kModeBwd>(P, pl.total, false, st);
}

}  // namespace

rlk_status current_device_supported(int* num_sms) { return check_device(num_sms); }

}  // namespace rlk

using namespace rlk;

extern "C" {

size_t rlk_linear_logp_workspace_bytes(int64_t T, int64_t H, int64_t V, int for_backward) {
  if (check_sizes(T, H, V, 1.0f) != RLK_OK) return 0;
  const Layout L = layout(T, H, V);
  return for_backward ? std::max(L.fwd_end, L.bwd_end) : L.fwd_end;
}

rlk_status rlk_linear_logp_fwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                               int64_t T, int64_t H, int64_t V, float temperature, float* logp,
                               float* entropy, float* lse, void* workspace,
                               size_t workspace_bytes, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (T == 0) return RLK_OK;
  if (!hidden || !W || !targets || !logp || !entropy || !lse || !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(workspace, 256) ||
      !aligned(targets, 8) || !aligned(logp, 4) || !aligned(entropy, 4) || !aligned(lse, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (workspace_bytes < L.fwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  s = enqueue_fwd(hidden, W, targets, T, H, V, temperature, logp, entropy, lse,
                  static_cast<uint8_t*>(workspace), L, st);
  if (s != RLK_OK) return s;
  g_calls[0].fetch_add(1);
  return RLK_OK;
}

// Test hook (declared in rlk.h): the short-batch forward with a chosen bound
// on every wait and, with stall set, one wait that nothing satisfies.
rlk_status rlk_test_linear_logp_fwd_stall(const rlk_bf16* hidden, const rlk_bf16* W,
                                          const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                          float temperature, float* logp, float* entropy,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          uint64_t wait_limit_ns, int stall, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (T < 1 || T > kDecMaxT || wait_limit_ns < 1000000ull || wait_limit_ns > kWaitLimitNs)
    return RLK_ERR_INVALID_ARG;
  if (!hidden || !W || !targets || !logp || !entropy || !lse || !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(workspace, 256) ||
      !aligned(targets, 8) || !aligned(logp, 4) || !aligned(entropy, 4) || !aligned(lse, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (workspace_bytes < L.fwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  float* pm = reinterpret_cast<float*>(ws + L.pm);
  float* ps = reinterpret_cast<float*>(ws + L.ps);
  float* pb = reinterpret_cast<float*>(ws + L.pb);
  float* yt = reinterpret_cast<float*>(ws + L.yt);
  s = enqueue_fwd_partials_short(hidden, W, targets, T, H, V, 0, temperature, pm, ps, pb,
                                 fwd_groups(V), yt, err, st, wait_limit_ns, stall != 0 ? 1 : 0);
  if (s != RLK_OK) return s;
  return enqueue_combine(pm, ps, pb, fwd_groups(V), yt, targets, T, V, logp, entropy, lse, err,
                         st);
}

rlk_status rlk_linear_logp_bwd(const rlk_bf16* hidden, const rlk_bf16* W, const int64_t* targets,
                               int64_t T, int64_t H, int64_t V, float temperature,
                               const float* lse, const float* entropy, const float* dlogp,
                               const float* dentropy, rlk_bf16* dHidden, float* dW,
                               void* workspace, size_t workspace_bytes, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (!dW) return RLK_ERR_INVALID_ARG;
  if (!aligned(dW, 16)) return RLK_ERR_MISALIGNED;
  int sms = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if ((s = check_device(&sms)) != RLK_OK) return s;
    if (cudaMemsetAsync(dW, 0, static_cast<size_t>(V) * H * 4, st) != cudaSuccess)
      return RLK_ERR_CUDA;
    g_calls[1].fetch_add(1);
    return RLK_OK;
  }
  if (!hidden || !W || !targets || !lse || !entropy || !dlogp || !dentropy || !dHidden ||
      !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(dHidden, 16) ||
      !aligned(workspace, 256) || !aligned(targets, 8) || !aligned(lse, 4) ||
      !aligned(entropy, 4) || !aligned(dlogp, 4) || !aligned(dentropy, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (workspace_bytes < L.bwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device(&sms)) != RLK_OK) return s;

  if ((s = enqueue_bwd(hidden, W, targets, T, H, V, 0, V, temperature, lse, entropy, dlogp,
                       dentropy, dHidden, nullptr, 0, 0, dW, static_cast<uint8_t*>(workspace), L,
                       st)) != RLK_OK)
    return s;
  g_calls[1].fetch_add(1);
  return RLK_OK;
}

// Test hook (declared in rlk.h): the backward with a chosen bound on every
// wait and, optionally, one dependency that is never met.
rlk_status rlk_test_linear_logp_bwd_stall(const rlk_bf16* hidden, const rlk_bf16* W,
                                          const int64_t* targets, int64_t T, int64_t H,
                                          int64_t V, float temperature, const float* lse,
                                          const float* entropy, const float* dlogp,
                                          const float* dentropy, rlk_bf16* dHidden, float* dW,
                                          void* workspace, size_t workspace_bytes,
                                          uint64_t wait_limit_ns, int stall,
                                          uint32_t* chunk_done, uint32_t seq, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (T == 0 || wait_limit_ns < 1000000ull || wait_limit_ns > kWaitLimitNs)
    return RLK_ERR_INVALID_ARG;  // 1 ms .. 2 s
  if (chunk_done != nullptr && (seq == 0 || !aligned(chunk_done, 4))) return RLK_ERR_INVALID_ARG;
  if (!hidden || !W || !targets || !lse || !entropy || !dlogp || !dentropy || !dHidden || !dW ||
      !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(dHidden, 16) || !aligned(dW, 16) ||
      !aligned(workspace, 256) || !aligned(targets, 8) || !aligned(lse, 4) ||
      !aligned(entropy, 4) || !aligned(dlogp, 4) || !aligned(dentropy, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (workspace_bytes < L.bwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  return enqueue_bwd(hidden, W, targets, T, H, V, 0, V, temperature, lse, entropy, dlogp,
                     dentropy, dHidden, nullptr, 0, 0, dW, static_cast<uint8_t*>(workspace), L,
                     static_cast<cudaStream_t>(stream), wait_limit_ns, stall != 0 ? 1 : 0,
                     chunk_done, seq);
}

// The backward that publishes each vocab chunk's completion (declared in
// rlk.h with the exchange it serves).
rlk_status rlk_linear_logp_bwd_signal(const rlk_bf16* hidden, const rlk_bf16* W,
                                      const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                      float temperature, const float* lse, const float* entropy,
                                      const float* dlogp, const float* dentropy,
                                      rlk_bf16* dHidden, float* dW, void* workspace,
                                      size_t workspace_bytes, uint32_t* chunk_done, uint32_t seq,
                                      void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (!chunk_done || seq == 0) return RLK_ERR_INVALID_ARG;
  if (!aligned(chunk_done, 4)) return RLK_ERR_MISALIGNED;
  if (T == 0) {
    // nothing to compute: dW is zero and every chunk is complete at once
    if ((s = rlk_linear_logp_bwd(hidden, W, targets, T, H, V, temperature, lse, entropy, dlogp,
                                 dentropy, dHidden, dW, workspace, workspace_bytes, stream)) !=
        RLK_OK)
      return s;
    return write_chunk_words(chunk_done, ceil_div(V, vchunk(V)), seq,
                             static_cast<cudaStream_t>(stream));
  }
  if (!dW || !hidden || !W || !targets || !lse || !entropy || !dlogp || !dentropy || !dHidden ||
      !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(dHidden, 16) || !aligned(dW, 16) ||
      !aligned(workspace, 256) || !aligned(targets, 8) || !aligned(lse, 4) ||
      !aligned(entropy, 4) || !aligned(dlogp, 4) || !aligned(dentropy, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (workspace_bytes < L.bwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  if ((s = enqueue_bwd(hidden, W, targets, T, H, V, 0, V, temperature, lse, entropy, dlogp,
                       dentropy, dHidden, nullptr, 0, 0, dW, static_cast<uint8_t*>(workspace), L,
                       static_cast<cudaStream_t>(stream), kWaitLimitNs, 0, chunk_done, seq)) !=
      RLK_OK)
    return s;
  g_calls[1].fetch_add(1);
  return RLK_OK;
}

rlk_status rlk_stream_wait_chunk(const uint32_t* chunk_word, uint32_t seq, void* stream) {
  if (!chunk_word || seq == 0) return RLK_ERR_INVALID_ARG;
  if (!aligned(chunk_word, 4)) return RLK_ERR_MISALIGNED;
  int sms = 0;
  rlk_status s = check_device(&sms);
  if (s != RLK_OK) return s;
  static const StreamWaitValueFn wait =
      reinterpret_cast<StreamWaitValueFn>(driver_fn("cuStreamWaitValue32"));
  if (!wait) return RLK_ERR_CUDA;
  return wait(static_cast<CUstream>(stream), reinterpret_cast<CUdeviceptr>(chunk_word), seq,
              CU_STREAM_WAIT_VALUE_GEQ) == CUDA_SUCCESS
             ? RLK_OK
             : RLK_ERR_CUDA;
}

size_t rlk_gemm_workspace_bytes(void) { return kHeader; }

rlk_status rlk_gemm_bf16_f32(const rlk_bf16* A, const rlk_bf16* B, int64_t M, int64_t N,
                             int64_t K, int a_mn_major, int b_mn_major, float* C,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return RLK_ERR_INVALID_ARG;
  // 16-byte row pitches for every tensor map and for C's vector stores
  if (K % 8 || N % 8 || (a_mn_major && M % 8) || M >= (int64_t{1} << 31) ||
      N >= (int64_t{1} << 31) || K >= (int64_t{1} << 31))
    return RLK_ERR_UNSUPPORTED_SHAPE;
  if (!A || !B || !C || !workspace) return RLK_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(workspace, 256))
    return RLK_ERR_MISALIGNED;
  if (workspace_bytes < kHeader) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  rlk_status s = check_device(&sms);
  if (s != RLK_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);

  if (!a_mn_major && !b_mn_major && M <= kDecGemmMaxM) {
    // Few rows: the short-batch kernel with the operands swapped (B's rows on
    // the MMA's M side, A's M rows on its N side) and a plain store epilogue.
    // Each C element is the same K-ordered dot product as in the pair tiles,
    // so the results do not depend on which path a row count takes.
    // A narrow C (up to 32 units of 256 columns, at most kDecHalfMaxN rows)
    // takes the half-height form: 64 rows of B per CTA on twice the CTAs
    // (2-5% faster; each CTA's chain of K steps sets the time here).
    const bool half = M <= kDecHalfMaxN && ceil_div(N, 4 * kDecHalfRows) <= 32;
    DecArgs d;
    d.wait_limit_ns = kWaitLimitNs;
    d.stall = 0;
    d.N = half ? static_cast<int>(std::max<int64_t>(16, ceil_div(M, 16) * 16)) : dec_width(M);
    if (!map_kmajor(&d.w_k, B, K, N, K, half ? kDecHalfRows : kBM) ||
        !map_kmajor(&d.hid_k, A, K, M, K, !half && d.N >= kDecPairMinN ? d.N / 2 : d.N))
      return RLK_ERR_CUDA;
    d.ep = EpiFwd::Params{};
    d.ep.part_m = C;
    d.ep.T = static_cast<int>(M);
    d.ep.V = static_cast<int>(N);
    d.ep.ldp = static_cast<int>(N);
    d.err = err;
    d.KB = static_cast<int>(ceil_div(K, kBK));
    d.NG = static_cast<int>(half ? ceil_div(N, 4 * kDecHalfRows) : fwd_groups(N));
    s = launch_short(d, true, st, half);
    if (s == RLK_OK) g_calls[2].fetch_add(1);
    return s;
  }
  GemmArgs a;
  a.a3 = a_mn_major && map_mnmajor3(&a.a, A, M, K, M) ? 1 : 0;
  a.b3 = b_mn_major && map_mnmajor3(&a.b, B, N, K, N) ? 1 : 0;
  a.ak3 = !a_mn_major && map_kmajor3(&a.a, A, K, M, K) ? 1 : 0;
  a.bk3 = !b_mn_major && map_kmajor3(&a.b, B, K, N, K) ? 1 : 0;
  bool ok = a.a3 || a.ak3 ||
            (a_mn_major ? map_mnmajor(&a.a, A, M, K, M) : map_kmajor(&a.a, A, K, M, K, kBM));
  ok = ok && (a.b3 || a.bk3 ||
              (b_mn_major ? map_mnmajor(&a.b, B, N, K, N) : map_kmajor(&a.b, B, K, N, K, kBM)));
  if (!ok) return RLK_ERR_CUDA;
  a.ep.out = C;
  a.ep.rows = static_cast<int>(M);
  a.ep.ncols = static_cast<int>(N);
  a.ep.ld = static_cast<int>(N);
  a.err = err;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.MT = static_cast<int>(ceil_div(M, kPairM));
  a.NT = static_cast<int>(ceil_div(N, kBN));
  a.KB = static_cast<int>(ceil_div(K, kBK));
  a.a_mn = a_mn_major ? 1 : 0;
  a.b_mn = b_mn_major ? 1 : 0;
  a.total = static_cast<long long>(a.MT) * a.NT;
  s = launch_pair<kModeGemm>(a, a.total, false, st);
  if (s == RLK_OK) g_calls[2].fetch_add(1);
  return s;
}

const char* rlk_backend_id(void) { return "rlk.linear_logp.bitwise.sm100a.v1"; }

uint64_t rlk_call_count(int which) {
  if (which < 0 || which > 2) return 0;
  return g_calls[which].load();
}

rlk_status rlk_read_device_error(void* workspace, uint32_t* flags, void* stream) {
  if (!workspace || !flags) return RLK_ERR_INVALID_ARG;
  if (!aligned(workspace, 4)) return RLK_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  *flags = v;
  return RLK_OK;
}

const char* rlk_status_string(rlk_status status) {
  switch (status) {
    case RLK_OK: return "RLK_OK";
    case RLK_ERR_INVALID_ARG: return "RLK_ERR_INVALID_ARG";
    case RLK_ERR_UNSUPPORTED_SHAPE: return "RLK_ERR_UNSUPPORTED_SHAPE";
    case RLK_ERR_MISALIGNED: return "RLK_ERR_MISALIGNED";
    case RLK_ERR_WORKSPACE_TOO_SMALL: return "RLK_ERR_WORKSPACE_TOO_SMALL";
    case RLK_ERR_UNSUPPORTED_DEVICE: return "RLK_ERR_UNSUPPORTED_DEVICE";
    case RLK_ERR_CUDA: return "RLK_ERR_CUDA";
  }
  return "RLK_ERR_UNKNOWN";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Vocab-parallel (tensor-parallel) forward: shards of W whose first rows are
// aligned to the 512-column splits produce exactly the single-GPU split
// triples, and the combine merges them in global split order.
// ---------------------------------------------------------------------------
extern "C" int64_t rlk_fwd_split_width(void) { return static_cast<int64_t>(kBN) * kFwdGroup; }

extern "C" rlk_status rlk_linear_logp_fwd_shard(const rlk_bf16* hidden, const rlk_bf16* W_shard,
                                                const int64_t* targets, int64_t T, int64_t H,
                                                int64_t V, int64_t v0, int64_t V_shard,
                                                float temperature, float* part_m, float* part_s,
                                                float* part_b, int64_t Gs, float* ytgt,
                                                void* workspace, size_t workspace_bytes,
                                                void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (v0 < 0 || V_shard < 1 || v0 + V_shard > V) return RLK_ERR_INVALID_ARG;
  if (Gs < fwd_groups(V_shard) || Gs > fwd_groups(V)) return RLK_ERR_INVALID_ARG;
  // splits must not straddle shards: every shard but the last is whole splits
  if (v0 % rlk_fwd_split_width() != 0 || (v0 + V_shard != V && V_shard % rlk_fwd_split_width()))
    return RLK_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return RLK_OK;
  if (!hidden || !W_shard || !targets || !part_m || !part_s || !part_b || !ytgt || !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W_shard, 16) || !aligned(workspace, 256) ||
      !aligned(targets, 8) || !aligned(part_m, 4) || !aligned(part_s, 4) || !aligned(part_b, 4) ||
      !aligned(ytgt, 4))
    return RLK_ERR_MISALIGNED;
  if (workspace_bytes < kHeader) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  return enqueue_fwd_partials(hidden, W_shard, targets, T, H, V_shard, v0, temperature, part_m,
                              part_s, part_b, Gs, ytgt, static_cast<uint32_t*>(workspace),
                              static_cast<cudaStream_t>(stream));
}

extern "C" rlk_status rlk_linear_logp_combine(const float* part_m, const float* part_s,
                                              const float* part_b, int64_t nshards, int64_t Gs,
                                              const float* ytgt, const int64_t* targets,
                                              int64_t T, int64_t V, float* logp, float* entropy,
                                              float* lse, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  rlk_status s = check_sizes(T, 64, V, 1.0f);
  if (s != RLK_OK) return s;
  const int64_t G = fwd_groups(V);
  if (nshards < 1 || Gs < 1 || (nshards - 1) * Gs >= G || nshards * Gs < G)
    return RLK_ERR_INVALID_ARG;
  if (T == 0) return RLK_OK;
  if (!part_m || !part_s || !part_b || !ytgt || !targets || !logp || !entropy || !lse ||
      !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(targets, 8) || !aligned(part_m, 4) ||
      !aligned(part_s, 4) || !aligned(part_b, 4) || !aligned(ytgt, 4) || !aligned(logp, 4) ||
      !aligned(entropy, 4) || !aligned(lse, 4))
    return RLK_ERR_MISALIGNED;
  if (workspace_bytes < kHeader) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  return enqueue_combine(part_m, part_s, part_b, Gs, ytgt, targets, T, V, logp, entropy, lse,
                         static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream));
}

// Vocab-parallel backward.  A shard's chunks are the full head's chunks
// (boundaries at multiples of rlk_bwd_chunk_width(V)), so its recompute,
// dlogits, per-chunk dHidden products and dW rows are bit for bit those of the
// single-GPU backward; rlk_dhidden_combine then adds the chunks' products in
// global chunk order with the same fp32 additions and bf16 rounding.
extern "C" int64_t rlk_bwd_chunk_width(int64_t V) {
  if (V <= 0 || V >= (int64_t{1} << 31)) return 0;
  return vchunk(V);
}

extern "C" rlk_status rlk_linear_logp_bwd_shard(
    const rlk_bf16* hidden, const rlk_bf16* W_shard, const int64_t* targets, int64_t T, int64_t H,
    int64_t V, int64_t v0, int64_t V_shard, float temperature, const float* lse,
    const float* entropy, const float* dlogp, const float* dentropy, float* dh_parts,
    int64_t part_rows, int64_t part_chunks, float* dW_shard, void* workspace,
    size_t workspace_bytes, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (v0 < 0 || V_shard < 1 || v0 + V_shard > V) return RLK_ERR_INVALID_ARG;
  const int64_t vc = vchunk(V);
  if (v0 % vc != 0 || (v0 + V_shard != V && V_shard % vc != 0)) return RLK_ERR_UNSUPPORTED_SHAPE;
  if (part_rows < 1 || part_rows >= (int64_t{1} << 31) || part_chunks < ceil_div(V_shard, vc) ||
      part_chunks > ceil_div(V, vc))
    return RLK_ERR_INVALID_ARG;
  if (!dW_shard) return RLK_ERR_INVALID_ARG;
  if (!aligned(dW_shard, 16)) return RLK_ERR_MISALIGNED;
  int sms = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if ((s = check_device(&sms)) != RLK_OK) return s;
    return cudaMemsetAsync(dW_shard, 0, static_cast<size_t>(V_shard) * H * 4, st) == cudaSuccess
               ? RLK_OK
               : RLK_ERR_CUDA;
  }
  if (!hidden || !W_shard || !targets || !lse || !entropy || !dlogp || !dentropy || !dh_parts ||
      !workspace)
    return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W_shard, 16) || !aligned(dh_parts, 16) ||
      !aligned(workspace, 256) || !aligned(targets, 8) || !aligned(lse, 4) ||
      !aligned(entropy, 4) || !aligned(dlogp, 4) || !aligned(dentropy, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);  // sized for the full head: covers any shard
  if (workspace_bytes < L.bwd_end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  return enqueue_bwd(hidden, W_shard, targets, T, H, V_shard, v0, V, temperature, lse, entropy,
                     dlogp, dentropy, nullptr, dh_parts, part_rows, part_chunks, dW_shard,
                     static_cast<uint8_t*>(workspace), L, st);
}

namespace rlk {
namespace {

// out[i] = bf16(((p_0[i] + p_1[i]) + p_2[i]) + ...), the same fp32 additions
// (old + new) and rounding as the dHidden epilogue's chunk chain.
__global__ void __launch_bounds__(256) dhidden_combine_kernel(const float* __restrict__ parts,
                                                              int nparts, int64_t count,
                                                              __nv_bfloat16* __restrict__ out) {
  const int64_t n4 = count / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += stride) {
    float4 a = reinterpret_cast<const float4*>(parts)[i];
    for (int k = 1; k < nparts; ++k) {
      const float4 v = reinterpret_cast<const float4*>(parts + k * count)[i];
      a.x = a.x + v.x;
      a.y = a.y + v.y;
      a.z = a.z + v.z;
      a.w = a.w + v.w;
    }
    uint2 w;
    w.x = pack_bf16x2(a.x, a.y);
    w.y = pack_bf16x2(a.z, a.w);
    reinterpret_cast<uint2*>(out)[i] = w;
  }
}

}  // namespace
}  // namespace rlk

extern "C" rlk_status rlk_dhidden_combine(const float* dh_parts, int64_t nparts, int64_t count,
                                          rlk_bf16* out, void* stream) {
  if (nparts < 1 || nparts > (int64_t{1} << 20) || count < 0) return RLK_ERR_INVALID_ARG;
  if (count % 4) return RLK_ERR_UNSUPPORTED_SHAPE;
  if (count == 0) return RLK_OK;
  if (!dh_parts || !out) return RLK_ERR_INVALID_ARG;
  if (!aligned(dh_parts, 16) || !aligned(out, 8)) return RLK_ERR_MISALIGNED;
  int sms = 0;
  rlk_status s = check_device(&sms);
  if (s != RLK_OK) return s;
  const int64_t blocks = std::min<int64_t>(ceil_div(count / 4, 256), static_cast<int64_t>(sms) * 8);
  dhidden_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      dh_parts, static_cast<int>(nparts), count, reinterpret_cast<__nv_bfloat16*>(out));
  return cudaGetLastError() == cudaSuccess ? RLK_OK : RLK_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Fixed-order sum of equally shaped fp32 buffers (the data-parallel exchange
// of dW: every rank's partial slice arrives at the slice's owner, which adds
// them in rank order, so the sum never depends on arrival order).
// ---------------------------------------------------------------------------
namespace rlk {
namespace {

constexpr int kMaxSumParts = 64;

struct SumParts {
  const float* p[kMaxSumParts];
};

__global__ void __launch_bounds__(256) sum_ordered_vec4_kernel(const __grid_constant__ SumParts P,
                                                               int n, float4* out,
                                                               int64_t count4) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(P.p[0])[i];
    for (int k = 1; k < n; ++k) {
      const float4 v = reinterpret_cast<const float4*>(P.p[k])[i];
      acc.x = acc.x + v.x;
      acc.y = acc.y + v.y;
      acc.z = acc.z + v.z;
      acc.w = acc.w + v.w;
    }
    out[i] = acc;
  }
}

__global__ void __launch_bounds__(256) sum_ordered_kernel(const __grid_constant__ SumParts P, int n,
                                                          float* out, int64_t count) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float acc = P.p[0][i];
    for (int k = 1; k < n; ++k) acc = acc + P.p[k][i];
    out[i] = acc;
  }
}

}  // namespace
}  // namespace rlk

extern "C" rlk_status rlk_sum_ordered(const float* const* parts, int nparts, float* out,
                                      int64_t count, void* stream) {
  if (!parts || !out || nparts < 1 || nparts > kMaxSumParts || count < 0)
    return RLK_ERR_INVALID_ARG;
  if (count == 0) return RLK_OK;
  SumParts P;
  bool vec = aligned(out, 16) && count % 4 == 0;
  for (int k = 0; k < nparts; ++k) {
    if (!parts[k]) return RLK_ERR_INVALID_ARG;
    if (!aligned(parts[k], 4)) return RLK_ERR_MISALIGNED;
    vec = vec && aligned(parts[k], 16);
    P.p[k] = parts[k];
  }
  if (!aligned(out, 4)) return RLK_ERR_MISALIGNED;
  int sms = 0;
  rlk_status s = check_device(&sms);
  if (s != RLK_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t items = vec ? count / 4 : count;
  const unsigned blocks =
      static_cast<unsigned>(std::min<int64_t>(ceil_div(items, 256), static_cast<int64_t>(sms) * 8));
  if (vec)
    sum_ordered_vec4_kernel<<<blocks, 256, 0, st>>>(P, nparts, reinterpret_cast<float4*>(out), items);
  else
    sum_ordered_kernel<<<blocks, 256, 0, st>>>(P, nparts, out, items);
  return cudaGetLastError() == cudaSuccess ? RLK_OK : RLK_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Forward without a caller-provided workspace.
//
// For callers that cannot allocate device memory at all: code that runs
// inside a host framework that owns every device byte (a serving engine with
// a pre-reserved pool, a plugin host that forbids allocation calls), or that
// cannot size a workspace ahead of time.  Their per-call scratch (the error
// word and the forward's per-split partials) lives in one file-scope device
// array that every GPU loading this library holds until the process exits.
// ---------------------------------------------------------------------------
namespace rlk {
namespace {

constexpr size_t kStaticScratchBytes = size_t{32} << 20;  // 32 MiB per device

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch per device, together with the id of the
// context it was looked up in.  In host code the array's name is only a
// host-side stand-in.  A context that is destroyed and created again (a
// device reset) reloads this library's module, so the array may move: the
// address is looked up again whenever the current context's id differs from
// the one stored.  Guarded by a mutex; host threads may call concurrently.
struct ScratchSlot {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch_slot[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the context current on this thread; false if there is none (the
// runtime has not bound one to this thread yet) or the driver cannot say.
bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_cur =
      reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
  static const CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

rlk_status static_scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return RLK_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch_slot[dev];
  unsigned long long id = 0;
  if (slot.addr && current_context_id(&id) && id == slot.ctx_id) {
    *out = slot.addr;
    return RLK_OK;
  }
  // First use on this device, a new context, or no context bound to this
  // thread yet: the lookup binds the device's primary context and returns
  // the array's address in it.
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return RLK_ERR_CUDA;
  }
  slot.addr = p;
  slot.ctx_id = current_context_id(&id) ? id : 0;
  *out = p;
  return RLK_OK;
}

// After a timed-out pipeline wait the outputs are not trustworthy; without a
// caller-visible error word they are overwritten with NaN instead.
__global__ void poison_on_timeout_kernel(const uint32_t* err, float* logp, float* entropy,
                                         float* lse, int T) {
  if ((*err & kDevErrTimeout) == 0) return;
  const float nan = __int_as_float(0x7fc00000);
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    logp[t] = nan;
    entropy[t] = nan;
    lse[t] = nan;
  }
}

}  // namespace
}  // namespace rlk

extern "C" {


rlk_status rlk_linear_logp_fwd_noalloc(const rlk_bf16* hidden, const rlk_bf16* W,
                                       const int64_t* targets, int64_t T, int64_t H, int64_t V,
                                       float temperature, float* logp, float* entropy,
                                       float* lse, void* stream) {
  rlk_status s = check_sizes(T, H, V, temperature);
  if (s != RLK_OK) return s;
  if (T == 0) return RLK_OK;
  if (!hidden || !W || !targets || !logp || !entropy || !lse) return RLK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(W, 16) || !aligned(targets, 8) || !aligned(logp, 4) ||
      !aligned(entropy, 4) || !aligned(lse, 4))
    return RLK_ERR_MISALIGNED;
  const Layout L = layout(T, H, V);
  if (L.fwd_end > kStaticScratchBytes) return RLK_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  if ((s = check_device(&sms)) != RLK_OK) return s;
  void* scratch = nullptr;
  if ((s = static_scratch_for_current_device(&scratch)) != RLK_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  uint8_t* ws = static_cast<uint8_t*>(scratch);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  // The array keeps the previous call's contents: only the error word must
  // start at zero (every partial this call reads, it writes first).
  if (cudaMemsetAsync(err, 0, kHeader, st) != cudaSuccess) return RLK_ERR_CUDA;
  if ((s = enqueue_fwd(hidden, W, targets, T, H, V, temperature, logp, entropy, lse, ws, L, st)) !=
      RLK_OK)
    return s;
  poison_on_timeout_kernel<<<std::min<int64_t>(ceil_div(T, 256), 1024), 256, 0, st>>>(
      err, logp, entropy, lse, static_cast<int>(T));
  if (cudaGetLastError() != cudaSuccess) return RLK_ERR_CUDA;
  g_calls[0].fetch_add(1);
  return RLK_OK;
}

}  // extern "C"
