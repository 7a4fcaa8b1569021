// rlk_transition.cu -- one step of a diffusion sampler's Gaussian transition
// and its log-probability, per sample, bitwise batch invariant (the RL-Kernel
// B200 report's transition gate, h3-runtime-integration-b200 report.json,
// transition[]: prev_sample and mean bitwise, logp batch invariant, scoring
// reproduces the sampling logprob).
//
//   mean[b, i] = a_b x[b, i] + c_b v[b, i]
//   prev[b, i] = mean[b, i] + s_b eps[b, i]                  (sampling only)
//   logp[b]    = -(sum_i (prev - mean)^2) / (2 s_b^2 n) - ln s_b - ln(2 pi) / 2
//
// One launch per call (no memset: the counters reset themselves).
// Elementwise arithmetic is one fp32 operation at a time, rounded to nearest
// (a x and c v, then their sum; s eps, then mean + that): what plain fp32
// tensor arithmetic gives, so the mean and prev_sample equal it bit for bit.
// The sum of squared residuals of a sample runs over fixed 4096-element
// chunks (one CTA each) in a fixed order inside the chunk, then over the
// chunks in index order; nothing depends on B, on the other samples or on
// which CTA finishes last.  Scoring a recorded prev_sample runs the same code
// on the same values as sampling, so its logp is the sampling logp.
//
// HBM-bound: sampling reads x, v, eps and writes mean, prev (20 bytes per
// element); scoring reads x, v, prev (12 bytes, +4 with the mean written).
#include <cmath>
#include <cstdint>

#include <cuda_runtime.h>

#include "rlk.h"
#include "rlk_device.h"

namespace rlk {
namespace {

constexpr int kTrThreads = 256;
constexpr int kTrVecs = 4;                                // float4 per thread
constexpr int64_t kTrChunk = kTrThreads * kTrVecs * 4;   // 4096 elements per CTA
constexpr size_t kTrHeader = 256;  // word 0: error word; word 1: samples finished
constexpr float kHalfLog2Pi = 0.918938533204672742f;      // ln(2 pi) / 2

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
int64_t tr_chunks(int64_t n) { return (n + kTrChunk - 1) / kTrChunk; }

// Counters are zero between calls: each call's last CTA of a sample resets
// that sample's counter and the last sample resets the finished count, so the
// workspace needs zero-filling once, before its first use, and no memset per
// call.
struct TrLayout {
  size_t done, flag, part, end;
};

TrLayout tr_layout(int64_t B, int64_t n) {
  TrLayout L;
  L.done = kTrHeader;
  L.flag = L.done + align256(static_cast<size_t>(B) * 4);
  L.part = L.flag + align256(static_cast<size_t>(B) * 4);
  L.end = L.part + align256(static_cast<size_t>(B) * tr_chunks(n) * 4);
  return L;
}

__device__ __forceinline__ float4 mean4(float a, float4 x, float c, float4 v) {
  return make_float4(__fadd_rn(__fmul_rn(a, x.x), __fmul_rn(c, v.x)),
                     __fadd_rn(__fmul_rn(a, x.y), __fmul_rn(c, v.y)),
                     __fadd_rn(__fmul_rn(a, x.z), __fmul_rn(c, v.z)),
                     __fadd_rn(__fmul_rn(a, x.w), __fmul_rn(c, v.w)));
}

// grid (chunks, B): CTA (k, b) covers elements [k * 4096, (k + 1) * 4096) of
// sample b.  kSample: third operand is eps and prev is written; otherwise it
// is the recorded prev.
template <bool kSample>
__global__ void __launch_bounds__(kTrThreads) transition_kernel(
    const float* __restrict__ x, const float* __restrict__ v, const float* __restrict__ third,
    const float* __restrict__ a, const float* __restrict__ c, const float* __restrict__ s,
    int64_t n, int nchunks, float* __restrict__ mean_out, float* __restrict__ prev_out,
    float* part, unsigned* done, unsigned* flag, float* __restrict__ logp, unsigned* err) {
  const int b = blockIdx.y;
  const int chunk = blockIdx.x;
  const float ab = a[b], cb = c[b], sb = s[b];
  const size_t base = static_cast<size_t>(b) * static_cast<size_t>(n);
  const int64_t c0 = static_cast<int64_t>(chunk) * kTrChunk;

  // squared residuals: per thread over its float4s in order, x+y and z+w
  // first; then a warp butterfly (every lane ends with the same sum); then
  // the warps in order
  // every load of the thread is issued before any arithmetic: the kernel is
  // one DRAM round trip deep
  float4 xs[kTrVecs], vs[kTrVecs], ts[kTrVecs];
#pragma unroll
  for (int k = 0; k < kTrVecs; ++k) {
    const int64_t i = c0 + (static_cast<int64_t>(k) * kTrThreads + threadIdx.x) * 4;
    if (i < n) {  // n % 4 == 0: the whole float4 is inside the sample
      xs[k] = __ldcs(reinterpret_cast<const float4*>(x + base + i));
      vs[k] = __ldcs(reinterpret_cast<const float4*>(v + base + i));
      ts[k] = __ldcs(reinterpret_cast<const float4*>(third + base + i));
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < kTrVecs; ++k) {
    const int64_t i = c0 + (static_cast<int64_t>(k) * kTrThreads + threadIdx.x) * 4;
    if (i < n) {
      const float4 xv = xs[k], vv = vs[k], tv = ts[k];
      const float4 mu = mean4(ab, xv, cb, vv);
      float4 pr = tv;
      if constexpr (kSample) {
        pr = make_float4(__fadd_rn(mu.x, __fmul_rn(sb, tv.x)), __fadd_rn(mu.y, __fmul_rn(sb, tv.y)),
                         __fadd_rn(mu.z, __fmul_rn(sb, tv.z)), __fadd_rn(mu.w, __fmul_rn(sb, tv.w)));
        *reinterpret_cast<float4*>(prev_out + base + i) = pr;
      }
      if (mean_out) *reinterpret_cast<float4*>(mean_out + base + i) = mu;
      const float dx = __fsub_rn(pr.x, mu.x), dy = __fsub_rn(pr.y, mu.y);
      const float dz = __fsub_rn(pr.z, mu.z), dw = __fsub_rn(pr.w, mu.w);
      const float q = __fadd_rn(__fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy)),
                                __fadd_rn(__fmul_rn(dz, dz), __fmul_rn(dw, dw)));
      acc = __fadd_rn(acc, q);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
  __shared__ float warp_sum[kTrThreads / 32];
  __shared__ int is_last;
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = warp_sum[0];
#pragma unroll
    for (int w = 1; w < kTrThreads / 32; ++w) t = __fadd_rn(t, warp_sum[w]);
    part[static_cast<size_t>(b) * nchunks + chunk] = t;
    __threadfence();
    is_last = atomicAdd(done + b, 1u) == static_cast<unsigned>(nchunks - 1);
  }
  __syncthreads();
  if (!is_last || threadIdx.x != 0) return;
  // the sample's last CTA: chunks in index order
  __threadfence();
  const volatile float* pp = part + static_cast<size_t>(b) * nchunks;
  float S = 0.f;
  for (int k = 0; k < nchunks; ++k) S = __fadd_rn(S, pp[k]);
  const bool bad = !(sb > 0.f) || !isfinite(sb);
  if (bad) {
    logp[b] = __int_as_float(0x7fc00000);
  } else {
    const float denom = __fmul_rn(__fmul_rn(2.f, __fmul_rn(sb, sb)), static_cast<float>(n));
    logp[b] = __fsub_rn(-__fdiv_rn(S, denom), __fadd_rn(logf(sb), kHalfLog2Pi));
  }
  flag[b] = bad ? RLK_DEVERR_SCALE : 0u;
  done[b] = 0u;  // every chunk of b has arrived: ready for the next call
  __threadfence();
  unsigned* finished = err + 1;
  if (atomicAdd(finished, 1u) == gridDim.y - 1) {
    // the call's last sample: this call's error word, then reset the count
    __threadfence();
    const volatile unsigned* fl = flag;
    unsigned e = 0u;
    for (unsigned k = 0; k < gridDim.y; ++k) e |= fl[k];
    *err = e;
    *finished = 0u;
  }
}

rlk_status tr_check(const float* x, const float* v, const float* third, const float* a,
                    const float* c, const float* s, int64_t B, int64_t n, const float* mean_out,
                    const float* prev_out, bool sample, const float* logp, const void* ws,
                    size_t ws_bytes) {
  if (B < 0 || n < 0) return RLK_ERR_INVALID_ARG;
  if (n % 4 != 0 || B > 65535 || tr_chunks(n) > (int64_t{1} << 31) - 1 ||
      static_cast<double>(n) > 16777216.0)   // n exact in fp32 for the 1/n of the mean
    return RLK_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || n == 0) return RLK_OK;
  if (!x || !v || !third || !a || !c || !s || !logp || !ws || (sample && !prev_out))
    return RLK_ERR_INVALID_ARG;
  auto al = [](const void* p, uintptr_t m) { return reinterpret_cast<uintptr_t>(p) % m == 0; };
  if (!al(x, 16) || !al(v, 16) || !al(third, 16) || !al(mean_out, 16) || !al(prev_out, 16) ||
      !al(a, 4) || !al(c, 4) || !al(s, 4) || !al(logp, 4) || !al(ws, 256))
    return RLK_ERR_MISALIGNED;
  if (ws_bytes < tr_layout(B, n).end) return RLK_ERR_WORKSPACE_TOO_SMALL;
  return RLK_OK;
}

template <bool kSample>
rlk_status tr_launch(const float* x, const float* v, const float* third, const float* a,
                     const float* c, const float* s, int64_t B, int64_t n, float* mean_out,
                     float* prev_out, float* logp, void* ws, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  const TrLayout L = tr_layout(B, n);
  const int nchunks = static_cast<int>(tr_chunks(n));
  transition_kernel<kSample><<<dim3(nchunks, static_cast<unsigned>(B)), kTrThreads, 0, st>>>(
      x, v, third, a, c, s, n, nchunks, mean_out, prev_out, reinterpret_cast<float*>(w + L.part),
      reinterpret_cast<unsigned*>(w + L.done), reinterpret_cast<unsigned*>(w + L.flag), logp,
      reinterpret_cast<unsigned*>(w));
  return cudaGetLastError() == cudaSuccess ? RLK_OK : RLK_ERR_CUDA;
}

}  // namespace
}  // namespace rlk

using namespace rlk;

extern "C" size_t rlk_transition_workspace_bytes(int64_t B, int64_t n) {
  if (B < 0 || n < 0 || B > 65535) return 0;
  return tr_layout(B, n).end;
}

extern "C" rlk_status rlk_transition_sample(const float* x, const float* v, const float* eps,
                                            const float* a, const float* c, const float* s,
                                            int64_t B, int64_t n, float* mean_out,
                                            float* prev_out, float* logp, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  rlk_status st = tr_check(x, v, eps, a, c, s, B, n, mean_out, prev_out, true, logp, workspace,
                           workspace_bytes);
  if (st != RLK_OK || B == 0 || n == 0) return st;
  int sms = 0;
  if ((st = current_device_supported(&sms)) != RLK_OK) return st;
  return tr_launch<true>(x, v, eps, a, c, s, B, n, mean_out, prev_out, logp, workspace,
                         static_cast<cudaStream_t>(stream));
}

extern "C" rlk_status rlk_transition_logp(const float* x, const float* v, const float* prev,
                                          const float* a, const float* c, const float* s,
                                          int64_t B, int64_t n, float* mean_out, float* logp,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  rlk_status st = tr_check(x, v, prev, a, c, s, B, n, mean_out, nullptr, false, logp, workspace,
                           workspace_bytes);
  if (st != RLK_OK || B == 0 || n == 0) return st;
  int sms = 0;
  if ((st = current_device_supported(&sms)) != RLK_OK) return st;
  return tr_launch<false>(x, v, prev, a, c, s, B, n, mean_out, nullptr, logp, workspace,
                          static_cast<cudaStream_t>(stream));
}
