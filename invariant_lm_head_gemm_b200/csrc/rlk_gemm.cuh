// rlk_gemm.cuh -- tile constants, the epilogues that turn 128 x 256 fp32
// accumulator tiles (one CTA's half of a pair tile, read from TMEM 32 columns
// at a time) into the operator's results, and the forward's fixed-order
// combine.  The mainloop that feeds them is pair_kernel (rlk_kernel.cuh).
//
// Batch invariance.  Every epilogue works row by row in a fixed column order,
// and each accumulator element comes from one fixed K loop; nothing depends on
// how many rows the problem has or on which CTA pair runs a tile.
#pragma once

#include <cuda_bf16.h>

#include "rlk_ptx.cuh"

namespace rlk {

constexpr int kBM = 128;     // accumulator rows per CTA
constexpr int kPairM = 256;  // accumulator rows per CTA pair
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kBox = 64 * 64 * 2;       // one MN-major 64x64 box, 8 KB

constexpr float kLog2e = 1.4426950408889634f;  // log2(e)
constexpr float kLn2 = 0.6931471805599453f;    // ln(2)
constexpr float kMaskLogit = -1.0e30f;         // stands for -inf without producing NaN

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// =====================================================================
// Epilogue policies.  Each provides Params, State and
//   begin_unit(p, st, row, mt, g)   once per unit, row = global M index
//   tile(p, st, taddr, nt, ...)     once per 128x256 accumulator tile
//   end_unit(p, st, g)              once per unit
// =====================================================================

// One 32-column chunk of the forward's online update for one row: columns
// col0 .. col0+31 of this W, y = x * log2(e) / tau already formed with
// fwd_scale.  Masks columns >= V, records y at the target's local column, then
// moves m to the chunk's max, rescales s and b, and adds the chunk's terms in
// column order.  Both forward kernels run exactly this code; the _rn
// intrinsics keep the compiler from fusing a product into a later add
// differently in the two.
__device__ __forceinline__ float fwd_scale(float x, float scale_log2) {
  return __fmul_rn(x, scale_log2);
}

__device__ __forceinline__ void fwd_chunk_update(float (&y)[32], int col0, int V, int64_t tgt,
                                                 float* ytgt_row, float& m, float& s,
                                                 float& b) {
  if (col0 + 32 > V) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j >= V) y[j] = kMaskLogit;
  }
  const int64_t d = tgt - col0;
  if (d >= 0 && d < 32) {
    float yt = y[0];
#pragma unroll
    for (int j = 1; j < 32; ++j) yt = (j == d) ? y[j] : yt;
    *ytgt_row = yt;
  }
  float cm = y[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) cm = fmaxf(cm, y[j]);
  const float mn = fmaxf(m, cm);
  const float dm = __fsub_rn(m, mn);
  const float a = ex2_approx(dm);
  b = __fmul_rn(a, fmaf(dm, s, b));
  s = __fmul_rn(s, a);
  m = mn;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float dd = __fsub_rn(y[j], mn);
    const float e = ex2_approx(dd);
    s = __fadd_rn(s, e);
    b = fmaf(e, dd, b);
  }
}

// Forward: per row, over the unit's vocab tiles in ascending order, keep the
// online triple in base-2 units of y = x * log2(e) / tau:
//   m = max y,  s = sum 2^(y - m),  b = sum 2^(y - m) (y - m)
// and pick up y at the row's target column.  The triple of each (row,
// vocab split) goes to the workspace for the fixed-order combine.
struct EpiFwd {
  struct Params {
    const int64_t* targets;
    float* part_m;  // [T][ldp] (row-major: a row's splits are contiguous)
    float* part_s;
    float* part_b;
    float* ytgt;
    int T;
    int V;             // vocab columns of this W (a shard's own count for a shard)
    int ldp;           // row stride of part_*: at least this W's vocab splits
    int64_t v0;        // global vocab index of this W's first row (0 unless a shard)
    float scale_log2;  // log2(e) / tau
  };
  struct State {
    float m, s, b;
    int64_t tgt;
    int row;
    bool valid;
  };

  __device__ static void begin_unit(const Params& p, State& st, int row, int, int) {
    st.row = row;
    st.valid = row < p.T;
    st.tgt = st.valid ? p.targets[row] - p.v0 : -1;  // local column of the target
    st.m = kMaskLogit;
    st.s = 0.f;
    st.b = 0.f;
  }

  __device__ static void tile(const Params& p, State& st, uint32_t taddr, int nt) {
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      float y[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) y[j] = fwd_scale(__uint_as_float(r[j]), p.scale_log2);
      fwd_chunk_update(y, nt * kBN + c * 32, p.V, st.tgt, p.ytgt + st.row, st.m, st.s, st.b);
    }
  }

  __device__ static void end_unit(const Params& p, State& st, int g) {
    if (st.valid) {
      const size_t i = static_cast<size_t>(st.row) * p.ldp + g;
      p.part_m[i] = st.m;
      p.part_s[i] = st.s;
      p.part_b[i] = st.b;
    }
  }
};

// Backward recompute: the same logits tile, turned into bf16 dlogits
//   dx = (dlogp (1[v = target] - p) - dentropy p (z - E_p z)) / tau
// with p = 2^(y - lse log2 e), written (through the store tensor map) to
// the chunk buffer dX[T, chunk width], columns local to the chunk at c0.
struct EpiDlogits {
  struct Params {
    const int64_t* targets;
    const float* lse;
    const float* entropy;
    const float* dlogp;
    const float* dentropy;
    uint32_t* err;
    int T;
    int V;             // vocab rows of this W (a shard's own count for a shard)
    int c0;            // first W row of the chunk
    int64_t v0;        // global vocab index of this W's first row (0 unless a shard)
    int64_t Vfull;     // full vocabulary (targets are global indices)
    float scale_log2;  // log2(e) / tau
    float inv_tau;
  };
  struct State {
    float A, k1, k2, hot;
    int64_t tloc;
    int row;
    bool valid;
  };

  __device__ static void begin_unit(const Params& p, State& st, int row, int, int) {
    st.row = row;
    st.valid = row < p.T;
    st.A = 0.f;
    st.k1 = st.k2 = st.hot = 0.f;
    st.tloc = -1;
    if (st.valid) {
      const float lse = p.lse[row], ent = p.entropy[row];
      const float dl = p.dlogp[row], de = p.dentropy[row];
      const int64_t tg = p.targets[row];
      const float ez = lse - ent;  // E_p z
      st.A = lse * kLog2e;
      // dx = hot*1[v=target] - p*(k1 + k2*y)
      st.k1 = p.inv_tau * (dl - de * ez);
      st.k2 = p.inv_tau * de * kLn2;
      st.hot = p.inv_tau * dl;
      if (tg >= 0 && tg < p.Vfull) {
        const int64_t t = tg - p.v0;  // shard-local; the target is elsewhere if out of [0, V)
        if (t >= 0 && t < p.V) st.tloc = t - p.c0;
      } else if (p.c0 == 0) {
        atomicOr(p.err, kDevErrTarget);
      }
    }
  }

  // One 128 x 256 tile, 32 columns at a time.  Each warp stages its 32 x 32
  // bf16 block in shared memory (two 2 KB buffers, `stage`, 1024-byte
  // aligned) and one lane writes it to dX[warp_row0 .. +32, col .. +32] with a
  // TMA store (rows past T are not written).  The staging layout is the
  // store map's 64-byte swizzle: the 16-byte piece q of row r sits at piece
  // q ^ ((r >> 1) & 3) of the row, so the warp's 16-byte stores spread over
  // all 32 banks (a plain 64-byte row pitch puts every even lane on the same
  // four banks).  The caller waits for the stores (bulk_wait_all) before
  // publishing the tile.
  __device__ static void tile(const Params& p, State& st, uint32_t taddr, int nt,
                              const CUtensorMap* store_map, uint32_t stage, int lane,
                              int warp_row0) {
    const bool any_row = warp_row0 < p.T;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      const int loc0 = nt * kBN + c * 32;
      const int col0 = p.c0 + loc0;
      float dx[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float y = __uint_as_float(r[j]) * p.scale_log2;
        const float pr = ex2_approx(y - st.A);
        dx[j] = -pr * fmaf(st.k2, y, st.k1);
      }
      if (col0 + 32 > p.V) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j >= p.V) dx[j] = 0.f;
      }
      const int64_t d = st.tloc - loc0;
      if (d >= 0 && d < 32) {
#pragma unroll
        for (int j = 0; j < 32; ++j) dx[j] = (j == d) ? dx[j] + st.hot : dx[j];
      }
      if (any_row) {
        const uint32_t buf = stage + (c & 1) * 2048u;
        if (lane == 0) bulk_wait_read_le1();  // the store two chunks back has read `buf`
        __syncwarp();
        const uint32_t row_addr = buf + lane * 64u;
        const uint32_t sw = static_cast<uint32_t>(lane >> 1) & 3u;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(row_addr + ((static_cast<uint32_t>(q) ^ sw) << 4), pack_bf16x2(dx[8 * q + 0], dx[8 * q + 1]),
                       pack_bf16x2(dx[8 * q + 2], dx[8 * q + 3]),
                       pack_bf16x2(dx[8 * q + 4], dx[8 * q + 5]),
                       pack_bf16x2(dx[8 * q + 6], dx[8 * q + 7]));
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(store_map, buf, loc0, warp_row0);
          bulk_commit_group();
        }
      }
    }
  }

  __device__ static void end_unit(const Params&, State&, int) {}
};

// dHidden: acc[T,H] (fp32 workspace) collects the vocab chunks in ascending
// order: chunk 0 stores, later chunks add (old + new), the last chunk writes
// the bf16 result.  kPart instead stores chunk c's own fp32 product into a
// parts buffer laid out [row slice s][chunk c][row r][H] (row = s * part_rows
// + r), for a sum in global chunk order elsewhere.
struct EpiDh {
  enum Mode { kFirst = 0, kMiddle = 1, kLast = 2, kOnly = 3, kPart = 4 };
  struct Params {
    float* acc;  // [T][H], or the parts buffer for kPart
    __nv_bfloat16* out;
    int T;
    int H;
    int mode;
    int c;            // kPart: the chunk
    int part_rows;    // kPart: rows per slice
    int part_chunks;  // kPart: chunk slots per slice
  };
  struct State {
    float* arow;
    __nv_bfloat16* orow;
    bool valid;
  };

  __device__ static void begin_unit(const Params& p, State& st, int row, int, int) {
    st.valid = row < p.T;
    size_t a = static_cast<size_t>(row) * p.H;
    if (p.mode == kPart) {
      const int s = row / p.part_rows, r = row - s * p.part_rows;
      a = ((static_cast<size_t>(s) * p.part_chunks + p.c) * p.part_rows + r) * p.H;
    }
    st.arow = p.acc + a;
    st.orow = p.out + static_cast<size_t>(row) * p.H;
  }

  __device__ static void tile(const Params& p, State& st, uint32_t taddr, int nt) {
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      const int col0 = nt * kBN + c * 32;
      if (col0 >= p.H) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      if (!st.valid) continue;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
      float4* pa = reinterpret_cast<float4*>(st.arow + col0);
      if (p.mode == kMiddle || p.mode == kLast) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 o = pa[q];
          v[4 * q + 0] = o.x + v[4 * q + 0];
          v[4 * q + 1] = o.y + v[4 * q + 1];
          v[4 * q + 2] = o.z + v[4 * q + 2];
          v[4 * q + 3] = o.w + v[4 * q + 3];
        }
      }
      if (p.mode == kFirst || p.mode == kMiddle || p.mode == kPart) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          pa[q] = make_float4(v[4 * q + 0], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(st.orow + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
          w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
          w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
          w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
          dst[q] = w;
        }
      }
    }
  }

  __device__ static void end_unit(const Params&, State&, int) {}
};

// Plain fp32 store of the tile into out[rows, ld] (dW rows of one vocab
// chunk, or the self-check GEMM's C).  Columns >= ncols are skipped.
struct EpiStore {
  struct Params {
    float* out;
    int rows;
    int ncols;
    int ld;
  };
  struct State {
    int row;
    bool valid;
  };

  __device__ static void begin_unit(const Params& p, State& st, int row, int, int) {
    st.row = row;
    st.valid = row < p.rows;
  }

  __device__ static void tile(const Params& p, State& st, uint32_t taddr, int nt) {
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      const int col0 = nt * kBN + c * 32;
      if (col0 >= p.ncols) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      if (!st.valid) continue;
      float* dst = p.out + static_cast<size_t>(st.row) * p.ld + col0;
      if (col0 + 32 <= p.ncols) {
        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          d4[q] = make_float4(__uint_as_float(r[4 * q + 0]), __uint_as_float(r[4 * q + 1]),
                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < p.ncols) dst[j] = __uint_as_float(r[j]);
      }
    }
  }

  __device__ static void end_unit(const Params&, State&, int) {}
};

// Fixed-order merge of the forward's per-split triples into
// lse = ln2 (M + log2 S), entropy = ln2 (log2 S - B / S),
// logp = ln2 (y_target - M - log2 S).
// One warp per row: lane l merges splits l, l + 32, l + 64, ... in ascending
// order, then the lanes combine by an xor butterfly.  merge(a, b) and
// merge(b, a) are bitwise equal (max and + are commutative), so every lane
// ends with the same triple, and the order depends only on the split count.
struct Triple {
  float m, s, b;
};

__device__ __forceinline__ Triple merge_triple(Triple x, Triple y) {
  const float mn = fmaxf(x.m, y.m);
  const float ax = ex2_approx(x.m - mn), ay = ex2_approx(y.m - mn);
  Triple r;
  r.m = mn;
  r.s = ax * x.s + ay * y.s;
  r.b = ax * fmaf(x.m - mn, x.s, x.b) + ay * fmaf(y.m - mn, y.s, y.b);
  return r;
}

// Partials are laid out [shard][T][Gs]: split g of row t sits in shard g / Gs
// at local split g % Gs (one shard of Gs = G splits without tensor
// parallelism).  The merge order depends only on G.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ pm,
                                                      const float* __restrict__ ps,
                                                      const float* __restrict__ pb,
                                                      const float* __restrict__ ytgt,
                                                      const int64_t* __restrict__ targets, int T,
                                                      int V, int G, int Gs,
                                                      float* __restrict__ logp,
                                                      float* __restrict__ entropy,
                                                      float* __restrict__ lse, uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;  // warp-uniform
  Triple acc{kMaskLogit, 0.f, 0.f};
  for (int g = lane; g < G; g += 32) {
    const size_t i = (static_cast<size_t>(g / Gs) * T + t) * Gs + g % Gs;
    acc = merge_triple(acc, Triple{pm[i], ps[i], pb[i]});
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Triple o;
    o.m = __shfl_xor_sync(0xffffffffu, acc.m, off);
    o.s = __shfl_xor_sync(0xffffffffu, acc.s, off);
    o.b = __shfl_xor_sync(0xffffffffu, acc.b, off);
    acc = merge_triple(acc, o);
  }
  if (lane != 0) return;
  const float l2s = log2f(acc.s);
  lse[t] = kLn2 * (acc.m + l2s);
  entropy[t] = kLn2 * (l2s - acc.b / acc.s);
  const int64_t tg = targets[t];
  if (tg < 0 || tg >= V) {
    logp[t] = __int_as_float(0x7fc00000);
    atomicOr(err, kDevErrTarget);
  } else {
    logp[t] = kLn2 * ((ytgt[t] - acc.m) - l2s);
  }
}

}  // namespace rlk
