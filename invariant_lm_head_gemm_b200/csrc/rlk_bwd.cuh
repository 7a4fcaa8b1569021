// rlk_bwd.cuh -- the whole backward pass in one persistent, dependency-driven
// launch.
//
// Work units (each one 128 x 256 accumulator tile, same mainloop as
// gemm_kernel):
//   R(c, m, j)  recompute the logits of row tile m and vocab tile j of chunk
//               c (K = H) and write bf16 dlogits into dX buffer c % 3;
//   H(c, m, n)  dHidden tile (m, n) += dX_c[m rows, :] . W[chunk c rows, n cols]
//               (K = the chunk's vocab entries), chunks added in ascending
//               order (old + new), the last one written as bf16;
//   D(c, v, n)  dW[chunk c rows v, n cols] = dX_c[:, v]^T . hidden[:, n]
//               (K = T, ascending, no atomics).
// Global order: R(0), R(1), then for g = 0 .. NC-1: H(g), D(g), R(g + 2).
// Every dependency points to an earlier unit, one group back or more:
//   H(c, m, .) needs every R(c, m, .)            (counter rdone_m[c][m])
//   D(c, v, .) needs every R(c, ., v / 2)        (counter rdone_j[c][v / 2])
//   H(c, m, n) needs H(c - 1, m, n)               (flag hdone[c - 1][m][n])
//   R(c, ., .) overwrites buffer c % 3 only after every H(c - 3), D(c - 3)
//                                                 (counter bufdone[c - 3])
// CTA b runs units b, b + grid, b + 2 grid, ... in ascending order and a
// unit only ever waits for smaller units, so with all CTAs resident (the
// launch is cooperative) every wait ends; each wait is also time-bounded.
// Producers of a counter store with generic stores, sync the epilogue warps,
// then one thread fences and increments; consumers acquire, and fence the
// async proxy before TMA reads of the data.
//
// The per-tile arithmetic, the K orders and the chunk order are exactly those
// of the per-chunk launches, so results do not depend on T or on scheduling.
#pragma once

#include "rlk_gemm.cuh"

namespace rlk {

constexpr int kDxBuffers = 3;

struct BwdMaps {
  CUtensorMap hid_k;              // hidden [T,H], K-major, box 64 x 128
  CUtensorMap w_k;                // W [V,H], K-major, box 64 x 256
  CUtensorMap w_mn;               // W read as MN-major (N = h, K = v), box 64 x 64
  CUtensorMap hid_mn;             // hidden read as MN-major (N = h, K = t), box 64 x 64
  CUtensorMap dx_k[kDxBuffers];   // dX buffer [T, ldx], K-major, box 64 x 128
  CUtensorMap dx_mn[kDxBuffers];  // dX buffer read as MN-major (M = v, K = t), box 64 x 64
};

struct BwdPlan {
  int T, H, V, ldx, NC, MT, NH;
  int RT_full, RT_last;  // 256-column recompute tiles per chunk
  int VT_full, VT_last;  // 128-row dW tiles per chunk
  int valid_last;        // vocab entries of the last chunk
  int KB_R;              // k-blocks of a recompute tile (H / 64)
  int KB_D;              // k-blocks of a dW tile (ceil(T / 64))
  long long total;       // number of units
};

struct BwdParams {
  BwdMaps maps;
  BwdPlan plan;
  const int64_t* targets;
  const float* lse;
  const float* entropy;
  const float* dlogp;
  const float* dentropy;
  __nv_bfloat16* dx[kDxBuffers];
  float* dh_acc;
  __nv_bfloat16* dhidden;
  float* dW;
  uint32_t* rdone_m;  // [NC][MT]
  uint32_t* rdone_j;  // [NC][RT_full]
  uint32_t* hdone;    // [NC][MT][NH]
  uint32_t* bufdone;  // [NC]
  uint32_t* err;
  float scale_log2;   // log2(e) / tau
  float inv_tau;
};

enum : int { kUnitR = 0, kUnitH = 1, kUnitD = 2 };

struct BwdUnit {
  int type, c, a, b;  // R: a = m, b = j;  H: a = m, b = n;  D: a = v, b = n
};

__host__ __device__ inline int bwd_chunk_valid(const BwdPlan& P, int c) {
  return c == P.NC - 1 ? P.valid_last : P.ldx;
}
__host__ __device__ inline int bwd_rt(const BwdPlan& P, int c) {
  return c == P.NC - 1 ? P.RT_last : P.RT_full;
}
__host__ __device__ inline long long bwd_nR(const BwdPlan& P, int c) {
  return static_cast<long long>(P.MT) * bwd_rt(P, c);
}
__host__ __device__ inline long long bwd_nH(const BwdPlan& P) {
  return static_cast<long long>(P.MT) * P.NH;
}
__host__ __device__ inline long long bwd_nD(const BwdPlan& P, int c) {
  return static_cast<long long>(P.NH) * (c == P.NC - 1 ? P.VT_last : P.VT_full);
}
__host__ __device__ inline long long bwd_group_size(const BwdPlan& P, int g) {
  return bwd_nH(P) + bwd_nD(P, g) + (g + 2 < P.NC ? bwd_nR(P, g + 2) : 0);
}

// Plan for T rows, H hidden, V vocab entries and vocab chunks of ldx columns
// (a multiple of 256).
__host__ inline long long bwd_total_units(const BwdPlan& P);

__host__ inline BwdPlan make_bwd_plan(int64_t T, int64_t H, int64_t V, int64_t ldx) {
  BwdPlan p;
  p.T = static_cast<int>(T);
  p.H = static_cast<int>(H);
  p.V = static_cast<int>(V);
  p.ldx = static_cast<int>(ldx);
  p.NC = static_cast<int>((V + ldx - 1) / ldx);
  p.MT = static_cast<int>((T + kBM - 1) / kBM);
  p.NH = static_cast<int>((H + kBN - 1) / kBN);
  p.RT_full = p.ldx / kBN;
  p.VT_full = p.ldx / kBM;
  p.valid_last = static_cast<int>(V - static_cast<int64_t>(p.NC - 1) * p.ldx);
  p.RT_last = (p.valid_last + kBN - 1) / kBN;
  p.VT_last = (p.valid_last + kBM - 1) / kBM;
  p.KB_R = static_cast<int>(H / kBK);
  p.KB_D = static_cast<int>((T + kBK - 1) / kBK);
  p.total = bwd_total_units(p);
  return p;
}

__host__ inline long long bwd_total_units(const BwdPlan& P) {
  long long t = 0;
  for (int c = 0; c < 2 && c < P.NC; ++c) t += bwd_nR(P, c);
  for (int g = 0; g < P.NC; ++g) t += bwd_group_size(P, g);
  return t;
}

__host__ __device__ inline BwdUnit bwd_seg_R(const BwdPlan& P, int c, long long i) {
  return BwdUnit{kUnitR, c, static_cast<int>(i % P.MT), static_cast<int>(i / P.MT)};
}
__host__ __device__ inline BwdUnit bwd_seg_H(const BwdPlan& P, int c, long long i) {
  return BwdUnit{kUnitH, c, static_cast<int>(i / P.NH), static_cast<int>(i % P.NH)};
}
__host__ __device__ inline BwdUnit bwd_seg_D(const BwdPlan& P, int c, long long i) {
  return BwdUnit{kUnitD, c, static_cast<int>(i / P.NH), static_cast<int>(i % P.NH)};
}

// Unit r of group g: H(g), then D(g), then R(g + 2).
__host__ __device__ inline BwdUnit bwd_group_unit(const BwdPlan& P, int g, long long r) {
  const long long h = bwd_nH(P);
  if (r < h) return bwd_seg_H(P, g, r);
  r -= h;
  const long long d = bwd_nD(P, g);
  if (r < d) return bwd_seg_D(P, g, r);
  return bwd_seg_R(P, g + 2, r - d);
}

__host__ __device__ inline BwdUnit bwd_decode(const BwdPlan& P, long long u) {
  for (int c = 0; c < 2 && c < P.NC; ++c) {
    const long long n = bwd_nR(P, c);
    if (u < n) return bwd_seg_R(P, c, u);
    u -= n;
  }
  // groups 0 .. NC-4 involve full chunks only and all have the same size
  const int nreg = P.NC > 3 ? P.NC - 3 : 0;
  const long long gs = bwd_nH(P) + static_cast<long long>(P.NH) * P.VT_full +
                       static_cast<long long>(P.MT) * P.RT_full;
  if (u < nreg * gs) {
    const int g = static_cast<int>(u / gs);
    return bwd_group_unit(P, g, u - g * gs);
  }
  u -= nreg * gs;
  for (int g = nreg; g < P.NC; ++g) {
    const long long n = bwd_group_size(P, g);
    if (u < n) return bwd_group_unit(P, g, u);
    u -= n;
  }
  return BwdUnit{-1, 0, 0, 0};
}

__global__ void __launch_bounds__(kThreads, 1) bwd_fused_kernel(const __grid_constant__ BwdParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kStages * kAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * (kAStage + kBStage));
  const uint32_t bar0 = smem_u32(bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);

  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);

  const BwdPlan& pl = P.plan;
  uint32_t* err = P.err;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *ep_ok = 1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&P.maps.hid_k);
    tma_prefetch_desc(&P.maps.w_k);
    tma_prefetch_desc(&P.maps.w_mn);
    tma_prefetch_desc(&P.maps.hid_mn);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  uint32_t issued = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < pl.total; u += gridDim.x) {
        const BwdUnit un = bwd_decode(pl, u);
        if (un.type < 0) break;
        const int buf = un.c % kDxBuffers;
        const CUtensorMap* mA;
        const CUtensorMap* mB;
        bool a_mn = false, b_mn = false;
        int kbs, m0, n0, bk0 = 0;
        if (un.type == kUnitR) {
          mA = &P.maps.hid_k;
          mB = &P.maps.w_k;
          kbs = pl.KB_R;
          m0 = un.a * kBM;
          n0 = un.c * pl.ldx + un.b * kBN;
        } else if (un.type == kUnitH) {
          ok = wait_counter_bounded(P.rdone_m + static_cast<size_t>(un.c) * pl.MT + un.a,
                                    static_cast<uint32_t>(bwd_rt(pl, un.c)), abort_flag, err);
          if (!ok) break;
          fence_proxy_async_global();
          mA = &P.maps.dx_k[buf];
          mB = &P.maps.w_mn;
          b_mn = true;
          kbs = (bwd_chunk_valid(pl, un.c) + kBK - 1) / kBK;
          m0 = un.a * kBM;
          n0 = un.b * kBN;
          bk0 = un.c * pl.ldx;
        } else {
          ok = wait_counter_bounded(P.rdone_j + static_cast<size_t>(un.c) * pl.RT_full + un.a / 2,
                                    static_cast<uint32_t>(pl.MT), abort_flag, err);
          if (!ok) break;
          fence_proxy_async_global();
          mA = &P.maps.dx_mn[buf];
          mB = &P.maps.hid_mn;
          a_mn = true;
          b_mn = true;
          kbs = pl.KB_D;
          m0 = un.a * kBM;
          n0 = un.b * kBN;
        }
        for (int kb = 0; kb < kbs; ++kb) {
          const int s = issued % kStages;
          const uint32_t ph = (issued / kStages) & 1u;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          const uint32_t dA = sA + s * kAStage;
          const uint32_t dB = sB + s * kBStage;
          uint32_t bytes = kAStage;
          if (!b_mn) {
            bytes += kBStage;
          } else {
#pragma unroll
            for (int j = 0; j < kBN / 64; ++j)
              if (n0 + 64 * j < pl.H) bytes += kBox;
          }
          mbar_arrive_expect_tx(full_bar(s), bytes);
          if (!a_mn) {
            tma_load_2d(dA, mA, full_bar(s), kb * kBK, m0);
          } else {
            tma_load_2d(dA, mA, full_bar(s), m0, kb * kBK);
            tma_load_2d(dA + kBox, mA, full_bar(s), m0 + 64, kb * kBK);
          }
          if (!b_mn) {
            tma_load_2d(dB, mB, full_bar(s), kb * kBK, n0);
          } else {
#pragma unroll
            for (int j = 0; j < kBN / 64; ++j)
              if (n0 + 64 * j < pl.H) tma_load_2d(dB + j * kBox, mB, full_bar(s), n0 + 64 * j, bk0 + kb * kBK);
          }
          ++issued;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (long long u = blockIdx.x; ok && u < pl.total; u += gridDim.x, ++tc) {
        const BwdUnit un = bwd_decode(pl, u);
        if (un.type < 0) break;
        const bool a_mn = un.type == kUnitD;
        const bool b_mn = un.type != kUnitR;
        const int kbs = un.type == kUnitR   ? pl.KB_R
                        : un.type == kUnitH ? (bwd_chunk_valid(pl, un.c) + kBK - 1) / kBK
                                            : pl.KB_D;
        const uint32_t idesc = idesc_bf16_f32(kBM, kBN, a_mn, b_mn);
        const uint32_t a_lbo = a_mn ? 8192u : 16u, b_lbo = b_mn ? 8192u : 16u;
        const uint32_t a_kstep = a_mn ? 2048u : 32u, b_kstep = b_mn ? 2048u : 32u;
        const int acc = tc & 1;
        const uint32_t use = tc >> 1;
        if (!mbar_wait_bounded(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (int kb = 0; kb < kbs; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sA + s * kAStage, b0 = sB + s * kBStage;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = smem_desc_sw128(a0 + k * a_kstep, a_lbo, 1024u);
            const uint64_t bd = smem_desc_sw128(b0 + k * b_kstep, b_lbo, 1024u);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(s));
        }
        if (ok) umma_commit(tfull_bar(acc));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const bool leader = threadIdx.x == 64;
    uint32_t tc = 0;
    for (long long u = blockIdx.x; u < pl.total; u += gridDim.x, ++tc) {
      const BwdUnit un = bwd_decode(pl, u);
      if (un.type < 0) break;
      const int acc = tc & 1;
      const uint32_t use = tc >> 1;
      if (leader) {
        bool ok = mbar_wait_bounded(tfull_bar(acc), use & 1u, abort_flag, err);
        if (ok && un.type == kUnitR && un.c >= kDxBuffers) {
          const int c3 = un.c - kDxBuffers;
          ok = wait_counter_bounded(P.bufdone + c3,
                                    static_cast<uint32_t>(bwd_nH(pl) + bwd_nD(pl, c3)),
                                    abort_flag, err);
        }
        if (ok && un.type == kUnitH && un.c >= 1) {
          ok = wait_counter_bounded(
              P.hdone + (static_cast<size_t>(un.c - 1) * pl.MT + un.a) * pl.NH + un.b, 1u,
              abort_flag, err);
        }
        *ep_ok = ok ? 1 : 0;
      }
      epilogue_bar();
      if (!*ep_ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kBN;
      if (un.type == kUnitR) {
        EpiDlogits::Params p;
        p.targets = P.targets;
        p.lse = P.lse;
        p.entropy = P.entropy;
        p.dlogp = P.dlogp;
        p.dentropy = P.dentropy;
        p.dX = P.dx[un.c % kDxBuffers];
        p.err = err;
        p.T = pl.T;
        p.V = pl.V;
        p.c0 = un.c * pl.ldx;
        p.ldx = pl.ldx;
        p.scale_log2 = P.scale_log2;
        p.inv_tau = P.inv_tau;
        EpiDlogits::State st;
        EpiDlogits::begin_unit(p, st, un.a * kBM + row_in_tile, un.a, 0);
        EpiDlogits::tile(p, st, taddr, un.b);
      } else if (un.type == kUnitH) {
        EpiDh::Params p;
        p.acc = P.dh_acc;
        p.out = P.dhidden;
        p.T = pl.T;
        p.H = pl.H;
        p.mode = pl.NC == 1 ? EpiDh::kOnly
                 : un.c == 0 ? EpiDh::kFirst
                 : un.c == pl.NC - 1 ? EpiDh::kLast
                                     : EpiDh::kMiddle;
        EpiDh::State st;
        EpiDh::begin_unit(p, st, un.a * kBM + row_in_tile, un.a, 0);
        EpiDh::tile(p, st, taddr, un.b);
      } else {
        EpiStore::Params p;
        p.out = P.dW + static_cast<size_t>(un.c) * pl.ldx * pl.H;
        p.rows = bwd_chunk_valid(pl, un.c);
        p.ncols = pl.H;
        p.ld = pl.H;
        EpiStore::State st;
        EpiStore::begin_unit(p, st, un.a * kBM + row_in_tile, un.a, 0);
        EpiStore::tile(p, st, taddr, un.b);
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      epilogue_bar();  // every store of this unit has been issued
      if (leader) {
        fence_proxy_async_global();
        __threadfence();
        if (un.type == kUnitR) {
          atomicAdd(P.rdone_m + static_cast<size_t>(un.c) * pl.MT + un.a, 1u);
          atomicAdd(P.rdone_j + static_cast<size_t>(un.c) * pl.RT_full + un.b, 1u);
        } else if (un.type == kUnitH) {
          atomicAdd(P.hdone + (static_cast<size_t>(un.c) * pl.MT + un.a) * pl.NH + un.b, 1u);
          atomicAdd(P.bufdone + un.c, 1u);
        } else {
          atomicAdd(P.bufdone + un.c, 1u);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      const uint32_t first = issued > static_cast<uint32_t>(kStages) ? issued - kStages : 0u;
      for (uint32_t i = first; i < issued; ++i)
        mbar_wait_drain(full_bar(i % kStages), (i / kStages) & 1u);
    }
    if (warp == 1 && lane == 0) {
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace rlk
