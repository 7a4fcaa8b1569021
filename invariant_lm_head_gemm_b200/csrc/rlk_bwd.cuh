// rlk_bwd.cuh -- plan and unit order of the backward pass, which runs as one
// persistent, dependency-driven launch of the pair kernel (rlk_kernel.cuh).
//
// Work units (each one 256 x 256 accumulator tile of a CTA pair):
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
//   D(c, v, .) needs every R(c, ., v)            (counter rdone_j[c][v])
//   H(c, m, n) needs H(c - 1, m, n)               (flag hdone[c - 1][m][n])
//   R(c, ., .) overwrites buffer c % 3 only after every H(c - 3), D(c - 3)
//                                                 (counter bufdone[c - 3])
// CTA pairs claim units from a global counter in ascending order and a unit
// only ever waits for smaller units, all of them claimed earlier by pairs that
// are running; so every wait ends without any co-residency guarantee (each
// wait is also time-bounded).  Both CTAs of a pair signal each unit, so the
// counters count CTA halves.
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
  CUtensorMap w_k;                // W [V,H], K-major, box 64 x 128
  CUtensorMap w_mn;               // W read as MN-major (N = h, K = v), box 64 x 64 (x 2 when 3-D)
  CUtensorMap hid_mn;             // hidden read as MN-major (N = h, K = t), box 64 x 64 (x 2)
  CUtensorMap dx_k[kDxBuffers];   // dX buffer [T, ldx], K-major, box 64 x 128
  CUtensorMap dx_mn[kDxBuffers];  // dX buffer read as MN-major (M = v, K = t), box 64 x 64 (x 2)
  CUtensorMap dx_st[kDxBuffers];  // dX buffer written by TMA stores, box 32 x 32, no swizzle
};

struct BwdPlan {
  int T, H, V, ldx, NC, MT, NH;
  int RT_full, RT_last;  // 256-column recompute tiles per chunk
  int VT_full, VT_last;  // 256-row dW tiles per chunk (equal to RT_*)
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
  float* dh_acc;
  __nv_bfloat16* dhidden;
  float* dh_parts;    // non-null: per-chunk dHidden products instead (EpiDh::kPart)
  int part_rows;
  int part_chunks;
  int64_t v0;         // global vocab index of W's first row (a vocab shard's offset)
  int64_t Vfull;      // full vocabulary
  float* dW;
  uint32_t* rdone_m;  // [NC][MT]
  uint32_t* rdone_j;  // [NC][RT_full]
  uint32_t* hdone;    // [NC][MT][NH]
  uint32_t* bufdone;  // [NC]
  uint32_t* next_unit;  // unit claim counter (one word)
  uint32_t* err;
  float scale_log2;   // log2(e) / tau
  float inv_tau;
  int mn3;            // w_mn, hid_mn, dx_mn are 3-D maps (one box per 128 MN columns)
  uint64_t wait_limit_ns;  // bound of every wait (kWaitLimitNs outside the test hook)
  int stall_first_h;  // test hook: the first dHidden unit waits for one R unit too many
  uint32_t* chunk_done;  // null, or [NC] words: chunk c's word is set to `seq` once its
                         // dHidden and dW units are done (for an exchange that overlaps)
  uint32_t seq;
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
// Unit counts and unit decoding use 32-bit arithmetic: the host rejects any
// plan with 2^31 units or more (bwd_total_units counts in 64 bits).
__host__ __device__ inline int bwd_nR(const BwdPlan& P, int c) { return P.MT * bwd_rt(P, c); }
__host__ __device__ inline int bwd_nH(const BwdPlan& P) { return P.MT * P.NH; }
__host__ __device__ inline int bwd_nD(const BwdPlan& P, int c) {
  return P.NH * (c == P.NC - 1 ? P.VT_last : P.VT_full);
}
__host__ __device__ inline int bwd_group_size(const BwdPlan& P, int g) {
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
  p.MT = static_cast<int>((T + kPairM - 1) / kPairM);
  p.NH = static_cast<int>((H + kBN - 1) / kBN);
  p.RT_full = p.ldx / kBN;
  p.VT_full = p.ldx / kPairM;
  p.valid_last = static_cast<int>(V - static_cast<int64_t>(p.NC - 1) * p.ldx);
  p.RT_last = (p.valid_last + kBN - 1) / kBN;
  p.VT_last = (p.valid_last + kPairM - 1) / kPairM;
  p.KB_R = static_cast<int>(H / kBK);
  p.KB_D = static_cast<int>((T + kBK - 1) / kBK);
  p.total = bwd_total_units(p);
  return p;
}

__host__ inline long long bwd_total_units(const BwdPlan& P) {
  // every chunk contributes its R, H and D units once
  long long t = 0;
  for (int c = 0; c < P.NC; ++c) {
    const long long rt = c == P.NC - 1 ? P.RT_last : P.RT_full;
    const long long vt = c == P.NC - 1 ? P.VT_last : P.VT_full;
    t += static_cast<long long>(P.MT) * rt + static_cast<long long>(P.MT) * P.NH +
         static_cast<long long>(P.NH) * vt;
  }
  return t;
}

// Recompute units: the row block varies fastest, in descending order on odd
// vocab tiles (serpentine), so a tile's first units reuse the hidden rows the
// previous tile's last units have just read.
__host__ __device__ inline BwdUnit bwd_seg_R(const BwdPlan& P, int c, int i) {
  const int j = i / P.MT;
  const int m = (j & 1) ? P.MT - 1 - i % P.MT : i % P.MT;
  return BwdUnit{kUnitR, c, m, j};
}
// dHidden units of one chunk in groups of kHGroup row blocks: inside a group
// the row block varies fastest, then the column block.  The units in flight
// then share a few W column blocks and a few dX row blocks, so neither the
// chunk's W columns nor its dX rows have to stream from DRAM many times.
// Odd groups take the column blocks in descending order, so a group starts on
// the W columns the previous group's last units are still reading.
constexpr int kHGroup = 8;

__host__ __device__ inline BwdUnit bwd_seg_H(const BwdPlan& P, int c, int i) {
  const int full = P.MT / kHGroup;
  const int per_group = kHGroup * P.NH;
  int g, m, n;
  if (i < full * per_group) {
    g = i / per_group;
    const int r = i % per_group;
    n = r / kHGroup;
    m = g * kHGroup + r % kHGroup;
  } else {
    const int rem = P.MT % kHGroup;
    const int r = i - full * per_group;
    g = full;
    n = r / rem;
    m = full * kHGroup + r % rem;
  }
  if (g & 1) n = P.NH - 1 - n;
  return BwdUnit{kUnitH, c, m, n};
}
// dW units: the column block varies fastest, in descending order on odd
// vocab blocks (serpentine, for the same reuse of hidden's columns).
__host__ __device__ inline BwdUnit bwd_seg_D(const BwdPlan& P, int c, int i) {
  const int v = i / P.NH;
  const int n = (v & 1) ? P.NH - 1 - i % P.NH : i % P.NH;
  return BwdUnit{kUnitD, c, v, n};
}

// Unit r of group g: H(g), then D(g), then R(g + 2).
__host__ __device__ inline BwdUnit bwd_group_unit(const BwdPlan& P, int g, int r) {
  const int h = bwd_nH(P);
  if (r < h) return bwd_seg_H(P, g, r);
  r -= h;
  const int d = bwd_nD(P, g);
  if (r < d) return bwd_seg_D(P, g, r);
  return bwd_seg_R(P, g + 2, r - d);
}

__host__ __device__ inline BwdUnit bwd_decode(const BwdPlan& P, int u) {
  for (int c = 0; c < 2 && c < P.NC; ++c) {
    const int n = bwd_nR(P, c);
    if (u < n) return bwd_seg_R(P, c, u);
    u -= n;
  }
  // groups 0 .. NC-4 involve full chunks only and all have the same size
  const int nreg = P.NC > 3 ? P.NC - 3 : 0;
  const int gs = bwd_nH(P) + P.NH * P.VT_full + P.MT * P.RT_full;
  if (u < nreg * gs) {
    const int g = u / gs;
    return bwd_group_unit(P, g, u - g * gs);
  }
  u -= nreg * gs;
  for (int g = nreg; g < P.NC; ++g) {
    const int n = bwd_group_size(P, g);
    if (u < n) return bwd_group_unit(P, g, u);
    u -= n;
  }
  return BwdUnit{-1, 0, 0, 0};
}

}  // namespace rlk
