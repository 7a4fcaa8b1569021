// rlk_kernel.cuh -- the persistent CTA-pair kernel behind the forward pass,
// the backward pass and the self-check GEMM.
//
// Each cluster of two CTAs computes 256 x 256 fp32 accumulator tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r of the pair
// loads rows [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r + 128)
// of the B tile (its half of N) into its own shared memory, the pair's leader
// (rank 0) issues the MMAs, and each CTA's TMEM receives its 128 accumulator
// rows.  Per CTA and 64-wide K block that is 16 KB of A and 16 KB of B.  A
// pipeline stage holds two K blocks (64 KB per CTA, eight MMAs), and three
// stages fit in shared memory.  The one MMA-issuing thread spends a roughly
// fixed time per stage (its barrier wait and its commit) on top of issuing the
// MMAs, so eight MMAs per stage keep the tensor pipe busier than four.
//
// Roles per CTA (192 threads): warp 0 TMA producer (both CTAs load; the
// leader arms its "full" barrier with both CTAs' bytes and both CTAs' loads
// complete on it); warp 1 allocates the pair's TMEM (two 256-column
// accumulators) and, in the leader, issues the MMAs and commits them to the
// "empty" / "full accumulator" barriers of both CTAs; warps 2-5 epilogue,
// one accumulator row per thread, releasing the accumulator to the leader.
//
// Units are walked in ascending order, pair p taking units p, p + pairs, ...;
// a unit is `ntiles` consecutive N tiles of one M tile (several only in the
// forward, whose epilogue carries its online reduction across them).  Every
// wait is time-bounded; on expiry the kernel records RLK_DEVERR_TIMEOUT,
// drains its in-flight copies and MMAs and returns.
#pragma once

#include "rlk_bwd.cuh"
#include "rlk_gemm.cuh"

namespace rlk {

constexpr uint32_t kSubA = kBM * kBK * 2;     // one K block of this CTA's 128 rows of A: 16 KB
constexpr uint32_t kSubB = kBM * kBK * 2;     // one K block of this CTA's 128 rows of B: 16 KB
constexpr int kSubK = 2;                      // K blocks per pipeline stage
constexpr uint32_t kPAStage = kSubK * kSubA;  // a stage's A: 32 KB
constexpr uint32_t kPBStage = kSubK * kSubB;  // a stage's B: 32 KB
constexpr int kRing = 4;                      // units in flight through the pair's broadcast ring

enum : int { kModeFwd = 0, kModeBwd = 1, kModeGemm = 2 };

// Shared memory per mode: three operand stages (192 KB); the backward's
// dlogit epilogue adds 16 KB of TMA store staging (two 2 KB buffers per
// epilogue warp).
template <int Mode>
struct PipeCfg {
  static constexpr int kStages = 3;
  static constexpr uint32_t kStaging = Mode == kModeBwd ? 4 * 4096 : 0;
  static constexpr int kNumBars = 2 * kStages + 5 + 2 * kRing;
  static constexpr size_t kSmemBytes =
      1024 + kStages * (kPAStage + kPBStage) + kStaging + kNumBars * 8 + 64;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};
enum : int { kJobFwd = 3, kJobGemm = 4 };  // backward jobs use kUnitR / kUnitH / kUnitD

struct FwdArgs {
  CUtensorMap hid_k;  // hidden [T,H], box 64 x 128 (64 x 128 x 2 when k3)
  CUtensorMap w_k;    // W [V,H], box 64 x 128 (64 x 128 x 2 when k3)
  EpiFwd::Params ep;
  uint32_t* err;
  int MT;             // 256-row M tiles
  int NT;             // 256-column vocab tiles
  int group;          // vocab tiles per unit
  int NG;             // vocab splits = ceil(NT / group)
  int KB;             // K blocks (H / 64)
  int k3;             // both maps 3-D: one copy per operand and stage
  long long total;    // MT * NG
};

struct GemmArgs {
  CUtensorMap a;      // K-major box 64 x 128, or MN-major box 64 x 64 (64 x 64 x 2 when a3)
  CUtensorMap b;
  EpiStore::Params ep;
  uint32_t* err;
  int M, N, MT, NT, KB;
  int a_mn, b_mn;
  int a3, b3;
  int ak3, bk3;       // K-major operand mapped 3-D (one copy per stage)
  long long total;
};

template <int Mode>
struct ModeArgs;
template <>
struct ModeArgs<kModeFwd> {
  using type = FwdArgs;
};
template <>
struct ModeArgs<kModeBwd> {
  using type = BwdParams;
};
template <>
struct ModeArgs<kModeGemm> {
  using type = GemmArgs;
};

// What one unit loads and computes.
struct Job {
  int type;
  int c;            // vocab chunk (backward)
  int mt;           // M tile (256 rows)
  int nt;           // first N tile (256 columns)
  int ntiles;       // N tiles in the unit
  int kbs;          // K blocks per tile
  bool a_mn, b_mn;  // operand majorness
  bool a3, b3;      // MN-major operand mapped 3-D: one box per 128 MN columns (else two 2-D boxes)
  bool ak3, bk3;    // K-major operand mapped 3-D (64 K, rows, K / 64) with box 64 x 128 x 2:
                    // one copy lands a stage's two K blocks (else one 2-D box per K block)
  const CUtensorMap* mA;
  const CUtensorMap* mB;
  int a_row0;       // M coordinate of the tile's first row in A's tensor map
  int b_col0;       // N coordinate of the first tile's first column in B's map
  int bk0;          // K offset of B's map
  int a_ext;        // M extent of A's map: boxes starting at or past it are skipped
  int b_ext;        // N extent of B's map
};

__device__ __forceinline__ Job make_job(const FwdArgs& P, long long u) {
  Job j;
  j.type = kJobFwd;
  j.c = 0;
  j.mt = static_cast<int>(u % P.MT);
  const int g = static_cast<int>(u / P.MT);
  j.nt = g * P.group;
  j.ntiles = min(P.group, P.NT - j.nt);
  j.kbs = P.KB;
  j.a_mn = j.b_mn = false;
  j.a3 = j.b3 = false;
  j.ak3 = j.bk3 = P.k3 != 0;
  j.mA = &P.hid_k;
  j.mB = &P.w_k;
  j.a_row0 = j.mt * kPairM;
  j.b_col0 = j.nt * kBN;
  j.bk0 = 0;
  j.a_ext = P.ep.T;
  j.b_ext = P.ep.V;
  return j;
}

__device__ __forceinline__ Job make_job(const GemmArgs& P, long long u) {
  Job j;
  j.type = kJobGemm;
  j.c = 0;
  j.mt = static_cast<int>(u % P.MT);
  j.nt = static_cast<int>(u / P.MT);
  j.ntiles = 1;
  j.kbs = P.KB;
  j.a_mn = P.a_mn != 0;
  j.b_mn = P.b_mn != 0;
  j.a3 = P.a3 != 0;
  j.b3 = P.b3 != 0;
  j.ak3 = P.ak3 != 0;
  j.bk3 = P.bk3 != 0;
  j.mA = &P.a;
  j.mB = &P.b;
  j.a_row0 = j.mt * kPairM;
  j.b_col0 = j.nt * kBN;
  j.bk0 = 0;
  j.a_ext = P.M;
  j.b_ext = P.N;
  return j;
}

__device__ __forceinline__ Job make_job(const BwdParams& P, long long u) {
  const BwdPlan& pl = P.plan;
  const BwdUnit un = bwd_decode(pl, static_cast<int>(u));
  Job j;
  j.type = un.type;
  j.c = un.c;
  j.mt = un.a;
  j.nt = un.b;
  j.ntiles = 1;
  j.bk0 = 0;
  j.a3 = j.b3 = false;
  j.ak3 = j.bk3 = false;
  const int buf = un.c % kDxBuffers;
  if (un.type == kUnitR) {
    j.kbs = pl.KB_R;
    j.a_mn = j.b_mn = false;
    j.mA = &P.maps.hid_k;
    j.mB = &P.maps.w_k;
    j.a_row0 = un.a * kPairM;
    j.b_col0 = un.c * pl.ldx + un.b * kBN;
    j.a_ext = pl.T;
    j.b_ext = pl.V;
  } else if (un.type == kUnitH) {
    j.kbs = (bwd_chunk_valid(pl, un.c) + kBK - 1) / kBK;
    j.a_mn = false;
    j.b_mn = true;
    j.mA = &P.maps.dx_k[buf];
    j.mB = &P.maps.w_mn;
    j.b3 = P.mn3 != 0;
    j.a_row0 = un.a * kPairM;
    j.b_col0 = un.b * kBN;
    j.bk0 = un.c * pl.ldx;
    j.a_ext = pl.T;
    j.b_ext = pl.H;
  } else {
    j.kbs = pl.KB_D;
    j.a_mn = j.b_mn = true;
    j.mA = &P.maps.dx_mn[buf];
    j.mB = &P.maps.hid_mn;
    j.a3 = j.b3 = P.mn3 != 0;
    j.a_row0 = un.a * kPairM;
    j.b_col0 = un.b * kBN;
    j.a_ext = pl.ldx;
    j.b_ext = pl.H;
  }
  return j;
}

__device__ __forceinline__ long long total_units(const FwdArgs& P) { return P.total; }
__device__ __forceinline__ long long total_units(const GemmArgs& P) { return P.total; }
__device__ __forceinline__ long long total_units(const BwdParams& P) { return P.plan.total; }
__device__ __forceinline__ uint32_t* err_word(const FwdArgs& P) { return P.err; }
__device__ __forceinline__ uint32_t* err_word(const GemmArgs& P) { return P.err; }
__device__ __forceinline__ uint32_t* err_word(const BwdParams& P) { return P.err; }
__device__ __forceinline__ uint64_t wait_limit(const FwdArgs&) { return kWaitLimitNs; }
__device__ __forceinline__ uint64_t wait_limit(const GemmArgs&) { return kWaitLimitNs; }
__device__ __forceinline__ uint64_t wait_limit(const BwdParams& P) { return P.wait_limit_ns; }

// K blocks of stage `st` of a tile of `kbs` K blocks (the last stage of an odd
// count holds one).
__device__ __forceinline__ int stage_kblocks(int kbs, int st) {
  return min(kSubK, kbs - st * kSubK);
}

// Bytes CTA `rank` loads in a stage of `nsub` K blocks of tile `t` of the job.
// A 3-D K-major box always lands both K blocks of a stage (a second block
// past K is filled, and a box counts in full), so it counts twice whatever
// nsub is; the other boxes count once per K block.
__device__ __forceinline__ uint32_t stage_bytes(const Job& j, int t, uint32_t rank, int nsub) {
  uint32_t bytes = 0;
  const int a0 = j.a_row0 + kBM * static_cast<int>(rank);
  if (!j.a_mn) {
    if (a0 < j.a_ext) bytes += j.ak3 ? kSubK * kSubA : nsub * kSubA;
  } else if (j.a3) {
    if (a0 < j.a_ext) bytes += nsub * 2 * kBox;  // the box counts in full, past-the-end half filled
  } else {
    if (a0 < j.a_ext) bytes += nsub * kBox;
    if (a0 + 64 < j.a_ext) bytes += nsub * kBox;
  }
  const int b0 = j.b_col0 + t * kBN + kBM * static_cast<int>(rank);
  if (!j.b_mn) {
    if (b0 < j.b_ext) bytes += j.bk3 ? kSubK * kSubB : nsub * kSubB;
  } else if (j.b3) {
    if (b0 < j.b_ext) bytes += nsub * 2 * kBox;
  } else {
    if (b0 < j.b_ext) bytes += nsub * kBox;
    if (b0 + 64 < j.b_ext) bytes += nsub * kBox;
  }
  return bytes;
}

template <int Mode>
__global__ void __launch_bounds__(kThreads, 1)
    pair_kernel(const __grid_constant__ typename ModeArgs<Mode>::type P) {
  constexpr int kPStages = PipeCfg<Mode>::kStages;
  constexpr uint32_t kPStaging = PipeCfg<Mode>::kStaging;
  constexpr int kPNumBars = PipeCfg<Mode>::kNumBars;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kPStages * kPAStage;
  const uint32_t sStage = sB + kPStages * kPBStage;
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(smem + kPStages * (kPAStage + kPBStage) + kPStaging);
  const uint32_t bar0 = smem_u32(bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kPNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* ep_unit = reinterpret_cast<volatile int*>(tmem_slot + 3);
  const uint32_t ring_addr = smem_u32(tmem_slot + 4);  // kRing unit indices

  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kPStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kPStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kPStages + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kPStages + 4);
  auto sfull_bar = [&](int i) { return bar0 + 8u * (2 * kPStages + 5 + i); };
  auto sempty_bar = [&](int i) { return bar0 + 8u * (2 * kPStages + 5 + kRing + i); };

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const long long pair = blockIdx.x >> 1;
  const long long npairs = gridDim.x >> 1;
  const long long total = total_units(P);
  uint32_t* err = err_word(P);
  const uint64_t lim = wait_limit(P);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(sfull_bar(i), 1);
      mbar_init(sempty_bar(i), 4);  // leader MMA + both CTAs' epilogues + the peer's producer
    }
    *abort_flag = 0;
    *ep_ok = 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Unit order.  Forward and self-check GEMM: pair p runs units p, p + pairs,
  // ...  Backward (units of unequal length that wait on each other): the
  // leader's producer claims the next unit from a global counter, in
  // ascending order, and broadcasts it through a kRing-slot ring to the
  // leader's MMA issuer, the peer's producer and both CTAs' epilogues.
  constexpr bool kDynamic = Mode == kModeBwd;
  auto static_unit = [&](uint32_t k) -> long long {
    const long long u = pair + static_cast<long long>(k) * npairs;
    return u < total ? u : -1;
  };
  // The peer's copy of a slot completes the peer's "full" barrier by the
  // store's own transaction count; the leader's copy by a CTA-scope arrival.
  // A slot is rewritten by the leader's producer once every consumer has
  // arrived on its "empty" barrier.  A consumer in the leader's own CTA orders
  // its read of the slot with a CTA-scope release (the writer is in its CTA);
  // a cluster-scope one held the MMA-issuing thread ~1.3k cycles per unit.
  // The peer's consumers read the peer's copy and release at cluster scope.
  auto fetch_unit = [&](uint32_t k, bool arm = false) -> long long {
    const int slot = k % kRing;
    // the peer's producer arms its own copy's barrier for the leader's 4-byte
    // asynchronous store (the phase completes once both have happened)
    if (arm) mbar_arrive_expect_tx(sfull_bar(slot), 4u);
    if (!mbar_wait_cluster_bounded(sfull_bar(slot), (k / kRing) & 1u, abort_flag, err, lim)) return -1;
    const int v = static_cast<int>(ld_shared_u32(ring_addr + 4u * slot));
    if (leader) {
      mbar_arrive(sempty_bar(slot));
    } else {
      mbar_arrive_cluster(mapa_shared(sempty_bar(slot), 0));
    }
    return v;
  };
  // The leader's producer claims each unit one unit ahead of publishing it
  // (the claim's atomic then runs while the current unit's copies are issued),
  // and publishes unit k in ring slot k % kRing.  Claiming ahead keeps the
  // order ascending, and a claimed unit is always processed by a running pair.
  auto publish_unit = [&](uint32_t k, long long u) -> long long {
    const int slot = k % kRing;
    if (!mbar_wait_bounded(sempty_bar(slot), ((k / kRing) & 1u) ^ 1u, abort_flag, err, lim)) return -1;
    if (u >= total) u = -1;
    // the own CTA's copy first, ordered at CTA scope (its MMA issuer waits for
    // it); the peer's copy by an asynchronous store that completes the peer's
    // barrier itself: a cluster-scope release here waited for this thread's
    // copies still in flight (~1.3k cycles per unit)
    tmem_slot[4 + slot] = static_cast<uint32_t>(u);
    mbar_arrive(sfull_bar(slot));
    st_async_cluster_u32(mapa_shared(ring_addr + 4u * slot, 1), static_cast<uint32_t>(u),
                         mapa_shared(sfull_bar(slot), 1));
    return u;
  };

  uint32_t issued = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      uint32_t claimed = 0;
      if constexpr (kDynamic) {
        if (leader) claimed = atomicAdd(P.next_unit, 1u);
      }
      for (uint32_t k = 0; ok; ++k) {
        long long u;
        if constexpr (kDynamic) {
          if (leader) {
            u = publish_unit(k, claimed);
            if (u >= 0) claimed = atomicAdd(P.next_unit, 1u);
          } else {
            u = fetch_unit(k, true);
          }
        } else {
          u = static_unit(k);
        }
        if (u < 0) break;
        const Job j = make_job(P, u);
        if (j.type < 0) break;
        if constexpr (Mode == kModeBwd) {
          const BwdPlan& pl = P.plan;
          if (j.type == kUnitH) {
            // the test hook asks one unit too many of the first dHidden unit
            const uint32_t extra =
                P.stall_first_h != 0 && j.c == 0 && j.mt == 0 && j.nt == 0 ? 1u : 0u;
            ok = wait_counter_bounded(P.rdone_m + static_cast<size_t>(j.c) * pl.MT + j.mt,
                                      2u * static_cast<uint32_t>(bwd_rt(pl, j.c)) + extra,
                                      abort_flag, err, lim);
          } else if (j.type == kUnitD) {
            ok = wait_counter_bounded(P.rdone_j + static_cast<size_t>(j.c) * pl.RT_full + j.mt,
                                      2u * static_cast<uint32_t>(pl.MT), abort_flag, err, lim);
          }
          if (!ok) break;
          if (j.type != kUnitR) fence_proxy_async_global();
        }
        if (k == 0) {
          tma_prefetch_desc(j.mA);
          tma_prefetch_desc(j.mB);
        }
        for (int t = 0; ok && t < j.ntiles; ++t) {
          const int a0 = j.a_row0 + kBM * static_cast<int>(rank);
          const int b0 = j.b_col0 + t * kBN + kBM * static_cast<int>(rank);
          const int nst = (j.kbs + kSubK - 1) / kSubK;
          // the leader's expected bytes of a full stage and of the last one,
          // worked out once per tile (they sit on the path from a free stage
          // to its copies)
          const uint32_t bytes_full =
              leader ? stage_bytes(j, t, 0, kSubK) + stage_bytes(j, t, 1, kSubK) : 0u;
          const int nsub_last = stage_kblocks(j.kbs, nst - 1);
          const uint32_t bytes_last =
              leader ? stage_bytes(j, t, 0, nsub_last) + stage_bytes(j, t, 1, nsub_last) : 0u;
          // A stage's copies are issued the moment its slot is free: everything
          // they need is worked out before the wait, and the leader arms the
          // full barrier after its own copies (its transaction count may run
          // below zero meanwhile, as it does whenever the peer's copies land
          // first).  In the load-bound backward this path sets when each
          // load starts.
          int s = static_cast<int>(issued % kPStages);
          uint32_t ph = (issued / kPStages) & 1u;
          for (int st = 0; st < nst; ++st) {
            const int nsub = stage_kblocks(j.kbs, st);
            const uint32_t fb = mapa_shared(full_bar(s), 0);
            const uint32_t dA = sA + s * kPAStage, dB = sB + s * kPBStage;
            const int k0 = st * kSubK * kBK, k1 = k0 + kBK;
            const uint32_t bytes = st + 1 < nst ? bytes_full : bytes_last;
            if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, err, lim)) {
              ok = false;
              break;
            }
            // 3-D K-major operands: one copy of the stage's two K blocks
            if (!j.a_mn && j.ak3 && a0 < j.a_ext)
              tma_load_3d_pair(dA, j.mA, fb, 0, a0, st * kSubK);
            if (!j.b_mn && j.bk3 && b0 < j.b_ext)
              tma_load_3d_pair(dB, j.mB, fb, 0, b0, st * kSubK);
            for (int sub = 0; sub < nsub; ++sub) {
              const uint32_t dAs = dA + sub * kSubA, dBs = dB + sub * kSubB;
              const int k = sub == 0 ? k0 : k1;
              if (!j.a_mn) {
                if (!j.ak3 && a0 < j.a_ext) tma_load_2d_pair(dAs, j.mA, fb, k, a0);
              } else if (j.a3) {
                if (a0 < j.a_ext) tma_load_3d_pair(dAs, j.mA, fb, 0, k, a0 >> 6);
              } else {
                if (a0 < j.a_ext) tma_load_2d_pair(dAs, j.mA, fb, a0, k);
                if (a0 + 64 < j.a_ext) tma_load_2d_pair(dAs + kBox, j.mA, fb, a0 + 64, k);
              }
              if (!j.b_mn) {
                if (!j.bk3 && b0 < j.b_ext) tma_load_2d_pair(dBs, j.mB, fb, k, b0);
              } else if (j.b3) {
                if (b0 < j.b_ext) tma_load_3d_pair(dBs, j.mB, fb, 0, j.bk0 + k, b0 >> 6);
              } else {
                if (b0 < j.b_ext) tma_load_2d_pair(dBs, j.mB, fb, b0, j.bk0 + k);
                if (b0 + 64 < j.b_ext) tma_load_2d_pair(dBs + kBox, j.mB, fb, b0 + 64, j.bk0 + k);
              }
            }
            if (leader) mbar_arrive_expect_tx(full_bar(s), bytes);
            ++issued;
            if (++s == kPStages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        long long u;
        if constexpr (kDynamic) {
          u = fetch_unit(k);
        } else {
          u = static_unit(k);
        }
        if (u < 0) break;
        const Job j = make_job(P, u);
        if (j.type < 0) break;
        const uint32_t idesc = idesc_bf16_f32(kPairM, kBN, j.a_mn, j.b_mn);
        const uint32_t a_lbo = j.a_mn ? 8192u : 16u, b_lbo = j.b_mn ? 8192u : 16u;
        const uint32_t a_kstep = j.a_mn ? 2048u : 32u, b_kstep = j.b_mn ? 2048u : 32u;
        for (int t = 0; ok && t < j.ntiles; ++t, ++tc) {
          const int acc = tc & 1;
          const uint32_t use = tc >> 1;
          if (!mbar_wait_bounded(tempty_bar(acc), (use & 1u) ^ 1u, abort_flag, err, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * kBN;
          const int nst = (j.kbs + kSubK - 1) / kSubK;
          for (int st = 0; st < nst; ++st, ++it) {
            const int s = it % kPStages;
            const uint32_t ph = (it / kPStages) & 1u;
            if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, err, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int nsub = stage_kblocks(j.kbs, st);
            for (int sub = 0; sub < nsub; ++sub) {
              const uint32_t a_s = sA + s * kPAStage + sub * kSubA;
              const uint32_t b_s = sB + s * kPBStage + sub * kSubB;
#pragma unroll
              for (int k = 0; k < kBK / 16; ++k) {
                const uint64_t ad = smem_desc_sw128(a_s + k * a_kstep, a_lbo, 1024u);
                const uint64_t bd = smem_desc_sw128(b_s + k * b_kstep, b_lbo, 1024u);
                umma_bf16_pair(d_tmem, ad, bd, idesc, (st | sub | k) != 0 ? 1u : 0u);
              }
            }
            umma_commit_pair_both(empty_bar(s));
          }
          if (ok) umma_commit_pair_both(tfull_bar(acc));
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const int row_off = kBM * static_cast<int>(rank) + row_in_tile;
    const bool ep_leader = threadIdx.x == 64;
    uint32_t tc = 0;
    bool go = true;
    for (uint32_t k = 0; go; ++k) {
      long long u;
      if constexpr (kDynamic) {
        if (ep_leader) *ep_unit = static_cast<int>(fetch_unit(k));
        epilogue_bar();
        u = *ep_unit;
      } else {
        u = static_unit(k);
      }
      if (u < 0) break;
      const Job j = make_job(P, u);
      if (j.type < 0) break;
      typename EpiFwd::State fst;
      if constexpr (Mode == kModeFwd) EpiFwd::begin_unit(P.ep, fst, j.mt * kPairM + row_off, 0, 0);
      for (int t = 0; t < j.ntiles; ++t, ++tc) {
        const int acc = tc & 1;
        const uint32_t use = tc >> 1;
        if (ep_leader) {
          bool ok = mbar_wait_bounded(tfull_bar(acc), use & 1u, abort_flag, err, lim);
          if constexpr (Mode == kModeBwd) {
            const BwdPlan& pl = P.plan;
            if (ok && j.type == kUnitR && j.c >= kDxBuffers) {
              const int c3 = j.c - kDxBuffers;
              ok = wait_counter_bounded(P.bufdone + c3,
                                        2u * static_cast<uint32_t>(bwd_nH(pl) + bwd_nD(pl, c3)),
                                        abort_flag, err, lim);
            }
            if (ok && j.type == kUnitH && j.c >= 1) {
              ok = wait_counter_bounded(
                  P.hdone + (static_cast<size_t>(j.c - 1) * pl.MT + j.mt) * pl.NH + j.nt, 2u,
                  abort_flag, err, lim);
            }
          }
          *ep_ok = ok ? 1 : 0;
        }
        epilogue_bar();
        if (!*ep_ok) {
          go = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kBN;
        const int row = j.mt * kPairM + row_off;
        if constexpr (Mode == kModeFwd) {
          EpiFwd::tile(P.ep, fst, taddr, j.nt + t);
        } else if constexpr (Mode == kModeGemm) {
          EpiStore::State st;
          EpiStore::begin_unit(P.ep, st, row, 0, 0);
          EpiStore::tile(P.ep, st, taddr, j.nt);
        } else {
          const BwdPlan& pl = P.plan;
          if (j.type == kUnitR) {
            EpiDlogits::Params p;
            p.targets = P.targets;
            p.lse = P.lse;
            p.entropy = P.entropy;
            p.dlogp = P.dlogp;
            p.dentropy = P.dentropy;
            p.err = err;
            p.T = pl.T;
            p.V = pl.V;
            p.c0 = j.c * pl.ldx;
            p.v0 = P.v0;
            p.Vfull = P.Vfull;
            p.scale_log2 = P.scale_log2;
            p.inv_tau = P.inv_tau;
            EpiDlogits::State st;
            EpiDlogits::begin_unit(p, st, row, 0, 0);
            EpiDlogits::tile(p, st, taddr, j.nt, &P.maps.dx_st[j.c % kDxBuffers],
                             sStage + q * 4096u, lane, row - lane);
          } else if (j.type == kUnitH) {
            EpiDh::Params p;
            p.acc = P.dh_acc;
            p.out = P.dhidden;
            p.T = pl.T;
            p.H = pl.H;
            p.mode = P.dh_parts          ? EpiDh::kPart
                     : pl.NC == 1        ? EpiDh::kOnly
                     : j.c == 0          ? EpiDh::kFirst
                     : j.c == pl.NC - 1  ? EpiDh::kLast
                                         : EpiDh::kMiddle;
            if (P.dh_parts) p.acc = P.dh_parts;
            p.c = j.c;
            p.part_rows = P.part_rows;
            p.part_chunks = P.part_chunks;
            EpiDh::State st;
            EpiDh::begin_unit(p, st, row, 0, 0);
            EpiDh::tile(p, st, taddr, j.nt);
          } else {
            EpiStore::Params p;
            p.out = P.dW + static_cast<size_t>(j.c) * pl.ldx * pl.H;
            p.rows = bwd_chunk_valid(pl, j.c);
            p.ncols = pl.H;
            p.ld = pl.H;
            EpiStore::State st;
            EpiStore::begin_unit(p, st, row, 0, 0);
            EpiStore::tile(p, st, taddr, j.nt);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {  // to the leader's MMA issuer: CTA scope from its own CTA
          if (leader) {
            mbar_arrive(tempty_bar(acc));
          } else {
            mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
          }
        }
        if constexpr (Mode == kModeBwd) {
          if (j.type == kUnitR && lane == 0) bulk_wait_all();  // dX tiles written
          epilogue_bar();  // every store of this CTA's half of the unit is done or issued
          if (ep_leader) {
            const BwdPlan& pl = P.plan;
            fence_proxy_async_global();
            __threadfence();
            if (j.type == kUnitR) {
              atomicAdd(P.rdone_m + static_cast<size_t>(j.c) * pl.MT + j.mt, 1u);
              atomicAdd(P.rdone_j + static_cast<size_t>(j.c) * pl.RT_full + j.nt, 1u);
            } else {
              if (j.type == kUnitH)
                atomicAdd(P.hdone + (static_cast<size_t>(j.c) * pl.MT + j.mt) * pl.NH + j.nt,
                          1u);
              const uint32_t done = atomicAdd(P.bufdone + j.c, 1u) + 1u;
              // the CTA that completes chunk c's dHidden and dW units publishes
              // it: every other CTA's stores were fenced before its increment
              if (P.chunk_done != nullptr &&
                  done == 2u * static_cast<uint32_t>(bwd_nH(pl) + bwd_nD(pl, j.c))) {
                __threadfence_system();
                st_release_sys_u32(P.chunk_done + j.c, P.seq);
              }
            }
          }
        }
      }
      if constexpr (Mode == kModeFwd) {
        if (go) EpiFwd::end_unit(P.ep, fst, j.nt / P.group);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (Mode == kModeBwd) {
    // After a timed-out wait some chunks never complete: publish every chunk
    // word anyway, so that a stream waiting on them is released (the error
    // word already says the results are not to be used).
    if (*abort_flag && threadIdx.x == 0 && P.chunk_done != nullptr) {
      __threadfence_system();
      for (int c = 0; c < P.plan.NC; ++c) st_release_sys_u32(P.chunk_done + c, P.seq);
    }
  }
  if (*abort_flag) {
    // Unwind after a timed-out wait: let TMA loads and MMAs in flight finish
    // before the shared memory and TMEM they touch go away.
    if (warp == 0 && lane == 0 && leader) {
      const uint32_t first = issued > static_cast<uint32_t>(kPStages) ? issued - kPStages : 0u;
      for (uint32_t i = first; i < issued; ++i)
        mbar_wait_drain(full_bar(i % kPStages), (i / kPStages) & 1u);
    }
    if (warp == 1 && lane == 0 && leader) {
      umma_commit_pair_both(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);  // 2 ms for the peer's copies
    __syncthreads();
  }
  cluster_sync();  // neither CTA frees TMEM or exits while the other may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace rlk
