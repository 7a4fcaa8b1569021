// rlk_decode.cuh -- forward for short batches (rollout / decode shapes, T <= 256
// rows): the same per-split triples as the pair kernel's forward, produced
// with the operands swapped so that the tensor cores do not pad T up to 256.
//
// With T small the pair kernel's work is set by its 256-row tile: it issues
// 2 * 256 * H * V flops whatever T is, about as long as streaming W from
// HBM.  Here the MMA's M side is the vocabulary (128 W rows per CTA) and its N
// side the T rows (16, or T rounded up to 32), so the tensor work shrinks
// with T and the kernel runs at the pace of the W stream.  That pace is set
// by the bytes of W in flight per SM and by how long each pipeline stage is
// held: a stage carries two K blocks, so each MMA / commit turn frees 32 KB
// of W (one K block per stage held the stages ~20% longer for the same
// bytes).
//
// Two forms of the MMA, chosen by N:
//  * single (kPair = false, N < 64): tcgen05.mma.cta_group::1, M = 128; each
//    CTA holds its 128 W rows and all N hidden rows per K block;
//  * pair (kPair = true, 64 <= N <= 256): tcgen05.mma.cta_group::2, M = 256
//    over CTAs (2i, 2i+1) of the cluster; each CTA still holds its own 128 W
//    rows but only half of the N hidden rows (B is split along N across the
//    pair), and each CTA's TMEM receives its 128 W rows x all N columns, so
//    the epilogue is the same.  Halving the hidden bytes per CTA lets N reach
//    256 (three stages) where the single form would hold 64 KB of hidden per
//    stage, and gives N = 128 four stages instead of three.
//
// A second epilogue (kStore) turns the kernel into the short-row path of the
// plain dense GEMM: no fold and no chain, each accumulator column is stored
// as C[t][n] (coalesced across the lanes of a warp).  For a narrow C (few
// W rows) the store path also has a half-height form (kHalf: single-CTA
// MMA with M = 64, 64 W rows per CTA), which spreads the same W over twice
// the CTAs.  It gains only 2-5%: a short GEMM's time follows K, not its
// bytes or its CTA count (about 7 us plus 0.42 us per 128-wide K stage at
// N = 512-8192 and 16-128 CTAs), i.e. each CTA's serial chain of 16-wide MMA
// steps sets it.  An M = 64 accumulator fills TMEM lanes 0-15 of each warp's
// lane quarter (rows 16q .. 16q+15 in quarter q).
//
// Numerics are those of the pair kernel, bit for bit:
//  * each logit is the same bf16 dot product over H in the same 64-wide K
//    blocks and 16-wide MMA steps (D = A . B^T gives the same fp32 element
//    with A and B exchanged and whatever the M / N shape: each element is its
//    own product sum);
//  * a vocab split is 512 columns = four 128-row W tiles, one per CTA of a
//    cluster of four.  CTA r runs the split's chunks r*4 .. r*4+3 with
//    fwd_chunk_update after receiving the running (m, s, b) of every row from
//    CTA r-1 through distributed shared memory, so the chunks of a split are
//    folded in the same ascending order by the same code as in the pair
//    kernel;
//  * CTA 3 writes the split's triple where the pair kernel's forward writes
//    it, and the same combine kernel merges the splits.
//
// Warp roles per CTA (192 threads): warp 0 producer (TMA), warp 1 MMA issuer
// (in the pair form only the even CTA of each pair issues), warps 2-5
// epilogue (the fold below, or the store of kStore).  Two TMEM accumulators of up to 128 (single) or 256 (pair)
// columns.  The epilogue is a pipeline over 32-row batch blocks: the warp
// that reads TMEM lane quarter q holds chunk q of the tile, transposes its
// 32 x 32 block through its own shared-memory tile so that each lane holds one
// batch row, folds that chunk and hands the row's (m, s, b) to the warp of
// chunk q+1; the warp of chunk 3 hands it on to CTA rank+1 block by block.
// So the four warps and the four CTAs of a split work on different blocks at
// once, while each row still folds its 16 chunks in ascending order.  With a
// single block (N <= 32) there is nothing to overlap: warp 2 folds all four
// chunks from the four warps' tiles, which keeps the chain of CTAs at one
// hand-off per CTA.
#pragma once

#include "rlk_gemm.cuh"

namespace rlk {

constexpr int kDecMaxRows = 256;    // largest N of the pair form (hand buffer rows)
constexpr int kDecMaxT = 256;       // largest T the forward sends here (one 256-row tile of
                                    // the pair kernel, whose 297 splits on 74 pairs take five
                                    // rounds, the last with one unit; here nine on 33 clusters)
constexpr int kDecGemmMaxM = 224;   // largest M of the plain GEMM's short path (store mode)
constexpr int kDecSingleMaxN = 128; // largest N of the single form
constexpr int kDecPairMinN = 64;    // N from which the pair form is launched
constexpr int kDecCluster = 4;      // CTAs per vocab split
constexpr int kDecThreads = 192;
constexpr int kDecMaxStages = 12;
constexpr int kDecXStride = 33;     // floats per row of a warp's 32 x 32 transposition tile
constexpr int kDecYStride = 132;    // floats per batch row of the one-block tile (same memory)
static_assert(32 * kDecYStride == 4 * 32 * kDecXStride, "the one-block tile reuses the four tiles");
constexpr int kDecMaxBlocks = kDecMaxRows / 32;  // 32-row batch blocks of the widest N
constexpr uint32_t kDecHandBytes = 32u * 3u * 4u;  // a block's (m, s, b) hand-off: 32 rows
constexpr int kDecSplit = kDecCluster * kBM;
constexpr int kDecKPerStage = 2;   // K blocks per pipeline stage
constexpr uint32_t kDecABox = kBM * kBK * 2;                    // one 128 x 64 W box
constexpr uint32_t kDecABytes = kDecKPerStage * kDecABox;       // a stage's W boxes
constexpr int kDecHalfRows = kBM / 2;  // W rows per CTA of the half-height store form
constexpr int kDecHalfMaxN = 128;      // largest N of the half-height form
// full, empty per stage; tfull, tempty per accumulator; hfull per (hand
// buffer, block), hempty per hand buffer; pfull, pempty per warp link; xfull,
// xfree of the one-block epilogue; drain
constexpr int kDecNumBars = 2 * kDecMaxStages + 4 + 2 * kDecMaxBlocks + 2 + 6 + 2 + 1;
// floats of the epilogue's shared memory besides the hand buffers: four 32 x 33
// transposition tiles and three (m, s, b) x 32 links between the warps
constexpr uint32_t kDecEpiFloats = 4u * 32u * kDecXStride + 3u * 3u * 32u;

// Batch rows (and TMEM columns per accumulator) of each form.
template <bool kPair>
struct DecForm {
  static constexpr int kMaxRows = kPair ? kDecMaxRows : kDecSingleMaxN;
  static constexpr uint32_t kTmemCols = 2u * kMaxRows;  // two accumulators (a power of 2)
};

struct DecArgs {
  CUtensorMap w_k;    // W [V, H], K-major, box 64 x 128
  CUtensorMap hid_k;  // hidden [T, H], K-major, box 64 x N
  EpiFwd::Params ep;  // outputs and layout of the pair kernel's forward; for the
                      // plain GEMM (kStore) part_m = C, T = rows, V = columns,
                      // ldp = C's row stride, the rest unused
  uint32_t* err;
  int N;              // MMA N: 16 for T <= 16, else T rounded up to 32
                      // (the hidden box holds N rows, or N / 2 in the pair form)
  int KB;             // H / 64
  int NG;             // vocab splits of this W
  int stages;
  uint64_t wait_limit_ns;  // bound of every wait (kWaitLimitNs outside the test hook)
  int stall;          // test hook: CTA 0 of each cluster waits for a second arrival on its
                      // first accumulator's "full" barrier, which never comes
};

// Dynamic shared memory of the kernel for MMA width N and `stages` stages
// (`half`: the half-height store form, whose W boxes hold 64 rows).
__host__ __device__ constexpr uint32_t dec_smem_bytes(int N, int stages, bool pair, bool half = false) {
  return 1024u +
         static_cast<uint32_t>(stages) *
             ((half ? kDecABytes / 2u : kDecABytes) +
              static_cast<uint32_t>(pair ? N / 2 : N) * kBK * 2u * kDecKPerStage) +
         kDecEpiFloats * 4u + 2u * 3u * static_cast<uint32_t>(pair ? kDecMaxRows : kDecSingleMaxN) * 4u +
         kDecNumBars * 8u + 32u;
}

// The stage count the launcher takes for MMA width N: the most, at most
// kDecMaxStages, whose plan fits in `limit` bytes; 0 if two stages do not fit.
__host__ __device__ constexpr int dec_stages(int N, bool pair, uint32_t limit, bool half = false) {
  int S = kDecMaxStages;
  while (S >= 2 && dec_smem_bytes(N, S, pair, half) > limit) --S;
  return S >= 2 ? S : 0;
}

template <bool kPair, bool kStore = false, bool kHalf = false>
__global__ void __launch_bounds__(kDecThreads, 1) decode_fwd_kernel(const __grid_constant__ DecArgs P) {
  static_assert(!kHalf || (kStore && !kPair), "the half-height form is a single-CTA store form");
  constexpr int MR = DecForm<kPair>::kMaxRows;  // batch rows a hand buffer holds
  constexpr int RB = kHalf ? kDecHalfRows : kBM;                  // W rows per CTA tile
  constexpr uint32_t kABox = static_cast<uint32_t>(RB) * kBK * 2u;  // one RB x 64 W box
  constexpr uint32_t kABytes = kDecKPerStage * kABox;
  constexpr int kUnitRows = kDecCluster * RB;                     // W rows per unit
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const int N = P.N, S = P.stages;
  const bool async_hand = N > 128;  // the chain's hand-off by asynchronous stores (see hfull)
  const int NB = kPair ? N / 2 : N;                              // hidden rows this CTA holds
  const uint32_t b_box = static_cast<uint32_t>(NB) * kBK * 2u;   // one NB x 64 hidden box
  const uint32_t b_bytes = kDecKPerStage * b_box;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + S * kABytes;
  float* XT = reinterpret_cast<float*>(smem + S * (kABytes + b_bytes));  // [4][32][kDecXStride]
  float* pass = XT + 4 * 32 * kDecXStride;           // [3][3][32] (m, s, b) from warp c to c+1
  float* hand = pass + 3 * 3 * 32;                   // [2][3][MR] incoming (m, s, b)
  uint64_t* bars = reinterpret_cast<uint64_t*>(hand + 2 * 3 * MR);
  const uint32_t bar0 = smem_u32(bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kDecNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kDecMaxStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kDecMaxStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kDecMaxStages + 2 + a); };
  // hfull(h, blk): rows blk*32 .. +31 of this CTA's hand buffer h were written
  //                by CTA rank-1: up to N = 128 one arrival per lane of its
  //                sending warp (each after its stores, release at cluster
  //                scope); above, that warp's asynchronous stores complete the
  //                barrier, which this CTA's first-chunk warp arms for their
  //                kDecHandBytes (no release on the chain: 3-6% faster at N =
  //                192-224, 0.5-1% slower at N <= 96)
  // hempty(h): CTA rank+1 has read every row this CTA wrote into its buffer h
  //            (one arrival per lane of its first-chunk warp)
  auto hfull_bar = [&](int h, int blk) {
    return bar0 + 8u * (2 * kDecMaxStages + 4 + h * kDecMaxBlocks + blk);
  };
  auto hempty_bar = [&](int h) { return bar0 + 8u * (2 * kDecMaxStages + 4 + 2 * kDecMaxBlocks + h); };
  // pfull(c) / pempty(c): the link from the warp of chunk c to that of c+1
  constexpr int kPBar = 2 * kDecMaxStages + 6 + 2 * kDecMaxBlocks;
  auto pfull_bar = [&](int c) { return bar0 + 8u * (kPBar + c); };
  auto pempty_bar = [&](int c) { return bar0 + 8u * (kPBar + 3 + c); };
  // xfull: the four transposition tiles of a one-block unit are written;
  // xfree: warp 2 has read them
  const uint32_t xfull_bar = bar0 + 8u * (kPBar + 6);
  const uint32_t xfree_bar = bar0 + 8u * (kPBar + 7);
  const uint32_t drain_bar = bar0 + 8u * (kPBar + 8);

  const uint32_t rank = cluster_ctarank();
  // the pair form: CTA 2i issues the MMAs of the pair (2i, 2i+1) and owns its
  // full / accumulator-empty barriers; commits arrive in both CTAs
  const uint32_t lead = kPair ? (rank & ~1u) : rank;
  const bool is_lead = rank == lead;
  const uint16_t pair_mask = static_cast<uint16_t>(3u << lead);
  const long long cluster = blockIdx.x / kDecCluster;
  const long long nclusters = gridDim.x / kDecCluster;
  const long long total = P.NG;
  uint32_t* err = P.err;
  const uint64_t lim = P.wait_limit_ns;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecMaxStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), P.stall != 0 && a == 0 && rank == 0 ? 2 : 1);
      mbar_init(tempty_bar(a), kPair ? 8 : 4);  // one arrival per epilogue warp (of both CTAs)
      for (int blk = 0; blk < kDecMaxBlocks; ++blk) mbar_init(hfull_bar(a, blk), async_hand ? 1 : 32);
      mbar_init(hempty_bar(a), 32);
    }
    for (int c = 0; c < 3; ++c) {
      mbar_init(pfull_bar(c), 32);
      mbar_init(pempty_bar(c), 32);
    }
    mbar_init(xfull_bar, 128);
    mbar_init(xfree_bar, 32);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), DecForm<kPair>::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), DecForm<kPair>::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every CTA's barriers exist before a neighbour signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto unit_of = [&](uint32_t k) -> long long {
    const long long u = cluster + static_cast<long long>(k) * nclusters;
    return u < total ? u : -1;
  };

  uint32_t issued = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&P.w_k);
      tma_prefetch_desc(&P.hid_k);
      const int h0 = kPair ? static_cast<int>(rank & 1u) * NB : 0;  // first hidden row held here
      bool ok = true;
      // stage slot and phase kept incrementally, and each stage's addresses
      // worked out before the wait for its slot: the copies go out as soon as
      // the slot is free
      int s = 0;
      uint32_t ph = 0;
      for (uint32_t k = 0; ok; ++k) {
        const long long u = unit_of(k);
        if (u < 0) break;
        const int w0 = static_cast<int>(u) * kUnitRows + static_cast<int>(rank) * RB;
        const bool a_in = w0 < P.ep.V;  // a tile wholly past V is masked anyway: skip its loads
        // bytes one K block delivers to the full barrier (both CTAs' in the pair form;
        // the odd CTA's W tile starts kBM rows after the even one's)
        uint32_t kb_bytes = (a_in ? kABox : 0u) + b_box;
        if (kPair) kb_bytes += (w0 + kBM < P.ep.V ? kABox : 0u) + b_box;
        for (int kb = 0; kb < P.KB; kb += kDecKPerStage) {
          const int nk = min(kDecKPerStage, P.KB - kb);  // K blocks in this stage
          const uint32_t dA = sA + s * kABytes, dB = sB + s * b_bytes;
          const uint32_t fb = kPair ? mapa_shared(full_bar(s), lead) : full_bar(s);
          const uint32_t tx = nk * kb_bytes;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, err, lim)) {
            ok = false;
            break;
          }
          if constexpr (kPair) {
            if (is_lead) mbar_arrive_expect_tx(full_bar(s), tx);
            for (int i = 0; i < nk; ++i) {
              if (a_in) tma_load_2d_pair(dA + i * kABox, &P.w_k, fb, (kb + i) * kBK, w0);
              tma_load_2d_pair(dB + i * b_box, &P.hid_k, fb, (kb + i) * kBK, h0);
            }
          } else {
            mbar_arrive_expect_tx(fb, tx);
            for (int i = 0; i < nk; ++i) {
              if (a_in) tma_load_2d(dA + i * kABox, &P.w_k, fb, (kb + i) * kBK, w0);
              tma_load_2d(dB + i * b_box, &P.hid_k, fb, (kb + i) * kBK, 0);
            }
          }
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && is_lead) {
      const uint32_t idesc = idesc_bf16_f32(kPair ? 2 * kBM : RB, N, false, false);
      int s = 0;  // stage slot and phase, kept incrementally
      uint32_t ph = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        if (unit_of(k) < 0) break;
        const int acc = k & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), ((k >> 1) & 1u) ^ 1u, abort_flag, err, lim)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MR;
        for (int kb = 0; kb < P.KB; kb += kDecKPerStage) {
          const int nk = min(kDecKPerStage, P.KB - kb);
          if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, err, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sA + s * kABytes, b_s = sB + s * b_bytes;
          for (int i = 0; i < nk; ++i) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(a_s + i * kABox + kk * 32u, 16u, 1024u);
              const uint64_t bd = smem_desc_sw128(b_s + i * b_box + kk * 32u, 16u, 1024u);
              const uint32_t accum = ((kb + i) | kk) != 0 ? 1u : 0u;
              if constexpr (kPair) {
                umma_bf16_pair(d_tmem, ad, bd, idesc, accum);
              } else {
                umma_bf16(d_tmem, ad, bd, idesc, accum);
              }
            }
          }
          if constexpr (kPair) {
            umma_commit_pair_mask(empty_bar(s), pair_mask);
          } else {
            umma_commit(empty_bar(s));
          }
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) {
          if constexpr (kPair) {
            umma_commit_pair_mask(tfull_bar(acc), pair_mask);
          } else {
            umma_commit(tfull_bar(acc));
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp q (q = warp & 3) reads TMEM lanes 32q .. 32q+31 = W rows 32q .. +31
    // of the tile = chunk q of the split's four 32-column chunks in this CTA.
    // Batch rows flow through the four warps in 32-row blocks: warp q folds
    // chunk q of a block's rows into their running (m, s, b), which it takes
    // from warp q-1 (or, for q = 0, from CTA rank-1 / fresh) and hands to warp
    // q+1 (or, for q = 3, to CTA rank+1 / the split's partial), so every row
    // still folds its chunks in ascending column order while the four warps
    // (and the four CTAs) work on different blocks at once.
    const int q = warp & 3;
    float* xt = XT + q * 32 * kDecXStride;
    const int nblk = (N + 31) / 32;
    // waits of one lane, shared with the warp; then each lane acquires
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded_sleep(bar, parity, abort_flag, err, lim) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) mbar_try_wait(bar, parity);
      return ok != 0;
    };
    auto warp_wait_cluster = [&](uint32_t bar, uint32_t parity) -> bool {
      int ok = 0;
      if (lane == 0) ok = mbar_wait_cluster_bounded_sleep(bar, parity, abort_flag, err, lim) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) mbar_try_wait_cluster(bar, parity);
      return ok != 0;
    };
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    if constexpr (kStore) {
      // The plain GEMM (C[T, V] = hidden . W^T, fp32): lane l of warp q holds
      // output column n = tile row 32q + l for the accumulator's batch rows;
      // each row t is stored as one coalesced 128-byte run of the warp.  In
      // the half-height form lanes 0-15 of warp q hold tile rows 16q + l
      // (64-byte runs) and lanes 16-31 read lanes no MMA wrote, which are
      // not stored.
      float* C = P.ep.part_m;
      const bool lane_row = !kHalf || lane < 16;
      for (uint32_t k = 0; ok; ++k) {
        const long long u = unit_of(k);
        if (u < 0) break;
        const int acc = k & 1;
        if (!warp_wait(tfull_bar(acc), (k >> 1) & 1u)) break;
        tc_fence_after();
        const int n = static_cast<int>(u) * kUnitRows + static_cast<int>(rank) * RB +
                      (kHalf ? q * 16 : q * 32) + lane;
        for (int blk = 0; blk < nblk; ++blk) {
          uint32_t r[32];
          const int cols = N == 16 ? 16 : 32;
          if (N == 16) {
            uint32_t r16[16];
            tmem_ld16(tl + acc * MR, r16);
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = r16[j];
          } else {
            tmem_ld32(tl + acc * MR + blk * 32, r);
          }
          if (blk == nblk - 1) {  // the accumulator's last columns are read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (kPair) {
                mbar_arrive_cluster(mapa_shared(tempty_bar(acc), lead));
              } else {
                mbar_arrive(tempty_bar(acc));
              }
            }
          }
          if (lane_row && n < P.ep.V) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int t = blk * 32 + j;
              if (j < cols && t < P.ep.T)
                C[static_cast<size_t>(t) * P.ep.ldp + n] = __uint_as_float(r[j]);
            }
          }
        }
      }
    } else {
      uint32_t g = 0;  // blocks this warp has passed on (phase of its links)
      for (uint32_t k = 0; ok; ++k) {
        const long long u = unit_of(k);
        if (u < 0) break;
        const int acc = k & 1, h = k & 1;
        const uint32_t hph = (k >> 1) & 1u;
        if (!warp_wait(tfull_bar(acc), hph)) break;
        tc_fence_after();
        const int tile0 = static_cast<int>(u) * kDecSplit + static_cast<int>(rank) * kBM;
        const int col0 = tile0 + q * 32;
        if (nblk == 1) {
          // One 32-row block (N <= 32): every warp transposes its chunk, then
          // warp 2 folds all four in order.  Passing the rows from warp to warp
          // would overlap nothing here and only lengthen the chain of CTAs by
          // three hand-offs; and warp 2 is the epilogue warp that shares its
          // scheduler with neither the producer (warp 0) nor the MMA issuer
          // (warp 1), whose issue latency sets the W stream.
          // The accumulator is read once the running triples have arrived from
          // CTA rank-1: releasing it sooner lets the four CTAs of a split drift
          // apart in their W streams, which measured ~2% slower.  The tile is
          // row-major per batch row (Y[row][W row of the tile]), in the memory of
          // the four transposition tiles.
          const int t = lane;
          const int64_t tgt = t < P.ep.T ? P.ep.targets[t] - P.ep.v0 : -1;
          float* Y = XT;
          if (warp != 2 && k > 0 && !warp_wait(xfree_bar, (k - 1) & 1u)) break;
          if (rank > 0 && !warp_wait_cluster(hfull_bar(h, 0), hph)) break;
          const int v_loc = q * 32 + lane;
          if (N == 16) {
            uint32_t r[16];
            tmem_ld16(tl + acc * MR, r);
#pragma unroll
            for (int j = 0; j < 16; ++j) Y[j * kDecYStride + v_loc] = __uint_as_float(r[j]);
          } else {
            uint32_t r[32];
            tmem_ld32(tl + acc * MR, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) Y[j * kDecYStride + v_loc] = __uint_as_float(r[j]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (kPair) {
              mbar_arrive_cluster(mapa_shared(tempty_bar(acc), lead));
            } else {
              mbar_arrive(tempty_bar(acc));
            }
          }
          mbar_arrive(xfull_bar);
          if (warp != 2) continue;
          if (!warp_wait(xfull_bar, k & 1u)) break;
          float m = kMaskLogit, s = 0.f, b = 0.f;
          if (rank > 0) {  // hfull(h, 0) has completed (waited above)
            const float* in = hand + h * 3 * MR;
            m = in[t];
            s = in[MR + t];
            b = in[2 * MR + t];
            mbar_arrive_cluster(mapa_shared(hempty_bar(h), rank - 1));
          }
          const float4* row = reinterpret_cast<const float4*>(Y + lane * kDecYStride);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float y[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 f = row[c * 8 + i];
              y[4 * i + 0] = fwd_scale(f.x, P.ep.scale_log2);
              y[4 * i + 1] = fwd_scale(f.y, P.ep.scale_log2);
              y[4 * i + 2] = fwd_scale(f.z, P.ep.scale_log2);
              y[4 * i + 3] = fwd_scale(f.w, P.ep.scale_log2);
            }
            if (t < P.ep.T) fwd_chunk_update(y, tile0 + c * 32, P.ep.V, tgt, P.ep.ytgt + t, m, s, b);
          }
          mbar_arrive(xfree_bar);
          if (rank + 1 < kDecCluster) {
            if (!warp_wait(hempty_bar(h), hph ^ 1u)) break;
            const uint32_t dst = mapa_shared(smem_u32(hand + h * 3 * MR), rank + 1);
            st_shared_cluster_u32(dst + 4u * t, __float_as_uint(m));
            st_shared_cluster_u32(dst + 4u * (MR + t), __float_as_uint(s));
            st_shared_cluster_u32(dst + 4u * (2 * MR + t), __float_as_uint(b));
            mbar_arrive_cluster(mapa_shared(hfull_bar(h, 0), rank + 1));
          } else if (t < P.ep.T) {
            const size_t i = static_cast<size_t>(t) * P.ep.ldp + static_cast<size_t>(u);
            P.ep.part_m[i] = m;
            P.ep.part_s[i] = s;
            P.ep.part_b[i] = b;
          }
          continue;
        }
        for (int blk = 0; blk < nblk; ++blk, ++g) {
          const int t = blk * 32 + lane;
          const int64_t tgt = t < P.ep.T ? P.ep.targets[t] - P.ep.v0 : -1;  // issued early
          // 1. this block's 32 columns of the accumulator, transposed through the
          //    warp's tile: lane l ends with batch row blk*32+l over the chunk
          if (N == 16) {
            uint32_t r[16];
            tmem_ld16(tl + acc * MR, r);
#pragma unroll
            for (int j = 0; j < 16; ++j) xt[lane * kDecXStride + j] = __uint_as_float(r[j]);
          } else {
            uint32_t r[32];
            tmem_ld32(tl + acc * MR + blk * 32, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) xt[lane * kDecXStride + j] = __uint_as_float(r[j]);
          }
          if (blk == nblk - 1) {  // the accumulator's last columns are read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (kPair) {
                mbar_arrive_cluster(mapa_shared(tempty_bar(acc), lead));
              } else {
                mbar_arrive(tempty_bar(acc));
              }
            }
          }
          __syncwarp();
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = fwd_scale(xt[i * kDecXStride + lane], P.ep.scale_log2);
          __syncwarp();  // the tile is free for the next block
          // 2. the rows' running triples
          float m = kMaskLogit, s = 0.f, b = 0.f;
          if (q == 0) {
            if (rank > 0) {
              if (async_hand && lane == 0) mbar_arrive_expect_tx(hfull_bar(h, blk), kDecHandBytes);
              if (!warp_wait_cluster(hfull_bar(h, blk), hph)) {
                ok = false;
                break;
              }
              const float* in = hand + h * 3 * MR;
              m = in[t];
              s = in[MR + t];
              b = in[2 * MR + t];
              if (blk == nblk - 1) mbar_arrive_cluster(mapa_shared(hempty_bar(h), rank - 1));
            }
          } else {
            if (!warp_wait(pfull_bar(q - 1), g & 1u)) {
              ok = false;
              break;
            }
            const float* in = pass + (q - 1) * 96;
            m = in[lane];
            s = in[32 + lane];
            b = in[64 + lane];
            mbar_arrive(pempty_bar(q - 1));
          }
          // 3. fold this chunk
          if (t < P.ep.T)
            fwd_chunk_update(y, col0, P.ep.V, tgt, P.ep.ytgt + t, m, s, b);
          // 4. pass the triples on
          if (q < 3) {
            if (!warp_wait(pempty_bar(q), (g & 1u) ^ 1u)) {
              ok = false;
              break;
            }
            float* out = pass + q * 96;
            out[lane] = m;
            out[32 + lane] = s;
            out[64 + lane] = b;
            mbar_arrive(pfull_bar(q));
          } else if (rank + 1 < kDecCluster) {
            if (blk == 0 && !warp_wait(hempty_bar(h), hph ^ 1u)) {
              ok = false;
              break;
            }
            const uint32_t dst = mapa_shared(smem_u32(hand + h * 3 * MR), rank + 1);
            const uint32_t bar = mapa_shared(hfull_bar(h, blk), rank + 1);
            if (async_hand) {
              st_async_cluster_u32(dst + 4u * t, __float_as_uint(m), bar);
              st_async_cluster_u32(dst + 4u * (MR + t), __float_as_uint(s), bar);
              st_async_cluster_u32(dst + 4u * (2 * MR + t), __float_as_uint(b), bar);
            } else {
              st_shared_cluster_u32(dst + 4u * t, __float_as_uint(m));
              st_shared_cluster_u32(dst + 4u * (MR + t), __float_as_uint(s));
              st_shared_cluster_u32(dst + 4u * (2 * MR + t), __float_as_uint(b));
              mbar_arrive_cluster(bar);
            }
          } else if (t < P.ep.T) {
            const size_t i = static_cast<size_t>(t) * P.ep.ldp + static_cast<size_t>(u);
            P.ep.part_m[i] = m;
            P.ep.part_s[i] = s;
            P.ep.part_b[i] = b;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Unwind after a timed-out wait: let TMA loads and MMAs in flight finish
    // before the shared memory and TMEM they touch go away.
    if (warp == 0 && lane == 0 && is_lead) {
      const uint32_t first = issued > static_cast<uint32_t>(S) ? issued - S : 0u;
      for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(full_bar(i % S), (i / S) & 1u);
    }
    if (warp == 1 && lane == 0 && is_lead) {
      if constexpr (kPair) {
        umma_commit_pair_mask(drain_bar, pair_mask);
      } else {
        umma_commit(drain_bar);
      }
      mbar_wait_drain(drain_bar, 0);
    }
    if constexpr (kPair) {
      // the odd CTA's copies signal the even CTA's barriers: give them time to land
      const uint64_t t_start = globaltimer_ns();
      while (globaltimer_ns() - t_start < 2000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  cluster_sync();  // no CTA exits while a neighbour may still write its shared memory
  tc_fence_after();
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_dealloc_pair(tmem_base, DecForm<kPair>::kTmemCols);
    } else {
      tmem_dealloc(tmem_base, DecForm<kPair>::kTmemCols);
    }
  }
}

}  // namespace rlk
