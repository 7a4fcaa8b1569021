// rlk_decode.cuh -- forward for short batches (rollout / decode shapes, T <= 128
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
// Numerics are those of the pair kernel, bit for bit:
//  * each logit is the same bf16 dot product over H in the same 64-wide K
//    blocks and 16-wide MMA steps (D = A . B^T gives the same fp32 element
//    with A and B exchanged: each element is its own product sum);
//  * a vocab split is 512 columns = four 128-row W tiles, one per CTA of a
//    cluster of four.  CTA r runs the split's chunks r*4 .. r*4+3 with
//    fwd_chunk_update after receiving the running (m, s, b) of every row from
//    CTA r-1 through distributed shared memory, so the chunks of a split are
//    folded in the same ascending order by the same code as in the pair
//    kernel;
//  * CTA 3 writes the split's triple where the pair kernel's forward writes
//    it, and the same combine kernel merges the splits.
//
// Warp roles per CTA (192 threads): warp 0 producer (TMA), warp 1 MMA issuer,
// warps 2-5 epilogue.  Two TMEM accumulators of up to 128 columns; the
// epilogue copies an accumulator to shared memory transposed (row-major per
// batch row), 32 rows at a time, and frees it after the last block.
#pragma once

#include "rlk_gemm.cuh"

namespace rlk {

constexpr int kDecMaxRows = 128;    // largest T this path takes
constexpr int kDecCluster = 4;      // CTAs per vocab split
constexpr int kDecThreads = 192;
constexpr int kDecMaxStages = 12;
constexpr int kDecYStride = 132;    // floats per batch row of the transposed tile
constexpr int kDecTmemCols = 256;   // two accumulators of up to 128 columns
constexpr int kDecSplit = kDecCluster * kBM;
constexpr int kDecKPerStage = 2;   // K blocks per pipeline stage
constexpr uint32_t kDecABox = kBM * kBK * 2;                    // one 128 x 64 W box
constexpr uint32_t kDecABytes = kDecKPerStage * kDecABox;       // a stage's W boxes
constexpr int kDecNumBars = 2 * kDecMaxStages + 9;

struct DecArgs {
  CUtensorMap w_k;    // W [V, H], K-major, box 64 x 128
  CUtensorMap hid_k;  // hidden [T, H], K-major, box 64 x N
  EpiFwd::Params ep;  // outputs and layout of the pair kernel's forward
  uint32_t* err;
  int N;              // MMA N: 16 for T <= 16, else T rounded up to 32
  int KB;             // H / 64
  int NG;             // vocab splits of this W
  int stages;
};

// Dynamic shared memory of the kernel for MMA width N and `stages` stages.
__host__ __device__ constexpr uint32_t dec_smem_bytes(int N, int stages) {
  return 1024u + static_cast<uint32_t>(stages) * (kDecABytes + N * kBK * 2u * kDecKPerStage) +
         32u * kDecYStride * 4u + 2u * 3u * kDecMaxRows * 4u +
         kDecNumBars * 8u + 32u;
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_fwd_kernel(const __grid_constant__ DecArgs P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const int N = P.N, S = P.stages;
  const uint32_t b_box = static_cast<uint32_t>(N) * kBK * 2u;   // one N x 64 hidden box
  const uint32_t b_bytes = kDecKPerStage * b_box;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + S * kDecABytes;
  float* Y = reinterpret_cast<float*>(smem + S * (kDecABytes + b_bytes));  // [32][kDecYStride]
  float* hand = Y + 32 * kDecYStride;                // [2][3][kDecMaxRows] incoming (m, s, b)
  uint64_t* bars = reinterpret_cast<uint64_t*>(hand + 2 * 3 * kDecMaxRows);
  const uint32_t bar0 = smem_u32(bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kDecNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ok1 = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* ok3 = reinterpret_cast<volatile int*>(tmem_slot + 4);

  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kDecMaxStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kDecMaxStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kDecMaxStages + 2 + a); };
  // hfull(h): this CTA's hand buffer h was written by CTA rank-1 (128 arrivals)
  // hempty(h): CTA rank+1 has read what this CTA wrote into its buffer h
  auto hfull_bar = [&](int h) { return bar0 + 8u * (2 * kDecMaxStages + 4 + h); };
  auto hempty_bar = [&](int h) { return bar0 + 8u * (2 * kDecMaxStages + 6 + h); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kDecMaxStages + 8);

  const uint32_t rank = cluster_ctarank();
  const long long cluster = blockIdx.x / kDecCluster;
  const long long nclusters = gridDim.x / kDecCluster;
  const long long total = P.NG;
  uint32_t* err = P.err;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecMaxStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);  // one arrival per epilogue warp
      mbar_init(hfull_bar(a), kDecMaxRows);
      mbar_init(hempty_bar(a), kDecMaxRows);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kDecTmemCols);
    tmem_relinquish();
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
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const long long u = unit_of(k);
        if (u < 0) break;
        const int w0 = static_cast<int>(u) * kDecSplit + static_cast<int>(rank) * kBM;
        const bool a_in = w0 < P.ep.V;  // a tile wholly past V is masked anyway: skip its loads
        for (int kb = 0; kb < P.KB; kb += kDecKPerStage) {
          const int nk = min(kDecKPerStage, P.KB - kb);  // K blocks in this stage
          const int s = issued % S;
          const uint32_t ph = (issued / S) & 1u;
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), nk * ((a_in ? kDecABox : 0u) + b_box));
          for (int i = 0; i < nk; ++i) {
            if (a_in)
              tma_load_2d(sA + s * kDecABytes + i * kDecABox, &P.w_k, full_bar(s),
                          (kb + i) * kBK, w0);
            tma_load_2d(sB + s * b_bytes + i * b_box, &P.hid_k, full_bar(s), (kb + i) * kBK, 0);
          }
          ++issued;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, N, false, false);
      uint32_t it = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        if (unit_of(k) < 0) break;
        const int acc = k & 1;
        if (!mbar_wait_bounded(tempty_bar(acc), ((k >> 1) & 1u) ^ 1u, abort_flag, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kDecMaxRows;
        for (int kb = 0; kb < P.KB; kb += kDecKPerStage, ++it) {
          const int nk = min(kDecKPerStage, P.KB - kb);
          const int s = it % S;
          if (!mbar_wait_bounded(full_bar(s), (it / S) & 1u, abort_flag, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = sA + s * kDecABytes, b_s = sB + s * b_bytes;
          for (int i = 0; i < nk; ++i) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(a_s + i * kDecABox + kk * 32u, 16u, 1024u);
              const uint64_t bd = smem_desc_sw128(b_s + i * b_box + kk * 32u, 16u, 1024u);
              umma_bf16(d_tmem, ad, bd, idesc, ((kb + i) | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(empty_bar(s));
        }
        if (ok) umma_commit(tfull_bar(acc));
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int v_loc = q * 32 + lane;     // W row of the tile held in this thread's lane
    const int t = (warp - 2) * 32 + lane;  // batch row whose chain this thread runs
    const bool tvalid = t < P.ep.T;
    const int64_t tgt = tvalid ? P.ep.targets[t] - P.ep.v0 : -1;
    const bool ep_leader = threadIdx.x == 64;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    for (uint32_t k = 0;; ++k) {
      const long long u = unit_of(k);
      if (u < 0) break;
      const int acc = k & 1, h = k & 1;
      const uint32_t hph = (k >> 1) & 1u;
      // 1. the accumulator, and the running triple from CTA rank-1 (or a fresh one)
      if (ep_leader) {
        bool ok = mbar_wait_bounded(tfull_bar(acc), hph, abort_flag, err);
        if (ok && rank > 0) ok = mbar_wait_cluster_bounded(hfull_bar(h), hph, abort_flag, err);
        *ok1 = ok ? 1 : 0;
      }
      epilogue_bar();
      if (!*ok1) break;
      tc_fence_after();
      float m = kMaskLogit, s = 0.f, b = 0.f;
      if (rank > 0) {
        mbar_try_wait_cluster(hfull_bar(h), hph);  // completed: acquire for this thread
        const float* in = hand + h * 3 * kDecMaxRows;
        m = in[t];
        s = in[kDecMaxRows + t];
        b = in[2 * kDecMaxRows + t];
        mbar_arrive_cluster(mapa_shared(hempty_bar(h), rank - 1));
      }
      // 2. 32 batch rows at a time: their accumulator columns go to Y transposed
      //    (all four warps, one TMEM lane quarter each), then the warp that owns
      //    those rows folds the tile's four chunks in column order; the
      //    accumulator is freed after its last columns are read
      const int col_base = static_cast<int>(u) * kDecSplit + static_cast<int>(rank) * kBM;
      const int nblk = (N + 31) / 32;
      for (int blk = 0; blk < nblk; ++blk) {
        if (N == 16) {
          uint32_t r[16];
          tmem_ld16(tl + acc * kDecMaxRows, r);
#pragma unroll
          for (int j = 0; j < 16; ++j) Y[j * kDecYStride + v_loc] = __uint_as_float(r[j]);
        } else {
          uint32_t r[32];
          tmem_ld32(tl + acc * kDecMaxRows + blk * 32, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) Y[j * kDecYStride + v_loc] = __uint_as_float(r[j]);
        }
        if (blk == nblk - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        epilogue_bar();  // Y holds batch rows blk*32 .. +31
        if (warp - 2 == blk && tvalid) {
          const float4* row = reinterpret_cast<const float4*>(Y + lane * kDecYStride);
#pragma unroll 1
          for (int c = 0; c < kBM / 32; ++c) {
            float y[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 f = row[c * 8 + i];
              y[4 * i + 0] = fwd_scale(f.x, P.ep.scale_log2);
              y[4 * i + 1] = fwd_scale(f.y, P.ep.scale_log2);
              y[4 * i + 2] = fwd_scale(f.z, P.ep.scale_log2);
              y[4 * i + 3] = fwd_scale(f.w, P.ep.scale_log2);
            }
            fwd_chunk_update(y, col_base + c * 32, P.ep.V, tgt, P.ep.ytgt + t, m, s, b);
          }
        }
        epilogue_bar();  // Y read: free for the next block
      }
      // 4. hand the triple on, or store the split's triple
      if (rank + 1 < kDecCluster) {
        if (ep_leader) *ok3 = mbar_wait_bounded(hempty_bar(h), hph ^ 1u, abort_flag, err) ? 1 : 0;
        epilogue_bar();
        if (!*ok3) break;
        const uint32_t dst = mapa_shared(smem_u32(hand + h * 3 * kDecMaxRows), rank + 1);
        st_shared_cluster_u32(dst + 4u * t, __float_as_uint(m));
        st_shared_cluster_u32(dst + 4u * (kDecMaxRows + t), __float_as_uint(s));
        st_shared_cluster_u32(dst + 4u * (2 * kDecMaxRows + t), __float_as_uint(b));
        mbar_arrive_cluster(mapa_shared(hfull_bar(h), rank + 1));
      } else if (tvalid) {
        const size_t i = static_cast<size_t>(t) * P.ep.ldp + static_cast<size_t>(u);
        P.ep.part_m[i] = m;
        P.ep.part_s[i] = s;
        P.ep.part_b[i] = b;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Unwind after a timed-out wait: let TMA loads and MMAs in flight finish
    // before the shared memory and TMEM they touch go away.
    if (warp == 0 && lane == 0) {
      const uint32_t first = issued > static_cast<uint32_t>(S) ? issued - S : 0u;
      for (uint32_t i = first; i < issued; ++i) mbar_wait_drain(full_bar(i % S), (i / S) & 1u);
    }
    if (warp == 1 && lane == 0) {
      umma_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
    __syncthreads();
  }
  cluster_sync();  // no CTA exits while a neighbour may still write its shared memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kDecTmemCols);
}

}  // namespace rlk
