// Host-only check of the short-batch forward kernel's shared-memory plan
// (rlk_decode.cuh), run by tests/test_decode_config.py on the CPU.  For every
// MMA width N and form the launcher takes (single-CTA: 16 and 32 .. up to the
// pair threshold; CTA pair: the threshold .. 256 in steps of 32; the
// half-height store form: 16 .. 128 in steps of 16, 64 W rows per box) it takes the
// stage count the launcher takes (dec_stages) and checks that the plan fits,
// that every stage's W and hidden boxes start on a 1024-byte boundary
// (128-byte swizzle atoms), that the barriers are 8-byte aligned, that every
// barrier the epilogue indexes (one per hand buffer and 32-row block) exists, that two stages at
// least remain, that a pair CTA's hidden rows (N / 2) fill whole 8-row
// swizzle groups, and that each form's two accumulators fit its TMEM
// allocation.  Prints one line per width and "OK", or the first violation.
#include <cstdio>

#include "rlk_decode.cuh"

using namespace rlk;

static int check(int N, bool pair, bool half = false) {
  const unsigned limit = 227u * 1024u;
  const int S = dec_stages(N, pair, limit, half);
  if (S < 2) { printf("N=%d: fewer than two stages\n", N); return 1; }
  const unsigned smem = dec_smem_bytes(N, S, pair, half);
  const unsigned a_box = (half ? kDecHalfRows : kBM) * kBK * 2, a_bytes = kDecKPerStage * a_box;
  const int NB = pair ? N / 2 : N;
  const int MR = pair ? DecForm<true>::kMaxRows : DecForm<false>::kMaxRows;
  const unsigned cols = pair ? DecForm<true>::kTmemCols : DecForm<false>::kTmemCols;
  const unsigned b_box = NB * kBK * 2, b_bytes = kDecKPerStage * b_box;
  const unsigned sB = S * a_bytes;
  const unsigned xt = S * (a_bytes + b_bytes);
  const unsigned hand = xt + kDecEpiFloats * 4u;
  const unsigned bars = hand + 2u * 3u * MR * 4u;
  if (smem > limit) { printf("N=%d: %u bytes of shared memory\n", N, smem); return 1; }
  if (half && (N > kDecHalfMaxN || N % 16)) { printf("N=%d: not a half-height width\n", N); return 1; }
  if (a_box % 1024 || a_bytes % 1024 || sB % 1024 || b_box % 1024 || b_bytes % 1024) {
    printf("N=%d: a box is off the 1024-byte grid\n", N);
    return 1;
  }
  if (NB % 8) { printf("N=%d: %d hidden rows per CTA\n", N, NB); return 1; }
  if (N > MR || 2u * MR > cols || (cols & (cols - 1)) || cols < 32 || cols > 512) {
    printf("N=%d: accumulators do not fit %u TMEM columns\n", N, cols);
    return 1;
  }
  if ((N + 31) / 32 > kDecMaxBlocks || MR / 32 > kDecMaxBlocks) {
    printf("N=%d: more 32-row blocks than hand-off barriers\n", N);
    return 1;
  }
  if (bars % 8) { printf("N=%d: barriers misaligned\n", N); return 1; }
  // the dynamic allocation holds the 1024-byte alignment slack, the plan,
  // the barriers and the words after them
  if (1024u + bars + kDecNumBars * 8u + 2u * 4u > smem) {
    printf("N=%d: plan overruns its allocation\n", N);
    return 1;
  }
  printf("%s N=%d stages=%d smem=%u\n", half ? "half" : pair ? "pair" : "single", N, S, smem);
  return 0;
}

int main() {
  if (check(16, false)) return 1;
  for (int N = 32; N <= kDecMaxRows; N += 32)
    if (check(N, N >= kDecPairMinN)) return 1;
  // the single form up to its own limit, for a launcher with a higher threshold
  for (int N = 32; N <= kDecSingleMaxN; N += 32)
    if (check(N, false)) return 1;
  for (int N = 16; N <= kDecHalfMaxN; N += 16)
    if (check(N, false, true)) return 1;
  printf("OK\n");
  return 0;
}
