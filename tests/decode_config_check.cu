// Host-only check of the short-batch forward kernel's shared-memory plan
// (rlk_decode.cuh), run by tests/test_decode_config.py on the CPU.  For every
// MMA width N the kernel takes (16, and 32..128 in steps of 32) it picks the
// stage count the launcher picks (the most stages, at most kDecMaxStages and
// at least 2, whose dec_smem_bytes fits in 227 KB) and checks that the plan
// fits, that every stage's W and hidden boxes start on a 1024-byte boundary
// (128-byte swizzle atoms), that the transposed rows are 16-byte aligned for
// float4 reads, that the barriers are 8-byte aligned, and that two stages at
// least remain.  Prints "OK" or the first violation.
#include <cstdio>

#include "rlk_decode.cuh"

using namespace rlk;

int main() {
  const unsigned limit = 227u * 1024u;
  const int widths[] = {16, 32, 64, 96, 128};
  for (int N : widths) {
    int S = kDecMaxStages;
    while (S > 2 && dec_smem_bytes(N, S) > limit) --S;  // as the launcher does
    const unsigned smem = dec_smem_bytes(N, S);
    const unsigned b_box = N * kBK * 2, b_bytes = kDecKPerStage * b_box;
    const unsigned sB = S * kDecABytes;
    const unsigned y = S * (kDecABytes + b_bytes);
    const unsigned hand = y + 32u * kDecYStride * 4u;
    const unsigned bars = hand + 2u * 3u * kDecMaxRows * 4u;
    if (S < 2) { printf("N=%d: fewer than two stages\n", N); return 1; }
    if (smem > limit) { printf("N=%d: %u bytes of shared memory\n", N, smem); return 1; }
    if (kDecABox % 1024 || kDecABytes % 1024 || sB % 1024 || b_box % 1024 || b_bytes % 1024) {
      printf("N=%d: a box is off the 1024-byte grid\n", N);
      return 1;
    }
    if (y % 16 || (kDecYStride * 4) % 16) { printf("N=%d: transposed rows misaligned\n", N); return 1; }
    if (bars % 8) { printf("N=%d: barriers misaligned\n", N); return 1; }
    // the dynamic allocation holds the 1024-byte alignment slack, the plan,
    // the barriers and the words after them
    if (1024u + bars + kDecNumBars * 8u + 5u * 4u > smem) {
      printf("N=%d: plan overruns its allocation\n", N);
      return 1;
    }
    printf("N=%d stages=%d smem=%u\n", N, S, smem);
  }
  printf("OK\n");
  return 0;
}
