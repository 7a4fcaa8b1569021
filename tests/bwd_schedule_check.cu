// Host-only check of the fused backward's unit schedule (rlk_bwd.cuh), run
// by tests/test_bwd_schedule.py on the CPU: every unit appears exactly once,
// every dependency is an earlier unit (so CTAs that walk their units in
// ascending order never wait on a later one), and every tile stays inside the
// buffers it touches.  Prints "OK <units>" or the first violation.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <tuple>

#include "rlk_bwd.cuh"

using namespace rlk;

int main(int argc, char** argv) {
  if (argc != 5) return 2;
  const long long T = atoll(argv[1]), H = atoll(argv[2]), V = atoll(argv[3]), ldx = atoll(argv[4]);
  const BwdPlan P = make_bwd_plan(T, H, V, ldx);
  std::map<std::tuple<int, int, int, int>, long long> index;
  for (long long u = 0; u < P.total; ++u) {
    const BwdUnit x = bwd_decode(P, u);
    if (x.type < 0 || x.c < 0 || x.c >= P.NC) { printf("BAD decode at %lld\n", u); return 1; }
    auto key = std::make_tuple(x.type, x.c, x.a, x.b);
    if (index.count(key)) { printf("DUP unit at %lld\n", u); return 1; }
    index[key] = u;
  }
  // every unit of every kind is present
  long long expect = 0;
  for (int c = 0; c < P.NC; ++c) expect += bwd_nR(P, c) + bwd_nH(P) + bwd_nD(P, c);
  if (expect != P.total || (long long)index.size() != P.total) {
    printf("COUNT %lld vs %lld\n", expect, P.total);
    return 1;
  }
  auto at = [&](int t, int c, int a, int b) -> long long {
    auto it = index.find(std::make_tuple(t, c, a, b));
    return it == index.end() ? -1 : it->second;
  };
  for (auto& kv : index) {
    const int t = std::get<0>(kv.first), c = std::get<1>(kv.first);
    const int a = std::get<2>(kv.first), b = std::get<3>(kv.first);
    const long long u = kv.second;
    const int valid = bwd_chunk_valid(P, c);
    if (t == kUnitR) {
      if (a >= P.MT || b >= bwd_rt(P, c)) { printf("R range\n"); return 1; }
      if ((long long)c * P.ldx + b * kBN >= V) { printf("R tile past V\n"); return 1; }
      if (b * kBN + kBN > P.ldx) { printf("R store past chunk buffer\n"); return 1; }
      if (c >= kDxBuffers) {
        const int c3 = c - kDxBuffers;
        for (int m = 0; m < P.MT; ++m)
          for (int n = 0; n < P.NH; ++n)
            if (at(kUnitH, c3, m, n) >= u) { printf("R waits on later H\n"); return 1; }
        for (int v = 0; v < (c3 == P.NC - 1 ? P.VT_last : P.VT_full); ++v)
          for (int n = 0; n < P.NH; ++n)
            if (at(kUnitD, c3, v, n) >= u) { printf("R waits on later D\n"); return 1; }
      }
    } else if (t == kUnitH) {
      if (a >= P.MT || b >= P.NH) { printf("H range\n"); return 1; }
      const int kbs = (valid + kBK - 1) / kBK;
      if (kbs * kBK > bwd_rt(P, c) * kBN) { printf("H reads unwritten dX columns\n"); return 1; }
      for (int j = 0; j < bwd_rt(P, c); ++j) {
        const long long d = at(kUnitR, c, a, j);
        if (d < 0 || d >= u) { printf("H dep on R not earlier\n"); return 1; }
      }
      if (c >= 1) {
        const long long d = at(kUnitH, c - 1, a, b);
        if (d < 0 || d >= u) { printf("H dep on previous chunk not earlier\n"); return 1; }
      }
    } else {
      const int vt = c == P.NC - 1 ? P.VT_last : P.VT_full;
      if (a >= vt || b >= P.NH) { printf("D range\n"); return 1; }
      if ((long long)c * P.ldx + a * kPairM >= V) { printf("D tile past V\n"); return 1; }
      if (a * kPairM + kPairM > bwd_rt(P, c) * kBN) { printf("D reads unwritten dX columns\n"); return 1; }
      for (int m = 0; m < P.MT; ++m) {
        const long long d = at(kUnitR, c, m, a);
        if (d < 0 || d >= u) { printf("D dep on R not earlier\n"); return 1; }
      }
    }
  }
  printf("OK %lld\n", P.total);
  return 0;
}
