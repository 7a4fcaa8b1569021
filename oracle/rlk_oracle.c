/*
 * rlk_oracle.c -- plain, slow fp64 CPU oracle for the linear-logp operator.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
 * benchmark's CPU-baseline leg are the only users.  The CUDA library and its
 * Python binding never load, call or link this file, and it shares no code,
 * header or constant with them.
 *
 * What it computes.  The RL-Kernel pages name a bitwise linear-logp route
 * ("rlkernel.linear_logp.bitwise.v1", h100-cp-gradient.json,
 * runs[].validation.runtime_readbacks.frameworks.*.modules.logp) that
 * replaces VIME's native calculate_log_probs_and_entropy (VIME Qwen3-8B
 * TP4/CP2 dense page, "User-facing operator matrix"), under "GRPO, BF16,
 * temperature 1" (same page, "Required gates").  The pages print no formula.
 * The plain reading of that name and of the route's outputs, for every row t
 * over the full vocabulary, is:
 *
 *   (1) x[t,v] = sum_h hidden[t,h] * W[v,h]      (bf16 inputs widened exactly)
 *   (2) z[t,v] = x[t,v] / tau
 *   (3) m = max_v z, s = sum_v exp(z - m), lse = m + log(s)
 *   (4) p = exp(z - lse); logp = z[target] - lse; entropy = lse - sum_v p z
 *   (5) dz = dlogp (1[v = target] - p) - dentropy p (z - sum_u p_u z_u);
 *       dx = dz / tau
 *   (6) dHidden[t,h] = sum_v dx[t,v] W[v,h];  dW[v,h] = sum_t dx[t,v] hidden[t,h]
 *
 * (5) is d/dz of  dlogp*logp + dentropy*entropy  (d logp/dz = onehot - p and
 * d entropy/dz_j = -p_j (z_j - E_p z)).  Everything is fp64, summed in
 * ascending index order, with a two-pass (max first) softmax.  Every product
 * of two bf16 values is exact in fp64.
 *
 * A mutation selector (rlk_oracle_set_mutation) plants one known mistake at a
 * time; the test suite uses it to show that its pins catch such mistakes.  It
 * is 0 (no mutation) unless a test sets it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum {
  MUT_NONE = 0,
  MUT_NO_TEMPERATURE = 1,   /* (2) drops the division by tau             */
  MUT_ENTROPY_SIGN = 2,     /* (4) entropy = sum p z - lse               */
  MUT_TARGET_SHIFT = 3,     /* (4),(5) reads target + 1                  */
  MUT_LSE_NO_MAX = 4,       /* (3) forgets to add m back                 */
  MUT_DX_NO_ENTROPY = 5,    /* (5) drops the entropy term                */
  MUT_DX_ONEHOT_SIGN = 6,   /* (5) p - onehot instead of onehot - p      */
  MUT_DW_ROW_INDEX = 7,     /* (6) dW pairs dx row t with hidden row t+1 */
  MUT_DX_NO_TAU = 8,        /* (5) forgets the final / tau               */
  MUT_EZ_IS_MAX = 9,        /* (5) uses max z in place of E_p z          */
  MUT_DOT_SKIP_LAST = 10,   /* (1) sums h over [0, H-1) only             */
  MUT_DH_TRANSPOSED = 11,   /* (6) dHidden reads W[h,v] (square V == H)  */
  MUT_COUNT = 12
};

static int g_mutation = MUT_NONE;

int rlk_oracle_set_mutation(int m) {
  if (m < 0 || m >= MUT_COUNT) return -1;
  g_mutation = m;
  return 0;
}

int rlk_oracle_num_mutations(void) { return MUT_COUNT; }

int rlk_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static void widen(const uint16_t* src, double* dst, int64_t n) {
  for (int64_t i = 0; i < n; ++i) dst[i] = bf16_to_f64(src[i]);
}

static int check_targets(const int64_t* targets, int64_t T, int64_t V) {
  for (int64_t t = 0; t < T; ++t)
    if (targets[t] < 0 || targets[t] >= V) return -2;
  return 0;
}

static int64_t target_of(const int64_t* targets, int64_t t, int64_t V) {
  int64_t k = targets[t];
  if (g_mutation == MUT_TARGET_SHIFT) k = (k + 1) % V;
  return k;
}

/* Steps (1)-(2): z[T,V] = (hidden[T,H] . W[V,H]^T) / tau.  Four rows share
 * each widened W row; every dot product is summed in ascending h. */
int rlk_oracle_logits(const uint16_t* hidden, const uint16_t* W, int64_t T, int64_t H,
                      int64_t V, double tau, double* z) {
  if (T < 0 || H <= 0 || V <= 0 || !(tau > 0.0)) return -1;
  if (T == 0) return 0;
  double* hd = (double*)malloc((size_t)(T * H) * sizeof(double));
  if (!hd) return -3;
  widen(hidden, hd, T * H);
  const double div = (g_mutation == MUT_NO_TEMPERATURE) ? 1.0 : tau;
  const int64_t hn = (g_mutation == MUT_DOT_SKIP_LAST) ? H - 1 : H;
#pragma omp parallel
  {
    double* w = (double*)malloc((size_t)H * sizeof(double));
#pragma omp for schedule(dynamic, 8)
    for (int64_t v = 0; v < V; ++v) {
      widen(W + v * H, w, H);
      int64_t t = 0;
      for (; t + 4 <= T; t += 4) {
        const double* a0 = hd + (t + 0) * H;
        const double* a1 = hd + (t + 1) * H;
        const double* a2 = hd + (t + 2) * H;
        const double* a3 = hd + (t + 3) * H;
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        for (int64_t h = 0; h < hn; ++h) {
          s0 += a0[h] * w[h];
          s1 += a1[h] * w[h];
          s2 += a2[h] * w[h];
          s3 += a3[h] * w[h];
        }
        z[(t + 0) * V + v] = s0 / div;
        z[(t + 1) * V + v] = s1 / div;
        z[(t + 2) * V + v] = s2 / div;
        z[(t + 3) * V + v] = s3 / div;
      }
      for (; t < T; ++t) {
        const double* a = hd + t * H;
        double s = 0.0;
        for (int64_t h = 0; h < hn; ++h) s += a[h] * w[h];
        z[t * V + v] = s / div;
      }
    }
    free(w);
  }
  free(hd);
  return 0;
}

/* Step (3) and the row statistics used by (4) and (5). */
static void row_stats(const double* zr, int64_t V, double* lse_out, double* ez_out) {
  double m = -INFINITY;
  for (int64_t v = 0; v < V; ++v)
    if (zr[v] > m) m = zr[v];
  double s = 0.0;
  for (int64_t v = 0; v < V; ++v) s += exp(zr[v] - m);
  const double lse = (g_mutation == MUT_LSE_NO_MAX) ? log(s) : m + log(s);
  double ez = 0.0;
  for (int64_t v = 0; v < V; ++v) ez += exp(zr[v] - lse) * zr[v];
  *lse_out = lse;
  *ez_out = ez;
}

/* Steps (3)-(4) from a dense z[T,V]. */
int rlk_oracle_softmax_stats(const double* z, int64_t T, int64_t V, const int64_t* targets,
                             double* logp, double* entropy, double* lse) {
  if (T < 0 || V <= 0) return -1;
  if (check_targets(targets, T, V)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    const double* zr = z + t * V;
    double l, ez;
    row_stats(zr, V, &l, &ez);
    lse[t] = l;
    entropy[t] = (g_mutation == MUT_ENTROPY_SIGN) ? ez - l : l - ez;
    logp[t] = zr[target_of(targets, t, V)] - l;
  }
  return 0;
}

/* Step (5): dx[T,V] from a dense z[T,V]. */
int rlk_oracle_dlogits(const double* z, int64_t T, int64_t V, const int64_t* targets,
                       double tau, const double* dlogp, const double* dentropy, double* dx) {
  if (T < 0 || V <= 0 || !(tau > 0.0)) return -1;
  if (check_targets(targets, T, V)) return -2;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    const double* zr = z + t * V;
    double l, ez;
    row_stats(zr, V, &l, &ez);
    if (g_mutation == MUT_EZ_IS_MAX) {
      ez = -INFINITY;
      for (int64_t v = 0; v < V; ++v)
        if (zr[v] > ez) ez = zr[v];
    }
    const int64_t k = target_of(targets, t, V);
    const double a = dlogp[t], b = dentropy[t];
    const double div = (g_mutation == MUT_DX_NO_TAU) ? 1.0 : tau;
    for (int64_t v = 0; v < V; ++v) {
      const double p = exp(zr[v] - l);
      const double onehot = (v == k) ? 1.0 : 0.0;
      double d_logp = (g_mutation == MUT_DX_ONEHOT_SIGN) ? a * (p - onehot) : a * (onehot - p);
      double d_ent = (g_mutation == MUT_DX_NO_ENTROPY) ? 0.0 : b * p * (zr[v] - ez);
      dx[t * V + v] = (d_logp - d_ent) / div;
    }
  }
  return 0;
}

/* Step (6a): dHidden[T,H] = dx[T,V] . W[V,H], v ascending.  Each thread owns
 * whole rows of dHidden and walks all of W. */
int rlk_oracle_dhidden(const double* dx, const uint16_t* W, int64_t T, int64_t H, int64_t V,
                       double* dH) {
  if (T < 0 || H <= 0 || V <= 0) return -1;
  if (T == 0) return 0;
  const int transposed = (g_mutation == MUT_DH_TRANSPOSED) && (V == H);
#pragma omp parallel
  {
    double* w = (double*)malloc((size_t)H * sizeof(double));
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      double* out = dH + t * H;
      for (int64_t h = 0; h < H; ++h) out[h] = 0.0;
      for (int64_t v = 0; v < V; ++v) {
        if (transposed) {
          for (int64_t h = 0; h < H; ++h) w[h] = bf16_to_f64(W[h * H + v]);
        } else {
          widen(W + v * H, w, H);
        }
        const double a = dx[t * V + v];
        for (int64_t h = 0; h < H; ++h) out[h] += a * w[h];
      }
    }
    free(w);
  }
  return 0;
}

/* Step (6b): dW[V,H] += dx[T,V]^T . hidden[T,H], t ascending.  Adds into dW
 * (the caller zeroes it), so row blocks can be streamed in order. */
int rlk_oracle_dw_accumulate(const double* dx, const uint16_t* hidden, int64_t T, int64_t H,
                             int64_t V, double* dW) {
  if (T < 0 || H <= 0 || V <= 0) return -1;
  if (T == 0) return 0;
  double* hd = (double*)malloc((size_t)(T * H) * sizeof(double));
  if (!hd) return -3;
  widen(hidden, hd, T * H);
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t v = 0; v < V; ++v) {
    double* out = dW + v * H;
    for (int64_t t = 0; t < T; ++t) {
      const int64_t tr = (g_mutation == MUT_DW_ROW_INDEX) ? (t + 1) % T : t;
      const double a = dx[t * V + v];
      const double* hr = hd + tr * H;
      for (int64_t h = 0; h < H; ++h) out[h] += a * hr[h];
    }
  }
  free(hd);
  return 0;
}

/* Forward, steps (1)-(4), over row blocks so that only a [block, V] slab of
 * z is held at a time. */
int rlk_oracle_forward(const uint16_t* hidden, const uint16_t* W, const int64_t* targets,
                       int64_t T, int64_t H, int64_t V, double tau, double* logp,
                       double* entropy, double* lse) {
  if (T < 0 || H <= 0 || V <= 0 || !(tau > 0.0)) return -1;
  if (check_targets(targets, T, V)) return -2;
  const int64_t B = 64;
  double* z = (double*)malloc((size_t)((T < B ? T : B) * V + 1) * sizeof(double));
  if (!z) return -3;
  int rc = 0;
  for (int64_t t0 = 0; t0 < T && rc == 0; t0 += B) {
    const int64_t tb = (T - t0 < B) ? T - t0 : B;
    rc = rlk_oracle_logits(hidden + t0 * H, W, tb, H, V, tau, z);
    if (rc == 0)
      rc = rlk_oracle_softmax_stats(z, tb, V, targets + t0, logp + t0, entropy + t0, lse + t0);
  }
  free(z);
  return rc;
}

/* Backward, steps (1)-(6), over row blocks.  dHidden[T,H] and dW[V,H] are
 * overwritten. */
int rlk_oracle_backward(const uint16_t* hidden, const uint16_t* W, const int64_t* targets,
                        int64_t T, int64_t H, int64_t V, double tau, const double* dlogp,
                        const double* dentropy, double* dH, double* dW) {
  if (T < 0 || H <= 0 || V <= 0 || !(tau > 0.0)) return -1;
  if (check_targets(targets, T, V)) return -2;
  memset(dW, 0, (size_t)(V * H) * sizeof(double));
  if (T == 0) return 0;
  const int64_t B = 64;
  const int64_t nb = (T < B ? T : B);
  double* z = (double*)malloc((size_t)(nb * V) * sizeof(double));
  double* dx = (double*)malloc((size_t)(nb * V) * sizeof(double));
  if (!z || !dx) {
    free(z);
    free(dx);
    return -3;
  }
  int rc = 0;
  for (int64_t t0 = 0; t0 < T && rc == 0; t0 += B) {
    const int64_t tb = (T - t0 < B) ? T - t0 : B;
    rc = rlk_oracle_logits(hidden + t0 * H, W, tb, H, V, tau, z);
    if (rc == 0)
      rc = rlk_oracle_dlogits(z, tb, V, targets + t0, tau, dlogp + t0, dentropy + t0, dx);
    if (rc == 0) rc = rlk_oracle_dhidden(dx, W, tb, H, V, dH + t0 * H);
    if (rc == 0) rc = rlk_oracle_dw_accumulate(dx, hidden + t0 * H, tb, H, V, dW);
  }
  free(z);
  free(dx);
  return rc;
}
