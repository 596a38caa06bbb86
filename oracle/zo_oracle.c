/*
 * zo_oracle.c -- plain, slow, single-threaded CPU oracle for the 1SPSA / 1.5-SPSA
 * zero-order step.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library; the product (libzo.so and its
 * Python binding) never does, and shares no code with it.
 *
 * Sources (cited by page title and section):
 *   [HOW]  "Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section
 *          "How 1.5-SPSA Works": Rademacher probes z_i in {-1,+1}^M, the losses at
 *          theta +/- eps*z_i, the projected difference (L+ - L-)/(2 eps) times the
 *          elementwise inverse of z_i (which is z_i itself for +/-1 entries).
 *   [PSP]  same page, section "Probe-Space Preconditioning": one extra clean loss,
 *          per-probe curvature from clean vs perturbed losses, weights |c_i|^alpha
 *          with alpha = 0.1, high-curvature probes down-weighted.
 *   [ABS]  "Probe-Space Preconditioning for Fast and Stable Zero-Order Training",
 *          abstract: inference-mode training with no stored activations, gradients
 *          or optimizer state; an 8-bit-packing random generator.
 *   [PHX]  Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3"
 *          (SC'11), the Philox-4x32 bijection with R = 10 rounds.
 *
 * Readings where the pages are silent (each restated in the design notes):
 *   - Probe bits, 8 signs per byte [ABS] with the byte holding the signs of one element
 *     under 8 consecutive probes: Philox4x32-10 with key = (seed low word, seed high
 *     word) and counter = (g low word, g high word, p, step), where g = j >> 4 is the
 *     index of the 16-element group of element j and p = probe >> 3 the index of the
 *     8-probe octet.  The 16 output bytes (little-endian words w0..w3) belong to the 16
 *     elements of the group: element j takes byte (j & 15), i.e. bits 8*(j & 3)..+7 of
 *     word ((j >> 2) & 3); probe i takes bit (i & 7) of that byte; bit 0 means z = +1,
 *     bit 1 means z = -1.  The packed form of ONE probe (an export format) holds its
 *     elements 8q..8q+7 in byte q (bit t <-> element 8q+t).
 *   - Perturbation: P_j = rd(theta_j + s*eps*z_j) as one fp32 add with
 *     round-to-nearest-even; bf16 weights are widened exactly, added in fp32, and
 *     rounded to bf16 (RNE).  theta itself is never written by a perturbation.
 *   - Estimator prefactor 1/n (the stray factor 2 in the printed formula is read as
 *     extraction damage); curvature c_i = (L+ + L- - 2 L0)/eps^2; step multiplier
 *     w_i = (|c_i| + damping)^(-alpha); a_i = lr * w_i * g_i / n; 1SPSA has w_i = 1.
 *   - Update: theta' = rd(theta - sum_i a_i z_i).  The "fp64" form sums in double;
 *     the "mirror" form fixes an fp32 order: probes in groups of 8, each group summed
 *     left to right starting from its first signed term, the group sums added left to
 *     right, then one fp32 subtraction.  Build with -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ Philox [PHX] */

/* The round multipliers and Weyl key increments published with Philox-4x32. */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void zo_oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                             uint32_t out[4]) {
  uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) { /* the key is bumped between rounds */
      k0 += PHILOX_W0;
      k1 += PHILOX_W1;
    }
    uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;
    uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)x2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t y0 = hi1 ^ x1 ^ k0;
    uint32_t y1 = lo1;
    uint32_t y2 = hi0 ^ x3 ^ k1;
    uint32_t y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The 128 sign bits of the 16-element group holding element j under the probe octet
 * holding `probe`, for (seed, step). */
static void probe_group_words(uint64_t seed, uint32_t step, uint32_t probe, int64_t j,
                              uint32_t out[4]) {
  uint64_t g = (uint64_t)j >> 4;
  uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), probe >> 3, step};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  zo_oracle_philox4x32_10(ctr, key, out);
}

/* z_ij in {+1, -1} [HOW]. */
int zo_oracle_probe_sign(uint64_t seed, uint32_t step, uint32_t probe, int64_t j) {
  uint32_t w[4];
  probe_group_words(seed, step, probe, j, w);
  uint32_t byte = (w[(j >> 2) & 3] >> (8 * (j & 3))) & 0xFFu;
  uint32_t bit = (byte >> (probe & 7)) & 1u;
  return bit ? -1 : +1;
}

/* Packed probe, 8 signs per byte [ABS]: out has ceil(M/8) bytes; bits past M are 0. */
void zo_oracle_pack_probe(uint64_t seed, uint32_t step, uint32_t probe, int64_t M,
                          uint8_t *out) {
  int64_t nbytes = (M + 7) / 8;
  memset(out, 0, (size_t)nbytes);
  for (int64_t j = 0; j < M; ++j) {
    if (zo_oracle_probe_sign(seed, step, probe, j) < 0)
      out[j >> 3] |= (uint8_t)(1u << (j & 7));
  }
}

/* ------------------------------------------------------------------ bf16 helpers */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
    return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

uint16_t zo_oracle_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
float zo_oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

/* ------------------------------------------------------------------ perturbation */

/* P_j = rd32(theta_j + s*eps*z_j), out of place; theta is not written [HOW].
 * Array element k holds global parameter j = j0 + k (the probe bits depend on j). */
void zo_oracle_perturb_f32(const float *theta, int64_t j0, int64_t count, uint64_t seed,
                           uint32_t step, uint32_t probe, int sign, float eps, float *out) {
  for (int64_t k = 0; k < count; ++k) {
    float delta = (float)(sign * zo_oracle_probe_sign(seed, step, probe, j0 + k)) * eps;
    out[k] = theta[k] + delta;
  }
}

void zo_oracle_perturb_bf16(const uint16_t *theta, int64_t j0, int64_t count, uint64_t seed,
                            uint32_t step, uint32_t probe, int sign, float eps, uint16_t *out) {
  for (int64_t k = 0; k < count; ++k) {
    float delta = (float)(sign * zo_oracle_probe_sign(seed, step, probe, j0 + k)) * eps;
    float sum = bf16_to_f32(theta[k]) + delta;
    out[k] = f32_to_bf16_rne(sum);
  }
}

/* ------------------------------------------------------------------ quadratic loss */

/* L = 1/2 sum_j D_j P_j^2, every term and the running sum in fp64, j ascending. */
double zo_oracle_quad_loss(const float *P, const float *D, int64_t M) {
  double sum = 0.0;
  for (int64_t j = 0; j < M; ++j) {
    double p = (double)P[j];
    sum += 0.5 * (double)D[j] * (p * p);
  }
  return sum;
}

/* ------------------------------------------------------------------ preconditioner */

/*
 * From the per-probe losses to the per-probe update coefficients, in fp64 [HOW][PSP]:
 *   g_i = (L+_i - L-_i) / (2 eps)
 *   c_i = (L+_i + L-_i - 2 L0) / eps^2             (1.5-SPSA only)
 *   w_i = (|c_i| + damping)^(-alpha)               (1.5-SPSA; 1SPSA: w_i = 1)
 *   a_i = lr * w_i * g_i / n
 * loss0 == NULL selects 1SPSA (c_i and w_i are then reported as 0 and 1).
 * Returns 0, or 1 if any loss is not finite (outputs are then untouched).
 */
int zo_oracle_precond(const double *loss_plus, const double *loss_minus,
                      const double *loss0, int n, double eps, double lr, double damping,
                      double alpha, double *g, double *c, double *w, double *a) {
  if (loss0 && !isfinite(*loss0)) return 1;
  for (int i = 0; i < n; ++i)
    if (!isfinite(loss_plus[i]) || !isfinite(loss_minus[i])) return 1;
  for (int i = 0; i < n; ++i) {
    double gi = (loss_plus[i] - loss_minus[i]) / (2.0 * eps);
    double ci = 0.0, wi = 1.0;
    if (loss0) {
      ci = (loss_plus[i] + loss_minus[i] - 2.0 * (*loss0)) / (eps * eps);
      wi = pow(fabs(ci) + damping, -alpha);
    }
    g[i] = gi;
    c[i] = ci;
    w[i] = wi;
    a[i] = lr * wi * gi / (double)n;
  }
  return 0;
}

/* ------------------------------------------------------------------ update */

/* theta' = rd32(theta - sum_i a_i z_i), the sum over probes taken in fp64.
 * Array element k holds global parameter j0 + k. */
void zo_oracle_update_f64_f32(float *theta, int64_t j0, int64_t count, const double *a, int n,
                              uint64_t seed, uint32_t step) {
  for (int64_t k = 0; k < count; ++k) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i)
      acc += a[i] * (double)zo_oracle_probe_sign(seed, step, (uint32_t)i, j0 + k);
    theta[k] = (float)((double)theta[k] - acc);
  }
}

/* bf16: the fp64 value is rounded to fp32 and then to bf16 (two roundings; the tests
 * allow one bf16 ulp against a single rounding). */
void zo_oracle_update_f64_bf16(uint16_t *theta, int64_t j0, int64_t count, const double *a,
                               int n, uint64_t seed, uint32_t step) {
  for (int64_t k = 0; k < count; ++k) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i)
      acc += a[i] * (double)zo_oracle_probe_sign(seed, step, (uint32_t)i, j0 + k);
    double v = (double)bf16_to_f32(theta[k]) - acc;
    theta[k] = f32_to_bf16_rne((float)v);
  }
}

/* The fixed fp32 summation order (groups of 8 probes) for coefficient a32. */
static float mirror_sum(const float *a32, int n, uint64_t seed, uint32_t step, int64_t j) {
  float acc = 0.0f;
  for (int g0 = 0; g0 < n; g0 += 8) {
    int g1 = g0 + 8 < n ? g0 + 8 : n;
    float s = (float)zo_oracle_probe_sign(seed, step, (uint32_t)g0, j) * a32[g0];
    for (int i = g0 + 1; i < g1; ++i)
      s = s + (float)zo_oracle_probe_sign(seed, step, (uint32_t)i, j) * a32[i];
    acc = acc + s;
  }
  return acc;
}

void zo_oracle_update_mirror_f32(float *theta, int64_t j0, int64_t count, const float *a32,
                                 int n, uint64_t seed, uint32_t step) {
  for (int64_t k = 0; k < count; ++k)
    theta[k] = theta[k] - mirror_sum(a32, n, seed, step, j0 + k);
}

void zo_oracle_update_mirror_bf16(uint16_t *theta, int64_t j0, int64_t count, const float *a32,
                                  int n, uint64_t seed, uint32_t step) {
  for (int64_t k = 0; k < count; ++k)
    theta[k] = f32_to_bf16_rne(bf16_to_f32(theta[k]) - mirror_sum(a32, n, seed, step, j0 + k));
}
