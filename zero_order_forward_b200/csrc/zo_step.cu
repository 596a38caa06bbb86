// zo_step.cu -- the probe-space preconditioner and the single-pass update.
//
// "Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation":
//   section "How 1.5-SPSA Works": g_i = (L(theta+eps z_i) - L(theta-eps z_i)) / (2 eps),
//     the estimate averages g_i z_i over the n probes (z_i is its own inverse);
//   section "Probe-Space Preconditioning": a clean loss L0 gives the per-probe curvature
//     c_i = (L+ + L- - 2 L0)/eps^2, and directions of high curvature get small weights
//     w_i = (|c_i| + damping)^(-alpha), alpha = 0.1; storage is O(n), not O(M).
// "Probe-Space Preconditioning for Fast and Stable Zero-Order Training", abstract: the
// update keeps no optimizer state; theta <- theta - sum_i a_i z_i with a_i = lr*w_i*g_i/n.
//
// The update regenerates all n probes in registers, so theta is read once and written
// once per step.  Its fp32 summation order is fixed (groups of 8 probes through a
// 256-entry table of signed partial sums per group, group sums added in order).
#include "zo_internal.cuh"

namespace zo {
namespace {

__device__ __forceinline__ double warp_min(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ double warp_add(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

constexpr int kPrecondThreads = 256;

// One CTA.  diag layout: g[0..MAX), c[MAX..2MAX), w[2MAX..3MAX), then 6 statistics:
// sum g^2, min c, max c, min w, max w, sum |a|.
__global__ void __launch_bounds__(kPrecondThreads)
precond_kernel(const double *__restrict__ lp, const double *__restrict__ lm,
               const double *__restrict__ l0, int n, double lr, double eps, double damping,
               double alpha, float *__restrict__ coef, double *__restrict__ diag,
               DevState *st) {
  __shared__ double red[6][kPrecondThreads / 32];
  bool bad = false;
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    bad |= !isfinite(lp[i]) || !isfinite(lm[i]);
  if (l0 != nullptr && threadIdx.x == 0) bad |= !isfinite(*l0);
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) {
      st->flags |= ZO_FLAG_NONFINITE;
      st->upd_ok = 0u;
    }
    return;
  }
  const double L0 = l0 ? *l0 : 0.0;
  double sg2 = 0.0, cmin = INFINITY, cmax = -INFINITY, wmin = INFINITY, wmax = -INFINITY,
         sa = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const double g = (lp[i] - lm[i]) / (2.0 * eps);
    double c = 0.0, w = 1.0;
    if (l0) {
      c = (lp[i] + lm[i] - 2.0 * L0) / (eps * eps);
      w = pow(fabs(c) + damping, -alpha);
    }
    const double a = lr * w * g / (double)n;
    coef[i] = __double2float_rn(a);
    diag[i] = g;
    diag[ZO_MAX_PROBES + i] = c;
    diag[2 * ZO_MAX_PROBES + i] = w;
    sg2 += g * g;
    cmin = fmin(cmin, c); cmax = fmax(cmax, c);
    wmin = fmin(wmin, w); wmax = fmax(wmax, w);
    sa += fabs(a);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  sg2 = warp_add(sg2); cmin = warp_min(cmin); cmax = warp_max(cmax);
  wmin = warp_min(wmin); wmax = warp_max(wmax); sa = warp_add(sa);
  if (lane == 0) {
    red[0][warp] = sg2; red[1][warp] = cmin; red[2][warp] = cmax;
    red[3][warp] = wmin; red[4][warp] = wmax; red[5][warp] = sa;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < kPrecondThreads / 32; ++k) {
      red[0][0] += red[0][k]; red[1][0] = fmin(red[1][0], red[1][k]);
      red[2][0] = fmax(red[2][0], red[2][k]); red[3][0] = fmin(red[3][0], red[3][k]);
      red[4][0] = fmax(red[4][0], red[4][k]); red[5][0] += red[5][k];
    }
    for (int k = 0; k < 6; ++k) diag[3 * ZO_MAX_PROBES + k] = red[k][0];
    st->upd_step = st->step;
    st->upd_ok = 1u;
    st->step = st->step + 1u;
  }
}

constexpr int kUpdWarps = 8;

// 4x4 byte transpose: out[k] byte t = w[t] byte k.
__device__ __forceinline__ void byte_transpose4(uint32_t w0, uint32_t w1, uint32_t w2,
                                                uint32_t w3, uint32_t out[4]) {
  const uint32_t t0 = __byte_perm(w0, w1, 0x5140), t1 = __byte_perm(w0, w1, 0x7362);
  const uint32_t t2 = __byte_perm(w2, w3, 0x5140), t3 = __byte_perm(w2, w3, 0x7362);
  out[0] = __byte_perm(t0, t2, 0x5410);
  out[1] = __byte_perm(t0, t2, 0x7632);
  out[2] = __byte_perm(t1, t3, 0x5410);
  out[3] = __byte_perm(t1, t3, 0x7632);
}

// Transpose the 8x8 bit matrix held in (lo = bytes 0..3, hi = bytes 4..7), byte = row,
// bit = column: afterwards bit i of byte j is the former bit j of byte i.
__device__ __forceinline__ void bit_transpose8(uint32_t &lo, uint32_t &hi) {
  uint32_t t;
  t = (lo ^ (lo >> 7)) & 0x00AA00AAu; lo ^= t ^ (t << 7);
  t = (hi ^ (hi >> 7)) & 0x00AA00AAu; hi ^= t ^ (t << 7);
  t = (lo ^ (lo >> 14)) & 0x0000CCCCu; lo ^= t ^ (t << 14);
  t = (hi ^ (hi >> 14)) & 0x0000CCCCu; hi ^= t ^ (t << 14);
  t = (lo ^ __funnelshift_r(lo, hi, 28)) & 0xF0F0F0F0u;
  lo ^= t;
  hi ^= t >> 4;
}

// Quad exchange: lane q of a quad holds the block r of probe p0+q; afterwards W[p] is
// word q of the block of probe p0+p.
__device__ __forceinline__ void quad_exchange(const uint4 &r, int q, int lane, uint32_t W[4]) {
  uint32_t R[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t send = word_of(r, (q - t) & 3);
    R[t] = __shfl_sync(0xFFFFFFFFu, send, (lane & ~3) | ((q + t) & 3));  // probe (q+t)&3
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // W[p] = R[(p - q) & 3]
    const int t = (p - q) & 3;
    W[p] = t == 0 ? R[0] : t == 1 ? R[1] : t == 2 ? R[2] : R[3];
  }
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ static void load32(const float *p, float v[32]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 x = reinterpret_cast<const float4 *>(p)[k];
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
  }
  __device__ static void store32(float *p, const float v[32]) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      reinterpret_cast<float4 *>(p)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  }
  __device__ static float get(const float *p, int64_t i) { return p[i]; }
  __device__ static void put(float *p, int64_t i, float v) { p[i] = v; }
};
template <> struct Elem<uint16_t> {
  __device__ static void load32(const uint16_t *p, float v[32]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 x = reinterpret_cast<const uint4 *>(p)[k];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[8 * k + 2 * t] = __uint_as_float(w[t] << 16);
        v[8 * k + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
      }
    }
  }
  __device__ static void store32(uint16_t *p, const float v[32]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        w[t] = (uint32_t)f32_to_bf16_bits(v[8 * k + 2 * t]) |
               ((uint32_t)f32_to_bf16_bits(v[8 * k + 2 * t + 1]) << 16);
      reinterpret_cast<uint4 *>(p)[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  __device__ static float get(const uint16_t *p, int64_t i) { return bf16_bits_to_f32(p[i]); }
  __device__ static void put(uint16_t *p, int64_t i, float v) { p[i] = f32_to_bf16_bits(v); }
};

// theta <- rd(theta - sum_i coef_i z_i).  A warp covers 8 groups (1024 elements) per
// slab: lane l owns the 32 elements of word slot (l & 3) of group (l >> 2).
template <typename T>
__global__ void __launch_bounds__(kUpdWarps * 32)
update_kernel(T *__restrict__ theta, int64_t M, const float *__restrict__ coef, int n,
              const uint32_t *step_ptr, const uint32_t *ok_ptr, uint32_t k0, uint32_t k1,
              int64_t n_slabs) {
  extern __shared__ float lut[];  // [ngroups][256]
  if (ok_ptr != nullptr && *ok_ptr == 0u) return;
  const uint32_t step = *step_ptr;
  const int ngroups = (n + 7) >> 3;
  // Tables of signed partial sums: entry b of group g is the fp32 sum, left to right,
  // of (bit t of b ? -a : +a) over the group's probes t.
  for (int idx = threadIdx.x; idx < ngroups * 256; idx += blockDim.x) {
    const int g = idx >> 8, b = idx & 255;
    const int p0 = 8 * g, cnt = min(8, n - p0);
    float a0 = __ldg(coef + p0);
    float s = (b & 1) ? -a0 : a0;
    for (int t = 1; t < cnt; ++t) {
      const float a = __ldg(coef + p0 + t);
      s = __fadd_rn(s, ((b >> t) & 1) ? -a : a);
    }
    lut[idx] = s;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, q = lane & 3;
  for (int64_t slab = (int64_t)blockIdx.x * kUpdWarps + warp; slab < n_slabs;
       slab += (int64_t)gridDim.x * kUpdWarps) {
    const uint64_t g = (uint64_t)slab * 8 + (lane >> 2);
    const int64_t e0 = (int64_t)g * kGroup + q * 32;
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.f;
    for (int grp = 0; grp < ngroups; ++grp) {
      const int pa = 8 * grp + q, pb = 8 * grp + 4 + q;
      const uint4 ra = pa < n ? probe_block(g, (uint32_t)pa, step, k0, k1) : make_uint4(0, 0, 0, 0);
      const uint4 rb = pb < n ? probe_block(g, (uint32_t)pb, step, k0, k1) : make_uint4(0, 0, 0, 0);
      uint32_t W[8];
      quad_exchange(ra, q, lane, W);
      quad_exchange(rb, q, lane, W + 4);
      uint32_t L[4], H[4];
      byte_transpose4(W[0], W[1], W[2], W[3], L);
      byte_transpose4(W[4], W[5], W[6], W[7], H);
      const float *tab = lut + grp * 256;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t lo = L[k], hi = H[k];
        bit_transpose8(lo, hi);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[8 * k + e] = __fadd_rn(acc[8 * k + e], tab[(lo >> (8 * e)) & 0xFFu]);
          acc[8 * k + 4 + e] = __fadd_rn(acc[8 * k + 4 + e], tab[(hi >> (8 * e)) & 0xFFu]);
        }
      }
    }
    if (e0 + 32 <= M) {
      float v[32];
      Elem<T>::load32(theta + e0, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __fsub_rn(v[e], acc[e]);
      Elem<T>::store32(theta + e0, v);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (e0 + e < M) Elem<T>::put(theta, e0 + e, __fsub_rn(Elem<T>::get(theta, e0 + e), acc[e]));
    }
  }
}

}  // namespace

zo_status launch_precond(zo_ctx *ctx, const double *lp, const double *lm, const double *l0,
                         int n, float lr, float eps, float damping) {
  precond_kernel<<<1, kPrecondThreads, 0, ctx->stream>>>(
      lp, lm, l0, n, (double)lr, (double)eps, (double)damping, (double)ctx->alpha, ctx->coef,
      ctx->diag, ctx->dstate);
  ctx->last_n = n;
  return check_launch(ctx, "precond_kernel");
}

zo_status launch_update(zo_ctx *ctx, const float *coef, int n, const uint32_t *step_ptr,
                        const uint32_t *ok_ptr) {
  const int64_t n_groups = (ctx->M + kGroup - 1) / kGroup;
  const int64_t n_slabs = (n_groups + 7) / 8;
  const size_t smem = (size_t)((n + 7) / 8) * 256 * sizeof(float);
  int64_t blocks = (n_slabs + kUpdWarps - 1) / kUpdWarps;
  if (blocks > (int64_t)kSmCount * 4) blocks = (int64_t)kSmCount * 4;
  ProbeKey pk = probe_key(ctx);
  if (ctx->dtype == ZO_F32) {
    cudaFuncSetAttribute(update_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    update_kernel<float><<<(unsigned)blocks, kUpdWarps * 32, smem, ctx->stream>>>(
        static_cast<float *>(ctx->params), ctx->M, coef, n, step_ptr, ok_ptr, pk.k0, pk.k1, n_slabs);
  } else {
    cudaFuncSetAttribute(update_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    update_kernel<uint16_t><<<(unsigned)blocks, kUpdWarps * 32, smem, ctx->stream>>>(
        static_cast<uint16_t *>(ctx->params), ctx->M, coef, n, step_ptr, ok_ptr, pk.k0, pk.k1, n_slabs);
  }
  return check_launch(ctx, "update_kernel");
}

}  // namespace zo
