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
// once per step.  Its fp32 summation order is fixed (octets of 8 probes through a
// 256-entry table of signed partial sums per octet, octet sums added in order).
#include "zo_internal.cuh"
#include "zo_tc.cuh"

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
  // Launched with programmatic dependent launch: the update may be scheduled now (it waits
  // for this grid before it reads anything); the losses are read only once the loss passes
  // before this kernel have completed.
  tc::pdl_launch_dependents();
  tc::pdl_wait();
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

template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ static void load16(const float *p, float v[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 x = __ldg(reinterpret_cast<const float4 *>(p) + k);
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
  }
  __device__ static void store16(float *p, const float v[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      reinterpret_cast<float4 *>(p)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  }
  __device__ static void load16s(const float *p, float v[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 x = reinterpret_cast<const float4 *>(p)[k];
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
  }
  __device__ static float get(const float *p, int64_t i) { return p[i]; }
  __device__ static void put(float *p, int64_t i, float v) { p[i] = v; }
};
template <> struct Elem<uint16_t> {
  __device__ static void load16(const uint16_t *p, float v[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint4 x = __ldg(reinterpret_cast<const uint4 *>(p) + k);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[8 * k + 2 * t] = __uint_as_float(w[t] << 16);
        v[8 * k + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
      }
    }
  }
  __device__ static void store16(uint16_t *p, const float v[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        w[t] = pack_bf16x2(v[8 * k + 2 * t], v[8 * k + 2 * t + 1]);
      reinterpret_cast<uint4 *>(p)[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  __device__ static void load16s(const uint16_t *p, float v[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint4 x = reinterpret_cast<const uint4 *>(p)[k];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[8 * k + 2 * t] = __uint_as_float(w[t] << 16);
        v[8 * k + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
      }
    }
  }
  __device__ static float get(const uint16_t *p, int64_t i) { return bf16_bits_to_f32(p[i]); }
  __device__ static void put(uint16_t *p, int64_t i, float v) { p[i] = f32_to_bf16_bits(v); }
};

// theta <- rd(theta - sum_i coef_i z_i).  One consumer thread per 16-element group: for each
// probe octet it computes the group's Philox block, whose byte b holds the octet's 8 signs of
// element b, and adds to element b the octet's table entry for that byte.  Entry e of an
// octet's table is the fp32 sum, left to right from its first signed term, of
// (bit t of e ? -a : +a) over the octet's probes t; the octet sums are added in order and
// subtracted once.  The tables are replicated R = 2^LOG_R times and lane l reads replica
// l mod R, so the 32 lookups of a warp meet at most 32/R to a bank (none at R = 32).  g_off is
// the global index of the context's first group: its elements take the signs of their
// global indices.
//
// theta streams in through shared memory: one or two CTAs per SM (section on the table
// budget below); warp 0 issues bulk copies of
// chunks of 8192 elements into a ring of stages, so that the loads are in flight while the
// 16 consumer warps regenerate the probes; a consumer thread copies its 16-element group from
// the stage into registers, the stage is released, and the updated group is written back with
// coalesced stores.  The last partial vector of theta (fewer than 16 bytes) is read directly.
constexpr int kUConsumers = 16;
constexpr int kUThreads = 32 * (1 + kUConsumers);
constexpr int kUChunk = kUConsumers * 32 * kGroup;  // 8192 elements

template <typename T, int STAGES> struct UpdPipe {
  static constexpr int kStages = STAGES;
  static constexpr int kStage = kUChunk * (int)sizeof(T);
  static constexpr int kRing = kStages * kStage;
  static constexpr int kLut = kRing + 2 * kStages * 8;  // after the ring and its barriers
  static constexpr int kFixed = kLut;
  // bf16 runs two CTAs per SM (registers capped at 56 per thread), fp32 one
  static constexpr int kMinBlocks = sizeof(T) == 2 ? 2 : 1;
};

// The octets' tables, R replicas each (all threads of the CTA take part).
template <int LOG_R>
__device__ __forceinline__ void build_tables(float *lut, const float *__restrict__ coef, int n) {
  const int octets = (n + 7) >> 3;
  // A warp computes 32 consecutive entries (one per lane) and writes their R replicas as
  // 32 R consecutive words, 32 per store: no bank conflicts.
  const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int base = (threadIdx.x >> 5) * 32; base < octets * 256; base += nwarps * 32) {
    const int idx = base + lane;  // octets * 256 is a multiple of 32
    const int o = idx >> 8, b = idx & 255;
    const int p0 = 8 * o, cnt = min(8, n - p0);
    const float a0 = __ldg(coef + p0);
    float s = (b & 1) ? -a0 : a0;
    for (int t = 1; t < cnt; ++t) {
      const float a = __ldg(coef + p0 + t);
      s = __fadd_rn(s, ((b >> t) & 1) ? -a : a);
    }
#pragma unroll
    for (int j = 0; j < (1 << LOG_R); ++j) {
      const int word = j * 32 + lane;  // replica (word & (R-1)) of entry base + (word >> LOG_R)
      lut[(base << LOG_R) + word] = __shfl_sync(0xFFFFFFFFu, s, word >> LOG_R);
    }
  }
}

// v[e] -= (sum over octets of the table entry of element e's sign byte), fixed order.
template <int LOG_R>
__device__ __forceinline__ void apply_probes(float v[16], const float *mine, uint64_t g, int octets,
                                             uint32_t step, const RoundKeys &rk) {
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int o = 0; o < octets; ++o) {
    const uint4 blk = sign_block(g, (uint32_t)o, step, rk);
    const uint32_t w[4] = {blk.x, blk.y, blk.z, blk.w};
    const float *tab = mine + ((o * 256) << LOG_R);
#pragma unroll
    for (int e = 0; e < 16; ++e)  // byte e & 3 of word e >> 2 selects the entry
      acc[e] = __fadd_rn(acc[e], tab[__byte_perm(w[e >> 2], 0u, 0x4440u | (uint32_t)(e & 3)) << LOG_R]);
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = __fsub_rn(v[e], acc[e]);
}

template <typename T, int LOG_R, int STAGES>
__global__ void __launch_bounds__(kUThreads, UpdPipe<T, STAGES>::kMinBlocks)
update_kernel(T *__restrict__ theta, int64_t M, const float *__restrict__ coef, int n,
              const uint32_t *step_ptr, const uint32_t *ok_ptr, const __grid_constant__ RoundKeys rk,
              uint64_t g_off, uint32_t *err) {
  using U = UpdPipe<T, STAGES>;
  constexpr int N = 16 / (int)sizeof(T);  // elements per 16-byte vector
  extern __shared__ __align__(128) uint8_t usm[];
  uint64_t *full = reinterpret_cast<uint64_t *>(usm + U::kRing);
  uint64_t *empty = full + U::kStages;
  float *lut = reinterpret_cast<float *>(usm + U::kLut);  // [octet][256 entries][R replicas]
  __shared__ volatile int abort_flag;
  // Launched with programmatic dependent launch: wait for the preconditioner (coefficients,
  // step, ok flag).  This kernel never signals early, so the next kernel of the stream, which
  // reads theta, starts only after it has completed.
  tc::pdl_wait();
  if (ok_ptr != nullptr && *ok_ptr == 0u) return;
  const uint32_t step = *step_ptr;
  const int octets = (n + 7) >> 3;
  if (threadIdx.x == 0) {
    for (int s = 0; s < U::kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kUConsumers);
    }
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  build_tables<LOG_R>(lut, coef, n);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_chunks = (M + kUChunk - 1) / kUChunk;
  if (warp == 0) {  // producer
    int it = 0, issued = 0;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
      const int s = it % U::kStages;
      const uint32_t ph = (uint32_t)(it / U::kStages) & 1u;
      int ok = 1;
      if (lane == 0) ok = tc::mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok || abort_flag) {
        if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
        break;
      }
      const int64_t cs = c * kUChunk;
      const int64_t copy = ((M - cs < kUChunk ? M - cs : kUChunk)) & ~(int64_t)(N - 1);
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&full[s], (uint32_t)(copy * (int64_t)sizeof(T)));
        if (copy > 0)
          tc::bulk_load(usm + s * U::kStage, theta + cs, (uint32_t)(copy * (int64_t)sizeof(T)), &full[s]);
      }
      __syncwarp();
      issued = it + 1;
    }
    if (abort_flag && lane == 0) {  // let this CTA's loads land before it exits (bounded)
      for (int s = 0; s < U::kStages; ++s) {
        int last = -1;
        for (int i = s; i < issued; i += U::kStages) last = i;
        if (last >= 0) tc::mbar_wait(&full[s], (uint32_t)(last / U::kStages) & 1u);
      }
    }
    return;
  }
  // consumers: thread ct updates group ct of each chunk: it copies the group from the stage
  // into registers, the warp releases the stage, and the updated group is written back with
  // coalesced 16-byte stores (a warp writes 1 KB (bf16) or 2 KB (fp32) of consecutive bytes)
  const int ct = threadIdx.x - 32;
  const float *mine = lut + (lane & ((1 << LOG_R) - 1));
  int it = 0;
  for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
    const int s = it % U::kStages;
    const uint32_t ph = (uint32_t)(it / U::kStages) & 1u;
    int ok = 1;
    if (lane == 0) ok = (!abort_flag && tc::mbar_wait(&full[s], ph)) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (ok && lane != 0) ok = tc::mbar_wait(&full[s], ph) ? 1 : 0;
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
      break;
    }
    const T *st = reinterpret_cast<const T *>(usm + s * U::kStage);
    const int64_t cs = c * kUChunk;
    const int64_t e0 = cs + (int64_t)ct * kGroup;
    if (cs + kUChunk <= M) {  // a full chunk: every group is whole and staged
      float v[16];
      Elem<T>::load16s(st + ct * kGroup, v);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[s]);  // the stage is free again
      apply_probes<LOG_R>(v, mine, (uint64_t)(e0 / kGroup) + g_off, octets, step, rk);
      Elem<T>::store16(theta + e0, v);
      continue;
    }
    const int64_t copy_end = cs + ((M - cs) & ~(int64_t)(N - 1));
    const bool whole = e0 + kGroup <= copy_end;
    float v[16];
    if (whole) {
      Elem<T>::load16s(st + ct * kGroup, v);
    } else {  // the last group: elements below copy_end are staged, the rest are read directly
#pragma unroll
      for (int e = 0; e < 16; ++e)
        v[e] = e0 + e < copy_end ? Elem<T>::get(st, e0 + e - cs)
                                 : (e0 + e < M ? Elem<T>::get(theta, e0 + e) : 0.f);
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[s]);  // the stage is free again
    if (e0 >= M) continue;
    apply_probes<LOG_R>(v, mine, (uint64_t)(e0 / kGroup) + g_off, octets, step, rk);
    if (whole) {
      Elem<T>::store16(theta + e0, v);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (e0 + e < M) Elem<T>::put(theta, e0 + e, v[e]);
    }
  }
}

// Shared-memory plan: table replicas R = 2^log_r and ring stages.  A lookup is conflict-free
// at R = 32 (lane l reads replica l); at R = 16 lanes l and l + 16 share a replica and split
// into two wavefronts whenever their entries differ in bank.  bf16 prefers two CTAs per SM
// (34 warps; the kernel is bound by instruction issue and shared-memory wavefronts): R = 32
// with the deepest ring (4 or 3 stages) that fits, else R = 16.  Otherwise (fp32, or large
// n) one CTA takes up to 226 KB with the largest R that fits beside its ring.
struct UpdPlan {
  int log_r, stages;
};

// Two CTAs per SM: 228 KB per SM, less 1 KB reserved per CTA and the kernel's static words.
constexpr int64_t kTwoCtaBudget = 113 * 1024 - 64;
constexpr int64_t kOneCtaBudget = 226 * 1024;

template <typename T>
UpdPlan update_plan(int n) {
  const int64_t per_replica = (int64_t)((n + 7) / 8) * 256 * 4;
  if constexpr (sizeof(T) == 2) {
    const int64_t ring4 = UpdPipe<T, 4>::kFixed, ring3 = UpdPipe<T, 3>::kFixed;
    for (int lr = 5; lr >= 4; --lr) {
      if (ring4 + (per_replica << lr) <= kTwoCtaBudget) return {lr, 4};
      if (ring3 + (per_replica << lr) <= kTwoCtaBudget) return {lr, 3};
    }
    int lr = 5;
    while (lr > 0 && ring4 + (per_replica << lr) > kOneCtaBudget) --lr;
    return {lr, 4};
  }
  const int64_t ring = UpdPipe<T, 3>::kFixed;
  int lr = 5;
  while (lr > 0 && ring + (per_replica << lr) > kOneCtaBudget) --lr;
  return {lr, 3};
}

template <typename T, int LOG_R, int STAGES>
zo_status launch_update_t(zo_ctx *ctx, const float *coef, int n, const uint32_t *step_ptr,
                          const uint32_t *ok_ptr, uint32_t k0, uint32_t k1) {
  const size_t smem = (size_t)UpdPipe<T, STAGES>::kFixed +
                      ((size_t)((n + 7) / 8) * 256 * sizeof(float) << LOG_R);
  auto kern = update_kernel<T, LOG_R, STAGES>;
  // the table size varies with n: raise the limit once to the largest a CTA may use (the
  // plan keeps every launch within 226 KB; the kernel's static shared memory comes on top,
  // within the 227 KB a CTA may have)
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), (int)kOneCtaBudget);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "update_kernel setup: %s", cudaGetErrorString(e));
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kUThreads, smem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const int64_t n_chunks = (ctx->M + kUChunk - 1) / kUChunk;
  const int64_t cap = (int64_t)kSmCount * per_sm;
  const int64_t blocks = n_chunks < cap ? n_chunks : cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kUThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = ctx->stream;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  const int slot = ktime_begin(ctx);
  e = cudaLaunchKernelEx(&cfg, kern, static_cast<T *>(ctx->params), ctx->M, coef, n, step_ptr,
                         ok_ptr, round_keys(k0, k1), (uint64_t)(ctx->first_element / kGroup),
                         &ctx->dstate->flags);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "update_kernel: %s", cudaGetErrorString(e));
  const zo_status st = check_launch(ctx, "update_kernel");
  if (st == ZO_OK) ktime_end(ctx, slot, ZO_KT_UPDATE, 2.0 * sizeof(T) * (double)ctx->M);
  return st;
}

template <typename T, int STAGES>
zo_status launch_update_s(zo_ctx *ctx, int log_r, const float *coef, int n,
                          const uint32_t *step_ptr, const uint32_t *ok_ptr, uint32_t k0,
                          uint32_t k1) {
  switch (log_r) {
    case 5: return launch_update_t<T, 5, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
    case 4: return launch_update_t<T, 4, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
    case 3: return launch_update_t<T, 3, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
    case 2: return launch_update_t<T, 2, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
    case 1: return launch_update_t<T, 1, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
    default: return launch_update_t<T, 0, STAGES>(ctx, coef, n, step_ptr, ok_ptr, k0, k1);
  }
}

template <typename T>
zo_status launch_update_r(zo_ctx *ctx, const float *coef, int n, const uint32_t *step_ptr,
                          const uint32_t *ok_ptr, uint32_t k0, uint32_t k1) {
  const UpdPlan p = update_plan<T>(n);
  if constexpr (sizeof(T) == 2) {
    if (p.stages == 4) return launch_update_s<T, 4>(ctx, p.log_r, coef, n, step_ptr, ok_ptr, k0, k1);
  }
  return launch_update_s<T, 3>(ctx, p.log_r, coef, n, step_ptr, ok_ptr, k0, k1);
}

}  // namespace

zo_status launch_precond(zo_ctx *ctx, const double *lp, const double *lm, const double *l0,
                         int n, float lr, float eps, float damping) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPrecondThreads);
  cfg.stream = ctx->stream;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, precond_kernel, lp, lm, l0, n, (double)lr, (double)eps,
                                           (double)damping, (double)ctx->alpha, ctx->coef, ctx->diag,
                                           ctx->dstate);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "precond_kernel: %s", cudaGetErrorString(e));
  ctx->last_n = n;
  return check_launch(ctx, "precond_kernel");
}

zo_status launch_update(zo_ctx *ctx, const float *coef, int n, const uint32_t *step_ptr,
                        const uint32_t *ok_ptr) {
  const ProbeKey pk = probe_key(ctx);
  return ctx->dtype == ZO_F32 ? launch_update_r<float>(ctx, coef, n, step_ptr, ok_ptr, pk.k0, pk.k1)
                              : launch_update_r<uint16_t>(ctx, coef, n, step_ptr, ok_ptr, pk.k0, pk.k1);
}

}  // namespace zo
