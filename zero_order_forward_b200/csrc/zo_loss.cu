// zo_loss.cu -- loss-only evaluations for the two small workloads: the diagonal
// quadratic (perturbation applied on load, fp64 accumulation) and the MLP classifier
// (fp32 CUDA-core arithmetic, no TF32).  Inference mode only: nothing but the scalar
// loss leaves the kernel ("Probe-Space Preconditioning for Fast and Stable Zero-Order
// Training", abstract).
//
// Reductions are deterministic: each block writes one fp64 partial, and the last block
// to finish (ticket on a counter) adds the partials in index order with a fixed tree.
#include <mutex>

#include "zo_internal.cuh"
#include "zo_tc.cuh"

namespace zo {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Sum `v` over the block (fixed shape); the result is valid in thread 0.
__device__ double block_sum(double v) {
  __shared__ double s[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) s[warp] = v;
  __syncthreads();
  const int nw = (blockDim.x + 31) >> 5;
  v = (threadIdx.x < nw) ? s[threadIdx.x] : 0.0;
  if (warp == 0) v = warp_sum(v);
  return v;
}

// Block `blockIdx.x` contributes v[0..NV) (valid in thread 0); the last block writes
// out[k] = (accumulate ? out[k] : 0) + scale * sum_b partials[k][b] for each k, summing
// the blocks in index order, and re-arms the counter.
template <int NV>
__device__ void finish_reduction_n(const double v[NV], double *partials, unsigned int *counter,
                                   double *const out[NV], int accumulate, double scale) {
  __shared__ bool last;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < NV; ++k) partials[k * gridDim.x + blockIdx.x] = v[k];
    __threadfence();
    const unsigned int ticket = atomicAdd(counter, 1u);
    last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    double s = 0.0;
    for (unsigned int i = threadIdx.x; i < gridDim.x; i += blockDim.x)
      s += __ldcg(partials + k * gridDim.x + i);
    s = block_sum(s);
    if (threadIdx.x == 0) {
      const double prev = accumulate ? *out[k] : 0.0;
      *out[k] = prev + scale * s;
    }
  }
  if (threadIdx.x == 0) *counter = 0u;
}

__device__ void finish_reduction(double v, double *partials, unsigned int *counter,
                                 double *out, int accumulate, double scale) {
  double *const o[1] = {out};
  finish_reduction_n<1>(&v, partials, counter, o, accumulate, scale);
}

// As finish_reduction_n, but returns the NV grid totals (in thread 0 of the last block,
// which alone gets true) for a caller that combines them non-linearly.
template <int NV>
__device__ bool last_block_totals(const double v[NV], double *partials, unsigned int *counter,
                                  double tot[NV]) {
  __shared__ bool last;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < NV; ++k) partials[k * gridDim.x + blockIdx.x] = v[k];
    __threadfence();
    last = (atomicAdd(counter, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (!last) return false;
  __threadfence();
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    double s = 0.0;
    for (unsigned int i = threadIdx.x; i < gridDim.x; i += blockDim.x)
      s += __ldcg(partials + k * gridDim.x + i);
    s = block_sum(s);
    if (threadIdx.x == 0) tot[k] = s;
  }
  if (threadIdx.x == 0) *counter = 0u;
  return threadIdx.x == 0;
}

// L = 1/2 sum_j D_j P_j^2 with P_j = rd(theta_j + s*eps*z_j) computed on load.
//
// A persistent producer/consumer pipeline: warp 0 streams 4096-element chunks of theta and
// D into a ring of shared-memory stages with bulk asynchronous copies; the 8 consumer warps
// regenerate the chunk's sign bits (each lane one Philox block: the 16 elements of one
// group that its warp reads, shared through warp shuffles), apply the perturbation and
// accumulate in fp64 (four independent partial sums per thread), then release the stage.
// Chunks are assigned round-robin (chunk = blockIdx.x + k * gridDim.x), so the grid size
// and every summation order depend on M only: the result is deterministic.
constexpr int kQChunk = 4096;
constexpr int kQStages = 3;
constexpr int kQConsumers = 8;
constexpr int kQThreads = 32 * (1 + kQConsumers);
constexpr int kQStageBytes = 2 * kQChunk * 4;  // theta, D
constexpr int kQSmemBytes = kQStages * kQStageBytes + 2 * kQStages * 8;

// PAIR: both losses of one probe, L(theta + eps z) into out and L(theta - eps z) into
// out_minus, from one pass over theta and D (pk.sign must be +1); each sum follows exactly
// the order of a single-sign pass, so the results are bit-identical to two passes.
//
// R > 0 adds the low-rank term of the conditioning-study quadratic,
//   L = 1/2 sum_j D_j P_j^2 + 1/2 sum_k (lam_k / M) (v_k . P)^2   (k < R),
// with the directions v_k in {-1,+1}^M regenerated like the probes (probes 0..R-1 of step 0
// under their own key): the same pass accumulates the R dot products in fp64 and the last
// block combines the grid totals.
struct LowRankArgs {
  float lam[4];       // eigenvalue each direction adds (0 for unused directions)
  uint32_t vk0, vk1;  // Philox key of the directions
};

template <bool PAIR, int R>
__global__ void __launch_bounds__(kQThreads)
quad_loss_kernel(const float *__restrict__ theta, const float *__restrict__ D, int64_t M,
                 ProbeKey pk, int64_t n_chunks, double *partials, unsigned int *counter,
                 double *out, double *out_minus, int accumulate, uint32_t *err, LowRankArgs lr) {
  extern __shared__ __align__(128) uint8_t qsm[];
  uint64_t *full = reinterpret_cast<uint64_t *>(qsm + kQStages * kQStageBytes);
  uint64_t *empty = full + kQStages;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kQConsumers);
    }
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  const uint32_t step = pk.sign ? *pk.step : 0u;
  const float delta = pk.sign > 0 ? pk.eps : -pk.eps;
  double acc4[4] = {0.0, 0.0, 0.0, 0.0};
  double accm4[4] = {0.0, 0.0, 0.0, 0.0};  // PAIR: the -eps loss
  double dot[R > 0 ? R : 1], dotm[R > 0 ? R : 1];  // R > 0: v_k . P (and for the -eps side)
#pragma unroll
  for (int k = 0; k < (R > 0 ? R : 1); ++k) dot[k] = dotm[k] = 0.0;

  if (warp == 0) {  // producer
    int it = 0, issued = 0;
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x, ++it) {
      const int s = it % kQStages;
      const uint32_t ph = (uint32_t)(it / kQStages) & 1u;
      int ok = 1;
      if (lane == 0) ok = tc::mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok || abort_flag) {
        if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
        break;
      }
      uint8_t *st = qsm + s * kQStageBytes;
      const int64_t base = chunk * kQChunk;
      const int cnt = (int)(M - base < (int64_t)kQChunk ? M - base : (int64_t)kQChunk);
      const int copy = cnt & ~3;
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)copy * 4u);
        if (copy) {
          tc::bulk_load(st, theta + base, (uint32_t)copy * 4u, &full[s]);
          tc::bulk_load(st + kQChunk * 4, D + base, (uint32_t)copy * 4u, &full[s]);
        }
      }
      __syncwarp();
      issued = it + 1;
    }
    if (abort_flag && lane == 0) {  // let this CTA's copies land before it exits
      for (int s = 0; s < kQStages; ++s) {
        int last = -1;
        for (int i = s; i < issued; i += kQStages) last = i;
        if (last >= 0) tc::mbar_wait(&full[s], (uint32_t)(last / kQStages) & 1u);
      }
    }
  } else {  // consumers
    const int ct = threadIdx.x - 32;  // 0 .. 255
    const int cw = ct >> 5;           // consumer warp: elements 4 (32 cw + lane + 256 k) + 0..3
    int it = 0;
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x, ++it) {
      const int s = it % kQStages;
      const uint32_t ph = (uint32_t)(it / kQStages) & 1u;
      // lane 0 decides for the warp (all lanes leave together or none), then every lane
      // observes the completed phase itself (immediate once lane 0 has seen it)
      int ok = 1;
      if (lane == 0) ok = (!abort_flag && tc::mbar_wait(&full[s], ph)) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (ok && lane != 0) ok = tc::mbar_wait(&full[s], ph) ? 1 : 0;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
        break;
      }
      const uint8_t *st = qsm + s * kQStageBytes;
      const float *sT = reinterpret_cast<const float *>(st);
      const float *sD = reinterpret_cast<const float *>(st + kQChunk * 4);
      const int64_t base = chunk * kQChunk;
      const int cnt = (int)(M - base < (int64_t)kQChunk ? M - base : (int64_t)kQChunk);
      const int copy = cnt & ~3;
      // The warp's 32 groups: slot q = 8 k + j is group 8 cw + 64 k + j of the chunk; lane q
      // computes its 16 bits (groups past M are computed and never used).
      const uint64_t my_group = (uint64_t)(base / kGroup) + 8 * cw + 64 * (lane >> 3) + (lane & 7);
      uint32_t mine = 0u;
      if (pk.sign) mine = probe_group_bits(my_group, pk.probe, step, pk.k0, pk.k1);
      uint4 vmine = make_uint4(0u, 0u, 0u, 0u);
      if (R > 0) vmine = sign_block(my_group, 0u, 0u, lr.vk0, lr.vk1);
#pragma unroll
      for (int k = 0; k < kQChunk / (4 * 32 * kQConsumers); ++k) {
        const int e = 4 * (ct + k * 32 * kQConsumers);
        const int src = 8 * k + (lane >> 2);
        const uint32_t bits = pk.sign ? __shfl_sync(0xFFFFFFFFu, mine, src) >> (4 * (lane & 3)) : 0u;
        uint32_t vw = 0u;  // R > 0: the direction bytes of this thread's 4 elements
        if (R > 0) {
          const uint32_t w0 = __shfl_sync(0xFFFFFFFFu, vmine.x, src);
          const uint32_t w1 = __shfl_sync(0xFFFFFFFFu, vmine.y, src);
          const uint32_t w2 = __shfl_sync(0xFFFFFFFFu, vmine.z, src);
          const uint32_t w3 = __shfl_sync(0xFFFFFFFFu, vmine.w, src);
          const int q = lane & 3;
          vw = q == 0 ? w0 : q == 1 ? w1 : q == 2 ? w2 : w3;
        }
        if (e >= cnt) continue;
        float tv[4], dv[4];
        if (e + 4 <= copy) {
          const float4 t = reinterpret_cast<const float4 *>(sT)[e >> 2];
          const float4 dd = reinterpret_cast<const float4 *>(sD)[e >> 2];
          tv[0] = t.x; tv[1] = t.y; tv[2] = t.z; tv[3] = t.w;
          dv[0] = dd.x; dv[1] = dd.y; dv[2] = dd.z; dv[3] = dd.w;
        } else {  // the last < 4 elements of theta (not covered by the 16-byte copies)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool in = e + q < cnt;
            tv[q] = in ? theta[base + e + q] : 0.f;
            dv[q] = in ? D[base + e + q] : 0.f;
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p = pk.sign ? perturb_f32(tv[q], delta, (bits >> q) & 1u) : tv[q];
          const double pd = (double)p;
          const double hd = __dmul_rn(0.5, (double)dv[q]);
          acc4[q] = __dadd_rn(acc4[q], __dmul_rn(hd, __dmul_rn(pd, pd)));
          double pm = 0.0;
          if (PAIR) {
            pm = (double)perturb_f32(tv[q], -delta, (bits >> q) & 1u);
            accm4[q] = __dadd_rn(accm4[q], __dmul_rn(hd, __dmul_rn(pm, pm)));
          }
          if (R > 0 && e + q < cnt) {
            const uint32_t vb = vw >> (8 * q);
#pragma unroll
            for (int r = 0; r < (R > 0 ? R : 1); ++r) {
              const bool neg = (vb >> r) & 1u;
              dot[r] = __dadd_rn(dot[r], neg ? -pd : pd);
              if (PAIR) dotm[r] = __dadd_rn(dotm[r], neg ? -pm : pm);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[s]);
    }
  }
  double acc = __dadd_rn(__dadd_rn(acc4[0], acc4[1]), __dadd_rn(acc4[2], acc4[3]));
  double accm = __dadd_rn(__dadd_rn(accm4[0], accm4[1]), __dadd_rn(accm4[2], accm4[3]));
  // The next loss pass may start streaming now; the reduction scratch (partials, counter,
  // out) is touched only after the previous kernel in the stream has fully completed.
  tc::pdl_launch_dependents();
  tc::pdl_wait();
  if (R > 0) {
    constexpr int NS = PAIR ? 2 : 1, NV = NS * (1 + (R > 0 ? R : 1));
    double v[NV], tot[NV];
    v[0] = block_sum(acc);
#pragma unroll
    for (int r = 0; r < (R > 0 ? R : 1); ++r) v[1 + r] = block_sum(dot[r]);
    if (PAIR) {
      v[1 + R] = block_sum(accm);
#pragma unroll
      for (int r = 0; r < (R > 0 ? R : 1); ++r) v[2 + R + r] = block_sum(dotm[r]);
    }
    if (last_block_totals<NV>(v, partials, counter, tot)) {
      const double inv_m = 1.0 / (double)M;
#pragma unroll
      for (int sgn = 0; sgn < NS; ++sgn) {
        const double *t = tot + sgn * (1 + R);
        double L = t[0];
#pragma unroll
        for (int r = 0; r < (R > 0 ? R : 1); ++r)
          L = __dadd_rn(L, __dmul_rn(__dmul_rn(0.5 * (double)lr.lam[r], inv_m), __dmul_rn(t[1 + r], t[1 + r])));
        double *o = sgn == 0 ? out : out_minus;
        *o = (accumulate ? *o : 0.0) + L;
      }
    }
    return;
  }
  acc = block_sum(acc);
  if (PAIR) {
    accm = block_sum(accm);
    const double v[2] = {acc, accm};
    double *const o[2] = {out, out_minus};
    finish_reduction_n<2>(v, partials, counter, o, accumulate, 1.0);
  } else {
    finish_reduction(acc, partials, counter, out, accumulate, 1.0);
  }
}

constexpr int kMlpMax = 1024;

// One block per sample: h = ReLU(W1 x + b1), logits = W2 h + b2, CE(logits, y).
__global__ void __launch_bounds__(256)
mlp_loss_kernel(const float *__restrict__ P, const float *__restrict__ X,
                const int32_t *__restrict__ y, int n_in, int n_hidden, int n_out,
                double *partials, unsigned int *counter, double *out, int accumulate,
                double scale) {
  __shared__ float xs[kMlpMax], hs[kMlpMax], ls[kMlpMax];
  const float *W1 = P;
  const float *b1 = W1 + (int64_t)n_hidden * n_in;
  const float *W2 = b1 + n_hidden;
  const float *b2 = W2 + (int64_t)n_out * n_hidden;
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int k = threadIdx.x; k < n_in; k += blockDim.x) xs[k] = X[(int64_t)b * n_in + k];
  __syncthreads();
  for (int j = threadIdx.x; j < n_hidden; j += blockDim.x) {
    const float *w = W1 + (int64_t)j * n_in;
    float a = 0.f;
    for (int k = 0; k < n_in; ++k) a = fmaf(w[k], xs[k], a);
    a = __fadd_rn(a, b1[j]);
    hs[j] = a > 0.f ? a : 0.f;
  }
  __syncthreads();
  for (int o = warp; o < n_out; o += nw) {
    const float *w = W2 + (int64_t)o * n_hidden;
    float a = 0.f;
    for (int k = lane; k < n_hidden; k += 32) a = fmaf(w[k], hs[k], a);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) a += __shfl_down_sync(0xFFFFFFFFu, a, s);
    if (lane == 0) ls[o] = __fadd_rn(a, b2[o]);
  }
  __syncthreads();
  double ce = 0.0;
  if (threadIdx.x == 0) {
    float m = ls[0];
    for (int o = 1; o < n_out; ++o) m = fmaxf(m, ls[o]);
    float s = 0.f;
    for (int o = 0; o < n_out; ++o) s += expf(ls[o] - m);
    const int label = y[b];
    // an out-of-range label poisons the loss (the step is then skipped as non-finite)
    ce = (label >= 0 && label < n_out) ? (double)(m + logf(s)) - (double)ls[label] : (double)NAN;
  }
  finish_reduction(ce, partials, counter, out, accumulate, scale);
}

}  // namespace

namespace {

template <bool PAIR, int R>
zo_status launch_quad(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out,
                      double *out_minus, int accumulate, double *partials, unsigned int *counter,
                      const LowRankArgs &lr = LowRankArgs{}) {
  const int64_t n_chunks = (ctx->M + kQChunk - 1) / kQChunk;
  int64_t blocks = n_chunks < (int64_t)kSmCount * 2 ? n_chunks : (int64_t)kSmCount * 2;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(quad_loss_kernel<PAIR, R>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "quad_loss_kernel attribute: %s", cudaGetErrorString(e));
    attr = true;
  }
  // Programmatic dependent launch: this pass may begin while the previous loss pass of
  // the stream finishes its reduction (see pdl_wait in the kernel).  Kernels that write
  // theta or the step counter never signal early, so they still complete first.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = kQSmemBytes;
  cfg.stream = ctx->stream;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, quad_loss_kernel<PAIR, R>,
                                           static_cast<const float *>(ctx->params), D, ctx->M, pk,
                                           n_chunks, partials, counter, out, out_minus, accumulate,
                                           &ctx->dstate->flags, lr);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "quad_loss_kernel: %s", cudaGetErrorString(e));
  return check_launch(ctx, "quad_loss_kernel");
}

}  // namespace

zo_status launch_quad_loss(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out,
                           int accumulate, double *partials, unsigned int *counter) {
  return launch_quad<false, 0>(ctx, pk, D, out, nullptr, accumulate, partials, counter);
}

zo_status launch_quad_loss_pair(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out_plus,
                                double *out_minus) {
  return launch_quad<true, 0>(ctx, pk, D, out_plus, out_minus, 0, ctx->partials, ctx->counter);
}

zo_status launch_lowrank_loss(zo_ctx *ctx, const ProbeKey &pk, const float *D, const float lam[4],
                              uint64_t vseed, double *out, double *out_minus, int accumulate) {
  LowRankArgs lr;
  for (int k = 0; k < 4; ++k) lr.lam[k] = lam[k];
  lr.vk0 = (uint32_t)vseed;
  lr.vk1 = (uint32_t)(vseed >> 32);
  if (out_minus)
    return launch_quad<true, 4>(ctx, pk, D, out, out_minus, 0, ctx->partials, ctx->counter, lr);
  return launch_quad<false, 4>(ctx, pk, D, out, nullptr, accumulate, ctx->partials, ctx->counter, lr);
}

zo_status launch_mlp_loss(zo_ctx *ctx, const float *P, const float *X, const int32_t *y,
                          int batch, int n_in, int n_hidden, int n_out, double scale,
                          double *out, int accumulate) {
  if (n_in > kMlpMax || n_hidden > kMlpMax || n_out > kMlpMax || batch > kMaxPartials)
    return fail(ctx, ZO_ERR_INVALID, "mlp shape beyond limits");
  mlp_loss_kernel<<<batch, 256, 0, ctx->stream>>>(P, X, y, n_in, n_hidden, n_out, ctx->partials,
                                                  ctx->counter, out, accumulate, scale);
  return check_launch(ctx, "mlp_loss_kernel");
}

}  // namespace zo

// ------------------------------------------------------------------ allocation-free MLP loss
// For callers that cannot allocate device memory: the same mlp_loss_kernel, with its
// per-sample partials and ticket counter in a static device array of this module instead
// of a context's cudaMalloc'd scratch.

namespace zo {
namespace {

constexpr size_t kNoallocPartialsBytes = (size_t)ZO_NOALLOC_MAX_BATCH * sizeof(double);
constexpr int kNoallocMaxDevices = 64;

// [0, kNoallocPartialsBytes): fp64 partials; then the unsigned ticket counter.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocPartialsBytes + 256];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoallocMaxDevices] = {};

// Device address of the scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up once per device.
cudaError_t noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoallocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace zo

extern "C" zo_status zo_mlp_loss_noalloc(const float *P, const float *X, const int32_t *labels,
                                         int batch, int n_in, int n_hidden, int n_out,
                                         double scale, double *loss_out, int accumulate,
                                         void *stream) {
  using namespace zo;
  if (!P || !X || !labels || !loss_out || batch < 1 || n_in < 1 || n_hidden < 1 || n_out < 1 ||
      n_in > kMlpMax || n_hidden > kMlpMax || n_out > kMlpMax || batch > ZO_NOALLOC_MAX_BATCH)
    return ZO_ERR_INVALID;
  void *base = nullptr;
  if (noalloc_scratch(&base) != cudaSuccess) {
    cudaGetLastError();
    return ZO_ERR_CUDA;
  }
  double *partials = static_cast<double *>(base);
  unsigned int *counter =
      reinterpret_cast<unsigned int *>(static_cast<unsigned char *>(base) + kNoallocPartialsBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counter, 0, sizeof(unsigned int), s) != cudaSuccess) {
    cudaGetLastError();
    return ZO_ERR_CUDA;
  }
  mlp_loss_kernel<<<batch, 256, 0, s>>>(P, X, labels, n_in, n_hidden, n_out, partials, counter,
                                        loss_out, accumulate, scale);
  if (cudaGetLastError() != cudaSuccess) return ZO_ERR_CUDA;
  return ZO_OK;
}
