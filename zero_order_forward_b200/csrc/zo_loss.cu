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

// Block `blockIdx.x` contributes `v` (valid in thread 0); the last block writes
// out = (accumulate ? out : 0) + scale * sum(partials[0..gridDim.x)) and re-arms counter.
__device__ void finish_reduction(double v, double *partials, unsigned int *counter,
                                 double *out, int accumulate, double scale) {
  __shared__ bool last;
  if (threadIdx.x == 0) {
    partials[blockIdx.x] = v;
    __threadfence();
    const unsigned int ticket = atomicAdd(counter, 1u);
    last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  double s = 0.0;
  for (unsigned int i = threadIdx.x; i < gridDim.x; i += blockDim.x) s += __ldcg(partials + i);
  s = block_sum(s);
  if (threadIdx.x == 0) {
    const double prev = accumulate ? *out : 0.0;
    *out = prev + scale * s;
    *counter = 0u;
  }
}

// L = 1/2 sum_j D_j P_j^2 with P_j = rd(theta_j + s*eps*z_j) computed on load.
__global__ void __launch_bounds__(kWarps * 32)
quad_loss_kernel(const float *__restrict__ theta, const float *__restrict__ D, int64_t M,
                 ProbeKey pk, int64_t n_tiles, double *partials, unsigned int *counter,
                 double *out, int accumulate) {
  constexpr int N = 4;
  constexpr int kIters = kTileElems / (32 * N);
  __shared__ uint4 blocks[kWarps][kTileGroups];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t step = pk.sign ? *pk.step : 0u;
  const float delta = pk.sign > 0 ? pk.eps : -pk.eps;
  const uint32_t *bw = reinterpret_cast<const uint32_t *>(blocks[warp]);
  double acc = 0.0;

  for (int64_t tile = (int64_t)blockIdx.x * kWarps + warp; tile < n_tiles;
       tile += (int64_t)gridDim.x * kWarps) {
    const int64_t base = tile * kTileElems;
    if (pk.sign) {
      const int64_t g = tile * kTileGroups + lane;
      if (g * kGroup < M) blocks[warp][lane] = probe_block(g, pk.probe, step, pk.k0, pk.k1);
      __syncwarp();
    }
#pragma unroll 4
    for (int k = 0; k < kIters; ++k) {
      const int e_rel = (k * 32 + lane) * N;
      const int64_t e = base + e_rel;
      uint32_t bits = 0;
      if (pk.sign) bits = bw[(e_rel >> 7) * 4 + ((e_rel >> 5) & 3)] >> (e_rel & 31);
      if (e + N <= M) {
        const float4 t = __ldcs(reinterpret_cast<const float4 *>(theta + e));
        const float4 d = __ldcs(reinterpret_cast<const float4 *>(D + e));
        const float tv[4] = {t.x, t.y, t.z, t.w}, dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p = pk.sign ? perturb_f32(tv[q], delta, (bits >> q) & 1u) : tv[q];
          const double pd = (double)p;
          acc = __dadd_rn(acc, __dmul_rn(__dmul_rn(0.5, (double)dv[q]), __dmul_rn(pd, pd)));
        }
      } else {
        for (int q = 0; q < N; ++q) {
          if (e + q >= M) break;
          const float tq = theta[e + q];
          const float p = pk.sign ? perturb_f32(tq, delta, (bits >> q) & 1u) : tq;
          const double pd = (double)p;
          acc = __dadd_rn(acc, __dmul_rn(__dmul_rn(0.5, (double)D[e + q]), __dmul_rn(pd, pd)));
        }
      }
    }
    if (pk.sign) __syncwarp();
  }
  acc = block_sum(acc);
  finish_reduction(acc, partials, counter, out, accumulate, 1.0);
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

zo_status launch_quad_loss(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out,
                           int accumulate, double *partials, unsigned int *counter) {
  const int64_t n_tiles = (ctx->M + kTileElems - 1) / kTileElems;
  int64_t blocks = (n_tiles + kWarps - 1) / kWarps;
  if (blocks > (int64_t)kSmCount * 4) blocks = (int64_t)kSmCount * 4;
  quad_loss_kernel<<<(unsigned)blocks, kWarps * 32, 0, ctx->stream>>>(
      static_cast<const float *>(ctx->params), D, ctx->M, pk, n_tiles, partials, counter, out,
      accumulate);
  return check_launch(ctx, "quad_loss_kernel");
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
