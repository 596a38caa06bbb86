// zo_core.cu -- the C ABI of libzo.so: context, perturbation state machine, argument
// checking, and the step drivers that order the kernels of one step.
//
// Step order ("Pretraining Transformers Without Backprop: What Two Zero-Order Papers
// Actually Measure", section "Backprop's memory tax", loop flowchart; the clean pass of
// 1.5-SPSA from "Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section
// "Probe-Space Preconditioning"):
//   clean loss L0 -> for each probe i: loss at theta+eps z_i, loss at theta-eps z_i ->
//   preconditioner -> update (step counter + 1).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>

#include <mutex>
#include <utility>
#include <vector>

#include "zo_internal.cuh"

namespace zo {

zo_status fail(zo_ctx *ctx, zo_status st, const char *fmt, ...) {
  if (ctx) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    ctx->err = buf;
  }
  return st;
}

zo_status check_launch(zo_ctx *ctx, const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(ctx, ZO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  ctx->launches += 1;
  return ZO_OK;
}

ProbeKey probe_key(const zo_ctx *ctx) {
  ProbeKey pk;
  pk.k0 = (uint32_t)ctx->seed;
  pk.k1 = (uint32_t)(ctx->seed >> 32);
  pk.step = &ctx->dstate->step;
  pk.probe = (uint32_t)ctx->probe;
  pk.sign = ctx->state == PState::Perturbed ? ctx->sign : 0;
  pk.eps = ctx->eps;
  pk.g_off = (uint64_t)(ctx->first_element / kGroup);
  return pk;
}

cudaError_t ensure_smem_limit(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void *, int>> done;  // (kernel, device)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto &d : done)
    if (d.first == kernel && d.second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.emplace_back(kernel, dev);
  else cudaGetLastError();  // reported by the caller; not left for a later launch check
  return e;
}

void phase_mark(zo_ctx *ctx, int which) {
  if (!ctx->phase_ev || ctx->phase_used >= ctx->phase_cap) return;
  cudaEventRecord(ctx->phase_ev[4 * ctx->phase_used + which], ctx->stream);
  if (which == 3) ctx->phase_used += 1;
}

// At most this many launches are recorded between two drains (zo_kernel_times); later ones
// are counted as dropped.
constexpr size_t kKtimeMaxRecords = 1u << 16;

int ktime_begin(zo_ctx *ctx) {
  if (!ctx->ktime_on) return -1;
  const size_t k = ctx->ktime_recs.size();
  if (k >= kKtimeMaxRecords) {
    ctx->ktime_dropped += 1;
    return -1;
  }
  while (ctx->ktime_ev.size() < 2 * (k + 1)) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) {
      cudaGetLastError();
      ctx->ktime_dropped += 1;
      return -1;
    }
    ctx->ktime_ev.push_back(ev);
  }
  if (cudaEventRecord(ctx->ktime_ev[2 * k], ctx->stream) != cudaSuccess) {
    cudaGetLastError();
    ctx->ktime_dropped += 1;
    return -1;
  }
  ctx->ktime_recs.push_back({-1, 0.0});
  return (int)k;
}

void ktime_end(zo_ctx *ctx, int slot, int cls, double work) {
  if (slot < 0) return;
  if (cudaEventRecord(ctx->ktime_ev[2 * (size_t)slot + 1], ctx->stream) != cudaSuccess) {
    cudaGetLastError();
    return;  // the record keeps class -1 and is skipped by the drain
  }
  ctx->ktime_recs[(size_t)slot] = {cls, work};
}

}  // namespace zo

using namespace zo;

namespace {
zo_status check_step_args(zo_ctx *ctx, int32_t n, float lr, float eps, float damping);
}

zo_status zo::step_device(zo_ctx *ctx, const double *loss_plus, const double *loss_minus,
                          int32_t n_pert, const double *loss0, float lr, float eps, float damping) {
  {
    const zo_status s0 = check_step_args(ctx, n_pert, lr, eps, damping);
    if (s0 != ZO_OK) return s0;
  }
  if (!loss_plus || !loss_minus) return fail(ctx, ZO_ERR_INVALID, "null loss arrays");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "zo_step while perturbed");
  const zo_status st = launch_precond(ctx, loss_plus, loss_minus, loss0, n_pert, lr, eps, damping);
  if (st != ZO_OK) return st;
  return launch_update(ctx, ctx->coef, n_pert, &ctx->dstate->upd_step, &ctx->dstate->upd_ok);
}

namespace {

size_t elem_size(int dtype) { return dtype == ZO_F32 ? 4 : 2; }

zo_status cuda_fail(zo_ctx *ctx, cudaError_t e, const char *what) {
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    return fail(ctx, ZO_ERR_OOM, "%s: out of device memory", what);
  }
  return fail(ctx, ZO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define ZO_CUDA(ctx, call, what)                      \
  do {                                                \
    const cudaError_t e_ = (call);                    \
    if (e_ != cudaSuccess) return cuda_fail(ctx, e_, what); \
  } while (0)

#define ZO_CHECK(expr)                 \
  do {                                 \
    const zo_status s_ = (expr);       \
    if (s_ != ZO_OK) return s_;        \
  } while (0)

zo_status check_ctx(zo_ctx *ctx) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  ZO_CUDA(ctx, cudaSetDevice(ctx->device), "cudaSetDevice");
  return ZO_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

zo_status check_step_args(zo_ctx *ctx, int32_t n, float lr, float eps, float damping) {
  if (n < 1 || n > ZO_MAX_PROBES)
    return fail(ctx, ZO_ERR_INVALID, "n_pert=%d outside [1, %d]", n, ZO_MAX_PROBES);
  if (!(eps > 0.f) || !std::isfinite(eps)) return fail(ctx, ZO_ERR_INVALID, "eps must be finite and > 0");
  if (!std::isfinite(lr)) return fail(ctx, ZO_ERR_INVALID, "lr must be finite");
  if (!(damping >= 0.f) || !std::isfinite(damping))
    return fail(ctx, ZO_ERR_INVALID, "damping must be finite and >= 0");
  return ZO_OK;
}

}  // namespace

extern "C" {

const char *zo_status_name(int s) {
  switch (s) {
    case ZO_OK: return "ZO_OK";
    case ZO_ERR_INVALID: return "ZO_ERR_INVALID";
    case ZO_ERR_STATE: return "ZO_ERR_STATE";
    case ZO_ERR_CUDA: return "ZO_ERR_CUDA";
    case ZO_ERR_OOM: return "ZO_ERR_OOM";
    case ZO_ERR_NONFINITE: return "ZO_ERR_NONFINITE";
    case ZO_ERR_UNSUPPORTED: return "ZO_ERR_UNSUPPORTED";
    case ZO_ERR_TIMEOUT: return "ZO_ERR_TIMEOUT";
    default: return "ZO_ERR_UNKNOWN";
  }
}

const char *zo_last_error(const zo_ctx *ctx) { return ctx ? ctx->err.c_str() : "null context"; }

zo_status zo_create(zo_ctx **out, void *params, int64_t M, int dtype, uint64_t seed,
                    void *stream) {
  if (!out) return ZO_ERR_INVALID;
  *out = nullptr;
  if (!params || M < 1 || M >= ((int64_t)1 << 39) || (dtype != ZO_F32 && dtype != ZO_BF16) ||
      !aligned16(params))
    return ZO_ERR_INVALID;
  zo_ctx *ctx = new (std::nothrow) zo_ctx();
  if (!ctx) return ZO_ERR_OOM;
  ctx->params = params;
  ctx->M = M;
  ctx->dtype = dtype;
  ctx->seed = seed;
  ctx->stream = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e == cudaSuccess) e = cudaMalloc(&ctx->dstate, sizeof(DevState));
  if (e == cudaSuccess) e = cudaMalloc(&ctx->coef, ZO_MAX_PROBES * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc(&ctx->diag, (3 * ZO_MAX_PROBES + 8) * sizeof(double));
  if (e == cudaSuccess) e = cudaMalloc(&ctx->partials, (kMaxPartials + 8) * sizeof(double));
  if (e == cudaSuccess) e = cudaMalloc(&ctx->counter, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->dstate, 0, sizeof(DevState), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->counter, 0, sizeof(unsigned int), ctx->stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctx->diag, 0, (3 * ZO_MAX_PROBES + 8) * sizeof(double), ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  if (e != cudaSuccess) {
    const zo_status st = e == cudaErrorMemoryAllocation ? ZO_ERR_OOM : ZO_ERR_CUDA;
    cudaGetLastError();
    zo_destroy(ctx);
    return st;
  }
  *out = ctx;
  return ZO_OK;
}

zo_status zo_destroy(zo_ctx *ctx) {
  if (!ctx) return ZO_OK;
  cudaSetDevice(ctx->device);
  cudaStreamSynchronize(ctx->stream);
  cudaFree(ctx->dstate);
  cudaFree(ctx->coef);
  cudaFree(ctx->diag);
  cudaFree(ctx->partials);
  cudaFree(ctx->counter);
  cudaFree(ctx->live);
  cudaFree(ctx->staging);
  cudaFree(ctx->loss_scratch);
  cudaFree(ctx->mlp_ce);
  cudaFree(ctx->lowrank_scratch);
  if (ctx->copy_stream) cudaStreamSynchronize(ctx->copy_stream);
  for (int b = 0; b < 2; ++b) {
    cudaFree(ctx->pipe_d[b]);
    cudaFree(ctx->pipe_l[b]);
    if (ctx->pipe_copied[b]) cudaEventDestroy(ctx->pipe_copied[b]);
    if (ctx->pipe_consumed[b]) cudaEventDestroy(ctx->pipe_consumed[b]);
  }
  if (ctx->copy_stream) cudaStreamDestroy(ctx->copy_stream);
  if (ctx->phase_ev) {
    for (int i = 0; i < 4 * ctx->phase_cap; ++i) cudaEventDestroy(ctx->phase_ev[i]);
    delete[] ctx->phase_ev;
  }
  for (cudaEvent_t ev : ctx->ktime_ev) cudaEventDestroy(ev);
  delete ctx;
  return ZO_OK;
}

zo_status zo_enable_phase_timing(zo_ctx *ctx, int32_t n_steps) {
  ZO_CHECK(check_ctx(ctx));
  if (n_steps < 0 || n_steps > 4096) return fail(ctx, ZO_ERR_INVALID, "n_steps outside [0, 4096]");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  if (ctx->phase_ev) {
    for (int i = 0; i < 4 * ctx->phase_cap; ++i) cudaEventDestroy(ctx->phase_ev[i]);
    delete[] ctx->phase_ev;
    ctx->phase_ev = nullptr;
  }
  ctx->phase_cap = ctx->phase_used = 0;
  if (n_steps == 0) return ZO_OK;
  ctx->phase_ev = new (std::nothrow) cudaEvent_t[4 * n_steps];
  if (!ctx->phase_ev) return fail(ctx, ZO_ERR_OOM, "phase events");
  for (int i = 0; i < 4 * n_steps; ++i) {
    const cudaError_t e = cudaEventCreate(&ctx->phase_ev[i]);
    if (e != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ctx->phase_ev[j]);
      delete[] ctx->phase_ev;
      ctx->phase_ev = nullptr;
      return cuda_fail(ctx, e, "cudaEventCreate");
    }
  }
  ctx->phase_cap = n_steps;
  return ZO_OK;
}

zo_status zo_phase_times(zo_ctx *ctx, int32_t n_steps, float *ms) {
  ZO_CHECK(check_ctx(ctx));
  if (!ms || n_steps < 1 || n_steps > ctx->phase_used)
    return fail(ctx, ZO_ERR_INVALID, "only %d steps were recorded", ctx->phase_used);
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  for (int k = 0; k < n_steps; ++k)
    for (int p = 0; p < 3; ++p)
      ZO_CUDA(ctx, cudaEventElapsedTime(&ms[3 * k + p], ctx->phase_ev[4 * k + p],
                                        ctx->phase_ev[4 * k + p + 1]), "cudaEventElapsedTime");
  return ZO_OK;
}

zo_status zo_enable_kernel_timing(zo_ctx *ctx, int enable) {
  ZO_CHECK(check_ctx(ctx));
  ctx->ktime_on = enable != 0;
  return ZO_OK;
}

zo_status zo_kernel_times(zo_ctx *ctx, zo_kernel_time *out, int64_t *dropped) {
  ZO_CHECK(check_ctx(ctx));
  if (!out) return fail(ctx, ZO_ERR_INVALID, "null output");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  for (int c = 0; c < ZO_KT_COUNT; ++c) out[c] = zo_kernel_time{0.0, 0, 0.0};
  zo_status st = ZO_OK;
  for (size_t k = 0; k < ctx->ktime_recs.size(); ++k) {
    const auto &r = ctx->ktime_recs[k];
    if (r.cls < 0 || r.cls >= ZO_KT_COUNT) continue;
    float ms = 0.f;
    const cudaError_t e = cudaEventElapsedTime(&ms, ctx->ktime_ev[2 * k], ctx->ktime_ev[2 * k + 1]);
    if (e != cudaSuccess) {
      st = cuda_fail(ctx, e, "cudaEventElapsedTime");
      break;
    }
    out[r.cls].ms += ms;
    out[r.cls].launches += 1;
    out[r.cls].work += r.work;
  }
  if (dropped) *dropped = ctx->ktime_dropped;
  ctx->ktime_recs.clear();
  ctx->ktime_dropped = 0;
  return st;
}

zo_status zo_launch_count(zo_ctx *ctx, int64_t *count) {
  if (!ctx || !count) return ZO_ERR_INVALID;
  *count = ctx->launches;
  return ZO_OK;
}

zo_status zo_set_loss_location(zo_ctx *ctx, int on_device) {
  ZO_CHECK(check_ctx(ctx));
  ctx->host_losses = on_device == 0;
  return ZO_OK;
}

zo_status zo_set_alpha(zo_ctx *ctx, float alpha) {
  ZO_CHECK(check_ctx(ctx));
  if (!std::isfinite(alpha) || alpha < 0.f) return fail(ctx, ZO_ERR_INVALID, "alpha must be finite and >= 0");
  ctx->alpha = alpha;
  return ZO_OK;
}

zo_status zo_set_live_buffer(zo_ctx *ctx, int enable) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "live buffer can only change when clean");
  if (enable && !ctx->live) {
    ZO_CUDA(ctx, cudaMalloc(&ctx->live, (size_t)ctx->M * elem_size(ctx->dtype)), "live buffer");
  } else if (!enable && ctx->live) {
    ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
    cudaFree(ctx->live);
    ctx->live = nullptr;
  }
  ctx->live_enabled = enable != 0;
  return ZO_OK;
}

const void *zo_live_params(const zo_ctx *ctx) {
  if (!ctx) return nullptr;
  if (ctx->state == PState::Perturbed && ctx->live_enabled) return ctx->live;
  return ctx->params;
}

zo_status zo_sync(zo_ctx *ctx, uint32_t *flags) {
  ZO_CHECK(check_ctx(ctx));
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "cudaStreamSynchronize");
  DevState s;
  ZO_CUDA(ctx, cudaMemcpy(&s, ctx->dstate, sizeof s, cudaMemcpyDeviceToHost), "read state");
  if (s.flags) {
    ZO_CUDA(ctx, cudaMemset(&ctx->dstate->flags, 0, sizeof(uint32_t)), "clear flags");
  }
  if (flags) *flags = s.flags;
  if (s.flags & ZO_FLAG_TIMEOUT) return fail(ctx, ZO_ERR_TIMEOUT, "a kernel gave up a bounded wait");
  if (s.flags & ZO_FLAG_NONFINITE) return fail(ctx, ZO_ERR_NONFINITE, "a loss was not finite; step skipped");
  return ZO_OK;
}

zo_status zo_get_step(zo_ctx *ctx, uint32_t *step) {
  ZO_CHECK(check_ctx(ctx));
  if (!step) return fail(ctx, ZO_ERR_INVALID, "null step");
  ZO_CUDA(ctx, cudaMemcpyAsync(step, &ctx->dstate->step, sizeof(uint32_t), cudaMemcpyDeviceToHost,
                               ctx->stream), "read step");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  return ZO_OK;
}

zo_status zo_set_step(zo_ctx *ctx, uint32_t step) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "set_step while perturbed");
  static_assert(sizeof(uint32_t) == 4, "");
  // cuMemsetD32-style enqueue through a tiny host->device copy of a pinned-free value.
  ZO_CUDA(ctx, cudaMemcpyAsync(&ctx->dstate->step, &step, sizeof step, cudaMemcpyHostToDevice,
                               ctx->stream), "write step");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  return ZO_OK;
}

zo_status zo_set_element_offset(zo_ctx *ctx, int64_t first_element) {
  ZO_CHECK(check_ctx(ctx));
  if (first_element < 0 || first_element % kGroup)
    return fail(ctx, ZO_ERR_INVALID, "element offset must be a non-negative multiple of %d", kGroup);
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "element offset set while perturbed");
  ctx->first_element = first_element;
  return ZO_OK;
}

zo_status zo_pack_probe(zo_ctx *ctx, uint32_t step, int32_t probe, int64_t first_byte,
                        int64_t nbytes, uint8_t *dev_out) {
  ZO_CHECK(check_ctx(ctx));
  const int64_t total = (ctx->M + 7) / 8;
  if (probe < 0 || !dev_out || first_byte < 0 || nbytes < 0 || first_byte + nbytes > total)
    return fail(ctx, ZO_ERR_INVALID, "pack range outside [0, %lld) bytes", (long long)total);
  return launch_pack(ctx, step, (uint32_t)probe, first_byte, nbytes, dev_out);
}

zo_status zo_perturb(zo_ctx *ctx, int sign, float eps, int32_t probe) {
  ZO_CHECK(check_ctx(ctx));
  if (sign != 1 && sign != -1) return fail(ctx, ZO_ERR_INVALID, "sign must be +1 or -1");
  if (!(eps > 0.f) || !std::isfinite(eps)) return fail(ctx, ZO_ERR_INVALID, "eps must be finite and > 0");
  if (probe < 0) return fail(ctx, ZO_ERR_INVALID, "probe must be >= 0");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "already perturbed; call zo_restore first");
  ctx->state = PState::Perturbed;
  ctx->sign = sign;
  ctx->eps = eps;
  ctx->probe = probe;
  if (ctx->live_enabled) {
    const zo_status st = launch_perturb(ctx, probe_key(ctx), 0, ctx->M, ctx->live);
    if (st != ZO_OK) {
      ctx->state = PState::Clean;
      return st;
    }
  }
  return ZO_OK;
}

zo_status zo_restore(zo_ctx *ctx) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->state != PState::Perturbed) return fail(ctx, ZO_ERR_STATE, "not perturbed");
  ctx->state = PState::Clean;
  ctx->sign = 0;
  return ZO_OK;
}

zo_status zo_perturb_range(zo_ctx *ctx, int64_t first, int64_t count, void *dev_out) {
  ZO_CHECK(check_ctx(ctx));
  if (!dev_out || first < 0 || count < 0 || first + count > ctx->M)
    return fail(ctx, ZO_ERR_INVALID, "range outside [0, M)");
  return launch_perturb(ctx, probe_key(ctx), first, count, dev_out);
}

zo_status zo_quad_loss(zo_ctx *ctx, const float *D, double *loss_out, int accumulate) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "quadratic loss needs an fp32 context");
  if (!D || !loss_out || !aligned16(D)) return fail(ctx, ZO_ERR_INVALID, "D must be a 16-byte aligned device pointer");
  return launch_quad_loss(ctx, probe_key(ctx), D, loss_out, accumulate, ctx->partials, ctx->counter);
}

zo_status zo_quad_loss_pair(zo_ctx *ctx, const float *D, int32_t probe, float eps,
                            double *loss_plus, double *loss_minus) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "quadratic loss needs an fp32 context");
  if (!D || !loss_plus || !loss_minus || !aligned16(D))
    return fail(ctx, ZO_ERR_INVALID, "D must be a 16-byte aligned device pointer; outputs non-null");
  if (probe < 0 || !(eps > 0.f) || !std::isfinite(eps)) return fail(ctx, ZO_ERR_INVALID, "bad probe or eps");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "pair evaluation needs the clean state");
  ProbeKey pk = probe_key(ctx);
  pk.sign = +1;
  pk.probe = (uint32_t)probe;
  pk.eps = eps;
  return launch_quad_loss_pair(ctx, pk, D, loss_plus, loss_minus);
}

zo_status zo_mlp_loss(zo_ctx *ctx, const float *X, const int32_t *labels, int batch, int n_in,
                      int n_hidden, int n_out, double scale, double *loss_out, int accumulate) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "MLP loss: not separable over parameter slices (element offset must be 0)");
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "MLP loss needs an fp32 context");
  if (!X || !labels || !loss_out || batch < 1 || n_in < 1 || n_hidden < 1 || n_out < 1)
    return fail(ctx, ZO_ERR_INVALID, "bad MLP arguments");
  const int64_t need = (int64_t)n_hidden * n_in + n_hidden + (int64_t)n_out * n_hidden + n_out;
  if (need != ctx->M) return fail(ctx, ZO_ERR_INVALID, "MLP shape needs M=%lld", (long long)need);
  if (ctx->state == PState::Perturbed && !ctx->live_enabled)
    return fail(ctx, ZO_ERR_STATE, "perturbed MLP loss needs the live buffer");
  return launch_mlp_loss(ctx, static_cast<const float *>(zo_live_params(ctx)), X, labels, batch,
                         n_in, n_hidden, n_out, scale, loss_out, accumulate);
}

zo_status zo_step(zo_ctx *ctx, const double *loss_plus, const double *loss_minus, int32_t n_pert,
                  const double *loss0, float lr, float eps, float damping) {
  ZO_CHECK(check_ctx(ctx));
  if (!ctx->host_losses) return step_device(ctx, loss_plus, loss_minus, n_pert, loss0, lr, eps, damping);
  // host losses: staged into the context's loss scratch [L0, L+..., L-...] on its stream
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!loss_plus || !loss_minus) return fail(ctx, ZO_ERR_INVALID, "null loss arrays");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "zo_step while perturbed");
  if (!ctx->loss_scratch)
    ZO_CUDA(ctx, cudaMalloc(&ctx->loss_scratch, (2 * ZO_MAX_PROBES + 1) * sizeof(double)), "loss scratch");
  double *L0 = ctx->loss_scratch, *Lp = L0 + 1, *Lm = L0 + 1 + n_pert;
  const size_t nb = (size_t)n_pert * sizeof(double);
  ZO_CUDA(ctx, cudaMemcpyAsync(Lp, loss_plus, nb, cudaMemcpyHostToDevice, ctx->stream), "copy L+");
  ZO_CUDA(ctx, cudaMemcpyAsync(Lm, loss_minus, nb, cudaMemcpyHostToDevice, ctx->stream), "copy L-");
  if (loss0)
    ZO_CUDA(ctx, cudaMemcpyAsync(L0, loss0, sizeof(double), cudaMemcpyHostToDevice, ctx->stream), "copy L0");
  // the copies read host memory that the caller may reuse once zo_step returns
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  return step_device(ctx, Lp, Lm, n_pert, loss0 ? L0 : nullptr, lr, eps, damping);
}

zo_status zo_update(zo_ctx *ctx, const float *coef, int32_t n_pert) {
  ZO_CHECK(check_ctx(ctx));
  if (n_pert < 1 || n_pert > ZO_MAX_PROBES) return fail(ctx, ZO_ERR_INVALID, "n_pert out of range");
  if (!coef) return fail(ctx, ZO_ERR_INVALID, "null coefficients");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "zo_update while perturbed");
  return launch_update(ctx, coef, n_pert, &ctx->dstate->step, nullptr);
}

zo_status zo_get_precond(zo_ctx *ctx, int32_t n, double *g, double *c, double *w, float *a) {
  ZO_CHECK(check_ctx(ctx));
  if (n < 1 || n > ctx->last_n) return fail(ctx, ZO_ERR_INVALID, "n outside [1, last n_pert]");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  if (g) ZO_CUDA(ctx, cudaMemcpy(g, ctx->diag, n * sizeof(double), cudaMemcpyDeviceToHost), "g");
  if (c) ZO_CUDA(ctx, cudaMemcpy(c, ctx->diag + ZO_MAX_PROBES, n * sizeof(double), cudaMemcpyDeviceToHost), "c");
  if (w) ZO_CUDA(ctx, cudaMemcpy(w, ctx->diag + 2 * ZO_MAX_PROBES, n * sizeof(double), cudaMemcpyDeviceToHost), "w");
  if (a) ZO_CUDA(ctx, cudaMemcpy(a, ctx->coef, n * sizeof(float), cudaMemcpyDeviceToHost), "a");
  return ZO_OK;
}

namespace {
zo_status check_lowrank(zo_ctx *ctx, const float *D, const zo_lowrank *q, float lam[4]) {
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "quadratic loss needs an fp32 context");
  if (!D || !aligned16(D)) return fail(ctx, ZO_ERR_INVALID, "D must be a 16-byte aligned device pointer");
  if (!q || q->rank < 1 || q->rank > 4) return fail(ctx, ZO_ERR_INVALID, "rank must be 1..4");
  for (int k = 0; k < 4; ++k) {
    lam[k] = k < q->rank ? q->lam[k] : 0.f;
    if (!std::isfinite(lam[k])) return fail(ctx, ZO_ERR_INVALID, "non-finite eigenvalue");
  }
  return ZO_OK;
}
}  // namespace

zo_status zo_lowrank_loss(zo_ctx *ctx, const float *D, const zo_lowrank *q, double *loss_out,
                          int accumulate) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "low-rank loss: not separable over parameter slices (element offset must be 0)");
  float lam[4];
  ZO_CHECK(check_lowrank(ctx, D, q, lam));
  if (!loss_out) return fail(ctx, ZO_ERR_INVALID, "null loss_out");
  return launch_lowrank_loss(ctx, probe_key(ctx), D, lam, q->vseed, loss_out, nullptr, accumulate);
}

zo_status zo_lowrank_loss_pair(zo_ctx *ctx, const float *D, const zo_lowrank *q, int32_t probe,
                               float eps, double *loss_plus, double *loss_minus) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "low-rank loss: not separable over parameter slices (element offset must be 0)");
  float lam[4];
  ZO_CHECK(check_lowrank(ctx, D, q, lam));
  if (!loss_plus || !loss_minus) return fail(ctx, ZO_ERR_INVALID, "null output");
  if (probe < 0 || !(eps > 0.f) || !std::isfinite(eps)) return fail(ctx, ZO_ERR_INVALID, "bad probe or eps");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "pair evaluation needs the clean state");
  ProbeKey pk = probe_key(ctx);
  pk.sign = +1;
  pk.probe = (uint32_t)probe;
  pk.eps = eps;
  return launch_lowrank_loss(ctx, pk, D, lam, q->vseed, loss_plus, loss_minus, 0);
}

zo_status zo_lowrank_step(zo_ctx *ctx, const float *D, const zo_lowrank *q, int32_t n_pert,
                          float eps, float lr, float damping, int preconditioned,
                          double *losses_out) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "low-rank step: not separable over parameter slices (element offset must be 0)");
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!losses_out) return fail(ctx, ZO_ERR_INVALID, "null losses_out");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "step while perturbed");
  float lam[4];
  ZO_CHECK(check_lowrank(ctx, D, q, lam));
  double *L0 = losses_out, *Lp = losses_out + 1, *Lm = losses_out + 1 + n_pert;
  // The loss of probe i is its diagonal part plus sum_r (lam_r / 2M) (v_r . P_i)^2: one
  // table pass per 64 probes for the diagonal part and one per direction for its dot
  // products (the clean values in the first pass), then their combination.
  const size_t per = (size_t)(2 * n_pert + 1), need = per * (size_t)(q->rank + 1);
  if (need > ctx->lowrank_cap) {
    cudaFree(ctx->lowrank_scratch);
    ctx->lowrank_scratch = nullptr;
    ctx->lowrank_cap = 0;
    ZO_CUDA(ctx, cudaMalloc(&ctx->lowrank_scratch, need * sizeof(double)), "low-rank scratch");
    ctx->lowrank_cap = need;
  }
  double *base = ctx->lowrank_scratch, *dots = base + per;
  phase_mark(ctx, 0);
  if (!preconditioned)
    ZO_CUDA(ctx, cudaMemsetAsync(L0, 0, sizeof(double), ctx->stream), "clear L0");
  phase_mark(ctx, 1);
  ProbeKey pk = probe_key(ctx);
  pk.sign = +1;
  pk.eps = eps;
  for (int32_t i = 0; i < n_pert; i += 64) {
    const int c = n_pert - i < 64 ? n_pert - i : 64;
    const bool clean = preconditioned && i == 0;
    ZO_CHECK(launch_quad_octet(ctx, pk, (uint32_t)(i / 8), c, D, base + 1 + i, base + 1 + n_pert + i,
                               clean ? base : nullptr));
    for (int r = 0; r < q->rank; ++r) {
      double *dr = dots + per * r;
      ZO_CHECK(launch_lowrank_dot_octet(ctx, pk, (uint32_t)(i / 8), c, r, q->vseed, dr + 1 + i,
                                        dr + 1 + n_pert + i, clean ? dr : nullptr));
    }
  }
  ZO_CHECK(launch_lowrank_combine(ctx, base, dots, q->rank, n_pert, lam, preconditioned ? 1 : 0,
                                  losses_out));
  phase_mark(ctx, 2);
  const zo_status st = step_device(ctx, Lp, Lm, n_pert, preconditioned ? L0 : nullptr, lr, eps, damping);
  phase_mark(ctx, 3);
  return st;
}

zo_status zo_quad_loss_octet(zo_ctx *ctx, const float *D, int32_t first_probe, int32_t count,
                             float eps, double *loss_plus, double *loss_minus, double *loss_clean) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "quadratic loss needs an fp32 context");
  if (!D || !loss_plus || !loss_minus || !aligned16(D))
    return fail(ctx, ZO_ERR_INVALID, "D must be a 16-byte aligned device pointer; outputs non-null");
  if (first_probe < 0 || first_probe % 8 || count < 1 || count > 64 || !(eps > 0.f) || !std::isfinite(eps))
    return fail(ctx, ZO_ERR_INVALID, "first_probe must be a multiple of 8, count 1..64, eps > 0");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "octet evaluation needs the clean state");
  ProbeKey pk = probe_key(ctx);
  pk.sign = +1;
  pk.eps = eps;
  return launch_quad_octet(ctx, pk, (uint32_t)(first_probe / 8), count, D, loss_plus, loss_minus,
                           loss_clean);
}

zo_status zo_quad_step(zo_ctx *ctx, const float *D, int32_t n_pert, float eps, float lr,
                       float damping, int preconditioned, double *losses_out) {
  ZO_CHECK(check_ctx(ctx));
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!losses_out) return fail(ctx, ZO_ERR_INVALID, "null losses_out");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "step while perturbed");
  double *L0 = losses_out, *Lp = losses_out + 1, *Lm = losses_out + 1 + n_pert;
  phase_mark(ctx, 0);
  if (!preconditioned)
    ZO_CUDA(ctx, cudaMemsetAsync(L0, 0, sizeof(double), ctx->stream), "clear L0");
  phase_mark(ctx, 1);
  // the 128 losses of eight probe octets from one pass; the first pass also adds the clean loss
  for (int32_t i = 0; i < n_pert; i += 64)
    ZO_CHECK(zo_quad_loss_octet(ctx, D, i, n_pert - i < 64 ? n_pert - i : 64, eps, Lp + i, Lm + i,
                                (preconditioned && i == 0) ? L0 : nullptr));
  phase_mark(ctx, 2);
  const zo_status st = step_device(ctx, Lp, Lm, n_pert, preconditioned ? L0 : nullptr, lr, eps, damping);
  phase_mark(ctx, 3);
  return st;
}

zo_status zo_quad_step_host_async(zo_ctx *ctx, const float *D_host, int32_t n_pert, float eps,
                                  float lr, float damping, int preconditioned, double *losses_host) {
  ZO_CHECK(check_ctx(ctx));
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!D_host || !losses_host) return fail(ctx, ZO_ERR_INVALID, "null host buffer");
  if (!ctx->copy_stream) {
    ZO_CUDA(ctx, cudaStreamCreateWithFlags(&ctx->copy_stream, cudaStreamNonBlocking), "copy stream");
    for (int b = 0; b < 2; ++b) {
      ZO_CUDA(ctx, cudaMalloc(&ctx->pipe_d[b], (size_t)ctx->M * sizeof(float)), "staging slot");
      ZO_CUDA(ctx, cudaMalloc(&ctx->pipe_l[b], (2 * ZO_MAX_PROBES + 1) * sizeof(double)), "loss slot");
      ZO_CUDA(ctx, cudaEventCreateWithFlags(&ctx->pipe_copied[b], cudaEventDisableTiming), "event");
      ZO_CUDA(ctx, cudaEventCreateWithFlags(&ctx->pipe_consumed[b], cudaEventDisableTiming), "event");
      ZO_CUDA(ctx, cudaEventRecord(ctx->pipe_consumed[b], ctx->stream), "event");
    }
  }
  const int b = (int)(ctx->pipe_k++ & 1u);
  // the slot's previous step must have finished reading it before it is refilled
  ZO_CUDA(ctx, cudaStreamWaitEvent(ctx->copy_stream, ctx->pipe_consumed[b], 0), "wait slot");
  ZO_CUDA(ctx, cudaMemcpyAsync(ctx->pipe_d[b], D_host, (size_t)ctx->M * sizeof(float),
                               cudaMemcpyHostToDevice, ctx->copy_stream), "copy D");
  ZO_CUDA(ctx, cudaEventRecord(ctx->pipe_copied[b], ctx->copy_stream), "event");
  ZO_CUDA(ctx, cudaStreamWaitEvent(ctx->stream, ctx->pipe_copied[b], 0), "wait copy");
  ZO_CHECK(zo_quad_step(ctx, ctx->pipe_d[b], n_pert, eps, lr, damping, preconditioned, ctx->pipe_l[b]));
  ZO_CUDA(ctx, cudaEventRecord(ctx->pipe_consumed[b], ctx->stream), "event");
  ZO_CUDA(ctx, cudaMemcpyAsync(losses_host, ctx->pipe_l[b], (2 * n_pert + 1) * sizeof(double),
                               cudaMemcpyDeviceToHost, ctx->stream), "copy losses");
  return ZO_OK;
}

zo_status zo_quad_step_host(zo_ctx *ctx, const float *D_host, int32_t n_pert, float eps,
                            float lr, float damping, int preconditioned, double *losses_host) {
  ZO_CHECK(check_ctx(ctx));
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!D_host || !losses_host) return fail(ctx, ZO_ERR_INVALID, "null host buffer");
  if (!ctx->staging)
    ZO_CUDA(ctx, cudaMalloc(&ctx->staging, (size_t)ctx->M * sizeof(float)), "staging buffer");
  if (!ctx->loss_scratch)
    ZO_CUDA(ctx, cudaMalloc(&ctx->loss_scratch, (2 * ZO_MAX_PROBES + 1) * sizeof(double)), "loss scratch");
  ZO_CUDA(ctx, cudaMemcpyAsync(ctx->staging, D_host, (size_t)ctx->M * sizeof(float),
                               cudaMemcpyHostToDevice, ctx->stream), "copy D");
  ZO_CHECK(zo_quad_step(ctx, ctx->staging, n_pert, eps, lr, damping, preconditioned, ctx->loss_scratch));
  ZO_CUDA(ctx, cudaMemcpyAsync(losses_host, ctx->loss_scratch, (2 * n_pert + 1) * sizeof(double),
                               cudaMemcpyDeviceToHost, ctx->stream), "copy losses");
  ZO_CUDA(ctx, cudaStreamSynchronize(ctx->stream), "sync");
  return ZO_OK;
}

zo_status zo_mlp_losses(zo_ctx *ctx, const float *X, const int32_t *labels, int batch, int n_in,
                        int n_hidden, int n_out, int32_t n_pert, float eps, double scale,
                        double *loss_plus, double *loss_minus, double *loss_clean) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "MLP losses: not separable over parameter slices (element offset must be 0)");
  if (ctx->dtype != ZO_F32) return fail(ctx, ZO_ERR_UNSUPPORTED, "MLP losses need an fp32 context");
  if (!X || !labels || !loss_plus || !loss_minus || batch < 1 || n_in < 1 || n_hidden < 1 ||
      n_out < 1 || n_pert < 1 || n_pert > ZO_MAX_PROBES || !(eps > 0.f) || !std::isfinite(eps))
    return fail(ctx, ZO_ERR_INVALID, "bad MLP loss arguments");
  if ((int64_t)n_hidden * n_in + n_hidden + (int64_t)n_out * n_hidden + n_out != ctx->M)
    return fail(ctx, ZO_ERR_INVALID, "MLP shape does not match M");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "MLP losses need the clean state");
  return launch_mlp_probes(ctx, X, labels, batch, n_in, n_hidden, n_out, n_pert, eps, scale,
                           loss_plus, loss_minus, loss_clean);
}

zo_status zo_mlp_step(zo_ctx *ctx, const float *X, const int32_t *labels, int batch, int n_in,
                      int n_hidden, int n_out, int32_t n_pert, float eps, float lr,
                      float damping, int preconditioned, double *losses_out) {
  ZO_CHECK(check_ctx(ctx));
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "MLP step: not separable over parameter slices (element offset must be 0)");
  ZO_CHECK(check_step_args(ctx, n_pert, lr, eps, damping));
  if (!losses_out) return fail(ctx, ZO_ERR_INVALID, "null losses_out");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "step while perturbed");
  const double scale = 1.0 / (double)batch;
  double *L0 = losses_out, *Lp = losses_out + 1, *Lm = losses_out + 1 + n_pert;
  if (ctx->dtype == ZO_F32 && ctx->M + n_hidden <= kMlpStageMax) {
    // every loss of the step from one launch (parameters staged per block), then zo_step
    phase_mark(ctx, 0);
    if (!preconditioned)
      ZO_CUDA(ctx, cudaMemsetAsync(L0, 0, sizeof(double), ctx->stream), "clear L0");
    phase_mark(ctx, 1);
    ZO_CHECK(zo_mlp_losses(ctx, X, labels, batch, n_in, n_hidden, n_out, n_pert, eps, scale, Lp,
                           Lm, preconditioned ? L0 : nullptr));
    phase_mark(ctx, 2);
    const zo_status st = step_device(ctx, Lp, Lm, n_pert, preconditioned ? L0 : nullptr, lr, eps, damping);
    phase_mark(ctx, 3);
    return st;
  }
  if (!ctx->live_enabled) ZO_CHECK(zo_set_live_buffer(ctx, 1));
  phase_mark(ctx, 0);
  if (preconditioned) {
    ZO_CHECK(zo_mlp_loss(ctx, X, labels, batch, n_in, n_hidden, n_out, scale, L0, 0));
  } else {
    ZO_CUDA(ctx, cudaMemsetAsync(L0, 0, sizeof(double), ctx->stream), "clear L0");
  }
  phase_mark(ctx, 1);
  for (int32_t i = 0; i < n_pert; ++i) {
    for (int s = +1; s >= -1; s -= 2) {
      ZO_CHECK(zo_perturb(ctx, s, eps, i));
      const zo_status st = zo_mlp_loss(ctx, X, labels, batch, n_in, n_hidden, n_out, scale,
                                       (s > 0 ? Lp : Lm) + i, 0);
      zo_restore(ctx);
      ZO_CHECK(st);
    }
  }
  phase_mark(ctx, 2);
  const zo_status st = step_device(ctx, Lp, Lm, n_pert, preconditioned ? L0 : nullptr, lr, eps, damping);
  phase_mark(ctx, 3);
  return st;
}

}  // extern "C"
