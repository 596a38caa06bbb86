// zo_internal.cuh -- shared definitions of libzo.so (context, device state, probe bits).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "zo.h"

namespace zo {

constexpr int kSmCount = 148;           // B200 SMs (two dies x 74)
constexpr int kGroup = 16;              // elements per Philox block (16 elements x 8 probes)
constexpr int kOctet = 8;               // probes per Philox block
constexpr int kTileElems = 4096;        // elements per tile / chunk of the streaming kernels
constexpr int kTileGroups = kTileElems / kGroup;  // 256

// Device-resident step state.  `step` keys the probes of the current step; the
// preconditioner copies it to `upd_step` and sets `upd_ok` before advancing it, so the
// update kernel of the same step reads a stable value.
struct DevState {
  uint32_t step;
  uint32_t flags;     // sticky ZO_FLAG_* bits
  uint32_t upd_step;  // step the pending update belongs to
  uint32_t upd_ok;    // 1 if the pending update may be applied
};

// Everything a streaming kernel needs to regenerate probe bits.
struct ProbeKey {
  uint32_t k0, k1;          // Philox key (seed low / high word)
  const uint32_t *step;     // device step counter
  uint32_t probe;
  int sign;                 // +1 / -1 ; 0 = clean (no perturbation)
  float eps;
  uint64_t g_off;           // global index of the context's first 16-element group
};

// ------------------------------------------------------------------ Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11):
// ten rounds of two 32x32->64 multiplies whose high halves are xor-ed with the other
// counter words and the round key; the key advances by the Weyl constants per round.
__device__ __forceinline__ uint4 philox10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t a = c.x, b = c.z;
    const uint32_t hi_a = __umulhi(0xD2511F53u, a), lo_a = 0xD2511F53u * a;
    const uint32_t hi_b = __umulhi(0xCD9E8D57u, b), lo_b = 0xCD9E8D57u * b;
    c = make_uint4(hi_b ^ c.y ^ k0, lo_b, hi_a ^ c.w ^ k1, lo_a);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// The ten rounds' keys (k0 + r W0, k1 + r W1), computed once on the host.  A kernel that takes
// them as a __grid_constant__ parameter reads each key from the constant bank inside the
// round's three-input xor, instead of advancing two key registers every round.
struct RoundKeys {
  uint32_t k[20];  // round r: k[2r] (xor-ed into word 0), k[2r + 1] (into word 2)
};

inline RoundKeys round_keys(uint32_t k0, uint32_t k1) {
  RoundKeys rk;
  for (int r = 0; r < 10; ++r) {
    rk.k[2 * r] = k0 + (uint32_t)r * 0x9E3779B9u;
    rk.k[2 * r + 1] = k1 + (uint32_t)r * 0xBB67AE85u;
  }
  return rk;
}

// The same ten rounds with the key schedule read from rk.
__device__ __forceinline__ uint4 philox10(uint4 c, const RoundKeys &rk) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t a = c.x, b = c.z;
    const uint32_t hi_a = __umulhi(0xD2511F53u, a), lo_a = 0xD2511F53u * a;
    const uint32_t hi_b = __umulhi(0xCD9E8D57u, b), lo_b = 0xCD9E8D57u * b;
    c = make_uint4(hi_b ^ c.y ^ rk.k[2 * r], lo_b, hi_a ^ c.w ^ rk.k[2 * r + 1], lo_a);
  }
  return c;
}

// Sign layout ("8 signs per byte"): one Philox block holds the signs of the 16 elements of
// group g (elements 16g .. 16g+15) under the 8 probes of one octet (probes 8p .. 8p+7).
// Byte b of the little-endian block (bits 8(b&3).. of word b>>2) belongs to element 16g+b,
// and bit k of that byte to probe 8p+k; bit 1 means z = -1.  The update, which needs every
// probe of an element, reads whole bytes; a single-probe pass extracts one bit per byte.
__device__ __forceinline__ uint4 sign_block(uint64_t g, uint32_t octet, uint32_t step,
                                            uint32_t k0, uint32_t k1) {
  return philox10(make_uint4((uint32_t)g, (uint32_t)(g >> 32), octet, step), k0, k1);
}

__device__ __forceinline__ uint4 sign_block(uint64_t g, uint32_t octet, uint32_t step,
                                            const RoundKeys &rk) {
  return philox10(make_uint4((uint32_t)g, (uint32_t)(g >> 32), octet, step), rk);
}

// The 16 sign bits of probe `probe` in the block of its octet: element 16g+b at bit b.
__device__ __forceinline__ uint32_t probe_bits16(const uint4 &v, uint32_t probe) {
  const uint32_t k = probe & 7u;
  // bits k, k+8, k+16, k+24 of a word -> bits 0..3 (the multiply gathers them at 24..27)
  auto nib = [k](uint32_t w) { return ((((w >> k) & 0x01010101u) * 0x01020408u) >> 24) & 0xFu; };
  return nib(v.x) | (nib(v.y) << 4) | (nib(v.z) << 8) | (nib(v.w) << 12);
}

// The 16 sign bits of probe `probe` for element group g.
__device__ __forceinline__ uint32_t probe_group_bits(uint64_t g, uint32_t probe, uint32_t step,
                                                     uint32_t k0, uint32_t k1) {
  return probe_bits16(sign_block(g, probe >> 3, step, k0, k1), probe);
}

__device__ __forceinline__ uint32_t probe_group_bits(uint64_t g, uint32_t probe, uint32_t step,
                                                     const RoundKeys &rk) {
  return probe_bits16(sign_block(g, probe >> 3, step, rk), probe);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int w) {
  return w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
}

// bf16 <-> fp32 on raw bits (round to nearest even, as __float2bfloat16_rn).
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float((uint32_t)h << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// Two values rounded to bf16 (round to nearest even) and packed, lo in the low half: one
// conversion instruction for the pair, the same bits as two f32_to_bf16_bits.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// P = rd(theta + s*eps*z) for one element given its sign bit (bit 1 -> z = -1).
// `delta` is s*eps; the xor of the bit into the sign flips it exactly.
__device__ __forceinline__ float perturb_f32(float theta, float delta, uint32_t bit) {
  return __fadd_rn(theta, __uint_as_float(__float_as_uint(delta) ^ (bit << 31)));
}

}  // namespace zo

// ------------------------------------------------------------------ context

enum class PState { Clean, Perturbed };

struct zo_ctx {
  void *params = nullptr;
  int64_t M = 0;
  int dtype = ZO_F32;
  uint64_t seed = 0;
  cudaStream_t stream = nullptr;
  int device = 0;
  float alpha = 0.1f;

  PState state = PState::Clean;
  int sign = 0;
  float eps = 0.f;
  int32_t probe = 0;

  int64_t first_element = 0;  // global index of params[0] (a multiple of 16)

  bool live_enabled = false;
  void *live = nullptr;        // M elements when enabled

  zo::DevState *dstate = nullptr;
  float *coef = nullptr;       // ZO_MAX_PROBES fp32 update coefficients
  double *diag = nullptr;      // 3 * ZO_MAX_PROBES fp64 (g, c, w) of the last step
  int32_t last_n = 0;
  double *partials = nullptr;  // reduction scratch (kMaxPartials doubles + 8 discard slots)
  unsigned int *counter = nullptr;  // last-block ticket for the reductions
  float *staging = nullptr;    // device staging for host-buffer entry points
  double *loss_scratch = nullptr;  // 2*ZO_MAX_PROBES+1 doubles for host-buffer steps

  // pipelined host-buffer steps: two staging slots, a copy stream, per-slot events
  float *pipe_d[2] = {nullptr, nullptr};
  double *pipe_l[2] = {nullptr, nullptr};
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t pipe_copied[2] = {nullptr, nullptr}, pipe_consumed[2] = {nullptr, nullptr};
  uint64_t pipe_k = 0;

  // per-probe sums of the batched low-rank step ((rank + 1) x (2 n + 1) doubles)
  double *lowrank_scratch = nullptr;
  size_t lowrank_cap = 0;

  // per-sample losses of the batched MLP evaluation ((2 n + 1) x batch doubles)
  double *mlp_ce = nullptr;
  size_t mlp_ce_cap = 0;

  // phase timing of the step drivers: 4 events per recorded step
  cudaEvent_t *phase_ev = nullptr;
  int32_t phase_cap = 0, phase_used = 0;

  // kernels this context has enqueued (every successful launch)
  int64_t launches = 0;

  // per-class kernel timing (zo_enable_kernel_timing): an event pair around every launch of
  // the timed classes, with the launch's algorithmic work; drained by zo_kernel_times
  struct KRec {
    int cls;      // ZO_KT_* or -1 (launch failed after its start event)
    double work;  // flops or bytes of this launch
  };
  bool ktime_on = false;
  std::vector<KRec> ktime_recs;
  std::vector<cudaEvent_t> ktime_ev;  // 2 per record, reused after each drain
  int64_t ktime_dropped = 0;

  // losses given to zo_step are host pointers (zo_set_loss_location(ctx, 0))
  bool host_losses = false;

  std::string err;
};

namespace zo {

constexpr int kMaxPartials = 32768;
// Parameters an MLP evaluation block stages in shared memory (192 KB of fp32).
constexpr int kMlpStageMax = 49152;

zo_status fail(zo_ctx *ctx, zo_status st, const char *fmt, ...);
zo_status check_launch(zo_ctx *ctx, const char *what);

ProbeKey probe_key(const zo_ctx *ctx);  // current perturbation (sign 0 when clean)

// Record phase event `which` (0..3) of the current step if phase timing is enabled;
// which == 3 closes the step.
void phase_mark(zo_ctx *ctx, int which);

// Kernel timing: ktime_begin records the start event of a launch of a timed class and
// returns its slot (-1 when timing is off or the record cap is reached); ktime_end records
// the end event after the launch, with the class and the launch's algorithmic work.
int ktime_begin(zo_ctx *ctx);
void ktime_end(zo_ctx *ctx, int slot, int cls, double work);

// zo_step's body for device-resident losses (what the step drivers call).
zo_status step_device(zo_ctx *ctx, const double *loss_plus, const double *loss_minus, int32_t n_pert,
                      const double *loss0, float lr, float eps, float damping);

// Launchers (each enqueues on ctx->stream and returns the launch status).
zo_status launch_perturb(zo_ctx *ctx, const ProbeKey &pk, int64_t first, int64_t count,
                         void *out);
zo_status launch_pack(zo_ctx *ctx, uint32_t step, uint32_t probe, int64_t first_byte,
                      int64_t nbytes, uint8_t *out);
zo_status launch_quad_loss(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out,
                           int accumulate, double *partials, unsigned int *counter);
zo_status launch_quad_loss_pair(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out_plus,
                                double *out_minus);
// The 2 count losses of probes 8 octet .. 8 octet + count - 1 (count <= 8) in one pass,
// and the clean loss into *out_clean in the same pass when out_clean is not null.
zo_status launch_quad_octet(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                            const float *D, double *out_plus, double *out_minus,
                            double *out_clean = nullptr);
// The conditioning-study quadratic (lam[4]: eigenvalue of each direction, 0 if unused;
// directions from vseed); out_minus != null evaluates both signs of pk's probe in one pass.
zo_status launch_lowrank_loss(zo_ctx *ctx, const ProbeKey &pk, const float *D, const float lam[4],
                              uint64_t vseed, double *out, double *out_minus, int accumulate);
zo_status launch_lowrank_dot_octet(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                                   int dir, uint64_t vseed, double *out_plus, double *out_minus,
                                   double *out_clean);
zo_status launch_lowrank_combine(zo_ctx *ctx, const double *base, const double *dots, int rank,
                                 int n, const float lam[4], int clean, double *out);
// Raise a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device): the attribute belongs to a device's context, so a process with contexts
// on several devices sets it on each.
cudaError_t ensure_smem_limit(const void *kernel, int bytes);
zo_status launch_mlp_probes(zo_ctx *ctx, const float *X, const int32_t *y, int batch, int n_in,
                            int n_hidden, int n_out, int n_pert, float eps, double scale,
                            double *lp, double *lm, double *l0);
zo_status launch_mlp_loss(zo_ctx *ctx, const float *P, const float *X, const int32_t *y,
                          int batch, int n_in, int n_hidden, int n_out, double scale,
                          double *out, int accumulate);
zo_status launch_precond(zo_ctx *ctx, const double *lp, const double *lm, const double *l0,
                         int n, float lr, float eps, float damping);
zo_status launch_update(zo_ctx *ctx, const float *coef, int n, const uint32_t *step_ptr,
                        const uint32_t *ok_ptr);

}  // namespace zo
