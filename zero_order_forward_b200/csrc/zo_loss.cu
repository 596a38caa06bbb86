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
// regenerate the chunk's sign bits (one Philox block per lane: a 16-element group of the
// elements its warp reads, shared through warp shuffles), apply the perturbation and
// accumulate in fp64, then release the stage.  Consumer thread ct takes the 4-element
// vectors 4 (ct + 256 k), k = 0..3, of every chunk and adds its terms to one accumulator
// per loss in that order; the grid walks chunks round-robin (chunk = blockIdx.x + i gridDim.x)
// and its size depends on M only, so every loss's summation order is fixed, and the same
// in the single-loss and pair forms (their results are bit-identical).
constexpr int kQChunk = 4096;
constexpr int kQStages = 3;
constexpr int kQConsumers = 8;
constexpr int kQThreads = 32 * (1 + kQConsumers);
constexpr int kQStageBytes = 2 * kQChunk * 4;  // theta, D
constexpr int kQSmemBytes = kQStages * kQStageBytes + 2 * kQStages * 8;
constexpr int kQIters = kQChunk / (4 * 32 * kQConsumers);  // 4 vectors per thread per chunk
// The octet pass is bound by its per-probe arithmetic, not by the stream: two stages of
// 2048-element chunks plus the 32 KB of nibble tables and at most 72 registers give three
// CTAs (27 warps) per SM.
constexpr int kOChunk = 2048;
constexpr int kOStages = 2;
constexpr int kOStageBytes = 2 * kOChunk * 4;
constexpr int kOIters = kOChunk / (4 * 32 * kQConsumers);  // 2 vectors per thread per chunk
constexpr int kOTableBytes = 16 * 32 * kQConsumers * 8;    // 16 fp64 entries per consumer thread
constexpr int kOTableOff = kOStages * kOStageBytes + 2 * kOStages * 8;
constexpr int kOSmemBytes = kOTableOff + kOTableBytes;
constexpr int kOBlocksPerSm = 3;

struct QuadPipe {
  uint8_t *sm;
  uint64_t *full, *empty;
  int stages;
  int chunk;  // elements per stage; a stage holds theta then D
};

__device__ __forceinline__ QuadPipe quad_pipe_init(uint8_t *qsm, volatile int *abort_flag,
                                                   int stages = kQStages, int chunk = kQChunk) {
  QuadPipe p{qsm, reinterpret_cast<uint64_t *>(qsm + stages * 2 * chunk * 4), nullptr, stages,
             chunk};
  p.empty = p.full + stages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      tc::mbar_init(&p.full[s], 1);
      tc::mbar_init(&p.empty[s], kQConsumers);
    }
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  return p;
}

// Warp 0: stream the CTA's chunks of theta and D into the stage ring (bounded waits).
__device__ __forceinline__ void quad_produce(const QuadPipe &p, const float *theta, const float *D,
                                             int64_t M, int64_t n_chunks, volatile int *abort_flag,
                                             uint32_t *err) {
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  int it = 0, issued = 0;
  for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x, ++it) {
    const int s = it % S;
    const uint32_t ph = (uint32_t)(it / S) & 1u;
    int ok = 1;
    if (lane == 0) ok = tc::mbar_wait(&p.empty[s], ph ^ 1u) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok || *abort_flag) {
      if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); *abort_flag = 1; }
      break;
    }
    uint8_t *st = p.sm + s * 2 * p.chunk * 4;
    const int64_t base = chunk * p.chunk;
    const int cnt = (int)(M - base < (int64_t)p.chunk ? M - base : (int64_t)p.chunk);
    const int copy = cnt & ~3;
    if (lane == 0) {  // D may be null (passes that read theta only)
      tc::mbar_arrive_expect_tx(&p.full[s], (D ? 2u : 1u) * (uint32_t)copy * 4u);
      if (copy) {
        tc::bulk_load(st, theta + base, (uint32_t)copy * 4u, &p.full[s]);
        if (D) tc::bulk_load(st + p.chunk * 4, D + base, (uint32_t)copy * 4u, &p.full[s]);
      }
    }
    __syncwarp();
    issued = it + 1;
  }
  if (*abort_flag && lane == 0) {  // let this CTA's copies land before it exits
    for (int s = 0; s < S; ++s) {
      int last = -1;
      for (int i = s; i < issued; i += S) last = i;
      if (last >= 0) tc::mbar_wait(&p.full[s], (uint32_t)(last / S) & 1u);
    }
  }
}

// A consumer warp takes stage s (phase ph): lane 0 decides for the warp (all lanes leave
// together or none), then every lane observes the completed phase itself.
__device__ __forceinline__ bool quad_acquire(const QuadPipe &p, int s, uint32_t ph,
                                             volatile int *abort_flag, uint32_t *err) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) ok = (!*abort_flag && tc::mbar_wait(&p.full[s], ph)) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok && lane != 0) ok = tc::mbar_wait(&p.full[s], ph) ? 1 : 0;
  if (__all_sync(0xFFFFFFFFu, ok)) return true;
  if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); *abort_flag = 1; }
  return false;
}

// The 4 theta and D values of vector e (0 past the end of the chunk: their terms are 0).
// WITH_D false: theta only (dv left 0).
template <int CHUNK = kQChunk, bool WITH_D = true>
__device__ __forceinline__ void quad_load4(const uint8_t *st, const float *theta, const float *D,
                                           int64_t base, int e, int cnt, float tv[4], float dv[4]) {
  if (e + 4 <= (cnt & ~3)) {
    const float4 t = reinterpret_cast<const float4 *>(st)[e >> 2];
    tv[0] = t.x; tv[1] = t.y; tv[2] = t.z; tv[3] = t.w;
    if (WITH_D) {
      const float4 dd = reinterpret_cast<const float4 *>(st + CHUNK * 4)[e >> 2];
      dv[0] = dd.x; dv[1] = dd.y; dv[2] = dd.z; dv[3] = dd.w;
    } else {
      dv[0] = dv[1] = dv[2] = dv[3] = 0.f;
    }
  } else {  // the last < 4 elements of theta (not covered by the 16-byte copies)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool in = e + q < cnt;
      tv[q] = in ? theta[base + e + q] : 0.f;
      dv[q] = (WITH_D && in) ? D[base + e + q] : 0.f;
    }
  }
}

// term = (D/2) P^2 in fp64 (P^2 of an fp32 value is exact in fp64).
__device__ __forceinline__ double quad_term(float d, float p) {
  const double pd = (double)p;
  return __dmul_rn(__dmul_rn(0.5, (double)d), __dmul_rn(pd, pd));
}

// PAIR: both losses of one probe, L(theta + eps z) into out and L(theta - eps z) into
// out_minus, from one pass over theta and D (pk.sign must be +1).
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
  __shared__ volatile int abort_flag;
  const QuadPipe pipe = quad_pipe_init(qsm, &abort_flag);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t step = pk.sign ? *pk.step : 0u;
  const float delta = pk.sign > 0 ? pk.eps : -pk.eps;
  constexpr int RR = R > 0 ? R : 1;
  double acc = 0.0, accm = 0.0;   // accm: PAIR, the -eps loss
  double dot[RR], dotm[RR];       // R > 0: v_k . P (and for the -eps side)
#pragma unroll
  for (int k = 0; k < RR; ++k) dot[k] = dotm[k] = 0.0;

  if (warp == 0) {
    quad_produce(pipe, theta, D, M, n_chunks, &abort_flag, err);
  } else {
    const int ct = threadIdx.x - 32;  // 0 .. 255
    const int cw = ct >> 5;           // consumer warp: elements 4 (32 cw + lane + 256 k) + 0..3
    int it = 0;
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x, ++it) {
      const int s = it % kQStages;
      if (!quad_acquire(pipe, s, (uint32_t)(it / kQStages) & 1u, &abort_flag, err)) break;
      const uint8_t *st = pipe.sm + s * kQStageBytes;
      const int64_t base = chunk * kQChunk;
      const int cnt = (int)(M - base < (int64_t)kQChunk ? M - base : (int64_t)kQChunk);
      // The warp's 32 groups: slot q = 8 k + j is group 8 cw + 64 k + j of the chunk; lane q
      // computes its 16 bits (groups past M are computed and never used).
      const uint64_t my_group = (uint64_t)(base / kGroup) + 8 * cw + 64 * (lane >> 3) + (lane & 7);
      uint32_t mine = 0u;
      if (pk.sign) mine = probe_group_bits(my_group + pk.g_off, pk.probe, step, pk.k0, pk.k1);
      uint4 vmine = make_uint4(0u, 0u, 0u, 0u);
      if (R > 0) vmine = sign_block(my_group, 0u, 0u, lr.vk0, lr.vk1);
#pragma unroll
      for (int k = 0; k < kQIters; ++k) {
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
        quad_load4(st, theta, D, base, e, cnt, tv, dv);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float p = pk.sign ? perturb_f32(tv[q], delta, (bits >> q) & 1u) : tv[q];
          acc = __dadd_rn(acc, quad_term(dv[q], p));
          float pm = 0.f;
          if (PAIR) {
            pm = perturb_f32(tv[q], -delta, (bits >> q) & 1u);
            accm = __dadd_rn(accm, quad_term(dv[q], pm));
          }
          if (R > 0 && e + q < cnt) {
            const uint32_t vb = vw >> (8 * q);
#pragma unroll
            for (int r = 0; r < RR; ++r) {
              const bool neg = (vb >> r) & 1u;
              const double pd = (double)p;
              dot[r] = __dadd_rn(dot[r], neg ? -pd : pd);
              if (PAIR) {
                const double pmd = (double)pm;
                dotm[r] = __dadd_rn(dotm[r], neg ? -pmd : pmd);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&pipe.empty[s]);
    }
  }
  // The next loss pass may start streaming now; the reduction scratch (partials, counter,
  // out) is touched only after the previous kernel in the stream has fully completed.
  tc::pdl_launch_dependents();
  tc::pdl_wait();
  if (R > 0) {
    constexpr int NS = PAIR ? 2 : 1, NV = NS * (1 + RR);
    double v[NV], tot[NV];
    v[0] = block_sum(acc);
#pragma unroll
    for (int r = 0; r < RR; ++r) v[1 + r] = block_sum(dot[r]);
    if (PAIR) {
      v[1 + RR] = block_sum(accm);
#pragma unroll
      for (int r = 0; r < RR; ++r) v[2 + RR + r] = block_sum(dotm[r]);
    }
    if (last_block_totals<NV>(v, partials, counter, tot)) {
      const double inv_m = 1.0 / (double)M;
#pragma unroll
      for (int sgn = 0; sgn < NS; ++sgn) {
        const double *t = tot + sgn * (1 + RR);
        double L = t[0];
#pragma unroll
        for (int r = 0; r < RR; ++r)
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

// Sign word of 4 elements: byte q holds element q's bits, bit t of a byte probe t of an
// octet.  Masking bits t and t + 4 of every byte ((w >> t) & 0x11111111, t < 4) and
// multiplying by 0x01020408 = 2^24 + 2^17 + 2^10 + 2^3 moves bit 8q + t to 24 + q and bit
// 8q + t + 4 to 28 + q: the nibbles of probes t and t + 4, bit q = element q.  Every other
// partial product lands at a distinct position below bit 24 or beyond bit 31, so nothing
// carries into them.  The table offsets 2048 * nibble follow with one shift and mask each.
// The losses L(theta +- eps z_i) of the 8 NOCT probes i = 8 octet + p, p < 8 NOCT (NOCT = 2,
// 4 or 8 consecutive octets: 32, 64 or 128 losses), from one pass over theta and D.
//
// Each element has only two perturbed values, P_a = rd(theta + eps) and P_b = rd(theta - eps),
// with terms t_a = (D/2) P_a^2 and t_b = (D/2) P_b^2 (fp64); the sign bit of probe i says
// which one L+_i takes (set: t_b, z = -1; clear: t_a) and L-_i takes the other, so
// L-_i = T - L+_i with T = sum_j (t_a + t_b)_j.
//
// A consumer thread holds 4 consecutive elements per vector; the 4 sign bits of one probe
// for them form a nibble, and the 16 possible sums (x_0 + x_1) + (x_2 + x_3), x_q in
// {t_a, t_b}, go into the thread's table in shared memory once per vector.  G neighbouring
// lanes (a pair for NOCT 2 and 4, a quad for NOCT 8; a quad's vectors are one 16-element
// group) read each other's tables, and each of them accumulates NOCT/G of the octets for
// all G vectors, so a thread keeps at most 16 accumulators while each vector's terms and
// table serve all 8 NOCT probes.  A pair gets its sign words from the quad's four Philox
// blocks through shuffles; a quad lane generates the blocks of its own two octets, whose
// four words are the quad's four vectors.  Per vector, two probes then cost one masked
// multiply of the sign word (above), and each probe a shift and mask, one table load and
// one fp64 add.  Summation order per
// loss: the vector steps of a thread in chunk order, each adding the G vectors in a fixed
// lane-dependent order; block and grid totals in a fixed order (LPV lanes per value over a
// fixed stride, then a butterfly).  Probes p >= count are computed and not stored.  CLEAN
// also adds the clean loss L(theta) to the same pass (into *out_clean).
//
// DOT: instead of the quadratic's terms, the terms of the dot product v . P with direction
// `dir` of the low-rank quadratic (v_j = -1 where bit dir of element j's byte of the
// directions' block, key (vk0, vk1), octet 0, step 0, is set; else +1): t_a = v_j P_a,
// t_b = v_j P_b and the clean term v_j theta_j, exact in fp64.  The same tables then give
// v . P(theta + eps z_i) and v . P(theta - eps z_i) = sum_j v_j (P_a + P_b)_j - v . P+; D is
// not read.
template <bool CLEAN, int NOCT, bool DOT>
__global__ void __launch_bounds__(kQThreads, kOBlocksPerSm)
quad_octet_kernel(const float *__restrict__ theta, const float *__restrict__ D, int64_t M,
                  ProbeKey pk, const __grid_constant__ RoundKeys rk, uint32_t octet, int count,
                  int64_t n_chunks, double *partials, unsigned int *counter, double *out_plus,
                  double *out_minus, double *out_clean, uint32_t *err, int dir, uint32_t vk0,
                  uint32_t vk1) {
  static_assert(NOCT == 2 || NOCT == 4 || NOCT == 8, "two, four or eight octets per pass");
  constexpr int G = NOCT == 8 ? 4 : 2;     // lanes sharing their tables (a pair or a quad)
  constexpr int LO = NOCT / G;             // octets per thread
  constexpr int NL = 8 * LO;               // accumulators per thread
  constexpr int NP = 8 * NOCT;             // probes per pass
  constexpr int NV = NP + 2;               // block values: probes, T, clean loss
  constexpr int LPV = NOCT == 8 ? 4 : 8;   // lanes per value in the epilogue
  static_assert(LPV * NV <= kQThreads, "lanes per value in the epilogue");
  static_assert(kOStages * kOStageBytes == 16 * 2048 && kOTableBytes == 16 * 2048 && NL + 2 <= 32,
                "epilogue rows: 16 in the stage buffers, the rest in the tables");
  extern __shared__ __align__(128) uint8_t qsm[];
  __shared__ volatile int abort_flag;
  __shared__ double totals[NV];
  __shared__ bool last;
  const QuadPipe pipe = quad_pipe_init(qsm, &abort_flag, kOStages, kOChunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t step = *pk.step;
  double lp[NL], tsum = 0.0, l0 = 0.0;
#pragma unroll
  for (int t = 0; t < NL; ++t) lp[t] = 0.0;
  const int ct = threadIdx.x - 32;  // consumer thread 0..255 (warp 0 produces)

  if (warp == 0) {
    quad_produce(pipe, theta, D, M, n_chunks, &abort_flag, err);
  } else {
    const int cw = ct >> 5;
    const int q = lane & 3, quad = lane >> 2, h = lane & 1;
    const uint32_t own8 = (uint32_t)ct * 8u, par8 = (uint32_t)(ct ^ 1) * 8u;
    // NOCT 8: round r reads the table of quad lane q ^ r (distinct per lane in every round)
    uint32_t col8[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) col8[r] = (uint32_t)(ct ^ r) * 8u;
    uint8_t *const tab = qsm + kOTableOff;  // entry n of thread c at byte 2048 n + 8 c
    int it = 0;
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x, ++it) {
      const int s = it % kOStages;
      if (!quad_acquire(pipe, s, (uint32_t)(it / kOStages) & 1u, &abort_flag, err)) break;
      const uint8_t *st = pipe.sm + s * kOStageBytes;
      const int64_t base = chunk * kOChunk;
      const int cnt = (int)(M - base < (int64_t)kOChunk ? M - base : (int64_t)kOChunk);
      // Vector k of this thread lies in group g_k = 8 cw + 64 k + quad of the chunk, bytes
      // 4q..4q+3 (word q of each block of that group); the pair's vectors are words
      // 2 (q >> 1) and 2 (q >> 1) + 1.  The quad's lanes generate the blocks it needs and
      // four shuffles hand each lane the pair's two words of each of its octets.
      const uint64_t g0 = pk.g_off + (uint64_t)(base / kGroup) + 8 * cw + quad;
      // NOCT 2: once per chunk, lane q generates (vector q >> 1, octet q & 1); lane l reads
      // lane l in rounds 0, 1 and lane l ^ 2 (the other vector) in rounds 2, 3.
      uint32_t wo2[kOIters], wp2[kOIters];
      if constexpr (NOCT == 2) {
        const uint4 blk = sign_block(g0 + 64 * (q >> 1), octet + (uint32_t)(q & 1), step, rk);
        uint32_t R[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int c = r >> 1;
          R[r] = __shfl_sync(0xFFFFFFFFu, word_of(blk, 2 * ((q >> 1) ^ c) + (r & 1)),
                             lane ^ (2 * c));
        }
        const bool x = q >> 1;  // rounds 0, 1 carried vector 1
        const uint32_t e0 = x ? R[2] : R[0], o0 = x ? R[3] : R[1];
        const uint32_t e1 = x ? R[0] : R[2], o1 = x ? R[1] : R[3];
        wo2[0] = h ? o0 : e0;
        wp2[0] = h ? e0 : o0;
        wo2[kOIters - 1] = h ? o1 : e1;
        wp2[kOIters - 1] = h ? e1 : o1;
      }
#pragma unroll
      for (int k = 0; k < kOIters; ++k) {
        // elements past the chunk's end load as 0 (terms 0): both lanes of a pair always
        // build a table
        const int e = 4 * (ct + k * 32 * kQConsumers);
        float tv[4], dv[4];
        quad_load4<kOChunk, !DOT>(st, theta, D, base, e, cnt, tv, dv);
        uint32_t vw = 0u;  // DOT: the directions' bits of this vector's 4 elements
        if constexpr (DOT) vw = word_of(sign_block(g0 + 64 * k, 0u, 0u, vk0, vk1), q);
        // wo / wp: the own / partner vector's word of each local octet j (pairs)
        uint32_t wo[LO], wp[LO];
        if constexpr (NOCT == 8) {
        } else if constexpr (NOCT == 4) {
          // lane q generates octet q; lane l reads octet sw(l) in rounds 0, 1 and octet
          // sw(l) ^ 1 in rounds 2, 3 (sw swaps the two bits of q), even word then odd
          const int sw = ((q & 1) << 1) | (q >> 1);
          const uint4 blk = sign_block(g0 + 64 * k, octet + (uint32_t)q, step, rk);
          uint32_t R[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int c = r >> 1;
            R[r] = __shfl_sync(0xFFFFFFFFu, word_of(blk, 2 * ((q & 1) ^ c) + (r & 1)),
                               (lane & ~3) | (sw ^ c));
          }
          const bool x = sw & 1;  // rounds 0, 1 carried local octet 1
          const uint32_t e0 = x ? R[2] : R[0], o0 = x ? R[3] : R[1];
          const uint32_t e1 = x ? R[0] : R[2], o1 = x ? R[1] : R[3];
          wo[0] = h ? o0 : e0;
          wp[0] = h ? e0 : o0;
          wo[LO - 1] = h ? o1 : e1;
          wp[LO - 1] = h ? e1 : o1;
        } else {
          wo[0] = wo2[k];
          wp[0] = wp2[k];
        }
        double ta[4], tb[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          if constexpr (DOT) {
            // elements past the chunk's end contribute nothing
            const bool in = e + qq < cnt, neg = (vw >> (8 * qq + dir)) & 1u;
            const double pa = in ? (double)__fadd_rn(tv[qq], pk.eps) : 0.0;
            const double pb = in ? (double)__fadd_rn(tv[qq], -pk.eps) : 0.0;
            ta[qq] = neg ? -pa : pa;
            tb[qq] = neg ? -pb : pb;
            if (CLEAN) l0 = __dadd_rn(l0, neg ? -(double)tv[qq] : (double)tv[qq]);
          } else {
            ta[qq] = quad_term(dv[qq], __fadd_rn(tv[qq], pk.eps));
            tb[qq] = quad_term(dv[qq], __fadd_rn(tv[qq], -pk.eps));
            if (CLEAN) l0 = __dadd_rn(l0, quad_term(dv[qq], tv[qq]));
          }
          tsum = __dadd_rn(tsum, __dadd_rn(ta[qq], tb[qq]));
        }
        // table entry n: element q takes t_b if bit q of n is set
        double lo[4], hi[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          lo[n] = __dadd_rn(n & 1 ? tb[0] : ta[0], n & 2 ? tb[1] : ta[1]);
          hi[n] = __dadd_rn(n & 1 ? tb[2] : ta[2], n & 2 ? tb[3] : ta[3]);
        }
        __syncwarp();  // the partner has read this table's previous contents
#pragma unroll
        for (int n = 0; n < 16; ++n)
          *reinterpret_cast<double *>(tab + 2048 * n + own8) = __dadd_rn(lo[n & 3], hi[n >> 2]);
        __syncwarp();  // the tables of the pair (quad) are written
        if constexpr (NOCT == 8) {
          // the quad holds the whole 16-element group: lane q generates the blocks of its
          // octets 2q, 2q + 1 itself; word m of a block is the vector of quad lane m
#pragma unroll
          for (int j = 0; j < LO; ++j) {
            const uint4 blk = sign_block(g0 + 64 * k, octet + (uint32_t)(LO * q + j), step, rk);
            uint32_t w[4] = {blk.x, blk.y, blk.z, blk.w};
            if (q & 1) {  // w[r] <- word q ^ r
              const uint32_t a = w[0], b = w[2];
              w[0] = w[1]; w[1] = a; w[2] = w[3]; w[3] = b;
            }
            if (q & 2) {
              const uint32_t a = w[0], b = w[1];
              w[0] = w[2]; w[1] = w[3]; w[2] = a; w[3] = b;
            }
            // probes t and t + 4 together: bits t and t + 4 of the word's 4 bytes, masked and
            // multiplied by 0x01020408, gather at bits 24..27 and 28..31 (the other partial
            // products fall at distinct positions below bit 24 or beyond bit 31)
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              double a0 = lp[8 * j + t], a1 = lp[8 * j + t + 4];
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const uint32_t pr = ((w[r] >> t) & 0x11111111u) * 0x01020408u;
                a0 = __dadd_rn(a0, *reinterpret_cast<const double *>(tab + (((pr >> 13) & 0x7800u) | col8[r])));
                a1 = __dadd_rn(a1, *reinterpret_cast<const double *>(tab + (((pr >> 17) & 0x7800u) | col8[r])));
              }
              lp[8 * j + t] = a0;
              lp[8 * j + t + 4] = a1;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < LO; ++j) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {  // probes t and t + 4 through one multiply per word
              const uint32_t po = ((wo[j] >> t) & 0x11111111u) * 0x01020408u;
              const uint32_t pp = ((wp[j] >> t) & 0x11111111u) * 0x01020408u;
              const double vo0 = *reinterpret_cast<const double *>(tab + (((po >> 13) & 0x7800u) | own8));
              const double vq0 = *reinterpret_cast<const double *>(tab + (((pp >> 13) & 0x7800u) | par8));
              const double vo1 = *reinterpret_cast<const double *>(tab + (((po >> 17) & 0x7800u) | own8));
              const double vq1 = *reinterpret_cast<const double *>(tab + (((pp >> 17) & 0x7800u) | par8));
              lp[8 * j + t] = __dadd_rn(__dadd_rn(lp[8 * j + t], vo0), vq0);
              lp[8 * j + t + 4] = __dadd_rn(__dadd_rn(lp[8 * j + t + 4], vo1), vq1);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&pipe.empty[s]);
    }
  }
  tc::pdl_launch_dependents();

  // Block totals through shared memory: row i holds accumulator i of the 256 consumer
  // threads (rows 0..15 in the stage buffers, the rest in the tables; the mbarriers between
  // them are left alone).  Both areas are idle once every warp has passed this barrier: the
  // producer returned only after its copies landed.
  __syncthreads();
  auto red_row = [](int i) {
    return reinterpret_cast<double *>(i < 16 ? qsm + 2048 * i : qsm + kOTableOff + 2048 * (i - 16));
  };
  if (warp > 0) {
#pragma unroll
    for (int i = 0; i < NL; ++i) red_row(i)[ct] = lp[i];
    red_row(NL)[ct] = tsum;
    red_row(NL + 1)[ct] = l0;
  }
  __syncthreads();
  // value v: probe v (accumulator v mod NL of the threads ct with ct mod G = v / NL), then
  // T, then the clean loss; lane g of the value's LPV sums a fixed stride, then a butterfly
  const int v = threadIdx.x / LPV, g = threadIdx.x % LPV;
  double bv = 0.0;
  if (v < NP) {
    const double *row = red_row(v % NL) + v / NL;
    for (int m = g; m < 256 / G; m += LPV) bv = __dadd_rn(bv, row[G * m]);
  } else if (v < NV) {
    const double *row = red_row(NL + v - NP);
    for (int c = g; c < 256; c += LPV) bv = __dadd_rn(bv, row[c]);
  }
#pragma unroll
  for (int o = LPV / 2; o > 0; o >>= 1) bv = __dadd_rn(bv, __shfl_xor_sync(0xFFFFFFFFu, bv, o));

  // The reduction scratch (partials, counter) is touched only after the previous kernel
  // in the stream has fully completed.
  tc::pdl_wait();
  if (g == 0 && v < NV) {
    partials[v * gridDim.x + blockIdx.x] = bv;
    __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  double tot = 0.0;
  if (v < NV)
    for (unsigned int b = g; b < gridDim.x; b += LPV) tot = __dadd_rn(tot, __ldcg(partials + v * gridDim.x + b));
#pragma unroll
  for (int o = LPV / 2; o > 0; o >>= 1) tot = __dadd_rn(tot, __shfl_xor_sync(0xFFFFFFFFu, tot, o));
  if (g == 0 && v < NV) totals[v] = tot;
  __syncthreads();
  const int p = threadIdx.x;
  if (p < NP && p < count) {
    out_plus[p] = totals[p];
    out_minus[p] = totals[NP] - totals[p];
  }
  if (p == 0) {
    if (CLEAN) *out_clean = totals[NP + 1];
    *counter = 0u;
  }
}

constexpr int kMlpMax = 1024;

// One sample's cross-entropy computed by the whole block (blockDim a multiple of 32), valid
// in thread 0: h = ReLU(W1 x + b1), logits = W2 h + b2, CE(logits, y).  The arithmetic of a
// sample does not depend on the block size: each hidden unit is one thread's fmaf chain over
// the inputs in order, each logit one warp's lane-strided fmaf chains combined by a fixed
// shuffle-down tree, the cross-entropy one thread's.  The weights may sit in global or
// shared memory; W1's rows are ld1 floats apart (ld1 >= n_in).  The caller may call it again
// for another sample right away: the first barrier of the next call orders its writes of hs
// and ls after this call's reads.
__device__ double mlp_sample_ce(const float *W1, int ld1, const float *b1, const float *W2,
                                const float *b2, const float *__restrict__ X,
                                const int32_t *__restrict__ y, int b, int n_in, int n_hidden,
                                int n_out, float *xs, float *hs, float *ls) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int k = threadIdx.x; k < n_in; k += blockDim.x) xs[k] = X[(int64_t)b * n_in + k];
  __syncthreads();
  for (int j = threadIdx.x; j < n_hidden; j += blockDim.x) {
    const float *w = W1 + (int64_t)j * ld1;
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
  return ce;
}

// One block per sample; the per-sample losses are summed in sample order by the last block.
__global__ void __launch_bounds__(256)
mlp_loss_kernel(const float *__restrict__ P, const float *__restrict__ X,
                const int32_t *__restrict__ y, int n_in, int n_hidden, int n_out,
                double *partials, unsigned int *counter, double *out, int accumulate,
                double scale) {
  __shared__ float xs[kMlpMax], hs[kMlpMax], ls[kMlpMax];
  const float *b1 = P + (int64_t)n_hidden * n_in;
  const float *W2 = b1 + n_hidden;
  const float *b2 = W2 + (int64_t)n_out * n_hidden;
  const double ce = mlp_sample_ce(P, n_in, b1, W2, b2, X, y, blockIdx.x, n_in, n_hidden, n_out,
                                  xs, hs, ls);
  finish_reduction(ce, partials, counter, out, accumulate, scale);
}

// All the losses of one MLP step in one launch: blockIdx.x = evaluation e (e < clean: the
// clean loss; then probe (e - clean) / 2 at +eps for even e - clean and at -eps for odd),
// blockIdx.y = a slice of per_cta samples.  The block stages its evaluation's parameters
// rd(theta + s eps z) in shared memory (the sign masks of the 16-element groups first, then
// one coalesced pass; W1's rows padded to n_in + 1 floats, so that the threads of the hidden
// layer, one row each, read distinct banks) and writes each sample's cross-entropy to ce[e][b].
__global__ void __launch_bounds__(256)
mlp_probes_kernel(const float *__restrict__ theta, int M, const float *__restrict__ X,
                  const int32_t *__restrict__ y, int batch, int n_in, int n_hidden, int n_out,
                  ProbeKey pk, int clean, int per_cta, double *__restrict__ ce) {
  extern __shared__ __align__(16) float Ps[];  // M + n_hidden parameters, then the masks
  __shared__ float xs[kMlpMax], hs[kMlpMax], ls[kMlpMax];
  const int n_w1 = n_hidden * n_in, ld1 = n_in + 1;
  uint16_t *masks = reinterpret_cast<uint16_t *>(Ps + M + n_hidden);
  const int e = blockIdx.x;
  const bool perturbed = e >= clean;
  const int k = e - clean;
  const float delta = (k & 1) ? -pk.eps : pk.eps;
  if (perturbed) {
    const uint32_t step = *pk.step;
    for (int g = threadIdx.x; g < (M + kGroup - 1) / kGroup; g += blockDim.x)
      masks[g] = (uint16_t)probe_group_bits((uint64_t)g, (uint32_t)(k >> 1), step, pk.k0, pk.k1);
    __syncthreads();
  }
  for (int j = threadIdx.x; j < M; j += blockDim.x) {
    const float t = theta[j];
    const float v = perturbed ? perturb_f32(t, delta, (masks[j >> 4] >> (j & 15)) & 1u) : t;
    Ps[j < n_w1 ? (j / n_in) * ld1 + j % n_in : j + n_hidden] = v;
  }
  __syncthreads();
  const float *b1s = Ps + n_hidden * ld1;
  const float *W2s = b1s + n_hidden;
  const float *b2s = W2s + n_out * n_hidden;
  const int bend = min(batch, (blockIdx.y + 1) * per_cta);
  for (int b = blockIdx.y * per_cta; b < bend; ++b) {
    const double v = mlp_sample_ce(Ps, ld1, b1s, W2s, b2s, X, y, b, n_in, n_hidden, n_out, xs, hs, ls);
    if (threadIdx.x == 0) ce[(int64_t)e * batch + b] = v;
  }
}

// Block e sums evaluation e's per-sample losses in the order of mlp_loss_kernel's reduction
// (same block size, strided sums, then the block tree) and stores scale * sum.
__global__ void __launch_bounds__(256)
mlp_probes_sum_kernel(const double *__restrict__ ce, int batch, double scale, int clean,
                      double *l0, double *lp, double *lm) {
  const int e = blockIdx.x;
  double s = 0.0;
  for (int i = threadIdx.x; i < batch; i += blockDim.x) s += ce[(int64_t)e * batch + i];
  s = block_sum(s);
  if (threadIdx.x == 0) {
    const int k = e - clean;
    double *o = e < clean ? l0 : ((k & 1) ? lm : lp) + (k >> 1);
    *o = 0.0 + scale * s;
  }
}

}  // namespace

namespace {

template <bool PAIR, int R>
zo_status launch_quad(zo_ctx *ctx, const ProbeKey &pk, const float *D, double *out,
                      double *out_minus, int accumulate, double *partials, unsigned int *counter,
                      const LowRankArgs &lr = LowRankArgs{}) {
  const int64_t n_chunks = (ctx->M + kQChunk - 1) / kQChunk;
  int64_t blocks = n_chunks < (int64_t)kSmCount * 2 ? n_chunks : (int64_t)kSmCount * 2;
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(quad_loss_kernel<PAIR, R>), kQSmemBytes);
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "quad_loss_kernel attribute: %s", cudaGetErrorString(e));
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

template <bool CLEAN, int NOCT, bool DOT>
zo_status launch_quad_octet_t(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                              const float *D, double *out_plus, double *out_minus, double *out_clean,
                              int dir, uint32_t vk0, uint32_t vk1) {
  const int64_t n_chunks = (ctx->M + kOChunk - 1) / kOChunk;
  const int64_t cap = (int64_t)kSmCount * kOBlocksPerSm;
  const int64_t blocks = n_chunks < cap ? n_chunks : cap;
  static_assert((8 * NOCT + 2) * kSmCount * kOBlocksPerSm <= kMaxPartials,
                "partials too small for the octet pass");
  {
    const cudaError_t e =
        ensure_smem_limit(reinterpret_cast<const void *>(quad_octet_kernel<CLEAN, NOCT, DOT>), kOSmemBytes);
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "quad_octet_kernel attribute: %s", cudaGetErrorString(e));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = kOSmemBytes;
  cfg.stream = ctx->stream;
  cudaLaunchAttribute attr_pdl[1];
  attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, quad_octet_kernel<CLEAN, NOCT, DOT>,
                                           static_cast<const float *>(ctx->params), D, ctx->M, pk,
                                           round_keys(pk.k0, pk.k1), octet, count, n_chunks, ctx->partials, ctx->counter,
                                           out_plus, out_minus, out_clean, &ctx->dstate->flags, dir, vk0,
                                           vk1);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "quad_octet_kernel: %s", cudaGetErrorString(e));
  return check_launch(ctx, "quad_octet_kernel");
}

// NOCT by count: 8 octets above 32 probes, 4 above 16, else 2.
template <bool DOT>
zo_status launch_octet_any(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                           const float *D, double *out_plus, double *out_minus, double *out_clean,
                           int dir, uint32_t vk0, uint32_t vk1) {
#define ZO_OCTET(C, N) launch_quad_octet_t<C, N, DOT>(ctx, pk, octet, count, D, out_plus, out_minus, \
                                                     C ? out_clean : nullptr, dir, vk0, vk1)
  if (count > 32) return out_clean ? ZO_OCTET(true, 8) : ZO_OCTET(false, 8);
  if (count > 16) return out_clean ? ZO_OCTET(true, 4) : ZO_OCTET(false, 4);
  return out_clean ? ZO_OCTET(true, 2) : ZO_OCTET(false, 2);
#undef ZO_OCTET
}

zo_status launch_quad_octet(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                            const float *D, double *out_plus, double *out_minus, double *out_clean) {
  return launch_octet_any<false>(ctx, pk, octet, count, D, out_plus, out_minus, out_clean, 0, 0u, 0u);
}

zo_status launch_lowrank_dot_octet(zo_ctx *ctx, const ProbeKey &pk, uint32_t octet, int count,
                                   int dir, uint64_t vseed, double *out_plus, double *out_minus,
                                   double *out_clean) {
  return launch_octet_any<true>(ctx, pk, octet, count, nullptr, out_plus, out_minus, out_clean, dir,
                                (uint32_t)vseed, (uint32_t)(vseed >> 32));
}

namespace {
// out[i] = base[i] + sum_r (lam_r / 2 / M) dots[r][i]^2 for the 2n + 1 values of a low-rank
// step ([L0, L+..., L-...]; i = 0 only with the clean loss), with the combination of the
// one-probe low-rank pass.
__global__ void lowrank_combine_kernel(const double *__restrict__ base, const double *__restrict__ dots,
                                       int rank, int n, LowRankArgs lr, int64_t M, int clean,
                                       double *__restrict__ out) {
  const double inv_m = 1.0 / (double)M;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x + (clean ? 0 : 1); i < 2 * n + 1;
       i += gridDim.x * blockDim.x) {
    double L = base[i];
    for (int r = 0; r < rank; ++r) {
      const double t = dots[(int64_t)r * (2 * n + 1) + i];
      L = __dadd_rn(L, __dmul_rn(__dmul_rn(0.5 * (double)lr.lam[r], inv_m), __dmul_rn(t, t)));
    }
    out[i] = L;
  }
}
}  // namespace

zo_status launch_lowrank_combine(zo_ctx *ctx, const double *base, const double *dots, int rank,
                                 int n, const float lam[4], int clean, double *out) {
  LowRankArgs lr;
  for (int k = 0; k < 4; ++k) lr.lam[k] = lam[k];
  lr.vk0 = lr.vk1 = 0u;
  const int blocks = (2 * n + 1 + 255) / 256;
  lowrank_combine_kernel<<<blocks, 256, 0, ctx->stream>>>(base, dots, rank, n, lr, ctx->M, clean, out);
  return check_launch(ctx, "lowrank_combine_kernel");
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

zo_status launch_mlp_probes(zo_ctx *ctx, const float *X, const int32_t *y, int batch, int n_in,
                            int n_hidden, int n_out, int n_pert, float eps, double scale,
                            double *lp, double *lm, double *l0) {
  if (n_in > kMlpMax || n_hidden > kMlpMax || n_out > kMlpMax || batch < 1)
    return fail(ctx, ZO_ERR_INVALID, "mlp shape beyond limits");
  if (ctx->M + n_hidden > kMlpStageMax)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "batched MLP losses need M + n_hidden <= %d", kMlpStageMax);
  const int clean = l0 ? 1 : 0;
  const int E = 2 * n_pert + clean;
  const size_t need = (size_t)E * (size_t)batch;
  if (need > ctx->mlp_ce_cap) {
    cudaFree(ctx->mlp_ce);
    ctx->mlp_ce = nullptr;
    ctx->mlp_ce_cap = 0;
    const cudaError_t e = cudaMalloc(&ctx->mlp_ce, need * sizeof(double));
    if (e != cudaSuccess) return fail(ctx, e == cudaErrorMemoryAllocation ? ZO_ERR_OOM : ZO_ERR_CUDA,
                                      "mlp loss scratch: %s", cudaGetErrorString(e));
    ctx->mlp_ce_cap = need;
  }
  const int M = (int)ctx->M;
  const size_t smem = (size_t)(M + n_hidden) * sizeof(float) +
                      (size_t)((M + kGroup - 1) / kGroup) * sizeof(uint16_t);
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(mlp_probes_kernel),
                                            (int)(kMlpStageMax * sizeof(float) + kMlpStageMax / 8));
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "mlp_probes_kernel attribute: %s", cudaGetErrorString(e));
  }
  ProbeKey pk = probe_key(ctx);
  pk.sign = +1;
  pk.eps = eps;
  // about 8 samples per block: the blocks of a step fill the GPU once at the pages' sizes
  const int per_cta = batch < 8 ? batch : 8;
  const dim3 grid((unsigned)E, (unsigned)((batch + per_cta - 1) / per_cta));
  mlp_probes_kernel<<<grid, 256, smem, ctx->stream>>>(static_cast<const float *>(ctx->params), M, X, y,
                                                      batch, n_in, n_hidden, n_out, pk, clean,
                                                      per_cta, ctx->mlp_ce);
  const zo_status st = check_launch(ctx, "mlp_probes_kernel");
  if (st != ZO_OK) return st;
  mlp_probes_sum_kernel<<<E, 256, 0, ctx->stream>>>(ctx->mlp_ce, batch, scale, clean, l0, lp, lm);
  return check_launch(ctx, "mlp_probes_sum_kernel");
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
constexpr int kNoallocMaxEntries = 64;

// [0, kNoallocPartialsBytes): fp64 partials; then the unsigned ticket counter.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocPartialsBytes + 256];

// The array's device address, looked up once per (device, CUDA context): a caller that makes
// a context of its own current gets that context's copy of the array.
struct NoallocEntry {
  int device;
  void *context;
  void *addr;
};
std::mutex g_noalloc_mu;
NoallocEntry g_noalloc_cache[kNoallocMaxEntries];
int g_noalloc_used = 0;

using CtxGetCurrentFn = int (*)(void **);  // cuCtxGetCurrent(CUcontext *)

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the scratch in the current device's current context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up (once per device
// and context, with that device current) with cudaGetSymbolAddress.
cudaError_t noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  void *context = nullptr;
  if (CtxGetCurrentFn fn = ctx_get_current()) fn(&context);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < g_noalloc_used; ++i)
    if (g_noalloc_cache[i].device == dev && g_noalloc_cache[i].context == context) {
      *out = g_noalloc_cache[i].addr;
      return cudaSuccess;
    }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  if (g_noalloc_used < kNoallocMaxEntries) g_noalloc_cache[g_noalloc_used++] = {dev, context, p};
  *out = p;
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
