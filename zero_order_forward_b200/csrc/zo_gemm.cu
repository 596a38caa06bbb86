// zo_gemm.cu -- bf16 GEMM on the 5th-generation tensor cores for the decoder forward:
//   out[M][N] = epilogue(A[M][K] . B[N][K]^T + bias[N])
// A (activations) and B (weights, nn.Linear layout) are both K-major.  This is the only
// dense contraction on the path (the decoder's QKV, output, FC1 and FC2 projections).
//
// Design (persistent, one CTA of 320 threads per SM, 128 x BN output tiles):
//   warp 0     one lane issues TMA tile loads (128-byte swizzle) into a STAGES-deep ring
//              of shared-memory stages, paced by "empty" mbarriers;
//   warp 1     allocates 2*BN TMEM columns (two accumulators); one lane issues
//              tcgen05.mma (M=128, N=BN, K=16, bf16 x bf16 -> fp32 in TMEM), commits each
//              stage back to its "empty" barrier and each finished accumulator to the
//              epilogue;
//   warps 2-9  the epilogue, two warps per TMEM lane quadrant (warp w reads TMEM lanes
//              32*(w%4)..+31 = its 32 output rows, half of the columns each): tcgen05.ld
//              32 columns at a time, bias and ReLU, a swizzled 32 x 32 staging tile in
//              shared memory, then one TMA tile store (bf16 outputs) or TMA add-reduce into
//              the fp32 residual stream (global += tile in L2, no load by the SM); the
//              accumulator is handed back after its last TMEM read.
// SwiGLU epilogue (ZO_EPI_SWIGLU_BF16): the weight is [Wg; Wu] (2N rows); a tile of BN/2
// output columns loads BN/2 gate rows and the matching BN/2 up rows into one BN-row
// operand stage, so TMEM columns c and BN/2 + c of the accumulator hold the gate and up
// products of output column c, combined as silu(g) * u in fp32 before one bf16 rounding.
// Tiles are visited in groups of row tiles (sized from K so that a group's rows of A, about
// 64 MB, stay in the 126 MB L2) so that both the group's A rows and each weight tile are reused
// from L2.  All waits are bounded (see zo_tc.cuh); a timeout sets an error bit.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "zo_internal.cuh"
#include "zo_tc.cuh"

namespace zo {

namespace {

constexpr int kBM = 128, kBK = 64;

struct GemmArgs {
  int M, N, K;
  int group_m;           // row tiles per group of the tile order
  const uint16_t *bias;  // [N] bf16 or null
  void *out;             // bf16 [M][ldo] or fp32 [M][ldo]
  int ldo;
  uint32_t *err;         // device error word (ZO_FLAG_TIMEOUT raised on a bounded-wait expiry)
  uint32_t extra_tx;     // 0; a test hook sets it so that the first stage never completes
  int64_t w_off;         // fused perturbation: flat index of B's element (0, 0) in the context
};

__device__ __forceinline__ void load_bias32(const uint16_t *bias, int col0, int N, float b[32]) {
  if (bias == nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) b[i] = 0.f;
    return;
  }
  if (col0 + 32 <= N) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 u = __ldg(reinterpret_cast<const uint4 *>(bias + col0) + k);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        b[8 * k + 2 * t] = __uint_as_float(w[t] << 16);
        b[8 * k + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) b[i] = (col0 + i < N) ? bf16_bits_to_f32(bias[col0 + i]) : 0.f;
  }
}

// Write one accumulator row chunk (32 columns of row `r` of a 32 x 32 tile) into the
// warp's staging tile in the layout the output tensor map's swizzle expects:
//   fp32: 128-byte rows, 16-byte chunk c stored at chunk c ^ (r & 7)   (128B swizzle);
//   bf16:  64-byte rows, 16-byte chunk c stored at chunk c ^ ((r >> 1) & 3) (64B swizzle).
__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + expf(-g)) * u; }

template <int EPI>
__device__ __forceinline__ void stage_row(uint8_t *stage, int r, const float v[32]) {
  if (EPI == ZO_EPI_RESID_F32) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<float4 *>(stage + r * 128 + ((c ^ (r & 7)) << 4)) =
          make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        w[t] = pack_bf16x2(v[8 * c + 2 * t], v[8 * c + 2 * t + 1]);
      *reinterpret_cast<uint4 *>(stage + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

constexpr int kEpiWarps = 8;                      // two warps per TMEM lane quadrant
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);  // producer, MMA, epilogue
constexpr int kXWarps = 4;                          // fused perturbation: transform warps
constexpr int kGemmThreadsX = kGemmThreads + 32 * kXWarps;
constexpr uint32_t kStageTile = 32 * 128;           // one 32 x 32 fp32 (or bf16) output tile

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOutOffset = STAGES * kStageBytes;         // 1024-aligned
  static constexpr uint32_t kBarOffset = kOutOffset + kEpiWarps * kStageTile;
  static constexpr uint32_t kBytes = kBarOffset + 256 + 1024;  // + barriers + alignment slack
  // full, empty, ready [STAGES]; acc_full, acc_empty [2]; mma_done; TMEM address; abort flag
  static_assert((3 * STAGES + 5) * 8 + 8 <= 256, "barrier area");
};

struct TileCoord {
  int m0, n0;
};

// Grouped order: group_m row tiles share each sweep over the column tiles, so a group's rows
// of A and each weight tile are reused from L2.
__device__ __forceinline__ TileCoord tile_coord(int t, int num_m, int num_n, int BN, int group_m) {
  const int group = t / (group_m * num_n);
  const int first_m = group * group_m;
  const int gsize = min(num_m - first_m, group_m);
  const int m_tile = first_m + (t % gsize);
  const int n_tile = (t % (group_m * num_n)) / gsize;
  return {m_tile * kBM, n_tile * BN};
}

// Row tiles per group: rows * K * 2 bytes of A near 128 MB, between 1 and 16 tiles (measured:
// K = 7168 pair tiles read 6.7 GB from DRAM with 16 per group against 9.7 GB with 8; K = 28672
// read 17.4 GB with 8 against 22 GB with 4).
int group_rows_for(int K, int rows_per_tile) {
  const int64_t per_tile = (int64_t)rows_per_tile * K * 2;
  int64_t g = ((int64_t)128 << 20) / (per_tile > 0 ? per_tile : 1);
  return (int)(g < 1 ? 1 : g > 16 ? 16 : g);
}

// Eight bf16 weights of one 16-byte chunk perturbed as the window kernel does it: element t
// takes sign bit t of `bits` (1: z = -1), P = rd_bf16(theta + (s eps) z) with the sign xor-ed
// into s eps (db: the bits of s eps).
__device__ __forceinline__ uint4 perturb8_bf16(uint4 v, uint32_t bits, uint32_t db) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float lo = __fadd_rn(__uint_as_float(w[t] << 16),
                               __uint_as_float(db ^ ((bits << (31 - 2 * t)) & 0x80000000u)));
    const float hi = __fadd_rn(__uint_as_float(w[t] & 0xFFFF0000u),
                               __uint_as_float(db ^ ((bits << (30 - 2 * t)) & 0x80000000u)));
    w[t] = pack_bf16x2(lo, hi);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// All lanes of the warp wait for `parity` on `bar` (lane 0 decides, bounded; then every lane
// observes the completed phase).  False on every lane on expiry or abort.
__device__ __forceinline__ bool gemm_warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) ok = (!*abort_flag && tc::mbar_wait(bar, parity)) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok && lane != 0) ok = tc::mbar_wait(bar, parity) ? 1 : 0;
  return __all_sync(0xFFFFFFFFu, ok) != 0;
}

// Persistent: one CTA per SM walks tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// The shared-memory ring runs across tile boundaries, and the accumulator is
// double-buffered in TMEM (2 x BN columns) so the epilogue of tile i overlaps the
// main loop of tile i+1.
//
// PERT (the perturbation fused into the operand path): B is a bf16 weight matrix inside the
// context's parameters (row n, column k at flat index args.w_off + n K + k), and the MMA
// multiplies by its perturbed copy P = rd(theta + s eps z_i) under `pk` without a window in
// HBM.  Four more warps wait for each stage, regenerate the probe's signs for its B tile
// (one Philox block per 16-column group of a row) and perturb the tile in shared memory in
// place (the 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7)), then
// release the stage to the MMA through ready[s].  Every row tile re-does this for the weight
// tiles it reads.
template <int BN, int STAGES, int EPI, bool PERT>
__global__ void __launch_bounds__(PERT ? kGemmThreadsX : kGemmThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, GemmArgs args, ProbeKey pk,
                 const __grid_constant__ RoundKeys rk) {
  using S = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * S::kABytes;
  uint8_t *sOut = smem + S::kOutOffset;  // one 32 x 32 staging tile per epilogue warp
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S::kBarOffset);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;   // [2] MMA -> epilogue
  uint64_t *acc_empty = acc_full + 2;    // [2] epilogue -> MMA
  uint64_t *mma_done = acc_empty + 2;    // all MMAs of this CTA retired
  uint64_t *ready = mma_done + 1;        // [STAGES] PERT: B tile of the stage perturbed
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(ready + STAGES);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  constexpr bool kSwiGLU = EPI == ZO_EPI_SWIGLU_BF16;
  static_assert(!(PERT && kSwiGLU), "the fused perturbation takes one weight matrix");
  constexpr int OUT_BN = kSwiGLU ? BN / 2 : BN;  // output columns per tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (args.M + kBM - 1) / kBM, num_n = (args.N + OUT_BN - 1) / OUT_BN;
  const int num_tiles = num_m * num_n;
  const int nk = (args.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], kEpiWarps);  // one arrival per epilogue warp
    }
    tc::mbar_init(mma_done, 1);
    if (PERT)
      for (int s = 0; s < STAGES; ++s) tc::mbar_init(&ready[s], kXWarps);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, 2 * BN);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  uint32_t issued = 0;  // producer: k-blocks issued (global ring position)
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      const TileCoord tc0 = tile_coord(t, num_m, num_n, OUT_BN, args.group_m);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t s = issued % STAGES, ph = (issued / STAGES) & 1u;
        if (*abort_flag || !tc::mbar_wait(&empty[s], ph ^ 1u)) {
          atomicOr(args.err, ZO_FLAG_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&full[s], S::kStageBytes + (issued == 0 ? args.extra_tx : 0u));
        tc::tma_load_2d(sA + s * S::kABytes, &tmA, &full[s], kb * kBK, tc0.m0);
        if (kSwiGLU) {  // gate rows n0.., then up rows N + n0.. (the map's box is BN/2 rows)
          tc::tma_load_2d(sB + s * S::kBBytes, &tmB, &full[s], kb * kBK, tc0.n0);
          tc::tma_load_2d(sB + s * S::kBBytes + S::kBBytes / 2, &tmB, &full[s], kb * kBK,
                          args.N + tc0.n0);
        } else {
          tc::tma_load_2d(sB + s * S::kBBytes, &tmB, &full[s], kb * kBK, tc0.n0);
        }
        ++issued;
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(kBM, BN);
    uint32_t consumed = 0;
    int i = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x, ++i) {
      const int b = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (!tc::mbar_wait(&acc_empty[b], aph ^ 1u)) {
        atomicOr(args.err, ZO_FLAG_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc::tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * BN);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t s = consumed % STAGES, ph = (consumed / STAGES) & 1u;
        // PERT: the stage is complete once its B tile has been perturbed (which follows the
        // transform warps' wait on full[s])
        if (*abort_flag || !tc::mbar_wait(PERT ? &ready[s] : &full[s], ph)) {
          atomicOr(args.err, ZO_FLAG_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc::tc_fence_after();
        const uint32_t a0 = tc::smem_addr(sA + s * S::kABytes);
        const uint32_t b0 = tc::smem_addr(sB + s * S::kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          tc::mma_bf16(d, tc::smem_desc_k128(a0 + 32 * k), tc::smem_desc_k128(b0 + 32 * k), idesc,
                       (kb | k) != 0 ? 1u : 0u);
        tc::mma_commit(&empty[s]);
        ++consumed;
      }
      if (*abort_flag) break;
      tc::mma_commit(&acc_full[b]);
    }
    tc::mma_commit(mma_done);  // arrives once every MMA issued above has retired
  } else if (PERT && warp >= 2 + kEpiWarps) {
    // transform warps: thread xt perturbs rows xt, xt + 128, ... of each stage's B tile
    const int xt = threadIdx.x - 32 * (2 + kEpiWarps);
    const uint32_t step = pk.sign ? *pk.step : 0u;
    const uint32_t db = __float_as_uint(pk.sign > 0 ? pk.eps : -pk.eps);
    uint32_t consumed = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
      const TileCoord tc0 = tile_coord(t, num_m, num_n, OUT_BN, args.group_m);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t s = consumed % STAGES, ph = (consumed / STAGES) & 1u;
        if (!gemm_warp_wait(&full[s], ph, abort_flag)) {
          if (lane == 0) atomicOr(args.err, ZO_FLAG_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (pk.sign) {
          uint8_t *st = sB + s * S::kBBytes;
#pragma unroll 1
          for (int r = xt; r < BN; r += 32 * kXWarps) {
            const int n = tc0.n0 + r;
            if (n >= args.N) break;  // rows past N stay as loaded (zero)
            const int64_t e0 = args.w_off + (int64_t)n * args.K + (int64_t)kb * kBK;
#pragma unroll
            for (int q = 0; q < kBK / 16; ++q) {
              if (kb * kBK + 16 * q >= args.K) break;  // K % 16 == 0: a group is whole or absent
              const uint32_t bits =
                  probe_group_bits(pk.g_off + (uint64_t)((e0 + 16 * q) >> 4), pk.probe, step, rk);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c = 2 * q + h;  // 16-byte chunk of the 128-byte row
                uint4 *p = reinterpret_cast<uint4 *>(st + r * 128 + ((c ^ (r & 7)) << 4));
                *p = perturb8_bf16(*p, bits >> (8 * h), db);
              }
            }
          }
          tc::fence_proxy_async_smem();  // these writes precede the tensor core's reads
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&ready[s]);
        ++consumed;
      }
    }
  } else if (warp >= 2) {
    const int q = warp & 3;                    // TMEM lanes 32q..32q+31 (this warp's rows)
    const int half = (warp - 2) / 4;           // which half of the output columns
    const int cbeg = half * (OUT_BN / 2), cend = cbeg + OUT_BN / 2;
    uint8_t *stage = sOut + (warp - 2) * kStageTile;
    if (lane == 0) tc::tma_prefetch_desc(&tmC);
    int i = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (*abort_flag || !tc::mbar_wait(&acc_full[b], aph)) {
        if (lane == 0) atomicOr(args.err, ZO_FLAG_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc::tc_fence_after();
      const TileCoord tc0 = tile_coord(t, num_m, num_n, OUT_BN, args.group_m);
      const int row0 = tc0.m0 + q * 32;
      const uint32_t base = tmem + (uint32_t)(b * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
        if (tc0.n0 + c0 >= args.N) break;
        float v[32];
        tc::tmem_ld32(base + (uint32_t)c0, v);
        if (kSwiGLU) {
          float u[32];
          tc::tmem_ld32(base + (uint32_t)(BN / 2 + c0), u);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = silu_mul(v[k], u[k]);
        } else {
          float bias[32];
          load_bias32(args.bias, tc0.n0 + c0, args.N, bias);
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            v[k] = __fadd_rn(v[k], bias[k]);
            if (EPI == ZO_EPI_RELU_BF16) v[k] = fmaxf(v[k], 0.f);
          }
        }
        // the previous chunk's bulk store must have finished reading the staging tile
        if (lane == 0) tc::bulk_wait_read0();
        __syncwarp();
        stage_row<EPI>(stage, lane, v);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.M) {
          if (EPI == ZO_EPI_RESID_F32) tc::tma_reduce_add_2d(&tmC, stage, tc0.n0 + c0, row0);
          else tc::tma_store_2d(&tmC, stage, tc0.n0 + c0, row0);
          tc::bulk_commit();
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
    }
    if (lane == 0) tc::bulk_wait0();  // this warp's stores and reductions have landed
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let this CTA's TMA loads still in flight land before it exits (bounded)
    for (uint32_t s = 0; s < STAGES; ++s) {
      if (issued <= s) continue;
      const uint32_t last = s + ((issued - 1 - s) / STAGES) * STAGES;
      if (!tc::mbar_wait(&full[s], (last / STAGES) & 1u)) atomicOr(args.err, ZO_FLAG_TIMEOUT);
    }
  }
  if (warp == 1) {
    if (lane == 0 && !tc::mbar_wait(mma_done, 0)) atomicOr(args.err, ZO_FLAG_TIMEOUT);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 2 * BN);
  }
}

// ------------------------------------------------------------------ CTA-pair form (cta_group::2)
// For the large projections: clusters of 2 CTAs on neighbouring SMs compute 256 x 256 tiles
// (SwiGLU: 256 rows x 128 output columns).  Each CTA holds its 128 A rows and its 128 of the
// 256 B rows per stage (32 KB instead of 48 KB per SM and stage), so the shared-memory traffic
// per MMA is two thirds of the single-CTA form's.  Warp 0 of each CTA loads its halves into
// its own stages, the bytes completing the leader's (CTA 0's) full barrier; one thread of the
// leader issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) and commits each stage and
// each finished accumulator to the barriers of both CTAs; the 8 epilogue warps of each CTA
// read their own tensor memory (their 128 rows) exactly as in the single-CTA form and release
// the accumulator on the leader's barrier.
constexpr int kPairBN = 256;  // accumulator columns of a pair tile (the MMA's N)

template <int STAGES>
struct PairSmem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;          // this CTA's 128 rows of A
  static constexpr uint32_t kBBytes = (kPairBN / 2) * kBK * 2;  // this CTA's 128 rows of B
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kOutOffset = STAGES * kStageBytes;  // 1024-aligned
  static constexpr uint32_t kBarOffset = kOutOffset + kEpiWarps * kStageTile;
  static constexpr uint32_t kBytes = kBarOffset + 256 + 1024;
};

__device__ __forceinline__ TileCoord pair_tile_coord(int t, int num_m, int num_n, int out_bn,
                                                    int group_m) {
  const TileCoord c = tile_coord(t, num_m, num_n, out_bn, group_m);
  return {c.m0 / kBM * (2 * kBM), c.n0};  // tile_coord's row tiles are pair tiles of 256 rows
}

template <int STAGES, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, GemmArgs args) {
  using S = PairSmem<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * S::kABytes;
  uint8_t *sOut = smem + S::kOutOffset;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + S::kBarOffset);  // used in the leader
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;  // [2]
  uint64_t *acc_empty = acc_full + 2;   // [2] used in the leader: both CTAs' epilogue warps
  uint64_t *mma_done = acc_empty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  constexpr bool kSwiGLU = EPI == ZO_EPI_SWIGLU_BF16;
  constexpr int OUT_BN = kSwiGLU ? kPairBN / 2 : kPairBN;  // output columns per tile
  const uint32_t rank = tc::cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (args.M + 2 * kBM - 1) / (2 * kBM), num_n = (args.N + OUT_BN - 1) / OUT_BN;
  const int num_tiles = num_m * num_n;
  const int nk = (args.K + kBK - 1) / kBK;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], 2 * kEpiWarps);  // the epilogue warps of both CTAs
    }
    tc::mbar_init(mma_done, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc_pair(tmem_holder, 2 * kPairBN);
  tc::tc_fence_before();
  tc::cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t full_leader = tc::map_to_rank(full, 0);
  const uint32_t acc_empty_leader = tc::map_to_rank(acc_empty, 0);
  const uint32_t abort_peer = tc::map_to_rank(const_cast<int *>(abort_flag), rank ^ 1u);
  auto raise_abort = [&]() {
    atomicOr(args.err, ZO_FLAG_TIMEOUT);
    *abort_flag = 1;
    tc::st_remote_u32(abort_peer, 1u);
  };

  uint32_t issued = 0;  // producer: k-blocks issued (global ring position)
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
    for (int t = cluster; t < num_tiles && !*abort_flag; t += n_clusters) {
      const TileCoord tc0 = pair_tile_coord(t, num_m, num_n, OUT_BN, args.group_m);
      // SwiGLU: CTA 0 loads the tile's gate rows, CTA 1 the matching up rows
      const int b_row = kSwiGLU ? (int)(rank ? args.N + tc0.n0 : tc0.n0) : tc0.n0 + (int)rank * (kPairBN / 2);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t s = issued % STAGES, ph = (issued / STAGES) & 1u;
        if (*abort_flag || !tc::mbar_wait(&empty[s], ph ^ 1u)) {
          raise_abort();
          break;
        }
        if (leader) tc::mbar_arrive_expect_tx(&full[s], 2 * S::kStageBytes);  // both CTAs' halves
        tc::tma_load_2d_pair(sA + s * S::kABytes, &tmA, full_leader + 8u * s, kb * kBK,
                             tc0.m0 + (int)rank * kBM);
        tc::tma_load_2d_pair(sB + s * S::kBBytes, &tmB, full_leader + 8u * s, kb * kBK, b_row);
        ++issued;
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(2 * kBM, kPairBN);
    uint32_t consumed = 0;
    int i = 0;
    for (int t = cluster; t < num_tiles && !*abort_flag; t += n_clusters, ++i) {
      const int b = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (!tc::mbar_wait(&acc_empty[b], aph ^ 1u)) {
        raise_abort();
        break;
      }
      tc::tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * kPairBN);
      for (int kb = 0; kb < nk; ++kb) {
        const uint32_t s = consumed % STAGES, ph = (consumed / STAGES) & 1u;
        if (*abort_flag || !tc::mbar_wait(&full[s], ph)) {
          raise_abort();
          break;
        }
        tc::tc_fence_after();
        const uint32_t a0 = tc::smem_addr(sA + s * S::kABytes);
        const uint32_t b0 = tc::smem_addr(sB + s * S::kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          tc::mma_bf16_pair(d, tc::smem_desc_k128(a0 + 32 * k), tc::smem_desc_k128(b0 + 32 * k), idesc,
                            (kb | k) != 0 ? 1u : 0u);
        tc::mma_commit_pair(&empty[s]);
        ++consumed;
      }
      if (*abort_flag) break;
      tc::mma_commit_pair(&acc_full[b]);
    }
    tc::mma_commit_pair(mma_done);  // arrives (in both CTAs) once every MMA above has retired
  } else if (warp >= 2) {
    const int q = warp & 3;           // TMEM lanes 32q..32q+31 (this warp's rows)
    const int half = (warp - 2) / 4;  // which half of the output columns
    const int cbeg = half * (OUT_BN / 2), cend = cbeg + OUT_BN / 2;
    uint8_t *stage = sOut + (warp - 2) * kStageTile;
    if (lane == 0) tc::tma_prefetch_desc(&tmC);
    int i = 0;
    for (int t = cluster; t < num_tiles; t += n_clusters, ++i) {
      const int b = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = (!*abort_flag && tc::mbar_wait(&acc_full[b], aph)) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (ok && lane != 0) ok = tc::mbar_wait(&acc_full[b], aph) ? 1 : 0;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) raise_abort();
        break;
      }
      tc::tc_fence_after();
      const TileCoord tc0 = pair_tile_coord(t, num_m, num_n, OUT_BN, args.group_m);
      const int row0 = tc0.m0 + (int)rank * kBM + q * 32;
      const uint32_t base = tmem + (uint32_t)(b * kPairBN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int c0 = cbeg; c0 < cend; c0 += 32) {
        if (tc0.n0 + c0 >= args.N) break;
        float v[32];
        tc::tmem_ld32(base + (uint32_t)c0, v);
        if (kSwiGLU) {
          float u[32];
          tc::tmem_ld32(base + (uint32_t)(kPairBN / 2 + c0), u);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = silu_mul(v[k], u[k]);
        } else {
          float bias[32];
          load_bias32(args.bias, tc0.n0 + c0, args.N, bias);
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            v[k] = __fadd_rn(v[k], bias[k]);
            if (EPI == ZO_EPI_RELU_BF16) v[k] = fmaxf(v[k], 0.f);
          }
        }
        // the previous chunk's bulk store must have finished reading the staging tile
        if (lane == 0) tc::bulk_wait_read0();
        __syncwarp();
        stage_row<EPI>(stage, lane, v);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.M) {
          if (EPI == ZO_EPI_RESID_F32) tc::tma_reduce_add_2d(&tmC, stage, tc0.n0 + c0, row0);
          else tc::tma_store_2d(&tmC, stage, tc0.n0 + c0, row0);
          tc::bulk_commit();
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) tc::mbar_arrive(&acc_empty[b]);
        else tc::mbar_arrive_remote(acc_empty_leader + 8u * (uint32_t)b);
      }
    }
    if (lane == 0) tc::bulk_wait0();  // this warp's stores and reductions have landed
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    if (leader) {
      // let the pair's loads still in flight land before either CTA exits (bounded)
      for (uint32_t s = 0; s < STAGES; ++s) {
        if (issued <= s) continue;
        const uint32_t last = s + ((issued - 1 - s) / STAGES) * STAGES;
        if (!tc::mbar_wait(&full[s], (last / STAGES) & 1u)) atomicOr(args.err, ZO_FLAG_TIMEOUT);
      }
    } else {
      __nanosleep(1000000);  // the peer cannot observe its loads' completion: give them time
    }
  }
  __syncwarp();
  if (warp == 1) {
    if (lane == 0 && !tc::mbar_wait(mma_done, 0)) atomicOr(args.err, ZO_FLAG_TIMEOUT);
    __syncwarp();
    tc::tc_fence_after();
  }
  tc::cluster_sync();  // no remote arrival or MMA touches either CTA after this point
  if (warp == 1) tc::tmem_dealloc_pair(tmem, 2 * kPairBN);
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Output tile map: [rows][cols] with row stride ld elements, box 32 x 32; fp32 uses the
// 128-byte swizzle (128-byte box rows), bf16 the 64-byte swizzle (64-byte box rows).
// Stores outside [rows][cols] are clipped by the hardware.
bool make_out_map(CUtensorMap *m, void *base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor [rows][cols] (row-major, cols contiguous), box = box_rows x 64 columns,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows,
              int64_t ld = 0) {  // ld: elements between row starts (0: cols)
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld ? ld : cols) * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int STAGES, int EPI, bool PERT = false>
cudaError_t launch_one(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tcm,
                       const GemmArgs &g, cudaStream_t st, const ProbeKey &pk = ProbeKey{},
                       const RoundKeys &rk = RoundKeys{}) {
  using S = GemmSmem<BN, STAGES>;
  auto kern = gemm_bf16_kernel<BN, STAGES, EPI, PERT>;
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), (int)S::kBytes);
    if (e != cudaSuccess) return e;
  }
  constexpr int OUT_BN = EPI == ZO_EPI_SWIGLU_BF16 ? BN / 2 : BN;
  const int num_m = (g.M + kBM - 1) / kBM, num_n = (g.N + OUT_BN - 1) / OUT_BN;
  const int tiles = num_m * num_n;
  kern<<<tiles < kSmCount ? tiles : kSmCount, PERT ? kGemmThreadsX : kGemmThreads, S::kBytes, st>>>(
      ta, tb, tcm, g, pk, rk);
  return cudaGetLastError();
}

template <int STAGES, int EPI>
cudaError_t launch_pair(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tcm,
                        const GemmArgs &g, cudaStream_t st) {
  using S = PairSmem<STAGES>;
  auto kern = gemm_pair_kernel<STAGES, EPI>;
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(kern), (int)S::kBytes);
    if (e != cudaSuccess) return e;
  }
  constexpr int OUT_BN = EPI == ZO_EPI_SWIGLU_BF16 ? kPairBN / 2 : kPairBN;
  const int tiles = ((g.M + 2 * kBM - 1) / (2 * kBM)) * ((g.N + OUT_BN - 1) / OUT_BN);
  const int clusters = tiles < kSmCount / 2 ? tiles : kSmCount / 2;
  kern<<<2 * clusters, kGemmThreads, S::kBytes, st>>>(ta, tb, tcm, g);
  return cudaGetLastError();
}

}  // namespace

zo_status launch_gemm_pair(zo_ctx *ctx, const void *A, const void *B, const void *bias, void *out,
                           int M, int N, int K, int ldo, int epi, int64_t lda) {
  const int NB = epi == ZO_EPI_SWIGLU_BF16 ? 2 * N : N;
  CUtensorMap ta, tb, tcm;
  if (!make_map(&ta, A, M, K, kBM, lda) || !make_map(&tb, B, NB, K, kPairBN / 2) ||
      !make_out_map(&tcm, out, M, N, ldo, epi == ZO_EPI_RESID_F32))
    return fail(ctx, ZO_ERR_CUDA, "gemm: cuTensorMapEncodeTiled failed");
  GemmArgs g{M, N, K, group_rows_for(K, 2 * kBM), static_cast<const uint16_t *>(bias), out, ldo,
             &ctx->dstate->flags, 0u};
  const int slot = ktime_begin(ctx);
  cudaError_t e;
  if (epi == ZO_EPI_BIAS_BF16) e = launch_pair<6, ZO_EPI_BIAS_BF16>(ta, tb, tcm, g, ctx->stream);
  else if (epi == ZO_EPI_RELU_BF16) e = launch_pair<6, ZO_EPI_RELU_BF16>(ta, tb, tcm, g, ctx->stream);
  else if (epi == ZO_EPI_RESID_F32) e = launch_pair<6, ZO_EPI_RESID_F32>(ta, tb, tcm, g, ctx->stream);
  else e = launch_pair<6, ZO_EPI_SWIGLU_BF16>(ta, tb, tcm, g, ctx->stream);
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "gemm (CTA pairs) launch: %s", cudaGetErrorString(e));
  ctx->launches += 1;
  ktime_end(ctx, slot, ZO_KT_GEMM, 2.0 * M * (double)NB * K);
  return ZO_OK;
}

// lda: elements between the starts of A's rows (0: K; a multiple of 8, at least K).  A padded
// row stride keeps the 128-byte pieces of A that a stage reads from colliding in L2 sets: at
// the OPT-30B FC2 shape (K = 28672) a stride of K + 64 measured 16 GB of DRAM reads per launch
// instead of 24 GB.
zo_status launch_gemm(zo_ctx *ctx, const void *A, const void *B, const void *bias, void *out,
                      int M, int N, int K, int ldo, int epi, uint32_t extra_tx, int64_t lda) {
  if (M < 1 || N < 1 || K < 1 || (K % 8) != 0 || (ldo % 8) != 0 || ldo < N)
    return fail(ctx, ZO_ERR_INVALID, "gemm: need M,N,K >= 1, K %% 8 == 0, ldo %% 8 == 0, ldo >= N");
  if (lda != 0 && (lda < K || lda % 8 != 0))
    return fail(ctx, ZO_ERR_INVALID, "gemm: lda must be a multiple of 8, at least K");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
       reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(bias)) & 15u)
    return fail(ctx, ZO_ERR_INVALID, "gemm: operands must be 16-byte aligned");
  if (epi < ZO_EPI_BIAS_BF16 || epi > ZO_EPI_SWIGLU_BF16) return fail(ctx, ZO_ERR_INVALID, "gemm: bad epilogue");
  const bool swiglu = epi == ZO_EPI_SWIGLU_BF16;
  if (swiglu && bias) return fail(ctx, ZO_ERR_INVALID, "gemm: the SwiGLU epilogue takes no bias");
  const int NB = swiglu ? 2 * N : N;  // rows of B, = accumulator columns over all tiles
  // CTA pairs for shapes that give every cluster at least two 256 x 256 tiles
  const int64_t pair_tiles = (int64_t)((M + 255) / 256) * ((NB + 255) / 256);
  if (extra_tx == 0 && M >= 256 && NB >= 256 && pair_tiles >= (int64_t)kSmCount)
    return launch_gemm_pair(ctx, A, B, bias, out, M, N, K, ldo, epi, lda);
  // N <= 128 tiles use BN = 128 to fill the machine on narrow outputs.
  const bool wide = NB > 128 && ((int64_t)((M + 127) / 128) * ((NB + 255) / 256) >= kSmCount);
  const int box_b = (wide ? 256 : 128) / (swiglu ? 2 : 1);
  CUtensorMap ta, tb, tcm;
  if (!make_map(&ta, A, M, K, kBM, lda) || !make_map(&tb, B, NB, K, box_b) ||
      !make_out_map(&tcm, out, M, N, ldo, epi == ZO_EPI_RESID_F32))
    return fail(ctx, ZO_ERR_CUDA, "gemm: cuTensorMapEncodeTiled failed");
  GemmArgs g{M, N, K, group_rows_for(K, kBM), static_cast<const uint16_t *>(bias), out, ldo,
             &ctx->dstate->flags, extra_tx};
  const int slot = ktime_begin(ctx);
  cudaError_t e;
  if (wide) {
    if (epi == ZO_EPI_BIAS_BF16) e = launch_one<256, 4, ZO_EPI_BIAS_BF16>(ta, tb, tcm, g, ctx->stream);
    else if (epi == ZO_EPI_RELU_BF16) e = launch_one<256, 4, ZO_EPI_RELU_BF16>(ta, tb, tcm, g, ctx->stream);
    else if (epi == ZO_EPI_RESID_F32) e = launch_one<256, 4, ZO_EPI_RESID_F32>(ta, tb, tcm, g, ctx->stream);
    else e = launch_one<256, 4, ZO_EPI_SWIGLU_BF16>(ta, tb, tcm, g, ctx->stream);
  } else {
    if (epi == ZO_EPI_BIAS_BF16) e = launch_one<128, 6, ZO_EPI_BIAS_BF16>(ta, tb, tcm, g, ctx->stream);
    else if (epi == ZO_EPI_RELU_BF16) e = launch_one<128, 6, ZO_EPI_RELU_BF16>(ta, tb, tcm, g, ctx->stream);
    else if (epi == ZO_EPI_RESID_F32) e = launch_one<128, 6, ZO_EPI_RESID_F32>(ta, tb, tcm, g, ctx->stream);
    else e = launch_one<128, 6, ZO_EPI_SWIGLU_BF16>(ta, tb, tcm, g, ctx->stream);
  }
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  ctx->launches += 1;
  ktime_end(ctx, slot, ZO_KT_GEMM, 2.0 * M * (double)NB * K);  // NB accumulator columns
  return ZO_OK;
}

// The GEMM with B = the context's bf16 parameters [w_off, w_off + N K) read under the
// context's current perturbation (fused into the operand path, single-CTA form).
zo_status launch_gemm_perturbed(zo_ctx *ctx, const void *A, int64_t w_off, const void *bias,
                                void *out, int M, int N, int K, int ldo, int epi) {
  if (ctx->dtype != ZO_BF16) return fail(ctx, ZO_ERR_INVALID, "perturbed gemm: needs a bf16 context");
  if (M < 1 || N < 1 || K < 16 || (K % 16) != 0 || (ldo % 8) != 0 || ldo < N)
    return fail(ctx, ZO_ERR_INVALID, "perturbed gemm: need M,N >= 1, K %% 16 == 0, ldo %% 8 == 0, ldo >= N");
  if (w_off < 0 || w_off % 16 != 0 || ctx->first_element % 16 != 0 || w_off + (int64_t)N * K > ctx->M)
    return fail(ctx, ZO_ERR_INVALID, "perturbed gemm: weights must lie in the context, 16-element aligned");
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(out) |
       reinterpret_cast<uintptr_t>(bias)) & 15u)
    return fail(ctx, ZO_ERR_INVALID, "perturbed gemm: operands must be 16-byte aligned");
  if (epi != ZO_EPI_BIAS_BF16 && epi != ZO_EPI_RELU_BF16 && epi != ZO_EPI_RESID_F32)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "perturbed gemm: bias, ReLU or residual epilogue only");
  const uint16_t *B = static_cast<const uint16_t *>(ctx->params) + w_off;
  const bool wide = N > 128 && ((int64_t)((M + 127) / 128) * ((N + 255) / 256) >= kSmCount);
  CUtensorMap ta, tb, tcm;
  if (!make_map(&ta, A, M, K, kBM) || !make_map(&tb, B, N, K, wide ? 256 : 128) ||
      !make_out_map(&tcm, out, M, N, ldo, epi == ZO_EPI_RESID_F32))
    return fail(ctx, ZO_ERR_CUDA, "perturbed gemm: cuTensorMapEncodeTiled failed");
  GemmArgs g{M, N, K, group_rows_for(K, kBM), static_cast<const uint16_t *>(bias), out, ldo,
             &ctx->dstate->flags, 0u, w_off};
  const ProbeKey pk = probe_key(ctx);
  const RoundKeys rk = round_keys(pk.k0, pk.k1);
  const int slot = ktime_begin(ctx);
  cudaError_t e;
  if (wide) {
    if (epi == ZO_EPI_BIAS_BF16) e = launch_one<256, 4, ZO_EPI_BIAS_BF16, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
    else if (epi == ZO_EPI_RELU_BF16) e = launch_one<256, 4, ZO_EPI_RELU_BF16, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
    else e = launch_one<256, 4, ZO_EPI_RESID_F32, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
  } else {
    if (epi == ZO_EPI_BIAS_BF16) e = launch_one<128, 6, ZO_EPI_BIAS_BF16, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
    else if (epi == ZO_EPI_RELU_BF16) e = launch_one<128, 6, ZO_EPI_RELU_BF16, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
    else e = launch_one<128, 6, ZO_EPI_RESID_F32, true>(ta, tb, tcm, g, ctx->stream, pk, rk);
  }
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "perturbed gemm launch: %s", cudaGetErrorString(e));
  ctx->launches += 1;
  ktime_end(ctx, slot, ZO_KT_GEMM, 2.0 * M * (double)N * K);
  return ZO_OK;
}

}  // namespace zo
