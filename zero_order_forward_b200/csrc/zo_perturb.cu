// zo_perturb.cu -- the fused unpack/apply kernel (perturbed copy of a parameter window)
// and the packed-probe writer.
//
// "Probe-Space Preconditioning for Fast and Stable Zero-Order Training", abstract:
// probes come from a packed random generator (8 signs per byte) and are applied to the
// weights by fused unpack/apply kernels.  Here the sign bits are regenerated in
// registers (never stored): the lanes of a warp compute the Philox blocks of the
// 16-element groups the warp streams, extract the probe's bit from each element byte, and
// share the 16-bit masks (through shared memory or warp shuffles) while every lane streams
// 16-byte vectors of theta -> rd(theta + s*eps*z).
#include <cstdio>

#include "zo_internal.cuh"
#include "zo_tc.cuh"

namespace zo {
namespace {

constexpr int kWarps = 8;  // warps per block

template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<uint16_t> { static constexpr int N = 8; };

// Apply the perturbation to one 16-byte vector of N elements whose sign bits are the
// low N bits of `bits`.
__device__ __forceinline__ uint4 apply_vec(uint4 v, uint32_t bits, float delta, float *) {
  const uint32_t db = __float_as_uint(delta);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
    f[t] = __fadd_rn(__uint_as_float(w[t]), __uint_as_float(db ^ ((bits << (31 - t)) & 0x80000000u)));
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 apply_vec(uint4 v, uint32_t bits, float delta, uint16_t *) {
  // element 2t takes sign bit 2t, element 2t+1 bit 2t+1: each shifted into bit 31 and xor-ed
  // into eps (the same sum as perturb_f32)
  const uint32_t db = __float_as_uint(delta);
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

__device__ __forceinline__ float apply_one(float v, uint32_t bit, float delta) {
  return perturb_f32(v, delta, bit);
}
__device__ __forceinline__ uint16_t apply_one(uint16_t v, uint32_t bit, float delta) {
  return f32_to_bf16_bits(perturb_f32(bf16_bits_to_f32(v), delta, bit));
}

// out[e - first] = P_e for e in [first, first + count).  Tiles of 256 groups (4096
// elements) are aligned to groups in the global element index; a warp owns a tile, its
// lane l computes the bits of groups l, l + 32, ..., l + 224 into the warp's 512-byte
// mask (element e of the tile at bit e), and then streams the tile.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
perturb_kernel(const T *__restrict__ theta, T *__restrict__ out, int64_t first, int64_t count,
               ProbeKey pk, int64_t n_tiles) {
  constexpr int N = Vec<T>::N;
  constexpr int kIters = kTileElems / (32 * N);
  __shared__ uint16_t masks[kWarps][kTileGroups];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t end = first + count;
  const int64_t g0 = first / kGroup;
  const uint32_t step = pk.sign ? *pk.step : 0u;
  const float delta = pk.sign > 0 ? pk.eps : -pk.eps;
  const uint32_t *bw = reinterpret_cast<const uint32_t *>(masks[warp]);

  for (int64_t tile = (int64_t)blockIdx.x * kWarps + warp; tile < n_tiles;
       tile += (int64_t)gridDim.x * kWarps) {
    const int64_t base = (g0 + tile * kTileGroups) * kGroup;  // first element of the tile
    if (pk.sign) {
#pragma unroll
      for (int i = 0; i < kTileGroups / 32; ++i) {
        const int64_t g = g0 + tile * kTileGroups + lane + 32 * i;
        masks[warp][lane + 32 * i] =
            g * kGroup < end ? (uint16_t)probe_group_bits(g + pk.g_off, pk.probe, step, pk.k0, pk.k1) : 0;
      }
      __syncwarp();
    }
#pragma unroll 4
    for (int k = 0; k < kIters; ++k) {
      const int e_rel = (k * 32 + lane) * N;
      const int64_t e = base + e_rel;
      uint32_t bits = 0;
      if (pk.sign) bits = bw[e_rel >> 5] >> (e_rel & 31);
      T *o = out + (e - first);
      if (e >= first && e + N <= end && ((reinterpret_cast<uintptr_t>(o) & 15) == 0)) {
        uint4 v = __ldg(reinterpret_cast<const uint4 *>(theta + e));
        if (pk.sign) v = apply_vec(v, bits, delta, (T *)nullptr);
        *reinterpret_cast<uint4 *>(o) = v;
      } else {
#pragma unroll
        for (int t = 0; t < N; ++t) {
          const int64_t et = e + t;
          if (et >= first && et < end) {
            T v = theta[et];
            if (pk.sign) v = apply_one(v, (bits >> t) & 1u, delta);
            out[et - first] = v;
          }
        }
      }
    }
    if (pk.sign) __syncwarp();
  }
}

// Pipelined form for 16-byte-aligned windows (first % (16 / sizeof(T)) == 0, out 16-byte
// aligned): chunks of 256 groups (4096 elements, aligned to groups in the global index)
// stream through a ring of shared-memory stages.  Warp 0 issues the bulk copy of a chunk
// into a stage; 8 consumer warps each regenerate the bits of the 32 groups of their slice
// (one Philox block per lane, shared by warp shuffles), copy the slice into registers and
// release the stage, then apply the perturbation and write the window with coalesced 16-byte
// stores.  Several CTAs per SM keep enough loads and stores in flight.
constexpr int kPChunk = kTileElems;  // 4096
constexpr int kPStages = 6;
constexpr int kPConsumers = 8;
constexpr int kPThreads = 32 * (1 + kPConsumers);

template <typename T>
struct PipeSmem {
  static constexpr int kData = kPChunk * (int)sizeof(T);
  static constexpr int kStage = kData;
  static constexpr int kBytes = kPStages * kStage + 2 * kPStages * 8;
};

template <typename T>
__global__ void __launch_bounds__(kPThreads)
perturb_pipe_kernel(const T *__restrict__ theta, T *__restrict__ out, int64_t first,
                    int64_t count, ProbeKey pk, const __grid_constant__ RoundKeys rk,
                    int64_t n_chunks, uint32_t *err) {
  using SM = PipeSmem<T>;
  constexpr int N = Vec<T>::N;
  extern __shared__ __align__(128) uint8_t psm[];
  uint64_t *full = reinterpret_cast<uint64_t *>(psm + kPStages * SM::kStage);
  uint64_t *empty = full + kPStages;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kPConsumers);
    }
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  const int64_t end = first + count;
  const int64_t g0 = first / kGroup;
  const uint32_t step = pk.sign ? *pk.step : 0u;
  const float delta = pk.sign > 0 ? pk.eps : -pk.eps;

  if (warp == 0) {
    int it = 0, issued = 0;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
      const int s = it % kPStages;
      const uint32_t ph = (uint32_t)(it / kPStages) & 1u;
      int ok = 1;
      if (lane == 0) ok = tc::mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok || abort_flag) {
        if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
        break;
      }
      uint8_t *st = psm + s * SM::kStage;
      const int64_t cs = (g0 + c * kTileGroups) * kGroup;
      const int64_t vs = cs > first ? cs : first;
      const int64_t ve = cs + kPChunk < end ? cs + kPChunk : end;
      const int64_t copy = (ve - vs) & ~(int64_t)(N - 1);
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&full[s], (uint32_t)(copy * (int64_t)sizeof(T)));
        if (copy > 0)
          tc::bulk_load(st + (vs - cs) * (int64_t)sizeof(T), theta + vs,
                        (uint32_t)(copy * (int64_t)sizeof(T)), &full[s]);
      }
      __syncwarp();
      issued = it + 1;
    }
    if (abort_flag && lane == 0) {
      for (int s = 0; s < kPStages; ++s) {
        int last = -1;
        for (int i = s; i < issued; i += kPStages) last = i;
        if (last >= 0) tc::mbar_wait(&full[s], (uint32_t)(last / kPStages) & 1u);
      }
    }
  } else {
    // Consumer warp cw owns the contiguous slice [cw * kSlice, (cw + 1) * kSlice) of each
    // chunk (32 sign groups, one Philox block per lane, computed before the data arrives):
    // its vectors are copied from the stage into registers, the stage is released at once,
    // and the perturbed vectors are written with coalesced 16-byte stores.
    constexpr int kSlice = kPChunk / kPConsumers;  // 512 elements = 32 groups
    constexpr int kVecs = kSlice / (N * 32);       // vectors per lane
    const int cw = warp - 1;
    int it = 0;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
      const int s = it % kPStages;
      const uint32_t ph = (uint32_t)(it / kPStages) & 1u;
      const int64_t cs = (g0 + c * kTileGroups) * kGroup;
      const int64_t ws = cs + (int64_t)cw * kSlice;  // this warp's slice
      uint32_t mine = 0u;
      if (pk.sign)
        mine = probe_group_bits(pk.g_off + (uint64_t)(ws / kGroup) + lane, pk.probe, step, rk);
      int ok = 1;  // decided per warp, as in the loss pipeline
      if (lane == 0) ok = (!abort_flag && tc::mbar_wait(&full[s], ph)) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (ok && lane != 0) ok = tc::mbar_wait(&full[s], ph) ? 1 : 0;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) { atomicOr(err, ZO_FLAG_TIMEOUT); abort_flag = 1; }
        break;
      }
      const uint8_t *st = psm + s * SM::kStage;
      if (cs >= first && cs + kPChunk <= end) {
        // the whole chunk lies in the window (every chunk but the window's edges): 32-bit
        // offsets, no per-vector bounds
        const uint4 *src = reinterpret_cast<const uint4 *>(st + (int64_t)cw * kSlice * (int64_t)sizeof(T));
        uint4 v[kVecs];
#pragma unroll
        for (int k = 0; k < kVecs; ++k) v[k] = src[lane + 32 * k];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[s]);  // the stage is free again
        uint4 *dst = reinterpret_cast<uint4 *>(out + (ws - first));
#pragma unroll
        for (int k = 0; k < kVecs; ++k) {
          const int vi = lane + 32 * k;
          uint4 x = v[k];
          if (pk.sign) {
            const uint32_t bits = __shfl_sync(0xFFFFFFFFu, mine, (vi * N) >> 4) >> ((vi * N) & 15);
            x = apply_vec(x, bits, delta, (T *)nullptr);
          }
          dst[vi] = x;
        }
        continue;
      }
      const int64_t vs = cs > first ? cs : first;
      const int64_t ve = cs + kPChunk < end ? cs + kPChunk : end;
      const int64_t copy_end = vs + ((ve - vs) & ~(int64_t)(N - 1));
      uint4 v[kVecs];
#pragma unroll
      for (int k = 0; k < kVecs; ++k) {
        const int64_t e = ws + (int64_t)(lane + 32 * k) * N;
        if (e >= vs && e + N <= copy_end)
          v[k] = *reinterpret_cast<const uint4 *>(st + (e - cs) * (int64_t)sizeof(T));
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[s]);  // the stage is free again
#pragma unroll
      for (int k = 0; k < kVecs; ++k) {
        const int vi = lane + 32 * k;  // vector of the slice
        const int64_t e = ws + (int64_t)vi * N;
        const uint32_t bits =
            pk.sign ? __shfl_sync(0xFFFFFFFFu, mine, (vi * N) >> 4) >> ((vi * N) & 15) : 0u;
        if (e + N <= vs || e >= ve) continue;
        if (e >= vs && e + N <= copy_end) {
          uint4 x = v[k];
          if (pk.sign) x = apply_vec(x, bits, delta, (T *)nullptr);
          *reinterpret_cast<uint4 *>(out + (e - first)) = x;
        } else {  // the window's last < N elements: plain loads and stores
#pragma unroll
          for (int t = 0; t < N; ++t) {
            const int64_t et = e + t;
            if (et >= first && et < end) {
              T x = theta[et];
              if (pk.sign) x = apply_one(x, (bits >> t) & 1u, delta);
              out[et - first] = x;
            }
          }
        }
      }
    }
  }
}

// Packed bytes of one probe [first_byte, first_byte + nbytes) (byte q: elements 8q..8q+7,
// bit t <-> element 8q+t): one thread per 16-element group, i.e. per 2 output bytes.
// Bits of elements >= M are cleared.
__global__ void pack_kernel(uint8_t *__restrict__ out, int64_t first_byte, int64_t nbytes,
                            int64_t M, uint32_t probe, uint32_t step, uint32_t k0, uint32_t k1,
                            uint64_t g_off) {
  const int64_t gfirst = first_byte / 2;
  const int64_t glast = (first_byte + nbytes - 1) / 2;
  const int64_t g = gfirst + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g > glast) return;
  const uint32_t m = probe_group_bits((uint64_t)g + g_off, probe, step, k0, k1);
  for (int q = 0; q < 2; ++q) {
    const int64_t byte = g * 2 + q;
    if (byte < first_byte || byte >= first_byte + nbytes) continue;
    uint32_t v = (m >> (8 * q)) & 0xFFu;
    const int64_t e0 = byte * 8;
    if (e0 + 8 > M) v &= (M > e0) ? ((1u << (M - e0)) - 1u) : 0u;
    out[byte - first_byte] = (uint8_t)v;
  }
}

}  // namespace

template <typename T>
zo_status launch_pipe(zo_ctx *ctx, const ProbeKey &pk, int64_t first, int64_t count, void *out) {
  using SM = PipeSmem<T>;
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(perturb_pipe_kernel<T>), SM::kBytes);
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "perturb_pipe_kernel attribute: %s", cudaGetErrorString(e));
  }
  const int64_t g0 = first / kGroup;
  const int64_t g1 = (first + count + kGroup - 1) / kGroup;
  const int64_t n_chunks = (g1 - g0 + kTileGroups - 1) / kTileGroups;
  int per_sm = 2;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, perturb_pipe_kernel<T>, kPThreads,
                                                    SM::kBytes) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const int64_t cap = (int64_t)kSmCount * per_sm;
  const int64_t blocks = n_chunks < cap ? n_chunks : cap;
  perturb_pipe_kernel<T><<<(unsigned)blocks, kPThreads, SM::kBytes, ctx->stream>>>(
      static_cast<const T *>(ctx->params), static_cast<T *>(out), first, count, pk,
      round_keys(pk.k0, pk.k1), n_chunks, &ctx->dstate->flags);
  return check_launch(ctx, "perturb_pipe_kernel");
}

zo_status launch_perturb_impl(zo_ctx *ctx, const ProbeKey &pk, int64_t first, int64_t count,
                              void *out);

// Timed as ZO_KT_PERTURB with its algorithmic bytes: theta read and the window written once.
zo_status launch_perturb(zo_ctx *ctx, const ProbeKey &pk, int64_t first, int64_t count,
                         void *out) {
  if (count <= 0) return ZO_OK;
  const int slot = ktime_begin(ctx);
  const zo_status st = launch_perturb_impl(ctx, pk, first, count, out);
  if (st == ZO_OK) ktime_end(ctx, slot, ZO_KT_PERTURB, 2.0 * (ctx->dtype == ZO_F32 ? 4 : 2) * (double)count);
  return st;
}

zo_status launch_perturb_impl(zo_ctx *ctx, const ProbeKey &pk, int64_t first, int64_t count,
                              void *out) {
  const int vec = ctx->dtype == ZO_F32 ? 4 : 8;
  if (count >= kPChunk && first % vec == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0)
    return ctx->dtype == ZO_F32 ? launch_pipe<float>(ctx, pk, first, count, out)
                                : launch_pipe<uint16_t>(ctx, pk, first, count, out);
  const int64_t g0 = first / kGroup;
  const int64_t g1 = (first + count + kGroup - 1) / kGroup;
  const int64_t n_tiles = (g1 - g0 + kTileGroups - 1) / kTileGroups;
  int64_t blocks = (n_tiles + kWarps - 1) / kWarps;
  if (blocks > (int64_t)kSmCount * 8) blocks = (int64_t)kSmCount * 8;
  if (ctx->dtype == ZO_F32)
    perturb_kernel<float><<<(unsigned)blocks, kWarps * 32, 0, ctx->stream>>>(
        static_cast<const float *>(ctx->params), static_cast<float *>(out), first, count, pk,
        n_tiles);
  else
    perturb_kernel<uint16_t><<<(unsigned)blocks, kWarps * 32, 0, ctx->stream>>>(
        static_cast<const uint16_t *>(ctx->params), static_cast<uint16_t *>(out), first,
        count, pk, n_tiles);
  return check_launch(ctx, "perturb_kernel");
}

zo_status launch_pack(zo_ctx *ctx, uint32_t step, uint32_t probe, int64_t first_byte,
                      int64_t nbytes, uint8_t *out) {
  if (nbytes <= 0) return ZO_OK;
  const int64_t groups = (first_byte + nbytes - 1) / 2 - first_byte / 2 + 1;
  const int threads = 256;
  const int64_t blocks = (groups + threads - 1) / threads;
  ProbeKey pk = probe_key(ctx);
  pack_kernel<<<(unsigned)blocks, threads, 0, ctx->stream>>>(
      out, first_byte, nbytes, ctx->M, probe, step, pk.k0, pk.k1, pk.g_off);
  return check_launch(ctx, "pack_kernel");
}

}  // namespace zo
