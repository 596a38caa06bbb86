// zo_attn_tc.cu -- causal multi-head / grouped-query attention on the 5th-generation tensor
// cores (inference forward only):
//
//   out[b, s, h, :] = sum_{s' <= s} softmax_s'( q[b,s,h,:] . k[b,s',g,:] / sqrt(hd) ) v[b,s',g,:]
//
// with g = h / (H / Hk).  Layout as zo_attn.cu: qkv is the fused projection output
// [B*S][(H + 2 Hk) hd] (query heads, key heads, value heads), out is [B*S][H hd].
//
// One CTA (6 warps) per (128-query tile, head, sequence), heavy (late) tiles first, two
// CTAs per SM so that one CTA's softmax overlaps the other's MMAs and loads:
//   warp 0     one lane issues TMA loads: the Q tile once (boxes of 64 columns x 128 rows),
//              then K and V tiles of 64 keys (boxes of 64 columns x 64 rows) into a 2-stage
//              ring (two tensor maps over the qkv buffer, 128-byte swizzle);
//   warp 1     allocates 256 TMEM columns (S: 64, P: 32, O: hd) and one lane issues
//              S = Q K^T (tcgen05.mma M=128, N=64, both operands K-major from shared
//              memory), the next tile's S as soon as the softmax has read this one, and,
//              once the softmax has written P, O += P V (P from tensor memory, V MN-major
//              from shared memory as loaded), committing to mbarriers;
//   warps 2-5  the softmax, one query row per thread (TMEM lane quadrant = warp % 4): read the
//              row of S from TMEM, scale, mask (diagonal and sequence-end tiles only), online
//              maximum with lazy rescaling (O and the row sum are rescaled only when the
//              maximum grows by more than 2^8, so exponentials stay below 256), P = 2^(s - m)
//              rounded to bf16 and stored to TMEM, row sum in fp32; at the end O / l is read
//              from TMEM, rounded to bf16 and stored.
// All waits are bounded (zo_tc.cuh); on expiry the kernel raises ZO_FLAG_TIMEOUT, lets its
// loads and MMAs drain and frees TMEM.
#include <cudaTypedefs.h>

#include <mutex>

#include "zo_internal.cuh"
#include "zo_tc.cuh"

namespace zo {
namespace {

constexpr int kTBM = 128, kTThreads = 192;
constexpr uint32_t kQBox = 128 * 128;  // bytes of one 128-row x 64-column bf16 box

// Key tiles of BN keys (hd 128: 64; hd 64: 128, so that a tile's MMAs amortise the
// softmax round trip), two K/V stages, 256 TMEM columns (S: BN, P: BN/2, O: hd) and 96 KB
// (hd 128) or 80 KB (hd 64) of shared memory per CTA: two CTAs per SM.
template <int HD> struct TcAttnCfg {
  static constexpr int kBN = HD == 128 ? 64 : 128;
  static constexpr int kStages = 2, kCtas = 2, kTmemCols = 256;
};

template <int HD>
struct TcAttnSmem {
  static constexpr int kStages = TcAttnCfg<HD>::kStages;
  static constexpr uint32_t kKBox = TcAttnCfg<HD>::kBN * 128;  // BN rows x 64 columns
  static constexpr uint32_t kQTile = (HD / 64) * kQBox;   // 128 rows x HD columns
  static constexpr uint32_t kKTile = (HD / 64) * kKBox;   // BN rows x HD columns
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQTile;                // [kStages]
  static constexpr uint32_t kV = kK + kStages * kKTile;      // [kStages]
  static constexpr uint32_t kBar = kV + kStages * kKTile;
  static constexpr uint32_t kBytes = kBar + 128 + 1024;      // barriers + alignment slack
};

struct TcAttnArgs {
  int S, H, Hk;
  int q0, k0, v0;  // column offsets of the query, key and value heads in a qkv row
  int ld_out;
  float scale_log2;
  uint16_t *out;
  uint32_t *err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  return pack_bf16x2(lo, hi);
}

// All lanes of the warp wait for `parity` on `bar`: lane 0 decides (bounded), then every lane
// observes the completed phase.  Returns false (on every lane) on expiry or abort.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) ok = (!*abort_flag && tc::mbar_wait(bar, parity)) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok && lane != 0) ok = tc::mbar_wait(bar, parity) ? 1 : 0;
  return __all_sync(0xFFFFFFFFu, ok) != 0;
}

template <int HD>
__global__ void __launch_bounds__(kTThreads, TcAttnCfg<HD>::kCtas)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmkv,
               TcAttnArgs a) {
  using SM = TcAttnSmem<HD>;
  constexpr int kTStages = SM::kStages;
  constexpr int kTBN = TcAttnCfg<HD>::kBN;
  constexpr uint32_t kKBox = SM::kKBox;
  constexpr uint32_t kCols = TcAttnCfg<HD>::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM::kBar);
  uint64_t *q_full = bars, *kv_full = bars + 1, *kv_empty = bars + 3, *s_full = bars + 5,
           *s_free = bars + 6, *p_full = bars + 7, *pv_done = bars + 8, *mma_done = bars + 9;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + 10);  // 10 barriers + 2 words < 128 B
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // heavy (late) query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (a.H / a.Hk);
  const int row0 = b * a.S;  // first token row of the sequence
  const int q_first = qt * kTBM;
  const int last_q = min(q_first + kTBM, a.S) - 1;
  const int n_kt = last_q / kTBN + 1;

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kTStages; ++s) {
      tc::mbar_init(&kv_full[s], 1);
      tc::mbar_init(&kv_empty[s], 1);
    }
    tc::mbar_init(s_full, 1);
    tc::mbar_init(s_free, 4);  // one arrival per softmax warp
    tc::mbar_init(p_full, 4);
    tc::mbar_init(pv_done, 1);
    tc::mbar_init(mma_done, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, kCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // S: BN columns, P: BN/2 (bf16 pairs), O: hd (hd 128: 0/64/128; hd 64: 0/128/192)
  const uint32_t tS = tmem, tP = tmem + kTBN, tO = tmem + kTBN + kTBN / 2 + (HD == 128 ? 32 : 0);

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      tc::tma_prefetch_desc(&tmq);
      tc::tma_prefetch_desc(&tmkv);
      tc::mbar_arrive_expect_tx(q_full, SM::kQTile);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c)
        tc::tma_load_2d(sm + SM::kQ + c * kQBox, &tmq, q_full, a.q0 + h * HD + 64 * c, row0 + q_first);
      int issued = 0;
      for (int j = 0; j < n_kt; ++j) {
        const int s = j % kTStages;
        const uint32_t ph = (uint32_t)(j / kTStages) & 1u;
        if (*abort_flag || !tc::mbar_wait(&kv_empty[s], ph ^ 1u)) {
          atomicOr(a.err, ZO_FLAG_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&kv_full[s], 2 * SM::kKTile);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c) {
          tc::tma_load_2d(sm + SM::kK + s * SM::kKTile + c * kKBox, &tmkv, &kv_full[s],
                          a.k0 + kvh * HD + 64 * c, row0 + j * kTBN);
          tc::tma_load_2d(sm + SM::kV + s * SM::kKTile + c * kKBox, &tmkv, &kv_full[s],
                          a.v0 + kvh * HD + 64 * c, row0 + j * kTBN);
        }
        issued = j + 1;
      }
      if (*abort_flag) {  // let this CTA's loads land before it exits (bounded)
        tc::mbar_wait(q_full, 0);
        for (int s = 0; s < kTStages; ++s) {
          int last = -1;
          for (int i = s; i < issued; i += kTStages) last = i;
          if (last >= 0) tc::mbar_wait(&kv_full[s], (uint32_t)(last / kTStages) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t idS = tc::idesc_bf16_f32(kTBM, kTBN);
      constexpr uint32_t idO = tc::idesc_bf16_f32(kTBM, HD) | (1u << 16);  // B (V) MN-major
      const uint32_t qa = tc::smem_addr(sm + SM::kQ);
      // S_j = Q K_j^T into TMEM once K_j has landed and the softmax has read S_{j-1}
      auto issue_s = [&](int j) -> bool {
        const int s = j % kTStages;
        if (*abort_flag || !tc::mbar_wait(&kv_full[s], (uint32_t)(j / kTStages) & 1u) ||
            (j > 0 && !tc::mbar_wait(s_free, (uint32_t)(j - 1) & 1u)))
          return false;
        tc::tc_fence_after();
        const uint32_t ka = tc::smem_addr(sm + SM::kK + s * SM::kKTile);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t kk = (uint32_t)(k & 3) * 32u;
          tc::mma_bf16(tS, tc::smem_desc_k128(qa + (uint32_t)(k >> 2) * kQBox + kk),
                       tc::smem_desc_k128(ka + (uint32_t)(k >> 2) * kKBox + kk), idS, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(s_full);
        return true;
      };
      bool ok = tc::mbar_wait(q_full, 0) && issue_s(0);
      for (int j = 0; ok && j < n_kt; ++j) {
        const int s = j % kTStages;
        // with two stages the next tile's scores overlap this tile's softmax; with one, the
        // next K arrives only after this tile's P V has released the stage
        if (kTStages > 1 && j + 1 < n_kt && !(ok = issue_s(j + 1))) break;
        ok = tc::mbar_wait(p_full, (uint32_t)j & 1u);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t va = tc::smem_addr(sm + SM::kV + s * SM::kKTile);
#pragma unroll
        for (int k = 0; k < kTBN / 16; ++k) {
          const uint32_t boff = (uint32_t)k * 16u * 128u;  // 16 keys of 128-byte V rows
          tc::mma_bf16_tmem_a(tO, tP + 8u * k, tc::smem_desc_mn128(va + boff, kKBox), idO,
                              (j > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(pv_done);
        tc::mma_commit(&kv_empty[s]);
        if (kTStages == 1 && j + 1 < n_kt && !(ok = issue_s(j + 1))) break;
      }
      if (!ok) {
        atomicOr(a.err, ZO_FLAG_TIMEOUT);
        *abort_flag = 1;
      }
      tc::mma_commit(mma_done);  // arrives once every MMA issued above has retired
    }
  } else {  // softmax warps: TMEM lane quadrant qd holds the tile's query rows 32 qd .. +31
    const int qd = warp & 3;
    const int tr = 32 * qd + lane;  // row within the tile
    const int r = q_first + tr;     // query position in the sequence
    const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      if (!warp_wait(s_full, (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
      tc::tc_fence_after();
      float s[kTBN];
#pragma unroll
      for (int c = 0; c < kTBN / 32; ++c) tc::tmem_ld32(tS + lane_off + 32u * c, s + 32 * c);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_free);  // S may be overwritten by the next tile
      const int key0 = j * kTBN;
      const bool edge = key0 + kTBN - 1 > q_first || key0 + kTBN > a.S;
      // the maximum of the raw scores (the scale is positive), then 2^(s * scale - m) with the
      // scaling folded into the exponent's fused multiply-add
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // 4 independent chains
#pragma unroll
      for (int c = 0; c < kTBN; ++c) {
        if (edge && (key0 + c > r || key0 + c >= a.S)) s[c] = -INFINITY;
        mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;
      const float m_new = fmaxf(m_used, mx);
      // Lazy rescaling: keep the running maximum unless it grows by more than 2^8 (then
      // O and l are rescaled below, once the previous tile's P V has completed).
      const bool need = j > 0 && m_new > m_used + 8.f;
      const float m_old = m_used;
      if (j == 0 || need) m_used = m_new;
      const float msc = m_used == -INFINITY ? 0.f : m_used;
      uint32_t pk[kTBN / 2];
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kTBN; c += 2) {
        const float p0 = ex2(fmaf(s[c], a.scale_log2, -msc)), p1 = ex2(fmaf(s[c + 1], a.scale_log2, -msc));
        ls4[(c >> 1) & 3] += p0 + p1;
        pk[c / 2] = pack2_bf16(p0, p1);
      }
      const float lsum = (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      if (j > 0) {
        // P and O are free once the previous tile's P V has completed
        if (!warp_wait(pv_done, (uint32_t)(j - 1) & 1u, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        if (__any_sync(0xFFFFFFFFu, need)) {
          const float f = need ? ex2(m_old - m_new) : 1.f;
          l *= f;
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float o[32];
            tc::tmem_ld32(tO + lane_off + 32u * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= f;
            tc::tmem_st32(tO + lane_off + 32u * c, o);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kTBN / 64; ++c) tc::tmem_st32u(tP + lane_off + 32u * c, pk + 32 * c);
      l += lsum;
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
    }
    if (ok && !warp_wait(pv_done, (uint32_t)(n_kt - 1) & 1u, abort_flag)) ok = false;
    if (ok) {
      tc::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t *orow = a.out + (int64_t)(row0 + r) * a.ld_out + h * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tc::tmem_ld32(tO + lane_off + 32u * c, o);
        if (r < a.S) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w = make_uint4(pack2_bf16(o[8 * q] * inv, o[8 * q + 1] * inv),
                                       pack2_bf16(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                       pack2_bf16(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                       pack2_bf16(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
            *reinterpret_cast<uint4 *>(orow + 32 * c + 8 * q) = w;
          }
        }
      }
    } else if (lane == 0) {
      atomicOr(a.err, ZO_FLAG_TIMEOUT);
      *abort_flag = 1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && !tc::mbar_wait(mma_done, 0)) atomicOr(a.err, ZO_FLAG_TIMEOUT);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 attn_encode_fn() {
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

template <int HD>
zo_status launch_tc(zo_ctx *ctx, const CUtensorMap &tmq, const CUtensorMap &tmkv, const TcAttnArgs &a,
                    int B) {
  using SM = TcAttnSmem<HD>;
  {
    const cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(attn_tc_kernel<HD>), (int)SM::kBytes);
    if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "attn_tc_kernel attribute: %s", cudaGetErrorString(e));
  }
  const dim3 grid((a.S + kTBM - 1) / kTBM, a.H, B);
  const int slot = ktime_begin(ctx);
  attn_tc_kernel<HD><<<grid, kTThreads, SM::kBytes, ctx->stream>>>(tmq, tmkv, a);
  const zo_status st = check_launch(ctx, "attn_tc_kernel");
  // algorithmic flops: Q K^T and P V over the causal pairs, 2 hd flops each per product
  if (st == ZO_OK)
    ktime_end(ctx, slot, ZO_KT_ATTENTION, 4.0 * HD * (double)B * a.H * ((double)a.S * (a.S + 1) / 2));
  return st;
}

}  // namespace

// Causal attention on the tensor cores for the grouped-query layout (Hk = H: multi-head).
zo_status launch_attention_tc(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S, int H,
                              int Hk, int hd) {
  if (B < 1 || S < 1 || H < 1 || Hk < 1 || H % Hk != 0)
    return fail(ctx, ZO_ERR_INVALID, "attention: bad shape");
  if (hd != 64 && hd != 128) return fail(ctx, ZO_ERR_UNSUPPORTED, "attention: head dim must be 64 or 128");
  if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return fail(ctx, ZO_ERR_INVALID, "attention: buffers must be 16-byte aligned");
  const int64_t ld = (int64_t)(H + 2 * Hk) * hd;
  auto fn = attn_encode_fn();
  if (!fn) return fail(ctx, ZO_ERR_CUDA, "attention: no tensor-map encoder");
  CUtensorMap tmq, tmkv;
  const cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)B * (cuuint64_t)S};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t boxq[2] = {64, (cuuint32_t)kTBM},
                   boxkv[2] = {64, (cuuint32_t)(hd == 128 ? TcAttnCfg<128>::kBN : TcAttnCfg<64>::kBN)};
  const cuuint32_t estr[2] = {1, 1};
  for (int m = 0; m < 2; ++m)
    if (fn(m ? &tmkv : &tmq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(qkv), dims,
           strides, m ? boxkv : boxq, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(ctx, ZO_ERR_CUDA, "attention: cuTensorMapEncodeTiled failed");
  TcAttnArgs a{S, H, Hk, 0, H * hd, (H + Hk) * hd, H * hd, 1.4426950408889634f / sqrtf((float)hd),
               out, &ctx->dstate->flags};
  return hd == 64 ? launch_tc<64>(ctx, tmq, tmkv, a, B) : launch_tc<128>(ctx, tmq, tmkv, a, B);
}

}  // namespace zo
