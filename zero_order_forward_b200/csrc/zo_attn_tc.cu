// zo_attn_tc.cu -- causal multi-head / grouped-query attention on the 5th-generation tensor
// cores (inference forward only):
//
//   out[b, s, h, :] = sum_{s' <= s} softmax_s'( q[b,s,h,:] . k[b,s',g,:] / sqrt(hd) ) v[b,s',g,:]
//
// with g = h / (H / Hk).  Layout as zo_attn.cu: qkv is the fused projection output
// [B*S][(H + 2 Hk) hd] (query heads, key heads, value heads), out is [B*S][H hd].
//
// One CTA (6 warps) per (128-query tile, head, sequence), heavy (late) tiles first, two
// CTAs per SM.  Key tiles of 64 keys flow through a software pipeline in which the softmax
// of tile j+1 overlaps the P V product of tile j:
//   warp 0     one lane issues TMA loads: the Q tile once (boxes of 64 columns x 128 rows),
//              then K_j and V_{j-1} alternately into separate K and V rings (128-byte
//              swizzle), each stage released by the MMA that reads it;
//   warp 1     allocates 256 TMEM columns (two 64-column score buffers, O: hd) and one lane
//              issues S_j = Q K_j^T into buffer j % 2 (tcgen05.mma M=128, N=64, both operands
//              K-major in shared memory), O += P_j V_j once the softmax has written P_j (P read
//              from TMEM as the A operand, V MN-major from shared memory as loaded), and
//              S_{j+2} into the same buffer once that P V has completed;
//   warps 2-5  the softmax, one query row per thread (TMEM lane quadrant = warp % 4): read the
//              row of S_j from TMEM, scale, mask (diagonal and sequence-end tiles only), online
//              maximum with lazy rescaling (O and the row sum are rescaled only when the
//              maximum grows by more than 2^8, so exponentials stay below 256; only then does
//              the softmax wait for the previous P V), P = 2^(s - m) rounded to bf16 and
//              written over S_j in TMEM, row sum in fp32; at the end O / l is read from TMEM,
//              rounded to bf16 and stored.
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

// Key tiles of 64 keys.  TMEM (256 columns per CTA, two CTAs per SM): two score buffers of
// 64 columns, each later overwritten in place by its tile's bf16 probabilities (32 columns),
// then O (hd columns).  Separate K and V rings in shared memory, so that a key tile is
// released (and the next one loaded) as soon as its score MMA has completed.
template <int HD> struct TcAttnCfg {
  // (Measured at head dim 64: key tiles of 32 with three CTAs per SM, or four, were slower
  // than this: a tile's softmax then carries its fixed costs over half as many scores.)
  static constexpr int kBN = 64;
  static constexpr int kKS = HD == 128 ? 2 : 4;  // K stages
  static constexpr int kVS = HD == 128 ? 2 : 4;  // V stages
  static constexpr int kCtas = 2;
  static constexpr int kTmemCols = 256;
  static constexpr uint32_t kKBox = kBN * 128;  // bytes of one kBN-row x 64-column bf16 box
};

template <int HD>
struct TcAttnSmem {
  static constexpr int kKS = TcAttnCfg<HD>::kKS, kVS = TcAttnCfg<HD>::kVS;
  static constexpr uint32_t kQTile = (HD / 64) * kQBox;   // 128 rows x HD columns
  static constexpr uint32_t kKTile = (HD / 64) * TcAttnCfg<HD>::kKBox;  // kBN rows x HD columns
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQTile;              // [kKS]
  static constexpr uint32_t kV = kK + kKS * kKTile;        // [kVS]
  static constexpr uint32_t kBar = kV + kVS * kKTile;
  static constexpr int kNumBars = 1 + 2 * kKS + 2 * kVS + 2 + 2 + 2 + 1;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;    // barriers + alignment slack
  static_assert(kNumBars * 8 + 8 <= 256, "barrier area");
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

// max(a, b, c): one three-input instruction instead of two.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two lanes of fp32 arithmetic per instruction (sm_100's packed f32x2 forms), each lane
// rounded exactly as the scalar instruction: (d0, d1) = (a0 * b + c, a1 * b + c).
__device__ __forceinline__ void fma2_bc(float a0, float a1, float b, float c, float &d0, float &d1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tmov.b64 c, {%5, %5};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// (s0, s1) += (a0, a1)
__device__ __forceinline__ void add2(float &s0, float &s1, float a0, float a1) {
  asm("{\n\t.reg .b64 s, a;\n\t"
      "mov.b64 s, {%0, %1};\n\tmov.b64 a, {%2, %3};\n\t"
      "add.rn.f32x2 s, s, a;\n\tmov.b64 {%0, %1}, s;\n\t}"
      : "+f"(s0), "+f"(s1) : "f"(a0), "f"(a1));
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

// Phase bookkeeping of a ring of `n` barriers used once per item i: item i uses barrier
// i % n, and its completion is phase i / n of that barrier.
__device__ __forceinline__ uint32_t ring_parity(int i, int n) { return (uint32_t)(i / n) & 1u; }

template <int HD>
__global__ void __launch_bounds__(kTThreads, TcAttnCfg<HD>::kCtas)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmkv,
               TcAttnArgs a) {
  using SM = TcAttnSmem<HD>;
  constexpr int KS = SM::kKS, VS = SM::kVS;
  constexpr uint32_t kCols = TcAttnCfg<HD>::kTmemCols;
  constexpr int kTBN = TcAttnCfg<HD>::kBN;
  constexpr uint32_t kKBox = TcAttnCfg<HD>::kKBox;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + SM::kBar);
  uint64_t *q_full = bars;
  uint64_t *k_full = q_full + 1, *k_empty = k_full + KS;
  uint64_t *v_full = k_empty + KS, *v_empty = v_full + VS;
  uint64_t *s_full = v_empty + VS;  // [2] scores of tile j in buffer j % 2
  uint64_t *p_full = s_full + 2;    // [2] probabilities of tile j written (4 softmax warps)
  uint64_t *pv_done = p_full + 2;   // [2] O += P_j V_j completed
  uint64_t *mma_done = pv_done + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
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
    for (int i = 0; i < SM::kNumBars; ++i) tc::mbar_init(&bars[i], 1);
    tc::mbar_init(&p_full[0], 4);  // one arrival per softmax warp
    tc::mbar_init(&p_full[1], 4);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, kCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tO = tmem + 2 * kTBN;  // S/P buffers at columns 0 and kTBN

  if (warp == 0) {
    if (lane == 0) {  // TMA producer: Q once, then K_j ahead of V_{j-1}
      tc::tma_prefetch_desc(&tmq);
      tc::tma_prefetch_desc(&tmkv);
      tc::mbar_arrive_expect_tx(q_full, SM::kQTile);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c)
        tc::tma_load_2d(sm + SM::kQ + c * kQBox, &tmq, q_full, a.q0 + h * HD + 64 * c, row0 + q_first);
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int j) -> bool {
        if (*abort_flag || !tc::mbar_wait(&k_empty[j % KS], ring_parity(j, KS) ^ 1u)) return false;
        tc::mbar_arrive_expect_tx(&k_full[j % KS], SM::kKTile);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c)
          tc::tma_load_2d(sm + SM::kK + (j % KS) * SM::kKTile + c * kKBox, &tmkv, &k_full[j % KS],
                          a.k0 + kvh * HD + 64 * c, row0 + j * kTBN);
        k_issued = j + 1;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        if (*abort_flag || !tc::mbar_wait(&v_empty[j % VS], ring_parity(j, VS) ^ 1u)) return false;
        tc::mbar_arrive_expect_tx(&v_full[j % VS], SM::kKTile);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c)
          tc::tma_load_2d(sm + SM::kV + (j % VS) * SM::kKTile + c * kKBox, &tmkv, &v_full[j % VS],
                          a.v0 + kvh * HD + 64 * c, row0 + j * kTBN);
        v_issued = j + 1;
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j <= n_kt; ++j) {
        if (j < n_kt) ok = load_k(j);
        if (ok && j >= 1) ok = load_v(j - 1);
      }
      if (!ok) {
        atomicOr(a.err, ZO_FLAG_TIMEOUT);
        *abort_flag = 1;
        // let this CTA's loads land before it exits (bounded)
        tc::mbar_wait(q_full, 0);
        for (int i = k_issued - KS > 0 ? k_issued - KS : 0; i < k_issued; ++i)
          tc::mbar_wait(&k_full[i % KS], ring_parity(i, KS));
        for (int i = v_issued - VS > 0 ? v_issued - VS : 0; i < v_issued; ++i)
          tc::mbar_wait(&v_full[i % VS], ring_parity(i, VS));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t idS = tc::idesc_bf16_f32(kTBM, kTBN);
      constexpr uint32_t idO = tc::idesc_bf16_f32(kTBM, HD) | (1u << 16);  // B (V) MN-major
      const uint32_t qa = tc::smem_addr(sm + SM::kQ);
      // S_j = Q K_j^T into score buffer j % 2
      auto issue_s = [&](int j) -> bool {
        if (*abort_flag || !tc::mbar_wait(&k_full[j % KS], ring_parity(j, KS))) return false;
        tc::tc_fence_after();
        const uint32_t ka = tc::smem_addr(sm + SM::kK + (j % KS) * SM::kKTile);
        const uint32_t tS = tmem + (uint32_t)((j & 1) * kTBN);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t kk = (uint32_t)(k & 3) * 32u;
          tc::mma_bf16(tS, tc::smem_desc_k128(qa + (uint32_t)(k >> 2) * kQBox + kk),
                       tc::smem_desc_k128(ka + (uint32_t)(k >> 2) * kKBox + kk), idS, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&s_full[j & 1]);
        tc::mma_commit(&k_empty[j % KS]);
        return true;
      };
      bool ok = tc::mbar_wait(q_full, 0) && issue_s(0) && (n_kt < 2 || issue_s(1));
      for (int j = 0; ok && j < n_kt; ++j) {
        // O += P_j V_j once the softmax has written P_j (in place of S_j) and V_j has landed
        ok = tc::mbar_wait(&p_full[j & 1], ring_parity(j, 2)) &&
             tc::mbar_wait(&v_full[j % VS], ring_parity(j, VS));
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t va = tc::smem_addr(sm + SM::kV + (j % VS) * SM::kKTile);
        const uint32_t tP = tmem + (uint32_t)((j & 1) * kTBN);
#pragma unroll
        for (int k = 0; k < kTBN / 16; ++k) {
          const uint32_t boff = (uint32_t)k * 16u * 128u;  // 16 keys of 128-byte V rows
          tc::mma_bf16_tmem_a(tO, tP + 8u * k, tc::smem_desc_mn128(va + boff, kKBox), idO,
                              (j > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(&pv_done[j & 1]);
        tc::mma_commit(&v_empty[j % VS]);
        if (j + 2 < n_kt) {
          // S_{j+2} reuses buffer j % 2: wait until P_j V_j has read it
          ok = tc::mbar_wait(&pv_done[j & 1], ring_parity(j, 2)) && issue_s(j + 2);
        }
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
      const uint32_t tS = tmem + (uint32_t)((j & 1) * kTBN) + lane_off;
      if (!warp_wait(&s_full[j & 1], ring_parity(j, 2), abort_flag)) { ok = false; break; }
      tc::tc_fence_after();
      float s[kTBN];
#pragma unroll
      for (int c = 0; c < kTBN / 32; ++c) tc::tmem_ld32(tS + 32u * c, s + 32 * c);
      const int key0 = j * kTBN;
      // the causal / sequence-end mask touches only the tiles that reach the diagonal or the
      // end (uniform across the CTA: a real branch, not per-element selects)
      if (key0 + kTBN - 1 > q_first || key0 + kTBN > a.S) {
#pragma unroll
        for (int c = 0; c < kTBN; ++c)
          if (key0 + c > r || key0 + c >= a.S) s[c] = -INFINITY;
      }
      // the maximum of the raw scores (the scale is positive), then 2^(s * scale - m) with the
      // scaling folded into the exponent's fused multiply-add
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // 4 independent chains
#pragma unroll
      for (int c = 0; c < kTBN; c += 2) mx4[(c >> 1) & 3] = max3f(mx4[(c >> 1) & 3], s[c], s[c + 1]);
      const float mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * a.scale_log2;
      const float m_new = fmaxf(m_used, mx);
      // Lazy rescaling: keep the running maximum unless it grows by more than 2^8 (then
      // O and l are rescaled, once the previous tile's P V has completed).
      const bool need = j > 0 && m_new > m_used + 8.f;
      const float m_old = m_used;
      if (j == 0 || need) m_used = m_new;
      const float msc = m_used == -INFINITY ? 0.f : m_used;
      uint32_t pk[kTBN / 2];
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};  // two packed pairs of partial sums
#pragma unroll
      for (int c = 0; c < kTBN; c += 2) {
        float x0, x1;
        fma2_bc(s[c], s[c + 1], a.scale_log2, -msc, x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        if ((c >> 1) & 1) add2(ls4[2], ls4[3], p0, p1);
        else add2(ls4[0], ls4[1], p0, p1);
        pk[c / 2] = pack2_bf16(p0, p1);
      }
      const float lsum = (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      if (__any_sync(0xFFFFFFFFu, need)) {
        // O holds P_{j-1} V_{j-1} only once that MMA has completed
        if (!warp_wait(&pv_done[(j - 1) & 1], ring_parity(j - 1, 2), abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
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
      // P_j overwrites the first kTBN / 2 columns of S_j (already read into registers)
      tc::tmem_st32u(tS, pk);
      l += lsum;
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[j & 1]);
    }
    if (ok && !warp_wait(&pv_done[(n_kt - 1) & 1], ring_parity(n_kt - 1, 2), abort_flag)) ok = false;
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
                   boxkv[2] = {64, (cuuint32_t)TcAttnCfg<128>::kBN};  // the same for both head dims
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
