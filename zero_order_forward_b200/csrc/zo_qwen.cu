// zo_qwen.cu -- the row kernels that the Qwen3-shaped decoder adds to the OPT-shaped one:
// RMSNorm and per-head query/key RMSNorm fused with the rotary position embedding.  The
// projections run on the tcgen05 GEMM (zo_gemm.cu, whose SwiGLU epilogue combines the gate
// and up projections), attention on the grouped-query kernel (zo_attn.cu); the layer loop
// is in zo_decoder.cu.
//
// Architecture of the family (public Qwen3 release): pre-RMSNorm layers, queries and keys
// RMS-normalised per head before rotary embeddings in the rotate-half convention (feature i
// pairs with feature i + e/2), SwiGLU feed-forward silu(g) * u.  Everything is computed in
// fp32 from bf16 inputs and rounded to bf16 once, where the next GEMM reads it.
#include "zo_internal.cuh"

namespace zo {
namespace {

constexpr int kVec = 8;            // columns per thread in the row kernels
constexpr int kMaxThreads = 1024;  // -> rows of up to 8192 columns

__device__ __forceinline__ float block_sum_fixed(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];  // same order in every thread
  __syncthreads();
  return s;
}

// y = bf16(x * rsqrt(mean(x^2) + eps) * w); one block per row, 8 consecutive columns per
// thread held in registers.
__global__ void __launch_bounds__(kMaxThreads)
rmsnorm_kernel(const float *__restrict__ x, const uint16_t *__restrict__ w, uint16_t *__restrict__ y,
               int d, float eps) {
  __shared__ float red[kMaxThreads / 32];
  const int c = threadIdx.x * kVec;
  const bool on = c < d;
  const float *row = x + (int64_t)blockIdx.x * d;
  float v[kVec];
  if (on) {
    const float4 a = reinterpret_cast<const float4 *>(row + c)[0];
    const float4 b = reinterpret_cast<const float4 *>(row + c)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < kVec; ++i) v[i] = 0.f;
  }
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) q = fmaf(v[i], v[i], q);
  const float rstd = rsqrtf(block_sum_fixed(q, red) / (float)d + eps);
  if (!on) return;
  const uint4 ww = *reinterpret_cast<const uint4 *>(w + c);
  const uint32_t wv[4] = {ww.x, ww.y, ww.z, ww.w};
  uint32_t o[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float y0 = v[2 * t] * rstd * __uint_as_float(wv[t] << 16);
    const float y1 = v[2 * t + 1] * rstd * __uint_as_float(wv[t] & 0xFFFF0000u);
    o[t] = pack_bf16x2(y0, y1);
  }
  *reinterpret_cast<uint4 *>(y + (int64_t)blockIdx.x * d + c) = make_uint4(o[0], o[1], o[2], o[3]);
}

// In place on bf16 rows of stride ld holding heads of HD features: heads hbeg ..
// hbeg+hcount-1 of every row t are RMS-normalised over their HD features with their
// weight (q_norm for heads < H, the query heads; k_norm for the key heads after them),
// then rotated by the angles of the row's position s (t mod S, or pos_fixed if >= 0):
//   out_i = x_i cos_i - x_{i+HD/2} sin_i,  out_{i+HD/2} = x_{i+HD/2} cos_i + x_i sin_i.
// One warp per (row, head); lane l owns features [l V, l V + V) of each half, V = HD / 64,
// so a rotation pair sits in one lane.
template <int HD>
__global__ void __launch_bounds__(256)
qk_norm_rope_kernel(uint16_t *__restrict__ qkv, int64_t ld, int hbeg, int hcount, int H,
                    const uint16_t *__restrict__ qn, const uint16_t *__restrict__ kn,
                    const float2 *__restrict__ rope, int64_t T, int S, int pos_fixed, float eps) {
  constexpr int V = HD / 64, HALF = HD / 2;
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= T * hcount) return;
  const int lane = threadIdx.x & 31;
  const int64_t t = wid / hcount;
  const int hh = hbeg + (int)(wid - t * hcount);
  const int s = pos_fixed >= 0 ? pos_fixed : (int)(t % S);
  uint16_t *x = qkv + t * ld + (int64_t)hh * HD;
  const uint16_t *w = hh < H ? qn : kn;
  const int f0 = lane * V;
  float a[V], b[V], wa[V], wb[V];
  if (V == 2) {  // one 4-byte load per half (f0 even, rows 16-byte aligned)
    const uint32_t xa = *reinterpret_cast<const uint32_t *>(x + f0);
    const uint32_t xb = *reinterpret_cast<const uint32_t *>(x + HALF + f0);
    const uint32_t ga = *reinterpret_cast<const uint32_t *>(w + f0);
    const uint32_t gb = *reinterpret_cast<const uint32_t *>(w + HALF + f0);
    a[0] = __uint_as_float(xa << 16); a[V - 1] = __uint_as_float(xa & 0xFFFF0000u);
    b[0] = __uint_as_float(xb << 16); b[V - 1] = __uint_as_float(xb & 0xFFFF0000u);
    wa[0] = __uint_as_float(ga << 16); wa[V - 1] = __uint_as_float(ga & 0xFFFF0000u);
    wb[0] = __uint_as_float(gb << 16); wb[V - 1] = __uint_as_float(gb & 0xFFFF0000u);
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      a[i] = bf16_bits_to_f32(x[f0 + i]);
      b[i] = bf16_bits_to_f32(x[HALF + f0 + i]);
      wa[i] = bf16_bits_to_f32(w[f0 + i]);
      wb[i] = bf16_bits_to_f32(w[HALF + f0 + i]);
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) ss = fmaf(a[i], a[i], fmaf(b[i], b[i], ss));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  const float rstd = rsqrtf(ss / (float)HD + eps);
  const float2 *cs = rope + (int64_t)s * HALF + f0;
  uint16_t oa[V], ob[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const float x1 = a[i] * rstd * wa[i], x2 = b[i] * rstd * wb[i];
    const float2 r = cs[i];
    oa[i] = f32_to_bf16_bits(x1 * r.x - x2 * r.y);
    ob[i] = f32_to_bf16_bits(x2 * r.x + x1 * r.y);
  }
  if (V == 2) {
    *reinterpret_cast<uint32_t *>(x + f0) = (uint32_t)oa[0] | ((uint32_t)oa[V - 1] << 16);
    *reinterpret_cast<uint32_t *>(x + HALF + f0) = (uint32_t)ob[0] | ((uint32_t)ob[V - 1] << 16);
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      x[f0 + i] = oa[i];
      x[HALF + f0 + i] = ob[i];
    }
  }
}

}  // namespace

zo_status launch_rmsnorm(zo_ctx *ctx, const float *x, const uint16_t *w, uint16_t *y, int rows,
                         int d, float eps) {
  if (rows < 1 || d < kVec || d % kVec || d > kVec * kMaxThreads ||
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) |
        reinterpret_cast<uintptr_t>(y)) & 15u))
    return fail(ctx, ZO_ERR_INVALID, "rmsnorm: need d %% 8 == 0, d <= 8192, 16-byte aligned rows");
  const int threads = ((d / kVec + 31) / 32) * 32;
  rmsnorm_kernel<<<rows, threads, 0, ctx->stream>>>(x, w, y, d, eps);
  return check_launch(ctx, "rmsnorm_kernel");
}

zo_status launch_qk_norm_rope(zo_ctx *ctx, uint16_t *x, int64_t ld, int hbeg, int hcount, int H,
                              const uint16_t *qn, const uint16_t *kn, const float2 *rope, int64_t T,
                              int S, int pos_fixed, int hd, float eps) {
  if (T < 1 || S < 1 || H < 1 || hbeg < 0 || hcount < 1 || ld < (int64_t)(hbeg + hcount) * hd)
    return fail(ctx, ZO_ERR_INVALID, "qk_norm_rope: bad shape");
  const int64_t warps = T * hcount;
  const unsigned blocks = (unsigned)((warps + 7) / 8);
  if (hd == 64)
    qk_norm_rope_kernel<64><<<blocks, 256, 0, ctx->stream>>>(x, ld, hbeg, hcount, H, qn, kn, rope, T,
                                                             S, pos_fixed, eps);
  else if (hd == 128)
    qk_norm_rope_kernel<128><<<blocks, 256, 0, ctx->stream>>>(x, ld, hbeg, hcount, H, qn, kn, rope, T,
                                                              S, pos_fixed, eps);
  else
    return fail(ctx, ZO_ERR_UNSUPPORTED, "qk_norm_rope: head dim must be 64 or 128");
  return check_launch(ctx, "qk_norm_rope_kernel");
}

}  // namespace zo
