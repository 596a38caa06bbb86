// zo_attn.cu -- attention entry points of the decoder forward, and the one-query attention
// of the pruned last layer.  Full causal attention runs on the tensor cores (zo_attn_tc.cu):
//
//   out[b, s, h, :] = sum_{s' <= s} softmax_s'( q[b,s,h,:] . k[b,s',g,:] / sqrt(hd) ) v[b,s',g,:]
//
// with g = h for multi-head attention (OPT) and g = h / (H / Hk) for grouped-query attention
// (Qwen3: H query heads share Hk key/value heads).  Layout: qkv is the bf16 output of the
// fused QKV projection, [B*S][(H + 2 Hk) hd] with the query heads, then the key heads, then
// the value heads (OPT: Hk = H, so q, k, v sit at column offsets 0, d, 2d); out is bf16
// [B*S][H hd].
#include "zo_internal.cuh"

namespace zo {
namespace {

// Column layout of the fused projection output: row stride ld_in, query head h at
// q0 + h*hd, its key/value head kvh = h / (H / Hk) at k0 + kvh*hd and v0 + kvh*hd; the
// output row stride is ld_out, head h at h*hd.
struct AttnLayout {
  int ld_in, q0, k0, v0, H, Hk, ld_out;
};

// Attention of one query per sequence (the last position), for the pruned last layer of a
// loss-only forward: q [B][ldq] bf16 with head h at h*HD (already projected, normalised and
// rotated), keys/values in the fused projection rows of sequence b (layout al), out
// [B][al.ld_out] bf16.  One CTA per (head, sequence): warps take keys round-robin (a lane
// holds HD/32 features; a warp reduction gives each score), softmax in fp32 over the S
// scores held in shared memory, then P V accumulated per warp and summed over the warps in
// a fixed order.
template <int HD>
__global__ void __launch_bounds__(256)
attn_last_kernel(const uint16_t *__restrict__ q, int ldq, const uint16_t *__restrict__ qkv, int S,
                 AttnLayout al, float scale, uint16_t *__restrict__ out) {
  constexpr int V = HD / 32, NW = 8;
  extern __shared__ float asm_f[];
  float *sc = asm_f;                // [S]
  float *part = asm_f + S;          // [NW][HD]
  __shared__ float red[NW];
  const int h = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = h / (al.H / al.Hk);
  const int64_t row0 = (int64_t)b * S;
  float qv[V];
  {
    const uint16_t *qp = q + (int64_t)b * ldq + h * HD + lane * V;
#pragma unroll
    for (int i = 0; i < V; ++i) qv[i] = bf16_bits_to_f32(qp[i]) * scale;
  }
  const uint16_t *Kb = qkv + al.k0 + kvh * HD + lane * V;
  const uint16_t *Vb = qkv + al.v0 + kvh * HD + lane * V;
  for (int s = warp; s < S; s += NW) {
    const uint16_t *kr = Kb + (row0 + s) * al.ld_in;
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i) d = fmaf(qv[i], bf16_bits_to_f32(kr[i]), d);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xFFFFFFFFu, d, o);
    if (lane == 0) sc[s] = d;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int s = threadIdx.x; s < S; s += blockDim.x) m = fmaxf(m, sc[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < NW; ++w) m = fmaxf(m, red[w]);
  __syncthreads();  // red is reused below
  float l = 0.f;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const float p = expf(sc[s] - m);
    sc[s] = p;
    l += p;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.f;
  for (int w = 0; w < NW; ++w) l += red[w];
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  for (int s = warp; s < S; s += NW) {
    const float p = sc[s];
    const uint16_t *vr = Vb + (row0 + s) * al.ld_in;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = fmaf(p, bf16_bits_to_f32(vr[i]), acc[i]);
  }
#pragma unroll
  for (int i = 0; i < V; ++i) part[warp * HD + lane * V + i] = acc[i];
  __syncthreads();
  const float inv = 1.f / l;
  for (int f = threadIdx.x; f < HD; f += blockDim.x) {
    float o = 0.f;
    for (int w = 0; w < NW; ++w) o += part[w * HD + f];
    out[(int64_t)b * al.ld_out + h * HD + f] = f32_to_bf16_bits(o * inv);
  }
}

}  // namespace

// The last query of each sequence only: q [B][ldq] (head h at h*hd), keys/values in the
// fused projection output qkv [B*S][(H + 2 Hk) hd], out [B][H hd].
zo_status launch_attention_last(zo_ctx *ctx, const uint16_t *q, int ldq, const uint16_t *qkv,
                                uint16_t *out, int B, int S, int H, int Hk, int hd) {
  if (B < 1 || S < 1 || H < 1 || Hk < 1 || H % Hk != 0 || ldq < H * hd)
    return fail(ctx, ZO_ERR_INVALID, "attention (last query): bad shape");
  if (hd != 64 && hd != 128) return fail(ctx, ZO_ERR_UNSUPPORTED, "attention: head dim must be 64 or 128");
  const size_t smem = ((size_t)S + 8 * (size_t)hd) * sizeof(float);
  if (smem > 200 * 1024) return fail(ctx, ZO_ERR_UNSUPPORTED, "attention (last query): sequence too long");
  const AttnLayout al{(H + 2 * Hk) * hd, 0, H * hd, (H + Hk) * hd, H, Hk, H * hd};
  const float scale = 1.f / sqrtf((float)hd);
  const dim3 grid(H, B);
  cudaError_t e;
  if (hd == 64) {
    e = cudaFuncSetAttribute(attn_last_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      attn_last_kernel<64><<<grid, 256, smem, ctx->stream>>>(q, ldq, qkv, S, al, scale, out);
  } else {
    e = cudaFuncSetAttribute(attn_last_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      attn_last_kernel<128><<<grid, 256, smem, ctx->stream>>>(q, ldq, qkv, S, al, scale, out);
  }
  if (e != cudaSuccess) return fail(ctx, ZO_ERR_CUDA, "attn_last_kernel attribute: %s", cudaGetErrorString(e));
  return check_launch(ctx, "attn_last_kernel");
}

zo_status launch_attention_tc(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S, int H,
                              int Hk, int hd);

zo_status launch_attention_gqa(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S,
                               int H, int Hk, int hd) {
  return launch_attention_tc(ctx, qkv, out, B, S, H, Hk, hd);
}

zo_status launch_attention(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S, int H,
                           int d) {
  if (H < 1 || d % H != 0) return fail(ctx, ZO_ERR_INVALID, "attention: bad shape");
  return launch_attention_tc(ctx, qkv, out, B, S, H, H, d / H);
}

}  // namespace zo
