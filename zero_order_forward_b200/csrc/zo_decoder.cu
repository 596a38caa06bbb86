// zo_decoder.cu -- loss-only forward of the two decoder families and the model-level C ABI:
// OPT-shaped (pre-LN, learned positions with offset 2, ReLU FFN, biases everywhere) and
// Qwen3-shaped (pre-RMSNorm, grouped-query attention with QK-norm and rotary embeddings,
// SwiGLU FFN, no biases); both tie the head to the token embedding.
//
// Inference mode only ("Probe-Space Preconditioning for Fast and Stable Zero-Order
// Training", abstract): each layer's activations overwrite the previous layer's, nothing is
// kept for a backward pass, and memory does not grow with the number of probes.
//
// Perturbed evaluation ("Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation",
// section "How 1.5-SPSA Works"): the loss at theta + s*eps*z_i.  theta is never written:
// before a layer runs, the fused unpack/apply kernel materialises that layer's perturbed
// parameters into one reusable layer window; the token/position embeddings, the final
// LayerNorm and the tied head rows are perturbed on load.
//
// OPT flat parameter order (bf16), d = d_model, f = d_ffn, V = vocab, P = max_pos + 2:
//   E[V][d], Pos[P][d],
//   per layer: ln1.g[d], ln1.b[d], Wqkv[3d][d], bqkv[3d], Wo[d][d], bo[d],
//              ln2.g[d], ln2.b[d], W1[f][d], b1[f], W2[d][f], b2[d],
//   final: lnf.g[d], lnf.b[d].
// Qwen3 flat parameter order (bf16), H / Hk query / key-value heads of e features:
//   E[V][d],
//   per layer: in_norm[d], Wqkv[(H+2Hk)e][d], q_norm[e], k_norm[e], Wo[d][He], post_norm[d],
//              Wgu[2f][d] (gate rows, then up rows), Wd[d][f],
//   final: final_norm[d].
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "zo_internal.cuh"

namespace zo {

zo_status launch_gemm(zo_ctx *ctx, const void *A, const void *B, const void *bias, void *out,
                      int M, int N, int K, int ldo, int epi, uint32_t extra_tx = 0,
                      int64_t lda = 0);
zo_status launch_gemm_perturbed(zo_ctx *ctx, const void *A, int64_t w_off, const void *bias,
                                void *out, int M, int N, int K, int ldo, int epi);
zo_status launch_attention(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S, int H,
                           int d);
zo_status launch_attention_gqa(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S,
                               int H, int Hk, int hd);
zo_status launch_rmsnorm(zo_ctx *ctx, const float *x, const uint16_t *w, uint16_t *y, int rows,
                         int d, float eps);
zo_status launch_qk_norm_rope(zo_ctx *ctx, uint16_t *x, int64_t ld, int hbeg, int hcount, int H,
                              const uint16_t *qn, const uint16_t *kn, const float2 *rope, int64_t T,
                              int S, int pos_fixed, int hd, float eps);
zo_status launch_attention_last(zo_ctx *ctx, const uint16_t *q, int ldq, const uint16_t *qkv,
                                uint16_t *out, int B, int S, int H, int Hk, int hd);

struct Layout {
  int64_t E, Pos, layers, layer_size, fin, total;  // Pos = -1: no position table (Qwen3)
  // offsets inside an OPT layer block
  int64_t ln1g, ln1b, wqkv, bqkv, wo, bo, ln2g, ln2b, w1, b1, w2, b2;
  // offsets inside a Qwen3 layer block (wqkv and wo above are shared)
  int64_t in_norm, q_norm, k_norm, post_norm, wgu, wd;
  int64_t qkv_cols, attn_cols;  // width of the QKV projection output and of attention's
};

bool common_cfg_ok(const zo_model_cfg &c) {
  return c.n_layers >= 1 && c.d_model >= 64 && c.d_model % 64 == 0 && c.d_model <= 8192 &&
         c.n_heads >= 1 && c.d_ffn >= 8 && c.d_ffn % 8 == 0 && c.vocab >= 2 && c.max_pos >= 1 &&
         c.class_ids[0] >= 0 && c.class_ids[0] < c.vocab && c.class_ids[1] >= 0 &&
         c.class_ids[1] < c.vocab;
}

bool make_qwen_layout(const zo_model_cfg &c, Layout *L) {
  if (!common_cfg_ok(c) || c.n_kv_heads < 1 || c.n_heads % c.n_kv_heads ||
      (c.head_dim != 64 && c.head_dim != 128) || !(c.rope_theta > 0.f) || !(c.norm_eps >= 0.f))
    return false;
  const int64_t d = c.d_model, f = c.d_ffn, e = c.head_dim, H = c.n_heads, Hk = c.n_kv_heads;
  L->E = 0;
  L->Pos = -1;
  L->layers = (int64_t)c.vocab * d;
  int64_t o = 0;
  L->in_norm = o; o += d;
  L->wqkv = o; o += (H + 2 * Hk) * e * d;
  L->q_norm = o; o += e;
  L->k_norm = o; o += e;
  L->wo = o; o += d * H * e;
  L->post_norm = o; o += d;
  L->wgu = o; o += 2 * f * d;
  L->wd = o; o += d * f;
  L->layer_size = o;
  L->fin = L->layers + (int64_t)c.n_layers * o;
  L->total = L->fin + d;
  L->qkv_cols = (H + 2 * Hk) * e;
  L->attn_cols = H * e;
  return true;
}

bool make_layout(const zo_model_cfg &c, Layout *L) {
  if (c.family == ZO_FAMILY_QWEN3) return make_qwen_layout(c, L);
  if (c.family != ZO_FAMILY_OPT || !common_cfg_ok(c) || c.d_model % c.n_heads) return false;
  const int64_t d = c.d_model, f = c.d_ffn;
  L->qkv_cols = 3 * d;
  L->attn_cols = d;
  L->E = 0;
  L->Pos = (int64_t)c.vocab * d;
  L->layers = L->Pos + (int64_t)(c.max_pos + 2) * d;
  int64_t o = 0;
  L->ln1g = o; o += d;
  L->ln1b = o; o += d;
  L->wqkv = o; o += 3 * d * d;
  L->bqkv = o; o += 3 * d;
  L->wo = o; o += d * d;
  L->bo = o; o += d;
  L->ln2g = o; o += d;
  L->ln2b = o; o += d;
  L->w1 = o; o += f * d;
  L->b1 = o; o += f;
  L->w2 = o; o += d * f;
  L->b2 = o; o += d;
  L->layer_size = o;
  L->fin = L->layers + (int64_t)c.n_layers * o;
  L->total = L->fin + 2 * d;
  return true;
}

namespace {

constexpr int kRowThreads = 256;

// 8 perturbed bf16 parameters starting at global element j (j % 8 == 0), widened to fp32.
__device__ __forceinline__ void load8_perturbed(const uint16_t *theta, int64_t j,
                                                const ProbeKey &pk, uint32_t step, float out[8]) {
  const uint4 v = *reinterpret_cast<const uint4 *>(theta + j);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    out[2 * t] = __uint_as_float(w[t] << 16);
    out[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
  }
  if (pk.sign) {
    // j % 8 == 0: the 8 elements are one half of a 16-element group
    const uint32_t bits = probe_group_bits((uint64_t)j >> 4, pk.probe, step, pk.k0, pk.k1) >> (j & 8);
    const float delta = pk.sign > 0 ? pk.eps : -pk.eps;
#pragma unroll
    for (int t = 0; t < 8; ++t)
      out[t] = bf16_bits_to_f32(f32_to_bf16_bits(perturb_f32(out[t], delta, (bits >> t) & 1u)));
  }
}

// h[t][:] = P_E[token] + P_Pos[s + 2] (fp32), one block per token; without a position
// table (pos_off < 0) h[t][:] = P_E[token].  An out-of-range token id writes NaN (the loss
// becomes non-finite and the step is skipped).
__global__ void __launch_bounds__(kRowThreads)
embed_kernel(const uint16_t *__restrict__ theta, const int32_t *__restrict__ tokens, int S, int d,
             int vocab, int64_t pos_off, ProbeKey pk, float *__restrict__ h) {
  const int64_t t = blockIdx.x;
  const int s = (int)(t % S);
  const int tok = tokens[t];
  const uint32_t step = pk.sign ? *pk.step : 0u;
  float *hrow = h + t * d;
  const bool ok = tok >= 0 && tok < vocab;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    if (!ok) {
#pragma unroll
      for (int i = 0; i < 8; ++i) hrow[c + i] = __int_as_float(0x7FC00000);
      continue;
    }
    float e[8], p[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    load8_perturbed(theta, (int64_t)tok * d + c, pk, step, e);
    if (pos_off >= 0) load8_perturbed(theta, pos_off + (int64_t)(s + 2) * d + c, pk, step, p);
    float4 *o = reinterpret_cast<float4 *>(hrow + c);
    o[0] = make_float4(e[0] + p[0], e[1] + p[1], e[2] + p[2], e[3] + p[3]);
    o[1] = make_float4(e[4] + p[4], e[5] + p[5], e[6] + p[6], e[7] + p[7]);
  }
}

__device__ __forceinline__ float block_allreduce_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];
  return s;
}

// xn = bf16(LayerNorm(x) * g + b), eps 1e-5, two passes in fp32 over registers.
// One block per row; each thread owns 8 consecutive columns (two 16-byte loads), so a
// block has ceil(d/8) threads rounded up to a warp (d <= 8192).
constexpr int kLnVec = 8;
constexpr int kLnMaxThreads = 1024;

__device__ __forceinline__ float ln_block_sum(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; ++i) s += red[i];  // same order in every thread
  __syncthreads();                           // red is reused by the next reduction
  return s;
}

__global__ void __launch_bounds__(kLnMaxThreads)
layernorm_kernel(const float *__restrict__ x, const uint16_t *__restrict__ g,
                 const uint16_t *__restrict__ b, uint16_t *__restrict__ y, int d) {
  __shared__ float red[kLnMaxThreads / 32];
  const int c = threadIdx.x * kLnVec;
  const bool on = c < d;
  const float *row = x + (int64_t)blockIdx.x * d;
  float v[kLnVec];
  if (on) {
    const float4 a = reinterpret_cast<const float4 *>(row + c)[0];
    const float4 bb = reinterpret_cast<const float4 *>(row + c)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = bb.x; v[5] = bb.y; v[6] = bb.z; v[7] = bb.w;
  } else {
#pragma unroll
    for (int i = 0; i < kLnVec; ++i) v[i] = 0.f;
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kLnVec; ++i) s += v[i];
  const float mean = ln_block_sum(s, red) / (float)d;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kLnVec; ++i) {
    const float u = on ? v[i] - mean : 0.f;
    q += u * u;
  }
  const float rstd = rsqrtf(ln_block_sum(q, red) / (float)d + 1e-5f);
  if (!on) return;
  const uint4 gg = *reinterpret_cast<const uint4 *>(g + c);
  const uint4 bv = *reinterpret_cast<const uint4 *>(b + c);
  const uint32_t gw[4] = {gg.x, gg.y, gg.z, gg.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
  uint32_t o[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float y0 = (v[2 * t] - mean) * rstd * __uint_as_float(gw[t] << 16) + __uint_as_float(bw[t] << 16);
    const float y1 = (v[2 * t + 1] - mean) * rstd * __uint_as_float(gw[t] & 0xFFFF0000u) +
                     __uint_as_float(bw[t] & 0xFFFF0000u);
    o[t] = pack_bf16x2(y0, y1);
  }
  *reinterpret_cast<uint4 *>(y + (int64_t)blockIdx.x * d + c) = make_uint4(o[0], o[1], o[2], o[3]);
}

int ln_threads(int d) { return ((d / kLnVec + 31) / 32) * 32; }

// dst[b][:] = src[b * S + S - 1][:] (rows of row_bytes, a multiple of 16): the last
// position of every sequence, for the pruned last layer.
__global__ void __launch_bounds__(kRowThreads)
gather_last_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst, int64_t row_bytes,
                   int S) {
  const int64_t b = blockIdx.x;
  const uint4 *from = reinterpret_cast<const uint4 *>(src + (b * S + S - 1) * row_bytes);
  uint4 *to = reinterpret_cast<uint4 *>(dst + b * row_bytes);
  for (int64_t i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) to[i] = from[i];
}

// Per sample: final norm of the last position (LayerNorm with gain and bias at fin_off, or
// with RMS = true RMSNorm with gain only), logits of the two class tokens through the tied
// head, 2-class cross-entropy.  Parameters perturbed on load.
template <bool RMS>
__global__ void __launch_bounds__(kRowThreads)
head_ce_kernel(const float *__restrict__ h, const uint16_t *__restrict__ theta, int S, int d,
               int64_t fin_off, int id0, int id1, const int32_t *__restrict__ labels,
               ProbeKey pk, double *partials, unsigned int *counter, double *out, int accumulate,
               double scale, float eps) {
  __shared__ float red[kRowThreads / 32];
  __shared__ bool last;
  const int b = blockIdx.x;
  const float *row = h + ((int64_t)b * S + S - 1) * d;
  const uint32_t step = pk.sign ? *pk.step : 0u;
  float mean = 0.f;
  if (!RMS) {
    float s = 0.f;
    for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8)
      for (int i = 0; i < 8; ++i) s += row[c + i];
    mean = block_allreduce_sum(s, red) / (float)d;
  }
  float q = 0.f;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8)
    for (int i = 0; i < 8; ++i) {
      const float u = row[c + i] - mean;
      q += u * u;
    }
  const float rstd = rsqrtf(block_allreduce_sum(q, red) / (float)d + eps);
  float l0 = 0.f, l1 = 0.f;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    float g[8], bb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, e0[8], e1[8];
    load8_perturbed(theta, fin_off + c, pk, step, g);
    if (!RMS) load8_perturbed(theta, fin_off + d + c, pk, step, bb);
    load8_perturbed(theta, (int64_t)id0 * d + c, pk, step, e0);
    load8_perturbed(theta, (int64_t)id1 * d + c, pk, step, e1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float xn = (row[c + i] - mean) * rstd * g[i] + bb[i];
      l0 = fmaf(xn, e0[i], l0);
      l1 = fmaf(xn, e1[i], l1);
    }
  }
  l0 = block_allreduce_sum(l0, red);
  l1 = block_allreduce_sum(l1, red);
  if (threadIdx.x == 0) {
    const int y = labels[b];
    const float m = fmaxf(l0, l1);
    const double lse = (double)m + (double)logf(expf(l0 - m) + expf(l1 - m));
    const double ce = (y == 0 || y == 1) ? lse - (double)(y == 0 ? l0 : l1) : (double)NAN;
    partials[b] = ce;
    __threadfence();
    last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last || threadIdx.x != 0) return;
  __threadfence();
  double tot = 0.0;
  for (unsigned int i = 0; i < gridDim.x; ++i) tot += __ldcg(partials + i);  // fixed order
  *out = (accumulate ? *out : 0.0) + scale * tot;
  *counter = 0u;
}

}  // namespace
}  // namespace zo

using namespace zo;

struct zo_model {
  zo_ctx *ctx = nullptr;
  zo_model_cfg cfg{};
  Layout L{};
  int64_t max_tokens = 0;
  uint16_t *window = nullptr;
  float *h = nullptr;
  uint16_t *xn = nullptr, *qkv = nullptr, *attn = nullptr, *mid = nullptr;
  int64_t ld_mid = 0;       // row stride of mid: d_ffn + 64 (see launch_gemm's lda)
  float2 *rope = nullptr;   // Qwen3: (cos, sin) of position s and pair i at [s][e/2]
  bool qwen = false;
  // pruned last layer of the loss forward: the last position of each sequence only
  int prune_rows = 0;       // capacity in sequences
  bool prune_enabled = true;
  float *hl = nullptr;      // residual rows [prune_rows][d]
  uint16_t *xl = nullptr, *ql = nullptr, *al = nullptr, *midl = nullptr;
  // zo_model_step_host: device copies of one step's tokens and labels, and its losses
  int32_t *stage = nullptr;
  size_t stage_cap = 0;     // int32 words
  double *stage_losses = nullptr;
};

namespace {

zo_status model_cuda(zo_ctx *ctx, cudaError_t e, const char *what) {
  if (e == cudaSuccess) return ZO_OK;
  cudaGetLastError();
  return fail(ctx, e == cudaErrorMemoryAllocation ? ZO_ERR_OOM : ZO_ERR_CUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

// Qwen3 layer: RMSNorm -> QKV projection -> per-head QK-norm + rotary -> grouped-query
// attention -> output projection added into the residual -> RMSNorm -> gate|up projection
// with the SwiGLU combination in its epilogue -> down projection added into the residual.
zo_status run_qwen_layer(zo_model *m, const uint16_t *lp, int B, int S) {
  zo_ctx *ctx = m->ctx;
  const zo_model_cfg &c = m->cfg;
  const Layout &L = m->L;
  const int d = c.d_model, f = c.d_ffn, e = c.head_dim, H = c.n_heads, Hk = c.n_kv_heads;
  const int T = B * S, nq = (int)L.qkv_cols, na = (int)L.attn_cols;
  const float eps = c.norm_eps;
  zo_status st;
  if ((st = launch_rmsnorm(ctx, m->h, lp + L.in_norm, m->xn, T, d, eps)) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->xn, lp + L.wqkv, nullptr, m->qkv, T, nq, d, nq,
                        ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
  if ((st = launch_qk_norm_rope(ctx, m->qkv, nq, 0, H + Hk, H, lp + L.q_norm, lp + L.k_norm, m->rope,
                                T, S, -1, e, eps)) != ZO_OK) return st;
  if ((st = launch_attention_gqa(ctx, m->qkv, m->attn, B, S, H, Hk, e)) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->attn, lp + L.wo, nullptr, m->h, T, d, na, d,
                        ZO_EPI_RESID_F32)) != ZO_OK) return st;
  if ((st = launch_rmsnorm(ctx, m->h, lp + L.post_norm, m->xn, T, d, eps)) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->xn, lp + L.wgu, nullptr, m->mid, T, f, d, (int)m->ld_mid,
                        ZO_EPI_SWIGLU_BF16)) != ZO_OK) return st;
  return launch_gemm(ctx, m->mid, lp + L.wd, nullptr, m->h, T, d, f, d, ZO_EPI_RESID_F32, 0,
                     m->ld_mid);
}

zo_status gather_last(zo_model *m, const void *src, void *dst, int64_t row_bytes, int B, int S) {
  gather_last_kernel<<<B, kRowThreads, 0, m->ctx->stream>>>(static_cast<const uint8_t *>(src),
                                                            static_cast<uint8_t *>(dst), row_bytes, S);
  return check_launch(m->ctx, "gather_last_kernel");
}

// The last layer of a loss-only forward, pruned to what the loss reads: keys and values
// for every position (the last query attends to all of them), everything else for the
// last position of each sequence only.  Leaves those residual rows in m->hl [B][d].
zo_status run_last_layer_pruned(zo_model *m, const uint16_t *lp, int B, int S) {
  zo_ctx *ctx = m->ctx;
  const zo_model_cfg &c = m->cfg;
  const Layout &L = m->L;
  const int d = c.d_model, f = c.d_ffn, T = B * S;
  const int nq = (int)L.qkv_cols, na = (int)L.attn_cols;
  zo_status st;
  if (m->qwen) {
    const int H = c.n_heads, Hk = c.n_kv_heads, e = c.head_dim;
    const float eps = c.norm_eps;
    if ((st = launch_rmsnorm(ctx, m->h, lp + L.in_norm, m->xn, T, d, eps)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->xn, lp + L.wqkv + (int64_t)H * e * d, nullptr, m->qkv + H * e, T,
                          2 * Hk * e, d, nq, ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
    if ((st = launch_qk_norm_rope(ctx, m->qkv, nq, H, Hk, H, lp + L.q_norm, lp + L.k_norm, m->rope, T,
                                  S, -1, e, eps)) != ZO_OK) return st;
    if ((st = gather_last(m, m->xn, m->xl, (int64_t)d * 2, B, S)) != ZO_OK) return st;
    if ((st = gather_last(m, m->h, m->hl, (int64_t)d * 4, B, S)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->xl, lp + L.wqkv, nullptr, m->ql, B, na, d, na,
                          ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
    if ((st = launch_qk_norm_rope(ctx, m->ql, na, 0, H, H, lp + L.q_norm, lp + L.k_norm, m->rope, B, S,
                                  S - 1, e, eps)) != ZO_OK) return st;
    if ((st = launch_attention_last(ctx, m->ql, na, m->qkv, m->al, B, S, H, Hk, e)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->al, lp + L.wo, nullptr, m->hl, B, d, na, d, ZO_EPI_RESID_F32)) != ZO_OK)
      return st;
    if ((st = launch_rmsnorm(ctx, m->hl, lp + L.post_norm, m->xl, B, d, eps)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->xl, lp + L.wgu, nullptr, m->midl, B, f, d, f,
                          ZO_EPI_SWIGLU_BF16)) != ZO_OK) return st;
    return launch_gemm(ctx, m->midl, lp + L.wd, nullptr, m->hl, B, d, f, d, ZO_EPI_RESID_F32);
  }
  layernorm_kernel<<<T, ln_threads(d), 0, ctx->stream>>>(m->h, lp + L.ln1g, lp + L.ln1b, m->xn, d);
  if ((st = check_launch(ctx, "layernorm_kernel")) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->xn, lp + L.wqkv + (int64_t)d * d, lp + L.bqkv + d, m->qkv + d, T,
                        2 * d, d, nq, ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
  if ((st = gather_last(m, m->xn, m->xl, (int64_t)d * 2, B, S)) != ZO_OK) return st;
  if ((st = gather_last(m, m->h, m->hl, (int64_t)d * 4, B, S)) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->xl, lp + L.wqkv, lp + L.bqkv, m->ql, B, d, d, d,
                        ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
  if ((st = launch_attention_last(ctx, m->ql, d, m->qkv, m->al, B, S, c.n_heads, c.n_heads,
                                  d / c.n_heads)) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->al, lp + L.wo, lp + L.bo, m->hl, B, d, d, d, ZO_EPI_RESID_F32)) != ZO_OK)
    return st;
  layernorm_kernel<<<B, ln_threads(d), 0, ctx->stream>>>(m->hl, lp + L.ln2g, lp + L.ln2b, m->xl, d);
  if ((st = check_launch(ctx, "layernorm_kernel")) != ZO_OK) return st;
  if ((st = launch_gemm(ctx, m->xl, lp + L.w1, lp + L.b1, m->midl, B, f, d, f, ZO_EPI_RELU_BF16)) != ZO_OK)
    return st;
  return launch_gemm(ctx, m->midl, lp + L.w2, lp + L.b2, m->hl, B, d, f, d, ZO_EPI_RESID_F32);
}

// Embedding plus the first n_run layers for one micro-batch; leaves the residual in m->h,
// or, when *pruned comes back true (prune requested and possible), the last layer ran
// pruned and the last positions' residual rows are in m->hl.
zo_status run_layers(zo_model *m, const int32_t *tokens, int B, int S, int n_run,
                     bool prune = false, bool *pruned = nullptr) {
  zo_ctx *ctx = m->ctx;
  const zo_model_cfg &c = m->cfg;
  const Layout &L = m->L;
  const int d = c.d_model, f = c.d_ffn;
  const int T = B * S;
  const uint16_t *theta = static_cast<const uint16_t *>(ctx->params);
  const ProbeKey pk = probe_key(ctx);
  embed_kernel<<<T, kRowThreads, 0, ctx->stream>>>(theta, tokens, S, d, c.vocab, L.Pos, pk, m->h);
  zo_status st = check_launch(ctx, "embed_kernel");
  if (st != ZO_OK) return st;
  const bool do_prune = prune && n_run >= 1 && S >= 2 && B <= m->prune_rows && S <= 32768;
  if (pruned) *pruned = do_prune;
  for (int l = 0; l < n_run; ++l) {
    const int64_t off = L.layers + (int64_t)l * L.layer_size;
    const uint16_t *lp = theta + off;
    if (pk.sign) {  // materialise this layer's perturbed parameters into the window
      st = launch_perturb(ctx, pk, off, L.layer_size, m->window);
      if (st != ZO_OK) return st;
      lp = m->window;
    }
    if (do_prune && l == n_run - 1) {
      if ((st = run_last_layer_pruned(m, lp, B, S)) != ZO_OK) return st;
      continue;
    }
    if (m->qwen) {
      if ((st = run_qwen_layer(m, lp, B, S)) != ZO_OK) return st;
      continue;
    }
    layernorm_kernel<<<T, ln_threads(d), 0, ctx->stream>>>(m->h, lp + L.ln1g, lp + L.ln1b, m->xn, d);
    if ((st = check_launch(ctx, "layernorm_kernel")) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->xn, lp + L.wqkv, lp + L.bqkv, m->qkv, T, 3 * d, d, 3 * d,
                          ZO_EPI_BIAS_BF16)) != ZO_OK) return st;
    if ((st = launch_attention(ctx, m->qkv, m->attn, B, S, c.n_heads, d)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->attn, lp + L.wo, lp + L.bo, m->h, T, d, d, d,
                          ZO_EPI_RESID_F32)) != ZO_OK) return st;
    layernorm_kernel<<<T, ln_threads(d), 0, ctx->stream>>>(m->h, lp + L.ln2g, lp + L.ln2b, m->xn, d);
    if ((st = check_launch(ctx, "layernorm_kernel")) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->xn, lp + L.w1, lp + L.b1, m->mid, T, f, d, (int)m->ld_mid,
                          ZO_EPI_RELU_BF16)) != ZO_OK) return st;
    if ((st = launch_gemm(ctx, m->mid, lp + L.w2, lp + L.b2, m->h, T, d, f, d,
                          ZO_EPI_RESID_F32, 0, m->ld_mid)) != ZO_OK) return st;
  }
  return ZO_OK;
}

zo_status check_batch(zo_model *m, const int32_t *tokens, int B, int S) {
  if (m->ctx->first_element != 0)
    return fail(m->ctx, ZO_ERR_UNSUPPORTED, "model: not separable over parameter slices (element offset must be 0)");
  if (!tokens || B < 1 || S < 1 || S > m->cfg.max_pos || (int64_t)B * S > m->max_tokens)
    return fail(m->ctx, ZO_ERR_INVALID, "batch %d x seq %d: need seq <= max_pos and B*S <= %lld",
                B, S, (long long)m->max_tokens);
  return ZO_OK;
}

}  // namespace

extern "C" {

zo_status zo_model_param_count(const zo_model_cfg *cfg, int64_t *M_out) {
  Layout L;
  if (!cfg || !M_out || !make_layout(*cfg, &L)) return ZO_ERR_INVALID;
  *M_out = L.total;
  return ZO_OK;
}

zo_status zo_model_create(zo_model **out, zo_ctx *ctx, const zo_model_cfg *cfg, int64_t max_tokens) {
  if (!out) return ZO_ERR_INVALID;
  *out = nullptr;
  if (!ctx || !cfg) return ZO_ERR_INVALID;
  Layout L;
  if (!make_layout(*cfg, &L)) return fail(ctx, ZO_ERR_INVALID, "invalid model configuration");
  if (ctx->dtype != ZO_BF16 || ctx->M != L.total)
    return fail(ctx, ZO_ERR_INVALID, "model needs a bf16 context with M = %lld", (long long)L.total);
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "model: not separable over parameter slices (element offset must be 0)");
  if (max_tokens < 1) return fail(ctx, ZO_ERR_INVALID, "max_tokens must be >= 1");
  zo_model *m = new (std::nothrow) zo_model();
  if (!m) return ZO_ERR_OOM;
  m->ctx = ctx;
  m->cfg = *cfg;
  m->L = L;
  m->max_tokens = max_tokens;
  m->qwen = cfg->family == ZO_FAMILY_QWEN3;
  const int64_t T = max_tokens, d = cfg->d_model, f = cfg->d_ffn;
  cudaError_t e = cudaMalloc(&m->window, (size_t)L.layer_size * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->h, (size_t)T * d * 4);
  if (e == cudaSuccess) e = cudaMalloc(&m->xn, (size_t)T * d * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->qkv, (size_t)T * L.qkv_cols * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->attn, (size_t)T * L.attn_cols * 2);
  m->ld_mid = f + 64;  // FC1 / SwiGLU output rows, padded (the FC2 / down GEMM's A)
  if (e == cudaSuccess) e = cudaMalloc(&m->mid, (size_t)T * m->ld_mid * 2);
  m->prune_rows = (int)(max_tokens < 512 ? max_tokens : 512);
  const int64_t R = m->prune_rows;
  if (e == cudaSuccess) e = cudaMalloc(&m->hl, (size_t)R * d * 4);
  if (e == cudaSuccess) e = cudaMalloc(&m->xl, (size_t)R * d * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->ql, (size_t)R * L.attn_cols * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->al, (size_t)R * L.attn_cols * 2);
  if (e == cudaSuccess) e = cudaMalloc(&m->midl, (size_t)R * f * 2);
  if (e == cudaSuccess && m->qwen) {
    // Rotary table: angle(s, i) = s * rope_theta^(-2i/e), evaluated in fp64 and rounded once.
    const int half = cfg->head_dim / 2;
    std::vector<float2> tab((size_t)cfg->max_pos * half);
    for (int s = 0; s < cfg->max_pos; ++s)
      for (int i = 0; i < half; ++i) {
        const double ang = (double)s * std::pow((double)cfg->rope_theta, -2.0 * i / cfg->head_dim);
        tab[(size_t)s * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    e = cudaMalloc(&m->rope, tab.size() * sizeof(float2));
    if (e == cudaSuccess)
      e = cudaMemcpy(m->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
  }
  if (e != cudaSuccess) {
    const zo_status st = model_cuda(ctx, e, "model buffers");
    zo_model_destroy(m);
    return st;
  }
  *out = m;
  return ZO_OK;
}

zo_status zo_model_destroy(zo_model *m) {
  if (!m) return ZO_OK;
  cudaStreamSynchronize(m->ctx->stream);
  cudaFree(m->window);
  cudaFree(m->h);
  cudaFree(m->xn);
  cudaFree(m->qkv);
  cudaFree(m->attn);
  cudaFree(m->mid);
  cudaFree(m->rope);
  cudaFree(m->hl);
  cudaFree(m->xl);
  cudaFree(m->ql);
  cudaFree(m->al);
  cudaFree(m->midl);
  cudaFree(m->stage);
  cudaFree(m->stage_losses);
  delete m;
  return ZO_OK;
}

zo_status zo_model_loss(zo_model *m, const int32_t *tokens, const int32_t *labels, int32_t batch,
                        int32_t seq, double scale, double *loss_out, int accumulate) {
  if (!m) return ZO_ERR_INVALID;
  zo_ctx *ctx = m->ctx;
  ctx->err.clear();
  zo_status st = check_batch(m, tokens, batch, seq);
  if (st != ZO_OK) return st;
  if (!labels || !loss_out) return fail(ctx, ZO_ERR_INVALID, "null labels or loss_out");
  if (batch > kMaxPartials) return fail(ctx, ZO_ERR_INVALID, "batch above %d", kMaxPartials);
  bool pruned = false;
  if ((st = run_layers(m, tokens, batch, seq, m->cfg.n_layers, m->prune_enabled, &pruned)) != ZO_OK)
    return st;
  const ProbeKey pk = probe_key(ctx);
  const uint16_t *theta = static_cast<const uint16_t *>(ctx->params);
  const zo_model_cfg &c = m->cfg;
  const float *hsrc = pruned ? m->hl : m->h;  // pruned: one row per sequence
  const int hS = pruned ? 1 : seq;
  if (m->qwen)
    head_ce_kernel<true><<<batch, kRowThreads, 0, ctx->stream>>>(
        hsrc, theta, hS, c.d_model, m->L.fin, c.class_ids[0], c.class_ids[1], labels, pk,
        ctx->partials, ctx->counter, loss_out, accumulate, scale, c.norm_eps);
  else
    head_ce_kernel<false><<<batch, kRowThreads, 0, ctx->stream>>>(
        hsrc, theta, hS, c.d_model, m->L.fin, c.class_ids[0], c.class_ids[1], labels, pk,
        ctx->partials, ctx->counter, loss_out, accumulate, scale, 1e-5f);
  return check_launch(ctx, "head_ce_kernel");
}

zo_status zo_model_set_pruning(zo_model *m, int enabled) {
  if (!m) return ZO_ERR_INVALID;
  m->prune_enabled = enabled != 0;
  return ZO_OK;
}

zo_status zo_model_hidden(zo_model *m, const int32_t *tokens, int32_t batch, int32_t seq,
                          int32_t n_layers_run, float *h_out) {
  if (!m) return ZO_ERR_INVALID;
  zo_ctx *ctx = m->ctx;
  ctx->err.clear();
  zo_status st = check_batch(m, tokens, batch, seq);
  if (st != ZO_OK) return st;
  if (!h_out || n_layers_run < 0 || n_layers_run > m->cfg.n_layers)
    return fail(ctx, ZO_ERR_INVALID, "bad hidden-state request");
  if ((st = run_layers(m, tokens, batch, seq, n_layers_run)) != ZO_OK) return st;
  return model_cuda(ctx,
                    cudaMemcpyAsync(h_out, m->h, (size_t)batch * seq * m->cfg.d_model * 4,
                                    cudaMemcpyDeviceToDevice, ctx->stream),
                    "copy hidden state");
}

zo_status zo_model_step(zo_model *m, const int32_t *tokens, const int32_t *labels, int32_t batch,
                        int32_t seq, int32_t n_micro, int32_t n_pert, float eps, float lr,
                        float damping, int preconditioned, double *losses_out) {
  if (!m) return ZO_ERR_INVALID;
  zo_ctx *ctx = m->ctx;
  if (n_micro < 1 || !losses_out) return fail(ctx, ZO_ERR_INVALID, "bad step arguments");
  if (ctx->first_element != 0)
    return fail(ctx, ZO_ERR_UNSUPPORTED, "model: not separable over parameter slices (element offset must be 0)");
  if (ctx->state != PState::Clean) return fail(ctx, ZO_ERR_STATE, "step while perturbed");
  const double scale = 1.0 / ((double)n_micro * batch);
  const int64_t tok_stride = (int64_t)batch * seq;
  double *L0 = losses_out, *Lp = losses_out + 1, *Lm = losses_out + 1 + n_pert;
  zo_status st;
  if (n_pert < 1 || n_pert > ZO_MAX_PROBES) return fail(ctx, ZO_ERR_INVALID, "n_pert out of range");
  phase_mark(ctx, 0);
  if (preconditioned) {
    for (int k = 0; k < n_micro; ++k)
      if ((st = zo_model_loss(m, tokens + k * tok_stride, labels + (int64_t)k * batch, batch, seq,
                              scale, L0, k > 0)) != ZO_OK)
        return st;
  } else if ((st = model_cuda(ctx, cudaMemsetAsync(L0, 0, sizeof(double), ctx->stream),
                              "clear L0")) != ZO_OK) {
    return st;
  }
  phase_mark(ctx, 1);
  for (int32_t i = 0; i < n_pert; ++i) {
    for (int s = +1; s >= -1; s -= 2) {
      if ((st = zo_perturb(ctx, s, eps, i)) != ZO_OK) return st;
      for (int k = 0; k < n_micro && st == ZO_OK; ++k)
        st = zo_model_loss(m, tokens + k * tok_stride, labels + (int64_t)k * batch, batch, seq,
                           scale, (s > 0 ? Lp : Lm) + i, k > 0);
      zo_restore(ctx);
      if (st != ZO_OK) return st;
    }
  }
  phase_mark(ctx, 2);
  st = step_device(ctx, Lp, Lm, n_pert, preconditioned ? L0 : nullptr, lr, eps, damping);
  phase_mark(ctx, 3);
  return st;
}

zo_status zo_model_step_host(zo_model *m, const int32_t *tokens_host, const int32_t *labels_host,
                             int32_t batch, int32_t seq, int32_t n_micro, int32_t n_pert, float eps,
                             float lr, float damping, int preconditioned, double *losses_host) {
  if (!m) return ZO_ERR_INVALID;
  zo_ctx *ctx = m->ctx;
  ctx->err.clear();
  if (!tokens_host || !labels_host || !losses_host || batch < 1 || seq < 1 || n_micro < 1 ||
      n_pert < 1 || n_pert > ZO_MAX_PROBES)
    return fail(ctx, ZO_ERR_INVALID, "bad host step arguments");
  const size_t n_tok = (size_t)n_micro * batch * seq, n_lab = (size_t)n_micro * batch;
  zo_status st;
  if (n_tok + n_lab > m->stage_cap) {
    if ((st = model_cuda(ctx, cudaStreamSynchronize(ctx->stream), "sync")) != ZO_OK) return st;
    cudaFree(m->stage);
    m->stage = nullptr;
    m->stage_cap = 0;
    if ((st = model_cuda(ctx, cudaMalloc(&m->stage, (n_tok + n_lab) * sizeof(int32_t)), "token staging")) != ZO_OK)
      return st;
    m->stage_cap = n_tok + n_lab;
  }
  if (!m->stage_losses &&
      (st = model_cuda(ctx, cudaMalloc(&m->stage_losses, (2 * ZO_MAX_PROBES + 1) * sizeof(double)),
                       "loss staging")) != ZO_OK)
    return st;
  int32_t *dtok = m->stage, *dlab = m->stage + n_tok;
  if ((st = model_cuda(ctx, cudaMemcpyAsync(dtok, tokens_host, n_tok * sizeof(int32_t), cudaMemcpyHostToDevice,
                                            ctx->stream), "copy tokens")) != ZO_OK ||
      (st = model_cuda(ctx, cudaMemcpyAsync(dlab, labels_host, n_lab * sizeof(int32_t), cudaMemcpyHostToDevice,
                                            ctx->stream), "copy labels")) != ZO_OK)
    return st;
  if ((st = zo_model_step(m, dtok, dlab, batch, seq, n_micro, n_pert, eps, lr, damping, preconditioned,
                          m->stage_losses)) != ZO_OK)
    return st;
  if ((st = model_cuda(ctx, cudaMemcpyAsync(losses_host, m->stage_losses, (2 * (size_t)n_pert + 1) * sizeof(double),
                                            cudaMemcpyDeviceToHost, ctx->stream), "copy losses")) != ZO_OK)
    return st;
  return model_cuda(ctx, cudaStreamSynchronize(ctx->stream), "sync");
}

zo_status zo_gemm_bf16(zo_ctx *ctx, const void *A, const void *B, const void *bias, void *out,
                       int32_t M, int32_t N, int32_t K, int32_t ldo, int32_t epilogue) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!A || !B || !out) return fail(ctx, ZO_ERR_INVALID, "null gemm operand");
  return launch_gemm(ctx, A, B, bias, out, M, N, K, ldo, epilogue);
}

zo_status zo_gemm_bf16_perturbed(zo_ctx *ctx, const void *A, int64_t w_offset, const void *bias,
                                 void *out, int32_t M, int32_t N, int32_t K, int32_t ldo,
                                 int32_t epilogue) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!A || !out) return fail(ctx, ZO_ERR_INVALID, "null gemm operand");
  return launch_gemm_perturbed(ctx, A, w_offset, bias, out, M, N, K, ldo, epilogue);
}

zo_status zo_debug_gemm_timeout(zo_ctx *ctx, const void *A, const void *B, void *out, int32_t M,
                                int32_t N, int32_t K) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!A || !B || !out) return fail(ctx, ZO_ERR_INVALID, "null gemm operand");
  return launch_gemm(ctx, A, B, nullptr, out, M, N, K, N, ZO_EPI_BIAS_BF16, 16u);
}

zo_status zo_attention(zo_ctx *ctx, const void *qkv, void *out, int32_t batch, int32_t seq,
                       int32_t n_heads, int32_t d_model) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!qkv || !out) return fail(ctx, ZO_ERR_INVALID, "null attention buffer");
  return launch_attention(ctx, static_cast<const uint16_t *>(qkv), static_cast<uint16_t *>(out),
                          batch, seq, n_heads, d_model);
}

zo_status zo_attention_gqa(zo_ctx *ctx, const void *qkv, void *out, int32_t batch, int32_t seq,
                           int32_t n_heads, int32_t n_kv_heads, int32_t head_dim) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!qkv || !out) return fail(ctx, ZO_ERR_INVALID, "null attention buffer");
  return launch_attention_gqa(ctx, static_cast<const uint16_t *>(qkv), static_cast<uint16_t *>(out),
                              batch, seq, n_heads, n_kv_heads, head_dim);
}

zo_status zo_rmsnorm(zo_ctx *ctx, const float *x, const void *w, void *out, int32_t rows, int32_t d,
                     float eps) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!x || !w || !out) return fail(ctx, ZO_ERR_INVALID, "null rmsnorm buffer");
  return launch_rmsnorm(ctx, x, static_cast<const uint16_t *>(w), static_cast<uint16_t *>(out), rows,
                        d, eps);
}

zo_status zo_layernorm(zo_ctx *ctx, const float *x, const void *gamma, const void *beta, void *out,
                       int32_t rows, int32_t d) {
  if (!ctx) return ZO_ERR_INVALID;
  ctx->err.clear();
  if (!x || !gamma || !beta || !out || rows < 1 || d < kLnVec || d % kLnVec ||
      d > kLnVec * kLnMaxThreads ||
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(gamma) |
        reinterpret_cast<uintptr_t>(beta) | reinterpret_cast<uintptr_t>(out)) & 15u))
    return fail(ctx, ZO_ERR_INVALID, "bad layernorm arguments (d %% 8 == 0, d <= 8192, 16-byte aligned)");
  layernorm_kernel<<<rows, ln_threads(d), 0, ctx->stream>>>(
      x, static_cast<const uint16_t *>(gamma), static_cast<const uint16_t *>(beta),
      static_cast<uint16_t *>(out), d);
  return check_launch(ctx, "layernorm_kernel");
}

}  // extern "C"
