// zo_attn.cu -- causal multi-head / grouped-query attention of the decoder forward
// (inference only).
//
//   out[b, s, h, :] = sum_{s' <= s} softmax_s'( q[b,s,h,:] . k[b,s',g,:] / sqrt(hd) ) v[b,s',g,:]
//
// with g = h for multi-head attention (OPT) and g = h / (H / Hk) for grouped-query attention
// (Qwen3: H query heads share Hk key/value heads).  Layout: qkv is the bf16 output of the
// fused QKV projection, [B*S][(H + 2 Hk) hd] with the query heads, then the key heads, then
// the value heads (OPT: Hk = H, so q, k, v sit at column offsets 0, d, 2d); out is bf16
// [B*S][H hd].
//
// One CTA (8 warps) per (128-query tile, head, sequence); each warp owns 16 query rows.
// Key/value tiles of 64 rows stream through shared memory (cp.async, double-buffered);
// scores and the probability-weighted sum use bf16 mma.sync (m16n8k16, fp32 accumulate)
// with an online softmax in fp32 (running max and sum per row).  Attention is a few per
// cent of the forward's FLOPs; the projections around it run on tcgen05.
#include "zo_internal.cuh"

namespace zo {
namespace {

constexpr int kQT = 128, kKT = 64, kThreads = 256;  // 8 warps x 16 query rows

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;  // 0 source bytes -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t r[4], const void *p) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t r[4], const void *p) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x via the multi-function unit (max error ~2 ulp; the probabilities are rounded to bf16).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

template <int HD>
struct AttnSmem {
  static constexpr int kStride = HD + 8;  // bf16 elements per smem row (16-byte pad)
  static constexpr int kQTile = kQT * kStride;
  static constexpr int kKVTile = kKT * kStride;
  static constexpr int kBytes = (kQTile + 4 * kKVTile) * 2;  // Q + 2 x (K, V)
};

// Column layout of the fused projection output: row stride ld_in, query head h at
// q0 + h*hd, its key/value head kvh = h / (H / Hk) at k0 + kvh*hd and v0 + kvh*hd; the
// output row stride is ld_out, head h at h*hd.
struct AttnLayout {
  int ld_in, q0, k0, v0, H, Hk, ld_out;
};

template <int HD>
__global__ void __launch_bounds__(kThreads)
attn_causal_kernel(const uint16_t *__restrict__ qkv, uint16_t *__restrict__ out, int S,
                   AttnLayout al, float scale_log2) {
  using SM = AttnSmem<HD>;
  constexpr int ST = SM::kStride;
  extern __shared__ __align__(16) uint16_t sm[];
  uint16_t *sQ = sm;
  // K and V tiles of buffer `buf` after the Q tile
  auto sK = [&](int buf) { return sm + SM::kQTile + buf * SM::kKVTile; };
  auto sV = [&](int buf) { return sm + SM::kQTile + (2 + buf) * SM::kKVTile; };

  const int qt = gridDim.x - 1 - blockIdx.x;  // heavy (late) query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)b * S;
  const int64_t ld = al.ld_in;
  const int kvh = h / (al.H / al.Hk);
  const uint16_t *Qg = qkv + al.q0 + h * HD;
  const uint16_t *Kg = qkv + al.k0 + kvh * HD;
  const uint16_t *Vg = qkv + al.v0 + kvh * HD;
  constexpr int kChunks = HD / 8;  // 16-byte chunks per row

  auto load_tile = [&](uint16_t *dst, const uint16_t *src, int r0, int rows) {
    for (int i = tid; i < rows * kChunks; i += kThreads) {
      const int r = i / kChunks, c = i % kChunks;
      const bool valid = r0 + r < S;
      const uint16_t *g = src + (row0 + (valid ? r0 + r : 0)) * ld + c * 8;
      cp_async16(dst + r * ST + c * 8, g, valid);
    }
  };

  load_tile(sQ, Qg, qt * kQT, kQT);
  load_tile(sK(0), Kg, 0, kKT);
  load_tile(sV(0), Vg, 0, kKT);
  cp_async_commit();

  float o[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[HD / 16][4];
  const int g = lane >> 2, t = lane & 3;
  const int qrow0 = qt * kQT + warp * 16;  // first query row of this warp

  // causal: the key tiles that hold keys <= the last query row of this CTA
  const int last_q = min(qt * kQT + kQT, S) - 1;
  const int n_kt = last_q / kKT + 1;
  for (int kt = 0; kt < n_kt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < n_kt) {
      load_tile(sK(buf ^ 1), Kg, (kt + 1) * kKT, kKT);
      load_tile(sV(buf ^ 1), Vg, (kt + 1) * kKT, kKT);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk)
        ldsm_x4(qf[kk], sQ + (warp * 16 + (lane & 15)) * ST + kk * 16 + (lane >> 4) * 8);
    }
    // scores S = Q K^T for 16 rows x 64 keys
    float s[kKT / 8][4];
#pragma unroll
    for (int j = 0; j < kKT / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int jj = 0; jj < kKT / 16; ++jj) {
        uint32_t kb[4];
        const int key = jj * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int dim = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(kb, sK(buf) + key * ST + dim);
        mma16816(s[2 * jj], qf[kk], kb[0], kb[1]);
        mma16816(s[2 * jj + 1], qf[kk], kb[2], kb[3]);
      }
    }
    // mask (keys after the query, or beyond S: only on tiles that reach past the warp's
    // first query row or the end of the sequence) and online softmax
    const int key0 = kt * kKT;
    float mnew[2] = {mrow[0], mrow[1]};
    if (key0 + kKT - 1 > qrow0 || key0 + kKT > S) {
#pragma unroll
      for (int j = 0; j < kKT / 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qr = qrow0 + g + (e >> 1) * 8;
          const int kc = key0 + 8 * j + 2 * t + (e & 1);
          if (kc > qr || kc >= S) s[j][e] = -INFINITY;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kKT / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) mnew[e >> 1] = fmaxf(mnew[e >> 1], s[j][e]);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xFFFFFFFFu, mnew[r], 1));
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xFFFFFFFFu, mnew[r], 2));
    }
    float corr[2], msc[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      // rows that have seen no key yet keep m = -inf; use 0 as the shift then
      msc[r] = (mnew[r] == -INFINITY) ? 0.f : mnew[r] * scale_log2;
      corr[r] = (mrow[r] == -INFINITY) ? 0.f : fast_exp2(mrow[r] * scale_log2 - msc[r]);
      mrow[r] = mnew[r];
      lrow[r] *= corr[r];
    }
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      o[j][0] *= corr[0]; o[j][1] *= corr[0];
      o[j][2] *= corr[1]; o[j][3] *= corr[1];
    }
    uint32_t pf[kKT / 16][4];
#pragma unroll
    for (int j = 0; j < kKT / 8; ++j) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = fast_exp2(s[j][e] * scale_log2 - msc[e >> 1]);
        lrow[e >> 1] += p[e];
      }
      pf[j >> 1][(j & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
      pf[j >> 1][(j & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
    }
    // O += P V
#pragma unroll
    for (int kb = 0; kb < kKT / 16; ++kb) {
      const uint32_t a[4] = {pf[kb][0], pf[kb][1], pf[kb][2], pf[kb][3]};
#pragma unroll
      for (int jj = 0; jj < HD / 16; ++jj) {
        uint32_t vb[4];
        const int key = kb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dim = jj * 16 + (lane >> 4) * 8;
        ldsm_x4_t(vb, sV(buf) + key * ST + dim);
        mma16816(o[2 * jj], a, vb[0], vb[1]);
        mma16816(o[2 * jj + 1], a, vb[2], vb[3]);
      }
    }
    __syncthreads();  // the buffer is refilled two iterations later
  }
  // normalise and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xFFFFFFFFu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xFFFFFFFFu, lrow[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qr = qrow0 + g + r * 8;
    if (qr >= S) continue;
    const float inv = lrow[r] > 0.f ? 1.f / lrow[r] : 0.f;
    uint16_t *orow = out + (row0 + qr) * (int64_t)al.ld_out + h * HD;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      const uint32_t v = pack_bf16(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
      *reinterpret_cast<uint32_t *>(orow + 8 * j + 2 * t) = v;
    }
  }
}

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

zo_status launch_attention_gqa(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S,
                               int H, int Hk, int hd) {
  if (B < 1 || S < 1 || H < 1 || Hk < 1 || H % Hk != 0)
    return fail(ctx, ZO_ERR_INVALID, "attention: bad shape");
  if (hd != 64 && hd != 128) return fail(ctx, ZO_ERR_UNSUPPORTED, "attention: head dim must be 64 or 128");
  if ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return fail(ctx, ZO_ERR_INVALID, "attention: buffers must be 16-byte aligned");
  const AttnLayout al{(H + 2 * Hk) * hd, 0, H * hd, (H + Hk) * hd, H, Hk, H * hd};
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)hd);
  dim3 grid((S + kQT - 1) / kQT, H, B);
  if (hd == 64) {
    constexpr int bytes = AttnSmem<64>::kBytes;
    cudaFuncSetAttribute(attn_causal_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    attn_causal_kernel<64><<<grid, kThreads, bytes, ctx->stream>>>(qkv, out, S, al, scale_log2);
  } else {
    constexpr int bytes = AttnSmem<128>::kBytes;
    cudaFuncSetAttribute(attn_causal_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    attn_causal_kernel<128><<<grid, kThreads, bytes, ctx->stream>>>(qkv, out, S, al, scale_log2);
  }
  return check_launch(ctx, "attn_causal_kernel");
}

zo_status launch_attention(zo_ctx *ctx, const uint16_t *qkv, uint16_t *out, int B, int S, int H,
                           int d) {
  if (H < 1 || d % H != 0) return fail(ctx, ZO_ERR_INVALID, "attention: bad shape");
  return launch_attention_gqa(ctx, qkv, out, B, S, H, H, d / H);
}

}  // namespace zo
