// Router: logits GEMM (fp32 SIMT), then per-token softmax, top-k with
// lowest-index tie-break, gates, and per-chunk statistics.
//
// Follows "Sharding d'experts" (Kvasir wiki), "Backbone x worker":
// ``ids, p = top_k(softmax(cur @ router), k)`` and moe_stream.py
// ``MoEFFN.forward`` (bias-free gate Linear, additive exploration bias on the
// logits, softmax, topk, gates divided by their sum, batch-local load-balance
// fractions).  Top-k is taken on the logits: softmax is monotone, and the
// logits carry the tie information that rounded probabilities can lose.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kChunk = 128;  // tokens per router / permute chunk (one CTA)

// ---------------------------------------------------------------------------
// logits_part[split][T][E] = sum over this split's K range of x[t,i] * W_r[e,i]
//   x bf16 [T, d], W_r fp32 [E, d].  128 x 64 output tile per CTA, 128 threads,
//   8 x 8 outputs per thread, K staged through shared memory 32 at a time.
constexpr int kLgBM = 128, kLgBN = 64, kLgBK = 32;

__global__ void __launch_bounds__(128) k_router_logits(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ W, float* __restrict__ part,
                                                       int T, int d, int E, int k_per_split) {
  __shared__ __align__(16) float As[kLgBK][kLgBM + 4];
  __shared__ __align__(16) float Bs[kLgBK][kLgBN + 4];
  const int m0 = blockIdx.x * kLgBM, n0 = blockIdx.y * kLgBN;
  const int kbeg = blockIdx.z * k_per_split;
  const int kend = min(d, kbeg + k_per_split);
  const int tid = threadIdx.x;
  const int tx = tid & 7, ty = tid >> 3;  // 8 x 16 threads: n block tx*8, m block ty*8
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kend; k0 += kLgBK) {
    // A: 128 rows x 32 bf16 = 512 chunks of 8 bf16; 4 per thread
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int c = tid + it * 128;
      const int r = c >> 2, kc = (c & 3) * 8;
      const int gm = m0 + r, gk = k0 + kc;
      float v[8];
      if (gm < T && gk + 8 <= kend) {
        const uint4 u = *reinterpret_cast<const uint4*>(x + (size_t)gm * d + gk);
        v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
        v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          v[q] = (gm < T && gk + q < kend) ? __bfloat162float(x[(size_t)gm * d + gk + q]) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) As[kc + q][r] = v[q];
    }
    // B: 64 rows x 32 fp32 = 512 chunks of 4; 4 per thread
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int c = tid + it * 128;
      const int r = c >> 3, kc = (c & 7) * 4;
      const int gn = n0 + r, gk = k0 + kc;
      float4 v;
      if (gn < E && gk + 4 <= kend) {
        v = *reinterpret_cast<const float4*>(W + (size_t)gn * d + gk);
      } else {
        v.x = (gn < E && gk + 0 < kend) ? W[(size_t)gn * d + gk + 0] : 0.f;
        v.y = (gn < E && gk + 1 < kend) ? W[(size_t)gn * d + gk + 1] : 0.f;
        v.z = (gn < E && gk + 2 < kend) ? W[(size_t)gn * d + gk + 2] : 0.f;
        v.w = (gn < E && gk + 3 < kend) ? W[(size_t)gn * d + gk + 3] : 0.f;
      }
      Bs[kc + 0][r] = v.x; Bs[kc + 1][r] = v.y; Bs[kc + 2][r] = v.z; Bs[kc + 3][r] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kLgBK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8 + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = part + (size_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + ty * 8 + i;
    if (gm >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + tx * 8 + j;
      if (gn < E) out[(size_t)gm * E + gn] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Exact three-way bf16 split of the fp32 router weight: W = hi + mid + lo with
// each part a bf16 value (24 significand bits = 3 x 8), written as one
// [E, 3d] bf16 operand [hi | mid | lo].  x is bf16, so every product x * part
// is exact in fp32 and x W^T = [x | x | x] [hi | mid | lo]^T.
__global__ void __launch_bounds__(256) k_router_split(const float* __restrict__ W, __nv_bfloat16* __restrict__ Ws,
                                                      int E, int d) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)E * d) return;
  const long long e = i / d, k = i - e * d;
  const float w = W[i];
  const __nv_bfloat16 hi = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
  __nv_bfloat16* row = Ws + e * 3 * d;
  row[k] = hi;
  row[d + k] = mid;
  row[2 * d + k] = lo;
}

// wmax[0] = max_e ||W_r[e]||_2 (one CTA, fixed order).
__global__ void __launch_bounds__(256) k_router_wmax(const float* __restrict__ W, float* __restrict__ wmax, int E,
                                                     int d) {
  __shared__ float s_m[8];
  float m = 0.f;
  for (int e = warp_id(); e < E; e += 8) {
    float ss = 0.f;
    for (int i = lane_id(); i < d; i += 32) ss = fmaf(W[(size_t)e * d + i], W[(size_t)e * d + i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    m = fmaxf(m, sqrtf(ss));
  }
  if (lane_id() == 0) s_m[warp_id()] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = s_m[0];
    for (int w = 1; w < 8; ++w) r = fmaxf(r, s_m[w]);
    *wmax = r;
  }
}

// ---------------------------------------------------------------------------
// Warp argmax over the lanes' (value, index) pairs: larger value first, lower
// index first among equal values (-0.0 == +0.0, so the index decides).
__device__ __forceinline__ void warp_argmax(float& bv, int& bi) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
}

// Exact fp32 logits of up to 8 experts for one token, computed by the whole
// warp: lane l accumulates inputs l, l+32, ... with fmaf (one chain per
// expert), then a fixed xor tree.  The order does not depend on how many
// experts are batched together.
__device__ __forceinline__ void warp_dot_multi(const __nv_bfloat16* __restrict__ xr, const float* __restrict__ W,
                                               int d, const int (&ex)[8], int n, float (&out)[8]) {
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  for (int i = lane_id(); i < d; i += 32) {
    const float xv = __bfloat162float(xr[i]);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c < n) acc[c] = fmaf(xv, W[(size_t)ex[c] * d + i], acc[c]);
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
    out[c] = acc[c];
  }
}

struct RefineArgs {
  const __nv_bfloat16* x;  // [T, d]; nullptr = logits are final
  const float* W;          // [E, d] fp32 router weight
  const float* bias;       // [E] or nullptr
  const float* wmax;       // max_e ||W_r[e]||_2 (one float)
  int d;
  float gamma;             // bound factor of the screening logits: |err| <= gamma * ||x_t|| * ||w_e||
};

// Per-token tail of the router, shared by every logit source: softmax, top-k
// (k rounds of warp argmax on (logit desc, index asc)), gates, and the
// per-warp running statistics (sum of p per expert, picks per expert).
template <int EPL>
__device__ __forceinline__ void route_token(const float (&z)[EPL], int t, int E, int k, int renorm,
                                            float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w, float (&pacc)[EPL], int (&cacc)[EPL]) {
  const int lane = lane_id();
  if (logits_out != nullptr) {
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (lane + 32 * i < E) logits_out[(size_t)t * E + lane + 32 * i] = z[i];
  }
  float m = z[0];
#pragma unroll
  for (int i = 1; i < EPL; ++i) m = fmaxf(m, z[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float ez[EPL], ssum = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    ez[i] = (lane + 32 * i < E) ? expf(z[i] - m) : 0.f;
    ssum += ez[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
  const float inv = 1.f / ssum;
#pragma unroll
  for (int i = 0; i < EPL; ++i) pacc[i] += ez[i] * inv;

  unsigned taken = 0u;
  float wv = 0.f, wsum = 0.f;
  int iv = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (z[i] > bv || (z[i] == bv && e < bi))) { bv = z[i]; bi = e; }
    }
    warp_argmax(bv, bi);
    if ((bi & 31) == lane) {
      const int i = bi >> 5;
      taken |= 1u << i;
#pragma unroll
      for (int q = 0; q < EPL; ++q)
        if (q == i) cacc[q] += 1;
    }
    const float pj = expf(bv - m) * inv;
    if (lane == j) { wv = pj; iv = bi; }
    wsum += pj;
  }
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = iv;
    topk_w[(size_t)t * k + lane] = renorm ? wv / wsum : wv;
  }
}

// Chunk statistics of a CTA of 8 warps, combined in fixed warp order.
template <int EPL>
__device__ __forceinline__ void chunk_stats(float (&s_p)[8][EPL * 32], int (&s_c)[8][EPL * 32],
                                            const float (&pacc)[EPL], const int (&cacc)[EPL], int chunk, int E,
                                            int32_t* __restrict__ cnt, float* __restrict__ psum) {
  const int lane = lane_id(), warp = warp_id();
#pragma unroll
  for (int i = 0; i < EPL; ++i) { s_p[warp][lane + 32 * i] = pacc[i]; s_c[warp][lane + 32 * i] = cacc[i]; }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float ps = 0.f;
    int cs = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) { ps += s_p[w][e]; cs += s_c[w][e]; }
    cnt[(size_t)chunk * E + e] = cs;
    psum[(size_t)chunk * E + e] = ps;
  }
}

// One warp per token.  Lane l holds the logits of experts l, l+32, ...
//   logits = sum_split part[split] (+ bias); softmax; top-k; gates.
// With refine.x set, `part` holds screening logits from the tensor cores whose
// error is at most gamma * ||x_t|| * ||w_e||.  Every expert that could still be
// in the top k under that bound (screening logit >= k-th largest - 2 bound) is
// recomputed as a plain fp32 dot product, so the top-k decision is made on
// fp32 FMA logits; the others are certified out of the top k.
// Per chunk of kChunk tokens (one CTA, 8 warps x 16 tokens):
//   cnt[chunk][e]  tokens of the chunk that chose e
//   psum[chunk][e] sum over the chunk's tokens of p[t,e] (fixed order)
template <int EPL>
__global__ void __launch_bounds__(256) k_router_topk(const float* __restrict__ part, int nsplit,
                                                     const float* __restrict__ bias, float* __restrict__ logits_out,
                                                     int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                     int32_t* __restrict__ cnt, float* __restrict__ psum, int T,
                                                     int E, int k, int renorm, const RefineArgs refine) {
  __shared__ float s_p[8][EPL * 32];
  __shared__ int s_c[8][EPL * 32];
  const int lane = lane_id(), warp = warp_id();
  const int chunk = blockIdx.x;
  float pacc[EPL];
  int cacc[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) { pacc[i] = 0.f; cacc[i] = 0; }
  float b[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    b[i] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  }
  const float wmax = refine.x != nullptr ? *refine.wmax : 0.f;
  const int t_first = chunk * kChunk + warp * (kChunk / 8);
  const int t_end = min(T, t_first + kChunk / 8);

  auto load_z = [&](int t, float (&z)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      float v = -INFINITY;
      if (e < E && t < t_end) {
        v = part[(size_t)t * E + e];
        for (int s = 1; s < nsplit; ++s) v += part[(size_t)s * T * E + (size_t)t * E + e];
        if (bias != nullptr) v += b[i];
      }
      z[i] = v;
    }
  };

  float znext[EPL];
  load_z(t_first, znext);
  for (int t = t_first; t < t_end; ++t) {
    float z[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) z[i] = znext[i];
    load_z(t + 1, znext);  // prefetch the next token's logits

    if (refine.x != nullptr) {
      // k-th largest screening logit
      unsigned tk = 0u;
      float kth = -INFINITY;
      for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (e < E && !((tk >> i) & 1u) && (z[i] > bv || (z[i] == bv && e < bi))) { bv = z[i]; bi = e; }
        }
        warp_argmax(bv, bi);
        if ((bi & 31) == lane) tk |= 1u << (bi >> 5);
        kth = bv;
      }
      const __nv_bfloat16* xr = refine.x + (size_t)t * refine.d;
      float ss = 0.f;
      for (int i = lane; i < refine.d; i += 32) {
        const float v = __bfloat162float(xr[i]);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float bound = refine.gamma * sqrtf(ss) * 1.001f * wmax * 1.001f + 1e-6f * (fabsf(kth) + 1.f);
      const float thr = kth - 2.f * bound;
      // recompute the candidates exactly, up to 8 experts per pass
      int ex[8];
      int n = 0;
      auto flush = [&]() {
        float v[8];
        warp_dot_multi(xr, refine.W, refine.d, ex, n, v);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          if (c < n) {
            const int e = ex[c];
            float zz = v[c];
            if (refine.bias != nullptr) zz += refine.bias[e];
            if ((e & 31) == lane) {
#pragma unroll
              for (int i = 0; i < EPL; ++i)
                if (i == (e >> 5)) z[i] = zz;
            }
          }
        }
        n = 0;
      };
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        unsigned cand = __ballot_sync(0xffffffffu, lane + 32 * i < E && z[i] >= thr);
        while (cand) {
          const int l = __ffs(cand) - 1;
          cand &= cand - 1;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            if (c == n) ex[c] = 32 * i + l;
          if (++n == 8) flush();
        }
      }
      if (n > 0) flush();
    }
    route_token<EPL>(z, t, E, k, renorm, logits_out, topk_idx, topk_w, pacc, cacc);
  }
  chunk_stats<EPL>(s_p, s_c, pacc, cacc, chunk, E, cnt, psum);
}

// Router fully in one kernel for small E * d: the CTA keeps W_r^T in shared
// memory ([d][32 EPL + 1] fp32, padded against bank conflicts); each warp
// computes its tokens' logits as plain fp32 FMA chains over the inputs (lane l
// owns experts l, l+32, ...), then softmax / top-k / gates as above.
template <int EPL>
__global__ void __launch_bounds__(256) k_router_fused(const __nv_bfloat16* __restrict__ x, const float* __restrict__ W,
                                                      const float* __restrict__ bias, float* __restrict__ logits_out,
                                                      int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                      int32_t* __restrict__ cnt, float* __restrict__ psum, int T,
                                                      int d, int E, int k, int renorm) {
  extern __shared__ float s_wt[];
  __shared__ float s_p[8][EPL * 32];
  __shared__ int s_c[8][EPL * 32];
  constexpr int EP = EPL * 32 + 1;
  for (int i = threadIdx.x; i < E * d; i += blockDim.x) {  // coalesced reads; odd row pitch: no bank conflicts
    const int e = i / d, c = i - e * d;
    s_wt[c * EP + e] = W[i];
  }
  __syncthreads();
  const int lane = lane_id(), warp = warp_id();
  const int chunk = blockIdx.x;
  float pacc[EPL];
  int cacc[EPL];
  float b[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    pacc[i] = 0.f;
    cacc[i] = 0;
    const int e = lane + 32 * i;
    b[i] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  }
  const int t_first = chunk * kChunk + warp * (kChunk / 8);
  const int t_end = min(T, t_first + kChunk / 8);
  for (int t = t_first; t < t_end; ++t) {
    float acc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * d);
#pragma unroll 2
    for (int c0 = 0; c0 < d; c0 += 8) {
      const uint4 u = xr[c0 >> 3];  // same address in every lane: one broadcast load
      const float xv[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                           bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float* wr = s_wt + (size_t)(c0 + q) * EP + lane;
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] = fmaf(xv[q], wr[32 * i], acc[i]);
      }
    }
    float z[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) z[i] = (lane + 32 * i < E) ? acc[i] + b[i] : -INFINITY;
    route_token<EPL>(z, t, E, k, renorm, logits_out, topk_idx, topk_w, pacc, cacc);
  }
  chunk_stats<EPL>(s_p, s_c, pacc, cacc, chunk, E, cnt, psum);
}

// Router logits for small T (decode): W_r is the large operand and is
// streamed once.  A CTA of 8 warps owns 2 experts; the 4 warps of an expert
// split the inputs into quarters, lane l of a warp takes inputs 4l..4l+3 of
// each 128-input step, and keeps one fp32 FMA chain per token (TT tokens per
// pass).  Lanes, then quarters, are combined in fixed order.
template <int TT>
__global__ void __launch_bounds__(256) k_router_skinny(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ W, float* __restrict__ logits, int T,
                                                       int d, int E) {
  __shared__ float s_part[8][TT];
  const int lane = lane_id(), warp = warp_id();
  const int e = blockIdx.x * 2 + (warp >> 2);
  const int quarter = warp & 3;
  const int span = ((d + 511) / 512) * 128;  // inputs per quarter, a multiple of 128
  const int i_beg = quarter * span, i_end = min(d, i_beg + span);
  for (int t0 = 0; t0 < T; t0 += TT) {
    float acc[TT];
#pragma unroll
    for (int j = 0; j < TT; ++j) acc[j] = 0.f;
    if (e < E) {
      for (int i = i_beg + lane * 4; i < i_end; i += 128) {
        const float4 w4 = *reinterpret_cast<const float4*>(W + (size_t)e * d + i);
#pragma unroll
        for (int j = 0; j < TT; ++j) {
          if (t0 + j < T) {
            const uint2 u = *reinterpret_cast<const uint2*>(x + (size_t)(t0 + j) * d + i);
            acc[j] = fmaf(bf16lo(u.x), w4.x, acc[j]);
            acc[j] = fmaf(bf16hi(u.x), w4.y, acc[j]);
            acc[j] = fmaf(bf16lo(u.y), w4.z, acc[j]);
            acc[j] = fmaf(bf16hi(u.y), w4.w, acc[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < TT; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < TT; ++j) s_part[warp][j] = acc[j];
    }
    __syncthreads();
    if (quarter == 0 && e < E) {
      for (int j = lane; j < TT && t0 + j < T; j += 32) {
        const int w0 = warp;  // warps w0..w0+3 hold the quarters of expert e
        logits[(size_t)(t0 + j) * E + e] =
            ((s_part[w0][j] + s_part[w0 + 1][j]) + s_part[w0 + 2][j]) + s_part[w0 + 3][j];
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Per-chunk expert histogram from caller routing (moe_permute without moe_route).
__global__ void __launch_bounds__(256) k_chunk_hist(const int32_t* __restrict__ topk_idx, int32_t* __restrict__ cnt,
                                                    int T, int E, int k) {
  extern __shared__ int s_h[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_h[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kChunk;
  const int n = min(kChunk, T - t0) * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = topk_idx[(size_t)t0 * k + i];
    atomicAdd(&s_h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[(size_t)blockIdx.x * E + e] = s_h[e];
}

// ---------------------------------------------------------------------------
// One warp per expert: cnt[c][e] -> exclusive prefix over chunks (in place),
// counts[e]; optional f[e] = counts/T, P[e] = sum_c psum[c][e] / T.
__global__ void __launch_bounds__(256) k_chunk_scan(int32_t* __restrict__ cnt, const float* __restrict__ psum,
                                                    int32_t* __restrict__ counts, float* __restrict__ f_out,
                                                    float* __restrict__ p_out, int nchunks, int E, int T) {
  const int e = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  if (e >= E) return;
  const int per = (nchunks + 31) / 32;
  const int c0 = min(nchunks, lane * per), c1 = min(nchunks, c0 + per);
  int seg = 0;
  float ps = 0.f;
  for (int c = c0; c < c1; ++c) {
    seg += cnt[(size_t)c * E + e];
    if (psum != nullptr) ps += psum[(size_t)c * E + e];
  }
  int incl = seg;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - seg;
  for (int c = c0; c < c1; ++c) {
    const int v = cnt[(size_t)c * E + e];
    cnt[(size_t)c * E + e] = run;
    run += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (psum != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
  }
  if (lane == 0) {
    if (counts != nullptr) counts[e] = total;
    if (f_out != nullptr) f_out[e] = (float)total / (float)T;
    if (p_out != nullptr && psum != nullptr) p_out[e] = ps / (float)T;
  }
}

// aux = E * sum_e f_e P_e, one warp, fixed order.
__global__ void k_aux_finalize(const float* __restrict__ f, const float* __restrict__ P, float* __restrict__ aux,
                               int E) {
  float s = 0.f;
  for (int e = lane_id(); e < E; e += 32) s += f[e] * P[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane_id() == 0) *aux = (float)E * s;
}

}  // namespace moe
