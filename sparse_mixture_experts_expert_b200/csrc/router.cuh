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

#include <cooperative_groups.h>

namespace moe {

namespace cg = cooperative_groups;

constexpr int kChunk = 32;         // tokens per router / grouping chunk (one warp)
constexpr int kMaxRouterE = 512;   // experts the routers handle

// ---------------------------------------------------------------------------
// logits_part[split][T][E] = sum over this split's K range of x[t,i] * W_r[e,i]
//   x bf16 [T, d], W_r fp32 [E, d].  128 x 64 output tile per CTA, 128 threads,
//   8 x 8 outputs per thread, K staged through shared memory 32 at a time.
constexpr int kLgBM = 128, kLgBN = 64, kLgBK = 32;

__global__ void __launch_bounds__(128) k_router_logits(const __nv_bfloat16* __restrict__ x,
                                                       const float* __restrict__ W, float* __restrict__ part,
                                                       int T, int d, int E, int k_per_split) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
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
// Router weight preparation for the tensor-core screening pass, one warp per
// expert row:
//  * two-term bf16 split W ~ hi + lo (hi = bf16(w), lo = bf16(w - hi): 16
//    significand bits, |w - hi - lo| <= 2^-16 |w|), written as one [E, 2d] bf16
//    operand [hi | lo]; x is bf16, so every product x * part is exact in fp32
//    and the screening logits x hi^T + x lo^T are one fp32 reduction of 2d
//    products (the screening GEMM accumulates both terms in one accumulator);
//  * the row norm ||W_r[e]||_2 for the screening error bound.
//  * with x set (the certified selection path), blocks past the weight rows
//    also compute xnorm2[t] = sum_i x[t,i]^2, one warp per token, every load of
//    the row in flight together (d <= 2048), and block 0 clears the list
//    lengths.
__global__ void __launch_bounds__(256) k_router_prep(const float* __restrict__ W, __nv_bfloat16* __restrict__ Ws,
                                                     float* __restrict__ wnorm, int E, int d,
                                                     int32_t* __restrict__ zero_counts, int n_zero,
                                                     const __nv_bfloat16* __restrict__ x, float* __restrict__ xnorm2,
                                                     int T) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  if (zero_counts != nullptr && blockIdx.x == 0)   // list lengths of the certified selection
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero_counts[i] = 0;
  const int wblocks = (E + 7) / 8;
  if ((int)blockIdx.x >= wblocks) {
    const long long t = (long long)(blockIdx.x - wblocks) * 8 + warp_id();
    if (x == nullptr || t >= T) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
    const int nv = d >> 3;
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = lane_id() + 32 * j < nv ? xr[lane_id() + 32 * j] : make_uint4(0, 0, 0, 0);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float q[8] = {bf16lo(u[j].x), bf16hi(u[j].x), bf16lo(u[j].y), bf16hi(u[j].y),
                          bf16lo(u[j].z), bf16hi(u[j].z), bf16lo(u[j].w), bf16hi(u[j].w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(q[i], q[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane_id() == 0) xnorm2[t] = ss;
    return;
  }
  const int e = blockIdx.x * 8 + warp_id();
  if (e >= E) return;
  const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d);
  __nv_bfloat16* row = Ws + (size_t)e * 2 * d;
  float ss = 0.f;
  // float4 per lane, four loads in flight per round (d % 16 == 0)
  for (int v0 = lane_id(); v0 < d / 4; v0 += 128) {
    float4 wv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) wv[j] = v0 + 32 * j < d / 4 ? __ldg(wr + v0 + 32 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int v = v0 + 32 * j;
      if (v >= d / 4) break;
      const float w4[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
      uint32_t hi2[2], lo2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __nv_bfloat162 hi = __floats2bfloat162_rn(w4[2 * h], w4[2 * h + 1]);
        const __nv_bfloat162 lo =
            __floats2bfloat162_rn(w4[2 * h] - __low2float(hi), w4[2 * h + 1] - __high2float(hi));
        hi2[h] = *reinterpret_cast<const uint32_t*>(&hi);
        lo2[h] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      reinterpret_cast<uint2*>(row)[v] = make_uint2(hi2[0], hi2[1]);
      reinterpret_cast<uint2*>(row + d)[v] = make_uint2(lo2[0], lo2[1]);
#pragma unroll
      for (int q = 0; q < 4; ++q) ss = fmaf(w4[q], w4[q], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane_id() == 0) wnorm[e] = sqrtf(ss);
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

struct RefineArgs {
  const __nv_bfloat16* x;  // [T, d]; nullptr = logits are final
  const float* W;          // [E, d] fp32 router weight
  const float* bias;       // [E] or nullptr
  const float* wnorm;      // [E] ||W_r[e]||_2
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

// Exact fp32 logit of one (token, expert) pair by the whole warp: lane l takes
// the 8-input slices l, l+32, ... (16-byte loads of x, 32-byte loads of W),
// one fmaf chain, then a fixed xor tree.  d % 8 == 0.
__device__ __forceinline__ float warp_dot(const __nv_bfloat16* __restrict__ xr, const float* __restrict__ wr, int d) {
  float acc = 0.f;
  const int nv = d >> 3;
  for (int v = lane_id(); v < nv; v += 32) {
    const uint4 u = reinterpret_cast<const uint4*>(xr)[v];
    const float4 w0 = reinterpret_cast<const float4*>(wr)[2 * v], w1 = reinterpret_cast<const float4*>(wr)[2 * v + 1];
    acc = fmaf(bf16lo(u.x), w0.x, acc); acc = fmaf(bf16hi(u.x), w0.y, acc);
    acc = fmaf(bf16lo(u.y), w0.z, acc); acc = fmaf(bf16hi(u.y), w0.w, acc);
    acc = fmaf(bf16lo(u.z), w1.x, acc); acc = fmaf(bf16hi(u.z), w1.y, acc);
    acc = fmaf(bf16lo(u.w), w1.z, acc); acc = fmaf(bf16hi(u.w), w1.w, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Warp argmax on (value desc, index asc) by two warp reductions: the largest
// value (redux.sync max.f32; NaNs are never chosen, -0.0 == +0.0), then the
// lowest index among the lanes holding it.
__device__ __forceinline__ void warp_argmax_redux(float& bv, int& bi) {
  float m;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(bv));
  bi = (int)__reduce_min_sync(0xffffffffu, bv == m ? (unsigned)bi : 0xffffffffu);
  bv = m;
}

// k rounds of warp argmax over the lanes' logits (lane l holds experts l, l+32, ...):
// fills sel_v / sel_i (lane j keeps pick j) and returns the k-th largest value.
template <int EPL>
__device__ __forceinline__ float warp_topk(const float (&z)[EPL], int E, int k, float& sel_v, int& sel_i,
                                           unsigned& taken) {
  const int lane = lane_id();
  taken = 0u;
  float kth = -INFINITY;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && z[i] > bv) { bv = z[i]; bi = e; }  // ascending e: first max wins
    }
    warp_argmax_redux(bv, bi);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) { sel_v = bv; sel_i = bi; }
    kth = bv;
  }
  return kth;
}

// The k-th largest of the lanes' logits (with multiplicity), without the
// indices: rounds of (warp maximum, how many entries equal it); the k-th
// largest is the maximum of the round at which the running count reaches k,
// and each earlier round removes its maximum's entries.  Entries past the
// expert count must be -inf.  At most k rounds (each removes at least one).
template <int EPL>
__device__ __forceinline__ float warp_kth(const float (&z)[EPL], int E, int k) {
  (void)E;
  float zz[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) zz[i] = z[i];
  int need = k;
  for (;;) {
    float lm = zz[0];
#pragma unroll
    for (int i = 1; i < EPL; ++i) lm = fmaxf(lm, zz[i]);
    float m;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(lm));
    int c = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) c += zz[i] == m ? 1 : 0;
    const int total = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
    if (total >= need) return m;
    need -= total;
#pragma unroll
    for (int i = 0; i < EPL; ++i) zz[i] = zz[i] == m ? -INFINITY : zz[i];
  }
}

// Exact fp32 logit of one (token, expert) pair with the token's inputs held in
// registers as fp32 (xf[8q + i] = x[8 (lane + 32 q) + i], d <= 1024): the same
// per-lane order and xor tree as warp_dot, without the bf16 unpacking.
__device__ __forceinline__ float warp_dot_reg(const float (&xf)[32], const float* __restrict__ wr, int d) {
  float acc = 0.f;
  const int nv = d >> 3, lane = lane_id();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int v = lane + 32 * q;
    if (v < nv) {
      const float4 w0 = reinterpret_cast<const float4*>(wr)[2 * v], w1 = reinterpret_cast<const float4*>(wr)[2 * v + 1];
      acc = fmaf(xf[8 * q + 0], w0.x, acc); acc = fmaf(xf[8 * q + 1], w0.y, acc);
      acc = fmaf(xf[8 * q + 2], w0.z, acc); acc = fmaf(xf[8 * q + 3], w0.w, acc);
      acc = fmaf(xf[8 * q + 4], w1.x, acc); acc = fmaf(xf[8 * q + 5], w1.y, acc);
      acc = fmaf(xf[8 * q + 6], w1.z, acc); acc = fmaf(xf[8 * q + 7], w1.w, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Router selection, one warp per token: lane l holds the logits of experts l,
// l+32, ...; a CTA of NW warps is one chunk of kChunk = 32 tokens (32 / NW
// tokens per warp).
//   logits = sum_split part[split] (+ bias); top-k (k rounds of warp argmax on
//   (value desc, index asc)); softmax; gates; chunk statistics.
// With refine.x set, `part` holds screening logits from the tensor cores whose
// error is at most gamma * ||x_t|| * max_e ||w_e||.  Every expert whose
// screening logit is >= (k-th largest - 2 bound) may still be in the top k and
// is recomputed exactly (warp_dot: a plain fp32 FMA dot product), then the top
// k is taken again; the others are certified out of the top k.  The softmax
// uses the exact values where they exist and the screening values elsewhere.
// Chunk statistics, expert-major: cnt[e][chunk] = picks, psum[e][chunk] = sum
// over the chunk's tokens of p[t,e].
//   STATS (large batches; a CTA of NW warps is one chunk of kChunk = 32
//   tokens, 32 / NW per warp): each warp accumulates its own row of the dynamic
//   shared memory (2 * NW * E words), then the rows are added in warp order.
//   !STATS (small batches; NW warps = NW tokens per CTA, so the tokens spread
//   over the SMs): the probabilities p[t,e] go to p_out and k_chunk_stats
//   forms the tables.  p_out may alias part: a warp writes row t only after
//   reading every split of row t.
template <int EPL, int NW, bool XREG, bool STATS>
__global__ void __launch_bounds__(NW * 32, 1) k_router_topk(const float* part, int nsplit,
                                                         const float* __restrict__ bias, float* __restrict__ logits_out,
                                                         int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                         int32_t* __restrict__ cnt, float* __restrict__ psum,
                                                         float* p_out, int T, int E, int k, int renorm,
                                                         const RefineArgs refine) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ float s_stat[];
  constexpr int TPW = STATS ? kChunk / NW : 1;
  const int lane = lane_id(), warp = warp_id();
  const int chunk = blockIdx.x;
  const int nchunks = (T + kChunk - 1) / kChunk;
  float* s_p = s_stat + (size_t)warp * E;
  int* s_c = reinterpret_cast<int*>(s_stat + (size_t)NW * E) + (size_t)warp * E;
  if (STATS)
    for (int e = lane; e < E; e += 32) { s_p[e] = 0.f; s_c[e] = 0; }
  float wmax = 0.f;
  if (refine.x != nullptr) {
    for (int e = lane; e < E; e += 32) wmax = fmaxf(wmax, refine.wnorm[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
  }
  for (int tt = 0; tt < TPW; ++tt) {
    const int t = STATS ? chunk * kChunk + warp * TPW + tt : blockIdx.x * NW + warp;
    if (t >= T) break;
    float z[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      float v = -INFINITY;
      if (e < E) {
        v = part[(size_t)t * E + e];
        for (int sp = 1; sp < nsplit; ++sp) v += part[(size_t)sp * T * E + (size_t)t * E + e];
        if (bias != nullptr) v += bias[e];
      }
      z[i] = v;
    }
    float sel_v = 0.f;
    int sel_i = 0;
    unsigned taken;
    // with the certified recompute only the k-th screening value is needed here: the picks come later
    float kth = refine.x != nullptr ? warp_kth<EPL>(z, E, k) : warp_topk<EPL>(z, E, k, sel_v, sel_i, taken);
    if (refine.x != nullptr) {
      const __nv_bfloat16* xr = refine.x + (size_t)t * refine.d;
      float ss = 0.f;
      float xf[XREG ? 32 : 1];
      if constexpr (XREG) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int v = lane + 32 * q;
          uint4 u = make_uint4(0, 0, 0, 0);
          if (v < (refine.d >> 3)) u = reinterpret_cast<const uint4*>(xr)[v];
          xf[8 * q + 0] = bf16lo(u.x); xf[8 * q + 1] = bf16hi(u.x); xf[8 * q + 2] = bf16lo(u.y);
          xf[8 * q + 3] = bf16hi(u.y); xf[8 * q + 4] = bf16lo(u.z); xf[8 * q + 5] = bf16hi(u.z);
          xf[8 * q + 6] = bf16lo(u.w); xf[8 * q + 7] = bf16hi(u.w);
#pragma unroll
          for (int j = 0; j < 8; ++j) ss = fmaf(xf[8 * q + j], xf[8 * q + j], ss);
        }
      } else {
        for (int v = lane; v < (refine.d >> 3); v += 32) {
          const uint4 u = reinterpret_cast<const uint4*>(xr)[v];
          const float q[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                              bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
          for (int j = 0; j < 8; ++j) ss = fmaf(q[j], q[j], ss);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float bound = refine.gamma * sqrtf(ss) * 1.001f * wmax * 1.001f + 1e-6f * (fabsf(kth) + 1.f);
      const float thr = kth - 2.f * bound;
      // candidate c (in expert order) is parked in lane c: exact value cv, index ci
      int nc = 0;
      float cv = -INFINITY;
      int ci = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        unsigned cand = __ballot_sync(0xffffffffu, lane + 32 * i < E && z[i] >= thr);
        while (cand) {
          const int l = __ffs(cand) - 1;
          cand &= cand - 1;
          const int e = 32 * i + l;
          float v;
          if constexpr (XREG) v = warp_dot_reg(xf, refine.W + (size_t)e * refine.d, refine.d);
          else v = warp_dot(xr, refine.W + (size_t)e * refine.d, refine.d);
          if (refine.bias != nullptr) v += refine.bias[e];
          if (lane == l) z[i] = v;
          if (lane == nc) { cv = v; ci = e; }
          ++nc;
        }
      }
      if (nc <= 32) {
        // The exact top k lies among the candidates: rank them by (value desc, index asc) with shuffles
        // instead of another k rounds over all experts.
        int rank = 0;
        for (int j = 0; j < nc; ++j) {
          const float vj = __shfl_sync(0xffffffffu, cv, j);
          const int ij = __shfl_sync(0xffffffffu, ci, j);
          rank += (vj > cv || (vj == cv && ij < ci)) ? 1 : 0;
        }
        for (int j = 0; j < nc; ++j) {
          const int rj = __shfl_sync(0xffffffffu, rank, j);
          const float vj = __shfl_sync(0xffffffffu, cv, j);
          const int ij = __shfl_sync(0xffffffffu, ci, j);
          if (lane == rj) { sel_v = vj; sel_i = ij; }
        }
        taken = 0u;
        for (int j = 0; j < k; ++j) {
          const int e = __shfl_sync(0xffffffffu, sel_i, j);
          if ((e & 31) == lane) taken |= 1u << (e >> 5);
        }
      } else {
        kth = warp_topk<EPL>(z, E, k, sel_v, sel_i, taken);
      }
    }
    if (logits_out != nullptr) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i < E) logits_out[(size_t)t * E + lane + 32 * i] = z[i];
    }
    // softmax (the largest logit is the first pick)
    const float m = __shfl_sync(0xffffffffu, sel_v, 0);
    float ssum = 0.f;
    float ez[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      ez[i] = (lane + 32 * i < E) ? __expf(z[i] - m) : 0.f;
      ssum += ez[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    const float inv = 1.f / ssum;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        if (STATS) {
          s_p[e] += ez[i] * inv;
          if ((taken >> i) & 1u) s_c[e] += 1;
        } else if (p_out != nullptr) {   // for the chunk probability sums, when they are wanted
          p_out[(size_t)t * E + e] = ez[i] * inv;
        }
      }
    }
    const float pj = lane < k ? __expf(sel_v - m) * inv : 0.f;
    float wsum = pj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (lane < k) {
      topk_idx[(size_t)t * k + lane] = sel_i;
      topk_w[(size_t)t * k + lane] = renorm ? pj / wsum : pj;
    }
  }
  if (!STATS) return;
  // chunk statistics: warps combined in fixed order
  __syncthreads();
  const int* s_c0 = reinterpret_cast<const int*>(s_stat + (size_t)NW * E);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float ps = 0.f;
    int cs = 0;
#pragma unroll 8
    for (int w = 0; w < NW; ++w) { ps += s_stat[(size_t)w * E + e]; cs += s_c0[(size_t)w * E + e]; }
    cnt[(size_t)e * nchunks + chunk] = cs;
    if (psum != nullptr) psum[(size_t)e * nchunks + chunk] = ps;
  }
}

// ---------------------------------------------------------------------------
// Certified selection over tensor-core screening logits, in three kernels that
// keep the exact fp32 work proportional to the candidates (about k + 0.1 per
// token) rather than to E:
//   k_router_select    one warp per token (lane l: experts l, l+32, ...): a
//                      lower bound L of the k-th largest screening logit,
//                      ||x_t|| for the error bound, the candidates
//                      (z >= L - 2 bound) in expert order, and the sum of
//                      exp(z - max) over the others; each candidate is listed
//                      under its expert;
//   k_router_recompute exact fp32 logits of the listed (token, expert) pairs,
//                      the flat list split evenly over the CTAs, W_r[e] in
//                      shared memory;
//   k_router_finish    top k among each token's exact candidates, softmax
//                      (exact candidates + screening rest), gates, picks per
//                      (expert, chunk).
// The decision equals the top k of exact fp32 logits: an expert outside the
// candidates has z < L - 2 bound <= (k-th screening value) - 2 bound, so its
// exact logit is below those of the k experts whose screening value reaches
// the k-th.
constexpr int kSelMaxD = 2048;      // largest input width of the selection path

struct SelectArgs {
  const float* zs;       // [T, E] screening logits (bias included)
  const float* xnorm2;   // [T] sum of x_t^2
  const __nv_bfloat16* x;
  const float* wnorm;    // [E] ||W_r[e]||_2
  float gamma;           // |screen - exact| <= gamma ||x_t|| max_e ||w_e||
  int T, d, E, k;
  uint8_t* cidx;         // [T][kSelMaxCand] candidate experts, expert order
  int32_t* ncand;        // [T] candidates (all of them)
  float* zmax;           // [T] largest screening logit
  float* snc;            // [T] sum over non-candidates of exp(z - zmax)
  int32_t* ecount;       // [E] list lengths (zero before k_router_select)
  int32_t* elist;        // [E][T] list entries t * kSelMaxCand + slot (a token at most once per expert)
  int32_t* cnt;          // [E][nchunks] pick counts, cleared here for k_router_finish
};

// One CTA = one 32-token chunk = 8 warps x 4 tokens.  A candidate takes its
// position in its expert's list in two steps: a shared-memory counter per
// expert inside the chunk, then one global reservation per (chunk, expert) for
// the chunk's whole run.  The tokens of a warp are loaded together (screening
// row and inputs), then processed side by side.  A token keeps its first
// kSelMaxCand candidates; with more, the finishing kernel recomputes every
// expert for it.
template <int EPL>
__global__ void __launch_bounds__(256, EPL <= 6 ? 3 : 2) k_router_select(const SelectArgs a) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  constexpr int TPW = kChunk / 8;
  __shared__ int s_cnt[kMaxRouterE];
  __shared__ int s_base[kMaxRouterE];
  __shared__ uint32_t s_rec[kChunk][kSelMaxCand];   // expert << 16 | index inside the chunk's run
  __shared__ int s_nk[kChunk];
  const int lane = lane_id(), warp = warp_id();
  const int chunk = blockIdx.x, nchunks = (a.T + kChunk - 1) / kChunk;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    s_cnt[e] = 0;
    a.cnt[(size_t)e * nchunks + chunk] = 0;
  }
  float wmax = 0.f;
  for (int e = lane; e < a.E; e += 32) wmax = fmaxf(wmax, a.wnorm[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  // screening rows and input norms of the warp's tokens, loads issued together
  float z[TPW][EPL];
  float x2s[TPW];
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt) {
    const int t = chunk * kChunk + warp * TPW + tt;
    const bool on = t < a.T;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      z[tt][i] = (on && e < a.E) ? a.zs[(size_t)t * a.E + e] : -INFINITY;
    }
    x2s[tt] = on ? a.xnorm2[t] : 0.f;
  }
  // A lower bound of each token's k-th largest screening value, the warp's tokens side by side: the k-th
  // largest of the 32 lane maxima (k lanes hold a maximum >= it, so at least k entries are >= it).  Rounds of
  // (warp maximum of the lane maxima, how many lanes hold it); the bound is the maximum of the round at which
  // the running count reaches k, and each earlier round retires its lanes.  Round 0's maximum is the token's
  // largest screening value.  Thresholding at this bound lists every expert the exact k-th value would, and
  // more only when two of a token's k largest share a lane.
  float lm[TPW], kth[TPW], m_s[TPW];
  int need[TPW];
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt) {
    float v = z[tt][0];
#pragma unroll
    for (int i = 1; i < EPL; ++i) v = fmaxf(v, z[tt][i]);
    lm[tt] = v;
    need[tt] = a.k;
    kth[tt] = -INFINITY;
  }
  for (int r = 0; r < a.k; ++r) {
    bool open = false;
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      float m;
      asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(lm[tt]));
      if (r == 0) m_s[tt] = m;
      const bool at = lm[tt] == m;
      const int c = __popc(__ballot_sync(0xffffffffu, at));
      if (need[tt] > 0) {
        if (c >= need[tt]) {
          kth[tt] = m;
          need[tt] = 0;
        } else {
          need[tt] -= c;
          if (at) lm[tt] = -INFINITY;
        }
      }
      open |= need[tt] > 0;
    }
    if (!open) break;   // warp-uniform
  }
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt) {
    const int tl = warp * TPW + tt;
    const int t = chunk * kChunk + tl;
    if (t >= a.T) {
      if (lane == 0) s_nk[tl] = 0;
      continue;
    }
    const float bound = a.gamma * sqrtf(x2s[tt]) * 1.001f * wmax * 1.001f + 1e-6f * (fabsf(kth[tt]) + 1.f);
    const float thr = kth[tt] - 2.f * bound;
    int nbefore = 0;      // candidates in earlier expert groups (warp-uniform)
    float snc = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      const bool cand = e < a.E && z[tt][i] >= thr;
      const unsigned m = __ballot_sync(0xffffffffu, cand);
      // non-candidates (experts past E hold -inf: their term is +0)
      snc += cand ? 0.f : __expf(z[tt][i] - m_s[tt]);
      if (cand) {
        const int slot = nbefore + __popc(m & lt);
        if (slot < kSelMaxCand) {
          a.cidx[(size_t)t * kSelMaxCand + slot] = (uint8_t)e;
          const int li = atomicAdd(&s_cnt[e], 1);
          s_rec[tl][slot] = ((uint32_t)e << 16) | (uint32_t)li;
        }
      }
      nbefore += __popc(m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) snc += __shfl_xor_sync(0xffffffffu, snc, o);
    if (lane == 0) {
      a.ncand[t] = nbefore;
      a.zmax[t] = m_s[tt];
      a.snc[t] = snc;
      s_nk[tl] = min(nbefore, kSelMaxCand);
    }
  }
  __syncthreads();
  // one reservation per expert for the chunk's run (all issued together), then the list entries
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    if (s_cnt[e] > 0) s_base[e] = atomicAdd(&a.ecount[e], s_cnt[e]);
  __syncthreads();
  for (int i = threadIdx.x; i < kChunk * kSelMaxCand; i += blockDim.x) {
    const int tl = i / kSelMaxCand, slot = i % kSelMaxCand;
    if (slot < s_nk[tl]) {
      const uint32_t r = s_rec[tl][slot];
      const int e = (int)(r >> 16);
      a.elist[(size_t)e * a.T + s_base[e] + (int)(r & 0xFFFFu)] =
          (int32_t)((chunk * kChunk + tl) * kSelMaxCand + slot);
    }
  }
}

// Exact fp32 logits of the listed (token, expert) pairs, expert-major.  A work
// item is a slice of kRecompSlice consecutive entries of one expert's list
// (popular experts give many items, so the load stays balanced whatever the
// routing skew) and belongs to one warp: warp g of the grid takes items g,
// g + (warps in the grid), ...  The warps run independently (no CTA barrier).
// Per item the warp holds the lane's slices of the expert's W_r row in
// registers, then computes NB entries at a time with all their input-row loads
// in flight together: lane l takes the 8-input slices l, l+32, ..., one fmaf
// chain, a fixed xor tree, then the bias -- the same value for a (token,
// expert) pair whichever warp computes it, and the same as warp_dot.
// zex[t][slot] = exact logit.
constexpr int kRecompSlice = 16;
// VPL: 16-byte input slices per lane (d <= 256 VPL); NB: entries per batch; MINB: resident CTAs per SM.
template <int VPL, int NB, int MINB>
__global__ void __launch_bounds__(256, MINB) k_router_recompute(const __nv_bfloat16* __restrict__ x,
                                                                const float* __restrict__ W,
                                                                const float* __restrict__ bias,
                                                                const int32_t* __restrict__ ecount,
                                                                const int32_t* __restrict__ elist,
                                                                float* __restrict__ zex, int T, int d, int E) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  static_assert(NB <= kRecompSlice && kRecompSlice <= 32, "one lane per entry of an item");
  __shared__ int s_ipre[kMaxRouterE + 1];   // items of experts < e
  const int lane = lane_id();
  if (warp_id() == 0) {
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += (ecount[e] + kRecompSlice - 1) / kRecompSlice;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int e = e0; e < e1; ++e) {
      s_ipre[e] = run;
      run += (ecount[e] + kRecompSlice - 1) / kRecompSlice;
    }
    if (lane == 31) s_ipre[E] = incl;
  }
  __syncthreads();
  const int nitems = s_ipre[E];
  const int nv = d >> 3;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int item = blockIdx.x * (blockDim.x >> 5) + warp_id(); item < nitems; item += nwarps) {
    int lo = 0, hi = E - 1;   // the item's expert: last e with s_ipre[e] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_ipre[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int a0 = (item - s_ipre[e]) * kRecompSlice;
    const int n = min(kRecompSlice, ecount[e] - a0);
    const int my_ent = lane < n ? elist[(size_t)e * T + a0 + lane] : 0;
    // this lane's slices of W_r[e]: inputs 8v .. 8v + 7 for v = lane + 32 q
    float4 w[VPL][2];
    const float4* wr = reinterpret_cast<const float4*>(W + (size_t)e * d);
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int v = lane + 32 * q;
      w[q][0] = v < nv ? __ldg(wr + 2 * v) : make_float4(0.f, 0.f, 0.f, 0.f);
      w[q][1] = v < nv ? __ldg(wr + 2 * v + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float be = bias != nullptr ? bias[e] : 0.f;
    for (int b0 = 0; b0 < n; b0 += NB) {
      int ent[NB];
      uint4 u[VPL][NB];
#pragma unroll
      for (int j = 0; j < NB; ++j) ent[j] = __shfl_sync(0xffffffffu, my_ent, min(b0 + j, n - 1));
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        const int v = lane + 32 * q;
#pragma unroll
        for (int j = 0; j < NB; ++j)
          u[q][j] = v < nv ? reinterpret_cast<const uint4*>(x + (size_t)(ent[j] / kSelMaxCand) * d)[v]
                           : make_uint4(0, 0, 0, 0);
      }
      float acc[NB];
#pragma unroll
      for (int j = 0; j < NB; ++j) acc[j] = 0.f;
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        if (lane + 32 * q < nv) {   // the slices warp_dot visits, in its order
          const float4 w0 = w[q][0], w1 = w[q][1];
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            float s2 = acc[j];
            s2 = fmaf(bf16lo(u[q][j].x), w0.x, s2); s2 = fmaf(bf16hi(u[q][j].x), w0.y, s2);
            s2 = fmaf(bf16lo(u[q][j].y), w0.z, s2); s2 = fmaf(bf16hi(u[q][j].y), w0.w, s2);
            s2 = fmaf(bf16lo(u[q][j].z), w1.x, s2); s2 = fmaf(bf16hi(u[q][j].z), w1.y, s2);
            s2 = fmaf(bf16lo(u[q][j].w), w1.z, s2); s2 = fmaf(bf16hi(u[q][j].w), w1.w, s2);
            acc[j] = s2;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NB; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
      }
      if (lane < NB) {
        float mine = acc[0];
        int me = ent[0];
#pragma unroll
        for (int j = 1; j < NB; ++j)
          if (lane == j) { mine = acc[j]; me = ent[j]; }
        if (b0 + lane < n) zex[me] = mine + be;
      }
    }
  }
}

// Top k of one token from exact fp32 logits of every expert (lane l: experts
// l, l+32, ...), for tokens with too many selection candidates.  Returns the
// softmax denominator; m receives the largest logit.  Kept out of line: the
// path is rare and must not weigh on the common one's registers.
template <int EPL>
__device__ __noinline__ float select_all_exact(const __nv_bfloat16* __restrict__ xr, const float* __restrict__ W,
                                               const float* __restrict__ bias, int d, int E, int k, float& sel_v,
                                               int& sel_i, float& m) {
  const int lane = lane_id();
  float z[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) z[i] = -INFINITY;
  for (int e = 0; e < E; ++e) {
    float v = warp_dot(xr, W + (size_t)e * d, d);
    if (bias != nullptr) v += bias[e];
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (e == lane + 32 * i) z[i] = v;
  }
  unsigned taken;
  warp_topk<EPL>(z, E, k, sel_v, sel_i, taken);
  m = __shfl_sync(0xffffffffu, sel_v, 0);
  float ez = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) ez += (lane + 32 * i < E) ? __expf(z[i] - m) : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ez += __shfl_xor_sync(0xffffffffu, ez, o);
  return ez;
}

// Selection finish, one warp per four tokens (8 warps per CTA).  Lane c holds candidate c
// (exact logit, expert); the top k among them by (value desc, index asc) --
// certified to be the top k of all experts -- come from k rounds of warp
// argmax.  Softmax: m = the first pick's value, sum = snc * exp(m_s - m) + the
// candidates' exp(z - m), where snc is the selection's sum of exp(z_e - m_s)
// over the non-candidates (screening values).  A token with more than
// kSelMaxCand candidates (degenerate logits) is finished from exact logits of
// every expert.  cnt[e][chunk] += picks (integer atomics: order-free).
template <int EPL>
__global__ void __launch_bounds__(256) k_router_finish(const int32_t* __restrict__ ncand,
                                                       const uint8_t* __restrict__ cidx, const float* __restrict__ zex,
                                                       const float* __restrict__ zmax, const float* __restrict__ snc,
                                                       const __nv_bfloat16* __restrict__ x, const float* __restrict__ W,
                                                       const float* __restrict__ bias, int32_t* __restrict__ topk_idx,
                                                       float* __restrict__ topk_w, int32_t* __restrict__ cnt, int T,
                                                       int d, int E, int k, int renorm) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  constexpr int TPW = 4;   // tokens per warp, their loads issued together
  const int lane = lane_id();
  const int t0 = (blockIdx.x * 8 + warp_id()) * TPW;
  const int nchunks = (T + kChunk - 1) / kChunk;
  int nc[TPW], cx[TPW];
  float zx[TPW], ms[TPW], sn[TPW];
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt) {
    const int t = min(t0 + tt, T - 1);
    nc[tt] = ncand[t];
    zx[tt] = zex[(size_t)t * kSelMaxCand + lane];      // slots past the count are masked below
    cx[tt] = (int)cidx[(size_t)t * kSelMaxCand + lane];
    ms[tt] = zmax[t];
    sn[tt] = snc[t];
  }
#pragma unroll
  for (int tt = 0; tt < TPW; ++tt) {
    const int t = t0 + tt;
    if (t >= T) break;
    float sel_v = 0.f, m, ssum;
    int sel_i = 0;
    if (nc[tt] <= kSelMaxCand) {
      float cv = lane < nc[tt] ? zx[tt] : -INFINITY;
      const int ci = lane < nc[tt] ? cx[tt] : 0x7fffffff;
      const float cv0 = cv;
      for (int j = 0; j < k; ++j) {
        float bv = cv;
        int bi = ci;
        warp_argmax_redux(bv, bi);
        if (lane == j) { sel_v = bv; sel_i = bi; }
        if (ci == bi) cv = -INFINITY;    // taken (candidate ids are distinct)
      }
      m = __shfl_sync(0xffffffffu, sel_v, 0);
      float ez = lane < nc[tt] ? __expf(cv0 - m) : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ez += __shfl_xor_sync(0xffffffffu, ez, o);
      ssum = ez + sn[tt] * __expf(ms[tt] - m);
    } else {
      ssum = select_all_exact<EPL>(x + (size_t)t * d, W, bias, d, E, k, sel_v, sel_i, m);
    }
    const float inv = 1.f / ssum;
    const float pj = lane < k ? __expf(sel_v - m) * inv : 0.f;
    float wsum = pj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    if (lane < k) {
      topk_idx[(size_t)t * k + lane] = sel_i;
      topk_w[(size_t)t * k + lane] = renorm ? pj / wsum : pj;
      atomicAdd(&cnt[(size_t)sel_i * nchunks + t / kChunk], 1);
    }
  }
}

// W_r [E][d] fp32 (global) -> shared memory as [d][pitch] (column e of row c =
// W_r[e][c]; columns E..pitch-1 untouched).  Coalesced float4 reads, eight in
// flight per thread before the transposed stores.  d % 4 == 0.
__device__ __forceinline__ void load_wt_transposed(const float* __restrict__ W, int E, int d, float* s_wt, int pitch) {
  const int n4 = E * d / 4;
  const float4* W4 = reinterpret_cast<const float4*>(W);
  for (int base = threadIdx.x; base < n4; base += 8 * blockDim.x) {
    float4 r[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i4 = base + j * blockDim.x;
      r[j] = i4 < n4 ? __ldg(W4 + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i4 = base + j * blockDim.x;
      if (i4 < n4) {
        const int e = (4 * i4) / d, c = 4 * i4 - e * d;
        s_wt[(c + 0) * pitch + e] = r[j].x;
        s_wt[(c + 1) * pitch + e] = r[j].y;
        s_wt[(c + 2) * pitch + e] = r[j].z;
        s_wt[(c + 3) * pitch + e] = r[j].w;
      }
    }
  }
}

// Router fully in one kernel for few experts (E <= EC <= 16).  KP lanes share
// one token (32 / KP tokens per warp, 256 / KP per CTA): lane part q takes the
// input pairs (2w, 2w + 1) for w = q, q + KP, q + 2 KP, ... and keeps E fp32
// FMA chains over them in order; an xor tree over the KP lanes then gives
// every lane of the token its full logits.  W_r^T sits in shared memory as
// [d][EC + 4] fp32: the lanes of a token read rows 2 apart, which the padded
// pitch puts in different banks, and the tokens of a warp read the same rows
// (broadcast).  Top-k runs per token (k
// ascending scans with a strict >: the lowest index wins ties), then softmax
// and gates.  Chunk statistics: fixed xor trees over the warp's tokens, then
// the KP warps of a 32-token chunk in warp order through shared memory.
template <int EC, int KP>
__global__ void __launch_bounds__(256) k_router_lanes(const __nv_bfloat16* __restrict__ x,
                                                      const float* __restrict__ W, const float* __restrict__ bias,
                                                      float* __restrict__ logits_out, int32_t* __restrict__ topk_idx,
                                                      float* __restrict__ topk_w, int32_t* __restrict__ cnt,
                                                      float* __restrict__ psum, int T, int d, int E, int k,
                                                      int renorm) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ __align__(16) float s_wt[];  // [d][EC]
  __shared__ float s_ps[8][EC];
  __shared__ int s_cn[8][EC];
  constexpr int PW = EC + 4;   // row pitch (floats)
  load_wt_transposed(W, E, d, s_wt, PW);
  for (int i = threadIdx.x; i < (EC - E) * d; i += blockDim.x) {   // zero columns E..EC-1
    const int c = i / (EC - E), e = E + (i - c * (EC - E));
    s_wt[c * PW + e] = 0.f;
  }
  __syncthreads();
  constexpr int TPW = 32 / KP;                 // tokens per warp
  const int lane = lane_id(), warp = warp_id();
  const int q = lane % KP, tw = lane / KP;
  const int t = blockIdx.x * (8 * TPW) + warp * TPW + tw;
  const bool on = t < T;
  float z[EC];
#pragma unroll
  for (int e = 0; e < EC; ++e) z[e] = 0.f;
  const uint32_t* xw = reinterpret_cast<const uint32_t*>(x + (size_t)(on ? t : 0) * d);
  const int nw = d >> 1;
  // the lane's input pairs w = q, q + KP, ...: sixteen loads in flight, then their FMAs
  for (int w0 = q; w0 < nw; w0 += 16 * KP) {
    uint32_t ub[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int w = w0 + j * KP;
      ub[j] = (on && w < nw) ? __ldg(xw + w) : 0u;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      // past the input end the loaded word is 0 and row 0 is read instead: the FMAs add zeros
      const int w = w0 + j * KP < nw ? w0 + j * KP : 0;
      const float x0 = bf16lo(ub[j]), x1 = bf16hi(ub[j]);
      const float4* r0 = reinterpret_cast<const float4*>(s_wt + (size_t)(2 * w) * PW);
      const float4* r1 = reinterpret_cast<const float4*>(s_wt + (size_t)(2 * w + 1) * PW);
#pragma unroll
      for (int e4 = 0; e4 < EC / 4; ++e4) {
        const float4 a4 = r0[e4];
        z[4 * e4 + 0] = fmaf(x0, a4.x, z[4 * e4 + 0]);
        z[4 * e4 + 1] = fmaf(x0, a4.y, z[4 * e4 + 1]);
        z[4 * e4 + 2] = fmaf(x0, a4.z, z[4 * e4 + 2]);
        z[4 * e4 + 3] = fmaf(x0, a4.w, z[4 * e4 + 3]);
      }
#pragma unroll
      for (int e4 = 0; e4 < EC / 4; ++e4) {
        const float4 b4 = r1[e4];
        z[4 * e4 + 0] = fmaf(x1, b4.x, z[4 * e4 + 0]);
        z[4 * e4 + 1] = fmaf(x1, b4.y, z[4 * e4 + 1]);
        z[4 * e4 + 2] = fmaf(x1, b4.z, z[4 * e4 + 2]);
        z[4 * e4 + 3] = fmaf(x1, b4.w, z[4 * e4 + 3]);
      }
    }
  }
#pragma unroll
  for (int o = 1; o < KP; o <<= 1)
#pragma unroll
    for (int e = 0; e < EC; ++e) z[e] += __shfl_xor_sync(0xffffffffu, z[e], o);
  const bool lead = on && q == 0;   // the lane that writes the token's outputs
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < EC; ++e) {
    if (e < E) {
      if (bias != nullptr) z[e] += bias[e];
      m = fmaxf(m, z[e]);
    } else {
      z[e] = -INFINITY;
    }
  }
  if (lead && logits_out != nullptr)
    for (int e = 0; e < E; ++e) logits_out[(size_t)t * E + e] = z[e];
  // softmax
  float ez[EC], ssum = 0.f;
#pragma unroll
  for (int e = 0; e < EC; ++e) {
    ez[e] = e < E ? expf(z[e] - m) : 0.f;
    ssum += ez[e];
  }
  const float inv = 1.f / ssum;
  // top-k: k scans in ascending index with a strict >, the picked entries masked
  uint32_t taken = 0u;
  float wsum = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = 0.f;
    int bi = -1;
#pragma unroll
    for (int e = 0; e < EC; ++e)
      if (e < E && !((taken >> e) & 1u) && (bi < 0 || z[e] > bv)) {
        bv = z[e];
        bi = e;
      }
    taken |= 1u << bi;
    float pj = 0.f;
#pragma unroll
    for (int e = 0; e < EC; ++e)
      if (e == bi) pj = ez[e] * inv;
    wsum += pj;
    if (lead) {
      topk_idx[(size_t)t * k + j] = bi;
      topk_w[(size_t)t * k + j] = pj;
    }
  }
  if (lead && renorm) {
    const float r = 1.f / wsum;
    for (int j = 0; j < k; ++j) topk_w[(size_t)t * k + j] *= r;
  }
  // chunk statistics: this warp's tokens (one lane each), then the chunk's KP warps in order
#pragma unroll
  for (int e = 0; e < EC; ++e) {
    if (e >= E) break;
    float pe = lead ? ez[e] * inv : 0.f;
#pragma unroll
    for (int o = KP; o < 32; o <<= 1) pe += __shfl_xor_sync(0xffffffffu, pe, o);
    const int ce = __popc(__ballot_sync(0xffffffffu, lead && ((taken >> e) & 1u)));
    if (lane == 0) {
      s_ps[warp][e] = pe;
      s_cn[warp][e] = ce;
    }
  }
  __syncthreads();
  const int nchunks = (T + kChunk - 1) / kChunk;
  constexpr int CPB = 8 / KP;                 // chunks per CTA
  for (int i = threadIdx.x; i < CPB * E; i += blockDim.x) {
    const int cl = i / E, e = i - cl * E;
    const int chunk = blockIdx.x * CPB + cl;
    if (chunk >= nchunks) continue;
    float ps = 0.f;
    int cs = 0;
#pragma unroll
    for (int w = 0; w < KP; ++w) {
      ps += s_ps[cl * KP + w][e];
      cs += s_cn[cl * KP + w][e];
    }
    if (psum != nullptr) psum[(size_t)e * nchunks + chunk] = ps;
    cnt[(size_t)e * nchunks + chunk] = cs;
  }
}

// Router fully in one kernel for small E * d: the CTA keeps W_r^T in shared
// memory ([d][32 EPL + 1] fp32, padded against bank conflicts); each warp
// computes its tokens' logits as plain fp32 FMA chains over the inputs (lane l
// owns experts l, l+32, ...), then softmax / top-k / gates as above.  A token's
// row is read once, 16 bytes per lane, and its values are broadcast by
// shuffles; the next token's row is prefetched.
template <int EPL, int NW>
__global__ void __launch_bounds__(NW * 32) k_router_fused(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ W, const float* __restrict__ bias,
                                                          float* __restrict__ logits_out,
                                                          int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                          int32_t* __restrict__ cnt, float* __restrict__ psum, int T,
                                                          int d, int E, int k, int renorm) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ float s_wt[];
  __shared__ float s_p[NW][EPL * 32];
  __shared__ int s_c[NW][EPL * 32];
  constexpr int EP = EPL * 32 + 1;
  load_wt_transposed(W, E, d, s_wt, EP);   // odd row pitch: no bank conflicts in the compute loop
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
  constexpr int TPW = (kChunk + NW - 1) / NW;  // tokens per warp
  const int t_first = chunk * kChunk + warp * TPW;
  const int t_end = min(T, t_first + TPW);
  const int nv = d >> 3;
  uint4 nxt = make_uint4(0, 0, 0, 0);
  if (t_first < t_end && lane < nv) nxt = reinterpret_cast<const uint4*>(x + (size_t)t_first * d)[lane];
  for (int t = t_first; t < t_end; ++t) {
    float acc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
    for (int v0 = 0; v0 < nv; v0 += 32) {
      const uint4 u = nxt;
      // prefetch: the next 256-input slice of this token, or the first slice of the next token
      if (v0 + 32 < nv) {
        nxt = (v0 + 32 + lane < nv) ? reinterpret_cast<const uint4*>(x + (size_t)t * d)[v0 + 32 + lane]
                                    : make_uint4(0, 0, 0, 0);
      } else if (t + 1 < t_end) {
        nxt = lane < nv ? reinterpret_cast<const uint4*>(x + (size_t)(t + 1) * d)[lane] : make_uint4(0, 0, 0, 0);
      }
      const int nl = min(32, nv - v0);
      for (int sl = 0; sl < nl; ++sl) {
        const uint32_t w0 = __shfl_sync(0xffffffffu, u.x, sl), w1 = __shfl_sync(0xffffffffu, u.y, sl);
        const uint32_t w2 = __shfl_sync(0xffffffffu, u.z, sl), w3 = __shfl_sync(0xffffffffu, u.w, sl);
        const float xv[8] = {bf16lo(w0), bf16hi(w0), bf16lo(w1), bf16hi(w1),
                             bf16lo(w2), bf16hi(w2), bf16lo(w3), bf16hi(w3)};
        const float* wr = s_wt + (size_t)((v0 + sl) * 8) * EP + lane;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
#pragma unroll
          for (int i = 0; i < EPL; ++i) acc[i] = fmaf(xv[q], wr[q * EP + 32 * i], acc[i]);
        }
      }
    }
    float z[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) z[i] = (lane + 32 * i < E) ? acc[i] + b[i] : -INFINITY;
    route_token<EPL>(z, t, E, k, renorm, logits_out, topk_idx, topk_w, pacc, cacc);
  }
  // chunk statistics: warps combined in fixed order
#pragma unroll
  for (int i = 0; i < EPL; ++i) { s_p[warp][lane + 32 * i] = pacc[i]; s_c[warp][lane + 32 * i] = cacc[i]; }
  __syncthreads();
  const int nchunks = (T + kChunk - 1) / kChunk;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float ps = 0.f;
    int cs = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) { ps += s_p[w][e]; cs += s_c[w][e]; }
    cnt[(size_t)e * nchunks + chunk] = cs;
    if (psum != nullptr) psum[(size_t)e * nchunks + chunk] = ps;
  }
}

// Router logits for small T (decode), exact fp32: W_r is the large operand and
// is streamed from HBM once (later token blocks re-read it from L2).
//   Grid: (ceil(E / 32), ceil(T / kSkTok), kSkSplit) with clusters of
//   kSkSplit CTAs along the inputs.  A CTA stages its kSkTok tokens x ks-input
//   slice of x in shared memory as fp32; each of its 8 warps owns 4 experts, and
//   lane l takes inputs 4l .. 4l+3 of every 128-input step: per step 4
//   coalesced float4 loads of W_r rows and kSkTok broadcast-free float4 reads
//   of x feed 16 kSkTok FMAs (one fp32 chain per (expert, token) per lane,
//   inputs in order), the W_r rows of the next three steps in flight.
//   The 4 kSkTok chains of a warp are combined across lanes by a transposing
//   xor tree, the kSkSplit partial tiles in cluster rank order through
//   distributed shared memory.  Logits are written without bias.
constexpr int kSkSplit = 4;
constexpr int kSkTok = 8;
constexpr int kSkExp = 4;   // experts per warp
static_assert(kSkTok == 2 * kSkSplit, "each rank of the cluster finishes two tokens");

__host__ __device__ constexpr int skinny_slice(int d) {
  return ((d + 128 * kSkSplit - 1) / (128 * kSkSplit)) * 128;   // inputs per split, a multiple of 128
}

__global__ void __cluster_dims__(1, 1, kSkSplit) __launch_bounds__(256, 2) k_router_skinny(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ W, float* __restrict__ logits,
                                                          int T, int d, int E) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ __align__(16) float s_x[];      // [kSkTok][ks]
  __shared__ float s_tile[kSkTok][8 * kSkExp];      // this CTA's partial [token][expert]
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int lane = lane_id(), warp = warp_id();
  const int ks = skinny_slice(d);
  const int k0 = rank * ks;
  const int kn = max(0, min(ks, d - k0));
  const int t0 = blockIdx.y * kSkTok;
  const int nt = min(kSkTok, T - t0);
  const int eb = blockIdx.x * 8 * kSkExp;
  // stage x (zeros for absent tokens and past the slice end)
  const int nv = ks >> 3;
  for (int i = threadIdx.x; i < kSkTok * nv; i += blockDim.x) {
    const int t = i / nv, v = i - t * nv;
    float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
    if (t < nt && 8 * v < kn) {
      const uint4 u = *reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d + k0 + 8 * v);
      lo = make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
      hi = make_float4(bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w));
    }
    float4* dst = reinterpret_cast<float4*>(s_x + (size_t)t * ks + 8 * v);
    dst[0] = lo;
    dst[1] = hi;
  }
  __syncthreads();
  float acc[kSkExp * kSkTok];
#pragma unroll
  for (int j = 0; j < kSkExp * kSkTok; ++j) acc[j] = 0.f;
  const int e_first = eb + warp * kSkExp;
  const int n_e = max(0, min(kSkExp, E - e_first));   // experts of this warp that exist
  const float* wbase = W + (size_t)(n_e > 0 ? e_first : 0) * d + k0 + 4 * lane;
  const int nsteps = (kn + 127) >> 7;
  auto load_w = [&](int st, int q) -> float4 {
    return (q < n_e && st < nsteps && st * 128 + 4 * lane < kn)
               ? __ldg(reinterpret_cast<const float4*>(wbase + (size_t)q * d + st * 128))
               : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  // the rows of the next three steps are in flight during a step's FMAs
  float4 w1[kSkExp], w2[kSkExp], w3[kSkExp];
#pragma unroll
  for (int q = 0; q < kSkExp; ++q) {
    w1[q] = load_w(0, q);
    w2[q] = load_w(1, q);
    w3[q] = load_w(2, q);
  }
  for (int st = 0; st < nsteps; ++st) {
    float4 w[kSkExp];
#pragma unroll
    for (int q = 0; q < kSkExp; ++q) {
      w[q] = w1[q];
      w1[q] = w2[q];
      w2[q] = w3[q];
      w3[q] = load_w(st + 3, q);
    }
#pragma unroll
    for (int t = 0; t < kSkTok; ++t) {
      const float4 xv = reinterpret_cast<const float4*>(s_x + (size_t)t * ks + st * 128)[lane];
#pragma unroll
      for (int q = 0; q < kSkExp; ++q) {
        float& a = acc[q * kSkTok + t];
        a = fmaf(xv.x, w[q].x, a);
        a = fmaf(xv.y, w[q].y, a);
        a = fmaf(xv.z, w[q].z, a);
        a = fmaf(xv.w, w[q].w, a);
      }
    }
  }
  // transposing xor tree: at offset o the lane keeps the half of its entries
  // selected by lane bit o and adds the partner's copy of that half
#pragma unroll
  for (int o = 16, n = kSkExp * kSkTok; o >= 1; o >>= 1, n >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = up ? acc[j] : acc[j + n / 2];
      const float keep = up ? acc[j + n / 2] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  // lane l holds entries EL l .. EL l + EL - 1 of (expert q, token t) = (idx / kSkTok, idx % kSkTok)
  constexpr int EL = kSkExp * kSkTok / 32;
#pragma unroll
  for (int j = 0; j < EL; ++j) {
    const int idx = EL * lane + j;
    s_tile[idx % kSkTok][warp * kSkExp + idx / kSkTok] = acc[j];
  }
  cluster.sync();
  // rank r finishes tokens 2r, 2r + 1 of the block (kSkTok / kSkSplit = 2) for the CTA's 32 experts
  if (threadIdx.x < 64) {
    const int tl = rank * 2 + (threadIdx.x >> 5), el = threadIdx.x & 31;
    float v = 0.f;
#pragma unroll
    for (int r = 0; r < kSkSplit; ++r) v += cluster.map_shared_rank(&s_tile[0][0], r)[tl * 32 + el];
    if (tl < nt && eb + el < E) logits[(size_t)(t0 + tl) * E + eb + el] = v;
  }
  cluster.sync();  // tiles stay alive until every CTA of the cluster has read them
}

// ---------------------------------------------------------------------------
// Per-chunk expert histogram from caller routing (moe_permute without moe_route).
__global__ void __launch_bounds__(256) k_chunk_hist(const int32_t* __restrict__ topk_idx, int32_t* __restrict__ cnt,
                                                    int T, int E, int k) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
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
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[(size_t)e * gridDim.x + blockIdx.x] = s_h[e];
}

// Chunk tables from per-token routing (small batches): one CTA per chunk of
// kChunk tokens.  cnt[e][c] by shared-memory integer counts (order-free),
// psum[e][c] = sum over the chunk's tokens, in token order, of p[t,e] (skipped
// when psum is null: no load-balance statistic requested).
__global__ void __launch_bounds__(256) k_chunk_stats(const int32_t* __restrict__ topk_idx,
                                                     const float* __restrict__ p, int32_t* __restrict__ cnt,
                                                     float* __restrict__ psum, int T, int E, int k) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ int s_h[kMaxRouterE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_h[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kChunk;
  const int nt = min(kChunk, T - t0);
  for (int i = threadIdx.x; i < nt * k; i += blockDim.x) atomicAdd(&s_h[topk_idx[(size_t)t0 * k + i]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    cnt[(size_t)e * gridDim.x + blockIdx.x] = s_h[e];
    if (psum != nullptr) {
      float ps = 0.f;
      for (int t = 0; t < nt; ++t) ps += p[(size_t)(t0 + t) * E + e];
      psum[(size_t)e * gridDim.x + blockIdx.x] = ps;
    }
  }
}

// ---------------------------------------------------------------------------
// Chunk tables are expert-major: cnt[e][c], psum[e][c].  One CTA of 8 warps per
// expert, each warp owning a contiguous run of 32-chunk rows:
// cnt[e][c] -> exclusive prefix over chunks (in place), counts[e]; optional
// f[e] = counts/T and P[e] = sum_c psum[e][c] / T (per lane in chunk order, a
// fixed xor tree per warp, then the warps in order).
__global__ void __launch_bounds__(256) k_chunk_scan(int32_t* __restrict__ cnt, const float* __restrict__ psum,
                                                    int32_t* __restrict__ counts, float* __restrict__ f_out,
                                                    float* __restrict__ p_out, int nchunks, int E, int T) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ int s_tot[8];
  __shared__ float s_ps[8];
  const int e = blockIdx.x;
  const int lane = lane_id(), warp = warp_id();
  int32_t* row = cnt + (size_t)e * nchunks;
  const float* prow = psum != nullptr ? psum + (size_t)e * nchunks : nullptr;
  const int nrows = (nchunks + 31) / 32;
  const int rpw = (nrows + 7) / 8;
  const int r0 = min(nrows, warp * rpw), r1 = min(nrows, r0 + rpw);
  // pass 1: this warp's total and probability sum (loads of all its rows in flight together)
  int wt = 0;
  float ps = 0.f;
  for (int r = r0; r < r1; ++r) {
    const int c = r * 32 + lane;
    if (c < nchunks) {
      wt += row[c];
      if (prow != nullptr) ps += prow[c];
    }
  }
  wt = (int)__reduce_add_sync(0xffffffffu, (unsigned)wt);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
  if (lane == 0) {
    s_tot[warp] = wt;
    s_ps[warp] = ps;
  }
  __syncthreads();
  int run = 0;
  for (int w = 0; w < warp; ++w) run += s_tot[w];
  // pass 2: exclusive scan of the warp's rows (re-read from cache), offset by the earlier warps
  for (int r = r0; r < r1; ++r) {
    const int c = r * 32 + lane;
    const int v = c < nchunks ? row[c] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (c < nchunks) row[c] = run + incl - v;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (threadIdx.x == 0) {
    int total = 0;
    float pt = 0.f;
    for (int w = 0; w < 8; ++w) {
      total += s_tot[w];
      pt += s_ps[w];
    }
    if (counts != nullptr) counts[e] = total;
    if (f_out != nullptr) f_out[e] = (float)total / (float)T;
    if (p_out != nullptr && prow != nullptr) p_out[e] = pt / (float)T;
  }
}

__global__ void k_aux_finalize(const float* __restrict__ f, const float* __restrict__ P, float* __restrict__ aux,
                               int E) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  float s = 0.f;
  for (int e = lane_id(); e < E; e += 32) s += f[e] * P[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane_id() == 0) *aux = (float)E * s;
}

}  // namespace moe
