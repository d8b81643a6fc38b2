// Input gradient of the layer (bf16 experts).  Training is the setting of the
// kieve-moe Features (load-balancing auxiliary loss), the MoEEvolve README
// (Architecture) and MoEFFN.forward in moe_stream.py ("Load balancing loss").
// For L = sum(dout * out) + aux_coef * aux the chain rule gives, per token t:
//   dx_t = sum over kept slots j of  w_tj * J_e(x_t)^T dout_t      (routed experts)
//        + J_shared(x_t)^T dout_t                                  (shared expert)
//        + W_r^T dz_t                                              (router)
// with the expert input gradient J^T dy = (dh u act'(g)) W1 + (dh act(g)) W3,
// dh = dy W2, and the router part: dw_tj = <dout_t, y_e(x_t)> on kept slots,
// the gate derivative (renormalised gates: (dw_j - sum_i dw_i w_i) / S), the
// statistic aux = E sum_e f_e P_e (d/dp = E f_e / T per expert, counts fixed),
// then the softmax: dz = p (dp - <p, dp>).  The routing decision passes no
// gradient.  Per routed row three GEMMs run on k_grouped_gemm: the recomputed
// [g | u] = x W13^T, dh' = dout W2 (unscaled; dh = w dh') and dx = [dg | du] W13
// (transposed weights).  The gate gradient needs no h or y: <dout, y> equals
// <act(g) u, dh'>.  The kernels here are the elementwise and gather steps.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace moe {

// wt[n][c][r] = w[n][r][c] (bf16), 32 x 32 tiles through shared memory.  Grid (ceil(cols/32),
// ceil(rows/32), n), block (32, 8).
__global__ void __launch_bounds__(256) k_transpose_bf16(const __nv_bfloat16* __restrict__ w,
                                                        __nv_bfloat16* __restrict__ wt, int rows, int cols) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ __nv_bfloat16 tile[32][34];
  const size_t base = (size_t)blockIdx.z * rows * cols;
  const int c = blockIdx.x * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = blockIdx.y * 32 + i;
    if (r < rows && c < cols) tile[i][threadIdx.x] = w[base + (size_t)r * cols + c];
  }
  __syncthreads();
  const int r = blockIdx.y * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int cc = blockIdx.x * 32 + i;
    if (cc < cols && r < rows) wt[base + (size_t)cc * rows + r] = tile[threadIdx.x][i];
  }
}

// W_r [E][d] fp32 -> W_r^T [d][ldE] bf16 (the B operand of dx_router = dz W_r), zeros in columns E .. ldE.
// Same tiling, grid (ceil(d/32), ceil(ldE/32)).
__global__ void __launch_bounds__(256) k_transpose_router(const float* __restrict__ w, __nv_bfloat16* __restrict__ wt,
                                                          int E, int d, int ldE) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ float tile[32][33];
  const int c = blockIdx.x * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int e = blockIdx.y * 32 + i;
    tile[i][threadIdx.x] = (e < E && c < d) ? w[(size_t)e * d + c] : 0.f;
  }
  __syncthreads();
  const int e = blockIdx.y * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int cc = blockIdx.x * 32 + i;
    if (cc < d && e < ldE) wt[(size_t)cc * ldE + e] = __float2bfloat16_rn(e < E ? tile[threadIdx.x][i] : 0.f);
  }
}

// d/dz of the activations: SiLU' = s (1 + z (1 - s)); GELU' = Phi(z) + z phi(z) (erf by Abramowitz & Stegun
// 7.1.26, as in the forward epilogue).
__device__ __forceinline__ float act_silu_grad(float z) {
  const float s = __fdividef(1.0f, 1.0f + __expf(-z));
  return s * (1.0f + z * (1.0f - s));
}
__device__ __forceinline__ float act_gelu_grad(float z) {
  return 0.5f * (1.0f + erf_as7126(z * 0.7071067811865476f)) + z * 0.3989422804014327f * __expf(-0.5f * z * z);
}

// GLU backward over rows of [g | u] (bf16 pre-activations, g in columns [0, H), u in [H, 2H)) and dh [., H]:
// in place, gu becomes [dg | du] with dg = dh u act'(g), du = dh act(g); with write_h, h = act(g) u (bf16)
// replaces dh.  One thread per 8 columns of a row.
template <int ACT>
__global__ void __launch_bounds__(256) k_glu_bwd(__nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ dh,
                                                 long long rows, int H, int write_h) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nv = H >> 3;
  if (i >= rows * nv) return;
  const long long r = i / nv;
  const int v = (int)(i - r * nv);
  uint4* g4 = reinterpret_cast<uint4*>(gu + r * 2 * H) + v;
  uint4* u4 = reinterpret_cast<uint4*>(gu + r * 2 * H + H) + v;
  uint4* d4 = reinterpret_cast<uint4*>(dh + r * H) + v;
  const uint4 G = *g4, U = *u4, D = *d4;
  const uint32_t gw[4] = {G.x, G.y, G.z, G.w}, uw[4] = {U.x, U.y, U.z, U.w}, dw[4] = {D.x, D.y, D.z, D.w};
  uint32_t og[4], ou[4], oh[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float dg[2], du[2], hh[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float g = h ? bf16hi(gw[q]) : bf16lo(gw[q]);
      const float u = h ? bf16hi(uw[q]) : bf16lo(uw[q]);
      const float d = h ? bf16hi(dw[q]) : bf16lo(dw[q]);
      const float a = ACT == kModeSwiGLU ? act_silu(g) : act_gelu(g);
      const float da = ACT == kModeSwiGLU ? act_silu_grad(g) : act_gelu_grad(g);
      dg[h] = d * u * da;
      du[h] = d * a;
      hh[h] = a * u;
    }
    og[q] = pack_bf16x2(dg[0], dg[1]);
    ou[q] = pack_bf16x2(du[0], du[1]);
    oh[q] = pack_bf16x2(hh[0], hh[1]);
  }
  *g4 = make_uint4(og[0], og[1], og[2], og[3]);
  *u4 = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  if (write_h) *d4 = make_uint4(oh[0], oh[1], oh[2], oh[3]);
}

// GLU backward of the routed rows with the gate gradients, one warp per (token, slot) i = t k + j with grouped row
// r = slot_pos[i]: from dh'_r = dout_t W2 (unscaled, bf16) and [g | u]_r, dw_tj = <act(g) u, dh'_r>, which is
// <dout_t, y_e(x_t)> since y = (act(g) u) W2^T, so neither h nor y is recomputed; then dh = w_tj dh' and
// gu_r becomes [dh u act'(g) | dh act(g)] in place.  With write_wh, w_tj h (bf16, the B operand of the W2
// gradient dout^T (w h)) replaces dh'_r.  Dropped slots: dw_tj = 0.  Lanes take 8-column slices in order,
// then a fixed xor tree.
template <int ACT>
__global__ void __launch_bounds__(256) k_glu_bwd_slots(__nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ dhp,
                                                       const int32_t* __restrict__ slot_pos,
                                                       const float* __restrict__ topk_w, long long n_slots, int H,
                                                       int write_wh, float* __restrict__ dw) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long i = (long long)blockIdx.x * 8 + warp_id();
  if (i >= n_slots) return;
  const int lane = lane_id();
  const int row = slot_pos[i];
  if (row < 0) {
    if (lane == 0) dw[i] = 0.f;
    return;
  }
  const float wj = topk_w[i];
  const int nv = H >> 3;
  uint4* g4 = reinterpret_cast<uint4*>(gu + (size_t)row * 2 * H);
  uint4* u4 = g4 + nv;
  uint4* d4 = reinterpret_cast<uint4*>(dhp + (size_t)row * H);
  float acc = 0.f;
  for (int v = lane; v < nv; v += 32) {
    const uint4 G = g4[v], U = u4[v], D = d4[v];
    const uint32_t gw[4] = {G.x, G.y, G.z, G.w}, uw[4] = {U.x, U.y, U.z, U.w}, dv[4] = {D.x, D.y, D.z, D.w};
    uint32_t og[4], ou[4], oh[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float dg[2], du[2], wh[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float g = h ? bf16hi(gw[q]) : bf16lo(gw[q]);
        const float u = h ? bf16hi(uw[q]) : bf16lo(uw[q]);
        const float d = h ? bf16hi(dv[q]) : bf16lo(dv[q]);
        const float a = ACT == kModeSwiGLU ? act_silu(g) : act_gelu(g);
        const float da = ACT == kModeSwiGLU ? act_silu_grad(g) : act_gelu_grad(g);
        acc = fmaf(a * u, d, acc);
        const float dh = wj * d;
        dg[h] = dh * u * da;
        du[h] = dh * a;
        wh[h] = wj * a * u;
      }
      og[q] = pack_bf16x2(dg[0], dg[1]);
      ou[q] = pack_bf16x2(du[0], du[1]);
      oh[q] = pack_bf16x2(wh[0], wh[1]);
    }
    g4[v] = make_uint4(og[0], og[1], og[2], og[3]);
    u4[v] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
    if (write_wh) d4[v] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) dw[i] = acc;
}

// Router backward, one warp per token (lane l: experts l, l + 32, ...): p = softmax(z_t); dp on the selected
// experts from dw (renormalised gates: (dw_j - sum_i dw_i w_i) / S, S = sum of the selected p); plus
// aux_coef E counts_e / T^2 on every expert; dz = p (dp - <p, dp>), written as bf16 (the A operand of dz W_r)
// into rows of ldz >= E columns, zeros past E (the reduction of dz W_r runs over whole 64-column steps).
template <int EPL>
__global__ void __launch_bounds__(256) k_router_bwd(const float* __restrict__ z, const int32_t* __restrict__ topk_idx,
                                                    const float* __restrict__ topk_w, const float* __restrict__ dw,
                                                    const int32_t* __restrict__ counts, float aux_coef, int T, int E,
                                                    int k, int renorm, int ldz, __nv_bfloat16* __restrict__ dz) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long t = (long long)blockIdx.x * 8 + warp_id();
  if (t >= T) return;
  const int lane = lane_id();
  float p[EPL], dp[EPL];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    p[i] = e < E ? z[t * E + e] : -INFINITY;
    m = fmaxf(m, p[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    p[i] = (lane + 32 * i < E) ? __expf(p[i] - m) : 0.f;
    sum += p[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  const float auxs = aux_coef * (float)E / ((float)T * (float)T);
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    p[i] *= inv;
    dp[i] = (e < E && aux_coef != 0.f) ? auxs * (float)counts[e] : 0.f;
  }
  // gates: S and sum_i dw_i w_i over the token's k slots (the same on every lane)
  float S = 0.f, dwsum = 0.f;
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[t * k + j];
    float pj = 0.f;   // p of expert e, held by lane e % 32
#pragma unroll
    for (int i = 0; i < EPL; ++i) pj = (lane + 32 * i == e) ? p[i] : pj;
    pj = __shfl_sync(0xffffffffu, pj, e & 31);
    S += pj;
    dwsum += dw[t * k + j] * topk_w[t * k + j];
  }
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[t * k + j];
    const float dpsel = renorm ? (dw[t * k + j] - dwsum) / S : dw[t * k + j];
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (lane + 32 * i == e) dp[i] += dpsel;
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) s = fmaf(p[i], dp[i], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) dz[t * ldz + e] = __float2bfloat16_rn(p[i] * (dp[i] - s));
  }
  for (int e = E + lane; e < ldz; e += 32) dz[t * ldz + e] = __float2bfloat16_rn(0.f);
}

// dx_t = sum over kept slots of dx_perm[slot] + dx_shared_t (if any) + dx_router_t, fp32, one thread per 8
// columns (slot order, then the shared and router terms).
__global__ void __launch_bounds__(256) k_bwd_final(const __nv_bfloat16* __restrict__ dx_perm,
                                                   const int32_t* __restrict__ slot_pos,
                                                   const __nv_bfloat16* __restrict__ dx_shared,
                                                   const __nv_bfloat16* __restrict__ dx_router, int T, int d, int k,
                                                   float* __restrict__ dx) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const int nv = d >> 3;
  if (i >= (long long)T * nv) return;
  const long long t = i / nv;
  const int v = (int)(i - t * nv);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto add = [&](const __nv_bfloat16* row) {
    const uint4 a = reinterpret_cast<const uint4*>(row)[v];
    acc[0] += bf16lo(a.x); acc[1] += bf16hi(a.x); acc[2] += bf16lo(a.y); acc[3] += bf16hi(a.y);
    acc[4] += bf16lo(a.z); acc[5] += bf16hi(a.z); acc[6] += bf16lo(a.w); acc[7] += bf16hi(a.w);
  };
  for (int j = 0; j < k; ++j) {
    const int slot = slot_pos[t * k + j];
    if (slot >= 0) add(dx_perm + (size_t)slot * d);
  }
  if (dx_shared != nullptr) add(dx_shared + t * d);
  add(dx_router + t * d);
  float4* o = reinterpret_cast<float4*>(dx + t * d) + 2 * v;
  o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

}  // namespace moe
