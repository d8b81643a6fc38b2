// Grouping by expert with (token, slot) identity kept, and the weighted combine.
//
// Grouping: ExpertMesh README ("Activation grouping that preserves token and
// top-k slot identity"; flowchart "Group activations by expert owner"), with
// the MoEEvolve README's capacity-factor static-shape dispatch: group e holds
// rows [e*C, e*C + kept_e), overflow dropped in token order.  The rank of an
// assignment is the number of earlier tokens that chose the same expert,
// computed from per-chunk prefix sums and in-warp ballots, never from atomics
// whose order varies, so the layout is canonical and bit-reproducible.
//
// Combine: ExpertMesh flowchart "Weighted top-k reduction", moe_stream.py
// ``out[mask] += w * expert_out``, Kvasir ``combine(p, partials) + shared(cur)``.
#pragma once

#include "common.cuh"
#include "router.cuh"

namespace moe {

constexpr int kMaxE = 512;

// Block-wide exclusive scan of group sizes (blockDim.x == 128, E <= 512):
// s_off[e] = first row of group e, s_off[E] = total.  With cap > 0 the groups
// are fixed slabs of cap rows.
__device__ __forceinline__ void group_offsets(const int32_t* __restrict__ counts, int E, int cap, int* s_off,
                                              int* s_kept, int* s_tmp) {
  const int tid = threadIdx.x;
  const int per = (E + 127) / 128;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int local = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    const int kv = cap > 0 ? min(c, cap) : c;
    s_kept[e] = kv;
    local += cap > 0 ? cap : kv;
  }
  int incl = local;
  const int lane = lane_id(), warp = warp_id();
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_tmp[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += s_tmp[w];
  int run = wbase + incl - local;
  for (int e = e0; e < e1; ++e) {
    s_off[e] = run;
    run += cap > 0 ? cap : s_kept[e];
  }
  if (tid == 127) s_off[E] = wbase + incl;
  __syncthreads();
}

// One CTA = 128 threads = four chunks of 32 tokens, one warp per chunk.
// rank = (tokens of earlier chunks that chose e, from the per-chunk prefix
// table) + (earlier tokens of the chunk that chose e).  The in-chunk part
// walks the chunk's (token, slot) pairs in order, 32 / kp tokens per step
// (kp = k rounded up to a power of two, lane = token * kp + slot): lanes with
// the same expert find each other with match.any, take consecutive ranks from
// a per-warp shared counter, and the last of them advances the counter.
template <int KMAX>
__global__ void __launch_bounds__(128) k_scatter(const __nv_bfloat16* __restrict__ x,
                                                 const int32_t* __restrict__ topk_idx,
                                                 const int32_t* __restrict__ cbase, const int32_t* __restrict__ counts,
                                                 int T, int d, int E, int k, int cap, int32_t* __restrict__ slot_pos,
                                                 uint8_t* __restrict__ drop, int32_t* __restrict__ row_src,
                                                 __nv_bfloat16* __restrict__ x_perm, int32_t* __restrict__ kept_out,
                                                 int32_t* __restrict__ offsets_out, const float* __restrict__ aux_f,
                                                 const float* __restrict__ aux_p, float* __restrict__ aux_out) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_kept[kMaxE];
  __shared__ int s_tmp[4];
  __shared__ int s_cnt[4][kMaxE];
  // load-balance statistic of the routing this call groups: aux = E * sum_e f_e P_e (lanes in expert
  // order, then a fixed xor tree), folded in here so the forward needs no launch of its own for it
  if (aux_out != nullptr && blockIdx.x == 0 && threadIdx.x < 32) {
    float a = 0.f;
    for (int e = threadIdx.x; e < E; e += 32) a += aux_f[e] * aux_p[e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (threadIdx.x == 0) *aux_out = (float)E * a;
  }
  __shared__ int s_ix[4][kChunk * KMAX];
  __shared__ int s_rk[4][kChunk * KMAX];
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int chunk = blockIdx.x * 4 + warp;
  const int nchunks = (T + kChunk - 1) / kChunk;

  group_offsets(counts, E, cap, s_off, s_kept, s_tmp);
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += 128) {
      if (kept_out) kept_out[e] = s_kept[e];
      if (offsets_out) offsets_out[e] = s_off[e];
    }
    if (tid == 0 && offsets_out) offsets_out[E] = s_off[E];
  }
  if (chunk >= nchunks) return;

  const int t0 = chunk * kChunk;
  const int ntok = min(kChunk, T - t0);
  int* ix = s_ix[warp];
  int* rk = s_rk[warp];
  int* cnt = s_cnt[warp];
  for (int q = lane; q < ntok * k; q += 32) ix[q] = topk_idx[(size_t)t0 * k + q];
  __syncwarp();
  for (int q = lane; q < ntok * k; q += 32) cnt[ix[q]] = 0;
  __syncwarp();
  const int kp = k == 1 ? 1 : 1 << (32 - __clz(k - 1));
  const int lg = 31 - __clz(kp);
  const unsigned lt = (1u << lane) - 1u;
  for (int tb = 0; tb < ntok; tb += 32 / kp) {
    const int tt = tb + (lane >> lg), j = lane & (kp - 1);
    const bool on = j < k && tt < ntok;
    const int e = on ? ix[tt * k + j] : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int base = on ? cnt[e] : 0;
    __syncwarp();
    if (on) {
      rk[tt * k + j] = base + __popc(peers & lt);
      if (lane == 31 - __clz(peers)) cnt[e] = base + __popc(peers);
    }
    __syncwarp();
  }

  if (lane < ntok) {
    const int t = t0 + lane;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        const int e = ix[lane * k + j];
        const int rank = cbase[(size_t)e * nchunks + chunk] + rk[lane * k + j];
        const bool dropped = cap > 0 && rank >= cap;
        const int pos = dropped ? -1 : s_off[e] + rank;
        slot_pos[(size_t)t * k + j] = pos;
        if (drop) drop[(size_t)t * k + j] = dropped ? 1 : 0;
        if (!dropped && row_src) row_src[pos] = t * k + j;
      }
    }
  }
}

// Row moves: one thread per (token, 16-byte column slice); it copies the slice
// of x[t] to every kept row of the token.  Fully parallel and coalesced.
template <int KMAX>
__global__ void __launch_bounds__(256) k_move_rows(const __nv_bfloat16* __restrict__ x,
                                                   const int32_t* __restrict__ slot_pos, int T, int d, int k,
                                                   __nv_bfloat16* __restrict__ x_perm) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const int nvec = d >> 3;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * nvec) return;
  const long long t = i / nvec;
  const int v = (int)(i - t * nvec);
  int p[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) p[j] = j < k ? slot_pos[t * k + j] : -1;
  const uint4 val = reinterpret_cast<const uint4*>(x + t * d)[v];
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (p[j] >= 0) reinterpret_cast<uint4*>(x_perm + (size_t)p[j] * d)[v] = val;
}

// Write the group table of moe_permute-style outputs without moving rows:
// used by moe_forward when only the tables are needed.  (kept, offsets)
__global__ void __launch_bounds__(128) k_group_table(const int32_t* __restrict__ counts, int E, int cap,
                                                     int32_t* __restrict__ kept_out, int32_t* __restrict__ offsets_out) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_kept[kMaxE];
  __shared__ int s_tmp[4];
  group_offsets(counts, E, cap, s_off, s_kept, s_tmp);
  for (int e = threadIdx.x; e < E; e += 128) {
    kept_out[e] = s_kept[e];
    offsets_out[e] = s_off[e];
  }
  if (threadIdx.x == 0) offsets_out[E] = s_off[E];
}

// ---------------------------------------------------------------------------
// Combine: one warp per (token, column range), fp32 sum over slots j = 0..k-1
// in order, then the shared expert, one bf16 rounding.  Each lane owns 16-byte
// column slices; the k row loads of a slice are issued together.  blockIdx.y
// splits the columns into gridDim.y ranges of `vec_per_range` 16-byte slices so
// that small batches (decode) still spread over every SM.
template <int KMAX>
__global__ void __launch_bounds__(256) k_combine(const __nv_bfloat16* __restrict__ y_perm,
                                                 const int32_t* __restrict__ slot_pos, const float* __restrict__ w,
                                                 const __nv_bfloat16* __restrict__ y_shared,
                                                 __nv_bfloat16* __restrict__ out, int T, int d, int k,
                                                 int vec_per_range) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const int t = blockIdx.x * 8 + warp_id();
  const int lane = lane_id();
  if (t >= T) return;
  const int v_begin = blockIdx.y * vec_per_range;
  const int nvec = min(d >> 3, v_begin + vec_per_range);
  int p[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    p[j] = j < k ? slot_pos[(size_t)t * k + j] : -1;
    g[j] = j < k ? w[(size_t)t * k + j] : 0.f;
  }
  for (int v = v_begin + lane; v < nvec; v += 32) {
    uint4 u[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      u[j] = p[j] >= 0 ? reinterpret_cast<const uint4*>(y_perm + (size_t)p[j] * d)[v] : make_uint4(0, 0, 0, 0);
    uint4 us = make_uint4(0, 0, 0, 0);
    if (y_shared != nullptr) us = reinterpret_cast<const uint4*>(y_shared + (size_t)t * d)[v];
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (p[j] >= 0) {
        acc[0] = fmaf(g[j], bf16lo(u[j].x), acc[0]); acc[1] = fmaf(g[j], bf16hi(u[j].x), acc[1]);
        acc[2] = fmaf(g[j], bf16lo(u[j].y), acc[2]); acc[3] = fmaf(g[j], bf16hi(u[j].y), acc[3]);
        acc[4] = fmaf(g[j], bf16lo(u[j].z), acc[4]); acc[5] = fmaf(g[j], bf16hi(u[j].z), acc[5]);
        acc[6] = fmaf(g[j], bf16lo(u[j].w), acc[6]); acc[7] = fmaf(g[j], bf16hi(u[j].w), acc[7]);
      }
    }
    if (y_shared != nullptr) {
      acc[0] += bf16lo(us.x); acc[1] += bf16hi(us.x); acc[2] += bf16lo(us.y); acc[3] += bf16hi(us.y);
      acc[4] += bf16lo(us.z); acc[5] += bf16hi(us.z); acc[6] += bf16lo(us.w); acc[7] += bf16hi(us.w);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]); o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]); o.w = pack_bf16x2(acc[6], acc[7]);
    reinterpret_cast<uint4*>(out + (size_t)t * d)[v] = o;
  }
}

}  // namespace moe
