// Hierarchical ("fractal") router (kieve-moe Features, "Fractal tiling routing": self-similar routing over a
// branch^levels expert tree, a cheap router for very large expert pools).  Expert e is the leaf whose
// base-branch digits d_0 .. d_{L-1} (most significant first) pick a child at each level; level l has its own
// router W_l [branch, d] shared by every node of the level, and the leaf probability is the product of the
// level softmaxes along the path: p(e) = q_0[d_0] q_1[d_1] ... q_{L-1}[d_{L-1}], q_l = softmax(x W_l^T + b_l).
// Per token that is levels * branch logits instead of E = branch^levels.  The level logits come from the
// router's tensor-core screen (two-term bf16 split of the fp32 weights, fp32 accumulation); this kernel takes
// the level softmaxes and the top-k of the leaf probabilities by a beam search, a small group of lanes per
// token: after each level only the k best partial paths survive, ordered by (product desc, path index asc).
// The product is monotone in each factor, so the k best leaves are never pruned; each leaf's product is formed
// in level order, as a direct evaluation would.  Gates are the leaf probabilities, renormalised over the k
// picks when asked.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kTreeMaxBranch = 32;   // one level's children on at most 8 lanes, 4 each
constexpr int kTreeMaxLogits = 256;  // levels * branch: one screening tile
constexpr long long kTreeMaxE = 1ll << 20;   // leaves

constexpr int kTreeCPL = 4;          // children per lane: a token takes branch / 4 lanes (rounded up to 2, 4 or 8)
constexpr int kTreeThreads = 128;

// G lanes per token (G = 2, 4 or 8, at least branch / 4).  z [T, L * B] fp32 level logits (bias included).
// Outputs topk_idx / topk_w [T, k]; counts [E] (zeroed beforehand) gains one per selection when not null.
// Per level:
//   1. softmax: lane g holds children c = g, g + G, g + 2 G, g + 3 G (c < B); group max and sum;
//   2. the level's kk = min(k, B) best children by (q desc, c asc), into shared memory: each lane offers its
//      best untaken child, a butterfly over the group picks the winner (exactly the order of a full sort);
//   3. the new beam: nsel = min(k, nb B) rounds over the candidates (bv[j] q[c], bi[j] B + c); lane g owns beam
//      entries g, g + G, ..., offers each entry's best untaken child (the first untaken in q order, or among
//      later ones whose product rounds to the same value, the lowest c), and a butterfly picks the largest
//      product, the lower path index among equal ones.  Only an entry's kk best children can reach the top k.
template <int KMAX, int G>
__global__ void __launch_bounds__(kTreeThreads) k_router_tree(const float* __restrict__ z, int T, int B, int L,
                                                              int k, int renorm, int32_t* __restrict__ topk_idx,
                                                              float* __restrict__ topk_w,
                                                              int32_t* __restrict__ counts) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  constexpr int kTreeGroup = G;
  constexpr int CPL = kTreeCPL;                              // children per lane
  constexpr int EPL = (KMAX + kTreeGroup - 1) / kTreeGroup;  // beam entries per lane
  __shared__ float s_cq[kTreeThreads / kTreeGroup][KMAX];
  __shared__ int s_cc[kTreeThreads / kTreeGroup][KMAX];
  const long long t = ((long long)blockIdx.x * kTreeThreads + threadIdx.x) / kTreeGroup;
  const int g = threadIdx.x % kTreeGroup;
  // whole groups leave together (T is a group boundary), so the group shuffles below see every lane
  if (t >= T) return;
  const unsigned gmask = ((1u << kTreeGroup) - 1u) << (lane_id() & ~(kTreeGroup - 1));
  float* cq = s_cq[threadIdx.x / kTreeGroup];
  int* cc = s_cc[threadIdx.x / kTreeGroup];
  const float* zr = z + t * (long long)(B * L);
  // this lane's beam entries g + 8 e: product and path index
  float bv[EPL];
  int bi[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) { bv[e] = (g + kTreeGroup * e == 0) ? 1.f : 0.f; bi[e] = 0; }
  int nb = 1;
  float nv[KMAX];   // the new beam, the same on every lane of the group
  int ni[KMAX];
  for (int l = 0; l < L; ++l) {
    // 1. level softmax
    const float* zl = zr + l * B;
    float q[CPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const int c = g + kTreeGroup * i;
      q[i] = c < B ? zl[c] : -INFINITY;
      m = fmaxf(m, q[i]);
    }
#pragma unroll
    for (int o = kTreeGroup / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(gmask, m, o, kTreeGroup));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      q[i] = g + kTreeGroup * i < B ? __expf(q[i] - m) : 0.f;
      sum += q[i];
    }
#pragma unroll
    for (int o = kTreeGroup / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(gmask, sum, o, kTreeGroup);
#pragma unroll
    for (int i = 0; i < CPL; ++i) q[i] = q[i] / sum;
    // 2. the level's best kk children, in order
    const int kk = min(k, B);
    uint32_t ctaken = 0u;
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      if (r >= kk) break;
      float best = -1.f;
      int bc = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int c = g + kTreeGroup * i;
        if (c < B && !((ctaken >> i) & 1u) && (q[i] > best || (q[i] == best && c < bc))) { best = q[i]; bc = c; }
      }
#pragma unroll
      for (int o = kTreeGroup / 2; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(gmask, best, o, kTreeGroup);
        const int oc = __shfl_xor_sync(gmask, bc, o, kTreeGroup);
        if (ov > best || (ov == best && oc < bc)) { best = ov; bc = oc; }
      }
      if (bc % kTreeGroup == g) ctaken |= 1u << (bc / kTreeGroup);
      if (g == 0) { cq[r] = best; cc[r] = bc; }
    }
    __syncwarp(gmask);
    // 3. the new beam
    const int nsel = min(k, nb * B);
    uint32_t tk[EPL];   // bit p: child cq[p] of this entry is taken
#pragma unroll
    for (int e = 0; e < EPL; ++e) tk[e] = 0u;
#pragma unroll
    for (int r = 0; r < KMAX; ++r) {
      nv[r] = 0.f;
      ni[r] = 0;
      if (r >= nsel) continue;
      float best = -1.f;
      int bidx = 0x7fffffff, be = -1, bp = 0;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        if (g + kTreeGroup * e >= nb) continue;
        const int p = __ffs(~tk[e]) - 1;
        if (p < 0 || p >= kk) continue;
        const float v = bv[e] * cq[p];
        int c = cc[p], pp = p;
        for (int p2 = p + 1; p2 < kk; ++p2) {   // later children whose product rounds to the same value
          if ((tk[e] >> p2) & 1u) continue;
          if (bv[e] * cq[p2] != v) break;
          if (cc[p2] < c) { c = cc[p2]; pp = p2; }
        }
        const int id = bi[e] * B + c;
        if (v > best || (v == best && id < bidx)) { best = v; bidx = id; be = e; bp = pp; }
      }
      const int mine = bidx;
#pragma unroll
      for (int o = kTreeGroup / 2; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(gmask, best, o, kTreeGroup);
        const int oi = __shfl_xor_sync(gmask, bidx, o, kTreeGroup);
        if (ov > best || (ov == best && oi < bidx)) { best = ov; bidx = oi; }
      }
      nv[r] = best;
      ni[r] = bidx;
      if (be >= 0 && mine == bidx) {
#pragma unroll
        for (int e = 0; e < EPL; ++e)
          if (e == be) tk[e] |= 1u << bp;
      }
    }
    __syncwarp(gmask);   // the children table is rewritten by the next level
    // hand the new beam to its owners
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      float v = 0.f;
      int id = 0;
#pragma unroll
      for (int r = 0; r < KMAX; ++r)
        if (r == g + kTreeGroup * e) { v = nv[r]; id = ni[r]; }
      bv[e] = v;
      bi[e] = id;
    }
    nb = nsel;
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < k) s += nv[j];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j >= k || j % kTreeGroup != g) continue;
    topk_idx[t * k + j] = ni[j];
    topk_w[t * k + j] = renorm ? nv[j] / s : nv[j];
    if (counts != nullptr) atomicAdd(counts + ni[j], 1);
  }
}

}  // namespace moe
