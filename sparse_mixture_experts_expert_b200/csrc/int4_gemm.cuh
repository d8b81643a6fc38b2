// Grouped expert GEMM over group-scaled signed INT4 weights (weight streaming).
//
// ExpertMesh README: "A HIP routed-expert correctness kernel for group-scaled
// signed INT4 weights ... unpacks signed INT4 weights, applies FP16 group
// scales, executes the routed expert product"; layout [expert, output,
// packed_input].  Scales here are bf16, one per 128 consecutive inputs of an
// output row; two's-complement nibbles, the even input in the low nibble.
//
// Decode batches put ~1-8 rows on each touched expert, so the kernel is bound
// by streaming the weights from HBM: every weight byte is read once, every
// row of the group reuses it from registers.
//   * one warp = one task = 16 output rows of one expert (gated mode: 16 gate
//     rows W1 and the matching 16 up rows W3) over the full reduction length;
//   * a thread loads 16 bytes (32 nibbles) per row per 128-input group; the
//     nibbles are turned into bf16 pairs with one LOP3 each (the nibble, with
//     its sign bit flipped, becomes the low mantissa bits of 128.0) and one
//     packed subtraction of 136;
//   * mma.sync m16n8k16 (bf16 in, fp32 out) multiplies the integer codes q
//     (exact in bf16) by up to 8 activation rows; the reduction order inside
//     a 128-group is permuted identically for weights and activations, so a
//     thread's 32 consecutive nibbles feed its fragments directly;
//   * the fp32 partial of each 128-group is scaled by its bf16 scale and
//     added to the fp32 total: w = q * s is applied exactly;
//   * gated mode writes h = act(x W1^T) * (x W3^T) in bf16, plain mode y.
// Groups with more than 8 rows are split into 8-row chunks, one task each;
// the chunks of one 16-row block run on neighbouring warps, so the repeat
// weight reads hit L2.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace moe {

struct Int4Params {
  const uint8_t* wq;             // [G, b_rows, K/2]
  const __nv_bfloat16* ws;       // [G, b_rows, K/128]
  const __nv_bfloat16* act;      // [R, K]
  const int32_t* group_start;    // [G] or nullptr (one group of R rows)
  const int32_t* group_rows;     // [G] or nullptr
  int n_groups;
  long long R;
  int K;
  int N;                         // output columns
  int b_rows;                    // rows per expert in wq (2H gated, d plain)
  int up_row0;                   // gated: first up row (H)
  __nv_bfloat16* out;            // [R, N]
  long long ldo;
};

__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t mask, uint32_t c) {
  // (a & mask) ^ c
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(r) : "r"(a), "r"(mask), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Word of 8 nibbles n0..n7 (n_i at bits 4i) -> four bf16 pairs of signed codes:
// p[0] = (n0, n4), p[1] = (n1, n5), p[2] = (n2, n6), p[3] = (n3, n7).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t kMask = 0x000F000Fu, kMagic = 0x43084308u, k136 = 0x43084308u;  // 136.0 in bf16 = 0x4308
  p[0] = bf16x2_sub(lop3_and_xor(w, kMask, kMagic), k136);
  p[1] = bf16x2_sub(lop3_and_xor(w >> 4, kMask, kMagic), k136);
  p[2] = bf16x2_sub(lop3_and_xor(w >> 8, kMask, kMagic), k136);
  p[3] = bf16x2_sub(lop3_and_xor(w >> 12, kMask, kMagic), k136);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t u4get(const uint4& v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// MMA of one 128-group for one 16-row block: acc += q[16 x 128] . x[8 x 128]^T.
// wa / wb: this thread's 16 bytes of rows g and g+8; xv[j]: activations
// x[token][32c + 8j .. +8] for j = 0..3 (zeros for absent tokens).
__device__ __forceinline__ void mma_group(float (&acc)[4], const uint4& wa, const uint4& wb, const uint4 (&xv)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t pa[4], pb[4];
    dequant_word(u4get(wa, j), pa);
    dequant_word(u4get(wb, j), pb);
    const uint4 xx = xv[j];
    const uint32_t x04 = prmt(xx.x, xx.z, 0x5410), x15 = prmt(xx.x, xx.z, 0x7632);
    const uint32_t x26 = prmt(xx.y, xx.w, 0x5410), x37 = prmt(xx.y, xx.w, 0x7632);
    mma_bf16_16816(acc, pa[0], pb[0], pa[1], pb[1], x04, x15);
    mma_bf16_16816(acc, pa[2], pb[2], pa[3], pb[3], x26, x37);
  }
}

template <bool GLU, int ACT>
__global__ void __launch_bounds__(256, 2) k_int4_gemm(const Int4Params p) {
  __shared__ int s_prefix[kMaxGroupsSmem + 1];
  const int lane = lane_id(), warp = warp_id();
  const bool single = p.group_rows == nullptr;
  const int G = single ? 1 : p.n_groups;
  const int oblocks = p.N / 16;
  // tasks of group g: oblocks x ceil(rows / 8) (16 output rows x 8 activation rows each)
  auto group_tasks = [&](int g) -> int {
    const long long rows = single ? p.R : (long long)p.group_rows[g];
    return (int)(oblocks * ((rows + 7) / 8));
  };
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g) local += group_tasks(g);
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
      s_prefix[g] = run;
      run += group_tasks(g);
    }
    if (lane == 31) s_prefix[G] = incl;
  }
  __syncthreads();
  const int total = s_prefix[G];
  const int gq = lane >> 2, c = lane & 3;
  const int ngroups_k = p.K / 128;
  const long long wrow_bytes = p.K / 2;

  for (int task = blockIdx.x * 8 + warp; task < total; task += gridDim.x * 8) {
    int lo = 0, hi = G - 1;  // last group with s_prefix[g] <= task
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= task) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const long long row0 = single ? 0 : p.group_start[g];
    const int n_rows = (int)(single ? p.R : (long long)p.group_rows[g]);
    const int nchunks = (n_rows + 7) / 8;
    const int tg = task - s_prefix[g];
    const int o0 = (tg / nchunks) * 16;  // chunks of one row block are adjacent tasks: the repeat reads hit L2
    const int n0 = (tg % nchunks) * 8;
    const long long wbase = (long long)g * p.b_rows;
    // this thread's weight rows: gate (or plain) rows o0+gq, o0+gq+8; up rows up_row0 + same
    const uint8_t* wg0 = p.wq + (wbase + o0 + gq) * wrow_bytes + c * 16;
    const uint8_t* wg1 = wg0 + 8 * wrow_bytes;
    const uint8_t* wu0 = p.wq + (wbase + p.up_row0 + o0 + gq) * wrow_bytes + c * 16;
    const uint8_t* wu1 = wu0 + 8 * wrow_bytes;
    const __nv_bfloat16* sg0 = p.ws + (wbase + o0 + gq) * ngroups_k;
    const __nv_bfloat16* sg1 = sg0 + 8 * ngroups_k;
    const __nv_bfloat16* su0 = p.ws + (wbase + p.up_row0 + o0 + gq) * ngroups_k;
    const __nv_bfloat16* su1 = su0 + 8 * ngroups_k;

    {
      const int tok = n0 + gq;            // B column this thread feeds
      const bool tok_ok = tok < n_rows;
      const __nv_bfloat16* xrow = p.act + (row0 + (tok_ok ? tok : 0)) * (long long)p.K + c * 32;
      float tg[4] = {0.f, 0.f, 0.f, 0.f}, tu[4] = {0.f, 0.f, 0.f, 0.f};
      uint4 a0 = ldg_stream(wg0), a1 = ldg_stream(wg1);
      uint4 u0 = make_uint4(0, 0, 0, 0), u1 = make_uint4(0, 0, 0, 0);
      if (GLU) { u0 = ldg_stream(wu0); u1 = ldg_stream(wu1); }
      for (int kg = 0; kg < ngroups_k; ++kg) {
        // prefetch the next group's weights
        uint4 na0 = a0, na1 = a1, nu0 = u0, nu1 = u1;
        if (kg + 1 < ngroups_k) {
          na0 = ldg_stream(wg0 + (kg + 1) * 64);
          na1 = ldg_stream(wg1 + (kg + 1) * 64);
          if (GLU) { nu0 = ldg_stream(wu0 + (kg + 1) * 64); nu1 = ldg_stream(wu1 + (kg + 1) * 64); }
        }
        uint4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xv[j] = tok_ok ? *reinterpret_cast<const uint4*>(xrow + kg * 128 + 8 * j) : make_uint4(0, 0, 0, 0);
        float pg[4] = {0.f, 0.f, 0.f, 0.f};
        mma_group(pg, a0, a1, xv);
        const float s0 = __bfloat162float(sg0[kg]), s1 = __bfloat162float(sg1[kg]);
        tg[0] = fmaf(pg[0], s0, tg[0]); tg[1] = fmaf(pg[1], s0, tg[1]);
        tg[2] = fmaf(pg[2], s1, tg[2]); tg[3] = fmaf(pg[3], s1, tg[3]);
        if (GLU) {
          float pu[4] = {0.f, 0.f, 0.f, 0.f};
          mma_group(pu, u0, u1, xv);
          const float r0 = __bfloat162float(su0[kg]), r1 = __bfloat162float(su1[kg]);
          tu[0] = fmaf(pu[0], r0, tu[0]); tu[1] = fmaf(pu[1], r0, tu[1]);
          tu[2] = fmaf(pu[2], r1, tu[2]); tu[3] = fmaf(pu[3], r1, tu[3]);
        }
        a0 = na0; a1 = na1; u0 = nu0; u1 = nu1;
      }
      // D fragment: (m = gq, n = 2c, 2c+1) in [0],[1]; (m = gq+8, same n) in [2],[3]
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = gq + (i >= 2 ? 8 : 0);
        const int n = n0 + 2 * c + (i & 1);
        if (n < n_rows) {
          float v = tg[i];
          if (GLU) v = (ACT == kModeSwiGLU ? act_silu(v) : act_gelu(v)) * tu[i];
          p.out[(row0 + n) * p.ldo + o0 + m] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

}  // namespace moe
