// Grouped expert GEMM over group-scaled signed INT4 weights (weight streaming).
//
// ExpertMesh README: "A HIP routed-expert correctness kernel for group-scaled
// signed INT4 weights ... unpacks signed INT4 weights, applies FP16 group
// scales, executes the routed expert product"; layout [expert, output,
// packed_input].  Scales here are bf16, one per 128 consecutive inputs of an
// output row; two's-complement nibbles, the even input in the low nibble.
//
// Decode batches put ~1-8 rows on each touched expert, so the GEMM is bound
// by streaming the weights from HBM: every weight byte is read once and every
// activation row of the group reuses it from registers.
//   * the nibbles become 16-bit float pairs with one LOP3 each (the nibble,
//     with its sign bit flipped, becomes mantissa bits of a power of two):
//     - offset codes (the forward's path): f16 codes 1032 + q (even inputs,
//       mantissa bits 0..3 of 1024.0) and 72 + q (odd inputs, mantissa bits
//       4..7 of 64.0), one shift per word of 8 nibbles; the activations are
//       f16 copies scaled by a power of two per 128-group, and the offsets'
//       share, sum(off_i x_i), is removed per group afterwards;
//     - exact codes (the per-step entry point): bf16 128 + (q + 8) followed by
//       one packed subtraction of 136, three shifts per word;
//   * mma.sync m16n8k16 (fp32 accumulation) multiplies the integer codes
//     (exact in f16 / bf16) by up to 8 activation rows; the reduction order
//     inside a 128-group is permuted identically for weights and activations,
//     so a thread's 32 consecutive nibbles feed its fragments directly;
//   * the fp32 partial of each 128-group is scaled by its bf16 scale and added
//     to the fp32 total: w = q * s is applied exactly;
//   * gated mode writes h = act(x W1^T) * (x W3^T) in bf16, plain mode y.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace moe {

struct Int4Params {
  const uint8_t* wq;             // [G, b_rows, K/2]
  const __nv_bfloat16* ws;       // [G, b_rows, K/128]
  const __nv_bfloat16* act;      // [R, K] (offset-code kernels: the f16 copy of k_int4_act_prep)
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
  int ksplit;                    // >= 1: each task's slabs are split into this many contiguous ranges
  float* part;                   // ksplit > 1: fp32 partials [ksplit, R, 2N] (gated: gate | up) or [ksplit, R, N]
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

// Word of 8 nibbles -> four f16 pairs of offset codes, one shift per word.  An
// f16 of exponent 2^10 has unit mantissa steps, so a nibble in mantissa bits
// 0..3 of 1024.0 reads 1024 + (nibble); one in bits 4..7 of 64.0 reads
// 64 + (nibble).  With the nibble's sign bit flipped (q + 8 in 0..15):
//   p[0] = (n0, n4), p[2] = (n2, n6): 1032 + q   (even inputs)
//   p[1] = (n1, n5), p[3] = (n3, n7):   72 + q   (odd inputs)
// All are integers below 2^11, exact in f16.
constexpr float kOffEven = 1032.f, kOffOdd = 72.f;
__device__ __forceinline__ void offset_word_f16(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  p[0] = lop3_and_xor(w, 0x000F000Fu, 0x64086408u);    // 1024.0 = 0x6400, sign bit of the nibble at bit 3
  p[1] = lop3_and_xor(w, 0x00F000F0u, 0x54805480u);    //   64.0 = 0x5400, sign bit of the nibble at bit 7
  p[2] = lop3_and_xor(w8, 0x000F000Fu, 0x64086408u);
  p[3] = lop3_and_xor(w8, 0x00F000F0u, 0x54805480u);
}

// acc += codes[16 x 128] . x'[8 x 128]^T for one 16-row block (rows g and g+8 of this thread), f16 operands.
// xf[j]: the scaled f16 activations of inputs 32c + 8j .. + 8 already in fragment order
// (x0,x4), (x1,x5), (x2,x6), (x3,x7) -- see k_int4_act_prep.
__device__ __forceinline__ void mma_group_offset(float (&acc)[4], const uint4& wa, const uint4& wb,
                                                 const uint4 (&xf)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t pa[4], pb[4];
    offset_word_f16(u4get(wa, j), pa);
    offset_word_f16(u4get(wb, j), pb);
    mma_f16_16816(acc, pa[0], pb[0], pa[1], pb[1], xf[j].x, xf[j].y);
    mma_f16_16816(acc, pa[2], pb[2], pa[3], pb[3], xf[j].z, xf[j].w);
  }
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

// ---------------------------------------------------------------------------
// Activation preparation of the offset-code product, one CTA per row (blockDim
// a multiple of 32, at most 1024: a row of up to 8192 inputs in one pass):
//   e:  the power of two that brings the row's largest |x| into [2^14, 2^15)
//       (0 for an all-zero row; clamped to [-100, 113]).  x' = x 2^-e is exact
//       in fp32, and its f16 rounding is exact from 2^-14 up (bf16 carries 8
//       significant bits, f16 11), so the f16 copy differs from x' only for
//       inputs below 2^-28 of the row's largest, by at most 2^-25;
//   Aq: x' in f16 with every 8 inputs x0..x7 stored as x0,x4,x1,x5,x2,x6,x3,x7,
//       the order in which the nibble pairs of a weight word come out, so the
//       streaming kernel uses 16-byte loads as B fragments without permutes;
//   csum[r][g]: c = sum of off_i x'_i over 128-group g (off = 1032 for even
//       inputs, 72 for odd ones: the offsets of offset_word_f16's codes), each
//       thread adding its 8 in order, then a fixed xor tree over the group's 16;
//   rscale[r] = 2^e.
// The product of the codes with x' minus c is sum(q x') = 2^-e sum(q x).
// With slot_pos (the grouping of a routed batch), block t converts token row t
// of A once and writes it to every grouped row slot_pos[t * kk + j] >= 0: the
// grouped copy of the activations is formed here, with no bf16 copy between;
// with Aq2 set, row t also goes to row t of (csum2, rscale2, Aq2): the ungrouped
// copy the shared expert reads.
__global__ void __launch_bounds__(1024) k_int4_act_prep(const __nv_bfloat16* __restrict__ A, int K,
                                                       float* __restrict__ csum, float* __restrict__ rscale,
                                                       __half* __restrict__ Aq,
                                                       const int32_t* __restrict__ slot_pos, int kk,
                                                       float* __restrict__ csum2, float* __restrict__ rscale2,
                                                       __half* __restrict__ Aq2) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  __shared__ float s_m[32];
  __shared__ int s_dst[16];
  __shared__ int s_nd;
  const long long row = blockIdx.x;   // source row
  int ndst = 1;
  if (slot_pos != nullptr) {          // destination rows of this token (kk <= 16), dropped slots skipped
    if (threadIdx.x == 0) {
      int nd = 0;
      for (int j = 0; j < kk; ++j) {
        const int pos = slot_pos[row * kk + j];
        if (pos >= 0) s_dst[nd++] = pos;
      }
      s_nd = nd;
    }
    __syncthreads();
    ndst = s_nd;
  } else if (threadIdx.x == 0) {
    s_dst[0] = (int)row;
  }
  const int nv = K / 8;   // 16 per 128-group; a pass covers whole groups
  const uint4* src = reinterpret_cast<const uint4*>(A + row * K);
  // the first pass's inputs stay in registers for the conversion (the whole row when nv <= blockDim)
  const uint4 u0 = (int)threadIdx.x < nv ? src[threadIdx.x] : make_uint4(0, 0, 0, 0);
  float m = 0.f;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    const uint4 u = v == (int)threadIdx.x ? u0 : src[v];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(u.x)), fabsf(bf16hi(u.x))), fmaxf(fabsf(bf16lo(u.y)), fabsf(bf16hi(u.y)))));
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(u.z)), fabsf(bf16hi(u.z))), fmaxf(fabsf(bf16lo(u.w)), fabsf(bf16hi(u.w)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane_id() == 0) s_m[warp_id()] = m;
  __syncthreads();
  m = s_m[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, s_m[w]);
  const int eb = (int)((__float_as_uint(m) >> 23) & 0xFFu);   // biased exponent of the row's largest |x|
  const int e = m == 0.f ? 0 : (eb == 0 ? -100 : max(-100, min(113, eb - 127 - 14)));
  const float down = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e, a normal float for e in [-100, 113]
  const float up = __uint_as_float((uint32_t)(127 + e) << 23);   // 2^e
  if ((int)threadIdx.x < ndst) rscale[s_dst[threadIdx.x]] = up;
  if (Aq2 != nullptr && threadIdx.x == 0) rscale2[row] = up;
  for (int base = 0; base < nv; base += blockDim.x) {   // every thread takes part in each pass's xor tree
    const int v = base + threadIdx.x;
    const bool on = v < nv;
    const uint4 u = base == 0 ? u0 : (on ? src[v] : make_uint4(0, 0, 0, 0));
    const float x[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                        bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
    __half h[8];
    float c = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      h[j] = __float2half_rn(x[j] * down);
      c = fmaf((j & 1) ? kOffOdd : kOffEven, __half2float(h[j]), c);
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (on) {
      auto pack = [](__half lo, __half hi) {
        return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
      };
      const uint4 q = make_uint4(pack(h[0], h[4]), pack(h[1], h[5]), pack(h[2], h[6]), pack(h[3], h[7]));
      for (int j = 0; j < ndst; ++j) {
        const long long dr = s_dst[j];
        reinterpret_cast<uint4*>(Aq + dr * K)[v] = q;
        if ((v & 15) == 0) csum[dr * (K / 128) + (v >> 4)] = c;
      }
      if (Aq2 != nullptr) {
        reinterpret_cast<uint4*>(Aq2 + row * K)[v] = q;
        if ((v & 15) == 0) csum2[row * (K / 128) + (v >> 4)] = c;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Streaming variant: the packed weights travel HBM -> shared memory by TMA
// (2-D tensor map over [experts * rows, K/2] bytes), each warp owning a ring
// of kI4Stages slabs of 32 rows x 128 bytes (256 inputs).  A warp's work is a
// sequence of (task, slab) items; its lane 0 keeps kI4Stages items in flight
// across task boundaries, so one SM has up to 16 x 3 x 4 KB of weight reads
// outstanding.  Each task covers 32 weight rows: the 16 gate rows and the 16
// matching up rows (gated mode) or 32 consecutive output rows (plain mode).
constexpr int kI4Warps = 16;
constexpr int kI4Coarse = 2048;   // entries of the stream kernel's task -> group table
constexpr int kI4Stages = 3;
constexpr int kI4SlabBytes = 32 * 128;
constexpr int kI4Smem = kI4Warps * kI4Stages * kI4SlabBytes;

// OFFS: multiply the f16 offset codes by the scaled f16 activations and remove
// the offsets' share c once per group, instead of one packed subtraction per
// pair of weights; p.act is then the fragment-ordered copy written by
// k_int4_act_prep, xcs[row][group] the offsets' share c of each group and
// xrs[row] = 2^e the row's scale, applied once to the finished sums.
template <bool GLU, int ACT, bool OFFS, bool SPLIT>
__global__ void __launch_bounds__(kI4Warps * 32, 1)
    k_int4_stream(const __grid_constant__ CUtensorMap tmW, const Int4Params p, unsigned long long wait_limit_ns,
                  const float* __restrict__ xcs, const float* __restrict__ xrs) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ __align__(128) uint8_t i4_smem[];
  __shared__ int s_prefix[kMaxGroupsSmem + 1];
  __shared__ int s_gstart[kMaxGroupsSmem];
  __shared__ int s_grows[kMaxGroupsSmem];
  __shared__ unsigned short s_cg[kI4Coarse];   // group of base task i * cstride
  __shared__ __align__(8) uint64_t s_bar[kI4Warps][kI4Stages];
  __shared__ volatile int s_abort[kI4Warps];
  const int lane = lane_id(), warp = warp_id();
  const bool single = p.group_rows == nullptr;
  const int G = single ? 1 : p.n_groups;
  const int oblocks = GLU ? p.N / 16 : p.N / 32;   // 32 weight rows per task
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
      s_gstart[g] = single ? 0 : p.group_start[g];
      s_grows[g] = (int)(single ? p.R : (long long)p.group_rows[g]);
      run += group_tasks(g);
    }
    if (lane == 31) s_prefix[G] = incl;
  }
  if (lane == 0) {
    for (int st = 0; st < kI4Stages; ++st) mbar_init(&s_bar[warp][st], 1);
    s_abort[warp] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmW);
  __syncthreads();
  // coarse task -> group table: entry i holds the group of base task i * cstride, so a lookup is one load
  // and a short forward scan instead of a binary search over the groups
  const int cstride = max(1, (s_prefix[G] + kI4Coarse - 1) / kI4Coarse);
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int a = (s_prefix[g] + cstride - 1) / cstride, b = (s_prefix[g + 1] + cstride - 1) / cstride;
    for (int i = a; i < b; ++i) s_cg[i] = (unsigned short)g;
  }
  __syncthreads();

  const int KS = SPLIT ? p.ksplit : 1;   // compile-time 1 unless the reduction is split
  const int total = s_prefix[G] * KS;
  const int nslab = (p.K + 255) / 256;               // slabs of a whole reduction (the last may hold one 128-group)
  const int tfirst = blockIdx.x * kI4Warps + warp;
  const int tstride = gridDim.x * kI4Warps;
  uint8_t* ring = i4_smem + (size_t)warp * kI4Stages * kI4SlabBytes;
  const int gq = lane >> 2, c = lane & 3;
  const int ngroups_k = p.K / 128;

  // task = base * KS + split: a base task is (group, 16 or 32 output rows, 8 tokens); split s covers
  // slabs [s * nslab / KS, (s + 1) * nslab / KS) of its reduction
  struct TaskPos { int g, o0, n0, n_rows, s, sb, se; long long row0; };
  auto locate = [&](int t) -> TaskPos {
    const int task = SPLIT ? t / KS : t;
    int lo = s_cg[task / cstride];   // the last group starting at or before task
    while (s_prefix[lo + 1] <= task) ++lo;
    TaskPos tp;
    tp.g = lo;
    tp.row0 = s_gstart[lo];
    tp.n_rows = s_grows[lo];
    const int nchunks = (tp.n_rows + 7) / 8;
    const int tg = task - s_prefix[lo];
    tp.o0 = (tg / nchunks) * (GLU ? 16 : 32);
    tp.n0 = (tg % nchunks) * 8;
    tp.s = SPLIT ? t - task * KS : 0;
    tp.sb = SPLIT ? tp.s * nslab / KS : 0;
    tp.se = SPLIT ? (tp.s + 1) * nslab / KS : nslab;
    return tp;
  };
  // weight rows of a task's two 16-row blocks (rows of the flattened [experts * b_rows] map)
  auto rows_of = [&](const TaskPos& tp, int& ra, int& rb) {
    ra = tp.g * p.b_rows + tp.o0;
    rb = GLU ? tp.g * p.b_rows + p.up_row0 + tp.o0 : ra + 16;
  };

  // Producer state (lane 0 issues the copies; the values are warp-uniform).
  // Items are (task, slab) pairs in order; issued - consumed <= kI4Stages.
  int issued = 0, consumed = 0;
  int p_task = tfirst, p_slab = 0, p_se = 0, p_st = 0, p_ra = 0, p_rb = 0;
  bool p_new = true;
  auto refill = [&]() {
    while (issued - consumed < kI4Stages) {
      if (p_new) {
        if (p_task >= total) return;
        const TaskPos tp = locate(p_task);
        rows_of(tp, p_ra, p_rb);
        p_slab = tp.sb;
        p_se = tp.se;
        p_new = false;
      }
      if (lane == 0) {
        uint8_t* dst = ring + p_st * kI4SlabBytes;
        mbar_arrive_expect_tx(&s_bar[warp][p_st], kI4SlabBytes);
        tma_load_2d(dst, &tmW, &s_bar[warp][p_st], p_slab * 128, p_ra);
        tma_load_2d(dst + 16 * 128, &tmW, &s_bar[warp][p_st], p_slab * 128, p_rb);
      }
      ++issued;
      if (++p_st == kI4Stages) p_st = 0;
      if (++p_slab == p_se) { p_new = true; p_task += tstride; }
    }
  };

  float tA[4], tB[4];
  TaskPos cur{0, 0, 0, 0, 0};
  const __nv_bfloat16* xrow = nullptr;   // this thread's activation row (token n0 + gq), inputs c*32 ..
  const __nv_bfloat16* sA = nullptr;     // scales of weight row ra + gq (row + 8: + 8 * ngroups_k)
  const __nv_bfloat16* sB = nullptr;     // scales of weight row rb + gq
  const float* xs0 = nullptr;            // offsets' shares c of tokens n0 + 2c, n0 + 2c + 1
  float rs0 = 1.f, rs1 = 1.f;            // their row scales 2^e
  bool tok_ok = false, ok0 = false, ok1 = false;
  const long long s8 = 8ll * ngroups_k;
  int c_task = tfirst, c_slab = 0, c_st = 0;
  uint32_t c_phase = 0;
  bool c_new = true;
  while (true) {
    if (c_new) {
      if (c_task >= total || s_abort[warp]) break;
      cur = locate(c_task);
      c_slab = cur.sb;
      c_new = false;
      int ra, rb;
      rows_of(cur, ra, rb);
      const int tok = cur.n0 + gq;
      tok_ok = tok < cur.n_rows;
      xrow = p.act + (cur.row0 + (tok_ok ? tok : 0)) * (long long)p.K + c * 32;
      sA = p.ws + (long long)(ra + gq) * ngroups_k;
      sB = p.ws + (long long)(rb + gq) * ngroups_k;
      ok0 = cur.n0 + 2 * c < cur.n_rows;
      ok1 = cur.n0 + 2 * c + 1 < cur.n_rows;
      if (OFFS) {
        xs0 = xcs + (cur.row0 + (ok0 ? cur.n0 + 2 * c : 0)) * (long long)ngroups_k;
        rs0 = ok0 ? xrs[cur.row0 + cur.n0 + 2 * c] : 0.f;
        rs1 = ok1 ? xrs[cur.row0 + cur.n0 + 2 * c + 1] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) { tA[i] = 0.f; tB[i] = 0.f; }
    }
    refill();
    // Operands that do not come through the ring are loaded before the wait so
    // that their latency overlaps it: activations and scales of the slab's two
    // 128-groups (the second absent when K % 256 == 128 on the last slab).
    const int kg0 = c_slab * 2;
    const bool two = kg0 + 1 < ngroups_k;
    uint4 xv[2][4];
    float sc[4][2];
    float xsv[2][2];
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      const bool on = tok_ok && (gi == 0 || two);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        xv[gi][q] = on ? *reinterpret_cast<const uint4*>(xrow + (kg0 + gi) * 128 + 8 * q) : make_uint4(0, 0, 0, 0);
    }
    {
      const __nv_bfloat16* sp[4] = {sA + kg0, sA + s8 + kg0, sB + kg0, sB + s8 + kg0};
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        if ((ngroups_k & 1) == 0) {
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(sp[rr]);
          sc[rr][0] = bf16lo(w2);
          sc[rr][1] = bf16hi(w2);
        } else {
          sc[rr][0] = __bfloat162float(sp[rr][0]);
          sc[rr][1] = two ? __bfloat162float(sp[rr][1]) : 0.f;
        }
      }
    }
    if (OFFS) {
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const bool on = gi == 0 || two;
        xsv[gi][0] = (ok0 && on) ? xs0[kg0 + gi] : 0.f;
        xsv[gi][1] = (ok1 && on) ? xs0[ngroups_k + kg0 + gi] : 0.f;
      }
    }
    if (!mbar_wait(&s_bar[warp][c_st], c_phase, wait_limit_ns, &s_abort[warp], 0x0201)) break;
    const uint8_t* slabp = ring + c_st * kI4SlabBytes;
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
      if (gi == 1 && !two) break;  // the slab's second half is TMA zero fill
      const uint4 a0 = *reinterpret_cast<const uint4*>(slabp + gq * 128 + gi * 64 + c * 16);
      const uint4 a1 = *reinterpret_cast<const uint4*>(slabp + (gq + 8) * 128 + gi * 64 + c * 16);
      const uint4 b0 = *reinterpret_cast<const uint4*>(slabp + (gq + 16) * 128 + gi * 64 + c * 16);
      const uint4 b1 = *reinterpret_cast<const uint4*>(slabp + (gq + 24) * 128 + gi * 64 + c * 16);
      float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
      if (OFFS) {
        mma_group_offset(pa, a0, a1, xv[gi]);
        mma_group_offset(pb, b0, b1, xv[gi]);
        // D columns are tokens n0 + 2c and n0 + 2c + 1: remove the offsets' share c of each, then the weight
        // row's group scale
        const float x0 = xsv[gi][0], x1 = xsv[gi][1];
        tA[0] = fmaf(pa[0] - x0, sc[0][gi], tA[0]); tA[1] = fmaf(pa[1] - x1, sc[0][gi], tA[1]);
        tA[2] = fmaf(pa[2] - x0, sc[1][gi], tA[2]); tA[3] = fmaf(pa[3] - x1, sc[1][gi], tA[3]);
        tB[0] = fmaf(pb[0] - x0, sc[2][gi], tB[0]); tB[1] = fmaf(pb[1] - x1, sc[2][gi], tB[1]);
        tB[2] = fmaf(pb[2] - x0, sc[3][gi], tB[2]); tB[3] = fmaf(pb[3] - x1, sc[3][gi], tB[3]);
      } else {
        mma_group(pa, a0, a1, xv[gi]);
        mma_group(pb, b0, b1, xv[gi]);
        tA[0] = fmaf(pa[0], sc[0][gi], tA[0]); tA[1] = fmaf(pa[1], sc[0][gi], tA[1]);
        tA[2] = fmaf(pa[2], sc[1][gi], tA[2]); tA[3] = fmaf(pa[3], sc[1][gi], tA[3]);
        tB[0] = fmaf(pb[0], sc[2][gi], tB[0]); tB[1] = fmaf(pb[1], sc[2][gi], tB[1]);
        tB[2] = fmaf(pb[2], sc[3][gi], tB[2]); tB[3] = fmaf(pb[3], sc[3][gi], tB[3]);
      }
    }
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // slab reads done before TMA reuses it
    ++consumed;
    if (++c_st == kI4Stages) { c_st = 0; c_phase ^= 1u; }
    refill();
    if (c_slab == cur.se - 1) {
      // D fragments: (m = gq, n = 2c, 2c+1) in [0],[1]; (m = gq + 8, same n) in [2],[3]
      if (OFFS) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // back from the scaled activations: the token's 2^e (exact)
          tA[i] *= (i & 1) ? rs1 : rs0;
          tB[i] *= (i & 1) ? rs1 : rs0;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = gq + (i >= 2 ? 8 : 0);
        const int n = cur.n0 + 2 * c + (i & 1);
        if (n < cur.n_rows) {
          if (SPLIT) {
            // fp32 partials of this slab range; k_int4_splitk_reduce adds the ranges in order
            float* prow = p.part + ((long long)cur.s * p.R + cur.row0 + n) * (GLU ? 2 * p.N : p.N) + cur.o0;
            if (GLU) {
              prow[m] = tA[i];
              prow[p.N + m] = tB[i];
            } else {
              prow[m] = tA[i];
              prow[m + 16] = tB[i];
            }
          } else {
            __nv_bfloat16* orow = p.out + (cur.row0 + n) * p.ldo + cur.o0;
            if (GLU) {
              const float a = ACT == kModeSwiGLU ? act_silu(tA[i]) : act_gelu(tA[i]);
              orow[m] = __float2bfloat16_rn(a * tB[i]);
            } else {
              orow[m] = __float2bfloat16_rn(tA[i]);
              orow[m + 16] = __float2bfloat16_rn(tB[i]);
            }
          }
        }
      }
    }
    if (++c_slab == cur.se) { c_new = true; c_task += tstride; }
  }
  // never leave the CTA with copies still landing in its shared memory
  {
    volatile int dummy = 0;
    for (int i = consumed; i < issued; ++i)
      mbar_wait(&s_bar[warp][i % kI4Stages], (uint32_t)((i / kI4Stages) & 1), wait_limit_ns, &dummy, 0x0202);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Dense small batches (one group of R <= 256 rows: the shared expert of a
// decode batch).  A CTA task is (kI4DWarps weight blocks, a block of 64 rows, a
// slab range of the reduction).  Warp w owns weight block kI4DWarps obg + w
// (16 gate + 16 up rows, or 32 output rows) and streams its packed weights by
// TMA through its own ring; the 64 rows' activations (the f16 copy written by
// k_int4_act_prep) and the slab's offset shares go to shared memory once per
// slab for all warps, by cp.async into two buffers, so slab s + 1 loads while
// slab s computes.  Each weight is read once per 64 rows and dequantised once
// per 32 (the MMAs of four 8-row chunks).  f16 offset codes as in k_int4_stream's OFFS
// mode; fp32 partials [ksplit][R][W] in its split layout, which
// k_int4_splitk_reduce adds in order.
constexpr int kI4DWarps = 8;
constexpr int kI4DStages = 4;
constexpr int kI4DChunks = 8;                      // 8-row chunks per task
constexpr int kI4DRows = 8 * kI4DChunks;           // rows per task
constexpr int kI4DActBytes = kI4DRows * 512;       // one slab of activations: 64 rows x 256 f16
constexpr int kI4DSmem = kI4DWarps * kI4DStages * kI4SlabBytes + 2 * kI4DActBytes;

// 16-byte chunk q (of the 32 in a 256-input activation row) of row r is stored at
// chunk q ^ (bit 3 of q, as bit 1 | bit 0 of r): the fragment reads of a
// quarter-warp (rows 2i, 2i+1; lanes c = 0..3 reading chunks 4c + j) then hit
// eight different bank groups.
__device__ __forceinline__ int dense_act_chunk(int q, int r) { return q ^ ((((q >> 3) & 1) << 1) | (r & 1)); }

template <bool GLU>
__global__ void __launch_bounds__(kI4DWarps * 32, 1)
    k_int4_dense(const __grid_constant__ CUtensorMap tmW, const Int4Params p, unsigned long long wait_limit_ns,
                 const float* __restrict__ xcs, const float* __restrict__ xrs) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  extern __shared__ __align__(128) uint8_t i4_smem[];
  __shared__ __align__(8) uint64_t s_bar[kI4DWarps][kI4DStages];
  __shared__ volatile int s_abort[kI4DWarps];
  __shared__ float s_c[2][kI4DRows][2];    // offsets' shares of a slab's two groups, per row
  const int lane = lane_id(), warp = warp_id();
  if (lane == 0) {
    for (int st = 0; st < kI4DStages; ++st) mbar_init(&s_bar[warp][st], 1);
    s_abort[warp] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmW);
  __syncthreads();
  uint8_t* ring = i4_smem + (size_t)warp * kI4DStages * kI4SlabBytes;
  uint8_t* act = i4_smem + (size_t)kI4DWarps * kI4DStages * kI4SlabBytes;
  const int KS = p.ksplit;
  const int oblocks = GLU ? p.N / 16 : p.N / 32;
  const int nobg = (oblocks + kI4DWarps - 1) / kI4DWarps;
  const int R = (int)p.R;
  const int nrh = (R + kI4DRows - 1) / kI4DRows;
  const int total = nobg * nrh * KS;       // task = (weight block group, row block, split), split fastest
  const int nslab = (p.K + 255) / 256;
  const int ngk = p.K / 128;
  const int gq = lane >> 2, c = lane & 3;
  auto task_pos = [&](int task, int& ob, int& rh, int& sb, int& se) {
    const int sp = task % KS;
    rh = (task / KS) % nrh;
    ob = (task / (KS * nrh)) * kI4DWarps + warp;
    sb = sp * nslab / KS;
    se = (sp + 1) * nslab / KS;
  };
  auto rows_of = [&](int ob, int& ra, int& rb) {
    ra = GLU ? ob * 16 : ob * 32;
    rb = GLU ? p.up_row0 + ob * 16 : ra + 16;
  };
  // weight producer (lane 0 issues; values warp-uniform): the warp's slabs of the CTA's tasks in order, at
  // most kI4DStages ahead; tasks whose weight block is past the last one have none
  int issued = 0, consumed = 0;
  int p_task = blockIdx.x, p_slab = 0, p_se = 0, p_st = 0, p_ra = 0, p_rb = 0;
  bool p_new = true;
  auto refill = [&]() {
    while (issued - consumed < kI4DStages && !s_abort[warp]) {
      if (p_new) {
        if (p_task >= total) return;
        int ob, rh, sb, se;
        task_pos(p_task, ob, rh, sb, se);
        if (ob >= oblocks || sb == se) { p_task += gridDim.x; continue; }
        rows_of(ob, p_ra, p_rb);
        p_slab = sb;
        p_se = se;
        p_new = false;
      }
      if (lane == 0) {
        uint8_t* dst = ring + p_st * kI4SlabBytes;
        mbar_arrive_expect_tx(&s_bar[warp][p_st], kI4SlabBytes);
        tma_load_2d(dst, &tmW, &s_bar[warp][p_st], p_slab * 128, p_ra);
        tma_load_2d(dst + 16 * 128, &tmW, &s_bar[warp][p_st], p_slab * 128, p_rb);
      }
      ++issued;
      if (++p_st == kI4DStages) p_st = 0;
      if (++p_slab == p_se) { p_new = true; p_task += gridDim.x; }
    }
  };
  // activations of slab s for rows r0 .. r0 + 63 into buffer b (zeros past R and past K)
  auto load_act = [&](int s, int b, int r0) {
    uint8_t* dst = act + (size_t)b * kI4DActBytes;
    for (int q = threadIdx.x; q < kI4DRows * 32; q += blockDim.x) {
      const int r = q >> 5, ch = q & 31;
      const int tok = r0 + r, kin = s * 256 + ch * 8;
      const bool on = tok < R && kin < p.K;
      const __nv_bfloat16* src = on ? p.act + (size_t)tok * p.K + kin : p.act;
      cp_async16(dst + r * 512 + dense_act_chunk(ch, r) * 16, src, on ? 16 : 0);
    }
  };
  // the offsets' share of group g of slab s for row r (thread i < 128: r = i / 2, g = i % 2)
  auto share = [&](int s, int r0) -> float {
    const int r = threadIdx.x >> 1, kg = 2 * s + (threadIdx.x & 1), tok = r0 + r;
    return (tok < R && kg < ngk) ? xcs[(size_t)tok * ngk + kg] : 0.f;
  };

  float tA[kI4DChunks][4], tB[kI4DChunks][4];
  int c_st = 0;
  uint32_t c_phase = 0;
  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    int ob, rh, sb, se;
    task_pos(task, ob, rh, sb, se);
    if (sb == se) continue;                  // the same for every warp of the CTA
    const bool mine = ob < oblocks;
    const int r0 = rh * kI4DRows;
    int ra = 0, rb = 0;
    if (mine) rows_of(ob, ra, rb);
#pragma unroll
    for (int ch = 0; ch < kI4DChunks; ++ch)
#pragma unroll
      for (int i = 0; i < 4; ++i) { tA[ch][i] = 0.f; tB[ch][i] = 0.f; }
    const __nv_bfloat16* sA = p.ws + (long long)(ra + gq) * ngk;
    const __nv_bfloat16* sB = p.ws + (long long)(rb + gq) * ngk;
    const long long s8 = 8ll * ngk;
    load_act(sb, 0, r0);
    if (threadIdx.x < kI4DRows * 2) s_c[0][threadIdx.x >> 1][threadIdx.x & 1] = share(sb, r0);
    for (int s = sb; s < se; ++s) {
      const int b = (s - sb) & 1;
      // slab s + 1's activations and shares start loading (buffer b ^ 1 was last read at slab s - 1, before the
      // barrier that closed it)
      float cnext = 0.f;
      if (s + 1 < se) {
        load_act(s + 1, b ^ 1, r0);
        if (threadIdx.x < kI4DRows * 2) cnext = share(s + 1, r0);
      }
      cp_async_commit();                     // an empty group on the last slab keeps the count uniform
      // the group scales of weight rows gq, gq + 8 (gate / first half) and the other half, before the waits
      float sc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      if (mine) {
        const __nv_bfloat16* sp4[4] = {sA, sA + s8, sB, sB + s8};
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
#pragma unroll
          for (int gi = 0; gi < 2; ++gi)
            sc[rr][gi] = 2 * s + gi < ngk ? __bfloat162float(sp4[rr][2 * s + gi]) : 0.f;
        refill();
      }
      cp_async_wait<1>();                    // this thread's copies of slab s have landed
      __syncthreads();                       // and everyone's: slab s's activations and shares are visible
      if (mine && !s_abort[warp] &&
          mbar_wait(&s_bar[warp][c_st], c_phase, wait_limit_ns, &s_abort[warp], 0x0203)) {
        const uint8_t* slabp = ring + c_st * kI4SlabBytes;
        const uint8_t* abuf = act + (size_t)b * kI4DActBytes;
#pragma unroll 1
        for (int gi = 0; gi < 2; ++gi) {
          if (2 * s + gi >= ngk) break;      // the slab's second half is TMA zero fill
          const uint4 a0 = *reinterpret_cast<const uint4*>(slabp + gq * 128 + gi * 64 + c * 16);
          const uint4 a1 = *reinterpret_cast<const uint4*>(slabp + (gq + 8) * 128 + gi * 64 + c * 16);
          const uint4 b0 = *reinterpret_cast<const uint4*>(slabp + (gq + 16) * 128 + gi * 64 + c * 16);
          const uint4 b1 = *reinterpret_cast<const uint4*>(slabp + (gq + 24) * 128 + gi * 64 + c * 16);
          // two halves of four 8-row chunks each (the weights are dequantised once per half: the group
          // partials of all eight chunks would not fit the registers beside the running sums)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            constexpr int HC = kI4DChunks / 2;
            float pA[HC][4], pB[HC][4];
#pragma unroll
            for (int ch = 0; ch < HC; ++ch)
#pragma unroll
              for (int i = 0; i < 4; ++i) { pA[ch][i] = 0.f; pB[ch][i] = 0.f; }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t qa0[4], qa1[4], qb0[4], qb1[4];
              offset_word_f16(u4get(a0, j), qa0);
              offset_word_f16(u4get(a1, j), qa1);
              offset_word_f16(u4get(b0, j), qb0);
              offset_word_f16(u4get(b1, j), qb1);
              const int q = gi * 16 + c * 4 + j;   // 16-byte chunk of the activation row
#pragma unroll
              for (int ch = 0; ch < HC; ++ch) {
                const int r = 8 * (hf * HC + ch) + gq;
                const uint4 xf = *reinterpret_cast<const uint4*>(abuf + r * 512 + dense_act_chunk(q, r) * 16);
                mma_f16_16816(pA[ch], qa0[0], qa1[0], qa0[1], qa1[1], xf.x, xf.y);
                mma_f16_16816(pA[ch], qa0[2], qa1[2], qa0[3], qa1[3], xf.z, xf.w);
                mma_f16_16816(pB[ch], qb0[0], qb1[0], qb0[1], qb1[1], xf.x, xf.y);
                mma_f16_16816(pB[ch], qb0[2], qb1[2], qb0[3], qb1[3], xf.z, xf.w);
              }
            }
            // offsets' share (columns = rows 8 ch + 2c, 8 ch + 2c + 1), then the weight rows' group scales
            const float s0 = gi ? sc[0][1] : sc[0][0], s1 = gi ? sc[1][1] : sc[1][0];
            const float s2 = gi ? sc[2][1] : sc[2][0], s3 = gi ? sc[3][1] : sc[3][0];
#pragma unroll
            for (int ch = 0; ch < HC; ++ch) {
              const int cc = hf * HC + ch;
              const float x0 = s_c[b][8 * cc + 2 * c][gi], x1 = s_c[b][8 * cc + 2 * c + 1][gi];
              tA[cc][0] = fmaf(pA[ch][0] - x0, s0, tA[cc][0]);
              tA[cc][1] = fmaf(pA[ch][1] - x1, s0, tA[cc][1]);
              tA[cc][2] = fmaf(pA[ch][2] - x0, s1, tA[cc][2]);
              tA[cc][3] = fmaf(pA[ch][3] - x1, s1, tA[cc][3]);
              tB[cc][0] = fmaf(pB[ch][0] - x0, s2, tB[cc][0]);
              tB[cc][1] = fmaf(pB[ch][1] - x1, s2, tB[cc][1]);
              tB[cc][2] = fmaf(pB[ch][2] - x0, s3, tB[cc][2]);
              tB[cc][3] = fmaf(pB[ch][3] - x1, s3, tB[cc][3]);
            }
          }
        }
        __syncwarp();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // slab reads done before TMA reuses it
        ++consumed;
        if (++c_st == kI4DStages) { c_st = 0; c_phase ^= 1u; }
      }
      // slab s + 1's shares into their buffer (its readers finished at slab s - 1)
      if (s + 1 < se && threadIdx.x < kI4DRows * 2) s_c[b ^ 1][threadIdx.x >> 1][threadIdx.x & 1] = cnext;
      __syncthreads();                       // buffer b is read by every warp before slab s + 2 refills it
    }
    cp_async_wait<0>();
    if (!mine || s_abort[warp]) continue;
    // partials of this slab range, in k_int4_stream's split layout, back from the scaled activations
    const int o0 = GLU ? ob * 16 : ob * 32;
    const int W = GLU ? 2 * p.N : p.N;
    const int sp = task % KS;
#pragma unroll
    for (int ch = 0; ch < kI4DChunks; ++ch) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = gq + (i >= 2 ? 8 : 0);
        const int n = r0 + 8 * ch + 2 * c + (i & 1);
        if (n < R) {
          float* prow = p.part + ((long long)sp * R + n) * W + o0;
          const float rs = xrs[n];
          if (GLU) {
            prow[m] = tA[ch][i] * rs;
            prow[p.N + m] = tB[ch][i] * rs;
          } else {
            prow[m] = tA[ch][i] * rs;
            prow[m + 16] = tB[ch][i] * rs;
          }
        }
      }
    }
  }
  // never leave the CTA with copies still landing in its shared memory
  cp_async_wait<0>();
  {
    volatile int dummy = 0;
    for (int i = consumed; i < issued; ++i)
      mbar_wait(&s_bar[warp][i % kI4DStages], (uint32_t)((i / kI4DStages) & 1), wait_limit_ns, &dummy, 0x0204);
  }
  __syncwarp();
}

// Split reduction of k_int4_stream: out[r, o] from the ksplit fp32 partials added
// in split order (gated: h = act(sum g) * (sum u); plain: y = sum).
template <bool GLU, int ACT>
__global__ void __launch_bounds__(256) k_int4_splitk_reduce(const float* __restrict__ part, int ksplit, long long R,
                                                            int N, __nv_bfloat16* __restrict__ out) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * N) return;
  const long long r = i / N;
  const int o = (int)(i - r * N);
  const int W = GLU ? 2 * N : N;
  float g = 0.f, u = 0.f;
  for (int sp = 0; sp < ksplit; ++sp) {
    const float* row = part + ((long long)sp * R + r) * W;
    g += row[o];
    if (GLU) u += row[N + o];
  }
  if (GLU) {
    const float a = ACT == kModeSwiGLU ? act_silu(g) : act_gelu(g);
    out[i] = __float2bfloat16_rn(a * u);
  } else {
    out[i] = __float2bfloat16_rn(g);
  }
}

}  // namespace moe
