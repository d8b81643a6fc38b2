// Weight gradients of the expert and router projections (training: kieve-moe
// Features, the MoEEvolve README Architecture, MoEFFN.forward in moe_stream.py).
// Every one has the form
//   out[g][m][n] = sum over the rows r of group g of A[r][m] * B[r][n]   (fp32)
// with A and B row-major activations that share their rows: for expert e,
// dW13_e = [dg | du]_e^T x_e and dW2_e = dout_e^T (w h)_e over the expert's
// grouped rows; dW_r = dz^T x and the shared expert's over all tokens.  The
// reduction runs down the rows, so both operands are MN-major: TMA brings
// 64 rows x 64 columns boxes (128-byte rows, 128-byte swizzle) and the
// tcgen05 MMA reads them through MN-major descriptors (the 64-column blocks
// of a tile LBO = 8 KB apart, 8-row groups SBO = 1 KB apart) with the
// transpose bits of the instruction descriptor set.  One CTA per SM walks
// (group, m tile, n tile) tiles; the K loop of a tile covers its group's rows
// in 64-row steps.  Rows of a step past the group's end belong to the next
// group: the MMA warp zeroes them in shared memory (async-proxy fence after)
// and skips the 16-row slices that hold none of the group's rows.  A group
// without rows gets zeros.  A group of many rows (a hot expert) is reduced in
// fixed-size row chunks, each its own set of tiles writing a partial that
// k_wgrad_reduce adds in order, so that one expert's tiles do not outlast the
// rest of the grid.  Dense gradients with few tiles split their rows into
// chunks (one partial output each) that k_sum_splits adds in order.
// Boxes wholly past the last output row or column are not loaded; what their
// stage space holds reaches only accumulator rows and columns that are never
// stored.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace moe {

struct WgradParams {
  const int32_t* group_start;   // [G] first row of each group, or nullptr: group g = rows [g chunk, (g+1) chunk)
  const int32_t* group_rows;    // [G] (ignored when group_start is nullptr)
  int G;
  long long R;                  // rows of A and B (the split groups' bound)
  int chunk;
  int M, N;                     // output rows (columns of A) and columns (columns of B)
  float* out;                   // group g: out + g * out_stride, [M][N] row-major
  long long out_stride;
  unsigned long long wait_limit_ns;
  // groups (group_start given) of more than split_rows rows are reduced in split_rows-row chunks, one tile
  // set each, into partials part + slot * out_stride; split_list gets [count, then (group, first slot,
  // chunks) per split group] for k_wgrad_reduce.  split_rows 0: no splitting.
  int split_rows;
  float* part;
  int32_t* split_list;
};

constexpr int kWgBox = 64 * 128;   // one 64-row x 64-column bf16 box (8 KB)

template <int BN>
struct WgradCfg {
  static constexpr int kABytes = 2 * kWgBox;          // 128 output rows
  static constexpr int kBBytes = (BN / 64) * kWgBox;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiBytes = 4 * 32 * 36 * 4;   // four warps x 32 rows x 36 floats
  static constexpr int kBudget = 219 * 1024 - 1024 - kEpiBytes;
  static constexpr int kStages = kBudget / kStageBytes > 8 ? 8 : kBudget / kStageBytes;
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + kEpiBytes;
};

// MN-major operand, 128-byte swizzle: 64 contiguous elements per 128-byte row (one row per reduction index),
// 8-row groups 1024 bytes apart (SBO), 64-column blocks `lbo` bytes apart (LBO).
__device__ __forceinline__ uint64_t smem_desc_mn128(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);   // start address
  d |= (uint64_t)(lbo >> 4) << 16;            // leading byte offset: next 64-column block
  d |= (uint64_t)(1024 >> 4) << 32;           // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;                     // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                     // swizzle: 128B
  return d;
}

// kind::f16, D fp32, A and B bf16, both MN-major (transpose bits 15 and 16).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_mn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 15) | (1u << 16);
}

template <int BN>
__global__ void __launch_bounds__(256, 1)
    k_wgrad_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const WgradParams p) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  using Cfg = WgradCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr int NBOX = 2 + BN / 64;   // boxes per stage
  constexpr uint32_t IDESC = idesc_bf16_f32_mn(kBM, BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[S], bar_empty[S], bar_tfull[2], bar_tempty[2], bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_uprefix[kMaxGroupsSmem + 1];   // row chunks before group g
  __shared__ int s_pslot[kMaxGroupsSmem];         // first partial slot of a split group, -1 otherwise

  const int warp = warp_id(), lane = lane_id();
  const int mt = (p.M + kBM - 1) / kBM, nt = (p.N + BN - 1) / BN;
  const long long per_group = (long long)mt * nt;
  const bool grouped = p.group_start != nullptr;
  const int CH = grouped ? p.split_rows : 0;

  // chunk table (warp 2): chunks per group, their prefix, the partial slots; CTA 0 also lists the split groups
  if (warp == 2) {
    const int per = (p.G + 31) / 32;
    const int g0 = min(p.G, lane * per), g1 = min(p.G, g0 + per);
    int units = 0, slots = 0, nsplit = 0;
    for (int g = g0; g < g1; ++g) {
      const int rows = grouped ? p.group_rows[g] : 0;
      const int nc = (CH > 0 && rows > CH) ? (rows + CH - 1) / CH : 1;
      units += nc;
      if (nc > 1) { slots += nc; ++nsplit; }
    }
    int iu = units, is = slots, in = nsplit;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, iu, o), b = __shfl_up_sync(0xffffffffu, is, o);
      const int c = __shfl_up_sync(0xffffffffu, in, o);
      if (lane >= o) { iu += a; is += b; in += c; }
    }
    int u = iu - units, sl = is - slots, li = in - nsplit;
    for (int g = g0; g < g1; ++g) {
      const int rows = grouped ? p.group_rows[g] : 0;
      const int nc = (CH > 0 && rows > CH) ? (rows + CH - 1) / CH : 1;
      s_uprefix[g] = u;
      s_pslot[g] = nc > 1 ? sl : -1;
      if (nc > 1 && blockIdx.x == 0 && p.split_list != nullptr) {
        p.split_list[1 + 3 * li] = g;
        p.split_list[2 + 3 * li] = sl;
        p.split_list[3 + 3 * li] = nc;
        ++li;
      }
      u += nc;
      if (nc > 1) sl += nc;
    }
    if (lane == 31) {
      s_uprefix[p.G] = iu;
      if (blockIdx.x == 0 && p.split_list != nullptr) p.split_list[0] = in;
    }
  }

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&bar_full[s], 1); mbar_init(&bar_empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bar_tfull[a], 1); mbar_init(&bar_tempty[a], 128); }
    mbar_init(&bar_final, 1);
    s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const long long total = per_group * s_uprefix[p.G];

  // tile -> group, its rows [start, start + rows), output tile, origin (m0, n0)
  auto locate = [&](long long tile, int& g, long long& start, int& rows, int& m0, int& n0, float*& out) {
    const int unit = (int)(tile / per_group);
    const int rem = (int)(tile - (long long)unit * per_group);
    m0 = (rem / nt) * kBM;
    n0 = (rem % nt) * BN;
    int lo = 0, hi = p.G - 1;   // last g with s_uprefix[g] <= unit
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_uprefix[mid] <= unit) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int c = unit - s_uprefix[g];
    if (grouped) {
      const int all = p.group_rows[g];
      start = (long long)p.group_start[g] + (long long)c * CH;
      rows = s_pslot[g] < 0 ? all : min(CH, all - c * CH);
      out = s_pslot[g] < 0 ? p.out + (long long)g * p.out_stride : p.part + (long long)(s_pslot[g] + c) * p.out_stride;
    } else {
      start = (long long)g * p.chunk;
      rows = (int)max(0ll, min((long long)p.chunk, p.R - start));
      out = p.out + (long long)g * p.out_stride;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    for (long long tile = blockIdx.x; tile < total && !__any_sync(0xffffffffu, s_abort); tile += gridDim.x) {
      int g, rows, m0, n0;
      long long start;
      float* out;
      locate(tile, g, start, rows, m0, n0, out);
      const int nk = (rows + 63) / 64;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        uint8_t* a_s = smem + (size_t)stage * Cfg::kStageBytes;
        uint8_t* b_s = a_s + Cfg::kABytes;
        if (lane == 0) {
          ok = mbar_wait(&bar_empty[stage], phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0701);
          if (ok) {
            // boxes wholly past the last column are not loaded: they only feed accumulator rows / columns
            // that are never stored
            const int na = min(2, (p.M - m0 + 63) / 64), nb = min(BN / 64, (p.N - n0 + 63) / 64);
            mbar_arrive_expect_tx(&bar_full[stage], (uint32_t)(na + nb) * kWgBox);
            const int r0 = (int)(start + 64ll * kb);
            for (int i = 0; i < na; ++i) tma_load_2d(a_s + i * kWgBox, &tmA, &bar_full[stage], m0 + 64 * i, r0);
            for (int j = 0; j < nb; ++j) tma_load_2d(b_s + j * kWgBox, &tmB, &bar_full[stage], n0 + 64 * j, r0);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++issued;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      __syncwarp();
      if (!ok) break;
    }
    // no copy may still be landing in shared memory when the CTA ends
    if (lane == 0) {
      const int last = (int)(issued < S ? issued : (long long)S);
      for (int i = 1; i <= last; ++i) {
        const long long n = issued - i;
        volatile int dummy = 0;
        mbar_wait(&bar_full[(int)(n % S)], (uint32_t)((n / S) & 1), p.wait_limit_ns, &dummy, 0x0702);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (lane 0), tail zeroing (whole warp)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (long long tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      int g, rows, m0, n0;
      long long start;
      float* out;
      locate(tile, g, start, rows, m0, n0, out);
      const int nk = (rows + 63) / 64;
      if (lane == 0) ok = mbar_wait(&bar_tempty[acc], acc_phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0703);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < nk; ++kb) {
        if (lane == 0) ok = mbar_wait(&bar_full[stage], phase, p.wait_limit_ns, &s_abort, 0x0704);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st_s = smem + (size_t)stage * Cfg::kStageBytes;
        const int valid = min(64, rows - 64 * kb);
        const int used = (valid + 15) & ~15;          // rows the issued 16-row slices read
        if (valid < used) {
          // rows [valid, used) of every box hold the next group's rows (or the fill): zero them
          const int per_box = (used - valid) * 8;     // 16-byte words
          for (int w = lane; w < NBOX * per_box; w += 32) {
            const int b = w / per_box, o = w - b * per_box;
            *reinterpret_cast<uint4*>(st_s + b * kWgBox + valid * 128 + o * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t a_addr = smem_u32(st_s);
          const uint32_t b_addr = a_addr + Cfg::kABytes;
          for (int kk = 0; kk < used / 16; ++kk)
            tc_mma_bf16(d_tmem, smem_desc_mn128(a_addr + kk * 2048, kWgBox),
                        smem_desc_mn128(b_addr + kk * 2048, kWgBox), IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bar_empty[stage]);
        }
        __syncwarp();
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&bar_tfull[acc]);   // a group without rows: arrives at once, nothing accumulated
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) {
      // all issued MMAs complete before TMEM is released
      tc_commit(&bar_final);
      volatile int dummy = 0;
      mbar_wait(&bar_final, 0, p.wait_limit_ns, &dummy, 0x0705);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue: TMEM -> fp32 staging -> 128-byte row segments
    const int q = warp & 3;
    constexpr int FR = 36;
    float* fstg = reinterpret_cast<float*>(smem + (size_t)S * Cfg::kStageBytes) + q * 32 * FR;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (long long tile = blockIdx.x; tile < total && !s_abort; tile += gridDim.x) {
      int g, rows, m0, n0;
      long long start;
      float* out;
      locate(tile, g, start, rows, m0, n0, out);
      if (!mbar_wait(&bar_tfull[acc], acc_phase, p.wait_limit_ns, &s_abort, 0x0706)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[2][16];
        if (rows > 0) {
          tmem_ld16(t_row + c0, v[0]);
          tmem_ld16(t_row + c0 + 16, v[1]);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[0][i] = v[1][i] = 0u;
        }
        if (c0 + 32 >= BN) {   // the accumulator goes back to the MMA warp after its last load
          tc_fence_before();
          mbar_arrive(&bar_tempty[acc]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(fstg + lane * FR + h * 16 + i) =
                make_float4(__uint_as_float(v[h][i]), __uint_as_float(v[h][i + 1]), __uint_as_float(v[h][i + 2]),
                            __uint_as_float(v[h][i + 3]));
        __syncwarp();
        const int cb = (lane & 7) * 4;
        const int col = n0 + c0 + cb;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + (lane >> 3);
          const int m = m0 + q * 32 + rr;
          if (m < p.M && col < p.N)
            *reinterpret_cast<float4*>(out + (long long)m * p.N + col) =
                *reinterpret_cast<const float4*>(fstg + rr * FR + cb);
        }
        __syncwarp();
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// The split groups of k_wgrad_gemm: out[g] = sum over its chunks c (in order) of part[slot + c], fp32.  The list
// ([count, then (group, slot, chunks)]) comes from the GEMM; a grid-stride loop covers count x mn / 4 vectors.
__global__ void __launch_bounds__(256) k_wgrad_reduce(const float* __restrict__ part,
                                                      const int32_t* __restrict__ split_list, long long mn,
                                                      float* __restrict__ out) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long nv = mn / 4;
  const long long total = (long long)split_list[0] * nv;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long item = i / nv, v = i - item * nv;
    const int g = split_list[1 + 3 * item], slot = split_list[2 + 3 * item], nc = split_list[3 + 3 * item];
    float4 a = reinterpret_cast<const float4*>(part + (long long)slot * mn)[v];
    for (int c = 1; c < nc; ++c) {
      const float4 b = reinterpret_cast<const float4*>(part + (long long)(slot + c) * mn)[v];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    reinterpret_cast<float4*>(out + (long long)g * mn)[v] = a;
  }
}

// out[i] = sum over s < n_splits of part[s][i] (in order), fp32, i < n (a multiple of 4).
__global__ void __launch_bounds__(256) k_sum_splits(const float* __restrict__ part, int n_splits, long long n,
                                                    float* __restrict__ out) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 a = *reinterpret_cast<const float4*>(part + i);
  for (int s = 1; s < n_splits; ++s) {
    const float4 b = *reinterpret_cast<const float4*>(part + (long long)s * n + i);
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
  }
  *reinterpret_cast<float4*>(out + i) = a;
}

}  // namespace moe
