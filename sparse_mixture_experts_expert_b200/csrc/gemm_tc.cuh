// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMA).
//
// out[rows of group g] = epilogue( A[rows of group g] . B_g^T )
//   GEMM 1 (gated): A = grouped tokens [R, d], B_g = w13[g] [2H, d]; the tile
//     loads H/..-wide slices of the gate rows W1 and of the up rows W3 side by
//     side, so one 128 x 256 fp32 accumulator holds g and u for 128 hidden
//     columns and the epilogue writes h = act(g) * u in bf16 (SwiGLU: SiLU;
//     GeGLU: exact-erf GELU).  MoEEvolve README "SwiGLU hidden 256",
//     kieve-moe "top-k GeGLU", the Kvasir worker's "3 mat-muls".
//   GEMM 2 (down): A = h [R, H], B_g = w2[g] [d, H], epilogue writes y in bf16.
//   Router screen: A = x [T, d], B = [W_hi | W_lo] [E, 2d] (the two bf16 terms
//     of W_r side by side); each k-step loads the A tile once and both terms'
//     B tiles, whose MMAs accumulate into one fp32 accumulator, so the 2d
//     products x_i W_hi[e,i] and x_i W_lo[e,i] are summed as one reduction;
//     the epilogue adds the bias and writes fp32 logits.
// The ExpertMesh README names a grouped GEMM with fused gate/up/down as the
// optimisation path of its routed-expert kernel; this is that GEMM for sm_100a.
//
// Structure: persistent CTAs (one per SM), 8 warps.
//   warp 0         TMA producer: A tile 128 x 64 and B tile N x 64 per stage
//                  (128-byte swizzle), ring of kStages stages.
//   warp 1         allocates 2 x BN TMEM columns; lane 0 issues tcgen05.mma
//                  (M=128, N=BN, K=16, bf16 -> fp32) and commits stages back.
//   warps 4..7     epilogue: tcgen05.ld of their 32 TMEM lanes, activation,
//                  bf16 rounding, masked row stores.  Two accumulators in
//                  TMEM let the epilogue of tile i overlap the MMAs of i+1.
// Tiles: for each group, ceil(rows/128) row tiles x ceil(N_out/cols) column
// tiles, enumerated from the device-side group table (no host sync).  Row tiles
// that run past a group's end read the next group's rows (or TMA zero fill);
// their outputs are masked.  Every wait is bounded.
//
// CTA-pair variant (CG = 2, launched as clusters of 2): the pair owns a tile of
// 256 rows x BN columns.  Each CTA loads its own 128 rows of A and half of the
// B tile (BN/2 rows: the gate slice in CTA 0 and the up slice in CTA 1 for the
// gated GEMM), both copies counting on the leader CTA's stage barrier; the
// leader issues one M = 256 MMA per k-step (tcgen05 cta_group::2), which reads
// both CTAs' shared memory and leaves each CTA's 128 x BN accumulator in that
// CTA's tensor memory.  Per CTA this moves (128 + BN/2) x 64 operand elements
// per k-step instead of (128 + BN) x 64 for the same MMA work, which is what
// bounds the single-CTA kernel (L2 -> SM bandwidth) for short reductions.
// Stage and accumulator releases are multicast commits to both CTAs; the
// epilogue warps of both CTAs release an accumulator on the leader's barrier.
#pragma once

#include "common.cuh"

namespace moe {

enum GemmMode { kModePlain = 0, kModeSwiGLU = 1, kModeGeGLU = 2, kModeScreen = 3 };

struct GemmParams {
  const int32_t* group_start;  // [n_groups] or nullptr (one group of R rows)
  const int32_t* group_rows;   // [n_groups] or nullptr
  int n_groups;
  long long R;
  int K;          // reduction length (screen: of A; B holds 2K columns)
  int N;          // output columns
  int up_row0;    // GLU: first row of the up half in B (= H)
  __nv_bfloat16* out;
  long long ldo;
  unsigned long long wait_limit_ns;
  float* out_f32;      // kModeScreen: fp32 output [R, N]
  const float* bias;   // kModeScreen: optional per-column bias [N]
};

#ifndef MOE_GEMM_MAX_STAGES
#define MOE_GEMM_MAX_STAGES 8   // TMA -> MMA ring depth cap (the shared-memory budget usually binds first)
#endif

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle atom of bf16
constexpr int kMaxGroupsSmem = 512;
constexpr int kEpiW = 64;                                   // columns staged per epilogue round
constexpr int kEpiRow = kEpiW + 8;                          // padded staging row (bf16), conflict-free
constexpr int kEpiBytes = 4 * 32 * kEpiRow * 2;             // four epilogue warps x 32 rows

template <int BN, int CG = 1, int NB = 1>   // NB: B tiles per k-step (2 for the router screen)
struct GemmCfg {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBox = (CG == 2 ? BN / 2 : BN) * kBK * 2;   // one B box, a whole number of 1 KB atoms
  static constexpr int kBBytes = kBBox * NB;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBudget = 219 * 1024 - 1024 - kEpiBytes;
  static constexpr int kStages = kBudget / kStageBytes > MOE_GEMM_MAX_STAGES ? MOE_GEMM_MAX_STAGES
                                                                            : kBudget / kStageBytes;
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);  // two accumulators, pow2
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + kEpiBytes;
};

// SiLU with the fast exponential and division: h is rounded to bf16 right after.
__device__ __forceinline__ float act_silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }
// erf by Abramowitz & Stegun, Handbook of Mathematical Functions, eq. 7.1.26 (rational-exponential
// approximation, |error| <= 1.5e-7 for the exact evaluation): a few ulps once evaluated in fp32, far below
// the bf16 rounding h receives right after.
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  const float t = __fdividef(1.0f, fmaf(0.3275911f, ax, 1.0f));
  const float poly =
      t * (0.254829592f + t * (-0.284496736f + t * (1.421413741f + t * (-1.453152027f + t * 1.061405429f))));
  return copysignf(1.0f - poly * __expf(-ax * ax), x);
}
__device__ __forceinline__ float act_gelu(float g) { return 0.5f * g * (1.0f + erf_as7126(g * 0.7071067811865476f)); }

template <int MODE, int BN, int CG = 1>
__global__ void __launch_bounds__(256, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  constexpr bool kScreen = MODE == kModeScreen;
  using Cfg = GemmCfg<BN, CG, kScreen ? 2 : 1>;
  constexpr bool kGLU = MODE == kModeSwiGLU || MODE == kModeGeGLU;
  constexpr bool kPair = CG == 2;
  constexpr int OUTN = kGLU ? BN / 2 : BN;  // output columns per tile
  constexpr int BOXB = kGLU ? BN / 2 : BN;  // rows per B box (single CTA)
  constexpr int TM = kBM * CG;              // rows per tile
  constexpr int S = Cfg::kStages;
  constexpr uint32_t IDESC = idesc_bf16_f32(TM, BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[S], bar_empty[S], bar_tfull[2], bar_tempty[2], bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_prefix[kMaxGroupsSmem + 1];
  __shared__ int s_gstart[kMaxGroupsSmem];
  __shared__ int s_grows[kMaxGroupsSmem];

  const int warp = warp_id(), lane = lane_id();
  const int crank = kPair ? (int)cluster_ctarank() : 0;   // 0 = leader of the pair
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int n_tiles = (p.N + OUTN - 1) / OUTN;
  const int nk = (p.K + kBK - 1) / kBK;
  const bool single = p.group_rows == nullptr;
  const int G = single ? 1 : p.n_groups;

  // group row-tile prefix (warp 2), barriers (warp 0), TMEM (warp 1)
  if (warp == 2) {
    const int per = (G + 31) / 32;
    const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
      const long long rows = single ? p.R : (long long)p.group_rows[g];
      local += (int)((rows + TM - 1) / TM);
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
      s_prefix[g] = run;
      const long long rows = single ? p.R : (long long)p.group_rows[g];
      s_grows[g] = (int)rows;
      s_gstart[g] = single ? 0 : p.group_start[g];
      run += (int)((rows + TM - 1) / TM);
    }
    if (lane == 31) s_prefix[G] = incl;
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&bar_full[s], 1); mbar_init(&bar_empty[s], 1); }
    // accumulator release: 128 epilogue threads, or (pair) one arrival per epilogue warp of both CTAs
    for (int a = 0; a < 2; ++a) { mbar_init(&bar_tfull[a], 1); mbar_init(&bar_tempty[a], kPair ? 8 : 128); }
    mbar_init(&bar_final, 1);
    s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&s_tmem, Cfg::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s_tmem, Cfg::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_all();  // both CTAs' barriers initialised before any cross-CTA arrival
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const int total_m = s_prefix[G];
  const long long total = (long long)total_m * n_tiles;

  auto locate = [&](long long tile, int& g, long long& row0, int& rows_valid, int& n0) {
    const int mt = (int)(tile / n_tiles);
    const int nt = (int)(tile - (long long)mt * n_tiles);
    int lo = 0, hi = G - 1;  // last g with s_prefix[g] <= mt
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const long long m_local = (long long)(mt - s_prefix[g]) * TM + (long long)crank * kBM;
    const long long start = s_gstart[g];
    const long long rows = s_grows[g];
    row0 = start + m_local;   // this CTA's first row
    rows_valid = (int)max(0ll, min((long long)kBM, rows - m_local));
    n0 = nt * OUTN;
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    // The whole warp walks the tiles; lane 0 waits, arms the barriers and issues the copies.
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    for (long long tile = unit; tile < total && !__any_sync(0xffffffffu, s_abort); tile += n_units) {
      int g, rows_valid, n0;
      long long row0;
      locate(tile, g, row0, rows_valid, n0);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        uint8_t* a_s = smem + (size_t)stage * Cfg::kStageBytes;
        uint8_t* b_s = a_s + Cfg::kABytes;
        if (lane == 0) {
          ok = mbar_wait(&bar_empty[stage], phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0101);
          // the leader's barrier counts the bytes of both CTAs of a pair
          if (ok && crank == 0) mbar_arrive_expect_tx(&bar_full[stage], CG * Cfg::kStageBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (kPair) {
          if (lane == 0) {
            const uint32_t fb = mapa_shared(smem_u32(&bar_full[stage]), 0);
            tma_load_2d_pair(a_s, &tmA, fb, kb * kBK, (int)row0);
            const int brow = kGLU ? (crank == 0 ? n0 : p.up_row0 + n0) : n0 + crank * (BN / 2);
            tma_load_3d_pair(b_s, &tmB, fb, kb * kBK, brow, g);
            if (kScreen) tma_load_3d_pair(b_s + Cfg::kBBox, &tmB, fb, p.K + kb * kBK, brow, g);
          }
        } else if (lane == 0) {
          tma_load_2d(a_s, &tmA, &bar_full[stage], kb * kBK, (int)row0);
          if (kGLU) {
            tma_load_3d(b_s, &tmB, &bar_full[stage], kb * kBK, n0, g);
            tma_load_3d(b_s + BOXB * 128, &tmB, &bar_full[stage], kb * kBK, p.up_row0 + n0, g);
          } else {
            tma_load_3d(b_s, &tmB, &bar_full[stage], kb * kBK, n0, g);
            if (kScreen) tma_load_3d(b_s + Cfg::kBBox, &tmB, &bar_full[stage], p.K + kb * kBK, n0, g);
          }
        }
        ++issued;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      __syncwarp();
      if (!ok) break;
    }
    // Make sure no copy is still landing in shared memory when the CTA ends (in a
    // pair the leader's barriers count both CTAs' copies; the pair leaves together).
    if (lane == 0 && crank == 0) {
      const int last = (int)(issued < S ? issued : (long long)S);
      for (int i = 1; i <= last; ++i) {
        const long long n = issued - i;
        const int st = (int)(n % S);
        const uint32_t ph = (uint32_t)((n / S) & 1);
        volatile int dummy = 0;
        mbar_wait(&bar_full[st], ph, p.wait_limit_ns, &dummy, 0x0102);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0 && crank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (long long tile = unit; tile < total && !s_abort; tile += n_units) {
        if (!mbar_wait(&bar_tempty[acc], acc_phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0103)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&bar_full[stage], phase, p.wait_limit_ns, &s_abort, 0x0104)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)stage * Cfg::kStageBytes);
          const uint32_t b_addr = a_addr + Cfg::kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            if (kPair)
              tc_mma_bf16_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                               (kb > 0 || kk > 0) ? 1u : 0u);
            else
              tc_mma_bf16(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                          (kb > 0 || kk > 0) ? 1u : 0u);
            if (kScreen) {   // the second term of W_r, same A tile, same accumulator
              const uint32_t b2 = b_addr + Cfg::kBBox + kk * 32;
              if (kPair) tc_mma_bf16_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b2), IDESC, 1u);
              else tc_mma_bf16(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b2), IDESC, 1u);
            }
          }
          if (kPair) tc_commit_pair_mc(&bar_empty[stage], 0x3);
          else tc_commit(&bar_empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (kPair) tc_commit_pair_mc(&bar_tfull[acc], 0x3);
        else tc_commit(&bar_tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // all issued MMAs complete before TMEM is released
      if (kPair) tc_commit_pair(&bar_final);
      else tc_commit(&bar_final);
      volatile int dummy = 0;
      mbar_wait(&bar_final, 0, p.wait_limit_ns, &dummy, 0x0105);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    // TMEM -> registers -> activation / bf16 -> per-warp staging rows in shared
    // memory -> coalesced row-segment stores (128 contiguous bytes per row per
    // 8 lanes).  The accumulator is handed back to the MMA warp as soon as its
    // last TMEM load has completed.
    const int q = warp & 3;  // TMEM lane quarter: this warp's 32 accumulator rows
    constexpr int OUTW = OUTN < kEpiW ? OUTN : kEpiW;
    constexpr int ROUNDS = OUTN / OUTW;
    constexpr int LPR = OUTW / 8;   // lanes per staged row in the copy-out
    constexpr int RPI = 32 / LPR;   // rows per copy-out iteration
    __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem + (size_t)S * Cfg::kStageBytes) + q * 32 * kEpiRow;
    int acc = 0;
    uint32_t acc_phase = 0;
    // accumulator release: each thread (single CTA) or each warp on the leader's barrier (pair)
    auto release_acc = [&](int a) {
      tc_fence_before();
      if (kPair) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bar_tempty[a]), 0));
      } else {
        mbar_arrive(&bar_tempty[a]);
      }
    };
    for (long long tile = unit; tile < total && !s_abort; tile += n_units) {
      int g, rows_valid, n0;
      long long row0;
      locate(tile, g, row0, rows_valid, n0);
      if (!mbar_wait(&bar_tfull[acc], acc_phase, p.wait_limit_ns, &s_abort, 0x0106)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if (kScreen) {
        // fp32 rows through the staging buffer, 32 columns (128 bytes per row) per round
        float* fstg = reinterpret_cast<float*>(stg);  // 32 rows x 36 floats per warp
        constexpr int FR = 36;
#pragma unroll 1
        for (int c0 = 0; c0 < OUTN; c0 += 32) {
          uint32_t v[2][16];
          tmem_ld16(t_row + c0, v[0]);
          tmem_ld16(t_row + c0 + 16, v[1]);
          tmem_ld_wait();
          if (c0 + 32 >= OUTN) release_acc(acc);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              float4 f;
              const int col = n0 + c0 + h * 16 + i;
              f.x = __uint_as_float(v[h][i]) + (p.bias != nullptr && col + 0 < p.N ? p.bias[col + 0] : 0.f);
              f.y = __uint_as_float(v[h][i + 1]) + (p.bias != nullptr && col + 1 < p.N ? p.bias[col + 1] : 0.f);
              f.z = __uint_as_float(v[h][i + 2]) + (p.bias != nullptr && col + 2 < p.N ? p.bias[col + 2] : 0.f);
              f.w = __uint_as_float(v[h][i + 3]) + (p.bias != nullptr && col + 3 < p.N ? p.bias[col + 3] : 0.f);
              *reinterpret_cast<float4*>(fstg + lane * FR + h * 16 + i) = f;
            }
          }
          __syncwarp();
          // 8 lanes per 128-byte row segment, 4 rows per step
          const int cb = (lane & 7) * 4;
          const int col = n0 + c0 + cb;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + (lane >> 3);
            if (q * 32 + rr < rows_valid && col < p.N) {
              const float4 val = *reinterpret_cast<const float4*>(fstg + rr * FR + cb);
              *reinterpret_cast<float4*>(p.out_f32 + (row0 + q * 32 + rr) * p.ldo + col) = val;
            }
          }
          __syncwarp();
        }
      } else {
#pragma unroll 1
        for (int rd = 0; rd < ROUNDS; ++rd) {
          // all TMEM loads of the round are issued before one wait
          constexpr int NCH = OUTW / 16;
          uint32_t v[NCH][16];
          uint32_t u[kGLU ? NCH : 1][16];
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            tmem_ld16(t_row + rd * OUTW + ch * 16, v[ch]);
            if (kGLU) tmem_ld16(t_row + OUTN + rd * OUTW + ch * 16, u[kGLU ? ch : 0]);
          }
          tmem_ld_wait();
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (kGLU) {
                const float g0 = __uint_as_float(v[ch][2 * i]), g1 = __uint_as_float(v[ch][2 * i + 1]);
                const float u0 = __uint_as_float(u[kGLU ? ch : 0][2 * i]);
                const float u1 = __uint_as_float(u[kGLU ? ch : 0][2 * i + 1]);
                const float a0 = MODE == kModeSwiGLU ? act_silu(g0) : act_gelu(g0);
                const float a1 = MODE == kModeSwiGLU ? act_silu(g1) : act_gelu(g1);
                o[i] = pack_bf16x2(a0 * u0, a1 * u1);
              } else {
                o[i] = pack_bf16x2(__uint_as_float(v[ch][2 * i]), __uint_as_float(v[ch][2 * i + 1]));
              }
            }
            uint4* sp = reinterpret_cast<uint4*>(stg + lane * kEpiRow + ch * 16);
            sp[0] = make_uint4(o[0], o[1], o[2], o[3]);
            sp[1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
          if (rd == ROUNDS - 1) release_acc(acc);
          __syncwarp();
          const int cb = (lane % LPR) * 8;
          const int col = n0 + rd * OUTW + cb;
#pragma unroll
          for (int it = 0; it < 32 / RPI; ++it) {
            const int rr = it * RPI + lane / LPR;
            if (q * 32 + rr < rows_valid && col < p.N) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * kEpiRow + cb);
              *reinterpret_cast<uint4*>(p.out + (row0 + q * 32 + rr) * p.ldo + col) = val;
            }
          }
          __syncwarp();
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_all();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    else tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace moe
