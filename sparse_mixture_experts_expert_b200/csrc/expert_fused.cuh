// Fused routed expert FFN for narrow experts (hidden H = 128 or 256) on the
// 5th-generation tensor cores: per row tile of one expert,
//   h = act(x W1^T) * (x W3^T)   (gate/up, K = d)     -> h stays in shared memory
//   y = h W2^T                   (down, K = H, N = d) -> y in bf16
// MoEEvolve README "Architecture" (granular SwiGLU experts of hidden 256), the
// Kvasir worker's "3 mat-muls"; the ExpertMesh README names fused gate/up/down
// projections as its routed-expert kernel's optimisation path.
//
// Why: with H <= 256 a row tile's whole h (128 rows x H bf16 = 64 KB per CTA)
// fits in shared memory, so h never makes the HBM round trip between two
// launches, and the down projection reads its A operand from shared memory
// (no L2 traffic), leaving only the W2 chunks to stream.
//
// Work of one tile (a "job" is one accumulator of 128 rows x 256 fp32 columns
// per CTA; jobs alternate between two TMEM slots, so an epilogue overlaps the
// next job's MMAs):
//   gate/up jobs j = 0 .. H/128 - 1: hidden columns [128 j, 128 j + 128), the
//     gate and up slices side by side (TMEM columns 0-127 gate, 128-255 up),
//     reduction over d; the epilogue writes h = act(g) * u in bf16 straight
//     into the tcgen05 operand layout (K-major, 128-byte swizzle, one 16 KB
//     atom per 64 hidden columns) and signals "h half j ready";
//   down jobs c = 0 .. ceil(d/256) - 1: output columns [256 c, 256 c + 256),
//     A = h from shared memory, B = W2 chunks streamed by TMA; the first down
//     job waits for each h half before its k-steps over that half; the
//     epilogue writes y rows (masked to the group).
// h is rewritten only by the next tile's gate/up epilogue, which runs after
// that gate/up job's MMAs completed -- and so after every earlier MMA,
// including this tile's down jobs that read h.
//
// Roles as in k_grouped_gemm: warp 0 TMA producer, warp 1 MMA issuer (TMEM
// owner), warps 4-7 epilogue.  CTA pairs (CG = 2, clusters of 2): 256-row
// tiles; each CTA loads its own 128 rows of x and half of every B chunk (gate
// rows in CTA 0, up rows in CTA 1; W2 rows split in halves); the leader issues
// M = 256 MMAs whose A operand is each CTA's own x rows or h rows.  Both
// CTAs' epilogue warps publish "h ready" on the leader's barrier with
// cluster-scope release after fencing their h writes to the async proxy.
// Every wait is bounded.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

template <int H, int CG>
struct FusedCfg {
  static constexpr int kAtoms = H / 64;                          // h atoms of 128 rows x 64 columns
  static constexpr int kHBytes = kAtoms * kBM * 128;             // 16 KB per atom
  static constexpr int kABytes = kBM * kBK * 2;                  // x chunk: 128 rows x 64
  static constexpr int kBBytes = (CG == 2 ? 128 : 256) * kBK * 2;  // 256-row B chunk (a half per CTA of a pair)
  static constexpr int kSlotBytes = kABytes + kBBytes;           // gate/up stage; a down stage uses the B part
  static constexpr int kBudget = 219 * 1024 - 1024 - kHBytes - kEpiBytes;
  static constexpr int kStages = kBudget / kSlotBytes > 8 ? 8 : kBudget / kSlotBytes;
  static constexpr size_t kSmemBytes = 1024 + (size_t)kHBytes + (size_t)kStages * kSlotBytes + kEpiBytes;
  static_assert(kStages >= 2, "shared memory budget");
};

// p.K = d (gate/up reduction), p.N = d (down output columns), p.up_row0 = H.
template <int MODE, int H, int CG>
__global__ void __launch_bounds__(256, 1)
    k_expert_fused(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW13,
                   const __grid_constant__ CUtensorMap tmW2, const GemmParams p) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  using Cfg = FusedCfg<H, CG>;
  static_assert(H == 128 || H == 256, "fused expert hidden width");
  static_assert(MODE == kModeSwiGLU || MODE == kModeGeGLU, "gated experts");
  constexpr bool kPair = CG == 2;
  constexpr int TM = kBM * CG;
  constexpr int S = Cfg::kStages;
  constexpr int NGU = H / 128;             // gate/up jobs per tile
  constexpr int NKD = H / kBK;             // down k-steps
  constexpr uint32_t IDESC = idesc_bf16_f32(TM, 256);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* h_s = smem;                                     // [atoms][128 rows][128 B], swizzled
  uint8_t* ring = smem + Cfg::kHBytes;
  __shared__ __align__(8) uint64_t bar_full[S], bar_empty[S], bar_tfull[2], bar_tempty[2], bar_hready[NGU],
      bar_final;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_prefix[kMaxGroupsSmem + 1];
  __shared__ int s_gstart[kMaxGroupsSmem];
  __shared__ int s_grows[kMaxGroupsSmem];

  const int warp = warp_id(), lane = lane_id();
  const int crank = kPair ? (int)cluster_ctarank() : 0;   // 0 = leader of the pair
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int nk = (p.K + kBK - 1) / kBK;
  const int nd = (p.N + 255) / 256;        // down jobs per tile
  const int jobs = NGU + nd;
  const bool single = p.group_rows == nullptr;
  const int G = single ? 1 : p.n_groups;

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
    for (int a = 0; a < 2; ++a) { mbar_init(&bar_tfull[a], 1); mbar_init(&bar_tempty[a], kPair ? 8 : 128); }
    for (int j = 0; j < NGU; ++j) mbar_init(&bar_hready[j], kPair ? 8 : 4);   // one arrival per epilogue warp
    mbar_init(&bar_final, 1);
    s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW13);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(&s_tmem, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&s_tmem, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_all();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = s_tmem;
  const int total = s_prefix[G];

  auto locate = [&](int tile, int& g, long long& row0, int& rows_valid) {
    int lo = 0, hi = G - 1;  // last g with s_prefix[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const long long m_local = (long long)(tile - s_prefix[g]) * TM + (long long)crank * kBM;
    row0 = s_gstart[g] + m_local;
    rows_valid = (int)max(0ll, min((long long)kBM, (long long)s_grows[g] - m_local));
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool ok = true;
    for (int tile = unit; tile < total && ok && !__any_sync(0xffffffffu, s_abort); tile += n_units) {
      int g, rows_valid;
      long long row0;
      locate(tile, g, row0, rows_valid);
      for (int job = 0; job < jobs && ok; ++job) {
        const bool gu = job < NGU;
        const int steps = gu ? nk : NKD;
        for (int kb = 0; kb < steps; ++kb) {
          uint8_t* a_s = ring + (size_t)stage * Cfg::kSlotBytes;
          uint8_t* b_s = a_s + Cfg::kABytes;
          if (lane == 0) {
            ok = mbar_wait(&bar_empty[stage], phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0301);
            if (ok && crank == 0)
              mbar_arrive_expect_tx(&bar_full[stage], CG * (gu ? Cfg::kSlotBytes : Cfg::kBBytes));
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (lane == 0) {
            if (kPair) {
              const uint32_t fb = mapa_shared(smem_u32(&bar_full[stage]), 0);
              if (gu) {
                tma_load_2d_pair(a_s, &tmX, fb, kb * kBK, (int)row0);
                tma_load_3d_pair(b_s, &tmW13, fb, kb * kBK, (crank == 0 ? 0 : p.up_row0) + 128 * job, g);
              } else {
                tma_load_3d_pair(b_s, &tmW2, fb, kb * kBK, 256 * (job - NGU) + 128 * crank, g);
              }
            } else {
              if (gu) {
                tma_load_2d(a_s, &tmX, &bar_full[stage], kb * kBK, (int)row0);
                tma_load_3d(b_s, &tmW13, &bar_full[stage], kb * kBK, 128 * job, g);
                tma_load_3d(b_s + 128 * 128, &tmW13, &bar_full[stage], kb * kBK, p.up_row0 + 128 * job, g);
              } else {
                tma_load_3d(b_s, &tmW2, &bar_full[stage], kb * kBK, 256 * (job - NGU), g);
              }
            }
          }
          ++issued;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
      }
      __syncwarp();
    }
    // no copy may still be landing in shared memory when the CTA ends
    if (lane == 0 && crank == 0) {
      const int last = (int)(issued < S ? issued : (long long)S);
      for (int i = 1; i <= last; ++i) {
        const long long n = issued - i;
        volatile int dummy = 0;
        mbar_wait(&bar_full[(int)(n % S)], (uint32_t)((n / S) & 1), p.wait_limit_ns, &dummy, 0x0302);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader CTA)
    if (lane == 0 && crank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int slot = 0;
      uint32_t slot_phase = 0;
      uint32_t tile_par = 0;
      const uint32_t h_addr = smem_u32(h_s);
      bool ok = true;
      for (int tile = unit; tile < total && ok && !s_abort; tile += n_units, tile_par ^= 1u) {
        for (int job = 0; job < jobs && ok; ++job) {
          if (!mbar_wait(&bar_tempty[slot], slot_phase ^ 1u, p.wait_limit_ns, &s_abort, 0x0303)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(slot * 256);
          const bool gu = job < NGU;
          const int steps = gu ? nk : NKD;
          for (int kb = 0; kb < steps; ++kb) {
            if (!gu && job == NGU && (kb * kBK) % 128 == 0) {
              // first down job: h half (kb * 64 / 128) written by both CTAs' epilogues
              if (!mbar_wait_cluster(&bar_hready[(kb * kBK) / 128], tile_par, p.wait_limit_ns, &s_abort, 0x0304)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            if (!mbar_wait(&bar_full[stage], phase, p.wait_limit_ns, &s_abort, 0x0305)) { ok = false; break; }
            tc_fence_after();
            const uint32_t slot_addr = smem_u32(ring + (size_t)stage * Cfg::kSlotBytes);
            const uint32_t a_addr = gu ? slot_addr : h_addr + (uint32_t)kb * (kBM * 128);
            const uint32_t b_addr = slot_addr + Cfg::kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              if (kPair)
                tc_mma_bf16_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                                 (kb > 0 || kk > 0) ? 1u : 0u);
              else
                tc_mma_bf16(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                            (kb > 0 || kk > 0) ? 1u : 0u);
            }
            if (kPair) tc_commit_pair_mc(&bar_empty[stage], 0x3);
            else tc_commit(&bar_empty[stage]);
            if (++stage == S) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          if (kPair) tc_commit_pair_mc(&bar_tfull[slot], 0x3);
          else tc_commit(&bar_tfull[slot]);
          if (++slot == 2) { slot = 0; slot_phase ^= 1u; }
        }
      }
      if (kPair) tc_commit_pair(&bar_final);
      else tc_commit(&bar_final);
      volatile int dummy = 0;
      mbar_wait(&bar_final, 0, p.wait_limit_ns, &dummy, 0x0306);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;                  // TMEM lane quarter: rows q*32 .. q*32+31 of this CTA's tile
    const int row = q * 32 + lane;           // this thread's row (TMEM lane)
    __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(ring + (size_t)S * Cfg::kSlotBytes) + q * 32 * kEpiRow;
    uint8_t* h_row = h_s + (size_t)row * 128;
    const uint32_t sw = (uint32_t)(row & 7);
    int slot = 0;
    uint32_t slot_phase = 0;
    auto release_slot = [&](int a) {
      tc_fence_before();
      if (kPair) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bar_tempty[a]), 0));
      } else {
        mbar_arrive(&bar_tempty[a]);
      }
    };
    bool ok = true;
    for (int tile = unit; tile < total && ok && !s_abort; tile += n_units) {
      int g, rows_valid;
      long long row0;
      locate(tile, g, row0, rows_valid);
      for (int job = 0; job < jobs; ++job) {
        if (!mbar_wait(&bar_tfull[slot], slot_phase, p.wait_limit_ns, &s_abort, 0x0307)) { ok = false; break; }
        tc_fence_after();
        const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(slot * 256);
        if (job < NGU) {
          // h = act(g) * u for hidden columns [128 job, 128 job + 128), 32 per round, into the swizzled atoms
#pragma unroll 1
          for (int r = 0; r < 4; ++r) {
            uint32_t gv[2][16], uv[2][16];
            tmem_ld16(t_row + 32 * r, gv[0]);
            tmem_ld16(t_row + 32 * r + 16, gv[1]);
            tmem_ld16(t_row + 128 + 32 * r, uv[0]);
            tmem_ld16(t_row + 128 + 32 * r + 16, uv[1]);
            tmem_ld_wait();
            if (r == 3) release_slot(slot);
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(gv[i >> 3][(2 * i) & 15]);
              const float g1 = __uint_as_float(gv[i >> 3][(2 * i + 1) & 15]);
              const float u0 = __uint_as_float(uv[i >> 3][(2 * i) & 15]);
              const float u1 = __uint_as_float(uv[i >> 3][(2 * i + 1) & 15]);
              const float a0 = MODE == kModeSwiGLU ? act_silu(g0) : act_gelu(g0);
              const float a1 = MODE == kModeSwiGLU ? act_silu(g1) : act_gelu(g1);
              o[i] = pack_bf16x2(a0 * u0, a1 * u1);
            }
            // hidden column hc = 128 job + 32 r + 8 cc lives in atom hc / 64, 16-byte chunk (hc % 64) / 8
            const int hc0 = 128 * job + 32 * r;
            uint8_t* atom = h_row + (size_t)(hc0 / 64) * (kBM * 128);
            const uint32_t c0 = (uint32_t)((hc0 % 64) / 8);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              *reinterpret_cast<uint4*>(atom + (((c0 + cc) ^ sw) << 4)) =
                  make_uint4(o[4 * cc], o[4 * cc + 1], o[4 * cc + 2], o[4 * cc + 3]);
          }
          // publish this h half to the tensor core (async proxy) and to the leader's MMA issuer
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (kPair) mbar_arrive_cluster_release(mapa_shared(smem_u32(&bar_hready[job]), 0));
            else mbar_arrive(&bar_hready[job]);
          }
        } else {
          // y columns [256 c, 256 c + 256): 64 per round through the staging rows, coalesced row stores
          const int n0 = 256 * (job - NGU);
#pragma unroll 1
          for (int rd = 0; rd < 4; ++rd) {
            uint32_t v[4][16];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) tmem_ld16(t_row + rd * 64 + ch * 16, v[ch]);
            tmem_ld_wait();
            if (rd == 3) release_slot(slot);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t o[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = pack_bf16x2(__uint_as_float(v[ch][2 * i]), __uint_as_float(v[ch][2 * i + 1]));
              uint4* sp = reinterpret_cast<uint4*>(stg + lane * kEpiRow + ch * 16);
              sp[0] = make_uint4(o[0], o[1], o[2], o[3]);
              sp[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
            __syncwarp();
            const int cb = (lane & 7) * 8;
            const int col = n0 + rd * 64 + cb;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int rr = it * 4 + (lane >> 3);
              if (q * 32 + rr < rows_valid && col < p.N) {
                const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * kEpiRow + cb);
                *reinterpret_cast<uint4*>(p.out + (row0 + q * 32 + rr) * p.ldo + col) = val;
              }
            }
            __syncwarp();
          }
        }
        if (++slot == 2) { slot = 0; slot_phase ^= 1u; }
      }
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_all();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace moe
