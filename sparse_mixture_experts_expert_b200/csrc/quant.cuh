// Group-scaled signed INT4 quantiser (ExpertMesh README: "A HIP routed-expert
// correctness kernel for group-scaled signed INT4 weights"; scales are bf16,
// one per 128 consecutive inputs of an output row).
//   s = bf16_rn(max|w_g| / 7), q = clamp(rint(w / s), -8, 7), q = 0 when s == 0.
// All decisions in fp32 with IEEE division, so the codes are reproducible.
#pragma once

#include "common.cuh"

namespace moe {

// One warp per (row, 128-input group); lane l owns inputs 4l .. 4l+3.
__global__ void __launch_bounds__(256) k_quantize_int4(const float* __restrict__ w, long long rows, int K,
                                                       uint8_t* __restrict__ q, __nv_bfloat16* __restrict__ scales) {
  pdl_wait();  // inputs written by the previous kernel on the stream are visible past this point
  const int groups = K / 128;
  const long long item = (long long)blockIdx.x * 8 + warp_id();
  if (item >= rows * groups) return;
  const long long row = item / groups;
  const int g = (int)(item - row * groups);
  const int lane = lane_id();
  const float4 v = reinterpret_cast<const float4*>(w + row * K + (long long)g * 128)[lane];
  float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __nv_bfloat16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
  const float s = __bfloat162float(sb);
  auto code = [&](float x) -> uint32_t {
    if (s == 0.0f) return 0u;
    float r = rintf(__fdiv_rn(x, s));
    r = fminf(fmaxf(r, -8.0f), 7.0f);
    return (uint32_t)((int)r & 0xF);
  };
  const uint32_t b0 = code(v.x) | (code(v.y) << 4);
  const uint32_t b1 = code(v.z) | (code(v.w) << 4);
  reinterpret_cast<uint16_t*>(q + row * (K / 2) + (long long)g * 64)[lane] = (uint16_t)(b0 | (b1 << 8));
  if (lane == 0) scales[row * groups + g] = sb;
}

}  // namespace moe
