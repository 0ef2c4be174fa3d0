// dec_quant.cuh -- FP8 (OCP E4M3) quantisation of one KV row held by a warp.
//
// The Baseten Qwen3-ASR article (KV cache quantization) stores the cache in
// FP8 and keeps the attention math in full precision.  The pages fix neither
// the FP8 variant nor the scale granularity; this library takes E4M3 with one
// fp32 scale per (layer, K/V, sequence, KV head, token):
//   scale = max(amax, 2^-126) / 448,  code_i = RNE-satfinite(x_i / scale),
// both divisions IEEE fp32, and the value attention reads back is
// code_i * scale.
#pragma once
#include "dec_ptx.cuh"

namespace dec {

// v[k] holds element lane + 32k of the row.  On return code[k] holds its E4M3
// code and v[k] the value the cache represents; returns the row scale.
template <int DL>
__device__ __forceinline__ float quantize_row_e4m3(float (&v)[DL], uint8_t (&code)[DL]) {
  float am = 0.f;
#pragma unroll
  for (int k = 0; k < DL; ++k) am = fmaxf(am, fabsf(v[k]));
  am = warp_max(am);
  am = fmaxf(am, 1.17549435e-38f);  // 2^-126
  const float sc = __fdiv_rn(am, 448.0f);
#pragma unroll
  for (int k = 0; k < DL; ++k) {
    const float q = __fdiv_rn(v[k], sc);
    code[k] = static_cast<uint8_t>(f2_to_e4m3x2(q, 0.f) & 0xFF);
    v[k] = e4m3x2_to_f2(static_cast<uint16_t>(code[k])).x * sc;
  }
  return sc;
}

}  // namespace dec
