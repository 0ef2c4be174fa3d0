// dec_rope.cuh -- sin/cos of the rotary angle, shared by the decode kernels.
//
// "Qwen3-ASR -- Latency & Bottleneck Analysis", 03 Decode (module table): the rotary
// embedding is computed in fp32.  The angle p * theta^(-2i/D) is an fp32
// product; its sine and cosine come from the routine below.
#pragma once

namespace dec {

// sin and cos of an fp32 rotary angle x (0 <= x < 2^16 * 2pi): Cody-Waite
// reduction by 2pi split into three fp32 parts (c1 has 8 significant bits,
// so k * c1 is exact for |k| < 2^16), then the fast hardware sin/cos on
// [-pi, pi], where its absolute error is about 2^-21.
__device__ __forceinline__ void rope_sincos(float x, float* sn, float* cs) {
  const float c1 = 6.28125f, c2 = 1.9353071693331003e-3f, c3 = 1.0253376273028358e-11f;
  const float k = rintf(x * 0.15915493667125702f);
  float r = fmaf(-k, c1, x);
  r = fmaf(-k, c2, r);
  r = fmaf(-k, c3, r);
  __sincosf(r, sn, cs);
}

}  // namespace dec
