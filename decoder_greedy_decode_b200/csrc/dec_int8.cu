// dec_int8.cu -- per-row symmetric int8 quantisation of bf16 weights, for
// weight-only int8 decoding (faster-qwen-asr GB10 benchmark record,
// "cuda_graph_int8" entries: int8 weight-only text decoder and lm_head).
//
// Format: one fp32 scale per output row, scale = amax / 127 (IEEE fp32
// division), code = round-half-even(w / scale) (IEEE fp32 division), clamped
// to [-127, 127]; a row of zeros has scale 0 and codes 0.  The weight the
// step multiplies is code * scale.
//
// One warp per row: a pass for the row's amax, then a pass that writes the
// codes (the row is L1/L2 resident by then).  A one-time conversion, not on
// the decode path.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dec_internal.h"
#include "dec_ptx.cuh"

namespace dec {
namespace {

constexpr int kQuantWarps = 8;

__device__ __forceinline__ uint32_t code_of(float w, float scale) {
  float r = rintf(__fdiv_rn(w, scale));  // ties to even
  r = fminf(fmaxf(r, -127.f), 127.f);
  return static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu;
}

__device__ __forceinline__ uint32_t pack4(uint32_t w0, uint32_t w1, float scale) {
  return code_of(bf16lo(w0), scale) | (code_of(bf16hi(w0), scale) << 8) |
         (code_of(bf16lo(w1), scale) << 16) | (code_of(bf16hi(w1), scale) << 24);
}

__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_int8_kernel(const uint16_t* __restrict__ w, int rows, int cols,
                         int8_t* __restrict__ codes, float* __restrict__ scales) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kQuantWarps + warp;
  if (r >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + static_cast<size_t>(r) * cols);
  const int nv = cols >> 3;
  float amax = 0.f;
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = src[v];
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(q.x)), fabsf(bf16hi(q.x))),
                             fmaxf(fabsf(bf16lo(q.y)), fabsf(bf16hi(q.y)))));
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(q.z)), fabsf(bf16hi(q.z))),
                             fmaxf(fabsf(bf16lo(q.w)), fabsf(bf16hi(q.w)))));
  }
  amax = warp_max(amax);
  const float scale = amax == 0.f ? 0.f : __fdiv_rn(amax, 127.f);
  if (lane == 0) scales[r] = scale;
  uint2* dst = reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * cols);
  for (int v = lane; v < nv; v += 32) {
    if (scale == 0.f) {
      dst[v] = make_uint2(0u, 0u);
    } else {
      const uint4 q = src[v];
      dst[v] = make_uint2(pack4(q.x, q.y, scale), pack4(q.z, q.w, scale));
    }
  }
}

// Per-row E4M3 weight-only quantisation ("Qwen3-ASR -- Latency & Bottleneck
// Analysis", 08 Optimization roadmap: an fp8 lm_head): the per-row E4M3
// quantiser of the KV rows applied to the fp32 values of a bf16 weight row,
// scale = max(amax, 2^-126) / 448 (IEEE fp32 division), code = E4M3(w /
// scale) (IEEE fp32 division, round to nearest even, saturating).  The
// weight the step multiplies is e4m3(code) * scale.
__device__ __forceinline__ uint32_t e4m3_pair(float a, float b, float scale) {
  return f2_to_e4m3x2(__fdiv_rn(a, scale), __fdiv_rn(b, scale));
}

__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_fp8_kernel(const uint16_t* __restrict__ w, int rows, int cols,
                        uint8_t* __restrict__ codes, float* __restrict__ scales) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kQuantWarps + warp;
  if (r >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(w + static_cast<size_t>(r) * cols);
  const int nv = cols >> 3;
  float amax = 0.f;
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = src[v];
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(q.x)), fabsf(bf16hi(q.x))),
                             fmaxf(fabsf(bf16lo(q.y)), fabsf(bf16hi(q.y)))));
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16lo(q.z)), fabsf(bf16hi(q.z))),
                             fmaxf(fabsf(bf16lo(q.w)), fabsf(bf16hi(q.w)))));
  }
  amax = fmaxf(warp_max(amax), 1.17549435e-38f);  // 2^-126
  const float scale = __fdiv_rn(amax, 448.0f);
  if (lane == 0) scales[r] = scale;
  uint2* dst = reinterpret_cast<uint2*>(codes + static_cast<size_t>(r) * cols);
  for (int v = lane; v < nv; v += 32) {
    const uint4 q = src[v];
    const uint32_t lo = e4m3_pair(bf16lo(q.x), bf16hi(q.x), scale) |
                        (e4m3_pair(bf16lo(q.y), bf16hi(q.y), scale) << 16);
    const uint32_t hi = e4m3_pair(bf16lo(q.z), bf16hi(q.z), scale) |
                        (e4m3_pair(bf16lo(q.w), bf16hi(q.w), scale) << 16);
    dst[v] = make_uint2(lo, hi);
  }
}

}  // namespace

cudaError_t launch_quantize_fp8w(const uint16_t* w, int rows, int cols, uint8_t* codes,
                                 float* scales, cudaStream_t s) {
  const int grid = (rows + kQuantWarps - 1) / kQuantWarps;
  quantize_fp8_kernel<<<grid, kQuantWarps * 32, 0, s>>>(w, rows, cols, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int8(const uint16_t* w, int rows, int cols, int8_t* codes,
                                 float* scales, cudaStream_t s) {
  const int grid = (rows + kQuantWarps - 1) / kQuantWarps;
  quantize_int8_kernel<<<grid, kQuantWarps * 32, 0, s>>>(w, rows, cols, codes, scales);
  return cudaGetLastError();
}

}  // namespace dec
