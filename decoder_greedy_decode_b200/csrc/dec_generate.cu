// dec_generate.cu -- the device-side bookkeeping between the steps of an
// on-device decode loop (dec_generate): the host launches n steps back to
// back and reads nothing until the end.
//
// The faster-qwen-asr GB10 record (notes.configuration) feeds the emitted
// token back on the device; the Baseten article ("Minimizing host-to-device
// syncs") keeps the host out of the per-step path.  Between two steps one
// tiny kernel advances each sequence's position and retires a sequence once
// it has emitted the end-of-sequence token: from then on its position stays
// and its outputs are that token.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dec_internal.h"

namespace dec {
namespace {

__global__ void gen_reset_kernel(int* done, int batch) {
  const int b = threadIdx.x;
  if (b < batch) done[b] = 0;
}

// out: the ids the step just wrote (the next step's input tokens);
// pos: the positions it used (the next step's, once advanced).
__global__ void gen_advance_kernel(int32_t* out, int32_t* pos, int* done, int batch, int eos) {
  const int b = threadIdx.x;
  if (b >= batch) return;
  if (done[b]) {
    out[b] = eos;  // a retired sequence keeps emitting the end token
    return;
  }
  if (eos >= 0 && out[b] == eos) {
    done[b] = 1;  // this step emitted the end token: the position stays
    return;
  }
  pos[b] += 1;
}

}  // namespace

cudaError_t launch_gen_reset(int* done, int batch, cudaStream_t s) {
  gen_reset_kernel<<<1, 64, 0, s>>>(done, batch);
  return cudaGetLastError();
}

cudaError_t launch_gen_advance(int32_t* out, int32_t* pos, int* done, int batch, int eos,
                               cudaStream_t s) {
  gen_advance_kernel<<<1, 64, 0, s>>>(out, pos, done, batch, eos);
  return cudaGetLastError();
}

}  // namespace dec
