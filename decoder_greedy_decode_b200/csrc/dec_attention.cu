// dec_attention.cu -- isolated split-K (flash-decoding) GQA decode attention.
//
// "Qwen3-ASR -- Latency & Bottleneck Analysis", 07 Root causes: the eager
// decode step spends ~10 launches per layer on attention (repeat_kv, QK^T,
// mask add, fp32 softmax, AV, transpose, contiguous) while the KV bytes alone
// would justify a fraction of the time.  Here one launch does all of it:
// every CTA takes a chunk of one (sequence, KV head) context, streams its K
// and V rows through shared memory with 1-D bulk copies, keeps an fp32 online
// softmax per query head of the group, and the last CTA of the (sequence, KV
// head) merges the chunks' partial states.  Up to 3 (head_dim 128) or 4
// (head_dim 64) query heads per KV head run the lane-octet kernel (4 rows per
// warp step); more run the one-row-per-warp kernel.  The Baseten Qwen3-ASR article
// (KV cache quantization) notes that decode attention is memory-bound: the
// roofline of this kernel is HBM bandwidth over the K/V bytes.
#include <cuda_runtime.h>

#include <mutex>

#include "dec.h"
#include "dec_internal.h"
#include "dec_ptx.cuh"
#include "dec_quant.cuh"

namespace dec {
namespace {

constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttStages = 4;
constexpr int kAttTileRows = 32;
constexpr int kAttMaxRep = 8;

template <int D>
__global__ void __launch_bounds__(kAttThreads) attention_kernel(const AttnArgs a) {
  constexpr int DL = D / 32;
  constexpr int kTileBytes = kAttTileRows * D * 2 * 2;  // K rows then V rows
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kAttStages * kTileBytes);
  float* merge = reinterpret_cast<float*>(full + kAttStages);  // [warps][rep][D+2]
  __shared__ int s_last;

  const int rep = a.Hq / a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ci = blockIdx.x % a.chunks_max;
  const int bg = blockIdx.x / a.chunks_max;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int len = a.lengths[b];
  if (len < 1 || len > a.max_len) {
    if (tid == 0 && ci == 0 && g == 0 && a.status) atomicOr(a.status, 1);
    return;
  }
  const int nchunk = (len + a.chunk_rows - 1) / a.chunk_rows;
  if (ci >= nchunk) return;
  const int j0 = ci * a.chunk_rows;
  const int j1 = min(j0 + a.chunk_rows, len);
  const int ntiles = (j1 - j0 + kAttTileRows - 1) / kAttTileRows;
  const size_t head_row0 = (static_cast<size_t>(b) * a.Hkv + g) * a.max_len;
  const uint16_t* kbase = a.k + head_row0 * D;
  const uint16_t* vbase = a.v + head_row0 * D;

  if (tid == 0) {
    for (int s = 0; s < kAttStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t) {
    const int j = j0 + t * kAttTileRows;
    const int nr = min(kAttTileRows, j1 - j);
    const uint32_t rb = static_cast<uint32_t>(nr) * D * 2;
    uint64_t* bar = &full[t % kAttStages];
    uint8_t* dst = ring + (t % kAttStages) * kTileBytes;
    mbar_arrive_expect_tx(bar, 2 * rb);
    bulk_g2s(dst, kbase + static_cast<size_t>(j) * D, rb, bar, pol);
    bulk_g2s(dst + kAttTileRows * D * 2, vbase + static_cast<size_t>(j) * D, rb, bar, pol);
  };
  if (tid == 0)
    for (int t = 0; t < ntiles && t < kAttStages; ++t) issue(t);

  const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  float qv[kAttMaxRep][DL], acc[kAttMaxRep][DL], m[kAttMaxRep], ls[kAttMaxRep];
#pragma unroll
  for (int h = 0; h < kAttMaxRep; ++h) {
    m[h] = -INFINITY;
    ls[h] = 0.f;
#pragma unroll
    for (int k = 0; k < DL; ++k) {
      acc[h][k] = 0.f;
      qv[h][k] = h < rep ? bf16_to_f(a.q[(static_cast<size_t>(b) * a.Hq + g * rep + h) * D +
                                         lane * DL + k]) * qscale
                         : 0.f;
    }
  }
  for (int t = 0; t < ntiles; ++t) {
    const int j = j0 + t * kAttTileRows;
    const int nr = min(kAttTileRows, j1 - j);
    // bounded wait: the copies always complete; the bound only guards the GPU
    {
      Spin1 sp;
      while (!mbar_test(&full[t % kAttStages], (t / kAttStages) & 1))
        if (sp.expired()) break;
    }
    const uint8_t* tb = ring + (t % kAttStages) * kTileBytes;
    for (int r = warp; r < nr; r += kAttWarps) {
      float kr[DL], vr[DL];
      const uint8_t* kp = tb + static_cast<size_t>(r) * D * 2 + lane * DL * 2;
      const uint8_t* vp = kp + kAttTileRows * D * 2;
      if (DL == 4) {
        const uint2 kw = *reinterpret_cast<const uint2*>(kp);
        const uint2 vw = *reinterpret_cast<const uint2*>(vp);
        kr[0] = bf16lo(kw.x); kr[1] = bf16hi(kw.x); kr[2] = bf16lo(kw.y); kr[3] = bf16hi(kw.y);
        vr[0] = bf16lo(vw.x); vr[1] = bf16hi(vw.x); vr[2] = bf16lo(vw.y); vr[3] = bf16hi(vw.y);
      } else {
        const uint32_t kw = *reinterpret_cast<const uint32_t*>(kp);
        const uint32_t vw = *reinterpret_cast<const uint32_t*>(vp);
        kr[0] = bf16lo(kw); kr[1] = bf16hi(kw);
        vr[0] = bf16lo(vw); vr[1] = bf16hi(vw);
      }
#pragma unroll
      for (int h = 0; h < kAttMaxRep; ++h) {
        if (h < rep) {
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < DL; ++k) s = fmaf(qv[h][k], kr[k], s);
          s = warp_sum(s);
          const float mn = fmaxf(m[h], s);
          const float al = exp2f(m[h] - mn);
          const float pe = exp2f(s - mn);
          ls[h] = ls[h] * al + pe;
#pragma unroll
          for (int k = 0; k < DL; ++k) acc[h][k] = fmaf(acc[h][k], al, pe * vr[k]);
          m[h] = mn;
        }
      }
    }
    __syncthreads();  // slot t % stages fully read
    if (tid == 0 && t + kAttStages < ntiles) issue(t + kAttStages);
  }
  // merge warps -> this chunk's partial (m in log2 units, l, unnormalised acc)
#pragma unroll
  for (int h = 0; h < kAttMaxRep; ++h) {
    if (h < rep) {
      float* mg = merge + (static_cast<size_t>(warp) * rep + h) * (D + 2);
#pragma unroll
      for (int k = 0; k < DL; ++k) mg[lane * DL + k] = acc[h][k];
      if (lane == 0) {
        mg[D] = m[h];
        mg[D + 1] = ls[h];
      }
    }
  }
  __syncthreads();
  for (int t = tid; t < rep * D; t += kAttThreads) {
    const int h = t / D, d = t % D;
    float M = -INFINITY;
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, merge[(w * rep + h) * (D + 2) + D]);
    float Ls = 0.f, A = 0.f;
    for (int w = 0; w < kAttWarps; ++w) {
      const float* mg = merge + (w * rep + h) * (D + 2);
      const float e = (mg[D] == -INFINITY) ? 0.f : exp2f(mg[D] - M);
      Ls += mg[D + 1] * e;
      A += mg[d] * e;
    }
    float* pp = a.part + ((static_cast<size_t>(b) * a.Hq + g * rep + h) * a.chunks_max + ci) * (D + 2);
    pp[d] = A;
    if (d == 0) {
      pp[D] = M;
      pp[D + 1] = Ls;
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(&a.cnt[b * a.Hkv + g], 1u);
    s_last = (old == static_cast<unsigned>(nchunk - 1));
    if (s_last) {
      atomicExch(&a.cnt[b * a.Hkv + g], 0u);
      __threadfence();
    }
  }
  __syncthreads();
  if (!s_last) return;
  for (int t = tid; t < rep * D; t += kAttThreads) {
    const int h = t / D, d = t % D;
    const float* pb = a.part + (static_cast<size_t>(b) * a.Hq + g * rep + h) * a.chunks_max * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < nchunk; ++c) M = fmaxf(M, __ldcg(pb + c * (D + 2) + D));
    float Ls = 0.f, A = 0.f;
    for (int c = 0; c < nchunk; ++c) {
      const float e = exp2f(__ldcg(pb + c * (D + 2) + D) - M);
      Ls += __ldcg(pb + c * (D + 2) + D + 1) * e;
      A += __ldcg(pb + c * (D + 2) + d) * e;
    }
    a.out[(static_cast<size_t>(b) * a.Hq + g * rep + h) * D + d] = A / Ls;
  }
}

// Lane-octet variant for up to 4 query heads per KV head: 8 warps, each
// taking 4 rows of a 32-row tile at once with 8 lanes per row (lane o holds
// elements [o*D/16, (o+1)*D/16) and the same span of the second half of the
// row: conflict-free 16-byte shared-memory reads; a dot product is 3
// shuffles), an fp32 online softmax per octet, merged at the end.  A CTA that
// holds a whole context writes the output directly.
constexpr int kOctWarps = 8;
constexpr int kOctThreads = kOctWarps * 32;
constexpr int kOctRows = kOctWarps * 4;  // rows of a tile

template <int D, int REP>
__global__ void __launch_bounds__(kOctThreads, 2) attention_octet(const AttnArgs a) {
  constexpr int HALF = D / 16;
  constexpr int RB = D * 2;                    // bytes per bf16 row
  constexpr int kHalfT = kOctRows * RB;        // K (or V) rows of one tile
  constexpr int kTile = 2 * kHalfT;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kAttStages * kTile);
  float* merge = reinterpret_cast<float*>(full + kAttStages);  // [warps][REP][D + 2]
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int oct = lane >> 3, o = lane & 7;
  const int ci = blockIdx.x % a.chunks_max;
  const int bg = blockIdx.x / a.chunks_max;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int len = a.lengths[b];
  if (len < 1 || len > a.max_len) {
    if (tid == 0 && ci == 0 && g == 0 && a.status) atomicOr(a.status, 1);
    return;
  }
  const int nchunk = (len + a.chunk_rows - 1) / a.chunk_rows;
  if (ci >= nchunk) return;
  const int j0 = ci * a.chunk_rows;
  const int j1 = min(j0 + a.chunk_rows, len);
  const int ntiles = (j1 - j0 + kOctRows - 1) / kOctRows;
  const size_t head_row0 = (static_cast<size_t>(b) * a.Hkv + g) * a.max_len;
  const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k + head_row0 * D);
  const uint8_t* vbase = reinterpret_cast<const uint8_t*>(a.v + head_row0 * D);

  if (tid == 0) {
    for (int s = 0; s < kAttStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t) {
    const int j = j0 + t * kOctRows;
    const int nr = min(kOctRows, j1 - j);
    const uint32_t rb = static_cast<uint32_t>(nr) * RB;
    uint64_t* bar = &full[t % kAttStages];
    uint8_t* dst = ring + (t % kAttStages) * kTile;
    mbar_arrive_expect_tx(bar, 2 * rb);
    bulk_g2s(dst, kbase + static_cast<size_t>(j) * RB, rb, bar, pol);
    bulk_g2s(dst + kHalfT, vbase + static_cast<size_t>(j) * RB, rb, bar, pol);
  };
  if (tid == 0)
    for (int t = 0; t < ntiles && t < kAttStages; ++t) issue(t);

  const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  float qv[REP][2][HALF], acc[REP][2][HALF], m[REP], ls[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) {
    m[h] = -INFINITY;
    ls[h] = 0.f;
    const uint16_t* qh = a.q + (static_cast<size_t>(b) * a.Hq + g * REP + h) * D;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int e = 0; e < HALF; ++e) {
        acc[h][i][e] = 0.f;
        qv[h][i][e] = bf16_to_f(qh[i * (D / 2) + o * HALF + e]) * qscale;
      }
  }
  auto span = [&](const uint8_t* row, int i, float (&x)[HALF]) {
    const uint8_t* pp = row + 2 * (i * (D / 2) + o * HALF);
    if constexpr (HALF == 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(pp);
      x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
      x[4] = bf16lo(w.z); x[5] = bf16hi(w.z); x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(pp);
      x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
    }
  };
  for (int t = 0; t < ntiles; ++t) {
    const int j = j0 + t * kOctRows;
    const int nr = min(kOctRows, j1 - j);
    {
      Spin1 sp;
      while (!mbar_test(&full[t % kAttStages], (t / kAttStages) & 1))
        if (sp.expired()) break;
    }
    const uint8_t* tb = ring + (t % kAttStages) * kTile;
    const int r = warp * 4 + oct;
    const bool valid = r < nr;  // every lane joins the shuffles; short rows are masked
    const uint8_t* krow = tb + static_cast<size_t>(valid ? r : 0) * RB;
    float s[REP];
#pragma unroll
    for (int h = 0; h < REP; ++h) s[h] = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float kx[HALF];
      span(krow, i, kx);
#pragma unroll
      for (int h = 0; h < REP; ++h)
#pragma unroll
        for (int e = 0; e < HALF; ++e) s[h] = fmaf(qv[h][i][e], kx[e], s[h]);
    }
#pragma unroll
    for (int sh = 4; sh > 0; sh >>= 1)
#pragma unroll
      for (int h = 0; h < REP; ++h) s[h] += __shfl_xor_sync(0xffffffffu, s[h], sh);
    if (valid) {
      float al[REP], p[REP];
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        const float mn = fmaxf(m[h], s[h]);
        al[h] = exp2f(m[h] - mn);
        p[h] = exp2f(s[h] - mn);
        ls[h] = ls[h] * al[h] + p[h];
        m[h] = mn;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float vx[HALF];
        span(krow + kHalfT, i, vx);
#pragma unroll
        for (int h = 0; h < REP; ++h)
#pragma unroll
          for (int e = 0; e < HALF; ++e) acc[h][i][e] = fmaf(acc[h][i][e], al[h], p[h] * vx[e]);
      }
    }
    __syncthreads();  // slot t % stages fully read
    if (tid == 0 && t + kAttStages < ntiles) issue(t + kAttStages);
  }
  // merge the four octets of the warp, then octet 0 writes the warp's state
#pragma unroll
  for (int sh = 8; sh <= 16; sh <<= 1) {
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], sh);
      const float lo = __shfl_xor_sync(0xffffffffu, ls[h], sh);
      const float mn = fmaxf(m[h], mo);
      const float e1 = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - mn);
      const float e2 = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
      ls[h] = ls[h] * e1 + lo * e2;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int e = 0; e < HALF; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[h][i][e], sh);
          acc[h][i][e] = acc[h][i][e] * e1 + ao * e2;
        }
      m[h] = mn;
    }
  }
  if (oct == 0) {
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      float* mg = merge + (static_cast<size_t>(warp) * REP + h) * (D + 2);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int e = 0; e < HALF; ++e) mg[i * (D / 2) + o * HALF + e] = acc[h][i][e];
      if (o == 0) {
        mg[D] = m[h];
        mg[D + 1] = ls[h];
      }
    }
  }
  __syncthreads();
  for (int t = tid; t < REP * D; t += kOctThreads) {
    const int h = t / D, d = t % D;
    float M = -INFINITY;
    for (int w = 0; w < kOctWarps; ++w) M = fmaxf(M, merge[(w * REP + h) * (D + 2) + D]);
    float Ls = 0.f, A = 0.f;
    for (int w = 0; w < kOctWarps; ++w) {
      const float* mg = merge + (w * REP + h) * (D + 2);
      const float e = (mg[D] == -INFINITY) ? 0.f : exp2f(mg[D] - M);
      Ls += mg[D + 1] * e;
      A += mg[d] * e;
    }
    if (nchunk == 1) {
      a.out[(static_cast<size_t>(b) * a.Hq + g * REP + h) * D + d] = A / Ls;
    } else {
      float* pp = a.part + ((static_cast<size_t>(b) * a.Hq + g * REP + h) * a.chunks_max + ci) * (D + 2);
      pp[d] = A;
      if (d == 0) {
        pp[D] = M;
        pp[D + 1] = Ls;
      }
    }
  }
  if (nchunk == 1) return;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned old = atomicAdd(&a.cnt[b * a.Hkv + g], 1u);
    s_last = (old == static_cast<unsigned>(nchunk - 1));
    if (s_last) {
      atomicExch(&a.cnt[b * a.Hkv + g], 0u);
      __threadfence();
    }
  }
  __syncthreads();
  if (!s_last) return;
  for (int t = tid; t < REP * D; t += kOctThreads) {
    const int h = t / D, d = t % D;
    const float* pb = a.part + (static_cast<size_t>(b) * a.Hq + g * REP + h) * a.chunks_max * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < nchunk; ++c) M = fmaxf(M, __ldcg(pb + c * (D + 2) + D));
    float Ls = 0.f, A = 0.f;
    for (int c = 0; c < nchunk; ++c) {
      const float e = exp2f(__ldcg(pb + c * (D + 2) + D) - M);
      Ls += __ldcg(pb + c * (D + 2) + D + 1) * e;
      A += __ldcg(pb + c * (D + 2) + d) * e;
    }
    a.out[(static_cast<size_t>(b) * a.Hq + g * REP + h) * D + d] = A / Ls;
  }
}

size_t octet_smem_bytes(int D, int rep) {
  return static_cast<size_t>(kAttStages) * kOctRows * D * 4 + kAttStages * sizeof(uint64_t) +
         static_cast<size_t>(kOctWarps) * rep * (D + 2) * sizeof(float);
}

template <int D, int REP>
cudaError_t launch_octet(const AttnArgs& a, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t set_err = cudaSuccess;
  const size_t smem = octet_smem_bytes(D, REP);
  std::call_once(once, [&] {
    set_err = cudaFuncSetAttribute(attention_octet<D, REP>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
  });
  if (set_err != cudaSuccess) return set_err;
  const dim3 grid(static_cast<unsigned>(a.B) * a.Hkv * a.chunks_max);
  attention_octet<D, REP><<<grid, kOctThreads, smem, s>>>(a);
  return cudaGetLastError();
}

// One warp per row: E4M3 codes and the fp32 row scale (the step kernel's
// append uses the same routine).
template <int D>
__global__ void quantize_kernel(const float* x, int rows, uint8_t* codes, float* scales) {
  constexpr int DL = D / 32;
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < rows; r += gridDim.x * warps) {
    float v[DL];
    uint8_t c[DL];
#pragma unroll
    for (int k = 0; k < DL; ++k) v[k] = x[static_cast<size_t>(r) * D + lane + 32 * k];
    const float sc = quantize_row_e4m3<DL>(v, c);
#pragma unroll
    for (int k = 0; k < DL; ++k) codes[static_cast<size_t>(r) * D + lane + 32 * k] = c[k];
    if (lane == 0) scales[r] = sc;
  }
}

}  // namespace

cudaError_t launch_quantize(const float* x, int rows, int dim, uint8_t* codes, float* scales,
                            cudaStream_t s) {
  const int threads = 256;
  long long blocks = (static_cast<long long>(rows) + 7) / 8;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  if (dim == 128) quantize_kernel<128><<<static_cast<int>(blocks), threads, 0, s>>>(x, rows, codes, scales);
  else if (dim == 64) quantize_kernel<64><<<static_cast<int>(blocks), threads, 0, s>>>(x, rows, codes, scales);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

size_t attention_smem_bytes(int D, int rep) {
  return static_cast<size_t>(kAttStages) * kAttTileRows * D * 4 + kAttStages * sizeof(uint64_t) +
         static_cast<size_t>(kAttWarps) * rep * (D + 2) * sizeof(float);
}

int attention_chunk_rows(int B, int Hkv, int max_len, int sms) {
  long long total = static_cast<long long>(B) * Hkv * max_len;
  long long target = 4LL * sms;
  long long c = (total + target - 1) / target;
  c = (c + kAttTileRows - 1) / kAttTileRows * kAttTileRows;
  if (c < kAttTileRows) c = kAttTileRows;
  if (c > 1024) c = 1024;
  return static_cast<int>(c);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  const int rep = a.Hq / a.Hkv;
  if (a.D == 128) {
    switch (rep) {
      case 1: return launch_octet<128, 1>(a, s);
      case 2: return launch_octet<128, 2>(a, s);
      case 3: return launch_octet<128, 3>(a, s);
      default: break;  // 4 heads of 128 would spill registers
    }
  } else if (a.D == 64) {
    switch (rep) {
      case 1: return launch_octet<64, 1>(a, s);
      case 2: return launch_octet<64, 2>(a, s);
      case 3: return launch_octet<64, 3>(a, s);
      case 4: return launch_octet<64, 4>(a, s);
      default: break;
    }
  }
  // 5..8 query heads per KV head: one row per warp step
  const size_t smem = attention_smem_bytes(a.D, rep);
  const dim3 grid(static_cast<unsigned>(a.B) * a.Hkv * a.chunks_max);
  cudaError_t e;
  if (a.D == 128) {
    e = cudaFuncSetAttribute(attention_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attention_kernel<128><<<grid, kAttThreads, smem, s>>>(a);
  } else if (a.D == 64) {
    e = cudaFuncSetAttribute(attention_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attention_kernel<64><<<grid, kAttThreads, smem, s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace dec

// ---------------------------------------------------------------------------
// dec_attention_noalloc: the same attention with its scratch in a fixed,
// library-owned device array instead of caller memory.
//
// The scratch holds what one call needs between its CTAs: the partial softmax
// state of every chunk and one arrival counter per (sequence, KV head).  It is
// a file-scope device array, so every GPU that loads the library holds it
// until the process exits, and every call on a device shares it.
using dec::AttnArgs;
using dec::attention_chunk_rows;
using dec::launch_attention;

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

size_t al256n(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" int dec_attention_noalloc(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                     const void* q, const void* k_cache, const void* v_cache,
                                     int max_len, const int32_t* lengths, float* out, int* status,
                                     void* stream) {
  if (!q || !k_cache || !v_cache || !lengths || !out) return DEC_ERR_NULL;
  if (batch < 1) return DEC_ERR_BATCH;
  if (head_dim != 64 && head_dim != 128) return DEC_ERR_SHAPE;
  if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads || n_q_heads / n_kv_heads > 8)
    return DEC_ERR_SHAPE;
  if (max_len < 1) return DEC_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return DEC_ERR_ALIGN;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DEC_ERR_DEVICE;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DEC_ERR_DEVICE;
  const int chunk_rows = attention_chunk_rows(batch, n_kv_heads, max_len, sms);
  const int chunks = (max_len + chunk_rows - 1) / chunk_rows;
  const size_t part_bytes =
      al256n(sizeof(float) * static_cast<size_t>(batch) * n_q_heads * chunks * (head_dim + 2));
  const size_t cnt_bytes = sizeof(unsigned) * static_cast<size_t>(batch) * n_kv_heads;
  if (part_bytes + cnt_bytes > kNoAllocScratchBytes) return DEC_ERR_TOO_LARGE;
  // once per device, with that device current: the device address of the array
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
        return DEC_ERR_DEVICE;
      g_noalloc_ptr[dev] = ptr;
    }
    base = g_noalloc_ptr[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* scratch = static_cast<uint8_t*>(base);
  // the array keeps the previous call's contents: the counters must start at zero
  if (cudaMemsetAsync(scratch + part_bytes, 0, cnt_bytes, st) != cudaSuccess) return DEC_ERR_CUDA;
  AttnArgs a{};
  a.B = batch;
  a.Hq = n_q_heads;
  a.Hkv = n_kv_heads;
  a.D = head_dim;
  a.max_len = max_len;
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k_cache);
  a.v = static_cast<const uint16_t*>(v_cache);
  a.lengths = lengths;
  a.out = out;
  a.chunk_rows = chunk_rows;
  a.chunks_max = chunks;
  a.part = reinterpret_cast<float*>(scratch);
  a.cnt = reinterpret_cast<unsigned*>(scratch + part_bytes);
  a.status = status;
  return launch_attention(a, st) == cudaSuccess ? DEC_OK : DEC_ERR_CUDA;
}
