// dec_step_small.cu -- persistent decode-step kernel for batch 1..4 (GEMV path).
//
// One cooperative launch runs the whole step of "Qwen3-ASR -- Latency &
// Bottleneck Analysis", 03 Decode: embed, 28 x [RMSNorm, QKV, q/k norm, RoPE,
// KV append, GQA attention, o_proj + residual, RMSNorm, gate/up, SiLU*up,
// down + residual], final norm, lm_head, argmax.  The page finds the eager
// step launch-bound (~300 attention kernels per token, 07 Root causes); here
// there is one launch per step and no host involvement inside it.
//
// Structure (one CTA per SM, 8 consumer warps + 1 producer warp):
//  * Every weight and KV byte the CTA will need is known before the step
//    starts, independent of activations.  The producer warp streams them with
//    1-D bulk copies (TMA engine) into a ring of 24 KB shared-memory slots,
//    running up to a whole ring (~170 KB, most of one layer's share) ahead of
//    the consumers.  HBM therefore keeps streaming while consumers wait for
//    activations.
//  * Activations move between CTAs as 8-byte words {fp32 value, 32-bit flag}
//    in global memory (L2).  A consumer polls the words it needs until their
//    flags equal the expected (step, layer) tag: data and readiness arrive
//    in one load, with no separate barrier round trip.
//  * Rows of every projection are split evenly over CTAs; each CTA owns the
//    same hidden rows in o_proj and down, so it keeps those residual entries
//    in shared memory.  Inside a CTA the K dimension of a projection is split
//    over the consumer warps in blocks of 128 columns: each warp polls only
//    the input words of its own blocks and computes its partial dot products
//    as soon as they are there, so the arrival skew of the producing CTAs
//    overlaps the arithmetic.  One CTA barrier per projection then sums the
//    warps' partials in a fixed order (deterministic) and applies the RMSNorm
//    factor of the input, computed from the warps' partial sums of squares:
//    W (g * x * s) = s * W (g * x).
//  * Attention is split-K over (sequence, KV head, chunk) items; every lane
//    octet scores a cached row against all query heads of its head group
//    (each K/V row is read once per group); the CTA of chunk 0 of a
//    (sequence, KV head) gathers the other chunks' partials as they are
//    published, merges them (flash-decoding combine) and publishes the head
//    outputs.
//  * Every wait is bounded (globaltimer).  A wait that runs out raises a
//    status bit and a global abort flag; all CTAs then drain their in-flight
//    copies without computing and leave; out_ids becomes -1.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dec_internal.h"
#include "dec_ptx.cuh"
#include "dec_quant.cuh"
#include "dec_rope.cuh"

namespace dec {
namespace {

constexpr int kCW = kConsumerWarps;
constexpr int kCT = kConsumerThreads;
constexpr int kMaxHRows = 64;  // hidden rows a CTA may own
constexpr int kDevTimeout = 4;
constexpr int kDevBadPos = 1;
constexpr int kDevBadTok = 2;
constexpr int kBlk = 128;                      // columns of one K block
constexpr int kWarpStage = 384;                // tagged words a warp stages per poll round
constexpr int kStageWords = kCW * kWarpStage;  // whole staging buffer (CTA-wide gathers)
constexpr int kMaxGainBlk = 6;                 // K blocks per warp of a normalised input (H <= 6144)
// bf16 projection rows sit in the ring kRowPad bytes apart beyond their
// length, so that the 8 rows an 8x8 matrix load touches fall in different
// banks (row stride = 16 mod 128 bytes); the activation planes likewise.
constexpr int kRowPad = 16;

// Stages of one layer; the lm_head runs as stage SQ of layer L (code SLM).
enum { SQ = 0, SA, SO, SU, SD, kStages, SLM = kStages };

// Optional per-phase timestamps (profiling builds only, -DDEC_PROFILE): thread
// 0 of every CTA records globaltimer at the phase boundaries of the step into
// prof[cta][kStampsPerLayer * L + 8] at the points named by the St* indices
// below (per layer), then lm_head start / gathered / done, consumer end and
// consumer start.
[[maybe_unused]] constexpr int kStampsPerLayer = kProfStampsPerLayer;
enum {
  StAttTile = 0, StQIn, StQDot, StQkv, StAttIn, StAttRows, StAtt, StOIn, StO, StUIn, StUDot,
  StU, StDIn, StD, StODot, StDDot,
  // the producer's issue time of the first tile of each stage
  StPQ, StPA, StPO, StPU, StPD,
  // SM cycles warp 0 spent waiting for ring tiles in each stage
  StWQ, StWA, StWO, StWU, StWD,
  // SM cycles of warp 0's GEMV of each stage (waits included)
  StCQ, StCO, StCU, StCD,
  // attention: partial state published (other chunks) / chunks gathered (chunk 0)
  StAttPub, StAttCmb
};
static_assert(StAttCmb < kStampsPerLayer, "profiling stamps of a layer");
enum { StLmStart = 0, StLmGath, StLmDone, StEnd, StBegin };
#ifdef DEC_PROFILE
#define DEC_STAMP(i)                                                                   \
  do {                                                                                 \
    if (a.prof && tid == 0)                                                            \
      a.prof[static_cast<size_t>(cta) * (kStampsPerLayer * a.L + 8) + (i)] = globaltimer(); \
  } while (0)
// the producer lane's stamps, and a stored value instead of a time
#define DEC_PSTAMP(i)                                                                  \
  do {                                                                                 \
    if (a.prof)                                                                        \
      a.prof[static_cast<size_t>(cta) * (kStampsPerLayer * a.L + 8) + (i)] = globaltimer(); \
  } while (0)
#define DEC_SVAL(i, v)                                                                 \
  do {                                                                                 \
    if (a.prof && tid == 0) a.prof[static_cast<size_t>(cta) * (kStampsPerLayer * a.L + 8) + (i)] = (v); \
  } while (0)
#else
#define DEC_STAMP(i) \
  do {               \
  } while (0)
#define DEC_PSTAMP(i) \
  do {                \
  } while (0)
#define DEC_SVAL(i, v) \
  do {                 \
  } while (0)
#endif

__host__ __device__ inline int split_at(int n, int parts, int i) {
  return static_cast<int>((static_cast<long long>(n) * i) / parts);
}

constexpr int kMaxLayers = 64;  // layer pointer table kept in shared memory
// Fewer, longer attention chunks keep the combine to one round of loads.
constexpr int kMinChunkRows = 96;

// The sequences of the current step and its attention work split: items
// (b, g, chunk) over contexts 0..p_b, chunk rows `crow`.  The consumers and
// the producer each keep their own copy (they reach a step at different
// times) and compute it identically.
struct Plan {
  int crow, n_items, all_done, bad;
  int nchunk[kMaxBatchSmall], pos[kMaxBatchSmall], tok[kMaxBatchSmall], done[kMaxBatchSmall];
};

struct Carve {
  size_t ring, bars, act, stg, xown, part, bred, ints, lw, wsc, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// prow: the most output rows one CTA computes in a K-split stage (gate and up
// rows counted separately).
__host__ __device__ inline Carve carve(int nslot, int slot_bytes, int B, int kmax, int D, int rep,
                                       int wsc_n, int prow) {
  Carve c;
  size_t o = 0;
  c.ring = o;
  o += static_cast<size_t>(nslot) * slot_bytes;
  c.bars = o;
  o += align_up(2 * nslot * sizeof(uint64_t), 16);
  // fp32 activations [B][kmax], or their bf16 hi/lo planes [B][2][kmax + pad]
  size_t act_b = static_cast<size_t>(B) * kmax * sizeof(float) + 2ull * B * kRowPad;
  // attention: qs[hm][D], kn/vn[B][D], merge[kCW][hm][D + 2] for hm query
  // heads per item (a verification block: B * rep of them, at most 8)
  const size_t hm = static_cast<size_t>(B * rep <= 8 && B * rep > rep ? B * rep : rep);
  size_t att_b = ((hm + 2ull * B) * D + static_cast<size_t>(kCW) * hm * (D + 2)) * sizeof(float);
  c.act = o;
  o += align_up(act_b > att_b ? act_b : att_b, 16);
  c.stg = o;
  o += static_cast<size_t>(kStageWords) * sizeof(uint64_t);
  c.xown = o;
  o += align_up(static_cast<size_t>(kMaxHRows) * B * sizeof(float), 16);
  c.part = o;  // two buffers of [kCW][prow][B] partial sums + [kCW][B] sums of squares
  o += align_up(2ull * kCW * (prow + 1) * B * sizeof(float), 16);
  c.bred = o;
  o += align_up(2ull * kCW * B * sizeof(float) + 2ull * kCW * B * sizeof(int), 16);
  c.ints = o;  // two Plans (consumers, producer), a few ints, a 16-byte zero row
  o += align_up(2 * sizeof(Plan) + 16 * sizeof(int), 16) + 16;
  c.lw = o;
  o += align_up(sizeof(LayerPtrs) * kMaxLayers, 16);
  c.wsc = o;
  o += align_up(static_cast<size_t>(wsc_n) * sizeof(float), 16);
  c.total = o;
  return c;
}

// Bounded spin.  `poll` waits (on other CTAs' data) also give up when some
// CTA has raised the abort flag; ring waits only give up on the time limit.
struct Spin {
  uint64_t t0 = 0;
  uint32_t it = 0;
  __device__ __forceinline__ bool tick(const StepArgs& a, bool poll) {
    if (it == 0) t0 = globaltimer();
    ++it;
    if ((it & 7) == 0) {
      if (poll && ld_relaxed_i32(a.abort_flag)) return true;
      if (globaltimer() - t0 > a.timeout_ns) {
        atomicOr(a.status, kDevTimeout);
        atomicExch(a.abort_flag, 1);
        return true;
      }
    }
    return false;
  }
};

__device__ __forceinline__ float dot8(const uint4 w, const float* x) {
  float s = bf16lo(w.x) * x[0];
  s = fmaf(bf16hi(w.x), x[1], s);
  s = fmaf(bf16lo(w.y), x[2], s);
  s = fmaf(bf16hi(w.y), x[3], s);
  s = fmaf(bf16lo(w.z), x[4], s);
  s = fmaf(bf16hi(w.z), x[5], s);
  s = fmaf(bf16lo(w.w), x[6], s);
  s = fmaf(bf16hi(w.w), x[7], s);
  return s;
}

// Dot products of R weight rows (shared memory, row i at rows[i]) with the
// activation rows of B sequences (shared memory, act_stride floats apart),
// K = 256 * nblk columns (group_dot: bf16 rows, group_dot_i8: int8 codes).
// The columns go in blocks of 256; lane l takes columns 4l..4l+3 and
// 128+4l..128+4l+3 of each block, so that a warp's weight reads (8 or 4
// bytes a lane) and activation reads (16 bytes a lane) are contiguous and
// free of bank conflicts.  Returns the transposed-butterfly reduction: every
// lane gets the full sum of row (R == 4: lane >> 3; R == 2: lane >> 4;
// R == 1: 0) for each b.  Compiled on their own (not inlined) so that their
// register allocation and scheduling do not depend on the rest of the
// persistent kernel.  (The lm_head: whole rows per warp.)
template <int R, int B>
struct GroupSums {
  float s[B];
};

template <int R>
__device__ __forceinline__ float tbfly_lane(float (&p)[R], int lane) {
  if constexpr (R == 1) {
    return warp_sum(p[0]);
  } else if constexpr (R == 2) {
    const bool hi = lane & 16;
    float k = hi ? p[1] : p[0];
    k += __shfl_xor_sync(0xffffffffu, hi ? p[0] : p[1], 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;
  } else {
    const bool h16 = lane & 16;
    float k0 = h16 ? p[2] : p[0], k1 = h16 ? p[3] : p[1];
    k0 += __shfl_xor_sync(0xffffffffu, h16 ? p[0] : p[2], 16);
    k1 += __shfl_xor_sync(0xffffffffu, h16 ? p[1] : p[3], 16);
    const bool h8 = lane & 8;
    float k = h8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;
  }
}

// Signed int8 byte j of w (given as w ^ 0x80808080, i.e. biased to code + 128)
// as a float, exactly: the byte becomes the low mantissa bits of 2^23, so the
// float is 2^23 + code + 128, and subtracting 2^23 + 128 leaves the code.
__device__ __forceinline__ float i8_at(uint32_t biased, uint32_t j) {
  return __uint_as_float(__byte_perm(biased, 0x4B000000u, 0x7540u + j)) - 8388736.0f;
}
__device__ __forceinline__ float dot8_i8(uint32_t w0, uint32_t w1, const float* x) {
  const uint32_t u0 = w0 ^ 0x80808080u, u1 = w1 ^ 0x80808080u;
  float s = i8_at(u0, 0) * x[0];
  s = fmaf(i8_at(u0, 1), x[1], s);
  s = fmaf(i8_at(u0, 2), x[2], s);
  s = fmaf(i8_at(u0, 3), x[3], s);
  s = fmaf(i8_at(u1, 0), x[4], s);
  s = fmaf(i8_at(u1, 1), x[5], s);
  s = fmaf(i8_at(u1, 2), x[6], s);
  s = fmaf(i8_at(u1, 3), x[7], s);
  return s;
}

// The four 8-bit weight codes of a word as floats (exact): W8 = 1 signed
// int8 codes, W8 = 2 E4M3 codes (two hardware e4m3x2 -> f16x2 conversions).
template <int W8>
__device__ __forceinline__ void codes4(uint32_t w, float (&f)[4]) {
  if constexpr (W8 == 2) {
    const float2 a = e4m3x2_to_f2(static_cast<uint16_t>(w & 0xFFFFu));
    const float2 b = e4m3x2_to_f2(static_cast<uint16_t>(w >> 16));
    f[0] = a.x;
    f[1] = a.y;
    f[2] = b.x;
    f[3] = b.y;
  } else {
    const uint32_t u = w ^ 0x80808080u;
#pragma unroll
    for (int e = 0; e < 4; ++e) f[e] = i8_at(u, static_cast<uint32_t>(e));
  }
}
template <int W8>
__device__ __forceinline__ float dot8_w8(uint32_t w0, uint32_t w1, const float* x) {
  if constexpr (W8 == 1) return dot8_i8(w0, w1, x);
  float a[4], b[4];
  codes4<W8>(w0, a);
  codes4<W8>(w1, b);
  float s = a[0] * x[0];
  s = fmaf(a[1], x[1], s);
  s = fmaf(a[2], x[2], s);
  s = fmaf(a[3], x[3], s);
  s = fmaf(b[0], x[4], s);
  s = fmaf(b[1], x[5], s);
  s = fmaf(b[2], x[6], s);
  return fmaf(b[3], x[7], s);
}

// 8-bit rows (K bytes, int8 or E4M3 codes): the sums of code * x; the caller
// applies the row scale.
template <int R, int B, int W8>
__device__ __noinline__ GroupSums<R, B> group_dot_i8(const uint32_t* rows, uint32_t act,
                                                     int act_stride, int nblk, int lane) {
  float acc[R][B], acc2[R][B];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[i][b] = acc2[i][b] = 0.f;
#pragma unroll 2
  for (int c = 0; c < nblk; ++c) {
    const bool odd = c & 1;
    const uint32_t col = static_cast<uint32_t>(c * 256 + lane * 4);
    uint32_t w[R][2];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[i][0]) : "r"(rows[i] + col));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[i][1]) : "r"(rows[i] + col + 128));
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float x[8];
      const uint32_t xa = act + static_cast<uint32_t>(b * act_stride) * 4u + col * 4u;
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]) : "r"(xa));
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7]) : "r"(xa + 512));
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const float d = dot8_w8<W8>(w[i][0], w[i][1], x);
        if (odd) acc2[i][b] += d;
        else acc[i][b] += d;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[i][b] += acc2[i][b];
  GroupSums<R, B> out;
#pragma unroll
  for (int b = 0; b < B; ++b) {
    float col[R];
#pragma unroll
    for (int i = 0; i < R; ++i) col[i] = acc[i][b];
    out.s[b] = tbfly_lane<R>(col, lane);
  }
  return out;
}

// bf16 rows (2K bytes).
template <int R, int B>
__device__ __noinline__ GroupSums<R, B> group_dot(const uint32_t* rows, uint32_t act,
                                                    int act_stride, int nblk, int lane) {
  float acc[R][B], acc2[R][B];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[i][b] = acc2[i][b] = 0.f;
#pragma unroll 2
  for (int c = 0; c < nblk; ++c) {
    const bool odd = c & 1;
    const uint32_t col = static_cast<uint32_t>(c * 256 + lane * 4);
    uint2 w[R][2];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                   : "=r"(w[i][0].x), "=r"(w[i][0].y) : "r"(rows[i] + col * 2));
      asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                   : "=r"(w[i][1].x), "=r"(w[i][1].y) : "r"(rows[i] + col * 2 + 256));
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float x[8];
      const uint32_t xa = act + static_cast<uint32_t>(b * act_stride) * 4u + col * 4u;
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]) : "r"(xa));
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(x[4]), "=f"(x[5]), "=f"(x[6]), "=f"(x[7]) : "r"(xa + 512));
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const uint4 wv = make_uint4(w[i][0].x, w[i][0].y, w[i][1].x, w[i][1].y);
        const float d = dot8(wv, x);
        if (odd) acc2[i][b] += d;
        else acc[i][b] += d;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[i][b] += acc2[i][b];
  GroupSums<R, B> out;
#pragma unroll
  for (int b = 0; b < B; ++b) {
    float col[R];
#pragma unroll
    for (int i = 0; i < R; ++i) col[i] = acc[i][b];
    out.s[b] = tbfly_lane<R>(col, lane);
  }
  return out;
}

// Partial dot products of R (4 or 8) tile rows (shared memory, row i at
// rows[i]) with the activations of B sequences over the K blocks blk0,
// blk0 + kCW, ... (nb of them): lane l takes columns 4l..4l+3 of each
// 128-column block, so that the warp reads 256 contiguous bytes of a bf16 row
// (128 of an int8 row) and 512 contiguous bytes of activations: no bank
// conflicts.  All R rows' loads of a block are issued before their
// multiply-adds, so R independent chains hide the shared-memory latency.
// Returns the transposed-butterfly reductions: lane gets the sums of rows
// (lane >> 3) and, for R == 8, 4 + (lane >> 3), for each b.
template <int R, int B>
struct KSums {
  float s[R / 4][B];
};

template <int R, int B, int W8>
__device__ __forceinline__ KSums<R, B> kdot(const uint32_t (&rows)[R], uint32_t act,
                                            int act_stride, int blk0, int nb, int lane) {
  float acc[R][B];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[i][b] = 0.f;
  for (int j = 0; j < nb; ++j) {
    const uint32_t col = static_cast<uint32_t>((blk0 + j * kCW) * kBlk + lane * 4);
    uint32_t w[R][2];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      if constexpr (W8) {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[i][0]) : "r"(rows[i] + col));
        w[i][1] = 0u;
      } else {
        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                     : "=r"(w[i][0]), "=r"(w[i][1]) : "r"(rows[i] + col * 2));
      }
    }
    float x[B][4];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      const uint32_t xa = act + static_cast<uint32_t>(b * act_stride + col) * 4u;
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(x[b][0]), "=f"(x[b][1]), "=f"(x[b][2]), "=f"(x[b][3]) : "r"(xa));
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
      float wf[4];
      if constexpr (W8) {
        codes4<W8>(w[i][0], wf);
      } else {
        wf[0] = bf16lo(w[i][0]);
        wf[1] = bf16hi(w[i][0]);
        wf[2] = bf16lo(w[i][1]);
        wf[3] = bf16hi(w[i][1]);
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float t = fmaf(wf[0], x[b][0], acc[i][b]);
        t = fmaf(wf[1], x[b][1], t);
        t = fmaf(wf[2], x[b][2], t);
        acc[i][b] = fmaf(wf[3], x[b][3], t);
      }
    }
  }
  KSums<R, B> out;
#pragma unroll
  for (int q = 0; q < R / 4; ++q)
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float c4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) c4[i] = acc[4 * q + i][b];
      out.s[q][b] = tbfly_lane<4>(c4, lane);
    }
  return out;
}

// Warp-level tensor-core pieces of the batch-1..4 projections: an 8x8
// matrix load per lane group and the m16n8k16 bf16 MMA with fp32
// accumulation.  With a handful of sequences the projections are matrix x
// vector products; one MMA multiplies 16 weight rows x 16 columns by the 8
// activation columns (hi and lo bf16 planes of up to 4 sequences), which
// replaces ~40 unpack/FMA/shuffle instructions per lane.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4],
                                          const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// The per-launch state of one CTA.  FP8: the cache holds E4M3 codes + scales.
// W8: 0 bf16 weights; 1 / 2: the projections and lm_head are int8 / E4M3
// codes with fp32 row scales.
template <int B, int D, bool FP8, int W8>
struct Cta {
  static constexpr int DL = D / 32;  // attention dims per lane (warp-wide vectors)
  static constexpr int DQ = D / 8;   // attention dims per lane (lane octets)
  const StepArgs& a;
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  float* act;
  float* xown;
  uint64_t* stg;  // gather staging: tagged words
  float* part;    // K-split partial sums, two buffers
  float* bredf;
  int* bredi;
  const LayerPtrs* slw;  // layer pointer table copied to shared memory
  float* wsc;                               // int8: row scales of the current stage
  static constexpr int eb = W8 ? 1 : 2;     // bytes per weight element
  int tid, warp, lane, cta, nc;
  int kmax, nqkv, prow;
  uint32_t seq0;  // step counter of the launch's first step
  uint32_t seq;   // step counter of the consumers' current step
  // per-CTA row ranges
  int q0, q1, h0, h1, f0, f1, v0, v1;
  int slot;  // bytes per ring slot
  int rpt_lm, rpt_h, rpt_o, rpt_u, rpt_d, art;
  uint32_t zrow;  // 16 zero bytes (shared memory)
  static constexpr int pad = W8 ? 0 : kRowPad;  // ring row padding of the projections
  // ring bytes between two rows of a projection with K columns
  __device__ __forceinline__ int rstride(int K) const { return K * eb + pad; }
  // this side's plan of the current step (shared memory)
  Plan* pl;
  Plan* cplan;  // the consumers' copy
  Plan* pplan;  // the producer's copy
  int* sints;   // a few shared ints after the plans

  __device__ Cta(const StepArgs& args, uint8_t* smem, int kmax_) : a(args), kmax(kmax_) {
    const int rep = a.Hq / a.Hkv;
    prow = a.prow;
    slot = a.slot_bytes;
    Carve c = carve(a.nslot, slot, B, kmax, D, rep, a.wsc_n, prow);
    ring = smem + c.ring;
    full = reinterpret_cast<uint64_t*>(smem + c.bars);
    empty = full + a.nslot;
    act = reinterpret_cast<float*>(smem + c.act);
    xown = reinterpret_cast<float*>(smem + c.xown);
    stg = reinterpret_cast<uint64_t*>(smem + c.stg);
    part = reinterpret_cast<float*>(smem + c.part);
    bredf = reinterpret_cast<float*>(smem + c.bred);
    bredi = reinterpret_cast<int*>(bredf + 2 * kCW * B);
    cplan = reinterpret_cast<Plan*>(smem + c.ints);
    pplan = cplan + 1;
    sints = reinterpret_cast<int*>(pplan + 1);
    zrow = smem_u32(smem + c.ints + align_up(2 * sizeof(Plan) + 16 * sizeof(int), 16));
    slw = reinterpret_cast<const LayerPtrs*>(smem + c.lw);
    wsc = reinterpret_cast<float*>(smem + c.wsc);
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    cta = blockIdx.x;
    nc = gridDim.x;
    nqkv = (a.Hq + 2 * a.Hkv) * D;
    q0 = split_at(nqkv, nc, cta);
    q1 = split_at(nqkv, nc, cta + 1);
    h0 = split_at(a.H, nc, cta);
    h1 = split_at(a.H, nc, cta + 1);
    f0 = split_at(a.F, nc, cta);
    f1 = split_at(a.F, nc, cta + 1);
    v0 = split_at(a.V, nc, cta);
    v1 = split_at(a.V, nc, cta + 1);
    rpt_lm = slot / (eb * a.H);
    rpt_h = slot / rstride(a.H);
    rpt_o = slot / rstride(a.Hq * D);
    rpt_u = slot / (2 * rstride(a.H));
    rpt_d = slot / rstride(a.F);
    if constexpr (FP8) {
      art = (slot / (2 * D + 8)) & ~15;
    } else {
      art = slot / (4 * D);
    }
    pl = warp == kCW ? pplan : cplan;
  }

  // Tag of the words a layer publishes in the current step (seq counts the
  // steps of all launches on the handle), and of the ids of step st of this
  // launch.
  __device__ __forceinline__ uint32_t flag(int layer) const {
    return seq * 256u + static_cast<uint32_t>(layer) + 1u;
  }
  __device__ __forceinline__ uint32_t tok_flag(int st) const {
    return (seq0 + static_cast<uint32_t>(st)) * 256u + 255u;
  }

  // The attention items of plan P's positions: chunk rows sized so that the
  // items fit the grid when possible.  Same on every CTA and both sides.
  // Block verification (a.vseq >= 0): the rows are consecutive tokens of one
  // cached sequence; its committed prefix [0, pos[0]) is split into chunks
  // shared by all rows, and chunk 0 also holds the block's own new rows.
  __device__ void make_plan(Plan& P) const {
    const bool ver = a.vseq >= 0;
    long long T = 0;
    if (ver) T = static_cast<long long>(P.pos[0] + a.B) * a.Hkv;
    else
      for (int b = 0; b < a.B; ++b) T += static_cast<long long>(P.pos[b] + 1) * a.Hkv;
    int slots = nc - (ver ? 1 : a.B) * a.Hkv;
    if (slots < 1) slots = 1;
    long long cr = (T + slots - 1) / slots;
    cr = (cr + 15) / 16 * 16;
    if (cr < kMinChunkRows) cr = kMinChunkRows;
    P.crow = static_cast<int>(cr);
    P.n_items = 0;
    int all = 1;
    if (ver) {
      const int nb = max(1, (P.pos[0] + P.crow - 1) / P.crow);
      P.nchunk[0] = nb;
      P.n_items = nb * a.Hkv;
    } else {
      for (int b = 0; b < a.B; ++b) {
        const int nb = (P.pos[b] + 1 + P.crow - 1) / P.crow;
        P.nchunk[b] = nb;
        P.n_items += nb * a.Hkv;
      }
    }
    for (int b = 0; b < a.B; ++b) all &= P.done[b];
    P.all_done = all;
  }
  __device__ void item(int it, int& b, int& g, int& ci) const {
    if (a.vseq >= 0) {
      b = 0;
      g = it / pl->nchunk[0];
      ci = it % pl->nchunk[0];
      return;
    }
    int bb = 0;
    while (bb < a.B - 1 && it >= pl->nchunk[bb] * a.Hkv) {
      it -= pl->nchunk[bb] * a.Hkv;
      ++bb;
    }
    b = bb;
    g = it / pl->nchunk[bb];
    ci = it % pl->nchunk[bb];
  }

  // The ids of step s (tagged words published by the CTA that finished the
  // step last), then plan P of step s + 1: a sequence that has emitted the
  // end token is retired (its position stays, its input is the end token,
  // the cache is not written); the others advance by one row.  Polled by one
  // thread; false when the wait gave up.
  __device__ bool next_step(Plan& P, uint32_t f) const {
    Spin sp;
    for (int b = 0; b < a.B; ++b) {
      uint64_t w;
      for (;;) {
        w = ld_tagged(a.tokw + b);
        if (static_cast<uint32_t>(w >> 32) == f) break;
        if (sp.tick(a, true)) return false;
      }
      const int id = static_cast<int>(static_cast<uint32_t>(w));
      if (!P.done[b]) {
        if (a.eos >= 0 && id == a.eos) P.done[b] = 1;
        else P.pos[b] += 1;
      }
      P.tok[b] = P.done[b] ? a.eos : id;
      if (!P.done[b] && P.pos[b] >= a.max_ctx) P.bad = 1;
    }
    make_plan(P);
    return true;
  }

  __device__ __forceinline__ size_t kv_row(int l, int kvsel, int b, int g, int j) const {
    return ((((static_cast<size_t>(l) * 2 + kvsel) * a.kv_batch + b) * a.Hkv + g) *
                static_cast<size_t>(a.max_ctx) + j);
  }

  // ================================================================ producer
  __device__ void producer() {
    if (lane == 0) produce();
    __syncwarp();
  }
  __device__ void produce() {
    const uint64_t pol = policy_evict_first();
    uint32_t n = 0;     // tiles issued
    int ps = 0;         // ring slot of tile n
    uint32_t lap = 0;   // n / nslot
    uint64_t* fb = full;
    bool dead = false;
    const int ns = a.nslot;
    // Slot for tile n, once the consumers released its previous use; arms its
    // full barrier with the tile's byte count.
    auto acquire = [&](uint32_t bytes) -> uint8_t* {
      if (lap > 0) {
        Spin sp;
        while (!mbar_wait(&empty[ps], (lap - 1) & 1, kWaitHintNs)) {
          if (sp.tick(a, false)) {
            dead = true;
            return nullptr;
          }
#ifdef DEC_PRODUCER_NAP
          __nanosleep(DEC_PRODUCER_NAP);  // the ring runs far ahead: issue slots go to the consumers
#endif
        }
      }
      fb = &full[ps];
      mbar_arrive_expect_tx(fb, bytes);
      return ring + static_cast<size_t>(ps) * slot;
    };
    auto advance = [&]() {
      ++n;
      if (++ps == ns) {
        ps = 0;
        ++lap;
      }
    };
    const int H = a.H, HqD = a.Hq * D, HkvD = a.Hkv * D;
    const uint32_t e = static_cast<uint32_t>(eb);
    // byte address of row r of a [rows, K] weight matrix
    auto wrow = [&](const void* base, int r, int K) {
      return static_cast<const uint8_t*>(base) + static_cast<size_t>(r) * K * e;
    };
    // cnt rows lo.. of a [rows, K] projection to dst, rstride(K) bytes apart
    auto rows_to = [&](uint8_t* dst, const void* base, int lo, int cnt, int K) {
      if (pad == 0) {
        bulk_g2s(dst, wrow(base, lo, K), static_cast<uint32_t>(cnt) * K * e, fb, pol);
      } else {
        for (int i = 0; i < cnt; ++i)
          bulk_g2s(dst + static_cast<size_t>(i) * rstride(K), wrow(base, lo + i, K),
                   static_cast<uint32_t>(K) * e, fb, pol);
      }
    };
    bool stop = false;
    for (int st = 0; !dead && !stop; ++st) {
    for (int l = 0; l < a.L && !dead; ++l) {
      const LayerPtrs& lw = slw[l];
      // The layer's tiles in consumption order: the four projection stages
      // (one copy of this code serves them all), the attention tiles before
      // o_proj.  s = 0: QKV rows [q0, q1) of [Wq; Wk; Wv]; 1: o_proj rows
      // [h0, h1), K = Hq*D; 2: gate/up rows [f0, f1), a tile is nr gate rows
      // then nr up rows; 3: down rows [h0, h1), K = F.
#pragma unroll 1
      for (int s = 0; s < 4 && !dead; ++s) {
        if (s == 1) {
          // A later step's attention rows depend on the ids of the step
          // before (a sequence that emitted the end token keeps its
          // position): wait for them once the first layer's QKV rows are on
          // their way.
          if (l == 0 && st > 0) {
            if (!next_step(*pplan, tok_flag(st - 1))) dead = true;
            if (dead || pplan->bad || pplan->all_done) {
              stop = true;
              break;
            }
          }
          // attention: cached rows [j0, min(j1, p_b)) of every item of this CTA
          for (int it = cta; it < pl->n_items && !dead; it += nc) {
            int b, g, ci;
            item(it, b, g, ci);
            const int j0 = ci * pl->crow;
            const int jc = min(j0 + pl->crow, pl->pos[b]);  // (verify: b = 0, the prefix end)
            if (a.vseq >= 0) b = a.vseq;                     // the cache sequence
            for (int j = j0; j < jc && !dead; j += art) {
              const int nr = min(art, jc - j);
              if constexpr (!FP8) {
                const uint32_t rb = static_cast<uint32_t>(nr) * D * 2;
                uint8_t* dst = acquire(2 * rb);
                if (!dst) break;
                if (j == j0) DEC_PSTAMP(kStampsPerLayer * l + StPA);
                const uint16_t* kvb = reinterpret_cast<const uint16_t*>(a.kv);
                bulk_g2s(dst, kvb + kv_row(l, 0, b, g, j) * D, rb, fb, pol);
                bulk_g2s(dst + rb, kvb + kv_row(l, 1, b, g, j) * D, rb, fb, pol);
              } else {
                const uint32_t rb = static_cast<uint32_t>(nr) * D;
                const uint32_t sb = static_cast<uint32_t>((nr + 3) & ~3) * 4;
                uint8_t* dst = acquire(2 * rb + 2 * sb);
                if (!dst) break;
                bulk_g2s(dst, a.kv + kv_row(l, 0, b, g, j) * D, rb, fb, pol);
                bulk_g2s(dst + rb, a.kv + kv_row(l, 1, b, g, j) * D, rb, fb, pol);
                bulk_g2s(dst + 2 * rb, a.kv_scales + kv_row(l, 0, b, g, j), sb, fb, pol);
                bulk_g2s(dst + 2 * rb + sb, a.kv_scales + kv_row(l, 1, b, g, j), sb, fb,
                         pol);
              }
              advance();
            }
          }
        }
        const int lo = s == 0 ? q0 : s == 2 ? f0 : h0;
        const int hi = s == 0 ? q1 : s == 2 ? f1 : h1;
        const int rpt = s == 0 ? rpt_h : s == 1 ? rpt_o : s == 2 ? rpt_u : rpt_d;
        const int K = s == 1 ? HqD : s == 3 ? a.F : H;
        const uint32_t mats = s == 2 ? 2u : 1u;
        for (int r = lo; r < hi && !dead; r += rpt) {
          const int nr = min(rpt, hi - r);
          uint8_t* dst = acquire(mats * static_cast<uint32_t>(nr) * K * e);
          if (!dst) break;
          if (r == lo)
            DEC_PSTAMP(kStampsPerLayer * l + (s == 0 ? StPQ : s == 1 ? StPO : s == 2 ? StPU : StPD));
          if (s == 0) {
            int rr = r, left = nr;
            while (left > 0) {
              const uint16_t* base;
              int r0, cnt;
              if (rr < HqD) {
                base = lw.w[1]; r0 = rr; cnt = min(left, HqD - rr);
              } else if (rr < HqD + HkvD) {
                base = lw.w[2]; r0 = rr - HqD; cnt = min(left, HqD + HkvD - rr);
              } else {
                base = lw.w[3]; r0 = rr - HqD - HkvD; cnt = left;
              }
              rows_to(dst, base, r0, cnt, H);
              dst += static_cast<size_t>(cnt) * rstride(H);
              rr += cnt;
              left -= cnt;
            }
          } else {
            rows_to(dst, s == 1 ? lw.w[6] : s == 2 ? lw.w[8] : lw.w[10], r, nr, K);
            if (s == 2) rows_to(dst + static_cast<size_t>(nr) * rstride(H), lw.w[9], r, nr, H);
          }
          advance();
        }
      }
      if (stop) break;
    }
    if (stop) break;
    // ---- lm_head rows [v0, v1)
    for (int r = v0; r < v1 && !dead; r += rpt_lm) {
      const int nr = min(rpt_lm, v1 - r);
      uint8_t* dst = acquire(static_cast<uint32_t>(nr) * H * e);
      if (!dst) break;
      bulk_g2s(dst, wrow(a.lm_head, r, H), static_cast<uint32_t>(nr) * H * e, fb, pol);
      advance();
    }
    if (st + 1 >= a.n_steps) break;
    }
    // Every copy issued must land before the CTA exits: wait for the last
    // phase armed on each slot (returns at once when consumers already did).
    const uint32_t armed = n;
    for (int s = 0; s < ns && static_cast<uint32_t>(s) < armed; ++s) {
      const uint32_t last = armed - 1 - ((armed - 1 - s) % ns);
      Spin sp;
      while (!mbar_test(&full[s], (last / ns) & 1)) {
        if (sp.tick(a, false)) break;
      }
    }
  }

  // ================================================================ consumers
  uint32_t rn = 0;         // ring tiles consumed
  int rs = 0;              // ring slot of tile rn
  uint32_t rph = 0;        // full-barrier phase parity of tile rn
  int ab = 0;              // aborted: keep the barrier sequence, compute nothing
  bool ring_dead = false;  // a ring wait ran out: stop waiting on the ring
  int pb = 0;              // partial-sum buffer of the current K-split stage
  uint64_t wacc = 0;       // profiling builds: ns spent in ring waits
  float best_v[B];         // lm_head argmax of this thread, per sequence
  int best_i[B];

  __device__ __forceinline__ void csync() { named_sync(1, kCT); }

  // Wait for ring tile rn.  Every consumer thread calls it for every tile, so
  // the barrier sequence stays uniform even when a wait runs out: the warp
  // then only stops computing (ab) and stops waiting on the ring.  Lane 0
  // polls; the outcome is broadcast so that it is warp-uniform.
  __device__ void wait_tile() {
    if (ring_dead) return;
    const int slot = rs;
    const uint32_t par = rph;
    int st = 1;
    if (lane == 0) {
#ifdef DEC_PROFILE
      const long long tw = clock64();
#endif
      Spin sp;
      while (!mbar_wait(&full[slot], par, kWaitHintNs)) {
        if (sp.tick(a, false)) {
          st = 0;
          break;
        }
      }
#ifdef DEC_PROFILE
      wacc += static_cast<uint64_t>(clock64() - tw);
#endif
    }
    st = __shfl_sync(0xffffffffu, st, 0);
    if (!st) {
      ring_dead = true;
      ab = 1;
      return;
    }
#ifdef DEC_LEAN_WAIT
    __syncwarp();  // lane 0 observed the completed phase; the warp is ordered after it
#else
    (void)mbar_test(&full[slot], par);  // every lane observes the completed phase
#endif
  }
  __device__ __forceinline__ void release_tile() {
    __syncwarp();
    if (lane == 0 && !ring_dead) mbar_arrive(&empty[rs]);
    ++rn;
    if (++rs == a.nslot) {
      rs = 0;
      rph ^= 1;
    }
  }

  // Fetch n (even, <= kStageWords) tagged words into stg, word w from
  // src_of(w) (16-byte aligned for even w), until every flag equals f.  All
  // copies of a pass are in flight at once (cp.async through L2); a pass
  // re-fetches only the words that were not ready, so the gather costs one
  // round trip after the last producer published.  Collective over the
  // consumer threads; ends with every word visible to every thread.
  template <class Src>
  __device__ void gather(int n, uint32_t f, Src src_of) {
    const int nch = n >> 1;
    uint32_t pend = 0;
    if (!ab) {
      int k = 0;
      for (int c = tid; c < nch; c += kCT, ++k) pend |= 1u << k;
    }
    int fail = 0;
    uint64_t t0 = 0;
    int more, round = 0;
    do {
      int k = 0;
      for (int c = tid; c < nch; c += kCT, ++k)
        if (pend & (1u << k)) cp_async16_cg(stg + 2 * c, src_of(2 * c));
      const int abf = (pend && round++ > 0) ? ld_relaxed_i32(a.abort_flag) : 0;
      cp_async_wait_all();
      k = 0;
      for (int c = tid; c < nch; c += kCT, ++k) {
        if (pend & (1u << k)) {
          if (static_cast<uint32_t>(stg[2 * c] >> 32) == f &&
              static_cast<uint32_t>(stg[2 * c + 1] >> 32) == f)
            pend &= ~(1u << k);
        }
      }
      if (pend) {
        const uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        if (now - t0 > a.timeout_ns) {
          atomicOr(a.status, kDevTimeout);
          atomicExch(a.abort_flag, 1);
          fail = 1;
        } else if (abf) {
          fail = 1;
        }
        if (fail) pend = 0;  // else re-poll at once: a hop costs one L2 round trip
      }
      more = named_sync_or(1, kCT, pend != 0);
    } while (more);
    ab = named_sync_or(1, kCT, fail | ab);
  }

  // Warp-collective version for one warp's own words: n (even, <=
  // kWarpStage) tagged words into ws (this warp's part of stg).  Sets ab
  // (warp-uniform) when the wait gave up; ends with every word visible to
  // every lane of the warp.
  template <class Src>
  __device__ void warp_gather(uint64_t* ws, int n, uint32_t f, Src src_of) {
    __syncwarp();  // the previous round's words are consumed
    const int np = n >> 1;
    constexpr int kPer = kWarpStage / 64;  // pairs per lane at most
    uint32_t pend = 0;
    const uint64_t* sp[kPer];  // this lane's source pairs, computed once
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int c = lane + 32 * k;
      sp[k] = c < np ? src_of(2 * c) : nullptr;
      if (!ab && c < np) pend |= 1u << k;
    }
    uint64_t t0 = 0;
    // A short pause before the first round: the words were only just being
    // written when a warp gets here, and every warp of every CTA polls the
    // same lines; starting a little later costs less than the rounds that
    // would fail meanwhile (0.6B batch 1: 774.7 -> 759.4 us/token with
    // 128 ns; 256 / 384 ns the same, 512 ns slower).
    __nanosleep(128);
    for (int round = 0;; ++round) {
#pragma unroll
      for (int k = 0; k < kPer; ++k)
        if (pend & (1u << k)) cp_async16_cg(ws + 2 * (lane + 32 * k), sp[k]);
      // every 8th round also reads the abort flag (its load overlaps the
      // copies' round trip) and checks the time limit
      const bool slow = (round & 7) == 7;
      const int abf = (lane == 0 && slow) ? ld_relaxed_i32(a.abort_flag) : 0;
      cp_async_wait_all();
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int c = lane + 32 * k;
        if ((pend & (1u << k)) && static_cast<uint32_t>(ws[2 * c] >> 32) == f &&
            static_cast<uint32_t>(ws[2 * c + 1] >> 32) == f)
          pend &= ~(1u << k);
      }
      if (!__any_sync(0xffffffffu, pend != 0)) break;
      if (!slow) continue;
      int fail = 0;
      if (lane == 0) {
        const uint64_t now = globaltimer();
        if (t0 == 0) t0 = now;
        if (now - t0 > a.timeout_ns) {
          atomicOr(a.status, kDevTimeout);
          atomicExch(a.abort_flag, 1);
          fail = 1;
        } else if (abf) {
          fail = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, fail, 0)) {
        ab = 1;
        break;
      }
    }
    __syncwarp();
  }

  // K blocks of 128 columns are dealt to the consumer warps round-robin:
  // warp w owns blocks w, w + kCW, ...
  __device__ __forceinline__ int my_blocks(int nblk) const {
    return nblk > warp ? (nblk - 1 - warp) / kCW + 1 : 0;
  }

  // This warp's share of a stage input: for every sequence b and every K
  // block the warp owns, the 128 values src[b][k] (tagged words, flag f; or,
  // with src == nullptr, the embedding row of the step's token) times the
  // gain g[k] (g == nullptr: 1) into act[b][k]; ss[b] gets the warp's share
  // of sum_k x[b][k]^2 (before the gain), reduced over the warp.
  // With `planes` (bf16 weights) the values go to act as two bf16 planes per
  // sequence instead, hi = bf16(x) and lo = bf16(x - hi) (row 2b + plane,
  // rstride(K) bytes apart): the operands of the tensor-core projections.
  // Unit u of a warp's input units: batch 1 in block order (u = j), larger
  // batches block-major (u = j * B + b, compile-time divisors).
  __device__ __forceinline__ void unit_of(int u, int nbw, int& b, int& blk) const {
    if constexpr (B == 1) {
      b = u / nbw;
      blk = warp + (u % nbw) * kCW;
    } else {
      b = u % B;
      blk = warp + (u / B) * kCW;
    }
  }
  __device__ void warp_input(const uint64_t* src, int K, uint32_t f, const uint16_t* g,
                             float (&ss)[B], bool planes) {
#pragma unroll
    for (int b = 0; b < B; ++b) ss[b] = 0.f;
    const int nbw = my_blocks(K / kBlk);
    const int units = B * nbw;  // 128-word units: (b, block)
    constexpr int per = kWarpStage / kBlk;
    uint64_t* ws = stg + warp * kWarpStage;
    // the gains of the warp's blocks, loaded before the polls so that their
    // latency overlaps them (K <= kMaxGainBlk * kCW * kBlk for a gained input)
    uint2 gv[kMaxGainBlk];
#pragma unroll
    for (int j = 0; j < kMaxGainBlk; ++j)
      gv[j] = (g && j < nbw) ? __ldg(reinterpret_cast<const uint2*>(
                                   g + (warp + j * kCW) * kBlk + lane * 4))
                             : make_uint2(0u, 0u);
    for (int u0 = 0; u0 < units; u0 += per) {
      const int nu = min(per, units - u0);
      if (src)
        warp_gather(ws, nu * kBlk, f, [=](int i) {
          const int u = u0 + i / kBlk;
          int b, blk;
          unit_of(u, nbw, b, blk);
          return src + static_cast<size_t>(b) * K + blk * kBlk + (i % kBlk);
        });
      if (ab) continue;
      for (int uu = 0; uu < nu; ++uu) {
        const int u = u0 + uu;
        int b, blk;
        unit_of(u, nbw, b, blk);
        const int k = blk * kBlk + lane * 4;
        float v[4];
        if (src) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            v[j] = __uint_as_float(static_cast<uint32_t>(ws[uu * kBlk + lane * 4 + j]));
        } else {
          const uint2 e = *reinterpret_cast<const uint2*>(
              a.embed + static_cast<size_t>(pl->tok[b]) * a.H + k);
          v[0] = bf16lo(e.x);
          v[1] = bf16hi(e.x);
          v[2] = bf16lo(e.y);
          v[3] = bf16hi(e.y);
        }
        const float q = v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3];
#pragma unroll
        for (int bb = 0; bb < B; ++bb)
          if (bb == b) ss[bb] += q;
        if (g) {
          const int j = B == 1 ? u % nbw : u / B;
          uint2 gs = gv[0];
#pragma unroll
          for (int jj = 1; jj < kMaxGainBlk; ++jj)
            if (jj == j) gs = gv[jj];
          v[0] *= bf16lo(gs.x);
          v[1] *= bf16hi(gs.x);
          v[2] *= bf16lo(gs.y);
          v[3] *= bf16hi(gs.y);
        }
        if (planes) {
          uint16_t hi[4], lo[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            hi[q] = f_to_bf16(v[q]);
            lo[q] = f_to_bf16(v[q] - bf16_to_f(hi[q]));
          }
          uint8_t* pl0 = reinterpret_cast<uint8_t*>(act) +
                         static_cast<size_t>(2 * b) * (K * 2 + kRowPad) + k * 2;
          *reinterpret_cast<uint2*>(pl0) =
              make_uint2(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]));
          *reinterpret_cast<uint2*>(pl0 + K * 2 + kRowPad) =
              make_uint2(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]));
        } else {
          *reinterpret_cast<float4*>(act + b * kmax + k) = make_float4(v[0], v[1], v[2], v[3]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < B; ++b) ss[b] = warp_sum(ss[b]);
  }

  // The bf16 K-split GEMV on the tensor cores: for every ring tile, 16-row
  // MMA tiles (rows past the tile repeat its last row; their sums are
  // dropped) over the warp's K blocks, 8 MMAs of k16 per block.  Matrix loads
  // of the A (weight rows, rstride(K) apart) and B (activation planes) tiles
  // are conflict-free thanks to the 16-byte row padding.  Output column n of
  // an MMA is plane n & 1 of sequence n >> 1 (zero for sequences past a.B), so
  // lane (g, t) holds rows g and g + 8 of sequence t as hi + lo.
  __device__ void kgemv_mma(int K, int nrows, int rpt, bool pair, float* pbuf) {
    const int nbw = my_blocks(K / kBlk);
    const uint32_t rsb = static_cast<uint32_t>(rstride(K));
    const uint32_t psb = static_cast<uint32_t>(K * 2 + kRowPad);
    // this lane's row address of the B matrix loads (lanes 0..15: rows n of
    // the k8 halves 0 / 1), or the zero row
    const int bn = lane & 7, bh = (lane >> 3) & 1;
    const bool bval = bn < 2 * B;
    const uint32_t bbase = bval ? smem_u32(act) + bn * psb + bh * 16 : zrow;
    const uint32_t bstep = bval ? 2u : 0u;  // bytes per column
    const int am = lane >> 3, ar = lane & 7;
    const int g = lane >> 2, t = lane & 3;
    for (int r0 = 0; r0 < nrows; r0 += rpt) {
      const int nr = min(rpt, nrows - r0);
      const int ntr = pair ? 2 * nr : nr;
      wait_tile();
      if (!ab && nbw > 0) {
        const uint32_t tb = smem_u32(ring + static_cast<size_t>(rs) * slot);
        for (int mt = 0; mt < ntr; mt += 16) {
          const int arow = min(mt + ar + 8 * (am & 1), ntr - 1);
          const uint32_t abase = tb + static_cast<uint32_t>(arow) * rsb + (am >> 1) * 16;
          // one accumulator per k16 step of a block: the MMAs of a block are
          // independent (a dependent chain would cost the MMA latency per step)
          float cs[kBlk / 16][4];
#pragma unroll
          for (int st = 0; st < kBlk / 16; ++st) cs[st][0] = cs[st][1] = cs[st][2] = cs[st][3] = 0.f;
          for (int j = 0; j < nbw; ++j) {
            const uint32_t k0 = static_cast<uint32_t>((warp + j * kCW) * kBlk);
            uint32_t af[kBlk / 16][4], bf[kBlk / 16][2];
#pragma unroll
            for (int st = 0; st < kBlk / 16; ++st) {
              const uint32_t k = k0 + st * 16;
              ldsm_x4(abase + k * 2, af[st]);
              ldsm_x2(bbase + k * bstep, bf[st]);
            }
#pragma unroll
            for (int st = 0; st < kBlk / 16; ++st) mma_16816(cs[st], af[st], bf[st]);
          }
          float c[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            c[q] = ((cs[0][q] + cs[1][q]) + (cs[2][q] + cs[3][q])) +
                   ((cs[4][q] + cs[5][q]) + (cs[6][q] + cs[7][q]));
          }
          if (t < B) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int tr = mt + g + 8 * h;
              if (tr < ntr) {
                const int r = pair ? (tr < nr ? r0 + tr : nrows + r0 + tr - nr) : r0 + tr;
                pbuf[(warp * prow + r) * B + t] = c[2 * h] + c[2 * h + 1];
              }
            }
          }
        }
      }
      release_tile();
    }
  }

  // The K-split GEMV of a stage over ring tiles: rows [0, nrows) of the
  // stage arrive rpt per tile (pair: rpt rows of the first matrix, then the
  // same rows of the second).  Every warp reads every tile and computes the
  // partial dot products of all its rows over the warp's own K blocks, 4 rows
  // at a time; the partials of row r (pair: the second matrix's row r at
  // nrows + r) go to pbuf[warp][r][b].
  __device__ void kgemv(int K, int nrows, int rpt, bool pair, float* pbuf) {
    if constexpr (!W8) {
      kgemv_mma(K, nrows, rpt, pair, pbuf);
      return;
    }
    const int nbw = my_blocks(K / kBlk);
    const uint32_t row_bytes = static_cast<uint32_t>(rstride(K));
    for (int r0 = 0; r0 < nrows; r0 += rpt) {
      const int nr = min(rpt, nrows - r0);
      const int ntr = pair ? 2 * nr : nr;
      wait_tile();
      if (!ab && nbw > 0) {
        const uint32_t tb = smem_u32(ring + static_cast<size_t>(rs) * slot);
        // the partials of tile row tr go to stage row r
        auto put = [&](int tr, const float (&v)[B]) {
          if ((lane & 7) == 0 && tr < ntr) {
            const int r = pair ? (tr < nr ? r0 + tr : nrows + r0 + tr - nr) : r0 + tr;
#pragma unroll
            for (int b = 0; b < B; ++b) pbuf[(warp * prow + r) * B + b] = v[b];
          }
        };
        int g0 = 0;
        for (; g0 + 4 < ntr; g0 += 8) {  // 8 rows at a time while more than 4 remain
          uint32_t rows[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            rows[i] = tb + static_cast<uint32_t>(min(g0 + i, ntr - 1)) * row_bytes;
          const KSums<8, B> s = kdot<8, B, W8>(rows, smem_u32(act), kmax, warp, nbw, lane);
          put(g0 + (lane >> 3), s.s[0]);
          put(g0 + 4 + (lane >> 3), s.s[1]);
        }
        if (g0 < ntr) {
          uint32_t rows[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            rows[i] = tb + static_cast<uint32_t>(min(g0 + i, ntr - 1)) * row_bytes;
          const KSums<4, B> s = kdot<4, B, W8>(rows, smem_u32(act), kmax, warp, nbw, lane);
          put(g0 + (lane >> 3), s.s[0]);
        }
      }
      release_tile();
    }
  }

  // End of a K-split stage: publish the warp's sums of squares, one CTA
  // barrier, then the sums of the warps' partials (fixed order) times the
  // RMSNorm factor of the input (norm) and the int8 row scales, through the
  // stage's epilogue.
  __device__ void kstage_end(int sc, int l, int K, int nrows, bool pair, bool norm,
                             const float (&ss)[B]) {
    float* pbuf = part + pb * (kCW * (prow + 1) * B);
    float* sbuf = pbuf + kCW * prow * B;
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < B; ++b) sbuf[warp * B + b] = ss[b];
    }
    cp_async_wait_all();  // int8 row scales of the stage
    ab = named_sync_or(1, kCT, ab);
    pb ^= 1;
    if (ab) return;
    const int nw = min(kCW, K / kBlk);
    // a fixed pairwise tree over the warps (deterministic; warps without K
    // blocks count as zero), all loads issued before the adds
    auto tree = [&](const float* p, int stride) {
      float v[kCW];
#pragma unroll
      for (int w = 0; w < kCW; ++w) v[w] = w < nw ? p[w * stride] : 0.f;
#pragma unroll
      for (int h = kCW / 2; h > 0; h >>= 1)
#pragma unroll
        for (int w = 0; w < h; ++w) v[w] += v[w + h];
      return v[0];
    };
    for (int t = tid; t < nrows * B; t += kCT) {
      const int r = t / B, b = t % B;
      const float s0 = tree(pbuf + r * B + b, prow * B);
      const float s1 = pair ? tree(pbuf + (nrows + r) * B + b, prow * B) : 0.f;
      float f = 1.f;
      if (norm) f = rsqrtf(tree(sbuf + b, B) / static_cast<float>(K) + a.eps);
      float c0 = f, c1 = f;
      if constexpr (W8) {
        c0 *= wsc[r];
        if (pair) c1 *= wsc[nrows + r];
      }
      epilogue(sc, l, r, b, s0 * c0, s1 * c1);
    }
  }

  // One K-split projection stage: this warp's input, the GEMV over the
  // stage's tiles, the CTA sum and the epilogue.
  __device__ void kstage(int sc, int l, const uint64_t* src, uint32_t f, const uint16_t* g,
                         int K, int nrows, int rpt, bool pair, bool norm) {
    float ss[B];
    if constexpr (W8) load_scales(sc, l);
    warp_input(src, K, f, g, ss, !W8);
    DEC_STAMP(kStampsPerLayer * l + (sc == SQ ? StQIn : sc == SO ? StOIn : sc == SU ? StUIn : StDIn));
    wacc = 0;
#ifdef DEC_PROFILE
    const long long tg = clock64();
#endif
    kgemv(K, nrows, rpt, pair, part + pb * (kCW * (prow + 1) * B));
    DEC_STAMP(kStampsPerLayer * l + (sc == SQ ? StQDot : sc == SO ? StODot : sc == SU ? StUDot : StDDot));
    DEC_SVAL(kStampsPerLayer * l + (sc == SQ ? StWQ : sc == SO ? StWO : sc == SU ? StWU : StWD), wacc);
#ifdef DEC_PROFILE
    DEC_SVAL(kStampsPerLayer * l + (sc == SQ ? StCQ : sc == SO ? StCO : sc == SU ? StCU : StCD),
             static_cast<uint64_t>(clock64() - tg));
#endif
    kstage_end(sc, l, K, nrows, pair, norm, ss);
  }

  // int8 weights: the row scales of this CTA's rows of stage sc of layer l
  // into wsc (cp.async, 4 bytes each), issued before the stage's input polls
  // so that their latency overlaps them; the stage end's wait and barrier
  // complete them.  QKV: rows [q0, q1) of [Wq; Wk; Wv]; gate/up: the gate
  // rows, then the up rows; lm_head: rows [v0, v1).
  __device__ void load_scales(int sc, int l) {
    const float* src0 = nullptr;
    const float* src1 = nullptr;
    int lo = 0, n = 0;
    if (sc == SLM) {
      src0 = a.lm_scale; lo = v0; n = v1 - v0;
    } else if (sc == SQ) {
      const LayerScales& ls = a.wscale[l];
      const int HqD = a.Hq * D, HkvD = a.Hkv * D;
      for (int i = tid; i < q1 - q0; i += kCT) {
        const int r = q0 + i;
        const float* p = r < HqD ? ls.s[1] + r
                       : r < HqD + HkvD ? ls.s[2] + (r - HqD)
                                        : ls.s[3] + (r - HqD - HkvD);
        cp_async4(wsc + i, p);
      }
      return;
    } else if (sc == SO) {
      src0 = a.wscale[l].s[6]; lo = h0; n = h1 - h0;
    } else if (sc == SU) {
      src0 = a.wscale[l].s[8]; src1 = a.wscale[l].s[9]; lo = f0; n = f1 - f0;
    } else {
      src0 = a.wscale[l].s[10]; lo = h0; n = h1 - h0;
    }
    for (int i = tid; i < n; i += kCT) {
      cp_async4(wsc + i, src0 + lo + i);
      if (src1) cp_async4(wsc + n + i, src1 + lo + i);
    }
  }

  // What each projection does with its output row r of sequence b.
  __device__ __forceinline__ void epilogue(int sc, int l, int r, int b, float s0, float s1) {
    switch (sc) {
      case SQ:
        st_tagged(a.x_qkv + static_cast<size_t>(b) * nqkv + q0 + r, s0, flag(l));
        break;
      case SO: {  // o_proj + residual
        const float x = xown[r * B + b] + s0;
        xown[r * B + b] = x;
        if (!(l == 0 && a.stall_cta == cta))
          st_tagged(a.x_mid + static_cast<size_t>(b) * a.H + h0 + r, x, flag(l));
        break;
      }
      case SU:  // SiLU(gate) * up
        st_tagged(a.x_u + static_cast<size_t>(b) * a.F + f0 + r, s0 / (1.0f + __expf(-s0)) * s1,
                  flag(l));
        break;
      case SD: {  // down + residual
        const float x = xown[r * B + b] + s0;
        xown[r * B + b] = x;
        st_tagged(a.x_out + static_cast<size_t>(b) * a.H + h0 + r, x, flag(l));
        if (a.hidden_out)
          a.hidden_out[(static_cast<size_t>(l + 1) * a.B + b) * a.H + h0 + r] = x;
        break;
      }
      default: {  // lm_head logit + running argmax (ties: lowest id)
        const int id = v0 + r;
        if (a.out_logits) a.out_logits[static_cast<size_t>(b) * a.V + id] = s0;
        if (s0 > best_v[b] || (s0 == best_v[b] && id < best_i[b])) {
          best_v[b] = s0;
          best_i[b] = id;
        }
      }
    }
  }

  // Row-group GEMV over ring tiles (the lm_head): rows [0, nrows) arrive
  // `rpt` per tile, K columns (K % 256 == 0); act holds the whole input.
  // One warp computes whole dot products for a group of R rows and reduces
  // its lanes' R partial sums with one transposed butterfly (R = 4: 6
  // shuffles instead of 20); every output is multiplied by rsc[b] (the final
  // RMSNorm factor) and, for int8 rows, the row scale.
  template <int R>
  __device__ void gemv(int K, int nrows, int rpt, int sc, int l, const float (&rsc)[B]) {
    const uint32_t row_bytes = static_cast<uint32_t>(K * eb);
    // A stage of many tiles gives each tile to one warp: only that warp waits
    // for it, computes all its groups and releases it for the whole CTA; the
    // other warps only advance their ring position.  The owner is the ring
    // slot's warp (slot mod warps), so a warp's consecutive tiles are never
    // more than one ring lap apart and its parity waits stay unambiguous.  A
    // stage of a few tiles spreads each tile's groups over the warps.
    const bool owned = (nrows + rpt - 1) / rpt > 2 * kCW && a.nslot >= kCW - 1;
    int gbase = 0;
    for (int r0 = 0; r0 < nrows; r0 += rpt) {
      const int nr = min(rpt, nrows - r0);
      const int ng = (nr + R - 1) / R;
      const bool mine = !owned || rs % kCW == warp;
      if (mine) wait_tile();
      if (mine && !ab) {
        const uint8_t* tb = ring + static_cast<size_t>(rs) * slot;
        int g0 = 0, gs = 1;
        if (!owned) {
          g0 = (warp - gbase) % kCW;
          if (g0 < 0) g0 += kCW;
          gs = kCW;
        }
        for (int gl = g0; gl < ng; gl += gs) {
          uint32_t rows[R];
#pragma unroll
          for (int i = 0; i < R; ++i) {
            const int j = gl * R + i;
            rows[i] = smem_u32(tb) + static_cast<uint32_t>(j < nr ? j : 0) * row_bytes;
          }
          const GroupSums<R, B> gs4 =
              W8 ? group_dot_i8<R, B, (W8 ? W8 : 1)>(rows, smem_u32(act), kmax, K >> 8, lane)
                 : group_dot<R, B>(rows, smem_u32(act), kmax, K >> 8, lane);
          const int ri = R == 4 ? (lane >> 3) : (R == 2 ? (lane >> 4) : 0);
          const bool leader = R == 4 ? ((lane & 7) == 0) : (R == 2 ? ((lane & 15) == 0) : lane == 0);
          const int j = gl * R + ri;
          float s0 = 1.f;
          if constexpr (W8) {
            if (j < nr) s0 = wsc[r0 + j];
          }
#pragma unroll
          for (int b = 0; b < B; ++b)
            if (leader && j < nr && b < a.B) epilogue(sc, l, r0 + j, b, gs4.s[b] * s0 * rsc[b], 0.f);
        }
      }
      gbase += ng;
      if (owned) {
        __syncwarp();
        if (mine && lane == 0 && !ring_dead) mbar_arrive_cnt(&empty[rs], kCW);
        ++rn;
        if (++rs == a.nslot) {
          rs = 0;
          rph ^= 1;
        }
      } else {
        release_tile();
      }
    }
  }

  // ------------------------------------------------------------- attention
  // One K (or V) row slice of the lane from a ring tile: the lane holds dims
  // [e8 * DQ, e8 * DQ + DQ) of tile row r (bf16 rows, or E4M3 codes with the
  // row scales stored after the codes).
  __device__ __forceinline__ void tile_row(const uint8_t* tb, int nr, int r, int e8, int kvsel,
                                           float (&o)[DQ]) const {
    if constexpr (!FP8) {
      const uint8_t* p = tb + (static_cast<size_t>(kvsel) * nr + r) * D * 2 + e8 * DQ * 2;
#pragma unroll
      for (int c = 0; c < DQ / 8; ++c) {
        const uint4 w = reinterpret_cast<const uint4*>(p)[c];
        o[8 * c + 0] = bf16lo(w.x); o[8 * c + 1] = bf16hi(w.x);
        o[8 * c + 2] = bf16lo(w.y); o[8 * c + 3] = bf16hi(w.y);
        o[8 * c + 4] = bf16lo(w.z); o[8 * c + 5] = bf16hi(w.z);
        o[8 * c + 6] = bf16lo(w.w); o[8 * c + 7] = bf16hi(w.w);
      }
    } else {
      const uint8_t* p = tb + (static_cast<size_t>(kvsel) * nr + r) * D + e8 * DQ;
      const int sb = ((nr + 3) & ~3) * 4;
      const float sc = reinterpret_cast<const float*>(tb + 2 * nr * D + kvsel * sb)[r];
#pragma unroll
      for (int c = 0; c < DQ; c += 2) {
        const float2 f2 = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(p + c));
        o[c] = f2.x * sc;
        o[c + 1] = f2.y * sc;
      }
    }
  }

  // Split-K attention of one layer.  Item (b, g, chunk): the query heads of KV
  // head g of sequence b over cached rows [j0, jc) streamed through the ring,
  // plus the new row p_b (from the gathered q/k/v, rotated and rounded as the
  // cache stores it; the CTA whose chunk holds p_b writes it to the cache).
  // In block verification (a.vseq >= 0) an item (g, chunk) serves the query
  // heads of every row of the block at once over the shared prefix, and
  // chunk 0 adds the block's new rows, causally: row i sees new rows 0..i.
  // The item's query heads form groups of two; every lane octet serves one
  // group and scores each of its rows against both heads, so a K/V row is
  // read once per group.  Octet i of a group takes rows i, i + octets per
  // group, ...; each lane holds a D/8-wide slice (3-shuffle dot products).
  // The CTA of chunk 0 combines the chunks' partial softmax states and
  // publishes the head outputs; other chunks publish their partial state and
  // move on.  act holds qs[hi][D], kn[nn][D], vn[nn][D], merge[kCW][hi][D + 2]
  // (hi heads and nn new rows of the item).
  __device__ void attention(int l) {
    const bool ver = a.vseq >= 0;
    const int rep = a.Hq / a.Hkv;
    const int hi = ver ? B * rep : rep;        // query heads of an item (<= 8 when verifying)
    const int nn = ver ? B : 1;                // new rows of an item
    const int ng0 = (hi + 1) >> 1;
    const int ngrp = ng0 <= 1 ? 1 : (ng0 <= 2 ? 2 : 4);  // head groups (of <= 2 heads)
    const int q8 = lane >> 3, e8 = lane & 7;
    const int octet = warp * 4 + q8;
    const int hg = octet % ngrp, oi = octet / ngrp, ostep = 32 / ngrp;
    const int hb = 2 * hg, nh = max(0, min(2, hi - hb));  // this octet's heads hb, hb + 1
    const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e)/sqrt(D)
    float* qs = act;
    float* kn = act + hi * D;
    float* vn = kn + nn * D;
    float* merge = vn + nn * D;
    const LayerPtrs& lw = slw[l];
    const uint32_t f = flag(l);
    const int HqD = a.Hq * D, HkvD = a.Hkv * D;
    // sequence (row) and query head of item head h
    auto hrow = [&](int h, int b) { return ver ? h / rep : b; };
    auto hq = [&](int h, int g) { return g * rep + (ver ? h % rep : h); };
    for (int it = cta; it < pl->n_items; it += nc) {
      int b, g, ci;
      item(it, b, g, ci);
      const int p = ver ? pl->pos[0] : pl->pos[b];  // verify: the prefix length
      const bool live = ver || !pl->done[b];        // a retired sequence writes no cache row
      const int cs = ver ? a.vseq : b;              // cache sequence
      const int j0 = ci * pl->crow;
      const int j1 = ver ? min(j0 + pl->crow, p) : min(j0 + pl->crow, p + 1);
      const int jc = min(j1, p);  // cached rows [j0, jc)
      const bool has_new = ver ? ci == 0 : (p >= j0 && p < j1);
      // -- inputs: vector v < hi is the query head v, then (only for the chunk
      //    holding the new rows) the keys and the values of the nn new rows;
      //    warp w takes vectors w, w + kCW, ...
      const int nvec = hi + (has_new ? 2 * nn : 0);
      for (int v0 = warp; v0 < nvec; v0 += kCW) {
        const int kind = v0 < hi ? 0 : (v0 < hi + nn ? 1 : 2);  // q, k, v
        const int j = kind == 0 ? 0 : (v0 - hi - (kind == 2 ? nn : 0));  // new row
        const int row = kind == 0 ? hrow(v0, b) : (ver ? j : b);
        const int prow = pl->pos[row];
        const uint16_t* gn = kind == 0 ? lw.w[4] : lw.w[5];
        float gq[DL], invf[DL / 2];
#pragma unroll
        for (int k = 0; k < DL; ++k) gq[k] = kind < 2 ? bf16_to_f(__ldg(gn + lane + 32 * k)) : 0.f;
#pragma unroll
        for (int k = 0; k < DL / 2; ++k) invf[k] = __ldg(a.inv_freq + lane + 32 * k);
        const uint64_t* src = a.x_qkv + static_cast<size_t>(row) * nqkv +
                              (kind == 0 ? hq(v0, g) * D : HqD + (kind - 1) * HkvD + g * D);
        uint64_t* ws = stg + warp * kWarpStage;
        warp_gather(ws, D, f, [=](int i) { return src + i; });
        if (!ab) {
          float v[DL];
#pragma unroll
          for (int k = 0; k < DL; ++k) v[k] = __uint_as_float(static_cast<uint32_t>(ws[lane + 32 * k]));
          if (kind < 2) {  // q/k RMSNorm + RoPE
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < DL; ++k) ss = fmaf(v[k], v[k], ss);
            ss = warp_sum(ss);
            const float inv = rsqrtf(ss / static_cast<float>(D) + a.eps);
#pragma unroll
            for (int k = 0; k < DL; ++k) v[k] = v[k] * inv * gq[k];
#pragma unroll
            for (int k = 0; k < DL / 2; ++k) {
              const float ang = __fmul_rn(static_cast<float>(prow), invf[k]);
              float sn, c;
              rope_sincos(ang, &sn, &c);
              const float x1 = v[k], x2 = v[k + DL / 2];
              v[k] = x1 * c - x2 * sn;
              v[k + DL / 2] = x2 * c + x1 * sn;
            }
          }
          if (kind > 0) {
            // the new K / V row as the cache stores it, written by this chunk
            const size_t crow = kv_row(l, kind - 1, cs, g, prow);
            if constexpr (!FP8) {
              uint16_t* dstp = reinterpret_cast<uint16_t*>(a.kv) + crow * D;
#pragma unroll
              for (int k = 0; k < DL; ++k) {
                const uint16_t h = f_to_bf16(v[k]);
                v[k] = bf16_to_f(h);
                if (live) dstp[lane + 32 * k] = h;
              }
            } else {
              uint8_t code[DL];
              const float sc = quantize_row_e4m3<DL>(v, code);
              if (live) {
                uint8_t* dstp = a.kv + crow * D;
#pragma unroll
                for (int k = 0; k < DL; ++k) dstp[lane + 32 * k] = code[k];
                if (lane == 0) a.kv_scales[crow] = sc;
              }
            }
          }
          float* x = kind == 0 ? qs + v0 * D : (kind == 1 ? kn : vn) + j * D;
#pragma unroll
          for (int k = 0; k < DL; ++k) x[lane + 32 * k] = v[k];
        }
      }
      ab = named_sync_or(1, kCT, ab);
      DEC_STAMP(kStampsPerLayer * l + StAttIn);
      wacc = 0;
      // -- this chunk's rows: online softmax per (lane octet, head)
      float qv[2][DQ], acc[2][DQ], m[2], ls[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        m[hh] = -INFINITY;
        ls[hh] = 0.f;
#pragma unroll
        for (int k = 0; k < DQ; ++k) {
          acc[hh][k] = 0.f;
          qv[hh][k] = (!ab && hh < nh) ? qs[(hb + hh) * D + e8 * DQ + k] * qscale : 0.f;
        }
      }
      for (int j = j0; j < jc; j += art) {
        const int nr = min(art, jc - j);
        wait_tile();
        if (j == j0) DEC_STAMP(kStampsPerLayer * l + StAttTile);
        if (!ab) {
          const uint8_t* tb = ring + static_cast<size_t>(rs) * slot;
          // two rows per octet per pass (independent chains; one rescale for both)
          for (int r0 = 0; r0 < nr; r0 += 2 * ostep) {  // warp-uniform trip count
            const int ra = r0 + oi, rb = r0 + ostep + oi;
            const bool oka = ra < nr, okb = rb < nr;
            float sa[2], sb[2];
            {
              float ka[DQ], kb[DQ];
              tile_row(tb, nr, oka ? ra : 0, e8, 0, ka);
              tile_row(tb, nr, okb ? rb : 0, e8, 0, kb);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                float ta[4] = {0.f, 0.f, 0.f, 0.f}, tb4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < DQ; ++k) {
                  ta[k & 3] = fmaf(qv[hh][k], ka[k], ta[k & 3]);
                  tb4[k & 3] = fmaf(qv[hh][k], kb[k], tb4[k & 3]);
                }
                sa[hh] = (ta[0] + ta[1]) + (ta[2] + ta[3]);
                sb[hh] = (tb4[0] + tb4[1]) + (tb4[2] + tb4[3]);
              }
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                sa[hh] += __shfl_xor_sync(0xffffffffu, sa[hh], o);
                sb[hh] += __shfl_xor_sync(0xffffffffu, sb[hh], o);
              }
            if (oka) {
              float va[DQ], vb[DQ];
              tile_row(tb, nr, ra, e8, 1, va);
              tile_row(tb, nr, okb ? rb : ra, e8, 1, vb);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                if (hh < nh) {
                  const float xb = okb ? sb[hh] : -INFINITY;
                  const float mn = fmaxf(m[hh], fmaxf(sa[hh], xb));
                  const float al = exp2f(m[hh] - mn), pa = exp2f(sa[hh] - mn);
                  const float pbv = exp2f(xb - mn);
                  ls[hh] = ls[hh] * al + (pa + pbv);
#pragma unroll
                  for (int k = 0; k < DQ; ++k)
                    acc[hh][k] = fmaf(acc[hh][k], al, fmaf(pa, va[k], pbv * vb[k]));
                  m[hh] = mn;
                }
              }
            }
          }
        }
        release_tile();
      }
      // the new rows, kept by the first octet of each group (a warp-uniform
      // loop: the warps holding those octets shuffle as a whole); head h sees
      // new row j when j <= its own row
      if (!ab && has_new && 4 * warp < ngrp) {
        for (int j = 0; j < nn; ++j) {
          float sv[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float t = 0.f;
#pragma unroll
            for (int k = 0; k < DQ; ++k) t = fmaf(qv[hh][k], kn[j * D + e8 * DQ + k], t);
            t += __shfl_xor_sync(0xffffffffu, t, 4);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            sv[hh] = t;
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh < nh && oi == 0 && (!ver || j <= (hb + hh) / rep)) {
              const float mn = fmaxf(m[hh], sv[hh]);
              const float al = exp2f(m[hh] - mn), pe = exp2f(sv[hh] - mn);
              ls[hh] = ls[hh] * al + pe;
#pragma unroll
              for (int k = 0; k < DQ; ++k) acc[hh][k] = fmaf(acc[hh][k], al, pe * vn[j * D + e8 * DQ + k]);
              m[hh] = mn;
            }
          }
        }
      }
      // merge the octets of the warp that serve the same head group (xor 16,
      // and xor 8 when there is one group; with four groups every octet of a
      // warp serves its own); the first octet of each group writes the warp's
      // state
      if (!ab) {
        if (ngrp < 4) {
#pragma unroll
          for (int o = 8; o <= 16; o <<= 1) {
            if (o == 8 && ngrp != 1) continue;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const float mo = __shfl_xor_sync(0xffffffffu, m[hh], o);
              const float lo = __shfl_xor_sync(0xffffffffu, ls[hh], o);
              const float mn = fmaxf(m[hh], mo);
              const float e1 = (m[hh] == -INFINITY) ? 0.f : exp2f(m[hh] - mn);
              const float e2 = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
              ls[hh] = ls[hh] * e1 + lo * e2;
#pragma unroll
              for (int k = 0; k < DQ; ++k) {
                const float ao = __shfl_xor_sync(0xffffffffu, acc[hh][k], o);
                acc[hh][k] = acc[hh][k] * e1 + ao * e2;
              }
              m[hh] = mn;
            }
          }
        }
        if (q8 < ngrp) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh < nh) {
              float* mg = merge + (static_cast<size_t>(warp) * hi + hb + hh) * (D + 2);
#pragma unroll
              for (int k = 0; k < DQ; ++k) mg[e8 * DQ + k] = acc[hh][k];
              if (e8 == 0) {
                mg[D] = m[hh];
                mg[D + 1] = ls[hh];
              }
            }
          }
        }
      }
      csync();
      DEC_STAMP(kStampsPerLayer * l + StAttRows);
      DEC_SVAL(kStampsPerLayer * l + StWA, wacc);
      // -- this chunk's partial state (m in log2 units, l, unnormalised acc)
      // for thread slots t = tid + kCT * i: (head, element) = t / D, t % D
      constexpr int kSlots = (8 * D + kCT - 1) / kCT;
      const bool combiner = (ci == 0);
      const int pc = a.part_chunks;
      // partial state of chunk c for item head h: the item's states are one
      // contiguous range [chunk][head][D + 2], so that the combiner's window
      // of chunks is a plain address range
      uint64_t* const pbase = a.part + (static_cast<size_t>(b) * a.Hkv + g) * pc * hi * (D + 2);
      auto pstate = [&](int h, int c) { return pbase + (static_cast<size_t>(c) * hi + h) * (D + 2); };
      float RM[kSlots], RL[kSlots], RA[kSlots];
#pragma unroll
      for (int i = 0; i < kSlots; ++i) {
        const int t = tid + kCT * i;
        RM[i] = -INFINITY;
        RL[i] = RA[i] = 0.f;
        if (!ab && t < hi * D) {
          const int h = t / D, d = t % D;
          float M = -INFINITY;
          for (int w = 0; w < kCW; ++w) M = fmaxf(M, merge[(w * hi + h) * (D + 2) + D]);
          float Ls = 0.f, A = 0.f;
          for (int w = 0; w < kCW; ++w) {
            const float* mg = merge + (w * hi + h) * (D + 2);
            const float e = (mg[D] == -INFINITY) ? 0.f : exp2f(mg[D] - M);
            Ls += mg[D + 1] * e;
            A += mg[d] * e;
          }
          if (combiner) {
            RM[i] = M;
            RL[i] = Ls;
            RA[i] = A;
          } else {
            uint64_t* pp = pstate(h, ci);
            st_tagged(pp + d, A, f);
            if (d == 0) {
              st_tagged(pp + D, M, f);
              st_tagged(pp + D + 1, Ls, f);
            }
          }
        }
      }
      DEC_STAMP(kStampsPerLayer * l + StAttPub);
      if (combiner) {  // uniform over the CTA: ci is the item's
        const int nc1 = pl->nchunk[ver ? 0 : b] - 1;
        const int win = kStageWords / (hi * (D + 2));
        for (int c0 = 1; c0 <= nc1; c0 += win) {
          const int nw = min(win, nc1 - c0 + 1);
          const uint64_t* const wsrc = pstate(0, c0);  // chunks c0 .. c0 + nw - 1, every head
          gather(nw * hi * (D + 2), f, [=](int w) { return wsrc + w; });
          if (!ab) {
#pragma unroll
            for (int i = 0; i < kSlots; ++i) {
              const int t = tid + kCT * i;
              if (t < hi * D) {
                const int h = t / D, d = t % D;
                for (int cc = 0; cc < nw; ++cc) {
                  const uint64_t* pw = stg + (cc * hi + h) * (D + 2);
                  const float Mc = __uint_as_float(static_cast<uint32_t>(pw[D]));
                  const float Lc = __uint_as_float(static_cast<uint32_t>(pw[D + 1]));
                  const float Ac = __uint_as_float(static_cast<uint32_t>(pw[d]));
                  const float mn = fmaxf(RM[i], Mc);
                  const float e1 = exp2f(RM[i] - mn), e2 = exp2f(Mc - mn);
                  RL[i] = RL[i] * e1 + Lc * e2;
                  RA[i] = RA[i] * e1 + Ac * e2;
                  RM[i] = mn;
                }
              }
            }
          }
          csync();  // stg is refilled by the next window
        }
        DEC_STAMP(kStampsPerLayer * l + StAttCmb);
        if (!ab) {
#pragma unroll
          for (int i = 0; i < kSlots; ++i) {
            const int t = tid + kCT * i;
            if (t < hi * D) {
              const int h = t / D, d = t % D;
              st_tagged(a.x_o + static_cast<size_t>(hrow(h, b)) * HqD + hq(h, g) * D + d,
                        RA[i] / RL[i], f);
            }
          }
        }
      }
      csync();
    }
  }

  // ------------------------------------------------------------- one step
  __device__ void one_step() {
    const int H = a.H, F = a.F, HqD = a.Hq * D;
#pragma unroll
    for (int b = 0; b < B; ++b) {
      best_v[b] = -INFINITY;
      best_i[b] = 0x7fffffff;
    }
    DEC_STAMP(kStampsPerLayer * a.L + StBegin);
    // the CTA's residual rows start as the embedding rows
    for (int i = tid; i < (h1 - h0) * B; i += kCT) {
      const int r = i / B, b = i % B;
      const float x = bf16_to_f(a.embed[static_cast<size_t>(pl->tok[b]) * H + h0 + r]);
      xown[r * B + b] = x;
      if (a.hidden_out) a.hidden_out[static_cast<size_t>(b) * H + h0 + r] = x;
    }
    for (int l = 0; l < a.L; ++l) {
      const LayerPtrs& lw = slw[l];
      const uint32_t f = flag(l);
      // QKV (the layer-0 input is the embedding row)
      // the four projection stages share one copy of the stage code
#pragma unroll 1
      for (int st = 0; st < 4; ++st) {
        if (st == 1) {
          attention(l);
          DEC_STAMP(kStampsPerLayer * l + StAtt);
        }
        const int sc = st == 0 ? SQ : st == 1 ? SO : st == 2 ? SU : SD;
        const uint64_t* src = st == 0 ? (l == 0 ? nullptr : a.x_out)
                              : st == 1 ? a.x_o : st == 2 ? a.x_mid : a.x_u;
        const uint16_t* gn = st == 0 ? lw.w[0] : st == 2 ? lw.w[7] : nullptr;
        const int K = st == 1 ? HqD : st == 3 ? F : H;
        const int nrows = st == 0 ? q1 - q0 : st == 2 ? f1 - f0 : h1 - h0;
        const int rpt = st == 0 ? rpt_h : st == 1 ? rpt_o : st == 2 ? rpt_u : rpt_d;
        kstage(sc, l, src, st == 0 ? flag(l - 1) : f, gn, K, nrows, rpt, st == 2, (st & 1) == 0);
        DEC_STAMP(kStampsPerLayer * l + (st == 0 ? StQkv : st == 1 ? StO : st == 2 ? StU : StD));
      }
    }
    // final norm + lm_head: the whole input in act, the norm factor applied
    // to every logit
    DEC_STAMP(kStampsPerLayer * a.L + StLmStart);
    {
      float ss[B], rsc[B];
      if constexpr (W8) load_scales(SLM, a.L);
      warp_input(a.x_out, H, flag(a.L - 1), a.final_norm, ss, false);
      float* sbuf = part + pb * (kCW * (prow + 1) * B) + kCW * prow * B;
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < B; ++b) sbuf[warp * B + b] = ss[b];
      }
      cp_async_wait_all();
      ab = named_sync_or(1, kCT, ab);
      pb ^= 1;
      const int nw = min(kCW, H / kBlk);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float t2 = 0.f;
        for (int w = 0; w < nw; ++w) t2 += sbuf[w * B + b];
        rsc[b] = rsqrtf(t2 / static_cast<float>(H) + a.eps);
      }
      DEC_STAMP(kStampsPerLayer * a.L + StLmGath);
      gemv<4>(H, v1 - v0, rpt_lm, SLM, a.L, rsc);
    }
    DEC_STAMP(kStampsPerLayer * a.L + StLmDone);
    // CTA argmax -> one 64-bit atomicMax per sequence (ties: lowest id)
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float v = best_v[b];
      int i = best_i[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) {
          v = ov;
          i = oi;
        }
      }
      if (lane == 0) {
        bredf[kCW * B + warp * B + b] = v;
        bredi[warp * B + b] = i;
      }
    }
    csync();
    if (tid < a.B && !ab) {
      const int b = tid;
      float v = bredf[kCW * B + b];
      int i = bredi[b];
      for (int w = 1; w < kCW; ++w) {
        const float ov = bredf[kCW * B + w * B + b];
        const int oi = bredi[w * B + b];
        if (ov > v || (ov == v && oi < i)) {
          v = ov;
          i = oi;
        }
      }
      if (i != 0x7fffffff) {
        const unsigned long long key =
            (static_cast<unsigned long long>(order_key(v)) << 32) | static_cast<uint32_t>(~i);
        atomicMax(&a.amax_key[b], key);
      }
    }
    DEC_STAMP(kStampsPerLayer * a.L + StEnd);
  }

  // After this CTA's argmax of step st is in: the CTA that arrives last takes
  // the step's ids from the argmax keys (clearing them for the next step),
  // writes out_ids[st] and publishes the ids as tagged words for the next
  // step.  A retired sequence keeps emitting the end token.  For a multi-step
  // launch it also advances the caller's positions (a sequence stays at the
  // row of the step that emitted the end token) and, when every sequence has
  // retired or the next step would be invalid, fills the remaining steps'
  // ids.  One thread.
  __device__ void step_end(int st) {
    __threadfence();
    const unsigned old = atomicAdd(a.step_cnt, 1u);
    if (old != static_cast<unsigned>(st + 1) * static_cast<unsigned>(nc) - 1u) return;
    __threadfence();
    int32_t* out = a.out_ids + static_cast<size_t>(st) * a.B;
    int all = 1, bad = 0;
    for (int b = 0; b < a.B; ++b) {
      const unsigned long long key = atomicExch(&a.amax_key[b], 0ull);
      int id = key == 0ull ? -1 : static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffull));
      const bool was_done = cplan->done[b] != 0;
      if (was_done) id = a.eos;
      out[b] = id;
      const bool done = was_done || (a.eos >= 0 && id == a.eos);
      const int np = done ? cplan->pos[b] : cplan->pos[b] + 1;
      if (a.gen_pos) a.gen_pos[b] = np;
      all &= done;
      if (!done && (id < 0 || id >= a.V)) bad |= kDevBadTok;
      if (!done && np >= a.max_ctx) bad |= kDevBadPos;
      st_tagged(a.tokw + b, __int_as_float(id), tok_flag(st));
    }
    if (st + 1 < a.n_steps && (all || bad)) {
      if (bad) atomicOr(a.status, bad);
      for (int s2 = st + 1; s2 < a.n_steps; ++s2)
        for (int b = 0; b < a.B; ++b)
          a.out_ids[static_cast<size_t>(s2) * a.B + b] = bad ? -1 : a.eos;
    }
  }

  // The consumers' step loop: one step per iteration, then the next step's
  // ids and plan (thread 0 polls, the others wait at the barrier).
  __device__ void consumer() {
    for (int st = 0;; ++st) {
      seq = seq0 + static_cast<uint32_t>(st);
      one_step();
      csync();  // this CTA's argmax keys are in
      if (tid == 0 && !ab) step_end(st);
      if (st + 1 >= a.n_steps || ab) break;
      if (tid == 0) sints[0] = next_step(*cplan, tok_flag(st)) ? 0 : 1;
      ab = named_sync_or(1, kCT, tid == 0 ? sints[0] : 0);
      if (ab || cplan->bad || cplan->all_done) break;
    }
  }
};

template <int B, int D, bool FP8, int W8>
__global__ void __launch_bounds__(kStepThreads, 1) step_kernel(const StepArgs a, int kmax) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Cta<B, D, FP8, W8> c(a, smem, kmax);
  // ---- set-up: layer pointer table, barriers, the first step's inputs and
  // plan (both sides' copies), validation
  {
    const uint64_t* src = reinterpret_cast<const uint64_t*>(a.layers);
    uint64_t* dst = reinterpret_cast<uint64_t*>(const_cast<LayerPtrs*>(c.slw));
    for (int i = threadIdx.x; i < a.L * kLayerPtrs; i += blockDim.x) dst[i] = src[i];
  }
  if (threadIdx.x < 4) asm volatile("st.shared.u32 [%0], %1;" ::"r"(c.zrow + 4 * threadIdx.x), "r"(0u));
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nslot; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], kCW);
    }
    fence_mbar_init();
    int bad = 0;
    Plan& P = *c.cplan;
    for (int b = 0; b < a.B; ++b) {
      const int p = a.positions[b], t = a.token_ids[b];
      P.pos[b] = p;
      P.tok[b] = t;
      P.done[b] = 0;
      if (p < 0 || p >= a.max_ctx) bad |= kDevBadPos;
      if (a.vseq >= 0 && p != a.positions[0] + b) bad |= kDevBadPos;  // a block is consecutive
      if (t < 0 || t >= a.V) bad |= kDevBadTok;
    }
    P.bad = bad;
    if (!bad) c.make_plan(P);
    *c.pplan = P;
    c.sints[1] = bad;
    c.sints[2] = static_cast<int>(ld_relaxed_u32(a.seq));
    if (bad && blockIdx.x == 0) atomicOr(a.status, bad);
  }
  __syncthreads();
  const int bad = c.sints[1];
  c.seq0 = c.seq = static_cast<uint32_t>(c.sints[2]);
  if (!bad) {
    if (c.warp == kCW) c.producer();
    else c.consumer();
  }
  __syncthreads();
  // ---- exit: the last CTA resets the launch state; a launch that saw an
  // invalid input or ran out of a wait reports -1 for every id
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.exit_cnt, 1u);
    if (old == gridDim.x - 1) {
      __threadfence();
      const int aborted = ld_relaxed_i32(a.abort_flag);
      if (bad || aborted) {
        for (int i = 0; i < a.n_steps * a.B; ++i) a.out_ids[i] = -1;
        for (int b = 0; b < a.B; ++b) atomicExch(&a.amax_key[b], 0ull);
      }
      atomicExch(a.abort_flag, 0);
      atomicExch(a.step_cnt, 0u);
      atomicExch(a.exit_cnt, 0u);
      atomicAdd(a.seq, static_cast<unsigned>(a.n_steps));
      __threadfence();
    }
  }
}

template <int B, int D, bool FP8, int W8>
cudaError_t launch_bd(const StepArgs& a, int ctas, size_t smem, int kmax,
                      cudaStream_t s) {
  auto k = step_kernel<B, D, FP8, W8>;
  StepArgs args = a;
  void* params[] = {&args, &kmax};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k), dim3(ctas),
                                     dim3(kStepThreads), params, smem, s);
}

template <int B, int D, bool FP8, int W8>
cudaError_t attr_bd(size_t smem) {
  return cudaFuncSetAttribute(step_kernel<B, D, FP8, W8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
}

}  // namespace

static int kmax_of(int H, int F, int HqD) {
  int k = H > F ? H : F;
  return k > HqD ? k : HqD;
}
size_t step_smem_bytes(int nslot, int slot_bytes, int B, int H, int F, int HqD, int D, int rep,
                       int wsc_n, int prow) {
  return carve(nslot, slot_bytes, B, kmax_of(H, F, HqD), D, rep, wsc_n, prow).total;
}

void step_ring(int B, int H, int F, int HqD, int D, int rep, int wsc_n, int prow, int smem_optin,
               int* nslot, int* slot_bytes) {
  auto most = [&](int sb) {
    int best = 0;
    for (int n = 1; n <= 16; ++n)
      if (step_smem_bytes(n, sb, B, H, F, HqD, D, rep, wsc_n, prow) <=
          static_cast<size_t>(smem_optin))
        best = n;
    return best;
  };
  const int nl = most(kSlotBytesLarge);
  if (nl >= kMinLargeSlots) {
    *nslot = nl;
    *slot_bytes = kSlotBytesLarge;
  } else {
    *nslot = most(kSlotBytesSmall);
    *slot_bytes = kSlotBytesSmall;
  }
}

// The largest split_at range of n over `ctas` parts.
static int most_rows(int n, int ctas) {
  int m = 0;
  for (int i = 0; i < ctas; ++i) {
    const int c = split_at(n, ctas, i + 1) - split_at(n, ctas, i);
    m = c > m ? c : m;
  }
  return m;
}

int step_wsc_slots(int H, int F, int nqkv, int V, int ctas) {
  int m = most_rows(nqkv, ctas);
  m = most_rows(H, ctas) > m ? most_rows(H, ctas) : m;
  m = 2 * most_rows(F, ctas) > m ? 2 * most_rows(F, ctas) : m;
  m = most_rows(V, ctas) > m ? most_rows(V, ctas) : m;
  return m;
}

int step_part_rows(int H, int F, int nqkv, int ctas) {
  int m = most_rows(nqkv, ctas);
  m = most_rows(H, ctas) > m ? most_rows(H, ctas) : m;
  m = 2 * most_rows(F, ctas) > m ? 2 * most_rows(F, ctas) : m;
  return m;
}

// Sets the dynamic shared-memory limit of the kernel instantiations a
// handle launches (once, when the handle is created).
cudaError_t step_set_smem(int B, int D, int w8, size_t smem) {
  cudaError_t e = cudaErrorInvalidValue;
#define DEC_ATTR_W(BB, DD, WW)                                                  \
  {                                                                             \
    e = attr_bd<BB, DD, false, WW>(smem);                                       \
    if (e == cudaSuccess) e = attr_bd<BB, DD, true, WW>(smem);                  \
  }
#define DEC_ATTR(BB, DD)                                                        \
  if (B == BB && D == DD) {                                                     \
    if (w8 == 1) DEC_ATTR_W(BB, DD, 1)                                          \
    else if (w8 == 2) DEC_ATTR_W(BB, DD, 2)                                     \
    else DEC_ATTR_W(BB, DD, 0)                                                  \
  }
  DEC_ATTR(1, 128) DEC_ATTR(2, 128) DEC_ATTR(3, 128) DEC_ATTR(4, 128)
  DEC_ATTR(1, 64) DEC_ATTR(2, 64) DEC_ATTR(3, 64) DEC_ATTR(4, 64)
#undef DEC_ATTR
#undef DEC_ATTR_W
  return e;
}

cudaError_t launch_step_small(const StepArgs& a, int ctas, size_t smem, cudaStream_t s) {
  const int HqD = a.Hq * a.D;
  const int kmax = kmax_of(a.H, a.F, HqD);
  const bool f8 = a.kv_fp8 != 0;
#define DEC_CASE_W(BB, DD, WW)                                                      \
  return f8 ? launch_bd<BB, DD, true, WW>(a, ctas, smem, kmax, s)                    \
            : launch_bd<BB, DD, false, WW>(a, ctas, smem, kmax, s);
#define DEC_CASE(BB, DD)                                                            \
  if (a.B == BB && a.D == DD) {                                                     \
    if (a.w8 == 1) DEC_CASE_W(BB, DD, 1)                                            \
    if (a.w8 == 2) DEC_CASE_W(BB, DD, 2)                                            \
    DEC_CASE_W(BB, DD, 0)                                                           \
  }
  DEC_CASE(1, 128) DEC_CASE(2, 128) DEC_CASE(3, 128) DEC_CASE(4, 128)
  DEC_CASE(1, 64) DEC_CASE(2, 64) DEC_CASE(3, 64) DEC_CASE(4, 64)
#undef DEC_CASE
#undef DEC_CASE_W
  return cudaErrorInvalidValue;
}

}  // namespace dec
