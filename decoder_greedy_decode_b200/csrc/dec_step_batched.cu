// dec_step_batched.cu -- the decode step for batches of 5..64 sequences.
//
// The step computes what the persistent single-sequence kernel computes
// (embed; 28 x [RMSNorm, QKV, q/k RMSNorm + RoPE, KV append, GQA attention,
// o_proj + residual, RMSNorm, SwiGLU MLP + residual]; final norm, lm_head,
// argmax: "Qwen3-ASR -- Latency & Bottleneck Analysis", 03 Decode), for
// many sequences at once.  With B sequences every weight row meets B
// activation rows, so the projections are dense [N x K] x [K x B]
// contractions and run on the tensor cores: tcgen05.mma with bf16 operands
// staged by TMA (128-byte swizzle) and fp32 accumulators in tensor memory,
// one 128-row weight tile x 64 sequences per CTA, split along K so that a
// layer's small matrices still cover every SM.  The split partials meet in
// L2 and small CUDA-core kernels finish each phase (residual add, RMSNorm,
// q/k norm, rotation and cache append, SwiGLU).  The Baseten Qwen3-ASR
// article ("KV cache quantization") notes that at high concurrency the
// attention over the cache takes the largest share of decode time: it is a
// split-K kernel over (sequence, KV head, chunk) streaming K/V rows (bf16
// or E4M3 codes + fp32 row scales) through shared memory.
//
// Numerics: weights and the KV cache as stored; the residual stream, norms,
// softmax and accumulators fp32.  A tensor-core activation operand (the
// normalised hidden state, the attention output, the SwiGLU output) is held
// as two bf16 planes, hi = bf16(x) and lo = bf16(x - hi), and every K step
// issues one MMA per plane: W x = W hi + W lo to about 2^-17 of x, so the
// batched step keeps the fp32-activation accuracy of the single-sequence
// kernel (the weights are exactly bf16).  The extra MMAs are free here: the
// step is bound by HBM, not by the tensor pipe.
#include <cuda.h>
#include <cuda_runtime.h>

#include <new>
#include <vector>

#include "dec.h"
#include "dec_internal.h"
#include "dec_ptx.cuh"
#include "dec_quant.cuh"
#include "dec_rope.cuh"
#include "dec_tc.cuh"

namespace dec {
namespace {

constexpr int kTileM = 128;                       // weight rows per tile (MMA M)
constexpr int kTileN = kMaxBatch;                 // sequences per tile (MMA N)
constexpr int kChunkK = 64;                       // K columns per pipeline stage
constexpr int kABytes = kTileM * kChunkK * 2;     // 16 KB
constexpr int kBRows = 2 * kTileN;               // activation rows: hi plane, then lo plane
constexpr int kBBytes = kBRows * kChunkK * 2;     // 16 KB
constexpr int kLoOffset = kTileN * kChunkK * 2;   // lo plane inside a B tile (8 KB)
constexpr int kStageBytes = kABytes + kBBytes;    // 32 KB
constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 128;                 // 4 warps = the 4 TMEM sub-partitions
constexpr uint32_t kTmemCols = 64;                // fp32 accumulator columns (= kTileN)
constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, kTileN);
constexpr int kLmStride = kTileM + 4;             // transposed logits tile row (floats)
constexpr size_t kGemmSmem = 1024 + kGemmStages * kStageBytes + 256;
constexpr int kMaxAttnChunks = 32;
constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttStages = 4;
constexpr int kAttTileRows = 32;
constexpr int kAttMaxRep = 8;
constexpr int kRowThreads = 256;

static_assert(kTileN == 64 && kTmemCols == 64, "epilogue reads 4 x 16 accumulator columns");
static_assert(kTileN * kLmStride * 4 <= kGemmStages * kStageBytes, "logits tile fits the ring");

// Bounded mbarrier wait: the copies and MMAs always complete; the bound only
// guards the GPU.  Returns false (and raises the timeout status) if it ran
// out; with `give_up` it also returns false as soon as another wait of the
// step has timed out, so that a stuck step ends quickly.
__device__ bool bt_wait(uint64_t* bar, uint32_t parity, unsigned long long limit, int* status,
                        bool give_up = true) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_wait(bar, parity, 20000)) return true;
    if (it == 0) {
      t0 = globaltimer();
    } else {
      if (give_up && (ld_relaxed_i32(status) & DEC_DEV_TIMEOUT)) return false;
      if (globaltimer() - t0 > limit) {
        atomicOr(status, DEC_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// ===================================================================== GEMM
// One launch computes, for up to three weight matrices stacked along their
// output rows, out[b][n] = sum_k W[n][k] * X[b][k] for b < 64 (X is the
// activation buffer: rows 0..63 the hi plane, 64..127 the lo plane; rows of
// sequences >= B are ignored).
// Grid: (stacked 128-row tiles, K splits).  MODE 0 writes the fp32 partial
// of split s to part[s][b][off + n]; MODE 1 (lm_head, one split) writes the
// logits (optional) and folds the tile's argmax into a 64-bit atomicMax key
// per sequence: (order-preserving bits of the logit << 32) | ~id, so equal
// logits keep the lowest id.
struct GemmArgs {
  int n_mat;
  int rows[3];   // output rows of each stacked matrix
  int tiles[3];  // ceil(rows / 128)
  int off[3];    // first partial column of each matrix
  int k_chunks;  // ceil(K / 64)
  int splits;
  int ldp;       // partial row length (sum of rows)
  int B;
  float* part;   // [splits][64][ldp]
  unsigned long long* keys;  // MODE 1: [64]
  float* logits;             // MODE 1: [B][rows[0]] or null
  int* status;
  unsigned long long timeout_ns;
};

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads) gemm_kernel(const __grid_constant__ CUtensorMap w0,
                                                            const __grid_constant__ CUtensorMap w1,
                                                            const __grid_constant__ CUtensorMap w2,
                                                            const __grid_constant__ CUtensorMap xm,
                                                            const GemmArgs g) {
  extern __shared__ uint8_t dsm[];
  const uint32_t raw = smem_u32(dsm);
  uint8_t* sm = dsm + (((raw + 1023u) & ~1023u) - raw);  // swizzle atoms need 1024-B alignment
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kGemmStages * kStageBytes);
  uint64_t* empty = full + kGemmStages;
  uint64_t* done = empty + kGemmStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // stacked tile -> (matrix, tile); selects rather than indexing keep the
  // parameter arrays out of local memory
  int mat = 0, tile = blockIdx.x;
  if (g.n_mat > 1 && tile >= g.tiles[0]) {
    tile -= g.tiles[0];
    mat = 1;
    if (g.n_mat > 2 && tile >= g.tiles[1]) {
      tile -= g.tiles[1];
      mat = 2;
    }
  }
  const CUtensorMap* wm = mat == 0 ? &w0 : (mat == 1 ? &w1 : &w2);
  const int mrows = mat == 0 ? g.rows[0] : (mat == 1 ? g.rows[1] : g.rows[2]);
  const int moff = mat == 0 ? g.off[0] : (mat == 1 ? g.off[1] : g.off[2]);
  const int split = blockIdx.y;
  const int c0 = split * g.k_chunks / g.splits;
  const int nch = (split + 1) * g.k_chunks / g.splits - c0;

  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: weight tile (streamed once: evict first) + activations
      tma_prefetch_map(wm);
      tma_prefetch_map(&xm);
      const uint64_t pw = policy_evict_first();
      const uint64_t px = policy_evict_last();
      int issued = 0;
      for (int i = 0; i < nch; ++i) {
        const int s = i % kGemmStages;
        if (i >= kGemmStages &&
            !bt_wait(&empty[s], ((i / kGemmStages) - 1) & 1, g.timeout_ns, g.status))
          break;
        const uint32_t st = smem_u32(sm + s * kStageBytes);
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(st, wm, (c0 + i) * kChunkK, tile * kTileM, smem_u32(&full[s]), pw);
        tma_load_2d(st + kABytes, &xm, (c0 + i) * kChunkK, 0, smem_u32(&full[s]), px);
        ++issued;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int s = 0; s < kGemmStages && s < issued; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % kGemmStages);
        bt_wait(&full[s], (last / kGemmStages) & 1, g.timeout_ns, g.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer: 4 x (128 x 64 x 16) per stage, accumulating in TMEM
      for (int i = 0; i < nch; ++i) {
        const int s = i % kGemmStages;
        if (!bt_wait(&full[s], (i / kGemmStages) & 1, g.timeout_ns, g.status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sm + s * kStageBytes);
        const uint64_t ad = sw128_desc(a_addr), bh = sw128_desc(a_addr + kABytes),
                       bl = sw128_desc(a_addr + kABytes + kLoOffset);
#pragma unroll
        for (int kk = 0; kk < kChunkK / 16; ++kk) {
          tc_mma_bf16(tmem, ad + 2 * kk, bh + 2 * kk, kIdesc, (i | kk) != 0 ? 1u : 0u);
          tc_mma_bf16(tmem, ad + 2 * kk, bl + 2 * kk, kIdesc, 1u);
        }
        tc_commit(smem_u32(&empty[s]));  // stage s is free once these MMAs are done
      }
      tc_commit(smem_u32(done));
    }
    __syncwarp();
  }

  // ---- epilogue: TMEM lane = weight row (warp w: rows 32w..32w+31), column = sequence
  bt_wait(done, 0, g.timeout_ns, g.status);
  tc_fence_after();
  float v[kTileN];
  const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
  for (int c = 0; c < kTileN; c += 16) tc_ld16(tl + c, v + c);
  tc_wait_ld();
  const int m = warp * 32 + lane;
  const int row = tile * kTileM + m;
  const bool valid = row < mrows;

  if constexpr (MODE == 0) {
    if (valid) {
      float* dst = g.part + static_cast<size_t>(split) * kTileN * g.ldp + moff + row;
#pragma unroll
      for (int b = 0; b < kTileN; ++b)
        if (b < g.B) dst[static_cast<size_t>(b) * g.ldp] = v[b];
    }
  } else {
    const int V = g.rows[0];
    if (g.logits && valid) {
#pragma unroll
      for (int b = 0; b < kTileN; ++b)
        if (b < g.B) g.logits[static_cast<size_t>(b) * V + row] = v[b];
    }
    // transpose through the (now idle) stage buffers: T[b][m]
    float* T = reinterpret_cast<float*>(sm);
#pragma unroll
    for (int b = 0; b < kTileN; ++b) T[b * kLmStride + m] = v[b];
    __syncthreads();
    // thread (b = tid / 2, half = tid % 2) scans rows half*64 .. half*64+63 of sequence b
    const int b = tid >> 1, half = tid & 1;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    if (b < g.B) {
      const float4* t4 = reinterpret_cast<const float4*>(T + b * kLmStride + half * 64);
      for (int j = 0; j < 16; ++j) {
        const float4 x = t4[j];
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int id = tile * kTileM + half * 64 + 4 * j + e;
          if (id < V && xs[e] > best) {  // ascending ids: strict > keeps the lowest on ties
            best = xs[e];
            bi = id;
          }
        }
      }
    }
    const float ob = __shfl_xor_sync(0xffffffffu, best, 1);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, 1);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
    if (half == 0 && b < g.B && bi != 0x7fffffff)
      atomicMax(&g.keys[b], (static_cast<unsigned long long>(order_key(best)) << 32) |
                                static_cast<uint32_t>(~bi));
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ================================================================ row kernels
struct StepArgs2 {
  int B, L, H, Hq, Hkv, D, F, V;
  float eps;
  const int32_t* tok;
  const int32_t* pos;
  int32_t* out;
  const uint16_t* embed;
  float* x;           // residual stream [64][H] fp32
  uint16_t* act_h;    // [2][64][H]   normalised hidden state (GEMM operand, hi/lo planes)
  uint16_t* act_o;    // [2][64][HqD] attention output
  uint16_t* act_u;    // [2][64][F]   SwiGLU output
  float* q;           // [64][Hq][D] fp32 rotated queries
  float* part;        // GEMM split partials
  unsigned long long* keys;  // [64]
  int* bad;           // this step's input-validation bits
  int* status;
  const float* inv_freq;
  float* hidden;      // [L+1][B][H] or null
  uint8_t* kv;
  float* kv_scales;
  int kv_batch, max_ctx;
};

// x as the two bf16 planes of a tensor-core activation buffer [2][64][K]
__device__ __forceinline__ void put_act(uint16_t* buf, int b, int n, int K, float x) {
  const uint16_t hi = f_to_bf16(x);
  buf[static_cast<size_t>(b) * K + n] = hi;
  buf[static_cast<size_t>(kTileN + b) * K + n] = f_to_bf16(x - bf16_to_f(hi));
}

__device__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read from a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

// Validation of every sequence's token and position (all CTAs reach the same
// answer), the embedding row, the first input RMSNorm.  Grid: B.
__global__ void __launch_bounds__(kRowThreads) embed_kernel(const StepArgs2 a, const uint16_t* g_in) {
  __shared__ float red[kRowThreads / 32];
  __shared__ int s_bad;
  const int b = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int i = tid; i < a.B; i += blockDim.x) {
    const int t = a.tok[i], p = a.pos[i];
    if (t < 0 || t >= a.V) atomicOr(&s_bad, DEC_DEV_BAD_TOKEN);
    if (p < 0 || p >= a.max_ctx) atomicOr(&s_bad, DEC_DEV_BAD_POSITION);
  }
  __syncthreads();
  const int bad = s_bad;
  if (b == 0 && tid == 0) {
    *a.bad = bad;
    if (bad) atomicOr(a.status, bad);
  }
  if (tid == 0) a.keys[b] = 0ull;
  int t = a.tok[b];
  if (t < 0 || t >= a.V) t = 0;
  const uint16_t* e = a.embed + static_cast<size_t>(t) * a.H;
  float* x = a.x + static_cast<size_t>(b) * a.H;
  float ss = 0.f;
  for (int n = tid; n < a.H; n += blockDim.x) {
    const float xv = bf16_to_f(e[n]);
    x[n] = xv;
    if (a.hidden) a.hidden[static_cast<size_t>(b) * a.H + n] = xv;
    ss = fmaf(xv, xv, ss);
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / static_cast<float>(a.H) + a.eps);
  for (int n = tid; n < a.H; n += blockDim.x)
    put_act(a.act_h, b, n, a.H, x[n] * inv * bf16_to_f(g_in[n]));
}

// x += sum of the GEMM split partials; optionally record x; act = bf16(RMSNorm(x) * g).
// Grid: B.
__global__ void __launch_bounds__(kRowThreads) resid_norm_kernel(const StepArgs2 a, int splits,
                                                                 const uint16_t* gain,
                                                                 float* hidden_slot) {
  __shared__ float red[kRowThreads / 32];
  const int b = blockIdx.x, tid = threadIdx.x, H = a.H;
  float* x = a.x + static_cast<size_t>(b) * H;
  float ss = 0.f;
  for (int n = tid; n < H; n += blockDim.x) {
    float xv = x[n];
    for (int s = 0; s < splits; ++s) xv += a.part[(static_cast<size_t>(s) * kTileN + b) * H + n];
    x[n] = xv;
    if (hidden_slot) hidden_slot[static_cast<size_t>(b) * H + n] = xv;
    ss = fmaf(xv, xv, ss);
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / static_cast<float>(H) + a.eps);
  for (int n = tid; n < H; n += blockDim.x) put_act(a.act_h, b, n, H, x[n] * inv * bf16_to_f(gain[n]));
}

// u = silu(gate) * up from the split partials [s][b][gate F | up F].  Grid: (ceil(F/256), B).
__global__ void __launch_bounds__(kRowThreads) swiglu_kernel(const StepArgs2 a, int splits) {
  const int b = blockIdx.y, n = blockIdx.x * blockDim.x + threadIdx.x, F = a.F;
  if (n >= F) return;
  float gs = 0.f, us = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* pr = a.part + (static_cast<size_t>(s) * kTileN + b) * (2 * F);
    gs += pr[n];
    us += pr[F + n];
  }
  put_act(a.act_u, b, n, F, gs / (1.0f + __expf(-gs)) * us);
}

// Per (sequence, head) of the stacked QKV output: sum the split partials,
// RMSNorm + rotate q and k heads, store the rotated query, append the new K
// and V rows to the cache (bf16, or E4M3 codes + row scale).  One warp per
// head; lane holds elements lane + 32 k, so rotation pairs (i, i + D/2) sit
// in the same lane.  Grid: (ceil((Hq + 2 Hkv) / 4), B).
template <int D, bool FP8>
__global__ void __launch_bounds__(128) qkv_post_kernel(const StepArgs2 a, int splits, int l,
                                                       const uint16_t* gq, const uint16_t* gk) {
  constexpr int DL = D / 32;
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int head = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int nh = a.Hq + 2 * a.Hkv;
  if (head >= nh) return;
  const int ldp = nh * D;
  float v[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) {
    const int n = head * D + lane + 32 * k;
    float s = 0.f;
    for (int sp = 0; sp < splits; ++sp) s += a.part[(static_cast<size_t>(sp) * kTileN + b) * ldp + n];
    v[k] = s;
  }
  const int p = a.pos[b];
  if (head < a.Hq + a.Hkv) {
    const uint16_t* gn = head < a.Hq ? gq : gk;
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < DL; ++k) ss = fmaf(v[k], v[k], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / static_cast<float>(D) + a.eps);
#pragma unroll
    for (int k = 0; k < DL; ++k) v[k] = v[k] * inv * bf16_to_f(gn[lane + 32 * k]);
#pragma unroll
    for (int k = 0; k < DL / 2; ++k) {
      const float ang = __fmul_rn(static_cast<float>(p), a.inv_freq[lane + 32 * k]);
      float sn, cs;
      rope_sincos(ang, &sn, &cs);
      const float x1 = v[k], x2 = v[k + DL / 2];
      v[k] = x1 * cs - x2 * sn;
      v[k + DL / 2] = x2 * cs + x1 * sn;
    }
  }
  if (head < a.Hq) {
    float* qd = a.q + (static_cast<size_t>(b) * a.Hq + head) * D;
#pragma unroll
    for (int k = 0; k < DL; ++k) qd[lane + 32 * k] = v[k];
    return;
  }
  if (*a.bad) return;  // an invalid step leaves the cache unchanged
  const int kvsel = head < a.Hq + a.Hkv ? 0 : 1;
  const int g = head - a.Hq - kvsel * a.Hkv;
  const size_t plane = ((static_cast<size_t>(l) * 2 + kvsel) * a.kv_batch + b) * a.Hkv + g;
  const size_t row = plane * a.max_ctx + p;
  if constexpr (!FP8) {
    uint16_t* dst = reinterpret_cast<uint16_t*>(a.kv) + row * D;
#pragma unroll
    for (int k = 0; k < DL; ++k) dst[lane + 32 * k] = f_to_bf16(v[k]);
  } else {
    uint8_t code[DL];
    const float sc = quantize_row_e4m3<DL>(v, code);
    uint8_t* dst = a.kv + row * D;
#pragma unroll
    for (int k = 0; k < DL; ++k) dst[lane + 32 * k] = code[k];
    if (lane == 0) a.kv_scales[row] = sc;
  }
}

// ================================================================ attention
// Split-K GQA decode attention over the step's cache: CTA = (sequence b, KV
// head g, chunk of chunk_rows rows of 0..p_b).  K and V rows of 32-row tiles
// arrive by 1-D bulk copies into a 4-stage ring; each warp keeps an fp32
// online softmax (base-2 exponent) per query head of the group; the last
// CTA of (b, g) merges the chunks and writes the bf16 o_proj operand.
struct AttnArgs2 {
  int B, Hq, Hkv, max_ctx, kv_batch, l;
  const uint8_t* kv;
  const float* kv_scales;
  const float* q;
  const int32_t* pos;
  const int* bad;
  uint16_t* out;   // act_o [2][64][Hq D]
  float* part;     // [B][Hq][chunks][D + 2]
  unsigned* cnt;   // [B][Hkv]
  int chunk_rows, chunks;
};

template <int D, bool FP8>
__global__ void __launch_bounds__(kAttThreads) attn_kernel(const AttnArgs2 a) {
  constexpr int DL = D / 32;
  constexpr int E = FP8 ? 1 : 2;                      // bytes per element
  constexpr int kHalf = kAttTileRows * D * E;          // K (or V) rows of one tile
  constexpr int kTile = 2 * kHalf;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kAttStages * kTile);
  float* merge = reinterpret_cast<float*>(full + kAttStages);  // [warps][rep][D + 2]
  __shared__ int s_last;

  if (*a.bad) return;
  const int rep = a.Hq / a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ci = blockIdx.x % a.chunks;
  const int bg = blockIdx.x / a.chunks;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int len = a.pos[b] + 1;
  const int nchunk = (len + a.chunk_rows - 1) / a.chunk_rows;
  if (ci >= nchunk) return;
  const int j0 = ci * a.chunk_rows;
  const int j1 = min(j0 + a.chunk_rows, len);
  const int ntiles = (j1 - j0 + kAttTileRows - 1) / kAttTileRows;
  const size_t kplane = ((static_cast<size_t>(a.l) * 2 + 0) * a.kv_batch + b) * a.Hkv + g;
  const size_t vplane = ((static_cast<size_t>(a.l) * 2 + 1) * a.kv_batch + b) * a.Hkv + g;
  const uint8_t* kbase = a.kv + kplane * a.max_ctx * D * E;
  const uint8_t* vbase = a.kv + vplane * a.max_ctx * D * E;
  const float* ksc = FP8 ? a.kv_scales + kplane * a.max_ctx : nullptr;
  const float* vsc = FP8 ? a.kv_scales + vplane * a.max_ctx : nullptr;

  if (tid == 0) {
    for (int s = 0; s < kAttStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t) {
    const int j = j0 + t * kAttTileRows;
    const int nr = min(kAttTileRows, j1 - j);
    const uint32_t rb = static_cast<uint32_t>(nr) * D * E;
    uint64_t* bar = &full[t % kAttStages];
    uint8_t* dst = ring + (t % kAttStages) * kTile;
    mbar_arrive_expect_tx(bar, 2 * rb);
    bulk_g2s(dst, kbase + static_cast<size_t>(j) * D * E, rb, bar, pol);
    bulk_g2s(dst + kHalf, vbase + static_cast<size_t>(j) * D * E, rb, bar, pol);
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
      qv[h][k] = h < rep ? a.q[(static_cast<size_t>(b) * a.Hq + g * rep + h) * D + lane * DL + k] *
                               qscale
                         : 0.f;
    }
  }
  for (int t = 0; t < ntiles; ++t) {
    const int j = j0 + t * kAttTileRows;
    const int nr = min(kAttTileRows, j1 - j);
    {
      Spin1 sp;
      while (!mbar_test(&full[t % kAttStages], (t / kAttStages) & 1))
        if (sp.expired()) break;
    }
    const uint8_t* tb = ring + (t % kAttStages) * kTile;
    for (int r = warp; r < nr; r += kAttWarps) {
      float kr[DL], vr[DL];
      const uint8_t* kp = tb + static_cast<size_t>(r) * D * E + lane * DL * E;
      const uint8_t* vp = kp + kHalf;
      if constexpr (!FP8) {
        if constexpr (DL == 4) {
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
      } else {
        const float ks = ksc[j + r], vs = vsc[j + r];
#pragma unroll
        for (int k = 0; k < DL; k += 2) {
          const float2 kf = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(kp + k));
          const float2 vf = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(vp + k));
          kr[k] = kf.x * ks; kr[k + 1] = kf.y * ks;
          vr[k] = vf.x * vs; vr[k + 1] = vf.y * vs;
        }
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
  // merge the warps -> this chunk's partial (m in log2 units, l, unnormalised acc)
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
    float* pp = a.part + ((static_cast<size_t>(b) * a.Hq + g * rep + h) * a.chunks + ci) * (D + 2);
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
  const int HqD = a.Hq * D;
  for (int t = tid; t < rep * D; t += kAttThreads) {
    const int h = t / D, d = t % D;
    const float* pb = a.part + (static_cast<size_t>(b) * a.Hq + g * rep + h) * a.chunks * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < nchunk; ++c) M = fmaxf(M, __ldcg(pb + c * (D + 2) + D));
    float Ls = 0.f, A = 0.f;
    for (int c = 0; c < nchunk; ++c) {
      const float e = exp2f(__ldcg(pb + c * (D + 2) + D) - M);
      Ls += __ldcg(pb + c * (D + 2) + D + 1) * e;
      A += __ldcg(pb + c * (D + 2) + d) * e;
    }
    put_act(a.out, b, (g * rep + h) * D + d, HqD, A / Ls);
  }
}

// out_ids from the argmax keys (-1 for every sequence of an invalid step).
__global__ void finish_kernel(const StepArgs2 a) {
  const int b = threadIdx.x;
  if (b >= a.B) return;
  const unsigned long long key = a.keys[b];
  a.out[b] = (*a.bad || key == 0ull) ? -1 : static_cast<int32_t>(~static_cast<uint32_t>(key));
}

size_t attn_smem(int D, int rep, bool fp8) {
  return static_cast<size_t>(kAttStages) * kAttTileRows * D * (fp8 ? 1 : 2) * 2 +
         kAttStages * sizeof(uint64_t) + static_cast<size_t>(kAttWarps) * rep * (D + 2) * sizeof(float);
}

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

// ================================================================ host plan
struct GemmPlan {
  GemmArgs args;
  CUtensorMap w[3];
  const CUtensorMap* x;  // activation map
  dim3 grid;
};

struct BtPlan {
  BtShape s;
  int sms = 0;
  const uint16_t* embed = nullptr;
  const uint16_t* final_norm = nullptr;
  std::vector<LayerPtrs> layers;
  const float* inv_freq = nullptr;
  CUtensorMap map_h{}, map_o{}, map_u{};
  std::vector<GemmPlan> qkv, o, gu, down;  // per layer
  GemmPlan lm{};
  uint8_t* ws = nullptr;
  float* x = nullptr;
  uint16_t *act_h = nullptr, *act_o = nullptr, *act_u = nullptr;
  float* q = nullptr;
  float* part = nullptr;
  float* att_part = nullptr;
  unsigned* att_cnt = nullptr;
  unsigned long long* keys = nullptr;
  int* bad = nullptr;
};

namespace {

bool encode_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunkK), box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Split count so that tiles x splits covers the SMs about once.
int pick_splits(int tiles, int k_chunks, int sms) {
  int s = (sms + tiles / 2) / tiles;
  if (s < 1) s = 1;
  if (s > k_chunks) s = k_chunks;
  return s;
}

bool make_gemm(EncodeTiledFn enc, GemmPlan& gp, int n_mat, const uint16_t* const* w,
               const int* rows, int K, const CUtensorMap* xmap, int sms, bool lm) {
  GemmArgs& g = gp.args;
  g = GemmArgs{};
  g.n_mat = n_mat;
  int tiles = 0, off = 0;
  for (int i = 0; i < 3; ++i) {
    if (i < n_mat) {
      g.rows[i] = rows[i];
      g.tiles[i] = (rows[i] + kTileM - 1) / kTileM;
      g.off[i] = off;
      off += rows[i];
      tiles += g.tiles[i];
      if (!encode_map(enc, &gp.w[i], w[i], K, rows[i], kTileM)) return false;
    } else {
      gp.w[i] = gp.w[0];
    }
  }
  g.ldp = off;
  g.k_chunks = (K + kChunkK - 1) / kChunkK;
  g.splits = lm ? 1 : pick_splits(tiles, g.k_chunks, sms);
  gp.x = xmap;
  gp.grid = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(g.splits));
  return true;
}

size_t part_floats(const GemmPlan& gp) {
  return static_cast<size_t>(gp.args.splits) * kTileN * gp.args.ldp;
}

cudaError_t launch_gemm(const GemmPlan& gp, int mode, int B, float* part,
                        unsigned long long* keys, float* logits, int* status,
                        unsigned long long timeout, cudaStream_t st) {
  GemmArgs g = gp.args;
  g.B = B;
  g.part = part;
  g.keys = keys;
  g.logits = logits;
  g.status = status;
  g.timeout_ns = timeout;
  if (mode == 0)
    gemm_kernel<0><<<gp.grid, kGemmThreads, kGemmSmem, st>>>(gp.w[0], gp.w[1], gp.w[2], *gp.x, g);
  else
    gemm_kernel<1><<<gp.grid, kGemmThreads, kGemmSmem, st>>>(gp.w[0], gp.w[1], gp.w[2], *gp.x, g);
  return cudaGetLastError();
}

}  // namespace

int bt_plan_create(const BtShape& s, const uint16_t* embed, const uint16_t* lm_head,
                   const uint16_t* final_norm, const LayerPtrs* layers_host,
                   const float* inv_freq_dev, int sms, BtPlan** out, cudaError_t* cerr) {
  *out = nullptr;
  *cerr = cudaSuccess;
  if (s.H % kChunkK || (s.Hq * s.D) % kChunkK || s.F % kChunkK) return DEC_ERR_SHAPE;
  if (s.Hq / s.Hkv > kAttMaxRep) return DEC_ERR_SHAPE;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
    *cerr = e != cudaSuccess ? e : cudaErrorNotSupported;
    return DEC_ERR_CUDA;
  }
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(fn);
  BtPlan* p = new (std::nothrow) BtPlan();
  if (!p) return DEC_ERR_ARG;
  p->s = s;
  p->sms = sms;
  p->embed = embed;
  p->final_norm = final_norm;
  p->inv_freq = inv_freq_dev;
  p->layers.assign(layers_host, layers_host + s.L);
  const int HqD = s.Hq * s.D, HkvD = s.Hkv * s.D;

  // ---- scratch
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += al256(bytes);
    return at;
  };
  const size_t x_off = take(sizeof(float) * kTileN * s.H);
  const size_t h_off = take(2ull * kBRows * s.H);
  const size_t ao_off = take(2ull * kBRows * HqD);
  const size_t au_off = take(2ull * kBRows * s.F);
  const size_t q_off = take(sizeof(float) * kTileN * HqD);
  const size_t ap_off = take(sizeof(float) * kTileN * s.Hq * kMaxAttnChunks * (s.D + 2));
  const size_t ac_off = take(sizeof(unsigned) * kTileN * s.Hkv);
  const size_t keys_off = take(sizeof(unsigned long long) * kTileN);
  const size_t bad_off = take(sizeof(int));
  // the activation maps need the buffers' addresses: allocate after sizing the partials,
  // which depend only on the shape (not on addresses), so plan the GEMMs twice
  size_t part_max = 0;
  {
    const int tiles_qkv = (HqD + kTileM - 1) / kTileM + 2 * ((HkvD + kTileM - 1) / kTileM);
    const int tiles_o = (s.H + kTileM - 1) / kTileM, tiles_gu = 2 * ((s.F + kTileM - 1) / kTileM);
    const size_t c[4] = {
        static_cast<size_t>(pick_splits(tiles_qkv, (s.H + 63) / 64, sms)) * (HqD + 2 * HkvD),
        static_cast<size_t>(pick_splits(tiles_o, (HqD + 63) / 64, sms)) * s.H,
        static_cast<size_t>(pick_splits(tiles_gu, (s.H + 63) / 64, sms)) * 2 * s.F,
        static_cast<size_t>(pick_splits(tiles_o, (s.F + 63) / 64, sms)) * s.H};
    for (size_t v : c) part_max = v > part_max ? v : part_max;
    part_max *= kTileN;
  }
  const size_t part_off = take(sizeof(float) * part_max);
  e = cudaMalloc(&p->ws, o);
  if (e == cudaSuccess) e = cudaMemset(p->ws, 0, o);
  if (e != cudaSuccess) {
    *cerr = e;
    cudaFree(p->ws);
    delete p;
    return DEC_ERR_CUDA;
  }
  p->x = reinterpret_cast<float*>(p->ws + x_off);
  p->act_h = reinterpret_cast<uint16_t*>(p->ws + h_off);
  p->act_o = reinterpret_cast<uint16_t*>(p->ws + ao_off);
  p->act_u = reinterpret_cast<uint16_t*>(p->ws + au_off);
  p->q = reinterpret_cast<float*>(p->ws + q_off);
  p->att_part = reinterpret_cast<float*>(p->ws + ap_off);
  p->att_cnt = reinterpret_cast<unsigned*>(p->ws + ac_off);
  p->keys = reinterpret_cast<unsigned long long*>(p->ws + keys_off);
  p->bad = reinterpret_cast<int*>(p->ws + bad_off);
  p->part = reinterpret_cast<float*>(p->ws + part_off);

  // ---- tensor maps and GEMM plans
  bool ok = encode_map(enc, &p->map_h, p->act_h, s.H, kBRows, kBRows) &&
            encode_map(enc, &p->map_o, p->act_o, HqD, kBRows, kBRows) &&
            encode_map(enc, &p->map_u, p->act_u, s.F, kBRows, kBRows);
  p->qkv.resize(s.L);
  p->o.resize(s.L);
  p->gu.resize(s.L);
  p->down.resize(s.L);
  for (int l = 0; ok && l < s.L; ++l) {
    const LayerPtrs& lp = p->layers[l];
    const uint16_t* wqkv[3] = {lp.w[DEC_LW_Q], lp.w[DEC_LW_K], lp.w[DEC_LW_V]};
    const int rqkv[3] = {HqD, HkvD, HkvD};
    const uint16_t* wo[1] = {lp.w[DEC_LW_O]};
    const int ro[1] = {s.H};
    const uint16_t* wgu[2] = {lp.w[DEC_LW_GATE], lp.w[DEC_LW_UP]};
    const int rgu[2] = {s.F, s.F};
    const uint16_t* wd[1] = {lp.w[DEC_LW_DOWN]};
    ok = make_gemm(enc, p->qkv[l], 3, wqkv, rqkv, s.H, &p->map_h, sms, false) &&
         make_gemm(enc, p->o[l], 1, wo, ro, HqD, &p->map_o, sms, false) &&
         make_gemm(enc, p->gu[l], 2, wgu, rgu, s.H, &p->map_h, sms, false) &&
         make_gemm(enc, p->down[l], 1, wd, ro, s.F, &p->map_u, sms, false);
    ok = ok && part_floats(p->qkv[l]) <= part_max && part_floats(p->o[l]) <= part_max &&
         part_floats(p->gu[l]) <= part_max && part_floats(p->down[l]) <= part_max;
  }
  if (ok) {
    const uint16_t* wl[1] = {lm_head};
    const int rl[1] = {s.V};
    ok = make_gemm(enc, p->lm, 1, wl, rl, s.H, &p->map_h, sms, true);
  }
  if (ok) {
    e = cudaFuncSetAttribute(gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kGemmSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kGemmSmem));
  }
  if (!ok || e != cudaSuccess) {
    *cerr = e;
    cudaFree(p->ws);
    delete p;
    return ok ? DEC_ERR_CUDA : DEC_ERR_SHAPE;
  }
  *out = p;
  return DEC_OK;
}

void bt_plan_destroy(BtPlan* p) {
  if (!p) return;
  cudaFree(p->ws);
  delete p;
}

namespace {

template <int D, bool FP8>
cudaError_t launch_attn(const AttnArgs2& a, int rep, cudaStream_t st) {
  const size_t smem = attn_smem(D, rep, FP8);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  attn_kernel<D, FP8><<<static_cast<unsigned>(a.B) * a.Hkv * a.chunks, kAttThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, bool FP8>
cudaError_t launch_qkv_post(const StepArgs2& a, int splits, int l, const LayerPtrs& lp,
                            cudaStream_t st) {
  const dim3 grid((a.Hq + 2 * a.Hkv + 3) / 4, a.B);
  qkv_post_kernel<D, FP8><<<grid, 128, 0, st>>>(a, splits, l, lp.w[DEC_LW_Q_NORM],
                                                lp.w[DEC_LW_K_NORM]);
  return cudaGetLastError();
}

}  // namespace

cudaError_t bt_step(BtPlan* p, const BtIO& io, cudaStream_t st) {
  const BtShape& s = p->s;
  StepArgs2 a{};
  a.B = io.B;
  a.L = s.L;
  a.H = s.H;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.D = s.D;
  a.F = s.F;
  a.V = s.V;
  a.eps = s.eps;
  a.tok = io.tok;
  a.pos = io.pos;
  a.out = io.out;
  a.embed = p->embed;
  a.x = p->x;
  a.act_h = p->act_h;
  a.act_o = p->act_o;
  a.act_u = p->act_u;
  a.q = p->q;
  a.part = p->part;
  a.keys = p->keys;
  a.bad = p->bad;
  a.status = io.status;
  a.inv_freq = p->inv_freq;
  a.hidden = io.hidden;
  a.kv = io.kv;
  a.kv_scales = io.kv_scales;
  a.kv_batch = io.kv_batch;
  a.max_ctx = io.max_ctx;

  // attention chunking: about 4 CTAs per SM over the cache capacity, at most
  // kMaxAttnChunks chunks per (sequence, KV head)
  int cr = attention_chunk_rows(io.B, s.Hkv, io.max_ctx, p->sms);
  const int min_cr = ((io.max_ctx + kMaxAttnChunks - 1) / kMaxAttnChunks + kAttTileRows - 1) /
                     kAttTileRows * kAttTileRows;
  if (cr < min_cr) cr = min_cr;
  AttnArgs2 at{};
  at.B = io.B;
  at.Hq = s.Hq;
  at.Hkv = s.Hkv;
  at.max_ctx = io.max_ctx;
  at.kv_batch = io.kv_batch;
  at.kv = io.kv;
  at.kv_scales = io.kv_scales;
  at.q = p->q;
  at.pos = io.pos;
  at.bad = p->bad;
  at.out = p->act_o;
  at.part = p->att_part;
  at.cnt = p->att_cnt;
  at.chunk_rows = cr;
  at.chunks = (io.max_ctx + cr - 1) / cr;
  const int rep = s.Hq / s.Hkv;
  const unsigned long long to = io.timeout_ns;

  cudaError_t e;
  embed_kernel<<<io.B, kRowThreads, 0, st>>>(a, p->layers[0].w[DEC_LW_IN_NORM]);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int l = 0; l < s.L; ++l) {
    const LayerPtrs& lp = p->layers[l];
    if ((e = launch_gemm(p->qkv[l], 0, io.B, p->part, nullptr, nullptr, io.status, to, st)))
      return e;
    const int sq = p->qkv[l].args.splits;
    if (s.D == 128)
      e = io.kv_fp8 ? launch_qkv_post<128, true>(a, sq, l, lp, st)
                    : launch_qkv_post<128, false>(a, sq, l, lp, st);
    else
      e = io.kv_fp8 ? launch_qkv_post<64, true>(a, sq, l, lp, st)
                    : launch_qkv_post<64, false>(a, sq, l, lp, st);
    if (e) return e;
    at.l = l;
    if (s.D == 128)
      e = io.kv_fp8 ? launch_attn<128, true>(at, rep, st) : launch_attn<128, false>(at, rep, st);
    else
      e = io.kv_fp8 ? launch_attn<64, true>(at, rep, st) : launch_attn<64, false>(at, rep, st);
    if (e) return e;
    if ((e = launch_gemm(p->o[l], 0, io.B, p->part, nullptr, nullptr, io.status, to, st))) return e;
    resid_norm_kernel<<<io.B, kRowThreads, 0, st>>>(a, p->o[l].args.splits,
                                                    lp.w[DEC_LW_POST_NORM], nullptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_gemm(p->gu[l], 0, io.B, p->part, nullptr, nullptr, io.status, to, st)))
      return e;
    swiglu_kernel<<<dim3((s.F + kRowThreads - 1) / kRowThreads, io.B), kRowThreads, 0, st>>>(
        a, p->gu[l].args.splits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_gemm(p->down[l], 0, io.B, p->part, nullptr, nullptr, io.status, to, st)))
      return e;
    const uint16_t* next_gain = l + 1 < s.L ? p->layers[l + 1].w[DEC_LW_IN_NORM] : p->final_norm;
    float* hs = io.hidden ? io.hidden + static_cast<size_t>(l + 1) * io.B * s.H : nullptr;
    resid_norm_kernel<<<io.B, kRowThreads, 0, st>>>(a, p->down[l].args.splits, next_gain, hs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = launch_gemm(p->lm, 1, io.B, nullptr, p->keys, io.logits, io.status, to, st))) return e;
  finish_kernel<<<1, kTileN, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dec
