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
// one 128-row weight tile x 64 sequences per CTA.
//
// Launches per layer: QKV GEMM, attention, o_proj GEMM, gate/up GEMM, down
// GEMM.  A GEMM is split along K over the CTAs of a thread-block cluster;
// the cluster sums the split accumulators through distributed shared memory
// (in a fixed order: deterministic) and the same launch finishes the phase:
//   QKV      q/k RMSNorm, rotation, query store, K/V append (bf16 or E4M3)
//   o_proj   residual add; the next RMSNorm's operand and sums of squares
//   gate/up  silu(gate) * up (a tile holds 64 gate rows and the same 64 up rows)
//   down     residual add; the next RMSNorm's operand and sums of squares
// RMSNorm is applied as a per-sequence scale: the producer of x stores g * x
// and per-tile sums of x^2, and the consumer GEMM multiplies its accumulator
// column b by rsqrt(mean x_b^2 + eps) (a column scale commutes with W).
// Every launch is a programmatic dependent launch: a GEMM's weight tiles
// (which no earlier kernel writes) stream in while its predecessor finishes.
//
// The Baseten Qwen3-ASR article ("KV cache quantization") notes that at high
// concurrency the attention over the cache takes the largest share of decode
// time: it is a split-K kernel over (sequence, KV head, chunk) streaming K/V
// rows (bf16, or E4M3 codes + fp32 row scales) through shared memory.
//
// Numerics: weights and the KV cache as stored; the residual stream, norms,
// softmax and accumulators fp32.  A tensor-core activation operand is held
// as two bf16 planes, hi = bf16(y) and lo = bf16(y - hi), and every K step
// issues one MMA per plane: W y = W hi + W lo to about 2^-17 of y, so the
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
constexpr int kBRows = 2 * kTileN;                // activation rows: hi plane, then lo plane
constexpr int kBBytes = kBRows * kChunkK * 2;     // 16 KB
constexpr int kLoOffset = kTileN * kChunkK * 2;   // lo plane inside a B tile (8 KB)
constexpr int kHalfA = kABytes / 2;               // gate/up tiles: up rows start here
constexpr int kStageBytes = kABytes + kBBytes;    // 32 KB
constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 256;                 // 8 warps: 2 per TMEM sub-partition
constexpr int kHalfN = kTileN / 2;                // accumulator columns read per warp
constexpr uint32_t kTmemCols = 64;                // fp32 accumulator columns (= kTileN)
constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, kTileN);
constexpr int kTStride = kTileM + 4;              // accumulator tile in smem: T[b][row]
constexpr int kWOffset = 40 * 1024;               // reduced rows of this CTA's sequences
constexpr size_t kGemmSmem = 1024 + kGemmStages * kStageBytes + 256;
// int8 weights: the codes of a weight tile land (TMA, no swizzle: row r at
// byte 64 r) in the upper half of the stage's bf16 weight tile; the CTA's
// epilogue warps, idle during the main loop, read them all into registers,
// then widen them into the whole bf16 tile.  The shared memory stays that of
// the bf16 GEMM, so two GEMM CTAs still fit an SM and a GEMM's prologue
// overlaps its predecessor (programmatic dependent launch).
constexpr int kA8Bytes = kTileM * kChunkK;        // 8 KB
constexpr int kA8Offset = kABytes - kA8Bytes;     // codes inside the weight tile
constexpr int kConvThreads = 128;                 // warps 4..7
constexpr int kConvBarrier = 1;                   // their named barrier
constexpr int kMaxSplits = 16;                    // cluster size (16: non-portable, allowed per kernel)
constexpr int kMaxAttnChunks = 32;
constexpr int kAttMinSplitRows = 1024;            // shortest chunk of a multi-wave split
constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttStages = 3;
constexpr int kAttTileRows = 32;                // passes of kAttWarps x 4 rows (lane octets)
constexpr int kAttMaxRep = 4;  // query heads per KV head (attention template)
constexpr int kRowThreads = 256;
[[maybe_unused]] constexpr int kProfCtas = 2048;                   // GEMM CTAs with timestamps (profiling builds)

enum GemmMode { kQKV = 0, kResid = 1, kSwiGLU = 2, kLm = 3 };

static_assert(kTileN == 64 && kTmemCols == 64, "epilogue reads 4 x 16 accumulator columns");
static_assert(kAttTileRows % (kAttWarps * 4) == 0, "a tile is whole passes of one row per octet");
static_assert(kTileN * kTStride * 4 <= kWOffset, "accumulator tile below the reduced rows");
static_assert((kTileN + kMaxSplits) * kTileM * 4 <= kWOffset, "split receive rows below them");
static_assert(kWOffset + kTileN * kTileM * 4 <= kGemmStages * kStageBytes, "both fit the ring");

// Bounded mbarrier wait: the copies and MMAs always complete; the bound only
// guards the GPU.  Returns false (and raises the timeout status) if it ran
// out; with `give_up` it also returns false as soon as another wait of the
// step has timed out, so that a stuck step ends quickly.
__device__ bool bt_wait(uint64_t* bar, uint32_t parity, unsigned long long limit, int* status,
                        bool give_up = true) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_wait(bar, parity, kWaitHintNs)) return true;
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

// y as the two bf16 planes of a tensor-core activation buffer [2][64][K]
__device__ __forceinline__ void put_act(uint16_t* buf, int b, int n, int K, float y) {
  const uint16_t hi = f_to_bf16(y);
  buf[static_cast<size_t>(b) * K + n] = hi;
  buf[static_cast<size_t>(kTileN + b) * K + n] = f_to_bf16(y - bf16_to_f(hi));
}

// sum over the threads of the CTA (every thread must call it)
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read from a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

// rsqrt(mean x_b^2 + eps) from the per-tile sums of squares [n_ssp][64]
__device__ __forceinline__ float rms_scale(const float* ssp, int n_ssp, int b, int H, float eps) {
  float ss = 0.f;
  for (int t = 0; t < n_ssp; ++t) ss += ssp[t * kTileN + b];
  return rsqrtf(ss / static_cast<float>(H) + eps);
}

// ===================================================================== GEMM
// out[b][n] = sum_k W[n][k] * Y[b][k] for the 64 sequence columns (Y is the
// activation buffer: rows 0..63 the hi plane, 64..127 the lo plane; columns
// of sequences >= B are computed and ignored), followed by the mode's
// epilogue.  Grid (tiles, splits); cluster (1, splits): the CTAs of a tile.
struct GemmArgs {
  int n_mat;     // kQKV: 3 (q, k, v); others 1
  int rows[3];   // output rows of each matrix (kSwiGLU: F; the tile pairs gate/up)
  int tiles[3];  // tiles of each matrix
  int k_chunks;  // ceil(K / 64)
  int splits;
  int B, H, D, Hq, Hkv, F;
  float eps;
  int n_ssp;             // tiles of the residual-producing GEMMs (ceil(H / 128))
  const float* ssp_in;   // [n_ssp][64] sums of squares of the residual (kQKV, kSwiGLU, kLm)
  float* ssp_out;        // kResid: [n_ssp][64]
  float* x;              // kResid: residual [64][H]
  float* hidden;         // kResid: [B][H] slot or null
  const uint16_t* gain;  // kResid: the next RMSNorm's gain; kQKV: q-norm gain
  const uint16_t* gain2; // kQKV: k-norm gain
  uint16_t* act;         // kResid: act_h; kSwiGLU: act_u
  float* q;              // kQKV: [64][Hq][D]
  uint8_t* kv;
  float* kv_scales;
  int kv_batch, max_ctx, layer, kv_fp8;
  int one_seq;           // -1: row b is cache sequence b; >= 0: every row is that sequence
  const int32_t* pos;
  const int* retired;    // [B] or null: rows whose cache row is not written
  const int* bad;
  const float* inv_freq;
  unsigned long long* keys;  // kLm: [64]
  float* logits;             // kLm: [B][V] or null
  int* status;
  unsigned long long timeout_ns;
  unsigned long long* prof;  // profiling builds: [4 modes][kProfCtas][16] timestamps, else null
  const float* wsc[3];       // int8 weights: fp32 row scales of each matrix (kSwiGLU: gate, up)
};

// Phase timestamps of one GEMM CTA (profiling builds only).
#ifdef DEC_PROFILE
#define BT_STAMP(k)                                                                      \
  do {                                                                                   \
    if (g.prof && blockIdx.y * gridDim.x + blockIdx.x < kProfCtas)                       \
      g.prof[((MODE * kProfCtas) + blockIdx.y * gridDim.x + blockIdx.x) * 16 + (k)] =    \
          globaltimer();                                                                 \
  } while (0)
#else
#define BT_STAMP(k) \
  do {              \
  } while (0)
#endif

template <int MODE, int W8>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap w0,
                                                            const __grid_constant__ CUtensorMap w1,
                                                            const __grid_constant__ CUtensorMap w2,
                                                            const __grid_constant__ CUtensorMap xm,
                                                            const GemmArgs g) {
  extern __shared__ uint8_t dsm[];
  __shared__ float s_red[kGemmThreads / 32][kTileN];  // per-warp partial sums, per slot
  __shared__ float s_inv[kTileN];      // rsqrt(mean x^2 + eps) per sequence
  __shared__ int s_pos[kTileN];
  const uint32_t raw = smem_u32(dsm);
  uint8_t* sm = dsm + (((raw + 1023u) & ~1023u) - raw);  // swizzle atoms need 1024-B alignment
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kGemmStages * kStageBytes);
  uint64_t* empty = full + kGemmStages;
  uint64_t* done = empty + kGemmStages;
  uint64_t* afull = done + 1;         // W8: the int8 codes of stage s landed
  uint64_t* conv = afull + kGemmStages;  // W8: stage s's bf16 weight tile written
  uint32_t* tslot = reinterpret_cast<uint32_t*>(conv + kGemmStages);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) BT_STAMP(0);
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
      if constexpr (W8) {
        mbar_init(&afull[s], 1);
        mbar_init(&conv[s], kConvThreads / 32);
      }
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    pdl_trigger();
    BT_STAMP(1);
  }
  const uint32_t tmem = *tslot;
  // per-row constants of the epilogue (weights: no earlier kernel writes them)
  float row_gain = 1.f, row_invf = 0.f, row_scale = 1.f;
  {
    const int r = tile * kTileM + (warp & 3) * 32 + lane;
    if constexpr (W8) {
      // the int8 row scale of accumulator row (warp & 3) * 32 + lane
      const int m = (warp & 3) * 32 + lane;
      if constexpr (MODE == kSwiGLU) {
        const int fr = tile * (kTileM / 2) + (m & (kTileM / 2 - 1));
        row_scale = fr < mrows ? (m < kTileM / 2 ? g.wsc[0] : g.wsc[1])[fr] : 0.f;
      } else {
        const float* sc = mat == 0 ? g.wsc[0] : (mat == 1 ? g.wsc[1] : g.wsc[2]);
        row_scale = r < mrows ? sc[r] : 0.f;
      }
    }
    if constexpr (MODE == kQKV) {
      const int d = r % g.D;
      if (mat < 2) row_gain = bf16_to_f((mat == 0 ? g.gain : g.gain2)[d]);
      row_invf = g.inv_freq[d < g.D / 2 ? d : d - g.D / 2];
    } else if constexpr (MODE == kResid) {
      if (r < mrows) row_gain = bf16_to_f(g.gain[r]);
    }
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer.  Weight tiles (streamed once: evict first) do not
      // depend on earlier kernels: the first stages load before pdl_wait().
      tma_prefetch_map(wm);
      tma_prefetch_map(&xm);
      const uint64_t pw = policy_evict_first();
      const uint64_t px = policy_evict_last();
      // bf16 weights: the tile into the stage, counted by full[s]; int8: the
      // codes into the staging area, counted by afull[s]
      auto load_a = [&](int i, int s) {
        const int x = (c0 + i) * kChunkK;
        uint32_t st, bar;
        if constexpr (W8) {
          st = smem_u32(sm + s * kStageBytes + kA8Offset);
          bar = smem_u32(&afull[s]);
          mbar_arrive_expect_tx(&afull[s], kA8Bytes);
        } else {
          st = smem_u32(sm + s * kStageBytes);
          bar = smem_u32(&full[s]);
        }
        constexpr uint32_t half = W8 ? kA8Bytes / 2 : kHalfA;
        if constexpr (MODE == kSwiGLU) {
          tma_load_2d(st, &w0, x, tile * (kTileM / 2), bar, pw);
          tma_load_2d(st + half, &w1, x, tile * (kTileM / 2), bar, pw);
        } else {
          tma_load_2d(st, wm, x, tile * kTileM, bar, pw);
        }
      };
      constexpr uint32_t kFullBytes = W8 ? kBBytes : kStageBytes;
      auto load_b = [&](int i, int s) {
        const uint32_t st = smem_u32(sm + s * kStageBytes);
        tma_load_2d(st + kABytes, &xm, (c0 + i) * kChunkK, 0, smem_u32(&full[s]), px);
      };
      const int pre = nch < kGemmStages ? nch : kGemmStages;
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], kFullBytes);
        load_a(i, i);
      }
      BT_STAMP(2);
      pdl_wait();
      BT_STAMP(3);
      for (int i = 0; i < pre; ++i) load_b(i, i);
      int issued = pre;
      for (int i = pre; i < nch; ++i) {
        const int s = i % kGemmStages;
        if (!bt_wait(&empty[s], ((i / kGemmStages) - 1) & 1, g.timeout_ns, g.status)) break;
        mbar_arrive_expect_tx(&full[s], kFullBytes);
        load_a(i, s);
        load_b(i, s);
        ++issued;
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int s = 0; s < kGemmStages && s < issued; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % kGemmStages);
        bt_wait(&full[s], (last / kGemmStages) & 1, g.timeout_ns, g.status, false);
        if constexpr (W8) bt_wait(&afull[s], (last / kGemmStages) & 1, g.timeout_ns, g.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer: per stage 4 K-steps x (hi, lo) of 128 x 64 x 16
      for (int i = 0; i < nch; ++i) {
        const int s = i % kGemmStages;
        if (!bt_wait(&full[s], (i / kGemmStages) & 1, g.timeout_ns, g.status)) break;
        if constexpr (W8)
          if (!bt_wait(&conv[s], (i / kGemmStages) & 1, g.timeout_ns, g.status)) break;
        if (i == 0) BT_STAMP(4);
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
      BT_STAMP(5);
      tc_commit(smem_u32(done));
    }
    __syncwarp();
  } else if (W8 && warp >= 4) {
    // ---- 8-bit weights: widen each stage's codes into the bf16 operand tile
    // (128-byte swizzle: row r at byte 128 r of its 8-row atom, 16-byte chunk
    // j at chunk position j ^ (r mod 8)).  An int8 code is sign-extended by a
    // byte permute and converted to fp32 (|c| <= 127: exact in bf16); E4M3
    // codes go through the hardware e4m3x2 -> f16x2 conversion; both are
    // packed to bf16 two at a time.
    const int ct = tid - 128;
    constexpr int kItems = kA8Bytes / 8 / kConvThreads;  // 8 codes each
    for (int i = 0; i < nch; ++i) {
      const int s = i % kGemmStages;
      // every converter waits; the barrier below makes the outcome uniform
      const bool ok = bt_wait(&afull[s], (i / kGemmStages) & 1, g.timeout_ns, g.status);
      uint8_t* dst = sm + s * kStageBytes;
      const uint8_t* src = dst + kA8Offset;
      uint2 c8s[kItems];
#pragma unroll
      for (int t = 0; t < kItems; ++t)
        c8s[t] = ok ? *reinterpret_cast<const uint2*>(src + (t * kConvThreads + ct) * 8)
                    : make_uint2(0u, 0u);
      // every code is read before the tile is rewritten; a wait that gave up
      // anywhere stops all converters together
      if (named_sync_or(kConvBarrier, kConvThreads, !ok)) break;
#pragma unroll
      for (int t = 0; t < kItems; ++t) {
        const int it = t * kConvThreads + ct;  // 8 codes: row it / 8, chunk it % 8
        const int r = it >> 3, j = it & 7;
        const uint2 c8 = c8s[t];
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x = h == 0 ? c8.x : c8.y;
          float f[4];
          if constexpr (W8 == 2) {
            // E4M3: every finite value is exact in bf16
            const float2 a = e4m3x2_to_f2(static_cast<uint16_t>(x & 0xFFFFu));
            const float2 b = e4m3x2_to_f2(static_cast<uint16_t>(x >> 16));
            f[0] = a.x;
            f[1] = a.y;
            f[2] = b.x;
            f[3] = b.y;
          } else {
            // selector 0x8880 + 0x1111 e: byte e, then its sign bit replicated
#pragma unroll
            for (int e = 0; e < 4; ++e)
              f[e] = static_cast<float>(static_cast<int>(prmt_b32(x, 0x8880u + 0x1111u * e)));
          }
          w[2 * h] = f2_to_bf16x2(f[0], f[1]);
          w[2 * h + 1] = f2_to_bf16x2(f[2], f[3]);
        }
        *reinterpret_cast<uint4*>(dst + (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&conv[s]);
    }
  }
  if (tid >= 64 && tid < 64 + kTileN) {
    // idle during the main loop: the epilogue's per-sequence inputs
    pdl_wait();
    const int b = tid - 64;
    if constexpr (MODE != kResid) s_inv[b] = b < g.B ? rms_scale(g.ssp_in, g.n_ssp, b, g.H, g.eps) : 0.f;
    if constexpr (MODE == kQKV) s_pos[b] = b < g.B ? g.pos[b] : 0;
  }

  // ---- accumulator: TMEM lane = tile row, column = sequence.  Warp w reads
  // the rows of its sub-partition (w % 4) and the 32 columns of half w / 4.
  bt_wait(done, 0, g.timeout_ns, g.status);
  if (tid == 0) BT_STAMP(6);
  tc_fence_after();
  const int quad = warp & 3, hg = warp >> 2;
  float v[kHalfN];  // v[c]: sequence hg * 32 + c
  const uint32_t tl =
      tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(hg * kHalfN);
  tc_ld16(tl, v);
  tc_ld16(tl + 16, v + 16);
  tc_wait_ld();
  if constexpr (W8) {
#pragma unroll
    for (int c = 0; c < kHalfN; ++c) v[c] *= row_scale;
  }
  const int m = quad * 32 + lane;
  if (tid == 0) BT_STAMP(7);
  pdl_wait();  // everything below reads or writes what earlier kernels use
  if (tid == 0) BT_STAMP(8);

  if constexpr (MODE == kLm) {
    // logits = rsqrt(mean x^2 + eps) * (W (g x)); argmax per sequence
    __syncthreads();  // s_inv
#pragma unroll
    for (int c = 0; c < kHalfN; ++c) v[c] *= s_inv[hg * kHalfN + c];
    const int V = g.rows[0];
    const int row = tile * kTileM + m;
    if (g.logits && row < V) {
#pragma unroll
      for (int c = 0; c < kHalfN; ++c)
        if (hg * kHalfN + c < g.B) g.logits[static_cast<size_t>(hg * kHalfN + c) * V + row] = v[c];
    }
    float* T = reinterpret_cast<float*>(sm);  // the (idle) ring: T[b][row]
#pragma unroll
    for (int c = 0; c < kHalfN; ++c) T[(hg * kHalfN + c) * kTStride + m] = v[c];
    __syncthreads();
    // thread (b = tid / 4, q = tid % 4) scans rows 32q .. 32q+31 of sequence b
    const int b = tid >> 2, q = tid & 3;
    float best = -INFINITY;
    int bi = 0x7fffffff;
    if (b < g.B) {
      const float4* t4 = reinterpret_cast<const float4*>(T + b * kTStride + q * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 x = t4[j];
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int id = tile * kTileM + q * 32 + 4 * j + e;
          if (id < V && xs[e] > best) {  // ascending ids: strict > keeps the lowest on ties
            best = xs[e];
            bi = id;
          }
        }
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    if (q == 0 && b < g.B && bi != 0x7fffffff)
      atomicMax(&g.keys[b], (static_cast<unsigned long long>(order_key(best)) << 32) |
                                static_cast<uint32_t>(~bi));
  } else {
    // ---- split-K reduction across the cluster, then the phase's epilogue.
    // CTA `rank` of the cluster finishes sequences b = rank, rank + S, ...
    // (slot bi = b / S).  Every CTA pushes its partial rows into the owner's
    // receive rows R[split][bi][row] with remote stores; after one cluster
    // barrier each owner sums them locally.  Thread (row m, half hg) then
    // finishes the slots bi = hg, hg + 2, ...
    const int S = g.splits;
    const int rank = static_cast<int>(cluster_rank());
    const int nbmax = (kTileN + S - 1) / S;
    const int nb = g.B > rank ? (g.B - rank + S - 1) / S : 0;
    float* R = reinterpret_cast<float*>(sm);                         // [S][nbmax][128]
    float* W = reinterpret_cast<float*>(sm + kWOffset);              // [nb][128]
    // R overlays the operand ring: wait until every CTA of the cluster is
    // past its MMAs before writing into another CTA's ring
    cluster_arrive();
    const bool bad = MODE == kQKV ? (*g.bad != 0) : false;
    cluster_wait();  // also orders s_inv / s_pos (written before the MMAs finished)
    const uint32_t r_addr = smem_u32(R) + 4u * static_cast<uint32_t>(rank * nbmax * kTileM + m);
    {
      int dst = (hg * kHalfN) % S, slot = (hg * kHalfN) / S;  // owner and slot of sequence b
#pragma unroll
      for (int c = 0; c < kHalfN; ++c) {
        if (hg * kHalfN + c < g.B)
          st_dsmem(map_rank(r_addr + 4u * static_cast<uint32_t>(slot * kTileM),
                            static_cast<uint32_t>(dst)),
                   v[c]);
        if (++dst == S) {
          dst = 0;
          ++slot;
        }
      }
    }
    cluster_sync();  // every split's rows have arrived
    if (tid == 0) BT_STAMP(9);
#pragma unroll 2
    for (int bi = hg; bi < nb; bi += 2) {
      float acc = 0.f;
      for (int sp = 0; sp < S; ++sp) acc += R[(sp * nbmax + bi) * kTileM + m];  // fixed order
      W[bi * kTileM + m] = acc;
    }
    if (tid == 0) BT_STAMP(10);
    const int row = tile * kTileM + m;  // row within the (first) matrix of this tile
    if constexpr (MODE == kQKV) {
      const int D = g.D, half = D / 2;
      const int head = row / D, d = row - head * D;
      const int wh = hg * 4 + (m / D) * (D / 32);  // first warp of this thread's head
#pragma unroll 4
      for (int bi = hg; bi < nb; bi += 2) W[bi * kTileM + m] *= s_inv[rank + S * bi];
      if (mat < 2) {
        // RMSNorm over the head (D / 32 warps of this half) and gain
#pragma unroll 4
        for (int bi = hg; bi < nb; bi += 2) {
          const float x = W[bi * kTileM + m];
          const float ss = warp_sum(x * x);
          if (lane == 0) s_red[warp][bi] = ss;
        }
        __syncthreads();
        const float gn = row_gain;
#pragma unroll 4
        for (int bi = hg; bi < nb; bi += 2) {
          float hs = 0.f;
          for (int w = 0; w < D / 32; ++w) hs += s_red[wh + w][bi];
          W[bi * kTileM + m] *= rsqrtf(hs / static_cast<float>(D) + g.eps) * gn;
        }
        __syncthreads();
      }
      // the rotated (q, k) or plain (v) value of slot bi
      const float invf = row_invf;
      auto value = [&](int bi) {
        const float x = W[bi * kTileM + m];
        if (mat == 2) return x;
        const float partner = W[bi * kTileM + (m ^ half)];
        const float ang = __fmul_rn(static_cast<float>(s_pos[rank + S * bi]), invf);
        float sn, cs;
        rope_sincos(ang, &sn, &cs);
        return d < half ? x * cs - partner * sn : x * cs + partner * sn;
      };
      if (mat == 0) {
#pragma unroll 4
        for (int bi = hg; bi < nb; bi += 2) {
          const int b = rank + S * bi;
          g.q[(static_cast<size_t>(b) * g.Hq + head) * D + d] = value(bi);
        }
      } else if (!bad) {  // an invalid step leaves the cache unchanged
        const int kvsel = mat - 1;
        auto crow_of = [&](int b) {
          const int cs = g.one_seq >= 0 ? g.one_seq : b;  // cache sequence of row b
          const size_t plane =
              ((static_cast<size_t>(g.layer) * 2 + kvsel) * g.kv_batch + cs) * g.Hkv + head;
          return plane * g.max_ctx + s_pos[b];
        };
        auto live = [&](int b) { return g.retired == nullptr || g.retired[b] == 0; };
        if (!g.kv_fp8) {
#pragma unroll 4
          for (int bi = hg; bi < nb; bi += 2) {
            const int b = rank + S * bi;
            if (live(b))
              reinterpret_cast<uint16_t*>(g.kv)[crow_of(b) * D + d] = f_to_bf16(value(bi));
          }
        } else {
          // E4M3 with one fp32 scale per row: scale = max(amax, 2^-126) / 448
#pragma unroll 4
          for (int bi = hg; bi < nb; bi += 2) {
            const float am = warp_max(fabsf(value(bi)));
            if (lane == 0) s_red[warp][bi] = am;
          }
          __syncthreads();
#pragma unroll 4
          for (int bi = hg; bi < nb; bi += 2) {
            const int b = rank + S * bi;
            float hm = 0.f;
            for (int w = 0; w < D / 32; ++w) hm = fmaxf(hm, s_red[wh + w][bi]);
            hm = fmaxf(hm, 1.17549435e-38f);
            const float sc = __fdiv_rn(hm, 448.0f);
            const size_t cr = crow_of(b);
            if (live(b)) {
              g.kv[cr * D + d] =
                  static_cast<uint8_t>(f2_to_e4m3x2(__fdiv_rn(value(bi), sc), 0.f) & 0xFF);
              if (d == 0) g.kv_scales[cr] = sc;
            }
          }
        }
      }
    } else if constexpr (MODE == kResid) {
      const bool ok = row < mrows;
      const float gn = row_gain;
      for (int bi0 = hg; bi0 < nb; bi0 += 16) {
        // the residual loads of the batch before any store (the stores may alias)
        float xv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          xv[j] = (ok && bi0 + 2 * j < nb)
                      ? g.x[static_cast<size_t>(rank + S * (bi0 + 2 * j)) * g.H + row] +
                            W[(bi0 + 2 * j) * kTileM + m]
                      : 0.f;
        float sq[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          sq[j] = xv[j] * xv[j];
          if (ok && bi0 + 2 * j < nb) {
            const int b = rank + S * (bi0 + 2 * j);
            g.x[static_cast<size_t>(b) * g.H + row] = xv[j];
            if (g.hidden) g.hidden[static_cast<size_t>(b) * g.H + row] = xv[j];
            put_act(g.act, b, row, g.H, xv[j] * gn);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int j = 0; j < 8; ++j) sq[j] += __shfl_xor_sync(0xffffffffu, sq[j], o);
        if (lane == 0) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (bi0 + 2 * j < nb) s_red[warp][bi0 + 2 * j] = sq[j];
        }
      }
      __syncthreads();
      if (tid < nb) {
        const int w0 = (tid & 1) * 4;  // the half that finished slot tid
        g.ssp_out[tile * kTileN + rank + S * tid] =
            s_red[w0][tid] + s_red[w0 + 1][tid] + s_red[w0 + 2][tid] + s_red[w0 + 3][tid];
      }
    } else {  // kSwiGLU: rows 0..63 gate, 64..127 up, of columns tile*64 ..
#pragma unroll 4
      for (int bi = hg; bi < nb; bi += 2) W[bi * kTileM + m] *= s_inv[rank + S * bi];
      __syncthreads();
      const int n = tile * (kTileM / 2) + m;
      if (m < kTileM / 2 && n < g.F) {
#pragma unroll 4
        for (int bi = hg; bi < nb; bi += 2) {
          const float gt = W[bi * kTileM + m], up = W[bi * kTileM + m + kTileM / 2];
          put_act(g.act, rank + S * bi, n, g.F, gt / (1.0f + __expf(-gt)) * up);
        }
      }
    }
    if (tid == 0) BT_STAMP(11);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0) BT_STAMP(13);
}

// ================================================================ small kernels
struct StepArgs2 {
  int B, H, V, n_ssp, max_ctx;
  const int32_t* tok;
  const int32_t* pos;
  int32_t* out;
  const uint16_t* embed;
  const uint16_t* g_in;   // layer 0 input RMSNorm gain
  float* x;               // residual stream [64][H] fp32
  uint16_t* act_h;        // [2][64][H]
  float* ssp;             // [n_ssp][64]
  unsigned long long* keys;
  int* bad;
  int* status;
  float* hidden;          // [B][H] slot 0 or null
};

// Validation of every sequence's token and position (all CTAs reach the same
// answer), the embedding row, the first RMSNorm's operand g * x and sum of
// squares.  Grid: B.
__global__ void __launch_bounds__(kRowThreads) embed_kernel(const StepArgs2 a) {
  __shared__ float red[kRowThreads / 32];
  __shared__ int s_bad;
  const int b = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) {
    pdl_trigger();
    s_bad = 0;
  }
  pdl_wait();
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
    put_act(a.act_h, b, n, a.H, xv * bf16_to_f(a.g_in[n]));
    ss = fmaf(xv, xv, ss);
  }
  ss = block_sum(ss, red);
  if (tid < a.n_ssp) a.ssp[tid * kTileN + b] = tid == 0 ? ss : 0.f;
}

// out_ids from the argmax keys (-1 for every sequence of an invalid step).
__global__ void finish_kernel(const StepArgs2 a) {
  pdl_wait();
  const int b = threadIdx.x;
  if (b >= a.B) return;
  const unsigned long long key = a.keys[b];
  a.out[b] = (*a.bad || key == 0ull) ? -1 : static_cast<int32_t>(~static_cast<uint32_t>(key));
}

// ================================================================ attention
// Split-K GQA decode attention over the step's cache: CTA = (sequence b, KV
// head g, chunk of chunk_rows rows of 0..p_b).  K and V rows of 32-row tiles
// arrive by 1-D bulk copies into a 3-stage ring.  4 warps (4 CTAs fit an SM,
// so a batch of 64 x 8 (sequence, KV head) pairs is one wave).  Lane octets:
// each warp takes 4 rows of a tile at once (two passes per 32-row tile), 8
// lanes per row; lane o of an octet holds elements
// [o*D/16, (o+1)*D/16) and the same span of the second half of the row (so
// the 8 lanes of a row read 8 consecutive 16-byte pieces: no bank conflicts),
// a dot product is 3 shuffles, and every octet keeps its own fp32 online
// softmax (base-2 exponent) per query head.  The octets and warps merge at
// the end; a CTA that holds the whole context writes the o_proj operand
// planes, otherwise the last chunk CTA of (b, g) merges the chunks.
struct AttnArgs2 {
  int B, Hq, Hkv, max_ctx, kv_batch, l;
  int one_seq;     // -1: row b is cache sequence b; >= 0: every row is that sequence
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

// (d0, d1) += (a0, a1) * (b0, b1) as one packed fp32x2 instruction.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0,
                                     float b1) {
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "mov.b64 pd, {%0, %1};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pd;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Elements [i*HALF, i*HALF + HALF) (i = 0, 1) of this lane's two spans of a
// K or V row as fp32: bf16 values, or E4M3 code values (the caller applies
// the row scale once per row).
template <int D, bool FP8>
__device__ __forceinline__ void load_span(const uint8_t* row, int o, int i, float (&x)[D / 16]) {
  constexpr int HALF = D / 16;
  const int e0 = i * (D / 2) + o * HALF;
  if constexpr (!FP8) {
    if constexpr (HALF == 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(row + 2 * e0);
      x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
      x[4] = bf16lo(w.z); x[5] = bf16hi(w.z); x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(row + 2 * e0);
      x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
    }
  } else {
    if constexpr (HALF == 8) {
      const uint2 w = *reinterpret_cast<const uint2*>(row + e0);
      const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 a0 = e4m3x2_to_f2(static_cast<uint16_t>(ws[j] & 0xFFFF));
        const float2 a1 = e4m3x2_to_f2(static_cast<uint16_t>(ws[j] >> 16));
        x[4 * j + 0] = a0.x; x[4 * j + 1] = a0.y;
        x[4 * j + 2] = a1.x; x[4 * j + 3] = a1.y;
      }
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(row + e0);
      const float2 a0 = e4m3x2_to_f2(static_cast<uint16_t>(w & 0xFFFF));
      const float2 a1 = e4m3x2_to_f2(static_cast<uint16_t>(w >> 16));
      x[0] = a0.x; x[1] = a0.y; x[2] = a1.x; x[3] = a1.y;
    }
  }
}

template <int D, bool FP8, int REP>
__global__ void __launch_bounds__(kAttThreads, 4) attn_kernel(const AttnArgs2 a) {
  constexpr int E = FP8 ? 1 : 2;                      // bytes per element
  constexpr int HALF = D / 16;                        // elements per span
  constexpr int RB = D * E;                           // bytes per row
  constexpr int kHalf = kAttTileRows * RB;            // K (or V) rows of one tile
  // a tile: K rows, V rows, then (E4M3) the K and V row scales
  constexpr int kTile = 2 * kHalf + (FP8 ? 2 * kAttTileRows * 4 : 0);
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kAttStages * kTile);
  float* merge = reinterpret_cast<float*>(full + kAttStages);  // [warps][REP][D + 2]
  __shared__ int s_last;

  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  if (*a.bad) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int oct = lane >> 3, o = lane & 7;            // row of the warp's 4, lane in the octet
  const int ci = blockIdx.x % a.chunks;
  const int bg = blockIdx.x / a.chunks;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int len = a.pos[b] + 1;
  const int nchunk = (len + a.chunk_rows - 1) / a.chunk_rows;
  if (ci >= nchunk) return;
  const int j0 = ci * a.chunk_rows;
  const int j1 = min(j0 + a.chunk_rows, len);
  const int ntiles = (j1 - j0 + kAttTileRows - 1) / kAttTileRows;
  const int cs = a.one_seq >= 0 ? a.one_seq : b;  // cache sequence of row b
  const size_t kplane = ((static_cast<size_t>(a.l) * 2 + 0) * a.kv_batch + cs) * a.Hkv + g;
  const size_t vplane = ((static_cast<size_t>(a.l) * 2 + 1) * a.kv_batch + cs) * a.Hkv + g;
  const uint8_t* kbase = a.kv + kplane * a.max_ctx * RB;
  const uint8_t* vbase = a.kv + vplane * a.max_ctx * RB;
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
    const uint32_t rb = static_cast<uint32_t>(nr) * RB;
    uint64_t* bar = &full[t % kAttStages];
    uint8_t* dst = ring + (t % kAttStages) * kTile;
    // scales: rows j .. j + nr rounded up to 4 (16 bytes; stays inside max_ctx,
    // a multiple of 16, since j is a multiple of 32)
    const uint32_t sb = FP8 ? static_cast<uint32_t>((nr + 3) & ~3) * 4u : 0u;
    mbar_arrive_expect_tx(bar, 2 * rb + 2 * sb);
    bulk_g2s(dst, kbase + static_cast<size_t>(j) * RB, rb, bar, pol);
    bulk_g2s(dst + kHalf, vbase + static_cast<size_t>(j) * RB, rb, bar, pol);
    if (FP8) {
      bulk_g2s(dst + 2 * kHalf, ksc + j, sb, bar, pol);
      bulk_g2s(dst + 2 * kHalf + kAttTileRows * 4, vsc + j, sb, bar, pol);
    }
  };
  if (tid == 0)
    for (int t = 0; t < ntiles && t < kAttStages; ++t) issue(t);

  // this lane's elements of the query heads of the group, scaled to base 2
  const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  float qv[REP][2][HALF], acc[REP][2][HALF], m[REP], ls[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) {
    m[h] = -INFINITY;
    ls[h] = 0.f;
    const float* qh = a.q + (static_cast<size_t>(b) * a.Hq + g * REP + h) * D;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int e = 0; e < HALF; ++e) {
        acc[h][i][e] = 0.f;
        qv[h][i][e] = qh[i * (D / 2) + o * HALF + e] * qscale;
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
    const float* tsc = reinterpret_cast<const float*>(tb + 2 * kHalf);
    // the tile's two passes of kAttWarps x 4 rows at once: this octet takes
    // rows r1 and r1 + kAttWarps * 4, scores both against every query head,
    // then folds both into its online softmax with one rescale, which it
    // skips when the running maximum did not move.  Dot products and the
    // value accumulation use packed fp32 pairs.  Every lane takes part in the
    // shuffles; rows past nr are masked out of the softmax.
    {
      static_assert(kAttTileRows == 2 * kAttWarps * 4, "two rows per octet per tile");
      const int r1 = warp * 4 + oct, r2 = r1 + kAttWarps * 4;
      const bool ok1 = r1 < nr, ok2 = r2 < nr;  // ok2 implies ok1
      const uint8_t* krow1 = tb + static_cast<size_t>(ok1 ? r1 : 0) * RB;
      const uint8_t* krow2 = tb + static_cast<size_t>(ok2 ? r2 : 0) * RB;
      float s1[REP], s2[REP];
      {
        float e1[REP], o1[REP], e2[REP], o2[REP];
#pragma unroll
        for (int h = 0; h < REP; ++h) e1[h] = o1[h] = e2[h] = o2[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          float kx1[HALF], kx2[HALF];
          load_span<D, FP8>(krow1, o, i, kx1);
          load_span<D, FP8>(krow2, o, i, kx2);
#pragma unroll
          for (int h = 0; h < REP; ++h)
#pragma unroll
            for (int e = 0; e < HALF; e += 2) {
              fma2(e1[h], o1[h], qv[h][i][e], qv[h][i][e + 1], kx1[e], kx1[e + 1]);
              fma2(e2[h], o2[h], qv[h][i][e], qv[h][i][e + 1], kx2[e], kx2[e + 1]);
            }
        }
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          s1[h] = e1[h] + o1[h];
          s2[h] = e2[h] + o2[h];
        }
      }
#pragma unroll
      for (int sh = 4; sh > 0; sh >>= 1)
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          s1[h] += __shfl_xor_sync(0xffffffffu, s1[h], sh);
          s2[h] += __shfl_xor_sync(0xffffffffu, s2[h], sh);
        }
      if (FP8) {  // q . (code x scale) = scale x (q . code)
        const float ks1 = tsc[ok1 ? r1 : 0], ks2 = tsc[ok2 ? r2 : 0];
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          s1[h] *= ks1;
          s2[h] *= ks2;
        }
      }
      if (ok1) {
        float p1[REP], p2[REP];
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          const float x2 = ok2 ? s2[h] : -INFINITY;
          const float mn = fmaxf(m[h], fmaxf(s1[h], x2));
          const float al = exp2f(m[h] - mn);
          p1[h] = exp2f(s1[h] - mn);
          p2[h] = exp2f(x2 - mn);
          ls[h] = ls[h] * al + (p1[h] + p2[h]);
          m[h] = mn;
          if (al != 1.f) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int e = 0; e < HALF; ++e) acc[h][i][e] *= al;
          }
        }
        if (FP8) {  // p (code x scale) = (p scale) code
          const float vs1 = tsc[kAttTileRows + r1], vs2 = tsc[kAttTileRows + (ok2 ? r2 : r1)];
#pragma unroll
          for (int h = 0; h < REP; ++h) {
            p1[h] *= vs1;
            p2[h] *= vs2;
          }
        }
        const uint8_t* vrow1 = krow1 + kHalf;
        const uint8_t* vrow2 = (ok2 ? krow2 : krow1) + kHalf;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          float vx1[HALF], vx2[HALF];
          load_span<D, FP8>(vrow1, o, i, vx1);
          load_span<D, FP8>(vrow2, o, i, vx2);
#pragma unroll
          for (int h = 0; h < REP; ++h)
#pragma unroll
            for (int e = 0; e < HALF; e += 2) {
              fma2(acc[h][i][e], acc[h][i][e + 1], p1[h], p1[h], vx1[e], vx1[e + 1]);
              fma2(acc[h][i][e], acc[h][i][e + 1], p2[h], p2[h], vx2[e], vx2[e + 1]);
            }
        }
      }
    }
    __syncthreads();  // slot t % stages fully read
    if (tid == 0 && t + kAttStages < ntiles) issue(t + kAttStages);
  }
  // merge the four octets of the warp (lanes o, o + 8, o + 16, o + 24 hold
  // the same elements), then octet 0 writes the warp's state
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
  const int HqD = a.Hq * D;
  // merge the warps: thread t -> (head, element)
  for (int t = tid; t < REP * D; t += kAttThreads) {
    const int h = t / D, d = t % D;
    float M = -INFINITY;
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, merge[(w * REP + h) * (D + 2) + D]);
    float Ls = 0.f, A = 0.f;
    for (int w = 0; w < kAttWarps; ++w) {
      const float* mg = merge + (w * REP + h) * (D + 2);
      const float e = (mg[D] == -INFINITY) ? 0.f : exp2f(mg[D] - M);
      Ls += mg[D + 1] * e;
      A += mg[d] * e;
    }
    if (nchunk == 1) {  // the whole context: this CTA writes the output
      put_act(a.out, b, (g * REP + h) * D + d, HqD, A / Ls);
    } else {
      float* pp =
          a.part + ((static_cast<size_t>(b) * a.Hq + g * REP + h) * a.chunks + ci) * (D + 2);
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
  for (int t = tid; t < REP * D; t += kAttThreads) {
    const int h = t / D, d = t % D;
    const float* pb = a.part + (static_cast<size_t>(b) * a.Hq + g * REP + h) * a.chunks * (D + 2);
    float M = -INFINITY;
    for (int c = 0; c < nchunk; ++c) M = fmaxf(M, __ldcg(pb + c * (D + 2) + D));
    float Ls = 0.f, A = 0.f;
    for (int c = 0; c < nchunk; ++c) {
      const float e = exp2f(__ldcg(pb + c * (D + 2) + D) - M);
      Ls += __ldcg(pb + c * (D + 2) + D + 1) * e;
      A += __ldcg(pb + c * (D + 2) + d) * e;
    }
    put_act(a.out, b, (g * REP + h) * D + d, HqD, A / Ls);
  }
}

size_t attn_smem(int D, int rep, bool fp8) {
  return static_cast<size_t>(kAttStages) * (kAttTileRows * D * (fp8 ? 1 : 2) * 2 +
                                            (fp8 ? 2 * kAttTileRows * 4 : 0)) +
         kAttStages * sizeof(uint64_t) + static_cast<size_t>(kAttWarps) * rep * (D + 2) * sizeof(float);
}

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Launch with the programmatic-dependent-launch attribute and, for split-K
// GEMMs, a (1, cluster_y, 1) cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, unsigned cluster_y, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_y > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = 1;
    at[n].val.clusterDim.y = cluster_y;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

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
  int w8 = 0;  // 1 / 2: int8 / E4M3 projections and lm_head (codes + fp32 row scales)
  int n_ssp = 0;
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
  float* ssp = nullptr;
  float* att_part = nullptr;
  unsigned* att_cnt = nullptr;
  unsigned long long* keys = nullptr;
  int* bad = nullptr;
  unsigned long long* prof = nullptr;  // profiling builds: GEMM phase timestamps
};

namespace {

// bf16 [rows][cols] (128-byte swizzle, the MMA's operand layout), or int8
// codes (i8: no swizzle, row r of a box at byte 64 r; widened by the CTA)
bool encode_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                uint32_t box_rows, bool i8 = false) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (i8 ? 1 : 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunkK), box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             i8 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K splits (= cluster size) so that tiles x splits covers the SMs about once.
int pick_splits(int tiles, int k_chunks, int sms) {
  int s = (sms + tiles / 2) / tiles;
  if (s < 1) s = 1;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s > k_chunks) s = k_chunks;
  return s;
}

// n_mat matrices stacked along their rows; box_rows = 128 (one matrix per
// tile) or 64 (gate/up pairs: 64 rows of each per tile).
// w8: the matrices are int8 codes with fp32 row scales sc[i]
bool make_gemm(EncodeTiledFn enc, GemmPlan& gp, int n_mat, const void* const* w,
               const int* rows, int K, uint32_t box_rows, const CUtensorMap* xmap, int sms,
               bool one_split, bool w8 = false, const float* const* sc = nullptr) {
  GemmArgs& g = gp.args;
  g = GemmArgs{};
  g.n_mat = box_rows == kTileM ? n_mat : 1;
  int tiles = 0;
  for (int i = 0; i < 3; ++i) {
    if (i < n_mat) {
      g.rows[i] = rows[i];
      g.tiles[i] = (rows[i] + static_cast<int>(box_rows) - 1) / static_cast<int>(box_rows);
      if (box_rows == kTileM || i == 0) tiles += g.tiles[i];
      if (!encode_map(enc, &gp.w[i], w[i], K, rows[i], box_rows, w8)) return false;
      g.wsc[i] = w8 ? sc[i] : nullptr;
    } else {
      gp.w[i] = gp.w[0];
      g.wsc[i] = g.wsc[0];
    }
  }
  g.k_chunks = (K + kChunkK - 1) / kChunkK;
  g.splits = one_split ? 1 : pick_splits(tiles, g.k_chunks, sms);
  gp.x = xmap;
  gp.grid = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(g.splits));
  return true;
}

template <int MODE>
cudaError_t launch_gemm(const GemmPlan& gp, const GemmArgs& g, int w8, cudaStream_t st) {
  if (w8 == 1)
    return launch_pdl(gemm_kernel<MODE, 1>, gp.grid, dim3(kGemmThreads), kGemmSmem, st,
                      static_cast<unsigned>(g.splits), gp.w[0], gp.w[1], gp.w[2], *gp.x, g);
  if (w8 == 2)
    return launch_pdl(gemm_kernel<MODE, 2>, gp.grid, dim3(kGemmThreads), kGemmSmem, st,
                      static_cast<unsigned>(g.splits), gp.w[0], gp.w[1], gp.w[2], *gp.x, g);
  return launch_pdl(gemm_kernel<MODE, 0>, gp.grid, dim3(kGemmThreads), kGemmSmem, st,
                    static_cast<unsigned>(g.splits), gp.w[0], gp.w[1], gp.w[2], *gp.x, g);
}

template <int MODE, int W8>
cudaError_t gemm_attrs() {
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel<MODE, W8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGemmSmem));
  if (e == cudaSuccess && MODE != kLm)
    e = cudaFuncSetAttribute(gemm_kernel<MODE, W8>,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int W8>
cudaError_t all_gemm_attrs() {
  cudaError_t e = gemm_attrs<kQKV, W8>();
  if (e == cudaSuccess) e = gemm_attrs<kResid, W8>();
  if (e == cudaSuccess) e = gemm_attrs<kSwiGLU, W8>();
  if (e == cudaSuccess) e = gemm_attrs<kLm, W8>();
  return e;
}

template <int D, int REP>
cudaError_t launch_attn_rep(const AttnArgs2& a, bool fp8, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(a.B) * a.Hkv * a.chunks);
  if (fp8)
    return launch_pdl(attn_kernel<D, true, REP>, grid, dim3(kAttThreads), attn_smem(D, REP, true),
                      st, 1u, a);
  return launch_pdl(attn_kernel<D, false, REP>, grid, dim3(kAttThreads), attn_smem(D, REP, false),
                    st, 1u, a);
}

template <int D>
cudaError_t launch_attn(const AttnArgs2& a, int rep, bool fp8, cudaStream_t st) {
  switch (rep) {
    case 1: return launch_attn_rep<D, 1>(a, fp8, st);
    case 2: return launch_attn_rep<D, 2>(a, fp8, st);
    case 3: return launch_attn_rep<D, 3>(a, fp8, st);
    case 4: return launch_attn_rep<D, 4>(a, fp8, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int REP>
cudaError_t attn_attrs() {
  const cudaFuncAttribute dyn = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, false, REP>, dyn,
                                       static_cast<int>(attn_smem(D, REP, false)));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_kernel<D, true, REP>, dyn,
                             static_cast<int>(attn_smem(D, REP, true)));
  return e;
}

template <int D>
cudaError_t attn_attrs_for(int rep) {
  switch (rep) {
    case 1: return attn_attrs<D, 1>();
    case 2: return attn_attrs<D, 2>();
    case 3: return attn_attrs<D, 3>();
    case 4: return attn_attrs<D, 4>();
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int bt_plan_create(const BtShape& s, const uint16_t* embed, const void* lm_head,
                   const uint16_t* final_norm, const LayerPtrs* layers_host,
                   const float* inv_freq_dev, int sms, BtPlan** out, cudaError_t* cerr,
                   const float* lm_scale, const LayerScales* scales_host, int w8) {
  *out = nullptr;
  if ((w8 != 0) != (scales_host != nullptr)) return DEC_ERR_ARG;
  *cerr = cudaSuccess;
  const int HqD = s.Hq * s.D, HkvD = s.Hkv * s.D;
  // tiles of 128 q / k / v rows hold whole heads; gate/up tiles pair 64 rows
  if (s.H % kChunkK || HqD % kTileM || HkvD % kTileM || s.F % (kTileM / 2)) return DEC_ERR_SHAPE;
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
  p->w8 = w8;
  p->n_ssp = (s.H + kTileM - 1) / kTileM;
  p->embed = embed;
  p->final_norm = final_norm;
  p->inv_freq = inv_freq_dev;
  p->layers.assign(layers_host, layers_host + s.L);

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
  const size_t ssp_off = take(sizeof(float) * kTileN * p->n_ssp);
  const size_t ap_off = take(sizeof(float) * kTileN * s.Hq * kMaxAttnChunks * (s.D + 2));
  const size_t ac_off = take(sizeof(unsigned) * kTileN * s.Hkv);
  const size_t keys_off = take(sizeof(unsigned long long) * kTileN);
  const size_t bad_off = take(sizeof(int));
#ifdef DEC_PROFILE
  const size_t prof_off = take(sizeof(unsigned long long) * 4 * kProfCtas * 16);
#endif
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
  p->ssp = reinterpret_cast<float*>(p->ws + ssp_off);
  p->att_part = reinterpret_cast<float*>(p->ws + ap_off);
  p->att_cnt = reinterpret_cast<unsigned*>(p->ws + ac_off);
  p->keys = reinterpret_cast<unsigned long long*>(p->ws + keys_off);
  p->bad = reinterpret_cast<int*>(p->ws + bad_off);
#ifdef DEC_PROFILE
  p->prof = reinterpret_cast<unsigned long long*>(p->ws + prof_off);
#endif

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
    const float* const* ls = w8 ? scales_host[l].s : nullptr;  // row scales of 8-bit codes
    auto sc = [&](int j) { return ls ? ls[j] : nullptr; };
    const void* wqkv[3] = {lp.w[DEC_LW_Q], lp.w[DEC_LW_K], lp.w[DEC_LW_V]};
    const float* sqkv[3] = {sc(DEC_LW_Q), sc(DEC_LW_K), sc(DEC_LW_V)};
    const int rqkv[3] = {HqD, HkvD, HkvD};
    const void* wo[1] = {lp.w[DEC_LW_O]};
    const float* so[1] = {sc(DEC_LW_O)};
    const int ro[1] = {s.H};
    const void* wgu[2] = {lp.w[DEC_LW_GATE], lp.w[DEC_LW_UP]};
    const float* sgu[2] = {sc(DEC_LW_GATE), sc(DEC_LW_UP)};
    const int rgu[2] = {s.F, s.F};
    const void* wd[1] = {lp.w[DEC_LW_DOWN]};
    const float* sd[1] = {sc(DEC_LW_DOWN)};
    ok = make_gemm(enc, p->qkv[l], 3, wqkv, rqkv, s.H, kTileM, &p->map_h, sms, false, w8, sqkv) &&
         make_gemm(enc, p->o[l], 1, wo, ro, HqD, kTileM, &p->map_o, sms, false, w8, so) &&
         make_gemm(enc, p->gu[l], 2, wgu, rgu, s.H, kTileM / 2, &p->map_h, sms, false, w8, sgu) &&
         make_gemm(enc, p->down[l], 1, wd, ro, s.F, kTileM, &p->map_u, sms, false, w8, sd);
  }
  if (ok) {
    const void* wl[1] = {lm_head};
    const float* sl[1] = {lm_scale};
    const int rl[1] = {s.V};
    ok = make_gemm(enc, p->lm, 1, wl, rl, s.H, kTileM, &p->map_h, sms, true, w8, sl);
  }
  // kernel attributes, once
  if (ok) e = w8 == 1 ? all_gemm_attrs<1>() : (w8 == 2 ? all_gemm_attrs<2>() : all_gemm_attrs<0>());
  const int rep = s.Hq / s.Hkv;
  if (ok && e == cudaSuccess) e = s.D == 128 ? attn_attrs_for<128>(rep) : attn_attrs_for<64>(rep);
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

cudaError_t bt_step(BtPlan* p, const BtIO& io, cudaStream_t st) {
  const BtShape& s = p->s;
  // fields every GEMM launch shares
  GemmArgs base{};
  base.B = io.B;
  base.H = s.H;
  base.D = s.D;
  base.Hq = s.Hq;
  base.Hkv = s.Hkv;
  base.F = s.F;
  base.eps = s.eps;
  base.n_ssp = p->n_ssp;
  base.ssp_in = p->ssp;
  base.ssp_out = p->ssp;
  base.x = p->x;
  base.q = p->q;
  base.kv = io.kv;
  base.kv_scales = io.kv_scales;
  base.kv_batch = io.kv_batch;
  base.max_ctx = io.max_ctx;
  base.kv_fp8 = io.kv_fp8;
  base.one_seq = io.one_seq;
  base.pos = io.pos;
  base.retired = io.retired;
  base.bad = p->bad;
  base.inv_freq = p->inv_freq;
  base.keys = p->keys;
  base.status = io.status;
  base.timeout_ns = io.timeout_ns;
  base.prof = p->prof;
  auto args_of = [&](const GemmPlan& gp) {
    GemmArgs g = base;
    g.n_mat = gp.args.n_mat;
    for (int i = 0; i < 3; ++i) {
      g.rows[i] = gp.args.rows[i];
      g.tiles[i] = gp.args.tiles[i];
    }
    g.k_chunks = gp.args.k_chunks;
    g.splits = gp.args.splits;
    for (int i = 0; i < 3; ++i) g.wsc[i] = gp.args.wsc[i];
    return g;
  };

  // attention chunking: one wave of CTAs (4 resident per SM) over the
  // (sequence, KV head) pairs, i.e. one chunk per pair once there are enough
  // pairs; at most kMaxAttnChunks chunks per pair
  int per_pair = (4 * p->sms) / (io.B * s.Hkv);
  // Long contexts: up to three waves, in chunks of at least kAttMinSplitRows
  // rows, so that the longest sequence of a ragged batch does not alone set
  // the kernel's length (1.7B shape, batch 64, contexts U[2048, 4064]:
  // attention -8 % with E4M3 rows, -4.5 % with bf16); below that the extra
  // merges cost more than the balance saves (0.6B, contexts U[200, 420]: +11 %).
  const int waves3 = (3 * 4 * p->sms) / (io.B * s.Hkv);
  const int by_len = io.max_ctx / kAttMinSplitRows;
  if (waves3 > per_pair) per_pair = max(per_pair, min(waves3, by_len));
  if (per_pair < 1) per_pair = 1;
  if (per_pair > kMaxAttnChunks) per_pair = kMaxAttnChunks;
  int cr = (io.max_ctx + per_pair - 1) / per_pair;
  cr = (cr + kAttTileRows - 1) / kAttTileRows * kAttTileRows;
  AttnArgs2 at{};
  at.B = io.B;
  at.Hq = s.Hq;
  at.Hkv = s.Hkv;
  at.max_ctx = io.max_ctx;
  at.kv_batch = io.kv_batch;
  at.one_seq = io.one_seq;
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

  StepArgs2 sa{};
  sa.B = io.B;
  sa.H = s.H;
  sa.V = s.V;
  sa.n_ssp = p->n_ssp;
  sa.max_ctx = io.max_ctx;
  sa.tok = io.tok;
  sa.pos = io.pos;
  sa.out = io.out;
  sa.embed = p->embed;
  sa.g_in = p->layers[0].w[DEC_LW_IN_NORM];
  sa.x = p->x;
  sa.act_h = p->act_h;
  sa.ssp = p->ssp;
  sa.keys = p->keys;
  sa.bad = p->bad;
  sa.status = io.status;
  sa.hidden = io.hidden;

  cudaError_t e = launch_pdl(embed_kernel, dim3(io.B), dim3(kRowThreads), 0, st, 1u, sa);
  if (e != cudaSuccess) return e;
  for (int l = 0; l < s.L; ++l) {
    const LayerPtrs& lp = p->layers[l];
    GemmArgs g = args_of(p->qkv[l]);
    g.layer = l;
    g.gain = lp.w[DEC_LW_Q_NORM];
    g.gain2 = lp.w[DEC_LW_K_NORM];
    if ((e = launch_gemm<kQKV>(p->qkv[l], g, p->w8, st)) != cudaSuccess) return e;
    at.l = l;
    e = s.D == 128 ? launch_attn<128>(at, rep, io.kv_fp8 != 0, st)
                   : launch_attn<64>(at, rep, io.kv_fp8 != 0, st);
    if (e != cudaSuccess) return e;
    g = args_of(p->o[l]);
    g.gain = lp.w[DEC_LW_POST_NORM];
    g.act = p->act_h;
    g.hidden = nullptr;
    if ((e = launch_gemm<kResid>(p->o[l], g, p->w8, st)) != cudaSuccess) return e;
    g = args_of(p->gu[l]);
    g.act = p->act_u;
    if ((e = launch_gemm<kSwiGLU>(p->gu[l], g, p->w8, st)) != cudaSuccess) return e;
    g = args_of(p->down[l]);
    g.gain = l + 1 < s.L ? p->layers[l + 1].w[DEC_LW_IN_NORM] : p->final_norm;
    g.act = p->act_h;
    g.hidden = io.hidden ? io.hidden + static_cast<size_t>(l + 1) * io.B * s.H : nullptr;
    if ((e = launch_gemm<kResid>(p->down[l], g, p->w8, st)) != cudaSuccess) return e;
  }
  GemmArgs g = args_of(p->lm);
  g.logits = io.logits;
  if ((e = launch_gemm<kLm>(p->lm, g, p->w8, st)) != cudaSuccess) return e;
  return launch_pdl(finish_kernel, dim3(1), dim3(kTileN), 0, st, 1u, sa);
}

}  // namespace dec

#ifdef DEC_PROFILE
namespace dec {
// Profiling builds: the GEMM phase timestamps of the last launch of each mode.
int bt_prof_read(BtPlan* p, unsigned long long* host, size_t n) {
  const size_t need = 4ull * kProfCtas * 16;
  if (!p || !p->prof || n < need) return -1;
  return cudaMemcpy(host, p->prof, need * sizeof(unsigned long long), cudaMemcpyDeviceToHost) ==
                 cudaSuccess
             ? 0
             : -1;
}
}  // namespace dec
#endif
