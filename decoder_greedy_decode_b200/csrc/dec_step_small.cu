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
//    running up to a whole ring (~190 KB, about one layer's share) ahead of
//    the consumers.  HBM therefore keeps streaming while consumers wait for
//    activations.
//  * Activations move between CTAs as 8-byte words {fp32 value, 32-bit flag}
//    in global memory (L2).  A consumer polls the words it needs until their
//    flags equal the expected (step, layer) tag: data and readiness arrive
//    in one load, with no separate barrier round trip.
//  * Rows of every projection are split evenly over CTAs.  Each CTA owns the
//    same hidden rows in o_proj and down, so it keeps those residual entries
//    in shared memory.  Attention is split-K over (sequence, KV head, chunk)
//    items; the last CTA to finish a (sequence, KV head) merges the partials
//    (flash-decoding combine) and publishes the head outputs.
//  * Every wait is bounded (globaltimer).  A wait that runs out raises a
//    status bit and a global abort flag; all CTAs then drain their in-flight
//    copies without computing and leave; out_ids becomes -1.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "dec_internal.h"
#include "dec_ptx.cuh"
#include "dec_quant.cuh"

namespace dec {
namespace {

constexpr int kCW = kConsumerWarps;
constexpr int kCT = kConsumerThreads;
constexpr int kMaxHRows = 64;  // hidden rows a CTA may own
constexpr int kDevTimeout = 4;
constexpr int kDevBadPos = 1;
constexpr int kDevBadTok = 2;

// Optional per-phase timestamps (profiling builds only, -DDEC_PROFILE): thread
// 0 of every CTA records globaltimer at the phase boundaries of the step into
// prof[cta][8 * L + 4]: 8l+0 layer start, +1 QKV published, +2 attention
// inputs gathered and rotated, +3 attention rows consumed and merged, +4
// attention done, +5 o_proj published, +6 gate/up published, +7 down
// published; 8L+0 lm_head start, +1 lm_head done, +2 consumer end,
// +3 consumer start.
#ifdef DEC_PROFILE
#define DEC_STAMP(i)                                                                   \
  do {                                                                                 \
    if (a.prof && tid == 0)                                                            \
      a.prof[static_cast<size_t>(cta) * (8 * a.L + 4) + (i)] = globaltimer();          \
  } while (0)
#else
#define DEC_STAMP(i) \
  do {               \
  } while (0)
#endif

__host__ __device__ inline int split_at(int n, int parts, int i) {
  return static_cast<int>((static_cast<long long>(n) * i) / parts);
}

struct Carve {
  size_t ring, bars, act, xown, red, bred, ints, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Carve carve(int nslot, int B, int kmax, int rmax, int D, int rep,
                                       int nchunks) {
  Carve c;
  size_t o = 0;
  c.ring = o;
  o += static_cast<size_t>(nslot) * kSlotBytes;
  c.bars = o;
  o += align_up(2 * nslot * sizeof(uint64_t), 16);
  size_t act_f = static_cast<size_t>(B) * kmax;
  size_t att_f = static_cast<size_t>(rep + 2) * D + static_cast<size_t>(kCW + rep) * (D + 2) +
                 static_cast<size_t>(nchunks) * rep * 2;
  c.act = o;
  o += align_up((act_f > att_f ? act_f : att_f) * sizeof(float), 16);
  c.xown = o;
  o += align_up(static_cast<size_t>(kMaxHRows) * B * sizeof(float), 16);
  c.red = o;
  o += align_up(2ull * rmax * B * kCW * sizeof(float), 16);
  c.bred = o;
  o += align_up(2ull * kCW * B * sizeof(float) + 2ull * kCW * B * sizeof(int), 16);
  c.ints = o;
  o += 64 * sizeof(int);
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

// The per-launch state of one CTA.
template <int B, int D>
struct Cta {
  static constexpr int DL = D / 32;  // attention dims per lane
  const StepArgs& a;
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  float* act;
  float* xown;
  float* red;
  float* bredf;
  int* bredi;
  int* sints;
  int tid, warp, lane, cta, nc;
  int kmax, rmax, nqkv;
  uint32_t seq;
  // per-CTA row ranges
  int q0, q1, h0, h1, f0, f1, v0, v1;
  int rpt_h, rpt_o, rpt_u, rpt_d, art;
  // attention work split
  int crow, n_items;
  int* pos;     // [B] positions (shared memory)
  int* tok;     // [B] tokens (shared memory)
  int* nchunk;  // [B] attention chunks per KV head (shared memory)

  __device__ Cta(const StepArgs& args, uint8_t* smem, int kmax_, int rmax_)
      : a(args), kmax(kmax_), rmax(rmax_) {
    const int rep = a.Hq / a.Hkv;
    Carve c = carve(a.nslot, B, kmax, rmax, D, rep, a.part_chunks);
    ring = smem + c.ring;
    full = reinterpret_cast<uint64_t*>(smem + c.bars);
    empty = full + a.nslot;
    act = reinterpret_cast<float*>(smem + c.act);
    xown = reinterpret_cast<float*>(smem + c.xown);
    red = reinterpret_cast<float*>(smem + c.red);
    bredf = reinterpret_cast<float*>(smem + c.bred);
    bredi = reinterpret_cast<int*>(bredf + 2 * kCW * B);
    sints = reinterpret_cast<int*>(smem + c.ints);
    pos = sints + 8;
    tok = sints + 16;
    nchunk = sints + 24;
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
    rpt_h = kSlotBytes / (2 * a.H);
    rpt_o = kSlotBytes / (2 * a.Hq * D);
    rpt_u = kSlotBytes / (4 * a.H);
    rpt_d = kSlotBytes / (2 * a.F);
    if (a.kv_fp8) {
      art = (kSlotBytes / (2 * D + 8)) & ~15;
    } else {
      art = kSlotBytes / (4 * D);
    }
  }

  __device__ __forceinline__ uint32_t flag(int layer) const {
    return seq * 256u + static_cast<uint32_t>(layer) + 1u;
  }

  // Attention items: (b, g, chunk) over contexts 0..p_b, chunk rows `crow`,
  // so that the items fit the grid when possible.  Same on every CTA.
  __device__ void plan_attention() {
    long long T = 0;
    for (int b = 0; b < a.B; ++b) T += static_cast<long long>(pos[b] + 1) * a.Hkv;
    int slots = nc - a.B * a.Hkv;
    if (slots < 1) slots = 1;
    long long cr = (T + slots - 1) / slots;
    cr = (cr + 15) / 16 * 16;
    if (cr < 16) cr = 16;
    crow = static_cast<int>(cr);
    n_items = 0;
    for (int b = 0; b < a.B; ++b) {
      const int nb = (pos[b] + 1 + crow - 1) / crow;
      if (tid == 0) nchunk[b] = nb;
      n_items += nb * a.Hkv;
    }
  }
  __device__ void item(int it, int& b, int& g, int& ci) const {
    int bb = 0;
    while (bb < a.B - 1 && it >= nchunk[bb] * a.Hkv) {
      it -= nchunk[bb] * a.Hkv;
      ++bb;
    }
    b = bb;
    g = it / nchunk[bb];
    ci = it % nchunk[bb];
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
    uint32_t n = 0;
    bool dead = false;
    const int ns = a.nslot;
    auto acquire = [&](uint32_t bytes) -> uint8_t* {
      const int slot = static_cast<int>(n % ns);
      if (n >= static_cast<uint32_t>(ns)) {
        const uint32_t par = ((n / ns) - 1) & 1;
        Spin sp;
        while (!mbar_test(&empty[slot], par)) {
          if (sp.tick(a, false)) {
            dead = true;
            return nullptr;
          }
        }
      }
      mbar_arrive_expect_tx(&full[slot], bytes);
      return ring + static_cast<size_t>(slot) * kSlotBytes;
    };
    const int H = a.H, HqD = a.Hq * D, HkvD = a.Hkv * D;
    for (int l = 0; l < a.L && !dead; ++l) {
      const LayerPtrs& lw = a.layers[l];
      // ---- QKV rows [q0, q1) of [Wq; Wk; Wv]
      for (int r = q0; r < q1 && !dead; r += rpt_h) {
        const int nr = min(rpt_h, q1 - r);
        uint8_t* dst = acquire(static_cast<uint32_t>(nr) * H * 2);
        if (!dst) break;
        int rr = r, left = nr;
        while (left > 0) {
          const uint16_t* base;
          int lo, cnt;
          if (rr < HqD) {
            base = lw.w[1]; lo = rr; cnt = min(left, HqD - rr);
          } else if (rr < HqD + HkvD) {
            base = lw.w[2]; lo = rr - HqD; cnt = min(left, HqD + HkvD - rr);
          } else {
            base = lw.w[3]; lo = rr - HqD - HkvD; cnt = left;
          }
          bulk_g2s(dst, base + static_cast<size_t>(lo) * H, static_cast<uint32_t>(cnt) * H * 2,
                   &full[n % ns], pol);
          dst += static_cast<size_t>(cnt) * H * 2;
          rr += cnt;
          left -= cnt;
        }
        ++n;
      }
      // ---- attention: cached rows [j0, min(j1, p_b)) of every item of this CTA
      for (int it = cta; it < n_items && !dead; it += nc) {
        int b, g, ci;
        item(it, b, g, ci);
        const int j0 = ci * crow;
        const int jc = min(j0 + crow, pos[b]);
        for (int j = j0; j < jc && !dead; j += art) {
          const int nr = min(art, jc - j);
          if (!a.kv_fp8) {
            const uint32_t rb = static_cast<uint32_t>(nr) * D * 2;
            uint8_t* dst = acquire(2 * rb);
            if (!dst) break;
            const uint16_t* kvb = reinterpret_cast<const uint16_t*>(a.kv);
            bulk_g2s(dst, kvb + kv_row(l, 0, b, g, j) * D, rb, &full[n % ns], pol);
            bulk_g2s(dst + rb, kvb + kv_row(l, 1, b, g, j) * D, rb, &full[n % ns], pol);
          } else {
            const uint32_t rb = static_cast<uint32_t>(nr) * D;
            const uint32_t sb = static_cast<uint32_t>((nr + 3) & ~3) * 4;
            uint8_t* dst = acquire(2 * rb + 2 * sb);
            if (!dst) break;
            bulk_g2s(dst, a.kv + kv_row(l, 0, b, g, j) * D, rb, &full[n % ns], pol);
            bulk_g2s(dst + rb, a.kv + kv_row(l, 1, b, g, j) * D, rb, &full[n % ns], pol);
            bulk_g2s(dst + 2 * rb, a.kv_scales + kv_row(l, 0, b, g, j), sb, &full[n % ns], pol);
            bulk_g2s(dst + 2 * rb + sb, a.kv_scales + kv_row(l, 1, b, g, j), sb, &full[n % ns],
                     pol);
          }
          ++n;
        }
      }
      // ---- o_proj rows [h0, h1), K = Hq*D
      for (int r = h0; r < h1 && !dead; r += rpt_o) {
        const int nr = min(rpt_o, h1 - r);
        uint8_t* dst = acquire(static_cast<uint32_t>(nr) * HqD * 2);
        if (!dst) break;
        bulk_g2s(dst, lw.w[6] + static_cast<size_t>(r) * HqD, static_cast<uint32_t>(nr) * HqD * 2,
                 &full[n % ns], pol);
        ++n;
      }
      // ---- gate / up rows [f0, f1): a tile is nr gate rows then nr up rows
      for (int r = f0; r < f1 && !dead; r += rpt_u) {
        const int nr = min(rpt_u, f1 - r);
        const uint32_t rb = static_cast<uint32_t>(nr) * H * 2;
        uint8_t* dst = acquire(2 * rb);
        if (!dst) break;
        bulk_g2s(dst, lw.w[8] + static_cast<size_t>(r) * H, rb, &full[n % ns], pol);
        bulk_g2s(dst + rb, lw.w[9] + static_cast<size_t>(r) * H, rb, &full[n % ns], pol);
        ++n;
      }
      // ---- down rows [h0, h1), K = F
      for (int r = h0; r < h1 && !dead; r += rpt_d) {
        const int nr = min(rpt_d, h1 - r);
        uint8_t* dst = acquire(static_cast<uint32_t>(nr) * a.F * 2);
        if (!dst) break;
        bulk_g2s(dst, lw.w[10] + static_cast<size_t>(r) * a.F,
                 static_cast<uint32_t>(nr) * a.F * 2, &full[n % ns], pol);
        ++n;
      }
    }
    // ---- lm_head rows [v0, v1)
    for (int r = v0; r < v1 && !dead; r += rpt_h) {
      const int nr = min(rpt_h, v1 - r);
      uint8_t* dst = acquire(static_cast<uint32_t>(nr) * H * 2);
      if (!dst) break;
      bulk_g2s(dst, a.lm_head + static_cast<size_t>(r) * H, static_cast<uint32_t>(nr) * H * 2,
               &full[n % ns], pol);
      ++n;
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
  uint32_t rn = 0;         // ring tile counter (consumer side)
  int ab = 0;              // aborted: keep the barrier sequence, compute nothing
  bool ring_dead = false;  // a ring wait ran out: stop waiting on the ring

  __device__ __forceinline__ void csync() { named_sync(1, kCT); }

  // Wait for ring tile rn.  Every consumer thread calls it for every tile, so
  // the barrier sequence stays uniform even when a wait runs out: the thread
  // then only stops computing (ab) and stops waiting on the ring.
  // The outcome is made warp-uniform (__all_sync / __any_sync) so that warp
  // collectives after it never see a split warp.
  __device__ void wait_tile() {
    if (ring_dead) return;
    const int slot = static_cast<int>(rn % a.nslot);
    const uint32_t par = (rn / a.nslot) & 1;
    Spin sp;
    while (true) {
      const bool done = mbar_test(&full[slot], par);
      if (__all_sync(0xffffffffu, done)) break;
      const bool out = sp.tick(a, false);
      if (__any_sync(0xffffffffu, out)) {
        ring_dead = true;
        ab = 1;
        return;
      }
    }
  }
  __device__ __forceinline__ void release_tile() {
    __syncwarp();
    if (lane == 0 && !ring_dead) mbar_arrive(&empty[rn % a.nslot]);
    ++rn;
  }

  // Poll `n` tagged words (element i at src[idx(i)]) until their flag is `f`,
  // store the values to dst[i].  Collective over the consumer threads.
  // All loads of a round are issued before any is checked, so a gather of up
  // to 16 words per thread costs one L2 round trip when the data is there.
  template <class Idx, class Didx>
  __device__ void gather(const uint64_t* src, int n, uint32_t f, float* dst, Idx idx, Didx didx) {
    constexpr int kRound = 8;
    int fail = 0;
    if (!ab) {
      for (int base = tid; base < n && !fail; base += kCT * kRound) {
        uint64_t w[kRound];
#pragma unroll
        for (int k = 0; k < kRound; ++k) {
          const int i = base + k * kCT;
          if (i < n) w[k] = ld_tagged(src + idx(i));
        }
#pragma unroll
        for (int k = 0; k < kRound; ++k) {
          const int i = base + k * kCT;
          if (i < n && !fail) {
            Spin sp;
            while (static_cast<uint32_t>(w[k] >> 32) != f) {
              if (sp.tick(a, true)) {
                fail = 1;
                break;
              }
              w[k] = ld_tagged(src + idx(i));
            }
            dst[didx(i)] = __uint_as_float(static_cast<uint32_t>(w[k]));
          }
        }
      }
    }
    ab = named_sync_or(1, kCT, fail | ab);
  }
  // In-place RMSNorm of rows act[b][0..K) with bf16 gains g.
  __device__ void rmsnorm_act(int K, const uint16_t* g) {
    if (!ab) {
      float ss[B];
#pragma unroll
      for (int b = 0; b < B; ++b) ss[b] = 0.f;
      for (int k = tid; k < K; k += kCT) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
          if (b < a.B) {
            const float x = act[b * kmax + k];
            ss[b] = fmaf(x, x, ss[b]);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        ss[b] = warp_sum(ss[b]);
        if (lane == 0) bredf[warp * B + b] = ss[b];
      }
    }
    csync();
    if (!ab) {
      float inv[B];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) t += bredf[w * B + b];
        inv[b] = rsqrtf(t / static_cast<float>(K) + a.eps);
      }
      for (int k = tid; k < K; k += kCT) {
        const float gk = bf16_to_f(g[k]);
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (b < a.B) act[b * kmax + k] = act[b * kmax + k] * inv[b] * gk;
      }
    }
    csync();
  }

  // Row-group GEMV over ring tiles.  Rows [0, nrows) of the stage arrive
  // `rpt` per tile, K columns (K % 256 == 0).  One warp computes whole dot
  // products for a group of R rows (pair: R/2 rows of the first matrix and the
  // same R/2 rows of the second, which follow them in the tile), reading the
  // activations act[b][k] from shared memory, and reduces its lanes' R partial
  // sums with one transposed butterfly (R = 4: 6 shuffles instead of 20).
  // Groups are dealt to warps round-robin over the whole stage, so there is no
  // CTA barrier per tile.  Every warp waits for every tile (no warp can run a
  // ring ahead of the others) and releases it.  epi(row, b, s0, s1) is called
  // once per output row and sequence; s1 is the second matrix's sum in pair
  // mode.
  template <int R, class Epi>
  __device__ void gemv(int K, int nrows, int rpt, bool pair, Epi epi) {
    const int nv = K >> 3;
    const int per = pair ? R / 2 : R;  // output rows per group
    int gbase = 0;
    for (int r0 = 0; r0 < nrows; r0 += rpt) {
      const int nr = min(rpt, nrows - r0);
      const int ng = (nr + per - 1) / per;
      wait_tile();
      if (!ab) {
        const uint8_t* tb = ring + static_cast<size_t>(rn % a.nslot) * kSlotBytes;
        int g0 = (warp - gbase) % kCW;
        if (g0 < 0) g0 += kCW;
        for (int gl = g0; gl < ng; gl += kCW) {
          const uint8_t* rp[R];
          bool rv[R];
#pragma unroll
          for (int i = 0; i < R; ++i) {
            const int j = gl * per + (i % per);
            rv[i] = j < nr;
            const int trow = (pair && i >= per) ? nr + j : j;
            rp[i] = tb + static_cast<size_t>(rv[i] ? trow : 0) * K * 2;
          }
          float acc[R][B];
#pragma unroll
          for (int i = 0; i < R; ++i)
#pragma unroll
            for (int b = 0; b < B; ++b) acc[i][b] = 0.f;
          for (int v = lane; v < nv; v += 32) {
            float x[B][8];
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const float4* xa = reinterpret_cast<const float4*>(act + b * kmax + v * 8);
              const float4 x0 = xa[0], x1 = xa[1];
              x[b][0] = x0.x; x[b][1] = x0.y; x[b][2] = x0.z; x[b][3] = x0.w;
              x[b][4] = x1.x; x[b][5] = x1.y; x[b][6] = x1.z; x[b][7] = x1.w;
            }
#pragma unroll
            for (int i = 0; i < R; ++i) {
              if (rv[i]) {
                const uint4 w = *reinterpret_cast<const uint4*>(rp[i] + v * 16);
#pragma unroll
                for (int b = 0; b < B; ++b) acc[i][b] += dot8(w, x[b]);
              }
            }
          }
          const int ri = R == 4 ? (lane >> 3) : (R == 2 ? (lane >> 4) : 0);
          const bool leader = R == 4 ? ((lane & 7) == 0) : (R == 2 ? ((lane & 15) == 0) : lane == 0);
          float sv[B], su[B];
#pragma unroll
          for (int b = 0; b < B; ++b) {
            float col[R];
#pragma unroll
            for (int i = 0; i < R; ++i) col[i] = acc[i][b];
            sv[b] = tbfly<R>(col);
            su[b] = __shfl_down_sync(0xffffffffu, sv[b], 16);
          }
          if (leader && (!pair || ri < per)) {
            const int j = gl * per + ri;
            if (j < nr) {
#pragma unroll
              for (int b = 0; b < B; ++b)
                if (b < a.B) epi(r0 + j, b, sv[b], su[b]);
            }
          }
        }
      }
      gbase += ng;
      release_tile();
    }
  }

  // Transposed butterfly: lane l holds partial sums p[i] of R rows; returns
  // the full sum of row (R == 4: l >> 3; R == 2: l >> 4; R == 1: 0).
  template <int R>
  __device__ __forceinline__ float tbfly(float (&p)[R]) const {
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

  // ------------------------------------------------------------- attention
  // Stage buffer (in act): qs[rep][D] (normed, rotated q), kn[D], vn[D] (the
  // new row as stored), merge[kCW][D + 2], ownb[rep][D + 2] (the
  // combiner's own partial), mlb[chunks][rep][2] (other chunks' m, l).
  __device__ void attention(int l) {
    const int rep = a.Hq / a.Hkv;
    const float qscale = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e)/sqrt(D)
    float* qs = act;
    float* kn = act + rep * D;
    float* vn = kn + D;
    float* merge = vn + D;
    float* ownb = merge + kCW * (D + 2);
    float* mlb = ownb + rep * (D + 2);
    const LayerPtrs& lw = a.layers[l];
    const uint32_t f = flag(l);
    const int HqD = a.Hq * D;
    for (int it = cta; it < n_items; it += nc) {
      int b, g, ci;
      item(it, b, g, ci);
      const int p = pos[b];
      const int j0 = ci * crow;
      const int j1 = min(j0 + crow, p + 1);
      const int jc = min(j1, p);  // cached rows [j0, jc)
      const bool has_new = (p >= j0 && p < j1);
      // -- gather q heads of the group, k_g and v_g of sequence b
      {
        const uint64_t* src = a.x_qkv + static_cast<size_t>(b) * nqkv;
        const int qn = rep * D;
        const int qoff = g * rep * D, koff = HqD + g * D, voff = HqD + a.Hkv * D + g * D;
        gather(
            src, qn + 2 * D, f, act,
            [=](int i) {
              return i < qn ? qoff + i : (i < qn + D ? koff + (i - qn) : voff + (i - qn - D));
            },
            [](int i) { return i; });
      }
      // -- q/k RMSNorm + RoPE (warp w < rep: q head; rep: k; rep+1: v)
      if (!ab && warp < rep + 2) {
        float* x = warp < rep ? qs + warp * D : (warp == rep ? kn : vn);
        float v[DL];
#pragma unroll
        for (int k = 0; k < DL; ++k) v[k] = x[lane + 32 * k];
        if (warp <= rep) {
          const uint16_t* gn = warp < rep ? lw.w[4] : lw.w[5];
          float ss = 0.f;
#pragma unroll
          for (int k = 0; k < DL; ++k) ss = fmaf(v[k], v[k], ss);
          ss = warp_sum(ss);
          const float inv = rsqrtf(ss / static_cast<float>(D) + a.eps);
#pragma unroll
          for (int k = 0; k < DL; ++k) v[k] = v[k] * inv * bf16_to_f(gn[lane + 32 * k]);
#pragma unroll
          for (int k = 0; k < DL / 2; ++k) {
            const int i = lane + 32 * k;
            const float ang = __fmul_rn(static_cast<float>(p), a.inv_freq[i]);
            float sn, cs;
            sincosf(ang, &sn, &cs);
            const float x1 = v[k], x2 = v[k + DL / 2];
            v[k] = x1 * cs - x2 * sn;
            v[k + DL / 2] = x2 * cs + x1 * sn;
          }
        }
        if (warp >= rep) {
          // the new K / V row as the cache stores it
          const int kvsel = warp - rep;
          const size_t row = kv_row(l, kvsel, b, g, p);
          if (!a.kv_fp8) {
            uint16_t* dstp = reinterpret_cast<uint16_t*>(a.kv) + row * D;
#pragma unroll
            for (int k = 0; k < DL; ++k) {
              const uint16_t h = f_to_bf16(v[k]);
              v[k] = bf16_to_f(h);
              if (has_new) dstp[lane + 32 * k] = h;
            }
          } else {
            uint8_t code[DL];
            const float sc = quantize_row_e4m3<DL>(v, code);
            uint8_t* dstp = a.kv + row * D;
            if (has_new) {
#pragma unroll
              for (int k = 0; k < DL; ++k) dstp[lane + 32 * k] = code[k];
              if (lane == 0) a.kv_scales[row] = sc;
            }
          }
        }
#pragma unroll
        for (int k = 0; k < DL; ++k) x[lane + 32 * k] = v[k];
      }
      csync();
      DEC_STAMP(8 * l + 2);
      // -- partial softmax over this item's rows: warp w serves query head
      // hw = w % rep of the group on rows rw, rw + rstep, ... (rw = w / rep),
      // with a warp-level online softmax.
      const int rstep = kCW / rep;
      const int hw = warp % rep, rw = warp / rep;
      const bool attw = warp < rstep * rep;
      float qv[DL], acc[DL];
      float m = -INFINITY, ls = 0.f;
#pragma unroll
      for (int k = 0; k < DL; ++k) {
        acc[k] = 0.f;
        qv[k] = (attw && !ab) ? qs[hw * D + lane * DL + k] * qscale : 0.f;
      }
      auto consume_row = [&](const float* kr, const float* vr) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < DL; ++k) s = fmaf(qv[k], kr[k], s);
        s = warp_sum(s);
        const float mn = fmaxf(m, s);
        const float al = exp2f(m - mn);
        const float pe = exp2f(s - mn);
        ls = ls * al + pe;
#pragma unroll
        for (int k = 0; k < DL; ++k) acc[k] = fmaf(acc[k], al, pe * vr[k]);
        m = mn;
      };
      for (int j = j0; j < jc; j += art) {
        const int nr = min(art, jc - j);
        wait_tile();
        if (!ab) {
          const uint8_t* tb = ring + static_cast<size_t>(rn % a.nslot) * kSlotBytes;
          for (int r = rw; attw && r < nr; r += rstep) {
            float kr[DL], vr[DL];
            if (!a.kv_fp8) {
              const uint8_t* kp = tb + static_cast<size_t>(r) * D * 2 + lane * DL * 2;
              const uint8_t* vp = kp + static_cast<size_t>(nr) * D * 2;
              if (DL == 4) {
                const uint2 kw = *reinterpret_cast<const uint2*>(kp);
                const uint2 vw = *reinterpret_cast<const uint2*>(vp);
                kr[0] = bf16lo(kw.x); kr[1] = bf16hi(kw.x);
                kr[2] = bf16lo(kw.y); kr[3] = bf16hi(kw.y);
                vr[0] = bf16lo(vw.x); vr[1] = bf16hi(vw.x);
                vr[2] = bf16lo(vw.y); vr[3] = bf16hi(vw.y);
              } else {
                const uint32_t kw = *reinterpret_cast<const uint32_t*>(kp);
                const uint32_t vw = *reinterpret_cast<const uint32_t*>(vp);
                kr[0] = bf16lo(kw); kr[1] = bf16hi(kw);
                vr[0] = bf16lo(vw); vr[1] = bf16hi(vw);
              }
            } else {
              const uint8_t* kp = tb + static_cast<size_t>(r) * D + lane * DL;
              const uint8_t* vp = kp + static_cast<size_t>(nr) * D;
              const int sb = ((nr + 3) & ~3) * 4;
              const float ks = reinterpret_cast<const float*>(tb + 2 * nr * D)[r];
              const float vs = reinterpret_cast<const float*>(tb + 2 * nr * D + sb)[r];
#pragma unroll
              for (int k = 0; k < DL; k += 2) {
                const float2 kk = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(kp + k));
                const float2 vv = e4m3x2_to_f2(*reinterpret_cast<const uint16_t*>(vp + k));
                kr[k] = kk.x * ks; kr[k + 1] = kk.y * ks;
                vr[k] = vv.x * vs; vr[k + 1] = vv.y * vs;
              }
            }
            consume_row(kr, vr);
          }
        }
        release_tile();
      }
      if (!ab && has_new && attw && rw == (jc - j0) % rstep) {
        float kr[DL], vr[DL];
#pragma unroll
        for (int k = 0; k < DL; ++k) {
          kr[k] = kn[lane * DL + k];
          vr[k] = vn[lane * DL + k];
        }
        consume_row(kr, vr);
      }
      // -- merge the warps' states, write this chunk's partial
      if (!ab && attw) {
        float* mg = merge + static_cast<size_t>(warp) * (D + 2);
#pragma unroll
        for (int k = 0; k < DL; ++k) mg[lane * DL + k] = acc[k];
        if (lane == 0) {
          mg[D] = m;
          mg[D + 1] = ls;
        }
      }
      csync();
      // -- this chunk's partial state (m in log2 units, l, unnormalised acc).
      // Chunk 0's CTA combines (b, g): it keeps its own partial in shared
      // memory; every other chunk publishes its partial as tagged words and
      // moves on without waiting.
      DEC_STAMP(8 * l + 3);
      const bool combiner = (ci == 0);
      const uint64_t* pbase =
          a.part + (static_cast<size_t>(b) * a.Hq + g * rep) * a.part_chunks * (D + 2);
      if (!ab) {
        for (int t = tid; t < rep * D; t += kCT) {
          const int h = t / D, d = t % D;
          float M = -INFINITY;
          for (int w = h; w < rstep * rep; w += rep) M = fmaxf(M, merge[w * (D + 2) + D]);
          float Ls = 0.f, A = 0.f;
          for (int w = h; w < rstep * rep; w += rep) {
            const float* mg = merge + w * (D + 2);
            const float e = (mg[D] == -INFINITY) ? 0.f : exp2f(mg[D] - M);
            Ls += mg[D + 1] * e;
            A += mg[d] * e;
          }
          if (combiner) {
            ownb[h * (D + 2) + d] = A;
            if (d == 0) {
              ownb[h * (D + 2) + D] = M;
              ownb[h * (D + 2) + D + 1] = Ls;
            }
          } else {
            uint64_t* pp = a.part + ((static_cast<size_t>(b) * a.Hq + g * rep + h) * a.part_chunks +
                                     ci) * (D + 2);
            st_tagged(pp + d, A, f);
            if (d == 0) {
              st_tagged(pp + D, M, f);
              st_tagged(pp + D + 1, Ls, f);
            }
          }
        }
      }
      if (combiner) {  // uniform over the CTA: ci is the item's
        const int nc1 = nchunk[b] - 1;
        const int pc = a.part_chunks;
        // (m, l) of chunks 1..nc1 -> mlb[(c - 1) * rep * 2 + h * 2 + e]
        gather(
            pbase, nc1 * rep * 2, f, mlb,
            [=](int i) {
              const int c = i / (rep * 2) + 1, h = (i >> 1) % rep, e = i & 1;
              return (h * pc + c) * (D + 2) + D + e;
            },
            [](int i) { return i; });
        int fail = 0;
        if (!ab) {
          for (int t = tid; t < rep * D; t += kCT) {
            const int h = t / D, d = t % D;
            const float* own = ownb + h * (D + 2);
            float M = own[D];
            for (int c = 0; c < nc1; ++c) M = fmaxf(M, mlb[(c * rep + h) * 2]);
            const float e0 = exp2f(own[D] - M);
            float Ls = own[D + 1] * e0, A = own[d] * e0;
            const uint64_t* ph = pbase + static_cast<size_t>(h) * pc * (D + 2) + d;
            for (int c0 = 0; c0 < nc1 && !fail; c0 += 8) {
              uint64_t wv[8];
#pragma unroll
              for (int k = 0; k < 8; ++k)
                if (c0 + k < nc1) wv[k] = ld_tagged(ph + static_cast<size_t>(c0 + k + 1) * (D + 2));
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                if (c0 + k < nc1 && !fail) {
                  Spin sp;
                  while (static_cast<uint32_t>(wv[k] >> 32) != f) {
                    if (sp.tick(a, true)) {
                      fail = 1;
                      break;
                    }
                    wv[k] = ld_tagged(ph + static_cast<size_t>(c0 + k + 1) * (D + 2));
                  }
                  const float* ml = mlb + ((c0 + k) * rep + h) * 2;
                  const float e = exp2f(ml[0] - M);
                  Ls += ml[1] * e;
                  A += __uint_as_float(static_cast<uint32_t>(wv[k])) * e;
                }
              }
            }
            if (!fail)
              st_tagged(a.x_o + static_cast<size_t>(b) * HqD + (g * rep + h) * D + d, A / Ls, f);
          }
        }
        ab = named_sync_or(1, kCT, fail | ab);
      }
      csync();
    }
  }

  // ------------------------------------------------------------- one step
  __device__ void consumer() {
    const int H = a.H, F = a.F, HqD = a.Hq * D;
    int best_i[B];
    float best_v[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      best_v[b] = -INFINITY;
      best_i[b] = 0x7fffffff;
    }
    DEC_STAMP(8 * a.L + 3);
    for (int l = 0; l < a.L; ++l) {
      const LayerPtrs& lw = a.layers[l];
      const uint32_t f = flag(l);
      DEC_STAMP(8 * l);
      // ---------------- input RMSNorm + QKV
      if (l == 0) {
        for (int i = tid; i < a.B * H; i += kCT) {
          const int b = i / H, k = i % H;
          act[b * kmax + k] = bf16_to_f(a.embed[static_cast<size_t>(tok[b]) * H + k]);
        }
        csync();
        for (int i = tid; i < (h1 - h0) * a.B; i += kCT) {
          const int r = i / a.B, b = i % a.B;
          xown[r * B + b] = act[b * kmax + h0 + r];
          if (a.hidden_out) a.hidden_out[static_cast<size_t>(b) * H + h0 + r] = xown[r * B + b];
        }
      } else {
        gather_x(a.x_out, H, flag(l - 1));
      }
      rmsnorm_act(H, lw.w[0]);
      {
        uint64_t* dst = a.x_qkv;
        const int nq = nqkv, base = q0;
        gemv<4>(H, q1 - q0, rpt_h, false, [=](int r, int b, float s, float) {
          st_tagged(dst + static_cast<size_t>(b) * nq + base + r, s, f);
        });
      }
      DEC_STAMP(8 * l + 1);
      // ---------------- attention
      attention(l);
      DEC_STAMP(8 * l + 4);
      // ---------------- o_proj + residual
      gather_x(a.x_o, HqD, f);
      {
        float* xo = xown;
        uint64_t* dst = a.x_mid;
        const int base = h0;
        const bool stall = (l == 0 && a.stall_cta == cta);
        gemv<1>(HqD, h1 - h0, rpt_o, false, [=](int r, int b, float s, float) {
          const float x = xo[r * B + b] + s;
          xo[r * B + b] = x;
          if (!stall) st_tagged(dst + static_cast<size_t>(b) * H + base + r, x, f);
        });
      }
      DEC_STAMP(8 * l + 5);
      // ---------------- post-attention RMSNorm + gate/up + SiLU * up
      gather_x(a.x_mid, H, f);
      rmsnorm_act(H, lw.w[7]);
      {
        uint64_t* dst = a.x_u;
        const int base = f0;
        gemv<4>(H, f1 - f0, rpt_u, true, [=](int r, int b, float gs, float us) {
          const float u = gs / (1.0f + __expf(-gs)) * us;
          st_tagged(dst + static_cast<size_t>(b) * F + base + r, u, f);
        });
      }
      DEC_STAMP(8 * l + 6);
      // ---------------- down + residual
      gather_x(a.x_u, F, f);
      {
        float* xo = xown;
        uint64_t* dst = a.x_out;
        const int base = h0;
        float* hid = a.hidden_out ? a.hidden_out + static_cast<size_t>(l + 1) * a.B * H : nullptr;
        gemv<1>(F, h1 - h0, rpt_d, false, [=](int r, int b, float s, float) {
          const float x = xo[r * B + b] + s;
          xo[r * B + b] = x;
          st_tagged(dst + static_cast<size_t>(b) * H + base + r, x, f);
          if (hid) hid[static_cast<size_t>(b) * H + base + r] = x;
        });
      }
      DEC_STAMP(8 * l + 7);
    }
    DEC_STAMP(8 * a.L);
    // ---------------- final norm + lm_head + argmax
    gather_x(a.x_out, H, flag(a.L - 1));
    rmsnorm_act(H, a.final_norm);
    {
      float* lg = a.out_logits;
      const int base = v0, V = a.V;
      gemv<4>(H, v1 - v0, rpt_h, false, [&](int r, int b, float s, float) {
        const int id = base + r;
        if (lg) lg[static_cast<size_t>(b) * V + id] = s;
#pragma unroll
        for (int bb = 0; bb < B; ++bb) {
          if (bb == b && (s > best_v[bb] || (s == best_v[bb] && id < best_i[bb]))) {
            best_v[bb] = s;
            best_i[bb] = id;
          }
        }
      });
    }
    DEC_STAMP(8 * a.L + 1);
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
    DEC_STAMP(8 * a.L + 2);
  }

  // B rows of K tagged words (row stride K) -> act rows (row stride kmax)
  __device__ void gather_x(const uint64_t* src, int K, uint32_t f) {
    const int km = kmax;
    gather(src, a.B * K, f, act, [](int i) { return i; },
           [K, km](int i) { return (i / K) * km + (i % K); });
  }
};

template <int B, int D>
__global__ void __launch_bounds__(kStepThreads, 1) step_kernel(const StepArgs a, int kmax, int rmax) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Cta<B, D> c(a, smem, kmax, rmax);
  // ---- set-up: barriers, step inputs, validation
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.nslot; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], kCW);
    }
    fence_mbar_init();
    int bad = 0;
    for (int b = 0; b < a.B; ++b) {
      const int p = a.positions[b], t = a.token_ids[b];
      c.sints[8 + b] = p;
      c.sints[16 + b] = t;
      if (p < 0 || p >= a.max_ctx) bad |= kDevBadPos;
      if (t < 0 || t >= a.V) bad |= kDevBadTok;
    }
    c.sints[1] = bad;
    c.sints[2] = static_cast<int>(ld_relaxed_u32(a.seq));
    if (bad && blockIdx.x == 0) atomicOr(a.status, bad);
  }
  __syncthreads();
  const int bad = c.sints[1];
  c.seq = static_cast<uint32_t>(c.sints[2]);
  if (!bad) c.plan_attention();
  __syncthreads();
  if (!bad) {
    if (c.warp == kCW) c.producer();
    else c.consumer();
  }
  __syncthreads();
  // ---- exit: the last CTA publishes the ids and resets the step state
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(a.exit_cnt, 1u);
    if (old == gridDim.x - 1) {
      __threadfence();
      const int aborted = ld_relaxed_i32(a.abort_flag);
      for (int b = 0; b < a.B; ++b) {
        const unsigned long long key = atomicExch(&a.amax_key[b], 0ull);
        a.out_ids[b] = (bad || aborted || key == 0ull)
                           ? -1
                           : static_cast<int32_t>(~static_cast<uint32_t>(key & 0xffffffffull));
      }
      atomicExch(a.abort_flag, 0);
      atomicExch(a.exit_cnt, 0u);
      atomicAdd(a.seq, 1u);
      __threadfence();
    }
  }
}

template <int B, int D>
cudaError_t launch_bd(const StepArgs& a, int ctas, size_t smem, int kmax, int rmax,
                      cudaStream_t s) {
  auto k = step_kernel<B, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  StepArgs args = a;
  void* params[] = {&args, &kmax, &rmax};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k), dim3(ctas),
                                     dim3(kStepThreads), params, smem, s);
}

}  // namespace

static int kmax_of(int H, int F, int HqD) {
  int k = H > F ? H : F;
  return k > HqD ? k : HqD;
}
static int rmax_of(int H, int F, int HqD) {
  int m = H < F ? H : F;
  m = m < HqD ? m : HqD;
  return kSlotBytes / (2 * m);
}

size_t step_smem_bytes(int nslot, int B, int H, int F, int HqD, int D, int rep, int nchunks) {
  return carve(nslot, B, kmax_of(H, F, HqD), rmax_of(H, F, HqD), D, rep, nchunks).total;
}

int step_max_slots(int B, int H, int F, int HqD, int D, int rep, int nchunks, int smem_optin) {
  int best = 0;
  for (int n = 1; n <= 16; ++n)
    if (step_smem_bytes(n, B, H, F, HqD, D, rep, nchunks) <= static_cast<size_t>(smem_optin))
      best = n;
  return best;
}

cudaError_t launch_step_small(const StepArgs& a, int ctas, size_t smem, cudaStream_t s) {
  const int HqD = a.Hq * a.D;
  const int kmax = kmax_of(a.H, a.F, HqD), rmax = rmax_of(a.H, a.F, HqD);
  if (a.D == 128) {
    switch (a.B) {
      case 1: return launch_bd<1, 128>(a, ctas, smem, kmax, rmax, s);
      case 2: return launch_bd<2, 128>(a, ctas, smem, kmax, rmax, s);
      case 3: return launch_bd<3, 128>(a, ctas, smem, kmax, rmax, s);
      case 4: return launch_bd<4, 128>(a, ctas, smem, kmax, rmax, s);
    }
  } else if (a.D == 64) {
    switch (a.B) {
      case 1: return launch_bd<1, 64>(a, ctas, smem, kmax, rmax, s);
      case 2: return launch_bd<2, 64>(a, ctas, smem, kmax, rmax, s);
      case 3: return launch_bd<3, 64>(a, ctas, smem, kmax, rmax, s);
      case 4: return launch_bd<4, 64>(a, ctas, smem, kmax, rmax, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace dec
