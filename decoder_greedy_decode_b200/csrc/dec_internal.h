// dec_internal.h -- host-side structures shared by the C ABI and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace dec {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kStepThreads = kConsumerThreads + 32;  // + one producer warp
// Ring slot sizes of the persistent step: the large one when at least
// kMinLargeSlots of them fit shared memory (fewer, larger tiles mean fewer
// waits per stage), else the small one.
constexpr int kSlotBytesLarge = 49152;
constexpr int kSlotBytesSmall = 24576;
constexpr int kMinLargeSlots = 3;
constexpr int kMaxBatchSmall = 4;                   // batch handled by the GEMV step kernel
constexpr int kMaxRep = 4;                          // query heads per KV head (step kernel)
constexpr int kMaxVerifyHeads = 8;                  // query heads per KV head of a block the step kernel verifies
constexpr int kVerifyPersistent = 1;  // verification blocks the persistent kernel takes when a batched step exists
constexpr int kLayerPtrs = 11;
constexpr int kMaxBatch = 64;                       // batched step: the N of the tensor-core tiles
constexpr int kProfStampsPerLayer = 32;             // profiling builds: timestamps per layer and CTA

struct LayerPtrs {
  const uint16_t* w[kLayerPtrs];  // dec_layer_weight order (int8 codes for the
                                  // projections of an int8 handle)
};
// fp32 row scales of an int8 handle's projections (norm slots unused).
struct LayerScales {
  const float* s[kLayerPtrs];
};

// Everything one launch of the persistent step kernel reads.
struct StepArgs {
  // shape
  int L, H, Hq, Hkv, D, F, V, B;
  float eps;
  // weights
  const uint16_t* embed;
  const uint16_t* lm_head;
  const uint16_t* final_norm;
  const LayerPtrs* layers;  // device array [L]
  // weight-only int8: projections and lm_head are int8 codes with one fp32
  // scale per output row (the embedding and the norm gains stay bf16)
  int w8;
  const float* lm_scale;        // [V]
  const LayerScales* wscale;    // device array [L]
  int wsc_n;                    // shared-memory scale slots (0 unless w8)
  // KV cache
  uint8_t* kv;          // values (bf16) or codes (fp8)
  float* kv_scales;     // fp8 only
  int kv_batch;         // batch dimension of the cache layout
  int max_ctx;
  int kv_fp8;
  // step inputs / outputs
  const int32_t* token_ids;
  const int32_t* positions;
  int32_t* out_ids;     // [n_steps][B]
  int n_steps;          // greedy steps this launch runs (ids fed back on the device)
  int eos;              // end-of-sequence id, or -1
  int32_t* gen_pos;     // n_steps > 1: the caller's positions, advanced in place; else null
  int vseq;             // >= 0: block verification, every row is a token of cache sequence vseq
  float* out_logits;    // [B, V] or null
  float* hidden_out;    // [L+1, B, H] or null
  // workspace
  uint64_t* x_qkv;      // tagged [B, (Hq+2Hkv)D]
  uint64_t* x_o;        // tagged [B, Hq D]
  uint64_t* x_mid;      // tagged [B, H]   residual after o_proj
  uint64_t* x_u;        // tagged [B, F]
  uint64_t* x_out;      // tagged [B, H]   residual after the MLP
  uint64_t* part;       // tagged attention partials [B, Hq, part_chunks, D + 2]
  int part_chunks;
  unsigned long long* amax_key;  // [B]
  uint64_t* tokw;       // tagged ids of the last finished step [B]
  unsigned* step_cnt;   // CTAs past their argmax, over the launch's steps
  unsigned* exit_cnt;
  unsigned* seq;
  int* status;
  int* abort_flag;
  const float* inv_freq;  // [D/2]
  unsigned long long timeout_ns;
  int stall_cta;        // -1: off
  int nslot;            // ring slots per CTA
  int slot_bytes;       // bytes per ring slot
  int prow;             // most output rows of one CTA in a K-split stage
  unsigned long long* prof;  // per-phase timestamps (profiling builds) or null
};

// Scratch layout inside the library workspace (byte offsets).
struct WorkspaceLayout {
  size_t x_qkv, x_o, x_mid, x_u, x_out, part, amax_key, tokw, step_cnt, exit_cnt, seq, status,
      abort_flag, inv_freq, tok_dev, pos_dev, out_dev, gen_done, prof, total;
  int part_chunks;
};

size_t step_smem_bytes(int nslot, int slot_bytes, int B, int H, int F, int HqD, int D, int rep,
                       int wsc_n, int prow);
// The ring of the persistent step for batch B: slot size and count (0 slots:
// the shape does not fit).
void step_ring(int B, int H, int F, int HqD, int D, int rep, int wsc_n, int prow, int smem_optin,
               int* nslot, int* slot_bytes);
// The most output rows one CTA computes in a K-split stage (gate and up rows
// counted separately).
int step_part_rows(int H, int F, int nqkv, int ctas);
// Dynamic shared-memory limit of the step kernels a handle launches.
cudaError_t step_set_smem(int B, int D, int w8, size_t smem);
// Shared-memory row-scale slots an int8 step needs: the most rows one CTA
// computes in any stage (gate and up rows counted twice).
int step_wsc_slots(int H, int F, int nqkv, int V, int ctas);
cudaError_t launch_quantize_int8(const uint16_t* w, int rows, int cols, int8_t* codes,
                                 float* scales, cudaStream_t s);
cudaError_t launch_quantize_fp8w(const uint16_t* w, int rows, int cols, uint8_t* codes,
                                 float* scales, cudaStream_t s);
cudaError_t launch_step_small(const StepArgs& a, int ctas, size_t smem, cudaStream_t s);

// Isolated split-K decode attention.
struct AttnArgs {
  int B, Hq, Hkv, D, max_len;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* lengths;
  float* out;
  float* part;          // [B, Hq, chunks_max, D + 2]
  unsigned* cnt;        // [B * Hkv]
  int chunk_rows;
  int chunks_max;
  int* status;
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);
size_t attention_smem_bytes(int D, int rep);
int attention_chunk_rows(int B, int Hkv, int max_len, int sms);
cudaError_t launch_quantize(const float* x, int rows, int dim, uint8_t* codes, float* scales,
                            cudaStream_t s);
// dec_generate's between-step bookkeeping (dec_generate.cu)
cudaError_t launch_gen_reset(int* done, int batch, cudaStream_t s);
cudaError_t launch_gen_advance(int32_t* out, int32_t* pos, int* done, int batch, int eos,
                               cudaStream_t s);

// ---- batched step (batch > kMaxBatchSmall): tensor-core projections
struct BtShape {
  int L, H, Hq, Hkv, D, F, V;
  float eps;
};
struct BtPlan;  // tensor maps, launch configuration and scratch (dec_step_batched.cu)
// Returns 0, or a DEC_ERR_* code (DEC_ERR_CUDA with *cerr set).
// 8-bit handles (w8 1: int8, 2: E4M3 codes) pass the lm_head row scales and
// every layer's projection row scales (host array of device pointers); bf16
// handles pass null for both and w8 = 0.
int bt_plan_create(const BtShape& s, const uint16_t* embed, const void* lm_head,
                   const uint16_t* final_norm, const LayerPtrs* layers_host,
                   const float* inv_freq_dev, int sms, BtPlan** out, cudaError_t* cerr,
                   const float* lm_scale, const LayerScales* scales_host, int w8);
void bt_plan_destroy(BtPlan* p);
struct BtIO {
  int B;
  const int32_t* tok;
  const int32_t* pos;
  int32_t* out;
  float* logits;   // [B, V] or null
  float* hidden;   // [L+1, B, H] or null
  uint8_t* kv;
  float* kv_scales;
  int kv_batch, max_ctx, kv_fp8;
  int one_seq;     // -1: row b is cache sequence b; >= 0: every row is that sequence
  const int* retired;  // [B] or null: rows whose new cache row is not written
  int* status;
  unsigned long long timeout_ns;
};
cudaError_t bt_step(BtPlan* p, const BtIO& io, cudaStream_t s);

}  // namespace dec
