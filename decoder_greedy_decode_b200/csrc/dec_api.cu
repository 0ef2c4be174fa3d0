// dec_api.cu -- the C ABI of libdec.so (declared and documented in dec.h):
// argument checking, the workspace, kernel configuration and launches.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <new>
#include <vector>

#include "dec.h"
#include "dec_internal.h"

using namespace dec;

namespace {
int g_last_cuda = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda = static_cast<int>(e);
  return DEC_ERR_CUDA;
}

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

struct dec_handle {
  dec_shape shape;
  int device = 0;
  int sms = 0;
  int ctas = 0;
  int smem_optin = 0;
  int nslot[kMaxBatchSmall + 1] = {0};
  int slot_bytes[kMaxBatchSmall + 1] = {0};
  size_t smem[kMaxBatchSmall + 1] = {0};
  const uint16_t* embed = nullptr;
  const uint16_t* lm_head = nullptr;
  const uint16_t* final_norm = nullptr;
  LayerPtrs* layers_dev = nullptr;
  int w8 = 0;                         // weight-only 8-bit handle: 1 int8, 2 E4M3 codes
  const float* lm_scale = nullptr;    // int8: lm_head row scales
  LayerScales* scales_dev = nullptr;  // int8: projection row scales
  int wsc_n = 0;
  int prow = 0;
  uint8_t* ws = nullptr;
  WorkspaceLayout wl{};
  float* logits_dev = nullptr;
  unsigned long long timeout_ns = 2000000000ull;
  int stall_cta = -1;
  BtPlan* bt = nullptr;  // batched path (max_batch > kMaxBatchSmall)
};

static int check_shape(const dec_shape* s) {
  if (!s) return DEC_ERR_NULL;
  if (s->n_layers < 1 || s->n_layers > 64) return DEC_ERR_SHAPE;
  if (s->hidden < 256 || s->hidden % 256 || s->hidden > 6144) return DEC_ERR_SHAPE;
  if (s->ffn < 256 || s->ffn % 256 || s->ffn > 6144) return DEC_ERR_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return DEC_ERR_SHAPE;
  if (s->n_kv_heads < 1 || s->n_q_heads < s->n_kv_heads || s->n_q_heads % s->n_kv_heads)
    return DEC_ERR_SHAPE;
  if (s->n_q_heads / s->n_kv_heads > kMaxRep) return DEC_ERR_SHAPE;
  const int hqd = s->n_q_heads * s->head_dim;
  if (hqd % 256 || hqd > 6144) return DEC_ERR_SHAPE;
  if (s->vocab < 1) return DEC_ERR_SHAPE;
  if (!(s->rms_eps >= 0.f) || !(s->rope_theta > 0.f)) return DEC_ERR_SHAPE;
  if (s->max_batch < 1 || s->max_batch > kMaxBatch) return DEC_ERR_BATCH;
  return DEC_OK;
}

namespace {
// The weights either entry point passes on (checked by the caller).
struct InitWeights {
  const void* embed;
  const void* lm_head;
  const void* final_norm;
  const void* const* layers;
  int w8;
  const float* lm_scale;
  const float* const* scales;
};
bool is_projection(int j) {
  return j == DEC_LW_Q || j == DEC_LW_K || j == DEC_LW_V || j == DEC_LW_O || j == DEC_LW_GATE ||
         j == DEC_LW_UP || j == DEC_LW_DOWN;
}
}  // namespace

static int init_handle(const dec_shape* shape, const InitWeights& w, dec_handle** out);

extern "C" int dec_init(const dec_shape* shape, const dec_weights* w, dec_handle** out) {
  if (!shape || !w || !out) return DEC_ERR_NULL;
  *out = nullptr;
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!w->embed || !w->lm_head || !w->final_norm || !w->layers) return DEC_ERR_NULL;
  if (!aligned(w->embed, 16) || !aligned(w->lm_head, 16) || !aligned(w->final_norm, 16))
    return DEC_ERR_ALIGN;
  const int L = shape->n_layers;
  for (int i = 0; i < L * DEC_LW_COUNT; ++i) {
    if (!w->layers[i]) return DEC_ERR_NULL;
    if (!aligned(w->layers[i], 16)) return DEC_ERR_ALIGN;
  }
  const InitWeights iw{w->embed, w->lm_head, w->final_norm, w->layers, 0, nullptr, nullptr};
  return init_handle(shape, iw, out);
}

static int init_8bit(const dec_shape* shape, const dec_weights_int8* w, int fmt,
                     dec_handle** out);

extern "C" int dec_init_int8(const dec_shape* shape, const dec_weights_int8* w,
                             dec_handle** out) {
  return init_8bit(shape, w, 1, out);
}

extern "C" int dec_init_fp8w(const dec_shape* shape, const dec_weights_int8* w,
                             dec_handle** out) {
  return init_8bit(shape, w, 2, out);
}

// fmt 1: int8 codes, 2: E4M3 codes (both with fp32 row scales)
static int init_8bit(const dec_shape* shape, const dec_weights_int8* w, int fmt,
                     dec_handle** out) {
  if (!shape || !w || !out) return DEC_ERR_NULL;
  *out = nullptr;
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!w->embed || !w->lm_head || !w->lm_head_scale || !w->final_norm || !w->layers ||
      !w->scales)
    return DEC_ERR_NULL;
  if (!aligned(w->embed, 16) || !aligned(w->lm_head, 16) || !aligned(w->final_norm, 16) ||
      !aligned(w->lm_head_scale, 4))
    return DEC_ERR_ALIGN;
  const int L = shape->n_layers;
  for (int i = 0; i < L * DEC_LW_COUNT; ++i) {
    if (!w->layers[i]) return DEC_ERR_NULL;
    if (!aligned(w->layers[i], 16)) return DEC_ERR_ALIGN;
    if (is_projection(i % DEC_LW_COUNT)) {
      if (!w->scales[i]) return DEC_ERR_NULL;
      if (!aligned(w->scales[i], 4)) return DEC_ERR_ALIGN;
    }
  }
  const InitWeights iw{w->embed, w->lm_head, w->final_norm, w->layers,
                       fmt, w->lm_head_scale, w->scales};
  return init_handle(shape, iw, out);
}

static int do_step(dec_handle* h, int batch, const int32_t* tok, const int32_t* pos,
                   const dec_kv* kv, int32_t* out_ids, float* logits, float* hidden,
                   cudaStream_t stream, int n_steps = 1, int eos = -1,
                   int32_t* gen_pos = nullptr, const int* retired = nullptr, int vseq = -1);

// The persistent step's time depends by a few per cent on where its
// workspace (above all the tagged exchange words, which every CTA polls)
// lands in device memory, and a placement keeps its time.  So a handle sets
// up kWsCandidates workspaces, times a few batch-1 steps on each over a
// small scratch cache (zero rows, token 0, position 0), keeps the fastest
// and frees the others.  h is bound to its first (filled) workspace on
// entry; on any failure the first one stays.
constexpr int kWsCandidates = 6;
template <class Fill, class Bind>
static cudaError_t pick_workspace(dec_handle* h, Fill&& fill, Bind&& bind) {
  uint8_t* cand[kWsCandidates] = {h->ws};
  float ms[kWsCandidates];
  void* scratch = nullptr;
  cudaStream_t st = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  const size_t kvb = dec_kv_bytes(h, 1, 16, DEC_KV_BF16);
  cudaError_t e = cudaMalloc(&scratch, kvb + 256);
  if (e == cudaSuccess) e = cudaMemset(scratch, 0, kvb + 256);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreate(&e0);
  if (e == cudaSuccess) e = cudaEventCreate(&e1);
  int n = 0;
  bool ok = e == cudaSuccess;
  for (int c = 0; ok && c < kWsCandidates; ++c) {
    if (c > 0) {
      ok = cudaMalloc(&cand[c], h->wl.total) == cudaSuccess;
      if (!ok) cand[c] = nullptr;
      ok = ok && fill(cand[c]) == cudaSuccess;
      if (!ok) break;
    }
    bind(cand[c]);
    n = c + 1;
    int32_t* io = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + kvb);  // tok, pos, out
    const dec_kv kv{scratch, kvb, 1, 16, DEC_KV_BF16};
    for (int i = 0; ok && i < 6; ++i) {  // 2 untimed, 4 timed steps
      if (i == 2) ok = cudaEventRecord(e0, st) == cudaSuccess;
      ok = ok && do_step(h, 1, io, io + 1, &kv, io + 2, nullptr, nullptr, st) == DEC_OK;
    }
    ok = ok && cudaEventRecord(e1, st) == cudaSuccess && cudaStreamSynchronize(st) == cudaSuccess;
    int status = 1;
    ok = ok && cudaMemcpy(&status, cand[c] + h->wl.status, sizeof(int),
                          cudaMemcpyDeviceToHost) == cudaSuccess && status == 0;
    ok = ok && cudaEventElapsedTime(&ms[c], e0, e1) == cudaSuccess;
  }
  int best = 0;
  if (ok) {
    for (int c = 1; c < n; ++c)
      if (ms[c] < ms[best]) best = c;
  } else {
    e = fill(cand[0]);  // a calibration step failed: keep the first, as new
  }
  bind(cand[best]);
  for (int c = 0; c < kWsCandidates; ++c)
    if (c != best && cand[c]) cudaFree(cand[c]);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (st) cudaStreamDestroy(st);
  cudaFree(scratch);
  return e;
}

static int init_handle(const dec_shape* shape, const InitWeights& w, dec_handle** out) {
  int rc = DEC_OK;
  const int L = shape->n_layers;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prop.major != 10) return DEC_ERR_DEVICE;
  if (!prop.cooperativeLaunch) return DEC_ERR_DEVICE;

  dec_handle* h = new (std::nothrow) dec_handle();
  if (!h) return DEC_ERR_ARG;
  h->shape = *shape;
  h->device = dev;
  h->sms = prop.multiProcessorCount;
  h->ctas = prop.multiProcessorCount;
  h->smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
  const int H = shape->hidden, F = shape->ffn, D = shape->head_dim;
  const int Hq = shape->n_q_heads, Hkv = shape->n_kv_heads;
  // the persistent kernel serves batches up to kMaxBatchSmall; larger ones
  // take the batched (tensor-core) path
  const int B = shape->max_batch < kMaxBatchSmall ? shape->max_batch : kMaxBatchSmall;
  const int Bfull = shape->max_batch;
  const int HqD = Hq * D, rep = Hq / Hkv;
  if ((H + h->ctas - 1) / h->ctas > 64) {
    delete h;
    return DEC_ERR_SHAPE;
  }
  const int nchunks = h->ctas + 1;
  const int nqkv = (Hq + 2 * Hkv) * D;
  h->w8 = w.w8;
  h->lm_scale = w.lm_scale;
  h->wsc_n = w.w8 ? step_wsc_slots(H, F, nqkv, shape->vocab, h->ctas) : 0;
  h->prow = step_part_rows(H, F, nqkv, h->ctas);
  for (int b = 1; b <= B; ++b) {
    step_ring(b, H, F, HqD, D, rep, h->wsc_n, h->prow, h->smem_optin, &h->nslot[b],
              &h->slot_bytes[b]);
    if (h->nslot[b] < 2) {
      delete h;
      return DEC_ERR_DEVICE;
    }
    h->smem[b] = step_smem_bytes(h->nslot[b], h->slot_bytes[b], b, H, F, HqD, D, rep, h->wsc_n,
                                 h->prow);
    e = step_set_smem(b, D, w.w8, h->smem[b]);
    if (e != cudaSuccess) {
      delete h;
      return cuda_fail(e);
    }
  }
  h->embed = static_cast<const uint16_t*>(w.embed);
  h->lm_head = static_cast<const uint16_t*>(w.lm_head);
  h->final_norm = static_cast<const uint16_t*>(w.final_norm);

  // ---- workspace
  WorkspaceLayout& wl = h->wl;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += al256(bytes);
    return at;
  };
  wl.part_chunks = nchunks;
  wl.x_qkv = take(sizeof(uint64_t) * B * nqkv);
  wl.x_o = take(sizeof(uint64_t) * B * HqD);
  wl.x_mid = take(sizeof(uint64_t) * B * H);
  wl.x_u = take(sizeof(uint64_t) * B * F);
  wl.x_out = take(sizeof(uint64_t) * B * H);
  wl.part = take(sizeof(uint64_t) * B * Hq * wl.part_chunks * (D + 2));
  wl.amax_key = take(sizeof(unsigned long long) * B);
  wl.tokw = take(sizeof(uint64_t) * B);
  wl.step_cnt = take(sizeof(unsigned));
  wl.exit_cnt = take(sizeof(unsigned));
  wl.seq = take(sizeof(unsigned));
  wl.status = take(sizeof(int));
  wl.abort_flag = take(sizeof(int));
  wl.inv_freq = take(sizeof(float) * D / 2);
  wl.tok_dev = take(sizeof(int32_t) * Bfull);
  wl.pos_dev = take(sizeof(int32_t) * Bfull);
  wl.out_dev = take(sizeof(int32_t) * Bfull);
  wl.gen_done = take(sizeof(int) * Bfull);
#ifdef DEC_PROFILE
  wl.prof = take(sizeof(unsigned long long) * h->ctas * (kProfStampsPerLayer * L + 8));
#endif
  size_t layers_off = take(sizeof(LayerPtrs) * L);
  size_t scales_off = w.w8 ? take(sizeof(LayerScales) * L) : 0;
  size_t logits_off = take(sizeof(float) * static_cast<size_t>(Bfull) * shape->vocab);
  wl.total = o;
  // host copies of the tables every workspace holds
  std::vector<float> inv(D / 2);  // rotary inverse frequencies theta^(-2i/D), rounded once to fp32
  for (int i = 0; i < D / 2; ++i)
    inv[i] = static_cast<float>(1.0 / pow(static_cast<double>(shape->rope_theta),
                                          (2.0 * i) / static_cast<double>(D)));
  std::vector<LayerPtrs> lp(L);
  for (int l = 0; l < L; ++l)
    for (int j = 0; j < DEC_LW_COUNT; ++j)
      lp[l].w[j] = static_cast<const uint16_t*>(w.layers[l * DEC_LW_COUNT + j]);
  std::vector<LayerScales> ls;
  if (w.w8) {
    ls.resize(L);
    for (int l = 0; l < L; ++l)
      for (int j = 0; j < DEC_LW_COUNT; ++j)
        ls[l].s[j] = is_projection(j) ? w.scales[l * DEC_LW_COUNT + j] : nullptr;
  }
  auto fill = [&](uint8_t* ws) {
    cudaError_t r = cudaMemset(ws, 0, wl.total);
    if (r == cudaSuccess)
      r = cudaMemcpy(ws + wl.inv_freq, inv.data(), sizeof(float) * inv.size(),
                     cudaMemcpyHostToDevice);
    if (r == cudaSuccess)
      r = cudaMemcpy(ws + layers_off, lp.data(), sizeof(LayerPtrs) * L, cudaMemcpyHostToDevice);
    if (r == cudaSuccess && w.w8)
      r = cudaMemcpy(ws + scales_off, ls.data(), sizeof(LayerScales) * L, cudaMemcpyHostToDevice);
    return r;
  };
  auto bind = [&](uint8_t* ws) {
    h->ws = ws;
    h->layers_dev = reinterpret_cast<LayerPtrs*>(ws + layers_off);
    h->scales_dev = w.w8 ? reinterpret_cast<LayerScales*>(ws + scales_off) : nullptr;
    h->logits_dev = reinterpret_cast<float*>(ws + logits_off);
  };
  uint8_t* ws0 = nullptr;
  e = cudaMalloc(&ws0, wl.total);
  if (e != cudaSuccess) {
    delete h;
    return cuda_fail(e);
  }
  e = fill(ws0);
  if (e == cudaSuccess) {
    bind(ws0);
    e = pick_workspace(h, fill, bind);
  }
  if (e != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return cuda_fail(e);
  }
  if (Bfull > kMaxBatchSmall) {
    const BtShape bs{L, H, Hq, Hkv, D, F, shape->vocab, shape->rms_eps};
    cudaError_t ce = cudaSuccess;
    rc = bt_plan_create(bs, h->embed, h->lm_head, h->final_norm, lp.data(),
                        reinterpret_cast<const float*>(h->ws + wl.inv_freq), h->sms, &h->bt, &ce,
                        w.w8 ? static_cast<const float*>(w.lm_scale) : nullptr,
                        w.w8 ? ls.data() : nullptr, w.w8);
    if (rc) {
      cudaFree(h->ws);
      delete h;
      if (rc == DEC_ERR_CUDA) g_last_cuda = static_cast<int>(ce);
      return rc;
    }
  }
  *out = h;
  return DEC_OK;
}

extern "C" void dec_free(dec_handle* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  bt_plan_destroy(h->bt);
  cudaFree(h->ws);
  delete h;
}

static size_t kv_code_bytes(const dec_shape& s, int batch, int max_ctx, int elt) {
  return static_cast<size_t>(s.n_layers) * 2 * batch * s.n_kv_heads * max_ctx * s.head_dim * elt;
}

extern "C" size_t dec_kv_scale_offset(const dec_handle* h, int batch, int max_ctx, int dtype) {
  if (!h || batch < 1 || max_ctx < 16 || dtype != DEC_KV_FP8_E4M3) return 0;
  return al256(kv_code_bytes(h->shape, batch, max_ctx, 1));
}

extern "C" size_t dec_kv_bytes(const dec_handle* h, int batch, int max_ctx, int dtype) {
  if (!h || batch < 1 || max_ctx < 16 || max_ctx % 16) return 0;
  if (dtype == DEC_KV_BF16) return kv_code_bytes(h->shape, batch, max_ctx, 2);
  if (dtype == DEC_KV_FP8_E4M3)
    return al256(kv_code_bytes(h->shape, batch, max_ctx, 1)) +
           static_cast<size_t>(h->shape.n_layers) * 2 * batch * h->shape.n_kv_heads * max_ctx *
               sizeof(float);
  return 0;
}

extern "C" int dec_kv_alloc(dec_handle* h, int batch, int max_ctx, int dtype, void* buf,
                            size_t buf_bytes, dec_kv* out) {
  if (!h || !buf || !out) return DEC_ERR_NULL;
  if (dtype != DEC_KV_BF16 && dtype != DEC_KV_FP8_E4M3) return DEC_ERR_DTYPE;
  if (batch < 1) return DEC_ERR_BATCH;
  if (max_ctx < 16 || max_ctx % 16) return DEC_ERR_ARG;
  if (!aligned(buf, 256)) return DEC_ERR_ALIGN;
  const size_t need = dec_kv_bytes(h, batch, max_ctx, dtype);
  if (need == 0) return DEC_ERR_ARG;
  if (buf_bytes < need) return DEC_ERR_KV_SIZE;
  out->base = buf;
  out->bytes = buf_bytes;
  out->batch = batch;
  out->max_ctx = max_ctx;
  out->dtype = dtype;
  return DEC_OK;
}

// n_steps > 1 (batch <= kMaxBatchSmall only): the persistent kernel runs the
// steps itself, feeding the ids back and advancing gen_pos (== pos) in place.
static int do_step(dec_handle* h, int batch, const int32_t* tok, const int32_t* pos,
                   const dec_kv* kv, int32_t* out_ids, float* logits, float* hidden,
                   cudaStream_t stream, int n_steps, int eos, int32_t* gen_pos,
                   const int* retired, int vseq) {
  if (!h || !kv || !tok || !pos || !out_ids || !kv->base) return DEC_ERR_NULL;
  if (batch < 1 || batch > h->shape.max_batch || (vseq < 0 && batch > kv->batch))
    return DEC_ERR_BATCH;
  if (kv->dtype != DEC_KV_BF16 && kv->dtype != DEC_KV_FP8_E4M3) return DEC_ERR_DTYPE;
  if (kv->bytes < dec_kv_bytes(h, kv->batch, kv->max_ctx, kv->dtype)) return DEC_ERR_KV_SIZE;
  const dec_shape& s = h->shape;
  if (batch > kMaxBatchSmall) {
    BtIO io{};
    io.B = batch;
    io.tok = tok;
    io.pos = pos;
    io.out = out_ids;
    io.logits = logits;
    io.hidden = hidden;
    io.kv = static_cast<uint8_t*>(kv->base);
    io.kv_fp8 = kv->dtype == DEC_KV_FP8_E4M3;
    io.kv_scales = io.kv_fp8 ? reinterpret_cast<float*>(
                                   static_cast<uint8_t*>(kv->base) +
                                   dec_kv_scale_offset(h, kv->batch, kv->max_ctx, kv->dtype))
                             : nullptr;
    io.kv_batch = kv->batch;
    io.max_ctx = kv->max_ctx;
    io.one_seq = -1;
    io.retired = retired;
    io.status = reinterpret_cast<int*>(h->ws + h->wl.status);
    io.timeout_ns = h->timeout_ns;
    cudaError_t e = bt_step(h->bt, io, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    return DEC_OK;
  }
  StepArgs a{};
  a.L = s.n_layers;
  a.H = s.hidden;
  a.Hq = s.n_q_heads;
  a.Hkv = s.n_kv_heads;
  a.D = s.head_dim;
  a.F = s.ffn;
  a.V = s.vocab;
  a.B = batch;
  a.eps = s.rms_eps;
  a.embed = h->embed;
  a.lm_head = h->lm_head;
  a.final_norm = h->final_norm;
  a.layers = h->layers_dev;
  a.w8 = h->w8;
  a.lm_scale = h->lm_scale;
  a.wscale = h->scales_dev;
  a.wsc_n = h->wsc_n;
  a.kv = static_cast<uint8_t*>(kv->base);
  a.kv_fp8 = kv->dtype == DEC_KV_FP8_E4M3;
  a.kv_scales = a.kv_fp8 ? reinterpret_cast<float*>(static_cast<uint8_t*>(kv->base) +
                                                    dec_kv_scale_offset(h, kv->batch, kv->max_ctx,
                                                                        kv->dtype))
                         : nullptr;
  a.kv_batch = kv->batch;
  a.max_ctx = kv->max_ctx;
  a.token_ids = tok;
  a.positions = pos;
  a.out_ids = out_ids;
  a.n_steps = n_steps;
  a.eos = eos;
  a.gen_pos = gen_pos;
  a.vseq = vseq;
  a.out_logits = logits;
  a.hidden_out = hidden;
  const WorkspaceLayout& wl = h->wl;
  a.x_qkv = reinterpret_cast<uint64_t*>(h->ws + wl.x_qkv);
  a.x_o = reinterpret_cast<uint64_t*>(h->ws + wl.x_o);
  a.x_mid = reinterpret_cast<uint64_t*>(h->ws + wl.x_mid);
  a.x_u = reinterpret_cast<uint64_t*>(h->ws + wl.x_u);
  a.x_out = reinterpret_cast<uint64_t*>(h->ws + wl.x_out);
  a.part = reinterpret_cast<uint64_t*>(h->ws + wl.part);
  a.part_chunks = wl.part_chunks;
  a.amax_key = reinterpret_cast<unsigned long long*>(h->ws + wl.amax_key);
  a.tokw = reinterpret_cast<uint64_t*>(h->ws + wl.tokw);
  a.step_cnt = reinterpret_cast<unsigned*>(h->ws + wl.step_cnt);
  a.exit_cnt = reinterpret_cast<unsigned*>(h->ws + wl.exit_cnt);
  a.seq = reinterpret_cast<unsigned*>(h->ws + wl.seq);
  a.status = reinterpret_cast<int*>(h->ws + wl.status);
  a.abort_flag = reinterpret_cast<int*>(h->ws + wl.abort_flag);
  a.inv_freq = reinterpret_cast<const float*>(h->ws + wl.inv_freq);
  a.timeout_ns = h->timeout_ns;
  a.stall_cta = h->stall_cta;
  a.nslot = h->nslot[batch];
  a.slot_bytes = h->slot_bytes[batch];
  a.prow = h->prow;
#ifdef DEC_PROFILE
  a.prof = reinterpret_cast<unsigned long long*>(h->ws + wl.prof);
#else
  a.prof = nullptr;
#endif
  cudaError_t e = launch_step_small(a, h->ctas, h->smem[batch], stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_step(dec_handle* h, int batch, const int32_t* token_ids,
                        const int32_t* positions, const dec_kv* kv, int32_t* out_ids,
                        float* out_logits, void* stream) {
  return do_step(h, batch, token_ids, positions, kv, out_ids, out_logits, nullptr,
                 static_cast<cudaStream_t>(stream));
}

extern "C" int dec_step_debug(dec_handle* h, int batch, const int32_t* token_ids,
                              const int32_t* positions, const dec_kv* kv, int32_t* out_ids,
                              float* out_logits, float* hidden_out, void* stream) {
  if (!hidden_out) return DEC_ERR_NULL;
  return do_step(h, batch, token_ids, positions, kv, out_ids, out_logits, hidden_out,
                 static_cast<cudaStream_t>(stream));
}

extern "C" int dec_step_host(dec_handle* h, int batch, const int32_t* tok_host,
                             const int32_t* pos_host, const dec_kv* kv, int32_t* out_host,
                             float* logits_host, void* stream) {
  if (!h || !tok_host || !pos_host || !out_host) return DEC_ERR_NULL;
  if (batch < 1 || batch > h->shape.max_batch) return DEC_ERR_BATCH;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* tok = reinterpret_cast<int32_t*>(h->ws + h->wl.tok_dev);
  int32_t* pos = reinterpret_cast<int32_t*>(h->ws + h->wl.pos_dev);
  int32_t* out = reinterpret_cast<int32_t*>(h->ws + h->wl.out_dev);
  cudaError_t e = cudaMemcpyAsync(tok, tok_host, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(pos, pos_host, sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e);
  int rc = do_step(h, batch, tok, pos, kv, out, logits_host ? h->logits_dev : nullptr, nullptr, st);
  if (rc) return rc;
  e = cudaMemcpyAsync(out_host, out, sizeof(int32_t) * batch, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && logits_host)
    e = cudaMemcpyAsync(logits_host, h->logits_dev,
                        sizeof(float) * static_cast<size_t>(batch) * h->shape.vocab,
                        cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_verify(dec_handle* h, int k, const int32_t* token_ids,
                          const int32_t* positions, int seq, const dec_kv* kv, int32_t* out_ids,
                          float* out_logits, void* stream) {
  if (!h || !kv || !token_ids || !positions || !out_ids || !kv->base) return DEC_ERR_NULL;
  if (k < 1 || k > h->shape.max_batch) return DEC_ERR_BATCH;
  if (seq < 0 || seq >= kv->batch) return DEC_ERR_ARG;
  if (kv->dtype != DEC_KV_BF16 && kv->dtype != DEC_KV_FP8_E4M3) return DEC_ERR_DTYPE;
  if (kv->bytes < dec_kv_bytes(h, kv->batch, kv->max_ctx, kv->dtype)) return DEC_ERR_KV_SIZE;
  const int rep = h->shape.n_q_heads / h->shape.n_kv_heads;
  // The persistent kernel (one launch, the prefix read once for the block)
  // takes blocks of up to kVerifyPersistent tokens, and blocks up to
  // kMaxBatchSmall when the handle has no batched step; from 2 tokens on the
  // batched step is as fast or faster (0.6B shape, context 795: 1.25-1.27 ms
  // per call for 2-4 tokens, against 1.2-1.4 / 1.5 / 1.9 ms).
  const bool small = k <= kMaxBatchSmall && k * rep <= kMaxVerifyHeads;
  if (small && (k <= kVerifyPersistent || !h->bt))
    return do_step(h, k, token_ids, positions, kv, out_ids, out_logits, nullptr,
                   static_cast<cudaStream_t>(stream), 1, -1, nullptr, nullptr, seq);
  if (!h->bt) return DEC_ERR_BATCH;  // larger blocks need the batched step (max_batch > 4)
  BtIO io{};
  io.B = k;
  io.tok = token_ids;
  io.pos = positions;
  io.out = out_ids;
  io.logits = out_logits;
  io.hidden = nullptr;
  io.kv = static_cast<uint8_t*>(kv->base);
  io.kv_fp8 = kv->dtype == DEC_KV_FP8_E4M3;
  io.kv_scales = io.kv_fp8 ? reinterpret_cast<float*>(
                                 static_cast<uint8_t*>(kv->base) +
                                 dec_kv_scale_offset(h, kv->batch, kv->max_ctx, kv->dtype))
                           : nullptr;
  io.kv_batch = kv->batch;
  io.max_ctx = kv->max_ctx;
  io.one_seq = seq;
  io.status = reinterpret_cast<int*>(h->ws + h->wl.status);
  io.timeout_ns = h->timeout_ns;
  cudaError_t e = bt_step(h->bt, io, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_accept_greedy(int k, const int32_t* tokens, const int32_t* out_ids,
                                 int32_t* emitted, int* n_emitted) {
  if (!tokens || !out_ids || !emitted || !n_emitted) return DEC_ERR_NULL;
  if (k < 1) return DEC_ERR_ARG;
  for (int i = 0; i < k; ++i)
    if (out_ids[i] < 0) return DEC_ERR_ARG;  // the verify step was invalid
  // draft token tokens[i + 1] is checked against the prediction made at the
  // position before it, out_ids[i]; the first mismatch ends the accepted run
  int j = 0;
  while (j < k - 1 && tokens[j + 1] == out_ids[j]) ++j;
  for (int i = 0; i < j; ++i) emitted[i] = tokens[i + 1];
  emitted[j] = out_ids[j];  // the correction, or the bonus token after a full match
  *n_emitted = j + 1;
  return DEC_OK;
}

extern "C" int dec_generate(dec_handle* h, int batch, int n_steps, const int32_t* token_ids,
                            int32_t* positions, const dec_kv* kv, int32_t* out_ids, int eos,
                            void* stream) {
  if (!h || !kv || !token_ids || !positions || !out_ids) return DEC_ERR_NULL;
  if (batch < 1 || batch > h->shape.max_batch || batch > 64) return DEC_ERR_BATCH;
  if (n_steps < 1 || eos < -1 || eos >= h->shape.vocab) return DEC_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (batch <= kMaxBatchSmall)  // one launch: the persistent kernel loops over the steps
    return do_step(h, batch, token_ids, positions, kv, out_ids, nullptr, nullptr, st, n_steps,
                   eos, positions);
  // the batched step: one step per launch, a small kernel in between feeds
  // the ids back, advances the positions and retires sequences at eos
  int* done = reinterpret_cast<int*>(h->ws + h->wl.gen_done);
  cudaError_t e = launch_gen_reset(done, batch, st);
  if (e != cudaSuccess) return cuda_fail(e);
  for (int i = 0; i < n_steps; ++i) {
    const int32_t* tok = i == 0 ? token_ids : out_ids + static_cast<size_t>(i - 1) * batch;
    int32_t* out = out_ids + static_cast<size_t>(i) * batch;
    const int rc = do_step(h, batch, tok, positions, kv, out, nullptr, nullptr, st, 1, -1,
                           nullptr, done);
    if (rc) return rc;
    e = launch_gen_advance(out, positions, done, batch, eos, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return DEC_OK;
}

extern "C" int dec_check(dec_handle* h, void* stream) {
  if (!h) return DEC_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpy(&v, h->ws + h->wl.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->ws + h->wl.status, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  return v;
}

extern "C" int dec_set_timeout_ns(dec_handle* h, unsigned long long ns) {
  if (!h) return DEC_ERR_NULL;
  if (ns < 1000000ull) return DEC_ERR_ARG;
  h->timeout_ns = ns;
  return DEC_OK;
}

extern "C" int dec_set_debug_stall(dec_handle* h, int cta_plus_one) {
  if (!h) return DEC_ERR_NULL;
  if (cta_plus_one < 0 || cta_plus_one > h->ctas) return DEC_ERR_ARG;
  h->stall_cta = cta_plus_one - 1;
  return DEC_OK;
}

extern "C" int dec_get_config(const dec_handle* h, int* ctas, int* ring_slots, int* slot_bytes) {
  if (!h) return DEC_ERR_NULL;
  if (ctas) *ctas = h->ctas;
  if (ring_slots) *ring_slots = h->nslot[1];
  if (slot_bytes) *slot_bytes = h->slot_bytes[1];
  return DEC_OK;
}

extern "C" const char* dec_error_string(int code) {
  switch (code) {
    case DEC_OK: return "ok";
    case DEC_ERR_NULL: return "a required pointer is NULL";
    case DEC_ERR_SHAPE: return "unsupported or inconsistent shape";
    case DEC_ERR_BATCH: return "batch out of range";
    case DEC_ERR_KV_SIZE: return "KV buffer too small";
    case DEC_ERR_DTYPE: return "unsupported KV dtype";
    case DEC_ERR_ALIGN: return "pointer not aligned";
    case DEC_ERR_CUDA: return "CUDA runtime error";
    case DEC_ERR_DEVICE: return "device not supported (needs compute capability 10.0)";
    case DEC_ERR_ARG: return "invalid argument";
    case DEC_ERR_TOO_LARGE: return "request exceeds the fixed scratch of dec_attention_noalloc";
    default: break;
  }
  if (code > 0) {
    static thread_local char buf[96];
    buf[0] = 0;
    if (code & DEC_DEV_BAD_POSITION) strcat(buf, "device: position out of range; ");
    if (code & DEC_DEV_BAD_TOKEN) strcat(buf, "device: token out of range; ");
    if (code & DEC_DEV_TIMEOUT) strcat(buf, "device: bounded wait ran out; ");
    return buf;
  }
  return "unknown status";
}

extern "C" int dec_last_cuda_error(void) { return g_last_cuda; }

// ------------------------------------------------------------ attention
extern "C" size_t dec_attention_workspace_bytes(int batch, int n_q_heads, int n_kv_heads,
                                                int head_dim, int max_len) {
  if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads || max_len < 1)
    return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cr = attention_chunk_rows(batch, n_kv_heads, max_len, sms);
  const int chunks = (max_len + cr - 1) / cr;
  return al256(sizeof(float) * static_cast<size_t>(batch) * n_q_heads * chunks * (head_dim + 2)) +
         al256(sizeof(unsigned) * static_cast<size_t>(batch) * n_kv_heads);
}

extern "C" int dec_attention(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                             const void* q, const void* k_cache, const void* v_cache, int max_len,
                             const int32_t* lengths, float* out, void* workspace,
                             size_t workspace_bytes, int* status, void* stream) {
  if (!q || !k_cache || !v_cache || !lengths || !out || !workspace) return DEC_ERR_NULL;
  if (batch < 1) return DEC_ERR_BATCH;
  if (head_dim != 64 && head_dim != 128) return DEC_ERR_SHAPE;
  if (n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads || n_q_heads / n_kv_heads > 8)
    return DEC_ERR_SHAPE;
  if (max_len < 1) return DEC_ERR_ARG;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(workspace, 256))
    return DEC_ERR_ALIGN;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t need = dec_attention_workspace_bytes(batch, n_q_heads, n_kv_heads, head_dim, max_len);
  if (workspace_bytes < need) return DEC_ERR_KV_SIZE;
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
  a.chunk_rows = attention_chunk_rows(batch, n_kv_heads, max_len, sms);
  a.chunks_max = (max_len + a.chunk_rows - 1) / a.chunk_rows;
  a.part = static_cast<float*>(workspace);
  a.cnt = reinterpret_cast<unsigned*>(
      static_cast<uint8_t*>(workspace) +
      al256(sizeof(float) * static_cast<size_t>(batch) * n_q_heads * a.chunks_max * (head_dim + 2)));
  a.status = status;
  e = launch_attention(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_kv_quantize_e4m3(const float* x, int rows, int dim, uint8_t* codes,
                                    float* scales, void* stream) {
  if (!x || !codes || !scales) return DEC_ERR_NULL;
  if (rows < 0) return DEC_ERR_ARG;
  if (dim != 64 && dim != 128) return DEC_ERR_SHAPE;
  if (rows == 0) return DEC_OK;
  cudaError_t e = launch_quantize(x, rows, dim, codes, scales, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_quantize_int8(const void* w, int rows, int cols, int8_t* codes,
                                 float* scales, void* stream) {
  if (!w || !codes || !scales) return DEC_ERR_NULL;
  if (rows < 0 || cols < 8 || cols % 8) return DEC_ERR_ARG;
  if (!aligned(w, 16) || !aligned(codes, 8) || !aligned(scales, 4)) return DEC_ERR_ALIGN;
  if (rows == 0) return DEC_OK;
  cudaError_t e = launch_quantize_int8(static_cast<const uint16_t*>(w), rows, cols, codes, scales,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

extern "C" int dec_quantize_fp8w(const void* w, int rows, int cols, uint8_t* codes,
                                 float* scales, void* stream) {
  if (!w || !codes || !scales) return DEC_ERR_NULL;
  if (rows < 0 || cols < 8 || cols % 8) return DEC_ERR_ARG;
  if (!aligned(w, 16) || !aligned(codes, 8) || !aligned(scales, 4)) return DEC_ERR_ALIGN;
  if (rows == 0) return DEC_OK;
  cudaError_t e = launch_quantize_fp8w(static_cast<const uint16_t*>(w), rows, cols, codes, scales,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return DEC_OK;
}

#ifdef DEC_PROFILE
namespace dec {
int bt_prof_read(BtPlan* p, unsigned long long* host, size_t n);
}
// Profiling builds only (not part of dec.h): GEMM phase timestamps of the
// batched step, [4 modes][2048 CTAs][16] globaltimer values.
extern "C" int dec_bt_prof_read(dec_handle* h, unsigned long long* host, size_t n) {
  if (!h || !h->bt || !host) return DEC_ERR_NULL;
  return dec::bt_prof_read(h->bt, host, n) == 0 ? DEC_OK : DEC_ERR_ARG;
}

// Profiling builds only (not part of dec.h): copy the per-phase timestamps of
// the last step, [ctas][32 * n_layers + 8] globaltimer values, to `host`.
extern "C" int dec_prof_read(dec_handle* h, unsigned long long* host, size_t n) {
  if (!h || !host) return DEC_ERR_NULL;
  const size_t need = static_cast<size_t>(h->ctas) * (kProfStampsPerLayer * h->shape.n_layers + 8);
  if (n < need) return DEC_ERR_ARG;
  cudaError_t e = cudaMemcpy(host, h->ws + h->wl.prof, need * sizeof(unsigned long long),
                             cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? DEC_OK : cuda_fail(e);
}
#endif
