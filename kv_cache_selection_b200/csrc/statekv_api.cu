// Host side of libstatekv: the C ABI declared in include/statekv.h, per-layer
// state (compressed C, detailed D) and the launch sequence of one step.
//
// One StateKV step ("Linear Scaling Video VLMs for Long Video Understanding",
// P1 section 方法步骤详情; P2 section 3.3) is enqueued as
//   (a) attention of the frame's queries over [C_{n-1}; frame]  -> out, lse
//   (b) score pass: column mass of the normalised weights       -> partials
//   (c) top-B select over the pool                              -> kept list
//   (d) gather of the kept rows into the other C buffer + append to D
// on the caller's stream with no host synchronisation.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "statekv.h"
#include "kernels.h"

namespace {

thread_local std::string g_free_error;  // errors of calls without a handle

struct LayerState {
  bool ready = false;
  int frames = 0;
  // entry point of the layer's last step (0 none, 1 device buffers on the
  // caller's stream, 2 host buffers on the library's compute stream) and the
  // completion of its last host-buffer step, which orders the layer's next
  // device-buffer step after it
  int last_entry = 0;
  cudaEvent_t ev_host_done = nullptr;
  int m = 0;    // current C length
  int cur = 0;  // index of the current C buffer
  void* kc[2] = {nullptr, nullptr};
  void* vc[2] = {nullptr, nullptr};
  int32_t* posc[2] = {nullptr, nullptr};
  float* scorec[2] = {nullptr, nullptr};
  void* kd = nullptr;
  void* vd = nullptr;
  int32_t* posd = nullptr;
  // per-step scratch of this layer (each layer has its own, so that steps of
  // different layers may run concurrently on different streams)
  float* lse = nullptr;         // [S][Hq][T]
  float* part = nullptr;        // [S][Hkv * query splits][B+T]
  float* pool_score = nullptr;  // [S][Hkv][B+T]
  int32_t* idx = nullptr;       // [S][Hkv][max(B,1)]
  __nv_bfloat16* o_part = nullptr;  // attention key-split partials (bf16 path)
  float* ml_part = nullptr;
  int pool_len = 0;             // pool size of the layer's last step
};

}  // namespace

struct statekv_handle {
  int S = 1, Hq = 0, Hkv = 0, d = 0, T = 0, B = 0, max_frames = 0;
  int dtype = 0, mask = 0, select = 0;
  int n_sm = 148;
  int device = 0;
  size_t esize = 2;
  std::vector<LayerState> layers;
  int* dev_err = nullptr;       // kernel error word (bounded-wait timeouts)
  unsigned long long wait_ns = 0;  // pipeline-wait limit of the tensor-core kernels (0: default)
  int max_split = 1;            // key splits the attention scratch is sized for
  int last_layer = -1;          // layer of the most recent prefill_frame
  // statekv_prefill_frame_host: two staging sets used in turn, a copy stream
  // for the host-to-device copies, and the events that order them (created on
  // first use)
  void* stage_q[2] = {nullptr, nullptr};
  void* stage_k[2] = {nullptr, nullptr};
  void* stage_v[2] = {nullptr, nullptr};
  void* stage_out[2] = {nullptr, nullptr};
  int32_t* stage_pos[2] = {nullptr, nullptr};
  int stage_next = 0;
  cudaStream_t copy_stream = nullptr;
  cudaStream_t compute_stream = nullptr;  // the steps of host-buffer calls
  cudaEvent_t ev_h2d[2] = {nullptr, nullptr};   // inputs of set b are on the device
  cudaEvent_t ev_step_done[2] = {nullptr, nullptr};  // the step that reads set b's inputs is done
  cudaEvent_t ev_stage_free[2] = {nullptr, nullptr};  // the copy-out of set b's output is done
  cudaEvent_t ev_caller = nullptr;  // tail of the caller's stream (device-buffer steps before a host call)
  // key-split partials of statekv_decode (float32), grown on demand
  float* dec_o = nullptr;
  float* dec_ml = nullptr;
  size_t dec_o_bytes = 0, dec_ml_bytes = 0;
  std::string err;
  std::vector<void*> allocs;
  // launch accounting and optional per-stage event timing
  long long launches = 0;
  int prof = 0;  // 0 off, 1 per-kernel events, 2 attention and its merge as one stage
  struct Rec {
    int stage;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> ev_free;
};

namespace {

int set_err(statekv_t h, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  else g_free_error = buf;
  return code;
}

int dev_alloc(statekv_t h, void** p, size_t bytes) {
  bytes = std::max<size_t>(bytes, 16);
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return set_err(h, STATEKV_ERR_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  e = cudaMemset(*p, 0, bytes);
  if (e != cudaSuccess) {
    cudaFree(*p);
    *p = nullptr;
    return set_err(h, STATEKV_ERR_CUDA, "cudaMemset failed: %s", cudaGetErrorString(e));
  }
  h->allocs.push_back(*p);
  return STATEKV_OK;
}

int check_shape(statekv_t h, int S, int Hq, int Hkv, int d, int T, int B, int max_frames, int dtype,
                int mask, int select) {
  if (S < 1 || Hq < 1 || Hkv < 1 || T < 1 || B < 0 || max_frames < 1)
    return set_err(h, STATEKV_ERR_INVALID_ARG,
                   "bad shape: S=%d Hq=%d Hkv=%d T=%d B=%d max_frames=%d", S, Hq, Hkv, T, B,
                   max_frames);
  if (Hq % Hkv != 0) return set_err(h, STATEKV_ERR_INVALID_ARG, "Hq (%d) %% Hkv (%d) != 0", Hq, Hkv);
  if (dtype != STATEKV_BF16 && dtype != STATEKV_F32)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (mask != STATEKV_MASK_FRAME_CAUSAL && mask != STATEKV_MASK_FRAME_BIDIR)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "bad mask_mode %d", mask);
  if (select != STATEKV_SELECT_GLOBAL && select != STATEKV_SELECT_PER_KV_HEAD && select != STATEKV_SELECT_RECENCY)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "bad select_mode %d", select);
  if (d != 64 && d != 128) return set_err(h, STATEKV_ERR_UNSUPPORTED, "head dim %d not in {64,128}", d);
  if ((long long)B + T > 28672)
    return set_err(h, STATEKV_ERR_UNSUPPORTED, "pool B+T=%lld above 28672", (long long)B + T);
  if ((long long)max_frames * T > (1LL << 30))
    return set_err(h, STATEKV_ERR_UNSUPPORTED, "max_frames*T too large");
  return STATEKV_OK;
}

int alloc_layer(statekv_t h, LayerState& L) {
  const size_t cbytes = (size_t)h->S * h->Hkv * h->B * h->d * h->esize;
  const size_t cint = (size_t)h->S * h->Hkv * h->B * 4;
  const size_t max_tok = (size_t)h->max_frames * h->T;
  const size_t dbytes = (size_t)h->S * h->Hkv * max_tok * h->d * h->esize;
  int rc;
  for (int b = 0; b < 2; ++b) {
    if ((rc = dev_alloc(h, &L.kc[b], cbytes))) return rc;
    if ((rc = dev_alloc(h, &L.vc[b], cbytes))) return rc;
    if ((rc = dev_alloc(h, (void**)&L.posc[b], cint))) return rc;
    if ((rc = dev_alloc(h, (void**)&L.scorec[b], cint))) return rc;
  }
  if ((rc = dev_alloc(h, &L.kd, dbytes))) return rc;
  if ((rc = dev_alloc(h, &L.vd, dbytes))) return rc;
  if ((rc = dev_alloc(h, (void**)&L.posd, (size_t)h->S * max_tok * 4))) return rc;
  const size_t S = h->S, pool = (size_t)h->B + h->T;
  if ((rc = dev_alloc(h, (void**)&L.lse, S * h->Hq * h->T * 4)) ||
      (rc = dev_alloc(h, (void**)&L.part, S * h->Hkv * skv::kMaxQsplit * pool * 4)) ||
      (rc = dev_alloc(h, (void**)&L.pool_score, S * h->Hkv * pool * 4)) ||
      (rc = dev_alloc(h, (void**)&L.idx, S * h->Hkv * std::max(h->B, 1) * 4)))
    return rc;
  if (h->max_split > 1 &&
      ((rc = dev_alloc(h, (void**)&L.o_part, S * h->Hq * h->max_split * h->T * h->d * 2)) ||
       (rc = dev_alloc(h, (void**)&L.ml_part, S * h->Hq * h->max_split * h->T * 4))))
    return rc;
  L.ready = true;
  return STATEKV_OK;
}

int get_layer(statekv_t h, int layer, LayerState** out) {
  if (layer < 0) return set_err(h, STATEKV_ERR_INVALID_ARG, "negative layer %d", layer);
  if ((size_t)layer >= h->layers.size()) h->layers.resize(layer + 1);
  LayerState& L = h->layers[layer];
  if (!L.ready) {
    int rc = alloc_layer(h, L);
    if (rc) return rc;
  }
  *out = &L;
  return STATEKV_OK;
}

cudaEvent_t take_event(statekv_t h) {
  if (!h->ev_free.empty()) {
    cudaEvent_t e = h->ev_free.back();
    h->ev_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// Brackets one kernel launch: counts it and, when profiling, records an event
// pair on the launch stream.
struct StageScope {
  statekv_t h;
  cudaStream_t st;
  int stage;
  cudaEvent_t a = nullptr;
  StageScope(statekv_t h_, cudaStream_t st_, int stage_) : h(h_), st(st_), stage(stage_) {
    if (h->prof && (a = take_event(h)) != nullptr) cudaEventRecord(a, st);
  }
  void done() {
    ++h->launches;
    if (!a) return;
    cudaEvent_t b = take_event(h);
    if (!b) {
      h->ev_free.push_back(a);
      return;
    }
    cudaEventRecord(b, st);
    h->recs.push_back({stage, a, b});
  }
};

// TMA maps of one step: q [S][T][Hq][d], K_C [S][Hkv][B][d], frame k [S][T][Hkv][d]
int encode_step_maps(statekv_t h, const void* q, const void* kc, const void* k, CUtensorMap* tq,
                     CUtensorMap* tkc, CUtensorMap* tkf, const void* vc = nullptr, const void* v = nullptr,
                     CUtensorMap* tvc = nullptr, CUtensorMap* tvf = nullptr) {
  const uint64_t d = h->d, Hq = h->Hq, Hkv = h->Hkv, T = h->T, S = h->S;
  const uint64_t B = std::max(h->B, 1);
  const uint64_t dq[4] = {d, Hq, T, S};
  const uint64_t sq[3] = {d * 2, Hq * d * 2, T * Hq * d * 2};
  const uint32_t bq[4] = {64, 1, 128, 1};
  const uint64_t dc[4] = {d, B, Hkv, S};
  const uint64_t sc[3] = {d * 2, B * d * 2, Hkv * B * d * 2};
  const uint32_t bc[4] = {64, 128, 1, 1};
  const uint64_t dk[4] = {d, Hkv, T, S};
  const uint64_t sk[3] = {d * 2, Hkv * d * 2, T * Hkv * d * 2};
  int r;
  if ((r = skv::encode_tmap_bf16_4d(tq, q, dq, sq, bq)) != 0 ||
      (r = skv::encode_tmap_bf16_4d(tkc, kc, dc, sc, bc)) != 0 ||
      (r = skv::encode_tmap_bf16_4d(tkf, k, dk, sk, bq)) != 0 ||
      (tvc && (r = skv::encode_tmap_bf16_4d(tvc, vc, dc, sc, bc)) != 0) ||
      (tvf && (r = skv::encode_tmap_bf16_4d(tvf, v, dk, sk, bq)) != 0))
    return set_err(h, STATEKV_ERR_CUDA, "TMA tensor map encoding failed (CUresult %d)", r);
  return STATEKV_OK;
}

int launch_err(statekv_t h, cudaError_t e, const char* what) {
  return set_err(h, STATEKV_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace skv {
void set_free_error(const char* msg) { g_free_error = msg; }
}  // namespace skv

namespace {

// Process-wide scratch of full_causal_prefill's key-split partials, grown on
// demand (one buffer per device, guarded by a mutex).
std::mutex g_fc_mu;
struct FcScratch {
  __nv_bfloat16* o = nullptr;
  float* ml = nullptr;
  int* err = nullptr;
  size_t o_bytes = 0, ml_bytes = 0;
};
FcScratch g_fc[64];

int full_causal_tc(const void* q, const void* k, const void* v, int n_seq, int N, int Hq, int Hkv, int d,
                   void* out, float* lse, cudaStream_t st) {
  int dev = 0, n_sm = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64)
    return set_err(nullptr, STATEKV_ERR_CUDA, "no usable CUDA device");
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  skv::AttnTcArgs ta{};
  ta.out = out;
  ta.out_s = (long long)N * Hq * d;
  ta.out_row = Hq * d;
  ta.lse = lse;
  ta.lse_s = (long long)Hq * N;
  ta.m = 0;
  ta.T = N;
  ta.Hq = Hq;
  ta.Hkv = Hkv;
  ta.causal = 1;
  ta.S = n_seq;
  ta.n_it = (N + 127) / 128;
  ta.n_pairs = ((Hq / Hkv) * ta.n_it + 1) / 2;
  ta.n_split = skv::attn_tc_splits(n_seq, Hq, Hkv, N, 0, n_sm);
  ta.nC = 0;
  ta.nF = ta.n_it;
  ta.stack = 0;
  ta.q_rows = 128;
  ta.scale_log2 = skv::kLog2e / sqrtf((float)d);
  {
    std::lock_guard<std::mutex> lk(g_fc_mu);
    FcScratch& sc = g_fc[dev];
    const size_t ob = ta.n_split > 1 ? (size_t)n_seq * Hq * ta.n_split * N * d * 2 : 16;
    const size_t mb = ta.n_split > 1 ? (size_t)n_seq * Hq * ta.n_split * N * 4 : 16;
    if (!sc.err && cudaMalloc((void**)&sc.err, 16) == cudaSuccess) cudaMemset(sc.err, 0, 16);
    if (sc.o_bytes < ob) {
      if (sc.o) cudaFree(sc.o);
      sc.o = nullptr;
      sc.o_bytes = 0;
      if (cudaMalloc((void**)&sc.o, ob) != cudaSuccess) {
        cudaGetLastError();
        return set_err(nullptr, STATEKV_ERR_OOM, "scratch allocation of %zu bytes failed", ob);
      }
      sc.o_bytes = ob;
    }
    if (sc.ml_bytes < mb) {
      if (sc.ml) cudaFree(sc.ml);
      sc.ml = nullptr;
      sc.ml_bytes = 0;
      if (cudaMalloc((void**)&sc.ml, mb) != cudaSuccess) {
        cudaGetLastError();
        return set_err(nullptr, STATEKV_ERR_OOM, "scratch allocation of %zu bytes failed", mb);
      }
      sc.ml_bytes = mb;
    }
    if (!sc.err) return set_err(nullptr, STATEKV_ERR_OOM, "error-word allocation failed");
    ta.o_part = sc.o;
    ta.ml_part = sc.ml;
    ta.err = sc.err;
  }
  // q [S][N][Hq][d] and k, v [S][N][Hkv][d]: the whole sequence is the "frame"
  const uint64_t D = d;
  const uint64_t dq[4] = {D, (uint64_t)Hq, (uint64_t)N, (uint64_t)n_seq};
  const uint64_t sq[3] = {D * 2, (uint64_t)Hq * D * 2, (uint64_t)N * Hq * D * 2};
  const uint64_t dk[4] = {D, (uint64_t)Hkv, (uint64_t)N, (uint64_t)n_seq};
  const uint64_t sk[3] = {D * 2, (uint64_t)Hkv * D * 2, (uint64_t)N * Hkv * D * 2};
  const uint32_t box[4] = {64, 1, 128, 1};
  CUtensorMap tq, tk, tv;
  int r;
  if ((r = skv::encode_tmap_bf16_4d(&tq, q, dq, sq, box)) || (r = skv::encode_tmap_bf16_4d(&tk, k, dk, sk, box)) ||
      (r = skv::encode_tmap_bf16_4d(&tv, v, dk, sk, box)))
    return set_err(nullptr, STATEKV_ERR_CUDA, "TMA tensor map encoding failed (CUresult %d)", r);
  // no compressed rows: the C maps are never read
  if ((e = skv::launch_attn_tc(tq, tk, tv, tk, tv, ta, d, st)) != cudaSuccess)
    return set_err(nullptr, STATEKV_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(e));
  if (ta.n_split > 1 && (e = skv::launch_attn_combine(ta, d, st)) != cudaSuccess)
    return set_err(nullptr, STATEKV_ERR_CUDA, "attention combine launch failed: %s", cudaGetErrorString(e));
  return STATEKV_OK;
}

}  // namespace

extern "C" {

int statekv_create_batched(statekv_t* out, int n_streams, int Hq, int Hkv, int d, int T, int B,
                           int max_frames, int dtype, int mask_mode, int select_mode) {
  if (!out) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle pointer");
  int rc = check_shape(nullptr, n_streams, Hq, Hkv, d, T, B, max_frames, dtype, mask_mode, select_mode);
  if (rc) return rc;
  statekv_t h = new (std::nothrow) statekv_handle();
  if (!h) return set_err(nullptr, STATEKV_ERR_OOM, "host allocation failed");
  h->S = n_streams;
  h->Hq = Hq;
  h->Hkv = Hkv;
  h->d = d;
  h->T = T;
  h->B = B;
  h->max_frames = max_frames;
  h->dtype = dtype;
  h->mask = mask_mode;
  h->select = select_mode;
  h->esize = dtype == STATEKV_BF16 ? 2 : 4;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device);
  if (e != cudaSuccess) {
    set_err(nullptr, STATEKV_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
    delete h;
    return STATEKV_ERR_CUDA;
  }
  if ((rc = dev_alloc(h, (void**)&h->dev_err, 16))) {
    g_free_error = h->err;
    statekv_destroy(h);
    return rc;
  }
  if (dtype == STATEKV_BF16) h->max_split = skv::attn_tc_splits(n_streams, Hq, Hkv, T, B, h->n_sm);
  *out = h;
  return STATEKV_OK;
}

int statekv_create(statekv_t* out, int Hq, int Hkv, int d, int T, int B, int max_frames, int dtype,
                   int mask_mode, int select_mode) {
  return statekv_create_batched(out, 1, Hq, Hkv, d, T, B, max_frames, dtype, mask_mode, select_mode);
}

int statekv_reserve_layers(statekv_t h, int n_layers) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (n_layers < 0) return set_err(h, STATEKV_ERR_INVALID_ARG, "negative layer count");
  for (int l = 0; l < n_layers; ++l) {
    LayerState* L;
    int rc = get_layer(h, l, &L);
    if (rc) return rc;
  }
  return STATEKV_OK;
}

namespace {
// One frame of one layer on `stream` (both entry points).
int prefill_step(statekv_t h, int layer, const void* q, const void* k, const void* v, const int32_t* pos,
                 void* out, void* stream) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (!q || !k || !v || !pos || !out)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "null input/output pointer");
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "q/k/v/out must be 16-byte aligned");
  if (layer >= 0 && (size_t)layer < h->layers.size() && h->layers[layer].ready &&
      h->layers[layer].frames >= h->max_frames)
    return set_err(h, STATEKV_ERR_CAPACITY, "layer %d already holds max_frames=%d frames", layer,
                   h->max_frames);
  LayerState* L;
  int rc = get_layer(h, layer, &L);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int S = h->S, Hq = h->Hq, Hkv = h->Hkv, d = h->d, T = h->T, B = h->B;
  const int m = L->m, cur = L->cur, nxt = cur ^ 1;
  const int pool = B + T;
  const int m_new = std::min(B, m + T);
  const float scale_log2 = skv::kLog2e / sqrtf((float)d);
  cudaError_t e;

  // (a) attention over [C_{n-1}; frame]
  skv::AttnArgs aa{};
  aa.q = q;
  aa.q_s = (long long)T * Hq * d;
  aa.q_row = Hq * d;
  aa.ka = L->kc[cur];
  aa.va = L->vc[cur];
  aa.a_s = (long long)Hkv * B * d;
  aa.a_g = (long long)B * d;
  aa.m = m;
  aa.kb = k;
  aa.vb = v;
  aa.b_s = (long long)T * Hkv * d;
  aa.b_row = Hkv * d;
  aa.nb = T;
  aa.out = out;
  aa.lse = L->lse;
  aa.lse_s = (long long)Hq * T;
  aa.n_rows = T;
  aa.Hq = Hq;
  aa.Hkv = Hkv;
  aa.causal = h->mask == STATEKV_MASK_FRAME_CAUSAL;
  aa.scale_log2 = scale_log2;
  CUtensorMap tq, tkc, tkf, tvc, tvf;
  skv::MergeArgs mrg{};  // key-split merge, run by the select launch (bf16 with splits)
  int n_split = 1;
  if (h->dtype == STATEKV_BF16) {
    if ((rc = encode_step_maps(h, q, L->kc[cur], k, &tq, &tkc, &tkf, L->vc[cur], v, &tvc, &tvf))) return rc;
    skv::AttnTcArgs ta{};
    ta.out = out;
    ta.out_s = (long long)T * Hq * d;
    ta.out_row = Hq * d;
    ta.lse = L->lse;
    ta.lse_s = (long long)Hq * T;
    ta.o_part = L->o_part;
    ta.ml_part = L->ml_part;
    ta.m = m;
    ta.T = T;
    ta.Hq = Hq;
    ta.Hkv = Hkv;
    ta.causal = aa.causal;
    ta.S = S;
    ta.n_it = (T + 127) / 128;
    ta.n_pairs = ((Hq / Hkv) * ta.n_it + 1) / 2;
    ta.n_split = std::min(h->max_split, skv::attn_tc_splits(S, Hq, Hkv, T, m, h->n_sm));
    ta.nC = (m + 127) / 128;
    ta.nF = ta.n_it;
    ta.stack = 0;
    ta.q_rows = 128;
    ta.scale_log2 = scale_log2;
    ta.err = h->dev_err;
    ta.wait_ns = h->wait_ns;
    {
      const bool chained = h->prof == 2 && ta.n_split > 1;
      StageScope sc(h, st, chained ? STATEKV_STAGE_ATTENTION_CHAINED : STATEKV_STAGE_ATTENTION);
      if ((e = skv::launch_attn_tc(tq, tkc, tvc, tkf, tvf, ta, d, st, true)) != cudaSuccess)
        return launch_err(h, e, "attention");
      if (chained) {
        // profiling mode 2: the merge right behind the attention, in the same event pair
        if ((e = skv::launch_attn_combine(ta, d, st, true)) != cudaSuccess) return launch_err(h, e, "attention merge");
        ++h->launches;
      }
      sc.done();
    }
    n_split = ta.n_split;
    if (n_split > 1 && h->prof != 2) {
      if (h->prof) {
        // timed runs charge the merge of the key splits to the attention stage
        // by launching it on its own; otherwise it rides in the select launch
        StageScope sc(h, st, STATEKV_STAGE_ATTENTION_COMBINE);
        if ((e = skv::launch_attn_combine(ta, d, st, true)) != cudaSuccess) return launch_err(h, e, "attention merge");
        sc.done();
      } else {
        mrg = skv::merge_args(ta, d);
      }
    }
  } else {
    StageScope sc(h, st, STATEKV_STAGE_ATTENTION);
    if ((e = skv::launch_attn_simt(aa, h->dtype, d, S, st)) != cudaSuccess) return launch_err(h, e, "attention");
    sc.done();
  }

  // (b) score pass
  int n_qsplit = 1;  // rows of the partial-sum buffer per KV group
  skv::ScoreArgs sa{};
  sa.q = q;
  sa.q_s = aa.q_s;
  sa.q_row = aa.q_row;
  sa.ka = aa.ka;
  sa.a_s = aa.a_s;
  sa.a_g = aa.a_g;
  sa.m = m;
  sa.kb = k;
  sa.b_s = aa.b_s;
  sa.b_row = aa.b_row;
  sa.nb = T;
  sa.lse = L->lse;
  sa.lse_s = aa.lse_s;
  sa.part = L->part;
  sa.part_s = (long long)Hkv * pool;
  sa.part_g = pool;
  sa.n_rows = T;
  sa.Hq = Hq;
  sa.Hkv = Hkv;
  sa.causal = aa.causal;
  sa.scale_log2 = scale_log2;
  if (h->dtype == STATEKV_BF16) {
    skv::ScoreTcArgs ta{};
    ta.lse = L->lse;
    ta.lse_s = aa.lse_s;
    ta.ml_part = L->ml_part;
    ta.n_split = n_split;
    ta.n_qsplit = skv::score_tc_qsplit(S, Hq, Hkv, T, m, h->n_sm);
    n_qsplit = ta.n_qsplit;
    ta.part = L->part;
    ta.part_s = (long long)Hkv * n_qsplit * pool;
    ta.part_g = pool;
    ta.m = m;
    ta.T = T;
    ta.Hq = Hq;
    ta.Hkv = Hkv;
    ta.causal = aa.causal;
    ta.n_c_tiles = (m + 127) / 128;
    ta.n_f_tiles = (T + 127) / 128;
    ta.S = S;
    ta.scale_log2 = scale_log2;
    ta.err = h->dev_err;
    ta.wait_ns = h->wait_ns;
    StageScope sc(h, st, STATEKV_STAGE_SCORE);
    if ((e = skv::launch_score_tc(tq, tkc, tkf, ta, d, st, true)) != cudaSuccess) return launch_err(h, e, "score");
    sc.done();
  } else {
    StageScope sc(h, st, STATEKV_STAGE_SCORE);
    if ((e = skv::launch_score_simt(sa, h->dtype, d, S, st)) != cudaSuccess) return launch_err(h, e, "score");
    sc.done();
  }

  // (c) top-B select
  skv::SelectArgs se{};
  se.part = L->part;
  se.part_s = (long long)Hkv * n_qsplit * pool;
  se.part_g = pool;
  se.n_qsplit = n_qsplit;
  se.pool_score = L->pool_score;
  se.pool_s = (long long)Hkv * pool;
  se.pos_c = L->posc[cur];
  se.pos_f = pos;
  se.idx = L->idx;
  se.Hkv = Hkv;
  se.m = m;
  se.T = T;
  se.B = B;
  se.global = h->select != STATEKV_SELECT_PER_KV_HEAD;  // recency keeps one set per layer too
  se.recency = h->select == STATEKV_SELECT_RECENCY;
  se.mrg = mrg;
  {
    StageScope sc(h, st, STATEKV_STAGE_SELECT);
    if ((e = skv::launch_select(se, S, st, true)) != cudaSuccess) return launch_err(h, e, "select");
    sc.done();
  }

  // (d) gather into C_n + append to D
  skv::GatherArgs ga{};
  ga.kc = L->kc[cur];
  ga.vc = L->vc[cur];
  ga.kf = k;
  ga.vf = v;
  ga.kc_new = L->kc[nxt];
  ga.vc_new = L->vc[nxt];
  ga.idx = L->idx;
  ga.kd = L->kd;
  ga.vd = L->vd;
  ga.pos_d = L->posd;
  ga.pos_f = pos;
  ga.pos_c = se.pos_c;
  ga.pool_score = se.pool_score;
  ga.pos_new = L->posc[nxt];
  ga.score_new = L->scorec[nxt];
  ga.pool_g = se.part_g;
  ga.Hkv = Hkv;
  ga.T = T;
  ga.B = B;
  ga.m = m;
  ga.m_new = m_new;
  ga.row_bytes = (int)(d * h->esize);
  ga.global = se.global;
  ga.d_len = L->frames * T;
  ga.max_tok = h->max_frames * T;
  ga.S = S;
  {
    StageScope sc(h, st, STATEKV_STAGE_GATHER);
    if ((e = skv::launch_gather(ga, h->n_sm, st, true)) != cudaSuccess) return launch_err(h, e, "gather");
    sc.done();
  }

  L->m = m_new;
  L->cur = nxt;
  L->frames += 1;
  L->pool_len = m + T;
  h->last_layer = layer;
  return STATEKV_OK;
}
}  // namespace

int statekv_prefill_frame(statekv_t h, int layer, const void* q, const void* k, const void* v,
                          const int32_t* pos, void* out, void* stream) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  LayerState* L = (layer >= 0 && (size_t)layer < h->layers.size()) ? &h->layers[layer] : nullptr;
  if (L && L->last_entry == 2 && L->ev_host_done) {
    // the layer's previous step came through the host-buffer call
    const cudaError_t e = cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), L->ev_host_done, 0);
    if (e != cudaSuccess) return set_err(h, STATEKV_ERR_CUDA, "stream wait failed: %s", cudaGetErrorString(e));
  }
  const int rc = prefill_step(h, layer, q, k, v, pos, out, stream);
  if (rc == STATEKV_OK) h->layers[layer].last_entry = 1;
  return rc;
}

int statekv_prefill_frame_host(statekv_t h, int layer, const void* q, const void* k, const void* v,
                               const int32_t* pos, void* out, void* stream) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (!q || !k || !v || !pos || !out)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "null input/output pointer");
  const size_t qb = (size_t)h->S * h->T * h->Hq * h->d * h->esize;
  const size_t kb = (size_t)h->S * h->T * h->Hkv * h->d * h->esize;
  const size_t pb = (size_t)h->S * h->T * 4;
  int rc;
  cudaError_t e;
  if (!h->stage_q[0]) {
    for (int b = 0; b < 2; ++b)
      if ((rc = dev_alloc(h, &h->stage_q[b], qb)) || (rc = dev_alloc(h, &h->stage_k[b], kb)) ||
          (rc = dev_alloc(h, &h->stage_v[b], kb)) || (rc = dev_alloc(h, &h->stage_out[b], qb)) ||
          (rc = dev_alloc(h, (void**)&h->stage_pos[b], pb)))
        return rc;
    if ((e = cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&h->compute_stream, cudaStreamNonBlocking)) != cudaSuccess)
      return set_err(h, STATEKV_ERR_CUDA, "staging streams: %s", cudaGetErrorString(e));
    for (int b = 0; b < 2; ++b)
      if ((e = cudaEventCreateWithFlags(&h->ev_h2d[b], cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&h->ev_step_done[b], cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&h->ev_stage_free[b], cudaEventDisableTiming)) != cudaSuccess)
        return set_err(h, STATEKV_ERR_CUDA, "staging events: %s", cudaGetErrorString(e));
    if ((e = cudaEventCreateWithFlags(&h->ev_caller, cudaEventDisableTiming)) != cudaSuccess)
      return set_err(h, STATEKV_ERR_CUDA, "staging events: %s", cudaGetErrorString(e));
  }
  // the step's own refusals, checked before anything is enqueued
  if (layer < 0) return set_err(h, STATEKV_ERR_INVALID_ARG, "negative layer %d", layer);
  if ((size_t)layer < h->layers.size() && h->layers[layer].ready && h->layers[layer].frames >= h->max_frames)
    return set_err(h, STATEKV_ERR_CAPACITY, "layer %d already holds max_frames=%d frames", layer, h->max_frames);
  LayerState* L;
  if ((rc = get_layer(h, layer, &L))) return rc;
  if (!L->ev_host_done && (e = cudaEventCreateWithFlags(&L->ev_host_done, cudaEventDisableTiming)) != cudaSuccess)
    return set_err(h, STATEKV_ERR_CUDA, "layer event: %s", cudaGetErrorString(e));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = h->compute_stream;
  const int b = h->stage_next;
  // Three streams: the inputs of this call go to staging set b on the copy
  // stream once set b's last step has read its inputs; the step runs on the
  // library's compute stream once they have arrived and set b's last output
  // has been copied out; `stream` waits for the step and copies out back.  So
  // the copy-in of call n+1 and the copy-out of call n overlap the steps, the
  // two directions overlap each other, and when `stream` has reached the end
  // of this call out is complete.
  if ((e = cudaStreamWaitEvent(h->copy_stream, h->ev_step_done[b], 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->stage_q[b], q, qb, cudaMemcpyHostToDevice, h->copy_stream)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->stage_k[b], k, kb, cudaMemcpyHostToDevice, h->copy_stream)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->stage_v[b], v, kb, cudaMemcpyHostToDevice, h->copy_stream)) != cudaSuccess ||
      (e = cudaMemcpyAsync(h->stage_pos[b], pos, pb, cudaMemcpyHostToDevice, h->copy_stream)) != cudaSuccess ||
      (e = cudaEventRecord(h->ev_h2d[b], h->copy_stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs, h->ev_h2d[b], 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs, h->ev_stage_free[b], 0)) != cudaSuccess)
    return set_err(h, STATEKV_ERR_CUDA, "host-to-device copy failed: %s", cudaGetErrorString(e));
  if (L->last_entry == 1) {
    // the layer's previous step came through the device-buffer call on the
    // caller's stream
    if ((e = cudaEventRecord(h->ev_caller, st)) != cudaSuccess || (e = cudaStreamWaitEvent(cs, h->ev_caller, 0)) != cudaSuccess)
      return set_err(h, STATEKV_ERR_CUDA, "stream wait failed: %s", cudaGetErrorString(e));
  }
  rc = prefill_step(h, layer, h->stage_q[b], h->stage_k[b], h->stage_v[b], h->stage_pos[b], h->stage_out[b], cs);
  if (rc) return rc;
  L->last_entry = 2;
  if ((e = cudaEventRecord(h->ev_step_done[b], cs)) != cudaSuccess ||
      (e = cudaEventRecord(L->ev_host_done, cs)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(st, h->ev_step_done[b], 0)) != cudaSuccess ||
      (e = cudaMemcpyAsync(out, h->stage_out[b], qb, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
      (e = cudaEventRecord(h->ev_stage_free[b], st)) != cudaSuccess)
    return set_err(h, STATEKV_ERR_CUDA, "device-to-host copy failed: %s", cudaGetErrorString(e));
  h->stage_next = b ^ 1;
  return STATEKV_OK;
}

int statekv_decode(statekv_t h, int layer, const void* q, const void* k, const void* v, int n_text, void* out,
                   float* lse, void* stream) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (!q || !k || !v || !out) return set_err(h, STATEKV_ERR_INVALID_ARG, "null input/output pointer");
  if (n_text < 1) return set_err(h, STATEKV_ERR_INVALID_ARG, "n_text=%d must be >= 1", n_text);
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "q/k/v/out must be 16-byte aligned");
  if (lse && ((uintptr_t)lse & 3)) return set_err(h, STATEKV_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (layer < 0 || (size_t)layer >= h->layers.size() || !h->layers[layer].ready)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "unknown layer %d", layer);
  const LayerState& L = h->layers[layer];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int S = h->S, Hq = h->Hq, Hkv = h->Hkv, d = h->d, T = h->T, G = Hq / Hkv;
  const int N = L.frames * T;                 // tokens in D
  const long long max_tok = (long long)h->max_frames * T;
  const float scale_log2 = skv::kLog2e / sqrtf((float)d);
  cudaError_t e;
  if (h->dtype != STATEKV_BF16) {
    skv::AttnArgs aa{};
    aa.q = q;
    aa.q_s = (long long)n_text * Hq * d;
    aa.q_row = Hq * d;
    aa.ka = L.kd;
    aa.va = L.vd;
    aa.a_s = (long long)Hkv * max_tok * d;
    aa.a_g = max_tok * d;
    aa.m = N;
    aa.kb = k;
    aa.vb = v;
    aa.b_s = (long long)n_text * Hkv * d;
    aa.b_row = Hkv * d;
    aa.nb = n_text;
    aa.out = out;
    aa.lse = lse;
    aa.lse_s = (long long)Hq * n_text;
    aa.n_rows = n_text;
    aa.Hq = Hq;
    aa.Hkv = Hkv;
    aa.causal = 1;
    aa.scale_log2 = scale_log2;
    StageScope sc(h, st, STATEKV_STAGE_DECODE);
    if ((e = skv::launch_attn_simt(aa, h->dtype, d, S, st)) != cudaSuccess) return launch_err(h, e, "decode");
    sc.done();
    return STATEKV_OK;
  }
  // tensor cores: each query tile stacks the G heads of a KV group, so every
  // D tile is read once per group; key splits fill the SMs
  skv::AttnTcArgs ta{};
  const int ri = 128 / G;
  ta.out = out;
  ta.out_s = (long long)n_text * Hq * d;
  ta.out_row = Hq * d;
  ta.lse = lse;
  ta.lse_s = (long long)Hq * n_text;
  ta.m = N;
  ta.T = n_text;
  ta.Hq = Hq;
  ta.Hkv = Hkv;
  ta.causal = 1;
  ta.S = S;
  ta.stack = G;
  ta.q_rows = G * ri;
  ta.n_it = (n_text + ri - 1) / ri;
  ta.n_pairs = (ta.n_it + 1) / 2;
  ta.nC = (N + 127) / 128;
  ta.nF = (n_text + 127) / 128;
  ta.scale_log2 = scale_log2;
  ta.err = h->dev_err;
  ta.wait_ns = h->wait_ns;
  const int units = S * Hkv * ta.n_pairs;
  int split = std::max(1, h->n_sm / std::max(units, 1));
  split = std::min(split, std::min(ta.nC + ta.nF, skv::kMaxMergeSplit));
  ta.n_split = split;
  if (split > 1) {
    const size_t ob = (size_t)S * Hq * split * n_text * d * 4, mb = (size_t)S * Hq * split * n_text * 4;
    if (h->dec_o_bytes < ob) {
      if (h->dec_o) cudaFree(h->dec_o);
      h->dec_o = nullptr;
      h->dec_o_bytes = 0;
      if (cudaMalloc((void**)&h->dec_o, ob) != cudaSuccess) {
        cudaGetLastError();
        return set_err(h, STATEKV_ERR_OOM, "decode scratch of %zu bytes", ob);
      }
      h->dec_o_bytes = ob;
    }
    if (h->dec_ml_bytes < mb) {
      if (h->dec_ml) cudaFree(h->dec_ml);
      h->dec_ml = nullptr;
      h->dec_ml_bytes = 0;
      if (cudaMalloc((void**)&h->dec_ml, mb) != cudaSuccess) {
        cudaGetLastError();
        return set_err(h, STATEKV_ERR_OOM, "decode scratch of %zu bytes", mb);
      }
      h->dec_ml_bytes = mb;
    }
    ta.o_part32 = h->dec_o;
    ta.ml_part = h->dec_ml;
  }
  const uint64_t D = d;
  const uint64_t dq[4] = {D, (uint64_t)Hq, (uint64_t)n_text, (uint64_t)S};
  const uint64_t sq[3] = {D * 2, (uint64_t)Hq * D * 2, (uint64_t)n_text * Hq * D * 2};
  const uint32_t bq[4] = {64, (uint32_t)G, (uint32_t)ri, 1};
  const uint64_t dd[4] = {D, (uint64_t)max_tok, (uint64_t)Hkv, (uint64_t)S};
  const uint64_t sd[3] = {D * 2, (uint64_t)max_tok * D * 2, (uint64_t)Hkv * max_tok * D * 2};
  const uint32_t bd[4] = {64, 128, 1, 1};
  const uint64_t dk[4] = {D, (uint64_t)Hkv, (uint64_t)n_text, (uint64_t)S};
  const uint64_t sk[3] = {D * 2, (uint64_t)Hkv * D * 2, (uint64_t)n_text * Hkv * D * 2};
  const uint32_t bk[4] = {64, 1, 128, 1};
  CUtensorMap tq, tkd, tvd, tk, tv;
  int r;
  if ((r = skv::encode_tmap_bf16_4d(&tq, q, dq, sq, bq)) || (r = skv::encode_tmap_bf16_4d(&tkd, L.kd, dd, sd, bd)) ||
      (r = skv::encode_tmap_bf16_4d(&tvd, L.vd, dd, sd, bd)) || (r = skv::encode_tmap_bf16_4d(&tk, k, dk, sk, bk)) ||
      (r = skv::encode_tmap_bf16_4d(&tv, v, dk, sk, bk)))
    return set_err(h, STATEKV_ERR_CUDA, "TMA tensor map encoding failed (CUresult %d)", r);
  {
    StageScope sc(h, st, STATEKV_STAGE_DECODE);
    if ((e = skv::launch_attn_tc(tq, tkd, tvd, tk, tv, ta, d, st)) != cudaSuccess) return launch_err(h, e, "decode");
    sc.done();
  }
  if (split > 1) {
    StageScope sc(h, st, STATEKV_STAGE_DECODE_COMBINE);
    if ((e = skv::launch_attn_merge_wide(ta, d, h->n_sm, st, true)) != cudaSuccess) return launch_err(h, e, "decode merge");
    sc.done();
  }
  return STATEKV_OK;
}

int statekv_get_compressed(statekv_t h, int layer, const void** k, const void** v, const int32_t** pos,
                           const float** score, int* len) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (layer < 0 || (size_t)layer >= h->layers.size() || !h->layers[layer].ready)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "unknown layer %d", layer);
  const LayerState& L = h->layers[layer];
  if (k) *k = L.kc[L.cur];
  if (v) *v = L.vc[L.cur];
  if (pos) *pos = L.posc[L.cur];
  if (score) *score = L.scorec[L.cur];
  if (len) *len = L.m;
  return STATEKV_OK;
}

int statekv_get_detailed(statekv_t h, int layer, const void** k, const void** v, const int32_t** pos,
                         int* len) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (layer < 0 || (size_t)layer >= h->layers.size() || !h->layers[layer].ready)
    return set_err(h, STATEKV_ERR_INVALID_ARG, "unknown layer %d", layer);
  const LayerState& L = h->layers[layer];
  if (k) *k = L.kd;
  if (v) *v = L.vd;
  if (pos) *pos = L.posd;
  if (len) *len = L.frames * h->T;
  return STATEKV_OK;
}

int statekv_get_step_stats(statekv_t h, const float** lse, const float** pool_score, int* pool_len) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (h->last_layer < 0) return set_err(h, STATEKV_ERR_INVALID_ARG, "no step has run yet");
  const LayerState& L = h->layers[h->last_layer];
  if (lse) *lse = L.lse;
  if (pool_score) *pool_score = L.pool_score;
  if (pool_len) *pool_len = L.pool_len;
  return STATEKV_OK;
}

int statekv_profile_enable(statekv_t h, int on) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  if (on < 0 || on > 2) return set_err(h, STATEKV_ERR_INVALID_ARG, "profiling mode %d (0, 1 or 2)", on);
  if (!on) {
    for (auto& r : h->recs) {
      h->ev_free.push_back(r.a);
      h->ev_free.push_back(r.b);
    }
    h->recs.clear();
  }
  h->prof = on;
  return STATEKV_OK;
}

int statekv_profile_read(statekv_t h, double* ms, long long* launches) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  double acc[STATEKV_N_STAGES] = {0};
  long long cnt[STATEKV_N_STAGES] = {0};
  int rc = STATEKV_OK;
  for (auto& r : h->recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess && rc == STATEKV_OK)
      rc = set_err(h, STATEKV_ERR_CUDA, "event timing failed: %s", cudaGetErrorString(e));
    acc[r.stage] += t;
    cnt[r.stage] += 1;
    h->ev_free.push_back(r.a);
    h->ev_free.push_back(r.b);
  }
  h->recs.clear();
  for (int i = 0; i < STATEKV_N_STAGES; ++i) {
    if (ms) ms[i] = acc[i];
    if (launches) launches[i] = cnt[i];
  }
  return rc;
}

long long statekv_kernel_launches(statekv_t h) { return h ? h->launches : 0; }

int statekv_device_status(statekv_t h, int* code) {
  if (!h || !code) return set_err(h, STATEKV_ERR_INVALID_ARG, "null argument");
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&v, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->dev_err, 0, sizeof(int));
  if (e != cudaSuccess) return set_err(h, STATEKV_ERR_CUDA, "status read failed: %s", cudaGetErrorString(e));
  *code = v;
  return STATEKV_OK;
}

int statekv_set_wait_limit(statekv_t h, long long ns) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  h->wait_ns = ns > 0 ? (unsigned long long)ns : 0ull;
  return STATEKV_OK;
}

int statekv_frames(statekv_t h, int layer) {
  if (!h || layer < 0 || (size_t)layer >= h->layers.size()) return 0;
  return h->layers[layer].frames;
}

int statekv_destroy(statekv_t h) {
  if (!h) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null handle");
  cudaDeviceSynchronize();
  for (auto& r : h->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (int b = 0; b < 2; ++b) {
    if (h->ev_h2d[b]) cudaEventDestroy(h->ev_h2d[b]);
    if (h->ev_step_done[b]) cudaEventDestroy(h->ev_step_done[b]);
    if (h->ev_stage_free[b]) cudaEventDestroy(h->ev_stage_free[b]);
  }
  if (h->ev_caller) cudaEventDestroy(h->ev_caller);
  for (auto& L : h->layers)
    if (L.ev_host_done) cudaEventDestroy(L.ev_host_done);
  if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
  if (h->compute_stream) cudaStreamDestroy(h->compute_stream);
  for (cudaEvent_t e : h->ev_free) cudaEventDestroy(e);
  for (void* p : h->allocs) cudaFree(p);
  if (h->dec_o) cudaFree(h->dec_o);
  if (h->dec_ml) cudaFree(h->dec_ml);
  delete h;
  return STATEKV_OK;
}

const char* statekv_last_error(statekv_t h) {
  return h ? h->err.c_str() : g_free_error.c_str();
}

int full_causal_prefill_batched(const void* q, const void* k, const void* v, int n_seq, int n_tokens,
                                int Hq, int Hkv, int d, int dtype, void* out, float* lse, void* stream) {
  if (!q || !k || !v || !out) return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "null pointer");
  if (n_seq < 1 || n_tokens < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv)
    return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "bad shape");
  if (dtype != STATEKV_BF16 && dtype != STATEKV_F32)
    return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (d != 64 && d != 128) return set_err(nullptr, STATEKV_ERR_UNSUPPORTED, "head dim %d", d);
  if (n_tokens == 0) return STATEKV_OK;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15)
    return set_err(nullptr, STATEKV_ERR_INVALID_ARG, "q/k/v/out must be 16-byte aligned");
  if (dtype == STATEKV_BF16) return full_causal_tc(q, k, v, n_seq, n_tokens, Hq, Hkv, d, out, lse,
                                                   static_cast<cudaStream_t>(stream));
  skv::AttnArgs aa{};
  aa.q = q;
  aa.q_s = (long long)n_tokens * Hq * d;
  aa.q_row = Hq * d;
  aa.ka = k;
  aa.va = v;
  aa.a_s = 0;
  aa.a_g = 0;
  aa.m = 0;
  aa.kb = k;
  aa.vb = v;
  aa.b_s = (long long)n_tokens * Hkv * d;
  aa.b_row = Hkv * d;
  aa.nb = n_tokens;
  aa.out = out;
  aa.lse = lse;
  aa.lse_s = (long long)Hq * n_tokens;
  aa.n_rows = n_tokens;
  aa.Hq = Hq;
  aa.Hkv = Hkv;
  aa.causal = 1;
  aa.scale_log2 = skv::kLog2e / sqrtf((float)d);
  cudaError_t e = skv::launch_attn_simt(aa, dtype, d, n_seq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return set_err(nullptr, STATEKV_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(e));
  return STATEKV_OK;
}

int full_causal_prefill(const void* q, const void* k, const void* v, int n_tokens, int Hq, int Hkv, int d,
                        int dtype, void* out, float* lse, void* stream) {
  return full_causal_prefill_batched(q, k, v, 1, n_tokens, Hq, Hkv, d, dtype, out, lse, stream);
}

}  // extern "C"
