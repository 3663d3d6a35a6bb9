// statekv_step_noalloc: one StateKV step that allocates no device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the step: an
// inference server or video pipeline that has already reserved nearly all of
// the GPU's memory for its own pool (so a library allocation would fail or
// break the pool's accounting), or a latency-critical loop in which
// cudaMalloc's implicit device-wide synchronisation is not acceptable.  This
// entry point takes every input and output from the caller (including C and
// D) and keeps its per-step scratch (row log-sum-exps, partial and pool
// scores, the kept index list) in one file-scope device array of fixed size.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "statekv.h"
#include "kernels.h"

namespace {

// Scratch shared by every call on a device; every GPU that loads the library
// holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device (the host-side
// name of the array is not a device address).
constexpr int kMaxDevices = 64;
std::once_flag g_setup_once[kMaxDevices];
void* g_scratch_addr[kMaxDevices];
cudaError_t g_setup_status[kMaxDevices];

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  skv::set_free_error(buf);
  return code;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" int statekv_step_noalloc(int Hq, int Hkv, int d, int T, int B, int dtype, int mask_mode,
                                    int select_mode, const void* q, const void* k, const void* v,
                                    const int32_t* pos, const void* kc, const void* vc,
                                    const int32_t* posc, int m, void* out, void* kc_new,
                                    void* vc_new, int32_t* posc_new, float* scorec_new, void* kd,
                                    void* vd, int32_t* posd, int d_len, int max_tok, void* stream) {
  if (Hq < 1 || Hkv < 1 || T < 1 || B < 0 || Hq % Hkv != 0)
    return fail(STATEKV_ERR_INVALID_ARG, "bad shape Hq=%d Hkv=%d T=%d B=%d", Hq, Hkv, T, B);
  if (d != 64 && d != 128) return fail(STATEKV_ERR_UNSUPPORTED, "head dim %d not in {64,128}", d);
  if (dtype != STATEKV_BF16 && dtype != STATEKV_F32) return fail(STATEKV_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (mask_mode != STATEKV_MASK_FRAME_CAUSAL && mask_mode != STATEKV_MASK_FRAME_BIDIR)
    return fail(STATEKV_ERR_INVALID_ARG, "bad mask_mode %d", mask_mode);
  if (select_mode != STATEKV_SELECT_GLOBAL && select_mode != STATEKV_SELECT_PER_KV_HEAD &&
      select_mode != STATEKV_SELECT_RECENCY)
    return fail(STATEKV_ERR_INVALID_ARG, "bad select_mode %d", select_mode);
  if (m < 0 || m > B) return fail(STATEKV_ERR_INVALID_ARG, "C length m=%d outside [0, B=%d]", m, B);
  if (d_len < 0 || (long long)d_len + T > max_tok)
    return fail(STATEKV_ERR_CAPACITY, "D holds %d tokens; appending %d at %d does not fit", max_tok, T, d_len);
  // scratch carve-up: lse [Hq][T], partial and pool scores [Hkv][B+T], kept [Hkv][B]
  const size_t pool = (size_t)B + T;
  const size_t lse_b = round256((size_t)Hq * T * 4);
  const size_t part_b = round256((size_t)Hkv * pool * 4);
  const size_t idx_b = round256((size_t)Hkv * (B > 0 ? B : 1) * 4);
  const size_t need = lse_b + 2 * part_b + idx_b;
  if (need > kNoAllocScratchBytes || pool > 28672)
    return fail(STATEKV_ERR_UNSUPPORTED,
                "shape needs %zu bytes of step scratch; statekv_step_noalloc has %zu (use statekv_create)",
                need, kNoAllocScratchBytes);

  if (!q || !k || !v || !pos || !out || !kc || !vc || !posc || !kc_new || !vc_new || !posc_new ||
      !scorec_new || !kd || !vd || !posd)
    return fail(STATEKV_ERR_INVALID_ARG, "null pointer argument");
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out | (uintptr_t)kc | (uintptr_t)vc |
       (uintptr_t)kc_new | (uintptr_t)vc_new | (uintptr_t)kd | (uintptr_t)vd) & 15)
    return fail(STATEKV_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (((uintptr_t)pos | (uintptr_t)posc | (uintptr_t)posc_new | (uintptr_t)scorec_new | (uintptr_t)posd) & 3)
    return fail(STATEKV_ERR_INVALID_ARG, "position and score pointers must be 4-byte aligned");

  // Every output range must be disjoint from every input range and from the
  // other outputs: the kernels read C_{n-1} and the frame while they write C_n
  // (another thread's row may be overwritten before it is read).  D is read
  // only in its appended region, which is an output.
  const size_t es = dtype == STATEKV_BF16 ? 2 : 4;
  const size_t cb = (size_t)Hkv * B * d * es, ci = (size_t)Hkv * B * 4;
  const size_t qb = (size_t)T * Hq * d * es, kb = (size_t)T * Hkv * d * es;
  const size_t db = (size_t)Hkv * max_tok * d * es, dpb = (size_t)max_tok * 4;
  struct Range {
    const void* p;
    size_t n;
    const char* name;
  };
  const Range outs[] = {{out, qb, "out"}, {kc_new, cb, "kc_new"}, {vc_new, cb, "vc_new"},
                        {posc_new, ci, "posc_new"}, {scorec_new, ci, "scorec_new"},
                        {kd, db, "kd"}, {vd, db, "vd"}, {posd, dpb, "posd"}};
  const Range ins[] = {{q, qb, "q"}, {k, kb, "k"}, {v, kb, "v"}, {pos, (size_t)T * 4, "pos"},
                       {kc, cb, "kc"}, {vc, cb, "vc"}, {posc, ci, "posc"}};
  auto overlap = [](const Range& x, const Range& y) {
    const uintptr_t a0 = (uintptr_t)x.p, b0 = (uintptr_t)y.p;
    return x.n > 0 && y.n > 0 && a0 < b0 + y.n && b0 < a0 + x.n;
  };
  for (const Range& o : outs) {
    for (const Range& i : ins)
      if (overlap(o, i)) return fail(STATEKV_ERR_INVALID_ARG, "output %s overlaps input %s", o.name, i.name);
    for (const Range& o2 : outs)
      if (&o2 < &o && overlap(o, o2))
        return fail(STATEKV_ERR_INVALID_ARG, "outputs %s and %s overlap", o2.name, o.name);
  }

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(STATEKV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(STATEKV_ERR_UNSUPPORTED, "device index %d", dev);
  std::call_once(g_setup_once[dev], [dev] {
    void* p = nullptr;
    g_setup_status[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_scratch_addr[dev] = p;
  });
  if (g_setup_status[dev] != cudaSuccess)
    return fail(STATEKV_ERR_CUDA, "cudaGetSymbolAddress of the scratch array: %s",
                cudaGetErrorString(g_setup_status[dev]));
  unsigned char* base = static_cast<unsigned char*>(g_scratch_addr[dev]);
  float* lse = reinterpret_cast<float*>(base);
  float* part = reinterpret_cast<float*>(base + lse_b);
  float* pool_score = reinterpret_cast<float*>(base + lse_b + part_b);
  int32_t* idx = reinterpret_cast<int32_t*>(base + lse_b + 2 * part_b);
  // Nothing here must start at zero: every kernel writes each scratch entry it
  // later reads (lse rows, partials j < m+T, kept slots < min(B, m+T)).

  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale_log2 = skv::kLog2e / sqrtf((float)d);
  const int causal = mask_mode == STATEKV_MASK_FRAME_CAUSAL;
  const int global = select_mode != STATEKV_SELECT_PER_KV_HEAD;
  const int m_new = m + T < B ? m + T : B;

  skv::AttnArgs aa{};
  aa.q = q;
  aa.q_s = (long long)T * Hq * d;
  aa.q_row = Hq * d;
  aa.ka = kc;
  aa.va = vc;
  aa.a_s = (long long)Hkv * B * d;
  aa.a_g = (long long)B * d;
  aa.m = m;
  aa.kb = k;
  aa.vb = v;
  aa.b_s = (long long)T * Hkv * d;
  aa.b_row = Hkv * d;
  aa.nb = T;
  aa.out = out;
  aa.lse = lse;
  aa.lse_s = (long long)Hq * T;
  aa.n_rows = T;
  aa.Hq = Hq;
  aa.Hkv = Hkv;
  aa.causal = causal;
  aa.scale_log2 = scale_log2;
  if ((e = skv::launch_attn_simt(aa, dtype, d, 1, st)) != cudaSuccess)
    return fail(STATEKV_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));

  skv::ScoreArgs sa{};
  sa.q = q;
  sa.q_s = aa.q_s;
  sa.q_row = aa.q_row;
  sa.ka = kc;
  sa.a_s = aa.a_s;
  sa.a_g = aa.a_g;
  sa.m = m;
  sa.kb = k;
  sa.b_s = aa.b_s;
  sa.b_row = aa.b_row;
  sa.nb = T;
  sa.lse = lse;
  sa.lse_s = aa.lse_s;
  sa.part = part;
  sa.part_s = (long long)Hkv * pool;
  sa.part_g = (int)pool;
  sa.n_rows = T;
  sa.Hq = Hq;
  sa.Hkv = Hkv;
  sa.causal = causal;
  sa.scale_log2 = scale_log2;
  if ((e = skv::launch_score_simt(sa, dtype, d, 1, st)) != cudaSuccess)
    return fail(STATEKV_ERR_CUDA, "score launch: %s", cudaGetErrorString(e));

  skv::SelectArgs se{};
  se.part = part;
  se.part_s = sa.part_s;
  se.part_g = (int)pool;
  se.n_qsplit = 1;
  se.pool_score = pool_score;
  se.pool_s = sa.part_s;
  se.pos_c = posc;
  se.pos_f = pos;
  se.idx = idx;
  se.Hkv = Hkv;
  se.m = m;
  se.T = T;
  se.B = B;
  se.global = global;
  se.recency = select_mode == STATEKV_SELECT_RECENCY;
  if ((e = skv::launch_select(se, 1, st)) != cudaSuccess)
    return fail(STATEKV_ERR_CUDA, "select launch: %s", cudaGetErrorString(e));

  skv::GatherArgs ga{};
  ga.kc = kc;
  ga.vc = vc;
  ga.kf = k;
  ga.vf = v;
  ga.kc_new = kc_new;
  ga.vc_new = vc_new;
  ga.idx = idx;
  ga.kd = kd;
  ga.vd = vd;
  ga.pos_d = posd;
  ga.pos_f = pos;
  ga.pos_c = se.pos_c;
  ga.pool_score = se.pool_score;
  ga.pos_new = posc_new;
  ga.score_new = scorec_new;
  ga.pool_g = se.part_g;
  ga.Hkv = Hkv;
  ga.T = T;
  ga.B = B;
  ga.m = m;
  ga.m_new = m_new;
  ga.row_bytes = d * (dtype == STATEKV_BF16 ? 2 : 4);
  ga.global = global;
  ga.d_len = d_len;
  ga.max_tok = max_tok;
  ga.S = 1;
  if ((e = skv::launch_gather(ga, n_sm, st)) != cudaSuccess)
    return fail(STATEKV_ERR_CUDA, "gather launch: %s", cudaGetErrorString(e));
  return STATEKV_OK;
}
