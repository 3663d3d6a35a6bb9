// Top-B selection of the candidate pool and the compaction of the kept rows
// into the next compressed state, plus the append of the frame to the detailed
// state.
//
// "Linear Scaling Video VLMs for Long Video Understanding", P1 section
// 方法步骤详情: the candidate pool is the previous compressed state plus every
// token of the current frame; the top-B candidates by score update the
// compressed state; the frame's KV pairs are added to the detailed state.
// P2 section 3.3: selection refreshes the capacity-limited state; virtual
// positions are kept.  Ties go to the lower original position and the kept
// set is stored in ascending position (the pool is already in that order:
// C_{n-1} is, and every frame position exceeds all earlier ones).
#include "common.cuh"
#include "kernels.h"
#include "merge.cuh"

namespace skv {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

__device__ __forceinline__ uint32_t score_bits(float x) {
  // scores are sums of exponentials: >= +0, so the IEEE bit pattern orders
  // them like the values
  return __float_as_uint(x);
}

// Block-wide exclusive scan of one 32-bit value per thread.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSelWarps ? warp_tot[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += n;
    }
    if (lane < kSelWarps) warp_tot[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  uint32_t r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------- select
//
// One block per (stream, selection group).  The pool's scores are staged in
// shared memory as their float32 bit patterns (scores are sums of
// exponentials, >= +0, so the bit patterns order like the values; in recency
// mode the non-negative positions take their place).  The threshold tau (the
// B-th largest value) is found by histogram refinement: the values still in
// play span [umin, umax]; a 4096-bin histogram over that span (bin width
// 2^shift) locates the bin holding the B-th largest; the bin becomes the new
// span.  As soon as that bin is one value wide (tau found), is kept whole
// (tau just below it), or holds at most 32 candidates, the refinement stops;
// in the last case one warp ranks those candidates exactly by (value desc,
// pool index asc).  The result is (tau, need_eq): keep
// every candidate above tau and the first need_eq candidates equal to tau in
// pool order, which is position order, so ties go to the lower position.
constexpr int kBins = 4096;
static_assert(kBins == 4 * kSelThreads, "each thread clears and scans four bins");

struct SelShared {
  alignas(16) uint32_t hist[kBins];
  uint32_t warp_a[kSelWarps];
  uint32_t warp_b[kSelWarps];
  uint32_t list_j[32];
  uint32_t list_u[32];
  uint32_t list_n;
  uint32_t sel_bin, sel_above;
  uint32_t vmin, vmax, total;
  uint32_t tau, need_eq;
};

__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) { return __reduce_min_sync(0xffffffffu, v); }
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xffffffffu, v); }

__global__ void __launch_bounds__(kSelThreads) select_topb_kernel(SelectArgs a) {
  extern __shared__ uint32_t su[];  // [L] value bits
  __shared__ SelShared sh;
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.x >= a.n_sel_blocks) {
    // extra blocks: merge of the attention's key-split partials
    const long long t = (long long)(blockIdx.x - a.n_sel_blocks) * kSelThreads + threadIdx.x;
    if (a.mrg.d == 128) merge_chunk<128>(a.mrg, t);
    else merge_chunk<64>(a.mrg, t);
    return;
  }
  const int n_groups = a.global ? 1 : a.Hkv;
  const int grp = blockIdx.x % n_groups, s = blockIdx.x / n_groups;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = a.m + a.T;
  const int G0 = a.global ? 0 : grp;
  const int G1 = a.global ? a.Hkv : grp + 1;

  // 1. scores of the pool: the KV groups' partial sums added in a fixed order
  //    (ascending group), written out as the pool scores and staged as bits
  const float* __restrict__ part = a.part + s * a.part_s;
  float* pool_score = a.pool_score + s * a.pool_s + (long long)G0 * a.part_g;
  // rows of part summed for this group: the KV groups' (and within a group the
  // query-row splits') partial sums, in ascending row order
  const int R0 = G0 * a.n_qsplit, R1 = G1 * a.n_qsplit;
  uint32_t tmin = 0xffffffffu, tmax = 0u;  // span of this thread's staged values (first level)
  if ((a.part_g & 3) == 0 && (reinterpret_cast<uintptr_t>(part) & 15) == 0) {
    // four consecutive candidates per thread and group as one 16-byte load
    const int n4 = (L + 3) / 4;
    // one row's four candidates at j0 (zeros past the pool or past row R1)
    auto load4 = [&](int j0, int row, float4& x) {
      x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row < R1 && j0 < L) {
        const float* src = part + (long long)row * a.part_g + j0;
        if (j0 + 3 < L) {
          x = __ldg(reinterpret_cast<const float4*>(src));
        } else {
          x.x = __ldg(src);
          if (j0 + 1 < L) x.y = __ldg(src + 1);
          if (j0 + 2 < L) x.z = __ldg(src + 2);
        }
      }
    };
    auto add4 = [](float4& v, const float4& x) {
      v.x += x.x;
      v.y += x.y;
      v.z += x.z;
      v.w += x.w;
    };
    // the four candidates' scores out, their bits staged, the span updated
    auto finish = [&](int j0, const float4& v) {
      if (j0 + 3 < L && (reinterpret_cast<uintptr_t>(pool_score) & 15) == 0) {
        *reinterpret_cast<float4*>(pool_score + j0) = v;
        if (!a.recency) {
          const uint4 b4 = make_uint4(score_bits(v.x), score_bits(v.y), score_bits(v.z), score_bits(v.w));
          *reinterpret_cast<uint4*>(su + j0) = b4;
          tmin = min(min(tmin, min(b4.x, b4.y)), min(b4.z, b4.w));
          tmax = max(max(tmax, max(b4.x, b4.y)), max(b4.z, b4.w));
        }
      } else {
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (j0 + e < L) {
            pool_score[j0 + e] = vv[e];
            if (!a.recency) {
              const uint32_t b = score_bits(vv[e]);
              su[j0 + e] = b;
              tmin = min(tmin, b);
              tmax = max(tmax, b);
            }
          }
        }
      }
    };
    if (R1 - R0 <= 4) {
      // at most four rows: two columns per thread, all eight loads in one
      // round (rows added in ascending order, as below)
      for (int c = threadIdx.x; c < n4; c += 2 * kSelThreads) {
        const int c1 = c + kSelThreads;
        float4 x[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          load4(4 * c, R0 + u, x[u]);
          load4(4 * c1, R0 + u, x[4 + u]);
        }
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          add4(v0, x[u]);
          add4(v1, x[4 + u]);
        }
        finish(4 * c, v0);
        if (c1 < n4) finish(4 * c1, v1);
      }
    } else {
      for (int c = threadIdx.x; c < n4; c += kSelThreads) {
        const int j0 = 4 * c;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int gb = R0; gb < R1; gb += 8) {
          float4 x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) load4(j0, gb + u, x[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) add4(v, x[u]);
        }
        finish(j0, v);
      }
    }
  } else {
    for (int j = threadIdx.x; j < L; j += kSelThreads) {
      float v = 0.f;
      for (int g = R0; g < R1; ++g) v += __ldg(part + (long long)g * a.part_g + j);
      pool_score[j] = v;
      if (!a.recency) {
        const uint32_t b = score_bits(v);
        su[j] = b;
        tmin = min(tmin, b);
        tmax = max(tmax, b);
      }
    }
  }
  if (a.recency) {
    // recency retention ranks by position: the bit pattern of a non-negative
    // int32 orders like its value, and positions are distinct (no ties).  The
    // score loops above leave su alone in this mode: each word of su is written
    // by one thread only (they map candidates to threads differently).
    const int* __restrict__ pos_c = a.pos_c + ((long long)s * a.Hkv + G0) * a.B;
    const int* __restrict__ pos_f = a.pos_f + (long long)s * a.T;
    for (int j = threadIdx.x; j < L; j += kSelThreads) {
      const uint32_t b = (uint32_t)max(j < a.m ? __ldg(pos_c + j) : __ldg(pos_f + (j - a.m)), 0);
      su[j] = b;
      tmin = min(tmin, b);
      tmax = max(tmax, b);
    }
  }
  // the first level of the threshold search takes its span from here
  reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
  tmin = warp_min_u32(tmin);
  tmax = warp_max_u32(tmax);
  if (lane == 0) {
    sh.warp_a[warp] = tmin;
    sh.warp_b[warp] = tmax;
  }
  __syncthreads();
  if (a.B <= 0) return;  // nothing is kept (block-uniform)

  // 2. threshold.  Shared memory serves one warp-wide access per clock, so
  //    block-wide results are reduced by one warp and read once per thread.
  const bool keep_all = L <= a.B;
  uint32_t tau = 0, need_eq = 0;
  if (!keep_all) {
    uint32_t lo = 0, hi = 0xffffffffu;  // span of the values still in play (inclusive)
    uint32_t need = (uint32_t)a.B;      // how many of them are kept
    for (int level = 0;; ++level) {
      // exact span of the values in play; the histogram is cleared meanwhile
      // (the first level's span and cleared histogram come from the load)
      uint32_t vmin = 0xffffffffu, vmax = 0u;
      if (level > 0) {
        for (int j = threadIdx.x; j < L; j += kSelThreads) {
          const uint32_t u = su[j];
          if (u >= lo && u <= hi) {
            vmin = min(vmin, u);
            vmax = max(vmax, u);
          }
        }
        reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
        vmin = warp_min_u32(vmin);
        vmax = warp_max_u32(vmax);
        if (lane == 0) {
          sh.warp_a[warp] = vmin;
          sh.warp_b[warp] = vmax;
        }
        __syncthreads();
      }
      if (warp == 0) {
        const uint32_t m0 = warp_min_u32(sh.warp_a[lane]), m1 = warp_max_u32(sh.warp_b[lane]);
        if (lane == 0) {
          sh.vmin = m0;
          sh.vmax = m1;
        }
      }
      __syncthreads();
      vmin = sh.vmin;
      vmax = sh.vmax;
      if (vmin == vmax) {  // every value in play is equal: it is tau
        tau = vmin;
        need_eq = need;
        break;
      }
      const uint32_t span = vmax - vmin;
      const int shift = max(0, 32 - __clz(span) - 12);  // (span >> shift) < kBins
      // histogram of the values in play (shared atomics; lanes of a warp that
      // hit one bin are serialised by the hardware)
      for (int j = threadIdx.x; j < L; j += kSelThreads) {
        const uint32_t u = su[j];
        if (u >= vmin && u <= vmax) atomicAdd(&sh.hist[(u - vmin) >> shift], 1u);
      }
      __syncthreads();
      // thread t owns bins [4t, 4t + 4): a block prefix sum (warp shuffles, then
      // warp 0 over the 32 warp totals) gives the values in bins below 4t; the
      // bin where the count from the top first reaches `need` holds the need-th
      // largest
      const uint4 h4 = reinterpret_cast<const uint4*>(sh.hist)[threadIdx.x];
      const uint32_t mine = h4.x + h4.y + h4.z + h4.w;
      uint32_t incl = mine;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      if (lane == 31) sh.warp_a[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        const uint32_t w = sh.warp_a[lane];
        uint32_t wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t n = __shfl_up_sync(0xffffffffu, wi, off);
          if (lane >= off) wi += n;
        }
        sh.warp_b[lane] = wi - w;  // values in the bins of lower warps
        if (lane == 31) sh.total = wi;
      }
      if (threadIdx.x == 0) sh.list_n = 0u;
      __syncthreads();
      const uint32_t total = sh.total;
      {
        const uint32_t hh[4] = {h4.x, h4.y, h4.z, h4.w};
        uint32_t below = sh.warp_b[warp] + incl - mine;  // values in bins below 4t
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t ge = total - below;  // values in bins >= 4t + e
          const uint32_t gt = ge - hh[e];     // values in bins > 4t + e
          if (ge >= need && gt < need) {
            sh.sel_bin = 4 * threadIdx.x + e;
            sh.sel_above = gt;
          }
          below += hh[e];
        }
      }
      __syncthreads();
      const uint32_t b = sh.sel_bin;
      const uint32_t in_bin = sh.hist[b];
      need -= sh.sel_above;
      lo = vmin + (b << shift);
      hi = shift == 0 ? lo : (uint32_t)min((unsigned long long)vmax, (unsigned long long)lo + (1ull << shift) - 1ull);
      if (shift == 0) {  // the bin is one value
        tau = lo;
        need_eq = need;
        break;
      }
      if (in_bin == need && lo > 0u) {
        // every candidate of the bin is kept: the kept set is every value
        // >= lo, with no tie to break (equal values share a bin)
        tau = lo - 1u;
        need_eq = 0u;
        break;
      }
      if (in_bin <= 32u) {
        // rank the bin's candidates exactly in one warp: order (value desc,
        // pool index asc); the need-th is tau, the kept ties are the
        // candidates equal to it ranked up to it
        for (int j = threadIdx.x; j < L; j += kSelThreads) {
          const uint32_t u = su[j];
          if (u >= lo && u <= hi) {
            const uint32_t slot = atomicAdd(&sh.list_n, 1u);
            sh.list_j[slot] = (uint32_t)j;
            sh.list_u[slot] = u;
          }
        }
        __syncthreads();
        if (warp == 0) {
          const uint32_t n = sh.list_n;
          const bool have = (uint32_t)lane < n;
          const uint32_t uj = have ? sh.list_u[lane] : 0u, jj = have ? sh.list_j[lane] : 0xffffffffu;
          uint32_t rank = 0;
          for (uint32_t k = 0; k < n; ++k) {
            const uint32_t uk = __shfl_sync(0xffffffffu, uj, k), jk = __shfl_sync(0xffffffffu, jj, k);
            rank += (uk > uj || (uk == uj && jk < jj)) ? 1u : 0u;
          }
          const uint32_t tmask = __ballot_sync(0xffffffffu, have && rank == need - 1);
          const uint32_t t = __shfl_sync(0xffffffffu, uj, __ffs(tmask) - 1);
          const uint32_t eq = __popc(__ballot_sync(0xffffffffu, have && uj == t && rank < need));
          if (lane == 0) {
            sh.tau = t;
            sh.need_eq = eq;
          }
        }
        __syncthreads();
        tau = sh.tau;
        need_eq = sh.need_eq;
        break;
      }
      __syncthreads();  // the bin's count and sel_* are read before the next level rewrites them
    }
  }

  // 3. compaction in pool (= position) order with one block-wide scan: thread
  //    t owns the consecutive candidates [t*C, t*C + C); the scan of its
  //    (greater, tied) counts gives its first output slot and how many tied
  //    candidates precede it, so the first need_eq ties in pool order are kept
  const int C = (L + kSelThreads - 1) / kSelThreads;
  const int j_lo = min(L, threadIdx.x * C), j_hi = min(L, j_lo + C);
  uint32_t n_gt = 0, n_eq = 0;
  for (int j = j_lo; j < j_hi; ++j) {
    if (keep_all) {
      ++n_gt;
    } else {
      const uint32_t u = su[j];
      n_gt += u > tau;
      n_eq += u == tau;
    }
  }
  __syncthreads();  // warp_a is reused by the scan
  const uint32_t packed = block_exclusive_scan(n_gt | (n_eq << 16), sh.warp_a);
  uint32_t eq_seen = packed >> 16;                                      // tied candidates before j_lo
  int dst = (int)(packed & 0xffffu) + (int)min(eq_seen, need_eq);       // kept candidates before j_lo
  int32_t* idx = a.idx + ((long long)s * a.Hkv + G0) * a.B;
  // Scattered 4-byte global stores cost several thousand cycles here; when B
  // fits the (now unused) histogram, the kept indices are placed there and
  // copied out with coalesced stores.
  const bool stage = a.B <= kBins;
  for (int j = j_lo; j < j_hi; ++j) {
    bool keep;
    if (keep_all) {
      keep = true;
    } else {
      const uint32_t u = su[j];
      keep = u > tau;
      if (u == tau) keep = eq_seen++ < need_eq;
    }
    if (keep) {
      if (dst < a.B) {
        if (stage) sh.hist[dst] = (uint32_t)j;
        else idx[dst] = j;
      }
      ++dst;
    }
  }
  if (stage) {
    __syncthreads();
    const int n_kept = min(a.B, L);
    for (int r = threadIdx.x; r < n_kept; r += kSelThreads) idx[r] = (int32_t)sh.hist[r];
  }
}

// ---------------------------------------------------------------- gather
//
// Warp tasks of R rows: a task copies R output rows of one (stream, KV head)
// -- K and V, VPR 16-byte vectors per row each -- so every lane moves four
// vectors, all four loads issued before any store.  Tasks [0, n_c) build C_n:
// the rows' kept pool indices are loaded once per task by R lanes and
// broadcast; tasks [n_c, n_c + n_d) append R frame tokens of one KV head to D.
template <int VPR>
struct GatherShape {
  static constexpr int kR = 64 / VPR;  // rows per task (four vectors per lane)
  static constexpr int kU = 4;
};

template <int VPR>
__global__ void __launch_bounds__(256) gather_append_kernel(GatherArgs a, int n_c_tasks, int n_tasks) {
  constexpr int R = GatherShape<VPR>::kR, U = GatherShape<VPR>::kU;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int c_blocks = (a.m_new + R - 1) / R;   // C tasks per (stream, KV head)
  const int d_blocks = (a.T + R - 1) / R;       // D tasks per (stream, KV head)
  for (int task = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < n_tasks; task += warps_total) {
    const bool is_c = task < n_c_tasks;
    const int t2 = is_c ? task : task - n_c_tasks;
    const int per = is_c ? c_blocks : d_blocks;
    const int sg = t2 / per;                     // s * Hkv + g
    const int r0 = (t2 - sg * per) * R;
    const int g = sg % a.Hkv, s = sg / a.Hkv;
    const int n_rows = min(R, (is_c ? a.m_new : a.T) - r0);
    const int4* src[U];
    int4* dst[U];
    bool ok[U];
    if (is_c) {
      const int gsel = a.global ? 0 : g;
      int j = -1;
      if (lane < n_rows) {
        j = __ldg(a.idx + ((long long)s * a.Hkv + gsel) * a.B + r0 + lane);
        if (j < 0 || j >= a.m + a.T) j = -1;  // never taken for a well-formed kept list
        if (j >= 0) {
          a.pos_new[(long long)sg * a.B + r0 + lane] =
              j < a.m ? __ldg(a.pos_c + (long long)sg * a.B + j) : __ldg(a.pos_f + (long long)s * a.T + (j - a.m));
          a.score_new[(long long)sg * a.B + r0 + lane] =
              __ldg(a.pool_score + ((long long)s * a.Hkv + gsel) * a.pool_g + j);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = lane + 32 * u;
        const int rl = e / (2 * VPR), w = e % (2 * VPR);
        const bool isv = w >= VPR;
        const int col = isv ? w - VPR : w;
        const int jr = __shfl_sync(0xffffffffu, j, rl);
        ok[u] = rl < n_rows && jr >= 0;
        const char* sb;
        if (jr < a.m) sb = static_cast<const char*>(isv ? a.vc : a.kc) + ((long long)sg * a.B + jr) * a.row_bytes;
        else sb = static_cast<const char*>(isv ? a.vf : a.kf) + (((long long)s * a.T + (jr - a.m)) * a.Hkv + g) * a.row_bytes;
        src[u] = reinterpret_cast<const int4*>(sb) + col;
        dst[u] = reinterpret_cast<int4*>(static_cast<char*>(isv ? a.vc_new : a.kc_new) +
                                         ((long long)sg * a.B + r0 + rl) * a.row_bytes) + col;
      }
    } else {
      if (g == 0 && lane < n_rows)
        a.pos_d[(long long)s * a.max_tok + a.d_len + r0 + lane] = __ldg(a.pos_f + (long long)s * a.T + r0 + lane);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = lane + 32 * u;
        const int rl = e / (2 * VPR), w = e % (2 * VPR);
        const bool isv = w >= VPR;
        const int col = isv ? w - VPR : w;
        const int t = r0 + rl;
        ok[u] = rl < n_rows;
        src[u] = reinterpret_cast<const int4*>(static_cast<const char*>(isv ? a.vf : a.kf) +
                                               (((long long)s * a.T + t) * a.Hkv + g) * a.row_bytes) + col;
        dst[u] = reinterpret_cast<int4*>(static_cast<char*>(isv ? a.vd : a.kd) +
                                         (((long long)s * a.Hkv + g) * a.max_tok + a.d_len + t) * a.row_bytes) + col;
      }
    }
    int4 x[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (ok[u]) x[u] = __ldg(src[u]);
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (ok[u]) *dst[u] = x[u];
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a_in, int S, cudaStream_t st, bool pdl) {
  SelectArgs a = a_in;
  const int L = a.m + a.T;
  const int n_groups = a.global ? 1 : a.Hkv;
  a.n_sel_blocks = n_groups * S;
  if (a.mrg.n_split > 1) {
    const long long mrg_threads = merge_threads((long long)a.mrg.S * a.mrg.Hq * a.mrg.T, a.mrg.d);
    a.n_mrg_blocks = (int)((mrg_threads + kSelThreads - 1) / kSelThreads);
  } else {
    a.n_mrg_blocks = 0;
  }
  const size_t smem = (size_t)L * sizeof(uint32_t);
  // the default 48 KB per block covers static and dynamic shared memory
  // together; the kernel's static arrays take ~19 KB, so opt in above 24 KB
  if (smem > 24 * 1024) {
    cudaError_t e = ensure_dynamic_smem(select_topb_kernel, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(select_topb_kernel, dim3(a.n_sel_blocks + a.n_mrg_blocks), dim3(kSelThreads), smem, st,
                       pdl, a);
}

template <int VPR>
static cudaError_t launch_gather_vpr(const GatherArgs& a, int n_sm, cudaStream_t st, bool pdl) {
  constexpr int R = GatherShape<VPR>::kR;
  const int per_c = (a.m_new + R - 1) / R, per_d = (a.T + R - 1) / R;
  const long long n_c = (long long)a.S * a.Hkv * per_c;
  const long long n_tasks = n_c + (long long)a.S * a.Hkv * per_d;
  if (n_tasks == 0) return cudaSuccess;
  long long blocks = (n_tasks + 7) / 8;        // eight warps per block
  const long long cap = (long long)n_sm * 8;   // one resident wave
  if (blocks > cap) blocks = cap;
  return launch_kernel(gather_append_kernel<VPR>, dim3((unsigned)blocks), dim3(256), 0, st, pdl, a, (int)n_c,
                       (int)n_tasks);
}

cudaError_t launch_gather(const GatherArgs& a, int n_sm, cudaStream_t st, bool pdl) {
  switch (a.row_bytes / 16) {
    case 8: return launch_gather_vpr<8>(a, n_sm, st, pdl);
    case 16: return launch_gather_vpr<16>(a, n_sm, st, pdl);
    case 32: return launch_gather_vpr<32>(a, n_sm, st, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace skv
