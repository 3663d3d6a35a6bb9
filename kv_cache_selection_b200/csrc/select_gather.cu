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

// One block per (selection group, stream).  Dynamic shared memory holds the
// pool's scores (L floats).  Radix select on 8-bit digits, most significant
// first; each pass is a histogram (warp-aggregated shared atomics) and a
// suffix count over the 256 bins done with warp shuffles.
// Appends frame token vectors to D: one 16-byte vector per thread.
__device__ __forceinline__ void append_vec(const SelectArgs& a, int v) {
  const int vpr = a.row_bytes / 16;
  const int per_row = 2 * vpr;  // K and V
  const int rr = v / per_row;   // (s, t, g) row of the frame
  if (rr >= a.S * a.T * a.Hkv) return;
  int e = v - rr * per_row;
  const bool isv = e >= vpr;
  if (isv) e -= vpr;
  const int g = rr % a.Hkv;
  const int st = rr / a.Hkv;  // s * T + t
  const int t = st % a.T, s = st / a.T;
  const long long src = (long long)rr * a.row_bytes;
  const long long dst = (((long long)s * a.Hkv + g) * a.max_tok + a.d_len + t) * a.row_bytes;
  const int4 x = __ldg(reinterpret_cast<const int4*>(static_cast<const char*>(isv ? a.vf : a.kf) + src) + e);
  reinterpret_cast<int4*>(static_cast<char*>(isv ? a.vd : a.kd) + dst)[e] = x;
  if (g == 0 && !isv && e == 0) a.pos_d[(long long)s * a.max_tok + a.d_len + t] = __ldg(a.pos_f + st);
}

__global__ void __launch_bounds__(kSelThreads) select_topb_kernel(SelectArgs a) {
  extern __shared__ float sc[];
  __shared__ uint32_t hist[257];
  __shared__ uint32_t bin_tot[8];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sel_bin, sel_above;
  pdl_wait();
  pdl_trigger();
  if ((int)blockIdx.x >= a.n_sel_blocks) {
    // extra blocks: D append, then the merge of key-split partials
    const int b = blockIdx.x - a.n_sel_blocks;
    if (b < a.n_app_blocks) {
      append_vec(a, b * kSelThreads + threadIdx.x);
    } else {
      const int t = (b - a.n_app_blocks) * kSelThreads + threadIdx.x;
      if (a.mrg.d == 128) merge_chunk<128>(a.mrg, t);
      else merge_chunk<64>(a.mrg, t);
    }
    return;
  }
  const int n_groups = a.global ? 1 : a.Hkv;
  const int grp = blockIdx.x % n_groups, s = blockIdx.x / n_groups;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = a.m + a.T;
  const int G0 = a.global ? 0 : grp;
  const int G1 = a.global ? a.Hkv : grp + 1;

  // 1. scores of the pool (global mode sums the KV groups in a fixed order)
  //    and the pool positions, staged in shared memory; every load of a
  //    candidate is independent of the others
  int* posp = reinterpret_cast<int*>(sc + L);
  const float* __restrict__ part = a.part + s * a.part_s;
  const int* __restrict__ pos_c = a.pos_c + ((long long)s * a.Hkv + G0) * a.B;
  const int* __restrict__ pos_f = a.pos_f + (long long)s * a.T;
  if ((a.part_g & 3) == 0 && (reinterpret_cast<uintptr_t>(part) & 15) == 0) {
    // four consecutive candidates per thread and group as one 16-byte load,
    // groups summed in the same fixed order
    const int n4 = (L + 3) / 4;
    for (int c = threadIdx.x; c < n4; c += kSelThreads) {
      const int j0 = 4 * c;
      const bool full = j0 + 3 < L;
      int pp[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + e;
        pp[e] = j < L ? (j < a.m ? __ldg(pos_c + j) : __ldg(pos_f + (j - a.m))) : 0;
      }
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      // groups in ascending order, eight loads in flight per chunk
      for (int gb = G0; gb < G1; gb += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (gb + u < G1) {
          const float* src = part + (long long)(gb + u) * a.part_g + j0;
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (full) {
            x = __ldg(reinterpret_cast<const float4*>(src));
          } else {
            x.x = __ldg(src);
            if (j0 + 1 < L) x.y = __ldg(src + 1);
            if (j0 + 2 < L) x.z = __ldg(src + 2);
          }
          v.x += x.x;
          v.y += x.y;
          v.z += x.z;
          v.w += x.w;
        }
      }
      }
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (j0 + e < L) {
          sc[j0 + e] = vv[e];
          posp[j0 + e] = pp[e];
        }
      }
    }
  } else {
    constexpr int kBatch = 4;  // candidates per thread whose loads are in flight together
    for (int jb = 0; jb < L; jb += kBatch * kSelThreads) {
      float acc[kBatch] = {};
      int pp[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int j = jb + q * kSelThreads + threadIdx.x;
        pp[q] = j < L ? (j < a.m ? __ldg(pos_c + j) : __ldg(pos_f + (j - a.m))) : 0;
      }
      // groups in ascending order, eight per chunk with their loads in flight
      for (int gb = G0; gb < G1; gb += 8) {
        float pv[kBatch][8];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int j = jb + q * kSelThreads + threadIdx.x;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            pv[q][u] = (j < L && gb + u < G1) ? __ldg(part + (long long)(gb + u) * a.part_g + j) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q)
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[q] += pv[q][u];
      }
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int j = jb + q * kSelThreads + threadIdx.x;
        if (j < L) {
          sc[j] = acc[q];
          posp[j] = pp[q];
        }
      }
    }
  }
  for (int b = threadIdx.x; b < 257; b += kSelThreads) hist[b] = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < L; j += kSelThreads) {
    a.pool_score[s * a.part_s + (long long)G0 * a.part_g + j] = sc[j];
    // recency retention ranks by position: the bit pattern of a non-negative
    // int32 orders like its value, and positions are distinct (no ties)
    if (a.recency) sc[j] = __int_as_float(max(posp[j], 0));
  }
  if (a.recency) __syncthreads();
  if (a.B <= 0) return;  // nothing is kept (block-uniform)

  // 2. threshold: the B-th largest score
  uint32_t tau = 0;
  int need_eq = 0;  // how many candidates equal to tau are kept
  const bool keep_all = L <= a.B;
  if (!keep_all) {
    uint32_t prefix = 0, pmask = 0;
    int k = a.B;
    const int n_iter = (L + kSelThreads - 1) / kSelThreads;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int it = 0; it < n_iter; ++it) {
        const int j = it * kSelThreads + threadIdx.x;
        // only candidates that still match the prefix are counted; warps with
        // none (most of them after the first passes) skip the match entirely
        bool match = false;
        uint32_t digit = 0;
        if (j < L) {
          const uint32_t u = score_bits(sc[j]);
          match = (u & pmask) == prefix;
          digit = (u >> shift) & 255u;
        }
        const uint32_t act = __ballot_sync(0xffffffffu, match);
        if (match) {
          const uint32_t peers = __match_any_sync(act, digit);
          if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
        }
      }
      __syncthreads();
      // suffix counts: warp w < 8 owns bins [32w, 32w+32)
      uint32_t suf = 0;
      if (warp < 8) {
        suf = hist[warp * 32 + lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          uint32_t n = __shfl_down_sync(0xffffffffu, suf, off);
          if (lane + off < 32) suf += n;
        }
        if (lane == 0) bin_tot[warp] = suf;  // all bins of this warp
      }
      __syncthreads();
      if (warp < 8) {
        uint32_t higher = 0;  // candidates in bins of higher warps
        for (int w2 = warp + 1; w2 < 8; ++w2) higher += bin_tot[w2];
        const uint32_t ge = suf + higher;                                   // digit >= bin
        const uint32_t gt = ge - hist[warp * 32 + lane];                    // digit > bin
        if (ge >= (uint32_t)k && gt < (uint32_t)k) {
          sel_bin = warp * 32 + lane;
          sel_above = gt;
        }
      }
      __syncthreads();
      const uint32_t b = sel_bin;
      k -= (int)sel_above;
      prefix |= b << shift;
      pmask |= 255u << shift;
      for (int bb = threadIdx.x; bb < 257; bb += kSelThreads) hist[bb] = 0;
      __syncthreads();
    }
    tau = prefix;
    need_eq = k;
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
      const uint32_t u = score_bits(sc[j]);
      n_gt += u > tau;
      n_eq += u == tau;
    }
  }
  const uint32_t packed = block_exclusive_scan(n_gt | (n_eq << 16), warp_tot);
  int eq_seen = (int)(packed >> 16);                               // tied candidates before j_lo
  int dst = (int)(packed & 0xffffu) + min(eq_seen, need_eq);       // kept candidates before j_lo
  int32_t* idx = a.idx + ((long long)s * a.Hkv + G0) * a.B;
  for (int j = j_lo; j < j_hi; ++j) {
    bool keep;
    if (keep_all) {
      keep = true;
    } else {
      const uint32_t u = score_bits(sc[j]);
      keep = u > tau;
      if (u == tau) keep = eq_seen++ < need_eq;
    }
    if (keep) {
      if (dst < a.B) idx[dst] = j;
      ++dst;
    }
  }
}

// One 16-byte vector per thread and step of the grid-stride loop, two steps
// unrolled so that two kept-index loads and then two row loads are in flight
// before any store.  Output row r of (stream, KV head): r < m_new gathers C_n
// from the pool, r >= m_new appends frame token r - m_new to D.  A row pair (K
// and V) is 2 * row_bytes / 16 vectors.
__device__ __forceinline__ bool gather_vec(const GatherArgs& a, int v, int per_row, int vpr, int rows,
                                           const int4** src, int4** dst) {
  const int rr = v / per_row;
  int e = v - rr * per_row;
  const bool isv = e >= vpr;
  if (isv) e -= vpr;
  const int row = rr % rows;
  const int sg = rr / rows;  // s * Hkv + g
  const int g = sg % a.Hkv;
  const int s = sg / a.Hkv;
  const char* sbase;
  char* dbase;
  if (row < a.m_new) {
    const int gsel = a.global ? 0 : g;
    const int j = __ldg(a.idx + ((long long)s * a.Hkv + gsel) * a.B + row);
    if (j < 0 || j >= a.m + a.T) return false;  // never taken for a well-formed kept list
    if (!isv && e == 0) {  // the row's position and score, once per (stream, KV head, slot)
      a.pos_new[(long long)sg * a.B + row] =
          j < a.m ? __ldg(a.pos_c + (long long)sg * a.B + j) : __ldg(a.pos_f + (long long)s * a.T + (j - a.m));
      a.score_new[(long long)sg * a.B + row] = __ldg(a.pool_score + ((long long)s * a.Hkv + gsel) * a.pool_g + j);
    }
    if (j < a.m) {
      sbase = static_cast<const char*>(isv ? a.vc : a.kc) + ((long long)sg * a.B + j) * a.row_bytes;
    } else {
      sbase = static_cast<const char*>(isv ? a.vf : a.kf) +
              (((long long)s * a.T + (j - a.m)) * a.Hkv + g) * a.row_bytes;
    }
    dbase = static_cast<char*>(isv ? a.vc_new : a.kc_new) + ((long long)sg * a.B + row) * a.row_bytes;
  } else {
    return false;  // rows past m_new do not exist
  }
  *src = reinterpret_cast<const int4*>(sbase) + e;
  *dst = reinterpret_cast<int4*>(dbase) + e;
  return true;
}

__global__ void __launch_bounds__(256) gather_append_kernel(GatherArgs a) {
  pdl_wait();
  pdl_trigger();
  const int vpr = a.row_bytes / 16;
  const int per_row = 2 * vpr;
  const int rows = a.m_new;
  const int total = a.S * a.Hkv * rows * per_row;
  const int stride = gridDim.x * blockDim.x;
  for (int v0 = blockIdx.x * blockDim.x + threadIdx.x; v0 < total; v0 += 2 * stride) {
    const int v1 = v0 + stride;
    const int4* s0 = nullptr;
    const int4* s1 = nullptr;
    int4* d0 = nullptr;
    int4* d1 = nullptr;
    const bool ok0 = gather_vec(a, v0, per_row, vpr, rows, &s0, &d0);
    const bool ok1 = v1 < total && gather_vec(a, v1, per_row, vpr, rows, &s1, &d1);
    int4 x0, x1;
    if (ok0) x0 = __ldg(s0);
    if (ok1) x1 = __ldg(s1);
    if (ok0) *d0 = x0;
    if (ok1) *d1 = x1;
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a_in, int S, cudaStream_t st, bool pdl) {
  SelectArgs a = a_in;
  const int L = a.m + a.T;
  const int n_groups = a.global ? 1 : a.Hkv;
  a.n_sel_blocks = n_groups * S;
  const long long app_vecs = (long long)S * a.T * a.Hkv * 2 * (a.row_bytes / 16);
  a.n_app_blocks = (int)((app_vecs + kSelThreads - 1) / kSelThreads);
  a.S = S;
  if (a.mrg.n_split > 1) {
    const long long mrg_threads = (long long)a.mrg.S * a.mrg.Hq * a.mrg.T * (a.mrg.d / 8);
    a.n_mrg_blocks = (int)((mrg_threads + kSelThreads - 1) / kSelThreads);
  } else {
    a.n_mrg_blocks = 0;
  }
  const size_t smem = (size_t)L * (sizeof(float) + sizeof(int));
  // the default 48 KB per block covers static and dynamic shared memory
  // together; the kernel's static arrays take ~1.2 KB, so opt in well before
  if (smem > 40 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_topb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(select_topb_kernel, dim3(a.n_sel_blocks + a.n_app_blocks + a.n_mrg_blocks),
                       dim3(kSelThreads), smem, st, pdl, a);
}

cudaError_t launch_gather(const GatherArgs& a, int n_sm, cudaStream_t st, bool pdl) {
  const long long vecs = (long long)a.S * a.Hkv * a.m_new * 2 * (a.row_bytes / 16);
  if (vecs == 0) return cudaSuccess;
  long long blocks = (vecs + 2 * 256 - 1) / (2 * 256);  // two vectors per thread
  const long long cap = (long long)n_sm * 8;           // one resident wave at 8 blocks per SM
  if (blocks > cap) blocks = cap;
  return launch_kernel(gather_append_kernel, dim3((unsigned)blocks), dim3(256), 0, st, pdl, a);
}

}  // namespace skv
