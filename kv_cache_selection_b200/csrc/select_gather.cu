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

namespace skv {
namespace {

constexpr int kSelThreads = 1024;

__device__ __forceinline__ uint32_t score_bits(float x) {
  // scores are sums of exponentials: >= +0, so the IEEE bit pattern orders
  // them like the values
  return __float_as_uint(x);
}

// Block-wide exclusive scan of one 32-bit value per thread (1024 threads).
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
    uint32_t w = warp_tot[lane];
    uint32_t wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  uint32_t r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

// One block per (selection group, stream).  Dynamic shared memory holds the
// pool's scores (L floats).
__global__ void __launch_bounds__(kSelThreads) select_topb_kernel(SelectArgs a) {
  extern __shared__ float sc[];
  __shared__ uint32_t hist[257];
  __shared__ uint32_t suffix[257];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t sel_bin;
  const int grp = blockIdx.x, s = blockIdx.y;
  const int L = a.m + a.T;
  const int G0 = a.global ? 0 : grp;
  const int G1 = a.global ? a.Hkv : grp + 1;

  // 1. scores of the pool: global mode sums the KV groups in a fixed order
  for (int j = threadIdx.x; j < L; j += kSelThreads) {
    float v = 0.f;
    for (int g = G0; g < G1; ++g) v += a.part[s * a.part_s + (long long)g * a.part_g + j];
    sc[j] = v;
    for (int g = G0; g < G1; ++g) a.pool_score[s * a.part_s + (long long)g * a.part_g + j] = v;
  }
  __syncthreads();
  if (a.B <= 0) return;  // nothing is kept (block-uniform)

  // 2. threshold: the B-th largest score (radix select, 8 bits per pass)
  uint32_t tau = 0;
  int need_eq = 0;  // how many candidates equal to tau are kept
  const bool keep_all = L <= a.B;
  if (!keep_all) {
    uint32_t prefix = 0, pmask = 0;
    int k = a.B;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = threadIdx.x; b < 257; b += kSelThreads) hist[b] = 0;
      __syncthreads();
      const int n_iter = (L + kSelThreads - 1) / kSelThreads;
      for (int it = 0; it < n_iter; ++it) {
        const int j = it * kSelThreads + threadIdx.x;
        uint32_t digit = 256;
        if (j < L) {
          uint32_t u = score_bits(sc[j]);
          if ((u & pmask) == prefix) digit = (u >> shift) & 255u;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, digit);
        if ((threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
      }
      __syncthreads();
      // suffix[b] = number of candidates (matching the prefix) with digit >= b
      if (threadIdx.x < 256) suffix[threadIdx.x] = hist[threadIdx.x];
      if (threadIdx.x == 0) suffix[256] = 0;
      __syncthreads();
      for (int off = 1; off < 256; off <<= 1) {
        uint32_t add = 0;
        if (threadIdx.x < 256 && threadIdx.x + off < 256) add = suffix[threadIdx.x + off];
        __syncthreads();
        if (threadIdx.x < 256) suffix[threadIdx.x] += add;
        __syncthreads();
      }
      if (threadIdx.x < 256) {
        const uint32_t b = threadIdx.x;
        if (suffix[b] >= (uint32_t)k && suffix[b + 1] < (uint32_t)k) sel_bin = b;
      }
      __syncthreads();
      const uint32_t b = sel_bin;
      k -= (int)suffix[b + 1];
      prefix |= b << shift;
      pmask |= 255u << shift;
      __syncthreads();
    }
    tau = prefix;
    need_eq = k;
  }

  // 3. keep flags and compaction in pool (= position) order
  const int chunk = (L + kSelThreads - 1) / kSelThreads;
  const int j0 = min(L, threadIdx.x * chunk), j1 = min(L, j0 + chunk);
  uint32_t gt = 0, eq = 0;
  if (!keep_all) {
    for (int j = j0; j < j1; ++j) {
      const uint32_t u = score_bits(sc[j]);
      gt += u > tau;
      eq += u == tau;
    }
  }
  // L <= 65535 (host-checked), so both counts fit 16 bits
  const uint32_t packed = block_exclusive_scan(gt | (eq << 16), warp_tot);
  const int gt_before = packed & 0xffffu;
  int eq_seen = packed >> 16;
  int dst = keep_all ? j0 : gt_before + min(eq_seen, need_eq);
  for (int j = j0; j < j1; ++j) {
    bool keep = keep_all;
    if (!keep_all) {
      const uint32_t u = score_bits(sc[j]);
      if (u > tau) keep = true;
      else if (u == tau) keep = eq_seen++ < need_eq;
    }
    if (!keep || dst >= a.B) continue;
    for (int g = G0; g < G1; ++g) {
      const long long row = ((long long)s * a.Hkv + g) * a.B;
      const int p = j < a.m ? a.pos_c[row + j] : a.pos_f[(long long)s * a.T + (j - a.m)];
      a.idx[row + dst] = j;
      a.pos_new[row + dst] = p;
      a.score_new[row + dst] = sc[j];
    }
    ++dst;
  }
}

// Copies 16-byte vectors.  Work item = (stream, KV head, output row, vector);
// rows [0, m_new) gather C_n, rows [m_new, m_new + T) append the frame to D.
__global__ void __launch_bounds__(256) gather_append_kernel(GatherArgs a) {
  const int vec_per_row = a.row_bytes / 16;
  const int rows = a.m_new + a.T;
  const long long total = (long long)a.S * a.Hkv * rows * vec_per_row;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int vec = (int)(w % vec_per_row);
    long long r = w / vec_per_row;
    const int row = (int)(r % rows);
    r /= rows;
    const int g = (int)(r % a.Hkv);
    const int s = (int)(r / a.Hkv);
    const long long sg = (long long)s * a.Hkv + g;
    const char* ksrc;
    const char* vsrc;
    char* kdst;
    char* vdst;
    if (row < a.m_new) {
      const int j = a.idx[sg * a.B + row];
      if (j < 0 || j >= a.m + a.T) continue;  // never taken for a well-formed kept list
      if (j < a.m) {
        const long long off = (sg * a.B + j) * a.row_bytes;
        ksrc = static_cast<const char*>(a.kc) + off;
        vsrc = static_cast<const char*>(a.vc) + off;
      } else {
        const long long off = (((long long)s * a.T + (j - a.m)) * a.Hkv + g) * a.row_bytes;
        ksrc = static_cast<const char*>(a.kf) + off;
        vsrc = static_cast<const char*>(a.vf) + off;
      }
      const long long doff = (sg * a.B + row) * a.row_bytes;
      kdst = static_cast<char*>(a.kc_new) + doff;
      vdst = static_cast<char*>(a.vc_new) + doff;
    } else {
      const int t = row - a.m_new;
      const long long off = (((long long)s * a.T + t) * a.Hkv + g) * a.row_bytes;
      ksrc = static_cast<const char*>(a.kf) + off;
      vsrc = static_cast<const char*>(a.vf) + off;
      const long long doff = (sg * a.max_tok + a.d_len + t) * a.row_bytes;
      kdst = static_cast<char*>(a.kd) + doff;
      vdst = static_cast<char*>(a.vd) + doff;
      if (g == 0 && vec == 0) a.pos_d[(long long)s * a.max_tok + a.d_len + t] = a.pos_f[(long long)s * a.T + t];
    }
    const int4 kv = __ldg(reinterpret_cast<const int4*>(ksrc) + vec);
    const int4 vv = __ldg(reinterpret_cast<const int4*>(vsrc) + vec);
    reinterpret_cast<int4*>(kdst)[vec] = kv;
    reinterpret_cast<int4*>(vdst)[vec] = vv;
  }
}

}  // namespace

cudaError_t launch_select(const SelectArgs& a, int S, cudaStream_t st) {
  const int L = a.m + a.T;
  const int n_groups = a.global ? 1 : a.Hkv;
  const size_t smem = (size_t)L * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_topb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_topb_kernel<<<dim3(n_groups, S), kSelThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs& a, int n_sm, cudaStream_t st) {
  const long long total = (long long)a.S * a.Hkv * (a.m_new + a.T) * (a.row_bytes / 16);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)n_sm * 8;
  if (blocks > cap) blocks = cap;
  gather_append_kernel<<<(int)blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace skv
