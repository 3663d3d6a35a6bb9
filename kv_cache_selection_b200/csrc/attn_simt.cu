// CUDA-core attention and score kernels (float32 arithmetic).
//
// These serve the float32 element type (the tensor-core kinds cannot hold a
// full float32 product) and every shape the tensor-core kernels do not take.
// Attention: "Linear Scaling Video VLMs for Long Video Understanding", P1
// section 方法步骤详情 — the frame's queries attend over the concatenation of
// the compressed memory and the frame's tokens; the score of candidate j is the
// sum over the frame's queries of the normalised attention weight.
#include "common.cuh"
#include "kernels.h"

namespace skv {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 4;
constexpr int kRowsPerBlock = kRowsPerWarp * kWarps;  // 16
constexpr int kKeyTile = 32;

template <typename T, int D>
__device__ __forceinline__ void load_rows_f32(float (*dst)[D + 1], const T* base, long long row_stride,
                                              int n_valid, int n_rows) {
  // n_rows x D tile, zero rows beyond n_valid
  for (int e = threadIdx.x; e < n_rows * D; e += blockDim.x) {
    int r = e / D, c = e % D;
    dst[r][c] = r < n_valid ? to_f(base[(long long)r * row_stride + c]) : 0.f;
  }
}

// One block: 16 query rows of one head h of stream s.  Online softmax in the
// log2 domain; each warp owns 4 rows, lanes split the key tile for the logits
// and the head dimension for the output.
template <typename T, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnArgs a) {
  __shared__ float Qs[kRowsPerBlock][D + 1];
  __shared__ float Ks[kKeyTile][D + 1];
  __shared__ float Vs[kKeyTile][D + 1];
  const int s = blockIdx.z, h = blockIdx.y, row0 = blockIdx.x * kRowsPerBlock;
  const int g = h / (a.Hq / a.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* q = static_cast<const T*>(a.q) + s * a.q_s + (long long)h * D;
  const T* ka = static_cast<const T*>(a.ka) + s * a.a_s + g * a.a_g;
  const T* va = static_cast<const T*>(a.va) + s * a.a_s + g * a.a_g;
  const T* kb = static_cast<const T*>(a.kb) + s * a.b_s + (long long)g * D;
  const T* vb = static_cast<const T*>(a.vb) + s * a.b_s + (long long)g * D;

  const int rows_valid = min(kRowsPerBlock, a.n_rows - row0);
  load_rows_f32<T, D>(Qs, q + (long long)row0 * a.q_row, a.q_row, rows_valid, kRowsPerBlock);

  float m_i[kRowsPerWarp], l_i[kRowsPerWarp], o[kRowsPerWarp][D / 32];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m_i[r] = -INFINITY;
    l_i[r] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[r][c] = 0.f;
  }
  // segment B keys needed by this block
  const int nb_needed = a.causal ? min(a.nb, row0 + kRowsPerBlock) : a.nb;
  const int n_tiles_a = (a.m + kKeyTile - 1) / kKeyTile;
  const int n_tiles_b = (nb_needed + kKeyTile - 1) / kKeyTile;

  for (int tile = 0; tile < n_tiles_a + n_tiles_b; ++tile) {
    const bool seg_a = tile < n_tiles_a;
    const int j0 = seg_a ? tile * kKeyTile : (tile - n_tiles_a) * kKeyTile;
    const int n_valid = seg_a ? min(kKeyTile, a.m - j0) : min(kKeyTile, nb_needed - j0);
    __syncthreads();
    if (seg_a) {
      load_rows_f32<T, D>(Ks, ka + (long long)j0 * D, D, n_valid, kKeyTile);
      load_rows_f32<T, D>(Vs, va + (long long)j0 * D, D, n_valid, kKeyTile);
    } else {
      load_rows_f32<T, D>(Ks, kb + (long long)j0 * a.b_row, a.b_row, n_valid, kKeyTile);
      load_rows_f32<T, D>(Vs, vb + (long long)j0 * a.b_row, a.b_row, n_valid, kKeyTile);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int lr = warp * kRowsPerWarp + r;
      const int row = row0 + lr;
      if (row >= a.n_rows) continue;  // warp-uniform
      float sc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) sc += Qs[lr][c] * Ks[lane][c];
      sc *= a.scale_log2;
      bool vis = lane < n_valid;
      if (!seg_a && a.causal) vis = vis && (j0 + lane <= row);
      sc = vis ? sc : -INFINITY;
      float tmax = sc;
#pragma unroll
      for (int off = 16; off; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      const float m_new = fmaxf(m_i[r], tmax);
      if (m_new == -INFINITY) continue;  // nothing visible yet (warp-uniform)
      const float p = vis ? exp2f(sc - m_new) : 0.f;
      const float alpha = exp2f(m_i[r] - m_new);
      float psum = p;
#pragma unroll
      for (int off = 16; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
      l_i[r] = l_i[r] * alpha + psum;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) o[r][c] *= alpha;
      for (int kk = 0; kk < kKeyTile; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) o[r][c] += pk * Vs[kk][lane + 32 * c];
      }
      m_i[r] = m_new;
    }
  }
  T* out = static_cast<T*>(a.out) + s * a.q_s + (long long)h * D;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = row0 + warp * kRowsPerWarp + r;
    if (row >= a.n_rows) continue;
    const float inv = 1.f / l_i[r];
#pragma unroll
    for (int c = 0; c < D / 32; ++c)
      out[(long long)row * a.q_row + lane + 32 * c] = from_f<T>(o[r][c] * inv);
    if (a.lse != nullptr && lane == 0)
      a.lse[s * a.lse_s + (long long)h * a.n_rows + row] = (m_i[r] + log2f(l_i[r])) * kLn2;
  }
}

// One block: 128 pool candidates (one per thread) of KV group g of stream s;
// loops over every query row of the group's heads.
constexpr int kScoreKeys = 128;
constexpr int kScoreRows = 32;

template <typename T, int D>
__global__ void __launch_bounds__(128) score_simt_kernel(ScoreArgs a) {
  __shared__ float Qs[kScoreRows][D];
  __shared__ float L2s[kScoreRows];
  const int s = blockIdx.z, g = blockIdx.y;
  const int j = blockIdx.x * kScoreKeys + threadIdx.x;
  const int G = a.Hq / a.Hkv;
  const int L = a.m + a.nb;
  const bool valid = j < L;
  const bool in_a = j < a.m;
  const int t = j - a.m;  // frame index for segment B
  float kreg[D];
  {
    const T* src = in_a ? static_cast<const T*>(a.ka) + s * a.a_s + g * a.a_g + (long long)j * D
                        : static_cast<const T*>(a.kb) + s * a.b_s + (long long)t * a.b_row +
                              (long long)g * D;
#pragma unroll
    for (int c = 0; c < D; ++c) kreg[c] = 0.f;
    if (valid) {
#pragma unroll
      for (int c = 0; c < D; ++c) kreg[c] = to_f(src[c]);
    }
  }
  float acc = 0.f;
  // first query row that can see this key: in causal mode frame token t is
  // seen by rows i >= t only
  const int n_groups_rows = G * a.n_rows;
  for (int r0 = 0; r0 < n_groups_rows; r0 += kScoreRows) {
    __syncthreads();
    for (int e = threadIdx.x; e < kScoreRows * D; e += blockDim.x) {
      int r = e / D, c = e % D;
      int rr = r0 + r;
      float val = 0.f;
      if (rr < n_groups_rows) {
        int hh = g * G + rr / a.n_rows, i = rr % a.n_rows;
        val = to_f(static_cast<const T*>(a.q)[s * a.q_s + (long long)i * a.q_row + (long long)hh * D + c]);
      }
      Qs[r][c] = val;
    }
    if (threadIdx.x < kScoreRows) {
      int rr = r0 + threadIdx.x;
      float v = INFINITY;
      if (rr < n_groups_rows) {
        int hh = g * G + rr / a.n_rows, i = rr % a.n_rows;
        v = a.lse[s * a.lse_s + (long long)hh * a.n_rows + i] * kLog2e;
      }
      L2s[threadIdx.x] = v;
    }
    __syncthreads();
    if (!valid) continue;
    for (int r = 0; r < kScoreRows; ++r) {
      const int rr = r0 + r;
      if (rr >= n_groups_rows) break;
      const int i = rr % a.n_rows;
      if (!in_a && a.causal && t > i) continue;
      float sc = 0.f;
#pragma unroll
      for (int c = 0; c < D; ++c) sc += Qs[r][c] * kreg[c];
      acc += exp2f(sc * a.scale_log2 - L2s[r]);
    }
  }
  if (valid) a.part[s * a.part_s + (long long)g * a.part_g + j] = acc;
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, int d, int S, cudaStream_t st) {
  dim3 grid((a.n_rows + kRowsPerBlock - 1) / kRowsPerBlock, a.Hq, S);
  if (dtype == kDtypeBF16) {
    if (d == 64) attn_simt_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(a);
    else attn_simt_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(a);
  } else {
    if (d == 64) attn_simt_kernel<float, 64><<<grid, 128, 0, st>>>(a);
    else attn_simt_kernel<float, 128><<<grid, 128, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_score_simt(const ScoreArgs& a, int dtype, int d, int S, cudaStream_t st) {
  const int L = a.m + a.nb;
  if (L == 0) return cudaSuccess;
  dim3 grid((L + kScoreKeys - 1) / kScoreKeys, a.Hkv, S);
  if (dtype == kDtypeBF16) {
    if (d == 64) score_simt_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(a);
    else score_simt_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(a);
  } else {
    if (d == 64) score_simt_kernel<float, 64><<<grid, 128, 0, st>>>(a);
    else score_simt_kernel<float, 128><<<grid, 128, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace skv
