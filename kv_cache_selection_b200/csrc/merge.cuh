// Merge of the attention's key-split partials: for one query row (stream s,
// head h, row i) and one 8-element chunk of d, the n_split partials (O/l in
// bf16 and the split's log2-sum-exp) are weighted by 2^(ml_u - max), summed
// and normalised; chunk 0 also writes the row's natural-log lse.
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace skv {

constexpr int kMaxSplit = 8;

template <int D>
__device__ __forceinline__ void merge_row_chunk(void* out, long long out_s, int out_row, float* lse, long long lse_s,
                                                const __nv_bfloat16* o_part, const float* ml_part, int Hq, int T,
                                                int n_split, int s, int h, int i, int chunk) {
  const long long prow0 = ((long long)s * Hq + h) * n_split * T + i;
  float ml[kMaxSplit];
  uint4 raw[kMaxSplit];
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u) {
    if (u < n_split) {
      ml[u] = __ldcg(ml_part + prow0 + (long long)u * T);
      raw[u] = __ldcg(reinterpret_cast<const uint4*>(o_part + (prow0 + (long long)u * T) * D) + chunk);
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u)
    if (u < n_split) mx = fmaxf(mx, ml[u]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u) {
    if (u < n_split) {
      const float w = ml[u] == -INFINITY ? 0.f : tc::ex2_approx(ml[u] - mx);
      wsum += w;
      const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += w * __bfloat162float(v[e]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4 o;
  uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int e = 0; e < 4; ++e) op[e] = tc::pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out) + s * out_s + (long long)i * out_row + (long long)h * D;
  reinterpret_cast<uint4*>(orow)[chunk] = o;
  if (chunk == 0 && lse) lse[s * lse_s + (long long)h * T + i] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
}

}  // namespace skv
