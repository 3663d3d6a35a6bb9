// Merge of attention key-split partials (device function shared by the
// standalone merge kernel and the extra blocks of the select launch).
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace skv {

constexpr int kMaxSplit = 8;

// Thread t handles (query row, 8-element chunk of d): it reads the row's
// n_split log2-sum-exps and its chunk of every split's O/l at once, weights
// them by 2^(ml_u - max), writes the bf16 result; chunk 0 also writes the
// row's natural-log lse.
template <int D>
__device__ __forceinline__ void merge_chunk(const MergeArgs& a, int t) {
  constexpr int kChunks = D / 8;
  const int rows = a.S * a.Hq * a.T;
  if (t >= rows * kChunks) return;
  const int chunk = t % kChunks;
  const int rw = t / kChunks;
  const int i = rw % a.T;
  const int sh = rw / a.T;  // s * Hq + h
  const int h = sh % a.Hq, s = sh / a.Hq;
  const long long prow0 = (long long)sh * a.n_split * a.T + i;
  float ml[kMaxSplit];
  uint4 raw[kMaxSplit];
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u) {
    if (u < a.n_split) {
      ml[u] = __ldg(a.ml_part + prow0 + (long long)u * a.T);
      raw[u] = __ldg(reinterpret_cast<const uint4*>(a.o_part + (prow0 + (long long)u * a.T) * D) + chunk);
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u)
    if (u < a.n_split) mx = fmaxf(mx, ml[u]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u) {
    if (u < a.n_split) {
      const float w = ml[u] == -INFINITY ? 0.f : tc::ex2_approx(ml[u] - mx);
      wsum += w;
      const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += w * __bfloat162float(v[e]);
    }
  }
  const float inv = 1.f / wsum;
  uint4 o;
  uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int e = 0; e < 4; ++e) op[e] = tc::pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + s * a.out_s + (long long)i * a.out_row +
                        (long long)h * D;
  reinterpret_cast<uint4*>(orow)[chunk] = o;
  if (chunk == 0 && a.lse) a.lse[s * a.lse_s + (long long)h * a.T + i] = (mx + __log2f(wsum)) * kLn2;
}

}  // namespace skv
