// Merge of attention key-split partials (device function shared by the
// standalone merge kernel and the extra blocks of the select launch).
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace skv {

constexpr int kMaxSplit = 8;

// Layout of the bf16 key-split partials: one plane of T x D values per
// (stream, query head, split), stored as [D/8 chunks of 8 values][T rows], so
// that a warp writing one 16-byte chunk of 32 consecutive rows (the attention
// epilogue, thread = row) covers 512 contiguous bytes.
__host__ __device__ __forceinline__ long long part_offset(long long plane, int chunk, int i, int T, int D) {
  return plane * T * D + ((long long)chunk * T + i) * 8;
}

// Threads of the merge: a warp takes 4 rows x 8 chunks (reads of 64
// contiguous bytes per chunk, writes of 128 contiguous bytes per row of out).
__host__ __device__ __forceinline__ long long merge_threads(long long rows, int D) {
  return (rows + 3) / 4 * 4 * (D / 8);
}

// Thread t handles (query row, 8-element chunk of d): it reads the row's
// n_split log2-sum-exps and its chunk of every split's O/l at once, weights
// them by 2^(ml_u - max), writes the bf16 result; chunk 0 also writes the
// row's natural-log lse.
template <int D>
__device__ __forceinline__ void merge_chunk(const MergeArgs& a, long long t) {
  constexpr int kHalves = D / 64;  // groups of 8 chunks per row
  const long long rows = (long long)a.S * a.Hq * a.T;
  const long long wid = t >> 5;
  const int lane = (int)(t & 31);
  const long long rw = (wid / kHalves) * 4 + (lane & 3);
  const int chunk = (int)(wid % kHalves) * 8 + (lane >> 2);
  if (rw >= rows) return;
  const int i = (int)(rw % a.T);
  const int sh = (int)(rw / a.T);  // s * Hq + h
  const int h = sh % a.Hq, s = sh / a.Hq;
  const long long plane0 = (long long)sh * a.n_split;
  float ml[kMaxSplit];
  uint4 raw[kMaxSplit];
#pragma unroll
  for (int u = 0; u < kMaxSplit; ++u) {
    if (u < a.n_split) {
      ml[u] = __ldg(a.ml_part + (plane0 + u) * a.T + i);
      raw[u] = __ldg(reinterpret_cast<const uint4*>(a.o_part + part_offset(plane0 + u, chunk, i, a.T, D)));
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
