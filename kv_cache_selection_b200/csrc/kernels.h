// Internal launchers of libstatekv (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace skv {

// Launch with an optional programmatic stream serialisation attribute (the
// kernel must call pdl_wait() before reading its predecessor's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit on the current device to at
// least `bytes`, calling the driver only when the recorded limit is lower
// (the attribute persists for the process).
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);
template <typename... KArgs>
cudaError_t ensure_dynamic_smem(void (*kernel)(KArgs...), int bytes) {
  return ensure_dynamic_smem(reinterpret_cast<const void*>(kernel), bytes);
}

// Most key splits the float32 merge of a decode takes (its weights sit in
// shared memory).
constexpr int kMaxMergeSplit = 256;

constexpr int kDtypeBF16 = 0;
constexpr int kDtypeF32 = 1;

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, int d, int S, cudaStream_t st);
cudaError_t launch_score_simt(const ScoreArgs& a, int dtype, int d, int S, cudaStream_t st);
cudaError_t launch_select(const SelectArgs& a, int S, cudaStream_t st, bool pdl = false);
cudaError_t launch_gather(const GatherArgs& a, int n_sm, cudaStream_t st, bool pdl = false);

// bf16 4-D tiled TMA map, 128-byte swizzle, zero fill out of bounds.  dims[0]
// is the innermost (contiguous) extent in elements; strides_bytes[i] is the
// byte stride of dims[i+1].  Returns 0 or a CUresult.
int encode_tmap_bf16_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                        const uint64_t strides_bytes[3], const uint32_t box[4]);

// Tensor-core score pass (bf16): the three maps cover q [S][T][Hq][d],
// K_C [S][Hkv][B][d] and the frame keys [S][T][Hkv][d], boxes of 64 x 128 rows.
struct ScoreTcArgs {
  const float* lse;  // [S][Hq][T] natural log (read when n_split == 1)
  long long lse_s;
  const float* ml_part;  // [S][Hq][n_split][T] log2-sum-exp per key split (n_split > 1)
  int n_split;
  float* part;       // [S][Hkv * n_qsplit][pool]: one row per (KV group, split of its query rows)
  long long part_s;
  int part_g;
  int n_qsplit;      // splits of a group's query-row chunks over CTAs (>= 1)
  int m, T, Hq, Hkv, causal, n_c_tiles, n_f_tiles, S;
  float scale_log2;
  int* err;          // device error word (timeouts)
  unsigned long long wait_ns;  // pipeline-wait limit; 0 = the default
};
cudaError_t launch_score_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_kc, const CUtensorMap& tm_kf,
                            const ScoreTcArgs& a, int d, cudaStream_t st, bool pdl = false);
// Splits of each group's query-row chunks for the score pass: enough CTAs to
// cover n_sm when the key tiles alone do not, at most kMaxQsplit.
constexpr int kMaxQsplit = 8;
int score_tc_qsplit(int S, int Hq, int Hkv, int T, int m, int n_sm);

// Tensor-core attention (bf16) over [compressed rows; frame tokens].
// Query tiles: with stack = 0 a tile is 128 consecutive rows of one query
// head (n_it tiles per head); with stack = G (the group size) a tile stacks
// the G query heads of a KV group for 128 / G consecutive rows, row r of the
// tile being (row i0 + r / G, head g*G + r % G), so every K/V tile is read
// once for the whole group (n_it tiles per group).  q_rows is the number of
// rows the Q tensor map's box fills (128, or G * (128 / G)).
struct AttnTcArgs {
  void* out;          // out[s][i][h][dd] bf16
  long long out_s;
  int out_row;        // Hq * d
  float* lse;         // [S][Hq][T] natural log, may be null
  long long lse_s;
  __nv_bfloat16* o_part;  // O/l per split (n_split > 1): planes [S][Hq][n_split] of [d/8][T][8]
  float* o_part32;    // [S][Hq][n_split][T][d] in float32; used instead of o_part when set
  float* ml_part;     // [S][Hq][n_split][T] log2-sum-exp
  int m, T, Hq, Hkv, causal, S;
  int n_it, n_pairs, n_split, nC, nF;
  int stack, q_rows;
  float scale_log2;
  int* err;
  unsigned long long wait_ns;  // pipeline-wait limit; 0 = the default
};
int attn_tc_splits(int S, int Hq, int Hkv, int T, int m, int n_sm);
cudaError_t launch_attn_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                           const CUtensorMap& tm_kf, const CUtensorMap& tm_vf, const AttnTcArgs& a, int d,
                           cudaStream_t st, bool pdl = false);
cudaError_t launch_attn_combine(const AttnTcArgs& a, int d, cudaStream_t st, bool pdl = false);
// Merge of up to kMaxMergeSplit float32 key-split partials (o_part32) into out
// and lse: thread-per-(row, chunk) when that gives a warp or more per SM (of
// n_sm), else one block per row.
cudaError_t launch_attn_merge_wide(const AttnTcArgs& a, int d, int n_sm, cudaStream_t st, bool pdl = false);
MergeArgs merge_args(const AttnTcArgs& a, int d);

// Message for statekv_last_error(NULL) (errors of calls without a handle).
void set_free_error(const char* msg);

}  // namespace skv
