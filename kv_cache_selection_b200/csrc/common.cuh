// Shared device helpers and kernel argument blocks of libstatekv (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace skv {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Programmatic dependent launch: wait until the preceding kernel in the stream
// has completed and its writes are visible (a no-op without a programmatic
// dependency), and let the next kernel start its prologue early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Attention of a block of query rows over a two-segment key pool:
//   segment A = compressed state rows j < m (always visible),
//   segment B = the frame's (or sequence's) tokens t < nb; with `causal`,
//   query row i sees t <= i.
// Element strides; every tensor is indexed [s] first.
struct AttnArgs {
  const void* q;       // q[s][i][h][dd]
  long long q_s;       // stride of s
  int q_row;           // stride of i (= Hq*d)
  const void* ka;      // ka[s][g][j][dd]
  const void* va;
  long long a_s, a_g;  // strides of s and g (row stride = d)
  int m;
  const void* kb;      // kb[s][t][g][dd]
  const void* vb;
  long long b_s;
  int b_row;           // stride of t (= Hkv*d)
  int nb;
  void* out;           // out[s][i][h][dd], same strides as q
  float* lse;          // lse[s][h][i] natural log, may be null
  long long lse_s;     // stride of s (= Hq*n_rows)
  int n_rows;          // query rows per head
  int Hq, Hkv;
  int causal;
  float scale_log2;    // log2(e)/sqrt(d)
};

// Column mass of the normalised softmax weights over one KV group's query
// heads: part[s][g][j] = sum_{h in g} sum_i exp(s_hij - lse_hi).
struct ScoreArgs {
  const void* q;
  long long q_s;
  int q_row;
  const void* ka;
  long long a_s, a_g;
  int m;
  const void* kb;
  long long b_s;
  int b_row;
  int nb;
  const float* lse;    // lse[s][h][i] natural log
  long long lse_s;
  float* part;         // part[s][g][j]
  long long part_s;
  int part_g;
  int n_rows, Hq, Hkv, causal;
  float scale_log2;
};

// Merge of the attention's key-split partials into out and lse.
struct MergeArgs {
  void* out;                     // out[s][i][h][dd] bf16
  long long out_s;
  int out_row;
  float* lse;                    // [S][Hq][T] natural log, may be null
  long long lse_s;
  const __nv_bfloat16* o_part;   // O/l per split: planes [S][Hq][n_split] of [d/8][T][8]
  const float* ml_part;          // [S][Hq][n_split][T] log2-sum-exp
  int S, Hq, T, n_split, d;
};

// Top-B selection over the pool of one (stream, selection group).  The same
// launch carries extra blocks that merge the attention's key-split partials
// (not on the path to C_n).
struct SelectArgs {
  const float* part;      // part[s][g * n_qsplit + q][j], j < m + T: the score pass's partial sums
  long long part_s;
  int part_g;             // row stride of part and pool_score
  int n_qsplit;           // rows of part per KV group
  float* pool_score;      // out [s][g][j] (row of the selection group only)
  long long pool_s;       // stream stride of pool_score
  const int32_t* pos_c;   // current C positions [s][g][B] (read in recency mode)
  const int32_t* pos_f;   // frame positions [s][T] (read in recency mode)
  int32_t* idx;           // out [s][g][B] kept pool indices, ascending (row 0 in global mode)
  int Hkv, m, T, B, global;
  int recency;            // keep the B largest positions instead of the B largest scores
  int n_sel_blocks;       // blocks [0, n_sel_blocks): one per (stream, selection group)
  // key-split merge (n_mrg_blocks > 0 only for the bf16 attention with splits)
  int n_mrg_blocks;
  MergeArgs mrg;
};

// Gather of the kept rows into the next C buffer, plus the append of the
// frame's K/V and positions to the detailed state D.
struct GatherArgs {
  const void* kc;  const void* vc;   // current C [s][g][B][d]
  const void* kf;  const void* vf;   // frame [s][t][g][d]
  void* kc_new;    void* vc_new;     // next C [s][g][B][d]
  const int32_t* idx;                // [s][g][B] kept pool indices (row 0 in global mode)
  void* kd;        void* vd;         // D [s][g][max_tok][d]
  int32_t* pos_d;                    // [s][max_tok]
  const int32_t* pos_f;              // [s][T]
  const int32_t* pos_c;              // current C positions [s][g][B]
  const float* pool_score;           // [s][g][pool_g] (row 0 only in global mode)
  int32_t* pos_new;                  // next C positions [s][g][B]
  float* score_new;                  // next C scores [s][g][B]
  int pool_g;                        // row stride of pool_score
  int Hkv, T, B, m, m_new, row_bytes, global, d_len, max_tok;
  int S;
};

}  // namespace skv
