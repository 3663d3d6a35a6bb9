// Attention of the frame's queries over [C_{n-1}; frame] on the 5th-generation
// tensor cores (bf16 in, f32 accumulate), with per-row log-sum-exp out.
//
// "Linear Scaling Video VLMs for Long Video Understanding", P1 section
// 方法步骤详情: the current frame's queries attend over the concatenation of
// the compressed memory and the current frame's tokens (softmax of the dot
// products, times the values); the frame is causal inside (P1 section
// 自注意力复杂度) and every compressed entry is visible.  The same kernel, with
// an empty compressed state and the whole sequence as "frame", is the full
// causal comparator.
//
// One CTA takes two 128-row query tiles (A, B) of one KV group and a range of
// 128-key tiles.  Per key tile and query tile:
//   S = Q K^T            tcgen05.mma, A = Q (smem), B = K (smem), D = S (TMEM)
//   P = exp2(S*c - m)    softmax warpgroup: TMEM -> registers -> bf16 P back
//                        into the same TMEM columns
//   O += P V             tcgen05.mma with A = P read from TMEM, B = V (smem,
//                        MN-major), D = O (TMEM)
// The two softmax warpgroups alternate with the tensor core (while one
// computes P, the other tile's MMAs run).  The running max is applied lazily:
// O and the row sum are rescaled only when a row's max grows by more than 2^8,
// so P stays below 256 and the result is exact up to rounding.  Key tiles are
// split across CTAs to fill the SMs; each split writes (O/l, log2-sum-exp)
// partials that attn_combine merges, or out and lse directly when unsplit.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 4..7 softmax of tile A, warps 8..11 softmax of tile B (warp w
// reads TMEM lanes 32*(w%4) .. +31, so each group covers all 128 rows).
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "merge.cuh"


namespace skv {
namespace {
using namespace tc;

constexpr int kSlots = 4;        // K/V ring slots (each one 128-key tile)
constexpr int kThreads = 384;
// registers: launched at 168 per thread (384 x 168 = 64512); warpgroup 0
// (producer, MMA issuer, two idle warps) drops to 72 and the two softmax
// warpgroups rise to 216: 128 x 72 + 256 x 216 = 64512.
constexpr int kRegsLow = 72;
constexpr int kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * 168, "register split exceeds the launch");
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct AttnSmem {
  static constexpr int kAtoms = D / 64;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kTileBytes = kAtoms * kAtomBytes;  // 128 rows x D bf16
  static constexpr int kQ = 0;                             // Q tiles A, B
  static constexpr int kKV = 2 * kTileBytes;               // ring
  static constexpr int kBar = kKV + kSlots * kTileBytes;
  // q_full (tile A), kv_full[kSlots], kv_empty[kSlots], s_full[2], p_full[2], o_done[2], done, pv_done,
  // q_full (tile B)
  static constexpr int kNumBars = 1 + 2 * kSlots + 6 + 1 + 1 + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  // at least 116 KB so that a second CTA (which would also need all 512 TMEM
  // columns) never shares the SM
  static constexpr int kAlloc = kBytes + 1024 > 116 * 1024 ? kBytes + 1024 : 116 * 1024;
};

struct TileInfo {
  bool valid;
  int h, i0, nk;  // head, first query row, key tiles it needs in total
};

__device__ __forceinline__ TileInfo tile_info(const AttnTcArgs& a, int g, int t) {
  TileInfo ti;
  const int G = a.Hq / a.Hkv;
  int i_max;
  if (a.stack) {
    const int ri = 128 / a.stack;  // rows of the tile per head
    ti.valid = t < a.n_it;
    if (!ti.valid) t = 0;
    ti.h = g * G;                  // first head of the stack
    ti.i0 = t * ri;
    i_max = min(ti.i0 + ri - 1, a.T - 1);
  } else {
    ti.valid = t < G * a.n_it;
    if (!ti.valid) t = 0;
    ti.h = g * G + t / a.n_it;
    ti.i0 = (t % a.n_it) * 128;
    i_max = min(ti.i0 + 127, a.T - 1);  // last row of the tile
  }
  int nf = a.nF;
  if (a.causal) nf = i_max / 128 + 1;   // frame tiles holding tokens <= i_max
  ti.nk = a.nC + nf;
  return ti;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kf,
                   const __grid_constant__ CUtensorMap tm_vf, AttnTcArgs a) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // unit -> (stream, KV group, query-tile pair, key split)
  int u = blockIdx.x;
  const int sp = u % a.n_split;
  u /= a.n_split;
  const int pair = a.n_pairs - 1 - u % a.n_pairs;  // later query tiles (more keys) first
  u /= a.n_pairs;
  const int g = u % a.Hkv;
  const int s = u / a.Hkv;
  const TileInfo tA = tile_info(a, g, 2 * pair), tB = tile_info(a, g, 2 * pair + 1);
  const int nk = max(tA.nk, tB.valid ? tB.nk : 0);
  const int kb = sp * nk / a.n_split, ke = (sp + 1) * nk / a.n_split;
  const int nA = max(0, min(ke, tA.nk) - kb);
  const int nB = tB.valid ? max(0, min(ke, tB.nk) - kb) : 0;
  const int n_load = max(nA, nB);

  const uint32_t bar_q = sb + L::kBar;  // Q tile A
  auto bar_kvfull = [&](int sl) { return sb + L::kBar + 8u * (1 + sl); };
  auto bar_kvempty = [&](int sl) { return sb + L::kBar + 8u * (1 + kSlots + sl); };
  auto bar_sfull = [&](int x) { return sb + L::kBar + 8u * (1 + 2 * kSlots + x); };
  auto bar_pfull = [&](int x) { return sb + L::kBar + 8u * (3 + 2 * kSlots + x); };
  auto bar_odone = [&](int x) { return sb + L::kBar + 8u * (5 + 2 * kSlots + x); };
  const uint32_t bar_done = sb + L::kBar + 8u * (7 + 2 * kSlots);
  const uint32_t bar_pvdone = sb + L::kBar + 8u * (8 + 2 * kSlots);
  const uint32_t bar_qb = sb + L::kBar + 8u * (9 + 2 * kSlots);  // Q tile B
  // With no keys for tile B in this CTA (a lone query tile: decode, or the
  // last tile of an odd count), tile A double-buffers S in the TMEM columns of
  // S_B: S(j+1) is computed while the softmax of tile j runs.
  const bool dbuf = nB == 0;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  const unsigned long long wait_lim = a.wait_ns ? a.wait_ns : kWaitLimitNs;  // pipeline-wait limit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  if (threadIdx.x == 0) {
    // the maps are kernel parameters, not outputs of the preceding kernel
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_vc);
    tma_prefetch_desc(&tm_kf);
    tma_prefetch_desc(&tm_vf);
    mbar_init(bar_q, 1);
    mbar_init(bar_qb, 1);
    for (int sl = 0; sl < kSlots; ++sl) {
      mbar_init(bar_kvfull(sl), 1);
      mbar_init(bar_kvempty(sl), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_sfull(x), 1);
      mbar_init(bar_pfull(x), 4);
      mbar_init(bar_odone(x), 1);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_pvdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  // TMEM columns: S/P of tile A at 0, of tile B at 128, O of A at 256, O of B at 384
  auto col_s = [](int x) { return (uint32_t)(x * 128); };
  auto col_o = [](int x) { return (uint32_t)(256 + x * 128); };

  if (warp < 4) regs_dec<kRegsLow>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Load order Q_A, K_0, Q_B, V_0, ...: S_A(0) needs only the first two
      auto load_q = [&](int x) {
        const uint32_t bar = x == 0 ? bar_q : bar_qb;
        const TileInfo& ti = x == 0 ? tA : tB;
        mbar_arrive_expect_tx(bar, L::kAtoms * a.q_rows * 128);
        for (int at = 0; at < L::kAtoms; ++at)
          tma_load_4d(sb + L::kQ + x * L::kTileBytes + at * L::kAtomBytes, &tm_q, bar, at * 64, ti.h, ti.i0, s);
      };
      if (nA > 0) load_q(0);
      bool qb_issued = false;
      int issued = 0;
      for (int idx = 0; idx < 2 * n_load; ++idx) {
        const int sl = idx % kSlots;
        if (!mbar_wait(bar_kvempty(sl), ((idx / kSlots) & 1) ^ 1, a.err, kErrWaitEmpty, abort_flag, wait_lim)) break;
        const int k = kb + (idx >> 1);
        const bool is_v = idx & 1;
        const bool is_c = k < a.nC;
        const int r0 = is_c ? k * 128 : (k - a.nC) * 128;
        mbar_arrive_expect_tx(bar_kvfull(sl), L::kTileBytes);
        const uint32_t dst = sb + L::kKV + sl * L::kTileBytes;
        for (int at = 0; at < L::kAtoms; ++at) {
          if (is_c) tma_load_4d(dst + at * L::kAtomBytes, is_v ? &tm_vc : &tm_kc, bar_kvfull(sl), at * 64, r0, g, s);
          else tma_load_4d(dst + at * L::kAtomBytes, is_v ? &tm_vf : &tm_kf, bar_kvfull(sl), at * 64, g, r0, s);
        }
        issued = idx + 1;
        if (idx == 0 && nB > 0) {
          load_q(1);
          qb_issued = true;
        }
      }
      if (nA > 0) drain_wait(bar_q, 0, a.err);
      if (qb_issued) drain_wait(bar_qb, 0, a.err);
      for (int idx = (issued > kSlots ? issued - kSlots : 0); idx < issued; ++idx)
        drain_wait(bar_kvfull(idx % kSlots), (idx / kSlots) & 1, a.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && n_load > 0) {
      constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16(128, D, false, true);
      const int nX[2] = {nA, nB};
      // Descriptors are formed once; per MMA only the start address (bits
      // 0..13, 16-byte units) advances, which never carries into the other
      // fields.
      const uint64_t dq0 = sdesc_sw128(sb + L::kQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(sb + L::kKV, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(sb + L::kKV, L::kAtomBytes, 1024);
      auto slot16 = [&](int idx) { return (uint64_t)((idx % kSlots) * (L::kTileBytes >> 4)); };
      auto wait_slot = [&](int idx) {
        return mbar_wait(bar_kvfull(idx % kSlots), (idx / kSlots) & 1, a.err, kErrWaitLoad, abort_flag, wait_lim);
      };
      auto issue_s = [&](int x, int j) {  // S_x = Q_x K_j^T
        const uint64_t dq = dq0 + (uint64_t)((x * L::kTileBytes) >> 4), dk = dk0 + slot16(2 * j);
        const uint32_t d_tmem = tmem + col_s(x);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * L::kAtomBytes + (kk & 3) * 32) >> 4);
          mma_ss(d_tmem, dq + off, dk + off, id_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_sfull(x));
      };
      auto issue_pv = [&](int x, int j) {  // O_x += P_x V_j
        const uint64_t dv = dv0 + slot16(2 * j + 1);
        const uint32_t d_tmem = tmem + col_o(x), a_tmem = tmem + col_s(x);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(d_tmem, a_tmem + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), id_o, (j > 0 || kk > 0) ? 1u : 0u);
        if (j == nX[x] - 1) mma_commit(bar_odone(x));
      };
      bool ok = wait_slot(0) && (nA == 0 || mbar_wait(bar_q, 0, a.err, kErrWaitLoad, abort_flag, wait_lim));
      if (dbuf) {
        // S of tile j goes to buffer j & 1 (the S columns of tile A or B); the
        // softmax of tile j overlaps S(j+1).  The tensor pipe runs MMAs in
        // issue order, so S(j+1) overwrites P(j-1) only after P.V(j-1) read it.
        auto issue_s_buf = [&](int buf, int j) {  // S_buf = Q_A K_j^T
          const uint64_t dk = dk0 + slot16(2 * j);
          const uint32_t d_tmem = tmem + col_s(buf);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * L::kAtomBytes + (kk & 3) * 32) >> 4);
            mma_ss(d_tmem, dq0 + off, dk + off, id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull(buf));
        };
        if (ok) {
          fence_after_sync();
          issue_s_buf(0, 0);
          mma_commit(bar_kvempty(0));
        }
        for (int j = 0; ok && j < nA; ++j) {
          const bool next_k = j + 1 < nA;
          if (next_k) {
            if (!(ok = wait_slot(2 * (j + 1)))) break;  // K_{j+1}
            issue_s_buf((j + 1) & 1, j + 1);
          }
          if (!(ok = wait_slot(2 * j + 1))) break;  // V_j
          if (!(ok = mbar_wait(bar_pfull(j & 1), (j >> 1) & 1, a.err, kErrWaitP, abort_flag, wait_lim))) break;
          fence_after_sync();
          const uint64_t dv = dv0 + slot16(2 * j + 1);
          const uint32_t a_tmem = tmem + col_s(j & 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + col_o(0), a_tmem + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), id_o,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_pvdone);
          if (j == nA - 1) mma_commit(bar_odone(0));
          mma_commit(bar_kvempty((2 * j + 1) % kSlots));                // V_j
          if (next_k) mma_commit(bar_kvempty((2 * (j + 1)) % kSlots));  // K_{j+1}
        }
        ok = false;  // the paired loop below is for two query tiles
      }
      if (ok) {
        fence_after_sync();
        if (nA > 0) issue_s(0, 0);
        if (nB > 0 && (ok = mbar_wait(bar_qb, 0, a.err, kErrWaitLoad, abort_flag, wait_lim))) {
          fence_after_sync();
          issue_s(1, 0);
        }
        if (ok) mma_commit(bar_kvempty(0));
      }
      // Ring order of tiles: K_0, V_0, K_1, V_1, ...; each slot is released
      // (kv_empty) after the last MMA reading it, in the same order.
      for (int j = 0; ok && j < n_load; ++j) {
        if (!(ok = wait_slot(2 * j + 1))) break;  // V_j
        const bool next_k = j + 1 < n_load;
        if (j < nA) {
          if (!(ok = mbar_wait(bar_pfull(0), j & 1, a.err, kErrWaitP, abort_flag, wait_lim))) break;
          fence_after_sync();
          issue_pv(0, j);
        }
        if (next_k && !(ok = wait_slot(2 * (j + 1)))) break;  // K_{j+1}
        if (j + 1 < nA) issue_s(0, j + 1);
        if (j < nB) {
          if (!(ok = mbar_wait(bar_pfull(1), j & 1, a.err, kErrWaitP, abort_flag, wait_lim))) break;
          fence_after_sync();
          issue_pv(1, j);
        }
        mma_commit(bar_kvempty((2 * j + 1) % kSlots));  // V_j read by both P.V
        if (j + 1 < nB) issue_s(1, j + 1);
        if (next_k) mma_commit(bar_kvempty((2 * (j + 1)) % kSlots));  // K_{j+1} read by both S
      }
      mma_commit(bar_done);
      drain_wait(bar_done, 0, a.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsHigh>();
    const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const TileInfo ti = x == 0 ? tA : tB;
    const int nX = x == 0 ? nA : nB;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row within the tile (= TMEM lane)
    // query row in the frame and query head of this TMEM lane
    const int i = a.stack ? ti.i0 + r / a.stack : ti.i0 + r;
    const int h = a.stack ? ti.h + r % a.stack : ti.h;
    const bool row_exists = !a.stack || r < a.q_rows;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_o = t_lane + col_o(x);
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = ti.valid;
    for (int j = 0; ok && j < nX; ++j) {
      // S of tile j: in buffer x, or in buffer j & 1 when tile A double-buffers
      const int sbuf = dbuf ? (j & 1) : x;
      const uint32_t sphase = dbuf ? ((j >> 1) & 1) : (j & 1);
      const uint32_t t_s = t_lane + col_s(sbuf);
      // S_j is on the critical chain: spin (a suspending wait wakes later)
      if (!(ok = warp_spin_wait(bar_sfull(sbuf), sphase, a.err, kErrWaitAcc, abort_flag, wait_lim))) break;
      fence_after_sync();
      const int k = kb + j;
      const bool is_c = k < a.nC;
      const int base = is_c ? k * 128 : (k - a.nC) * 128;
      // visible columns of this row form a prefix [0, lim)
      int lim = is_c ? a.m - base : (a.causal ? min(a.T, i + 1) : a.T) - base;
      lim = max(0, min(128, lim));
      const bool masked = __any_sync(0xffffffffu, lim < 128);
      // the whole 128-column row of S in one batch of TMEM loads
      uint32_t sv[128];
      tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
      tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      tmem_ld_wait();
      if (masked) {
#pragma unroll
        for (int jj = 0; jj < 128; ++jj)
          if (jj >= lim) sv[jj] = __float_as_uint(-INFINITY);
      }
      // row max of the raw logits (c > 0): eight independent chains
      float m8[8];
#pragma unroll
      for (int q8 = 0; q8 < 8; ++q8) {
        m8[q8] = __uint_as_float(sv[16 * q8]);
#pragma unroll
        for (int jj = 1; jj < 15; jj += 2)
          m8[q8] = max3f(m8[q8], __uint_as_float(sv[16 * q8 + jj]), __uint_as_float(sv[16 * q8 + jj + 1]));
        m8[q8] = fmaxf(m8[q8], __uint_as_float(sv[16 * q8 + 15]));
      }
      const float mx = fmaxf(fmaxf(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5])), fmaxf(m8[6], m8[7]));
      float m_new = fmaxf(m_used, mx * c);
      if (m_new == -INFINITY) m_new = 0.f;  // nothing visible yet in this row
      if (j == 0) {
        m_used = m_new;
      } else {
        const bool need = m_new > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold P.V of every earlier tile: S_j was issued after them,
          // except with double-buffered S, where P.V(j-1) may still run
          if (dbuf && !(ok = warp_wait(bar_pvdone, (j - 1) & 1, a.err, kErrWaitAcc, abort_flag, wait_lim))) break;
          fence_after_sync();
          const float f = need ? ex2_approx(m_used - m_new) : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D / 32; ++c0) {
            uint32_t v[32];
            tmem_ld32(t_o + c0 * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) v[jj] = __float_as_uint(__uint_as_float(v[jj]) * f);
            tmem_st32(t_o + c0 * 32, v);
          }
          tmem_st_wait();
          l *= f;
          if (need) m_used = m_new;
        }
      }
      // P = exp2(S*c - m_used) (masked entries hold -inf -> 0), as bf16 into
      // the first 64 columns of the same TMEM region
      // (the scale-and-shift and the row sums in paired float32 instructions)
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_used, -m_used);
      float2 ls = make_float2(0.f, 0.f);
#pragma unroll
      for (int c0 = 0; c0 < 4; ++c0) {
        uint32_t pk[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[c0 * 32 + 2 * jj]),
                                             __uint_as_float(sv[c0 * 32 + 2 * jj + 1])), c2, nm2);
          const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          ls = fadd2(ls, pp);
          pk[jj] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st16(t_s + c0 * 16, pk);
      }
      tmem_st_wait();
      l += ls.x + ls.y;
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull(sbuf));
    }
    // ---- epilogue: O / l and the row's log2-sum-exp
    if (ok && nX > 0) ok = warp_wait(bar_odone(x), 0, a.err, kErrWaitAcc, abort_flag, wait_lim);
    if (ok && ti.valid && !*abort_flag) {
      fence_after_sync();
      const bool row_ok = row_exists && i < a.T;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m_used + __log2f(l) : -INFINITY;
      if (a.n_split == 1) {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + s * a.out_s + (long long)i * a.out_row +
                              (long long)h * D;
#pragma unroll
        for (int c0 = 0; c0 < D / 32; ++c0) {
          uint32_t v[32];
          tmem_ld32(t_o + c0 * 32, v);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            pk[jj] = pack_bf16x2(__uint_as_float(v[2 * jj]) * inv, __uint_as_float(v[2 * jj + 1]) * inv);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c0 * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          }
        }
        if (row_ok && a.lse) a.lse[s * a.lse_s + (long long)h * a.T + i] = lse2 * kLn2;
      } else {
        const long long prow = ((long long)(s * a.Hq + h) * a.n_split + sp) * a.T + i;
#pragma unroll
        for (int c0 = 0; c0 < D / 32; ++c0) {
          uint32_t v[32];
          if (nX > 0) {
            tmem_ld32(t_o + c0 * 32, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) v[jj] = 0u;
          }
          if (a.o_part32) {
            if (row_ok) {
              float4* dst = reinterpret_cast<float4*>(a.o_part32 + prow * D + c0 * 32);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(__uint_as_float(v[4 * q4]) * inv, __uint_as_float(v[4 * q4 + 1]) * inv,
                                      __uint_as_float(v[4 * q4 + 2]) * inv, __uint_as_float(v[4 * q4 + 3]) * inv);
            }
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              pk[jj] = pack_bf16x2(__uint_as_float(v[2 * jj]) * inv, __uint_as_float(v[2 * jj + 1]) * inv);
            if (row_ok) {
              const long long plane = ((long long)(s * a.Hq + h) * a.n_split + sp);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4*>(a.o_part + part_offset(plane, c0 * 4 + q4, i, a.T, D)) =
                    make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
            }
          }
        }
        if (row_ok) a.ml_part[prow] = nX > 0 ? lse2 : -INFINITY;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(MergeArgs a) {
  pdl_wait();
  pdl_trigger();
  merge_chunk<D>(a, (long long)blockIdx.x * blockDim.x + threadIdx.x);
}

// Merge of n_split float32 partials (O/l and log2-sum-exp per split) when the
// rows alone fill the GPU: thread = (row, 4-element chunk of d); pass 1 takes
// the largest log2-sum-exp, pass 2 adds the splits' O/l weighted by
// 2^(ml_u - max).
template <int D>
__global__ void __launch_bounds__(256) attn_merge_wide_kernel(AttnTcArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int kChunks = D / 4;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long rows = (long long)a.S * a.Hq * a.T;
  if (t >= rows * kChunks) return;
  const int chunk = (int)(t % kChunks);
  const long long rw = t / kChunks;
  const int i = (int)(rw % a.T);
  const long long sh = rw / a.T;  // s * Hq + h
  const int h = (int)(sh % a.Hq), s = (int)(sh / a.Hq);
  const long long prow0 = sh * a.n_split * a.T + i;
  // eight splits' loads in flight per round (a decode has tens of splits)
  constexpr int kB = 8;
  float mx = -INFINITY;
  for (int u0 = 0; u0 < a.n_split; u0 += kB) {
    float m8[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k)
      m8[k] = u0 + k < a.n_split ? __ldg(a.ml_part + prow0 + (long long)(u0 + k) * a.T) : -INFINITY;
#pragma unroll
    for (int k = 0; k < kB; ++k) mx = fmaxf(mx, m8[k]);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  for (int u0 = 0; u0 < a.n_split; u0 += kB) {
    float m8[kB];
    float4 o8[kB];
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      m8[k] = -INFINITY;
      if (u0 + k < a.n_split) {
        m8[k] = __ldg(a.ml_part + prow0 + (long long)(u0 + k) * a.T);
        o8[k] = __ldg(reinterpret_cast<const float4*>(a.o_part32 + (prow0 + (long long)(u0 + k) * a.T) * D) + chunk);
      }
    }
#pragma unroll
    for (int k = 0; k < kB; ++k) {
      if (m8[k] == -INFINITY) continue;
      const float w = ex2_approx(m8[k] - mx);
      wsum += w;
      acc.x += w * o8[k].x;
      acc.y += w * o8[k].y;
      acc.z += w * o8[k].z;
      acc.w += w * o8[k].w;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + s * a.out_s + (long long)i * a.out_row + (long long)h * D;
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(orow)[chunk] = pk;
  if (chunk == 0 && a.lse)
    a.lse[s * a.lse_s + (long long)h * a.T + i] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
}

// The same merge when the rows are few (a decode of a few text tokens has
// tens of splits per row): one block per query row, so that the work still
// spreads over many threads with every load of a pass in flight at once:
//   1. each thread takes a split's log2-sum-exp ml_u; block maximum mx;
//   2. w_u = 2^(ml_u - mx) into shared memory, wsum = sum of the w_u (a fixed
//      reduction tree);
//   3. thread (group g, 4-element chunk c) adds w_u * (O/l)_u[c] over the
//      splits u = g, g + kG, ...; the kG group sums are added in group order.
// out = sum / wsum; lse = mx + log2(wsum), in natural-log units.
template <int D>
__global__ void __launch_bounds__(256) attn_merge_split_kernel(AttnTcArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int kT = 256;
  constexpr int kChunks = D / 4;       // 4-float chunks of a row
  constexpr int kG = kT / kChunks;     // split groups
  constexpr int kBatch = 8;            // loads in flight per thread and round
  __shared__ float s_w[kMaxMergeSplit];
  __shared__ float s_red[kT / 32];
  __shared__ float4 s_acc[kG][kChunks];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long rw = blockIdx.x;     // (s, h, i)
  const int i = (int)(rw % a.T);
  const long long sh = rw / a.T;       // s * Hq + h
  const int h = (int)(sh % a.Hq), s = (int)(sh / a.Hq);
  const long long prow0 = sh * a.n_split * a.T + i;
  const int n = a.n_split;
  // 1. largest log2-sum-exp of the row
  float mx = -INFINITY;
  for (int u = tid; u < n; u += kT) mx = fmaxf(mx, __ldg(a.ml_part + prow0 + (long long)u * a.T));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  mx = s_red[0];
#pragma unroll
  for (int w = 1; w < kT / 32; ++w) mx = fmaxf(mx, s_red[w]);
  __syncthreads();  // s_red is reused below
  // 2. split weights (0 for a split that saw no key of the row)
  float wpart = 0.f;
  for (int u = tid; u < n; u += kT) {
    const float ml = __ldg(a.ml_part + prow0 + (long long)u * a.T);
    const float w = ml == -INFINITY ? 0.f : ex2_approx(ml - mx);
    s_w[u] = w;
    wpart += w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wpart += __shfl_xor_sync(0xffffffffu, wpart, off);
  if (lane == 0) s_red[warp] = wpart;
  __syncthreads();
  float wsum = 0.f;
#pragma unroll
  for (int w = 0; w < kT / 32; ++w) wsum += s_red[w];
  // 3. weighted sum of the splits' O/l, kBatch loads in flight per round
  const int c = tid % kChunks, g = tid / kChunks;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int u0 = g; u0 < n; u0 += kG * kBatch) {
    float4 o[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int u = u0 + k * kG;
      if (u < n) o[k] = __ldg(reinterpret_cast<const float4*>(a.o_part32 + (prow0 + (long long)u * a.T) * D) + c);
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int u = u0 + k * kG;
      if (u < n) {
        const float w = s_w[u];
        acc.x += w * o[k].x;
        acc.y += w * o[k].y;
        acc.z += w * o[k].z;
        acc.w += w * o[k].w;
      }
    }
  }
  s_acc[g][c] = acc;
  __syncthreads();
  if (g == 0) {
#pragma unroll
    for (int gg = 1; gg < kG; ++gg) {
      const float4 x = s_acc[gg][c];
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    __nv_bfloat16* orow =
        static_cast<__nv_bfloat16*>(a.out) + s * a.out_s + (long long)i * a.out_row + (long long)h * D;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(orow)[c] = pk;
    if (c == 0 && a.lse)
      a.lse[s * a.lse_s + (long long)h * a.T + i] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attn_merge_wide(const AttnTcArgs& a, int d, int n_sm, cudaStream_t st, bool pdl) {
  const long long rows = (long long)a.S * a.Hq * a.T;
  if (a.n_split > kMaxMergeSplit) return cudaErrorInvalidValue;
  const long long threads = rows * (d / 4);  // one thread per (row, 4-element chunk)
  if (threads >= (long long)n_sm * 32) {
    // a warp or more per SM: the rows give enough parallel loads
    const int blocks = (int)((threads + 255) / 256);
    if (d == 128) return launch_kernel(attn_merge_wide_kernel<128>, dim3(blocks), dim3(256), 0, st, pdl, a);
    return launch_kernel(attn_merge_wide_kernel<64>, dim3(blocks), dim3(256), 0, st, pdl, a);
  }
  if (d == 128) return launch_kernel(attn_merge_split_kernel<128>, dim3((unsigned)rows), dim3(256), 0, st, pdl, a);
  return launch_kernel(attn_merge_split_kernel<64>, dim3((unsigned)rows), dim3(256), 0, st, pdl, a);
}

int attn_tc_splits(int S, int Hq, int Hkv, int T, int m, int n_sm) {
  const int G = Hq / Hkv;
  const int n_it = (T + 127) / 128;
  const int n_pairs = (G * n_it + 1) / 2;
  const int units = S * Hkv * n_pairs;
  const int nk = (m + 127) / 128 + n_it;
  int split = n_sm / units;
  if (split < 1) split = 1;
  if (split > nk) split = nk;
  if (split > kMaxSplit) split = kMaxSplit;  // the merge holds at most kMaxSplit partials
  return split;
}

cudaError_t launch_attn_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_kc, const CUtensorMap& tm_vc,
                           const CUtensorMap& tm_kf, const CUtensorMap& tm_vf, const AttnTcArgs& a, int d,
                           cudaStream_t st, bool pdl) {
  const int units = a.S * a.Hkv * a.n_pairs * a.n_split;
  cudaError_t e;
  if (d == 128) {
    const int smem = AttnSmem<128>::kAlloc;
    if ((e = ensure_dynamic_smem(attn_tc_kernel<128>, smem)))
      return e;
    return launch_kernel(attn_tc_kernel<128>, dim3(units), dim3(kThreads), smem, st, pdl, tm_q, tm_kc, tm_vc,
                         tm_kf, tm_vf, a);
  } else {
    const int smem = AttnSmem<64>::kAlloc;
    if ((e = ensure_dynamic_smem(attn_tc_kernel<64>, smem)))
      return e;
    return launch_kernel(attn_tc_kernel<64>, dim3(units), dim3(kThreads), smem, st, pdl, tm_q, tm_kc, tm_vc,
                         tm_kf, tm_vf, a);
  }
  return cudaGetLastError();
}

MergeArgs merge_args(const AttnTcArgs& a, int d) {
  MergeArgs m{};
  m.out = a.out;
  m.out_s = a.out_s;
  m.out_row = a.out_row;
  m.lse = a.lse;
  m.lse_s = a.lse_s;
  m.o_part = a.o_part;
  m.ml_part = a.ml_part;
  m.S = a.S;
  m.Hq = a.Hq;
  m.T = a.T;
  m.n_split = a.n_split;
  m.d = d;
  return m;
}

cudaError_t launch_attn_combine(const AttnTcArgs& a, int d, cudaStream_t st, bool pdl) {
  const MergeArgs m = merge_args(a, d);
  const long long rows = (long long)a.S * a.Hq * a.T;
  const int blocks = (int)((merge_threads(rows, d) + 255) / 256);
  if (d == 128) return launch_kernel(attn_combine_kernel<128>, dim3(blocks), dim3(256), 0, st, pdl, m);
  return launch_kernel(attn_combine_kernel<64>, dim3(blocks), dim3(256), 0, st, pdl, m);
}

}  // namespace skv
