// Score pass on the 5th-generation tensor cores (bf16 in, f32 accumulate).
//
// The score of pool candidate j is the sum, over the frame's query rows i and
// the query heads h of its KV group, of the normalised attention weight
// P_hij = exp(s_hij - lse_hi) ("Linear Scaling Video VLMs for Long Video
// Understanding", P1 section 方法步骤详情: sum the attention weights over all
// queries; P2 A.3 "Kernel considerations": fused attention kernels do not
// expose the weights, so they are recomputed here from the row statistics and
// never written to memory).
//
// Transposed formulation: one CTA owns 128 candidates (keys) of one KV group
// and computes S^T = K Q^T, 128 keys (TMEM lanes) x 128 query rows (TMEM
// columns) per chunk, streaming the group's G*T query rows through a TMA ring.
// Each epilogue thread owns one key's TMEM lane, so the column sum of P is a
// private running sum: no shuffles, no atomics, deterministic.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 4..15 epilogue: three warpgroups (each covers the 128 TMEM
// lanes) take chunks round robin, so up to three chunks are in the epilogue
// while the MMA fills the fourth of the four TMEM accumulators.  Each
// epilogue warp reads its lanes 16 columns at a time with the next TMEM load
// in flight, and frees the accumulator as soon as its last load has landed.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace skv {
namespace {
using namespace tc;

constexpr int kStages = 4;
constexpr int kGroups = 3;                      // epilogue warpgroups (take chunks round robin)
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kThreads = 128 + 32 * kEpiWarps;  // warpgroup 0: producer, MMA, two idle warps
// registers: the launch gives each thread kRegsLaunch; warpgroup 0 drops to
// kRegsLow and the epilogue warpgroups rise to kRegsHigh within that total
constexpr int kRegsLaunch = (65536 / kThreads) / 8 * 8 > 168 ? 168 : (65536 / kThreads) / 8 * 8;
constexpr int kRegsLow = kGroups == 2 ? 72 : 56;
constexpr int kRegsHigh = ((kThreads * kRegsLaunch - 128 * kRegsLow) / (128 * kGroups)) / 8 * 8;
static_assert(128 * kRegsLow + 128 * kGroups * kRegsHigh <= kThreads * kRegsLaunch, "register split exceeds the launch");

template <int D>
struct Smem {
  static constexpr int kAtoms = D / 64;                  // 64-element (128-byte) swizzle atoms
  static constexpr int kAtomBytes = 128 * 128;           // 128 rows x 128 bytes
  static constexpr int kTileBytes = kAtoms * kAtomBytes;
  static constexpr int kK = 0;
  static constexpr int kQ = kK + kTileBytes;
  static constexpr int kRed = kQ + kStages * kTileBytes;  // (kGroups - 1) x 128 floats
  static constexpr int kBar = kRed + (kGroups - 1) * 128 * 4;
  // k_full, q_full[kStages], q_empty[kStages], acc_full[4], acc_empty[4], done
  static constexpr int kNumBars = 1 + 2 * kStages + 8 + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kLse = (kAbort + 4 + 15) & ~15;    // [kGroups][2][128] row statistics
  static constexpr int kBytes = kLse + kGroups * 2 * 128 * 4;
  static constexpr int kAlloc = kBytes + 1024;            // + room to align the base to 1024
};

// Exponentials of 16 columns (query rows i0 .. i0+15) of one key's TMEM lane,
// weighted by the rows' negated log2-sum-exps, added to four running sums.
__device__ __forceinline__ void score_cols16(const uint32_t (&rr)[16], const float* lse2, float scale_log2,
                                             bool need_mask, bool diag, int i0, int key, int T, float& acc0,
                                             float& acc1, float& acc2, float& acc3) {
  const float4* l4 = reinterpret_cast<const float4*>(lse2);
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    const float4 lv = l4[j4];  // -lse2 of 4 columns
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    const float2 x01 = ffma2(make_float2(__uint_as_float(rr[4 * j4 + 0]), __uint_as_float(rr[4 * j4 + 1])), sc2,
                             make_float2(lv.x, lv.y));
    const float2 x23 = ffma2(make_float2(__uint_as_float(rr[4 * j4 + 2]), __uint_as_float(rr[4 * j4 + 3])), sc2,
                             make_float2(lv.z, lv.w));
    float p0 = ex2_approx(x01.x);
    float p1 = ex2_approx(x01.y);
    float p2 = ex2_approx(x23.x);
    float p3 = ex2_approx(x23.y);
    if (need_mask) {
      // frame token `key` is seen by rows i >= key (frame-causal); rows past T do not exist
      const int i = i0 + 4 * j4;
      p0 = (i + 0 < T && (!diag || key <= i + 0)) ? p0 : 0.f;
      p1 = (i + 1 < T && (!diag || key <= i + 1)) ? p1 : 0.f;
      p2 = (i + 2 < T && (!diag || key <= i + 2)) ? p2 : 0.f;
      p3 = (i + 3 < T && (!diag || key <= i + 3)) ? p3 : 0.f;
    }
    const float2 a01 = fadd2(make_float2(acc0, acc1), make_float2(p0, p1));
    const float2 a23 = fadd2(make_float2(acc2, acc3), make_float2(p2, p3));
    acc0 = a01.x;
    acc1 = a01.y;
    acc2 = a23.x;
    acc3 = a23.y;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_kf, ScoreTcArgs a) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.y = (KV group, split of the group's query-row chunks)
  const int s = blockIdx.z, g = blockIdx.y / a.n_qsplit, qs = blockIdx.y % a.n_qsplit, tile = blockIdx.x;
  const bool is_c = tile < a.n_c_tiles;
  const int r0 = is_c ? tile * 128 : (tile - a.n_c_tiles) * 128;  // first C row / frame token
  const int G = a.Hq / a.Hkv;
  const int n_ic = (a.T + 127) / 128;
  // frame-causal: frame token t is seen only by query rows i >= t, so chunks
  // ending before r0 hold nothing visible for this tile
  const int ic_min = (!is_c && a.causal) ? r0 / 128 : 0;
  const int per_head = n_ic - ic_min;
  // this CTA takes chunks [c_lo, c_lo + n_chunks) of the group's G * per_head
  const int c_lo = qs * (G * per_head) / a.n_qsplit;
  const int n_chunks = (qs + 1) * (G * per_head) / a.n_qsplit - c_lo;

  const uint32_t bar_k = sb + L::kBar;
  auto bar_qfull = [&](int st) { return sb + L::kBar + 8u * (1 + st); };
  auto bar_qempty = [&](int st) { return sb + L::kBar + 8u * (1 + kStages + st); };
  auto bar_accfull = [&](int b) { return sb + L::kBar + 8u * (1 + 2 * kStages + b); };
  auto bar_accempty = [&](int b) { return sb + L::kBar + 8u * (5 + 2 * kStages + b); };
  const uint32_t bar_done = sb + L::kBar + 8u * (9 + 2 * kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  const unsigned long long wait_lim = a.wait_ns ? a.wait_ns : kWaitLimitNs;  // pipeline-wait limit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);

  if (threadIdx.x == 0) {
    mbar_init(bar_k, 1);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(bar_qfull(st), 1);
      mbar_init(bar_qempty(st), 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(bar_accfull(b), 1);
      mbar_init(bar_accempty(b), 4);  // the four warps of the group that owns chunk c's buffer
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);  // four 128-column f32 accumulators
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp < 4) regs_dec<kRegsLow>();
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(is_c ? &tm_kc : &tm_kf);
      mbar_arrive_expect_tx(bar_k, L::kTileBytes);
      for (int at = 0; at < L::kAtoms; ++at) {
        if (is_c) tma_load_4d(sb + L::kK + at * L::kAtomBytes, &tm_kc, bar_k, at * 64, r0, g, s);
        else tma_load_4d(sb + L::kK + at * L::kAtomBytes, &tm_kf, bar_k, at * 64, g, r0, s);
      }
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % kStages;
        if (!mbar_wait(bar_qempty(st), ((c / kStages) & 1) ^ 1, a.err, kErrWaitEmpty, abort_flag, wait_lim)) break;
        const int h = g * G + (c_lo + c) / per_head;
        const int i0 = (ic_min + (c_lo + c) % per_head) * 128;
        mbar_arrive_expect_tx(bar_qfull(st), L::kTileBytes);
        for (int at = 0; at < L::kAtoms; ++at)
          tma_load_4d(sb + L::kQ + st * L::kTileBytes + at * L::kAtomBytes, &tm_q, bar_qfull(st), at * 64, h,
                      i0, s);
        issued = c + 1;
      }
      // every armed load must land before the CTA may exit
      drain_wait(bar_k, 0, a.err);
      for (int c = (issued > kStages ? issued - kStages : 0); c < issued; ++c)
        drain_wait(bar_qfull(c % kStages), (c / kStages) & 1, a.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, false, false);
      bool ok = mbar_wait(bar_k, 0, a.err, kErrWaitLoad, abort_flag, wait_lim);
      for (int c = 0; ok && c < n_chunks; ++c) {
        const int st = c % kStages, buf = c & 3;
        if (!mbar_wait(bar_qfull(st), (c / kStages) & 1, a.err, kErrWaitLoad, abort_flag, wait_lim)) break;
        if (!mbar_wait(bar_accempty(buf), ((c >> 2) & 1) ^ 1, a.err, kErrWaitAccFree, abort_flag, wait_lim)) break;
        fence_after_sync();
        const uint32_t qbase = sb + L::kQ + st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kAtomBytes + (kk & 3) * 32;
          mma_ss(tmem + buf * 128, sdesc_sw128(sb + L::kK + off, 16, 1024), sdesc_sw128(qbase + off, 16, 1024),
                 idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_qempty(st));
        mma_commit(bar_accfull(buf));
      }
      mma_commit(bar_done);
      drain_wait(bar_done, 0, a.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    regs_inc<kRegsHigh>();
    const int ew = warp - 4;              // 0..7
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int half = ew >> 2;             // group: takes chunks half, half + kGroups, ...
    const int row = quarter * 32 + lane;  // key row within the tile
    const int key = r0 + row;
    // Row statistics in log2 units, negated, -inf past the frame: for each of
    // its chunks a warpgroup loads the 128 rows' statistics (one row per
    // thread: log2-sum-exp = max + log2(sum 2^(ml_u - max)) over the
    // attention's key splits, or the stored lse when unsplit) into its own
    // shared buffer; the loads for the next chunk are in flight while the
    // current chunk is processed.
    float* lse_wg = reinterpret_cast<float*>(smem + L::kLse) + half * 256;  // [2 slots][128 rows]
    const int r_wg = threadIdx.x & 127;                                     // row of the chunk this thread loads
    const int bar_wg = 3 + half;                                            // named barrier of the warpgroup
    float mlv[8];
    auto load_stats = [&](int c) {
      const int hh = (c_lo + c) / per_head;
      const int i = (ic_min + (c_lo + c) % per_head) * 128 + r_wg;
      const bool valid = i < a.T;
      const long long rowbase = (long long)(s * a.Hq + g * G + hh);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        mlv[u] = -INFINITY;
        if (valid && a.n_split > 1 && u < a.n_split) mlv[u] = __ldg(a.ml_part + (rowbase * a.n_split + u) * a.T + i);
      }
      if (valid && a.n_split <= 1) mlv[0] = __ldg(a.lse + rowbase * a.T + i) * kLog2e;
    };
    auto publish_stats = [&](float* dst) {
      float mx = mlv[0];
#pragma unroll
      for (int u = 1; u < 8; ++u) mx = fmaxf(mx, mlv[u]);
      float l2 = mx;
      if (a.n_split > 1 && mx > -INFINITY) {
        float ssum = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) ssum += mlv[u] == -INFINITY ? 0.f : ex2_approx(mlv[u] - mx);
        l2 = mx + __log2f(ssum);
      }
      // rows past the frame have no statistics: -inf makes their weight 0
      dst[r_wg] = mx == -INFINITY ? -INFINITY : -l2;
    };
    if (half < n_chunks) load_stats(half);
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    bool ok = true;
    for (int c = half, it = 0; c < n_chunks; c += kGroups, ++it) {
      const int buf = c & 3;
      const int i0 = (ic_min + (c_lo + c) % per_head) * 128;
      float* lse2 = lse_wg + (it & 1) * 128;
      publish_stats(lse2);
      if (c + kGroups < n_chunks) load_stats(c + kGroups);
      uint32_t got = 1;
      if (lane == 0) got = mbar_wait(bar_accfull(buf), (c >> 2) & 1, a.err, kErrWaitAcc, abort_flag, wait_lim) ? 1u : 0u;
      got = __shfl_sync(0xffffffffu, got, 0);
      // the warpgroup's four warps pass together (also when a wait gave up);
      // the barrier also publishes the chunk's row statistics
      if (named_bar_red_or(bar_wg, 128, got == 0)) {
        ok = false;
        break;
      }
      fence_after_sync();
      // some columns of this chunk precede some key of the tile (frame-causal),
      // or lie past the frame
      const bool diag = !is_c && a.causal && (i0 < r0 + 127);
      const bool need_mask = diag || i0 + 128 > a.T;
      // 16 columns at a time; the TMEM load of the next 16 is in flight while
      // the current 16 are exponentiated, and the accumulator is handed back
      // to the MMA issuer as soon as its last columns are in registers
      const uint32_t tb = tmem_addr(tmem, quarter * 32, buf * 128);
      uint32_t ra[16], rb[16];
      tmem_ld16(tb, ra);
      tmem_ld_wait();
#pragma unroll 1
      for (int q = 0; q < 8; q += 2) {
        tmem_ld16(tb + 16 * (q + 1), rb);
        score_cols16(ra, lse2 + 16 * q, a.scale_log2, need_mask, diag, i0 + 16 * q, key, a.T, acc0, acc1, acc2,
                     acc3);
        tmem_ld_wait();
        if (q + 2 < 8) tmem_ld16(tb + 16 * (q + 2), ra);
        if (q + 2 == 8) {
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_accempty(buf));
        }
        score_cols16(rb, lse2 + 16 * (q + 1), a.scale_log2, need_mask, diag, i0 + 16 * (q + 1), key, a.T, acc0,
                     acc1, acc2, acc3);
        if (q + 2 < 8) tmem_ld_wait();
      }
    }
    // combine the groups' partial sums of each key row (fixed order)
    float tot = (acc0 + acc1) + (acc2 + acc3);
    float* red = reinterpret_cast<float*>(smem + L::kRed);
    if (half > 0) red[(half - 1) * 128 + row] = tot;
    named_bar_sync(1, 32 * kEpiWarps);
    if (half == 0 && ok && !*abort_flag) {
      for (int gr = 1; gr < kGroups; ++gr) tot += red[(gr - 1) * 128 + row];
      const bool valid = is_c ? key < a.m : key < a.T;
      if (valid) {
        const int j = is_c ? key : a.m + key;
        a.part[s * a.part_s + (long long)(g * a.n_qsplit + qs) * a.part_g + j] = tot;
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

}  // namespace

int score_tc_qsplit(int S, int Hq, int Hkv, int T, int m, int n_sm) {
  const int n_tiles = (m + 127) / 128 + (T + 127) / 128;
  const int ctas = S * Hkv * n_tiles;
  if (ctas <= 0 || Hkv <= 0) return 1;
  const int chunks = (Hq / Hkv) * ((T + 127) / 128);  // query-row chunks of a group
  int q = n_sm / ctas;
  q = std::min(q, std::min(chunks, kMaxQsplit));
  return std::max(q, 1);
}

cudaError_t launch_score_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_kc, const CUtensorMap& tm_kf,
                            const ScoreTcArgs& a, int d, cudaStream_t st, bool pdl) {
  const int n_tiles = a.n_c_tiles + a.n_f_tiles;
  if (n_tiles == 0) return cudaSuccess;
  dim3 grid(n_tiles, a.Hkv * a.n_qsplit, a.S);
  cudaError_t e;
  if (d == 128) {
    const int smem = Smem<128>::kAlloc;
    if ((e = ensure_dynamic_smem(score_tc_kernel<128>, smem)))
      return e;
    return launch_kernel(score_tc_kernel<128>, grid, dim3(kThreads), smem, st, pdl, tm_q, tm_kc, tm_kf, a);
  } else {
    const int smem = Smem<64>::kAlloc;
    if ((e = ensure_dynamic_smem(score_tc_kernel<64>, smem)))
      return e;
    return launch_kernel(score_tc_kernel<64>, grid, dim3(kThreads), smem, st, pdl, tm_q, tm_kc, tm_kf, a);
  }
  return cudaGetLastError();
}

}  // namespace skv
