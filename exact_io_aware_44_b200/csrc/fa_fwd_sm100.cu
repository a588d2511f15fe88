// fa_fwd_sm100.cu -- attention forward on sm_100a tensor cores (bf16, or E4M3 inputs).
//
// The method is the tiled forward with the online softmax: each query tile
// streams the key/value tiles through on-chip memory, keeps a running row max m
// and denominator l, rescales the partial output when m grows, and divides by l
// once at the end ("FlashAttention Kernel & Online Softmax", first paragraph;
// "FlashAttention" blog, mechanics of the running m, ell and O). The N x N score
// matrix only ever exists as one 128 x 128 tile in Tensor Memory.
//
// The kernel is persistent: one CTA per SM, 384 threads, looping over work units
// of two 128-row query tiles of one (batch, head). Units are
// dealt to the CTAs in rounds, in snake order over a heavy-first list; Tensor
// Memory, the barriers and the K/V ring stay set up from one unit to the next,
// and the next unit's Q and K/V loads overlap the current unit's last tiles.
//   warp 0      TMA producer: per unit, Q (once the previous unit's score MMAs
//               are done with it), then K_0, V_0, K_1, V_1, ... through one ring
//               of shared-memory stages guarded by mbarriers (full / empty).
//   warp 1      allocates Tensor Memory; lane 0 issues every tcgen05.mma:
//               S_t = Q_t K_j^T into TMEM, then O_t += P_t V_j with P_t read
//               from TMEM.
//   warps 4-7   softmax for query tile 0 (thread = query row = TMEM lane).
//   warps 8-11  softmax for query tile 1.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 [384,384+d);
// P_t (bf16 pairs, 64 columns) overwrites the first half of S_t once it is read.
//
// E4M3 or E5M2 inputs (d = 128) run the same kernel with kind::f8f6f4 MMAs: a
// tile is 16 KB (one 128-byte swizzle block wide), the ring holds 10 stages, an
// MMA steps 32 elements of K, and P is rounded to the inputs' format, four keys
// per TMEM column (32 columns), so both operands of every MMA share one type. The
// Q and K descales fold into c; V's descale multiplies the final 1/l.
//
// Per key tile j, a softmax thread loads its row of S_t, applies the causal
// mask on the diagonal tile, updates the running max, and computes
// P = 2^(S c - m c) with c = scale * log2(e) on the SFU. It rescales its row
// of O_t in TMEM only when the max grew by more than 2^8; otherwise the stale
// max stays the reference, which is exact because the final division uses the
// same reference. It stores P as bf16 into Tensor Memory, where the P V product
// reads it: P never touches shared memory, whose bandwidth the score MMAs and
// the K/V loads already use. The epilogue divides O by l, stores O as bf16 and
// writes LSE = (m c + log2 l) ln 2.
//
// MMA issue order: S_0(0), S_1(0), then per key tile j: PV_0(j), S_0(j+1),
// PV_1(j), S_1(j+1). S_t(j+1) overwrites the columns PV_t(j) reads; one
// thread's MMAs execute in issue order. The commit after S_t(j+1) also covers
// PV_t(j), so when a softmax warpgroup sees S_t(j+1), O_t is complete and may be
// rescaled. While one softmax warpgroup exponentiates, the tensor core runs the
// other tile's P V and scores.
//
// d = 256 (fwd256_kernel, further down): the O tile alone takes 256 columns, so a
// CTA holds one query tile, and the spare 128 columns double-buffer its scores.
#include <math.h>

#include <algorithm>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kFwdThreads = 384;
// Register split: 384 threads x 168 at launch = 64512 = 128 x 88 (producer /
// MMA warpgroup) + 256 x 208 (the two softmax warpgroups).
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
static_assert(kFwdThreads * kRegsLaunch == 128 * kRegsControl + 256 * kRegsSoftmax, "register split");
constexpr uint32_t kRescaleThresholdLog2 = 8;  // rescale only when m grows by > 2^8
// Launch persistently when an average work unit visits at most this many key tiles.
constexpr int kPersistentMaxKv = 8;
#ifndef FA_FWD_POLY_PAIRS
#define FA_FWD_POLY_PAIRS 0
#endif
// Of every 8 key pairs, how many take 2^x by polynomial on the FMA pipe instead
// of the SFU (0 = all on the SFU).
constexpr int kPolyPairs = FA_FWD_POLY_PAIRS;
#ifndef FA_FWD64_POLY_PAIRS
#define FA_FWD64_POLY_PAIRS 2
#endif
constexpr int kPolyPairs64 = FA_FWD64_POLY_PAIRS;  // the same, for d = 64 (bf16)

// D: head dim; FP8: 8-bit Q, K, V and P (E4M3 or E5M2, kind::f8f6f4 MMAs), else bf16 (kind::f16).
template <int D, bool FP8>
struct FwdCfg {
  static constexpr int kElem = FP8 ? 1 : 2;                      // bytes per element
  static_assert(D == 64 || D == 128, "d = 256 has a kernel of its own (fwd256_kernel)");
  static constexpr int kTiles = 2;  // query tiles per CTA
  // K/V ring: K_0, V_0, K_1, V_1, ...
  static constexpr int kStages = (FP8 || D == 64) ? 10 : 5;
  static constexpr int kTileBytes = kTileM * D * kElem;          // one Q, K or V tile
  static constexpr int kRegion = kTileM * 128;                   // one 128-byte-wide column block
  static constexpr int kRegions = D * kElem / 128;               // column blocks per tile
  static constexpr int kBoxCols = 128 / kElem;                   // elements per block row
  static constexpr int kKStep = 32 / kElem;                      // K per MMA (32 bytes of each row)
  static constexpr int kSSteps = D / kKStep;                     // MMAs per S tile
  static constexpr int kPvSteps = kTileN / kKStep;               // MMAs per P V (8 TMEM columns each)
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kOffQ + kTiles * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  // q_full, q_empty, full[S], empty[S], s_ready[2], p_ready[2], o_done[2], mma_final
  static constexpr int kNumBars = 2 + 2 * kStages + 7;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base to 1024
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Element kinds: bf16 (kind::f16 MMAs), or an 8-bit float for Q, K, V and P
// (kind::f8f6f4 MMAs with E4M3 or E5M2 in both operands).
constexpr int kKindBf16 = 0, kKindE4M3 = 1, kKindE5M2 = 2;

// kind::f8f6f4 instruction descriptor with both operand formats set (E4M3 = 0, E5M2 = 1).
__host__ __device__ constexpr uint32_t idesc_f8_f32(int kind, int M, int N, bool a_mn, bool b_mn) {
  return idesc_e4m3_f32(M, N, a_mn, b_mn) | ((kind == kKindE5M2 ? 1u : 0u) << 7) |
         ((kind == kKindE5M2 ? 1u : 0u) << 10);
}
// Four fp32 values to E5M2 (round to nearest, saturating), packed low byte first.
__device__ __forceinline__ uint32_t pack_e5m2x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e5m2x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e5m2x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// Work units: one (batch, head, block of kTiles query tiles) each. Heads are taken in
// groups of p.head_group, whose K/V fit in L2 together, so that CTAs running at the
// same time share them; within a group the longest (last) query blocks of all its
// heads come first, so that the causal tail ends on short blocks.
struct FwdUnit {
  int b, h, kv_head, q0, n_kv;
  int n_iter[2];  // key tiles each query tile visits (0: the tile is past N)
};

template <int kTiles>
__device__ __forceinline__ FwdUnit fwd_unit(const FwdParams& p, int u) {
  FwdUnit U;
  const int grp0 = (u / (p.head_group * p.n_qblk)) * p.head_group;
  const int gsz = min(p.head_group, p.B * p.Hq - grp0);
  const int r = u - grp0 * p.n_qblk;
  const int bh = grp0 + r % gsz;
  const int qb = p.n_qblk - 1 - r / gsz;
  U.b = bh / p.Hq;
  U.h = bh % p.Hq;
  U.kv_head = U.b * p.Hkv + U.h / (p.Hq / p.Hkv);
  U.q0 = qb * kTiles * kTileM;
  const int n_kv_all = (p.N + kTileN - 1) / kTileN;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = U.q0 / kTileM + t;
    const bool active = t < kTiles && U.q0 + t * kTileM < p.N;
    U.n_iter[t] = !active ? 0 : (p.causal ? qt + 1 : n_kv_all);
  }
  U.n_kv = max(U.n_iter[0], U.n_iter[1]);
  return U;
}

// The k-th unit of this CTA in a persistent grid of gridDim.x CTAs: rounds of
// gridDim.x consecutive units, taken in snake order (CTA i takes the i-th unit of
// even rounds and the i-th from the end of odd rounds), so that a CTA given a long
// unit in one round gets a short one in the next. Returns n_units when done. (With
// one CTA per unit the 0-th unit is blockIdx.x.)
__device__ __forceinline__ int fwd_unit_index(int k, int n_units) {
  const int G = (int)gridDim.x;
  const int c = (int)blockIdx.x;
  const long long u = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
  return u < n_units ? (int)u : n_units;
}

// PERSIST: the grid has fewer CTAs than units and every CTA loops over its share;
// otherwise each CTA runs exactly one unit (blockIdx.x) and the unit loops fold away.
template <int D, int KIND, bool PERSIST>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  constexpr bool FP8 = KIND != kKindBf16;
  using C = FwdCfg<D, FP8>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* ring_full = bars + 2;
  uint64_t* ring_empty = ring_full + S;
  uint64_t* s_ready = ring_empty + S;
  uint64_t* p_ready = s_ready + 2;
  uint64_t* o_done = p_ready + 2;
  uint64_t* mma_final = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.B * p.Hq * p.n_qblk;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_ready[t], 1);
      mbar_init(&p_ready[t], kTileM);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx w{abort_flag, p.status, p.wait_budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Per unit: Q (once the previous unit's score MMAs are done with it), then
    // K_0, V_0, K_1, V_1, ... through the ring, whose position carries across units.
    regs_dec<kRegsControl, kRegsLaunch>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;
      int q_loads = 0;  // Q loads issued (one per unit)
      auto push = [&](const CUtensorMap* map, int kv_tile, int kv_head) -> bool {
        const int s = it % S;
        if (!mbar_wait_spin(&ring_empty[s], ((it / S) & 1) ^ 1, w)) return false;
        mbar_arrive_expect_tx(&ring_full[s], C::kTileBytes);
#pragma unroll
        for (int z = 0; z < C::kRegions; ++z)
          tma_load_3d(smem + C::kOffKV + s * C::kTileBytes + z * C::kRegion, map, &ring_full[s], z * C::kBoxCols,
                      kv_tile * kTileN, kv_head);
        ++it;
        return true;
      };
      bool ok = true;
      for (int k = 0; ok && (PERSIST || k == 0); ++k) {
        const int u = fwd_unit_index(k, n_units);
        if (u >= n_units) break;
        const FwdUnit U = fwd_unit<C::kTiles>(p, u);
        if (k > 0 && !(ok = mbar_wait_spin(q_empty, (k - 1) & 1, w))) break;
        const int n_qt = U.n_iter[1] > 0 ? 2 : 1;
        mbar_arrive_expect_tx(q_full, n_qt * C::kTileBytes);
        for (int t = 0; t < n_qt; ++t)
#pragma unroll
          for (int z = 0; z < C::kRegions; ++z)
            tma_load_3d(smem + C::kOffQ + t * C::kTileBytes + z * C::kRegion, &tmQ, q_full, z * C::kBoxCols,
                        U.q0 + t * kTileM, U.b * p.Hq + U.h);
        ++q_loads;
        for (int j = 0; j < U.n_kv && ok; ++j) {
          ok = push(&tmK, j, U.kv_head);
          if (ok) ok = push(&tmV, j, U.kv_head);
        }
      }
      if (!ok) {
        // Error path: let the loads already issued land before the CTA exits.
        WaitCtx drain{abort_flag, p.status, 20000000ull};
        volatile int zero = 0;
        drain.abort_flag = &zero;
        for (int kk = max(0, it - S); kk < it; ++kk) mbar_wait(&ring_full[kk % S], (kk / S) & 1, drain);
        if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this role so that descriptors are warp-uniform; lane 0
    // alone issues tcgen05.mma and tcgen05.commit. Descriptors are built once and
    // advanced by constant offsets of the start-address field.
    regs_dec<kRegsControl, kRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdescS =
        FP8 ? idesc_f8_f32(KIND, kTileM, kTileN, false, false) : idesc_bf16_f32(kTileM, kTileN, false, false);
    constexpr uint32_t kIdescPV =
        FP8 ? idesc_f8_f32(KIND, kTileM, D, false, true) : idesc_bf16_f32(kTileM, D, false, true);
    const uint64_t d_q = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t d_k = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);           // K-major view
    const uint64_t d_v = sdesc_sw128(smem_u32(smem + C::kOffKV), C::kRegion, 1024);   // MN-major view
    int cnt = 0;
    auto take = [&](int& slot) -> bool {  // next stage of the ring
      slot = cnt % S;
      const bool res = warp_wait_spin(&ring_full[slot], (cnt / S) & 1, w);
      ++cnt;
      tc_fence_after();
      return res;
    };
    auto issue_s = [&](int t, int slot) {
      const uint64_t a0 = desc_advance(d_q, t * C::kTileBytes);
      const uint64_t b0 = desc_advance(d_k, slot * C::kTileBytes);
#pragma unroll
      for (int k = 0; k < C::kSSteps; ++k) {
        const uint32_t off = (k >> 2) * C::kRegion + (k & 3) * 32;
        if (leader) {
          if constexpr (FP8)
            mma_e4m3_ss(tmem + t * 128, desc_advance(a0, off), desc_advance(b0, off), kIdescS, k > 0 ? 1u : 0u);
          else
            mma_bf16_ss(tmem + t * 128, desc_advance(a0, off), desc_advance(b0, off), kIdescS, k > 0 ? 1u : 0u);
        }
      }
      if (leader) mma_commit(&s_ready[t]);
    };
    auto issue_pv = [&](int t, int slot, int j) {
      const uint64_t b0 = desc_advance(d_v, slot * C::kTileBytes);
#pragma unroll
      for (int k = 0; k < C::kPvSteps; ++k) {
        if (leader) {
          const uint64_t bk = desc_advance(b0, k * C::kKStep * 128);
          if constexpr (FP8)
            mma_e4m3_ts(tmem + 256 + t * 128, tmem + t * 128 + k * 8, bk, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
          else
            mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + k * 8, bk, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
        }
      }
    };
    int p_base[2] = {0, 0};  // p_ready phases completed in earlier units, per tile
    // progress record: the P V products this CTA has issued (both tiles, all its units)
    unsigned* const prog = (int)blockIdx.x < p.progress_n ? p.progress : nullptr;
    unsigned pv_count = 0;
    if (leader && prog) prog[blockIdx.x] = 0u;
    bool ok = true;
    for (int k = 0; ok && (PERSIST || k == 0); ++k) {
      const int u = fwd_unit_index(k, n_units);
      if (u >= n_units) break;
      const FwdUnit U = fwd_unit<C::kTiles>(p, u);
      if (!(ok = warp_wait_spin(q_full, k & 1, w))) break;
      tc_fence_after();
      {
        int kslot;
        if (!(ok = take(kslot))) break;
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (U.n_iter[t] > 0) issue_s(t, kslot);
        if (leader) {
          mma_commit(&ring_empty[kslot]);
          if (U.n_kv == 1) mma_commit(q_empty);  // the unit's score MMAs are all issued
        }
      }
      for (int j = 0; j < U.n_kv && ok; ++j) {
        int vslot, kslot = -1;
        if (!(ok = take(vslot))) break;
#pragma unroll
        for (int t = 0; t < 2; ++t) {  // unrolled: t, the TMEM columns and barriers are constants
          if (j >= U.n_iter[t]) continue;
          if (!(ok = warp_wait_spin(&p_ready[t], (p_base[t] + j) & 1, w))) break;
          if (leader && prog) prog[blockIdx.x] = (unsigned)(++pv_count);
          tc_fence_after();
          issue_pv(t, vslot, j);
          if (j + 1 < U.n_iter[t]) {
            if (kslot < 0 && !(ok = take(kslot))) break;
            issue_s(t, kslot);
          } else if (leader) {
            mma_commit(&o_done[t]);
          }
        }
        if (!ok) break;
        if (leader) {
          mma_commit(&ring_empty[vslot]);
          if (kslot >= 0) mma_commit(&ring_empty[kslot]);
          // the unit's last score MMAs were issued in this iteration: Q may be replaced
          if (j + 2 == U.n_kv) mma_commit(q_empty);
        }
      }
      p_base[0] += U.n_iter[0];
      p_base[1] += U.n_iter[1];
    }
    // Every MMA issued above must finish before TMEM is released.
    if (leader) mma_commit(mma_final);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_final, 0, drain);
  } else if (warp < 4) {
    regs_dec<kRegsControl, kRegsLaunch>();
  } else {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsSoftmax, kRegsLaunch>();
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    const float c = p.scale_log2;
    int s_base = 0;  // s_ready phases of this tile completed in earlier units
    int o_base = 0;  // o_done phases of this tile completed in earlier units
    bool ok = true;
    for (int k = 0; ok && (PERSIST || k == 0); ++k) {
      const int u = fwd_unit_index(k, n_units);
      if (u >= n_units) break;
      const FwdUnit U = fwd_unit<C::kTiles>(p, u);
      const int n = U.n_iter[t];
      if (n == 0) continue;
      const int qrow = U.q0 + t * kTileM + row;
      float m_ref = -INFINITY;  // reference max (raw score units)
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        if (!(ok = consumer_wait(&s_ready[t], (s_base + j) & 1, w))) break;
        tc_fence_after();
        float s[kTileN];
#pragma unroll
        for (int cc = 0; cc < kTileN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tS + cc * 32, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
        }

        const int k0 = j * kTileN;
        if (p.causal && j == n - 1) {
          const int lim = qrow - k0;  // keys with column > lim are in the future
#pragma unroll
          for (int i = 0; i < kTileN; ++i)
            if (i > lim) s[i] = -INFINITY;
        } else if (!p.causal && j == n - 1 && p.N - k0 < kTileN) {
          const int lim = p.N - k0;
#pragma unroll
          for (int i = 0; i < kTileN; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
        // row max: four independent chains of 3-input max
        float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int i = 4; i < kTileN; i += 8) {
          mq[0] = fmax3(mq[0], s[i], s[i + 1]);
          mq[1] = fmax3(mq[1], s[i + 2], s[i + 3]);
          if (i + 4 < kTileN) mq[2] = fmax3(mq[2], s[i + 4], s[i + 5]);  // the last step has 4 left
          if (i + 6 < kTileN) mq[3] = fmax3(mq[3], s[i + 6], s[i + 7]);
        }
        const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
        const float m_new = fmaxf(m_ref, mx);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_ref = m_new;
        } else if ((m_new - m_ref) * c > (float)kRescaleThresholdLog2) {
          alpha = ex2((m_ref - m_new) * c);
          m_ref = m_new;
          l *= alpha;
          rescale = true;
        }
        const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
        // P = 2^(S c - m c), packed at once (bf16 pairs, or E4M3 quads: one TMEM column
        // each); l sums the fp32 values. P <= 2^8 fits E4M3; E4M3 flushes P < 2^-10 to zero.
        uint32_t pk[kTileN / (FP8 ? 4 : 2)];
        uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
        const uint64_t c2 = f2_pack(c, c), nmc2 = f2_pack(-mc, -mc);
#pragma unroll
        for (int i = 0; i < kTileN; i += 4) {
          // x = S c - m c for four keys (two packed FMAs), then 2^x: on the SFU, or for
          // kPolyPairs of every 8 key pairs by the polynomial on the FMA pipe.
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(s[i], s[i + 1]), c2, nmc2), x0, x1);
          f2_unpack(f2_fma(f2_pack(s[i + 2], s[i + 3]), c2, nmc2), x2, x3);
          float e0, e1, e2, e3;
          if (((i / 2) & 7) < (D == 64 ? kPolyPairs64 : kPolyPairs)) {
            ex2_poly2(x0, x1, e0, e1);
          } else {
            e0 = ex2(x0);
            e1 = ex2(x1);
          }
          if (((i / 2 + 1) & 7) < (D == 64 ? kPolyPairs64 : kPolyPairs)) {
            ex2_poly2(x2, x3, e2, e3);
          } else {
            e2 = ex2(x2);
            e3 = ex2(x3);
          }
          rs2[0] = f2_add(rs2[0], f2_pack(e0, e1));
          rs2[1] = f2_add(rs2[1], f2_pack(e2, e3));
          if constexpr (FP8) {
            pk[i / 4] = KIND == kKindE5M2 ? pack_e5m2x4(e0, e1, e2, e3) : pack_e4m3x4(e0, e1, e2, e3);
          } else {
            pk[i / 2] = pack_bf16x2(e0, e1);
            pk[i / 2 + 1] = pack_bf16x2(e2, e3);
          }
        }
        float ra, rb, rc, rd;
        f2_unpack(rs2[0], ra, rb);
        f2_unpack(rs2[1], rc, rd);
        l += (ra + rb) + (rc + rd);

        // PV(j-1) has completed (the commit of S(j) covers it): O may be rescaled.
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            tmem_ld32(tO + cc * 32, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tO + cc * 32, r);
          }
        }
        // P into the first columns of S_t (its scores are in registers now).
        if constexpr (FP8) {
          tmem_st32(tS, pk);
        } else {
          uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(&pk[0]);
          uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(&pk[32]);
          tmem_st32(tS, lo);
          tmem_st32(tS + 32, hi);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_ready[t]);
      }
      if (ok && (ok = consumer_wait(&o_done[t], o_base & 1, w))) {
        tc_fence_after();
        const float inv_l = p.o_scale / l;
        const bool valid = qrow < p.N;
        const size_t row_idx = (size_t)(U.b * p.Hq + U.h) * p.N + qrow;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row_idx * D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tO + cc * 32, r);
          tmem_ld_wait(r);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 pk4;
              const int i = v4 * 8;
              pk4.x = pack_bf16x2(__uint_as_float(r[i + 0]) * inv_l, __uint_as_float(r[i + 1]) * inv_l);
              pk4.y = pack_bf16x2(__uint_as_float(r[i + 2]) * inv_l, __uint_as_float(r[i + 3]) * inv_l);
              pk4.z = pack_bf16x2(__uint_as_float(r[i + 4]) * inv_l, __uint_as_float(r[i + 5]) * inv_l);
              pk4.w = pack_bf16x2(__uint_as_float(r[i + 6]) * inv_l, __uint_as_float(r[i + 7]) * inv_l);
              dst[cc * 4 + v4] = pk4;
            }
          }
        }
        if (valid) p.lse[row_idx] = (m_ref * c + log2f(l)) * 0.6931471805599453f;
      }
      s_base += n;
      ++o_base;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------
// fwd256_kernel (bf16, d = 256): one 128-row query tile per CTA, one CTA per unit.
// The O tile takes 256 TMEM columns, which leaves room for two score buffers, so the
// scores of key tile j+1 are computed while the softmax works on tile j, and the
// chain P(j) -> P V(j) -> S(j+1) -> softmax(j+1) of the one-buffer design leaves the
// critical path: the tensor core does P V(j-1) and S(j+1) while the softmax works. What
// bounds it then is the tensor core itself: an S product reads both operands from shared
// memory (8 KB per 64-cycle MMA, the SM's whole shared-memory bandwidth) while the K/V
// loads write into it, so it runs at about 60 % of the MMA rate.
//   TMEM: S buffers [0,128) and [128,256) (key tile parity), O [256,512).
//   warp 0      TMA producer: Q (64 KB), then K and V in 32 KB halves (128 of the
//               256 columns) through a ring of 5 stages, in the order the MMAs use
//               them: K_0, K_1, V_0, K_2, V_1, K_3, ...
//   warp 1      MMA issuer: S(0), S(1); then per key tile j, once P(j) is stored,
//               O += P(j) V_j (two N = 128 halves per K step) and S(j+2) into the
//               buffer P(j) came from (issued after P V(j), and one thread's MMAs run
//               in issue order).
//   warps 4-7   softmax (thread = query row = TMEM lane), as in fwd_kernel; before it
//               stores P(j) it waits for P V(j-1) to finish (which it normally already
//               has), so that O may be rescaled.
// P (bf16 pairs, 64 columns) overwrites the first half of its S buffer.
struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kRegion = kTileM * 128;     // 16 KB: 128 rows x 64 columns (128-byte swizzle)
  static constexpr int kHalf = 2 * kRegion;        // 32 KB: 128 columns of a K or V tile
  static constexpr int kStages = 5;
  static constexpr int kOffQ = 0;                  // Q: 4 regions
  static constexpr int kOffKV = 4 * kRegion;
  static constexpr int kOffBar = kOffKV + kStages * kHalf;
  // q_full, full[S], empty[S], s_ready[2], p_ready, o_ready, mma_final
  static constexpr int kNumBars = 1 + 2 * kStages + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
};

__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Fwd256Cfg;
  constexpr int S = C::kStages;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* ring_full = bars + 1;
  uint64_t* ring_empty = ring_full + S;
  uint64_t* s_ready = ring_empty + S;
  uint64_t* p_ready = s_ready + 2;
  uint64_t* o_ready = p_ready + 1;
  uint64_t* mma_final = o_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const FwdUnit U = fwd_unit<1>(p, (int)blockIdx.x);
  const int n = U.n_iter[0];  // key tiles of this query tile (>= 1: the tile starts below N)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    mbar_init(&s_ready[0], 1);
    mbar_init(&s_ready[1], 1);
    mbar_init(p_ready, kTileM);
    mbar_init(o_ready, 1);
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx w{abort_flag, p.status, p.wait_budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    regs_dec<kRegsControl, kRegsLaunch>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 4 * C::kRegion);
#pragma unroll
      for (int z = 0; z < 4; ++z)
        tma_load_3d(smem + C::kOffQ + z * C::kRegion, &tmQ, q_full, z * 64, U.q0, U.b * p.Hq + U.h);
      int it = 0;
      // one K or V tile: its two 32 KB halves, each in a stage of its own
      auto push = [&](const CUtensorMap* map, int kv_tile) -> bool {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int s = it % S;
          if (!mbar_wait_spin(&ring_empty[s], ((it / S) & 1) ^ 1, w)) return false;
          mbar_arrive_expect_tx(&ring_full[s], C::kHalf);
#pragma unroll
          for (int z = 0; z < 2; ++z)
            tma_load_3d(smem + C::kOffKV + s * C::kHalf + z * C::kRegion, map, &ring_full[s], (half * 2 + z) * 64,
                        kv_tile * kTileN, U.kv_head);
          ++it;
        }
        return true;
      };
      bool ok = push(&tmK, 0);
      if (ok && n > 1) ok = push(&tmK, 1);
      for (int j = 0; j < n && ok; ++j) {
        ok = push(&tmV, j);
        if (ok && j + 2 < n) ok = push(&tmK, j + 2);
      }
      if (!ok) {
        // Error path: let the loads already issued land before the CTA exits.
        WaitCtx drain{abort_flag, p.status, 20000000ull};
        volatile int zero = 0;
        drain.abort_flag = &zero;
        for (int kk = max(0, it - S); kk < it; ++kk) mbar_wait(&ring_full[kk % S], (kk / S) & 1, drain);
        mbar_wait(q_full, 0, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kRegsControl, kRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, 128, false, true);  // one 128-column half of O
    const uint64_t d_q = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t d_k = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);          // K-major view
    const uint64_t d_v = sdesc_sw128(smem_u32(smem + C::kOffKV), C::kRegion, 1024);  // MN-major view
    int cnt = 0;
    auto take = [&](int& slot) -> bool {  // next stage of the ring
      slot = cnt % S;
      const bool res = warp_wait_spin(&ring_full[slot], (cnt / S) & 1, w);
      ++cnt;
      tc_fence_after();
      return res;
    };
    // S(j) = Q K_j^T into buffer buf: 16 K steps, the first 8 from K's first half
    auto issue_s = [&](int buf) -> bool {
      int sa, sb;
      if (!take(sa) || !take(sb)) return false;
      const uint64_t ka = desc_advance(d_k, sa * C::kHalf), kb = desc_advance(d_k, sb * C::kHalf);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint32_t qoff = (k >> 2) * C::kRegion + (k & 3) * 32;
        const uint32_t koff = ((k >> 2) & 1) * C::kRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + buf * 128, desc_advance(d_q, qoff), desc_advance(k < 8 ? ka : kb, koff), kIdescS,
                      k > 0 ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&s_ready[buf]);
        mma_commit(&ring_empty[sa]);
        mma_commit(&ring_empty[sb]);
      }
      return true;
    };
    // O += P(j) V_j: P from buffer buf, V's halves give O's column halves
    auto issue_pv = [&](int buf, int j) -> bool {
      int sa, sb;
      if (!take(sa) || !take(sb)) return false;
      const uint64_t va = desc_advance(d_v, sa * C::kHalf), vb = desc_advance(d_v, sb * C::kHalf);
#pragma unroll
      for (int k = 0; k < kTileN / 16; ++k) {
        if (leader) {
          const uint32_t acc = (j > 0 || k > 0) ? 1u : 0u;
          mma_bf16_ts(tmem + 256, tmem + buf * 128 + k * 8, desc_advance(va, k * 16 * 128), kIdescPV, acc);
          mma_bf16_ts(tmem + 384, tmem + buf * 128 + k * 8, desc_advance(vb, k * 16 * 128), kIdescPV, acc);
        }
      }
      if (leader) {
        mma_commit(o_ready);
        mma_commit(&ring_empty[sa]);
        mma_commit(&ring_empty[sb]);
      }
      return true;
    };
    unsigned* const prog = (int)blockIdx.x < p.progress_n ? p.progress : nullptr;
    if (leader && prog) prog[blockIdx.x] = 0u;
    bool ok = warp_wait_spin(q_full, 0, w);
    tc_fence_after();
    if (ok) ok = issue_s(0);
    if (ok && n > 1) ok = issue_s(1);
    for (int j = 0; j < n && ok; ++j) {
      if (!(ok = warp_wait_spin(p_ready, j & 1, w))) break;
      tc_fence_after();
      if (leader && prog) prog[blockIdx.x] = (unsigned)(j + 1);
      if (!(ok = issue_pv(j & 1, j))) break;
      if (j + 2 < n) ok = issue_s(j & 1);
    }
    // Every MMA issued above must finish before TMEM is released.
    if (leader) mma_commit(mma_final);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_final, 0, drain);
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsSoftmax, kRegsLaunch>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + 256;
    const float c = p.scale_log2;
    const int qrow = U.q0 + row;
    float m_ref = -INFINITY;  // reference max (raw score units)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int buf = j & 1;
      const uint32_t tS = tmem + lane_off + buf * 128;
      if (!(ok = consumer_wait(&s_ready[buf], (j >> 1) & 1, w))) break;
      tc_fence_after();
      float s[kTileN];
#pragma unroll
      for (int cc = 0; cc < kTileN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tS + cc * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
      }
      const int k0 = j * kTileN;
      if (p.causal && j == n - 1) {
        const int lim = qrow - k0;  // keys with column > lim are in the future
#pragma unroll
        for (int i = 0; i < kTileN; ++i)
          if (i > lim) s[i] = -INFINITY;
      } else if (!p.causal && j == n - 1 && p.N - k0 < kTileN) {
        const int lim = p.N - k0;
#pragma unroll
        for (int i = 0; i < kTileN; ++i)
          if (i >= lim) s[i] = -INFINITY;
      }
      float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int i = 4; i < kTileN; i += 8) {
        mq[0] = fmax3(mq[0], s[i], s[i + 1]);
        mq[1] = fmax3(mq[1], s[i + 2], s[i + 3]);
        if (i + 4 < kTileN) mq[2] = fmax3(mq[2], s[i + 4], s[i + 5]);  // the last step has 4 left
        if (i + 6 < kTileN) mq[3] = fmax3(mq[3], s[i + 6], s[i + 7]);
      }
      const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
      const float m_new = fmaxf(m_ref, mx);
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_ref = m_new;
      } else if ((m_new - m_ref) * c > (float)kRescaleThresholdLog2) {
        alpha = ex2((m_ref - m_new) * c);
        m_ref = m_new;
        l *= alpha;
        rescale = true;
      }
      const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
      uint32_t pk[kTileN / 2];
      uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
      const uint64_t c2 = f2_pack(c, c), nmc2 = f2_pack(-mc, -mc);
#pragma unroll
      for (int i = 0; i < kTileN; i += 4) {
        float x0, x1, x2, x3;
        f2_unpack(f2_fma(f2_pack(s[i], s[i + 1]), c2, nmc2), x0, x1);
        f2_unpack(f2_fma(f2_pack(s[i + 2], s[i + 3]), c2, nmc2), x2, x3);
        const float e0 = ex2(x0), e1 = ex2(x1), e2 = ex2(x2), e3 = ex2(x3);
        rs2[0] = f2_add(rs2[0], f2_pack(e0, e1));
        rs2[1] = f2_add(rs2[1], f2_pack(e2, e3));
        pk[i / 2] = pack_bf16x2(e0, e1);
        pk[i / 2 + 1] = pack_bf16x2(e2, e3);
      }
      float ra, rb, rc, rd;
      f2_unpack(rs2[0], ra, rb);
      f2_unpack(rs2[1], rc, rd);
      l += (ra + rb) + (rc + rd);
      // P V(j-1) must be done before O is rescaled; it was issued a whole softmax ago.
      if (j > 0) {
        if (!(ok = consumer_wait(o_ready, (j - 1) & 1, w))) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tO + cc * 32, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(tO + cc * 32, r);
        }
      }
      tmem_st32(tS, *reinterpret_cast<uint32_t (*)[32]>(&pk[0]));
      tmem_st32(tS + 32, *reinterpret_cast<uint32_t (*)[32]>(&pk[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready);
    }
    if (ok && (ok = consumer_wait(o_ready, (n - 1) & 1, w))) {
      tc_fence_after();
      const float inv_l = p.o_scale / l;
      const bool valid = qrow < p.N;
      const size_t row_idx = (size_t)(U.b * p.Hq + U.h) * p.N + qrow;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row_idx * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tO + cc * 32, r);
        tmem_ld_wait(r);
        if (valid) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 pk4;
            const int i = v4 * 8;
            pk4.x = pack_bf16x2(__uint_as_float(r[i + 0]) * inv_l, __uint_as_float(r[i + 1]) * inv_l);
            pk4.y = pack_bf16x2(__uint_as_float(r[i + 2]) * inv_l, __uint_as_float(r[i + 3]) * inv_l);
            pk4.z = pack_bf16x2(__uint_as_float(r[i + 4]) * inv_l, __uint_as_float(r[i + 5]) * inv_l);
            pk4.w = pack_bf16x2(__uint_as_float(r[i + 6]) * inv_l, __uint_as_float(r[i + 7]) * inv_l);
            dst[cc * 4 + v4] = pk4;
          }
        }
      }
      if (valid) p.lse[row_idx] = (m_ref * c + log2f(l)) * 0.6931471805599453f;
    }
  } else {
    regs_dec<kRegsControl, kRegsLaunch>();  // warps 2-3 and 8-11 have no role here
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int KIND>
cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                         cudaStream_t stream) {
  using C = FwdCfg<D, KIND != kKindBf16>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  // Short units (a few key tiles each) run persistently, one CTA per SM (the shared memory
  // and the 512 TMEM columns allow no more): the per-CTA set-up and ring fill would weigh on
  // every unit. Longer units get one CTA each, and the hardware's dynamic block scheduling
  // balances their uneven causal lengths better than a static deal (measured: persistent
  // grids lost 5 % to 11 % on N = 8K to 64K, and won 7 % on N = 2K).
  const long long units = (long long)p.B * p.Hq * p.n_qblk;
  const int n_kv_all = (p.N + kTileN - 1) / kTileN;
  const int mean_kv = p.causal ? (n_kv_all + 1) / 2 : n_kv_all;  // key tiles of an average unit
  const bool persist = mean_kv <= kPersistentMaxKv && units > sm_count();
  if (persist) {
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = ensure_smem_limit(fwd_kernel<D, KIND, true>, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    fwd_kernel<D, KIND, true><<<(unsigned)sm_count(), kFwdThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  } else {
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = ensure_smem_limit(fwd_kernel<D, KIND, false>, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    fwd_kernel<D, KIND, false><<<(unsigned)units, kFwdThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_fwd256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p,
                          cudaStream_t stream) {
  static_assert(Fwd256Cfg::kSmemBytes <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(fwd256_kernel, Fwd256Cfg::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  const long long units = (long long)p.B * p.Hq * p.n_qblk;
  fwd256_kernel<<<(unsigned)units, kFwdThreads, Fwd256Cfg::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int d, cudaStream_t s) {
  if (d == 256) return launch_fwd256(tq, tk, tv, p, s);
  return d == 128 ? launch_fwd_d<128, kKindBf16>(tq, tk, tv, p, s) : launch_fwd_d<64, kKindBf16>(tq, tk, tv, p, s);
}

int fwd_tiles_per_cta(int d) { return d == 256 ? 1 : 2; }

cudaError_t launch_fwd_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t s) {
  return launch_fwd_d<128, kKindE4M3>(tq, tk, tv, p, s);
}

cudaError_t launch_fwd_e5m2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t s) {
  return launch_fwd_d<128, kKindE5M2>(tq, tk, tv, p, s);
}

}  // namespace fa
