// fa_bwd_sm100.cu -- bf16 attention backward on sm_100a, by recomputation.
//
// The backward pass does not store the score matrix: it recomputes S and P
// block by block from Q, K and the saved log-sum-exp ("Walk through what
// FlashAttention does differently from standard attention", second paragraph:
// the backward recomputes attention from the saved Q, K, V and statistics).
// For L = sum(O o dO), with D_i = sum_c dO_ic O_ic and dS = P o (dP - D):
//   dV = P^T dO,   dP = dO V^T,   dK = scale dS^T Q,   dQ = scale dS K.
//
// Kernels:
//   bwd_preprocess  D = rowsum(dO o O) (fp32) and zeroes the fp32 dQ accumulator.
//   bwd_main        one CTA per 128-key tile of one (batch, kv head). It keeps K
//                   and V in shared memory and dK, dV in Tensor Memory, and loops
//                   over the query heads of its GQA group and the 128-row query
//                   tiles that can see its keys. Per query tile i:
//                     S^T = K Q_i^T, dP^T = V dO_i^T          (tcgen05.mma -> TMEM)
//                     P^T = 2^(S^T c - LSE_i log2 e), dS^T = P^T o (dP^T - D_i)
//                     dV += P^T dO_i, dK += dS^T Q_i            (TMEM accumulators)
//                     dQ_i partial -> TMEM, then added to the fp32 accumulator
//                     with red.global.add.
//                   Two variants, one per head dim: bwd_main_kernel<64> and
//                   bwd_main_d128_kernel (described where each is defined).
//   bwd_convert     dQ = bf16(scale * accumulator).
//
// bwd_main roles (512 threads):
//   warp 0      producer: K, V once (TMA); per query tile Q_i, dO_i (TMA) and
//               -LSE_i log2(e), D_i (plain loads) into shared-memory slots.
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma.
//   warps 4-11  two warpgroups, thread = key row; warpgroup h computes P^T and
//               dS^T for query columns [64 h, 64 h + 64).
//   warps 12-15 thread = TMEM lane of the dQ tile: reads it and issues the fp32
//               reductions; at the end, writes dK and dV.
#include <math.h>

#include <algorithm>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kBwdThreads = 512;
#ifndef FA_BWD_POLY_PAIRS
#define FA_BWD_POLY_PAIRS 0
#endif
// Of every 8 pairs of P^T values, how many take 2^x by polynomial on the FMA pipe
// instead of the SFU (128-row kernel).
constexpr int kBwdPolyPairs = FA_BWD_POLY_PAIRS;
// Register split: the launch gives 128 per thread (512 x 128 = 65536). The
// control and dQ warpgroups lower to 96 and the two P/dS warpgroups raise to
// 160: 128 x (96 + 2 x 160 + 96) = 65536.
constexpr int kBwdRegsLaunch = 128;
constexpr int kBwdRegsControl = 96;
constexpr int kBwdRegsSoftmax = 160;
constexpr int kBwdRegsDq = 96;
static_assert(128 * (kBwdRegsControl + 2 * kBwdRegsSoftmax + kBwdRegsDq) <= kBwdThreads * kBwdRegsLaunch,
              "register split");

// ---------------------------------------------------------------------------
// main backward kernel, d = 64
// ---------------------------------------------------------------------------
// Query tiles of BR = 128 rows; dQ = dS K has M = 128 query rows (TMEM lanes)
// and N = d = 64. TMEM columns: S^T [0, 128), dP^T [128, 256), dQ [256, 320),
// dV [384, 448), dK [448, 512). P^T and dS^T go through shared memory in the
// 128-byte-swizzled K-major layout. MMA issue order per query tile i: S(i+1),
// dV(i), dP(i+1), dK(i), dQ(i): the next tile's scores are issued as soon as the
// current ones have been read out of TMEM, and dP(i+1) as soon as dP(i) has.
template <int D>
struct BwdCfg {
  static_assert(D == 64, "bwd_main_kernel serves d = 64; d = 128 has bwd_main_d128_kernel");
  static constexpr int BR = 128;                    // query rows per tile
  static constexpr int kStages = 3;
  static constexpr int kKVBytes = kTileN * D * 2;   // K or V tile (128 keys)
  static constexpr int kKVRegion = kTileN * 128;    // 64-column block of a K/V tile
  static constexpr int kQBytes = BR * D * 2;        // Q or dO tile
  static constexpr int kQRegion = BR * 128;         // 64-column block of a Q/dO tile
  static constexpr int kPBytes = kTileN * BR * 2;   // P^T or dS^T tile (128 keys x BR queries)
  static constexpr int kPRegion = kTileN * 128;
  static constexpr int kStageBytes = 2 * kQBytes + 1024;  // Q, dO, then LSE2 and D vectors
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVBytes;
  static constexpr int kOffStage = kOffV + kKVBytes;
  static constexpr int kOffP = kOffStage + kStages * kStageBytes;
  static constexpr int kOffDS = kOffP + kPBytes;
  static constexpr int kOffBar = kOffDS + kPBytes;
  // kv_full, st_full[S], st_empty[S], s_full, s_free, dp_full, dp_free, p_full, p_free,
  // ds_full, ds_free, dq_full, dq_free, mma_done
  static constexpr int kNumBars = 1 + 2 * kStages + 11;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // TMEM columns
  static constexpr int kColS = 0;
  static constexpr int kColDP = BR;
  static constexpr int kColDQ = 2 * BR;
  static constexpr int kColDV = 512 - 2 * D;
  static constexpr int kColDK = 512 - D;
  static_assert(kColDQ + 64 <= kColDV, "TMEM layout");
};

__device__ __forceinline__ uint8_t* align1024b(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void red_add(float* p, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

// ---------------------------------------------------------------------------
// D = rowsum(dO o O); dQ accumulator = 0. One thread per 8 columns of a row.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             float* __restrict__ delta, float* __restrict__ dq_acc,
                                                             long long rows) {
  constexpr int kPer = D / 8;  // threads per row (16 or 8)
  const long long total = rows * kPer;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t - threadIdx.x < total;
       t += (long long)gridDim.x * blockDim.x) {
    const bool in = t < total;
    const long long row = t / kPer;
    const int part = (int)(t % kPer);
    float acc = 0.f;
    if (in) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(a2[i]);
        const float2 y = __bfloat1622float2(b2[i]);
        acc = fmaf(x.x, y.x, acc);
        acc = fmaf(x.y, y.y, acc);
      }
      float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = kPer / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in && part == 0) delta[row] = acc;
  }
}

// ---------------------------------------------------------------------------
// dQ = bf16(scale * accumulator), 8 elements per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                          long long n8, float scale) {
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    uint4 u;
    u.x = pack_bf16x2(a.x * scale, a.y * scale);
    u.y = pack_bf16x2(a.z * scale, a.w * scale);
    u.z = pack_bf16x2(b.x * scale, b.y * scale);
    u.w = pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[t] = u;
  }
}

// ---------------------------------------------------------------------------
// main backward kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BR = C::BR;
  constexpr int ST = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024b(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* st_full = bars + 1;
  uint64_t* st_empty = st_full + ST;
  uint64_t* s_full = st_empty + ST;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_free + 1;
  uint64_t* dp_free = dp_full + 1;
  uint64_t* p_full = dp_free + 1;
  uint64_t* p_free = p_full + 1;
  uint64_t* ds_full = p_free + 1;
  uint64_t* ds_free = ds_full + 1;
  uint64_t* dq_full = ds_free + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* mma_done = dq_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key tile). (batch, kv head) pairs in groups of
  // p.head_group, whose Q, dO and dQ accumulators fit in L2 together; within a group
  // key tile 0 of every pair first (it sees the most query tiles under the causal mask).
  const int n_kt = (p.N + kTileN - 1) / kTileN;
  const int grp0 = (int)(blockIdx.x / (unsigned)(p.head_group * n_kt)) * p.head_group;
  const int gsz = min(p.head_group, p.B * p.Hkv - grp0);
  const int r = (int)blockIdx.x - grp0 * n_kt;
  const int bkv = grp0 + r % gsz;
  const int kt = r / gsz;
  const int b = bkv / p.Hkv;
  const int kvh = bkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int j0 = kt * kTileN;
  const int n_qt = (p.N + BR - 1) / BR;
  const int qt_first = p.causal ? j0 / BR : 0;
  const int per_head = n_qt - qt_first;
  const int n_it = g * per_head;
  const float c = p.scale_log2;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&st_full[s], 1 + 32);
      mbar_init(&st_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(dp_full, 1);
    mbar_init(dp_free, 256);
    mbar_init(p_full, 256);
    mbar_init(p_free, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(mma_done, 1);
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
    regs_dec<kBwdRegsControl, kBwdRegsLaunch>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(kv_full, 2 * C::kKVBytes);
#pragma unroll
      for (int z = 0; z < D / 64; ++z) {
        tma_load_3d(smem + C::kOffK + z * C::kKVRegion, &tmK, kv_full, z * 64, j0, bkv);
        tma_load_3d(smem + C::kOffV + z * C::kKVRegion, &tmV, kv_full, z * 64, j0, bkv);
      }
    }
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % ST;
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      const int q_head = b * p.Hq + h;
      ok = mbar_wait_spin(&st_empty[s], ((it / ST) & 1) ^ 1, w);
      if (!ok) break;
      uint8_t* stage = smem + C::kOffStage + s * C::kStageBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&st_full[s], 2 * C::kQBytes);
#pragma unroll
        for (int z = 0; z < D / 64; ++z) {
          tma_load_3d(stage + z * C::kQRegion, &tmQ, &st_full[s], z * 64, i0, q_head);
          tma_load_3d(stage + C::kQBytes + z * C::kQRegion, &tmDO, &st_full[s], z * 64, i0, q_head);
        }
      }
      float* lse2 = reinterpret_cast<float*>(stage + 2 * C::kQBytes);
      float* dl = lse2 + BR;
      const size_t rbase = (size_t)q_head * p.N;
#pragma unroll
      for (int r = lane; r < BR; r += 32) {
        const int i = i0 + r;
        const bool in = i < p.N;
        lse2[r] = in ? -p.lse[rbase + i] * 1.4426950408889634f : -INFINITY;  // -LSE log2(e)
        dl[r] = in ? p.delta[rbase + i] : 0.f;
      }
      mbar_arrive(&st_full[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this role (warp-uniform descriptors, built once and
    // advanced by constant offsets); lane 0 alone issues tcgen05.mma / commit.
    regs_dec<kBwdRegsControl, kBwdRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, BR, false, false);   // S^T, dP^T
    constexpr uint32_t kIdKV = idesc_bf16_f32(128, D, false, true);    // dV, dK
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, 64, true, true);     // dQ (or dQ^T)
    const uint32_t k_addr = smem_u32(smem + C::kOffK);
    const uint32_t v_addr = smem_u32(smem + C::kOffV);
    const uint32_t st_addr = smem_u32(smem + C::kOffStage);
    const uint32_t pt_addr = smem_u32(smem + C::kOffP);
    const uint32_t ds_addr = smem_u32(smem + C::kOffDS);
    // K-major views (LBO unused) and MN-major views (LBO = distance of 64-column blocks)
    const uint64_t dK_k = sdesc_sw128(k_addr, 16, 1024), dV_k = sdesc_sw128(v_addr, 16, 1024);
    const uint64_t dSt_k = sdesc_sw128(st_addr, 16, 1024);
    const uint64_t dSt_mn = sdesc_sw128(st_addr, C::kQRegion, 1024);
    const uint64_t dPt_k = sdesc_sw128(pt_addr, 16, 1024), dDs_k = sdesc_sw128(ds_addr, 16, 1024);
    const uint64_t dK_mn = sdesc_sw128(k_addr, C::kKVRegion, 1024);
    const uint64_t dDs_mn = sdesc_sw128(ds_addr, C::kPRegion, 1024);
    // X^T = A B^T over the head dim: A = K or V tile, B = Q or dO tile (both K-major)
    auto mma_scores = [&](uint64_t a0, uint64_t b0, uint32_t col) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kKVRegion + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * C::kQRegion + (k & 3) * 32;
        if (leader) mma_bf16_ss(tmem + col, desc_advance(a0, ao), desc_advance(b0, bo), kIdS, k > 0 ? 1u : 0u);
      }
    };
    // acc += A B over the query rows: A = P^T or dS^T (K-major), B = dO or Q (MN-major)
    auto mma_accum = [&](uint64_t a0, uint64_t b0, uint32_t col, bool first) {
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kPRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + col, desc_advance(a0, ao), desc_advance(b0, k * 2048), kIdKV,
                      (!first || k > 0) ? 1u : 0u);
      }
    };
    // dQ = dS K: A = dS (MN-major view of dS^T), B = K (MN-major), over the 128 keys.
    auto mma_dq = [&]() {
      const uint64_t a0 = dDs_mn;
      const uint64_t b0 = dK_mn;
#pragma unroll
      for (int k = 0; k < kTileN / 16; ++k)
        if (leader) mma_bf16_ss(tmem + C::kColDQ, desc_advance(a0, k * 2048), desc_advance(b0, k * 2048), kIdQ,
                                k > 0 ? 1u : 0u);
    };
    auto stage_off = [&](int it) -> uint32_t { return (uint32_t)((it % ST) * C::kStageBytes); };
    bool ok = mbar_wait_spin(kv_full, 0, w);
    if (ok && n_it > 0) ok = mbar_wait_spin(&st_full[0], 0, w);
    tc_fence_after();
    if (ok && n_it > 0) {
      mma_scores(dK_k, dSt_k, C::kColS);
      if (leader) mma_commit(s_full);
      mma_scores(dV_k, desc_advance(dSt_k, C::kQBytes), C::kColDP);
      if (leader) mma_commit(dp_full);
    }
    for (int it = 0; it < n_it && ok; ++it) {
      const uint32_t so = stage_off(it);
      const uint32_t ph = it & 1;
      // the next tile's S^T as soon as the current one has been read out of TMEM
      if (it + 1 < n_it) {
        if (!(ok = mbar_wait_spin(&st_full[(it + 1) % ST], ((it + 1) / ST) & 1, w))) break;
        if (!(ok = mbar_wait_spin(s_free, ph, w))) break;
        tc_fence_after();
        mma_scores(dK_k, desc_advance(dSt_k, stage_off(it + 1)), C::kColS);
        if (leader) mma_commit(s_full);
      }
      // dV += P^T dO_i
      if (!(ok = mbar_wait_spin(p_full, ph, w))) break;
      tc_fence_after();
      mma_accum(dPt_k, desc_advance(dSt_mn, so + C::kQBytes), C::kColDV, it == 0);
      if (leader) mma_commit(p_free);
      // the next tile's dP^T once the current one has been read out
      if (it + 1 < n_it) {
        if (!(ok = mbar_wait_spin(dp_free, ph, w))) break;
        tc_fence_after();
        mma_scores(dV_k, desc_advance(dSt_k, stage_off(it + 1) + C::kQBytes), C::kColDP);
        if (leader) mma_commit(dp_full);
      }
      // dK += dS^T Q_i ; dQ_i
      if (!(ok = mbar_wait_spin(ds_full, ph, w))) break;
      tc_fence_after();
      mma_accum(dDs_k, desc_advance(dSt_mn, so), C::kColDK, it == 0);
      if (it >= 1 && !(ok = mbar_wait_spin(dq_free, ph ^ 1, w))) break;
      tc_fence_after();
      mma_dq();
      if (leader) {
        mma_commit(dq_full);
        mma_commit(ds_free);
        mma_commit(&st_empty[it % ST]);
      }
    }
    if (leader) mma_commit(mma_done);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_done, 0, drain);
  } else if (warp < 4) {
    regs_dec<kBwdRegsControl, kBwdRegsLaunch>();
  } else if (warp < 12) {
    // ------------------------------------------------------------ P^T and dS^T (half the columns each)
    regs_inc<kBwdRegsSoftmax, kBwdRegsLaunch>();
    constexpr int HB = BR / 2;  // query columns per warpgroup
    const int half = (warp - 4) >> 2;
    const int col0 = half * HB;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row within the tile
    const int key = j0 + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t pt_tile = smem_u32(smem + C::kOffP);
    const uint32_t ds_tile = smem_u32(smem + C::kOffDS);
    const bool key_valid = key < p.N;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % ST;
      const uint32_t ph = it & 1;
      const int i0 = (qt_first + it % per_head) * BR + col0;  // first query of this half
      const float* lse2 =
          reinterpret_cast<const float*>(smem + C::kOffStage + s * C::kStageBytes + 2 * C::kQBytes) + col0;
      const float* dl = lse2 + BR;
      if (!mbar_wait_ns(&st_full[s], (it / ST) & 1, w, kConsumerPollNs)) break;
      if (!mbar_wait_ns(s_full, ph, w, kConsumerPollNs)) break;
      tc_fence_after();
      float pr[HB];
#pragma unroll
      for (int cc = 0; cc < HB / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + C::kColS + col0 + cc * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) pr[cc * 32 + i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      mbar_arrive(s_free);
      // P^T[key][q] = 2^(S c - LSE_q log2 e), zero for future queries and invalid keys.
      // The stage holds -LSE log2(e) per query (-inf past N), read as broadcast pairs.
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t* nl2 = reinterpret_cast<const uint64_t*>(lse2);
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[i], pr[i + 1]), c2, nl2[i / 2]), x0, x1);
        pr[i] = ex2(x0);
        pr[i + 1] = ex2(x1);
      }
      if (p.causal && i0 < j0 + kTileN) {  // diagonal tiles only
#pragma unroll
        for (int i = 0; i < HB; ++i)
          if (i0 + i < key) pr[i] = 0.f;
      }
      if (!key_valid) {
#pragma unroll
        for (int i = 0; i < HB; ++i) pr[i] = 0.f;
      }
      if (it >= 1 && !mbar_wait_ns(p_free, ph ^ 1, w, kConsumerPollNs)) break;
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch) {
        const int c0 = ch * 8;
        const int chunk = col0 / 8 + ch;
        st_shared_v4(pt_tile + (chunk >> 3) * C::kPRegion + sw128_offset(row, chunk & 7),
                     pack_bf16x2(pr[c0], pr[c0 + 1]), pack_bf16x2(pr[c0 + 2], pr[c0 + 3]),
                     pack_bf16x2(pr[c0 + 4], pr[c0 + 5]), pack_bf16x2(pr[c0 + 6], pr[c0 + 7]));
      }
      fence_async_smem();
      mbar_arrive(p_full);
      // dS^T = P^T o (dP^T - D_q); dP^T is read out whole first so the next
      // tile's dP^T can be issued at once.
      if (!mbar_wait_ns(dp_full, ph, w, kConsumerPollNs)) break;
      tc_fence_after();
      float dp[HB];
#pragma unroll
      for (int cc = 0; cc < HB / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + C::kColDP + col0 + cc * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) dp[cc * 32 + i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      mbar_arrive(dp_free);
      uint32_t dsp[HB / 2];
      const uint64_t* dl2 = reinterpret_cast<const uint64_t*>(dl);
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        float a, bb;
        f2_unpack(f2_mul(f2_pack(pr[i], pr[i + 1]), f2_sub(f2_pack(dp[i], dp[i + 1]), dl2[i / 2])), a, bb);
        dsp[i / 2] = pack_bf16x2(a, bb);
      }
      if (it >= 1 && !mbar_wait_ns(ds_free, ph ^ 1, w, kConsumerPollNs)) break;
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch) {
        const int chunk = col0 / 8 + ch;
        st_shared_v4(ds_tile + (chunk >> 3) * C::kPRegion + sw128_offset(row, chunk & 7), dsp[ch * 4],
                     dsp[ch * 4 + 1], dsp[ch * 4 + 2], dsp[ch * 4 + 3]);
      }
      fence_async_smem();
      mbar_arrive(ds_full);
    }
  } else {
    // ------------------------------------------------------------ dQ reductions, dK / dV epilogue
    regs_dec<kBwdRegsDq, kBwdRegsLaunch>();
    const int quarter = warp & 3;
    const int tl = quarter * 32 + lane;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      const size_t head_row0 = (size_t)(b * p.Hq + h) * p.N;
      if (!(ok = mbar_wait_ns(dq_full, it & 1, w, kConsumerPollNs))) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lane_off + C::kColDQ, r0);
      tmem_ld_wait(r0);
      tmem_ld32(tmem + lane_off + C::kColDQ + 32, r1);
      tmem_ld_wait(r1);
      tc_fence_before();
      mbar_arrive(dq_free);
      // lane = query row, TMEM columns = the 64 head-dim columns
      if (i0 + tl < p.N) {
        float* base = p.dq_acc + (head_row0 + i0 + tl) * D;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          red_add_v4(base + v * 4, __uint_as_float(r0[v * 4]), __uint_as_float(r0[v * 4 + 1]),
                     __uint_as_float(r0[v * 4 + 2]), __uint_as_float(r0[v * 4 + 3]));
#pragma unroll
        for (int v = 0; v < 8; ++v)
          red_add_v4(base + 32 + v * 4, __uint_as_float(r1[v * 4]), __uint_as_float(r1[v * 4 + 1]),
                     __uint_as_float(r1[v * 4 + 2]), __uint_as_float(r1[v * 4 + 3]));
      }
    }
    if (ok && n_it > 0 && mbar_wait(mma_done, 0, w)) {
      tc_fence_after();
      // dK, dV rows: TMEM lane = key row
      const int key = j0 + tl;
      const bool valid = key < p.N;
      const size_t row_idx = (size_t)bkv * p.N + key;
      uint4* dk_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + row_idx * D);
      uint4* dv_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + row_idx * D);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which ? C::kColDK : C::kColDV;
        const float mul = which ? p.scale : 1.f;
        uint4* dst = which ? dk_dst : dv_dst;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + col + cc * 32, r);
          tmem_ld_wait(r);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int i = v4 * 8;
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[i]) * mul, __uint_as_float(r[i + 1]) * mul);
              u.y = pack_bf16x2(__uint_as_float(r[i + 2]) * mul, __uint_as_float(r[i + 3]) * mul);
              u.z = pack_bf16x2(__uint_as_float(r[i + 4]) * mul, __uint_as_float(r[i + 5]) * mul);
              u.w = pack_bf16x2(__uint_as_float(r[i + 6]) * mul, __uint_as_float(r[i + 7]) * mul);
              dst[cc * 4 + v4] = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// main backward kernel, d = 128, 128-row query tiles
// ---------------------------------------------------------------------------
// With 128 query rows per tile every MMA has M = N = 128 (an N = 64 MMA runs at
// about half the rate). Tensor Memory then holds exactly S^T [0,128),
// dP^T [128,256), dV [256,384) and dK [384,512):
//   * P^T(i) is written back as bf16 over the S^T columns it came from (each
//     warpgroup over the first half of its own 64 columns) and dV += P^T dO_i
//     reads it from there, so P^T never goes through shared memory; S^T(i+1) is
//     issued after dV(i).
//   * dQ_i^T = K^T dS^T (head-dim columns in TMEM lanes, so each warp's fp32
//     reduction of one query row is one coalesced 128-byte access) reuses the
//     dP^T columns once dP^T(i) has been read, and dP^T(i+1) waits until dQ_i has
//     been read out.
// Shared memory (226 KB): K, V, two Q slots, two dO slots, the dS^T tile and the
// per-row -LSE log2 e and D of the two Q slots. That leaves no slack to align the
// base by hand, so it is declared 1024-byte aligned and checked at entry.
//
// Hand-offs per query tile i (mbarriers; every wait bounded):
//   q_full/q_empty[2], do_full/do_empty[2]   producer <-> MMA (TMA slots)
//   s_full   S^T(i) in TMEM          p_full   P^T(i) in TMEM (S^T(i) has been read)
//   dp_full  dP^T(i) in TMEM         ds_full  dS^T(i) in shared memory (dP^T(i) read)
//   ds_free  dQ(i) and dK(i) done: the dS^T tile may take dS^T(i+1)
//   dq_full  dQ(i) in TMEM           dq_free  dQ(i) read: dP^T(i+1) may be issued
// MMA order per i: dV(i), S^T(i+1), dQ(i), dK(i), dP^T(i+1).
struct Bwd128Cfg {
  static constexpr int D = 128;
  static constexpr int BR = 128;
  static constexpr int kTile = 128 * 128 * 2;       // K, V, Q, dO, dS^T tiles (32 KB)
  static constexpr int kRegion = 128 * 128;         // 64-column block of a tile
  static constexpr int kVecBytes = 2 * BR * 4;      // -LSE log2 e and D of one query tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;       // two slots
  static constexpr int kOffDO = kOffQ + 2 * kTile;  // two slots
  static constexpr int kOffDS = kOffDO + 2 * kTile;
  static constexpr int kOffVec = kOffDS + kTile;    // two slots
  static constexpr int kOffBar = kOffVec + 2 * kVecBytes;
  // kv_full, q_full[2], q_empty[2], do_full[2], do_empty[2], s_full, p_full, dp_full,
  // ds_full, ds_free, dq_full, dq_free, mma_done
  static constexpr int kNumBars = 17;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kOffDS % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kColS = 0, kColDP = 128, kColDQ = 128, kColDV = 256, kColDK = 384;
};
// Register split for this kernel: 128 x (80 + 2 x 160 + 112) = 65536.
constexpr int kB128RegsControl = 80;
constexpr int kB128RegsSoftmax = 160;
constexpr int kB128RegsDq = 112;
static_assert(128 * (kB128RegsControl + 2 * kB128RegsSoftmax + kB128RegsDq) <= kBwdThreads * kBwdRegsLaunch,
              "register split");

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_d128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const BwdParams p) {
  using C = Bwd128Cfg;
  constexpr int D = C::D;
  constexpr int BR = C::BR;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // uniform across the CTA: nothing has started yet
    if (threadIdx.x == 0) record_error(p.status, FA_ERR_LAUNCH);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = bars + 3;
  uint64_t* do_full = bars + 5;
  uint64_t* do_empty = bars + 7;
  uint64_t* s_full = bars + 9;
  uint64_t* p_full = bars + 10;
  uint64_t* dp_full = bars + 11;
  uint64_t* ds_full = bars + 12;
  uint64_t* ds_free = bars + 13;
  uint64_t* dq_full = bars + 14;
  uint64_t* dq_free = bars + 15;
  uint64_t* mma_done = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key tile). (batch, kv head) pairs in groups of
  // p.head_group, whose Q, dO and dQ accumulators fit in L2 together; within a group
  // key tile 0 of every pair first (it sees the most query tiles under the causal mask).
  const int n_kt = (p.N + kTileN - 1) / kTileN;
  const int grp0 = (int)(blockIdx.x / (unsigned)(p.head_group * n_kt)) * p.head_group;
  const int gsz = min(p.head_group, p.B * p.Hkv - grp0);
  const int r = (int)blockIdx.x - grp0 * n_kt;
  const int bkv = grp0 + r % gsz;
  const int kt = r / gsz;
  const int b = bkv / p.Hkv;
  const int kvh = bkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int j0 = kt * kTileN;
  const int n_qt = (p.N + BR - 1) / BR;
  const int qt_first = p.causal ? j0 / BR : 0;
  const int per_head = n_qt - qt_first;
  const int n_it = g * per_head;
  const float c = p.scale_log2;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1 + 32);
      mbar_init(&q_empty[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(mma_done, 1);
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
    regs_dec<kB128RegsControl, kBwdRegsLaunch>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(kv_full, 2 * C::kTile);
#pragma unroll
      for (int z = 0; z < 2; ++z) {
        tma_load_3d(smem + C::kOffK + z * C::kRegion, &tmK, kv_full, z * 64, j0, bkv);
        tma_load_3d(smem + C::kOffV + z * C::kRegion, &tmV, kv_full, z * 64, j0, bkv);
      }
    }
    // Q_i (with its row vectors) and dO_i, each as soon as its slot is free.
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it & 1;
      const uint32_t use_par = ((it >> 1) & 1) ^ 1;  // parity of the slot's previous release
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      const int q_head = b * p.Hq + h;
      if (!(ok = mbar_wait_spin(&q_empty[s], use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[s], C::kTile);
#pragma unroll
        for (int z = 0; z < 2; ++z)
          tma_load_3d(smem + C::kOffQ + s * C::kTile + z * C::kRegion, &tmQ, &q_full[s], z * 64, i0, q_head);
      }
      float* lse2 = reinterpret_cast<float*>(smem + C::kOffVec + s * C::kVecBytes);
      float* dl = lse2 + BR;
      const size_t rbase = (size_t)q_head * p.N;
#pragma unroll
      for (int r = lane; r < BR; r += 32) {
        const int i = i0 + r;
        const bool in = i < p.N;
        lse2[r] = in ? -p.lse[rbase + i] * 1.4426950408889634f : -INFINITY;  // -LSE log2(e)
        dl[r] = in ? p.delta[rbase + i] : 0.f;
      }
      mbar_arrive(&q_full[s]);
      if (!(ok = mbar_wait_spin(&do_empty[s], use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&do_full[s], C::kTile);
#pragma unroll
        for (int z = 0; z < 2; ++z)
          tma_load_3d(smem + C::kOffDO + s * C::kTile + z * C::kRegion, &tmDO, &do_full[s], z * 64, i0, q_head);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kB128RegsControl, kBwdRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T: A, B K-major
    constexpr uint32_t kIdKV = idesc_bf16_f32(128, 128, false, true);  // dV, dK: B MN-major
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, 128, true, true);    // dQ^T: A, B MN-major
    const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
    const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::kOffV), 16, 1024);
    const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + C::kOffK), C::kRegion, 1024);
    const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t dQ_mn = sdesc_sw128(smem_u32(smem + C::kOffQ), C::kRegion, 1024);
    const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + C::kOffDO), 16, 1024);
    const uint64_t dDO_mn = sdesc_sw128(smem_u32(smem + C::kOffDO), C::kRegion, 1024);
    const uint64_t dS_k = sdesc_sw128(smem_u32(smem + C::kOffDS), 16, 1024);
    const uint64_t dS_mn = sdesc_sw128(smem_u32(smem + C::kOffDS), C::kRegion, 1024);
    // X^T = A B^T over the head dim (A = K or V, B = Q_i or dO_i, both K-major)
    auto mma_scores = [&](uint64_t a0, uint64_t b0, uint32_t col) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * C::kRegion + (k & 3) * 32;
        if (leader) mma_bf16_ss(tmem + col, desc_advance(a0, off), desc_advance(b0, off), kIdS, k > 0 ? 1u : 0u);
      }
    };
    // dV += P^T dO_i: A = P^T in TMEM (query columns q: warpgroup q / 64's packed
    // pairs at S^T columns 64 (q / 64) + (q % 64) / 2), B = dO_i (MN-major)
    auto mma_dv = [&](uint64_t b0, bool first) {
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t acol = C::kColS + (k >> 2) * 64 + (k & 3) * 8;
        if (leader)
          mma_bf16_ts(tmem + C::kColDV, tmem + acol, desc_advance(b0, k * 2048), kIdKV, (!first || k > 0) ? 1u : 0u);
      }
    };
    // dK += dS^T Q_i (A = dS^T, K-major; B = Q_i, MN-major)
    auto mma_dk = [&](uint64_t b0, bool first) {
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColDK, desc_advance(dS_k, ao), desc_advance(b0, k * 2048), kIdKV,
                      (!first || k > 0) ? 1u : 0u);
      }
    };
    // dQ_i^T = K^T dS^T over the 128 keys (A = K^T: MN-major view of K; B = dS^T, MN-major)
    auto mma_dq = [&]() {
#pragma unroll
      for (int k = 0; k < kTileN / 16; ++k)
        if (leader)
          mma_bf16_ss(tmem + C::kColDQ, desc_advance(dK_mn, k * 2048), desc_advance(dS_mn, k * 2048), kIdQ,
                      k > 0 ? 1u : 0u);
    };
    bool ok = mbar_wait_spin(kv_full, 0, w);
    if (ok && n_it > 0) ok = mbar_wait_spin(&q_full[0], 0, w);
    if (ok && n_it > 0) ok = mbar_wait_spin(&do_full[0], 0, w);
    tc_fence_after();
    if (ok && n_it > 0) {
      mma_scores(dK_k, dQ_k, C::kColS);
      if (leader) mma_commit(s_full);
      mma_scores(dV_k, dDO_k, C::kColDP);
      if (leader) mma_commit(dp_full);
    }
    for (int it = 0; it < n_it && ok; ++it) {
      const uint32_t ph = it & 1;
      const int s = it & 1;
      // dV += P^T dO_i, then S^T(i+1) into the columns P^T(i) came from (one
      // thread's MMAs execute in issue order)
      if (!(ok = mbar_wait_spin(p_full, ph, w))) break;
      tc_fence_after();
      mma_dv(desc_advance(dDO_mn, s * C::kTile), it == 0);
      if (leader) mma_commit(&do_empty[s]);
      if (it + 1 < n_it) {
        if (!(ok = mbar_wait_spin(&q_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
        tc_fence_after();
        mma_scores(dK_k, desc_advance(dQ_k, (s ^ 1) * C::kTile), C::kColS);
        if (leader) mma_commit(s_full);
      }
      // dQ_i into the dP^T columns (already read), then dK += dS^T Q_i
      if (!(ok = mbar_wait_spin(ds_full, ph, w))) break;
      tc_fence_after();
      mma_dq();
      if (leader) mma_commit(dq_full);
      mma_dk(desc_advance(dQ_mn, s * C::kTile), it == 0);
      if (leader) {
        mma_commit(&q_empty[s]);
        mma_commit(ds_free);
      }
      // dP^T(i+1) once dQ_i has been read out of TMEM
      if (it + 1 < n_it) {
        if (!(ok = mbar_wait_spin(dq_free, ph, w))) break;
        if (!(ok = mbar_wait_spin(&do_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
        tc_fence_after();
        mma_scores(dV_k, desc_advance(dDO_k, (s ^ 1) * C::kTile), C::kColDP);
        if (leader) mma_commit(dp_full);
      }
    }
    if (leader) mma_commit(mma_done);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_done, 0, drain);
  } else if (warp < 4) {
    regs_dec<kB128RegsControl, kBwdRegsLaunch>();
  } else if (warp < 12) {
    // ------------------------------------------------------------ P^T and dS^T, 64 query columns each
    regs_inc<kB128RegsSoftmax, kBwdRegsLaunch>();
    constexpr int HB = 64;
    const int half = (warp - 4) >> 2;
    const int col0 = half * HB;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row within the tile
    const int key = j0 + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t ds_tile = smem_u32(smem + C::kOffDS) + half * C::kRegion;
    const bool key_valid = key < p.N;
    for (int it = 0; it < n_it; ++it) {
      const int s = it & 1;
      const uint32_t ph = it & 1;
      const int i0 = (qt_first + it % per_head) * BR + col0;  // first query of this half
      const float* lse2 = reinterpret_cast<const float*>(smem + C::kOffVec + s * C::kVecBytes) + col0;
      const float* dl = lse2 + BR;
      if (!mbar_wait_ns(&q_full[s], (it >> 1) & 1, w, kConsumerPollNs)) break;
      if (!mbar_wait_ns(s_full, ph, w, kConsumerPollNs)) break;
      tc_fence_after();
      float pr[HB];
      {
        uint32_t r0[32], r1[32];  // both loads in flight before the one wait
        tmem_ld32(tmem + lane_off + C::kColS + col0, r0);
        tmem_ld32(tmem + lane_off + C::kColS + col0 + 32, r1);
        tmem_ld_wait(r0);
        tmem_ld_wait(r1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          pr[i] = __uint_as_float(r0[i]);
          pr[32 + i] = __uint_as_float(r1[i]);
        }
      }
      // P^T[key][q] = 2^(S c - LSE_q log2 e), zero for future queries and invalid keys.
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t* nl2 = reinterpret_cast<const uint64_t*>(lse2);
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[i], pr[i + 1]), c2, nl2[i / 2]), x0, x1);
        if (((i / 2) & 7) < kBwdPolyPairs) {  // part of the exponentials on the FMA pipe
          ex2_poly2(x0, x1, pr[i], pr[i + 1]);
        } else {
          pr[i] = ex2(x0);
          pr[i + 1] = ex2(x1);
        }
      }
      if (p.causal && i0 < j0 + kTileN) {  // the diagonal tile only
#pragma unroll
        for (int i = 0; i < HB; ++i)
          if (i0 + i < key) pr[i] = 0.f;
      }
      if (!key_valid) {
#pragma unroll
        for (int i = 0; i < HB; ++i) pr[i] = 0.f;
      }
      // P^T as bf16 pairs over the first 32 of this warpgroup's S^T columns (read above)
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(pr[2 * i], pr[2 * i + 1]);
        tmem_st32(tmem + lane_off + C::kColS + col0, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(p_full);
      // dS^T = P^T o (dP^T - D_q), 32 columns at a time
      if (!mbar_wait_ns(dp_full, ph, w, kConsumerPollNs)) break;
      tc_fence_after();
      uint32_t dsp[HB / 2];
      const uint64_t* dl2 = reinterpret_cast<const uint64_t*>(dl);
#pragma unroll
      for (int cc = 0; cc < HB / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + C::kColDP + col0 + cc * 32, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int q = cc * 32 + i;
          float a, bb;
          f2_unpack(f2_mul(f2_pack(pr[q], pr[q + 1]),
                           f2_sub(f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), dl2[q / 2])),
                    a, bb);
          dsp[q / 2] = pack_bf16x2(a, bb);
        }
      }
      // the dS^T tile is free once dQ and dK of the previous query tile are done
      if (it >= 1 && !mbar_wait_ns(ds_free, ph ^ 1, w, kConsumerPollNs)) break;
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch)
        st_shared_v4(ds_tile + sw128_offset(row, ch), dsp[ch * 4], dsp[ch * 4 + 1], dsp[ch * 4 + 2],
                     dsp[ch * 4 + 3]);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
  } else {
    // ------------------------------------------------------------ dQ reductions, dK / dV epilogue
    regs_dec<kB128RegsDq, kBwdRegsLaunch>();
    const int quarter = warp & 3;
    const int tl = quarter * 32 + lane;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      // lane = head-dim column, TMEM columns = the 128 query rows
      float* base = p.dq_acc + ((size_t)(b * p.Hq + h) * p.N + i0) * D + tl;
      const int nq = min(BR, p.N - i0);
      if (!(ok = mbar_wait_ns(dq_full, it & 1, w, kConsumerPollNs))) break;
      tc_fence_after();
      auto reduce32 = [&](const uint32_t (&r)[32], int q0) {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (q0 + q < nq) red_add(base + (size_t)(q0 + q) * D, __uint_as_float(r[q]));
      };
      // four 32-column loads into three buffers; dq_free as soon as the last one has
      // landed (only one chunk's reductions are issued before it: they queue behind
      // the memory system and would hold up the next dP^T)
      uint32_t ra[32], rb[32], rc[32];
      tmem_ld32(tmem + lane_off + C::kColDQ, ra);
      tmem_ld32(tmem + lane_off + C::kColDQ + 32, rb);
      tmem_ld32(tmem + lane_off + C::kColDQ + 64, rc);
      tmem_ld_wait(ra);
      tmem_ld_wait(rb);
      tmem_ld_wait(rc);
      reduce32(ra, 0);
      tmem_ld32(tmem + lane_off + C::kColDQ + 96, ra);
      tmem_ld_wait(ra);
      tc_fence_before();
      mbar_arrive(dq_free);
      reduce32(rb, 32);
      reduce32(rc, 64);
      reduce32(ra, 96);
    }
    if (ok && n_it > 0 && mbar_wait(mma_done, 0, w)) {
      tc_fence_after();
      // dK, dV rows: TMEM lane = key row
      const int key = j0 + tl;
      const bool valid = key < p.N;
      const size_t row_idx = (size_t)bkv * p.N + key;
      uint4* dk_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + row_idx * D);
      uint4* dv_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + row_idx * D);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which ? C::kColDK : C::kColDV;
        const float mul = which ? p.scale : 1.f;
        uint4* dst = which ? dk_dst : dv_dst;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + col + cc * 32, r);
          tmem_ld_wait(r);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int i = v4 * 8;
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[i]) * mul, __uint_as_float(r[i + 1]) * mul);
              u.y = pack_bf16x2(__uint_as_float(r[i + 2]) * mul, __uint_as_float(r[i + 3]) * mul);
              u.z = pack_bf16x2(__uint_as_float(r[i + 4]) * mul, __uint_as_float(r[i + 5]) * mul);
              u.w = pack_bf16x2(__uint_as_float(r[i + 6]) * mul, __uint_as_float(r[i + 7]) * mul);
              dst[cc * 4 + v4] = u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int D>
cudaError_t launch_preprocess_d(const BwdParams& p, cudaStream_t s) {
  const long long rows = (long long)p.B * p.Hq * p.N;
  const int blocks = (int)std::min<long long>((rows * (D / 8) + 255) / 256, 8LL * sm_count());
  bwd_preprocess_kernel<D><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(p.o),
                                                   static_cast<const __nv_bfloat16*>(p.dout), p.delta, p.dq_acc, rows);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_main_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                          const BwdParams& p, cudaStream_t s) {
  const long long grid = (long long)p.B * p.Hkv * ((p.N + kTileN - 1) / kTileN);
  if constexpr (D == 128) {
    using C = Bwd128Cfg;
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = ensure_smem_limit(bwd_main_d128_kernel, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    bwd_main_d128_kernel<<<(unsigned)grid, kBwdThreads, C::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
  } else {
    using C = BwdCfg<D>;
    static_assert(C::kSmemBytes <= 232448, "shared memory budget");
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = ensure_smem_limit(bwd_main_kernel<D>, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    bwd_main_kernel<D><<<(unsigned)grid, kBwdThreads, C::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
  }
  return cudaGetLastError();
}

}  // namespace

int bwd_query_rows(int) { return 128; }

cudaError_t launch_bwd_preprocess(const BwdParams& p, cudaStream_t s) {
  return p.d == 128 ? launch_preprocess_d<128>(p, s) : launch_preprocess_d<64>(p, s);
}

cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, cudaStream_t s) {
  return p.d == 128 ? launch_main_d<128>(tq, tk, tv, tdo, p, s) : launch_main_d<64>(tq, tk, tv, tdo, p, s);
}

cudaError_t launch_bwd_convert(const BwdParams& p, cudaStream_t s) {
  const long long n8 = (long long)p.B * p.Hq * p.N * p.d / 8;
  const int blocks = (int)std::min<long long>((n8 + 255) / 256, 8LL * sm_count());
  bwd_convert_kernel<<<blocks, 256, 0, s>>>(p.dq_acc, static_cast<__nv_bfloat16*>(p.dq), n8, p.scale);
  return cudaGetLastError();
}

}  // namespace fa
