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
//                     (d = 128: red.global.add; d = 64: TMA reduce-add).
//                   Two variants, one per head dim: bwd_main_d64_kernel and
//                   bwd_main_d128_kernel (described where each is defined).
//   bwd_convert     dQ = bf16(scale * accumulator).
//
// bwd_main roles (512 threads):
//   warp 0      producer: K, V once (TMA); per query tile Q_i, dO_i (TMA) and
//               -LSE_i log2(e), D_i (plain loads) into shared-memory slots.
//   warp 1      allocates TMEM; one lane issues every tcgen05.mma.
//   warps 4-11  two warpgroups, thread = key row; warpgroup h computes P^T and
//               dS^T for query columns [64 h, 64 h + 64).
//   warps 12-15 thread = TMEM lane of the dQ tile: reads it and adds it into the
//               fp32 accumulator; at the end, writes dK and dV.
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
#ifndef FA_BWD64_POLY_PAIRS
#define FA_BWD64_POLY_PAIRS 1
#endif
constexpr int kBwd64PolyPairs = FA_BWD64_POLY_PAIRS;  // the same, for the d = 64 kernel
// Register split: the launch gives 128 per thread (512 x 128 = 65536). The
// control and dQ warpgroups lower to 96 and the two P/dS warpgroups raise to
// 160: 128 x (96 + 2 x 160 + 96) = 65536.
constexpr int kBwdRegsLaunch = 128;
constexpr int kBwdRegsControl = 96;
constexpr int kBwdRegsSoftmax = 160;
constexpr int kBwdRegsDq = 96;
static_assert(128 * (kBwdRegsControl + 2 * kBwdRegsSoftmax + kBwdRegsDq) <= kBwdThreads * kBwdRegsLaunch,
              "register split");

__device__ __forceinline__ void red_add(float* p, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

// ---------------------------------------------------------------------------
// D = rowsum(dO o O); dQ accumulator = 0. One thread per 8 columns of a row, and
// kPrepItems such (row, 8 columns) items per thread per round, whose loads are all
// issued before any is used (more bytes in flight per thread).
// ---------------------------------------------------------------------------
constexpr int kPrepItems = 4;

template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             float* __restrict__ delta, float* __restrict__ dq_acc,
                                                             long long rows) {
  constexpr int kPer = D / 8;  // threads per row (32, 16 or 8)
  const long long total = rows * kPer;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // rounds are taken by whole warps (t - threadIdx.x is the same across a block), so the
  // shuffles below always see converged warps
  for (long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; t0 - threadIdx.x < total;
       t0 += kPrepItems * stride) {
    uint4 a[kPrepItems], b[kPrepItems];
#pragma unroll
    for (int j = 0; j < kPrepItems; ++j) {
      const long long t = t0 + j * stride;
      if (t < total) {
        const long long row = t / kPer;
        const int part = (int)(t % kPer);
        a[j] = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
        b[j] = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
      }
    }
#pragma unroll
    for (int j = 0; j < kPrepItems; ++j) {
      const long long t = t0 + j * stride;
      const bool in = t < total;
      const long long row = t / kPer;
      const int part = (int)(t % kPer);
      float acc = 0.f;
      if (in) {
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[j]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b[j]);
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
}

// ---------------------------------------------------------------------------
// dQ = bf16(scale * accumulator), 8 elements per item, kPrepItems items per thread
// per round with all their loads in flight together.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                          long long n8, float scale) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; t0 < n8; t0 += kPrepItems * stride) {
    float4 a[kPrepItems], b[kPrepItems];
#pragma unroll
    for (int j = 0; j < kPrepItems; ++j) {
      const long long t = t0 + j * stride;
      if (t < n8) {
        a[j] = reinterpret_cast<const float4*>(acc)[2 * t];
        b[j] = reinterpret_cast<const float4*>(acc)[2 * t + 1];
      }
    }
#pragma unroll
    for (int j = 0; j < kPrepItems; ++j) {
      const long long t = t0 + j * stride;
      if (t < n8) {
        uint4 u;
        u.x = pack_bf16x2(a[j].x * scale, a[j].y * scale);
        u.y = pack_bf16x2(a[j].z * scale, a[j].w * scale);
        u.z = pack_bf16x2(b[j].x * scale, b[j].y * scale);
        u.w = pack_bf16x2(b[j].z * scale, b[j].w * scale);
        reinterpret_cast<uint4*>(dq)[t] = u;
      }
    }
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
// Register split: 128 x (48 + 2 x 160 + 144) = 65536. The dQ warpgroup holds a whole
// 128-column dQ tile in registers; the producer and MMA warps need few.
constexpr int kB128RegsControl = 48;
constexpr int kB128RegsSoftmax = 160;
constexpr int kB128RegsDq = 144;
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
      if (!(ok = warp_wait_spin(&q_empty[s], use_par, w))) break;
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
      if (!(ok = warp_wait_spin(&do_empty[s], use_par, w))) break;
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
    // progress record: the query tiles whose dV MMA this CTA has issued
    unsigned* const prog = (int)blockIdx.x < p.progress_n ? p.progress : nullptr;
    if (leader && prog) prog[blockIdx.x] = 0u;
    bool ok = warp_wait_spin(kv_full, 0, w);
    if (ok && n_it > 0) ok = warp_wait_spin(&q_full[0], 0, w);
    if (ok && n_it > 0) ok = warp_wait_spin(&do_full[0], 0, w);
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
      if (!(ok = warp_wait_spin(p_full, ph, w))) break;
      if (leader && prog) prog[blockIdx.x] = (unsigned)(it + 1);
      tc_fence_after();
      mma_dv(desc_advance(dDO_mn, s * C::kTile), it == 0);
      if (leader) mma_commit(&do_empty[s]);
      if (it + 1 < n_it) {
        if (!(ok = warp_wait_spin(&q_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
        tc_fence_after();
        mma_scores(dK_k, desc_advance(dQ_k, (s ^ 1) * C::kTile), C::kColS);
        if (leader) mma_commit(s_full);
      }
      // dQ_i into the dP^T columns (already read), then dK += dS^T Q_i
      if (!(ok = warp_wait_spin(ds_full, ph, w))) break;
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
        if (!(ok = warp_wait_spin(dq_free, ph, w))) break;
        if (!(ok = warp_wait_spin(&do_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
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
      if (!consumer_wait(&q_full[s], (it >> 1) & 1, w)) break;
      if (!consumer_wait(s_full, ph, w)) break;
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
      const ulonglong2* nl4 = reinterpret_cast<const ulonglong2*>(lse2);  // 16-byte broadcast loads
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        const ulonglong2 nv = nl4[i / 4];
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[i], pr[i + 1]), c2, (i & 2) ? nv.y : nv.x), x0, x1);
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
      // dS^T = P^T o (dP^T - D_q); both halves of dP^T in flight before the one wait
      if (!consumer_wait(dp_full, ph, w)) break;
      tc_fence_after();
      uint32_t dsp[HB / 2];
      const ulonglong2* dl4 = reinterpret_cast<const ulonglong2*>(dl);  // 16-byte broadcast loads
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + lane_off + C::kColDP + col0, r0);
        tmem_ld32(tmem + lane_off + C::kColDP + col0 + 32, r1);
        tmem_ld_wait(r0);
        tmem_ld_wait(r1);
#pragma unroll
        for (int i = 0; i < HB; i += 2) {
          const uint32_t d0 = i < 32 ? r0[i] : r1[i - 32], d1 = i < 32 ? r0[i + 1] : r1[i - 31];
          float a, bb;
          f2_unpack(f2_mul(f2_pack(pr[i], pr[i + 1]),
                           f2_sub(f2_pack(__uint_as_float(d0), __uint_as_float(d1)),
                                  (i & 2) ? dl4[i / 4].y : dl4[i / 4].x)),
                    a, bb);
          dsp[i / 2] = pack_bf16x2(a, bb);
        }
      }
      // the dS^T tile is free once dQ and dK of the previous query tile are done
      if (it >= 1 && !consumer_wait(ds_free, ph ^ 1, w)) break;
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
    regs_inc<kB128RegsDq, kBwdRegsLaunch>();
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
      if (!(ok = consumer_wait(dq_full, it & 1, w))) break;
      tc_fence_after();
      auto reduce32 = [&](const uint32_t (&r)[32], int q0) {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (q0 + q < nq) red_add(base + (size_t)(q0 + q) * D, __uint_as_float(r[q]));
      };
      // all four 32-column loads in flight, one wait, then dq_free at once: the next
      // dP^T waits for these columns, the reductions do not hold it up
      uint32_t ra[32], rb[32], rc[32], rd[32];
      tmem_ld32(tmem + lane_off + C::kColDQ, ra);
      tmem_ld32(tmem + lane_off + C::kColDQ + 32, rb);
      tmem_ld32(tmem + lane_off + C::kColDQ + 64, rc);
      tmem_ld32(tmem + lane_off + C::kColDQ + 96, rd);
      tmem_ld_wait(ra);
      tmem_ld_wait(rb);
      tmem_ld_wait(rc);
      tmem_ld_wait(rd);
      tc_fence_before();
      mbar_arrive(dq_free);
      reduce32(ra, 0);
      reduce32(rb, 32);
      reduce32(rc, 64);
      reduce32(rd, 96);
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
// main backward kernel, d = 64, 128-row query tiles
// ---------------------------------------------------------------------------
// The d = 128 kernel's design at half the head dim. S^T, dP^T, dV and dK now
// take 384 TMEM columns, so dQ gets columns of its own, twice over:
//   S^T [0,128), dP^T [128,256), dQ_0 [256,320), dQ_1 [320,384), dV [384,448),
//   dK [448,512).
// dQ_i = dS_i K (M = 128 query rows in TMEM lanes, N = d = 64) goes to buffer
// i % 2, so no MMA ever waits for a dQ read-out except two query tiles later.
// P^T(i) is written back as bf16 over the S^T columns it came from and dV reads
// it from TMEM (TS MMA), as at d = 128.
//
// dQ leaves through shared memory: the dQ warpgroup copies its 128 x 64 fp32
// tile from TMEM into a 128-byte-swizzled staging buffer (two 16 KB boxes of 32
// columns; thread = query row, so every warp store covers whole 128-byte lines
// without bank conflicts), and one thread hands each box to the TMA unit as a
// reduce-add into the fp32 accumulator (cp.reduce.async.bulk.tensor ... add).
// Two staging buffers alternate; rows past N are clipped by the tensor map.
//
// Shared memory (196 KB): K, V, two Q slots, two dO slots (16 KB each), the
// dS^T tile (32 KB), two dQ staging buffers (32 KB each), the row vectors of
// the two Q slots.
//
// MMA order per query tile i: dV(i), S^T(i+1), dQ(i), dK(i), dP^T(i+1).
struct Bwd64Cfg {
  static constexpr int D = 64;
  static constexpr int BR = 128;
  static constexpr int kTile = 128 * 64 * 2;        // K, V, Q or dO tile (16 KB, one 64-column block)
  static constexpr int kDsTile = 128 * 128 * 2;     // dS^T tile: 128 keys x 128 queries (two blocks)
  static constexpr int kDsRegion = 128 * 128;       // one 64-query block of it
  static constexpr int kDqBox = 128 * 32 * 4;       // 128 rows x 32 fp32 (one TMA box, 16 KB)
  static constexpr int kDqStage = 2 * kDqBox;       // a 128 x 64 fp32 dQ tile
  static constexpr int kVecBytes = 2 * BR * 4;      // -LSE log2 e and D of one query tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTile;
  static constexpr int kOffQ = kOffV + kTile;       // two slots
  static constexpr int kOffDO = kOffQ + 2 * kTile;  // two slots
  static constexpr int kOffDS = kOffDO + 2 * kTile;
  static constexpr int kOffDQ = kOffDS + kDsTile;   // two staging buffers
  static constexpr int kOffVec = kOffDQ + 2 * kDqStage;
  static constexpr int kOffBar = kOffVec + 2 * kVecBytes;
  // kv_full, q_full[2], q_empty[2], do_full[2], do_empty[2], s_full, p_full, dp_full,
  // ds_full, ds_free, dq_full[2], dq_free[2], mma_done
  static constexpr int kNumBars = 19;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kOffDS % 1024 == 0 && kOffDQ % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kColS = 0, kColDP = 128, kColDQ = 256, kColDV = 384, kColDK = 448;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_d64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using C = Bwd64Cfg;
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
  uint64_t* dq_full = bars + 14;  // two
  uint64_t* dq_free = bars + 16;  // two
  uint64_t* mma_done = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key tile), scheduled as in the d = 128 kernel.
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
      mbar_init(&dq_full[s], 1);
      mbar_init(&dq_free[s], 128);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
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
      tma_prefetch_desc(&tmDQ);
      mbar_arrive_expect_tx(kv_full, 2 * C::kTile);
      tma_load_3d(smem + C::kOffK, &tmK, kv_full, 0, j0, bkv);
      tma_load_3d(smem + C::kOffV, &tmV, kv_full, 0, j0, bkv);
    }
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it & 1;
      const uint32_t use_par = ((it >> 1) & 1) ^ 1;  // parity of the slot's previous release
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      const int q_head = b * p.Hq + h;
      if (!(ok = warp_wait_spin(&q_empty[s], use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[s], C::kTile);
        tma_load_3d(smem + C::kOffQ + s * C::kTile, &tmQ, &q_full[s], 0, i0, q_head);
      }
      float* lse2 = reinterpret_cast<float*>(smem + C::kOffVec + s * C::kVecBytes);
      float* dl = lse2 + BR;
      const size_t rbase = (size_t)q_head * p.N;
#pragma unroll
      for (int rr = lane; rr < BR; rr += 32) {
        const int i = i0 + rr;
        const bool in = i < p.N;
        lse2[rr] = in ? -p.lse[rbase + i] * 1.4426950408889634f : -INFINITY;  // -LSE log2(e)
        dl[rr] = in ? p.delta[rbase + i] : 0.f;
      }
      mbar_arrive(&q_full[s]);
      if (!(ok = warp_wait_spin(&do_empty[s], use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&do_full[s], C::kTile);
        tma_load_3d(smem + C::kOffDO + s * C::kTile, &tmDO, &do_full[s], 0, i0, q_head);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kB128RegsControl, kBwdRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T: A, B K-major
    constexpr uint32_t kIdKV = idesc_bf16_f32(128, D, false, true);    // dV, dK: B MN-major, N = d
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, true, true);      // dQ: A, B MN-major, N = d
    const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
    const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::kOffV), 16, 1024);
    const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + C::kOffK), C::kTile, 1024);
    const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t dQ_mn = sdesc_sw128(smem_u32(smem + C::kOffQ), C::kTile, 1024);
    const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + C::kOffDO), 16, 1024);
    const uint64_t dDO_mn = sdesc_sw128(smem_u32(smem + C::kOffDO), C::kTile, 1024);
    const uint64_t dS_k = sdesc_sw128(smem_u32(smem + C::kOffDS), 16, 1024);
    const uint64_t dS_mn = sdesc_sw128(smem_u32(smem + C::kOffDS), C::kDsRegion, 1024);
    // X^T = A B^T over the head dim (A = K or V, B = Q_i or dO_i, both K-major, one block)
    auto mma_scores = [&](uint64_t a0, uint64_t b0, uint32_t col) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        if (leader) mma_bf16_ss(tmem + col, desc_advance(a0, k * 32), desc_advance(b0, k * 32), kIdS, k > 0 ? 1u : 0u);
    };
    // dV += P^T dO_i: A = P^T in TMEM (query q of warpgroup q / 64 packed at S^T column
    // 64 (q / 64) + (q % 64) / 2), B = dO_i (MN-major)
    auto mma_dv = [&](uint64_t b0, bool first) {
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t acol = C::kColS + (k >> 2) * 64 + (k & 3) * 8;
        if (leader)
          mma_bf16_ts(tmem + C::kColDV, tmem + acol, desc_advance(b0, k * 2048), kIdKV, (!first || k > 0) ? 1u : 0u);
      }
    };
    // dK += dS^T Q_i (A = dS^T, K-major over the queries; B = Q_i, MN-major)
    auto mma_dk = [&](uint64_t b0, bool first) {
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kDsRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColDK, desc_advance(dS_k, ao), desc_advance(b0, k * 2048), kIdKV,
                      (!first || k > 0) ? 1u : 0u);
      }
    };
    // dQ_i = dS K over the 128 keys (A = dS: MN-major view of dS^T; B = K, MN-major)
    auto mma_dq = [&](uint32_t col) {
#pragma unroll
      for (int k = 0; k < kTileN / 16; ++k)
        if (leader)
          mma_bf16_ss(tmem + col, desc_advance(dS_mn, k * 2048), desc_advance(dK_mn, k * 2048), kIdQ,
                      k > 0 ? 1u : 0u);
    };
    // progress record: the query tiles whose dV MMA this CTA has issued
    unsigned* const prog = (int)blockIdx.x < p.progress_n ? p.progress : nullptr;
    if (leader && prog) prog[blockIdx.x] = 0u;
    bool ok = warp_wait_spin(kv_full, 0, w);
    if (ok && n_it > 0) ok = warp_wait_spin(&q_full[0], 0, w);
    if (ok && n_it > 0) ok = warp_wait_spin(&do_full[0], 0, w);
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
      const int qb = it & 1;  // dQ buffer
      if (!(ok = warp_wait_spin(p_full, ph, w))) break;
      if (leader && prog) prog[blockIdx.x] = (unsigned)(it + 1);
      tc_fence_after();
      mma_dv(desc_advance(dDO_mn, s * C::kTile), it == 0);
      if (leader) mma_commit(&do_empty[s]);
      if (it + 1 < n_it) {
        if (!(ok = warp_wait_spin(&q_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
        tc_fence_after();
        mma_scores(dK_k, desc_advance(dQ_k, (s ^ 1) * C::kTile), C::kColS);
        if (leader) mma_commit(s_full);
      }
      if (!(ok = warp_wait_spin(ds_full, ph, w))) break;
      // the dQ buffer is free once dQ(it - 2) has been read out
      if (it >= 2 && !(ok = warp_wait_spin(&dq_free[qb], ((it >> 1) & 1) ^ 1, w))) break;
      tc_fence_after();
      mma_dq(C::kColDQ + qb * 64);
      if (leader) mma_commit(&dq_full[qb]);
      mma_dk(desc_advance(dQ_mn, s * C::kTile), it == 0);
      if (leader) {
        mma_commit(&q_empty[s]);
        mma_commit(ds_free);
      }
      if (it + 1 < n_it) {
        if (!(ok = warp_wait_spin(&do_full[s ^ 1], ((it + 1) >> 1) & 1, w))) break;
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
    const uint32_t ds_tile = smem_u32(smem + C::kOffDS) + half * C::kDsRegion;
    const bool key_valid = key < p.N;
    for (int it = 0; it < n_it; ++it) {
      const int s = it & 1;
      const uint32_t ph = it & 1;
      const int i0 = (qt_first + it % per_head) * BR + col0;  // first query of this half
      const float* lse2 = reinterpret_cast<const float*>(smem + C::kOffVec + s * C::kVecBytes) + col0;
      const float* dl = lse2 + BR;
      if (!consumer_wait(&q_full[s], (it >> 1) & 1, w)) break;
      if (!consumer_wait(s_full, ph, w)) break;
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
      const ulonglong2* nl4 = reinterpret_cast<const ulonglong2*>(lse2);  // 16-byte broadcast loads
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        const ulonglong2 nv = nl4[i / 4];
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[i], pr[i + 1]), c2, (i & 2) ? nv.y : nv.x), x0, x1);
        if (((i / 2) & 7) < kBwd64PolyPairs) {  // part of the exponentials on the FMA pipe
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
      // dS^T = P^T o (dP^T - D_q); both halves of dP^T in flight before the one wait
      if (!consumer_wait(dp_full, ph, w)) break;
      tc_fence_after();
      uint32_t dsp[HB / 2];
      const ulonglong2* dl4 = reinterpret_cast<const ulonglong2*>(dl);  // 16-byte broadcast loads
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + lane_off + C::kColDP + col0, r0);
        tmem_ld32(tmem + lane_off + C::kColDP + col0 + 32, r1);
        tmem_ld_wait(r0);
        tmem_ld_wait(r1);
#pragma unroll
        for (int i = 0; i < HB; i += 2) {
          const uint32_t d0 = i < 32 ? r0[i] : r1[i - 32], d1 = i < 32 ? r0[i + 1] : r1[i - 31];
          float a, bb;
          f2_unpack(f2_mul(f2_pack(pr[i], pr[i + 1]),
                           f2_sub(f2_pack(__uint_as_float(d0), __uint_as_float(d1)),
                                  (i & 2) ? dl4[i / 4].y : dl4[i / 4].x)),
                    a, bb);
          dsp[i / 2] = pack_bf16x2(a, bb);
        }
      }
      // the dS^T tile is free once dQ and dK of the previous query tile are done
      if (it >= 1 && !consumer_wait(ds_free, ph ^ 1, w)) break;
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch)
        st_shared_v4(ds_tile + sw128_offset(row, ch), dsp[ch * 4], dsp[ch * 4 + 1], dsp[ch * 4 + 2],
                     dsp[ch * 4 + 3]);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
  } else {
    // ------------------------------------------------------------ dQ out through the TMA, dK / dV epilogue
    regs_inc<kB128RegsDq, kBwdRegsLaunch>();
    const int quarter = warp & 3;
    const int tl = quarter * 32 + lane;  // TMEM lane = query row of the dQ tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool issuer = threadIdx.x == 384;
    constexpr int kBarDq = 1;  // named barrier of these 128 threads
    // Every thread takes both named barriers of every iteration, whatever its waits
    // returned, so that a wait that ran out cannot leave the others at a barrier.
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int qb = it & 1;
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      uint32_t ra[32], rb[32];
      ok = ok && consumer_wait(&dq_full[qb], (it >> 1) & 1, w);
      ok = __all_sync(0xffffffffu, ok);  // the tcgen05.ld below are warp-wide
      if (ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_off + C::kColDQ + qb * 64, ra);
        tmem_ld32(tmem + lane_off + C::kColDQ + qb * 64 + 32, rb);
        tmem_ld_wait(ra);
        tmem_ld_wait(rb);
        tc_fence_before();
        mbar_arrive(&dq_free[qb]);
      }
      // staging buffer qb was last read by the reduction issued two tiles ago
      if (issuer) bulk_wait_read<1>();
      named_barrier(kBarDq, 128);
      uint8_t* stage = smem + C::kOffDQ + qb * C::kDqStage;
      if (ok) {
        const uint32_t box0 = smem_u32(stage), box1 = box0 + C::kDqBox;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          st_shared_v4(box0 + sw128_offset(tl, ch), ra[ch * 4], ra[ch * 4 + 1], ra[ch * 4 + 2], ra[ch * 4 + 3]);
          st_shared_v4(box1 + sw128_offset(tl, ch), rb[ch * 4], rb[ch * 4 + 1], rb[ch * 4 + 2], rb[ch * 4 + 3]);
        }
        fence_async_smem();
      }
      named_barrier(kBarDq, 128);
      if (issuer && ok && !*abort_flag) {
        const int q_head = b * p.Hq + h;
        tma_reduce_add_3d(&tmDQ, stage, 0, i0, q_head);
        tma_reduce_add_3d(&tmDQ, stage + C::kDqBox, 32, i0, q_head);
        bulk_commit();
      }
    }
    if (issuer) bulk_wait_all();
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
          uint32_t rr[32];
          tmem_ld32(tmem + lane_off + col + cc * 32, rr);
          tmem_ld_wait(rr);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int i = v4 * 8;
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(rr[i]) * mul, __uint_as_float(rr[i + 1]) * mul);
              u.y = pack_bf16x2(__uint_as_float(rr[i + 2]) * mul, __uint_as_float(rr[i + 3]) * mul);
              u.z = pack_bf16x2(__uint_as_float(rr[i + 4]) * mul, __uint_as_float(rr[i + 5]) * mul);
              u.w = pack_bf16x2(__uint_as_float(rr[i + 6]) * mul, __uint_as_float(rr[i + 7]) * mul);
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


template <int D>
cudaError_t launch_preprocess_d(const BwdParams& p, cudaStream_t s) {
  const long long rows = (long long)p.B * p.Hq * p.N;
  const int blocks = (int)std::min<long long>((rows * (D / 8) + 256 * kPrepItems - 1) / (256 * kPrepItems),
                                              8LL * sm_count());
  bwd_preprocess_kernel<D><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(p.o),
                                                   static_cast<const __nv_bfloat16*>(p.dout), p.delta, p.dq_acc, rows);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// main backward kernel, d = 256, 64-row query tiles, two passes over the head dim
// ---------------------------------------------------------------------------
// At d = 256 the dK and dV accumulators of a 128-key tile alone would fill all 512
// TMEM columns, and K, V, Q and dO tiles are 64 KB each. So the kernel keeps K and V
// resident (128 KB), takes 64-row query tiles (Q_i, dO_i: 32 KB each, one slot), and
// runs the query loop twice: pass h accumulates columns [128 h, 128 h + 128) of dK and
// dV, and of dQ. S^T and dP^T (the full-d contractions) and P^T, dS^T are recomputed
// in each pass. TMEM columns: S^T [0,64), dP^T [64,128), dQ_h^T [128,192),
// dV_h [256,384), dK_h [384,512). After pass 0 the dQ warpgroup writes dK and dV's
// first halves and hands the accumulators back.
//
// MMAs per query tile i (pass h): S^T = K Q_i^T and dP^T = V dO_i^T (M = 128 keys,
// N = 64 queries, K = 256); dV_h += P^T dO_i[:, h] (P^T from TMEM) and
// dK_h += dS^T Q_i[:, h] (M = 128, N = 128, K = 64); dQ_h^T = K[:, h]^T dS^T
// (M = 128, N = 64, K = 128 keys). Each thread of the two P/dS warpgroups owns one key
// row and 32 of the 64 query columns.
struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr int BR = 64;                     // query rows per tile
  static constexpr int kKV = 128 * 256 * 2;         // K or V tile (64 KB): four 64-column blocks
  static constexpr int kKVRegion = 128 * 128;       // one 64-column block of K / V (16 KB)
  static constexpr int kQ = BR * 256 * 2;           // Q or dO tile (32 KB): four 64-column blocks
  static constexpr int kQRegion = BR * 128;         // one 64-column block of Q / dO (8 KB)
  static constexpr int kDs = 128 * BR * 2;          // dS^T tile: 128 keys x 64 queries (16 KB)
  static constexpr int kVecBytes = 2 * BR * 4;      // -LSE log2 e and D of one query tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKV;
  static constexpr int kOffQ = kOffV + kKV;
  static constexpr int kOffDO = kOffQ + kQ;
  static constexpr int kOffDS = kOffDO + kQ;
  static constexpr int kOffVec = kOffDS + kDs;
  static constexpr int kOffBar = kOffVec + kVecBytes;
  // kv_full, q_full, q_empty, do_full, do_empty, s_full, p_full, dp_full, ds_full, ds_free,
  // dq_full, dq_free, acc_done[2], acc_free, mma_done
  static constexpr int kNumBars = 16;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kOffDS % 1024 == 0 && kOffQ % 1024 == 0 && kOffDO % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kColS = 0, kColDP = 64, kColDQ = 128, kColDV = 256, kColDK = 384;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_main_d256_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const BwdParams p) {
  using C = Bwd256Cfg;
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
  uint64_t* q_empty = bars + 2;
  uint64_t* do_full = bars + 3;
  uint64_t* do_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* dp_full = bars + 7;
  uint64_t* ds_full = bars + 8;
  uint64_t* ds_free = bars + 9;
  uint64_t* dq_full = bars + 10;
  uint64_t* dq_free = bars + 11;
  uint64_t* acc_done = bars + 12;  // two: one per pass
  uint64_t* acc_free = bars + 14;
  uint64_t* mma_done = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key tile), scheduled as in the d = 128 kernel.
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
  const int n_it = g * per_head;   // query tiles per pass
  const int n_all = 2 * n_it;      // both passes
  const float c = p.scale_log2;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(q_full, 1 + 32);
    mbar_init(q_empty, 1);
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 256);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(&acc_done[0], 1);
    mbar_init(&acc_done[1], 1);
    mbar_init(acc_free, 128);
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
      mbar_arrive_expect_tx(kv_full, 2 * C::kKV);
#pragma unroll
      for (int z = 0; z < 4; ++z) {
        tma_load_3d(smem + C::kOffK + z * C::kKVRegion, &tmK, kv_full, z * 64, j0, bkv);
        tma_load_3d(smem + C::kOffV + z * C::kKVRegion, &tmV, kv_full, z * 64, j0, bkv);
      }
    }
    // Q_i (with its row vectors) and dO_i, one slot each, once the previous tile's MMAs
    // are done with it
    bool ok = true;
    for (int gi = 0; gi < n_all && ok; ++gi) {
      const int it = gi % n_it;
      const uint32_t use_par = (gi & 1) ^ 1;  // parity of the slot's previous release
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      const int q_head = b * p.Hq + h;
      if (!(ok = warp_wait_spin(q_empty, use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, C::kQ);
#pragma unroll
        for (int z = 0; z < 4; ++z)
          tma_load_3d(smem + C::kOffQ + z * C::kQRegion, &tmQ, q_full, z * 64, i0, q_head);
      }
      float* lse2 = reinterpret_cast<float*>(smem + C::kOffVec);
      float* dl = lse2 + BR;
      const size_t rbase = (size_t)q_head * p.N;
#pragma unroll
      for (int rr = lane; rr < BR; rr += 32) {
        const int i = i0 + rr;
        const bool in = i < p.N;
        lse2[rr] = in ? -p.lse[rbase + i] * 1.4426950408889634f : -INFINITY;  // -LSE log2(e)
        dl[rr] = in ? p.delta[rbase + i] : 0.f;
      }
      mbar_arrive(q_full);
      if (!(ok = warp_wait_spin(do_empty, use_par, w))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(do_full, C::kQ);
#pragma unroll
        for (int z = 0; z < 4; ++z)
          tma_load_3d(smem + C::kOffDO + z * C::kQRegion, &tmDO, do_full, z * 64, i0, q_head);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<kB128RegsControl, kBwdRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, BR, false, false);  // S^T, dP^T
    constexpr uint32_t kIdKV = idesc_bf16_f32(128, 128, false, true);  // dV_h, dK_h: B MN-major
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, BR, true, true);     // dQ_h^T: A, B MN-major
    const uint64_t dK_k = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
    const uint64_t dV_k = sdesc_sw128(smem_u32(smem + C::kOffV), 16, 1024);
    const uint64_t dQ_k = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t dDO_k = sdesc_sw128(smem_u32(smem + C::kOffDO), 16, 1024);
    const uint64_t dS_k = sdesc_sw128(smem_u32(smem + C::kOffDS), 16, 1024);
    const uint64_t dS_mn = sdesc_sw128(smem_u32(smem + C::kOffDS), C::kDs, 1024);
    // X^T = A B^T over the head dim (A = K or V, B = Q_i or dO_i, K-major, four blocks each)
    auto mma_scores = [&](uint64_t a0, uint64_t b0, uint32_t col) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kKVRegion + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * C::kQRegion + (k & 3) * 32;
        if (leader) mma_bf16_ss(tmem + col, desc_advance(a0, ao), desc_advance(b0, bo), kIdS, k > 0 ? 1u : 0u);
      }
    };
    // progress record: the query tiles (both passes) whose dV MMA this CTA has issued
    unsigned* const prog = (int)blockIdx.x < p.progress_n ? p.progress : nullptr;
    if (leader && prog) prog[blockIdx.x] = 0u;
    bool ok = warp_wait_spin(kv_full, 0, w);
    for (int gi = 0; gi < n_all && ok; ++gi) {
      const int it = gi % n_it;
      const int hp = gi / n_it;  // pass: head-dim half of dK, dV, dQ
      const uint32_t ph = gi & 1;
      const bool first = it == 0;
      // head-dim half hp of Q_i / dO_i (MN-major: LBO = distance of the two 64-column blocks)
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(smem + C::kOffQ + 2 * hp * C::kQRegion), C::kQRegion, 1024);
      const uint64_t dDO_mn = sdesc_sw128(smem_u32(smem + C::kOffDO + 2 * hp * C::kQRegion), C::kQRegion, 1024);
      // K's head-dim half hp as the MN-major A operand of dQ_h^T (M = 128 head-dim rows)
      const uint64_t dK_mn = sdesc_sw128(smem_u32(smem + C::kOffK + 2 * hp * C::kKVRegion), C::kKVRegion, 1024);
      if (!(ok = warp_wait_spin(q_full, ph, w))) break;
      tc_fence_after();
      mma_scores(dK_k, dQ_k, C::kColS);
      if (leader) mma_commit(s_full);
      if (!(ok = warp_wait_spin(do_full, ph, w))) break;
      tc_fence_after();
      mma_scores(dV_k, dDO_k, C::kColDP);
      if (leader) mma_commit(dp_full);
      // dV_h += P^T dO_i[:, h] (A = P^T in TMEM: warpgroup q / 32's packed pairs)
      if (!(ok = warp_wait_spin(p_full, ph, w))) break;
      if (leader && prog) prog[blockIdx.x] = (unsigned)(gi + 1);
      if (first && hp == 1 && !(ok = warp_wait_spin(acc_free, 0, w))) break;  // pass-0 dK, dV written out
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < BR / 16; ++k) {
        const uint32_t acol = C::kColS + (k >> 1) * 32 + (k & 1) * 8;
        if (leader)
          mma_bf16_ts(tmem + C::kColDV, tmem + acol, desc_advance(dDO_mn, k * 2048), kIdKV,
                      (!first || k > 0) ? 1u : 0u);
      }
      if (leader) mma_commit(do_empty);
      // dQ_h^T = K[:, h]^T dS^T, then dK_h += dS^T Q_i[:, h]
      if (!(ok = warp_wait_spin(ds_full, ph, w))) break;
      if (gi >= 1 && !(ok = warp_wait_spin(dq_free, ph ^ 1, w))) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kTileN / 16; ++k)
        if (leader)
          mma_bf16_ss(tmem + C::kColDQ, desc_advance(dK_mn, k * 2048), desc_advance(dS_mn, k * 2048), kIdQ,
                      k > 0 ? 1u : 0u);
      if (leader) mma_commit(dq_full);
#pragma unroll
      for (int k = 0; k < BR / 16; ++k)
        if (leader)
          mma_bf16_ss(tmem + C::kColDK, desc_advance(dS_k, k * 32), desc_advance(dQ_mn, k * 2048), kIdKV,
                      (!first || k > 0) ? 1u : 0u);
      if (leader) {
        mma_commit(q_empty);
        mma_commit(ds_free);
        if (it == n_it - 1) mma_commit(&acc_done[hp]);  // this pass's dK_h, dV_h are complete
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
    // ------------------------------------------------------------ P^T and dS^T, 32 query columns each
    regs_inc<kB128RegsSoftmax, kBwdRegsLaunch>();
    constexpr int HB = 32;
    const int half = (warp - 4) >> 2;
    const int col0 = half * HB;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row within the tile
    const int key = j0 + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t ds_tile = smem_u32(smem + C::kOffDS);
    const bool key_valid = key < p.N;
    for (int gi = 0; gi < n_all; ++gi) {
      const int it = gi % n_it;
      const uint32_t ph = gi & 1;
      const int i0 = (qt_first + it % per_head) * BR + col0;  // first query of this half
      const float* lse2 = reinterpret_cast<const float*>(smem + C::kOffVec) + col0;
      const float* dl = lse2 + BR;
      if (!consumer_wait(q_full, ph, w)) break;
      if (!consumer_wait(s_full, ph, w)) break;
      tc_fence_after();
      float pr[HB];
      {
        uint32_t r0[32];
        tmem_ld32(tmem + lane_off + C::kColS + col0, r0);
        tmem_ld_wait(r0);
#pragma unroll
        for (int i = 0; i < 32; ++i) pr[i] = __uint_as_float(r0[i]);
      }
      // P^T[key][q] = 2^(S c - LSE_q log2 e), zero for future queries and invalid keys.
      const uint64_t c2 = f2_pack(c, c);
      const ulonglong2* nl4 = reinterpret_cast<const ulonglong2*>(lse2);  // 16-byte broadcast loads
#pragma unroll
      for (int i = 0; i < HB; i += 2) {
        const ulonglong2 nv = nl4[i / 4];
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(pr[i], pr[i + 1]), c2, (i & 2) ? nv.y : nv.x), x0, x1);
        pr[i] = ex2(x0);
        pr[i + 1] = ex2(x1);
      }
      if (p.causal && i0 < j0 + kTileN) {  // tiles that reach the diagonal
#pragma unroll
        for (int i = 0; i < HB; ++i)
          if (i0 + i < key) pr[i] = 0.f;
      }
      if (!key_valid) {
#pragma unroll
        for (int i = 0; i < HB; ++i) pr[i] = 0.f;
      }
      // P^T as bf16 pairs over the first 16 of this warpgroup's S^T columns (read above)
      {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pr[2 * i], pr[2 * i + 1]);
        tmem_st16(tmem + lane_off + C::kColS + col0, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(p_full);
      // dS^T = P^T o (dP^T - D_q)
      if (!consumer_wait(dp_full, ph, w)) break;
      tc_fence_after();
      uint32_t dsp[HB / 2];
      const ulonglong2* dl4 = reinterpret_cast<const ulonglong2*>(dl);
      {
        uint32_t r0[32];
        tmem_ld32(tmem + lane_off + C::kColDP + col0, r0);
        tmem_ld_wait(r0);
#pragma unroll
        for (int i = 0; i < HB; i += 2) {
          float a, bb;
          f2_unpack(f2_mul(f2_pack(pr[i], pr[i + 1]),
                           f2_sub(f2_pack(__uint_as_float(r0[i]), __uint_as_float(r0[i + 1])),
                                  (i & 2) ? dl4[i / 4].y : dl4[i / 4].x)),
                    a, bb);
          dsp[i / 2] = pack_bf16x2(a, bb);
        }
      }
      // the dS^T tile is free once dQ and dK of the previous query tile are done
      if (gi >= 1 && !consumer_wait(ds_free, ph ^ 1, w)) break;
#pragma unroll
      for (int ch = 0; ch < HB / 8; ++ch)
        st_shared_v4(ds_tile + sw128_offset(row, half * 4 + ch), dsp[ch * 4], dsp[ch * 4 + 1], dsp[ch * 4 + 2],
                     dsp[ch * 4 + 3]);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
  } else {
    // ------------------------------------------------------------ dQ reductions, dK / dV epilogues
    regs_inc<kB128RegsDq, kBwdRegsLaunch>();
    const int quarter = warp & 3;
    const int tl = quarter * 32 + lane;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // dK, dV columns [128 hp, 128 hp + 128): TMEM lane = key row
    auto write_kv = [&](int hp) {
      const int key = j0 + tl;
      const bool valid = key < p.N;
      const size_t row_idx = (size_t)bkv * p.N + key;
      uint4* dk_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + row_idx * D + hp * 128);
      uint4* dv_dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + row_idx * D + hp * 128);
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which ? C::kColDK : C::kColDV;
        const float mul = which ? p.scale : 1.f;
        uint4* dst = which ? dk_dst : dv_dst;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_off + col + cc * 32, rr);
          tmem_ld_wait(rr);
          if (valid) {
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int i = v4 * 8;
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(rr[i]) * mul, __uint_as_float(rr[i + 1]) * mul);
              u.y = pack_bf16x2(__uint_as_float(rr[i + 2]) * mul, __uint_as_float(rr[i + 3]) * mul);
              u.z = pack_bf16x2(__uint_as_float(rr[i + 4]) * mul, __uint_as_float(rr[i + 5]) * mul);
              u.w = pack_bf16x2(__uint_as_float(rr[i + 6]) * mul, __uint_as_float(rr[i + 7]) * mul);
              dst[cc * 4 + v4] = u;
            }
          }
        }
      }
    };
    bool ok = true;
    for (int gi = 0; gi < n_all; ++gi) {
      const int it = gi % n_it;
      const int hp = gi / n_it;
      const int h = kvh * g + it / per_head;
      const int i0 = (qt_first + it % per_head) * BR;
      // lane = head-dim column of half hp, TMEM columns = the 64 query rows
      float* base = p.dq_acc + ((size_t)(b * p.Hq + h) * p.N + i0) * D + hp * 128 + tl;
      const int nq = min(BR, p.N - i0);
      if (!(ok = consumer_wait(dq_full, gi & 1, w))) break;
      tc_fence_after();
      uint32_t ra[32], rb[32];
      tmem_ld32(tmem + lane_off + C::kColDQ, ra);
      tmem_ld32(tmem + lane_off + C::kColDQ + 32, rb);
      tmem_ld_wait(ra);
      tmem_ld_wait(rb);
      tc_fence_before();
      mbar_arrive(dq_free);
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (q < nq) red_add(base + (size_t)q * D, __uint_as_float(ra[q]));
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (32 + q < nq) red_add(base + (size_t)(32 + q) * D, __uint_as_float(rb[q]));
      if (it == n_it - 1 && hp == 0) {
        // pass 0 done: write the first halves of dK and dV, then hand the columns back
        if (!(ok = consumer_wait(&acc_done[0], 0, w))) break;
        tc_fence_after();
        write_kv(0);
        tc_fence_before();
        mbar_arrive(acc_free);
      }
    }
    if (ok && n_it > 0 && mbar_wait(&acc_done[1], 0, w)) {
      tc_fence_after();
      write_kv(1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_main_d128(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const BwdParams& p, cudaStream_t s) {
  const long long grid = (long long)p.B * p.Hkv * ((p.N + kTileN - 1) / kTileN);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(bwd_main_d128_kernel, Bwd128Cfg::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  bwd_main_d128_kernel<<<(unsigned)grid, kBwdThreads, Bwd128Cfg::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

cudaError_t launch_main_d64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdParams& p, cudaStream_t s) {
  const long long grid = (long long)p.B * p.Hkv * ((p.N + kTileN - 1) / kTileN);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(bwd_main_d64_kernel, Bwd64Cfg::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  bwd_main_d64_kernel<<<(unsigned)grid, kBwdThreads, Bwd64Cfg::kSmemBytes, s>>>(tq, tk, tv, tdo, tdq, p);
  return cudaGetLastError();
}

cudaError_t launch_main_d256(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tdo, const BwdParams& p, cudaStream_t s) {
  const long long grid = (long long)p.B * p.Hkv * ((p.N + kTileN - 1) / kTileN);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(bwd_main_d256_kernel, Bwd256Cfg::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  bwd_main_d256_kernel<<<(unsigned)grid, kBwdThreads, Bwd256Cfg::kSmemBytes, s>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

}  // namespace

int bwd_query_rows(int d) { return d == 256 ? Bwd256Cfg::BR : 128; }

cudaError_t launch_bwd_preprocess(const BwdParams& p, cudaStream_t s) {
  if (p.d == 256) return launch_preprocess_d<256>(p, s);
  return p.d == 128 ? launch_preprocess_d<128>(p, s) : launch_preprocess_d<64>(p, s);
}

cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdParams& p, cudaStream_t s) {
  if (p.d == 256) return launch_main_d256(tq, tk, tv, tdo, p, s);
  return p.d == 128 ? launch_main_d128(tq, tk, tv, tdo, p, s) : launch_main_d64(tq, tk, tv, tdo, tdq, p, s);
}

cudaError_t launch_bwd_convert(const BwdParams& p, cudaStream_t s) {
  const long long n8 = (long long)p.B * p.Hq * p.N * p.d / 8;
  const int blocks = (int)std::min<long long>((n8 + 256 * kPrepItems - 1) / (256 * kPrepItems), 8LL * sm_count());
  bwd_convert_kernel<<<blocks, 256, 0, s>>>(p.dq_acc, static_cast<__nv_bfloat16*>(p.dq), n8, p.scale);
  return cudaGetLastError();
}

}  // namespace fa
