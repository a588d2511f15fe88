// fa_decode_sm100.cu -- attention of a few new queries against a long key/value
// cache (decode), split along the keys, on sm_100a tensor cores.
//
// In serving, FlashAttention runs against a KV cache; the decode step is bound
// by reading that cache from device memory, which the kernel cannot avoid
// ("FlashAttention Kernel & Online Softmax" card: the relation to the KV cache
// and the decode bandwidth bottleneck). So the design goal is to read K and V
// exactly once at full bandwidth: one CTA handles all query rows of one GQA
// group (g query heads x Nq queries, at most 32 rows) against one slice of the
// keys, and enough slices run side by side to fill the GPU.
//
// Each split produces an unnormalised-then-normalised partial output O_s and its
// log-sum-exp LSE_s; decode_merge_kernel combines them with the online-softmax
// merge (running max and rescaled denominators, the same update the pages give
// for key blocks): LSE = log sum_s e^(LSE_s), O = sum_s e^(LSE_s - LSE) O_s.
//
// decode_split_kernel (192 threads, d = 128):
//   warp 0      TMA producer: the group's query rows once, then K and V chunks of
//               128 keys through a 3-stage ring.
//   warp 1      allocates TMEM (64 or 128 columns); lane 0 issues the MMAs:
//                 S^T(c) = K_c Q^T   M = 128 keys, N = R query rows, K = d -> TMEM
//                 O^T   += V_c^T P^T  M = d = 128, N = R, K = 128 keys      -> TMEM
//               so keys, and then head-dim columns, sit in TMEM lanes and the few
//               query rows are the MMA's N (tcgen05 needs M >= 64, N may be 16).
//   warps 2-5   thread = TMEM lane: key row of S^T, head-dim row of O^T.
// The kernel is instantiated for R = 16 and R = 32 query rows (the host takes the
// smaller that holds the group). Per chunk a thread loads its R scores, and the CTA keeps one reference max per
// query row, raised only when some score exceeds it by more than 2^8 (the exact
// column max is then reduced across the 128 threads and O^T and the per-thread
// partial denominators are rescaled); otherwise P = 2^(S c - m_ref) directly.
// P^T goes to shared memory as the MMA's B operand (K-major, 128-byte swizzle).
// The denominators are per-thread partial sums, reduced once at the end.
//
// TMEM columns: S^T buffers [0,R) and [R,2R) (chunk parity), O^T [2R,3R).
#include <math.h>

#include "fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 192;
constexpr int kDecChunk = 128;   // keys per chunk (the MMA M)
constexpr int kDecStages = 3;
constexpr uint32_t kDecRescaleLog2 = 8;

// R: query rows per CTA (the MMA N: 16 or 32).
template <int R>
struct DecCfg {
  static constexpr int D = 128;
  static constexpr int kKV = kDecChunk * D * 2;          // one K or V chunk (32 KB)
  static constexpr int kRegion = kDecChunk * 128;        // 64-column block of a chunk (16 KB)
  static constexpr int kQRegion = R * 128;               // 64-column block of the query tile
  static constexpr int kPRegion = R * 128;               // 64-key block of a P^T tile
  static constexpr int kOffQ = 0;                        // 2 blocks
  static constexpr int kOffP = kOffQ + 2 * kQRegion;     // 2 buffers x 2 blocks
  static constexpr int kOffKV = kOffP + 4 * kPRegion;    // stages of K then V
  static constexpr int kOffRed = kOffKV + kDecStages * 2 * kKV;   // [3][4][R] floats, then flags [2][4]
  static constexpr int kOffBar = kOffRed + 3 * 4 * R * 4 + 64;
  // q_full, kv_full[3], kv_empty[3], s_full[2], p_full[2], pv_done[2], vote[2], red_bar, mma_done
  static constexpr int kNumBars = 17;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kOffKV % 1024 == 0 && kOffP % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // TMEM: S^T buffers [0, R) and [R, 2R) (chunk parity), O^T [2R, 3R)
  static constexpr int kColS = 0, kColO = 2 * R;
  static constexpr int kTmemCols = R == 16 ? 64 : 128;
};

__device__ __forceinline__ uint8_t* align1024d(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// tcgen05.ld / tcgen05.st, shape 32x32b, 16 columns (thread = TMEM lane).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// R-column forms (R = 16 or 32).
template <int R>
__device__ __forceinline__ void tmem_ld_r(uint32_t taddr, uint32_t (&r)[R]) {
  if constexpr (R == 16) {
    tmem_ld16(taddr, r);
    tmem_ld_wait16(r);
  } else {
    tmem_ld32(taddr, r);
    tmem_ld_wait(r);
  }
}
template <int R>
__device__ __forceinline__ void tmem_st_r(uint32_t taddr, const uint32_t (&r)[R]) {
  if constexpr (R == 16)
    tmem_st16(taddr, r);
  else
    tmem_st32(taddr, r);
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// A bounded wait whose outcome the whole warp agrees on, so that a warp never
// splits between leaving the loop and reaching a warp-synchronous instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  return __all_sync(0xffffffffu, mbar_wait_ns(bar, parity, w, kConsumerPollNs));
}

// All 128 threads of the softmax warpgroup arrive on `bar` and wait for the phase
// to complete (a bounded stand-in for a named barrier).
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, const WaitCtx& w) {
  mbar_arrive(bar);
  const bool ok = warp_wait(bar, phase, w);
  phase ^= 1u;
  return ok;
}

template <int R>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecCfg<R>;
  constexpr int kDecRows = R;
  constexpr int S = kDecStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024d(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 4;
  uint64_t* s_full = bars + 7;
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 11;
  uint64_t* vote_bar = bars + 13;
  uint64_t* red_bar = bars + 15;
  uint64_t* mma_done = bars + 16;
  // [3][4][R]: column maxima by chunk parity, then the final denominators
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kOffRed + 3 * 4 * R * 4);  // [2][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bkv = blockIdx.y;  // b * Hkv + kv head
  const int b = bkv / p.Hkv;
  const int kvh = bkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int rows = g * p.Nq;                                 // valid query rows (<= R)
  const int row0 = (b * p.Hq + kvh * g) * p.Nq;              // first global query row
  const int n_chunks_all = (p.Nk + kDecChunk - 1) / kDecChunk;
  const int c_begin = min(split * p.chunks_per_split, n_chunks_all);
  const int c_end = min(c_begin + p.chunks_per_split, n_chunks_all);
  const int n = c_end - c_begin;                             // chunks of this split
  const int k_end = min(c_end * kDecChunk, p.Nk);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&pv_done[t], 1);
      mbar_init(&vote_bar[t], 128);
    }
    mbar_init(red_bar, 128);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx w{abort_flag, p.status, p.wait_budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::kQRegion);
      for (int z = 0; z < 2; ++z) tma_load_3d(smem + C::kOffQ + z * C::kQRegion, &tmQ, q_full, z * 64, row0, 0);
      bool ok = true;
      int issued = 0;
      for (int c = 0; c < n && ok; ++c) {
        const int s = c % S;
        if (!(ok = mbar_wait_spin(&kv_empty[s], ((c / S) & 1) ^ 1, w))) break;
        ++issued;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::kKV);
        const int key0 = (c_begin + c) * kDecChunk;
        uint8_t* st = smem + C::kOffKV + s * 2 * C::kKV;
        for (int z = 0; z < 2; ++z) {
          tma_load_3d(st + z * C::kRegion, &tmK, &kv_full[s], z * 64, key0, bkv);
          tma_load_3d(st + C::kKV + z * C::kRegion, &tmV, &kv_full[s], z * 64, key0, bkv);
        }
      }
      if (!ok) {  // error path: let the loads already issued land before the CTA exits
        WaitCtx drain{abort_flag, p.status, 20000000ull};
        volatile int zero = 0;
        drain.abort_flag = &zero;
        for (int c = max(0, issued - S); c < issued; ++c) mbar_wait(&kv_full[c % S], (c / S) & 1, drain);
        mbar_wait(q_full, 0, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, kDecRows, false, false);  // S^T = K Q^T
    constexpr uint32_t kIdO = idesc_bf16_f32(128, kDecRows, true, false);   // O^T = V^T P^T
    const uint64_t d_q = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t d_p = sdesc_sw128(smem_u32(smem + C::kOffP), 16, 1024);
    const uint64_t d_k = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);           // K-major K
    const uint64_t d_v = sdesc_sw128(smem_u32(smem + C::kOffKV + C::kKV), C::kRegion, 1024);  // V^T
    auto issue_s = [&](int c) {
      const uint64_t a0 = desc_advance(d_k, (c % S) * 2 * C::kKV);
#pragma unroll
      for (int k = 0; k < C::D / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kRegion + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * C::kQRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColS + (c & 1) * R, desc_advance(a0, ao), desc_advance(d_q, bo), kIdS,
                      k > 0 ? 1u : 0u);
      }
      if (leader) mma_commit(&s_full[c & 1]);
    };
    auto issue_pv = [&](int c) {
      const uint64_t a0 = desc_advance(d_v, (c % S) * 2 * C::kKV);
      const uint64_t b0 = desc_advance(d_p, (c & 1) * 2 * C::kPRegion);
#pragma unroll
      for (int k = 0; k < kDecChunk / 16; ++k) {
        const uint32_t bo = (k >> 2) * C::kPRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColO, desc_advance(a0, k * 2048), desc_advance(b0, bo), kIdO,
                      (c > 0 || k > 0) ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&pv_done[c & 1]);
        mma_commit(&kv_empty[c % S]);
      }
    };
    bool ok = n == 0 || mbar_wait_spin(q_full, 0, w);
    tc_fence_after();
    for (int c = 0; c < 2 && c < n && ok; ++c) {
      if (!(ok = mbar_wait_spin(&kv_full[c % S], (c / S) & 1, w))) break;
      tc_fence_after();
      issue_s(c);
    }
    for (int c = 0; c < n && ok; ++c) {
      if (!(ok = mbar_wait_spin(&p_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      issue_pv(c);
      // S^T(c + 2) into the buffer whose scores the softmax has read (p_full(c))
      if (c + 2 < n) {
        if (!(ok = mbar_wait_spin(&kv_full[(c + 2) % S], ((c + 2) / S) & 1, w))) break;
        tc_fence_after();
        issue_s(c + 2);
      }
    }
    if (leader) mma_commit(mma_done);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_done, 0, drain);
  } else {
    // ------------------------------------------------------------ softmax (thread = TMEM lane)
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const int wq = warp - 2;  // 0..3, index into the reduction arrays
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c2 = p.scale_log2;
    float m_ref[kDecRows], l_part[kDecRows];
#pragma unroll
    for (int j = 0; j < kDecRows; ++j) {
      m_ref[j] = -INFINITY;
      l_part[j] = 0.f;
    }
    // Row j is query i = j mod Nq of its head; with the causal mask it sees keys up to
    // Nk - Nq + i. Keys up to all_vis are seen by every valid row.
    const uint32_t row_mask = rows >= 32 ? 0xffffffffu : ((1u << rows) - 1u);
    const int all_vis = p.causal ? p.Nk - p.Nq : p.Nk - 1;
    uint32_t vote_ph[2] = {0, 0}, red_ph = 0;
    bool ok = true;
    for (int c = 0; c < n && ok; ++c) {
      if (!(ok = warp_wait(&s_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      uint32_t r[R];
      tmem_ld_r<R>(tmem + lane_off + C::kColS + (c & 1) * R, r);
      const int key = (c_begin + c) * kDecChunk + t;
      uint32_t vis = key < k_end ? row_mask : 0u;  // bit j: row j sees this key
      if (key < k_end && key > all_vis) {           // the causal edge, in the last chunk only
        vis = 0u;
        for (int j = 0; j < rows; ++j)
          if (key <= p.Nk - p.Nq + j % p.Nq) vis |= 1u << j;
      }
      float x[kDecRows];
      bool over = false;
#pragma unroll
      for (int j = 0; j < kDecRows; ++j) {
        x[j] = (vis >> j) & 1u ? __uint_as_float(r[j]) * c2 : -INFINITY;
        over |= x[j] > m_ref[j] + (float)kDecRescaleLog2;
      }
      // does any thread need a higher reference max for some row?
      const int wv = __any_sync(0xffffffffu, over);
      if (lane == 0) flags[(c & 1) * 4 + wq] = wv;
      if (!(ok = group_sync(&vote_bar[c & 1], vote_ph[c & 1], w))) break;
      const bool rescale = flags[(c & 1) * 4 + 0] | flags[(c & 1) * 4 + 1] | flags[(c & 1) * 4 + 2] |
                           flags[(c & 1) * 4 + 3];
      if (rescale) {
        // exact column max of this chunk over the 128 threads
        float* rd = red + (c & 1) * 4 * R;
#pragma unroll
        for (int j = 0; j < kDecRows; ++j) {
          float v = x[j];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rd[wq * R + j] = v;
        }
        if (!(ok = group_sync(red_bar, red_ph, w))) break;
        float alpha[kDecRows];
#pragma unroll
        for (int j = 0; j < kDecRows; ++j) {
          const float cm = fmaxf(fmaxf(rd[j], rd[R + j]), fmaxf(rd[2 * R + j], rd[3 * R + j]));
          const float m_new = fmaxf(m_ref[j], cm);
          alpha[j] = (m_new == -INFINITY || m_ref[j] == m_new) ? 1.f : ex2(m_ref[j] - m_new);
          m_ref[j] = m_new;
          l_part[j] *= alpha[j];
        }
        // O^T (thread = head-dim row) once every earlier P V is complete
        if (c > 0) {
          if (!(ok = warp_wait(&pv_done[(c - 1) & 1], ((c - 1) >> 1) & 1, w))) break;
          tc_fence_after();
          uint32_t o[R];
          tmem_ld_r<R>(tmem + lane_off + C::kColO, o);
#pragma unroll
          for (int j = 0; j < kDecRows; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha[j]);
          tmem_st_r<R>(tmem + lane_off + C::kColO, o);
          tmem_st_wait();
        }
      }
      // P^T(c) -> shared memory, once P V(c - 2) has read this buffer
      if (c >= 2) {
        if (!(ok = warp_wait(&pv_done[c & 1], ((c - 2) >> 1) & 1, w))) break;
      }
      const uint32_t pbuf = smem_u32(smem + C::kOffP + (c & 1) * 2 * C::kPRegion) + (t >> 6) * C::kPRegion;
      const uint32_t kb = (uint32_t)(t & 63) * 2;  // byte offset of this key within a 128-byte row
#pragma unroll
      for (int j = 0; j < kDecRows; ++j) {
        const float e = x[j] == -INFINITY ? 0.f : ex2(x[j] - m_ref[j]);
        l_part[j] += e;
        const uint16_t hb = (uint16_t)(pack_bf16x2(e, 0.f) & 0xFFFFu);
        st_shared_u16(pbuf + sw128_offset(j, kb >> 4) + (kb & 15), hb);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[c & 1]);
    }
    // epilogue: denominators reduced over the 128 threads, O^T / l -> partial outputs
    if (ok && n > 0) {
      float* rd = red + 2 * 4 * R;  // its own slot: a slower thread may still read the last maxima
#pragma unroll
      for (int j = 0; j < kDecRows; ++j) {
        float v = l_part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rd[wq * R + j] = v;
      }
      ok = group_sync(red_bar, red_ph, w);
      if (ok) ok = warp_wait(mma_done, 0, w);
      if (ok) {
        tc_fence_after();
        uint32_t o[R];
        tmem_ld_r<R>(tmem + lane_off + C::kColO, o);
        float* opart = p.o_part + (size_t)split * p.rows_total * C::D;
#pragma unroll
        for (int j = 0; j < kDecRows; ++j) {
          if (j < rows) {
            const float l = rd[j] + rd[R + j] + rd[2 * R + j] + rd[3 * R + j];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            opart[(size_t)(row0 + j) * C::D + t] = __uint_as_float(o[j]) * inv;
            if (t == 0)
              p.lse_part[(size_t)split * p.rows_total + row0 + j] =
                  l > 0.f ? (m_ref[j] + log2f(l)) * 0.6931471805599453f : -INFINITY;
          }
        }
      }
    }
    if (n == 0 && t < rows) {  // an empty split contributes nothing
      p.lse_part[(size_t)split * p.rows_total + row0 + t] = -INFINITY;
      float* opart = p.o_part + ((size_t)split * p.rows_total + row0 + t) * C::D;
      for (int dd = 0; dd < C::D; ++dd) opart[dd] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// One block per query row, one thread per head-dim column: the split partials
// combined with the online-softmax merge, O in bf16 and LSE.
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p) {
  const long long row = blockIdx.x;
  const int t = threadIdx.x;
  float m = -INFINITY;
  for (int s = 0; s < p.n_splits; ++s) m = fmaxf(m, p.lse_part[(size_t)s * p.rows_total + row]);
  float wsum = 0.f, acc = 0.f;
  for (int s = 0; s < p.n_splits; ++s) {
    const float ls = p.lse_part[(size_t)s * p.rows_total + row];
    const float wgt = ls == -INFINITY ? 0.f : __expf(ls - m);
    wsum += wgt;
    acc += wgt * p.o_part[((size_t)s * p.rows_total + row) * 128 + t];
  }
  const float o = wsum > 0.f ? acc / wsum : 0.f;
  static_cast<__nv_bfloat16*>(p.o)[row * 128 + t] = __float2bfloat16_rn(o);
  if (t == 0) p.lse[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

template <int R>
cudaError_t launch_decode_r(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const DecodeParams& p, cudaStream_t s) {
  using C = DecCfg<R>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid((unsigned)p.n_splits, (unsigned)(p.B * p.Hkv));
  decode_split_kernel<R><<<grid, kDecThreads, C::kSmemBytes, s>>>(tq, tk, tv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<<<(unsigned)p.rows_total, 128, 0, s>>>(p);
  return cudaGetLastError();
}

int decode_rows_per_cta(int rows) { return rows <= 16 ? 16 : 32; }

cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          cudaStream_t s) {
  const int rows = (p.Hq / p.Hkv) * p.Nq;
  return decode_rows_per_cta(rows) == 16 ? launch_decode_r<16>(tq, tk, tv, p, s) : launch_decode_r<32>(tq, tk, tv, p, s);
}

}  // namespace fa
