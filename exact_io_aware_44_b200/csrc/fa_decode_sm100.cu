// fa_decode_sm100.cu -- attention of a few new queries against a long key/value
// cache (decode), split along the keys, on sm_100a tensor cores.
//
// In serving, FlashAttention runs against a KV cache; the decode step is bound
// by reading that cache from device memory, which the kernel cannot avoid
// ("FlashAttention Kernel & Online Softmax" card: the relation to the KV cache
// and the decode bandwidth bottleneck). So the design goal is to read K and V
// exactly once at full bandwidth. A GQA group (one batch entry and kv head: g
// query heads x Nq queries) of up to 32 rows is the unit that shares K and V
// (decode_split_kernel<R>); a larger group is cut into 128-row blocks, each a unit
// (decode_split_wide_kernel, below; every group at d = 64, where a group of at most
// 64 rows fills both halves of its block with the same rows, each half taking half of
// every chunk's keys). A unit's keys form n_chunks chunks of 128.
// All units' chunks are laid end to end, and CTA i of the persistent grid (one CTA
// per SM) takes the i-th of n_ctas equal slices of that sequence. A slice may
// cross unit boundaries: each piece of it that lies in one unit is a segment, with
// its own partial output O_s and log-sum-exp LSE_s, stored in slot (unit + i) of
// the workspace. The key ring
// keeps streaming across segments, so an SM never waits for a new CTA to fill it.
// decode_merge_kernel combines a unit's segments with the online-softmax merge
// (running max and rescaled denominators, the same update the pages give for key
// blocks): LSE = log sum_s e^(LSE_s), O = sum_s e^(LSE_s - LSE) O_s.
//
// decode_split_kernel<R> (R = 16 or 32 query rows; 64 + 128 * R / 16 threads; d = 128):
//   warp 0      TMA producer: each segment's query rows (two buffers, by segment
//               parity), and K and V chunks of 128 keys through a 3-stage ring.
//   warp 1      allocates TMEM (4R columns); lane 0 issues the MMAs:
//                 S^T(c) = K_c Q^T   M = 128 keys, N = R query rows, K = d -> TMEM
//                 O^T   += V_c^T P^T  M = d = 128, N = R, K = 128 keys      -> TMEM
//               so keys, and then head-dim columns, sit in TMEM lanes and the few
//               query rows are the MMA's N (tcgen05 needs M >= 64, N may be 16).
//   warps 2-5   thread = TMEM lane: key row of S^T, head-dim row of O^T; query rows
//               (TMEM columns) 0-15. For R = 32, warps 6-9 do the same for rows 16-31,
//               so every softmax thread handles 16 rows and two softmax warps share
//               each SM sub-partition.
// The kernel is instantiated for R = 16 and R = 32 query rows (the host takes the
// smaller that holds the group). Per chunk a thread loads its 16 scores, and the
// CTA keeps one reference max per query row for the segment, raised only when
// some score exceeds it by more than 2^8 (the exact column max is then reduced
// across the 128 threads and O^T and the per-thread partial denominators are
// rescaled); otherwise P = 2^(S c - m_ref) directly. P^T goes to shared memory as
// the MMA's B operand (K-major, 128-byte swizzle). The denominators are per-thread
// partial sums, reduced at the end of each segment.
//
// TMEM columns: S^T buffers [0,R) and [R,2R) (chunk parity), O^T buffers [2R,3R)
// and [3R,4R) (segment parity), so a segment's output is read while the next
// segment accumulates.
#include <math.h>

#include "fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kDecChunk = 128;   // keys per chunk (the MMA M)
constexpr int kDecStages = 3;
constexpr uint32_t kDecRescaleLog2 = 8;

// R: query rows per CTA (the MMA N: 16 or 32).
template <int R>
struct DecCfg {
  static constexpr int D = 128;
  static constexpr int kHalves = R / 16;                 // softmax warpgroups, 16 query rows each
  static constexpr int kThreads = 64 + 128 * kHalves;
  static constexpr int kKV = kDecChunk * D * 2;          // one K or V chunk (32 KB)
  static constexpr int kRegion = kDecChunk * 128;        // 64-column block of a chunk (16 KB)
  static constexpr int kQRegion = R * 128;               // 64-column block of the query tile
  static constexpr int kPRegion = R * 128;               // 64-key block of a P^T tile
  static constexpr int kOffQ = 0;                        // 2 buffers x 2 blocks
  static constexpr int kOffP = kOffQ + 4 * kQRegion;     // 2 buffers x 2 blocks
  static constexpr int kOffKV = kOffP + 4 * kPRegion;    // stages of K then V
  static constexpr int kOffRed = kOffKV + kDecStages * 2 * kKV;   // [3][4][R] floats, then flags [2][8]
  static constexpr int kOffBar = kOffRed + 3 * 4 * R * 4 + 64;
  // q_full[2], q_empty[2], kv_full[3], kv_empty[3], s_full[2], p_full[2], pv_done[2], vote[2],
  // red_bar, mma_done
  static constexpr int kNumBars = 20;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kOffKV % 1024 == 0 && kOffP % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kColS = 0, kColO = 2 * R;
  static constexpr int kTmemCols = 4 * R;
};

// Position in a CTA's chunk sequence: group G, chunk of the group cig, segment seg.
struct ChunkPos {
  int G, cig, seg;
  __device__ __forceinline__ void next(int n_chunks) {
    if (++cig == n_chunks) {
      cig = 0;
      ++G;
      ++seg;
    }
  }
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
// One TMEM column (thread = lane).
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& v) {
  asm volatile(
      "{\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t"
      "}"
      : "=r"(v)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// A bounded wait whose outcome the whole warp agrees on, so that a warp never
// splits between leaving the loop and reaching a warp-synchronous instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  return __all_sync(0xffffffffu, mbar_wait_ns(bar, parity, w, kConsumerPollNs));
}

// Every softmax warp arrives on `bar` once (lane 0, after the warp's own shared-memory
// accesses are ordered by __syncwarp) and waits for the phase to complete: a bounded
// stand-in for a named barrier. The barrier counts warps.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, const WaitCtx& w) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = warp_wait(bar, phase, w);
  phase ^= 1u;
  return ok;
}

template <int R>
__global__ void __launch_bounds__(DecCfg<R>::kThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecCfg<R>;
  constexpr int kRows = 16;  // query rows (TMEM columns) per softmax thread
  constexpr int kSoftmax = 128 * C::kHalves;
  constexpr int S = kDecStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024d(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = bars + 7;
  uint64_t* s_full = bars + 10;
  uint64_t* p_full = bars + 12;
  uint64_t* pv_done = bars + 14;
  uint64_t* vote_bar = bars + 16;
  uint64_t* red_bar = bars + 18;
  uint64_t* mma_done = bars + 19;
  // [3][4][R]: column maxima by chunk parity, then the final denominators
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::kOffRed + 3 * 4 * R * 4);  // [2][8]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nch = p.n_chunks;                     // chunks per group
  const int rows = p.rows;                        // query rows of a group (<= R)
  // this CTA's slice [f0, f1) of all groups' chunks laid end to end
  const long long f0 = (long long)blockIdx.x * p.total_chunks / p.n_ctas;
  const long long f1 = (long long)(blockIdx.x + 1) * p.total_chunks / p.n_ctas;
  const int n = (int)(f1 - f0);                   // >= 1: the host launches at most one CTA per chunk
  const ChunkPos pos0{(int)(f0 / nch), (int)(f0 % nch), 0};

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kSoftmax / 32);
      mbar_init(&pv_done[b], 1);
      mbar_init(&vote_bar[b], kSoftmax / 32);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(red_bar, kSoftmax / 32);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      bool ok = true;
      int issued = 0, q_issued = 0;
      ChunkPos ps = pos0;
      for (int c = 0; c < n && ok; ++c, ps.next(nch)) {
        if (c == 0 || ps.cig == 0) {  // a new segment: its group's query rows
          const int k = ps.seg;
          if (!(ok = mbar_wait_spin(&q_empty[k & 1], ((k >> 1) & 1) ^ 1, w))) break;
          ++q_issued;
          mbar_arrive_expect_tx(&q_full[k & 1], 2 * C::kQRegion);
          for (int z = 0; z < 2; ++z)
            tma_load_3d(smem + C::kOffQ + ((k & 1) * 2 + z) * C::kQRegion, &tmQ, &q_full[k & 1], z * 64,
                        ps.G * rows, 0);
        }
        const int s = c % S;
        if (!(ok = mbar_wait_spin(&kv_empty[s], ((c / S) & 1) ^ 1, w))) break;
        ++issued;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::kKV);
        const int key0 = ps.cig * kDecChunk;
        uint8_t* st = smem + C::kOffKV + s * 2 * C::kKV;
        for (int z = 0; z < 2; ++z) {
          tma_load_3d(st + z * C::kRegion, &tmK, &kv_full[s], z * 64, key0, ps.G);
          tma_load_3d(st + C::kKV + z * C::kRegion, &tmV, &kv_full[s], z * 64, key0, ps.G);
        }
      }
      if (!ok) {  // error path: let the loads already issued land before the CTA exits
        WaitCtx drain{abort_flag, p.status, 20000000ull};
        volatile int zero = 0;
        drain.abort_flag = &zero;
        for (int c = max(0, issued - S); c < issued; ++c) mbar_wait(&kv_full[c % S], (c / S) & 1, drain);
        for (int k = max(0, q_issued - 2); k < q_issued; ++k) mbar_wait(&q_full[k & 1], (k >> 1) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, R, false, false);  // S^T = K Q^T
    constexpr uint32_t kIdO = idesc_bf16_f32(128, R, true, false);   // O^T = V^T P^T
    const uint64_t d_q = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t d_p = sdesc_sw128(smem_u32(smem + C::kOffP), 16, 1024);
    const uint64_t d_k = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);           // K-major K
    const uint64_t d_v = sdesc_sw128(smem_u32(smem + C::kOffKV + C::kKV), C::kRegion, 1024);  // V^T
    // S^T(c) with the query rows of its segment; the Q buffer is released after the
    // segment's last S^T
    auto issue_s = [&](int c, const ChunkPos& ps) -> bool {
      const int qb = ps.seg & 1;
      if (c == 0 || ps.cig == 0) {
        if (!mbar_wait_spin(&q_full[qb], (ps.seg >> 1) & 1, w)) return false;
      }
      if (!mbar_wait_spin(&kv_full[c % S], (c / S) & 1, w)) return false;
      tc_fence_after();
      const uint64_t a0 = desc_advance(d_k, (c % S) * 2 * C::kKV);
      const uint64_t b0 = desc_advance(d_q, qb * 2 * C::kQRegion);
#pragma unroll
      for (int k = 0; k < C::D / 16; ++k) {
        const uint32_t ao = (k >> 2) * C::kRegion + (k & 3) * 32;
        const uint32_t bo = (k >> 2) * C::kQRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColS + (c & 1) * R, desc_advance(a0, ao), desc_advance(b0, bo), kIdS,
                      k > 0 ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&s_full[c & 1]);
        if (c == n - 1 || ps.cig == nch - 1) mma_commit(&q_empty[qb]);
      }
      return true;
    };
    // O^T += V^T P^T(c) into the O^T buffer of its segment, overwriting at a segment's first chunk
    auto issue_pv = [&](int c, const ChunkPos& pp) {
      const uint64_t a0 = desc_advance(d_v, (c % S) * 2 * C::kKV);
      const uint64_t b0 = desc_advance(d_p, (c & 1) * 2 * C::kPRegion);
      const bool first = c == 0 || pp.cig == 0;
#pragma unroll
      for (int k = 0; k < kDecChunk / 16; ++k) {
        const uint32_t bo = (k >> 2) * C::kPRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColO + (pp.seg & 1) * R, desc_advance(a0, k * 2048), desc_advance(b0, bo), kIdO,
                      (!first || k > 0) ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&pv_done[c & 1]);
        mma_commit(&kv_empty[c % S]);
      }
    };
    bool ok = true;
    ChunkPos ps = pos0, pp = pos0;  // ps runs two chunks ahead of pp
    for (int c = 0; c < 2 && c < n && ok; ++c, ps.next(nch)) ok = issue_s(c, ps);
    for (int c = 0; c < n && ok; ++c, pp.next(nch)) {
      if (!(ok = mbar_wait_spin(&p_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      issue_pv(c, pp);
      // S^T(c + 2) into the buffer whose scores the softmax has read (p_full(c))
      if (c + 2 < n) {
        if (!(ok = issue_s(c + 2, ps))) break;
        ps.next(nch);
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
    // Warpgroup h (warps 2 + 4h .. 5 + 4h) owns query rows [16h, 16h + 16).
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;
    const int wq = (warp - 2) & 3;   // 0..3 within the warpgroup, index into the reduction arrays
    const int h = (warp - 2) >> 2;   // warpgroup
    const int jr0 = h * kRows;       // first query row of this warpgroup
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c2 = p.scale_log2;
    float m_ref[kRows], l_part[kRows];
    // Row j is query i = j mod Nq of its head; with the causal mask it sees keys up to
    // Nk - Nq + i. Keys up to all_vis are seen by every valid row.
    const int my_rows = min(max(rows - jr0, 0), kRows);
    const uint32_t row_mask = (1u << my_rows) - 1u;
    const int all_vis = p.causal ? p.Nk - p.Nq : p.Nk - 1;
    uint32_t vote_ph[2] = {0, 0}, red_ph = 0;
    bool ok = true;
    ChunkPos pos = pos0;
    for (int c = 0; c < n && ok; ++c, pos.next(nch)) {
      const bool seg_first = c == 0 || pos.cig == 0;
      const bool seg_last = c == n - 1 || pos.cig == nch - 1;
      const uint32_t o_col = C::kColO + (pos.seg & 1) * R + jr0;
      if (seg_first) {
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          m_ref[j] = -INFINITY;
          l_part[j] = 0.f;
        }
      }
      if (!(ok = warp_wait(&s_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      uint32_t r[kRows];
      tmem_ld16(tmem + lane_off + C::kColS + (c & 1) * R + jr0, r);
      tmem_ld_wait16(r);
      const int key = pos.cig * kDecChunk + t;
      uint32_t vis = key < p.Nk ? row_mask : 0u;  // bit j: row jr0 + j sees this key
      if (key < p.Nk && key > all_vis) {          // the causal edge, in a group's last chunk only
        vis = 0u;
        for (int j = 0; j < my_rows; ++j)
          if (key <= p.Nk - p.Nq + (jr0 + j) % p.Nq) vis |= 1u << j;
      }
      float x[kRows];
      bool over = false;
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        x[j] = (vis >> j) & 1u ? __uint_as_float(r[j]) * c2 : -INFINITY;
        over |= x[j] > m_ref[j] + (float)kDecRescaleLog2;
      }
      // does any thread need a higher reference max for some row?
      const int wv = __any_sync(0xffffffffu, over);
      if (lane == 0) flags[(c & 1) * 8 + (warp - 2)] = wv;
      if (!(ok = group_sync(&vote_bar[c & 1], vote_ph[c & 1], w))) break;
      int any = 0;
#pragma unroll
      for (int f = 0; f < 4 * C::kHalves; ++f) any |= flags[(c & 1) * 8 + f];
      if (any) {
        // exact column max of this chunk over the 128 threads of the warpgroup
        float* rd = red + (c & 1) * 4 * R;
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          float v = x[j];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rd[wq * R + jr0 + j] = v;
        }
        if (!(ok = group_sync(red_bar, red_ph, w))) break;
        float alpha[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const int q = jr0 + j;
          const float cm = fmaxf(fmaxf(rd[q], rd[R + q]), fmaxf(rd[2 * R + q], rd[3 * R + q]));
          const float m_new = fmaxf(m_ref[j], cm);
          alpha[j] = (m_new == -INFINITY || m_ref[j] == m_new) ? 1.f : ex2(m_ref[j] - m_new);
          m_ref[j] = m_new;
          l_part[j] *= alpha[j];
        }
        // the segment's O^T (thread = head-dim row) once every earlier P V of it is complete
        if (!seg_first) {
          if (!(ok = warp_wait(&pv_done[(c - 1) & 1], ((c - 1) >> 1) & 1, w))) break;
          tc_fence_after();
          uint32_t o[kRows];
          tmem_ld16(tmem + lane_off + o_col, o);
          tmem_ld_wait16(o);
#pragma unroll
          for (int j = 0; j < kRows; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha[j]);
          tmem_st16(tmem + lane_off + o_col, o);
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
      for (int j = 0; j < kRows; ++j) {
        const float e = x[j] == -INFINITY ? 0.f : ex2(x[j] - m_ref[j]);
        l_part[j] += e;
        const uint16_t hb = (uint16_t)(pack_bf16x2(e, 0.f) & 0xFFFFu);
        st_shared_u16(pbuf + sw128_offset(jr0 + j, kb >> 4) + (kb & 15), hb);
      }
      fence_async_smem();  // every thread's P^T stores, visible to the MMA (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[c & 1]);
      if (seg_last) {
        // end of a segment: denominators reduced over the 128 threads, O^T / l -> its slot
        float* rd = red + 2 * 4 * R;  // its own slot: a slower thread may still read the last maxima
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          float v = l_part[j];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) rd[wq * R + jr0 + j] = v;
        }
        if (!(ok = group_sync(red_bar, red_ph, w))) break;
        if (!(ok = warp_wait(&pv_done[c & 1], (c >> 1) & 1, w))) break;
        tc_fence_after();
        uint32_t o[kRows];
        tmem_ld16(tmem + lane_off + o_col, o);
        tmem_ld_wait16(o);
        const size_t slot_row = (size_t)(pos.G + (int)blockIdx.x) * rows;
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          if (j < my_rows) {
            const int q = jr0 + j;
            const float l = rd[q] + rd[R + q] + rd[2 * R + q] + rd[3 * R + q];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            p.o_part[(slot_row + q) * C::D + t] = __uint_as_float(o[j]) * inv;
            if (t == 0)
              p.lse_part[slot_row + q] = l > 0.f ? (m_ref[j] + log2f(l)) * 0.6931471805599453f : -INFINITY;
          }
        }
        tc_fence_before();  // the O^T reads, before a later segment's P V overwrites the buffer
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Groups of more than 32 query rows: the query rows are the MMA's M, as in the
// forward pass. A group's rows are cut into blocks of 128 (row blocks); each row
// block is a unit of its own in the chunk sequence, so a group of more than 128
// rows reads its keys once per row block.
//   warp 0      TMA producer: the row block's 128 query rows (one buffer, released
//               after the segment's last S), K and V chunks through a 3-stage ring.
//   warp 1      allocates TMEM (512 columns); lane 0 issues
//                 S(c) = Q K_c^T   M = 128 query rows, N = 128 keys, K = d -> S buffer c & 1
//                 O   += P(c) V_c  A = P from TMEM (TS MMA), N = d            -> O buffer
//               with S two chunks ahead of O and one O buffer per segment parity.
//   warps 4-11  the forward pass's online softmax (reference max raised only when the
//               row max grows by more than 2^8), thread = query row = TMEM lane; warps
//               4-7 take keys [0,64) of every chunk and warps 8-11 keys [64,128), so two
//               warps share each sub-partition (warps 2 and 3 only complete the first
//               warpgroup, whose registers go to the softmax: 120 / 192 of 168 at
//               launch). The two threads of a row exchange their maxima through shared
//               memory every chunk (a thread writes the next chunk's only once p_full of
//               this one is complete, i.e. after its partner has read it) and their
//               shares of the denominator at a segment's end (through the S buffer's
//               unused columns). P in bf16 over the first 64 columns of the S
//               buffer; at a segment's end O / l and the LSE go to the segment's slot.
//               Warps whose rows all lie past the group's end compute nothing and store
//               P = 0.
// TMEM columns: S buffers [0,128) and [128,256), O buffers [256,384) and [384,512).
template <int D_>
struct DecWideCfg {
  static constexpr int D = D_;                             // head dim: 64 or 128
  static constexpr int kRegions = D * 2 / 128;             // 64-column blocks of a row
  static constexpr int kBlockRows = 128;
  static constexpr int kThreads = 384;
  static constexpr int kRegsLaunch = 168, kRegsControl = 120, kRegsSoftmax = 192;
  static_assert(kThreads * kRegsLaunch == 128 * kRegsControl + 256 * kRegsSoftmax, "register split");
  static constexpr int kKV = kDecChunk * D * 2;           // one K or V chunk (16 or 32 KB)
  static constexpr int kRegion = kDecChunk * 128;         // 64-column block of a 128-row tile (16 KB)
  static constexpr int kOffQ = 0;                         // one buffer of kRegions blocks
  static constexpr int kOffKV = kOffQ + kRegions * kRegion;  // stages of K then V
  static constexpr int kOffBar = kOffKV + kDecStages * 2 * kKV;
  // q_full, q_empty, kv_full[3], kv_empty[3], s_full[2], p_full[2], pv_done[2], mma_done, xch
  static constexpr int kNumBars = 16;
  static constexpr int kOffRed = kOffBar + kNumBars * 8;  // [2][128] floats: row maxima by key half
  static constexpr int kOffMisc = kOffRed + 2 * kBlockRows * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kOffKV % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kColS = 0, kColO = 256;
};

// DUP: the block's rows 64-127 repeat rows 0-63 (p.dup), lanes 64-127 taking keys 64-127 of
// every chunk; a template parameter so that the other blocks' code stays as it was
template <int D, bool DUP>
__global__ void __launch_bounds__(DecWideCfg<D>::kThreads, 1)
    decode_split_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using C = DecWideCfg<D>;
  constexpr int S = kDecStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024d(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = bars + 5;
  uint64_t* s_full = bars + 8;
  uint64_t* p_full = bars + 10;
  uint64_t* pv_done = bars + 12;
  uint64_t* mma_done = bars + 14;
  uint64_t* xch = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nch = p.n_chunks;  // chunks per row block
  const long long f0 = (long long)blockIdx.x * p.total_chunks / p.n_ctas;
  const long long f1 = (long long)(blockIdx.x + 1) * p.total_chunks / p.n_ctas;
  const int n = (int)(f1 - f0);
  const ChunkPos pos0{(int)(f0 / nch), (int)(f0 % nch), 0};  // G: row block (group * n_rb + block)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(xch, 256);
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
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
    regs_dec<C::kRegsControl, C::kRegsLaunch>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      bool ok = true;
      int issued = 0, q_issued = 0;
      ChunkPos ps = pos0;
      for (int c = 0; c < n && ok; ++c, ps.next(nch)) {
        const int grp = ps.G / p.n_rb;
        if (c == 0 || ps.cig == 0) {
          const int k = ps.seg;
          if (!(ok = mbar_wait_spin(q_empty, (k & 1) ^ 1, w))) break;
          ++q_issued;
          mbar_arrive_expect_tx(q_full, C::kRegions * C::kRegion);
          const int row0 = grp * p.rows + (ps.G % p.n_rb) * C::kBlockRows;
          for (int z = 0; z < C::kRegions; ++z)
            tma_load_3d(smem + C::kOffQ + z * C::kRegion, &tmQ, q_full, z * 64, row0, 0);
        }
        const int s = c % S;
        if (!(ok = mbar_wait_spin(&kv_empty[s], ((c / S) & 1) ^ 1, w))) break;
        ++issued;
        mbar_arrive_expect_tx(&kv_full[s], 2 * C::kKV);
        const int key0 = ps.cig * kDecChunk;
        uint8_t* st = smem + C::kOffKV + s * 2 * C::kKV;
        for (int z = 0; z < C::kRegions; ++z) {
          tma_load_3d(st + z * C::kRegion, &tmK, &kv_full[s], z * 64, key0, grp);
          tma_load_3d(st + C::kKV + z * C::kRegion, &tmV, &kv_full[s], z * 64, key0, grp);
        }
      }
      if (!ok) {
        WaitCtx drain{abort_flag, p.status, 20000000ull};
        volatile int zero = 0;
        drain.abort_flag = &zero;
        for (int c = max(0, issued - S); c < issued; ++c) mbar_wait(&kv_full[c % S], (c / S) & 1, drain);
        if (q_issued > 0) mbar_wait(q_full, (q_issued - 1) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    regs_dec<C::kRegsControl, C::kRegsLaunch>();
    const bool leader = lane == 0;
    constexpr uint32_t kIdS = idesc_bf16_f32(128, kDecChunk, false, false);  // S = Q K^T
    constexpr uint32_t kIdO = idesc_bf16_f32(128, C::D, false, true);        // O += P V
    const uint64_t d_q = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
    const uint64_t d_k = sdesc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);
    const uint64_t d_v = sdesc_sw128(smem_u32(smem + C::kOffKV + C::kKV), C::kRegion, 1024);
    // S(c) with the query rows of its segment; the Q buffer is released after the
    // segment's last S
    auto issue_s = [&](int c, const ChunkPos& ps) -> bool {
      if (c == 0 || ps.cig == 0) {
        if (!warp_wait_spin(q_full, ps.seg & 1, w)) return false;
        if constexpr (DUP) {
          // rows 64-127 of every 64-column block := rows 0-63 (8 KB each; a row's 128-byte
          // swizzle depends on the row mod 8, which the copy keeps), for the tensor core
          constexpr int kPer = C::kRegion / 2 / 16;  // 16-byte pieces of half a block
          for (int i = lane; i < C::kRegions * kPer; i += 32) {
            uint8_t* src = smem + C::kOffQ + (i / kPer) * C::kRegion + (i % kPer) * 16;
            *reinterpret_cast<uint4*>(src + C::kRegion / 2) = *reinterpret_cast<const uint4*>(src);
          }
          fence_async_smem();
          __syncwarp();
        }
      }
      if (!warp_wait_spin(&kv_full[c % S], (c / S) & 1, w)) return false;
      tc_fence_after();
      const uint64_t b0 = desc_advance(d_k, (c % S) * 2 * C::kKV);
#pragma unroll
      for (int k = 0; k < C::D / 16; ++k) {
        const uint32_t off = (k >> 2) * C::kRegion + (k & 3) * 32;
        if (leader)
          mma_bf16_ss(tmem + C::kColS + (c & 1) * 128, desc_advance(d_q, off), desc_advance(b0, off), kIdS,
                      k > 0 ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&s_full[c & 1]);
        if (c == n - 1 || ps.cig == nch - 1) mma_commit(q_empty);
      }
      return true;
    };
    // O += P(c) V_c into the O buffer of its segment, overwriting at a segment's first chunk
    auto issue_pv = [&](int c, const ChunkPos& pp) -> bool {
      const uint64_t b0 = desc_advance(d_v, (c % S) * 2 * C::kKV);
      const bool first = c == 0 || pp.cig == 0;
      const uint32_t a = tmem + C::kColS + (c & 1) * 128;
#pragma unroll
      for (int k = 0; k < kDecChunk / 16; ++k) {
        if (leader)
          mma_bf16_ts(tmem + C::kColO + (pp.seg & 1) * 128, a + k * 8, desc_advance(b0, k * 16 * 128), kIdO,
                      (!first || k > 0) ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&pv_done[c & 1]);
        mma_commit(&kv_empty[c % S]);
      }
      return true;
    };
    bool ok = true;
    ChunkPos ps = pos0, pp = pos0;  // ps runs two chunks ahead of pp
    for (int c = 0; c < 2 && c < n && ok; ++c, ps.next(nch)) ok = issue_s(c, ps);
    for (int c = 0; c < n && ok; ++c, pp.next(nch)) {
      if (!(ok = warp_wait_spin(&p_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      if (!(ok = issue_pv(c, pp))) break;
      // S(c + 2) into the columns of P(c): the MMAs run in issue order, so P V(c) reads
      // P(c) before S(c + 2) overwrites it
      if (c + 2 < n) {
        if (!(ok = issue_s(c + 2, ps))) break;
        ps.next(nch);
      }
    }
    if (leader) mma_commit(mma_done);
    __syncwarp();
    WaitCtx drain{abort_flag, p.status, 20000000ull};
    volatile int zero = 0;
    drain.abort_flag = &zero;
    mbar_wait(mma_done, 0, drain);
  } else if (warp < 4) {
    regs_dec<C::kRegsControl, C::kRegsLaunch>();
  } else {
    // ------------------------------------------------------------ softmax (thread = query row)
    regs_inc<C::kRegsSoftmax, C::kRegsLaunch>();
    const int quarter = warp & 3;
    const int h = (warp - 4) >> 2;      // key half of every chunk: [64h, 64h + 64)
    const int r = quarter * 32 + lane;  // row of the block, TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c2 = p.scale_log2;
    // every valid row sees the keys up to all_vis
    const int all_vis = p.causal ? p.Nk - p.Nq : p.Nk - 1;
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    float m_ref = -INFINITY;  // reference max, log2 units (S c)
    float l = 0.f;            // this half's share of the denominator
    int lim = -1;             // last key this row sees; -1 for rows past the group's end
    bool dead = true;         // every row of this warp lies past the group's end
    uint32_t xph = 0;
    auto exchange = [&]() -> bool {  // all 256 softmax threads
      mbar_arrive(xch);
      const bool res = warp_wait(xch, xph, w);
      xph ^= 1u;
      return res;
    };
    bool ok = true;
    ChunkPos pos = pos0;
    for (int c = 0; c < n && ok; ++c, pos.next(nch)) {
      const bool seg_first = c == 0 || pos.cig == 0;
      const bool seg_last = c == n - 1 || pos.cig == nch - 1;
      if (seg_first) {
        // row of the group: query j mod Nq of its head (with dup, lanes r and r + 64 hold row r)
        const int j = DUP ? (r & 63) : (pos.G % p.n_rb) * C::kBlockRows + r;
        m_ref = -INFINITY;
        l = 0.f;
        lim = j >= p.rows ? -1 : (p.causal ? p.Nk - p.Nq + j % p.Nq : p.Nk - 1);
        dead = __all_sync(0xffffffffu, lim < 0);
      }
      if (!(ok = warp_wait(&s_full[c & 1], (c >> 1) & 1, w))) break;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + C::kColS + (c & 1) * 128;
      constexpr int kHalf = kDecChunk / 2;
      float x[kHalf];
      float mx = -INFINITY;
      // with dup, lanes 0-63 take keys [0, 64) of the chunk and lanes 64-127 keys [64, 128);
      // the warpgroup of the other half only stores zeros for P (and still writes its
      // columns of O at the end)
      const bool keys_off = DUP && h != (quarter >> 1);
      if (!dead && !keys_off) {
#pragma unroll
        for (int cc = 0; cc < kHalf / 32; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tS + h * kHalf + cc * 32, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[cc * 32 + i] = __uint_as_float(rr[i]) * c2;
        }
        const int k0 = pos.cig * kDecChunk + h * kHalf;
        // the causal edge and keys past Nk; rows past the group's end (lim < 0) are left
        // unmasked: their results are never written, and masking them cost a loop per chunk
        if (k0 + kHalf - 1 > all_vis) {
#pragma unroll
          for (int i = 0; i < kHalf; ++i)
            if (k0 + i > lim) x[i] = -INFINITY;
        }
        float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int i = 4; i < kHalf; i += 8) {
          mq[0] = fmax3(mq[0], x[i], x[i + 1]);
          mq[1] = fmax3(mq[1], x[i + 2], x[i + 3]);
          if (i + 4 < kHalf) mq[2] = fmax3(mq[2], x[i + 4], x[i + 5]);  // the last step has 4 left
          if (i + 6 < kHalf) mq[3] = fmax3(mq[3], x[i + 6], x[i + 7]);
        }
        mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
      }
      // the row max over the whole chunk: this half's and the partner's. The slot is written
      // once p_full of the previous chunk is complete, i.e. once the partner has read it.
      if (c > 0 && !(ok = warp_wait(&p_full[(c - 1) & 1], ((c - 1) >> 1) & 1, w))) break;
      red[h * C::kBlockRows + r] = mx;
      if (!(ok = exchange())) break;
      const float m_new = fmaxf(m_ref, fmaxf(mx, red[(1 - h) * C::kBlockRows + r]));
      float alpha = 1.f;
      bool rescale = false;
      if (m_new > m_ref + (float)kDecRescaleLog2) {
        // O holds earlier chunks of this segment only if some of them had a visible key
        if (!seg_first && m_ref != -INFINITY) {
          alpha = ex2(m_ref - m_new);
          l *= alpha;
          rescale = true;
        }
        m_ref = m_new;
      }
      const float mc = m_ref == -INFINITY ? 0.f : m_ref;
      uint32_t pk[kHalf / 2];
      if (!dead && !keys_off) {
        uint64_t rs2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kHalf; i += 2) {
          const float e0 = ex2(x[i] - mc), e1 = ex2(x[i + 1] - mc);
          rs2 = f2_add(rs2, f2_pack(e0, e1));
          pk[i / 2] = pack_bf16x2(e0, e1);
        }
        float ra, rb;
        f2_unpack(rs2, ra, rb);
        l += ra + rb;
      } else {
#pragma unroll
        for (int i = 0; i < kHalf / 2; ++i) pk[i] = 0u;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // this half's columns of the segment's O once P V(c - 1) is complete
        if (!(ok = warp_wait(&pv_done[(c - 1) & 1], ((c - 1) >> 1) & 1, w))) break;
        tc_fence_after();
        const uint32_t tO = tmem + lane_off + C::kColO + (pos.seg & 1) * 128 + h * (C::D / 2);
#pragma unroll
        for (int cc = 0; cc < C::D / 64; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tO + cc * 32, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(tO + cc * 32, rr);
        }
      }
      float l_row = 0.f;
      if (seg_last) {
        // the row's denominator: both halves' shares, through column 64 + h of S(c), which
        // both halves have read by now and P does not reach
        tmem_st1(tS + kHalf + h, __float_as_uint(l));
        tmem_st_wait();
        tc_fence_before();
        if (!(ok = exchange())) break;
        tc_fence_after();
        uint32_t other;
        tmem_ld1(tS + kHalf + 1 - h, other);
        l_row = l + __uint_as_float(other);
      }
      tmem_st32(tS + h * (kHalf / 2), pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[c & 1]);
      if (seg_last && !dead) {
        // end of a segment: this half's columns of O / l, and the LSE, into the segment's slot
        if (!(ok = warp_wait(&pv_done[c & 1], (c >> 1) & 1, w))) break;
        tc_fence_after();
        const uint32_t tO = tmem + lane_off + C::kColO + (pos.seg & 1) * 128 + h * (C::D / 2);
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        const size_t slot_row = (size_t)(pos.G + (int)blockIdx.x) * p.slot_rows + r;
        float4* dst = reinterpret_cast<float4*>(p.o_part + slot_row * C::D + h * (C::D / 2));
#pragma unroll
        for (int cc = 0; cc < C::D / 64; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tO + cc * 32, rr);
          tmem_ld_wait(rr);
          if (lim >= 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              dst[(cc * 32 + i) / 4] = make_float4(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv,
                                                   __uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
          }
        }
        if (h == 0 && lim >= 0)
          p.lse_part[slot_row] = l_row > 0.f ? (m_ref + log2f(l_row)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();  // the O reads, before a later segment's P V overwrites the buffer
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

// The CTA whose slice of the chunk sequence holds chunk x: the largest i with
// floor(i * total / n_ctas) <= x.
__device__ __forceinline__ int decode_cta_of(long long x, const DecodeParams& p) {
  return (int)(((x + 1) * p.n_ctas - 1) / p.total_chunks);
}

// One warp per query row, four head-dim columns per lane: the row's group's
// segments (slots group + i for the CTAs i that covered it) combined in one pass
// with the online-softmax merge (running max, rescaled weight sum and output),
// then O in bf16 and LSE.
constexpr int kMergeRowsPerBlock = 8;

// D / 32 head-dim columns per lane (D = 64 or 128).
template <int D>
__global__ void __launch_bounds__(32 * kMergeRowsPerBlock) decode_merge_kernel(const DecodeParams p) {
  constexpr int kPer = D / 32;
  const long long row = (long long)blockIdx.x * kMergeRowsPerBlock + (threadIdx.x >> 5);
  if (row >= p.rows_total) return;
  const int lane = threadIdx.x & 31;
  const int q = (int)(row % p.rows);                                // row of its group
  const int G = (int)(row / p.rows) * p.n_rb + q / p.slot_rows;     // its row block's unit
  const int sq = q % p.slot_rows;                                   // row within the slot
  const int i0 = decode_cta_of((long long)G * p.n_chunks, p);
  const int i1 = decode_cta_of((long long)(G + 1) * p.n_chunks - 1, p);
  float m = -INFINITY, wsum = 0.f;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  // one partial row (o_part, lse_part at slot_row) into the running merge (the same steps
  // as the loop below, which the single-partial case keeps as it was measured)
  auto take = [&](size_t slot_row) {
    const float ls = p.lse_part[slot_row];
    float o[kPer];
    const float* src = p.o_part + slot_row * D + lane * kPer;
    if constexpr (kPer == 4) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(src);
      o[0] = v.x, o[1] = v.y;
    }
    if (ls == -INFINITY) return;  // no visible key in this segment
    const float m_new = fmaxf(m, ls);
    const float a = __expf(m - m_new);  // 0 while m is still -inf
    const float wgt = __expf(ls - m_new);
    wsum = wsum * a + wgt;
#pragma unroll
    for (int e = 0; e < kPer; ++e) acc[e] = acc[e] * a + wgt * o[e];
    m = m_new;
  };
  if (p.dup) {
    // each CTA's slot holds two partial rows of the query row, sq and sq + 64 (one per half
    // of every key chunk)
#pragma unroll 2
    for (int i = i0; i <= i1; ++i) {
      take((size_t)(G + i) * p.slot_rows + sq);
      take((size_t)(G + i) * p.slot_rows + sq + 64);
    }
  } else {
#pragma unroll 4
    for (int i = i0; i <= i1; ++i) {
      const size_t slot_row = (size_t)(G + i) * p.slot_rows + sq;
      const float ls = p.lse_part[slot_row];
      float o[kPer];
      const float* src = p.o_part + slot_row * D + lane * kPer;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        o[0] = v.x, o[1] = v.y;
      }
      if (ls == -INFINITY) continue;  // no visible key in this segment
      const float m_new = fmaxf(m, ls);
      const float a = __expf(m - m_new);  // 0 while m is still -inf
      const float wgt = __expf(ls - m_new);
      wsum = wsum * a + wgt;
#pragma unroll
      for (int e = 0; e < kPer; ++e) acc[e] = acc[e] * a + wgt * o[e];
      m = m_new;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint32_t packed[kPer / 2];
#pragma unroll
  for (int e = 0; e < kPer / 2; ++e) packed[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) + row * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = packed[0];
  }
  if (lane == 0) p.lse[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

template <int R>
cudaError_t launch_decode_r(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const DecodeParams& p, cudaStream_t s) {
  using C = DecCfg<R>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(decode_split_kernel<R>, C::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  decode_split_kernel<R><<<(unsigned)p.n_ctas, C::kThreads, C::kSmemBytes, s>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<128><<<(unsigned)((p.rows_total + kMergeRowsPerBlock - 1) / kMergeRowsPerBlock),
                             32 * kMergeRowsPerBlock, 0, s>>>(p);
  return cudaGetLastError();
}

template <int D, bool DUP>
cudaError_t launch_decode_wide(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const DecodeParams& p, cudaStream_t s) {
  using C = DecWideCfg<D>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = ensure_smem_limit(decode_split_wide_kernel<D, DUP>, C::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  decode_split_wide_kernel<D, DUP><<<(unsigned)p.n_ctas, C::kThreads, C::kSmemBytes, s>>>(tq, tk, tv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<D><<<(unsigned)((p.rows_total + kMergeRowsPerBlock - 1) / kMergeRowsPerBlock),
                           32 * kMergeRowsPerBlock, 0, s>>>(p);
  return cudaGetLastError();
}

// d = 128: groups of up to 32 rows take the kernels with the rows as the MMA's N (the
// cache read once); larger groups, and every group at d = 64 (whose O^T would need an
// M = 64 MMA), take 128-row blocks.
int decode_rows_per_cta(int rows, int d) {
  if (d != 128) return DecWideCfg<64>::kBlockRows;
  return rows <= 16 ? 16 : rows <= 32 ? 32 : DecWideCfg<128>::kBlockRows;
}

cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          cudaStream_t s) {
  if (p.d == 64)
    return p.dup ? launch_decode_wide<64, true>(tq, tk, tv, p, s) : launch_decode_wide<64, false>(tq, tk, tv, p, s);
  switch (decode_rows_per_cta(p.rows, p.d)) {
    case 16: return launch_decode_r<16>(tq, tk, tv, p, s);
    case 32: return launch_decode_r<32>(tq, tk, tv, p, s);
    default: return launch_decode_wide<128, false>(tq, tk, tv, p, s);
  }
}

}  // namespace fa
