// fa_fwd_f32.cu -- float32 attention forward on the CUDA cores.
//
// The same tiled online-softmax forward as the tensor-core kernel, in fp32
// throughout: a tile of 32 query rows stays in shared memory while 32-key tiles
// of K and V stream through; each row keeps a running max m and denominator l
// and rescales its output accumulator by 2^(m - m_new) when a tile raises the
// max ("FlashAttention Kernel & Online Softmax", first paragraph). Scores are
// kept in the log2 domain (x c, c = scale * log2(e)) so the exponentials are 2^x.
//
// CTA: 128 threads, 4 per query row. For S = Q K^T a thread computes 8 scores
// of its row (columns lane%4 + 4i); for O += P V it owns d/4 output columns
// (lane%4 + 4i) of its row.
#include <math.h>

#include "fa.h"
#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kBr = 32;
constexpr int kBc = 32;
constexpr int kF32Threads = 128;
constexpr int kLoadBatch = 8;  // float4 loads a thread has in flight at once

// Copy `rows` rows of d floats (row-major, 16-byte aligned rows: d % 4 == 0) from global
// memory at src + r0 * d into shared memory with row pitch `pitch`; rows past n read as
// zero. Each thread issues kLoadBatch 16-byte loads before it stores any of them, so the
// loads' latencies overlap instead of following one another.
__device__ __forceinline__ void load_rows_f32(float* dst, int pitch, const float* src, int r0, int rows, int n,
                                              int d) {
  const int n4 = rows * d / 4;
  for (int e0 = 0; e0 < n4; e0 += kF32Threads * kLoadBatch) {
    float4 v[kLoadBatch];
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      const int e = e0 + u * kF32Threads + (int)threadIdx.x;
      const int rr = (e * 4) / d, cc = (e * 4) % d;
      v[u] = (e < n4 && r0 + rr < n) ? *reinterpret_cast<const float4*>(src + (size_t)(r0 + rr) * d + cc)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kLoadBatch; ++u) {
      const int e = e0 + u * kF32Threads + (int)threadIdx.x;
      if (e < n4) {
        const int rr = (e * 4) / d, cc = (e * 4) % d;
        float* t = dst + rr * pitch + cc;
        t[0] = v[u].x;
        t[1] = v[u].y;
        t[2] = v[u].z;
        t[3] = v[u].w;
      }
    }
  }
}

__global__ void __launch_bounds__(kF32Threads) fwd_f32_kernel(const FwdF32Params p) {
  extern __shared__ float sm[];
  const int d = p.d;
  const int ldq = d + 1;  // padded row pitch of Q and K in shared memory
  float* sQ = sm;                   // [kBr][d + 1]
  float* sK = sQ + kBr * ldq;       // [kBc][d + 1]
  float* sV = sK + kBc * ldq;       // [kBc][d]
  float* sP = sV + kBc * d;         // [kBr][kBc + 1]

  const int n_qt = (p.N + kBr - 1) / kBr;
  const int bh = blockIdx.x / n_qt;
  const int qt = n_qt - 1 - (blockIdx.x % n_qt);
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int kvh = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int q0 = qt * kBr;
  const int tid = threadIdx.x;
  const int r = tid >> 2;   // query row within the tile
  const int sub = tid & 3;  // which quarter of the columns
  const int qrow = q0 + r;

  const float* qg = p.q + ((size_t)(b * p.Hq + h) * p.N) * d;
  const float* kg = p.k + ((size_t)kvh * p.N) * d;
  const float* vg = p.v + ((size_t)kvh * p.N) * d;

  load_rows_f32(sQ, ldq, qg, q0, kBr, p.N, d);

  const float c = p.scale_log2;
  float m = -INFINITY, l = 0.f;
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;
  const int n_cols = d / 4;  // output columns owned by this thread

  const int n_kv_all = (p.N + kBc - 1) / kBc;
  const int n_kv = p.causal ? min(n_kv_all, (q0 + kBr - 1) / kBc + 1) : n_kv_all;
  for (int j = 0; j < n_kv; ++j) {
    const int k0 = j * kBc;
    __syncthreads();  // previous tile's K, V and P are no longer read
    load_rows_f32(sK, ldq, kg, k0, kBc, p.N, d);
    load_rows_f32(sV, d, vg, k0, kBc, p.N, d);
    __syncthreads();

    float s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = 0.f;
    for (int kk = 0; kk < d; ++kk) {
      const float qv = sQ[r * ldq + kk];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = fmaf(qv, sK[(sub + 4 * i) * ldq + kk], s[i]);
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int key = k0 + sub + 4 * i;
      const bool visible = key < p.N && (!p.causal || key <= qrow);
      s[i] = visible ? s[i] * c : -INFINITY;
      mx = fmaxf(mx, s[i]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    // A row with nothing visible yet keeps m = -inf and contributes nothing.
    const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
    const float ref = (m_new == -INFINITY) ? 0.f : m_new;
    float rs = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float e = exp2f(s[i] - ref);
      sP[r * (kBc + 1) + sub + 4 * i] = e;
      rs += e;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = l * alpha + rs;
    m = m_new;
    __syncwarp();  // the four threads of a row share its P values
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] *= alpha;
    for (int jj = 0; jj < kBc; ++jj) {
      const float pv = sP[r * (kBc + 1) + jj];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < n_cols) acc[i] = fmaf(pv, sV[jj * d + sub + 4 * i], acc[i]);
    }
  }

  if (qrow < p.N) {
    const size_t row_idx = (size_t)(b * p.Hq + h) * p.N + qrow;
    const float inv = 1.f / l;
    float* og = p.o + row_idx * d;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < n_cols) og[sub + 4 * i] = acc[i] * inv;
    if (sub == 0) p.lse[row_idx] = (m + log2f(l)) * 0.6931471805599453f;
  }
}

// Failure-detection self test: wait on a barrier that nothing completes.
__global__ void wait_selftest_kernel(int* status, uint64_t budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"((uint32_t)__cvta_generic_to_shared(&bar)));
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(&bar);
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    const uint64_t max_iter = budget_ns / 8 + 1024;
    for (uint64_t i = 0; i < max_iter; ++i) {
      uint32_t ok;
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(a)
          : "memory");
      if (ok) return;
      uint64_t t1;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
      if (t1 - t0 > budget_ns) break;
    }
    abort_flag = 1;
    atomicCAS(status, 0, (int)FA_ERR_DEVICE_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdF32Params& p, cudaStream_t s) {
  const int ldq = p.d + 1;
  const size_t smem = sizeof(float) * (size_t)(kBr * ldq + kBc * ldq + kBc * p.d + kBr * (kBc + 1));
  cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_qt = (p.N + kBr - 1) / kBr;
  const long long grid = (long long)p.B * p.Hq * n_qt;
  fwd_f32_kernel<<<(unsigned)grid, kF32Threads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int* status, uint64_t budget_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, budget_ns);
  return cudaGetLastError();
}

}  // namespace fa
