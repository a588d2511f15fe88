// fa_internal.h -- parameter blocks and launchers shared by the host C ABI
// (fa_api.cu) and the kernel translation units. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace fa {

constexpr int kTileM = 128;  // query rows per tile (TMEM lanes)
constexpr int kTileN = 128;  // keys per tile

struct FwdParams {
  void* o;            // bf16 [B, Hq, N, d]
  float* lse;         // [B, Hq, N]
  int* status;        // device status word
  int B, Hq, Hkv, N;
  int causal;
  int n_qblk;         // query blocks of 2 tiles (256 rows) per head
  int head_group;     // consecutive (batch, head) pairs scheduled together (a multiple of Hq / Hkv)
  float scale_log2;   // scale * log2(e) (times the Q and K descales for E4M3 inputs)
  float o_scale;      // multiplies O at the end (the V descale for E4M3 inputs, else 1)
  uint64_t wait_budget_ns;
  unsigned* progress;  // per-CTA progress record (blockIdx.x < progress_n), or null
  int progress_n;
};

struct FwdF32Params {
  const float *q, *k, *v;
  float* o;
  float* lse;
  int B, Hq, Hkv, N, d;
  int causal;
  float scale_log2;
};

struct BwdParams {
  const void *q, *k, *v, *o, *dout;
  const float* lse;
  void *dq, *dk, *dv;
  float* delta;      // workspace: D = rowsum(dO o O), [B, Hq, N]
  float* dq_acc;     // workspace: fp32 dQ accumulator, [B, Hq, N, d]
  int* status;
  int B, Hq, Hkv, N, d;
  int causal;
  float scale;
  float scale_log2;
  int head_group;    // consecutive (batch, kv head) pairs scheduled together
  uint64_t wait_budget_ns;
  unsigned* progress;  // per-CTA progress record (blockIdx.x < progress_n), or null
  int progress_n;
};

struct DecodeParams {
  void* o;            // bf16 [B, Hq, Nq, d]
  float* lse;         // [B, Hq, Nq]
  float* o_part;      // workspace: per segment slot, normalised partial O [n_slots, slot_rows, d]
  float* lse_part;    // workspace: per segment slot, partial LSE (natural log) [n_slots, slot_rows]
  int* status;
  int B, Hq, Hkv, Nq, Nk, d;
  int causal;
  int rows;                        // query rows of a GQA group: (Hq / Hkv) * Nq
  int n_rb;                        // row blocks per group (units of the chunk sequence)
  int slot_rows;                   // query rows of a workspace slot (of a row block)
  int dup;                         // d = 64, at most 64 rows a group (128-row-block kernel): rows r and
                                   // r + 64 of the block are query row r, lanes 64-127 taking keys
                                   // 64-127 of every chunk; both write a partial (slot rows r, r + 64)
  int n_chunks;                    // 128-key chunks per row block
  int n_ctas;                      // split-kernel CTAs (equal slices of all row blocks' chunks)
  long long total_chunks;          // B * Hkv * n_rb * n_chunks
  long long rows_total;            // B * Hq * Nq
  float scale_log2;
  uint64_t wait_budget_ns;
};

// Launchers (return a cudaError_t from the launch).
cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int d, cudaStream_t s);
// Query tiles of 128 rows per forward CTA for head dim d (the grid's query blocks).
int fwd_tiles_per_cta(int d);
cudaError_t launch_fwd_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t s);
cudaError_t launch_fwd_e5m2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, cudaStream_t s);
cudaError_t launch_fwd_f32(const FwdF32Params& p, cudaStream_t s);
// Decode: the split kernel, then the merge of the splits.
// Query rows per decode CTA for a GQA group of `rows` rows: 16 or 32 (one CTA's
// MMA N covers the group), else 128 (a row block, the MMA M).
int decode_rows_per_cta(int rows, int d);
cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          cudaStream_t s);
// Query rows per tile of the main backward kernel for head dim d (its TMA box height).
int bwd_query_rows(int d);
// Backward phases: D and zeroed dQ accumulator; main kernel; dQ conversion.
cudaError_t launch_bwd_preprocess(const BwdParams& p, cudaStream_t s);
// `tdq`: fp32 map over the dQ accumulator (d = 64 only; 32-column, 128-row box, 128-byte swizzle).
cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdParams& p, cudaStream_t s);
cudaError_t launch_bwd_convert(const BwdParams& p, cudaStream_t s);
cudaError_t launch_wait_selftest(int* status, uint64_t budget_ns, cudaStream_t s);
// Streaming multiprocessors of the current device (148 on a B200).
int sm_count();
// Slots of the per-CTA progress record: CTAs with blockIdx.x below this record.
constexpr int kProgressSlots = 1 << 16;

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current device,
// once per device (the attribute is per device; `done` holds one bit per device
// ordinal below 64, larger ordinals set it on every call). Thread-safe: a race
// only repeats the idempotent call.
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace fa
