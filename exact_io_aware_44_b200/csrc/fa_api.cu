// fa_api.cu -- the library's C ABI (declared in include/fa.h): argument
// validation, TMA descriptor encoding, the device status word, and launches.
// Nothing here computes attention; every step of the path runs in the kernels.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace fa {

// First device-side error since the last fa_get_status(); 0 = none.
__device__ int g_status = 0;

// Progress record of the last forward / backward main-kernel launch on this device:
// word i is how far CTA i got (see fa_get_progress).
__device__ unsigned g_progress[kProgressSlots];

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

namespace {

constexpr int kMaxDevices = 64;
std::atomic<uint64_t> g_wait_budget_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

struct DeviceInfo {
  int checked = 0;  // 0 = not yet, 1 = sm_100, -1 = not sm_100
  int* status = nullptr;
  unsigned* progress = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device if it is an sm_100 part, with its status-word address.
int current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.checked == 0) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    if (major != 10) {
      di.checked = -1;
    } else {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_LAUNCH;
      }
      di.status = static_cast<int*>(ptr);
      if (cudaGetSymbolAddress(&ptr, g_progress) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_LAUNCH;
      }
      di.progress = static_cast<unsigned*>(ptr);
      di.checked = 1;
    }
  }
  if (di.checked != 1) return FA_ERR_NO_DEVICE;
  *out = &di;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common size checks. Returns FA_OK, or the code to return; *empty is set when
// there is nothing to do.
int check_sizes(int B, int Hq, int Hkv, int N, int d, float scale, bool* empty) {
  *empty = false;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 0 || d < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if ((long long)B * Hq * (long long)N >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  if (N == 0) *empty = true;
  return FA_OK;
}

// 3-D tensor map over [heads, N, d] (bf16, or E4M3 as bytes) with a box one
// 128-byte block wide and `box_rows` high, and the 128-byte swizzle; rows past N
// read as zero.
int make_map(CUtensorMap* m, const void* base, int d, int N, int heads, int box_rows = kTileM, bool e4m3 = false) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return FA_ERR_LAUNCH;
  const cuuint64_t elem = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * elem, (cuuint64_t)N * d * elem};
  cuuint32_t box[3] = {(cuuint32_t)(128 / elem), (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

// 3-D fp32 tensor map over the dQ accumulator [heads, N, d] with a 32-column
// (128-byte), 128-row box and the 128-byte swizzle: the target of the d = 64
// backward's TMA reduce-adds. Rows past N are never written.
int make_map_acc(CUtensorMap* m, const float* base, int d, int N, int heads) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return FA_ERR_LAUNCH;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)kTileM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

// Consecutive heads that the kernels schedule together (the causal work order runs
// longest-first across them): `per_unit` heads share one unit (a kv head) whose
// operands are re-read, `reuse_bytes` of them. As many units as keep those within
// 48 MB, well inside the 126 MB L2, and a divisor of the unit count, so that no
// short last group ends the launch with long blocks.
int head_group(double reuse_bytes, int per_unit, int total) {
  const double budget = 48.0 * 1024 * 1024;
  const int units = total / per_unit;
  // groups of more than 1024 units schedule no better and would only lengthen the search
  const int max_units = (int)std::min(1024.0, std::max(1.0, budget / std::max(reuse_bytes, 1.0)));
  if (units <= max_units) return total;
  for (int u = max_units; u > 1; --u)
    if (units % u == 0) return u * per_unit;
  return per_unit;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

int fa_version(void) { return 100; }

const char* fa_error_string(int code) {
  switch (code) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported shape";
    case FA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case FA_ERR_LAUNCH: return "CUDA launch or query failed";
    case FA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case FA_ERR_NO_DEVICE: return "no sm_100 device is current";
    default: return "unknown status";
  }
}

void fa_set_wait_budget_ns(uint64_t ns) {
  if (ns < 100000ull) ns = 100000ull;
  if (ns > 60000000000ull) ns = 60000000000ull;
  g_wait_budget_ns.store(ns);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d,
           int causal, float scale, void* stream) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (rc != FA_OK) return rc;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, d, N, B * Hq)) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, d, N, B * Hkv)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, d, N, B * Hkv)) != FA_OK) return rc;
  FwdParams p;
  p.o = o;
  p.lse = lse;
  p.status = di->status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.causal = causal ? 1 : 0;
  const int rows_per_cta = fwd_tiles_per_cta(d) * kTileM;
  p.n_qblk = (N + rows_per_cta - 1) / rows_per_cta;
  p.head_group = head_group(2.0 * N * d * 2, Hq / Hkv, B * Hq);  // K and V of a kv head
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_scale = 1.f;
  p.wait_budget_ns = g_wait_budget_ns.load();
  p.progress = di->progress;
  p.progress_n = kProgressSlots;
  if (launch_fwd_bf16(tq, tk, tv, p, d, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

static int fwd_f8(bool e5m2, const void* q, const void* k, const void* v, float descale_q, float descale_k,
                  float descale_v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                  void* stream) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (rc != FA_OK) return rc;
  for (float ds : {descale_q, descale_k, descale_v})
    if (!(ds > 0.f) || !isfinite(ds)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  const float c = scale * descale_q * descale_k * 1.4426950408889634f;
  if (!isfinite(c) || !(c > 0.f) || !isfinite(descale_v)) return FA_ERR_INVALID_ARG;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, d, N, B * Hq, kTileM, true)) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, d, N, B * Hkv, kTileM, true)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, d, N, B * Hkv, kTileM, true)) != FA_OK) return rc;
  FwdParams p;
  p.o = o;
  p.lse = lse;
  p.status = di->status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.causal = causal ? 1 : 0;
  p.n_qblk = (N + 2 * kTileM - 1) / (2 * kTileM);
  p.head_group = head_group(2.0 * N * d, Hq / Hkv, B * Hq);  // K and V of a kv head, one byte each
  p.scale_log2 = c;
  p.o_scale = descale_v;
  p.wait_budget_ns = g_wait_budget_ns.load();
  p.progress = di->progress;
  p.progress_n = kProgressSlots;
  const cudaError_t e = e5m2 ? launch_fwd_e5m2(tq, tk, tv, p, static_cast<cudaStream_t>(stream))
                             : launch_fwd_e4m3(tq, tk, tv, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k, float descale_v,
               void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  return fwd_f8(false, q, k, v, descale_q, descale_k, descale_v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

int fa_fwd_e5m2(const void* q, const void* k, const void* v, float descale_q, float descale_k, float descale_v,
                void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  return fwd_f8(true, q, k, v, descale_q, descale_k, descale_v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int Hq, int Hkv, int N,
               int d, int causal, float scale, void* stream) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (rc != FA_OK) return rc;
  if (d % 4 != 0 || d > 128) return FA_ERR_UNSUPPORTED;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  FwdF32Params p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (launch_fwd_f32(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

}  // extern "C"

namespace fa {
namespace {

// Decode work split. A GQA group's query rows ((Hq / Hkv) * Nq) are one unit when
// they fit one CTA's MMA (at most 32 rows), else blocks of 128 rows, each a unit
// of its own (row blocks). All units' 128-key chunks are laid end to end and cut
// into n_ctas equal slices, one per split-kernel CTA. Automatic: one CTA per SM of
// a 148-SM part (the kernels keep one CTA per SM), so the slices run as one wave;
// num_splits > 0: units * num_splits CTAs. Never more CTAs than chunks. A fixed
// rule of the sizes, not of the current device, so that the workspace size can be
// computed without one. A slice may cross unit boundaries; each (unit, CTA) piece
// is a segment with its own slot (unit + CTA index) in the workspace.
constexpr int kDecodeSms = 148;
constexpr int kDecodeBlockRows = 128;

struct DecodeSplit {
  int n_rb, slot_rows, n_chunks, n_ctas, dup;
  long long total_chunks;
  long long n_units() const { return total_chunks / n_chunks; }
  long long n_slots() const { return n_units() + n_ctas - 1; }
};

DecodeSplit decode_split(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits) {
  const int rows = (Hq / Hkv) * Nq;
  const int n_rb = rows <= 32 ? 1 : (rows + kDecodeBlockRows - 1) / kDecodeBlockRows;
  // d = 64 groups of at most 64 rows (128-row-block kernel): each query row has two partial
  // rows in a slot, one per half of every key chunk, so that all four SM sub-partitions
  // exponentiate (+15 % measured; at d = 128 the cache read bounds such groups instead)
  const int dup = d == 64 && rows <= 64;
  const int slot_rows = dup ? kDecodeBlockRows : n_rb == 1 ? rows : kDecodeBlockRows;
  const int n_chunks = (Nk + kTileN - 1) / kTileN;
  const long long units = (long long)B * Hkv * n_rb;
  const long long total = units * n_chunks;
  const long long want = num_splits > 0 ? units * num_splits : kDecodeSms;
  return {n_rb, slot_rows, n_chunks, (int)std::min(want, total), dup, total};
}

int check_decode(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, Nq, d, scale, &empty);
  if (rc != FA_OK) return rc;
  if (Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  if (causal && Nq > Nk) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long rows = (long long)(Hq / Hkv) * Nq;
  const long long n_rb = rows <= 32 ? 1 : (rows + kDecodeBlockRows - 1) / kDecodeBlockRows;
  if (rows >= (1ll << 31) || (long long)B * Hkv * n_rb * ((Nk + kTileN - 1) / kTileN) >= (1ll << 31) ||
      (long long)B * Hkv * Nk >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t decode_workspace(int d, const DecodeSplit& sp) {
  const size_t slot_rows = (size_t)sp.slot_rows;
  const size_t opart = ((size_t)sp.n_slots() * slot_rows * d * sizeof(float) + 255) & ~size_t(255);
  return opart + (size_t)sp.n_slots() * slot_rows * sizeof(float);
}

}  // namespace
}  // namespace fa

extern "C" {

size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits) {
  if (check_decode(B, Hq, Hkv, Nq, Nk, d, 0, 1.f) != FA_OK) return 0;
  return decode_workspace(d, decode_split(B, Hq, Hkv, Nq, Nk, d, num_splits));
}

int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace, int B, int Hq,
              int Hkv, int Nq, int Nk, int d, int causal, float scale, int num_splits, void* stream) {
  int rc = check_decode(B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != FA_OK) return rc;
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_ALIGNMENT;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  const DecodeSplit sp = decode_split(B, Hq, Hkv, Nq, Nk, d, num_splits);
  const long long rows = (long long)B * Hq * Nq;
  CUtensorMap tq, tk, tv;
  if ((rc = make_map(&tq, q, d, (int)rows, 1, decode_rows_per_cta((Hq / Hkv) * Nq, d))) != FA_OK) return rc;
  if ((rc = make_map(&tk, k, d, Nk, B * Hkv)) != FA_OK) return rc;
  if ((rc = make_map(&tv, v, d, Nk, B * Hkv)) != FA_OK) return rc;
  DecodeParams p;
  p.o = o;
  p.lse = lse;
  p.o_part = static_cast<float*>(workspace);
  const int g_rows = (Hq / Hkv) * Nq;
  const size_t opart = ((size_t)sp.n_slots() * sp.slot_rows * d * sizeof(float) + 255) & ~size_t(255);
  p.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + opart);
  p.status = di->status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.rows = g_rows;
  p.n_rb = sp.n_rb;
  p.slot_rows = sp.slot_rows;
  p.dup = sp.dup;
  p.n_chunks = sp.n_chunks;
  p.n_ctas = sp.n_ctas;
  p.total_chunks = sp.total_chunks;
  p.rows_total = rows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_budget_ns = g_wait_budget_ns.load();
  if (launch_decode(tq, tk, tv, p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  bool empty;
  if (check_sizes(B, Hq, Hkv, N, d, 1.f, &empty) != FA_OK) return 0;
  const size_t rows = (size_t)B * Hq * N;
  const size_t delta = (rows * sizeof(float) + 255) & ~size_t(255);
  return delta + rows * (size_t)d * sizeof(float);
}

}  // extern "C"

namespace fa {
namespace {

enum BwdPhase { kPhasePre = 1, kPhaseMain = 2, kPhaseConvert = 4, kPhaseAll = 7 };

// Validates the arguments each requested phase reads, then launches the phases
// in order on `stream`. Nothing is launched unless every check passes.
int run_bwd(int phases, const void* q, const void* k, const void* v, const void* o, const float* lse,
            const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int N, int d,
            int causal, float scale, void* stream) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (rc != FA_OK) return rc;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (empty) return FA_OK;
  const bool pre = phases & kPhasePre, main = phases & kPhaseMain, conv = phases & kPhaseConvert;
  if (!workspace) return FA_ERR_INVALID_ARG;
  if (pre && (!o || !dout)) return FA_ERR_INVALID_ARG;
  if (main && (!q || !k || !v || !lse || !dout || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if (conv && !dq) return FA_ERR_INVALID_ARG;
  const void* need16[] = {pre ? o : nullptr,     pre || main ? dout : nullptr, main ? q : nullptr,
                          main ? k : nullptr,    main ? v : nullptr,           main ? lse : nullptr,
                          main ? dk : nullptr,   main ? dv : nullptr,          conv ? dq : nullptr};
  for (const void* ptr : need16)
    if (ptr && !aligned16(ptr)) return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_ALIGNMENT;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  CUtensorMap tq, tk, tv, tdo, tdq;
  memset(&tdq, 0, sizeof(tdq));
  if (main) {
    const int q_rows = bwd_query_rows(d);  // query rows per backward tile
    if ((rc = make_map(&tq, q, d, N, B * Hq, q_rows)) != FA_OK) return rc;
    if ((rc = make_map(&tk, k, d, N, B * Hkv)) != FA_OK) return rc;
    if ((rc = make_map(&tv, v, d, N, B * Hkv)) != FA_OK) return rc;
    if ((rc = make_map(&tdo, dout, d, N, B * Hq, q_rows)) != FA_OK) return rc;
  }
  const size_t rows = (size_t)B * Hq * N;
  const size_t delta_bytes = (rows * sizeof(float) + 255) & ~size_t(255);
  BwdParams p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.delta = static_cast<float*>(workspace);
  p.dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + delta_bytes);
  if (main && d == 64 && (rc = make_map_acc(&tdq, p.dq_acc, d, N, B * Hq)) != FA_OK) return rc;
  p.status = di->status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  // per kv head, for its Hq / Hkv query heads: Q and dO (bf16), the fp32 dQ accumulator, LSE and D
  p.head_group = head_group((double)(Hq / Hkv) * N * (8.0 * d + 8), 1, B * Hkv);
  p.wait_budget_ns = g_wait_budget_ns.load();
  p.progress = di->progress;
  p.progress_n = kProgressSlots;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pre && launch_bwd_preprocess(p, s) != cudaSuccess) return FA_ERR_LAUNCH;
  if (main && launch_bwd_main(tq, tk, tv, tdo, tdq, p, s) != cudaSuccess) return FA_ERR_LAUNCH;
  if (conv && launch_bwd_convert(p, s) != cudaSuccess) return FA_ERR_LAUNCH;
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" {

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
           void* dk, void* dv, void* workspace, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
           void* stream) {
  return run_bwd(kPhaseAll, q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, N, d, causal, scale, stream);
}

int fa_bwd_preprocess(const void* o, const void* dout, void* workspace, int B, int Hq, int Hkv, int N, int d,
                      void* stream) {
  return run_bwd(kPhasePre, nullptr, nullptr, nullptr, o, nullptr, dout, nullptr, nullptr, nullptr, workspace, B, Hq,
                 Hkv, N, d, 0, 1.f, stream);
}

int fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dk, void* dv,
                void* workspace, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  return run_bwd(kPhaseMain, q, k, v, nullptr, lse, dout, nullptr, dk, dv, workspace, B, Hq, Hkv, N, d, causal, scale,
                 stream);
}

int fa_bwd_convert(void* dq, const void* workspace, int B, int Hq, int Hkv, int N, int d, float scale, void* stream) {
  return run_bwd(kPhaseConvert, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq, nullptr, nullptr,
                 const_cast<void*>(workspace), B, Hq, Hkv, N, d, 0, scale, stream);
}

int fa_get_status(void* stream) {
  DeviceInfo* di;
  int rc = current_device(&di);
  if (rc != FA_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  int v = 0;
  if (cudaMemcpy(&v, di->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_LAUNCH;
  const int zero = 0;
  if (v != 0 && cudaMemcpy(di->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return FA_ERR_LAUNCH;
  return v;
}

int fa_get_progress(unsigned* out, int n, void* stream) {
  if (!out || n < 0) return FA_ERR_INVALID_ARG;
  if (n > kProgressSlots) n = kProgressSlots;
  DeviceInfo* di;
  int rc = current_device(&di);
  if (rc != FA_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  if (n > 0 && cudaMemcpy(out, di->progress, (size_t)n * sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FA_ERR_LAUNCH;
  return n;
}

int fa_selftest_wait_timeout(uint64_t budget_ns, void* stream) {
  DeviceInfo* di;
  int rc = current_device(&di);
  if (rc != FA_OK) return rc;
  if (budget_ns < 1000ull) budget_ns = 1000ull;
  if (budget_ns > 2000000000ull) budget_ns = 2000000000ull;
  if (launch_wait_selftest(di->status, budget_ns, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_LAUNCH;
  return fa_get_status(stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_bwd_noalloc: the backward pass without a caller-provided workspace, for
// callers that cannot allocate device memory (see include/fa.h).
// ---------------------------------------------------------------------------
namespace fa {
namespace {

// D and the fp32 dQ accumulator of fa_bwd_noalloc. In host code this name is
// only a stand-in for the device array: the kernels get its device address,
// looked up per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device
std::mutex g_noalloc_mu;

}  // namespace
}  // namespace fa

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                              int causal, float scale, void* stream) {
  bool empty;
  int rc = check_sizes(B, Hq, Hkv, N, d, scale, &empty);
  if (rc != FA_OK) return rc;
  if (fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  DeviceInfo* di;
  if ((rc = current_device(&di)) != FA_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
      // Once per device, with that device current.
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) {
        cudaGetLastError();
        return FA_ERR_LAUNCH;
      }
      g_noalloc_addr[dev] = addr;
    }
    scratch = g_noalloc_addr[dev];
  }
  return run_bwd(kPhaseAll, q, k, v, o, lse, dout, dq, dk, dv, scratch, B, Hq, Hkv, N, d, causal, scale, stream);
}
