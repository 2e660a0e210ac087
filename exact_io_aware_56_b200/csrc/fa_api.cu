// C-ABI layer of libfa: argument checks, device check, TMA tensor maps,
// watchdog word, status strings. Declared in include/fa.h.

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "../../include/fa_profile.h"
#include "../../include/fa_test.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

__global__ void test_exp2_kernel(const float* x, float* yp, float* ye, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    yp[i] = exp2_poly(x[i]);
    ye[i] = ex2(x[i]);
  }
}

__global__ void test_exp2_accurate_kernel(const float* x, float* y, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) y[i] = exp2_accurate(x[i]);
}

constexpr int kMaxDevices = 64;

// Device error word written by the kernels' watchdog.
__device__ unsigned int g_err_word;

std::atomic<uint64_t> g_budget_ns{2000000000ull};
std::atomic<int> g_fault{0};
std::atomic<void*> g_ev_pre{nullptr};
std::atomic<void*> g_ev_main{nullptr};
std::atomic<void*> g_ev_dec{nullptr};
thread_local char t_cuda_msg[256] = "no CUDA error recorded";

struct DevState {
  std::once_flag once;
  bool supported = false;
  unsigned int* err = nullptr;
  int sms = 0;
};
DevState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

int record_cuda(cudaError_t e) {
  snprintf(t_cuda_msg, sizeof(t_cuda_msg), "CUDA error %d: %s", static_cast<int>(e), cudaGetErrorString(e));
  return FA_ERR_CUDA;
}

// Checks the current device once: compute capability 10.0 (sm_100a) and the
// address of its error word. Returns FA_OK or an error status.
int device_state(DevState** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  DevState& st = g_dev[dev];
  std::call_once(st.once, [&] {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return;
    if (major != 10 || minor != 0) return;
    if (cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || st.sms <= 0) return;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return;
    st.err = static_cast<unsigned int*>(p);
    st.supported = true;
  });
  if (!st.supported) return FA_ERR_UNSUPPORTED;
  *out = &st;
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int Hq, int Hkv, int N, int d, int causal, float scale) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0) return FA_ERR_INVALID_ARGUMENT;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  // Index arithmetic limits: (B*Hq) fits the grid and a TMA coordinate; the
  // element count of one tensor stays below 2^40.
  const long long bh = static_cast<long long>(B) * Hq;
  if (bh > (1LL << 30)) return FA_ERR_UNSUPPORTED;
  if (bh * N * d >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

int check_decode_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || Nq > Nk) return FA_ERR_INVALID_ARGUMENT;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0) return FA_ERR_UNSUPPORTED;
  // Query rows per KV head and (batch, KV head) pairs stay TMA coordinates;
  // element counts of the query and cache tensors stay below 2^40.
  const long long rows = static_cast<long long>(Hq / Hkv) * Nq;
  const long long bkv = static_cast<long long>(B) * Hkv;
  if (rows > (1LL << 30) || bkv > (1LL << 30)) return FA_ERR_UNSUPPORTED;
  if (bkv * rows * d >= (1LL << 40) || bkv * Nk * d >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

LaunchCtl make_ctl(const DevState* st) {
  LaunchCtl c;
  c.err = st->err;
  c.budget_ns = g_budget_ns.load(std::memory_order_relaxed);
  c.fault = g_fault.load(std::memory_order_relaxed);
  c.ev_after_pre = static_cast<cudaEvent_t>(g_ev_pre.load(std::memory_order_relaxed));
  c.ev_after_main = static_cast<cudaEvent_t>(g_ev_main.load(std::memory_order_relaxed));
  return c;
}

}  // namespace

int check_current_device() {
  DevState* st = nullptr;
  return device_state(&st);
}

int record_cuda_error(cudaError_t e) { return record_cuda(e); }

namespace {
bool encode_map(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, int cols, int rows,
                int outer, int box_cols, int box_rows) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * elem_bytes,
                           static_cast<cuuint64_t>(cols) * elem_bytes * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

bool encode_tile_map(CUtensorMap* map, const void* base, int cols, int rows, int outer, int box_rows) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, cols, rows, outer, 64, box_rows);
}

bool encode_f32_tile_map(CUtensorMap* map, const void* base, int cols, int rows, int outer, int box_cols,
                         int box_rows) {
  if (box_cols * 4 > 128) return false;
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, cols, rows, outer, box_cols, box_rows);
}

}  // namespace fa

using namespace fa;

extern "C" {

static int fwd_impl(const void* q, const void* k, const void* v, void* o, void* o_resid, float* lse, int B,
                    int Hq, int Hkv, int N, int d, int causal, float scale, void* stream, int window = -1,
                    int prefix = 0) {
  if (window < -1 || prefix < 0) return FA_ERR_INVALID_ARGUMENT;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(o_resid))
    return FA_ERR_INVALID_ARGUMENT;
  int rc = check_shape(B, Hq, Hkv, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  DevState* st = nullptr;
  if ((rc = device_state(&st)) != FA_OK) return rc;
  CUtensorMap tq, tk, tv, to, tr;
  if (!encode_tile_map(&tq, q, d, N, B * Hq, 128) || !encode_tile_map(&tk, k, d, N, B * Hkv, 128) ||
      !encode_tile_map(&tv, v, d, N, B * Hkv, 128) || !encode_tile_map(&to, o, d, N, B * Hq, 128) ||
      !encode_tile_map(&tr, o_resid ? o_resid : o, d, N, B * Hq, 128))
    return FA_ERR_UNSUPPORTED;
  AttnShape s{B, Hq, Hkv, N, d, causal, scale};
  s.window = window;
  s.prefix = prefix;
  cudaError_t e =
      launch_fwd(s, tq, tk, tv, to, tr, o, o_resid, lse, make_ctl(st), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
           int d, int causal, float scale, void* stream) {
  return fwd_impl(q, k, v, o, nullptr, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

int fa_fwd_with_residual(const void* q, const void* k, const void* v, void* o, void* o_resid, float* lse, int B,
                         int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  if (!o_resid) return FA_ERR_INVALID_ARGUMENT;
  return fwd_impl(q, k, v, o, o_resid, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  if (check_shape(B, Hq, Hkv, N, d, 0, 1.f) != FA_OK) return 0;
  AttnShape s{B, Hq, Hkv, N, d, 0, 1.f};
  return bwd_workspace_bytes(s);
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                    int d, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream,
                    int window = -1, int prefix = 0) {
  if (window < -1 || prefix < 0) return FA_ERR_INVALID_ARGUMENT;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {q, k, v, o, o_resid, dout, lse, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_INVALID_ARGUMENT;
  int rc = check_shape(B, Hq, Hkv, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  AttnShape s{B, Hq, Hkv, N, d, causal, scale};
  s.window = window;
  s.prefix = prefix;
  if (workspace_bytes < bwd_workspace_bytes(s)) return FA_ERR_INVALID_ARGUMENT;
  DevState* st = nullptr;
  if ((rc = device_state(&st)) != FA_OK) return rc;
  // The backward streams 64-row query tiles past 128-row key tiles.
  CUtensorMap tq, tk, tv, tdo, tdk, tdv;
  if (!encode_tile_map(&tq, q, d, N, B * Hq, 64) || !encode_tile_map(&tk, k, d, N, B * Hkv, 128) ||
      !encode_tile_map(&tv, v, d, N, B * Hkv, 128) || !encode_tile_map(&tdo, dout, d, N, B * Hq, 64) ||
      !encode_tile_map(&tdk, dk, d, N, B * Hkv, 128) || !encode_tile_map(&tdv, dv, d, N, B * Hkv, 128))
    return FA_ERR_UNSUPPORTED;
  cudaError_t e = launch_bwd(s, tq, tk, tv, tdo, tdk, tdv, o, o_resid, dout, lse, dq, dk, dv, workspace, make_ctl(st),
                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
           void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, nullptr, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, workspace,
                  workspace_bytes, stream);
}

int fa_bwd_with_residual(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                         int N, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (!o_resid) return FA_ERR_INVALID_ARGUMENT;
  return bwd_impl(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale, workspace,
                  workspace_bytes, stream);
}

int fa_fwd_masked(const void* q, const void* k, const void* v, void* o, void* o_resid, float* lse, int B, int Hq,
                  int Hkv, int N, int d, int window, int prefix, float scale, void* stream) {
  return fwd_impl(q, k, v, o, o_resid, lse, B, Hq, Hkv, N, d, 1, scale, stream, window, prefix);
}

int fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* o_resid, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int window,
                  int prefix, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, 1, scale, workspace,
                  workspace_bytes, stream, window, prefix);
}

int fa_quantize_fp8(const void* x, void* codes, float* scales, int BH, int N, int d, int per_head, void* stream) {
  if (!x || !codes || !scales) return FA_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FA_ERR_INVALID_ARGUMENT;
  if (BH <= 0 || N <= 0 || (per_head != 0 && per_head != 1)) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(BH) * N * d >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
  DevState* st = nullptr;
  int rc = device_state(&st);
  if (rc != FA_OK) return rc;
  cudaError_t e = launch_quantize_fp8(x, codes, scales, BH, N, d, per_head, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

int fa_fwd_fp8(const void* q8, const float* sq, const void* k8, const float* sk, const void* v8, const float* sv,
               void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream) {
  if (!q8 || !sq || !k8 || !sk || !v8 || !sv || !o || !lse) return FA_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {q8, k8, v8, o, lse};
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_INVALID_ARGUMENT;
  const void* sptrs[] = {sq, sk, sv};
  for (const void* p : sptrs)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return FA_ERR_INVALID_ARGUMENT;
  int rc = check_shape(B, Hq, Hkv, N, d, causal, scale);
  if (rc != FA_OK) return rc;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  DevState* st = nullptr;
  if ((rc = device_state(&st)) != FA_OK) return rc;
  // e4m3 tensors: 128 one-byte columns per row, boxes of 128 columns x 128 rows.
  CUtensorMap tq, tk, tv, to;
  if (!encode_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q8, d, N, B * Hq, 128, 128) ||
      !encode_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k8, d, N, B * Hkv, 128, 128) ||
      !encode_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v8, d, N, B * Hkv, 128, 128) ||
      !encode_tile_map(&to, o, d, N, B * Hq, 128))
    return FA_ERR_UNSUPPORTED;
  AttnShape s{B, Hq, Hkv, N, d, causal, scale};
  cudaError_t e =
      launch_fwd_fp8(s, tq, tk, tv, to, o, lse, sq, sk, sv, make_ctl(st), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  if (check_decode_shape(B, Hq, Hkv, Nq, Nk, d, 0, 1.f) != FA_OK) return 0;
  DecodeShape s{B, Hq, Hkv, Nq, Nk, d, 0, 1.f};
  return decode_workspace_bytes(s);
}

int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
              int Nk, int d, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARGUMENT;
  const void* ptrs[] = {q, k, v, o, lse, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_INVALID_ARGUMENT;
  int rc = check_decode_shape(B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (rc != FA_OK) return rc;
  DecodeShape s{B, Hq, Hkv, Nq, Nk, d, causal, scale};
  if (workspace_bytes < decode_workspace_bytes(s)) return FA_ERR_INVALID_ARGUMENT;
  DevState* st = nullptr;
  if ((rc = device_state(&st)) != FA_OK) return rc;
  const DecodePlan plan = make_decode_plan(s, st->sms);
  // The partials of this plan must fit the shape's workspace bound.
  if (static_cast<long long>(plan.G) * plan.MS > plan.W / plan.T + 2LL * plan.G) return FA_ERR_UNSUPPORTED;
  // Queries as [B*Hkv][R][d] (the query heads of a KV head are adjacent),
  // boxes of one row chunk; K and V as [B*Hkv][Nk][d], boxes of 128 keys.
  CUtensorMap tq, tk, tv;
  if (!encode_tile_map(&tq, q, d, plan.R, B * Hkv, 128 / plan.rho) || !encode_tile_map(&tk, k, d, Nk, B * Hkv, 128) ||
      !encode_tile_map(&tv, v, d, Nk, B * Hkv, 128))
    return FA_ERR_UNSUPPORTED;
  LaunchCtl ctl = make_ctl(st);
  ctl.ev_after_pre = nullptr;
  ctl.ev_after_main = static_cast<cudaEvent_t>(g_ev_dec.load(std::memory_order_relaxed));
  cudaError_t e = launch_decode(s, plan, tq, tk, tv, o, lse, workspace, ctl, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK:
      return "ok";
    case FA_ERR_INVALID_ARGUMENT:
      return "invalid argument (null or misaligned pointer, non-positive size, bad causal flag, "
             "non-finite or non-positive scale, or workspace too small)";
    case FA_ERR_UNSUPPORTED:
      return "unsupported (head dim not 64/128, Hq not a multiple of Hkv, size limit, or device is not "
             "compute capability 10.0)";
    case FA_ERR_CUDA:
      return t_cuda_msg;
    case FA_ERR_TIMEOUT:
      return "a kernel wait ran past the watchdog budget and the kernel gave up";
    default:
      return "unknown status";
  }
}

int fa_check_device_error(void* stream) {
  DevState* st = nullptr;
  int rc = device_state(&st);
  if (rc != FA_OK) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return record_cuda(e);
  unsigned int word = 0;
  e = cudaMemcpy(&word, st->err, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return record_cuda(e);
  if (word == 0) return FA_OK;
  e = cudaMemset(st->err, 0, sizeof(word));
  if (e != cudaSuccess) return record_cuda(e);
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return record_cuda(e);
  return FA_ERR_TIMEOUT;
}

void fa_set_watchdog_ns(uint64_t ns) { g_budget_ns.store(ns < 1000000ull ? 1000000ull : ns); }

// Test hook, declared in include/fa_test.h: selects a deliberate stall
// (1 = the forward producer never loads the first K tile) so that the
// watchdog path can be exercised without faulting the GPU.
void fa_test_set_fault(int code) { g_fault.store(code); }

int fa_test_exp2(const float* x, float* y_poly, float* y_ex2, int n, void* stream) {
  if (!x || !y_poly || !y_ex2 || n < 0) return FA_ERR_INVALID_ARGUMENT;
  if (n == 0) return FA_OK;
  const int blocks = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  test_exp2_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_ex2, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

int fa_test_exp2_accurate(const float* x, float* y, int n, void* stream) {
  if (!x || !y || n < 0) return FA_ERR_INVALID_ARGUMENT;
  if (n == 0) return FA_OK;
  const int blocks = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  test_exp2_accurate_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : record_cuda(e);
}

int fa_test_decode_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas, long long* out) {
  if (!out || num_ctas < 1) return FA_ERR_INVALID_ARGUMENT;
  const int rc = check_decode_shape(B, Hq, Hkv, Nq, Nk, d, 0, 1.f);
  if (rc != FA_OK) return rc;
  const DecodeShape s{B, Hq, Hkv, Nq, Nk, d, 0, 1.f};
  const DecodePlan p = make_decode_plan(s, num_ctas);
  const long long v[8] = {p.W, p.T, p.G, p.MS, p.R, p.rho, p.rv, p.n_chunks};
  for (int i = 0; i < 8; ++i) out[i] = v[i];
  return FA_OK;
}

void fa_profile_set_decode_event(void* after_main) { g_ev_dec.store(after_main); }

void fa_profile_set_bwd_events(void* after_pre, void* after_main) {
  g_ev_pre.store(after_pre);
  g_ev_main.store(after_main);
}

}  // extern "C"
