// Internal interface between the C-ABI layer (fa_api.cpp) and the kernel
// launchers (fa_fwd.cu, fa_bwd.cu). Not installed, not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

struct AttnShape {
  int B, Hq, Hkv, N, d;
  int causal;
  float scale;
  int window = -1;  // left window of the causal mask, -1 = none
  int prefix = 0;   // keys below this index are visible to every query
  // 0: no mask; 1: causal; 2: causal with a window and/or a prefix
  // (key j visible to query i iff (j <= i and i - j <= window) or j < prefix).
  int mask_kind() const { return !causal ? 0 : (window < 0 && prefix == 0 ? 1 : 2); }
};

struct LaunchCtl {
  unsigned int* err;        // device error word (watchdog)
  uint64_t budget_ns;       // watchdog budget per wait
  int fault;                // test-only fault injection selector (0 = none)
  cudaEvent_t ev_after_pre;   // optional timing events (see fa_profile.h)
  cudaEvent_t ev_after_main;
};

// Number of heads to schedule together so that their per-head working set
// (`bytes_per_head`) stays within a share of L2 that the resident CTAs can
// keep hot; at least 1, at most `heads`.
inline int l2_head_group(long long bytes_per_head, int heads) {
  constexpr long long kBudget = 48ll << 20;
  long long g = bytes_per_head > 0 ? kBudget / bytes_per_head : heads;
  if (g < 1) g = 1;
  if (g > heads) g = heads;
  return static_cast<int>(g);
}

// Encodes a 3-D bf16 tensor map over [outer][rows][cols] with a box of
// 64 columns x box_rows rows and 128-byte swizzle. Returns false on failure.
bool encode_tile_map(CUtensorMap* map, const void* base, int cols, int rows, int outer, int box_rows);

// Same for an fp32 tensor, box of box_cols x box_rows (box_cols * 4 <= 128).
bool encode_f32_tile_map(CUtensorMap* map, const void* base, int cols, int rows, int outer, int box_cols,
                         int box_rows);

// Checks that the current device is supported (compute capability 10.0),
// once per device, as every entry point does before its first launch.
// Returns FA_OK or the entry points' error status.
int check_current_device();

// Keeps `e` as the message of FA_ERR_CUDA for fa_status_string and returns
// FA_ERR_CUDA.
int record_cuda_error(cudaError_t e);

// o_resid may be null (no residual written). to and tr are bf16 tensor maps
// of o and o_resid laid out like q (tr unused without a residual).
cudaError_t launch_fwd(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const CUtensorMap& tr, void* o, void* o_resid, float* lse,
                       const LaunchCtl& ctl, cudaStream_t stream);

// FP8 mode (d = 128, masks 0 and 1): q, k, v are e4m3 codes behind 1-byte
// tensor maps with 128-column boxes; sq, sk, sv the block scales; to the
// bf16 tensor map of o.
cudaError_t launch_fwd_fp8(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, void* o, float* lse, const float* sq, const float* sk,
                           const float* sv, const LaunchCtl& ctl, cudaStream_t stream);

// e4m3 block quantization of a bf16 tensor [BH][N][d]: scales per 128-row
// block ([BH][ceil(N/128)]) or per head ([BH]); see fa.h.
cudaError_t launch_quantize_fp8(const void* x, void* codes, float* scales, int BH, int N, int d, int per_head,
                                cudaStream_t stream);

size_t bwd_workspace_bytes(const AttnShape& s);

// tdk and tdv: bf16 tensor maps of dk and dv laid out like k (128-row boxes).
cudaError_t launch_bwd(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const void* o,
                       const void* o_resid, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       void* workspace, const LaunchCtl& ctl, cudaStream_t stream);

// Decode / short-query attention: Nq queries per head against an Nk-key
// cache, queries at the last Nq positions.
struct DecodeShape {
  int B, Hq, Hkv, Nq, Nk, d;
  int causal;
  float scale;
};

// At most this many CTAs run the decode kernel (one per SM up to here); the
// workspace bound below depends on it.
constexpr int kDecodeMaxCtas = 256;

// Stream-K partition of the decode work. Units are (batch, KV head, chunk of
// 128/rho query rows) with T key tiles of 128 keys each; the W = units * T
// tiles, in unit order, are cut into G contiguous runs of nearly equal
// length, run c being tiles [lo(c), lo(c+1)). A run touches at most MS units.
struct DecodePlan {
  long long W;
  int T, G, MS;
  int R;         // query rows per KV head: (Hq / Hkv) * Nq
  int rho;       // replication of the chunk's rows over the 128 lanes (4, 2 or 1)
  int rv;        // stored rows per copy and partial: min(128 / rho, R)
  int n_chunks;  // row chunks per KV head
  __host__ __device__ long long lo(long long c) const { return c * W / G; }
  // The run holding tile t: the largest c with lo(c) <= t.
  __host__ __device__ int cta_of(long long t) const { return static_cast<int>(((t + 1) * G + W - 1) / W) - 1; }
};

DecodePlan make_decode_plan(const DecodeShape& s, int num_ctas);

// Workspace for any plan of this shape with G <= kDecodeMaxCtas: partial O
// (fp32, d per row) and logsumexp for (units + 2 * G) partials of rho * rv rows
// (G * MS <= W / T + 2 G).
size_t decode_workspace_bytes(const DecodeShape& s);

cudaError_t launch_decode(const DecodeShape& s, const DecodePlan& plan, const CUtensorMap& tq,
                          const CUtensorMap& tk, const CUtensorMap& tv, void* o, float* lse, void* workspace,
                          const LaunchCtl& ctl, cudaStream_t stream);

}  // namespace fa
