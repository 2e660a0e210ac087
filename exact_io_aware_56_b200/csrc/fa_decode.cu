// Decode / short-query attention for sm_100a: Nq new queries per head
// against an Nk-key cache (Nq <= Nk), the queries sitting at the last Nq
// positions (bottom-right alignment when causal).
//
// Where the prefill is bound by tensor cores and the exponential unit, the
// decode loop reads the whole KV cache for a handful of queries and is
// bound by HBM bandwidth (FlashAttention: IO-aware exact attention,
// "PREFILL PATH" diagram, the decode loop "bound by KV-cache bandwidth";
// "Two notes"). The design therefore aims at streaming K and V once, at
// full bandwidth, from every SM:
//
// * Work: a unit is (batch, KV head, chunk of <= 128 query rows). All
//   query heads of a KV head share its K/V stream: the unit's rows are the
//   R = (Hq/Hkv) * Nq rows [B][Hkv][R][d] of the query tensor. The units'
//   key tiles (128 keys each) are concatenated and cut into G = #SM equal
//   contiguous runs ("stream-K"): one CTA per SM, one wave, no tail. A CTA
//   whose run crosses unit boundaries processes it as segments; each
//   segment leaves a partial (O / l, logsumexp) for its unit, and a second
//   kernel merges a unit's partials by their logsumexp
//   (O = sum_s e^(L_s - L) O_s, L = log sum_s e^(L_s)).
// * Rows: the unit's RB = 128 / RHO rows are replicated RHO times over the
//   128 tensor-memory lanes (RHO = 4 when R <= 32, 2 when R <= 64, else 1).
//   Copy c runs its own online softmax over key columns
//   [c * 128/RHO, (c+1) * 128/RHO) of every tile, so the exponentials of a
//   tile spread over all four softmax warps without any cross-lane
//   reduction; the copies are merged like split partials. The S MMA then
//   computes RHO times more scores than needed, which costs nothing that
//   matters here: the tensor pipe is far from busy in an HBM-bound loop.
//
// Warp roles (192 threads):
//   warps 0-3  softmax, one thread per tensor-memory lane (Q slot).
//   warp 4     TMA producer: K_j / V_j into a ring of stages, Q per segment.
//   warp 5     tensor-memory owner and MMA issuer (one thread):
//              S = Q K_j^T (both in shared memory), O += P V_j (P in TMEM).
//
// Tensor memory (512 columns allocated):
//   [0,128) S | [128,192) P (bf16 pairs) | [192,192+D) O_0 | [192+D,192+2D) O_1
// Copy c writes P only at its own 128/RHO key columns; the rest of its
// lanes' P columns hold zeros written once at start, so P V sums exactly
// the copy's keys. Two O buffers let the epilogue of one segment overlap
// the next segment's MMAs.
//
// Per tile the MMA thread issues S_j, waits for P_j, issues P_j V_j, so
// S_(j+1) is issued after P_j V_j; tcgen05 operations complete in issue
// order, hence once S_(j+1) is complete O holds every earlier product and
// the softmax may rescale it in place (same argument as the forward).

#include <cuda_bf16.h>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kT = 128;  // keys per K/V tile = tensor-memory lanes = Q slots
constexpr int kDecThreads = 192;
constexpr int kDecProducer = 4;
constexpr int kDecMma = 5;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColO = 192;

template <int D>
struct DecCfg {
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kQBufs = (D == 128) ? 1 : 2;
  static constexpr int kBoxBytes = kT * 128;  // 128 rows x 64 bf16 columns
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxBytes * kBoxes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBufs * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kColO + 2 * D <= kTmemCols, "tensor memory budget");
};

struct DecArgs {
  float* part_o;  // [G * MS][RHO * RV][D] partial O / l
  float* part_l;  // [G * MS][RHO * RV]    partial logsumexp (natural log, -inf if no key)
  int Nq, Nk, R, n_chunks, causal;
  DecodePlan plan;
  float scale_log2;
  LaunchCtl ctl;
};

struct DecBars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[6], v_full[6], kv_empty[6];
  uint64_t s_full, p_ready;
  uint64_t o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// The j-th segment of this CTA's run: unit u, tiles [j0, j1) of the unit.
struct Segment {
  int u, j0, j1;
};

__device__ __forceinline__ Segment segment_of(const DecodePlan& p, long long t_lo, long long t_hi, int e) {
  const long long u = t_lo / p.T + e;
  const long long a = max(t_lo, u * p.T), b = min(t_hi, (u + 1) * p.T);
  return Segment{static_cast<int>(u), static_cast<int>(a - u * p.T), static_cast<int>(b - u * p.T)};
}

template <int D, int RHO>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const DecArgs a) {
  using C = DecCfg<D>;
  constexpr int ST = C::kStages;
  constexpr int QB = C::kQBufs;
  constexpr int RB = kT / RHO;  // rows per unit chunk
  constexpr int CW = kT / RHO;  // key columns per copy
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  DecBars* bars = reinterpret_cast<DecBars*>(smem + C::kOffBar);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const DecodePlan& P = a.plan;
  const long long t_lo = P.lo(blockIdx.x), t_hi = P.lo(blockIdx.x + 1);
  const int n_seg = static_cast<int>((t_hi - 1) / P.T - t_lo / P.T) + 1;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->q_full[b], 1);
      mbar_init(&bars->q_empty[b], 1);
      mbar_init(&bars->o_full[b], 1);
      mbar_init(&bars->o_empty[b], kT);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_ready, kT);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kDecMma) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const Watch w{&bars->abort, a.ctl.err, a.ctl.budget_ns};

  if (warp == kDecProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int k_last[ST], q_last[2] = {-1, -1};
#pragma unroll
      for (int s = 0; s < ST; ++s) k_last[s] = -1;
      int g = 0;  // tile counter of this CTA
      bool ok = true;
      for (int e = 0; ok && e < n_seg; ++e) {
        const Segment sg = segment_of(P, t_lo, t_hi, e);
        const int bkv = sg.u / a.n_chunks;
        const int chunk = sg.u - bkv * a.n_chunks;
        for (int j = sg.j0; j < sg.j1; ++j, ++g) {
          const int s = g % ST;
          const int use = g / ST;
          if (g >= ST && !(ok = wait_bar(&bars->kv_empty[s], (use - 1) & 1, w))) break;
          mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
#pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(&tmK, &bars->k_full[s], smem + C::kOffK + s * C::kTileBytes + x * C::kBoxBytes, x * 64,
                        j * kT, bkv);
          mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
#pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(&tmV, &bars->v_full[s], smem + C::kOffV + s * C::kTileBytes + x * C::kBoxBytes, x * 64,
                        j * kT, bkv);
          k_last[s] = use;
          if (j == sg.j0) {
            // The segment's Q, after its first K/V tile is on its way: RHO
            // copies of the chunk's RB rows fill the 128 slots.
            const int qb = e % QB;
            if (e >= QB && !(ok = wait_bar(&bars->q_empty[qb], ((e / QB) - 1) & 1, w))) break;
            mbar_arrive_expect_tx(&bars->q_full[qb], C::kTileBytes);
#pragma unroll
            for (int x = 0; x < C::kBoxes; ++x)
#pragma unroll
              for (int c = 0; c < RHO; ++c)
                tma_load_3d(&tmQ, &bars->q_full[qb],
                            smem + C::kOffQ + qb * C::kTileBytes + x * C::kBoxBytes + c * RB * 128, x * 64,
                            chunk * RB, bkv);
            q_last[qb] = e / QB;
          }
        }
      }
      // Every copy issued must land before the CTA may exit.
      for (int b = 0; b < QB; ++b)
        if (q_last[b] >= 0) drain_bar(&bars->q_full[b], q_last[b] & 1, w);
#pragma unroll
      for (int s = 0; s < ST; ++s)
        if (k_last[s] >= 0) {
          drain_bar(&bars->k_full[s], k_last[s] & 1, w);
          drain_bar(&bars->v_full[s], k_last[s] & 1, w);
        }
    }
  } else if (warp == kDecMma) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(kT, kT, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(kT, D, false, true);
      const uint32_t sQ = smem_u32(smem + C::kOffQ);
      const uint32_t sK = smem_u32(smem + C::kOffK);
      const uint32_t sV = smem_u32(smem + C::kOffV);
      int g = 0;
      bool ok = true;
      for (int e = 0; ok && e < n_seg; ++e) {
        const Segment sg = segment_of(P, t_lo, t_hi, e);
        const int qb = e % QB, ob = e & 1;
        const uint32_t tO = tmem + kColO + ob * D;
        if (!(ok = wait_bar(&bars->q_full[qb], (e / QB) & 1, w))) break;
        if (e >= 2 && !(ok = wait_bar(&bars->o_empty[ob], ((e >> 1) - 1) & 1, w))) break;
        for (int j = sg.j0; j < sg.j1; ++j, ++g) {
          const int s = g % ST;
          const uint32_t par = (g / ST) & 1;
          if (!(ok = wait_bar(&bars->k_full[s], par, w))) break;
          tc_fence_after();
          const uint32_t qa = sQ + qb * C::kTileBytes;
          const uint32_t ka = sK + s * C::kTileBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * C::kBoxBytes + (k % 4) * 32;
            mma_ss(tmem, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), idesc_qk, k > 0);
          }
          mma_commit(&bars->s_full);
          if (!(ok = wait_bar(&bars->p_ready, g & 1, w) && wait_bar(&bars->v_full[s], par, w))) break;
          tc_fence_after();
          const uint32_t va = sV + s * C::kTileBytes;
#pragma unroll
          for (int k = 0; k < kT / 16; ++k)
            mma_ts(tO, tmem + kColP + k * 8, sdesc_sw128(va + k * 2048, C::kBoxBytes, 1024), idesc_pv,
                   (j > sg.j0 || k > 0) ? 1u : 0u);
          mma_commit(&bars->kv_empty[s]);
        }
        if (!ok) break;
        mma_commit(&bars->o_full[ob]);
        mma_commit(&bars->q_empty[qb]);
      }
      // All MMAs issued by this thread must finish before tensor memory is freed.
      mma_commit(&bars->drain);
      drain_bar(&bars->drain, 0, w);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int slot = warp * 32 + lane;  // tensor-memory lane = Q slot
    const int cp = slot / RB;           // copy: key columns [cp*CW, cp*CW + CW) of each tile
    const int rr = slot - cp * RB;      // row within the chunk
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off;
    const uint32_t tP = tmem + lane_off + kColP;
    const float sl2 = a.scale_log2;
    if (RHO > 1) {
      // P columns of the other copies stay zero for the whole kernel.
      uint32_t z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st16(tP + c * 16, z);
      tmem_st_wait();
    }
    const int RV = min(RB, a.R);
    int g = 0;
    bool ok = true;
    for (int e = 0; ok && e < n_seg; ++e) {
      const Segment sg = segment_of(P, t_lo, t_hi, e);
      const int ob = e & 1;
      const uint32_t tO = tmem + lane_off + kColO + ob * D;
      const int chunk = sg.u % a.n_chunks;
      const int grow = chunk * RB + rr;  // row within the KV head's R rows
      const bool valid = rr < RV && grow < a.R;
      // Last visible key of this row.
      const int pos = a.causal ? a.Nk - a.Nq + (grow % a.Nq) : a.Nk - 1;
      float m = -CUDART_INF_F;
      float l = 0.f;
      for (int j = sg.j0; j < sg.j1; ++j, ++g) {
        ok = __all_sync(0xffffffffu, wait_bar(&bars->s_full, g & 1, w));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[CW];
        if constexpr (CW == 128) {
          tmem_ld128(tS, sr);
        } else {
#pragma unroll
          for (int c = 0; c < CW / 32; ++c) {
            uint32_t t32[32];
            tmem_ld32(tS + cp * CW + c * 32, t32);
#pragma unroll
            for (int i = 0; i < 32; ++i) sr[c * 32 + i] = t32[i];
          }
        }
        const int k0 = j * kT + cp * CW;
        if (k0 + CW - 1 > pos) {
#pragma unroll
          for (int i = 0; i < CW; ++i)
            if (k0 + i > pos) sr[i] = __float_as_uint(-CUDART_INF_F);
        }
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = fmaxf(__uint_as_float(sr[u]), __uint_as_float(sr[8 + u]));
#pragma unroll
        for (int i = 16; i < CW; i += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            pm[u] = fmax3(pm[u], __uint_as_float(sr[i + u]), __uint_as_float(sr[i + 8 + u]));
        pm[0] = fmax3(pm[0], pm[1], pm[2]);
        pm[3] = fmax3(pm[3], pm[4], pm[5]);
        pm[6] = fmaxf(pm[6], pm[7]);
        const float m_cand = fmax3(pm[0], pm[3], pm[6]) * sl2;
        bool rescale = false;
        float alpha = 1.f;
        if (j == sg.j0) {
          m = m_cand;
        } else if (__any_sync(0xffffffffu, m_cand > m)) {
          const float m_new = fmaxf(m, m_cand);
          alpha = (m_new == -CUDART_INF_F) ? 1.f : ex2(m - m_new);
          m = m_new;
          l *= alpha;
          rescale = true;
        }
        // A row with no visible key so far keeps m = -inf; its masked
        // scores must give exp(-inf) = 0, not exp(-inf + inf).
        const float neg_m = (m == -CUDART_INF_F) ? 0.f : -m;
        float ps[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) ps[u] = 0.f;
#pragma unroll
        for (int c = 0; c < CW / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2(fmaf(__uint_as_float(sr[c * 32 + 2 * i]), sl2, neg_m));
            const float p1 = ex2(fmaf(__uint_as_float(sr[c * 32 + 2 * i + 1]), sl2, neg_m));
            ps[(2 * i) & 7] += p0;
            ps[(2 * i + 1) & 7] += p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tP + cp * (CW / 2) + c * 16, pk);
        }
        const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        if (rescale) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o32[32];
            tmem_ld32(tO + c * 32, o32);
#pragma unroll
            for (int i = 0; i < 32; ++i) o32[i] = __float_as_uint(__uint_as_float(o32[i]) * alpha);
            tmem_st32(tO + c * 32, o32);
          }
        }
        l += sum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar(&bars->o_full[ob], (e >> 1) & 1, w));
      if (!ok) break;
      tc_fence_after();
      // Partial of this copy: O / l and logsumexp, or zeros and -inf when
      // no key of the segment is visible to the row.
      const long long pidx = static_cast<long long>(blockIdx.x) * P.MS + e;
      const long long prow = (pidx * RHO + cp) * RV + rr;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t oo[32];
        tmem_ld32(tO + c * 32, oo);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(a.part_o + prow * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(oo[4 * i]) * inv_l, __uint_as_float(oo[4 * i + 1]) * inv_l,
                                 __uint_as_float(oo[4 * i + 2]) * inv_l, __uint_as_float(oo[4 * i + 3]) * inv_l);
        }
      }
      if (valid) a.part_l[prow] = l > 0.f ? (m + lg2(l)) * 0.69314718055994530942f : -CUDART_INF_F;
      tc_fence_before();
      mbar_arrive(&bars->o_empty[ob]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDecMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Merges each row's partials (every copy of every segment of its unit):
// one warp per query row, lanes across the head dimension.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_l,
                                                             __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                             const DecodePlan plan, int rows, int R, int rb,
                                                             int rho, int n_chunks) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;  // = bkv * R + grow
  if (row >= rows) return;
  const int bkv = static_cast<int>(row / R);
  const int grow = static_cast<int>(row - static_cast<long long>(bkv) * R);
  const int chunk = grow / rb;
  const int rr = grow - chunk * rb;
  const int rv = min(rb, R);
  const long long u = static_cast<long long>(bkv) * n_chunks + chunk;
  const int c0 = plan.cta_of(u * plan.T);
  const int c1 = plan.cta_of(u * plan.T + plan.T - 1);
  float mx = -CUDART_INF_F;
  for (int c = c0; c <= c1; ++c) {
    const long long pidx = static_cast<long long>(c) * plan.MS + (u - plan.lo(c) / plan.T);
    for (int cp = 0; cp < rho; ++cp) mx = fmaxf(mx, part_l[(pidx * rho + cp) * rv + rr]);
  }
  float den = 0.f;
  for (int c = c0; c <= c1; ++c) {
    const long long pidx = static_cast<long long>(c) * plan.MS + (u - plan.lo(c) / plan.T);
    for (int cp = 0; cp < rho; ++cp) den += expf(part_l[(pidx * rho + cp) * rv + rr] - mx);
  }
  const float L = mx + logf(den);
  float acc[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) acc[i] = 0.f;
  for (int c = c0; c <= c1; ++c) {
    const long long pidx = static_cast<long long>(c) * plan.MS + (u - plan.lo(c) / plan.T);
    for (int cp = 0; cp < rho; ++cp) {
      const long long prow = (pidx * rho + cp) * rv + rr;
      const float wgt = expf(part_l[prow] - L);
      if (wgt == 0.f) continue;  // also skips rows of segments without a visible key
#pragma unroll
      for (int i = 0; i < D / 32; ++i) acc[i] = fmaf(wgt, part_o[prow * D + i * 32 + lane], acc[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < D / 32; ++i) o[row * D + i * 32 + lane] = __float2bfloat16_rn(acc[i]);
  if (lane == 0) lse[row] = L;
}

template <int D, int RHO>
cudaError_t launch_decode_t(const DecodeShape& s, const DecodePlan& plan, const CUtensorMap& tq,
                            const CUtensorMap& tk, const CUtensorMap& tv, void* o, float* lse, void* workspace,
                            const LaunchCtl& ctl, cudaStream_t stream) {
  using C = DecCfg<D>;
  auto kern = decode_kernel<D, RHO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  DecArgs a;
  const long long parts = static_cast<long long>(plan.G) * plan.MS * plan.rho * plan.rv;
  a.part_o = static_cast<float*>(workspace);
  a.part_l = a.part_o + parts * D;
  a.Nq = s.Nq;
  a.Nk = s.Nk;
  a.R = plan.R;
  a.n_chunks = plan.n_chunks;
  a.causal = s.causal;
  a.plan = plan;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.ctl = ctl;
  kern<<<plan.G, kDecThreads, C::kSmemBytes, stream>>>(tq, tk, tv, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long rows = static_cast<long long>(s.B) * s.Hkv * plan.R;
  decode_combine_kernel<D><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, stream>>>(
      a.part_o, a.part_l, static_cast<__nv_bfloat16*>(o), lse, plan, static_cast<int>(rows), plan.R, kT / RHO,
      RHO, plan.n_chunks);
  return cudaGetLastError();
}

}  // namespace

DecodePlan make_decode_plan(const DecodeShape& s, int num_ctas) {
  DecodePlan p{};
  p.R = (s.Hq / s.Hkv) * s.Nq;
  p.rho = p.R <= 32 ? 4 : (p.R <= 64 ? 2 : 1);
  const int rb = kT / p.rho;
  p.n_chunks = (p.R + rb - 1) / rb;
  p.rv = p.R < rb ? p.R : rb;
  p.T = (s.Nk + kT - 1) / kT;
  const long long units = static_cast<long long>(s.B) * s.Hkv * p.n_chunks;
  p.W = units * p.T;
  long long g = num_ctas < kDecodeMaxCtas ? num_ctas : kDecodeMaxCtas;
  if (g > p.W) g = p.W;
  if (g < 1) g = 1;
  p.G = static_cast<int>(g);
  const long long len = (p.W + p.G - 1) / p.G;
  p.MS = static_cast<int>((len + p.T - 1) / p.T) + 1;
  return p;
}

size_t decode_workspace_bytes(const DecodeShape& s) {
  const DecodePlan p = make_decode_plan(s, kDecodeMaxCtas);
  const long long units = p.W / p.T;
  const long long g = p.W < kDecodeMaxCtas ? p.W : kDecodeMaxCtas;
  const long long parts = (units + 2 * g) * p.rho * p.rv;
  return static_cast<size_t>(parts) * (s.d + 1) * sizeof(float);
}

cudaError_t launch_decode(const DecodeShape& s, const DecodePlan& plan, const CUtensorMap& tq,
                          const CUtensorMap& tk, const CUtensorMap& tv, void* o, float* lse, void* workspace,
                          const LaunchCtl& ctl, cudaStream_t stream) {
#define FA_DEC_ARGS s, plan, tq, tk, tv, o, lse, workspace, ctl, stream
  if (s.d == 64) {
    if (plan.rho == 4) return launch_decode_t<64, 4>(FA_DEC_ARGS);
    if (plan.rho == 2) return launch_decode_t<64, 2>(FA_DEC_ARGS);
    return launch_decode_t<64, 1>(FA_DEC_ARGS);
  }
  if (plan.rho == 4) return launch_decode_t<128, 4>(FA_DEC_ARGS);
  if (plan.rho == 2) return launch_decode_t<128, 2>(FA_DEC_ARGS);
  return launch_decode_t<128, 1>(FA_DEC_ARGS);
#undef FA_DEC_ARGS
}

}  // namespace fa
