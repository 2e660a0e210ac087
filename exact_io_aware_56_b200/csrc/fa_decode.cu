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
//   warp 5     tensor-memory owner and MMA issuer (the whole warp runs the
//              issue loop so descriptors stay warp-uniform; one elected lane
//              issues): S = Q K_j^T (both in shared memory), O += P V_j (P in
//              TMEM).
//
// Tensor memory (512 columns allocated):
//   [0,256) S_0, S_1 | [256,384) P_0, P_1 (bf16 pairs) | [384,...) O_0 (, O_1)
// S and P are double-buffered by tile parity, so S_(j+1) runs on the
// tensor pipe while the softmax turns S_j into P_j. Copy c writes P only
// at its own 128/RHO key columns; the rest of its lanes' P columns hold
// zeros written once at start, so P V sums exactly the copy's keys. With
// two O buffers (d = 64) the epilogue of one segment overlaps the next
// segment's MMAs.
//
// Ordering. The MMA thread issues, per tile j, S_(j+1) and then P_j V_j,
// so S_(j+1) follows P_(j-1) V_(j-1): once S_(j+1) is complete, the P
// buffer of parity j+1 is free again. O, however, may still be receiving
// P_j V_j while the softmax works on tile j+1, so a warp that must rescale
// O first waits for the pv_done phase of tile j (P_(j+1) V_(j+1) cannot
// start before this warp hands P_(j+1) back, so that phase is unambiguous).

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
constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 256;
constexpr uint32_t kColO = 384;

template <int D>
struct DecCfg {
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kQBufs = (D == 128) ? 1 : 2;
  static constexpr int kOBufs = (kColO + 2 * D <= 512) ? 2 : 1;
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
  static_assert(kColO + kOBufs * D <= kTmemCols, "tensor memory budget");
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
  uint64_t s_full[2], p_ready, pv_done;
  uint64_t o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(DecBars) <= 256, "barrier block exceeds its shared-memory reservation");

// Walks the tiles of this CTA's run [t_lo, t_hi) in order, tracking the
// unit u, its segment e (0 = the run's first unit) and tile j of the unit
// without dividing per tile.
struct TileCursor {
  long long t, t_hi;
  int T, u, e, j;
  __device__ __forceinline__ TileCursor(const DecodePlan& p, long long lo, long long hi) : t(lo), t_hi(hi), T(p.T) {
    const long long u0 = lo / p.T;
    u = static_cast<int>(u0);
    e = 0;
    j = static_cast<int>(lo - u0 * p.T);
  }
  __device__ __forceinline__ bool first(long long lo) const { return t == lo || j == 0; }
  __device__ __forceinline__ bool last() const { return t == t_hi - 1 || j == T - 1; }
  __device__ __forceinline__ void next() {
    ++t;
    if (++j == T) {
      j = 0;
      ++u;
      ++e;
    }
  }
};

template <int D, int RHO>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const DecArgs a) {
  using C = DecCfg<D>;
  constexpr int ST = C::kStages;
  constexpr int QB = C::kQBufs;
  constexpr int OB = C::kOBufs;
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

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->q_full[b], 1);
      mbar_init(&bars->q_empty[b], 1);
      mbar_init(&bars->o_full[b], 1);
      mbar_init(&bars->o_empty[b], kT);
      mbar_init(&bars->s_full[b], 1);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->p_ready, kT);
    mbar_init(&bars->pv_done, 1);
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
  // The merge kernel may be scheduled now; it waits for this grid's results.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;");

  if (warp == kDecProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int k_last[ST], q_last[2] = {-1, -1};
#pragma unroll
      for (int s = 0; s < ST; ++s) k_last[s] = -1;
      for (TileCursor ta(P, t_lo, t_hi); ta.t < t_hi; ta.next()) {
        const int g = static_cast<int>(ta.t - t_lo);
        const int s = g % ST;
        const int use = g / ST;
        const int bkv = ta.u / a.n_chunks;
        if (g >= ST && !wait_bar(&bars->kv_empty[s], (use - 1) & 1, w)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
#pragma unroll
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(&tmK, &bars->k_full[s], smem + C::kOffK + s * C::kTileBytes + x * C::kBoxBytes, x * 64,
                      ta.j * kT, bkv);
        mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
#pragma unroll
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(&tmV, &bars->v_full[s], smem + C::kOffV + s * C::kTileBytes + x * C::kBoxBytes, x * 64,
                      ta.j * kT, bkv);
        k_last[s] = use;
        if (ta.first(t_lo)) {
          // The segment's Q, after its first K/V tile is on its way: RHO
          // copies of the chunk's RB rows fill the 128 slots.
          const int qb = ta.e % QB;
          const int chunk = ta.u - bkv * a.n_chunks;
          if (ta.e >= QB && !wait_bar(&bars->q_empty[qb], ((ta.e / QB) - 1) & 1, w)) break;
          mbar_arrive_expect_tx(&bars->q_full[qb], C::kTileBytes);
#pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
#pragma unroll
            for (int c = 0; c < RHO; ++c)
              tma_load_3d(&tmQ, &bars->q_full[qb], smem + C::kOffQ + qb * C::kTileBytes + x * C::kBoxBytes + c * RB * 128,
                          x * 64, chunk * RB, bkv);
          q_last[qb] = ta.e / QB;
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
    // The whole warp runs this loop (descriptors stay warp-uniform); the
    // elected lane issues the tcgen05 instructions.
    const bool leader = elect_one();
    auto all = [](bool b) { return __all_sync(0xffffffffu, b); };
    {
      constexpr uint32_t idesc_qk = idesc_bf16(kT, kT, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16(kT, D, false, true);
      // Operand descriptors computed once and stepped by byte offsets.
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + C::kOffQ), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(smem + C::kOffK), 16, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(smem + C::kOffV), C::kBoxBytes, 1024);
      auto ofs_kmaj = [](int k) { return static_cast<uint32_t>((k / 4) * C::kBoxBytes + (k % 4) * 32); };
      // S_t = Q K_t^T into S buffer (t - t_lo) & 1.
      auto issue_s = [&](const TileCursor& ta) -> bool {
        const int g = static_cast<int>(ta.t - t_lo);
        const int s = g % ST;
        const int qb = ta.e % QB;
        if (ta.first(t_lo) && !all(wait_bar(&bars->q_full[qb], (ta.e / QB) & 1, w))) return false;
        if (!all(wait_bar(&bars->k_full[s], (g / ST) & 1, w))) return false;
        tc_fence_after();
        const uint64_t qa = sdesc_step(dQ, qb * C::kTileBytes);
        const uint64_t ka = sdesc_step(dK, s * C::kTileBytes);
        const uint32_t d_s = tmem + kColS + (g & 1) * kT;
#pragma unroll
        for (int k = 0; k < D / 16; k += 4)
          mma_ss_x4(d_s, sdesc_step(qa, ofs_kmaj(k)), sdesc_step(qa, ofs_kmaj(k + 1)), sdesc_step(qa, ofs_kmaj(k + 2)),
                    sdesc_step(qa, ofs_kmaj(k + 3)), sdesc_step(ka, ofs_kmaj(k)), sdesc_step(ka, ofs_kmaj(k + 1)),
                    sdesc_step(ka, ofs_kmaj(k + 2)), sdesc_step(ka, ofs_kmaj(k + 3)), idesc_qk, k > 0, leader);
        mma_commit(&bars->s_full[g & 1], leader);
        if (ta.last()) mma_commit(&bars->q_empty[qb], leader);  // the segment's last read of its Q buffer
        return true;
      };
      // O += P_t V_t.
      auto issue_pv = [&](const TileCursor& ta) -> bool {
        const int g = static_cast<int>(ta.t - t_lo);
        const int s = g % ST;
        const int ob = ta.e % OB;
        if (!all(wait_bar(&bars->p_ready, g & 1, w)) || !all(wait_bar(&bars->v_full[s], (g / ST) & 1, w))) return false;
        const bool first = ta.first(t_lo);
        if (first && ta.e >= OB && !all(wait_bar(&bars->o_empty[ob], ((ta.e / OB) - 1) & 1, w))) return false;
        tc_fence_after();
        const uint64_t va = sdesc_step(dV, s * C::kTileBytes);
        const uint32_t d_o = tmem + kColO + ob * D;
        const uint32_t a_p = tmem + kColP + (g & 1) * 64;
#pragma unroll
        for (int k = 0; k < kT / 16; k += 4)
          mma_ts_x4(d_o, a_p + k * 8, a_p + (k + 1) * 8, a_p + (k + 2) * 8, a_p + (k + 3) * 8,
                    sdesc_step(va, k * 2048), sdesc_step(va, (k + 1) * 2048), sdesc_step(va, (k + 2) * 2048),
                    sdesc_step(va, (k + 3) * 2048), idesc_pv, (!first || k > 0) ? 1u : 0u, leader);
        mma_commit(&bars->kv_empty[s], leader);
        mma_commit(&bars->pv_done, leader);
        if (ta.last()) mma_commit(&bars->o_full[ob], leader);
        return true;
      };
      TileCursor cur(P, t_lo, t_hi), nxt(P, t_lo, t_hi);
      bool ok = issue_s(nxt);
      for (nxt.next(); ok && cur.t < t_hi; cur.next(), nxt.next()) {
        const bool more = nxt.t < t_hi;
        // With one Q buffer the next segment's Q lands only after this
        // segment's last S: hand P_t V_t to the tensor pipe before waiting.
        if (QB == 1 && more && nxt.first(t_lo)) {
          ok = issue_pv(cur) && issue_s(nxt);
        } else {
          ok = (!more || issue_s(nxt)) && issue_pv(cur);
        }
      }
      // All MMAs issued by this thread must finish before tensor memory is freed.
      mma_commit(&bars->drain, leader);
      all(drain_bar(&bars->drain, 0, w));
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int slot = warp * 32 + lane;  // tensor-memory lane = Q slot
    const int cp = slot / RB;           // copy: key columns [cp*CW, cp*CW + CW) of each tile
    const int rr = slot - cp * RB;      // row within the chunk
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    if (RHO > 1) {
      // P columns of the other copies stay zero for the whole kernel.
      uint32_t z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
      for (int c = 0; c < 8; ++c) tmem_st16(tmem + lane_off + kColP + c * 16, z);
      tmem_st_wait();
    }
    const int RV = min(RB, a.R);
    float m = -CUDART_INF_F;
    float l = 0.f;
    int pos = 0;
    bool valid = false;
    for (TileCursor ta(P, t_lo, t_hi); ta.t < t_hi; ta.next()) {
      const int g = static_cast<int>(ta.t - t_lo);
      const bool first = ta.first(t_lo);
      const int ob = ta.e % OB;
      const uint32_t tS = tmem + lane_off + kColS + (g & 1) * kT;
      const uint32_t tP = tmem + lane_off + kColP + (g & 1) * 64;
      const uint32_t tO = tmem + lane_off + kColO + ob * D;
      if (first) {
        const int chunk = ta.u % a.n_chunks;
        const int grow = chunk * RB + rr;  // row within the KV head's R rows
        valid = rr < RV && grow < a.R;
        pos = a.causal ? a.Nk - a.Nq + (grow % a.Nq) : a.Nk - 1;  // last visible key
        m = -CUDART_INF_F;
        l = 0.f;
      }
      if (!__all_sync(0xffffffffu, wait_bar(&bars->s_full[g & 1], (g >> 1) & 1, w))) break;
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
      const int k0 = ta.j * kT + cp * CW;
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
      if (first) {
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
          // Exponent arguments and partial sums two at a time (packed f32x2).
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(sr[c * 32 + 2 * i]), __uint_as_float(sr[c * 32 + 2 * i + 1]), sl2, sl2,
                neg_m, neg_m);
          const float p0 = ex2(x0);
          const float p1 = ex2(x1);
          fadd2(ps[(2 * i) & 7], ps[(2 * i + 1) & 7], ps[(2 * i) & 7], ps[(2 * i + 1) & 7], p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tP + cp * (CW / 2) + c * 16, pk);
      }
      const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      if (rescale) {
        // O may still be receiving the previous tile's product.
        if (!__all_sync(0xffffffffu, wait_bar(&bars->pv_done, (g - 1) & 1, w))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o32[32];
          tmem_ld32(tO + c * 32, o32);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float x0, x1;
            fmul2(x0, x1, __uint_as_float(o32[i]), __uint_as_float(o32[i + 1]), alpha, alpha);
            o32[i] = __float_as_uint(x0);
            o32[i + 1] = __float_as_uint(x1);
          }
          tmem_st32(tO + c * 32, o32);
        }
      }
      l += sum;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_ready);
      if (ta.last()) {
        if (!__all_sync(0xffffffffu, wait_bar(&bars->o_full[ob], (ta.e / OB) & 1, w))) break;
        tc_fence_after();
        // Partial of this copy: O / l and logsumexp, or zeros and -inf when
        // no key of the segment is visible to the row.
        const long long pidx = static_cast<long long>(blockIdx.x) * P.MS + ta.e;
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDecMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Loads 2 or 4 consecutive floats (8- or 16-byte aligned) into registers.
__device__ __forceinline__ void load_vec(const float* p, float (&x)[4]) {
  const float4 t = *reinterpret_cast<const float4*>(p);
  x[0] = t.x;
  x[1] = t.y;
  x[2] = t.z;
  x[3] = t.w;
}
__device__ __forceinline__ void load_vec(const float* p, float (&x)[2]) {
  const float2 t = *reinterpret_cast<const float2*>(p);
  x[0] = t.x;
  x[1] = t.y;
}

// Merges each row's partials (every copy of every segment of its unit):
// one warp per query row. Lanes first take one partial each for the max and
// the sum of e^(L_s - max); the weighted sum of the partial O rows then runs
// over the head dimension across lanes, four partials per step so their
// loads overlap. Launched as a programmatic dependent of the decode kernel:
// it may become resident early and waits for that grid's results here.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_l,
                                                             __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                             const DecodePlan plan, int rows, int R, int rb,
                                                             int rho, int n_chunks) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
  const int n_parts = (plan.cta_of(u * plan.T + plan.T - 1) - c0 + 1) * rho;
  // Partial p = (run c0 + p / rho, copy p % rho) -> its row in the workspace.
  auto prow_of = [&](int p) -> long long {
    const int c = c0 + p / rho;
    const long long pidx = static_cast<long long>(c) * plan.MS + (u - plan.lo(c) / plan.T);
    return (pidx * rho + p % rho) * rv + rr;
  };
  float mx = -CUDART_INF_F;
  for (int p = lane; p < n_parts; p += 32) mx = fmaxf(mx, part_l[prow_of(p)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float den = 0.f;
  for (int p = lane; p < n_parts; p += 32) den += expf(part_l[prow_of(p)] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  const float L = mx + logf(den);
  // Lane l owns columns [l * VW, (l + 1) * VW) of the row: one vector load
  // per partial, eight partials in flight per step.
  constexpr int VW = D / 32;
  float acc[VW];
#pragma unroll
  for (int i = 0; i < VW; ++i) acc[i] = 0.f;
  for (int base = 0; base < n_parts; base += 32) {
    // Lane i holds the weight and row of partial base + i (weight 0 past the
    // end, and for partials without a visible key, whose L is -inf).
    const int p = base + lane;
    float wl = 0.f;
    long long rl = 0;
    if (p < n_parts) {
      rl = prow_of(p);
      wl = expf(part_l[rl] - L);
    }
    const int n = min(32, n_parts - base);
    for (int i = 0; i < n; i += 8) {
      float wv[8], x[8][VW];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        wv[q] = __shfl_sync(0xffffffffu, wl, (i + q) & 31);
        const long long r = __shfl_sync(0xffffffffu, rl, (i + q) & 31);
        if (i + q < n && wv[q] != 0.f) {
          load_vec(part_o + r * D + lane * VW, x[q]);
        } else {
          wv[q] = 0.f;
#pragma unroll
          for (int k = 0; k < VW; ++k) x[q][k] = 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int k = 0; k < VW; ++k) acc[k] = fmaf(wv[q], x[q][k], acc[k]);
    }
  }
  uint32_t packed[VW / 2];
#pragma unroll
  for (int k = 0; k < VW / 2; ++k) packed[k] = pack_bf16x2(acc[2 * k], acc[2 * k + 1]);
  if constexpr (VW == 4) {
    *reinterpret_cast<uint2*>(o + row * D + lane * VW) = make_uint2(packed[0], packed[1]);
  } else {
    *reinterpret_cast<uint32_t*>(o + row * D + lane * VW) = packed[0];
  }
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
  if (ctl.ev_after_main && (e = cudaEventRecord(ctl.ev_after_main, stream)) != cudaSuccess) return e;
  const long long rows = static_cast<long long>(s.B) * s.Hkv * plan.R;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, static_cast<const float*>(a.part_o),
                            static_cast<const float*>(a.part_l), static_cast<__nv_bfloat16*>(o), lse, plan,
                            static_cast<int>(rows), plan.R, kT / RHO, RHO, plan.n_chunks);
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
