// Backward attention kernels for sm_100a.
//
// Gradients of sum(dO * O) for O = softmax(scale * Q K^T [causal]) V, with P
// rebuilt on chip from Q, K and the forward's row logsumexp L instead of
// being stored (FlashAttention: IO-aware exact attention, "Four ideas" list,
// item "Recomputation in the backward pass"; Flash Attention: memory-
// efficient transformers, "Recomputation in the Backward Pass"). The pages
// give no formulas; these are the gradient of the definition:
//   P = exp(scale S - L), dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij
//   (= sum_c dO_ic O_ic), dS = P o (dP - D), dQ = scale dS K,
//   dK = scale dS^T Q, KV heads summing over their query heads.
//
// Three kernels:
//   bwd_pre   D_i = sum_c dO_ic O_ic (fp32) and zero the fp32 dQ accumulator.
//             O is the bf16 o plus, when given, its rounding residual: D_i
//             multiplies every error of O by dO and sums it over d, and the
//             bf16 rounding of O alone moves D by ~1e-2 at d = 128.
//   bwd_main  one CTA per (batch, KV head, 128-key tile j). K_j and V_j stay in
//             shared memory; the CTA loops over the query heads of the KV
//             group and the 64-row query tiles i that can see tile j
//             (i >= 2j when causal). Per (head, i):
//               S^T  = K_j Q_i^T          (tcgen05 -> tensor memory, M=128 N=64)
//               dP^T = V_j dO_i^T         (tcgen05 -> tensor memory)
//               P^T  = 2^(S^T scale log2e - L_i log2e), dS^T = P^T o (dP^T - D_i)
//                                         (one thread per key row)
//               dV_j += P^T dO_i          (P^T read from tensor memory)
//               dK_j += dS^T Q_i          (dS^T read from tensor memory)
//               dQ_i^T = K_j^T dS_i^T     (M = d: one thread per column of dQ)
//             dQ_i is added to the fp32 accumulator by coalesced reductions
//             issued from registers, which overlap the next tiles.
//             dK_j (times scale) and dV_j are written once.
//   bwd_post  dq = bf16(scale * accumulator).
//
// Warp roles of bwd_main (512 threads):
//   warps 0-3   softmax-gradient warpgroup for even query tiles (buffer 0),
//   warps 4-7   the same for odd tiles (buffer 1): thread = key row; writes
//               P^T and dS^T to tensor memory and dS^T to shared memory (the
//               B operand of dQ^T); epilogue stores dV (half of the columns
//               each).
//   warp 8      producer: K_j, V_j once; Q_i, dO_i by TMA and L_i, D_i by
//               plain loads into a three-stage ring.
//   warp 9      tensor-memory owner and MMA issuer (the whole warp runs the
//               issue loop so operand descriptors stay warp-uniform; one
//               elected lane issues).
//   warps 10-11 idle (keep the third warpgroup whole).
//   warps 12-15 dQ warpgroup: thread = column c of dQ; reads dQ_i^T out of
//               tensor memory, releases it and issues the reductions;
//               epilogue stores dK.
// Tensor memory (512 columns): S^T[2] (64 each; dS^T in bf16 over its first
// 32 columns once S^T is loaded) | dP^T[2] (64 each; P^T in bf16 over its
// first 32 columns, then dQ_i^T over all 64) | dV (D) | dK (D).
// S^T and dP^T are double-buffered so that one warpgroup's softmax-gradient
// work overlaps the MMAs of the other's tile. Every tcgen05 operation of the
// MMA thread completes in issue order, which orders the P^T reads of dV
// before the dQ^T write into the same columns, and the dS^T reads of dK
// before the next S^T write into its columns.

#include <cuda_bf16.h>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100.cuh"


namespace fa {
namespace {

constexpr int kKT = 128;   // keys per key tile (MMA M of the key-side products)
constexpr int kQT = 64;    // queries per query tile
constexpr int kThreads = 512;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kDqWarp0 = 12;
constexpr int kQStages = 3;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kKBox = kKT * 128;                  // one 64-column box of a 128-row tile
  static constexpr int kKTile = kKBox * (D / 64);          // K_j or V_j
  static constexpr int kQBox = kQT * 128;                  // one 64-column box of a 64-row tile
  static constexpr int kQTile = kQBox * (D / 64);          // Q_i or dO_i
  static constexpr int kDSTile = kKT * kQT * 2;            // dS^T: 128 keys x 64 queries bf16 (one box)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKTile;
  static constexpr int kOffQ = kOffV + kKTile;
  static constexpr int kOffDO = kOffQ + kQStages * kQTile;
  static constexpr int kOffDS = kOffDO + kQStages * kQTile;
  static constexpr int kOffLD = kOffDS + 2 * kDSTile;      // [stage] L2[64], D[64]
  static constexpr int kOffBar = kOffLD + kQStages * 2 * kQT * 4;
  static constexpr int kUsed = kOffBar + 256;
  static constexpr int kSmemBytes = (kUsed + 1024 <= 232448) ? kUsed + 1024 : 232448;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static_assert(kUsed <= 232448, "shared memory budget");
  static_assert(kSmemBytes > 114 * 1024, "one CTA per SM (owns all tensor memory)");
};

struct BwdArgs {
  const float* lse;
  const float* dsum;    // D_i, fp32 [B*Hq*N]
  float* dq_acc;        // fp32 [B*Hq*N*d]
  int N, Hq, Hkv, BHkv, nk, nq;
  int group;  // KV heads per scheduling group (see the work-unit comment)
  int band;   // causal: key tiles per scheduling band (0: strict longest-first)
  int window;  // left window (a huge value when there is none), mask kind 2
  int prefix;  // prefix length, mask kind 2
  float scale, scale_log2;
  LaunchCtl ctl;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t s_full[2], dp_full[2], p_ready[2], ds_free[2], dq_full[2], dq_empty[2];
  uint64_t acc_final, drain;
  uint64_t epi_dv, epi_dk;  // output staging: all rows of dV / dK written to shared memory
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BwdBars) <= 256, "barrier block exceeds its shared-memory reservation");

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

// MASK: 0 none, 1 causal, 2 causal with a left window and/or a prefix
// (key j visible to query i iff (j <= i and i - j <= window) or j < prefix).
template <int D, int MASK>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                    const BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  if (pad + C::kUsed > static_cast<uint32_t>(C::kSmemBytes)) {
    // Not enough room to align the tiles: report instead of overrunning.
    if (threadIdx.x == 0) atomicOr(a.ctl.err, 2u);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::kOffBar);
  float* sLD = reinterpret_cast<float*>(smem + C::kOffLD);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, KV head, key tile j). KV heads are taken in groups
  // (all of them when causal, where longest-first order matters most;
  // otherwise small enough that their query heads' Q, dO and dQ-accumulator
  // tiles stay in L2 while the resident CTAs sweep them); within a group the
  // longest units (smallest j when causal) come first.
  int bkv, j;
  if (MASK == 1 && a.band > 0) {
    // Bands of a.band key tiles, longest band first; within a band,
    // KV-head-major with the key tiles of a head adjacent, so that the
    // resident CTAs share the dQ accumulator, Q and dO of a few heads.
    const int per_band = a.band * a.BHkv;
    const int band = blockIdx.x / per_band;
    const int rem = blockIdx.x - band * per_band;
    const int bw = min(a.band, a.nk - band * a.band);
    bkv = rem / bw;
    j = band * a.band + rem % bw;
  } else {
    const int per_group = a.group * a.nk;
    const int grp = blockIdx.x / per_group;
    const int rem = blockIdx.x - grp * per_group;
    const int gsize = min(a.group, a.BHkv - grp * a.group);
    bkv = grp * a.group + rem % gsize;
    j = rem / gsize;
  }
  const int r = a.Hq / a.Hkv;
  const int b = bkv / a.Hkv;
  const int g = bkv % a.Hkv;
  // Query tiles [i0, i0 + nqi) that see some key of tile j: all of them
  // without a mask or when the tile holds a prefix key; otherwise from the
  // tile's first key on (causal) up to its last key plus the window.
  int i0 = 0, i1 = a.nq;
  if (MASK == 1) i0 = 2 * j;
  if (MASK == 2 && j * kKT >= a.prefix) {
    i0 = 2 * j;
    const long long last = static_cast<long long>(j) * kKT + kKT - 1 + a.window;
    i1 = static_cast<int>(min(static_cast<long long>(a.nq), last / kQT + 1));
  }
  const int nqi = i1 - i0;             // query tiles per head
  const int n_it = r * nqi;            // (head, query tile) iterations

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->dp_full[x], 1);
      mbar_init(&bars->p_ready[x], kKT);
      mbar_init(&bars->ds_free[x], 1);
      mbar_init(&bars->dq_full[x], 1);
      mbar_init(&bars->dq_empty[x], 128);
    }
    mbar_init(&bars->acc_final, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->epi_dv, 256);
    mbar_init(&bars->epi_dk, 128);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const Watch w{&bars->abort, a.ctl.err, a.ctl.budget_ns};

  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sDO = smem_u32(smem + C::kOffDO);
  const uint32_t sDS = smem_u32(smem + C::kOffDS);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    int q_last[kQStages];
#pragma unroll
    for (int s = 0; s < kQStages; ++s) q_last[s] = -1;
    bool kv_issued = false;
    bool ok = true;
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * C::kKTile);
      for (int x = 0; x < D / 64; ++x) {
        tma_load_3d(&tmK, &bars->kv_full, smem + C::kOffK + x * C::kKBox, x * 64, j * kKT, bkv);
        tma_load_3d(&tmV, &bars->kv_full, smem + C::kOffV + x * C::kKBox, x * 64, j * kKT, bkv);
      }
      kv_issued = true;
    }
    for (int it = 0; it < n_it; ++it) {
      const int s = it % kQStages;
      const int u = it / kQStages;
      if (it >= kQStages) {
        ok = __all_sync(0xffffffffu, wait_bar(&bars->q_empty[s], (u - 1) & 1, w));
        if (!ok) break;
      }
      const int h = g * r + it / nqi;
      const int i = i0 + it % nqi;
      const int bh = b * a.Hq + h;
      // L (in log2 units) and D for the 64 query rows of this tile; rows
      // past N get L = +inf so that their P is exactly 0.
      float* l2 = sLD + s * 2 * kQT;
      float* dd = l2 + kQT;
#pragma unroll
      for (int e = 0; e < kQT / 32; ++e) {
        const int rr = e * 32 + lane;
        const int row = i * kQT + rr;
        const bool in = row < a.N;
        const size_t idx = static_cast<size_t>(bh) * a.N + row;
        l2[rr] = in ? a.lse[idx] * kLog2e : CUDART_INF_F;
        dd[rr] = in ? a.dsum[idx] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::kQTile);
        for (int x = 0; x < D / 64; ++x) {
          tma_load_3d(&tmQ, &bars->q_full[s], smem + C::kOffQ + s * C::kQTile + x * C::kQBox, x * 64, i * kQT,
                      bh);
          tma_load_3d(&tmDO, &bars->q_full[s], smem + C::kOffDO + s * C::kQTile + x * C::kQBox, x * 64, i * kQT,
                      bh);
        }
        q_last[s] = u;
      }
    }
    if (lane == 0) {
      if (kv_issued) drain_bar(&bars->kv_full, 0, w);
      for (int s = 0; s < kQStages; ++s)
        if (q_last[s] >= 0) drain_bar(&bars->q_full[s], q_last[s] & 1, w);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- MMA issue
    // The whole warp runs this loop (descriptors stay warp-uniform); the
    // elected lane issues the tcgen05 instructions.
    const bool leader = elect_one();
    auto all = [](bool b) { return __all_sync(0xffffffffu, b); };
    {
      constexpr uint32_t id_sdp = idesc_bf16(kKT, kQT, false, false);  // S^T, dP^T: 128 x 64
      constexpr uint32_t id_dvk = idesc_bf16(kKT, D, false, true);     // dV (A in TMEM), dK
      constexpr uint32_t id_dq = idesc_bf16(128, kQT, true, true);     // dQ^T: A = K^T, B = dS^T
      // Operand descriptors, computed once and stepped by byte offsets
      // (sdesc_step). K step k (16 elements) of a K-major operand: 32 bytes
      // within a 128-byte swizzle row, boxes of 64 columns kKBox / kQBox
      // bytes apart; of an MN-major operand: 16 rows of 128 bytes (2048).
      const uint64_t kK = sdesc_sw128(sK, 16, 1024), kV = sdesc_sw128(sV, 16, 1024);
      const uint64_t kQ = sdesc_sw128(sQ, 16, 1024), kO = sdesc_sw128(sDO, 16, 1024);
      const uint64_t kDS = sdesc_sw128(sDS, 16, 1024);
      const uint64_t mQ = sdesc_sw128(sQ, C::kQBox, 1024), mO = sdesc_sw128(sDO, C::kQBox, 1024);
      const uint64_t mK = sdesc_sw128(sK, C::kKBox, 1024), mDS = sdesc_sw128(sDS, C::kKBox, 1024);
      auto ofs_k = [](int k) { return static_cast<uint32_t>((k / 4) * (kKT * 128) + (k % 4) * 32); };
      auto ofs_q = [](int k) { return static_cast<uint32_t>((k / 4) * (kQT * 128) + (k % 4) * 32); };
      auto ofs_m = [](int k) { return static_cast<uint32_t>(k * 2048); };
      // Four MMAs, K steps k0..k0+3, into d; A and B stepped by their offsets.
      auto ss4 = [&](uint32_t d, uint64_t a, uint64_t b, auto oa, auto ob, int k0, uint32_t id, uint32_t acc0) {
        mma_ss_x4(d, sdesc_step(a, oa(k0)), sdesc_step(a, oa(k0 + 1)), sdesc_step(a, oa(k0 + 2)),
                  sdesc_step(a, oa(k0 + 3)), sdesc_step(b, ob(k0)), sdesc_step(b, ob(k0 + 1)),
                  sdesc_step(b, ob(k0 + 2)), sdesc_step(b, ob(k0 + 3)), id, acc0, leader);
      };
      auto ts4 = [&](uint32_t d, uint32_t a, uint64_t b, auto ob, int k0, uint32_t id, uint32_t acc0) {
        mma_ts_x4(d, a + 8 * k0, a + 8 * (k0 + 1), a + 8 * (k0 + 2), a + 8 * (k0 + 3), sdesc_step(b, ob(k0)),
                  sdesc_step(b, ob(k0 + 1)), sdesc_step(b, ob(k0 + 2)), sdesc_step(b, ob(k0 + 3)), id, acc0,
                  leader);
      };
      auto issue_sdp = [&](int it) {
        const int x = it & 1;
        const uint32_t st = (it % kQStages) * C::kQTile;
        const uint64_t q = sdesc_step(kQ, st), o = sdesc_step(kO, st);
        const uint32_t tS = tmem + C::kColS + 64 * x, tDP = tmem + C::kColDP + 64 * x;
#pragma unroll
        for (int k = 0; k < D / 16; k += 4) ss4(tS, kK, q, ofs_k, ofs_q, k, id_sdp, k > 0);
        mma_commit(&bars->s_full[x], leader);
        return [=] {
#pragma unroll
          for (int k = 0; k < D / 16; k += 4) ss4(tDP, kV, o, ofs_k, ofs_q, k, id_sdp, k > 0);
        };
      };
      const uint32_t tDV = tmem + C::kColDV, tDK = tmem + C::kColDK;
      // M(it): dV += P^T dO, dK += dS^T Q, dQ^T = K^T dS^T for tile it.
      auto issue_main = [&](int it) {
        const int x = it & 1;
        const int s = it % kQStages;
        const uint32_t tDP = tmem + C::kColDP + 64 * x;
        const uint32_t st = s * C::kQTile;
        const uint64_t qm = sdesc_step(mQ, st), om = sdesc_step(mO, st);
        const uint32_t acc = it > 0;
        ts4(tDV, tDP, om, ofs_m, 0, id_dvk, acc);  // dV += P^T dO (K = 64 queries)
        ts4(tDK, tmem + C::kColS + 64 * x, qm, ofs_m, 0, id_dvk, acc);  // dK += dS^T Q (dS^T in tensor memory)
        const uint64_t dsm = sdesc_step(mDS, x * C::kDSTile);
#pragma unroll
        for (int k = 0; k < kKT / 16; k += 4) ss4(tDP, mK, dsm, ofs_m, ofs_m, k, id_dq, k > 0);  // dQ^T = K^T dS^T
        mma_commit(&bars->dq_full[x], leader);
        mma_commit(&bars->ds_free[x], leader);
        mma_commit(&bars->q_empty[s], leader);
      };
      bool ok = all(wait_bar(&bars->kv_full, 0, w));
      // Tiles 0 and 1: S^T and dP^T into their own buffers.
      for (int it = 0; ok && it < 2 && it < n_it; ++it) {
        if (!(ok = all(wait_bar(&bars->q_full[it % kQStages], (it / kQStages) & 1, w)))) break;
        tc_fence_after();
        auto dp = issue_sdp(it);
        dp();
        mma_commit(&bars->dp_full[it & 1], leader);
      }
      // Then, per tile it: M(it) once the softmax-gradient warps hand it
      // back; S^T and dP^T of tile it + 2 into the same buffers (dP^T after
      // dQ^T of tile it has been read out of its columns).
      for (int it = 0; ok && it < n_it; ++it) {
        const int x = it & 1;
        if (!(ok = all(wait_bar(&bars->p_ready[x], (it >> 1) & 1, w)))) break;
        tc_fence_after();
        issue_main(it);
        const int nx = it + 2;
        if (nx < n_it) {
          if (!(ok = all(wait_bar(&bars->q_full[nx % kQStages], (nx / kQStages) & 1, w)))) break;
          tc_fence_after();
          auto dp = issue_sdp(nx);
          if (!(ok = all(wait_bar(&bars->dq_empty[x], (it >> 1) & 1, w)))) break;
          tc_fence_after();
          dp();
          mma_commit(&bars->dp_full[x], leader);
        }
      }
      mma_commit(&bars->acc_final, leader);
      mma_commit(&bars->drain, leader);
      all(drain_bar(&bars->drain, 0, w));
    }
  } else if (warp < 8) {
    // ------------------------------------------- P^T and dS^T (key rows)
    const int x = warp >> 2;                               // buffer = parity of the tiles handled
    const int quad = warp & 3;
    const int kr = quad * 32 + lane;                       // key row in tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + 64 * x;
    const uint32_t tDP = tmem + lane_off + C::kColDP + 64 * x;
    const float sl2 = a.scale_log2;
    uint8_t* ds_row = smem + C::kOffDS + x * C::kDSTile + kr * 128;
    const uint32_t sw = static_cast<uint32_t>(kr & 7);
    bool ok = true;
    for (int it = x; it < n_it; it += 2) {
      const int s = it % kQStages;
      const int i = i0 + it % nqi;
      const uint32_t par = (it >> 1) & 1;
      const float* l2 = sLD + s * 2 * kQT;
      const float* dd = l2 + kQT;
      // q_full orders the producer's plain stores of L and D before these reads.
      ok = __all_sync(0xffffffffu, wait_bar(&bars->q_full[s], (it / kQStages) & 1, w));
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bars->s_full[x], par, w));
      if (ok && it >= 2) ok = __all_sync(0xffffffffu, wait_bar(&bars->ds_free[x], par ^ 1, w));
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bars->dp_full[x], par, w));
      if (!ok) break;
      tc_fence_after();
      // Kinds 0, 1: local query ql is masked when its position is below this
      // key's. Kind 2: the general predicate, unless every pair of the tile
      // pair is visible (all keys in the prefix, or below every query's
      // diagonal and inside every query's window).
      const int diag_lim = MASK == 1 ? kKT * j + kr - kQT * i : -1;
      const int key = kKT * j + kr;
      const bool gmask = MASK == 2 && !((kKT * j + kKT <= a.prefix) ||
                                        (kKT * j + kKT - 1 <= kQT * i && kQT * i + kQT - 1 - kKT * j <= a.window));
#pragma unroll
      for (int c = 0; c < kQT / 32; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld32_nowait(tS + c * 32, sv);
        tmem_ld32_nowait(tDP + c * 32, dv);
        tmem_ld_wait(sv);
        tmem_ld_tie(dv);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int y = 0; y < 8; ++y) {
          const int q0 = c * 32 + 4 * y;
          const float4 lq = *reinterpret_cast<const float4*>(l2 + q0);
          const float4 dq = *reinterpret_cast<const float4*>(dd + q0);
          // Exponent arguments, dP - D and the products two at a time
          // (packed f32x2, same rounding as the scalar form).
          float p[4];
          ffma2(p[0], p[1], __uint_as_float(sv[4 * y]), __uint_as_float(sv[4 * y + 1]), sl2, sl2, -lq.x, -lq.y);
          ffma2(p[2], p[3], __uint_as_float(sv[4 * y + 2]), __uint_as_float(sv[4 * y + 3]), sl2, sl2, -lq.z, -lq.w);
#pragma unroll
          for (int e = 0; e < 4; ++e) p[e] = ex2(p[e]);
          if (q0 < diag_lim) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (q0 + e < diag_lim) p[e] = 0.f;
          }
          if (gmask) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int qg = kQT * i + q0 + e;
              if (!((key <= qg && qg - key <= a.window) || key < a.prefix)) p[e] = 0.f;
            }
          }
          float g0, g1, g2, g3;
          fsub2(g0, g1, __uint_as_float(dv[4 * y]), __uint_as_float(dv[4 * y + 1]), dq.x, dq.y);
          fsub2(g2, g3, __uint_as_float(dv[4 * y + 2]), __uint_as_float(dv[4 * y + 3]), dq.z, dq.w);
          fmul2(g0, g1, p[0], p[1], g0, g1);
          fmul2(g2, g3, p[2], p[3], g2, g3);
          pk[2 * y] = pack_bf16x2(p[0], p[1]);
          pk[2 * y + 1] = pack_bf16x2(p[2], p[3]);
          dk[2 * y] = pack_bf16x2(g0, g1);
          dk[2 * y + 1] = pack_bf16x2(g2, g3);
        }
        // P^T chunk -> columns [16c, 16c+16) of this buffer's dP^T columns
        // (their dP^T values were loaded by this or the previous chunk).
        tmem_st16(tDP + c * 16, pk);
        // dS^T chunk -> columns [16c, 16c+16) of this buffer's S^T columns
        // (their S^T values were loaded by this or the previous chunk): the
        // A operand of dK += dS^T Q straight from tensor memory.
        tmem_st16(tS + c * 16, dk);
        // dS^T chunk: queries [32c, 32c+32) of key row kr, 128-byte swizzled.
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = static_cast<uint32_t>(c * 4 + u);
          *reinterpret_cast<uint4*>(ds_row + ((chunk ^ sw) << 4)) =
              make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_ready[x]);
    }
    // Epilogue: dV_j rows (this thread's key row), half of the columns per
    // warpgroup, staged over V_j (no MMA reads it any more) in its 128-byte
    // swizzled box layout and written by TMA stores once all 256 threads
    // have staged theirs (whole lines instead of one thread per row writing
    // half sectors). Key rows past N are clipped by the copy.
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bars->acc_final, 0, w));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int c = x * (D / 64) + cc;  // 32-column chunk
        uint32_t vv[32];
        tmem_ld32(tmem + lane_off + C::kColDV + c * 32, vv);
        uint8_t* row = smem + C::kOffV + (c / 2) * C::kKBox + kr * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = static_cast<uint32_t>((c % 2) * 4 + u);
          *reinterpret_cast<uint4*>(row + ((chunk ^ (kr & 7)) << 4)) =
              make_uint4(pack_bf16x2(__uint_as_float(vv[8 * u]), __uint_as_float(vv[8 * u + 1])),
                         pack_bf16x2(__uint_as_float(vv[8 * u + 2]), __uint_as_float(vv[8 * u + 3])),
                         pack_bf16x2(__uint_as_float(vv[8 * u + 4]), __uint_as_float(vv[8 * u + 5])),
                         pack_bf16x2(__uint_as_float(vv[8 * u + 6]), __uint_as_float(vv[8 * u + 7])));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->epi_dv);
      if (threadIdx.x == 0 && wait_bar(&bars->epi_dv, 0, w)) {
#pragma unroll
        for (int b = 0; b < D / 64; ++b) tma_store_3d(&tmDV, smem + C::kOffV + b * C::kKBox, b * 64, j * kKT, bkv);
        bulk_commit();
      }
      if (threadIdx.x == 0) bulk_wait_read<0>();
    }
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------- dQ_i^T readout (columns of dQ)
    // Lane m of the four warps holds column m of dQ_i for the 64 query rows,
    // so for each row the 32 lanes of a warp cover 32 consecutive floats: one
    // fully coalesced 128-byte reduction per warp instruction, straight from
    // registers (no shared-memory staging, which would compete with the MMA
    // operand reads for shared-memory bandwidth).
    const int quad = warp & 3;
    const int m = quad * 32 + lane;                        // column of dQ (tensor-memory lane)
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int x = it & 1;
      ok = __all_sync(0xffffffffu, wait_bar(&bars->dq_full[x], (it >> 1) & 1, w));
      if (!ok) break;
      tc_fence_after();
      const int h = g * r + it / nqi;
      const int i = i0 + it % nqi;
      const int bh = b * a.Hq + h;
      uint32_t v0[32], v1[32];
      const uint32_t tDQ = tmem + lane_off + C::kColDP + 64 * x;
      tmem_ld32(tDQ, v0);
      tmem_ld32(tDQ + 32, v1);
      tc_fence_before();
      mbar_arrive(&bars->dq_empty[x]);
      if (m < D) {
        const int row0 = i * kQT;
        float* col = a.dq_acc + (static_cast<size_t>(bh) * a.N + row0) * D + m;
        const int rows = min(kQT, a.N - row0);
        if (rows == kQT) {
#pragma unroll
          for (int q = 0; q < 32; ++q) red_add_f32(col + static_cast<size_t>(q) * D, __uint_as_float(v0[q]));
#pragma unroll
          for (int q = 0; q < 32; ++q) red_add_f32(col + static_cast<size_t>(q + 32) * D, __uint_as_float(v1[q]));
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (q < rows) red_add_f32(col + static_cast<size_t>(q) * D, __uint_as_float(v0[q]));
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (q + 32 < rows) red_add_f32(col + static_cast<size_t>(q + 32) * D, __uint_as_float(v1[q]));
        }
      }
    }
    // Epilogue: dK_j = scale * accumulated dS^T Q (row m = key row), staged
    // over K_j and written by TMA stores as dV is.
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bars->acc_final, 0, w));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t vv[32];
        tmem_ld32(tmem + lane_off + C::kColDK + c * 32, vv);
        uint8_t* row = smem + C::kOffK + (c / 2) * C::kKBox + m * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t chunk = static_cast<uint32_t>((c % 2) * 4 + u);
          *reinterpret_cast<uint4*>(row + ((chunk ^ (m & 7)) << 4)) = make_uint4(
              pack_bf16x2(__uint_as_float(vv[8 * u]) * a.scale, __uint_as_float(vv[8 * u + 1]) * a.scale),
              pack_bf16x2(__uint_as_float(vv[8 * u + 2]) * a.scale, __uint_as_float(vv[8 * u + 3]) * a.scale),
              pack_bf16x2(__uint_as_float(vv[8 * u + 4]) * a.scale, __uint_as_float(vv[8 * u + 5]) * a.scale),
              pack_bf16x2(__uint_as_float(vv[8 * u + 6]) * a.scale, __uint_as_float(vv[8 * u + 7]) * a.scale));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->epi_dk);
      const bool issuer = warp == kDqWarp0 && lane == 0;
      if (issuer && wait_bar(&bars->epi_dk, 0, w)) {
#pragma unroll
        for (int b = 0; b < D / 64; ++b) tma_store_3d(&tmDK, smem + C::kOffK + b * C::kKBox, b * 64, j * kKT, bkv);
        bulk_commit();
      }
      if (issuer) bulk_wait_read<0>();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// D_i = sum_c dO_ic O_ic for every query row, and zero the dQ accumulator.
// One warp per row; each lane handles 8 columns per step (one uint4 each).
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ o_resid,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ dsum, float* __restrict__ dq_acc,
                                                      long long rows) {
  const long long warp_g = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long row = warp_g; row < rows; row += nwarps) {
    float acc = 0.f;
    if (lane * 8 < D) {
      const uint4 a4 = reinterpret_cast<const uint4*>(o + row * D)[lane];
      const uint4 b4 = reinterpret_cast<const uint4*>(dout + row * D)[lane];
      const uint4 r4 = o_resid ? reinterpret_cast<const uint4*>(o_resid + row * D)[lane] : make_uint4(0, 0, 0, 0);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a4);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b4);
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&r4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fr = __bfloat1622float2(r2[e]);
        const float2 fb = __bfloat1622float2(b2[e]);
        acc = fmaf(fa.x + fr.x, fb.x, acc);
        acc = fmaf(fa.y + fr.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dsum[row] = acc;
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D);
    for (int e = lane; e < D / 4; e += 32) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dq = bf16(scale * accumulator), 8 elements per thread per step.
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* __restrict__ dq_acc,
                                                       __nv_bfloat16* __restrict__ dq, float scale,
                                                       long long n8) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n8; e += stride) {
    const float4 x = reinterpret_cast<const float4*>(dq_acc)[2 * e];
    const float4 y = reinterpret_cast<const float4*>(dq_acc)[2 * e + 1];
    uint4 out;
    out.x = pack_bf16x2(x.x * scale, x.y * scale);
    out.y = pack_bf16x2(x.z * scale, x.w * scale);
    out.z = pack_bf16x2(y.x * scale, y.y * scale);
    out.w = pack_bf16x2(y.z * scale, y.w * scale);
    reinterpret_cast<uint4*>(dq)[e] = out;
  }
}

int grid_for(long long work, int per_block, int cap) {
  long long g = (work + per_block - 1) / per_block;
  if (g < 1) g = 1;
  return static_cast<int>(g < cap ? g : cap);
}

template <int D, int MASK>
cudaError_t launch_bwd_t(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const void* o,
                         const void* o_resid, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                         void* workspace, const LaunchCtl& ctl, cudaStream_t stream) {
  using C = BwdCfg<D>;
  const long long rows = static_cast<long long>(s.B) * s.Hq * s.N;
  float* dsum = static_cast<float*>(workspace);
  const size_t dsum_bytes = ((static_cast<size_t>(rows) * 4 + 255) / 256) * 256;
  float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dsum_bytes);

  bwd_pre_kernel<D><<<grid_for(rows, 8, 148 * 64), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(o_resid),
      static_cast<const __nv_bfloat16*>(dout), dsum, dq_acc, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ctl.ev_after_pre && (e = cudaEventRecord(ctl.ev_after_pre, stream)) != cudaSuccess) return e;

  auto kern = bwd_main_kernel<D, MASK>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  BwdArgs a;
  a.lse = lse;
  a.dsum = dsum;
  a.dq_acc = dq_acc;
  (void)dk;  // written through tdk and tdv
  (void)dv;
  a.N = s.N;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.BHkv = s.B * s.Hkv;
  a.nk = (s.N + kKT - 1) / kKT;
  a.nq = (s.N + kQT - 1) / kQT;
  // Causal units differ in length: keep strict longest-first order over all
  // KV heads. Non-causal units are equal: group KV heads for L2 locality.
  a.group = MASK == 1 ? a.BHkv : l2_head_group(static_cast<long long>(8) * (s.Hq / s.Hkv) * s.N * D, a.BHkv);
  // Causal: strict longest-first order over all KV heads keeps the tail
  // short but spreads the resident CTAs over every head, whose dQ
  // accumulators, Q and dO then fall out of L2 between visits. When those
  // (8 bytes per element of a KV group's query heads) exceed a share of L2
  // and a head has enough key tiles for bands of 16 to stay longest-first
  // overall, order by bands of 16 key tiles, head-major within a band
  // (measured on B200, B=2 H=16 N=8192 d=128: +4.8% on this kernel; at
  // N=2048 the head-major order costs more in tail than it saves).
  const long long group_bytes = static_cast<long long>(8) * (s.Hq / s.Hkv) * s.N * D;
  a.band = (MASK == 1 && a.nk >= 64 && group_bytes * a.BHkv > (48ll << 20)) ? 16 : 0;
  a.window = s.window < 0 ? 0x3fffffff : s.window;
  a.prefix = s.prefix;
  a.scale = s.scale;
  a.scale_log2 = s.scale * kLog2e;
  a.ctl = ctl;
  const long long grid = static_cast<long long>(a.nk) * a.BHkv;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdk, tdv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ctl.ev_after_main && (e = cudaEventRecord(ctl.ev_after_main, stream)) != cudaSuccess) return e;

  const long long n8 = rows * D / 8;
  bwd_post_kernel<<<grid_for(n8, 256, 148 * 32), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq),
                                                                     s.scale, n8);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(const AttnShape& s) {
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * s.N;
  const size_t dsum_bytes = ((rows * 4 + 255) / 256) * 256;
  return dsum_bytes + rows * static_cast<size_t>(s.d) * 4;
}

cudaError_t launch_bwd(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv, const void* o,
                       const void* o_resid, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                       void* workspace, const LaunchCtl& ctl, cudaStream_t stream) {
#define FA_BWD_ARGS s, tq, tk, tv, tdo, tdk, tdv, o, o_resid, dout, lse, dq, dk, dv, workspace, ctl, stream
  switch (s.mask_kind() + (s.d == 64 ? 0 : 3)) {
    case 0: return launch_bwd_t<64, 0>(FA_BWD_ARGS);
    case 1: return launch_bwd_t<64, 1>(FA_BWD_ARGS);
    case 2: return launch_bwd_t<64, 2>(FA_BWD_ARGS);
    case 3: return launch_bwd_t<128, 0>(FA_BWD_ARGS);
    case 4: return launch_bwd_t<128, 1>(FA_BWD_ARGS);
    default: return launch_bwd_t<128, 2>(FA_BWD_ARGS);
  }
#undef FA_BWD_ARGS
}

}  // namespace fa
