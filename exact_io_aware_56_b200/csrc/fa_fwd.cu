// Forward attention kernel for sm_100a.
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V and the row
// logsumexp L, tile by tile, without writing the N x N scores anywhere
// (FlashAttention: IO-aware exact attention, "FLASH" box of the "NAIVE
// ATTENTION vs FLASHATTENTION" diagram, and the "PREFILL PATH" diagram:
// a 128-row Q block stays on chip, 128-column K/V blocks stream through
// shared memory and are dropped, only m, l and O persist, O is written once
// together with one logsumexp per row).
//
// Two forms of one kernel template (FwdCfg, parameter T = Q tiles per CTA):
//   two-tile form (T = 2, d = 128 in bf16): one CTA per SM owns two 128-row
//     Q tiles of one (batch, query head), streams the K/V tiles of its KV
//     head once for both, and holds all 512 tensor-memory columns;
//   one-tile form (T = 1, d = 64 in bf16, and the FP8 mode: 128-byte rows):
//     one Q tile per CTA, two CTAs per SM with 256 columns each, so that one
//     CTA's start and epilogue run under the other's key-tile loop.
// Warp roles (w0 = 4T):
//   warps 0 .. w0-1  softmax, one warpgroup per Q tile: one thread per query
//                    row (warp w reads tensor-memory lanes 32*(w%4)..).
//   warp w0          TMA producer of the Q tiles (once) and of K_j into the
//                    K ring (mbarrier full / empty pairs).
//   warp w0+1        tensor-memory owner and MMA issuer:
//                    S_t = Q_t K_j^T (tcgen05, both operands in shared memory),
//                    O_t += P_t V_j (tcgen05, P_t read from tensor memory).
//   warp w0+2        TMA producer of V_j into the V ring.
//   warp w0+3        idle (keeps the last warpgroup whole).
// The softmax is the online form of the "Four ideas" list (item "Online
// softmax"): running max m, running sum l, O rescaled by e^(m - m_new)
// when the max grows (by more than the rescale threshold below). P_t goes
// back to the MMA thread in two halves of 64 keys, one barrier each; the O
// rescale precedes the first, and the first half's share of O_t += P_t V_j
// runs while the second half's exponentials are computed.
//
// Tensor memory (128 lanes, fp32 columns): S_t at [128t, 128t + 128), O_t
// at kColO + D t. P_t is written over the first columns of S_t (bf16 two
// per column, e4m3 four per column), except at d = 64, where it has its own
// 64 columns at kColP + 64t (the separate-P schedule below). Two-tile form:
//   [0,128) S_0 | [128,256) S_1 | [256,384) O_0 | [384,512) O_1;
// one-tile form: [0,128) S | [128,128+D) O | at d = 64 [192,256) P.
//
// Ordering argument used by the softmax warps when P is written over S: the
// MMA thread issues, for each tile t, S_t^(j+1) after both halves of
// O_t += P_t^j V_j, and tcgen05 operations complete in issue order, so once
// S_t^(j+1) is signalled complete the O_t accumulator holds every earlier
// product and may be rescaled in place until the first half of P_t^(j+1) is
// handed back.
//
// Separate-P schedule (d = 64): the MMA thread issues S_t^(j+1) as soon as
// the softmax has loaded S_t^j (barrier s_free), before O_t += P_t^j V_j.
// The softmax then waits for that product's completion (barrier pv_done)
// before it writes P_t^(j+1) or rescales O_t, instead of relying on the
// order above.
//
// The exponentials are base 2: scores are scaled by scale*log2(e), and
// L = (m + log2 l) * ln 2. A warp whose rows' maxima did not grow on a tile
// skips the tensor-memory round trip of the O rescale.
//
// Epilogue (bf16 mode): each softmax warpgroup stages its normalised O tile
// (and the residual) in shared memory in the 128-byte-swizzled box layout
// and writes it with TMA tensor stores (o and o_resid tensor maps); the FP8
// mode stores its rows from registers.

#include <cuda_bf16.h>
#include <math_constants.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;   // query rows per Q tile
constexpr int kBN = 128;   // keys per K/V tile
// One-tile form (two CTAs per SM): register shares of the softmax
// warpgroup and of the producer / MMA warpgroup (setmaxnreg), summing to
// what a launch at 128 registers per thread gives the CTA.
constexpr int kSoftmaxRegs1 = 192;
constexpr int kOtherRegs1 = 64;
static_assert(kSoftmaxRegs1 + kOtherRegs1 == 2 * 128, "register split of the one-tile form");
// Rescale threshold (log2 units): a warp rescales its O rows only when some
// row's running max grew by more than this. With the O residual (the
// training path, whose backward forms D from O to ~16 bits) it is 0: every
// row's reference max stays exact, so the largest weight of a row is exactly
// 1, which bf16 represents without error; a stale reference turns that
// weight into 2^delta, whose bf16 rounding moves O by up to 2^-9 |V| on
// peaky rows and, through D, dQ and dK past their bound. A forward-only call
// (no residual) takes kRescaleLazy: the same rounding as the output's own,
// L exact, and most rescales skipped (measured on B200: +7 to 9% at N = 8192
// to 16384, d = 128).
constexpr float kRescaleExact = 0.0f;
constexpr float kRescaleLazy = 8.0f;
// FP8 mode has no backward to serve and its weights are e4m3 anyway: a warp
// rescales only when some row's max grew by more than kF8Rescale (log2
// units), which skips most rescales (measured on B200, B=2 H=16 N=8192
// causal: 1168 -> 1290 TFLOP/s). P is written as e4m3 of 2^(x + kF8Offset)
// with x <= kF8Rescale against the stale max, so it stays <= 2^8 < 448, and a
// row's largest weight is at least 2^kF8Offset.
constexpr float kF8Rescale = 4.0f;
constexpr float kF8Offset = 8.0f - kF8Rescale;
// Of every 32 exponentials of a row, this many are evaluated on the FMA pipe
// (exp2_poly, exact at integer arguments like the exponential unit) and the
// rest on the exponential unit. At d = 128 the softmax is one link of a
// chain with P V and the next S, so FMA-pipe instructions mostly lengthen
// it: measured on B200 at N = 8192, 4, 8, 12 of 32 cost 3%, 8%, 14% (with
// per-row epilogue stores and default waits); with the current kernel 2 of
// 32 gains ~1% at 8192 tokens and 1-4% on the 16384-token GQA forward, 1 of
// 32 nothing, 3 and 4 of 32 no better than 2. FP8 mode, one-tile form
// (B = 2, H = 16, N = 8192 and the 16384-token GQA shape): 3 of every 16
// is fastest (+1.2 to +1.6% against 2 of 16, which gained 1.6 and 2.9%
// against 4 of 16, itself 0.6 to 2.4% ahead of none; 1 of 16 -2%, 6 of
// 16 -6%, 8 of 16 -12%). At d = 64 the softmax alone sets the pace (S of the
// next tile is computed while it runs) and its weights need twice the
// exponential unit's time of the MMAs. With two one-tile CTAs per SM
// (B = 4, H = 16, N = 2048): 4 of 32 gains 2 to 4% without a mask and
// loses 2.5% causal (0 fastest there; 2 of 32 -0.6%); 5 and 6 of 32 lose 1 to
// 2.5% against 4, 8 of 32 loses 4 to 7%.
constexpr int kPolyPer32 = 2;
constexpr int kPolyPer16F8 = 3;
template <int D, int MASK>
constexpr int poly_per32() {
  return D == 64 ? (MASK == 0 ? 4 : 0) : kPolyPer32;
}

// F8: e4m3 Q, K, V with block scales (the FP8 mode); otherwise bf16.
// T: Q tiles per CTA. T = 2 (one CTA per SM, all of its tensor memory) is
// the general form; T = 1 (d = 64 in bf16, and the FP8 mode: 128-byte rows)
// runs two CTAs per SM, each with half the tensor memory and shared memory,
// so that one CTA's start and epilogue overlap the other's key-tile loop.
template <int D, bool F8 = false, int T = 2>
struct FwdCfg {
  static_assert(T == 2 || (T == 1 && D * (F8 ? 1 : 2) == 128), "the one-tile form takes 128-byte rows (d = 64 bf16, FP8)");
  static constexpr int kThreads = T == 1 ? 256 : 384;
  static constexpr int kMinBlocks = T == 1 ? 2 : 1;  // CTAs per SM
  static constexpr int kProducerWarp = 4 * T;        // Q and K
  static constexpr int kMmaWarp = 4 * T + 1;
  static constexpr int kVProducerWarp = 4 * T + 2;   // V
  static constexpr int kElem = F8 ? 1 : 2;              // bytes per element
  static constexpr int kBoxCols = 128 / kElem;          // elements per 128-byte swizzle row
  static constexpr int kKStep = 32 / kElem;             // MMA K per instruction (16 bf16, 32 e4m3)
  // K and V rings: K_j is free once both S products of tile j are issued,
  // V_j only after both P V products, so K gets the deeper ring where
  // shared memory is short (d = 128 in bf16: 3 K stages, 2 V stages).
  static constexpr int kKStages = T == 1 ? 2 : (D * kElem == 256) ? 3 : 4;
  static constexpr int kVStages = T == 1 ? 2 : (D * kElem == 256) ? 2 : 4;
  static constexpr int kBoxBytes = kBN * 128;           // one 128-byte-wide TMA box of a 128-row tile
  static constexpr int kBoxes = D * kElem / 128;
  static constexpr int kTileBytes = kBoxBytes * kBoxes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = T * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  // Output staging (the epilogue, bf16 mode): two 16-KB boxes per Q tile.
  // At d = 128 the finished Q_t buffer holds them; at d = 64 they get their
  // own region, except in the one-tile form, whose two boxes are the Q
  // buffer and one box of its own.
  static constexpr bool kOwnStage = !F8 && (T == 1 || kTileBytes < 2 * 16384);
  static constexpr int kOffStage = (kOffBar + kBarBytes + 1023) / 1024 * 1024;
  static constexpr int kStageBytes = T == 1 ? 16384 : 4 * 16384;
  // + alignment slack
  static constexpr int kSmemBytes = (kOwnStage ? kOffStage + kStageBytes : kOffBar + kBarBytes) + 1024;
  // Tensor memory: S_t at [128t, 128t + 128), O_t at kColO + D t, P_t (the
  // separate-P schedule) at kColP + 64t.
  static constexpr uint32_t kTmemCols = T == 1 ? 256 : 512;
  static constexpr uint32_t kColO = T == 1 ? 128 : 256;
  static constexpr uint32_t kColP = T == 1 ? 192 : 384;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // One CTA per SM (it owns all tensor memory), or exactly two.
  static_assert(T == 1 ? (kSmemBytes <= 228 * 1024 / 2 - 1024 && 3 * kSmemBytes > 228 * 1024)
                       : kSmemBytes > 114 * 1024,
                "CTAs per SM");
};

// Block scales of the FP8 mode: Q and K per 128-row block of a head
// ([B*Hq][nb], [B*Hkv][nb]), V per head ([B*Hkv]).
struct Fp8Scales {
  const float* sq;
  const float* sk;
  const float* sv;
};

struct FwdArgs {
  void* o;              // stored through tmO, except in FP8 mode
  const void* o_resid;  // optional: bf16(O - bf16(O)), the rounding residual of o (stored through tmR)
  float* lse;
  int N, Hq, Hkv, BH, nk;
  int n_pairs;  // work units per head: pairs of Q tiles (single tiles in the one-tile form)
  int group;  // heads per scheduling group (see the work-unit comment)
  int window;  // left window (a huge value when there is none), mask kind 2
  int prefix;  // prefix length, mask kind 2
  float scale_log2;
  float rescale_tau;  // rescale threshold (log2 units), see kRescaleExact
  Fp8Scales f8;
  LaunchCtl ctl;
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
  uint64_t s_full[2], p_ready[2][2], o_final[2];  // p_ready: [Q tile][half of P]
  uint64_t s_free[2], pv_done[2];  // separate-P schedule (d = 64) only
  uint64_t epi_full[2], epi_free[2];  // output staging (see the epilogue)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FwdBars) <= FwdCfg<128>::kBarBytes && sizeof(FwdBars) <= FwdCfg<64, false, 1>::kBarBytes,
              "barrier block exceeds its shared-memory reservation");

// Key j visible to query i under mask kind 2.
__device__ __forceinline__ bool visible2(int i, int j, int window, int prefix) {
  return (j <= i && i - j <= window) || j < prefix;
}

// MASK: 0 none, 1 causal, 2 causal with a left window and/or a prefix.
// F8: e4m3 operands with block scales (FP8 mode, masks 0 and 1).
// T: Q tiles per CTA (see FwdCfg).
template <int D, int MASK, bool F8 = false, int T = 2>
__global__ void __launch_bounds__(FwdCfg<D, F8, T>::kThreads, FwdCfg<D, F8, T>::kMinBlocks)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmR, const FwdArgs a) {
  using C = FwdCfg<D, F8, T>;
  static_assert(!F8 || MASK != 2, "FP8 mode covers the unmasked and causal forward");
  // Separate-P schedule: at d = 64 tensor memory has room for P next to S
  // and O (P_t at kColP + 64t), so S_t of the next key tile is computed as
  // soon as the softmax has loaded S_t, while it still turns the scores
  // into P, and the softmax warps never wait for P V and S to pass through
  // the tensor pipe between tiles.
  constexpr bool SEP = (D == 64) && !F8;
  constexpr int KS = C::kKStages;  // K ring stages
  constexpr int VS = C::kVStages;  // V ring stages
  static_assert(KS <= 4 && VS <= 4, "barrier arrays hold four stages");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::kOffBar);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch*head, T consecutive Q tiles: a pair, or one tile in the
  // one-tile form). Heads are taken in groups
  // (all heads in one group when causal, where longest-first order matters
  // most; otherwise small enough that a group's K/V tiles stay in L2 while
  // the resident CTAs stream them); within a group the heaviest pairs
  // (largest query index, most K/V tiles when causal) come first and heads
  // sharing a KV head are adjacent.
  const int per_group = a.group * a.n_pairs;
  const int grp = blockIdx.x / per_group;
  const int rem = blockIdx.x - grp * per_group;
  const int gsize = min(a.group, a.BH - grp * a.group);
  const int bh = grp * a.group + rem % gsize;
  const int pair = a.n_pairs - 1 - rem / gsize;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int kvh = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int q0 = pair * T * kBM;
  int n_t[2];
  // Mask kind 2: both Q tiles walk one K/V stream, the prefix tiles [0, pre)
  // then the window tiles [win0, win1): stream position u holds key tile
  // u < pre ? u : win0 + (u - pre). Tiles in the gap are never visited.
  int pre = 0, win0 = 0;
  if (MASK == 2) {
    const int q_hi = min(q0 + T * kBM, a.N) - 1;   // highest real query of the unit
    pre = min(a.nk, (a.prefix + kBN - 1) / kBN);
    const int lo_key = (a.window >= q0) ? 0 : q0 - a.window;
    win0 = max(pre, lo_key / kBN);
    const int win1 = min(a.nk, q_hi / kBN + 1);
    n_t[0] = n_t[1] = pre + max(0, win1 - win0);
  } else {
#pragma unroll
    for (int t = 0; t < 2; ++t) n_t[t] = MASK == 1 ? min(a.nk, T * pair + min(t, T - 1) + 1) : a.nk;
  }
  // n_t[1] is the unit's K/V stream length (n_t[0] in the one-tile form).
  auto key_tile = [&](int u) { return (MASK == 2 && u >= pre) ? win0 + (u - pre) : u; };

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_ready[t][0], kBM);
      mbar_init(&bars->p_ready[t][1], kBM);
      mbar_init(&bars->o_final[t], 1);
      mbar_init(&bars->s_free[t], kBM);
      mbar_init(&bars->pv_done[t], 1);
      mbar_init(&bars->epi_full[t], kBM);
      mbar_init(&bars->epi_free[t], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const Watch w{&bars->abort, a.ctl.err, a.ctl.budget_ns};

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);

  if (warp >= 4 * T) {
    // Producers and the MMA warp (one-tile form: the smaller register share).
    if constexpr (T == 1) regs_dec<kOtherRegs1>();
    if (warp == C::kProducerWarp) {
      // ------------------------------------------------------- Q, K producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        int k_last[KS];
    #pragma unroll
        for (int s = 0; s < KS; ++s) k_last[s] = -1;
        mbar_arrive_expect_tx(&bars->q_full, T * C::kTileBytes);
    #pragma unroll
        for (int t = 0; t < T; ++t)
    #pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(&tmQ, &bars->q_full, smem + C::kOffQ + t * C::kTileBytes + x * C::kBoxBytes,
                        x * C::kBoxCols, q0 + t * kBM, bh);
        const int n = n_t[1];
        for (int j = 0; j < n; ++j) {
          const int s = j % KS;
          const int u = j / KS;
          if (j >= KS && !wait_bar(&bars->k_empty[s], (u - 1) & 1, w)) break;
          if (a.ctl.fault == 1 && j == 0) continue;  // test hook: K_0 never arrives
          mbar_arrive_expect_tx(&bars->k_full[s], C::kTileBytes);
    #pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(&tmK, &bars->k_full[s], smem + C::kOffK + s * C::kTileBytes + x * C::kBoxBytes,
                        x * C::kBoxCols, key_tile(j) * kBN, kvh);
          k_last[s] = u;
        }
        // Every copy issued must land before the CTA may exit.
        drain_bar(&bars->q_full, 0, w);
    #pragma unroll
        for (int s = 0; s < KS; ++s)
          if (k_last[s] >= 0) drain_bar(&bars->k_full[s], k_last[s] & 1, w);
      }
    } else if (warp == C::kVProducerWarp) {
      // ----------------------------------------------------------- V producer
      if (lane == 0) {
        tma_prefetch_desc(&tmV);
        int v_last[VS];
    #pragma unroll
        for (int s = 0; s < VS; ++s) v_last[s] = -1;
        const int n = n_t[1];
        for (int j = 0; j < n; ++j) {
          const int s = j % VS;
          const int u = j / VS;
          if (j >= VS && !wait_bar(&bars->v_empty[s], (u - 1) & 1, w)) break;
          mbar_arrive_expect_tx(&bars->v_full[s], C::kTileBytes);
    #pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(&tmV, &bars->v_full[s], smem + C::kOffV + s * C::kTileBytes + x * C::kBoxBytes,
                        x * C::kBoxCols, key_tile(j) * kBN, kvh);
          v_last[s] = u;
        }
    #pragma unroll
        for (int s = 0; s < VS; ++s)
          if (v_last[s] >= 0) drain_bar(&bars->v_full[s], v_last[s] & 1, w);
      }
    } else if (warp == C::kMmaWarp) {
      // ----------------------------------------------------------- MMA issue
      // The whole warp runs this loop (descriptors stay warp-uniform); the
      // elected lane issues the tcgen05 instructions.
      const bool leader = elect_one();
      auto all = [](bool b) { return __all_sync(0xffffffffu, b); };
      {
        constexpr uint32_t idesc_qk = F8 ? idesc_e4m3(kBM, kBN, false, false) : idesc_bf16(kBM, kBN, false, false);
        constexpr uint32_t idesc_pv = F8 ? idesc_e4m3(kBM, D, false, true) : idesc_bf16(kBM, D, false, true);
        constexpr int KSTEP = C::kKStep;  // MMA K per instruction (16 bf16, 32 e4m3)
        const uint32_t tS[2] = {tmem, tmem + 128u};
        // A operand (P) of O += P V: over S, or in its own columns (SEP).
        const uint32_t tP[2] = {SEP ? tmem + C::kColP : tmem, SEP ? tmem + C::kColP + 64u : tmem + 128u};
        const uint32_t tO[2] = {tmem + C::kColO, tmem + C::kColO + D};
        // Operand descriptors computed once and stepped by byte offsets
        // (sdesc_step): K step k of a K-major tile is 32 bytes within a
        // 128-byte swizzle row, boxes kBoxBytes apart; of the MN-major V tile,
        // KSTEP rows of 128 bytes.
        const uint64_t dQ = sdesc_sw128(sQ, 16, 1024), dK = sdesc_sw128(sK, 16, 1024);
        const uint64_t dV = sdesc_sw128(sV, C::kBoxBytes, 1024);
        auto ofs_kmaj = [](int k) { return static_cast<uint32_t>((k / 4) * C::kBoxBytes + (k % 4) * 32); };
        auto issue_s = [&](int t, int j) {
          const uint64_t qa = sdesc_step(dQ, t * C::kTileBytes);
          const uint64_t ka = sdesc_step(dK, (j % KS) * C::kTileBytes);
          if constexpr (F8) {
            // Each K step is 32 bytes of a 128-byte swizzle row (32 e4m3).
    #pragma unroll
            for (int k = 0; k < D / KSTEP; ++k)
              mma_ss_f8(tS[t], sdesc_step(qa, ofs_kmaj(k)), sdesc_step(ka, ofs_kmaj(k)), idesc_qk, k > 0, leader);
          } else {
    #pragma unroll
            for (int k = 0; k < D / KSTEP; k += 4)
              mma_ss_x4(tS[t], sdesc_step(qa, ofs_kmaj(k)), sdesc_step(qa, ofs_kmaj(k + 1)),
                        sdesc_step(qa, ofs_kmaj(k + 2)), sdesc_step(qa, ofs_kmaj(k + 3)), sdesc_step(ka, ofs_kmaj(k)),
                        sdesc_step(ka, ofs_kmaj(k + 1)), sdesc_step(ka, ofs_kmaj(k + 2)),
                        sdesc_step(ka, ofs_kmaj(k + 3)), idesc_qk, k > 0, leader);
          }
          mma_commit(&bars->s_full[t], leader);
        };
        // Half h of P V: keys [64h, 64h + 64).
        auto issue_pv = [&](int t, int j, int h) {
          const uint64_t va = sdesc_step(dV, (j % VS) * C::kTileBytes);
          // P: KSTEP keys per step = 8 tensor-memory columns (bf16 pairs or e4m3
          // quads); V: KSTEP key rows of 128 bytes (MN-major).
          constexpr int KH = kBN / KSTEP / 2;
          if constexpr (F8) {
    #pragma unroll
            for (int k = h * KH; k < h * KH + KH; ++k)
              mma_ts_f8(tO[t], tP[t] + k * 8, sdesc_step(va, k * KSTEP * 128), idesc_pv, (j > 0 || k > 0) ? 1u : 0u,
                        leader);
          } else {
            static_assert(F8 || KH == 4, "one group of four MMAs per half");
            const int k = h * KH;
            mma_ts_x4(tO[t], tP[t] + k * 8, tP[t] + (k + 1) * 8, tP[t] + (k + 2) * 8, tP[t] + (k + 3) * 8,
                      sdesc_step(va, k * KSTEP * 128), sdesc_step(va, (k + 1) * KSTEP * 128),
                      sdesc_step(va, (k + 2) * KSTEP * 128), sdesc_step(va, (k + 3) * KSTEP * 128), idesc_pv,
                      (j > 0 || k > 0) ? 1u : 0u, leader);
          }
        };
        const int n0 = n_t[0], n1 = n_t[1];
        bool ok = all(wait_bar(&bars->q_full, 0, w)) && all(wait_bar(&bars->k_full[0], 0, w));
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          if constexpr (T == 2) issue_s(1, 0);
          mma_commit(&bars->k_empty[0], leader);  // K_0 read by the S products
        }
        // One-tile form, P over S (FP8): this tile's P V, then S of the next
        // key tile over the P it has consumed.
        for (int j = 0; T == 1 && !SEP && ok && j < n0; ++j) {
          const int s = j % VS;
          const uint32_t par = (j / VS) & 1;
          const int jn = j + 1;
          if (!(ok = all(wait_bar(&bars->p_ready[0][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
          tc_fence_after();
          issue_pv(0, j, 0);
          if (!(ok = all(wait_bar(&bars->p_ready[0][1], j & 1, w)))) break;
          tc_fence_after();
          issue_pv(0, j, 1);
          mma_commit(&bars->v_empty[s], leader);
          if (j == n0 - 1) mma_commit(&bars->o_final[0], leader);
          if (jn < n0) {
            if (!(ok = all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w)))) break;
            issue_s(0, jn);
            mma_commit(&bars->k_empty[jn % KS], leader);
          }
        }
        // One-tile form, separate P (d = 64): S of the next key tile once the
        // softmax has loaded this one, then this tile's P V.
        for (int j = 0; T == 1 && SEP && ok && j < n0; ++j) {
          const int s = j % VS;
          const uint32_t par = (j / VS) & 1;
          const int jn = j + 1;
          if (jn < n0) {
            if (!(ok = all(wait_bar(&bars->s_free[0], j & 1, w)) && all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w))))
              break;
            tc_fence_after();
            issue_s(0, jn);
            mma_commit(&bars->k_empty[jn % KS], leader);
          }
          if (!(ok = all(wait_bar(&bars->p_ready[0][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
          tc_fence_after();
          issue_pv(0, j, 0);
          if (!(ok = all(wait_bar(&bars->p_ready[0][1], j & 1, w)))) break;
          tc_fence_after();
          issue_pv(0, j, 1);
          mma_commit(&bars->pv_done[0], leader);
          mma_commit(&bars->v_empty[s], leader);
          if (j == n0 - 1) mma_commit(&bars->o_final[0], leader);
        }
        for (int j = 0; T == 2 && ok && j < n1; ++j) {
          const int s = j % VS;                   // V_j stage
          const uint32_t par = (j / VS) & 1;
          const int jn = j + 1;
          if constexpr (SEP) {
            // S_t of tile j + 1 as soon as the softmax has loaded S_t of tile
            // j; then this tile's P V. pv_done tells the softmax when P_t and
            // O_t may be written again.
            if (j < n0) {
              if (jn < n0) {
                if (!(ok = all(wait_bar(&bars->s_free[0], j & 1, w)) && all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w))))
                  break;
                tc_fence_after();
                issue_s(0, jn);
              }
              if (!(ok = all(wait_bar(&bars->p_ready[0][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
              tc_fence_after();
              issue_pv(0, j, 0);
              if (!(ok = all(wait_bar(&bars->p_ready[0][1], j & 1, w)))) break;
              tc_fence_after();
              issue_pv(0, j, 1);
              mma_commit(&bars->pv_done[0], leader);
              if (j == n0 - 1) mma_commit(&bars->o_final[0], leader);
            }
            if (jn < n1) {
              if (!(ok = all(wait_bar(&bars->s_free[1], j & 1, w)) && all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w))))
                break;
              tc_fence_after();
              issue_s(1, jn);
              mma_commit(&bars->k_empty[jn % KS], leader);
            }
            if (!(ok = all(wait_bar(&bars->p_ready[1][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
            tc_fence_after();
            issue_pv(1, j, 0);
            if (!(ok = all(wait_bar(&bars->p_ready[1][1], j & 1, w)))) break;
            tc_fence_after();
            issue_pv(1, j, 1);
            mma_commit(&bars->pv_done[1], leader);
            mma_commit(&bars->v_empty[s], leader);
            if (j == n1 - 1) mma_commit(&bars->o_final[1], leader);
            continue;
          }
          if (j < n0) {
            if (!(ok = all(wait_bar(&bars->p_ready[0][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
            tc_fence_after();
            issue_pv(0, j, 0);
            if (!(ok = all(wait_bar(&bars->p_ready[0][1], j & 1, w)))) break;
            tc_fence_after();
            issue_pv(0, j, 1);
            if (j == n0 - 1) mma_commit(&bars->o_final[0], leader);
            if (jn < n0) {
              if (!(ok = all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w)))) break;
              issue_s(0, jn);
            }
          }
          if (!(ok = all(wait_bar(&bars->p_ready[1][0], j & 1, w)) && all(wait_bar(&bars->v_full[s], par, w)))) break;
          tc_fence_after();
          issue_pv(1, j, 0);
          if (!(ok = all(wait_bar(&bars->p_ready[1][1], j & 1, w)))) break;
          tc_fence_after();
          issue_pv(1, j, 1);
          mma_commit(&bars->v_empty[s], leader);
          if (j == n1 - 1) mma_commit(&bars->o_final[1], leader);
          if (jn < n1) {
            if (!(ok = all(wait_bar(&bars->k_full[jn % KS], (jn / KS) & 1, w)))) break;
            issue_s(1, jn);
            mma_commit(&bars->k_empty[jn % KS], leader);
          }
        }
        // All MMAs issued by this thread must finish before tensor memory is freed.
        mma_commit(&bars->drain, leader);
        all(drain_bar(&bars->drain, 0, w));
      }
    }
  } else {
    if constexpr (T == 1) regs_inc<kSoftmaxRegs1>();
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;                   // Q tile of this warpgroup
    const int quad = warp & 3;                 // tensor-memory lane quadrant
    const int r = quad * 32 + lane;            // row within the tile
    const int row = q0 + t * kBM + r;          // query position
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128u;
    const uint32_t tPw = SEP ? tmem + lane_off + C::kColP + t * 64u : tS;  // where this tile's P goes
    const uint32_t tO = tmem + lane_off + C::kColO + t * D;
    const int n = n_t[t];
    // FP8 mode: the scores come out of the MMA in units of sq * sk (the Q
    // tile's and the K tile's block scales); both fold into the exponent's
    // scale, per tile.
    // (The second tile of the last pair may start past N; its rows are never
    // written, and its block index is clamped into the scale array.)
    const float sl2_q =
        F8 ? a.scale_log2 * a.f8.sq[static_cast<size_t>(bh) * a.nk + min((q0 + t * kBM) / kBM, a.nk - 1)]
           : a.scale_log2;
    const int lim = MASK == 1 ? min(row, a.N - 1) : a.N - 1;  // last visible key (kinds 0, 1)
    const int qt0 = q0 + t * kBM;                               // first query of this tile
    float m = -CUDART_INF_F;  // running max of scale*log2(e)*s
    float l = 0.f;            // running sum, relative to m
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, wait_bar(&bars->s_full[t], j & 1, w));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kBN];
      // (With the register split, no instruction may name more than 64
      // destination registers.)
      if constexpr (T == 1)
        tmem_ld64x2(tS, sr);
      else
        tmem_ld128(tS, sr);
      if constexpr (SEP) {
        // S_t is in registers: the MMA thread may compute the next tile's S_t.
        tc_fence_before();
        mbar_arrive(&bars->s_free[t]);
      }
      const float sl2 = F8 ? sl2_q * a.f8.sk[static_cast<size_t>(kvh) * a.nk + key_tile(j)] : sl2_q;
      if (MASK != 2) {
        if (j == n - 1) {
          const int k0 = j * kBN;
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (k0 + i > lim) sr[i] = __float_as_uint(-CUDART_INF_F);
        }
      } else {
        const int k0 = key_tile(j) * kBN;
        // Tile visible to every row of this Q tile: all inside the prefix, or
        // below every row's diagonal and inside every row's window.
        const bool full = (k0 + kBN <= a.N) &&
                          ((k0 + kBN <= a.prefix) || (k0 + kBN - 1 <= qt0 && qt0 + kBM - 1 - k0 <= a.window));
        if (!full) {
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (k0 + i >= a.N || !visible2(row, k0 + i, a.window, a.prefix)) sr[i] = __float_as_uint(-CUDART_INF_F);
        }
      }
      // Row max as 8 independent partial maxima of three-input max
      // instructions (a linear chain would put 127 dependent instructions on
      // the softmax's critical path).
      static_assert(kBN % 16 == 0, "the partial maxima take 16 columns per step");
      float pm[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) pm[u] = fmaxf(__uint_as_float(sr[u]), __uint_as_float(sr[8 + u]));
#pragma unroll
      for (int i = 16; i < kBN; i += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          pm[u] = fmax3(pm[u], __uint_as_float(sr[i + u]), __uint_as_float(sr[i + 8 + u]));
      pm[0] = fmax3(pm[0], pm[1], pm[2]);
      pm[3] = fmax3(pm[3], pm[4], pm[5]);
      pm[6] = fmaxf(pm[6], pm[7]);
      const float m_cand = fmax3(pm[0], pm[3], pm[6]) * sl2;
      // Warp-uniform: rescale O when some row of the warp has a new max.
      bool rescale = false;
      float alpha = 1.f;
      if (j == 0) {
        m = m_cand;  // -inf for a row with no visible key yet (mask kind 2)
      } else if (__any_sync(0xffffffffu, m_cand > m + a.rescale_tau)) {
        const float m_new = fmaxf(m, m_cand);
        // On the FMA pipe: an ex2 here would queue behind the other tile's
        // exponentials on the exponential unit.
        alpha = (MASK == 2 && m_new == -CUDART_INF_F) ? 1.f : exp2_accurate(m - m_new);
        m = m_new;
        l *= alpha;
        rescale = true;
      }
      // A row with no visible key so far has m = -inf: its masked scores
      // must give exp(-inf) = 0, not exp(-inf + inf).
      // FP8 mode writes P as e4m3 of 2^kF8Offset p (headroom against
      // underflow, exact to undo): the offset rides on the exponent.
      const float neg_m = ((MASK == 2 && m == -CUDART_INF_F) ? 0.f : -m) + (F8 ? kF8Offset : 0.f);
      if constexpr (SEP) {
        // P_t and O_t of the previous key tile must have passed through P V
        // before this tile's P overwrites P_t or O_t is rescaled.
        if (j > 0) {
          ok = __all_sync(0xffffffffu, wait_bar(&bars->pv_done[t], (j - 1) & 1, w));
          if (!ok) break;
          tc_fence_after();
        }
      }
      float ps[8];  // 8 independent partial row sums
#pragma unroll
      for (int u = 0; u < 8; ++u) ps[u] = 0.f;
      // P goes to tensor memory in two halves of 64 keys. The first half is
      // released to the MMA thread (after the O rescale, which must precede
      // any of this tile's P V) while the second half's exponentials run, so
      // half of P V overlaps the softmax.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if constexpr (F8) {
          // 64 scores -> 16 columns of four e4m3 each.
          const int c = h;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float p4[4];
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              float x0, x1;
              ffma2(x0, x1, __uint_as_float(sr[c * 64 + 4 * i + e]), __uint_as_float(sr[c * 64 + 4 * i + e + 1]),
                    sl2, sl2, neg_m, neg_m);
              p4[e] = (((4 * i + e) & 15) < kPolyPer16F8) ? exp2_poly(x0) : ex2(x0);
              p4[e + 1] = (((4 * i + e + 1) & 15) < kPolyPer16F8) ? exp2_poly(x1) : ex2(x1);
              fadd2(ps[(4 * i + e) & 7], ps[(4 * i + e + 1) & 7], ps[(4 * i + e) & 7], ps[(4 * i + e + 1) & 7],
                    p4[e], p4[e + 1]);
            }
            pk[i] = pack_e4m3x4(p4[0], p4[1], p4[2], p4[3]);
          }
          tmem_st16(tPw + c * 16, pk);
        } else {
#pragma unroll
          for (int c = 2 * h; c < 2 * h + 2; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              // Exponent arguments and partial sums two at a time (packed
              // f32x2: half the FMA and add instructions of the scalar form).
              float x0, x1;
              ffma2(x0, x1, __uint_as_float(sr[c * 32 + 2 * i]), __uint_as_float(sr[c * 32 + 2 * i + 1]), sl2,
                    sl2, neg_m, neg_m);
              constexpr int kPoly = poly_per32<D, MASK>();
              const float p0 = (2 * i < kPoly) ? exp2_poly(x0) : ex2(x0);
              const float p1 = (2 * i + 1 < kPoly) ? exp2_poly(x1) : ex2(x1);
              fadd2(ps[(2 * i) & 7], ps[(2 * i + 1) & 7], ps[(2 * i) & 7], ps[(2 * i + 1) & 7], p0, p1);
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tPw + c * 16, pk);
          }
        }
        if (h == 0 && rescale) {
          // O holds every earlier product (see the ordering argument above);
          // scale this row by alpha before P V is added to it, two columns
          // per packed multiply. d = 64: one tensor-memory round trip (two
          // loads, one wait); d = 128: 32 columns per round trip (64 would
          // spill, with 64 scores still live here).
          if constexpr (D == 64) {
            uint32_t oo[64];
            uint32_t(&o0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&oo[0]);
            uint32_t(&o1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&oo[32]);
            tmem_ld32_nowait(tO, o0);
            tmem_ld32_nowait(tO + 32, o1);
            tmem_ld_wait(o0);
            tmem_ld_tie(o1);
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
              float y0, y1;
              fmul2(y0, y1, __uint_as_float(oo[i]), __uint_as_float(oo[i + 1]), alpha, alpha);
              oo[i] = __float_as_uint(y0);
              oo[i + 1] = __float_as_uint(y1);
            }
            tmem_st32(tO, o0);
            tmem_st32(tO + 32, o1);
          } else {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o32[32];
              tmem_ld32(tO + c * 32, o32);
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                float y0, y1;
                fmul2(y0, y1, __uint_as_float(o32[i]), __uint_as_float(o32[i + 1]), alpha, alpha);
                o32[i] = __float_as_uint(y0);
                o32[i + 1] = __float_as_uint(y1);
              }
              tmem_st32(tO + c * 32, o32);
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready[t][h]);
      }
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(&bars->o_final[t], 0, w));
    if (ok) {
      tc_fence_after();
      // FP8 mode: l sums 2^kF8Offset p, O sums the same weights times V's
      // codes; V's head scale turns codes into values.
      const float inv_l = F8 ? a.f8.sv[kvh] / l : 1.f / l;
      if constexpr (!F8) {
        // O (then its residual) leaves through two staging boxes (the Q_t
        // buffer, which no MMA reads any more, where it is large enough):
        // each job is one 64-column box of 128 rows, written by the rows'
        // threads in the tensor map's 128-byte swizzle and stored by one TMA
        // copy, so that global memory sees whole lines (one thread per row
        // storing its own row writes half sectors; measured on B200 the
        // staged form takes ~6000 cycles off each CTA's epilogue at d = 128
        // with the residual). Rows past N are clipped by the copy; a tile
        // that starts past N has no job.
        constexpr int kBoxesO = D / 64;  // bf16 output boxes
        constexpr int kSlots = 2;        // 16-KB boxes staged at a time
        const int jobs = qt0 < a.N ? kBoxesO * (a.o_resid ? 2 : 1) : 0;
        // Box i of this tile stages in slot i % 2: two boxes of the own region
        // or of the Q_t buffer; in the one-tile form the Q buffer, then the
        // own box.
        uint8_t* const slots[2] = {
            T == 1 ? smem + C::kOffQ : (C::kOwnStage ? smem + C::kOffStage + t * 2 * 16384 : smem + C::kOffQ + t * C::kTileBytes),
            T == 1 ? smem + C::kOffStage
                   : (C::kOwnStage ? smem + C::kOffStage + t * 2 * 16384 : smem + C::kOffQ + t * C::kTileBytes) + 16384};
        const bool issuer = r == 0;
        for (int i = 0; i < jobs; ++i) {
          const int x = i % kBoxesO;
          const bool resid = i >= kBoxesO;
          uint8_t* slot = slots[i % kSlots];
          // The slot's previous box must have been read by its copy.
          if (i >= kSlots && !(ok = __all_sync(0xffffffffu, wait_bar(&bars->epi_free[t], (i - kSlots) & 1, w)))) break;
          uint32_t oo[64];
          uint32_t(&o0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&oo[0]);
          uint32_t(&o1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&oo[32]);
          tmem_ld32_nowait(tO + x * 64, o0);
          tmem_ld32_nowait(tO + x * 64 + 32, o1);
          tmem_ld_wait(o0);
          tmem_ld_tie(o1);
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint4 v;
            uint32_t* pv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(oo[8 * cc + 2 * e]) * inv_l;
              const float x1 = __uint_as_float(oo[8 * cc + 2 * e + 1]) * inv_l;
              pv[e] = pack_bf16x2(x0, x1);
              if (resid) {
                const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&pv[e]);
                pv[e] = pack_bf16x2(x0 - __low2float(hi), x1 - __high2float(hi));
              }
            }
            *reinterpret_cast<uint4*>(slot + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
          }
          fence_proxy_async_smem();
          mbar_arrive(&bars->epi_full[t]);
          if (issuer) {
            if (!(ok = wait_bar(&bars->epi_full[t], i & 1, w))) break;
            tma_store_3d(resid ? &tmR : &tmO, slot, x * 64, qt0, bh);
            bulk_commit();
            if (i + 1 < jobs && i + 1 >= kSlots) {
              bulk_wait_read<kSlots - 1>();
              mbar_arrive(&bars->epi_free[t]);
            }
          }
        }
        // The copies must have read the staged boxes before the CTA exits.
        if (issuer) bulk_wait_read<0>();
      } else {
        // FP8 mode (no residual): one thread per row stores its own row
        // (measured on B200: staging costs 1 to 2% here).
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (static_cast<size_t>(bh) * a.N + row) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t oo[32];
          tmem_ld32(tO + c * 32, oo);
          uint4 v[4];
          uint32_t* pv = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pv[i] = pack_bf16x2(__uint_as_float(oo[2 * i]) * inv_l, __uint_as_float(oo[2 * i + 1]) * inv_l);
          if (row < a.N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = v[i];
          }
        }
      }
      if (row < a.N)
        a.lse[static_cast<size_t>(bh) * a.N + row] = (m + lg2(l) - (F8 ? kF8Offset : 0.f)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// 128-byte rows (d = 64 in bf16, the FP8 mode) take the one-tile form (two
// CTAs per SM).
template <int D, int MASK, bool F8 = false, int T = (D * (F8 ? 1 : 2) == 128) ? 1 : 2>
cudaError_t launch_fwd_t(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& to, const CUtensorMap& tr, void* o, void* o_resid, float* lse,
                         const LaunchCtl& ctl, cudaStream_t stream,
                         Fp8Scales f8 = Fp8Scales{nullptr, nullptr, nullptr}) {
  using C = FwdCfg<D, F8, T>;
  auto kern = fwd_kernel<D, MASK, F8, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  if constexpr (T == 1) {
    // The register split (setmaxnreg) hands out exactly what a launch at 128
    // registers per thread gives the CTA; with any other count the softmax
    // warps' increase could never be granted.
    static const int launch_regs = [&] {
      cudaFuncAttributes at{};
      return cudaFuncGetAttributes(&at, kern) == cudaSuccess ? at.numRegs : -1;
    }();
    if (launch_regs != 128) return cudaErrorLaunchOutOfResources;
  }
  FwdArgs a;
  a.o = o;
  a.o_resid = o_resid;
  a.lse = lse;
  a.N = s.N;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.BH = s.B * s.Hq;
  a.nk = (s.N + kBN - 1) / kBN;
  a.n_pairs = (s.N + T * kBM - 1) / (T * kBM);  // units per head
  // Causal units differ in length: keep strict longest-first order over all
  // heads. Non-causal units are equal: group heads for L2 locality.
  a.group = MASK == 1 ? a.BH
                      : l2_head_group(static_cast<long long>(2 * C::kElem) * s.N * D / (s.Hq / s.Hkv), a.BH);
  a.window = s.window < 0 ? 0x3fffffff : s.window;
  a.prefix = s.prefix;
  a.scale_log2 = s.scale * 1.4426950408889634f;
  a.rescale_tau = F8 ? kF8Rescale : (o_resid ? kRescaleExact : kRescaleLazy);
  a.f8 = f8;
  a.ctl = ctl;
  const long long grid = static_cast<long long>(a.n_pairs) * a.BH;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  kern<<<static_cast<unsigned>(grid), C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, tr, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const CUtensorMap& tr, void* o, void* o_resid, float* lse,
                       const LaunchCtl& ctl, cudaStream_t stream) {
#define FA_FWD_ARGS s, tq, tk, tv, to, tr, o, o_resid, lse, ctl, stream
  switch (s.mask_kind() + (s.d == 64 ? 0 : 3)) {
    case 0: return launch_fwd_t<64, 0>(FA_FWD_ARGS);
    case 1: return launch_fwd_t<64, 1>(FA_FWD_ARGS);
    case 2: return launch_fwd_t<64, 2>(FA_FWD_ARGS);
    case 3: return launch_fwd_t<128, 0>(FA_FWD_ARGS);
    case 4: return launch_fwd_t<128, 1>(FA_FWD_ARGS);
    default: return launch_fwd_t<128, 2>(FA_FWD_ARGS);
  }
#undef FA_FWD_ARGS
}

cudaError_t launch_fwd_fp8(const AttnShape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, void* o, float* lse, const float* sq, const float* sk,
                           const float* sv, const LaunchCtl& ctl, cudaStream_t stream) {
  if (s.d != 128 || s.mask_kind() == 2) return cudaErrorInvalidValue;
  const Fp8Scales f8{sq, sk, sv};
  if (s.causal) return launch_fwd_t<128, 1, true>(s, tq, tk, tv, to, to, o, nullptr, lse, ctl, stream, f8);
  return launch_fwd_t<128, 0, true>(s, tq, tk, tv, to, to, o, nullptr, lse, ctl, stream, f8);
}

}  // namespace fa
