// fb_attn_sm100.cu -- fused forward of attention with an additive bias on
// B200 (sm_100a): TMA -> shared memory -> tcgen05 MMA -> TMEM -> softmax on
// the CUDA cores -> tcgen05 MMA -> TMEM -> HBM.
//
// Method: FlashBias (arXiv 2505.12044). The bias b = phi_q phi_k^T joins the
// QK^T tile product: q' = [q, phi_q], k' = [k, phi_k] gives q'k'^T = qk^T +
// phi_q phi_k^T (rebuttal, reply to Reviewer UJUf, Q2, "Eq. (3) of main
// text"). Here the concatenation is never formed: the Q tile and the phi_q
// tile sit in two shared-memory tiles and the two MMAs (bf16 QK^T, then fp16
// phi_q' phi_k^T with phi_q' = phi_q / scale) accumulate into one fp32 TMEM
// accumulator, so the N x N bias is never read or written (Figure 2). For
// rank <= 4 (the ALiBi factors, Example 3.4) the factor tile is created next
// to the scores on the CUDA cores in fp32 instead, as the rebuttal describes
// for ALiBi (reply to Reviewer BRmd, Q2 (2): Block x 2 factor tiles made "in
// JIT"). The dense mode streams a materialised bias tile per tile pair: the
// "FlashAttention w/ Bias" comparison path of Figure 1(c).
//
// CTA organisation (QT = 1 or 2 query tiles of 128 rows per CTA):
//   warps 0..4QT-1  softmax warpgroups; warpgroup t owns query tile t, one
//                   thread per row (TMEM lane), so row max and row sum are
//                   thread-local; it also rescales O in TMEM when the running
//                   max grows by more than 2^8 and writes the epilogue.
//   warp 4QT        TMA producer (one thread): Q|phi_q once, then K|phi_k and
//                   V per 128-key step into a KS-deep ring, plus the
//                   softmax-side tiles (dense bias / rank<=4 factors).
//   warp 4QT+1      TMEM allocator and MMA issuer (one elected lane).
// TMEM columns: S_t at 128 t, O_t at 128 QT + 128 t; P_t (bf16) overwrites
// the first 64 columns of S_t and feeds the PV MMA as the TMEM A operand.
// MMA issue order per key step i: S_0(i), PV_1(i-1), S_1(i), PV_0(i), so the
// tensor core works on one tile while the softmax of the other runs. With
// that order the commit that publishes S_t(i) also covers PV_t(i-1), so the
// softmax may rescale O_t right after seeing S_t(i), and S_t(i+1) (which
// overwrites P_t(i)) is issued after PV_t(i) (tcgen05 MMAs of one thread run
// in order).
#include <algorithm>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8
// Of every 16 element pairs of P, this many get exp2 from the packed FMA-pipe
// polynomial (ex2_fma_pair) and the rest from the MUFU unit, which balances
// the MUFU against the issue slots of the two softmax warps per scheduler.
constexpr int kEmuPairs = 4;
constexpr uint32_t kSmemLimit = 227u * 1024u;

template <int DP, int RP, int MODE, int QT>
struct Sm100Cfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int DCH = DP > 64 ? 64 : DP;  // columns per TMA box / swizzle atom
  static constexpr int NDCH = DP / DCH;
  static constexpr int RCH = (MODE == kBiasMma) ? (RP > 64 ? 64 : RP) : 16;
  static constexpr int NRCH = (MODE == kBiasMma) ? RP / RCH : 0;
  static constexpr uint32_t Q_TILE = BM * DP * 2;
  static constexpr uint32_t KV_TILE = BN * DP * 2;
  static constexpr uint32_t FQ_TILE = MODE == kBiasMma ? BM * RP * 2 : 0;
  static constexpr uint32_t FK_TILE = MODE == kBiasMma ? BN * RP * 2 : 0;
  static constexpr uint32_t AUX_TILE = MODE == kBiasReg ? BN * 16 : (MODE == kBiasDense ? BM * BN * 2 : 0);
  static constexpr bool HAS_AUX = AUX_TILE > 0;
  static constexpr uint32_t FIXED = QT * (Q_TILE + FQ_TILE);
  static constexpr uint32_t STAGE = 2 * KV_TILE + FK_TILE + QT * AUX_TILE;
  static constexpr uint32_t CTRL = 1024;  // barriers + TMEM address + abort flag
  static constexpr uint32_t ALIGN_SLACK = 1024;
  static constexpr int KS_FIT = (kSmemLimit > FIXED + CTRL + ALIGN_SLACK)
                                    ? int((kSmemLimit - FIXED - CTRL - ALIGN_SLACK) / STAGE)
                                    : 0;
  static constexpr int KS = KS_FIT > 3 ? 3 : KS_FIT;
  static constexpr uint32_t SMEM = FIXED + uint32_t(KS) * STAGE + CTRL + ALIGN_SLACK;
  // QT softmax warpgroups + one warpgroup holding the producer warp, the MMA
  // warp and two idle warps. Registers are moved from that warpgroup to the
  // softmax warpgroups with setmaxnreg: the launch allocation is
  // THREADS * LAUNCH_REGS and the shares below add up to exactly that.
  static constexpr int THREADS = QT * 128 + 128;
  static constexpr int MIN_BLOCKS = QT == 1 ? 2 : 1;
  static constexpr int LAUNCH_REGS = QT == 1 ? 128 : 168;
  static constexpr int REG_SOFTMAX = QT == 1 ? 208 : 216;
  static constexpr int REG_OTHER = QT == 1 ? 48 : 72;
  static_assert(QT * 128 * REG_SOFTMAX + 128 * REG_OTHER == THREADS * LAUNCH_REGS, "register split");
  static constexpr int PRODUCER_WARP = QT * 4;
  static constexpr int MMA_WARP = QT * 4 + 1;
  static constexpr uint32_t TMEM_COLS = QT == 2 ? 512 : 256;
  // With DP <= 64 the bf16 P tile gets its own 64 TMEM columns, so S(i+1)
  // can be computed while the softmax of S(i) is still running; with DP = 128
  // P overwrites the first 64 columns of S.
  static constexpr bool SEP_P = DP <= 64;
  static constexpr uint32_t S_COL0 = 0;                                // + 128 t
  static constexpr uint32_t P_COL0 = SEP_P ? 128 * QT : 0;             // + (SEP_P ? 64 : 128) t
  static constexpr uint32_t P_STRIDE = SEP_P ? 64 : 128;
  static constexpr uint32_t O_COL0 = SEP_P ? 128 * QT + 64 * QT : 128 * QT;  // + O_STRIDE t
  static constexpr uint32_t O_STRIDE = SEP_P ? DP : 128;
  static_assert(O_COL0 + O_STRIDE * QT <= TMEM_COLS, "TMEM layout");
  // MMA issuer warps (one per query tile with separate P, else one), each of
  // which releases every K/V stage once per key step.
  static constexpr int RELEASERS = SEP_P ? QT : 1;
  static constexpr uint32_t IDESC_QK = make_idesc_f16(true, true, 128, 128, false);
  static constexpr uint32_t IDESC_F = make_idesc_f16(false, false, 128, 128, false);
  static constexpr uint32_t IDESC_PV = make_idesc_f16(true, true, 128, DP, true);
};

struct SmemCtrl {
  uint64_t q_full;
  uint64_t o_final[2];
  uint64_t drain[2];
  uint64_t s_free[2], pv_done[2];  // separate-P schedule only
  uint64_t k_full[3], v_full[3];
  uint64_t k_empty[3], v_empty[3];  // one arrival per MMA issuer per key step
  uint64_t s_full[2], p_full[2];
  uint64_t aux_full[2][3], aux_empty[2][3];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(SmemCtrl) <= 1024, "control block too large");

// K-major tile of 128 rows x (NCH * CH) 16-bit elements, stored as NCH
// swizzled column chunks of CH elements: descriptor of the chunk base, and
// the start-address offset (in 16-byte units) of the 16-column MMA step kk.
template <int CH>
__device__ __forceinline__ uint64_t desc_kmajor_base(uint32_t base) {
  return make_smem_desc(base, 16, 8 * CH * 2, swizzle_code(CH * 2));
}
template <int CH>
__host__ __device__ constexpr uint32_t kmajor_step(int kk) {
  return uint32_t((kk / (CH / 16)) * (128 * CH * 2) + (kk % (CH / 16)) * 32) >> 4;
}

// V tile, [128 keys] x (NCH * CH) values, as the MN-major B operand of the PV
// MMA: descriptor of the tile base and the offset of the 16-key step kk.
template <int CH>
__device__ __forceinline__ uint64_t desc_v_base(uint32_t base) {
  return make_smem_desc(base, 128 * CH * 2, 8 * CH * 2, swizzle_code(CH * 2));
}
template <int CH>
__host__ __device__ constexpr uint32_t v_step(int kk) {
  return uint32_t(kk * 16 * CH * 2) >> 4;
}

template <int DP, int RP, int MODE, int QT>
__global__ void __launch_bounds__(Sm100Cfg<DP, RP, MODE, QT>::THREADS, Sm100Cfg<DP, RP, MODE, QT>::MIN_BLOCKS)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_fq,
                   const __grid_constant__ CUtensorMap tm_fk, const __grid_constant__ CUtensorMap tm_bias,
                   const FwdArgs args) {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  constexpr int KS = C::KS;
  static_assert(KS >= 1, "configuration does not fit in shared memory");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                                     // QT x Q_TILE
  uint8_t *sFQ = sQ + QT * C::Q_TILE;                     // QT x FQ_TILE
  uint8_t *sK = sFQ + QT * C::FQ_TILE;                    // KS x KV_TILE
  uint8_t *sFK = sK + KS * C::KV_TILE;                    // KS x FK_TILE
  uint8_t *sV = sFK + KS * C::FK_TILE;                    // KS x KV_TILE
  uint8_t *sAux = sV + KS * C::KV_TILE;                   // QT x KS x AUX_TILE
  SmemCtrl *ctrl = reinterpret_cast<SmemCtrl *>(sAux + QT * KS * C::AUX_TILE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int b = bh / args.H;
  const int h = bh - b * args.H;
  const int qg = args.n_cta_q - 1 - int(blockIdx.y);  // heaviest causal row groups first
  const int N = args.N;
  const int fb_slice = (args.fac_B > 1 ? b : 0) * args.fac_H + (args.fac_H > 1 ? h : 0);

  // Per query tile: first row and number of key tiles. Key tiles are visited
  // from the last one down (step i reads key tile n_steps - 1 - i), so for a
  // causal mask the diagonal comes first: biases that decay away from the
  // diagonal then set the running max at once and O is rarely rescaled. Tile
  // t is active for steps first[t] .. n_steps - 1 (its local step j = i -
  // first[t]); in causal attention tile 0 skips the first step.
  int q0[2], nk[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = qg * QT + t;
    q0[t] = qt * 128;
    const bool active = (t < QT) && (q0[t] < N);
    nk[t] = active ? (args.causal ? min(qt + 1, args.n_kv) : args.n_kv) : 0;
  }
  const int n_steps = max(nk[0], nk[1]);
  const int first[2] = {n_steps - nk[0], n_steps - nk[1]};

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctrl->k_full[s], 1);
      mbar_init(&ctrl->v_full[s], 1);
      mbar_init(&ctrl->k_empty[s], C::RELEASERS);
      mbar_init(&ctrl->v_empty[s], C::RELEASERS);
      for (int t = 0; t < QT; ++t) {
        mbar_init(&ctrl->aux_full[t][s], 1);
        mbar_init(&ctrl->aux_empty[t][s], 128);
      }
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 128);
      mbar_init(&ctrl->o_final[t], 1);
      mbar_init(&ctrl->drain[t], 1);
      mbar_init(&ctrl->s_free[t], 128);
      mbar_init(&ctrl->pv_done[t], 1);
    }
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(&ctrl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int *abort = &ctrl->abort;

  if (warp >= QT * 4) {
  setmaxnreg_dec<C::REG_OTHER>();
  // The producer and MMA warps run their loops with all 32 lanes so that
  // coordinates and descriptors stay warp-uniform; lane 0 alone issues each
  // TMA copy, expect-tx arrival, MMA and commit (predicated inside the asm).
  const uint32_t leader = lane == 0 ? 1u : 0u;
  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (leader) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      if (MODE == kBiasMma) {
        tma_prefetch_map(&tm_fq);
        tma_prefetch_map(&tm_fk);
      }
      if (MODE == kBiasReg) tma_prefetch_map(&tm_fk);
      if (MODE == kBiasDense) tma_prefetch_map(&tm_bias);
    }
    uint32_t qbytes = 0;
    for (int t = 0; t < QT; ++t)
      if (nk[t] > 0) qbytes += C::Q_TILE + C::FQ_TILE;
    mbar_arrive_expect_tx_leader(&ctrl->q_full, qbytes, leader);
    for (int t = 0; t < QT; ++t) {
      if (nk[t] == 0) continue;
      for (int ch = 0; ch < C::NDCH; ++ch)
        tma_load_3d_leader(sQ + t * C::Q_TILE + ch * (128 * C::DCH * 2), &tm_q, &ctrl->q_full, ch * C::DCH, q0[t], bh,
                           leader);
      if (MODE == kBiasMma)
        for (int ch = 0; ch < C::NRCH; ++ch)
          tma_load_3d_leader(sFQ + t * C::FQ_TILE + ch * (128 * C::RCH * 2), &tm_fq, &ctrl->q_full, ch * C::RCH,
                             q0[t], fb_slice, leader);
    }
    int hb = 0, bb = 0;
    if (MODE == kBiasDense) {
      hb = args.bias_H > 1 ? h : 0;
      bb = args.bias_B > 1 ? b : 0;
    }
    bool ok = true;
    for (int i = 0; i < n_steps && ok; ++i) {
      const int s = i % KS;
      const uint32_t ph = uint32_t(i / KS) & 1u;
      const int kv = (n_steps - 1 - i) * 128;  // first key of this step's tile
      // stage s last held step i - KS: wait until every issuer released it
      if (i >= KS && !(ok = mbar_wait(&ctrl->k_empty[s], ph ^ 1u, abort))) break;
      mbar_arrive_expect_tx_leader(&ctrl->k_full[s], C::KV_TILE + C::FK_TILE, leader);
      for (int ch = 0; ch < C::NDCH; ++ch)
        tma_load_3d_leader(sK + s * C::KV_TILE + ch * (128 * C::DCH * 2), &tm_k, &ctrl->k_full[s], ch * C::DCH, kv,
                           bh, leader);
      if (MODE == kBiasMma)
        for (int ch = 0; ch < C::NRCH; ++ch)
          tma_load_3d_leader(sFK + s * C::FK_TILE + ch * (128 * C::RCH * 2), &tm_fk, &ctrl->k_full[s], ch * C::RCH,
                             kv, fb_slice, leader);
      if (C::HAS_AUX) {
        for (int t = 0; t < QT; ++t) {
          const int j = i - first[t];  // the tile's local step; its own ring
          if (j < 0) continue;
          const int sa = j % KS;
          if (j >= KS && !(ok = mbar_wait(&ctrl->aux_empty[t][sa], (uint32_t(j / KS) & 1u) ^ 1u, abort))) break;
          uint8_t *dst = sAux + (t * KS + sa) * C::AUX_TILE;
          mbar_arrive_expect_tx_leader(&ctrl->aux_full[t][sa], C::AUX_TILE, leader);
          if (MODE == kBiasReg) {
            tma_load_3d_leader(dst, &tm_fk, &ctrl->aux_full[t][sa], 0, kv, fb_slice, leader);
          } else {
            tma_load_4d_leader(dst, &tm_bias, &ctrl->aux_full[t][sa], kv, q0[t], hb, bb, leader);
            tma_load_4d_leader(dst + 128 * 128, &tm_bias, &ctrl->aux_full[t][sa], kv + 64, q0[t], hb, bb, leader);
          }
        }
        if (!ok) break;
      }
      if (i >= KS && !(ok = mbar_wait(&ctrl->v_empty[s], ph ^ 1u, abort))) break;
      mbar_arrive_expect_tx_leader(&ctrl->v_full[s], C::KV_TILE, leader);
      for (int ch = 0; ch < C::NDCH; ++ch)
        tma_load_3d_leader(sV + s * C::KV_TILE + ch * (128 * C::DCH * 2), &tm_v, &ctrl->v_full[s], ch * C::DCH, kv,
                           bh, leader);
    }
    if (!ok) {
      // Aborted: let the copies already issued land before the CTA exits.
      for (int s = 0; s < KS; ++s) {
        mbar_wait_for(&ctrl->k_full[s], 0, 100000000ull);
        mbar_wait_for(&ctrl->k_full[s], 1, 100000000ull);
        mbar_wait_for(&ctrl->v_full[s], 0, 100000000ull);
        mbar_wait_for(&ctrl->v_full[s], 1, 100000000ull);
      }
      if (leader) atomicOr(args.flags, kFlagTimeout);
    }
  } else if (warp == C::MMA_WARP || (C::SEP_P && QT == 2 && warp == C::MMA_WARP + 1)) {
    // ---------------------------------------------------------- MMA issuer
    // Descriptors of every tile base, computed once; each MMA adds a
    // compile-time step offset (the start address is the low field, and
    // shared addresses >> 4 stay below 2^14, so plain adds cannot carry).
    const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
    const uint64_t dk0 = desc_kmajor_base<C::DCH>(smem_u32(sK));
    const uint64_t dfk0 = desc_kmajor_base<C::RCH>(smem_u32(sFK));
    const uint64_t dv0 = desc_v_base<C::DCH>(smem_u32(sV));
    auto issue_s = [&](int t, int s) {  // S_t = Q_t K_s^T (+ phi_q' phi_k^T)
      const uint32_t d_tm = tm_u + C::S_COL0 + uint32_t(128 * t);
      const uint64_t dq = desc_kmajor_base<C::DCH>(smem_u32(sQ + t * C::Q_TILE));
      const uint64_t dk = dk0 + uint64_t((uint32_t(s) * C::KV_TILE) >> 4);
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)
        mma_ss_elect(d_tm, dq + kmajor_step<C::DCH>(kk), dk + kmajor_step<C::DCH>(kk), C::IDESC_QK,
                     kk > 0 ? 1u : 0u);
      if (MODE == kBiasMma) {
        const uint64_t dfq = desc_kmajor_base<C::RCH>(smem_u32(sFQ + t * C::FQ_TILE));
        const uint64_t dfk = dfk0 + uint64_t((uint32_t(s) * C::FK_TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < (MODE == kBiasMma ? RP / 16 : 0); ++kk)
          mma_ss_elect(d_tm, dfq + kmajor_step<C::RCH>(kk), dfk + kmajor_step<C::RCH>(kk), C::IDESC_F, 1u);
      }
    };
    auto issue_pv = [&](int t, int s, bool acc) {  // O_t += P_t V_s, P_t read from TMEM
      const uint32_t d_tm = tm_u + C::O_COL0 + C::O_STRIDE * uint32_t(t);
      const uint32_t p_tm = tm_u + C::P_COL0 + C::P_STRIDE * uint32_t(t);
      const uint64_t dv = dv0 + uint64_t((uint32_t(s) * C::KV_TILE) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_elect(d_tm, p_tm + uint32_t(kk * 8), dv + v_step<C::DCH>(kk), C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
    };
    bool ok = mbar_wait(&ctrl->q_full, 0, abort);
    tc_fence_after();
    if constexpr (C::SEP_P) {
      // One issuer warp per query tile t: S_t(i+1) as soon as the softmax has
      // read S_t(i) into registers, PV_t(i) once P_t(i) is written. The two
      // tiles' chains are independent and share the tensor core. Every issuer
      // walks all key steps and releases each K/V stage once per step, also
      // for steps its tile does not use.
      const int t = warp - C::MMA_WARP;
      for (int i = 0; i < n_steps && ok; ++i) {
        const int s = i % KS;
        const uint32_t ph = uint32_t(i / KS) & 1u;
        const int j = i - first[t];
        if (j < 0) {
          if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
          tc_commit_elect(&ctrl->k_empty[s]);
          if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
          tc_commit_elect(&ctrl->v_empty[s]);
          continue;
        }
        if (j == 0) {
          if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
          tc_fence_after();
          issue_s(t, s);
          tc_commit_elect(&ctrl->s_full[t]);
          tc_commit_elect(&ctrl->k_empty[s]);
        }
        if (i + 1 < n_steps) {
          const int s1 = (i + 1) % KS;
          if (!(ok = mbar_wait(&ctrl->k_full[s1], uint32_t((i + 1) / KS) & 1u, abort))) break;
          if (!(ok = mbar_wait(&ctrl->s_free[t], uint32_t(j) & 1u, abort))) break;
          tc_fence_after();
          issue_s(t, s1);
          tc_commit_elect(&ctrl->s_full[t]);
          tc_commit_elect(&ctrl->k_empty[s1]);
        }
        if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
        if (!(ok = mbar_wait(&ctrl->p_full[t], uint32_t(j) & 1u, abort))) break;
        tc_fence_after();
        issue_pv(t, s, j > 0);
        tc_commit_elect(&ctrl->pv_done[t]);
        tc_commit_elect(&ctrl->v_empty[s]);
      }
      tc_commit_elect(&ctrl->o_final[t]);
      if (!ok) {
        tc_commit_elect(&ctrl->drain[t]);
        mbar_wait_for(&ctrl->drain[t], 0, 100000000ull);
        if (leader) atomicOr(args.flags, kFlagTimeout);
      }
    } else {
      // One issuer for both tiles, in the order S_0(i), PV_1(i-1), S_1(i),
      // PV_0(i) (P overwrites S, so S_t(i+1) must follow PV_t(i)).
      auto act = [&](int t, int i) { return t < QT && i >= first[t] && i < n_steps; };
      for (int i = 0; i < n_steps && ok; ++i) {
        const int s = i % KS;
        const uint32_t ph = uint32_t(i / KS) & 1u;
        if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
        tc_fence_after();
        if (act(0, i)) {
          issue_s(0, s);
          tc_commit_elect(&ctrl->s_full[0]);
        }
        if (QT == 2) {
          const int ip = i - 1;  // PV of tile 1 for the previous step
          if (act(1, ip)) {
            const int sp = ip % KS;
            const uint32_t php = uint32_t(ip / KS) & 1u;
            if (!act(0, ip) && !(ok = mbar_wait(&ctrl->v_full[sp], php, abort))) break;
            if (!(ok = mbar_wait(&ctrl->p_full[1], uint32_t(ip - first[1]) & 1u, abort))) break;
            tc_fence_after();
            issue_pv(1, sp, ip > first[1]);
            tc_commit_elect(&ctrl->v_empty[sp]);
          }
          if (act(1, i)) {
            issue_s(1, s);
            tc_commit_elect(&ctrl->s_full[1]);
          }
        }
        tc_commit_elect(&ctrl->k_empty[s]);
        if (act(0, i)) {
          if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
          if (!(ok = mbar_wait(&ctrl->p_full[0], uint32_t(i - first[0]) & 1u, abort))) break;
          tc_fence_after();
          issue_pv(0, s, i > first[0]);
          if (!act(1, i)) tc_commit_elect(&ctrl->v_empty[s]);
        } else if (!act(1, i)) {
          tc_commit_elect(&ctrl->v_empty[s]);  // no tile used this step's V
        }
      }
      if (ok && act(1, n_steps - 1)) {
        const int ip = n_steps - 1;
        const int sp = ip % KS;
        const uint32_t php = uint32_t(ip / KS) & 1u;
        ok = act(0, ip) || mbar_wait(&ctrl->v_full[sp], php, abort);
        ok = ok && mbar_wait(&ctrl->p_full[1], uint32_t(ip - first[1]) & 1u, abort);
        if (ok) {
          tc_fence_after();
          issue_pv(1, sp, ip > first[1]);
          tc_commit_elect(&ctrl->v_empty[sp]);
        }
      }
      for (int t = 0; t < QT; ++t) tc_commit_elect(&ctrl->o_final[t]);
      if (!ok) {
        // Aborted: wait (bounded) for the MMAs already issued to finish.
        tc_commit_elect(&ctrl->drain[0]);
        mbar_wait_for(&ctrl->drain[0], 0, 100000000ull);
        if (leader) atomicOr(args.flags, kFlagTimeout);
      }
    }
  }
  } else {
    setmaxnreg_inc<C::REG_SOFTMAX>();
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;  // TMEM lane quarter
    const int r_loc = wq * 32 + lane;
    const int row = q0[t] + r_loc;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t s_tm = lane_base + C::S_COL0 + uint32_t(128 * t);
    const uint32_t p_tm = lane_base + C::P_COL0 + C::P_STRIDE * uint32_t(t);
    const uint32_t o_tm = lane_base + C::O_COL0 + C::O_STRIDE * uint32_t(t);
    const float sl2 = args.scale_log2;

    float aq0 = 0.f, aq1 = 0.f, aq2 = 0.f, aq3 = 0.f;
    if (MODE == kBiasReg && row < N) {
      const float4 v = *reinterpret_cast<const float4 *>(args.phiq_reg + (size_t(fb_slice) * N + row) * 4);
      aq0 = v.x, aq1 = v.y, aq2 = v.z, aq3 = v.w;
    }

    float m_use = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int i = 0; i < nk[t]; ++i) {  // i: this tile's local step (key tile nk[t] - 1 - i)
      const int s = i % KS;             // its own ring of softmax-side tiles
      const uint32_t ph = uint32_t(i / KS) & 1u;
      if (C::HAS_AUX && !(ok = mbar_wait(&ctrl->aux_full[t][s], ph, abort))) break;
      if (!(ok = mbar_wait(&ctrl->s_full[t], uint32_t(i) & 1u, abort))) break;
      tc_fence_after();

      // Raw scores of this thread's row; with a softmax-side bias they are
      // turned into log2-domain logits in place, otherwise the scale is
      // folded into the exponent below.
      uint32_t x[128];
      tmem_ld32(s_tm + 0, x + 0);
      tmem_ld32(s_tm + 32, x + 32);
      tmem_ld32(s_tm + 64, x + 64);
      tmem_ld32(s_tm + 96, x + 96);
      tmem_ld_wait32(x + 0);
      tmem_ld_wait32(x + 32);
      tmem_ld_wait32(x + 64);
      tmem_ld_wait32(x + 96);
      if (C::SEP_P) {  // S_t(i) is in registers: the tensor core may overwrite it
        tc_fence_before();
        mbar_arrive(&ctrl->s_free[t]);
      }
      float mul = sl2;  // logit = raw * mul
      if (MODE == kBiasReg) {
        const uint8_t *fk = sAux + (t * KS + s) * C::AUX_TILE;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          float v;
          if (RP <= 2) {
            const float2 f = *reinterpret_cast<const float2 *>(fk + c * 16);
            v = fmaf(aq0, f.x, fmaf(aq1, f.y, __uint_as_float(x[c]) * sl2));
          } else {
            const float4 f = *reinterpret_cast<const float4 *>(fk + c * 16);
            v = fmaf(aq0, f.x, fmaf(aq1, f.y, fmaf(aq2, f.z, fmaf(aq3, f.w, __uint_as_float(x[c]) * sl2))));
          }
          x[c] = __float_as_uint(v);
        }
        mbar_arrive(&ctrl->aux_empty[t][s]);
        mul = 1.f;
      } else if (MODE == kBiasDense) {
        const uint8_t *tile = sAux + (t * KS + s) * C::AUX_TILE;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
          for (int ck = 0; ck < 8; ++ck) {
            const uint4 u =
                *reinterpret_cast<const uint4 *>(tile + hh * 16384 + r_loc * 128 + ((ck ^ (r_loc & 7)) * 16));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = hh * 64 + ck * 8 + 2 * e;
              x[c] = __float_as_uint(fmaf(__uint_as_float(w[e] << 16), kLog2e, __uint_as_float(x[c]) * sl2));
              x[c + 1] =
                  __float_as_uint(fmaf(__uint_as_float(w[e] & 0xFFFF0000u), kLog2e, __uint_as_float(x[c + 1]) * sl2));
            }
          }
        }
        mbar_arrive(&ctrl->aux_empty[t][s]);
        mul = 1.f;
      }
      // Causal diagonal tile and the ragged last key tile.
      const int key0 = (nk[t] - 1 - i) * 128;
      if ((args.causal && key0 + 127 > q0[t]) || key0 + 128 > N) {
        const int lim = args.causal ? min(row + 1, N) : N;  // keys [0, lim) are visible
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (key0 + c >= lim) x[c] = __float_as_uint(-INFINITY);
      }
      float mx;
      {
        float mp[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mp[e] = __uint_as_float(x[e]);
#pragma unroll
        for (int c = 8; c < 128; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) mp[e] = fmaxf(mp[e], __uint_as_float(x[c + e]));
        mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      }
      const float m_new = fmaxf(m_use, mx * mul);
      float alpha = 1.f;
      bool resc = false;
      if (m_use == -INFINITY || m_new > m_use + kRescaleThreshold) {
        alpha = (m_use == -INFINITY) ? 0.f : ex2_approx(m_use - m_new);
        resc = (i > 0) && (m_use != -INFINITY);
        m_use = m_new;
      }
      l_sum *= alpha;
      if (C::SEP_P && i > 0) {
        // O_t and P_t are still read by PV_t(i-1); wait until it has completed.
        if (!(ok = mbar_wait(&ctrl->pv_done[t], uint32_t(i - 1) & 1u, abort))) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
        // PV_t(i-1) has completed (pv_done, or, when P aliases S, the commit
        // that published S_t(i) covers it).
#pragma unroll
        for (int c0 = 0; c0 < DP; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(o_tm + c0, r);
          tmem_ld_wait16(r);
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(o_tm + c0, r);
        }
      }
      const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
      const uint64_t mul2 = f2_pack(mul, mul), negm2 = f2_pack(neg_m, neg_m);
      uint64_t ls[4] = {0, 0, 0, 0};  // packed partial row sums
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t a = f2_fma(f2_pack(__uint_as_float(x[q4 * 32 + 2 * e]), __uint_as_float(x[q4 * 32 + 2 * e + 1])),
                                    mul2, negm2);
          float a0, a1, p0, p1;
          f2_unpack(a, a0, a1);
          if (e < kEmuPairs) {
            ex2_fma_pair(a0, a1, p0, p1);
          } else {
            p0 = ex2_approx(a0);
            p1 = ex2_approx(a1);
          }
          ls[e & 3] = f2_add(ls[e & 3], f2_pack(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_tm + uint32_t(q4 * 16), pk);
      }
      {
        float s0, s1, s2, s3, s4, s5, s6, s7;
        f2_unpack(ls[0], s0, s1);
        f2_unpack(ls[1], s2, s3);
        f2_unpack(ls[2], s4, s5);
        f2_unpack(ls[3], s6, s7);
        l_sum += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctrl->p_full[t]);
    }

    // ------------------------------------------------------------ epilogue
    if (ok && nk[t] > 0) ok = mbar_wait(&ctrl->o_final[t], 0, abort);
    if (ok && nk[t] > 0) {
      tc_fence_after();
      const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
      __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(args.O) + (size_t(bh) * N + row) * args.d;
#pragma unroll
      for (int c0 = 0; c0 < DP; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(o_tm + c0, r);
        tmem_ld_wait16(r);
        if (row < N) {
#pragma unroll
          for (int v8 = 0; v8 < 2; ++v8) {
            const int col = c0 + v8 * 8;
            if (col < args.d) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(r[v8 * 8 + 0]) * inv_l, __uint_as_float(r[v8 * 8 + 1]) * inv_l);
              u.y = pack_bf16x2(__uint_as_float(r[v8 * 8 + 2]) * inv_l, __uint_as_float(r[v8 * 8 + 3]) * inv_l);
              u.z = pack_bf16x2(__uint_as_float(r[v8 * 8 + 4]) * inv_l, __uint_as_float(r[v8 * 8 + 5]) * inv_l);
              u.w = pack_bf16x2(__uint_as_float(r[v8 * 8 + 6]) * inv_l, __uint_as_float(r[v8 * 8 + 7]) * inv_l);
              *reinterpret_cast<uint4 *>(orow + col) = u;
            }
          }
        }
      }
      if (row < N)
        args.LSE[size_t(bh) * N + row] = l_sum > 0.f ? (m_use + __log2f(l_sum)) * kLn2 : -INFINITY;
    }
    if (!ok) atomicOr(args.flags, kFlagTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DP, int RP, int MODE, int QT>
static cudaError_t launch_one(const FwdMaps &m, const FwdArgs &a, cudaStream_t stream) {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  if constexpr (C::KS < 1) {
    return cudaErrorInvalidConfiguration;
  } else {
    auto kern = attn_fwd_sm100<DP, RP, MODE, QT>;
    // setmaxnreg.inc waits until the block's pool has the registers, so the
    // launch allocation must be exactly what the split assumes.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.H, a.n_cta_q);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(m.q, m.k, m.v, m.fq, m.fk, m.bias, a);
    return cudaGetLastError();
  }
}

template <int DP, int RP, int MODE, int QT>
static constexpr size_t smem_of() {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  return C::KS >= 1 ? size_t(C::SMEM) : 0;
}

#define FB_DISPATCH_QT(DPv, RPv, MODEv)                                          \
  if (p.QT == 1) return FB_ACTION(DPv, RPv, MODEv, 1);                           \
  if (p.QT == 2) return FB_ACTION(DPv, RPv, MODEv, 2);

#define FB_DISPATCH_MODE(DPv)                                                    \
  if (p.mode == kBiasNone) { FB_DISPATCH_QT(DPv, 0, kBiasNone) }                 \
  if (p.mode == kBiasReg) {                                                      \
    if (p.RP == 2) { FB_DISPATCH_QT(DPv, 2, kBiasReg) }                          \
    if (p.RP == 4) { FB_DISPATCH_QT(DPv, 4, kBiasReg) }                          \
  }                                                                              \
  if (p.mode == kBiasDense) { FB_DISPATCH_QT(DPv, 0, kBiasDense) }               \
  if (p.mode == kBiasMma) {                                                      \
    if (p.RP == 16) { FB_DISPATCH_QT(DPv, 16, kBiasMma) }                        \
    if (p.RP == 32) { FB_DISPATCH_QT(DPv, 32, kBiasMma) }                        \
    if (p.RP == 64) { FB_DISPATCH_QT(DPv, 64, kBiasMma) }                        \
    if (p.RP == 128) { FB_DISPATCH_QT(DPv, 128, kBiasMma) }                      \
  }

#define FB_DISPATCH_ALL                                                          \
  if (p.DP == 16) { FB_DISPATCH_MODE(16) }                                       \
  if (p.DP == 32) { FB_DISPATCH_MODE(32) }                                       \
  if (p.DP == 64) { FB_DISPATCH_MODE(64) }                                       \
  if (p.DP == 128) { FB_DISPATCH_MODE(128) }

size_t sm100_smem_bytes(const FwdPlan &p) {
#define FB_ACTION(DPv, RPv, MODEv, QTv) smem_of<DPv, RPv, MODEv, QTv>()
  FB_DISPATCH_ALL
#undef FB_ACTION
  return 0;
}

cudaError_t sm100_launch(const FwdPlan &p, const FwdMaps &maps, const FwdArgs &a, cudaStream_t stream) {
#define FB_ACTION(DPv, RPv, MODEv, QTv) launch_one<DPv, RPv, MODEv, QTv>(maps, a, stream)
  FB_DISPATCH_ALL
#undef FB_ACTION
  return cudaErrorInvalidConfiguration;
}

}  // namespace fb
