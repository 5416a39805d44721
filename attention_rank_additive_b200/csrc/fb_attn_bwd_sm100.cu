// fb_attn_bwd_sm100.cu -- backward of attention with a low-rank additive bias
// on B200 (sm_100a): TMA -> shared memory -> tcgen05 MMA -> TMEM -> CUDA cores
// -> tcgen05 MMA (A operand from TMEM) -> TMEM -> HBM.
//
// Method: FlashBias (arXiv 2505.12044) trains by concatenating the factors to
// the queries and keys, q' = [q, phi_q], k' = [k, phi_k] (rebuttal, reply to
// Reviewer UJUf, Q2 and the training speedup of Q1 (3); reply to Reviewer
// Bp2x, Q3), so the backward is the attention backward of the concatenated
// operands and the factor gradients are the extra columns of dq' and dk':
//   P = exp(s - LSE), dP = dO V^T, dS = P * (dP - D) with D = rowsum(dO * O),
//   dV = P^T dO, dK = scale dS^T Q, dphi_k = dS^T phi_q,
//   dQ = scale dS K, dphi_q = dS phi_k.
// S is recomputed exactly as the forward computes it (bf16 QK^T plus the
// fp16 or tf32 factor MMA into one fp32 accumulator), so P matches the
// forward's P; the gradient products run in bf16 with fp32 accumulation, the
// factors entering them as bf16 copies.
//
// At head dim 64 (fixed factors, or 33 <= R <= 64) one persistent kernel,
// attn_bwd_fused_sm100 (below), computes every gradient of a 128-key tile and
// adds each query block's dQ and dphi_q into an fp32 accumulator with TMA
// reduce-adds. Otherwise two kernels, no atomics:
//   attn_bwd_dkdv_sm100  one CTA per (b, h, 128-key tile). The key tile K|phi_k
//       and V stay in shared memory; query blocks of BQ rows (64, or 32 at
//       head dim 128 so that TMEM holds everything) stream through a ring.
//       Per block: S^T = K Q^T (+ phi_k' phi_q'^T), dP^T = V dO^T; the CUDA
//       cores turn them into P^T and dS^T (bf16, written back over S^T and
//       dP^T in TMEM); then dV += P^T dO, dK += dS^T Q, dphi_k += dS^T phi_q
//       with the A operand read from TMEM and dO, Q, phi_q as MN-major B.
//   attn_bwd_dq_sm100    one CTA per (b, h, 128-query tile), key blocks of 64:
//       S = Q K^T (+ ...), dP = dO V^T, dS over S in TMEM, dQ += dS K,
//       dphi_q += dS phi_k.
// In all of them, two compute warpgroups take alternate blocks, each with its
// own S and dP buffers in TMEM (ping-pong): while one turns its scores into P
// and dS, the tensor core runs the other's products.
// The factor gradients of a broadcast factor (stride 0) sum over the heads
// and batches sharing it: each head writes its rows to per-head partials and
// a reduction over the sharing heads follows; a per-head factor gets its rows
// written directly.
//
// Two-kernel CTA: warps 0-7 compute (two warpgroups, one thread per TMEM lane
// = tile row in each), warp 8 TMA producer, warp 9 TMEM allocator and MMA
// issuer. Every wait is bounded (the abort flag and the device flag word
// report a timeout).
#include <algorithm>
#include <atomic>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {
namespace {

constexpr uint32_t kSmemLimitB = 227u * 1024u;

// Bulk copy (no tensor map) of `bytes` (multiple of 16, both addresses
// 16-byte aligned) into shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load_leader(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                 uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\t"
      "@q cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%4];\n\t}" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(leader), "r"(smem_u32(bar))
      : "memory");
}

// Packed f32x2 multiply (one instruction for two lanes' worth of products).
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// K-major tile of ROWS rows x (NCH * CH) 16-bit units stored as NCH swizzled
// chunks of CH units: descriptor of the base and offset (>> 4) of K-step kk
// (32 bytes of a row).
template <int CH>
__device__ __forceinline__ uint64_t kdesc(uint32_t base) {
  return make_smem_desc(base, 16, 8 * CH * 2, swizzle_code(CH * 2));
}
template <int CH, int ROWS>
__host__ __device__ constexpr uint32_t kstep(int kk) {
  return uint32_t((kk / (CH / 16)) * (ROWS * CH * 2) + (kk % (CH / 16)) * 32) >> 4;
}
// The same tile read as an MN-major B operand (rows = the MMA's K dimension,
// columns = N): chunk stride as leading offset, 8 rows as stride offset;
// offset of the 16-row step kk.
template <int CH, int ROWS>
__device__ __forceinline__ uint64_t mndesc(uint32_t base) {
  return make_smem_desc(base, ROWS * CH * 2, 8 * CH * 2, swizzle_code(CH * 2));
}
template <int CH>
__host__ __device__ constexpr uint32_t mnstep(int kk) {
  return uint32_t(kk * 16 * CH * 2) >> 4;
}

}  // namespace

template <int DP, int RP, int MODE, int RG>
struct BwdCfg {
  // Two compute warpgroups take alternate row blocks (ping-pong): each has
  // its own S and dP buffers in TMEM, so the tensor core computes one
  // block's scores while the CUDA cores turn the other's into P and dS.
  // dK/dV kernel: streamed query blocks of BQ rows (32 at head dim 128 so
  // that TMEM holds both buffers and the dV, dK, dphi_k accumulators).
  static constexpr int BQ = DP == 128 ? 32 : 64;
  // dQ kernel: streamed key blocks of BK rows.
  static constexpr int BK = 64;
  static constexpr int DCH = DP > 64 ? 64 : DP;
  static constexpr int NDCH = DP / DCH;
  static constexpr bool FAC = MODE == kBiasMma || MODE == kBiasTf32;
  // S-side factor tile: fp16 [rows x RP] or fp32 [rows x RP] (tf32); width in
  // 16-bit units of one chunk (tf32 rows are one chunk of RP floats).
  static constexpr int FCH = MODE == kBiasMma ? (RP > 64 ? 64 : RP) : (MODE == kBiasTf32 ? 2 * RP : 16);
  static constexpr int NFCH = MODE == kBiasMma ? RP / FCH : (MODE == kBiasTf32 ? 1 : 0);
  static constexpr int FESZ = MODE == kBiasTf32 ? 4 : 2;
  // bf16 gradient factor tile [rows x RG].
  static constexpr int GCH = RG > 64 ? 64 : (RG > 0 ? RG : 16);
  static constexpr int NGCH = RG > 0 ? RG / GCH : 0;
  static constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }
  static constexpr uint32_t CTRL = 1024;
  static constexpr uint32_t SLACK = 1024;
  static constexpr int MAX_STAGES = 4;
  // dK/dV kernel: fixed K, V, phi_k' tiles; per stage Q, dO, phi_q', phi_q (bf16), LSE2, D
  static constexpr uint32_t KV_FIXED = 2u * 128u * DP * 2u + (FAC ? 128u * RP * FESZ : 0u);
  static constexpr uint32_t KV_STAGE_BYTES =
      2u * BQ * DP * 2u + (FAC ? BQ * RP * FESZ : 0u) + BQ * RG * 2u + 2u * BQ * 4u;
  static constexpr uint32_t KV_STAGE = align1k(KV_STAGE_BYTES);
  static constexpr int KV_KS_FIT =
      kSmemLimitB > KV_FIXED + CTRL + SLACK ? int((kSmemLimitB - KV_FIXED - CTRL - SLACK) / KV_STAGE) : 0;
  static constexpr int KV_KS = KV_KS_FIT > MAX_STAGES ? MAX_STAGES : KV_KS_FIT;
  static constexpr uint32_t KV_SMEM = KV_FIXED + uint32_t(KV_KS) * KV_STAGE + CTRL + SLACK;
  // dQ kernel: fixed Q, dO, phi_q' tiles; per stage K, V, phi_k', phi_k (bf16)
  static constexpr uint32_t DQ_FIXED = 2u * 128u * DP * 2u + (FAC ? 128u * RP * FESZ : 0u);
  static constexpr uint32_t DQ_STAGE_BYTES = 2u * BK * DP * 2u + (FAC ? BK * RP * FESZ : 0u) + BK * RG * 2u;
  static constexpr uint32_t DQ_STAGE = align1k(DQ_STAGE_BYTES);
  static constexpr int DQ_KS_FIT =
      kSmemLimitB > DQ_FIXED + CTRL + SLACK ? int((kSmemLimitB - DQ_FIXED - CTRL - SLACK) / DQ_STAGE) : 0;
  static constexpr int DQ_KS = DQ_KS_FIT > MAX_STAGES ? MAX_STAGES : DQ_KS_FIT;
  static constexpr uint32_t DQ_SMEM = DQ_FIXED + uint32_t(DQ_KS) * DQ_STAGE + CTRL + SLACK;
  static constexpr int THREADS = 320;  // 2 compute warpgroups, producer warp, MMA warp
  static constexpr int PRODUCER_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns, dK/dV kernel: buffer t holds S^T at t 2BQ and dP^T at t 2BQ + BQ
  static constexpr uint32_t KV_DV = 4 * BQ, KV_DK = 4 * BQ + DP, KV_DF = 4 * BQ + 2 * DP;
  static_assert(KV_DF + RG <= TMEM_COLS, "dK/dV TMEM layout");
  // TMEM columns, dQ kernel: buffer t holds S at t 2BK and dP at t 2BK + BK
  static constexpr uint32_t DQ_DQ = 4 * BK, DQ_DF = 4 * BK + DP;
  static_assert(DQ_DF + RG <= TMEM_COLS, "dQ TMEM layout");
  static constexpr uint32_t IDESC_KV_S = make_idesc_f16(true, true, 128, BQ, false);
  static constexpr uint32_t IDESC_KV_F =
      MODE == kBiasTf32 ? make_idesc_tf32(128, BQ) : make_idesc_f16(false, false, 128, BQ, false);
  static constexpr uint32_t IDESC_DQ_S = make_idesc_f16(true, true, 128, BK, false);
  static constexpr uint32_t IDESC_DQ_F =
      MODE == kBiasTf32 ? make_idesc_tf32(128, BK) : make_idesc_f16(false, false, 128, BK, false);
  static constexpr uint32_t IDESC_GD = make_idesc_f16(true, true, 128, DP, true);
  static constexpr uint32_t IDESC_GR = make_idesc_f16(true, true, 128, RG > 0 ? RG : 16, true);
};

namespace {

struct BwdCtrl {
  uint64_t fixed_full;
  uint64_t full[4], empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_done;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(BwdCtrl) <= 1024, "control block too large");

// fp32 -> bf16 pairs of a TMEM row segment, scaled, stored to a global row
// (columns [c0, c0 + 16) of which those below d are written).
__device__ __forceinline__ void store_row16_bf16(const uint32_t *r, float mul, uint16_t *row, int c0, int d) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
  if (c0 + 8 <= d) *reinterpret_cast<uint4 *>(row + c0) = make_uint4(w[0], w[1], w[2], w[3]);
  if (c0 + 16 <= d) *reinterpret_cast<uint4 *>(row + c0 + 8) = make_uint4(w[4], w[5], w[6], w[7]);
}

// The factor-gradient row of head (b, h) and row n: in the caller's tensor
// when every head has its own factor slice (each row is then written by
// exactly one CTA), else in the per-head partial rows [BH, N, R] that a
// reduction over the heads sharing a slice sums afterwards. No atomics.
__device__ __forceinline__ float *factor_grad_row(const BwdArgs &a, float *dphi, float *part, int b, int h, int bh,
                                                  int n) {
  if (a.dphi_direct)
    return dphi + (a.fac_B > 1 ? int64_t(b) * a.phi_bs : 0) + (a.fac_H > 1 ? int64_t(h) * a.phi_hs : 0) +
           int64_t(n) * a.R;
  return part + (int64_t(bh) * a.N + n) * a.R;
}

// The first `valid` of the RG fp32 columns of this thread's TMEM lane to a
// global row (16-byte stores when the row allows them). TMEM loads are
// warp-collective: every lane loads, lanes with valid = 0 store nothing.
template <int RG>
__device__ __forceinline__ void store_factor_grad_row(uint32_t taddr, float *row, int valid) {
  const bool vec = (valid & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0;
#pragma unroll 1
  for (int c0 = 0; c0 < RG; c0 += 16) {
    uint32_t r[16];
    tmem_ld16(taddr + uint32_t(c0), r);
    tmem_ld_wait16(r);
    if (vec) {
#pragma unroll
      for (int e = 0; e < 16; e += 4)
        if (c0 + e < valid)
          *reinterpret_cast<float4 *>(row + c0 + e) = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                                                  __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c0 + e < valid) row[c0 + e] = __uint_as_float(r[e]);
    }
  }
}

}  // namespace

// ------------------------------------------------------------ dK, dV, dphi_k
template <int DP, int RP, int MODE, int RG>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_fk, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_fq,
                        const __grid_constant__ CUtensorMap tm_gq, const BwdArgs args) {
  using C = BwdCfg<DP, RP, MODE, RG>;
  constexpr int KS = C::KV_KS;
  constexpr int BQ = C::BQ;
  static_assert(KS >= 2, "configuration does not fit in shared memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem;                    // 128 x DP bf16
  uint8_t *sV = sK + 128 * DP * 2;       // 128 x DP bf16
  uint8_t *sFK = sV + 128 * DP * 2;      // 128 x RP (fp16 / fp32)
  uint8_t *sStage = smem + C::KV_FIXED;  // KS x KV_STAGE
  BwdCtrl *ctrl = reinterpret_cast<BwdCtrl *>(sStage + KS * C::KV_STAGE);
  // offsets inside a stage
  constexpr uint32_t O_Q = 0, O_DO = BQ * DP * 2, O_FQ = 2 * BQ * DP * 2;
  constexpr uint32_t O_GQ = O_FQ + (C::FAC ? BQ * RP * C::FESZ : 0);
  constexpr uint32_t O_L = O_GQ + BQ * RG * 2, O_D = O_L + BQ * 4;
  static_assert(O_D + BQ * 4 == C::KV_STAGE_BYTES, "stage layout");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = args.B * args.H;
  const int kb = int(blockIdx.x) / BH;  // key tile; the heaviest causal tiles come first
  const int bh = int(blockIdx.x) % BH;
  const int b = bh / args.H, h = bh % args.H;
  const int k0 = kb * 128;
  const int fslice = (args.fac_B > 1 ? b : 0) * args.fac_H + (args.fac_H > 1 ? h : 0);
  const int j0 = args.causal ? k0 / BQ : 0;  // query blocks before the diagonal see none of these keys
  const int nb = (args.N + BQ - 1) / BQ - j0;  // >= 1

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->fixed_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 128);
    }
    mbar_init(&ctrl->acc_done, 1);
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
  const uint32_t leader = lane == 0 ? 1u : 0u;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (leader) {
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_do);
      if (C::FAC) {
        tma_prefetch_map(&tm_fk);
        tma_prefetch_map(&tm_fq);
      }
      if (RG > 0) tma_prefetch_map(&tm_gq);
    }
    mbar_arrive_expect_tx_leader(&ctrl->fixed_full, C::KV_FIXED, leader);
    for (int ch = 0; ch < C::NDCH; ++ch) {
      tma_load_3d_leader(sK + ch * (128 * C::DCH * 2), &tm_k, &ctrl->fixed_full, ch * C::DCH, k0, bh, leader);
      tma_load_3d_leader(sV + ch * (128 * C::DCH * 2), &tm_v, &ctrl->fixed_full, ch * C::DCH, k0, bh, leader);
    }
    if (C::FAC)
      for (int ch = 0; ch < C::NFCH; ++ch)
        tma_load_3d_leader(sFK + ch * (128 * C::FCH * 2), &tm_fk, &ctrl->fixed_full, ch * C::FCH, k0, fslice,
                           leader);
    bool ok = true;
    for (int u = 0; u < nb; ++u) {
      const int s = u % KS;
      if (u >= KS && !(ok = mbar_wait(&ctrl->empty[s], (uint32_t(u / KS) & 1u) ^ 1u, abort))) break;
      uint8_t *st = sStage + s * C::KV_STAGE;
      const int q0 = (j0 + u) * BQ;
      mbar_arrive_expect_tx_leader(&ctrl->full[s], C::KV_STAGE_BYTES, leader);
      for (int ch = 0; ch < C::NDCH; ++ch) {
        tma_load_3d_leader(st + O_Q + ch * (BQ * C::DCH * 2), &tm_q, &ctrl->full[s], ch * C::DCH, q0, bh, leader);
        tma_load_3d_leader(st + O_DO + ch * (BQ * C::DCH * 2), &tm_do, &ctrl->full[s], ch * C::DCH, q0, bh, leader);
      }
      if (C::FAC)
        for (int ch = 0; ch < C::NFCH; ++ch)
          tma_load_3d_leader(st + O_FQ + ch * (BQ * C::FCH * 2), &tm_fq, &ctrl->full[s], ch * C::FCH, q0, fslice,
                             leader);
      for (int ch = 0; ch < C::NGCH; ++ch)
        tma_load_3d_leader(st + O_GQ + ch * (BQ * C::GCH * 2), &tm_gq, &ctrl->full[s], ch * C::GCH, q0, fslice,
                           leader);
      const size_t roff = size_t(bh) * args.Npad + q0;
      bulk_load_leader(st + O_L, args.nlse2 + roff, BQ * 4, &ctrl->full[s], leader);
      bulk_load_leader(st + O_D, args.delta + roff, BQ * 4, &ctrl->full[s], leader);
    }
    if (!ok) {
      // Aborted: let the copies already issued land before the CTA exits.
      mbar_wait_for(&ctrl->fixed_full, 0, 100000000ull);
      for (int s = 0; s < KS; ++s) {
        mbar_wait_for(&ctrl->full[s], 0, 100000000ull);
        mbar_wait_for(&ctrl->full[s], 1, 100000000ull);
      }
      if (leader) atomicOr(args.flags, kFlagTimeout);
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------------------------------------------------- MMA issuer
    // Order: S(0), S(1), G(0), S(2), G(1), S(3), ... where S(u) computes the
    // scores of block u into buffer u & 1 and G(u) the gradient products of
    // block u from that buffer; S(u + 2) follows G(u) (tcgen05 MMAs of one
    // thread run in order), so it overwrites P and dS only after their use.
    const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->fixed_full, 0, abort));  // warp-uniform for elect.sync
    tc_fence_after();
    const uint64_t dK = kdesc<C::DCH>(smem_u32(sK));
    const uint64_t dV = kdesc<C::DCH>(smem_u32(sV));
    const uint64_t dFK = kdesc<C::FCH>(smem_u32(sFK));
    auto issue_s = [&](int u) -> bool {
      const int s = u % KS;
      if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->full[s], uint32_t(u / KS) & 1u, abort))) return false;
      tc_fence_after();
      const uint32_t st = smem_u32(sStage + s * C::KV_STAGE);
      const uint32_t s_col = tm_u + uint32_t((u & 1) * 2 * BQ);
      uint64_t dq = kdesc<C::DCH>(st + O_Q), ddo = kdesc<C::DCH>(st + O_DO);
      asm volatile("" : "+l"(dq), "+l"(ddo));
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)  // S^T = K Q^T
        mma_ss_elect(s_col, dK + kstep<C::DCH, 128>(kk), dq + kstep<C::DCH, BQ>(kk), C::IDESC_KV_S, kk > 0 ? 1u : 0u);
      if constexpr (C::FAC) {  // S^T += phi_k' phi_q'^T
        uint64_t dfq = kdesc<C::FCH>(st + O_FQ);
        asm volatile("" : "+l"(dfq));
#pragma unroll
        for (int kk = 0; kk < C::FCH * C::NFCH / 16; ++kk) {
          if (MODE == kBiasTf32)
            mma_ss_elect_tf32(s_col, dFK + kstep<C::FCH, 128>(kk), dfq + kstep<C::FCH, BQ>(kk), C::IDESC_KV_F, 1u);
          else
            mma_ss_elect(s_col, dFK + kstep<C::FCH, 128>(kk), dfq + kstep<C::FCH, BQ>(kk), C::IDESC_KV_F, 1u);
        }
      }
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)  // dP^T = V dO^T
        mma_ss_elect(s_col + BQ, dV + kstep<C::DCH, 128>(kk), ddo + kstep<C::DCH, BQ>(kk), C::IDESC_KV_S,
                     kk > 0 ? 1u : 0u);
      tc_commit_elect(&ctrl->s_full[u & 1]);
      __syncwarp();
      return true;
    };
    auto issue_g = [&](int u) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->p_full[u & 1], uint32_t(u >> 1) & 1u, abort))) return false;
      tc_fence_after();
      const int s = u % KS;
      const uint32_t st = smem_u32(sStage + s * C::KV_STAGE);
      const uint32_t p_col = tm_u + uint32_t((u & 1) * 2 * BQ);  // P^T bf16 over S^T; dS^T over dP^T
      uint64_t bdo = mndesc<C::DCH, BQ>(st + O_DO), bq = mndesc<C::DCH, BQ>(st + O_Q);
      asm volatile("" : "+l"(bdo), "+l"(bq));
#pragma unroll
      for (int kk = 0; kk < BQ / 16; ++kk) {
        const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
        mma_ts_elect(tm_u + C::KV_DV, p_col + uint32_t(kk * 8), bdo + mnstep<C::DCH>(kk), C::IDESC_GD, acc);
        mma_ts_elect(tm_u + C::KV_DK, p_col + BQ + uint32_t(kk * 8), bq + mnstep<C::DCH>(kk), C::IDESC_GD, acc);
      }
      if constexpr (RG > 0) {
        uint64_t bg = mndesc<C::GCH, BQ>(st + O_GQ);
        asm volatile("" : "+l"(bg));
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_ts_elect(tm_u + C::KV_DF, p_col + BQ + uint32_t(kk * 8), bg + mnstep<C::GCH>(kk), C::IDESC_GR,
                       (u > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit_elect(&ctrl->empty[s]);
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    if (ok && nb > 1) ok = issue_s(1);
    for (int u = 0; u < nb && ok; ++u) {
      ok = issue_g(u);
      if (ok && u + 2 < nb) ok = issue_s(u + 2);
    }
    if (ok) {
      tc_commit_elect(&ctrl->acc_done);
      __syncwarp();
    }
    if (!ok && leader) atomicOr(args.flags, kFlagTimeout);
  } else {
    // ------------------------------- compute: warpgroup t takes blocks u = t mod 2
    const int t = warp >> 2, quarter = warp & 3;
    const int r_loc = quarter * 32 + lane;
    const int krow = k0 + r_loc;  // this thread's key
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_tm = lane_base + uint32_t(t * 2 * BQ), dp_tm = s_tm + BQ;
    const float sl2 = args.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    for (int u = t; u < nb; u += 2) {
      const int s = u % KS;
      // the whole warp leaves together: the TMEM accesses below are warp-collective
      ok = mbar_wait(&ctrl->full[s], uint32_t(u / KS) & 1u, abort) &&
           mbar_wait(&ctrl->s_full[t], uint32_t(u >> 1) & 1u, abort);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint8_t *st = sStage + s * C::KV_STAGE;
      const float *sL = reinterpret_cast<const float *>(st + O_L);
      const float *sD = reinterpret_cast<const float *>(st + O_D);
      const int q0 = (j0 + u) * BQ;
      const bool diag = args.causal && q0 < k0 + 127;  // some query of the block precedes some key
#pragma unroll
      for (int c = 0; c < BQ / 32; ++c) {
        uint32_t sx[32], dx[32];
        tmem_ld32(s_tm + uint32_t(32 * c), sx);
        tmem_ld32(dp_tm + uint32_t(32 * c), dx);
        tmem_ld_wait32(sx);
        tmem_ld_wait32(dx);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          // sL holds -LSE log2(e): x = S scale log2(e) - LSE log2(e), two columns per instruction
          const float4 l4 = *reinterpret_cast<const float4 *>(sL + 32 * c + 4 * e4);
          const float4 d4 = *reinterpret_cast<const float4 *>(sD + 32 * c + 4 * e4);
          const uint64_t l2[2] = {f2_pack(l4.x, l4.y), f2_pack(l4.z, l4.w)};
          const uint64_t d2[2] = {f2_pack(d4.x, d4.y), f2_pack(d4.z, d4.w)};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int i = 4 * e4 + 2 * h2;
            float a0, a1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sx[i]), __uint_as_float(sx[i + 1])), sl2x2, l2[h2]), a0, a1);
            float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
            if (diag) {
              const int col = 32 * c + i;
              if (q0 + col < krow) p0 = 0.f;
              if (q0 + col + 1 < krow) p1 = 0.f;
            }
            const uint64_t p2 = f2_pack(p0, p1);
            float g0, g1;
            f2_unpack(f2_mul(p2, f2_sub(f2_pack(__uint_as_float(dx[i]), __uint_as_float(dx[i + 1])), d2[h2])), g0, g1);
            pp[2 * e4 + h2] = pack_bf16x2(p0, p1);
            dd[2 * e4 + h2] = pack_bf16x2(g0, g1);
          }
        }
        tmem_st16(s_tm + uint32_t(16 * c), pp);
        tmem_st16(dp_tm + uint32_t(16 * c), dd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctrl->p_full[t]);
    }
    if (ok) ok = mbar_wait(&ctrl->acc_done, 0, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      // epilogue: warpgroup 0 writes dV and dphi_k, warpgroup 1 dK. TMEM loads
      // are warp-collective: every lane loads, rows past N store nothing.
      tc_fence_after();
      const bool valid = krow < args.N;
      const int d_st = valid ? args.d : 0;
      const size_t row_off = (size_t(bh) * args.N + (valid ? krow : 0)) * args.d;
      uint16_t *dst = static_cast<uint16_t *>(t == 0 ? args.dV : args.dK) + row_off;
      const uint32_t acc_tm = lane_base + (t == 0 ? C::KV_DV : C::KV_DK);
      const float mul = t == 0 ? 1.f : args.scale;
#pragma unroll 1
      for (int c0 = 0; c0 < DP; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(acc_tm + uint32_t(c0), r);
        tmem_ld_wait16(r);
        store_row16_bf16(r, mul, dst, c0, d_st);
      }
      if constexpr (RG > 0) {
        if (t == 0) {
          const int r_st = valid ? args.R : 0;
          store_factor_grad_row<RG>(lane_base + C::KV_DF, factor_grad_row(args, args.dphi_k, args.dphi_k_part, b, h,
                                                                           bh, valid ? krow : 0),
                                    r_st);
        }
      }
    }
    if (!ok && lane == 0) atomicOr(args.flags, kFlagTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ dQ, dphi_q
template <int DP, int RP, int MODE, int RG>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_dq_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ CUtensorMap tm_fq, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_fk,
                      const __grid_constant__ CUtensorMap tm_gk, const BwdArgs args) {
  using C = BwdCfg<DP, RP, MODE, RG>;
  constexpr int KS = C::DQ_KS;
  constexpr int BK = C::BK;
  static_assert(KS >= 2, "configuration does not fit in shared memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                    // 128 x DP bf16
  uint8_t *sDO = sQ + 128 * DP * 2;      // 128 x DP bf16
  uint8_t *sFQ = sDO + 128 * DP * 2;     // 128 x RP (fp16 / fp32)
  uint8_t *sStage = smem + C::DQ_FIXED;  // KS x DQ_STAGE
  BwdCtrl *ctrl = reinterpret_cast<BwdCtrl *>(sStage + KS * C::DQ_STAGE);
  constexpr uint32_t O_K = 0, O_V = BK * DP * 2, O_FK = 2 * BK * DP * 2;
  constexpr uint32_t O_GK = O_FK + (C::FAC ? BK * RP * C::FESZ : 0);
  static_assert(O_GK + BK * RG * 2 == C::DQ_STAGE_BYTES, "stage layout");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = args.B * args.H;
  const int qb = args.n_kv - 1 - int(blockIdx.x) / BH;  // the heaviest causal tiles come first
  const int bh = int(blockIdx.x) % BH;
  const int b = bh / args.H, h = bh % args.H;
  const int q0 = qb * 128;
  const int fslice = (args.fac_B > 1 ? b : 0) * args.fac_H + (args.fac_H > 1 ? h : 0);
  // key blocks this query tile sees: keys [0, min(q0 + 128, N)) when causal
  const int key_end = args.causal ? min(q0 + 128, args.N) : args.N;
  const int nb = (key_end + BK - 1) / BK;

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->fixed_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 128);
    }
    mbar_init(&ctrl->acc_done, 1);
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
  const uint32_t leader = lane == 0 ? 1u : 0u;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (leader) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_do);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      if (C::FAC) {
        tma_prefetch_map(&tm_fq);
        tma_prefetch_map(&tm_fk);
      }
      if (RG > 0) tma_prefetch_map(&tm_gk);
    }
    mbar_arrive_expect_tx_leader(&ctrl->fixed_full, C::DQ_FIXED, leader);
    for (int ch = 0; ch < C::NDCH; ++ch) {
      tma_load_3d_leader(sQ + ch * (128 * C::DCH * 2), &tm_q, &ctrl->fixed_full, ch * C::DCH, q0, bh, leader);
      tma_load_3d_leader(sDO + ch * (128 * C::DCH * 2), &tm_do, &ctrl->fixed_full, ch * C::DCH, q0, bh, leader);
    }
    if (C::FAC)
      for (int ch = 0; ch < C::NFCH; ++ch)
        tma_load_3d_leader(sFQ + ch * (128 * C::FCH * 2), &tm_fq, &ctrl->fixed_full, ch * C::FCH, q0, fslice,
                           leader);
    bool ok = true;
    for (int u = 0; u < nb; ++u) {
      const int s = u % KS;
      if (u >= KS && !(ok = mbar_wait(&ctrl->empty[s], (uint32_t(u / KS) & 1u) ^ 1u, abort))) break;
      uint8_t *st = sStage + s * C::DQ_STAGE;
      const int kv = u * BK;
      mbar_arrive_expect_tx_leader(&ctrl->full[s], C::DQ_STAGE_BYTES, leader);
      for (int ch = 0; ch < C::NDCH; ++ch) {
        tma_load_3d_leader(st + O_K + ch * (BK * C::DCH * 2), &tm_k, &ctrl->full[s], ch * C::DCH, kv, bh, leader);
        tma_load_3d_leader(st + O_V + ch * (BK * C::DCH * 2), &tm_v, &ctrl->full[s], ch * C::DCH, kv, bh, leader);
      }
      if (C::FAC)
        for (int ch = 0; ch < C::NFCH; ++ch)
          tma_load_3d_leader(st + O_FK + ch * (BK * C::FCH * 2), &tm_fk, &ctrl->full[s], ch * C::FCH, kv, fslice,
                             leader);
      for (int ch = 0; ch < C::NGCH; ++ch)
        tma_load_3d_leader(st + O_GK + ch * (BK * C::GCH * 2), &tm_gk, &ctrl->full[s], ch * C::GCH, kv, fslice,
                           leader);
    }
    if (!ok) {
      mbar_wait_for(&ctrl->fixed_full, 0, 100000000ull);
      for (int s = 0; s < KS; ++s) {
        mbar_wait_for(&ctrl->full[s], 0, 100000000ull);
        mbar_wait_for(&ctrl->full[s], 1, 100000000ull);
      }
      if (leader) atomicOr(args.flags, kFlagTimeout);
    }
  } else if (warp == C::MMA_WARP) {
    // ---------------------------------------------------------- MMA issuer
    // S(0), S(1), G(0), S(2), G(1), ... as in the dK/dV kernel.
    const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->fixed_full, 0, abort));
    tc_fence_after();
    const uint64_t aQ = kdesc<C::DCH>(smem_u32(sQ));
    const uint64_t aDO = kdesc<C::DCH>(smem_u32(sDO));
    const uint64_t aFQ = kdesc<C::FCH>(smem_u32(sFQ));
    auto issue_s = [&](int u) -> bool {
      const int s = u % KS;
      if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->full[s], uint32_t(u / KS) & 1u, abort))) return false;
      tc_fence_after();
      const uint32_t st = smem_u32(sStage + s * C::DQ_STAGE);
      const uint32_t s_col = tm_u + uint32_t((u & 1) * 2 * BK);
      uint64_t bk = kdesc<C::DCH>(st + O_K), bv = kdesc<C::DCH>(st + O_V);
      asm volatile("" : "+l"(bk), "+l"(bv));
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)  // S = Q K^T
        mma_ss_elect(s_col, aQ + kstep<C::DCH, 128>(kk), bk + kstep<C::DCH, BK>(kk), C::IDESC_DQ_S, kk > 0 ? 1u : 0u);
      if constexpr (C::FAC) {  // S += phi_q' phi_k'^T
        uint64_t bfk = kdesc<C::FCH>(st + O_FK);
        asm volatile("" : "+l"(bfk));
#pragma unroll
        for (int kk = 0; kk < C::FCH * C::NFCH / 16; ++kk) {
          if (MODE == kBiasTf32)
            mma_ss_elect_tf32(s_col, aFQ + kstep<C::FCH, 128>(kk), bfk + kstep<C::FCH, BK>(kk), C::IDESC_DQ_F, 1u);
          else
            mma_ss_elect(s_col, aFQ + kstep<C::FCH, 128>(kk), bfk + kstep<C::FCH, BK>(kk), C::IDESC_DQ_F, 1u);
        }
      }
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)  // dP = dO V^T
        mma_ss_elect(s_col + BK, aDO + kstep<C::DCH, 128>(kk), bv + kstep<C::DCH, BK>(kk), C::IDESC_DQ_S,
                     kk > 0 ? 1u : 0u);
      tc_commit_elect(&ctrl->s_full[u & 1]);
      __syncwarp();
      return true;
    };
    auto issue_g = [&](int u) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->p_full[u & 1], uint32_t(u >> 1) & 1u, abort))) return false;
      tc_fence_after();
      const int s = u % KS;
      const uint32_t st = smem_u32(sStage + s * C::DQ_STAGE);
      const uint32_t ds_col = tm_u + uint32_t((u & 1) * 2 * BK);  // dS bf16 over S
      uint64_t bk = mndesc<C::DCH, BK>(st + O_K);
      asm volatile("" : "+l"(bk));
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)  // dQ += dS K
        mma_ts_elect(tm_u + C::DQ_DQ, ds_col + uint32_t(kk * 8), bk + mnstep<C::DCH>(kk), C::IDESC_GD,
                     (u > 0 || kk > 0) ? 1u : 0u);
      if constexpr (RG > 0) {  // dphi_q += dS phi_k
        uint64_t bg = mndesc<C::GCH, BK>(st + O_GK);
        asm volatile("" : "+l"(bg));
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          mma_ts_elect(tm_u + C::DQ_DF, ds_col + uint32_t(kk * 8), bg + mnstep<C::GCH>(kk), C::IDESC_GR,
                       (u > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit_elect(&ctrl->empty[s]);
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    if (ok && nb > 1) ok = issue_s(1);
    for (int u = 0; u < nb && ok; ++u) {
      ok = issue_g(u);
      if (ok && u + 2 < nb) ok = issue_s(u + 2);
    }
    if (ok) {
      tc_commit_elect(&ctrl->acc_done);
      __syncwarp();
    }
    if (!ok && leader) atomicOr(args.flags, kFlagTimeout);
  } else {
    // ------------------------------- compute: warpgroup t takes blocks u = t mod 2
    const int t = warp >> 2, quarter = warp & 3;
    const int r_loc = quarter * 32 + lane;
    const int row = q0 + r_loc;  // this thread's query
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_tm = lane_base + uint32_t(t * 2 * BK), dp_tm = s_tm + BK;
    const float sl2 = args.scale_log2;
    const float neg_lse2 = args.nlse2[size_t(bh) * args.Npad + row];  // -inf past N: P = 0
    const float drow = args.delta[size_t(bh) * args.Npad + row];
    const uint64_t sl2x2 = f2_pack(sl2, sl2), nl2 = f2_pack(neg_lse2, neg_lse2), d2 = f2_pack(drow, drow);
    const int lim = args.causal ? min(row + 1, args.N) : args.N;  // keys [0, lim) are visible
    bool ok = true;
    for (int u = t; u < nb; u += 2) {
      ok = mbar_wait(&ctrl->s_full[t], uint32_t(u >> 1) & 1u, abort);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = u * BK;
      const bool edge = key0 + BK > lim;
#pragma unroll
      for (int c = 0; c < BK / 32; ++c) {
        uint32_t sx[32], dx[32];
        tmem_ld32(s_tm + uint32_t(32 * c), sx);
        tmem_ld32(dp_tm + uint32_t(32 * c), dx);
        tmem_ld_wait32(sx);
        tmem_ld_wait32(dx);
        uint32_t dd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {  // two keys per packed f32x2 instruction
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sx[2 * e]), __uint_as_float(sx[2 * e + 1])), sl2x2, nl2), a0, a1);
          float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
          if (edge) {
            const int col = 32 * c + 2 * e;
            if (key0 + col >= lim) p0 = 0.f;
            if (key0 + col + 1 >= lim) p1 = 0.f;
          }
          float g0, g1;
          f2_unpack(f2_mul(f2_pack(p0, p1), f2_sub(f2_pack(__uint_as_float(dx[2 * e]), __uint_as_float(dx[2 * e + 1])), d2)),
                    g0, g1);
          dd[e] = pack_bf16x2(g0, g1);
        }
        tmem_st16(s_tm + uint32_t(16 * c), dd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctrl->p_full[t]);
    }
    if (ok) ok = mbar_wait(&ctrl->acc_done, 0, abort);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      // epilogue: warpgroup 0 writes dQ, warpgroup 1 dphi_q
      tc_fence_after();
      const bool valid = row < args.N;
      if (t == 0) {
        const int d_st = valid ? args.d : 0;
        uint16_t *dq_row = static_cast<uint16_t *>(args.dQ) + (size_t(bh) * args.N + (valid ? row : 0)) * args.d;
#pragma unroll 1
        for (int c0 = 0; c0 < DP; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(lane_base + C::DQ_DQ + uint32_t(c0), r);
          tmem_ld_wait16(r);
          store_row16_bf16(r, args.scale, dq_row, c0, d_st);
        }
      }
      if constexpr (RG > 0) {
        if (t == 1) {
          const int r_st = valid ? args.R : 0;
          store_factor_grad_row<RG>(lane_base + C::DQ_DF, factor_grad_row(args, args.dphi_q, args.dphi_q_part, b, h,
                                                                           bh, valid ? row : 0),
                                    r_st);
        }
      }
    }
    if (!ok && lane == 0) atomicOr(args.flags, kFlagTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}


// ------------------------------------------ fused: dK, dV, dphi_k and dQ, dphi_q
// At head dim 64 with gradient factor width 0 or 64, one kernel does the
// whole backward of a 128-key tile: besides dV, dK and dphi_k (as above),
// each query block contributes dq' = dS [K | phi_k] for its BQ queries. The
// compute warps also write dS^T (bf16) to shared memory, one MMA computes
// dq'^T = [K | phi_k]^T dS^T into TMEM (128 lanes: the concatenated columns;
// BQ TMEM columns: the queries), and a fourth warpgroup reads it out and adds
// it into an fp32 accumulator [BH, Npad, 64 + RG] with TMA reduce-adds
// (performed at L2). The per-row pass zeroes the accumulator beforehand; a
// conversion pass turns it into dQ (bf16, times the scale) and dphi_q. This
// replaces the dQ kernel and with it the second evaluation of S, dP and
// the exponentials.
template <int RP, int MODE, int RG>
struct FusedCfg {
  using B = BwdCfg<64, RP, MODE, RG>;
  static_assert(RG == 0 || RG == 64, "fused backward: gradient factor width 0 or 64");
  static constexpr int BQ = 64;
  static constexpr int DQW = 64 + RG;                // accumulator columns (dQ | dphi_q)
  static constexpr uint32_t TILE = 128u * 64u * 2u;  // one 128-row x 64-column bf16 tile
  static constexpr uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }
  // fixed tiles: K, then phi_k (bf16, RG = 64), V, phi_k' (S side). [K | phi_k]
  // read as one MN-major A operand of 128 rows: its second 64-row chunk is the
  // tile after K (phi_k, or V when RG = 0, whose products are not read).
  static constexpr uint32_t O_K = 0, O_GK = TILE, O_V = O_GK + (RG ? TILE : 0u), O_FK = O_V + TILE;
  static constexpr uint32_t FIXED = O_FK + (B::FAC ? 128u * RP * B::FESZ : 0u);
  static constexpr uint32_t O_DS = align1k(FIXED);    // dS^T [128 keys][64 queries] bf16, one per warpgroup
  // dq' leaves in pieces of QR queries through two staging tiles [QR][DQW]
  // fp32 (8 KB each), so that one is written while the other is being read
  // by its TMA reduce.
  static constexpr int QR = DQW == 128 ? 16 : 32;
  static constexpr uint32_t O_DQS = O_DS + 2 * TILE;
  static constexpr uint32_t DQS_ONE = uint32_t(QR) * DQW * 4u, DQS = 2 * DQS_ONE;
  static constexpr uint32_t O_ST = align1k(O_DQS + DQS);
  static constexpr uint32_t STAGE_BYTES = B::KV_STAGE_BYTES, STAGE = B::KV_STAGE;
  static constexpr uint32_t CTRL = 1024, SLACK = 1024;
  static constexpr int KS_FIT = kSmemLimitB > O_ST + CTRL + SLACK ? int((kSmemLimitB - O_ST - CTRL - SLACK) / STAGE) : 0;
  static constexpr int KS = KS_FIT > 4 ? 4 : KS_FIT;
  static constexpr uint32_t SMEM = O_ST + uint32_t(KS) * STAGE + CTRL + SLACK;
  // warpgroups: 0, 1 compute; 2 the producer warp (8), the MMA warp (9), the
  // warp issuing the dq' MMAs (10: its waits for the readout then hold up
  // nothing else) and an idle warp; 3 the dq' readout. Registers move to the
  // compute warpgroups (shares chosen so that no role spills).
  static constexpr int THREADS = 512;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, DQ_MMA_WARP = 10, DQ_WARP0 = 12;
  static constexpr uint32_t LAUNCH_REGS = 128, REG_COMPUTE = 176, REG_OTHER = 72, REG_DQ = 88;
  static_assert(2 * 128 * REG_COMPUTE + 128 * REG_OTHER + 128 * REG_DQ == THREADS * LAUNCH_REGS, "register split");
  // TMEM columns: buffer t (S^T at t 2BQ, dP^T at t 2BQ + BQ), dV, dK, dphi_k,
  // then dq'^T, twice where the columns allow (the MMA of block u then waits
  // for the readout of block u - 2 instead of u - 1)
  static constexpr uint32_t C_DV = 4 * BQ, C_DK = C_DV + 64, C_DF = C_DK + 64, C_DQ = C_DF + RG;
  static constexpr int NDQ = C_DQ + 2 * BQ <= 512 ? 2 : 1;
  static_assert(C_DQ + NDQ * BQ <= 512, "fused TMEM layout");
  static constexpr uint32_t IDESC_DQ = make_idesc_bf16_mn(128, BQ);
};

struct FusedCtrl {
  uint64_t fixed_full, fixed_empty;  // the item's fixed tiles: loaded / read by its last S and dq' MMAs
  uint64_t full[4], empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t ds_free[2];              // the dq' MMA has read warpgroup t's dS^T tile
  uint64_t dq_full[2], dq_free[2];  // dq'^T buffer b in TMEM: written by the MMA / read by the readout
  uint64_t acc_done, acc_empty;     // the item's dV, dK, dphi_k: complete / read out of TMEM
  uint64_t item_full[4], item_empty[4];  // the work-item ring (producer -> every other warp)
  int item[4];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(FusedCtrl) <= 1024, "control block too large");

// Warps that read each published work item: the MMA warp, the dq' MMA warp,
// the four readout warps and the eight compute warps (lane 0 of each frees
// the ring slot).
constexpr int kFusedItemReaders = 1 + 1 + 4 + 8;

// A work item (key tile, head) of the fused kernel; items are numbered
// heaviest causal key tile first.
struct FusedItem {
  int kb, bh, b, h, k0, fslice, j0, nb;
};
__device__ __forceinline__ FusedItem fused_item(int k, const BwdArgs &a) {
  FusedItem w;
  const int BH = a.B * a.H;
  w.kb = k / BH;
  w.bh = k - w.kb * BH;
  w.b = w.bh / a.H;
  w.h = w.bh - w.b * a.H;
  w.k0 = w.kb * 128;
  w.fslice = (a.fac_B > 1 ? w.b : 0) * a.fac_H + (a.fac_H > 1 ? w.h : 0);
  w.j0 = a.causal ? w.k0 / 64 : 0;  // query blocks before the diagonal see none of these keys
  w.nb = (a.N + 63) / 64 - w.j0;    // >= 1
  return w;
}

// The item of the CTA's pass p: its own index first, then the next unclaimed
// one from the counter (zeroed by the per-row pass before the launch).
__device__ __forceinline__ int fused_claim(int p, int n_items, unsigned int *sched) {
  if (p == 0) return int(blockIdx.x);
  const unsigned int k = gridDim.x + atomicAdd(sched, 1u);
  return k < unsigned(n_items) ? int(k) : -1;
}

// Ring read by one warp: wait for pass p's item, read it, free the slot.
__device__ __forceinline__ int fused_read_item(FusedCtrl *ctrl, int p, volatile int *abort, bool &ok) {
  const int slot = p & 3;
  ok = mbar_wait(&ctrl->item_full[slot], uint32_t(p >> 2) & 1u, abort);
  if (!ok) return -1;
  const int k = *reinterpret_cast<const volatile int *>(&ctrl->item[slot]);
  __syncwarp();
  if ((threadIdx.x & 31u) == 0) mbar_arrive(&ctrl->item_empty[slot]);
  return k;
}

// Persistent: one CTA per SM walks work items (key tile, head). Every
// barrier phase runs on counters that continue across items: g counts query
// blocks (stage ring, score buffers, dq' buffers), p counts items (fixed
// tiles, accumulators).
template <int RP, int MODE, int RG>
__global__ void __launch_bounds__(512, 1)
    attn_bwd_fused_sm100(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_fk, const __grid_constant__ CUtensorMap tm_gk,
                         const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_fq, const __grid_constant__ CUtensorMap tm_gq,
                         const __grid_constant__ CUtensorMap tm_acc, const BwdArgs args) {
  using F = FusedCfg<RP, MODE, RG>;
  using C = typename F::B;
  constexpr int KS = F::KS;
  constexpr int BQ = F::BQ;
  constexpr int DP = 64;
  static_assert(KS >= 3, "configuration does not fit in shared memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem + F::O_K, *sGK = smem + F::O_GK, *sV = smem + F::O_V, *sFK = smem + F::O_FK;
  uint8_t *sDS = smem + F::O_DS;
  float *sDQ = reinterpret_cast<float *>(smem + F::O_DQS);
  uint8_t *sStage = smem + F::O_ST;
  FusedCtrl *ctrl = reinterpret_cast<FusedCtrl *>(sStage + KS * F::STAGE);
  constexpr uint32_t O_Q = 0, O_DO = BQ * DP * 2, O_FQ = 2 * BQ * DP * 2;
  constexpr uint32_t O_GQ = O_FQ + (C::FAC ? BQ * RP * C::FESZ : 0);
  constexpr uint32_t O_L = O_GQ + BQ * RG * 2, O_D = O_L + BQ * 4;
  static_assert(O_D + BQ * 4 == F::STAGE_BYTES, "stage layout");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = args.n_kv * args.B * args.H;

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->fixed_full, 1);
    mbar_init(&ctrl->fixed_empty, 2);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 128);
      mbar_init(&ctrl->ds_free[t], 1);
      mbar_init(&ctrl->dq_full[t], 1);
      mbar_init(&ctrl->dq_free[t], 128);
    }
    mbar_init(&ctrl->acc_done, 1);
    mbar_init(&ctrl->acc_empty, 256);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ctrl->item_full[i], 1);
      mbar_init(&ctrl->item_empty[i], kFusedItemReaders);
    }
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == F::MMA_WARP) {
    tmem_alloc(&ctrl->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;
  volatile int *abort = &ctrl->abort;
  const uint32_t leader = lane == 0 ? 1u : 0u;
  // The set-up above reads no global memory; the per-row terms, the zeroed
  // accumulator and work counter of the kernel before are read only once it
  // has completed.
  griddep_launch_dependents();
  griddep_wait();

  if (warp >= F::PRODUCER_WARP && warp < F::DQ_WARP0) {
    setmaxnreg_dec<F::REG_OTHER>();
    if (warp == F::PRODUCER_WARP) {
      // ---------------------------------------------------------- producer
      // Per item: the first KS query blocks' stages (they free up during the
      // previous item's last blocks), the fixed tiles once the previous item's
      // last S and dq' MMAs have read them, then the remaining stages. The
      // next item is claimed and published after the item's loads.
      if (leader) {
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_do);
        if (C::FAC) {
          tma_prefetch_map(&tm_fk);
          tma_prefetch_map(&tm_fq);
        }
        if (RG > 0) {
          tma_prefetch_map(&tm_gk);
          tma_prefetch_map(&tm_gq);
        }
      }
      bool ok = true;
      int cur = __shfl_sync(0xffffffffu, leader ? fused_claim(0, n_items, args.sched) : 0, 0);
      if (leader) {
        ctrl->item[0] = cur;
        mbar_arrive(&ctrl->item_full[0]);
      }
      int g = 0;
      for (int p = 0; ok && cur >= 0; ++p) {
        const FusedItem w = fused_item(cur, args);
        auto load_stage = [&](int u) -> bool {
          const int gg = g + u;
          const int s = gg % KS;
          if (gg >= KS && !mbar_wait(&ctrl->empty[s], (uint32_t(gg / KS) & 1u) ^ 1u, abort)) return false;
          uint8_t *st = sStage + s * F::STAGE;
          const int q0 = (w.j0 + u) * BQ;
          mbar_arrive_expect_tx_leader(&ctrl->full[s], F::STAGE_BYTES, leader);
          tma_load_3d_leader(st + O_Q, &tm_q, &ctrl->full[s], 0, q0, w.bh, leader);
          tma_load_3d_leader(st + O_DO, &tm_do, &ctrl->full[s], 0, q0, w.bh, leader);
          if (C::FAC)
            for (int ch = 0; ch < C::NFCH; ++ch)
              tma_load_3d_leader(st + O_FQ + ch * (BQ * C::FCH * 2), &tm_fq, &ctrl->full[s], ch * C::FCH, q0,
                                 w.fslice, leader);
          if (RG > 0) tma_load_3d_leader(st + O_GQ, &tm_gq, &ctrl->full[s], 0, q0, w.fslice, leader);
          const size_t roff = size_t(w.bh) * args.Npad + q0;
          bulk_load_leader(st + O_L, args.nlse2 + roff, BQ * 4, &ctrl->full[s], leader);
          bulk_load_leader(st + O_D, args.delta + roff, BQ * 4, &ctrl->full[s], leader);
          return true;
        };
        const int early = w.nb < KS ? w.nb : KS;
        for (int u = 0; u < early && ok; ++u) ok = load_stage(u);
        if (!ok) break;
        if (p > 0 && !(ok = mbar_wait(&ctrl->fixed_empty, uint32_t(p - 1) & 1u, abort))) break;
        mbar_arrive_expect_tx_leader(&ctrl->fixed_full, F::FIXED, leader);
        tma_load_3d_leader(sK, &tm_k, &ctrl->fixed_full, 0, w.k0, w.bh, leader);
        tma_load_3d_leader(sV, &tm_v, &ctrl->fixed_full, 0, w.k0, w.bh, leader);
        if (RG > 0) tma_load_3d_leader(sGK, &tm_gk, &ctrl->fixed_full, 0, w.k0, w.fslice, leader);
        if (C::FAC)
          for (int ch = 0; ch < C::NFCH; ++ch)
            tma_load_3d_leader(sFK + ch * (128 * C::FCH * 2), &tm_fk, &ctrl->fixed_full, ch * C::FCH, w.k0, w.fslice,
                               leader);
        for (int u = early; u < w.nb && ok; ++u) ok = load_stage(u);
        if (!ok) break;
        g += w.nb;
        // the next item, published once its ring slot is free
        const int nxt = __shfl_sync(0xffffffffu, leader ? fused_claim(p + 1, n_items, args.sched) : 0, 0);
        const int slot = (p + 1) & 3;
        if (p + 1 >= 4 && !(ok = mbar_wait(&ctrl->item_empty[slot], uint32_t((p + 1) / 4 - 1) & 1u, abort))) break;
        if (leader) {
          ctrl->item[slot] = nxt;
          mbar_arrive(&ctrl->item_full[slot]);
        }
        cur = nxt;
      }
      if (!ok) {
        // Aborted: let the copies already issued land before the CTA exits.
        mbar_wait_for(&ctrl->fixed_full, 0, 100000000ull);
        mbar_wait_for(&ctrl->fixed_full, 1, 100000000ull);
        for (int s = 0; s < KS; ++s) {
          mbar_wait_for(&ctrl->full[s], 0, 100000000ull);
          mbar_wait_for(&ctrl->full[s], 1, 100000000ull);
        }
        if (leader) atomicOr(args.flags, kFlagTimeout);
      }
    } else if (warp == F::MMA_WARP) {
      // -------------------------------------------------------- MMA issuer
      // Per item: S(0), S(1), then per block u: G(u), S(u + 2), where G(u) is
      // the key-side gradient products (from TMEM P^T, dS^T); the first G of
      // an item waits for the previous item's accumulators to be read out.
      const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
      const uint64_t dK = kdesc<64>(smem_u32(sK));
      const uint64_t dV = kdesc<64>(smem_u32(sV));
      const uint64_t dFK = kdesc<C::FCH>(smem_u32(sFK));
      bool ok = true;
      int g = 0;
      auto issue_s = [&](int gg, int u, int j0) -> bool {
        const int s = gg % KS;
        if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->full[s], uint32_t(gg / KS) & 1u, abort))) return false;
        tc_fence_after();
        const uint32_t st = smem_u32(sStage + s * F::STAGE);
        const uint32_t s_col = tm_u + uint32_t((gg & 1) * 2 * BQ);
        uint64_t dq = kdesc<64>(st + O_Q), ddo = kdesc<64>(st + O_DO);
        asm volatile("" : "+l"(dq), "+l"(ddo));
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk)  // S^T = K Q^T
          mma_ss_elect(s_col, dK + kstep<64, 128>(kk), dq + kstep<64, BQ>(kk), C::IDESC_KV_S, kk > 0 ? 1u : 0u);
        if constexpr (C::FAC) {  // S^T += phi_k' phi_q'^T
          uint64_t dfq = kdesc<C::FCH>(st + O_FQ);
          asm volatile("" : "+l"(dfq));
#pragma unroll
          for (int kk = 0; kk < C::FCH * C::NFCH / 16; ++kk) {
            if (MODE == kBiasTf32)
              mma_ss_elect_tf32(s_col, dFK + kstep<C::FCH, 128>(kk), dfq + kstep<C::FCH, BQ>(kk), C::IDESC_KV_F, 1u);
            else
              mma_ss_elect(s_col, dFK + kstep<C::FCH, 128>(kk), dfq + kstep<C::FCH, BQ>(kk), C::IDESC_KV_F, 1u);
          }
        }
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk)  // dP^T = V dO^T
          mma_ss_elect(s_col + BQ, dV + kstep<64, 128>(kk), ddo + kstep<64, BQ>(kk), C::IDESC_KV_S, kk > 0 ? 1u : 0u);
        tc_commit_elect(&ctrl->s_full[gg & 1]);
        __syncwarp();
        return true;
      };
      auto issue_g = [&](int gg, int u) -> bool {
        if (!__all_sync(0xffffffffu, mbar_wait(&ctrl->p_full[gg & 1], uint32_t(gg >> 1) & 1u, abort))) return false;
        tc_fence_after();
        const int s = gg % KS;
        const uint32_t st = smem_u32(sStage + s * F::STAGE);
        const uint32_t p_col = tm_u + uint32_t((gg & 1) * 2 * BQ);  // P^T bf16 over S^T; dS^T over dP^T
        uint64_t bdo = mndesc<64, BQ>(st + O_DO), bq = mndesc<64, BQ>(st + O_Q);
        asm volatile("" : "+l"(bdo), "+l"(bq));
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
          mma_ts_elect(tm_u + F::C_DV, p_col + uint32_t(kk * 8), bdo + mnstep<64>(kk), C::IDESC_GD, acc);
          mma_ts_elect(tm_u + F::C_DK, p_col + BQ + uint32_t(kk * 8), bq + mnstep<64>(kk), C::IDESC_GD, acc);
        }
        if constexpr (RG > 0) {
          uint64_t bg = mndesc<64, BQ>(st + O_GQ);
          asm volatile("" : "+l"(bg));
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk)
            mma_ts_elect(tm_u + F::C_DF, p_col + BQ + uint32_t(kk * 8), bg + mnstep<64>(kk), C::IDESC_GR,
                         (u > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit_elect(&ctrl->empty[s]);
        __syncwarp();
        return true;
      };
      for (int p = 0; ok; ++p) {
        const int k = fused_read_item(ctrl, p, abort, ok);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || k < 0) break;
        const FusedItem w = fused_item(k, args);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->fixed_full, uint32_t(p) & 1u, abort)))) break;
        tc_fence_after();
        ok = issue_s(g, 0, w.j0);
        if (ok && w.nb > 1) ok = issue_s(g + 1, 1, w.j0);
        if (ok && w.nb <= 2) tc_commit_elect(&ctrl->fixed_empty);  // the item's last S is issued
        for (int u = 0; u < w.nb && ok; ++u) {
          if (u == 0 && p > 0 &&
              !(ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->acc_empty, uint32_t(p - 1) & 1u, abort))))
            break;
          ok = issue_g(g + u, u);
          if (ok && u + 2 < w.nb) {
            ok = issue_s(g + u + 2, u + 2, w.j0);
            if (ok && u + 2 == w.nb - 1) tc_commit_elect(&ctrl->fixed_empty);
          }
        }
        if (!ok) break;
        tc_commit_elect(&ctrl->acc_done);
        __syncwarp();
        g += w.nb;
      }
      if (!ok && leader) atomicOr(args.flags, kFlagTimeout);
    } else if (warp == F::DQ_MMA_WARP) {
      // ------------------------------------------------ dq' MMA issuer
      // Q(g): dq'^T = [K | phi_k]^T dS^T over the item's 128 keys, into TMEM
      // buffer g mod NDQ once the readout has emptied it, as soon as block g's
      // dS^T is in shared memory. After the item's last Q the fixed tiles are
      // free (together with the MMA warp's commit after the last S).
      const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
      const uint64_t aKT = mndesc<64, 128>(smem_u32(sK));  // [K | phi_k]^T, 128 rows
      bool ok = true;
      int g = 0;
      for (int p = 0; ok; ++p) {
        const int k = fused_read_item(ctrl, p, abort, ok);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok || k < 0) break;
        const FusedItem w = fused_item(k, args);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->fixed_full, uint32_t(p) & 1u, abort)))) break;
        for (int u = 0; u < w.nb && ok; ++u, ++g) {
          const int bq = g % F::NDQ;
          ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->p_full[g & 1], uint32_t(g >> 1) & 1u, abort) &&
                                           (g < F::NDQ || mbar_wait(&ctrl->dq_free[bq],
                                                                    uint32_t(g / F::NDQ - 1) & 1u, abort)));
          if (!ok) break;
          tc_fence_after();
          uint64_t bds = mndesc<64, 128>(smem_u32(sDS + (g & 1) * F::TILE));
          asm volatile("" : "+l"(bds));
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ss_elect(tm_u + F::C_DQ + uint32_t(bq * BQ), aKT + mnstep<64>(kk), bds + mnstep<64>(kk), F::IDESC_DQ,
                         kk > 0 ? 1u : 0u);
          tc_commit_elect(&ctrl->dq_full[bq]);
          tc_commit_elect(&ctrl->ds_free[g & 1]);
          __syncwarp();
        }
        if (!ok) break;
        tc_commit_elect(&ctrl->fixed_empty);
        __syncwarp();
      }
      if (!ok && leader) atomicOr(args.flags, kFlagTimeout);
    }
  } else if (warp >= F::DQ_WARP0) {
    setmaxnreg_dec<F::REG_DQ>();
    // ------------------------------------------------------ dq' readout
    // Each thread holds one accumulator column (TMEM lane) for the block's
    // queries and hands TMEM back at once; the block leaves in pieces of QR
    // queries through the two staging tiles, one thread adding each piece
    // into the accumulator with a TMA reduce.
    const int qw = warp & 3;
    const int col = qw * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(qw * 32) << 16);
    const bool has_col = col < F::DQW;
    const bool issuer = warp == F::DQ_WARP0 && lane == 0;
    constexpr int QR = F::QR;
    bool ok = true;
    int pc = 0;  // pieces issued
    int g = 0;
    for (int p = 0; ok; ++p) {
      const int k = fused_read_item(ctrl, p, abort, ok);
      ok = named_bar_and(2, 128, ok);
      if (!ok || k < 0) break;
      const FusedItem w = fused_item(k, args);
      for (int u = 0; u < w.nb; ++u, ++g) {
        const int bq = g % F::NDQ;
        ok = named_bar_and(2, 128, mbar_wait(&ctrl->dq_full[bq], uint32_t(g / F::NDQ) & 1u, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[64];
        tmem_ld32(lane_base + F::C_DQ + uint32_t(bq * BQ), v);
        tmem_ld32(lane_base + F::C_DQ + uint32_t(bq * BQ) + 32, v + 32);
        tmem_ld_wait32(v);
        tmem_ld_wait32(v + 32);
        tc_fence_before();
        mbar_arrive(&ctrl->dq_free[bq]);
        const int q0 = (w.j0 + u) * BQ;
#pragma unroll
        for (int piece = 0; piece < BQ / QR; ++piece, ++pc) {
          float *stg = sDQ + (pc & 1) * (QR * F::DQW);
          if (issuer) bulk_wait_group_read1();  // the reduce that last read this tile is done reading
          named_bar_sync(1, 128);
          if (has_col) {
#pragma unroll
            for (int i = 0; i < QR; ++i) stg[i * F::DQW + col] = __uint_as_float(v[QR * piece + i]);
          }
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (issuer) {
            tma_reduce_add_3d(&tm_acc, stg, 0, q0 + QR * piece, w.bh);
            bulk_commit_group();
          }
        }
      }
    }
    // the staging tiles must outlive the reads of the last reduces; the adds
    // themselves complete with the kernel
    if (issuer) bulk_wait_group_read0();
    if (!ok && lane == 0) atomicOr(args.flags, kFlagTimeout);
  } else {
    setmaxnreg_inc<F::REG_COMPUTE>();
    // ------------------------------- compute: warpgroup t takes blocks g = t mod 2
    const int t = warp >> 2, quarter = warp & 3;
    const int r_loc = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_tm = lane_base + uint32_t(t * 2 * BQ), dp_tm = s_tm + BQ;
    // this thread's row of the dS^T tile (128-byte rows, 16-byte chunks swizzled by row)
    const uint32_t ds_row = smem_u32(sDS + t * F::TILE) + uint32_t(r_loc) * 128u;
    const uint32_t sw = uint32_t(r_loc) & 7u;
    const float sl2 = args.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    int g0 = 0;  // the item's first block
    for (int p = 0; ok; ++p) {
      const int k = fused_read_item(ctrl, p, abort, ok);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok || k < 0) break;
      const FusedItem w = fused_item(k, args);
      const int krow = w.k0 + r_loc;  // this thread's key
      for (int g = g0 + ((g0 & 1) != t ? 1 : 0); g < g0 + w.nb; g += 2) {
        const int u = g - g0;
        const int s = g % KS;
        ok = mbar_wait(&ctrl->full[s], uint32_t(g / KS) & 1u, abort) &&
             mbar_wait(&ctrl->s_full[t], uint32_t(g >> 1) & 1u, abort) &&
             (g < 2 || mbar_wait(&ctrl->ds_free[t], uint32_t((g >> 1) - 1) & 1u, abort));
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t *st = sStage + s * F::STAGE;
        const float *sL = reinterpret_cast<const float *>(st + O_L);
        const float *sD = reinterpret_cast<const float *>(st + O_D);
        const int q0 = (w.j0 + u) * BQ;
        const bool diag = args.causal && q0 < w.k0 + 127;
#pragma unroll
        for (int c = 0; c < BQ / 32; ++c) {
          uint32_t sx[32], dx[32];
          tmem_ld32(s_tm + uint32_t(32 * c), sx);
          tmem_ld32(dp_tm + uint32_t(32 * c), dx);
          tmem_ld_wait32(sx);
          tmem_ld_wait32(dx);
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = *reinterpret_cast<const float4 *>(sL + 32 * c + 4 * e4);
            const float4 d4 = *reinterpret_cast<const float4 *>(sD + 32 * c + 4 * e4);
            const uint64_t l2[2] = {f2_pack(l4.x, l4.y), f2_pack(l4.z, l4.w)};
            const uint64_t d2[2] = {f2_pack(d4.x, d4.y), f2_pack(d4.z, d4.w)};
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int i = 4 * e4 + 2 * h2;
              float a0, a1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sx[i]), __uint_as_float(sx[i + 1])), sl2x2, l2[h2]), a0, a1);
              float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
              if (diag) {
                const int cq = 32 * c + i;
                if (q0 + cq < krow) p0 = 0.f;
                if (q0 + cq + 1 < krow) p1 = 0.f;
              }
              const uint64_t p2 = f2_pack(p0, p1);
              float g0f, g1f;
              f2_unpack(f2_mul(p2, f2_sub(f2_pack(__uint_as_float(dx[i]), __uint_as_float(dx[i + 1])), d2[h2])),
                        g0f, g1f);
              pp[2 * e4 + h2] = pack_bf16x2(p0, p1);
              dd[2 * e4 + h2] = pack_bf16x2(g0f, g1f);
            }
          }
          tmem_st16(s_tm + uint32_t(16 * c), pp);
          tmem_st16(dp_tm + uint32_t(16 * c), dd);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            st_shared_v4(ds_row + (((uint32_t(4 * c + jj)) ^ sw) << 4), dd[4 * jj], dd[4 * jj + 1], dd[4 * jj + 2],
                         dd[4 * jj + 3]);
        }
        tmem_st_wait();
        fence_proxy_async_smem();  // dS^T in shared memory, for the dq' MMA
        tc_fence_before();
        mbar_arrive(&ctrl->p_full[t]);
      }
      if (!ok) break;
      g0 += w.nb;
      // epilogue of the item: warpgroup 0 writes dV, warpgroup 1 dK, each half
      // of dphi_k's columns; the accumulators are handed back once loaded
      ok = __all_sync(0xffffffffu, mbar_wait(&ctrl->acc_done, uint32_t(p) & 1u, abort));
      if (!ok) break;
      tc_fence_after();
      const bool valid = krow < args.N;
      const int d_st = valid ? args.d : 0;
      const size_t row_off = (size_t(w.bh) * args.N + (valid ? krow : 0)) * args.d;
      uint16_t *dst = static_cast<uint16_t *>(t == 0 ? args.dV : args.dK) + row_off;
      const uint32_t acc_tm = lane_base + (t == 0 ? F::C_DV : F::C_DK);
      const float mul = t == 0 ? 1.f : args.scale;
      uint32_t r[64], gr[RG > 0 ? 32 : 1];
      tmem_ld32(acc_tm, r);
      tmem_ld32(acc_tm + 32, r + 32);
      if constexpr (RG > 0) tmem_ld32(lane_base + F::C_DF + uint32_t(32 * t), gr);
      tmem_ld_wait32(r);
      tmem_ld_wait32(r + 32);
      if constexpr (RG > 0) tmem_ld_wait32(gr);
      tc_fence_before();
      mbar_arrive(&ctrl->acc_empty);
#pragma unroll
      for (int c0 = 0; c0 < DP; c0 += 16) store_row16_bf16(r + c0, mul, dst, c0, d_st);
      if constexpr (RG > 0) {
        // columns [32 t, 32 t + 32) of this key's dphi_k row, those below R
        float *frow =
            factor_grad_row(args, args.dphi_k, args.dphi_k_part, w.b, w.h, w.bh, valid ? krow : 0) + 32 * t;
        const int n_st = valid ? min(32, max(0, args.R - 32 * t)) : 0;
        const bool vec = (n_st & 3) == 0 && (reinterpret_cast<uintptr_t>(frow) & 15u) == 0;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          if (vec) {
            if (e < n_st)
              *reinterpret_cast<float4 *>(frow + e) = make_float4(
                  __uint_as_float(gr[e]), __uint_as_float(gr[e + 1]), __uint_as_float(gr[e + 2]), __uint_as_float(gr[e + 3]));
          } else {
#pragma unroll
            for (int x = 0; x < 4; ++x)
              if (e + x < n_st) frow[e + x] = __uint_as_float(gr[e + x]);
          }
        }
      }
    }
    if (!ok && lane == 0) atomicOr(args.flags, kFlagTimeout);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == F::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

namespace {

constexpr int kMaxDevicesB = 64;

// The fused kernel serves head dim 64 with gradient factor width 0 or 64.
template <int DP, int RP, int MODE, int RG>
constexpr bool fused_ok() {
  if constexpr (DP == 64 && (RG == 0 || RG == 64))
    return FusedCfg<RP, MODE, RG>::KS >= 3;
  else
    return false;
}

template <int RP, int MODE, int RG>
cudaError_t launch_bwd_fused(const BwdMaps &m, const BwdArgs &a, cudaStream_t stream) {
  using F = FusedCfg<RP, MODE, RG>;
  auto kern = attn_bwd_fused_sm100<RP, MODE, RG>;
  static std::atomic<int> ready[kMaxDevicesB];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesB) return cudaErrorInvalidDevice;
  if (!ready[dev].load(std::memory_order_acquire)) {
    // setmaxnreg.inc waits until the block's pool has the registers, so the
    // launch allocation must be exactly what the split assumes.
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    if (fa.numRegs != int(F::LAUNCH_REGS)) return cudaErrorInvalidConfiguration;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(F::SMEM))) != cudaSuccess)
      return e;
    ready[dev].store(1, std::memory_order_release);
  }
  // persistent: one CTA per SM (the TMEM allocation and the shared memory
  // admit one), never more than there are work items
  int sms = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long items = (long long)a.n_kv * a.B * a.H;
  const unsigned grid = unsigned(std::min<long long>(items, sms));
  return launch_programmatic(kern, dim3(grid), dim3(F::THREADS), F::SMEM, stream, m.k, m.v, m.fk, m.gk, m.q_blk,
                             m.do_blk, m.fq_blk, m.gq_blk, m.acc, a);
}

template <int DP, int RP, int MODE, int RG>
cudaError_t launch_bwd_one(const BwdMaps &m, const BwdArgs &a, cudaStream_t stream) {
  using C = BwdCfg<DP, RP, MODE, RG>;
  if constexpr (fused_ok<DP, RP, MODE, RG>()) {
    return launch_bwd_fused<RP, MODE, RG>(m, a, stream);
  } else if constexpr (C::KV_KS < 1 || C::DQ_KS < 1) {
    return cudaErrorInvalidConfiguration;
  } else {
    auto kv = attn_bwd_dkdv_sm100<DP, RP, MODE, RG>;
    auto dq = attn_bwd_dq_sm100<DP, RP, MODE, RG>;
    static std::atomic<int> ready[kMaxDevicesB];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevicesB) return cudaErrorInvalidDevice;
    if (!ready[dev].load(std::memory_order_acquire)) {
      if ((e = cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::KV_SMEM))) != cudaSuccess)
        return e;
      if ((e = cudaFuncSetAttribute(dq, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::DQ_SMEM))) != cudaSuccess)
        return e;
      ready[dev].store(1, std::memory_order_release);
    }
    const unsigned grid = unsigned((long long)a.n_kv * a.B * a.H);
    kv<<<grid, C::THREADS, C::KV_SMEM, stream>>>(m.k, m.v, m.fk, m.q_blk, m.do_blk, m.fq_blk, m.gq_blk, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dq<<<grid, C::THREADS, C::DQ_SMEM, stream>>>(m.q, m.dO, m.fq, m.k_blk, m.v_blk, m.fk_blk, m.gk_blk, a);
    return cudaGetLastError();
  }
}

template <int DP, int RP, int MODE, int RG>
constexpr int bwd_block_rows() {
  return BwdCfg<DP, RP, MODE, RG>::BQ;
}
template <int DP, int RP, int MODE, int RG>
constexpr int bwd_key_block_rows() {
  return BwdCfg<DP, RP, MODE, RG>::BK;
}

}  // namespace

// RG = 0: the factors are fixed (no factor gradients requested)
#define FB_BWD_MODE(DPv)                                                            \
  if (p.mode == kBiasNone) return FB_BWD_ACTION(DPv, 0, kBiasNone, 0);              \
  if (p.mode == kBiasTf32) {                                                        \
    if (p.RP == 8) return p.RG ? FB_BWD_ACTION(DPv, 8, kBiasTf32, 16) : FB_BWD_ACTION(DPv, 8, kBiasTf32, 0);    \
    if (p.RP == 16) return p.RG ? FB_BWD_ACTION(DPv, 16, kBiasTf32, 16) : FB_BWD_ACTION(DPv, 16, kBiasTf32, 0); \
  }                                                                                 \
  if (p.mode == kBiasMma) {                                                         \
    if (p.RP == 16) return p.RG ? FB_BWD_ACTION(DPv, 16, kBiasMma, 16) : FB_BWD_ACTION(DPv, 16, kBiasMma, 0);   \
    if (p.RP == 32) return p.RG ? FB_BWD_ACTION(DPv, 32, kBiasMma, 32) : FB_BWD_ACTION(DPv, 32, kBiasMma, 0);   \
    if (p.RP == 64) return p.RG ? FB_BWD_ACTION(DPv, 64, kBiasMma, 64) : FB_BWD_ACTION(DPv, 64, kBiasMma, 0);   \
    if (p.RP == 128) return p.RG ? FB_BWD_ACTION(DPv, 128, kBiasMma, 128) : FB_BWD_ACTION(DPv, 128, kBiasMma, 0); \
  }

#define FB_BWD_ALL                                                                  \
  if (p.DP == 16) { FB_BWD_MODE(16) }                                               \
  if (p.DP == 32) { FB_BWD_MODE(32) }                                               \
  if (p.DP == 64) { FB_BWD_MODE(64) }                                               \
  if (p.DP == 128) { FB_BWD_MODE(128) }

int bwd_query_block_rows(const BwdPlan &p) {
#define FB_BWD_ACTION(DPv, RPv, MODEv, RGv) bwd_block_rows<DPv, RPv, MODEv, RGv>()
  FB_BWD_ALL
#undef FB_BWD_ACTION
  return 0;
}

bool bwd_fused(const BwdPlan &p) {
#define FB_BWD_ACTION(DPv, RPv, MODEv, RGv) fused_ok<DPv, RPv, MODEv, RGv>()
  FB_BWD_ALL
#undef FB_BWD_ACTION
  return false;
}

int bwd_key_block_rows(const BwdPlan &p) {
#define FB_BWD_ACTION(DPv, RPv, MODEv, RGv) bwd_key_block_rows<DPv, RPv, MODEv, RGv>()
  FB_BWD_ALL
#undef FB_BWD_ACTION
  return 0;
}

cudaError_t bwd_launch(const BwdPlan &p, const BwdMaps &maps, const BwdArgs &a, cudaStream_t stream) {
#define FB_BWD_ACTION(DPv, RPv, MODEv, RGv) launch_bwd_one<DPv, RPv, MODEv, RGv>(maps, a, stream)
  FB_BWD_ALL
#undef FB_BWD_ACTION
  return cudaErrorInvalidConfiguration;
}

}  // namespace fb
