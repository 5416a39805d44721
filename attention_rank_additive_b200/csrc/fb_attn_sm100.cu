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
// rank <= 4 (the ALiBi factors, Example 3.4; rebuttal, reply to Reviewer
// BRmd, Q2 (2)) fp16 cannot hold the factors, and they enter as a tf32 MMA
// of hi/lo split fp32 values instead (q' = [qh, qh, ql], k' = [kh, kl, kh]),
// which keeps fp32-level accuracy at one extra K = 8 or 16 MMA per tile.
// The dense mode streams a materialised bias tile per tile pair: the
// "FlashAttention w/ Bias" comparison path of Figure 1(c).
//
// Work items: one (batch, head, group of QT query tiles of 128 rows) each.
// The grid is persistent (at most as many CTAs as are resident at once); CTA
// c takes items c, 2G-1-c, 2G+c, ... (G CTAs), heaviest causal groups first,
// so the heavy and light items of successive passes even out. Barrier phases
// run on counters that continue across items, so the next item's Q and K/V
// stream in while the current one finishes, and O is handed back through an
// o_free barrier once the epilogue has read it.
//
// CTA organisation (QT = 1 or 2 query tiles of 128 rows per CTA):
//   warps 0..4QT-1  softmax warpgroups; warpgroup t owns query tile t, one
//                   thread per row (TMEM lane), so row max and row sum are
//                   thread-local; it also rescales O in TMEM when the running
//                   max grows by more than 2^8 and writes the epilogue.
//   warp 4QT        TMA producer (one thread): Q|phi_q per item, then K|phi_k
//                   and V per 128-key step into a KS-deep ring, plus the
//                   softmax-side tiles (dense bias / rank<=4 factors).
//   warp 4QT+1      TMEM allocator and MMA issuer (one elected lane); with
//   (and 4QT+2)     a separate P tile (head dim <= 64) one issuer per tile.
// Head dim <= 64: TMEM holds S_t (128 columns), P_t (64 columns of bf16
// pairs) and O_t per tile, so S_t(i+1) is computed as soon as the softmax has
// read S_t(i) into registers, while P_t(i) waits for PV_t(i).
// Head dim 128: P_t overwrites the first 64 columns of S_t, and one issuer
// runs S_0(i), PV_1(i-1), S_1(i), PV_0(i), so the tensor core works on one
// tile while the softmax of the other runs; the commit that publishes S_t(i)
// also covers PV_t(i-1), and S_t(i+1) (which overwrites P_t(i)) follows
// PV_t(i) (tcgen05 MMAs of one thread run in order).
#include <algorithm>
#include <atomic>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

#ifndef FB_KS_MAX
#define FB_KS_MAX 2
#endif

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
  // Factor tiles: fp16 [128 x RP] (mma) or fp32 [128 x RP] (tf32). RCH is a
  // chunk's width in 16-bit units (the descriptors and swizzle are made from
  // the chunk's byte width, so a tf32 row of RP floats is 2 RP such units).
  static constexpr bool FAC_MMA = MODE == kBiasMma || MODE == kBiasTf32;
  static constexpr int RCH = MODE == kBiasMma ? (RP > 64 ? 64 : RP) : (MODE == kBiasTf32 ? 2 * RP : 16);
  static constexpr int NRCH = MODE == kBiasMma ? RP / RCH : (MODE == kBiasTf32 ? 1 : 0);
  static constexpr uint32_t Q_TILE = BM * DP * 2;
  static constexpr uint32_t KV_TILE = BN * DP * 2;
  static constexpr uint32_t FQ_TILE = MODE == kBiasMma ? BM * RP * 2 : (MODE == kBiasTf32 ? BM * RP * 4 : 0);
  static constexpr uint32_t FK_TILE = MODE == kBiasMma ? BN * RP * 2 : (MODE == kBiasTf32 ? BN * RP * 4 : 0);
  static constexpr uint32_t AUX_TILE = MODE == kBiasDense ? BM * BN * 2 : 0;
  static constexpr bool HAS_AUX = AUX_TILE > 0;
  static constexpr uint32_t FIXED = QT * (Q_TILE + FQ_TILE);
  static constexpr uint32_t STAGE = 2 * KV_TILE + FK_TILE + QT * AUX_TILE;
  // Key split (head dim 128, one query tile): two softmax warpgroups share
  // the tile's rows, warpgroup h taking keys 64h .. 64h+63 of every key tile
  // with its own running max, row sum and O accumulator; the two partial
  // results are merged once per item in the epilogue. TMEM: S 128 + P 64 +
  // 2 x O 128 = 448 columns, so S(i+1) never waits for PV(i).
  static constexpr bool KSPLIT = DP == 128 && QT == 1;
  static constexpr int NSWG = KSPLIT ? 2 : QT;  // softmax warpgroups
  static constexpr uint32_t XCH = KSPLIT ? 4u * 2u * 2u * 2u * 32u * 4u : 0u;  // [quarter][half][slot][m,l][lane]
  static constexpr uint32_t CTRL = 1024 + XCH;  // barriers, TMEM address, abort flag, exchange
  static constexpr uint32_t ALIGN_SLACK = 1024;
  static constexpr int KS_FIT = (kSmemLimit > FIXED + CTRL + ALIGN_SLACK)
                                    ? int((kSmemLimit - FIXED - CTRL - ALIGN_SLACK) / STAGE)
                                    : 0;
  static constexpr int KS_MAX = FB_KS_MAX;
  static constexpr int KS = KS_FIT > KS_MAX ? KS_MAX : KS_FIT;
  // QT softmax warpgroups + one warpgroup holding the producer warp, the MMA
  // warp and two idle warps. Registers are moved from that warpgroup to the
  // softmax warpgroups with setmaxnreg: the launch allocation is
  // THREADS * LAUNCH_REGS and the shares below add up to exactly that.
  static constexpr int THREADS = NSWG * 128 + 128;
  static constexpr bool SMALL = QT == 1 && !KSPLIT;  // two CTAs per SM
  // Epilogue: O leaves through shared memory and TMA stores, EPI_E columns of
  // a warp's 32 rows at a time (one staging slot per softmax warp), when the
  // slots fit beside the rings (for a two-per-SM plan: within half an SM);
  // otherwise each thread stores its own row.
  static constexpr uint32_t SMEM_BASE = FIXED + uint32_t(KS) * STAGE + CTRL + ALIGN_SLACK;
  static constexpr uint32_t kPairLimit = 228u * 1024u / 2u - 1024u;
  static constexpr uint32_t SMEM_CAP = (SMALL && SMEM_BASE <= kPairLimit) ? kPairLimit : kSmemLimit;
  // a whole 64-column row chunk per warp where it fits (one store per warp
  // for head dims up to 64), else 32 columns (the key split always uses 32)
  static constexpr int EPI_E_WIDE = DP < 64 ? DP : 64;
  static constexpr bool WIDE_FITS =
      !KSPLIT && SMEM_BASE + uint32_t(NSWG) * 4u * 32u * uint32_t(EPI_E_WIDE) * 2u <= SMEM_CAP;
  static constexpr int EPI_E = WIDE_FITS ? EPI_E_WIDE : (DP < 32 ? DP : 32);
  static constexpr uint32_t STG_WARP = 32u * uint32_t(EPI_E) * 2u;
  static constexpr uint32_t STG = uint32_t(NSWG) * 4u * STG_WARP;
  static constexpr bool TMA_EPI = SMEM_BASE + STG <= SMEM_CAP;
  static constexpr uint32_t SMEM = SMEM_BASE + (TMA_EPI ? STG : 0u);
  static constexpr int MIN_BLOCKS = SMALL ? 2 : 1;
  static constexpr int LAUNCH_REGS = SMALL ? 128 : 168;
  static constexpr int REG_SOFTMAX = SMALL ? 192 : 216;
  static constexpr int REG_OTHER = SMALL ? 64 : 72;
  static_assert(NSWG * 128 * REG_SOFTMAX + 128 * REG_OTHER == THREADS * LAUNCH_REGS, "register split");
  static constexpr int PRODUCER_WARP = NSWG * 4;
  static constexpr int MMA_WARP = NSWG * 4 + 1;
  static constexpr uint32_t TMEM_COLS = SMALL ? 256 : 512;
  // With DP <= 64 (and with the key split) the bf16 P tile gets its own 64
  // TMEM columns, so S(i+1) can be computed while the softmax of S(i) is
  // still running; with DP = 128 and two query tiles P overwrites the first
  // 64 columns of S.
  static constexpr bool SEP_P = DP <= 64 || KSPLIT;
  static constexpr uint32_t S_COL0 = 0;                                // + 128 t
  static constexpr uint32_t P_COL0 = SEP_P ? 128 * QT : 0;             // + (SEP_P ? 64 : 128) t
  static constexpr uint32_t P_STRIDE = SEP_P ? 64 : 128;
  static constexpr uint32_t O_COL0 = SEP_P ? 128 * QT + 64 * QT : 128 * QT;  // + O_STRIDE t (or half h)
  static constexpr uint32_t O_STRIDE = SEP_P ? DP : 128;
  static_assert(O_COL0 + O_STRIDE * (KSPLIT ? 2 : QT) <= TMEM_COLS, "TMEM layout");
  // MMA issuer warps (one per query tile or key half with separate P, else
  // one), each of which releases every K/V stage once per key step.
  static constexpr int RELEASERS = SEP_P ? NSWG : 1;
  // Warps that read the work-item ring: the MMA issuers and the softmax warps.
  static constexpr int ITEM_READERS = RELEASERS + 4 * NSWG;
  static constexpr uint32_t IDESC_QK = make_idesc_f16(true, true, 128, 128, false);
  static constexpr uint32_t IDESC_F =
      MODE == kBiasTf32 ? make_idesc_tf32(128, 128) : make_idesc_f16(false, false, 128, 128, false);
  static constexpr uint32_t IDESC_PV = make_idesc_f16(true, true, 128, DP, true);
};

struct SmemCtrl {
  uint64_t q_full, q_empty;
  uint64_t o_final[2], o_free[2];
  uint64_t drain[2];
  uint64_t s_free[2], pv_done[2];  // separate-P schedule only
  uint64_t k_full[3], v_full[3];
  uint64_t k_empty[3], v_empty[3];  // one arrival per MMA issuer per key step
  uint64_t s_full[2], p_full[2];
  uint64_t aux_full[2][3], aux_empty[2][3];
  uint64_t pair[4];  // key split: the two halves of a 32-row quarter exchange (m, l)
  uint64_t item_full[4], item_empty[4];  // the work-item ring (producer -> every other role)
  int item[4];
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

// Maximum of the NC floats (bit patterns) in x: eight independent chains of
// three-input max, one instruction per two elements.
template <int NC>
__device__ __forceinline__ float row_max(const uint32_t *x) {
  static_assert(NC % 8 == 0 && NC >= 24, "row_max");
  float mp[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mp[e] = fmax3(__uint_as_float(x[e]), __uint_as_float(x[8 + e]), __uint_as_float(x[16 + e]));
#pragma unroll
  for (int c = 24; c + 16 <= NC; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) mp[e] = fmax3(mp[e], __uint_as_float(x[c + e]), __uint_as_float(x[c + 8 + e]));
  if constexpr ((NC - 24) % 16 == 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) mp[e] = fmaxf(mp[e], __uint_as_float(x[NC - 8 + e]));
  }
  return fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
}

// One chunk of the epilogue: a warp's 32 rows x E bf16 columns (thread =
// row; pk holds its E/2 packed pairs) go into the warp's staging slot, laid
// out in the TMA swizzle of an E*2-byte row (128 B: 16-byte chunk j of row r
// at j ^ (r & 7); 64 B: at j ^ ((r >> 1) & 3); 32 B: at j ^ ((r >> 2) & 1)), so that the
// row-per-thread writes are free of bank conflicts; lane 0 then issues one
// tiled store of the slot at (col, row0, bh). The slot is rewritten only
// after its previous store has read it.
template <int E>
__device__ __forceinline__ void stage_and_store_o(uint8_t *slot, const uint32_t *pk, int lane, const CUtensorMap *map,
                                                  int col, int row0, int bh) {
  static_assert(E == 16 || E == 32 || E == 64, "staging chunk");
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
#pragma unroll
  for (int j = 0; j < E / 8; ++j) {
    const int pj = E == 64 ? (j ^ (lane & 7)) : (E == 32 ? (j ^ ((lane >> 1) & 3)) : (j ^ ((lane >> 2) & 1)));
    *reinterpret_cast<uint4 *>(slot + lane * (E * 2) + pj * 16) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(map, slot, col, row0, bh);
    bulk_commit_group();
  }
}

// Dense-bias comparison path: x[c] = scale * x[c] + bias[c] (natural-log
// units; the softmax then multiplies by log2 e) for 64 columns of this
// thread's row, the bias read from its 128-byte-swizzled bf16 tile in shared
// memory (16-byte chunk j of row r at j ^ (r & 7)). A bf16 pair becomes an
// fp32 pair by a shift and a mask, then one packed fma per pair.
__device__ __forceinline__ void add_dense_bias(uint32_t *x, const uint8_t *tile, int r_loc, float scale) {
  const uint64_t sc2 = f2_pack(scale, scale);
#pragma unroll
  for (int ck = 0; ck < 8; ++ck) {
    const uint4 u = *reinterpret_cast<const uint4 *>(tile + r_loc * 128 + ((ck ^ (r_loc & 7)) * 16));
    const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = ck * 8 + 2 * e;
      const uint64_t b2 = f2_pack(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
      const uint64_t r2 = f2_fma(f2_pack(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), sc2, b2);
      float lo, hi;
      f2_unpack(r2, lo, hi);
      x[c] = __float_as_uint(lo);
      x[c + 1] = __float_as_uint(hi);
    }
  }
}

// One schedulable work item: a group of QT query tiles of one (b, h) head.
struct WorkItem {
  int bh, b, h, fb_slice;
  int q0[2], nk[2], first[2], n_steps;
};

template <int QT, bool GROUPED>
__device__ __forceinline__ WorkItem make_item(int k, const FwdArgs &a) {
  // Items in groups of head_group heads, and within a group heaviest query
  // groups first (causal work grows with the query index): the CTAs at work
  // then share few heads, whose K and V stay in L2 while every query group of
  // the head reads them. One group (the plain heaviest-first order) when all
  // heads' K and V fit in L2 anyway. Only the head-dim-128 kernels carry the
  // grouped form (GROUPED): at the smaller head dims all heads' K and V fit
  // for the sequence lengths at hand, and the extra code cost the d = 16
  // kernel 3 % through register allocation.
  const int BH = a.B * a.H;
  WorkItem w;
  const int G = GROUPED ? a.head_group : BH;
  int qg;
  if (!GROUPED || G >= BH) {
    w.bh = k % BH;
    qg = a.n_cta_q - 1 - k / BH;
  } else {
    const int per_group = G * a.n_cta_q;
    const int n_groups = (BH + G - 1) / G;
    const int grp = min(k / per_group, n_groups - 1);
    const int first = grp * G;
    const int gh = min(G, BH - first);  // heads in this group
    const int i = k - grp * per_group;
    w.bh = first + i % gh;
    qg = a.n_cta_q - 1 - i / gh;
  }
  w.b = w.bh / a.H;
  w.h = w.bh - w.b * a.H;
  w.fb_slice = (a.fac_B > 1 ? w.b : 0) * a.fac_H + (a.fac_H > 1 ? w.h : 0);
  // Key tiles are visited from the last one down (step i reads key tile
  // n_steps - 1 - i), so for a causal mask the diagonal comes first: biases
  // that decay away from the diagonal then set the running max at once and O
  // is rarely rescaled. Tile t is active for steps first[t] .. n_steps - 1.
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = qg * QT + t;
    w.q0[t] = qt * 128;
    const bool active = (t < QT) && (w.q0[t] < a.N);
    w.nk[t] = active ? (a.causal ? min(qt + 1, a.n_kv) : a.n_kv) : 0;
  }
  w.n_steps = max(w.nk[0], w.nk[1]);
  w.first[0] = w.n_steps - w.nk[0];
  w.first[1] = w.n_steps - w.nk[1];
  return w;
}

// Entry t of a per-tile pair, by select: t is warp-dependent, and indexing
// the pair with it would put the work item in local memory.
__device__ __forceinline__ int pick(const int (&v)[2], int t) { return t == 0 ? v[0] : v[1]; }

// Work item of this CTA's p-th pass, or -1: items are dealt out in passes of
// gridDim.x, alternating direction each pass so that the heavy items of one
// pass and the light items of the next even out across CTAs.
__device__ __forceinline__ int item_of_pass(int p, int n_items) {
  const int G = int(gridDim.x), c = int(blockIdx.x);
  const int k = p * G + ((p & 1) ? (G - 1 - c) : c);
  return k < n_items ? k : -1;
}

// The p-th work item of this CTA. With a work counter (sched), CTA c starts
// with item c (items are numbered heaviest first and the grid is never larger
// than the item count) and then takes the items after the first gridDim.x in
// order, each when it gets to it, so that the CTAs finish together whatever
// their item mix and speed; without a counter, the fixed passes above. Items
// are claimed by the producer's lane 0 only.
__device__ __forceinline__ int claim_item(int p, int n_items, unsigned int *sched) {
  if (sched == nullptr) return item_of_pass(p, n_items);
  if (p == 0) return int(blockIdx.x);
  const unsigned int k = gridDim.x + atomicAdd(sched, 1u);
  return k < unsigned(n_items) ? int(k) : -1;
}

// After its last claim, each CTA counts itself out on sched[1]; the last one
// resets both words, so the counter starts at zero for the next launch in
// stream order (the factor preparation zeroes it before the first).
__device__ __forceinline__ void release_sched(unsigned int *sched) {
  if (sched == nullptr) return;
  __threadfence();
  if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
    sched[0] = 0u;
    sched[1] = 0u;
    __threadfence();
  }
}

// Work-item ring: the producer publishes the item of pass p (or -1: no more)
// in slot p % 4; every reading warp waits for it, reads it and frees the slot.
__device__ __forceinline__ int read_item(uint64_t *full, uint64_t *empty, const int *items, int p,
                                         volatile int *abort, bool &ok) {
  const int slot = p & 3;
  ok = mbar_wait(&full[slot], uint32_t(p >> 2) & 1u, abort);
  if (!ok) return -1;
  const int k = *reinterpret_cast<const volatile int *>(&items[slot]);
  __syncwarp();
  if ((threadIdx.x & 31u) == 0) mbar_arrive(&empty[slot]);
  return k;
}

template <int DP, int RP, int MODE, int QT>
__global__ void __launch_bounds__(Sm100Cfg<DP, RP, MODE, QT>::THREADS, Sm100Cfg<DP, RP, MODE, QT>::MIN_BLOCKS)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_fq,
                   const __grid_constant__ CUtensorMap tm_fk, const __grid_constant__ CUtensorMap tm_bias,
                   const __grid_constant__ CUtensorMap tm_o, const FwdArgs args) {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  constexpr int KS = C::KS;
  static_assert(KS >= 1, "configuration does not fit in shared memory");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                    // QT x Q_TILE
  uint8_t *sFQ = sQ + QT * C::Q_TILE;    // QT x FQ_TILE
  uint8_t *sK = sFQ + QT * C::FQ_TILE;   // KS x KV_TILE
  uint8_t *sFK = sK + KS * C::KV_TILE;   // KS x FK_TILE
  uint8_t *sV = sFK + KS * C::FK_TILE;   // KS x KV_TILE
  uint8_t *sAux = sV + KS * C::KV_TILE;  // QT x KS x AUX_TILE
  constexpr uint32_t STG_OFF = QT * (C::Q_TILE + C::FQ_TILE) + KS * (2 * C::KV_TILE + C::FK_TILE + QT * C::AUX_TILE);
  uint8_t *sStg = smem + STG_OFF;  // NSWG x 4 x STG_WARP (TMA_EPI), 1024-aligned
  SmemCtrl *ctrl = reinterpret_cast<SmemCtrl *>(sStg + (C::TMA_EPI ? C::STG : 0u));
  // The epilogue's staging slot of softmax warp wi, recomputed from the
  // shared-memory base where it is needed rather than kept live in a register.
  auto stg_slot = [&](int wi) {
    const uintptr_t base = (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023);
    return reinterpret_cast<uint8_t *>(base) + STG_OFF + uint32_t(wi) * C::STG_WARP;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = args.N;
  const int n_items = args.n_cta_q * args.B * args.H;

  if (threadIdx.x == 0) {
    mbar_init(&ctrl->q_full, 1);
    mbar_init(&ctrl->q_empty, C::RELEASERS);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&ctrl->k_full[s], 1);
      mbar_init(&ctrl->v_full[s], 1);
      mbar_init(&ctrl->k_empty[s], C::RELEASERS);
      mbar_init(&ctrl->v_empty[s], C::RELEASERS);
      for (int t = 0; t < QT; ++t) {
        mbar_init(&ctrl->aux_full[t][s], 1);
        mbar_init(&ctrl->aux_empty[t][s], C::KSPLIT ? 256 : 128);
      }
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(&ctrl->s_full[t], 1);
      mbar_init(&ctrl->p_full[t], 128);
      mbar_init(&ctrl->o_final[t], 1);
      mbar_init(&ctrl->o_free[t], C::KSPLIT ? 256 : 128);
      mbar_init(&ctrl->drain[t], 1);
      mbar_init(&ctrl->s_free[t], C::KSPLIT ? 256 : 128);
      mbar_init(&ctrl->pv_done[t], 1);
    }
    if (C::KSPLIT) {
      for (int t = 0; t < 2; ++t) {  // per key half: P hand-over, PV completion, final O
        mbar_init(&ctrl->p_full[t], 128);
        mbar_init(&ctrl->pv_done[t], 1);
        mbar_init(&ctrl->o_final[t], 1);
        mbar_init(&ctrl->drain[t], 1);
      }
      for (int q = 0; q < 4; ++q) mbar_init(&ctrl->pair[q], 64);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&ctrl->item_full[q], 1);
      mbar_init(&ctrl->item_empty[q], C::ITEM_READERS);
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
  // The set-up above touches no global memory; what the previous kernel in
  // the stream writes (the prepared factors, the work counter) is read only
  // after it has completed.
  griddep_wait();

  // Barrier phases run on per-role counters that continue across work items:
  // g counts key steps (K/V ring), it counts items (Q, O), L_t counts the
  // key steps query tile t has processed (S, P, softmax-side ring).
  if (warp >= C::PRODUCER_WARP) {
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
      if (C::FAC_MMA) {
        tma_prefetch_map(&tm_fq);
        tma_prefetch_map(&tm_fk);
      }
      if (MODE == kBiasDense) tma_prefetch_map(&tm_bias);
    }
    bool ok = true;
    int g = 0, it = 0, la[2] = {0, 0};
    // The item of pass 0 is claimed and published before the loop; each pass
    // p claims and publishes the item of pass p + 1 once its own loads are
    // issued, the last published item being -1.
    int cur = __shfl_sync(0xffffffffu, leader ? claim_item(0, n_items, args.sched) : 0, 0);
    if (leader) {
      ctrl->item[0] = cur;
      mbar_arrive(&ctrl->item_full[0]);
    }
    for (int p = 0; ok && cur >= 0; ++p) {
      const WorkItem w = make_item<QT, (DP == 128)>(cur, args);
      // Q and phi_q of the item, once the previous item's last S MMAs are done.
      if (it > 0 && !(ok = mbar_wait(&ctrl->q_empty, uint32_t(it - 1) & 1u, abort))) break;
      uint32_t qbytes = 0;
      for (int t = 0; t < QT; ++t)
        if (w.nk[t] > 0) qbytes += C::Q_TILE + C::FQ_TILE;
      mbar_arrive_expect_tx_leader(&ctrl->q_full, qbytes, leader);
      for (int t = 0; t < QT; ++t) {
        if (w.nk[t] == 0) continue;
        for (int ch = 0; ch < C::NDCH; ++ch)
          tma_load_3d_leader(sQ + t * C::Q_TILE + ch * (128 * C::DCH * 2), &tm_q, &ctrl->q_full, ch * C::DCH,
                             w.q0[t], w.bh, leader);
        if (C::FAC_MMA)
          for (int ch = 0; ch < C::NRCH; ++ch)
            tma_load_3d_leader(sFQ + t * C::FQ_TILE + ch * (128 * C::RCH * 2), &tm_fq, &ctrl->q_full,
                               ch * C::RCH, w.q0[t], w.fb_slice, leader);
      }
      const int hb = args.bias_H > 1 ? w.h : 0;
      const int bb = args.bias_B > 1 ? w.b : 0;
      for (int i = 0; i < w.n_steps && ok; ++i, ++g) {
        const int s = g % KS;
        const uint32_t ph = uint32_t(g / KS) & 1u;
        const int kv = (w.n_steps - 1 - i) * 128;  // first key of this step's tile
        // stage s last held step g - KS: wait until every issuer released it
        if (g >= KS && !(ok = mbar_wait(&ctrl->k_empty[s], ph ^ 1u, abort))) break;
        mbar_arrive_expect_tx_leader(&ctrl->k_full[s], C::KV_TILE + C::FK_TILE, leader);
        for (int ch = 0; ch < C::NDCH; ++ch)
          tma_load_3d_leader(sK + s * C::KV_TILE + ch * (128 * C::DCH * 2), &tm_k, &ctrl->k_full[s], ch * C::DCH,
                             kv, w.bh, leader);
        if (C::FAC_MMA)
          for (int ch = 0; ch < C::NRCH; ++ch)
            tma_load_3d_leader(sFK + s * C::FK_TILE + ch * (128 * C::RCH * 2), &tm_fk, &ctrl->k_full[s],
                               ch * C::RCH, kv, w.fb_slice, leader);
        if (C::HAS_AUX) {
          for (int t = 0; t < QT; ++t) {
            if (i < w.first[t]) continue;
            const int ja = la[t]++;  // this tile's running step: its own ring
            const int sa = ja % KS;
            if (ja >= KS && !(ok = mbar_wait(&ctrl->aux_empty[t][sa], (uint32_t(ja / KS) & 1u) ^ 1u, abort))) break;
            uint8_t *dst = sAux + (t * KS + sa) * C::AUX_TILE;
            mbar_arrive_expect_tx_leader(&ctrl->aux_full[t][sa], C::AUX_TILE, leader);
            tma_load_4d_leader(dst, &tm_bias, &ctrl->aux_full[t][sa], kv, w.q0[t], hb, bb, leader);
            tma_load_4d_leader(dst + 128 * 128, &tm_bias, &ctrl->aux_full[t][sa], kv + 64, w.q0[t], hb, bb, leader);
          }
          if (!ok) break;
        }
        if (g >= KS && !(ok = mbar_wait(&ctrl->v_empty[s], ph ^ 1u, abort))) break;
        mbar_arrive_expect_tx_leader(&ctrl->v_full[s], C::KV_TILE, leader);
        for (int ch = 0; ch < C::NDCH; ++ch)
          tma_load_3d_leader(sV + s * C::KV_TILE + ch * (128 * C::DCH * 2), &tm_v, &ctrl->v_full[s], ch * C::DCH,
                             kv, w.bh, leader);
      }
      if (!ok) break;
      // All of this item's loads are issued: claim and publish the item of
      // pass p + 1 now, close to when the CTA will get to it. Slot (p + 1) % 4
      // last held pass p - 3, which every reader has freed by now (the
      // issuers are past the last S of pass p - 1).
      const int q1 = p + 1;
      if (q1 >= 4 && !(ok = mbar_wait(&ctrl->item_empty[q1 & 3], uint32_t((q1 >> 2) - 1) & 1u, abort))) break;
      const int nxt = __shfl_sync(0xffffffffu, leader ? claim_item(q1, n_items, args.sched) : 0, 0);
      if (leader) {
        ctrl->item[q1 & 3] = nxt;
        mbar_arrive(&ctrl->item_full[q1 & 3]);
        // its Q and phi_q tiles go to L2 now, so their load at the item
        // change waits for L2, not HBM
        if (nxt >= 0) {
          const WorkItem w2 = make_item<QT, (DP == 128)>(nxt, args);
          for (int t = 0; t < QT; ++t) {
            if (w2.nk[t] == 0) continue;
            for (int ch = 0; ch < C::NDCH; ++ch) tma_prefetch_l2_3d(&tm_q, ch * C::DCH, w2.q0[t], w2.bh);
            if (C::FAC_MMA)
              for (int ch = 0; ch < C::NRCH; ++ch) tma_prefetch_l2_3d(&tm_fq, ch * C::RCH, w2.q0[t], w2.fb_slice);
          }
        }
      }
      ++it;
      cur = nxt;
    }
    if (leader) release_sched(args.sched);  // this CTA claims nothing more
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
  } else if (warp == C::MMA_WARP || (C::SEP_P && C::NSWG == 2 && warp == C::MMA_WARP + 1)) {
    // ---------------------------------------------------------- MMA issuer
    // Descriptors of every tile base, computed once; each MMA adds a
    // compile-time step offset (the start address is the low field, and
    // shared addresses >> 4 stay below 2^14, so plain adds cannot carry).
    const uint32_t tm_u = __shfl_sync(0xffffffffu, tmem, 0);
    const uint64_t dk0 = desc_kmajor_base<C::DCH>(smem_u32(sK));
    const uint64_t dfk0 = desc_kmajor_base<C::RCH>(smem_u32(sFK));
    const uint64_t dv0 = desc_v_base<C::DCH>(smem_u32(sV));
    // The descriptors are made opaque at each call, so that the compiler
    // does not keep every per-step descriptor of the loop-invariant tiles
    // live in registers across the issue loop (this warpgroup runs on few).
    auto issue_s = [&](int t, int s) {  // S_t = Q_t K_s^T (+ phi_q' phi_k^T)
      const uint32_t d_tm = tm_u + C::S_COL0 + uint32_t(128 * t);
      uint64_t dq = desc_kmajor_base<C::DCH>(smem_u32(sQ + t * C::Q_TILE));
      uint64_t dk = dk0 + uint64_t((uint32_t(s) * C::KV_TILE) >> 4);
      asm volatile("" : "+l"(dq), "+l"(dk));
#pragma unroll
      for (int kk = 0; kk < DP / 16; ++kk)
        mma_ss_elect(d_tm, dq + kmajor_step<C::DCH>(kk), dk + kmajor_step<C::DCH>(kk), C::IDESC_QK,
                     kk > 0 ? 1u : 0u);
      if (C::FAC_MMA) {
        uint64_t dfq = desc_kmajor_base<C::RCH>(smem_u32(sFQ + t * C::FQ_TILE));
        uint64_t dfk = dfk0 + uint64_t((uint32_t(s) * C::FK_TILE) >> 4);
        asm volatile("" : "+l"(dfq), "+l"(dfk));
#pragma unroll
        // one MMA step covers 32 bytes of a row: 16 fp16 or 8 tf32 factor columns
        for (int kk = 0; kk < (C::FAC_MMA ? C::RCH * C::NRCH / 16 : 0); ++kk) {
          if (MODE == kBiasTf32)
            mma_ss_elect_tf32(d_tm, dfq + kmajor_step<C::RCH>(kk), dfk + kmajor_step<C::RCH>(kk), C::IDESC_F, 1u);
          else
            mma_ss_elect(d_tm, dfq + kmajor_step<C::RCH>(kk), dfk + kmajor_step<C::RCH>(kk), C::IDESC_F, 1u);
        }
      }
    };
    auto issue_pv = [&](int t, int s, bool acc) {  // O_t += P_t V_s, P_t read from TMEM
      const uint32_t d_tm = tm_u + C::O_COL0 + C::O_STRIDE * uint32_t(t);
      const uint32_t p_tm = tm_u + C::P_COL0 + C::P_STRIDE * uint32_t(t);
      uint64_t dv = dv0 + uint64_t((uint32_t(s) * C::KV_TILE) >> 4);
      asm volatile("" : "+l"(dv));
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_elect(d_tm, p_tm + uint32_t(kk * 8), dv + v_step<C::DCH>(kk), C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
    };
    // Key split: O_h += P[:, keys of half h] V_s[keys of half h] (MMA K-steps
    // 4h .. 4h+3 of the 128 keys).
    auto issue_pv_half = [&](int hh, int s, bool acc) {
      const uint32_t d_tm = tm_u + C::O_COL0 + C::O_STRIDE * uint32_t(hh);
      const uint32_t p_tm = tm_u + C::P_COL0;
      uint64_t dv = dv0 + uint64_t((uint32_t(s) * C::KV_TILE) >> 4);
      asm volatile("" : "+l"(dv));
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = 4 * hh + q;
        mma_ts_elect(d_tm, p_tm + uint32_t(kk * 8), dv + v_step<C::DCH>(kk), C::IDESC_PV, (acc || q > 0) ? 1u : 0u);
      }
    };
    bool ok = true;
    int g = 0, it = 0;
    if constexpr (C::KSPLIT) {
      // Issuer hh runs the PV MMAs of key half hh into O_hh; issuer 0 also
      // issues every S, S(i+1) as soon as both halves have read S(i). Each
      // issuer releases every K/V stage once per key step, and Q once per item.
      const int hh = warp - C::MMA_WARP;
      int L = 0;
      for (int p = 0; ok; ++p) {
        const int k = read_item(ctrl->item_full, ctrl->item_empty, ctrl->item, p, abort, ok);
        if (k < 0) break;
        const WorkItem w = make_item<QT, (DP == 128)>(k, args);
        const int n = w.n_steps;
        if (hh == 0) {
          if (!(ok = mbar_wait(&ctrl->q_full, uint32_t(it) & 1u, abort))) break;
          tc_fence_after();
        }
        for (int i = 0; i < n && ok; ++i) {
          const int gi = g + i;
          const int s = gi % KS;
          const uint32_t ph = uint32_t(gi / KS) & 1u;
          if (hh == 0) {
            if (i == 0) {
              if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
              // S overwrites the columns both halves read at their last step
              if (L > 0 && !(ok = mbar_wait(&ctrl->s_free[0], uint32_t(L - 1) & 1u, abort))) break;
              tc_fence_after();
              issue_s(0, s);
              tc_commit_elect(&ctrl->s_full[0]);
              tc_commit_elect(&ctrl->k_empty[s]);
            }
            if (i + 1 < n) {
              const int s1 = (gi + 1) % KS;
              if (!(ok = mbar_wait(&ctrl->k_full[s1], uint32_t((gi + 1) / KS) & 1u, abort))) break;
              if (!(ok = mbar_wait(&ctrl->s_free[0], uint32_t(L) & 1u, abort))) break;
              tc_fence_after();
              issue_s(0, s1);
              tc_commit_elect(&ctrl->s_full[0]);
              tc_commit_elect(&ctrl->k_empty[s1]);
            } else {
              tc_commit_elect(&ctrl->q_empty);  // last S of this item issued
            }
          } else {
            if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
            tc_commit_elect(&ctrl->k_empty[s]);  // only issuer 0's MMAs read K
          }
          if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
          if (!(ok = mbar_wait(&ctrl->p_full[hh], uint32_t(L) & 1u, abort))) break;
          // the first PV of an item overwrites O_hh: the epilogue must have read it
          if (i == 0 && it > 0 && !(ok = mbar_wait(&ctrl->o_free[0], uint32_t(it - 1) & 1u, abort))) break;
          tc_fence_after();
          issue_pv_half(hh, s, i > 0);
          tc_commit_elect(&ctrl->pv_done[hh]);
          tc_commit_elect(&ctrl->v_empty[s]);
          ++L;
        }
        if (!ok) break;
        tc_commit_elect(&ctrl->o_final[hh]);
        if (hh == 1) tc_commit_elect(&ctrl->q_empty);
        g += n;
        ++it;
      }
      if (!ok) {
        tc_commit_elect(&ctrl->drain[hh]);
        mbar_wait_for(&ctrl->drain[hh], 0, 100000000ull);
        if (leader) atomicOr(args.flags, kFlagTimeout);
      }
    } else if constexpr (C::SEP_P) {
      // One issuer warp per query tile t: S_t(i+1) as soon as the softmax has
      // read S_t(i) into registers, PV_t(i) once P_t(i) is written. The two
      // tiles' chains are independent and share the tensor core. Every issuer
      // walks all key steps and releases each K/V stage and the Q tiles once
      // per step or item, also where its query tile does no work.
      const int t = warp - C::MMA_WARP;
      int L = 0;
      for (int p = 0; ok; ++p) {
        const int k = read_item(ctrl->item_full, ctrl->item_empty, ctrl->item, p, abort, ok);
        if (k < 0) break;
        const WorkItem w = make_item<QT, (DP == 128)>(k, args);
        const int nk_t = pick(w.nk, t), first_t = pick(w.first, t);
        if (!(ok = mbar_wait(&ctrl->q_full, uint32_t(it) & 1u, abort))) break;
        tc_fence_after();
        if (nk_t == 0) tc_commit_elect(&ctrl->q_empty);  // this tile reads no Q in this item
        for (int i = 0; i < w.n_steps && ok; ++i) {
          const int gi = g + i;
          const int s = gi % KS;
          const uint32_t ph = uint32_t(gi / KS) & 1u;
          const int j = i - first_t;
          if (j < 0) {
            if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
            tc_commit_elect(&ctrl->k_empty[s]);
            if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
            tc_commit_elect(&ctrl->v_empty[s]);
            continue;
          }
          if (j == 0) {
            if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
            // S_t overwrites the columns the softmax read at its last step
            if (L > 0 && !(ok = mbar_wait(&ctrl->s_free[t], uint32_t(L - 1) & 1u, abort))) break;
            tc_fence_after();
            issue_s(t, s);
            tc_commit_elect(&ctrl->s_full[t]);
            tc_commit_elect(&ctrl->k_empty[s]);
          }
          if (i + 1 < w.n_steps) {
            const int s1 = (gi + 1) % KS;
            if (!(ok = mbar_wait(&ctrl->k_full[s1], uint32_t((gi + 1) / KS) & 1u, abort))) break;
            if (!(ok = mbar_wait(&ctrl->s_free[t], uint32_t(L) & 1u, abort))) break;
            tc_fence_after();
            issue_s(t, s1);
            tc_commit_elect(&ctrl->s_full[t]);
            tc_commit_elect(&ctrl->k_empty[s1]);
          }
          if (i + 1 == w.n_steps && nk_t > 0) tc_commit_elect(&ctrl->q_empty);  // last S of this item issued
          if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
          if (!(ok = mbar_wait(&ctrl->p_full[t], uint32_t(L) & 1u, abort))) break;
          // the first PV of an item overwrites O_t: its epilogue must have read it
          if (j == 0 && it > 0 && !(ok = mbar_wait(&ctrl->o_free[t], uint32_t(it - 1) & 1u, abort))) break;
          tc_fence_after();
          issue_pv(t, s, j > 0);
          tc_commit_elect(&ctrl->pv_done[t]);
          tc_commit_elect(&ctrl->v_empty[s]);
          ++L;
        }
        if (!ok) break;
        tc_commit_elect(&ctrl->o_final[t]);
        g += w.n_steps;
        ++it;
      }
      if (!ok) {
        tc_commit_elect(&ctrl->drain[t]);
        mbar_wait_for(&ctrl->drain[t], 0, 100000000ull);
        if (leader) atomicOr(args.flags, kFlagTimeout);
      }
    } else {
      // One issuer for both tiles, in the order S_0(i), PV_1(i-1), S_1(i),
      // PV_0(i) (P overwrites S, so S_t(i+1) must follow PV_t(i); tcgen05 MMAs
      // of one thread run in order).
      int L[2] = {0, 0};
      for (int p = 0; ok; ++p) {
        const int k = read_item(ctrl->item_full, ctrl->item_empty, ctrl->item, p, abort, ok);
        if (k < 0) break;
        const WorkItem w = make_item<QT, (DP == 128)>(k, args);
        auto act = [&](int t, int i) { return t < QT && i >= w.first[t] && i < w.n_steps; };
        if (!(ok = mbar_wait(&ctrl->q_full, uint32_t(it) & 1u, abort))) break;
        tc_fence_after();
        for (int i = 0; i < w.n_steps && ok; ++i) {
          const int gi = g + i;
          const int s = gi % KS;
          const uint32_t ph = uint32_t(gi / KS) & 1u;
          if (!(ok = mbar_wait(&ctrl->k_full[s], ph, abort))) break;
          tc_fence_after();
          if (act(0, i)) {
            issue_s(0, s);
            tc_commit_elect(&ctrl->s_full[0]);
          }
          if (QT == 2) {
            const int ip = i - 1;  // PV of tile 1 for the previous step
            if (act(1, ip)) {
              const int sp = (gi - 1) % KS;
              const uint32_t php = uint32_t((gi - 1) / KS) & 1u;
              if (!act(0, ip) && !(ok = mbar_wait(&ctrl->v_full[sp], php, abort))) break;
              if (!(ok = mbar_wait(&ctrl->p_full[1], uint32_t(L[1]) & 1u, abort))) break;
              if (ip == w.first[1] && it > 0 && !(ok = mbar_wait(&ctrl->o_free[1], uint32_t(it - 1) & 1u, abort)))
                break;
              tc_fence_after();
              issue_pv(1, sp, ip > w.first[1]);
              tc_commit_elect(&ctrl->v_empty[sp]);
              ++L[1];
            }
            if (act(1, i)) {
              issue_s(1, s);
              tc_commit_elect(&ctrl->s_full[1]);
            }
          }
          tc_commit_elect(&ctrl->k_empty[s]);
          if (i + 1 == w.n_steps) tc_commit_elect(&ctrl->q_empty);  // last S of this item issued
          if (act(0, i)) {
            if (!(ok = mbar_wait(&ctrl->v_full[s], ph, abort))) break;
            if (!(ok = mbar_wait(&ctrl->p_full[0], uint32_t(L[0]) & 1u, abort))) break;
            if (i == w.first[0] && it > 0 && !(ok = mbar_wait(&ctrl->o_free[0], uint32_t(it - 1) & 1u, abort)))
              break;
            tc_fence_after();
            issue_pv(0, s, i > w.first[0]);
            ++L[0];
            if (!act(1, i)) tc_commit_elect(&ctrl->v_empty[s]);
          } else if (!act(1, i)) {
            tc_commit_elect(&ctrl->v_empty[s]);  // no tile used this step's V
          }
        }
        if (ok && act(1, w.n_steps - 1)) {
          const int ip = w.n_steps - 1;
          const int gp = g + ip;
          const int sp = gp % KS;
          const uint32_t php = uint32_t(gp / KS) & 1u;
          ok = act(0, ip) || mbar_wait(&ctrl->v_full[sp], php, abort);
          ok = ok && mbar_wait(&ctrl->p_full[1], uint32_t(L[1]) & 1u, abort);
          ok = ok && (ip != w.first[1] || it == 0 || mbar_wait(&ctrl->o_free[1], uint32_t(it - 1) & 1u, abort));
          if (ok) {
            tc_fence_after();
            issue_pv(1, sp, ip > w.first[1]);
            tc_commit_elect(&ctrl->v_empty[sp]);
            ++L[1];
          }
        }
        if (!ok) break;
        for (int t = 0; t < QT; ++t) tc_commit_elect(&ctrl->o_final[t]);
        g += w.n_steps;
        ++it;
      }
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
    if constexpr (C::KSPLIT) {
      // Key split: warpgroup h takes keys 64h .. 64h+63 of every key tile of
      // the item, with its own running max m_h, row sum l_h and O_h; the two
      // are merged in the epilogue (O = sum_h 2^(m_h - M) O_h / sum_h 2^(m_h - M) l_h).
      const int h = warp >> 2;
      const int wq = warp & 3;  // TMEM lane quarter
      const int r_loc = wq * 32 + lane;
      const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
      const uint32_t s_tm = lane_base + C::S_COL0 + uint32_t(64 * h);
      const uint32_t p_tm = lane_base + C::P_COL0 + uint32_t(32 * h);
      const uint32_t o0_tm = lane_base + C::O_COL0;
      const uint32_t o1_tm = lane_base + C::O_COL0 + C::O_STRIDE;
      const uint32_t own_tm = h ? o1_tm : o0_tm;
      const float sl2 = args.scale_log2;
      float *xch = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(ctrl) + 1024);
      auto xslot = [&](int half, int slot, int v) { return xch + (((wq * 2 + half) * 2 + slot) * 2 + v) * 32 + lane; };
      int n_ex = 0;
      bool ok = true;
      int L = 0, it = 0;
      for (int p = 0; ok; ++p) {
        const int k = read_item(ctrl->item_full, ctrl->item_empty, ctrl->item, p, abort, ok);
        if (k < 0) break;
        const WorkItem w = make_item<QT, (DP == 128)>(k, args);
        const int q0 = w.q0[0], n = w.n_steps;
        const int row = q0 + r_loc;
        float m_use = -INFINITY, l_sum = 0.f;
        for (int i = 0; i < n; ++i) {  // key tile n - 1 - i
          const int s = L % KS;
          const uint32_t ph = uint32_t(L / KS) & 1u;
          if (C::HAS_AUX && !(ok = mbar_wait(&ctrl->aux_full[0][s], ph, abort))) break;
          if (!(ok = mbar_wait(&ctrl->s_full[0], uint32_t(L) & 1u, abort))) break;
          tc_fence_after();
          uint32_t x[64];
          tmem_ld32(s_tm, x);
          tmem_ld32(s_tm + 32, x + 32);
          tmem_ld_wait32(x);
          tmem_ld_wait32(x + 32);
          tc_fence_before();
          mbar_arrive(&ctrl->s_free[0]);  // S is in registers: the tensor core may overwrite it
          float mul = sl2;  // log2-domain logit = x * mul
          if (MODE == kBiasDense) {
            add_dense_bias(x, sAux + s * C::AUX_TILE + h * 16384, r_loc, args.scale);
            mbar_arrive(&ctrl->aux_empty[0][s]);
            mul = kLog2e;
          }
          // Causal diagonal tile and the ragged last key tile.
          const int key0 = (n - 1 - i) * 128 + 64 * h;  // first key of this half
          if ((args.causal && key0 + 63 > q0) || key0 + 64 > N) {
            const int lim = args.causal ? min(row + 1, N) : N;  // keys [0, lim) are visible
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (key0 + c >= lim) x[c] = __float_as_uint(-INFINITY);
          }
          const float m_new = fmaxf(m_use, row_max<64>(x) * mul);
          float alpha = 1.f;
          bool resc = false;
          if (m_use == -INFINITY || m_new > m_use + kRescaleThreshold) {
            alpha = (m_use == -INFINITY) ? 0.f : ex2_approx(m_use - m_new);
            resc = (i > 0) && (m_use != -INFINITY);
            m_use = m_new;
          }
          l_sum *= alpha;
          const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
          const uint64_t mul2 = f2_pack(mul, mul), negm2 = f2_pack(neg_m, neg_m);
          uint64_t ls[4] = {0, 0, 0, 0};
          uint32_t pk[32];
#pragma unroll
          for (int q4 = 0; q4 < 2; ++q4) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t a =
                  f2_fma(f2_pack(__uint_as_float(x[q4 * 32 + 2 * e]), __uint_as_float(x[q4 * 32 + 2 * e + 1])),
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
              pk[q4 * 16 + e] = pack_bf16x2(p0, p1);
            }
          }
          {
            float s0, s1, s2, s3, s4, s5, s6, s7;
            f2_unpack(ls[0], s0, s1);
            f2_unpack(ls[1], s2, s3);
            f2_unpack(ls[2], s4, s5);
            f2_unpack(ls[3], s6, s7);
            l_sum += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
          }
          if (L > 0) {  // P_h and O_h are still read by the previous PV_h
            if (!(ok = mbar_wait(&ctrl->pv_done[h], uint32_t(L - 1) & 1u, abort))) break;
            tc_fence_after();
          }
          if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
            for (int c0 = 0; c0 < DP; c0 += 16) {
              uint32_t r[16];
              tmem_ld16(own_tm + c0, r);
              tmem_ld_wait16(r);
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st16(own_tm + c0, r);
            }
          }
          tmem_st32(p_tm, pk);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&ctrl->p_full[h]);
          ++L;
        }
        if (!ok) break;

        // ---------------------------------------------------- epilogue (merge)
        if (!(ok = mbar_wait(&ctrl->o_final[0], uint32_t(it) & 1u, abort))) break;
        if (!(ok = mbar_wait(&ctrl->o_final[1], uint32_t(it) & 1u, abort))) break;
        tc_fence_after();
        const int slot = n_ex & 1;
        *xslot(h, slot, 0) = m_use;
        *xslot(h, slot, 1) = l_sum;
        mbar_arrive(&ctrl->pair[wq]);
        if (!(ok = mbar_wait(&ctrl->pair[wq], uint32_t(n_ex) & 1u, abort))) break;
        const float m_o = *xslot(h ^ 1, slot, 0), l_o = *xslot(h ^ 1, slot, 1);
        ++n_ex;
        const float m0 = h ? m_o : m_use, l0 = h ? l_o : l_sum;
        const float m1 = h ? m_use : m_o, l1 = h ? l_sum : l_o;
        const float M = fmaxf(m0, m1);
        const float w0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M);
        const float w1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - M);
        const float l_tot = w0 * l0 + w1 * l1;
        const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
        const float c0s = w0 * inv_l, c1s = w1 * inv_l;
        if constexpr (C::TMA_EPI) {
          // this half stores O columns 64h .. 64h+63 of the warp's rows in two
          // staged chunks; both O accumulators are handed back after the last read
          const bool rows_live = q0 + 32 * wq < N;  // warp-uniform
          uint8_t *slot = stg_slot(warp);
#pragma unroll
          for (int cc = 0; cc < 64; cc += 32) {
            const int col0 = 64 * h + cc;
            uint32_t r0[32], r1[32];
            tmem_ld32(o0_tm + col0, r0);
            tmem_ld32(o1_tm + col0, r1);
            tmem_ld_wait32(r0);
            tmem_ld_wait32(r1);
            if (cc == 32) {
              tc_fence_before();
              mbar_arrive(&ctrl->o_free[0]);  // both O accumulators have been read
            }
            if (rows_live && col0 < args.d) {  // chunks past the head dim hold padding only
              uint32_t pkd[16];
#pragma unroll
              for (int e = 0; e < 16; ++e)
                pkd[e] = pack_bf16x2(fmaf(__uint_as_float(r0[2 * e]), c0s, __uint_as_float(r1[2 * e]) * c1s),
                                     fmaf(__uint_as_float(r0[2 * e + 1]), c0s, __uint_as_float(r1[2 * e + 1]) * c1s));
              stage_and_store_o<32>(slot, pkd, lane, &tm_o, col0, q0 + 32 * wq, w.bh);
            }
          }
          if (h == 0 && row < N)
            args.LSE[size_t(w.bh) * N + row] = l_tot > 0.f ? (M + __log2f(l_tot)) * kLn2 : -INFINITY;
          ++it;
          continue;
        }
        __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(args.O) + (size_t(w.bh) * N + row) * args.d;
#pragma unroll
        for (int cc = 0; cc < 64; cc += 16) {  // this half writes O columns 64h .. 64h+63
          const int col0 = 64 * h + cc;
          uint32_t r0[16], r1[16];
          tmem_ld16(o0_tm + col0, r0);
          tmem_ld16(o1_tm + col0, r1);
          tmem_ld_wait16(r0);
          tmem_ld_wait16(r1);
          if (row < N) {
#pragma unroll
            for (int v8 = 0; v8 < 2; ++v8) {
              const int col = col0 + v8 * 8;
              if (col < args.d) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  o[e] = fmaf(__uint_as_float(r0[v8 * 8 + e]), c0s, __uint_as_float(r1[v8 * 8 + e]) * c1s);
                uint4 u;
                u.x = pack_bf16x2(o[0], o[1]);
                u.y = pack_bf16x2(o[2], o[3]);
                u.z = pack_bf16x2(o[4], o[5]);
                u.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4 *>(orow + col) = u;
              }
            }
          }
        }
        if (h == 0 && row < N)
          args.LSE[size_t(w.bh) * N + row] = l_tot > 0.f ? (M + __log2f(l_tot)) * kLn2 : -INFINITY;
        tc_fence_before();
        mbar_arrive(&ctrl->o_free[0]);  // both O accumulators have been read
        ++it;
      }
      if (!ok) atomicOr(args.flags, kFlagTimeout);
    } else {
      // ------------------------------------------------------------- softmax
      const int t = warp >> 2;  // query tile of this warpgroup
      const int wq = warp & 3;  // TMEM lane quarter
      const int r_loc = wq * 32 + lane;
      const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
      const uint32_t s_tm = lane_base + C::S_COL0 + uint32_t(128 * t);
      const uint32_t p_tm = lane_base + C::P_COL0 + C::P_STRIDE * uint32_t(t);
      const uint32_t o_tm = lane_base + C::O_COL0 + C::O_STRIDE * uint32_t(t);
      const float sl2 = args.scale_log2;
      bool ok = true;
      int L = 0, it = 0;
      for (int p = 0; ok; ++p) {
        const int k = read_item(ctrl->item_full, ctrl->item_empty, ctrl->item, p, abort, ok);
        if (k < 0) break;
        const WorkItem w = make_item<QT, (DP == 128)>(k, args);
        const int q0_t = pick(w.q0, t), nk_t = pick(w.nk, t), first_t = pick(w.first, t);
        const int row = q0_t + r_loc;
        float m_use = -INFINITY, l_sum = 0.f;
        for (int i = first_t; i < w.n_steps; ++i) {  // key tile n_steps - 1 - i
          const int s = L % KS;  // the softmax-side ring runs on L
          const uint32_t ph = uint32_t(L / KS) & 1u;
          if (C::HAS_AUX && !(ok = mbar_wait(&ctrl->aux_full[t][s], ph, abort))) break;
          if (!(ok = mbar_wait(&ctrl->s_full[t], uint32_t(L) & 1u, abort))) break;
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
          if (C::SEP_P) {  // S_t is in registers: the tensor core may overwrite it
            tc_fence_before();
            mbar_arrive(&ctrl->s_free[t]);
          }
          float mul = sl2;  // log2-domain logit = x * mul
          if (MODE == kBiasDense) {
            const uint8_t *tile = sAux + (t * KS + s) * C::AUX_TILE;
            add_dense_bias(x, tile, r_loc, args.scale);
            add_dense_bias(x + 64, tile + 16384, r_loc, args.scale);
            mbar_arrive(&ctrl->aux_empty[t][s]);
            mul = kLog2e;
          }
          // Causal diagonal tile and the ragged last key tile.
          const int key0 = (w.n_steps - 1 - i) * 128;
          if ((args.causal && key0 + 127 > q0_t) || key0 + 128 > N) {
            const int lim = args.causal ? min(row + 1, N) : N;  // keys [0, lim) are visible
  #pragma unroll
            for (int c = 0; c < 128; ++c)
              if (key0 + c >= lim) x[c] = __float_as_uint(-INFINITY);
          }
          float mx;
          {
            // eight independent chains of three-input max (one instruction per
            // two elements)
            float mp[8];
  #pragma unroll
            for (int e = 0; e < 8; ++e) mp[e] = fmax3(__uint_as_float(x[e]), __uint_as_float(x[8 + e]), __uint_as_float(x[16 + e]));
  #pragma unroll
            for (int c = 24; c < 120; c += 16)
  #pragma unroll
              for (int e = 0; e < 8; ++e) mp[e] = fmax3(mp[e], __uint_as_float(x[c + e]), __uint_as_float(x[c + 8 + e]));
  #pragma unroll
            for (int e = 0; e < 8; ++e) mp[e] = fmaxf(mp[e], __uint_as_float(x[120 + e]));
            mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
          }
          const float m_new = fmaxf(m_use, mx * mul);
          float alpha = 1.f;
          bool resc = false;
          if (m_use == -INFINITY || m_new > m_use + kRescaleThreshold) {
            alpha = (m_use == -INFINITY) ? 0.f : ex2_approx(m_use - m_new);
            resc = (i > first_t) && (m_use != -INFINITY);
            m_use = m_new;
          }
          l_sum *= alpha;
          // P of the whole row stays in registers (each 32-column group of x
          // dies as its 16 bf16 pairs are made) and goes to TMEM at the end, so
          // the wait for the previous PV_t overlaps the exponentials.
          const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;
          const uint64_t mul2 = f2_pack(mul, mul), negm2 = f2_pack(neg_m, neg_m);
          uint64_t ls[4] = {0, 0, 0, 0};  // packed partial row sums
          uint32_t pk[64];
  #pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
  #pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t a =
                  f2_fma(f2_pack(__uint_as_float(x[q4 * 32 + 2 * e]), __uint_as_float(x[q4 * 32 + 2 * e + 1])), mul2,
                         negm2);
              float a0, a1, p0, p1;
              f2_unpack(a, a0, a1);
              if (e < kEmuPairs) {
                ex2_fma_pair(a0, a1, p0, p1);
              } else {
                p0 = ex2_approx(a0);
                p1 = ex2_approx(a1);
              }
              ls[e & 3] = f2_add(ls[e & 3], f2_pack(p0, p1));
              pk[q4 * 16 + e] = pack_bf16x2(p0, p1);
            }
          }
          {
            float s0, s1, s2, s3, s4, s5, s6, s7;
            f2_unpack(ls[0], s0, s1);
            f2_unpack(ls[1], s2, s3);
            f2_unpack(ls[2], s4, s5);
            f2_unpack(ls[3], s6, s7);
            l_sum += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
          }
          if (C::SEP_P && L > 0) {
            // P_t (and O_t) are still read by the previous PV_t; wait for it.
            if (!(ok = mbar_wait(&ctrl->pv_done[t], uint32_t(L - 1) & 1u, abort))) break;
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
          tmem_st32(p_tm, pk);
          tmem_st32(p_tm + 32, pk + 32);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&ctrl->p_full[t]);
          ++L;
        }
        if (!ok) break;

        // ---------------------------------------------------------- epilogue
        if (!(ok = mbar_wait(&ctrl->o_final[t], uint32_t(it) & 1u, abort))) break;
        tc_fence_after();
        if constexpr (C::TMA_EPI) {
          // O leaves in chunks of EPI_E columns through this warp's staging
          // slot; O_t is handed back to the MMA warp as soon as its last chunk
          // is in registers, and the TMA stores complete on their own.
          if (nk_t > 0) {
            const uint32_t tid = tid_x_fresh();
            const int e_lane = int(tid & 31u), e_warp = int(tid >> 5);
            const int row0 = q0_t + 32 * (e_warp & 3);  // first row of this warp's TMEM lane quarter
            const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
            const bool rows_live = row0 < N;  // warp-uniform
            uint8_t *slot = stg_slot(e_warp);
#pragma unroll
            for (int c0 = 0; c0 < DP; c0 += C::EPI_E) {
              uint32_t r[C::EPI_E];
              if constexpr (C::EPI_E == 64) {
                tmem_ld32(o_tm + c0, r);
                tmem_ld32(o_tm + c0 + 32, r + 32);
                tmem_ld_wait32(r);
                tmem_ld_wait32(r + 32);
              } else if constexpr (C::EPI_E == 32) {
                tmem_ld32(o_tm + c0, r);
                tmem_ld_wait32(r);
              } else {
                tmem_ld16(o_tm + c0, r);
                tmem_ld_wait16(r);
              }
              if (c0 + C::EPI_E == DP) {
                tc_fence_before();
                mbar_arrive(&ctrl->o_free[t]);  // O_t has been read
              }
              if (rows_live && c0 < args.d) {  // chunks past the head dim hold padding only
                uint32_t pkd[C::EPI_E / 2];
#pragma unroll
                for (int e = 0; e < C::EPI_E / 2; ++e)
                  pkd[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
                stage_and_store_o<C::EPI_E>(slot, pkd, e_lane, &tm_o, c0, row0, w.bh);
              }
            }
            if (row0 + e_lane < N)
              args.LSE[size_t(w.bh) * N + row0 + e_lane] = l_sum > 0.f ? (m_use + __log2f(l_sum)) * kLn2 : -INFINITY;
          } else {
            tc_fence_before();
            mbar_arrive(&ctrl->o_free[t]);
          }
          ++it;
          continue;
        }
        if (nk_t > 0) {
          const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
          __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(args.O) + (size_t(w.bh) * N + row) * args.d;
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
            args.LSE[size_t(w.bh) * N + row] = l_sum > 0.f ? (m_use + __log2f(l_sum)) * kLn2 : -INFINITY;
        }
        tc_fence_before();
        mbar_arrive(&ctrl->o_free[t]);  // O_t has been read
        ++it;
      }
      if (!ok) atomicOr(args.flags, kFlagTimeout);
    }
  }

  if constexpr (C::TMA_EPI) {
    // the staging slots must outlive the stores that read them
    if (warp < C::PRODUCER_WARP && lane == 0) bulk_wait_group0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Per device: the resident CTA capacity of one kernel instantiation (SMs x
// CTAs per SM), found once together with the attribute checks and settings.
constexpr int kMaxDevices = 64;

template <int DP, int RP, int MODE, int QT>
static cudaError_t launch_one(const FwdMaps &m, const FwdArgs &a, cudaStream_t stream) {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  if constexpr (C::KS < 1) {
    return cudaErrorInvalidConfiguration;
  } else {
    auto kern = attn_fwd_sm100<DP, RP, MODE, QT>;
    static std::atomic<int> capacity[kMaxDevices];  // 0: not set up on that device yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int cap = capacity[dev].load(std::memory_order_acquire);
    if (cap == 0) {
      // setmaxnreg.inc waits until the block's pool has the registers, so the
      // launch allocation must be exactly what the split assumes.
      cudaFuncAttributes fa;
      if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
      if (fa.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
      if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM))) != cudaSuccess)
        return e;
      // All of the SM's unified L1/shared storage as shared memory, so that
      // MIN_BLOCKS CTAs fit side by side.
      if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    int(cudaSharedmemCarveoutMaxShared))) != cudaSuccess)
        return e;
      // CTAs per SM from the per-SM limits: shared memory, registers,
      // threads and the 512 TMEM columns (which no occupancy query knows of).
      int sms = 0, smem_sm = 0, smem_res = 0, regs_sm = 0, thr_sm = 0;
      if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess)
        return e;
      int per_sm = int(512 / C::TMEM_COLS);
      per_sm = std::min(per_sm, smem_sm / (int(C::SMEM) + smem_res));
      per_sm = std::min(per_sm, regs_sm / (C::THREADS * C::LAUNCH_REGS));
      per_sm = std::min(per_sm, thr_sm / C::THREADS);
      if (per_sm < 1 || sms < 1) return cudaErrorInvalidConfiguration;
      cap = sms * per_sm;
      capacity[dev].store(cap, std::memory_order_release);
    }
    // Persistent grid: at most as many CTAs as are resident at once, each
    // walking its share of the work items.
    const long long items = (long long)a.n_cta_q * a.B * a.H;
    const long long ctas = std::min<long long>(items, cap);
    // Programmatic stream serialization: the CTAs may start their set-up
    // while the preparation kernel before them finishes (they wait for it
    // before reading anything it writes).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(ctas));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, m.q, m.k, m.v, m.fq, m.fk, m.bias, m.o, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
}

template <int DP, int RP, int MODE, int QT>
static constexpr size_t smem_of() {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  return C::KS >= 1 ? size_t(C::SMEM) : 0;
}

template <int DP, int RP, int MODE, int QT>
static constexpr int epi_cols_of() {
  using C = Sm100Cfg<DP, RP, MODE, QT>;
  return C::EPI_E;
}

#define FB_DISPATCH_QT(DPv, RPv, MODEv)                                          \
  if (p.QT == 1) return FB_ACTION(DPv, RPv, MODEv, 1);                           \
  if (p.QT == 2) return FB_ACTION(DPv, RPv, MODEv, 2);

#define FB_DISPATCH_MODE(DPv)                                                    \
  if (p.mode == kBiasNone) { FB_DISPATCH_QT(DPv, 0, kBiasNone) }                 \
  if (p.mode == kBiasTf32) {                                                     \
    if (p.RP == 8) { FB_DISPATCH_QT(DPv, 8, kBiasTf32) }                         \
    if (p.RP == 16) { FB_DISPATCH_QT(DPv, 16, kBiasTf32) }                       \
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

int sm100_epi_cols(const FwdPlan &p) {
#define FB_ACTION(DPv, RPv, MODEv, QTv) epi_cols_of<DPv, RPv, MODEv, QTv>()
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
