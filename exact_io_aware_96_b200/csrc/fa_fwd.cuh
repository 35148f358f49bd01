// fa_fwd.cuh — fused attention forward for sm_100a, fp16/bf16 inputs (fa_fwd;
// the e4m3 forward is fa_fwd_e4m3.cuh).
//
// One CTA computes O and LSE for 256 query rows (two 128-row tiles, t = 0, 1)
// of one (batch, head), streaming 128-key K/V blocks through shared memory:
// S_t = Q_t K_j^T, the online softmax and O_t += P_t V_j happen in one kernel
// and the Sq x Sk score matrix never reaches device memory ([P1] "性能引擎":
// the three steps fused into one kernel; [P2] item 2 "分块处理": tiles in
// on-chip memory with an online softmax; [P5] "第三招": the next block is
// prefetched while the current one is computed).
//
// Softmax per row in base 2: x = s * scale * log2(e), running max m and sum
// l; the accumulator O_t stays unscaled and is divided by l once at the end,
// and only LSE = ln2 * (m + log2 l) is stored ([P4] §3.1). The running max is
// raised (and O_t, l rescaled) only when a block's max exceeds it by more than
// 8, a factor 256; otherwise the stale max is kept, which is still exact
// because l, O_t and LSE all use the same m.
//
// Per tile the work is a chain: softmax of block j, then P V(j) and S(j+1) on
// the tensor core, then the softmax of block j + 1. The two tiles alternate,
// so one tile's softmax runs while the tensor core works on the other's
// products. Two warpgroups share every row of a tile, one per 64-key half of
// each block, so a block's exponentials are spread over eight warps (two per
// SM sub-partition) and the softmax link of the chain is short.
//
// Warp roles (576 threads):
//   warps 8t + 4c + r  softmax/epilogue of tile t, key half c (keys 64c ..
//              64c + 63 of every block), TMEM lanes 32r .. 32r + 31, one query
//              row per thread (r = warp % 4 is the warp's TMEM lane quarter)
//   warp  16   TMA loader: Q tiles once, then K_j and V_j into a ring
//   warp  17   MMA issuer (the whole warp; elect.sync picks the issuing lane)
// Tensor memory (512 columns x 128 lanes of fp32):
//   D = 128 (and e4m3): [128t, 128t + 128) S_t   [256 + tD, 256 + tD + D) O_t
//   D = 64: three S buffers [0, 384) that the S products rotate over (see
//   the MMA issuer), O_t at [384 + 64t, 448 + 64t).
//   Half c of an S buffer is its columns 64c .. 64c + 63; its P (16-bit, two
//   values per column) overwrites the first 32 of them, so each warpgroup only
//   touches its own columns. P V(j) reads the two halves of P from their two
//   places.
// The two warps that own the same 32 rows of a tile (one per half) agree on
// the running max once per block: each puts its partial row max in shared
// memory and both meet at a 64-thread named barrier that also ANDs their
// "still running" flags, so an abort seen by one side ends both sides at the
// same point and neither waits for a partner that has left. Each half
// rescales its own D/2 columns of O_t and keeps its own partial sum l; the two
// sums meet the same way in the epilogue.
//
// Exponentials: 2^t on the MUFU unit (ex2.approx), except that on blocks
// with no masked entry one pair in four goes through a polynomial on the FMA
// pipe (sm100::exp2_poly2). Masked blocks use the MUFU unit for every entry,
// so masked P entries are exactly 0.
//
// Work split over batch x heads x 256-row blocks ([P4] §3.2); for causal masks
// the grid is ordered so the longest rows start first, key blocks past the
// diagonal are skipped and only diagonal and tail blocks are masked element
// by element ([P4] §4: causal skips about half the blocks).
//
// Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
// [P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P4] the FlashAttention-2
// walkthrough titled "企业官网建设流程全解析"; [P5] the FlashAttention
// "IO感知" overview (0539edu.com/news/165270).
#pragma once

#include "fa_common.cuh"

namespace fa {

// Number of 128-key blocks that rows [r0, r0 + 128) of the query range need.
__host__ __device__ inline int fwd_kv_blocks(int r0, int Sq, int Sk, int causal) {
  if (r0 >= Sq) return 0;
  const int nk = (Sk + 127) / 128;
  if (!causal) return nk;
  const int last = (r0 + 127 < Sq - 1 ? r0 + 127 : Sq - 1) + (Sk - Sq);
  if (last < 0) return 0;
  return nk < last / 128 + 1 ? nk : last / 128 + 1;
}

// ESZ: bytes per Q/K/V element (2 for fp16/bf16, 1 for e4m3).
template <int D, int ESZ = 2>
struct FwdLayout {
  static constexpr int kThreads = 576;
  static constexpr int kLoaderWarp = 16;
  static constexpr int kMmaWarp = 17;
  static constexpr int RB = D * ESZ;             // bytes of one tile row
  static constexpr int KB = RB / 128;            // 128-byte column blocks per row
  static constexpr int TILE = 128 * RB;          // bytes of one 128-row tile
  static constexpr int BLK = 128 * 128;          // one 128-row x 128-byte block
  static constexpr int STAGES = (RB == 256) ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  // Partial row maxima [block parity][tile][half][row] and partial sums
  // [tile][half][row], fp32.
  static constexpr int OFF_PMAX = OFF_V + STAGES * TILE;
  static constexpr int OFF_LSUM = OFF_PMAX + 2 * 2 * 2 * 128 * 4;
  static constexpr int OFF_BAR = OFF_LSUM + 2 * 2 * 128 * 4;
  // q_full, k_full/k_empty/v_full/v_empty[STAGES], s_full[2], p_full[2],
  // o_final[2], drain, pv_done[2]
  static constexpr int NBAR = 1 + 4 * STAGES + 2 + 2 + 2 + 1 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // room to align the base to 1024
  static constexpr int TMEM_COLS = 512;
};

// P = 2^(s * sl2 - mu) for 32 S values of one row (raw fp32 bits in sv),
// packed to 16 words of two 16-bit values; adds the P values into acc0/acc1.
// MASKED: entries past column `lim` are -inf (P = 0) and every exponential
// runs on the MUFU unit, which returns exactly 0 for them.
template <bool BF16, bool MASKED>
__device__ __forceinline__ void fwd_exp32(const uint32_t (&sv)[32], int col0, int lim, uint64_t sl2x2,
                                          uint64_t negmu2, uint64_t& acc0, uint64_t& acc1, uint32_t (&pw)[16]) {
  using namespace sm100;
#pragma unroll
  for (int cc = 0; cc < 16; ++cc) {
    float s0 = __uint_as_float(sv[2 * cc]);
    float s1 = __uint_as_float(sv[2 * cc + 1]);
    if constexpr (MASKED) {
      s0 = (col0 + 2 * cc <= lim) ? s0 : -INFINITY;
      s1 = (col0 + 2 * cc + 1 <= lim) ? s1 : -INFINITY;
    }
    const uint64_t tt = fma2(f2(s0, s1), sl2x2, negmu2);
    uint64_t e;
    if (!MASKED && (cc & 3) == 3) {
      e = exp2_poly2(tt);
    } else {
      float t0, t1;
      f2_split(tt, t0, t1);
      e = f2(ex2(t0), ex2(t1));
    }
    if (cc & 1)
      acc1 = add2(acc1, e);
    else
      acc0 = add2(acc0, e);
    float e0, e1;
    f2_split(e, e0, e1);
    pw[cc] = pack2<BF16>(e0, e1);
  }
}

// Epilogue of a CTA that covers one half of its rows' key blocks (FwdArgs::
// n_split). Every softmax warp of the CTA calls it. The CTA's partial result
// for a row, (m, l = l_0 + l_1, unnormalised O), is exact for that half of the
// keys; two halves merge exactly:
//   m = max(m_a, m_b),  l = l_a 2^(m_a - m) + l_b 2^(m_b - m),
//   O = (O_a 2^(m_a - m) + O_b 2^(m_b - m)) / l,
// the same rescaling the online softmax applies from one key block to the
// next ([P4] §3.1), here between the two halves. Each CTA writes its partial
// into its workspace slot; the 16 softmax warps meet; one thread fences and
// swaps the pair's ticket to this launch's epoch; the CTA that finds the
// epoch already there (the second to finish) fences again and reads its
// partner's partial through L2, then writes O and LSE. The barrier orders the
// other threads' partial stores before that thread's fence (fences are
// cumulative), so one fence per CTA suffices.
// Partial O layout: float4 units [CTA][tile][D / 4][128 rows], so a warp's
// stores and loads of one 4-column group cover 512 contiguous bytes.
template <int D, bool BF16>
__device__ __forceinline__ void fwd_split_epilogue(const FwdArgs& a, uint8_t* flag_smem, float* lsum, uint64_t* o_final,
                                                   volatile int* abort_flag, uint32_t tO, bool ok, int t, int c, int r,
                                                   int pair_bar, int n, float m, float l, int pair, int cta, int pcta,
                                                   int b, int h, int row, int r0) {
  using namespace sm100;
  constexpr int kSplitBar = 9;  // named barrier of the 16 softmax warps
  const bool rows = r0 < a.Sq;  // the same for both warps of a pair
  bool go = ok && !*abort_flag;
  float lt = 0.f;
  if (rows) {
    lsum[(t * 2 + c) * 128 + r] = l;
    go = named_bar_and(pair_bar, 64, go);
    lt = l + lsum[(t * 2 + (c ^ 1)) * 128 + r];
  }
  const int n_ctas = 2 * a.n_split * a.H * a.B;
  // first float4 of this thread's columns in a CTA's partial O; step 128 per 4 columns
  auto o_base = [&](int k) {
    return reinterpret_cast<float4*>(a.part_o) + (static_cast<int64_t>(k) * 2 + t) * (D / 4) * 128 +
           static_cast<int64_t>(c * (D / 8)) * 128 + r;
  };
  bool have_o = false;  // O_t holds this CTA's sums (n > 0 and its MMAs are done)
  if (go && rows && n > 0) {
    have_o = __all_sync(0xffffffffu, wait_bar(o_final, 0, abort_flag, kRoleSoftmax, n));
    go = have_o;
    if (have_o) tc_fence_after();
  }
  // (Conditions around tcgen05.ld are warp-uniform: the load is collective.)
  if (__all_sync(0xffffffffu, go && rows && checked(cta < n_ctas, 110))) {
    float4* po = o_base(cta);
#pragma unroll 1
    for (int q = 0; q < D / 64; ++q) {
      uint32_t ov[32];
      if (have_o) {
        tmem_ld32(tO + 32 * q, ov);
        tmem_ld_wait();
        reg_fence(ov);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
        po[(8 * q + i) * 128] = make_float4(__uint_as_float(ov[4 * i]), __uint_as_float(ov[4 * i + 1]),
                                            __uint_as_float(ov[4 * i + 2]), __uint_as_float(ov[4 * i + 3]));
    }
    if (c == 0) a.part_ml[static_cast<int64_t>(cta) * 256 + t * 128 + r] = make_float2(m, lt);
  }
  go = named_bar_and(kSplitBar, 512, go);
  volatile uint32_t* second_flag = reinterpret_cast<volatile uint32_t*>(flag_smem);
  if (threadIdx.x == 0) {
    uint32_t second = 0;
    if (go && checked(pair < a.n_split * a.H * a.B, 112)) {
      __threadfence();
      second = atomicExch(&a.tickets[pair], a.epoch) == a.epoch;
      if (second) __threadfence();
    }
    *second_flag = second;
  }
  named_bar_sync(kSplitBar, 512);
  if (!__all_sync(0xffffffffu, go && rows && *second_flag && checked(pcta >= 0 && pcta < n_ctas, 111))) return;
  const float2 mo = __ldcg(a.part_ml + static_cast<int64_t>(pcta) * 256 + t * 128 + r);  // the partner's (m, l)
  const float mn = fmaxf(m, mo.x);
  const float as = (m == -INFINITY) ? 0.f : ex2(m - mn);
  const float ao = (mo.x == -INFINITY) ? 0.f : ex2(mo.x - mn);
  // Products rounded separately and then added (no fused multiply-add), so
  // the result is the same whichever of the two CTAs merges.
  const float lsum_all = __fadd_rn(__fmul_rn(lt, as), __fmul_rn(mo.y, ao));
  const bool has = (mn != -INFINITY) && lsum_all > 0.f;  // false only for rows with no allowed key
  const float inv = has ? a.o_scale / lsum_all : 0.f;
  const float ws = as * inv, wo = ao * inv;
  const bool valid = row < a.Sq;
  const int cb = c * (D / 2);  // first O column of this half
  const float4* ppo = o_base(pcta);
  uint16_t* orow = reinterpret_cast<uint16_t*>(a.o) + static_cast<int64_t>(b) * a.o_sb +
                   static_cast<int64_t>(row) * a.o_ss + static_cast<int64_t>(h) * a.o_sh;
#pragma unroll 1
  for (int q = 0; q < D / 64; ++q) {
    float4 pv[8];  // the partner's 32 columns, loaded while this CTA's come out of TMEM
#pragma unroll
    for (int i = 0; i < 8; ++i) pv[i] = __ldcg(ppo + (8 * q + i) * 128);
    uint32_t ov[32];
    if (have_o) {
      tmem_ld32(tO + 32 * q, ov);
      tmem_ld_wait();
      reg_fence(ov);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] = 0u;
    }
    auto mix = [&](uint32_t own, float other) {
      return __fadd_rn(__fmul_rn(__uint_as_float(own), ws), __fmul_rn(other, wo));
    };
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pk[2 * i] = pack2<BF16>(mix(ov[4 * i], pv[i].x), mix(ov[4 * i + 1], pv[i].y));
      pk[2 * i + 1] = pack2<BF16>(mix(ov[4 * i + 2], pv[i].z), mix(ov[4 * i + 3], pv[i].w));
    }
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(orow + cb + 32 * q);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (cb + 32 * q + 8 * i < a.d && checked(row < a.Sq && b < a.B && h < a.H, 107))
          dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
  }
  if (valid && c == 0 && checked(b < a.B && h < a.H && row < a.Sq, 108))
    a.lse[(static_cast<int64_t>(b) * a.H + h) * a.Sq + row] =
        has ? (mn + __log2f(lsum_all)) * 0.69314718055994531f : -INFINITY;
}

// Q, K, V and O are fp16 (BF16 = false) or bf16 (BF16 = true).
template <int D, bool BF16>
__global__ void __launch_bounds__(576, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using L = FwdLayout<D>;
  using namespace sm100;
  constexpr int S = L::STAGES;
  constexpr int KCOL = 64;  // elements per 128-byte column block
  // D = 64 leaves room in TMEM for a third S buffer: S products rotate over
  // three buffers (see the MMA issuer), so a tile's next S is ready before
  // its softmax finishes the current block.
  constexpr bool kRot3 = (D == 64);
  constexpr int OBASE = kRot3 ? 384 : 256;  // first TMEM column of O_0

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + S;
  uint64_t* v_full = k_empty + S;
  uint64_t* v_empty = v_full + S;
  uint64_t* s_full = v_empty + S;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_final = p_full + 2;
  uint64_t* drain = o_final + 2;
  uint64_t* pv_done = drain + 1;  // D = 64: P_t(j) V_j has completed
  float* pmax = reinterpret_cast<float*>(smem + L::OFF_PMAX);
  float* lsum = reinterpret_cast<float*>(smem + L::OFF_LSUM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Grid order: unit-major over (b, h). Ranks count query blocks from the
  // last one (the most key blocks) down with a causal mask, from the first
  // without. Unsplit, unit = rank. With a split the units come from
  // FwdArgs::order, longest first: a whole rank, or one half of a split rank
  // (half 0: key blocks [0, hs), half 1: [hs, n), hs = ceil(n / 2) of the
  // block's longer tile).
  // Without a mask and unsplit, every CTA has the same length and the grid
  // is head-major instead: the CTAs running at one time then share a few
  // heads' K and V, which stay in L2.
  const int hb_count = a.H * a.B;
  const bool head_major = !a.causal && a.n_split == 0;
  const int unit = head_major ? static_cast<int>(blockIdx.x) % a.n_qblocks : blockIdx.x / hb_count;
  const int hb = head_major ? static_cast<int>(blockIdx.x) / a.n_qblocks : blockIdx.x % hb_count;
  int rank = unit, half = 0;
  bool split = false;
  if (a.n_split > 0) {
    const int e = a.order[unit < 2 * FwdArgs::kMaxSplitRanks ? unit : 0];
    checked(unit < a.n_qblocks + a.n_split && unit < 2 * FwdArgs::kMaxSplitRanks, 113);
    rank = e / 3;
    split = (e % 3) != 0;
    half = split ? (e % 3) - 1 : 0;
  }
  const int h = hb % a.H;
  const int b = hb / a.H;
  const int qb = a.causal ? (a.n_qblocks - 1 - rank) : rank;
  const int q0 = qb * 256;
  // This CTA's key blocks of tile t: [jlo, jlo + nkv[t]).
  int nkv[2];
  nkv[0] = fwd_kv_blocks(q0, a.Sq, a.Sk, a.causal);
  nkv[1] = fwd_kv_blocks(q0 + 128, a.Sq, a.Sk, a.causal);
  int jlo = 0;
  if (split) {
    const int hs = (max(nkv[0], nkv[1]) + 1) / 2;
    if (half == 0) {
      nkv[0] = min(nkv[0], hs);
      nkv[1] = min(nkv[1], hs);
    } else {
      jlo = hs;
      nkv[0] = max(0, nkv[0] - hs);
      nkv[1] = max(0, nkv[1] - hs);
    }
  }
  const int nmax = max(nkv[0], nkv[1]);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 8);  // one arrival per softmax warp of the tile
      mbar_init(&o_final[t], 1);
      mbar_init(&pv_done[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == L::kLoaderWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == L::kMmaWarp) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == L::kLoaderWarp) {
    // ------------------------------------------------------------ loader
    if (lane == 0 && nmax > 0) {
      int q_bytes = 0;
      for (int t = 0; t < 2; ++t) q_bytes += nkv[t] > 0 ? L::TILE : 0;
      mbar_arrive_expect_tx(q_full, q_bytes);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0) {
          // TMA zero-fills tiles past the tensor's end; the check build still
          // records a tile that starts outside it (a scheduling error).
          checked(q0 + 128 * t < a.Sq && b < a.B && h < a.H, 101);
          for (int kb = 0; kb < L::KB; ++kb)
            tma_load_4d(smem + L::OFF_Q + t * L::TILE + kb * L::BLK, &tmQ, q_full, kb * KCOL, q0 + 128 * t, h, b);
        }
      int j = 0;
      for (; j < nmax; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        if (!wait_bar(&k_empty[st], ph ^ 1, abort_flag, kRoleLoader, j)) break;
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
        checked((jlo + j) * 128 < a.Sk && st < S, 102);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_4d(smem + L::OFF_K + st * L::TILE + kb * L::BLK, &tmK, &k_full[st], kb * KCOL, (jlo + j) * 128, h,
                      b);
        if (!wait_bar(&v_empty[st], ph ^ 1, abort_flag, kRoleLoader, j)) {
          ++j;  // K_j was issued
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
        checked((jlo + j) * 128 < a.Sk && st < S, 102);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_4d(smem + L::OFF_V + st * L::TILE + kb * L::BLK, &tmV, &v_full[st], kb * KCOL, (jlo + j) * 128, h,
                      b);
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA exits. A V copy
        // may be missing for the last K issued; its wait then runs out.
        drain_wait(q_full, 0);
        for (int i = max(0, j - S); i < j; ++i) {
          drain_wait(&k_full[i % S], (i / S) & 1);
          drain_wait(&v_full[i % S], (i / S) & 1);
        }
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged; elect.sync picks the lane that
    // issues each MMA and commit, and every wait is voted warp-wide.
    if (nmax > 0) {
      auto wait = [&](uint64_t* bar, uint32_t parity, int iter) {
        return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, kRoleMma, iter));
      };
      constexpr uint32_t idS = idesc_f16(BF16, 128, 128, 0, 0);
      constexpr uint32_t idO = idesc_f16(BF16, 128, D, 0, 1);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sK = smem_u32(smem + L::OFF_K);
      const uint32_t sV = smem_u32(smem + L::OFF_V);
      // S_t = Q_t K^T into the 128 TMEM columns at `buf`.
      auto issue_S = [&](int t, int st, uint32_t buf) {
        checked(buf + 128 <= OBASE && st < S && t < 2, 103);
        const uint64_t qd = desc_sw128(sQ + t * L::TILE, 16, 1024);
        const uint64_t kd = desc_sw128(sK + st * L::TILE, 16, 1024);
        // 32 bytes of the head dim per instruction, four instructions per
        // 128-byte column block, issued under one elect.
#pragma unroll
        for (int kb = 0; kb < L::KB; ++kb) {
          uint64_t ad[4], bd[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ad[u] = desc_add(qd, kb * L::BLK + u * 32);
            bd[u] = desc_add(kd, kb * L::BLK + u * 32);
          }
          mma_ss_x4(tmem + buf, ad, bd, idS, kb > 0);
        }
      };
      // O_t += P_t V with P_t over the S buffer at `buf`.
      auto issue_PV = [&](int t, int st, uint32_t buf, int acc) {
        checked(buf + 128 <= OBASE && OBASE + (t + 1) * D <= L::TMEM_COLS && st < S, 104);
        const uint64_t vd = desc_sw128(sV + st * L::TILE, L::BLK, 1024);
        // Keys 16kk .. 16kk + 15: P of half kk >> 2 at columns buf + 64(kk >> 2)
        // + 8(kk & 3) (8 columns per 16 keys); V advances 16 rows of 128 bytes.
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // the two halves of P, four instructions each under one elect
          uint32_t pa[4];
          uint64_t vb[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            pa[u] = tmem + buf + 64 * h + u * 8;
            vb[u] = desc_add(vd, (4 * h + u) * 2048);
          }
          mma_ts_x4(tmem + OBASE + t * D, pa, vb, idO, (acc || h > 0) ? 1u : 0u);
        }
      };
      bool ok = wait(q_full, 0, -1);
      if constexpr (kRot3) {
        // S products in the order k = 2j + t (block j, tile t), the k-th into
        // buffer k % 3; P_t(j) overwrites its S there. S(k + 3) is issued
        // right after P V(k), the last reader of the buffer it reuses (the
        // tensor core runs them in issue order), so every S is ready well
        // before the softmax warps reach it. s_full[t] completes once per
        // block of tile t, pv_done[t] once per P_t(j) V_j.
        int kwait = -1, vwait = -1;  // last block whose K / V arrival was awaited
        auto s_exists = [&](int k) { return (k >> 1) < ((k & 1) ? nkv[1] : nkv[0]); };
        auto issue_S_k = [&](int k) {
          const int t = k & 1, j = k >> 1;
          if (j > kwait) {
            if (!wait(&k_full[j % S], (j / S) & 1, j)) return false;
            tc_fence_after();
            kwait = j;
          }
          issue_S(t, j % S, 128 * (k % 3));
          mma_commit_w(&s_full[t]);
          // K_j is free after its last S (tile 1's, or tile 0's where tile 1
          // has no block j).
          if (t == 1 || j >= nkv[1]) mma_commit_w(&k_empty[j % S]);
          return true;
        };
        for (int k = 0; ok && k < 3; ++k)
          if (s_exists(k)) ok = issue_S_k(k);
        for (int k = 0; ok && k < 2 * nmax; ++k) {
          const int t = k & 1, j = k >> 1;
          const int nt = t ? nkv[1] : nkv[0];
          if (j < nt) {
            if (j > vwait) {
              if (!(ok = wait(&v_full[j % S], (j / S) & 1, j))) break;
              vwait = j;
            }
            if (!(ok = wait(&p_full[t], j & 1, j))) break;
            tc_fence_after();
            issue_PV(t, j % S, 128 * (k % 3), j > 0);
            mma_commit_w(&pv_done[t]);
            if (j == nt - 1) mma_commit_w(&o_final[t]);
            if (t == 1 || j >= nkv[1]) mma_commit_w(&v_empty[j % S]);
          }
          if (s_exists(k + 3)) ok = issue_S_k(k + 3);
        }
      } else if (ok && (ok = wait(&k_full[0], 0, 0))) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (nkv[t] > 0) {
            issue_S(t, 0, 128 * t);
            mma_commit_w(&s_full[t]);
          }
        mma_commit_w(&k_empty[0]);
      }
      for (int j = 0; ok && !kRot3 && j < nmax; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        const int jn = j + 1;
        const int stn = jn % S;
        const uint32_t phn = (jn / S) & 1;
        if (!(ok = wait(&v_full[st], ph, j))) break;
        bool kn_ready = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok) break;
          if (j < nkv[t]) {
            if (!(ok = wait(&p_full[t], j & 1, j))) break;
            tc_fence_after();
            issue_PV(t, st, 128 * t, j > 0);
            if (j == nkv[t] - 1) mma_commit_w(&o_final[t]);
            // V_j is free once the last P V that reads it has run (tile 1's,
            // or tile 0's where tile 1 has no block j): the loader may refill
            // its stage while S(j+1) is still on the tensor core.
            if (t == 1 || j >= nkv[1]) mma_commit_w(&v_empty[st]);
          }
          if (jn < nkv[t]) {
            if (!kn_ready) {
              if (!(ok = wait(&k_full[stn], phn, jn))) break;
              tc_fence_after();
              kn_ready = true;
            }
            issue_S(t, stn, 128 * t);
            mma_commit_w(&s_full[t]);
          }
        }
        if (kn_ready) mma_commit_w(&k_empty[stn]);
      }
      // Wait for every MMA this warp issued before TMEM is released.
      mma_commit_w(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------- softmax / epilogue
    const int t = warp >> 3;            // query tile
    const int c = (warp >> 2) & 1;      // key half of every block
    const int quarter = warp & 3;       // TMEM lane quarter
    const int r = quarter * 32 + lane;  // row within the tile
    const int r0 = q0 + 128 * t;
    const int row = r0 + r;
    const int n = t ? nkv[1] : nkv[0];
    const int pair_bar = 1 + t * 4 + quarter;  // named barrier of the two warps that share these rows
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_base + OBASE + t * D + c * (D / 2);  // this half's O columns
    const float sl2 = a.scale_log2;
    const int off = a.Sk - a.Sq;
    float m = -INFINITY;  // running max of x = s * scale * log2(e), the same in both halves
    float l = 0.f;        // this half's running sum of 2^(x - m)
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      // `ok` false here: a wait of the previous block ran out; this warp goes
      // straight to the pair barrier, which then ends both warps.
      const bool ready = ok && __all_sync(0xffffffffu, wait_bar(&s_full[t], j & 1, abort_flag, kRoleSoftmax, j));
      const int k0 = (jlo + j) * 128 + 64 * c;  // first key of this half
      const bool masked = k0 + 64 > a.Sk || (a.causal && k0 + 63 > r0 + off);
      int lim = a.Sk - 1 - k0;  // last allowed column of this half
      if (a.causal) lim = min(lim, row + off - k0);
      float* slot = pmax + (((j & 1) * 2 + t) * 2) * 128;
      // This half's S of block j, then its P (D = 64: buffer (2j + t) % 3).
      const uint32_t tS = tmem + lane_base + 128 * (kRot3 ? (2 * j + t) % 3 : t) + 64 * c;
      checked(128 * (kRot3 ? (2 * j + t) % 3 : t) + 64 * c + 64 <= OBASE && (((j & 1) * 2 + t) * 2 + 2) * 128 <= 1024,
              105);
      float pm = -INFINITY;
      if (ready) {
        tc_fence_after();
        uint32_t rr[2][32];
        tmem_ld32(tS, rr[0]);
        tmem_ld32(tS + 32, rr[1]);
        tmem_ld_wait();
        reg_fence(rr[0]);
        reg_fence(rr[1]);
        if (masked) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              rr[q][i] = (32 * q + i <= lim) ? rr[q][i] : __float_as_uint(-INFINITY);
        }
        auto xf = [&](int i) { return __uint_as_float(rr[i >> 5][i & 31]); };
        float mx0 = max3(xf(0), xf(1), xf(2)), mx1 = max3(xf(3), xf(4), xf(5));
        float mx2 = max3(xf(6), xf(7), xf(8)), mx3 = max3(xf(9), xf(10), xf(11));
#pragma unroll
        for (int i = 12; i < 60; i += 8) {
          mx0 = max3(mx0, xf(i), xf(i + 1));
          mx1 = max3(mx1, xf(i + 2), xf(i + 3));
          mx2 = max3(mx2, xf(i + 4), xf(i + 5));
          mx3 = max3(mx3, xf(i + 6), xf(i + 7));
        }
        mx0 = max3(mx0, xf(60), xf(61));
        mx1 = max3(mx1, xf(62), xf(63));
        pm = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        // The slot of block j is written again in block j + 2, after the
        // partner has passed the barrier of block j + 1, i.e. after it has
        // read this value.
        slot[c * 128 + r] = pm;
      }
      // Both warps of the pair reach this barrier in every block, running or
      // not; it publishes the partial maxima and ANDs the two "ready" flags.
      if (!named_bar_and(pair_bar, 64, ready)) {
        ok = false;
        break;
      }
      const float m_blk = fmaxf(pm, slot[(c ^ 1) * 128 + r]) * sl2;
      const bool raise = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (raise) {
        alpha = ex2(m - m_blk);  // 0 when m was -inf
        m = m_blk;
      }
      l *= alpha;
      // P_t(j-1) V_{j-1} must have completed before O_t is rescaled. D = 128:
      // S_t(j) was issued after it and s_full covers both. D = 64: S_t(j) may
      // have been issued before it, so wait for pv_done.
      const bool rescale = j > 0 && __any_sync(0xffffffffu, raise);
      if (kRot3 && rescale &&
          !__all_sync(0xffffffffu, wait_bar(&pv_done[t], (j - 1) & 1, abort_flag, kRoleSoftmax, j))) {
        ok = false;  // the next pair barrier (or the epilogue's) ends both warps
        continue;
      }
      if (rescale) {
        // Rescale this warp's 32 rows of this half's D/2 columns of O_t. The
        // fence orders the TMEM loads after the wait above.
        tc_fence_after();
#pragma unroll 1
        for (int q = 0; q < D / 64; ++q) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * q, ov);
          tmem_ld_wait();
          reg_fence(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tO + 32 * q, ov);
        }
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      const uint64_t sl2x2 = f2(sl2, sl2);
      const uint64_t negmu2 = f2(-mu, -mu);
      uint64_t acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
      // S is read again from tensor memory 32 columns at a time, so the 64 S
      // values need not stay in registers across the exchange: P of columns
      // 0-31 goes to columns 0-15, P of 32-63 to 16-31, each after the S
      // values under it have been read.
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t sv[32];
        tmem_ld32(tS + 32 * q, sv);
        tmem_ld_wait();
        reg_fence(sv);
        uint32_t pw[16];
        if (masked)
          fwd_exp32<BF16, true>(sv, 32 * q, lim, sl2x2, negmu2, acc0, acc1, pw);
        else
          fwd_exp32<BF16, false>(sv, 32 * q, lim, sl2x2, negmu2, acc0, acc1, pw);
        tmem_st16(tS + 16 * q, pw);
      }
      {
        const uint64_t acc = add2(acc0, acc1);
        float a0, a1;
        f2_split(acc, a0, a1);
        l += a0 + a1;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }

    // Epilogue: O = O_t / (l_0 + l_1), LSE = ln2 * (m + log2(l_0 + l_1)).
    // Both warps of the pair arrive here with the same `ok` (the loop's
    // barrier ANDs it), so both take the barrier below or neither does.
    if (split) {
      // Workspace slots: split rank `rank`, half `half`, (b, h) `hb`.
      fwd_split_epilogue<D, BF16>(a, smem + L::OFF_MISC + 8, lsum, &o_final[t], abort_flag, tO, ok, t, c, r, pair_bar,
                                  n, m, l, rank * hb_count + hb, (2 * rank + half) * hb_count + hb,
                                  (2 * rank + 1 - half) * hb_count + hb, b, h, row, r0);
    } else if (r0 < a.Sq) {
      lsum[(t * 2 + c) * 128 + r] = l;
      const bool go = named_bar_and(pair_bar, 64, ok && !*abort_flag);
      const bool valid = row < a.Sq;
      const int cb = c * (D / 2);  // first O column of this half
      uint16_t* orow = reinterpret_cast<uint16_t*>(a.o) + static_cast<int64_t>(b) * a.o_sb +
                       static_cast<int64_t>(row) * a.o_ss + static_cast<int64_t>(h) * a.o_sh;
      if (go && n > 0) {
        const float lt = l + lsum[(t * 2 + (c ^ 1)) * 128 + r];
        const bool has = (m != -INFINITY) && lt > 0.f;  // m stays -inf only for rows with no allowed key
        const float inv_l = has ? a.o_scale / lt : 0.f;
        if (__all_sync(0xffffffffu, wait_bar(&o_final[t], 0, abort_flag, kRoleSoftmax, n))) {
          tc_fence_after();
#pragma unroll 1
          for (int q = 0; q < D / 64; ++q) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * q, ov);
            tmem_ld_wait();
            reg_fence(ov);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + cb + 32 * q);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (cb + 32 * q + 8 * i < a.d && checked(row < a.Sq && b < a.B && h < a.H, 107))
                  dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
          if (valid && c == 0 && checked(b < a.B && h < a.H && row < a.Sq, 108))
            a.lse[(static_cast<int64_t>(b) * a.H + h) * a.Sq + row] =
                has ? (m + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
        }
      } else if (go && valid) {
        // No key reaches these rows: O = 0, LSE = -inf.
        uint4* dst = reinterpret_cast<uint4*>(orow);
        if (checked(row < a.Sq && b < a.B && h < a.H, 109)) {
          for (int i = cb / 8; i < min(a.d, cb + D / 2) / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
          if (c == 0) a.lse[(static_cast<int64_t>(b) * a.H + h) * a.Sq + row] = -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
