// fa_fwd_e4m3.cuh — fused attention forward for sm_100a, e4m3 inputs with
// per-tensor descales (fa_fwd_fp8).
//
// One CTA computes O and LSE for 256 query rows (two 128-row tiles, t = 0, 1)
// of one (batch, head), streaming 128-key K/V blocks of E4M3 bytes through
// shared memory: S = Q K^T on tcgen05.mma kind::f8f6f4, the online softmax in
// fp32, P rounded to E4M3 for O += P V, and the Sq x Sk score matrix never
// reaches device memory ([P1] "性能引擎"; [P2] item 2 "分块处理"; [P5]
// "H100的FP8加速能力": FP8 in FlashAttention-3). The row sum l uses the
// unrounded P, so LSE is as exact as in 16-bit.
//
// The 16-bit forward (fa_fwd.cuh) shares each tile's softmax between two
// warpgroups. Here one warpgroup owns each tile, one whole 128-key row per
// thread: with kind::f8f6f4 the tensor core finishes a block's two products
// in half the time, and the exchange between two warpgroups would then cost
// more than the longer per-thread exponential loop it saves.
//
// Warp roles (320 threads):
//   warps 0-3  softmax/epilogue for tile 0 (one query row per thread)
//   warps 4-7  softmax/epilogue for tile 1
//   warp  8    TMA loader: Q tiles once, then K_j and V_j into a ring
//   warp  9    MMA issuer (the whole warp; elect.sync picks the issuing lane):
//              S_t = Q_t K_j^T and O_t += P_t V_j
// Tensor memory (512 columns x 128 lanes of fp32):
//   [0,128) S_0   [128,256) S_1   [256,384) O_0   [384,512) O_1
//   P_t (four E4M3 values per column) overwrites the first 32 columns of S_t
//   and feeds P V as the TMEM-resident A operand.
// Softmax per row in base 2: x = s * scale * log2(e) (the Q and K descales
// folded into the scale); running max m and sum l; O_t stays unscaled and is
// divided by l (times V's descale) once at the end, and only LSE = ln2 * (m +
// log2 l) is stored ([P4] §3.1). The running max is raised (and O_t, l
// rescaled) only when a block's max exceeds it by more than 8; otherwise the
// stale max is kept, which is still exact because l, O_t and LSE share it.
// Work split over batch x heads x 256-row blocks ([P4] §3.2); causal grids
// start with the longest rows, skip key blocks past the diagonal and mask only
// diagonal and tail blocks element by element ([P4] §4).
//
// Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
// [P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P4] the FlashAttention-2
// walkthrough titled "企业官网建设流程全解析"; [P5] the FlashAttention
// "IO感知" overview (0539edu.com/news/165270).
#pragma once

#include "fa_common.cuh"
#include "fa_fwd.cuh"  // fwd_kv_blocks, FwdArgs users

namespace fa {

// ESZ: bytes per Q/K/V element (1: e4m3).
template <int D, int ESZ = 1>
struct FwdE4m3Layout {
  static constexpr int kThreads = 320;
  static constexpr int RB = D * ESZ;          // bytes of one tile row
  static constexpr int KB = RB / 128;         // 128-byte column blocks per row
  static constexpr int TILE = 128 * RB;       // bytes of one 128-row tile
  static constexpr int BLK = 128 * 128;       // bytes of one 128-row x 128-byte block
  static constexpr int STAGES = (RB == 256) ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE;
  static constexpr int NBAR = 1 + 4 * STAGES + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // room to align the base to 1024
  static constexpr int TMEM_COLS = 512;
};

// Q, K, V are e4m3 with per-tensor descale factors (folded into a.scale_log2
// and a.o_scale), P is rounded to e4m3 for the P V product, and O is bf16
// (BF16 = true) or fp16.
template <int D, bool BF16>
__global__ void __launch_bounds__(320, 1)
    fa_fwd_e4m3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  static_assert(D == 128, "e4m3 tiles are one 128-byte swizzle block wide");
  using L = FwdE4m3Layout<D, 1>;
  constexpr int KCOL = 128;  // elements per 128-byte column block
  using namespace sm100;
  constexpr int S = L::STAGES;

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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Linear block order: all heads' heaviest query blocks first (causal).
  const int hb_count = a.H * a.B;
  const int rank = blockIdx.x / hb_count;
  const int hb = blockIdx.x % hb_count;
  const int h = hb % a.H;
  const int b = hb / a.H;
  const int qb = a.causal ? (a.n_qblocks - 1 - rank) : rank;
  const int q0 = qb * 256;
  int nkv[2];
  nkv[0] = fwd_kv_blocks(q0, a.Sq, a.Sk, a.causal);
  nkv[1] = fwd_kv_blocks(q0 + 128, a.Sq, a.Sk, a.causal);
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
      mbar_init(&p_full[t], 128);
      mbar_init(&o_final[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ loader
    if (lane == 0 && nmax > 0) {
      int q_bytes = 0;
      for (int t = 0; t < 2; ++t) q_bytes += nkv[t] > 0 ? L::TILE : 0;
      mbar_arrive_expect_tx(q_full, q_bytes);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0) {
          checked(q0 + 128 * t < a.Sq && b < a.B && h < a.H, 301);
          for (int kb = 0; kb < L::KB; ++kb)
            tma_load_4d(smem + L::OFF_Q + t * L::TILE + kb * L::BLK, &tmQ, q_full, kb * KCOL, q0 + 128 * t, h, b);
        }
      int j = 0;
      for (; j < nmax; ++j) {
        const int st = j % S;
        const uint32_t ph = (j / S) & 1;
        if (!wait_bar(&k_empty[st], ph ^ 1, abort_flag, kRoleLoader, j)) break;
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
        checked(j * 128 < a.Sk && st < S, 302);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_4d(smem + L::OFF_K + st * L::TILE + kb * L::BLK, &tmK, &k_full[st], kb * KCOL, j * 128, h, b);
        if (!wait_bar(&v_empty[st], ph ^ 1, abort_flag, kRoleLoader, j)) {
          ++j;  // K_j was issued
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_4d(smem + L::OFF_V + st * L::TILE + kb * L::BLK, &tmV, &v_full[st], kb * KCOL, j * 128, h, b);
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA exits.
        drain_wait(q_full, 0);
        for (int i = max(0, j - S); i < j; ++i) {
          drain_wait(&k_full[i % S], (i / S) & 1);
          drain_wait(&v_full[i % S], (i / S) & 1);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged; elect.sync picks the lane that
    // issues each MMA and commit, and every wait is voted warp-wide.
    if (nmax > 0) {
      auto wait = [&](uint64_t* bar, uint32_t parity, int iter) {
        return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, kRoleMma, iter));
      };
      const uint32_t idS = idesc_e4m3(128, 128, 0, 0);
      const uint32_t idO = idesc_e4m3(128, D, 0, 1);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sK = smem_u32(smem + L::OFF_K);
      const uint32_t sV = smem_u32(smem + L::OFF_V);
      auto issue_S = [&](int t, int st) {
        const uint64_t qd = desc_sw128(sQ + t * L::TILE, 16, 1024);
        const uint64_t kd = desc_sw128(sK + st * L::TILE, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < L::RB / 32; ++kk) {  // 32 bytes of K per instruction
          const uint32_t o = (kk >> 2) * L::BLK + (kk & 3) * 32;
          mma_ss_f8_w(tmem + t * 128, desc_add(qd, o), desc_add(kd, o), idS, kk > 0);
        }
      };
      auto issue_PV = [&](int t, int st, int acc) {
        const uint64_t vd = desc_sw128(sV + st * L::TILE, L::BLK, 1024);
        // P occupies 8 TMEM columns per instruction (32 keys of e4m3); V
        // advances by as many 128-byte rows.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_f8_w(tmem + 256 + t * D, tmem + t * 128 + kk * 8, desc_add(vd, kk * 4096), idO,
                      (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait(q_full, 0, -1) && wait(&k_full[0], 0, 0);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (nkv[t] > 0) {
            issue_S(t, 0);
            mma_commit_w(&s_full[t]);
          }
        mma_commit_w(&k_empty[0]);
      }
      for (int j = 0; ok && j < nmax; ++j) {
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
            issue_PV(t, st, j > 0);
            if (j == nkv[t] - 1) mma_commit_w(&o_final[t]);
          }
          if (jn < nkv[t]) {
            if (!kn_ready) {
              if (!(ok = wait(&k_full[stn], phn, jn))) break;
              tc_fence_after();
              kn_ready = true;
            }
            issue_S(t, stn);
            mma_commit_w(&s_full[t]);
          }
        }
        mma_commit_w(&v_empty[st]);
        if (kn_ready) mma_commit_w(&k_empty[stn]);
      }
      // Wait for every MMA this warp issued before TMEM is released.
      mma_commit_w(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------- softmax / epilogue
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int r0 = q0 + 128 * t;
    const int row = r0 + quarter * 32 + lane;
    const int n = nkv[t];
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + 256 + t * D;
    const float sl2 = a.scale_log2;
    const int off = a.Sk - a.Sq;
    float m = -INFINITY;  // running max of x = s * scale * log2(e)
    float l = 0.f;        // running sum of 2^(x - m)
    bool ok = true;

    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, wait_bar(&s_full[t], j & 1, abort_flag, kRoleSoftmax, j));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      const int k0 = j * 128;
      if (k0 + 128 > a.Sk || (a.causal && k0 + 127 > r0 + off)) {
        int lim = a.Sk - 1 - k0;  // last allowed column of this block
        if (a.causal) lim = min(lim, row + off - k0);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) r[c][i] = (32 * c + i <= lim) ? r[c][i] : __float_as_uint(-INFINITY);
      }
      auto xf = [&](int i) { return __uint_as_float(r[i >> 5][i & 31]); };
      float mx0 = max3(xf(0), xf(1), xf(2)), mx1 = max3(xf(3), xf(4), xf(5));
      float mx2 = max3(xf(6), xf(7), xf(8)), mx3 = max3(xf(9), xf(10), xf(11));
#pragma unroll
      for (int i = 12; i < 124; i += 8) {
        mx0 = max3(mx0, xf(i), xf(i + 1));
        mx1 = max3(mx1, xf(i + 2), xf(i + 3));
        mx2 = max3(mx2, xf(i + 4), xf(i + 5));
        mx3 = max3(mx3, xf(i + 6), xf(i + 7));
      }
      mx0 = max3(mx0, xf(124), xf(125));
      mx1 = max3(mx1, xf(126), xf(127));
      const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      const bool raise = m_blk > m + 8.0f;
      float alpha = 1.f;
      if (raise) {
        alpha = ex2(m - m_blk);  // 0 when m was -inf
        m = m_blk;
      }
      l *= alpha;
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        // Rescale this warp's 32 rows of the unscaled accumulator O_t.
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * c, ov);
          tmem_ld_wait();
          reg_fence(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tO + 32 * c, ov);
        }
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      // P = 2^(s * scale * log2e - m) for pairs of columns; one pair in four
      // takes the polynomial exp2 on the FMA pipe, the rest the MUFU unit.
      // The polynomial gives 2^-126 rather than 0 for a masked (-inf) entry:
      // that rounds to an exact 0 in E4M3 (smallest subnormal 2^-9), so P V
      // never sees it, and it is far below an ulp of l (l >= 2^-8).
      const uint64_t sl2x2 = f2(sl2, sl2);
      const uint64_t negmu2 = f2(-mu, -mu);
      uint64_t acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 32 columns at a time -> 8 words of four E4M3 values
        uint32_t pw[8];
        float h0 = 0.f, h1 = 0.f;  // the even pair, packed with the odd one
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const int c = 16 * q + cc;
          const uint64_t tt = fma2(f2(xf(2 * c), xf(2 * c + 1)), sl2x2, negmu2);
          uint64_t e;
          if ((c & 3) == 3) {
            e = exp2_poly2(tt);
          } else {
            float t0, t1;
            f2_split(tt, t0, t1);
            e = f2(ex2(t0), ex2(t1));
          }
          if (c & 1)
            acc1 = add2(acc1, e);
          else
            acc0 = add2(acc0, e);
          float e0, e1;
          f2_split(e, e0, e1);
          if (cc & 1)
            pw[cc >> 1] = pack4_e4m3(h0, h1, e0, e1);
          else
            h0 = e0, h1 = e1;
        }
        // Every S column of this row is in registers already.
        tmem_st8(tS + 8 * q, pw);
      }
      {
        const uint64_t acc = add2(acc0, acc1);
        float a0, a1;
        f2_split(acc, a0, a1);
        l += a0 + a1;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }

    // Epilogue: O = O_t / l, LSE = ln2 * (m + log2 l).
    if (ok && !*abort_flag && r0 < a.Sq) {
      const bool valid = row < a.Sq;
      const bool has = (m != -INFINITY) && l > 0.f;  // m stays -inf only for rows with no allowed key
      const float inv_l = has ? a.o_scale / l : 0.f;  // o_scale: V's descale (1 for 16-bit inputs)
      uint16_t* orow = reinterpret_cast<uint16_t*>(a.o) + static_cast<int64_t>(b) * a.o_sb +
                       static_cast<int64_t>(row) * a.o_ss + static_cast<int64_t>(h) * a.o_sh;
      if (n > 0) {
        if (__all_sync(0xffffffffu, wait_bar(&o_final[t], 0, abort_flag, kRoleSoftmax, n))) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < (a.d + 31) / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov);
            tmem_ld_wait();
            reg_fence(ov);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (32 * c + 8 * i < a.d && checked(row < a.Sq && b < a.B && h < a.H, 307))
                  dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      } else if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
        if (checked(row < a.Sq && b < a.B && h < a.H, 309))
          for (int i = 0; i < a.d / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
      }
      if (valid && checked(b < a.B && h < a.H && row < a.Sq, 308))
        a.lse[(static_cast<int64_t>(b) * a.H + h) * a.Sq + row] =
            has ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
