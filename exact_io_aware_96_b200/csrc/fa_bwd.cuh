// fa_bwd.cuh — attention backward for sm_100a.
//
// Three kernels on the caller's stream:
//  1. fa_bwd_pre:  Dvec_i = sum_d dO_id O_id and lse2_i = LSE_i * log2(e)
//                  (+inf for rows with no key and for padding rows) into the
//                  workspace; zero the fp32 dQ accumulator.
//  2. fa_bwd_main: one CTA per (batch, head, 128-key block). Keeps K, V and the
//                  fp32 dK, dV accumulators on chip and walks the query blocks
//                  that can see its keys (from the diagonal block on when
//                  causal). Per query block it recomputes S^T = K Q^T and
//                  P^T = 2^(S^T scale log2e - lse2) from the saved logsumexp
//                  instead of reading P ([P1] "性能引擎" recomputation; [P2]
//                  item 3 "重计算"; [P4] §3.1: only the logsumexp is kept),
//                  forms dP^T = V dO^T, dS^T = P^T (dP^T - Dvec), and runs the
//                  five matrix products of the backward ([P4] §3.3):
//                  S^T, dP^T, dV += P^T dO, dK += dS^T Q, and dQ = dS K, whose
//                  block result is added into the fp32 accumulator in global
//                  memory.
//  3. fa_bwd_dq:   dq = scale * accumulator, rounded to the input dtype.
//
// The formulas are the textbook gradient of softmax(x) V: with P = softmax(X),
// dV = P^T dO, dP = dO V^T, dX = P (dP - rowsum(P dP)), dQ = scale dX K,
// dK = scale dX^T Q, and rowsum(P dP)_i = sum_d dO_id O_id.
//
// Main kernel, warp roles (320 threads):
//   warps 0-3  one key row per thread: P^T, dS^T; at the end dK
//   warps 4-7  read the dQ block from TMEM, add it into the accumulator; at the end dV
//   warp  8    TMA loader: K, V once; Q_i, dO_i, lse2_i, Dvec_i per query block
//   warp  9    MMA issuer
// D = 128 uses 64-row query blocks and two S^T/dP^T buffers so the softmax of
// block i+1 overlaps the products of block i; dQ is computed transposed
// (dQ^T = K^T dS^T, M = head_dim) into the dP^T buffer it follows. D = 64 uses
// 128-row query blocks, one buffer, and dQ = dS K into its own columns.
//
// Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
// [P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P4] the FlashAttention-2
// walkthrough titled "企业官网建设流程全解析".
#pragma once

#include "fa.h"
#include "fa_common.cuh"

namespace fa {

// ------------------------------------------------------------- preprocess
// One group of D/8 threads per (b, h, i) row, i in [0, Sq_pad).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre(const BwdArgs a) {
  constexpr int G = D / 8;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gid / G;
  const int part = static_cast<int>(gid % G);
  const int64_t nrows = static_cast<int64_t>(a.B) * a.H * a.Sq_pad;
  if (row >= nrows) return;  // whole groups leave together: G divides 32
  const int i = static_cast<int>(row % a.Sq_pad);
  const int bh = static_cast<int>(row / a.Sq_pad);
  const int h = bh % a.H;
  const int b = bh / a.H;
  float acc = 0.f;
  if (i < a.Sq) {
    const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.o) + b * a.o_sb +
                                                      static_cast<int64_t>(i) * a.o_ss + h * a.o_sh + part * 8);
    const uint4 dv = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.dO) + b * a.do_sb +
                                                      static_cast<int64_t>(i) * a.do_ss + h * a.do_sh + part * 8);
    const uint32_t* o32 = reinterpret_cast<const uint32_t*>(&ov);
    const uint32_t* d32 = reinterpret_cast<const uint32_t*>(&dv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 x = sm100::unpack2<BF16>(o32[k]);
      const float2 y = sm100::unpack2<BF16>(d32[k]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int s = G / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  float4* dq = reinterpret_cast<float4*>(a.dq_acc + row * D + part * 8);
  dq[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  dq[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (part == 0) {
    a.dvec[row] = acc;
    float l2 = INFINITY;
    if (i < a.Sq) {
      const float lse = a.lse[static_cast<int64_t>(bh) * a.Sq + i];
      if (lse != -INFINITY) l2 = lse * 1.4426950408889634f;
    }
    a.lse2[row] = l2;
  }
}

// ------------------------------------------------------------- dq convert
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq(const BwdArgs a) {
  constexpr int G = D / 8;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gid / G;  // (b, h, i) with i < Sq
  const int part = static_cast<int>(gid % G);
  if (row >= static_cast<int64_t>(a.B) * a.H * a.Sq) return;
  const int i = static_cast<int>(row % a.Sq);
  const int bh = static_cast<int>(row / a.Sq);
  const int h = bh % a.H;
  const int b = bh / a.H;
  const float4* src = reinterpret_cast<const float4*>(a.dq_acc + (static_cast<int64_t>(bh) * a.Sq_pad + i) * D +
                                                      part * 8);
  const float4 x = src[0], y = src[1];
  const float s = a.scale;
  uint4 out;
  out.x = sm100::pack2<BF16>(x.x * s, x.y * s);
  out.y = sm100::pack2<BF16>(x.z * s, x.w * s);
  out.z = sm100::pack2<BF16>(y.x * s, y.y * s);
  out.w = sm100::pack2<BF16>(y.z * s, y.w * s);
  *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.dq) + b * a.dq_sb + static_cast<int64_t>(i) * a.dq_ss +
                            h * a.dq_sh + part * 8) = out;
}

// ------------------------------------------------------------- main kernel
template <int D>
struct BwdLayout {
  static constexpr int kThreads = 320;
  static constexpr int BN = 128;                 // keys per CTA
  static constexpr int BM = (D == 128) ? 64 : 128;  // query rows per block
  static constexpr int NBUF = (D == 128) ? 2 : 1;   // S^T/dP^T buffers in TMEM
  static constexpr int QS = 2;                   // Q/dO stages
  static constexpr int KB = D / 64;              // 64-column blocks per row
  static constexpr int KV_TILE = BN * D * 2;     // K or V tile bytes
  static constexpr int KV_BLK = BN * 128;        // one [128 rows][64 cols] block
  static constexpr int Q_TILE = BM * D * 2;      // Q or dO tile bytes
  static constexpr int Q_BLK = BM * 128;         // one [BM rows][64 cols] block
  static constexpr int DS_TILE = BN * BM * 2;    // dS^T tile bytes [128 keys][BM]
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int OFF_Q = OFF_V + KV_TILE;
  static constexpr int OFF_DO = OFF_Q + QS * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + QS * Q_TILE;
  static constexpr int OFF_LSE = OFF_DS + 2 * DS_TILE;
  static constexpr int OFF_DVEC = OFF_LSE + QS * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + QS * BM * 4;
  // kv_full, q_full[QS], q_empty[QS], s_full[NBUF], ds_ready[NBUF], ds_free[2],
  // dq_full[NBUF], dq_free[NBUF], mma_done, drain
  static constexpr int NBAR = 1 + 2 * QS + 4 * NBUF + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static constexpr int TMEM_COLS = 512;
  // TMEM columns
  static constexpr int COL_DK = 0;
  static constexpr int COL_DV = D;
  __host__ __device__ static constexpr int col_s(int b) { return 2 * D + b * 2 * BM; }
  __host__ __device__ static constexpr int col_dp(int b) { return 2 * D + b * 2 * BM + BM; }
  __host__ __device__ static constexpr int col_dq(int b) { return NBUF == 2 ? col_dp(b) : 2 * D + 2 * BM; }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_main(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO, const BwdArgs a) {
  using L = BwdLayout<D>;
  using namespace sm100;
  constexpr int BM = L::BM, NBUF = L::NBUF, QS = L::QS;
  static_assert(L::col_dq(NBUF - 1) + (NBUF == 2 ? BM : D) <= L::TMEM_COLS, "TMEM budget");
  static_assert(L::BYTES + 1024 <= 232448, "smem budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* s_full = q_empty + QS;
  uint64_t* ds_ready = s_full + NBUF;
  uint64_t* dq_full = ds_ready + NBUF;
  uint64_t* dq_free = dq_full + NBUF;
  uint64_t* ds_free = dq_free + NBUF;
  uint64_t* mma_done = ds_free + 2;
  uint64_t* drain = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_dvec = reinterpret_cast<const float*>(smem + L::OFF_DVEC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int hb_count = a.H * a.B;
  const int kvb = blockIdx.x / hb_count;  // causal: the first key blocks see the most queries
  const int hb = blockIdx.x % hb_count;
  const int h = hb % a.H;
  const int b = hb / a.H;
  const int n0 = kvb * L::BN;
  const int off = a.Sk - a.Sq;
  const int nqb = (a.Sq + BM - 1) / BM;
  int i_start = 0;
  if (a.causal) {
    const int qmin = n0 - off;  // smallest query row that may see key n0
    i_start = qmin <= 0 ? 0 : qmin / BM;
  }
  const int n = max(0, nqb - i_start);
  const int64_t bh_row0 = static_cast<int64_t>(b * a.H + h) * a.Sq_pad;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < NBUF; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&ds_ready[s], 128);
      mbar_init(&dq_full[s], 1);
      mbar_init(&dq_free[s], 128);
    }
    mbar_init(&ds_free[0], 1);
    mbar_init(&ds_free[1], 1);
    mbar_init(mma_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
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
    // ---------------------------------------------------------------- loader
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(kv_full, 2 * L::KV_TILE);
      for (int kb = 0; kb < L::KB; ++kb) {
        tma_load_4d(smem + L::OFF_K + kb * L::KV_BLK, &tmK, kv_full, kb * 64, n0, h, b);
        tma_load_4d(smem + L::OFF_V + kb * L::KV_BLK, &tmV, kv_full, kb * 64, n0, h, b);
      }
      int i = 0;
      for (; i < n; ++i) {
        const int st = i % QS;
        const uint32_t ph = (i / QS) & 1;
        if (!wait_bar(&q_empty[st], ph ^ 1, abort_flag, kRoleLoader, i)) break;
        const int i0 = (i_start + i) * BM;
        mbar_arrive_expect_tx(&q_full[st], 2 * L::Q_TILE + 2 * BM * 4);
        for (int kb = 0; kb < L::KB; ++kb) {
          tma_load_4d(smem + L::OFF_Q + st * L::Q_TILE + kb * L::Q_BLK, &tmQ, &q_full[st], kb * 64, i0, h, b);
          tma_load_4d(smem + L::OFF_DO + st * L::Q_TILE + kb * L::Q_BLK, &tmdO, &q_full[st], kb * 64, i0, h, b);
        }
        bulk_load(smem + L::OFF_LSE + st * BM * 4, a.lse2 + bh_row0 + i0, BM * 4, &q_full[st]);
        bulk_load(smem + L::OFF_DVEC + st * BM * 4, a.dvec + bh_row0 + i0, BM * 4, &q_full[st]);
      }
      if (*abort_flag) {
        drain_wait(kv_full, 0);
        for (int j = max(0, i - QS); j < i; ++j) drain_wait(&q_full[j % QS], (j / QS) & 1);
      }
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      const uint32_t sK = smem_u32(smem + L::OFF_K);
      const uint32_t sV = smem_u32(smem + L::OFF_V);
      const uint32_t sQ = smem_u32(smem + L::OFF_Q);
      const uint32_t sdO = smem_u32(smem + L::OFF_DO);
      const uint32_t sDS = smem_u32(smem + L::OFF_DS);
      // S^T = K Q^T and dP^T = V dO^T: M = 128 keys, N = BM queries, K = D.
      const uint32_t id_s = idesc_f16(BF16, 128, BM, 0, 0);
      // dV += P^T dO, dK += dS^T Q: M = 128 keys, N = D, K = BM (B operand MN-major).
      const uint32_t id_kv = idesc_f16(BF16, 128, D, 0, 1);
      // dQ^T = K^T dS^T (D = 128): M = D, N = BM; dQ = dS K (D = 64): M = BM, N = D. Both operands MN-major.
      const uint32_t id_q = (NBUF == 2) ? idesc_f16(BF16, 128, BM, 1, 1) : idesc_f16(BF16, 128, D, 1, 1);

      auto issue_sdp = [&](int i) {
        const int bf = i % NBUF;
        const int st = i % QS;
        const uint32_t qa = sQ + st * L::Q_TILE;
        const uint32_t da = sdO + st * L::Q_TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * L::KV_BLK + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * L::Q_BLK + (kk & 3) * 32;
          mma_ss(tmem + L::col_s(bf), desc_sw128(sK + okv, 16, 1024), desc_sw128(qa + oq, 16, 1024), id_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * L::KV_BLK + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * L::Q_BLK + (kk & 3) * 32;
          mma_ss(tmem + L::col_dp(bf), desc_sw128(sV + okv, 16, 1024), desc_sw128(da + oq, 16, 1024), id_s, kk > 0);
        }
        mma_commit(&s_full[bf]);
      };

      bool ok = wait_bar(kv_full, 0, abort_flag, kRoleMma, -1) && wait_bar(&q_full[0], 0, abort_flag, kRoleMma, 0);
      if (ok) {
        tc_fence_after();
        issue_sdp(0);
      }
      for (int i = 0; ok && i < n; ++i) {
        const int bf = i % NBUF;
        const int st = i % QS;
        const int db = i & 1;
        if (NBUF == 2 && i + 1 < n) {
          // The other buffer held S^T/dP^T(i-1) and then dQ^T(i-1): wait until it is drained.
          if (i >= 1 && !(ok = wait_bar(&dq_free[(i - 1) % NBUF], ((i - 1) / NBUF) & 1, abort_flag, kRoleMma, i)))
            break;
          if (!(ok = wait_bar(&q_full[(i + 1) % QS], ((i + 1) / QS) & 1, abort_flag, kRoleMma, i + 1))) break;
          tc_fence_after();
          issue_sdp(i + 1);
        }
        if (!(ok = wait_bar(&ds_ready[bf], (i / NBUF) & 1, abort_flag, kRoleMma, i))) break;
        tc_fence_after();
        const uint32_t qa = sQ + st * L::Q_TILE;
        const uint32_t da = sdO + st * L::Q_TILE;
        const uint32_t dsa = sDS + db * L::DS_TILE;
        // dV += P^T dO  (P^T in TMEM, 16-bit pairs in the S^T columns)
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + L::COL_DV, tmem + L::col_s(bf) + kk * 8, desc_sw128(da + kk * 2048, L::Q_BLK, 1024), id_kv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q  (dS^T K-major in smem: [128 keys][BM] in 64-column blocks)
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ss(tmem + L::COL_DK, desc_sw128(dsa + (kk >> 2) * L::KV_BLK + (kk & 3) * 32, 16, 1024),
                 desc_sw128(qa + kk * 2048, L::Q_BLK, 1024), id_kv, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&q_empty[st]);
        if (NBUF == 1 && i >= 1)
          if (!(ok = wait_bar(&dq_free[0], (i - 1) & 1, abort_flag, kRoleMma, i))) break;
        if (NBUF == 2) {
          // dQ^T = K^T dS^T: A = K viewed MN-major (M = head_dim), B = dS^T MN-major (N = queries).
#pragma unroll
          for (int kk = 0; kk < L::BN / 16; ++kk)
            mma_ss(tmem + L::col_dq(bf), desc_sw128(sK + kk * 2048, L::KV_BLK, 1024),
                   desc_sw128(dsa + kk * 2048, L::KV_BLK, 1024), id_q, kk > 0);
        } else {
          // dQ = dS K: A = dS^T viewed MN-major (M = queries), B = K MN-major (N = head_dim).
#pragma unroll
          for (int kk = 0; kk < L::BN / 16; ++kk)
            mma_ss(tmem + L::col_dq(0), desc_sw128(dsa + kk * 2048, L::KV_BLK, 1024),
                   desc_sw128(sK + kk * 2048, L::KV_BLK, 1024), id_q, kk > 0);
        }
        mma_commit(&dq_full[bf]);
        mma_commit(&ds_free[db]);
        if (NBUF == 1 && i + 1 < n) {
          if (!(ok = wait_bar(&q_full[(i + 1) % QS], ((i + 1) / QS) & 1, abort_flag, kRoleMma, i + 1))) break;
          tc_fence_after();
          issue_sdp(i + 1);
        }
      }
      mma_commit(mma_done);
      mma_commit(drain);
      drain_wait(drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------ P^T, dS^T (one key per thread)
    const int kr = warp * 32 + lane;
    const int key = n0 + kr;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int bf = i % NBUF;
      const int st = i % QS;
      const int db = i & 1;
      ok = __all_sync(0xffffffffu, wait_bar(&s_full[bf], (i / NBUF) & 1, abort_flag, kRoleSoftmax, i) &&
                                       wait_bar(&q_full[st], (i / QS) & 1, abort_flag, kRoleSoftmax, i) &&
                                       wait_bar(&ds_free[db], ((i >> 1) & 1) ^ 1, abort_flag, kRoleSoftmax, i));
      if (!ok) break;
      tc_fence_after();
      const int i0 = (i_start + i) * BM;
      // columns c < cmin are masked for this key (causal), all columns if key >= Sk
      int cmin = a.causal ? key - off - i0 : -1;
      if (key >= a.Sk) cmin = BM;
      const float* lse_s = s_lse + st * BM;
      const float* dvec_s = s_dvec + st * BM;
      const uint32_t ds_row = smem_u32(smem + L::OFF_DS + db * L::DS_TILE) + kr * 128;
#pragma unroll
      for (int c = 0; c < BM / 32; ++c) {
        uint32_t sv[32], dpv[32];
        tmem_ld32(tmem + lane_base + L::col_s(bf) + 32 * c, sv);
        tmem_ld32(tmem + lane_base + L::col_dp(bf) + 32 * c, dpv);
        tmem_ld_wait();
        reg_fence(sv);
        reg_fence(dpv);
        uint32_t pp[16], dsp[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int q = 32 * c + e;
          float s0 = __uint_as_float(sv[e]), s1 = __uint_as_float(sv[e + 1]);
          s0 = (q < cmin) ? -INFINITY : s0;
          s1 = (q + 1 < cmin) ? -INFINITY : s1;
          const float p0 = ex2(fmaf(s0, sl2, -lse_s[q]));
          const float p1 = ex2(fmaf(s1, sl2, -lse_s[q + 1]));
          const float d0 = p0 * (__uint_as_float(dpv[e]) - dvec_s[q]);
          const float d1 = p1 * (__uint_as_float(dpv[e + 1]) - dvec_s[q + 1]);
          pp[e >> 1] = pack2<BF16>(p0, p1);
          dsp[e >> 1] = pack2<BF16>(d0, d1);
        }
        tmem_st16(tmem + lane_base + L::col_s(bf) + 16 * c, pp);
        // dS^T row kr, query columns [32c, 32c + 32): four 16-byte chunks,
        // 128-byte swizzle within each 64-column block.
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = 4 * (c & 1) + u;
          const uint32_t addr = ds_row + (c >> 1) * L::KV_BLK + ((chunk ^ (kr & 7)) << 4);
          st_shared_v4(addr, dsp[4 * u], dsp[4 * u + 1], dsp[4 * u + 2], dsp[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ds_ready[bf]);
    }
    // epilogue: dK = scale * accumulator
    const bool have = n > 0;
    if (ok && !*abort_flag) {
      bool done = !have || __all_sync(0xffffffffu, wait_bar(mma_done, 0, abort_flag, kRoleSoftmax, n));
      if (done) {
        tc_fence_after();
        uint16_t* dst = reinterpret_cast<uint16_t*>(a.dk) + b * a.dk_sb + static_cast<int64_t>(key) * a.dk_ss +
                        h * a.dk_sh;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tmem + lane_base + L::COL_DK + 32 * c, v);
            tmem_ld_wait();
            reg_fence(v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (key < a.Sk) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = pack2<BF16>(__uint_as_float(v[8 * u + 2 * e]) * a.scale,
                                   __uint_as_float(v[8 * u + 2 * e + 1]) * a.scale);
              d4[u] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------- dQ drain (warps 4-7), then dV
    const int wq = warp - 4;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int tr = wq * 32 + lane;  // TMEM lane: head_dim index (D = 128) or query row (D = 64)
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int bf = i % NBUF;
      ok = __all_sync(0xffffffffu, wait_bar(&dq_full[bf], (i / NBUF) & 1, abort_flag, kRoleSoftmax, i));
      if (!ok) break;
      tc_fence_after();
      const int i0 = (i_start + i) * BM;
      if constexpr (NBUF == 2) {
        // dQ^T: lane = head_dim index d, columns = BM = 64 query rows.
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_base + L::col_dq(bf), v0);
        tmem_ld32(tmem + lane_base + L::col_dq(bf) + 32, v1);
        tmem_ld_wait();
        reg_fence(v0);
        reg_fence(v1);
        tc_fence_before();
        mbar_arrive(&dq_free[bf]);
        float* base = a.dq_acc + (bh_row0 + i0) * D + tr;
#pragma unroll
        for (int c = 0; c < 32; ++c) red_add_f32(base + c * D, __uint_as_float(v0[c]));
#pragma unroll
        for (int c = 0; c < 32; ++c) red_add_f32(base + (32 + c) * D, __uint_as_float(v1[c]));
      } else {
        // dQ: lane = query row, columns = head_dim (64).
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_base + L::col_dq(0), v0);
        tmem_ld32(tmem + lane_base + L::col_dq(0) + 32, v1);
        tmem_ld_wait();
        reg_fence(v0);
        reg_fence(v1);
        tc_fence_before();
        mbar_arrive(&dq_free[0]);
        float* base = a.dq_acc + (bh_row0 + i0 + tr) * D;
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          red_add_v4_f32(base + c, __uint_as_float(v0[c]), __uint_as_float(v0[c + 1]), __uint_as_float(v0[c + 2]),
                         __uint_as_float(v0[c + 3]));
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          red_add_v4_f32(base + 32 + c, __uint_as_float(v1[c]), __uint_as_float(v1[c + 1]),
                         __uint_as_float(v1[c + 2]), __uint_as_float(v1[c + 3]));
      }
    }
    // epilogue: dV
    const int key = n0 + tr;
    const bool have = n > 0;
    if (ok && !*abort_flag) {
      bool done = !have || __all_sync(0xffffffffu, wait_bar(mma_done, 0, abort_flag, kRoleSoftmax, n));
      if (done) {
        tc_fence_after();
        uint16_t* dst = reinterpret_cast<uint16_t*>(a.dv) + b * a.dv_sb + static_cast<int64_t>(key) * a.dv_ss +
                        h * a.dv_sh;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tmem + lane_base + L::COL_DV + 32 * c, v);
            tmem_ld_wait();
            reg_fence(v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (key < a.Sk) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = pack2<BF16>(__uint_as_float(v[8 * u + 2 * e]), __uint_as_float(v[8 * u + 2 * e + 1]));
              d4[u] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
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
