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
// Main kernel, warp roles (448 threads):
//   warps 0-7   P^T and dS^T, one key row per thread; warps 0-3 take query
//               columns [0, 64), warps 4-7 [64, 128). At the end warps 0-3
//               write dK and warps 4-7 write dV.
//   warps 8-11  read the dQ block out of TMEM and add it into the fp32
//               accumulator. D = 128: dQ^T (one head_dim index per thread),
//               staged in shared memory a quarter (32 query rows) at a time
//               and added by TMA bulk reductions, which keeps the reduction
//               traffic off the load/store queues the softmax warps use.
//               D = 64: each warp stages its 32 query rows (8 KB) and has the
//               TMA add them. Deterministic mode: plain stores into the
//               block's own slot.
//   warp  12    TMA loader: K, V once; Q_i with lse2_i and dO_i with Dvec_i per
//               query block, on separate rings (Q runs ahead of dO)
//   warp  13    MMA issuer (the whole warp; elect.sync picks the issuing lane)
// Blocks are 128 keys x 128 queries. Tensor memory: dK and dV accumulators,
// X (S^T, then 16-bit P^T written back by the softmax warps and used as the
// TMEM A operand of dV += P^T dO) and Y (dP^T, then dQ^T = K^T dS^T (D = 128)
// or dQ = dS K (D = 64)). dS^T goes to 128-byte swizzled smem, where it is
// the A operand of dK += dS^T Q and an operand of the dQ product. The MMA
// order per block i is dV(i), S^T(i+1), dK(i), dQ(i), dP^T(i+1): X is free as
// soon as dV(i) has read P^T(i), so the softmax warps start on block i+1
// while the tensor core runs dK(i) and dQ(i), and dP^T(i+1) follows once
// dQ(i) has been drained out of Y.
//
// Page legend: [P1] "Miniconda-Python3.9环境下使用FlashAttention优化训练";
// [P2] "使用FlashAttention优化PyTorch模型注意力计算"; [P4] the FlashAttention-2
// walkthrough titled "企业官网建设流程全解析".
#pragma once

#include <type_traits>

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
  if (i < a.Sq && part * 8 < a.d && checked(b < a.B && h < a.H && part * 8 + 8 <= D, 201)) {
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
  if (a.dq_part == nullptr && checked(row < nrows && part * 8 + 8 <= D, 202)) {  // the atomic accumulator starts from zero
    float4* dq = reinterpret_cast<float4*>(a.dq_acc + row * D + part * 8);
    dq[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    dq[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (part == 0 && checked(row < nrows, 203)) {
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
  if (row >= static_cast<int64_t>(a.B) * a.H * a.Sq || part * 8 >= a.d) return;
  const int i = static_cast<int>(row % a.Sq);
  const int bh = static_cast<int>(row / a.Sq);
  const int h = bh % a.H;
  const int b = bh / a.H;
  if (!checked(b < a.B && i < a.Sq_pad && part * 8 + 8 <= D, 206)) return;
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

// ------------------------------------------------ deterministic dq reduction
// D = 128: the accumulator is [b][h][d][Sq_pad] (the main kernel adds dQ^T
// blocks into it). One block of 256 threads per (b, h, 32 queries): the 128 x
// 32 floats are read along the query axis into shared memory and written out
// as dq rows of 128 head-dim values.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_t(const BwdArgs a) {
  constexpr int D = 128;
  __shared__ float tile[D][33];  // +1 column: the write-out reads hit different banks
  const int bh = blockIdx.y;
  const int h = bh % a.H;
  const int b = bh / a.H;
  const int i0 = blockIdx.x * 32;
  if (!checked(b < a.B && i0 < a.Sq, 205)) return;
  {
    const int d = threadIdx.x >> 1, half = threadIdx.x & 1;
    const float4* src = reinterpret_cast<const float4*>(a.dq_acc + (static_cast<int64_t>(bh) * D + d) * a.Sq_pad + i0 +
                                                        16 * half);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 x = src[u];
      tile[d][16 * half + 4 * u] = x.x;
      tile[d][16 * half + 4 * u + 1] = x.y;
      tile[d][16 * half + 4 * u + 2] = x.z;
      tile[d][16 * half + 4 * u + 3] = x.w;
    }
  }
  __syncthreads();
  const float s = a.scale;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int task = threadIdx.x + 256 * r;
    const int ii = task >> 4, dc = task & 15;  // query row of the tile, 8-column group
    const int i = i0 + ii;
    if (i >= a.Sq || dc * 8 >= a.d) continue;
    uint4 out;
    out.x = sm100::pack2<BF16>(tile[8 * dc][ii] * s, tile[8 * dc + 1][ii] * s);
    out.y = sm100::pack2<BF16>(tile[8 * dc + 2][ii] * s, tile[8 * dc + 3][ii] * s);
    out.z = sm100::pack2<BF16>(tile[8 * dc + 4][ii] * s, tile[8 * dc + 5][ii] * s);
    out.w = sm100::pack2<BF16>(tile[8 * dc + 6][ii] * s, tile[8 * dc + 7][ii] * s);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.dq) + b * a.dq_sb + static_cast<int64_t>(i) * a.dq_ss +
                              h * a.dq_sh + dc * 8) = out;
  }
}

// dq = scale * sum over key blocks, in increasing key-block order, of the
// dQ blocks the main kernel stored in their (query block, key block) slots.
// A key block contributes to query block qb iff qb >= bwd_first_qblock(kvb),
// which is where the main kernel starts its query loop. One group of 8
// columns per thread, as fa_bwd_dq.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_sum(const BwdArgs a) {
  constexpr int G = D / 8;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gid / G;  // (b, h, i) with i < Sq
  const int part = static_cast<int>(gid % G);
  if (row >= static_cast<int64_t>(a.B) * a.H * a.Sq || part * 8 >= a.d) return;
  const int i = static_cast<int>(row % a.Sq);
  const int bh = static_cast<int>(row / a.Sq);
  const int h = bh % a.H;
  const int b = bh / a.H;
  const int qb = i / 128;
  if (!checked(b < a.B && qb < a.nqb && part * 8 + 8 <= D, 207)) return;
  const float* slot = a.dq_part + (static_cast<int64_t>(bh) * a.nqb + qb) * a.nkb * (128 * D) +
                      (i % 128) * D + part * 8;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int kvb = 0; kvb < a.nkb; ++kvb) {
    if (qb < bwd_first_qblock(kvb, a.Sq, a.Sk, a.causal)) break;  // later key blocks start later still
    const float4* src = reinterpret_cast<const float4*>(slot + static_cast<int64_t>(kvb) * (128 * D));
    const float4 x = src[0], y = src[1];
    acc[0] += x.x, acc[1] += x.y, acc[2] += x.z, acc[3] += x.w;
    acc[4] += y.x, acc[5] += y.y, acc[6] += y.z, acc[7] += y.w;
  }
  const float s = a.scale;
  uint4 out;
  out.x = sm100::pack2<BF16>(acc[0] * s, acc[1] * s);
  out.y = sm100::pack2<BF16>(acc[2] * s, acc[3] * s);
  out.z = sm100::pack2<BF16>(acc[4] * s, acc[5] * s);
  out.w = sm100::pack2<BF16>(acc[6] * s, acc[7] * s);
  *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.dq) + b * a.dq_sb + static_cast<int64_t>(i) * a.dq_ss +
                            h * a.dq_sh + part * 8) = out;
}

// ------------------------------------------------------------- main kernel
template <int D>
struct BwdLayout {
  static constexpr int kThreads = 448;   // 14 warps
  static constexpr int BN = 128;         // keys per CTA
  static constexpr int BM = 128;         // query rows per block
  // Q (with lse2) and dO (with Dvec) travel on separate rings: S^T(i+1)
  // needs Q(i+1) right after dV(i), dP^T(i+1) needs dO(i+1) later in block
  // i, after dO(i) has been released.
  // Q stages: three where shared memory allows (D = 64); D = 128 spends the
  // third stage's 32 KB on the dQ staging buffers below.
  static constexpr int QS = (D == 128) ? 2 : 3;
  static constexpr int OS = 1;           // dO stages
  // D = 128: dQ is computed transposed (TMEM lane = head_dim index), so each
  // warp's reductions into the accumulator cover one contiguous 128-byte line.
  static constexpr bool DQ_T = (D == 128);
  static constexpr int KB = D / 64;      // 64-column blocks per row
  static constexpr int TILE = 128 * D * 2;  // one K, V, Q or dO tile
  static constexpr int BLK = 128 * 128;     // one [128 rows][64 cols] block
  static constexpr int DS_TILE = 128 * 128 * 2;  // dS^T [128 keys][128 queries]
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + QS * TILE;
  static constexpr int OFF_DS = OFF_DO + OS * TILE;
  // dQ staging, from which the TMA adds a dQ block into the accumulator.
  // D = 128: two 16 KB buffers, each 32 query rows x 128 fp32. D = 64: one
  // 8 KB buffer per drain warp (its 32 query rows x 64 fp32).
  static constexpr int DQ_PART = 32 * D * 4;
  static constexpr int OFF_DQS = OFF_DS + DS_TILE;
  static constexpr int OFF_LSE = OFF_DQS + (DQ_T ? 2 * DQ_PART : 4 * DQ_PART);
  static constexpr int OFF_DVEC = OFF_LSE + QS * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + OS * BM * 4;
  // kv_full, q_full[QS], q_empty[QS], o_full[OS], o_empty[OS], sx_full,
  // dp_full, p_ready, ds_ready, ds_free, dq_full, dq_free, mma_done, drain
  static constexpr int NBAR = 1 + 2 * QS + 2 * OS + 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_MAX = 232448;
  // 1024 bytes of slack to align the base when it fits; otherwise the kernel
  // requires (and checks) a 1024-aligned dynamic shared memory base.
  static constexpr int SMEM_ALLOC = (BYTES + 1024 <= SMEM_MAX) ? BYTES + 1024 : BYTES;
  static constexpr int TMEM_COLS = 512;
  // TMEM columns: dK, dV accumulators; X holds S^T, then P^T (16-bit); Y
  // holds dP^T, then dQ.
  static constexpr int COL_DK = 0;
  static constexpr int COL_DV = D;
  static constexpr int COL_X = 2 * D;
  static constexpr int COL_Y = 2 * D + 128;
  // Softmax warpgroup g owns queries [64g, 64g + 64): it packs their P^T into
  // X columns [64g, 64g + 32).
  __host__ __device__ static constexpr int col_p(int kk) { return COL_X + (kk >> 2) * 64 + (kk & 3) * 8; }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(448, 1)
    fa_bwd_main(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
  using L = BwdLayout<D>;
  using namespace sm100;
  constexpr int BM = L::BM, QS = L::QS;
  static_assert(L::COL_Y + 128 <= L::TMEM_COLS, "TMEM budget");
  static_assert(L::BYTES <= L::SMEM_MAX, "smem budget");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024 - (smem_u32(smem_raw) & 1023)) & 1023;
  uint8_t* smem = smem_raw + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (L::BYTES + pad > L::SMEM_ALLOC) {
    // The tiles need a 1024-byte aligned base and there is no room to align it.
    if (threadIdx.x == 0) atomicCAS(&g_status[0], 0, -2);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* o_full = q_empty + QS;
  uint64_t* o_empty = o_full + L::OS;
  uint64_t* sx_full = o_empty + L::OS;
  uint64_t* dp_full = sx_full + 1;
  uint64_t* p_ready = dp_full + 1;
  uint64_t* ds_ready = p_ready + 1;
  uint64_t* ds_free = ds_ready + 1;
  uint64_t* dq_full = ds_free + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* mma_done = dq_free + 1;
  uint64_t* drain = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_dvec = reinterpret_cast<const float*>(smem + L::OFF_DVEC);
  constexpr int kLoaderWarp = 12, kMmaWarp = 13;

  // Causal: key-block-major, the first key blocks (the most query blocks)
  // first. Without a mask every CTA has the same length and the grid is
  // head-major: the CTAs running at one time then share a few heads' Q, dO
  // and dQ accumulator, which stay in L2.
  const int hb_count = a.H * a.B;
  const int kvb = a.causal ? static_cast<int>(blockIdx.x) / hb_count : static_cast<int>(blockIdx.x) % a.nkb;
  const int hb = a.causal ? static_cast<int>(blockIdx.x) % hb_count : static_cast<int>(blockIdx.x) / a.nkb;
  const int h = hb % a.H;
  const int b = hb / a.H;
  const int n0 = kvb * L::BN;
  const int off = a.Sk - a.Sq;
  const int nqb = (a.Sq + BM - 1) / BM;
  const int i_start = bwd_first_qblock(kvb, a.Sq, a.Sk, a.causal);
  const int n = max(0, nqb - i_start);
  const int64_t bh_row0 = static_cast<int64_t>(b * a.H + h) * a.Sq_pad;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < L::OS; ++s) {
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 1);
    }
    mbar_init(sx_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(mma_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kLoaderWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 12) {
    if (warp == kLoaderWarp) {
      // ---------------------------------------------------------------- loader
      if (lane == 0 && n > 0) {
        mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
        // TMA zero-fills tiles past the tensor's end; the check build still
        // records a tile that starts outside it (a scheduling error).
        checked(n0 < a.Sk && b < a.B && h < a.H, 210);
        for (int kb = 0; kb < L::KB; ++kb) {
          tma_load_4d(smem + L::OFF_K + kb * L::BLK, &tmK, kv_full, kb * 64, n0, h, b);
          tma_load_4d(smem + L::OFF_V + kb * L::BLK, &tmV, kv_full, kb * 64, n0, h, b);
        }
        // Q(j) with lse2(j) runs QS - 1 blocks ahead, dO(j) with Dvec(j)
        // OS - 1 blocks ahead: per step i, dO(i + OS - 1) (at OS = 1 its slot
        // frees first) and then Q(i + QS - 1).
        int nq = 0, no = 0;  // loads issued
        auto load_q = [&](int j) -> bool {
          const int st = j % QS;
          if (!wait_bar(&q_empty[st], ((j / QS) & 1) ^ 1, abort_flag, kRoleLoader, j)) return false;
          const int j0 = (i_start + j) * BM;
          checked(j0 < a.Sq, 211);
          mbar_arrive_expect_tx(&q_full[st], L::TILE + BM * 4);
          for (int kb = 0; kb < L::KB; ++kb)
            tma_load_4d(smem + L::OFF_Q + st * L::TILE + kb * L::BLK, &tmQ, &q_full[st], kb * 64, j0, h, b);
          // Skipped on a failed check: its wait then runs out (FA_ERR_BOUNDS stays recorded).
          if (checked(bh_row0 + j0 + BM <= static_cast<int64_t>(a.B) * a.H * a.Sq_pad, 212))
            bulk_load(smem + L::OFF_LSE + st * BM * 4, a.lse2 + bh_row0 + j0, BM * 4, &q_full[st]);
          ++nq;
          return true;
        };
        auto load_o = [&](int j) -> bool {
          const int st = j % L::OS;
          if (!wait_bar(&o_empty[st], ((j / L::OS) & 1) ^ 1, abort_flag, kRoleLoader, j)) return false;
          const int j0 = (i_start + j) * BM;
          checked(j0 < a.Sq, 211);
          mbar_arrive_expect_tx(&o_full[st], L::TILE + BM * 4);
          for (int kb = 0; kb < L::KB; ++kb)
            tma_load_4d(smem + L::OFF_DO + st * L::TILE + kb * L::BLK, &tmdO, &o_full[st], kb * 64, j0, h, b);
          if (checked(bh_row0 + j0 + BM <= static_cast<int64_t>(a.B) * a.H * a.Sq_pad, 212))
            bulk_load(smem + L::OFF_DVEC + st * BM * 4, a.dvec + bh_row0 + j0, BM * 4, &o_full[st]);
          ++no;
          return true;
        };
        bool lok = true;
        for (int j = 0; lok && j < QS - 1 && j < n; ++j) lok = load_q(j);
        for (int j = 0; lok && j < L::OS - 1 && j < n; ++j) lok = load_o(j);
        for (int i = 0; lok && i < n; ++i) {
          if (i + L::OS - 1 < n) lok = load_o(i + L::OS - 1);
          if (lok && i + QS - 1 < n) lok = load_q(i + QS - 1);
        }
        if (*abort_flag) {
          drain_wait(kv_full, 0);
          for (int j = max(0, nq - QS); j < nq; ++j) drain_wait(&q_full[j % QS], (j / QS) & 1);
          for (int j = max(0, no - L::OS); j < no; ++j) drain_wait(&o_full[j % L::OS], (j / L::OS) & 1);
        }
      }
    } else if (warp == kMmaWarp) {
      // ----------------------------------------------------------- MMA issuer
      // The whole warp runs this loop converged; elect.sync picks the lane
      // that issues each MMA and commit, and every wait is voted warp-wide.
      if (n > 0) {
        auto wait = [&](uint64_t* bar, uint32_t parity, int iter) {
          return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, kRoleMma, iter));
        };
        const uint32_t sK = smem_u32(smem + L::OFF_K);
        const uint32_t sV = smem_u32(smem + L::OFF_V);
        const uint32_t sQ = smem_u32(smem + L::OFF_Q);
        const uint32_t sdO = smem_u32(smem + L::OFF_DO);
        const uint32_t sDS = smem_u32(smem + L::OFF_DS);
        // S^T = K Q^T, dP^T = V dO^T: M = 128 keys, N = 128 queries, K = D (both K-major).
        const uint32_t id_s = idesc_f16(BF16, 128, 128, 0, 0);
        // dV += P^T dO, dK += dS^T Q: M = 128 keys, N = D, K = 128 queries; A in TMEM, B MN-major.
        const uint32_t id_kv = idesc_f16(BF16, 128, D, 0, 1);
        // D = 128: dQ^T = K^T dS^T, M = head_dim, N = 128 queries, K = 128 keys; A = K viewed
        // MN-major, B = dS^T MN-major. D = 64: dQ = dS K, M = 128 queries, N = D; A = dS^T
        // viewed MN-major, B = K MN-major.
        const uint32_t id_q = L::DQ_T ? idesc_f16(BF16, 128, 128, 1, 1) : idesc_f16(BF16, 128, D, 1, 1);
        // Operand descriptors are formed once per tile and advanced by adds.
        auto issue_kt = [&](uint32_t dcol, uint32_t kv, uint32_t qa) {  // dcol = kv-tile x qa-tile^T
          const uint64_t a0 = desc_sw128(kv, 16, 1024), b0 = desc_sw128(qa, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk >> 2) * L::BLK + (kk & 3) * 32;
            mma_ss_w(tmem + dcol, desc_add(a0, o), desc_add(b0, o), id_s, kk > 0);
          }
        };
        const uint64_t ds_k = desc_sw128(sDS, 16, 1024);         // dS^T, K-major (A of dK)
        const uint64_t ds_mn = desc_sw128(sDS, L::BLK, 1024);    // dS^T, MN-major (dQ)
        const uint64_t k_mn = desc_sw128(sK, L::BLK, 1024);      // K, MN-major (dQ)
        bool ok = wait(kv_full, 0, -1) && wait(&q_full[0], 0, 0);
        if (ok) {
          tc_fence_after();
          issue_kt(L::COL_X, sK, sQ);
          mma_commit_w(sx_full);
          ok = wait(&o_full[0], 0, 0);
        }
        if (ok) {
          tc_fence_after();
          issue_kt(L::COL_Y, sV, sdO);
          mma_commit_w(dp_full);
        }
        for (int i = 0; ok && i < n; ++i) {
          const int st = i % QS;
          const uint32_t ph = i & 1;
          const int ost = i % L::OS;
          const uint32_t qa = sQ + st * L::TILE;
          const uint64_t q_mn = desc_sw128(qa, L::BLK, 1024);
          const uint64_t do_mn = desc_sw128(sdO + ost * L::TILE, L::BLK, 1024);
          if (!(ok = wait(p_ready, ph, i))) break;
          tc_fence_after();
          // dV += P^T dO
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts_w(tmem + L::COL_DV, tmem + L::col_p(kk), desc_add(do_mn, kk * 2048), id_kv,
                   (i > 0 || kk > 0) ? 1u : 0u);
          if (i + 1 < n) {
            // S^T(i+1) into X as soon as dV(i) has been issued: X held only
            // P^T(i), which dV(i) reads first (the tensor pipe runs in issue
            // order). The softmax of block i+1 then overlaps dK(i) and dQ(i).
            const int sn = (i + 1) % QS;
            if (!(ok = wait(&q_full[sn], ((i + 1) / QS) & 1, i + 1))) break;
            tc_fence_after();
            issue_kt(L::COL_X, sK, sQ + sn * L::TILE);
            mma_commit_w(sx_full);
          }
          if (!(ok = wait(ds_ready, ph, i))) break;
          tc_fence_after();
          // dO(i) and Dvec(i) are free once dV(i) is done (the softmax warps
          // have read Dvec(i): ds_ready).
          mma_commit_w(&o_empty[ost]);
          // dQ (or dQ^T) into Y first, so that its drain overlaps dK(i): dP^T(i)
          // there has been read by the softmax warps.
#pragma unroll
          for (int kk = 0; kk < L::BN / 16; ++kk) {
            const uint64_t dk_desc = desc_add(ds_mn, kk * 2048);
            const uint64_t k_desc = desc_add(k_mn, kk * 2048);
            if constexpr (L::DQ_T)
              mma_ss_w(tmem + L::COL_Y, k_desc, dk_desc, id_q, kk > 0);
            else
              mma_ss_w(tmem + L::COL_Y, dk_desc, k_desc, id_q, kk > 0);
          }
          mma_commit_w(dq_full);
          // dK += dS^T Q, dS^T from shared memory (K-major: 128 keys x 128 queries)
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk) {
            const uint32_t o = (kk >> 2) * L::BLK + (kk & 3) * 32;
            mma_ss_w(tmem + L::COL_DK, desc_add(ds_k, o), desc_add(q_mn, kk * 2048), id_kv,
                   (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_w(&q_empty[st]);
          mma_commit_w(ds_free);
          if (i + 1 < n) {
            // dP^T(i+1) into Y once dQ(i) has been read out of it.
            const int on = (i + 1) % L::OS;
            if (!(ok = wait(dq_free, ph, i))) break;
            if (!(ok = wait(&o_full[on], ((i + 1) / L::OS) & 1, i + 1))) break;
            tc_fence_after();
            issue_kt(L::COL_Y, sV, sdO + on * L::TILE);
            mma_commit_w(dp_full);
          }
        }
        mma_commit_w(mma_done);
        mma_commit_w(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp < 8) {
    // --------------- P^T and dS^T: one key row per thread, 64 query columns per warpgroup
    const int g = warp >> 2;
    const int kr = (warp & 3) * 32 + lane;
    const int key = n0 + kr;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tX = tmem + lane_base + L::COL_X + 64 * g;
    const uint32_t tY = tmem + lane_base + L::COL_Y + 64 * g;
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int st = i % QS;
      const uint32_t ph = i & 1;
      ok = __all_sync(0xffffffffu, wait_bar(sx_full, ph, abort_flag, kRoleSoftmax, i) &&
                                       wait_bar(&q_full[st], (i / QS) & 1, abort_flag, kRoleSoftmax, i));
      if (!ok) break;
      tc_fence_after();
      const int i0 = (i_start + i) * BM;
      // query columns c < cmin are masked for this key (causal); all of them if key >= Sk
      int cmin = a.causal ? key - off - i0 : -1;
      if (key >= a.Sk) cmin = BM;
      const float* lse_s = s_lse + st * BM + 64 * g;
      const float* dvec_s = s_dvec + (i % L::OS) * BM + 64 * g;
      const int cm = cmin - 64 * g;  // in this warpgroup's column numbering
      // Phase A: P^T = 2^(S^T scale log2e - lse2) -> 16-bit pairs into X.
      uint32_t pp[2][16];
      {
        uint32_t sv[2][32];
        tmem_ld32(tX, sv[0]);
        tmem_ld32(tX + 32, sv[1]);
        tmem_ld_wait();
        reg_fence(sv[0]);
        reg_fence(sv[1]);
        // Blocks with a masked entry in this warp (causal diagonal, key tail,
        // query rows with no key) take the MUFU exp2 everywhere, so that masked
        // entries give exact zeros. Other blocks send one pair in four through
        // the polynomial exp2 on the FMA pipe.
        auto block = [&](auto masked) {
          const uint64_t sl2x2 = f2(sl2, sl2);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float4 lv[8];  // lse2 of these 32 queries
#pragma unroll
            for (int u = 0; u < 8; ++u) lv[u] = reinterpret_cast<const float4*>(lse_s + 32 * c)[u];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int q = 32 * c + e;
              const float4 L4 = lv[e >> 2];
              float s0 = __uint_as_float(sv[c][e]), s1 = __uint_as_float(sv[c][e + 1]);
              const float l0 = (e & 2) ? L4.z : L4.x, l1 = (e & 2) ? L4.w : L4.y;
              if constexpr (decltype(masked)::value) {
                s0 = (q < cm) ? -INFINITY : s0;
                s1 = (q + 1 < cm) ? -INFINITY : s1;
                pp[c][e >> 1] = pack2<BF16>(ex2(fmaf(s0, sl2, -l0)), ex2(fmaf(s1, sl2, -l1)));
              } else {
                const uint64_t t = fma2(f2(s0, s1), sl2x2, f2(-l0, -l1));
                float p0, p1;
                if (((e >> 1) & 3) == 3) {
                  f2_split(exp2_poly2(t), p0, p1);
                } else {
                  f2_split(t, p0, p1);
                  p0 = ex2(p0);
                  p1 = ex2(p1);
                }
                pp[c][e >> 1] = pack2<BF16>(p0, p1);
              }
            }
          }
        };
        if (__any_sync(0xffffffffu, cm > 0))
          block(std::true_type{});
        else
          block(std::false_type{});
      }
      tmem_st16(tX, pp[0]);       // X columns [64g, 64g + 32): read above
      tmem_st16(tX + 16, pp[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready);
      // Phase B: dS^T = P^T (dP^T - Dvec) -> 16-bit pairs into swizzled smem
      // (the A operand of dK, the B operand of dQ^T / A of dQ).
      ok = __all_sync(0xffffffffu, wait_bar(dp_full, ph, abort_flag, kRoleSoftmax, i) &&
                                       wait_bar(ds_free, ph ^ 1, abort_flag, kRoleSoftmax, i) &&
                                       wait_bar(&o_full[i % L::OS], (i / L::OS) & 1, abort_flag, kRoleSoftmax, i));
      if (!ok) break;
      tc_fence_after();
      const uint32_t ds_row = smem_u32(smem + L::OFF_DS + g * L::BLK) + kr * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dpv[32];
        tmem_ld32(tY + 32 * c, dpv);
        float4 dv4[8];  // Dvec of these 32 queries, loaded while the TMEM load is in flight
#pragma unroll
        for (int u = 0; u < 8; ++u) dv4[u] = reinterpret_cast<const float4*>(dvec_s + 32 * c)[u];
        tmem_ld_wait();
        reg_fence(dpv);
        uint32_t dsp[16];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 V4 = dv4[e >> 2];
          const float2 pa = unpack2<BF16>(pp[c][e >> 1]);
          const float2 pb = unpack2<BF16>(pp[c][(e >> 1) + 1]);
          dsp[e >> 1] = pack2<BF16>(pa.x * (__uint_as_float(dpv[e]) - V4.x), pa.y * (__uint_as_float(dpv[e + 1]) - V4.y));
          dsp[(e >> 1) + 1] =
              pack2<BF16>(pb.x * (__uint_as_float(dpv[e + 2]) - V4.z), pb.y * (__uint_as_float(dpv[e + 3]) - V4.w));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int chunk = 4 * c + u;
          st_shared_v4(ds_row + ((chunk ^ (kr & 7)) << 4), dsp[4 * u], dsp[4 * u + 1], dsp[4 * u + 2],
                       dsp[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_ready);
    }
    // epilogue: warpgroup 0 writes dK = scale * accumulator, warpgroup 1 writes dV
    const bool have = n > 0;
    if (ok && !*abort_flag) {
      bool done = !have || __all_sync(0xffffffffu, wait_bar(mma_done, 0, abort_flag, kRoleSoftmax, n));
      if (done) {
        tc_fence_after();
        const float mul = g == 0 ? a.scale : 1.f;
        uint16_t* dst = g == 0 ? reinterpret_cast<uint16_t*>(a.dk) + b * a.dk_sb +
                                     static_cast<int64_t>(key) * a.dk_ss + h * a.dk_sh
                               : reinterpret_cast<uint16_t*>(a.dv) + b * a.dv_sb +
                                     static_cast<int64_t>(key) * a.dv_ss + h * a.dv_sh;
        const int col = g == 0 ? L::COL_DK : L::COL_DV;
#pragma unroll 1
        for (int c = 0; c < (a.d + 31) / 32; ++c) {
          uint32_t v[32];
          if (have) {
            tmem_ld32(tmem + lane_base + col + 32 * c, v);
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
                w[e] = pack2<BF16>(__uint_as_float(v[8 * u + 2 * e]) * mul,
                                   __uint_as_float(v[8 * u + 2 * e + 1]) * mul);
              if (32 * c + 8 * u < a.d && checked(b < a.B && h < a.H, 217)) d4[u] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------- dQ drain (warps 8-11)
    const int tr = (warp & 3) * 32 + lane;  // TMEM lane
    const uint32_t tY = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + L::COL_Y;
    // DET: store the block into its own slot (deterministic mode) instead of
    // adding it into the shared accumulator.
    auto drain = [&](auto det) {
      constexpr bool DET = decltype(det)::value;
      bool in_range = true;  // set per block below
      auto put = [&](float* p, float x) {
        if (!in_range) return;
        if constexpr (DET)
          *p = x;
        else
          red_add_f32(p, x);
      };
      for (int i = 0; i < n; ++i) {
        const bool ok = __all_sync(0xffffffffu, wait_bar(dq_full, i & 1, abort_flag, kRoleSoftmax, i));
        if (!ok) break;
        tc_fence_after();
        const int qb = i_start + i;
        // block base: row0 of the accumulator, or the (qb, kvb) slot
        // (D = 128 adds through the TMA and tmDQ and does not use `base`.)
        float* base = DET ? a.dq_part + ((static_cast<int64_t>(hb) * a.nqb + qb) * a.nkb + kvb) * (BM * D)
                          : a.dq_acc + (bh_row0 + static_cast<int64_t>(qb) * BM) * D;
        // Every write of this block lands in [base, base + BM * D); the check
        // build skips the block if that range leaves its buffer.
        in_range =
            DET ? checked(hb < a.B * a.H && qb < a.nqb && kvb < a.nkb, 216)
                : checked(bh_row0 + static_cast<int64_t>(qb) * BM + BM <= static_cast<int64_t>(a.B) * a.H * a.Sq_pad, 216);
        if constexpr (L::DQ_T) {
          // lane = head_dim index d, columns = 128 query rows: for each query the
          // warp writes 32 consecutive floats (one 128-byte line). Three quarters
          // of the block are read before any write is issued and the last
          // quarter after the first quarter's writes, so that Y is released
          // (and dP^T(i+1) may start) after 32 of the 128 writes.
          float* col = base + tr;
          uint32_t v[3][32];
#pragma unroll
          for (int part = 0; part < 3; ++part) tmem_ld32(tY + 32 * part, v[part]);
          tmem_ld_wait();
#pragma unroll
          for (int part = 0; part < 3; ++part) reg_fence(v[part]);
          if constexpr (DET) {
#pragma unroll
            for (int c = 0; c < 32; ++c) put(col + c * D, __uint_as_float(v[0][c]));
            tmem_ld32(tY + 96, v[0]);
            tmem_ld_wait();
            reg_fence(v[0]);
            tc_fence_before();
            mbar_arrive(dq_free);  // Y may take dP^T(i+1) now
#pragma unroll
            for (int part = 1; part < 4; ++part)
#pragma unroll
              for (int c = 0; c < 32; ++c)
                put(col + (32 * part + c) * D, __uint_as_float(v[part == 3 ? 0 : part][c]));
          } else {
            // The accumulator is kept transposed at D = 128, [b][h][d][Sq_pad]:
            // this warp's 32 head-dim rows of quarter p (32 queries) are one
            // 32 x 32-float box of it. The warp stages the box in the 128-byte
            // swizzled layout (row d's 16-byte chunk c at d * 128 + ((c ^ (d %
            // 8)) * 16): eight 16-byte stores per thread, no bank conflicts)
            // and has the TMA add it through tmDQ. Each warp owns a quarter of
            // each of the two staging buffers, so the four drain warps do not
            // wait for one another. Y is released after the first quarter is
            // staged and the last one read.
            const int wq = warp & 3;
            auto store = [&](int part, const uint32_t (&x)[32]) {
              uint8_t* buf = smem + L::OFF_DQS + (part & 1) * L::DQ_PART + wq * (32 * 128);
              if (lane == 0) bulk_wait_read1();  // the reduction that read this buffer last
              __syncwarp();
              const uint32_t rbase = smem_u32(buf) + lane * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                st_shared_v4(rbase + ((c ^ (lane & 7)) << 4), x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                const int64_t drow = static_cast<int64_t>(hb) * D + 32 * wq;  // (b, h, d) row of the accumulator
                if (checked(qb * BM + 32 * part + 32 <= a.Sq_pad && drow + 32 <= static_cast<int64_t>(a.B) * a.H * D,
                            214))
                  tma_reduce_add_2d(&tmDQ, buf, qb * BM + 32 * part, static_cast<int>(drow));
                bulk_commit();
              }
            };
            store(0, v[0]);
            tmem_ld32(tY + 96, v[0]);
            tmem_ld_wait();
            reg_fence(v[0]);
            tc_fence_before();
            mbar_arrive(dq_free);  // Y may take dP^T(i+1) now
            store(1, v[1]);
            store(2, v[2]);
            store(3, v[0]);
          }
        } else {
          // lane = query row, columns = head_dim (64): the whole block fits in
          // registers, so Y is released before the writes.
          float* row = base + tr * D;
          uint32_t v[D / 32][32];
#pragma unroll
          for (int part = 0; part < D / 32; ++part) tmem_ld32(tY + 32 * part, v[part]);
          tmem_ld_wait();
#pragma unroll
          for (int part = 0; part < D / 32; ++part) reg_fence(v[part]);
          tc_fence_before();
          mbar_arrive(dq_free);
          if constexpr (DET) {
#pragma unroll
            for (int part = 0; part < D / 32; ++part)
#pragma unroll
              for (int c = 0; c < 32; c += 4)
                if (in_range)
                  *reinterpret_cast<float4*>(row + 32 * part + c) =
                      make_float4(__uint_as_float(v[part][c]), __uint_as_float(v[part][c + 1]),
                                  __uint_as_float(v[part][c + 2]), __uint_as_float(v[part][c + 3]));
          } else {
            // This warp's 32 rows are contiguous in the accumulator. They are
            // staged as two boxes of 32 rows x 32 floats (columns 0-31 and
            // 32-63) in the 128-byte swizzled layout: row r's 16-byte chunk c
            // sits at r * 128 + ((c ^ (r % 8)) * 16), so the eight lanes of
            // each store phase hit eight different bank groups (rows of 256
            // plain bytes would put all 32 lanes on the same banks). The TMA
            // reads the swizzle through tmDQ and adds each box into the
            // accumulator.
            const int wq = warp & 3;
            uint8_t* wbuf = smem + L::OFF_DQS + wq * L::DQ_PART;
            if (lane == 0) bulk_wait_read0();  // this warp's previous reduction has read the buffer
            __syncwarp();
            const uint32_t rbase = smem_u32(wbuf) + lane * 128;
#pragma unroll
            for (int part = 0; part < D / 32; ++part)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                st_shared_v4(rbase + part * (32 * 128) + ((c ^ (lane & 7)) << 4), v[part][4 * c],
                             v[part][4 * c + 1], v[part][4 * c + 2], v[part][4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const int row0 = static_cast<int>(bh_row0 + static_cast<int64_t>(qb) * BM) + 32 * wq;
#pragma unroll
              if (checked(row0 + 32 <= static_cast<int64_t>(a.B) * a.H * a.Sq_pad, 215))
                for (int part = 0; part < D / 32; ++part)
                  tma_reduce_add_2d(&tmDQ, wbuf + part * (32 * 128), 32 * part, row0);
              bulk_commit();
            }
          }
        }
      }
    };
    if (a.dq_part != nullptr) {
      drain(std::true_type{});
    } else {
      drain(std::false_type{});
      // Let the TMA finish the last reductions before shared memory goes away
      // (lane 0 of each drain warp issued its own).
      if (lane == 0) bulk_wait0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
