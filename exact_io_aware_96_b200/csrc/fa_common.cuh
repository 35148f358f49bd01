// fa_common.cuh — pieces shared by the forward and backward kernels: the
// device status word, bounded pipeline waits, and the kernel argument structs.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fa {

// Status word written by kernels whose pipeline wait ran out:
// [0] code (FA_ERR_TIMEOUT), [1] linear block index, [2] role, [3] loop index.
// One per device (the library is loaded once per process; every device gets
// its own copy of a __device__ variable).
__device__ int g_status[4];

enum Role : int { kRoleLoader = 1, kRoleMma = 2, kRoleSoftmax = 3, kRoleSelfTest = 4, kRoleCheck = 5 };

// The check build (-DFA_CHECK=1, libfa_check.so): checked(ok, site) records a
// failed index or bounds test in the status word (FA_ERR_BOUNDS, role 5, the
// site number in place of the loop index) and returns false, so that the
// caller skips the access. In the normal build it is `true` and the test is
// not compiled. Sites: 1xx 16-bit forward, 2xx backward, 3xx e4m3 forward.
#ifndef FA_CHECK
#define FA_CHECK 0
#endif
__device__ __forceinline__ bool checked(bool ok, int site) {
#if FA_CHECK
  if (!ok && atomicCAS(&g_status[0], 0, -9) == 0) {
    g_status[1] = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    g_status[2] = kRoleCheck;
    g_status[3] = site;
  }
  return ok;
#else
  (void)ok;
  (void)site;
  return true;
#endif
}

// A wait longer than this is treated as a hang: the kernel records it and
// winds down instead of spinning forever. Real waits last microseconds.
constexpr uint64_t kWaitLimitNs = 4000000000ull;

__device__ __forceinline__ void record_timeout(int role, int iter) {
  if (atomicCAS(&g_status[0], 0, -5) == 0) {
    g_status[1] = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    g_status[2] = role;
    g_status[3] = iter;
  }
}

// Wait for phase `parity` of `bar` to complete. Returns false (and raises the
// CTA-wide abort flag) if it has not after kWaitLimitNs, or if another warp of
// the CTA has already aborted.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int role,
                                         int iter, uint64_t limit_ns = kWaitLimitNs) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::globaltimer_ns();
  while (true) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (sm100::globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      record_timeout(role, iter);
      return false;
    }
  }
}

// Bounded wait used only on wind-down paths, to let copies or MMAs already in
// flight land before the CTA exits or releases tensor memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = sm100::globaltimer_ns();
  while (!sm100::mbar_try_wait(bar, parity)) {
    if (sm100::globaltimer_ns() - t0 > 500000000ull) break;
  }
}

// Self-test of the failure path: warp 0 waits on an mbarrier that nothing
// arrives on, with a limit of limit_ns; it records the timeout in the status
// word and raises the block's abort flag. Warp 1 waits on the same barrier
// with the normal limit and leaves as soon as it sees the abort flag, the way
// the other roles of a pipeline wind down.
__global__ void __launch_bounds__(64) fa_selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == 0)
    wait_bar(&bar, 0, &abort_flag, kRoleSelfTest, 0, limit_ns);
  else
    wait_bar(&bar, 0, &abort_flag, kRoleSelfTest, 1);
}

struct FwdArgs {
  void* o;
  float* lse;
  int64_t o_sb, o_ss, o_sh;  // element strides of o
  int B, H, Sq, Sk;
  int d;             // head_dim of the tensors (<= the kernel's padded D; columns past it read as 0)
  float scale_log2;  // scale * log2(e) (times the Q and K descale factors for e4m3 inputs)
  float o_scale;     // factor applied to O with 1/l: 1, or V's descale factor for e4m3 inputs
  int causal;
  int n_qblocks;     // ceil(Sq / 256)
  // Key-range split (fa_fwd_kernel only; 0 elsewhere). The first n_split
  // ranks (the heaviest query blocks when causal) each run as two CTAs, one
  // per half of the key blocks; the two leave unnormalised partial results in
  // the workspace and the second to finish merges them. 0: every CTA covers
  // its whole key range and the grid is rank-major. Otherwise the grid runs
  // the units order[0 .. n_qblocks + n_split) (B * H CTAs each), every entry
  // rank * 3 + kind (kind 0: the whole rank, 1 and 2: its first and second
  // half), longest first.
  static constexpr int kMaxSplitRanks = 64;
  int n_split;
  uint8_t order[2 * kMaxSplitRanks];
  float* part_o;                // fp32 [split CTA][256 rows][D]: unnormalised O
  float2* part_ml;              // [split CTA][256 rows]: (running max m, row sum l), base 2
  unsigned long long* tickets;  // [split pair]: the epoch of the first of its two CTAs to finish
  unsigned long long epoch;     // distinct for every launch
};

// First query block that key block kvb contributes to: with a causal mask,
// the block holding the smallest query row i with kvb * 128 <= i + (Sk - Sq).
__host__ __device__ inline int bwd_first_qblock(int kvb, int Sq, int Sk, int causal) {
  if (!causal) return 0;
  const int qmin = kvb * 128 - (Sk - Sq);
  return qmin <= 0 ? 0 : qmin / 128;
}

struct BwdArgs {
  const void* o;
  const void* dO;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;  // fp32 [B, H, Sq_pad, D]
  float* dvec;    // fp32 [B, H, Sq_pad]: sum_d dO_id O_id
  float* lse2;    // fp32 [B, H, Sq_pad]: LSE * log2(e); +inf where no key or padding
  // Deterministic mode (non-null): fp32 [B*H][nqb][nkb][128][D] slots, one per
  // (query block, key block) pair; each key block stores its dQ block there
  // and fa_bwd_dq_sum adds the slots in key-block order. Null: dQ blocks are
  // added into dq_acc with atomics.
  float* dq_part;
  int nqb, nkb;   // ceil(Sq / 128), ceil(Sk / 128)
  int64_t o_sb, o_ss, o_sh;
  int64_t do_sb, do_ss, do_sh;
  int64_t dq_sb, dq_ss, dq_sh;
  int64_t dk_sb, dk_ss, dk_sh;
  int64_t dv_sb, dv_ss, dv_sh;
  int B, H, Sq, Sk, Sq_pad;
  int d;  // head_dim of the tensors (<= the kernel's padded D)
  float scale;
  float scale_log2;
  int causal;
};

}  // namespace fa
