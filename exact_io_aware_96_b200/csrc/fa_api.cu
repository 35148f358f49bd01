// fa_api.cu — the C ABI declared in include/fa.h: argument checks, TMA tensor
// maps, launch configuration. No allocation per call; no host synchronisation
// except in fa_last_device_status().
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <vector>

#include "fa.h"
#include "fa_fwd.cuh"
#include "fa_fwd_e4m3.cuh"
#include "fa_bwd.cuh"

namespace {

constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks shared by every tensor view of a call.
int check_view(const fa_tensor& t, bool allow_null = false) {
  if (t.ptr == nullptr) return allow_null ? FA_OK : FA_ERR_INVALID_ARG;
  if (t.stride_b < 0 || t.stride_s < 0 || t.stride_h < 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return FA_ERR_MISALIGNED;
  if ((t.stride_b % 8) || (t.stride_s % 8) || (t.stride_h % 8)) return FA_ERR_MISALIGNED;
  return FA_OK;
}

int check_common(int B, int H, int Sq, int Sk, int D, float scale, int causal, int dtype) {
  if (B < 1 || H < 1 || Sq < 1 || Sk < 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (D < 8 || D > 128 || D % 8) return FA_ERR_UNSUPPORTED;
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (int64_t(B) * H * Sq > lim || int64_t(B) * H * Sk > lim) return FA_ERR_INVALID_ARG;
  if (int64_t(B) * H * ((Sq + 255) / 256) > lim) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_tensor dense(const void* p, int S, int H, int D) {
  fa_tensor t;
  t.ptr = const_cast<void*>(p);
  t.stride_h = D;
  t.stride_s = int64_t(H) * D;
  t.stride_b = int64_t(S) * H * D;
  return t;
}

// 4-D tiled map over a [B, S, H, D] view: dims (D, S, H, B), box (128 bytes of
// columns, rows, 1, 1), 128-byte swizzle, out-of-range rows and columns read
// as zeros. `dtype` is FA_FP16, FA_BF16 or kE4M3 (one byte per element).
constexpr int kE4M3 = 100;
int make_map(CUtensorMap* map, const fa_tensor& t, int B, int S, int H, int D, int dtype, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const int esz = dtype == kE4M3 ? 1 : 2;
  const CUtensorMapDataType dt = dtype == kE4M3   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(S), cuuint64_t(H), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(t.stride_s) * esz, cuuint64_t(t.stride_h) * esz, cuuint64_t(t.stride_b) * esz};
  // A stride the driver rejects (0 for an extent-1 axis) is replaced by a
  // harmless positive one: with extent 1 it is never stepped over.
  if (S == 1 && strides[0] == 0) strides[0] = 16;
  if (H == 1 && strides[1] == 0) strides[1] = 16;
  if (B == 1 && strides[2] == 0) strides[2] = 16;
  cuuint32_t box[4] = {cuuint32_t(128 / esz), cuuint32_t(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dt, 4, t.ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// 2-D map over the fp32 dQ accumulator, [rows][cols] with cols innermost,
// boxes of 32 rows x 32 floats (128 bytes) in the 128-byte swizzled
// shared-memory layout: the backward stages dQ blocks that way and has the TMA
// add them. D = 64: [B*H*Sq_pad][64]. D = 128: the accumulator is transposed,
// [B*H*128][Sq_pad].
int make_dq_map(CUtensorMap* map, float* acc, int64_t rows, int64_t cols) {
  auto fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * sizeof(float)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, acc, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Raises the dynamic shared memory limit of `fn` once per device, and asks
// for the largest shared-memory carveout. Every kernel of the library asks
// for the same carveout, so consecutive launches (forward, backward
// preprocess, main, dQ convert) never make the SM reconfigure its L1/shared
// split between them.
template <typename F>
int prepare(F* fn, int smem_bytes, bool (&done)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (!done[dev]) {
    if (smem_bytes > 0 &&
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
      return FA_ERR_CUDA;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    done[dev] = true;
  }
  return FA_OK;
}

// ------------------------------------------------------- key-range split plan
// Workspace of a split over the first n_split ranks: tickets (one u64 per
// split (b, h, rank)), then (m, l) per row and the fp32 O partial per row of
// every split CTA; sections 256-byte aligned.
struct SplitLayout {
  uint64_t off_ml, off_o, bytes;
};
uint64_t round256(uint64_t x) { return (x + 255) / 256 * 256; }
SplitLayout split_layout(int B, int H, int n_split, int Dk) {
  const uint64_t pairs = uint64_t(B) * H * n_split;
  const uint64_t ctas = 2 * pairs;
  SplitLayout l;
  l.off_ml = round256(pairs * 8);
  l.off_o = l.off_ml + round256(ctas * 256 * 8);
  l.bytes = n_split > 0 ? l.off_o + ctas * 256 * uint64_t(Dk) * 4 : 0;
  return l;
}

int sm_count() {
  static int count[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    count[dev] = n;
  }
  return count[dev];
}

// A split plan: n_split ranks split, and the grid's unit order (see
// FwdArgs::order), longest unit first.
struct SplitPlan {
  int ns = 0;
  int units = 0;
  uint8_t order[2 * fa::FwdArgs::kMaxSplitRanks] = {};
};

// Unit costs in 128 x 128 tile-blocks: a CTA's key blocks over both tiles,
// plus a start-up cost (loading Q, filling the pipeline, the epilogue), plus
// for a split half the exchange through the workspace and the merge. The
// constants are fitted to per-CTA timings of the kernel on B200.
constexpr double kSplitStart = 3.0;
double split_merge_cost(int Dk) { return Dk <= 64 ? 4.0 : 5.0; }

void split_costs(const int* c0, const int* c1, int r, double merge, double* whole, double* h0, double* h1) {
  const int hs = (std::max(c0[r], c1[r]) + 1) / 2;
  *whole = kSplitStart + c0[r] + c1[r];
  *h0 = kSplitStart + merge + std::min(c0[r], hs) + std::min(c1[r], hs);
  *h1 = kSplitStart + merge + std::max(0, c0[r] - hs) + std::max(0, c1[r] - hs);
}

// The order for `ns` split ranks: units sorted by cost, longest first (ties
// in rank, then half order), so that CTAs starting in grid order on
// whichever SM frees first is longest-processing-time-first list scheduling.
SplitPlan split_order(const int* c0, const int* c1, int nq, int ns, double merge) {
  SplitPlan p;
  p.ns = ns;
  std::vector<std::pair<double, int>> u;
  for (int r = 0; r < nq; ++r) {
    double w, a, b;
    split_costs(c0, c1, r, merge, &w, &a, &b);
    if (r < ns) {
      u.push_back({a, r * 3 + 1});
      u.push_back({b, r * 3 + 2});
    } else {
      u.push_back({w, r * 3});
    }
  }
  std::stable_sort(u.begin(), u.end(), [](const std::pair<double, int>& x, const std::pair<double, int>& y) {
    return x.first > y.first;
  });
  p.units = int(u.size());
  for (size_t i = 0; i < u.size(); ++i) p.order[i] = uint8_t(u[i].second);
  return p;
}

// Finish time of the plan's grid: CTAs start in grid order on whichever SM
// frees first, one CTA per SM.
double split_makespan(const int* c0, const int* c1, const SplitPlan& p, int HB, int sms, double merge) {
  std::vector<double> heap(size_t(sms), 0.0);  // min-heap of SM free times
  std::make_heap(heap.begin(), heap.end(), std::greater<double>());
  for (int i = 0; i < p.units; ++i) {
    const int r = p.order[i] / 3, kind = p.order[i] % 3;
    double w, a, b;
    split_costs(c0, c1, r, merge, &w, &a, &b);
    const double cost = kind == 0 ? w : (kind == 1 ? a : b);
    for (int j = 0; j < HB; ++j) {
      std::pop_heap(heap.begin(), heap.end(), std::greater<double>());
      heap.back() += cost;
      std::push_heap(heap.begin(), heap.end(), std::greater<double>());
    }
  }
  return *std::max_element(heap.begin(), heap.end());
}

// The plan for split_ranks (see fa_fwd_params): -1 none, k > 0 min(k, ranks),
// 0 the estimate's best (kept only if it beats the unsplit grid by more than
// 8%). No split past kMaxSplitRanks ranks. Automatic plans are cached per
// shape.
SplitPlan plan_split(int B, int H, int Sq, int Sk, int Dk, int causal, int split_ranks, int sms) {
  const int nq = (Sq + 255) / 256;
  SplitPlan none;
  if (split_ranks < 0 || nq > fa::FwdArgs::kMaxSplitRanks) return none;
  std::vector<int> c0(static_cast<size_t>(nq)), c1(static_cast<size_t>(nq));
  for (int r = 0; r < nq; ++r) {
    const int qb = causal ? nq - 1 - r : r;
    c0[size_t(r)] = fa::fwd_kv_blocks(qb * 256, Sq, Sk, causal);
    c1[size_t(r)] = fa::fwd_kv_blocks(qb * 256 + 128, Sq, Sk, causal);
  }
  const double merge = split_merge_cost(Dk);
  if (split_ranks > 0) return split_order(c0.data(), c1.data(), nq, std::min(split_ranks, nq), merge);
  const int64_t HB = int64_t(B) * H;
  if (sms <= 0 || HB * nq >= 4 * int64_t(sms)) return none;
  struct Entry {
    int B, H, Sq, Sk, Dk, causal, sms;
    SplitPlan plan;
  };
  static Entry cache[32];
  static int cache_n = 0, cache_next = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < cache_n; ++i) {
      const Entry& e = cache[i];
      if (e.B == B && e.H == H && e.Sq == Sq && e.Sk == Sk && e.Dk == Dk && e.causal == causal && e.sms == sms)
        return e.plan;
    }
  }
  SplitPlan best = split_order(c0.data(), c1.data(), nq, 0, merge);
  const double base = split_makespan(c0.data(), c1.data(), best, int(HB), sms, merge);
  double best_t = base;
  for (int ns = 1; ns <= nq; ++ns) {
    const SplitPlan p = split_order(c0.data(), c1.data(), nq, ns, merge);
    const double t = split_makespan(c0.data(), c1.data(), p, int(HB), sms, merge);
    if (t < best_t) {
      best_t = t;
      best = p;
    }
  }
  if (best_t > 0.92 * base) best = none;
  std::lock_guard<std::mutex> g(mu);
  cache[cache_next] = Entry{B, H, Sq, Sk, Dk, causal, sms, best};
  cache_next = (cache_next + 1) % 32;
  cache_n = std::min(cache_n + 1, 32);
  return best;
}

// Distinct for every launch of the split forward (the tickets compare it).
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> epoch{
      (uint64_t(std::chrono::steady_clock::now().time_since_epoch().count()) * 0x9E3779B97F4A7C15ull) | 1ull};
  return epoch.fetch_add(2);
}

template <int D, bool BF16>
int launch_fwd(const fa_fwd_params* p, cudaStream_t stream) {
  using L = fa::FwdLayout<D>;
  static bool done[kMaxDevices] = {};
  auto* kern = &fa::fa_fwd_kernel<D, BF16>;
  int st = prepare(kern, L::SMEM_ALLOC, done);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, p->q, p->B, p->Sq, p->H, p->D, p->dtype, 128)) != FA_OK) return st;
  if ((st = make_map(&mk, p->k, p->B, p->Sk, p->H, p->D, p->dtype, 128)) != FA_OK) return st;
  if ((st = make_map(&mv, p->v, p->B, p->Sk, p->H, p->D, p->dtype, 128)) != FA_OK) return st;
  fa::FwdArgs a{};
  a.o = p->o.ptr;
  a.lse = p->lse;
  a.o_sb = p->o.stride_b;
  a.o_ss = p->o.stride_s;
  a.o_sh = p->o.stride_h;
  a.B = p->B;
  a.H = p->H;
  a.Sq = p->Sq;
  a.Sk = p->Sk;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.o_scale = 1.f;
  a.causal = p->causal;
  a.n_qblocks = (p->Sq + 255) / 256;
  a.d = p->D;
  if (p->workspace != nullptr) {
    const SplitPlan plan = plan_split(p->B, p->H, p->Sq, p->Sk, D, p->causal, p->split_ranks, sm_count());
    const int ns = plan.ns;
    const SplitLayout sl = split_layout(p->B, p->H, ns, D);
    if (ns > 0) {
      if (p->workspace_bytes < sl.bytes) return FA_ERR_WORKSPACE;
      uint8_t* ws = static_cast<uint8_t*>(p->workspace);
      a.n_split = ns;
      std::memcpy(a.order, plan.order, sizeof(a.order));
      a.tickets = reinterpret_cast<unsigned long long*>(ws);
      a.part_ml = reinterpret_cast<float2*>(ws + sl.off_ml);
      a.part_o = reinterpret_cast<float*>(ws + sl.off_o);
      a.epoch = next_epoch();
    }
  }
  const unsigned grid = unsigned(int64_t(a.n_qblocks + a.n_split) * p->B * p->H);
  kern<<<grid, L::kThreads, L::SMEM_ALLOC, stream>>>(mq, mk, mv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// e4m3 inputs: one kernel width (128 bytes = 128 columns) for every head_dim.
template <bool OUT_BF16>
int launch_fwd_fp8(const fa_fwd_fp8_params* p, cudaStream_t stream) {
  using L = fa::FwdE4m3Layout<128, 1>;
  static bool done[kMaxDevices] = {};
  auto* kern = &fa::fa_fwd_e4m3_kernel<128, OUT_BF16>;
  int st = prepare(kern, L::SMEM_ALLOC, done);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map(&mq, p->q, p->B, p->Sq, p->H, p->D, kE4M3, 128)) != FA_OK) return st;
  if ((st = make_map(&mk, p->k, p->B, p->Sk, p->H, p->D, kE4M3, 128)) != FA_OK) return st;
  if ((st = make_map(&mv, p->v, p->B, p->Sk, p->H, p->D, kE4M3, 128)) != FA_OK) return st;
  fa::FwdArgs a{};
  a.o = p->o.ptr;
  a.lse = p->lse;
  a.o_sb = p->o.stride_b;
  a.o_ss = p->o.stride_s;
  a.o_sh = p->o.stride_h;
  a.B = p->B;
  a.H = p->H;
  a.Sq = p->Sq;
  a.Sk = p->Sk;
  // S = (q8 . k8) * q_descale * k_descale; O = (P v8 / l) * v_descale.
  a.scale_log2 = float(double(p->scale) * p->q_descale * p->k_descale * 1.4426950408889634);
  a.o_scale = p->v_descale;
  a.causal = p->causal;
  a.n_qblocks = (p->Sq + 255) / 256;
  a.d = p->D;
  const unsigned grid = unsigned(int64_t(a.n_qblocks) * p->B * p->H);
  kern<<<grid, L::kThreads, L::SMEM_ALLOC, stream>>>(mq, mk, mv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Byte offset of the deterministic-mode dQ slots in the workspace: after the
// fp32 accumulator, Dvec and base-2 LSE, rounded up to 256 bytes.
uint64_t det_part_offset(int B, int H, int Sq, int D) {
  const uint64_t dpad = D <= 64 ? 64 : 128;
  const uint64_t rows = uint64_t(B) * H * ((uint64_t(Sq) + 127) / 128 * 128);
  return (rows * (dpad + 2) * 4 + 255) / 256 * 256;
}

template <int D, bool BF16>
int launch_bwd(const fa_bwd_params* p, cudaStream_t stream) {
  using L = fa::BwdLayout<D>;
  static bool done[kMaxDevices] = {};
  auto* kern = &fa::fa_bwd_main<D, BF16>;
  int st = prepare(kern, L::SMEM_ALLOC, done);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_map(&mq, p->q, p->B, p->Sq, p->H, p->D, p->dtype, L::BM)) != FA_OK) return st;
  if ((st = make_map(&mk, p->k, p->B, p->Sk, p->H, p->D, p->dtype, L::BN)) != FA_OK) return st;
  if ((st = make_map(&mv, p->v, p->B, p->Sk, p->H, p->D, p->dtype, L::BN)) != FA_OK) return st;
  static_assert(L::BM == 128 && L::BN == 128, "tensor maps assume 128-row boxes");
  if ((st = make_map(&mdo, p->dO, p->B, p->Sq, p->H, p->D, p->dtype, L::BM)) != FA_OK) return st;
  fa::BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.o = p->o.ptr;
  a.dO = p->dO.ptr;
  a.lse = p->lse;
  a.dq = p->dq.ptr;
  a.dk = p->dk.ptr;
  a.dv = p->dv.ptr;
  a.Sq_pad = (p->Sq + 127) / 128 * 128;
  const int64_t rows = int64_t(p->B) * p->H * a.Sq_pad;
  a.dq_acc = static_cast<float*>(p->workspace);
  a.dvec = a.dq_acc + rows * D;
  a.lse2 = a.dvec + rows;
  a.nqb = (p->Sq + 127) / 128;
  a.nkb = (p->Sk + 127) / 128;
  a.dq_part = p->deterministic ? reinterpret_cast<float*>(static_cast<char*>(p->workspace) +
                                                          det_part_offset(p->B, p->H, p->Sq, p->D))
                               : nullptr;
  a.o_sb = p->o.stride_b, a.o_ss = p->o.stride_s, a.o_sh = p->o.stride_h;
  a.do_sb = p->dO.stride_b, a.do_ss = p->dO.stride_s, a.do_sh = p->dO.stride_h;
  a.dq_sb = p->dq.stride_b, a.dq_ss = p->dq.stride_s, a.dq_sh = p->dq.stride_h;
  a.dk_sb = p->dk.stride_b, a.dk_ss = p->dk.stride_s, a.dk_sh = p->dk.stride_h;
  a.dv_sb = p->dv.stride_b, a.dv_ss = p->dv.stride_s, a.dv_sh = p->dv.stride_h;
  a.B = p->B;
  a.H = p->H;
  a.Sq = p->Sq;
  a.Sk = p->Sk;
  a.scale = p->scale;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.causal = p->causal;
  a.d = p->D;
  constexpr int G = D / 8;
  {
    static bool done_pre[kMaxDevices] = {}, done_dq[kMaxDevices] = {}, done_sum[kMaxDevices] = {};
    if ((st = prepare(&fa::fa_bwd_pre<D, BF16>, 0, done_pre)) != FA_OK) return st;
    if ((st = prepare(&fa::fa_bwd_dq<D, BF16>, 0, done_dq)) != FA_OK) return st;
    if ((st = prepare(&fa::fa_bwd_dq_sum<D, BF16>, 0, done_sum)) != FA_OK) return st;
    static bool done_t[kMaxDevices] = {};
    if ((st = prepare(&fa::fa_bwd_dq_t<BF16>, 0, done_t)) != FA_OK) return st;
  }
  const int64_t pre_threads = rows * G;
  fa::fa_bwd_pre<D, BF16><<<unsigned((pre_threads + 255) / 256), 256, 0, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = unsigned(int64_t((p->Sk + L::BN - 1) / L::BN) * p->B * p->H);
  CUtensorMap mdq = mq;  // not read in deterministic mode
  if (!p->deterministic) {
    st = D == 64 ? make_dq_map(&mdq, a.dq_acc, rows, 64)
                 : make_dq_map(&mdq, a.dq_acc, int64_t(p->B) * p->H * D, a.Sq_pad);
    if (st != FA_OK) return st;
  }
  kern<<<grid, L::kThreads, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mdo, mdq, a);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const int64_t dq_threads = int64_t(p->B) * p->H * p->Sq * G;
  if (a.dq_part != nullptr)
    fa::fa_bwd_dq_sum<D, BF16><<<unsigned((dq_threads + 255) / 256), 256, 0, stream>>>(a);
  else if (D == 128)
    fa::fa_bwd_dq_t<BF16><<<dim3(unsigned((p->Sq + 31) / 32), unsigned(p->B * p->H)), 256, 0, stream>>>(a);
  else
    fa::fa_bwd_dq<D, BF16><<<unsigned((dq_threads + 255) / 256), 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

// Device scratch of fa_bwd_noalloc: a file-scope array, so the library never
// allocates for it. Host code cannot use the name as an address; its device
// address is looked up once per device (noalloc_scratch) and passed to the
// kernels like a caller's workspace.
constexpr size_t kNoAllocScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device; set up on the
// first call per device (cudaGetSymbolAddress), cached afterwards.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 300; }

const char* fa_strerror(int s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument (null pointer, size < 1, scale or causal flag)";
    case FA_ERR_UNSUPPORTED: return "unsupported dtype or head_dim (fp16/bf16: D a multiple of 8 in [8, 128]; e4m3: a multiple of 16)";
    case FA_ERR_MISALIGNED: return "tensor base or stride not 16-byte aligned";
    case FA_ERR_CUDA: return "CUDA runtime or driver call failed";
    case FA_ERR_TIMEOUT: return "device-side pipeline wait exceeded its time limit";
    case FA_ERR_NOT_IMPLEMENTED: return "not implemented";
    case FA_ERR_WORKSPACE: return "workspace missing or smaller than fa_bwd_workspace_size()";
    case FA_ERR_SCRATCH_LIMIT: return "fa_bwd_noalloc: the problem needs more scratch than FA_NOALLOC_SCRATCH_BYTES (64 MiB)";
    case FA_ERR_BOUNDS: return "a device-side index or bounds check failed (check build); the access was skipped";
    default: return "unknown status";
  }
}

int fa_fwd_ex(const fa_fwd_params* p, fa_stream_t stream) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  int st = check_common(p->B, p->H, p->Sq, p->Sk, p->D, p->scale, p->causal, p->dtype);
  if (st != FA_OK) return st;
  const fa_tensor* views[4] = {&p->q, &p->k, &p->v, &p->o};
  for (const fa_tensor* v : views)
    if ((st = check_view(*v)) != FA_OK) return st;
  if (p->lse == nullptr) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p->lse) & 3u) return FA_ERR_MISALIGNED;
  if (p->workspace != nullptr && (reinterpret_cast<uintptr_t>(p->workspace) & 255u)) return FA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // head_dim <= 64 runs the 64-column kernels, <= 128 the 128-column ones;
  // the tensor maps read the columns past head_dim as zeros.
  if (p->D <= 64) return p->dtype == FA_BF16 ? launch_fwd<64, true>(p, s) : launch_fwd<64, false>(p, s);
  return p->dtype == FA_BF16 ? launch_fwd<128, true>(p, s) : launch_fwd<128, false>(p, s);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk, int D,
           float scale, int causal, int dtype, fa_stream_t stream) {
  fa_fwd_params p;
  std::memset(&p, 0, sizeof(p));
  p.q = dense(q, Sq, H, D);
  p.k = dense(k, Sk, H, D);
  p.v = dense(v, Sk, H, D);
  p.o = dense(o, Sq, H, D);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.D = D;
  p.scale = scale;
  p.causal = causal;
  p.dtype = dtype;
  return fa_fwd_ex(&p, stream);
}

int fa_fwd_fp8_ex(const fa_fwd_fp8_params* p, fa_stream_t stream) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  if (p->o_dtype != FA_FP16 && p->o_dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  int st = check_common(p->B, p->H, p->Sq, p->Sk, p->D, p->scale, p->causal, p->o_dtype);
  if (st != FA_OK) return st;
  if (p->D % 16) return FA_ERR_UNSUPPORTED;
  for (float f : {p->q_descale, p->k_descale, p->v_descale})
    if (!(std::isfinite(f) && f > 0.f)) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(float(double(p->scale) * p->q_descale * p->k_descale * 1.4426950408889634)))
    return FA_ERR_INVALID_ARG;
  const fa_tensor* in[3] = {&p->q, &p->k, &p->v};
  for (const fa_tensor* v : in) {
    if ((st = check_view(*v)) != FA_OK) return st;
    if ((v->stride_b % 16) || (v->stride_s % 16) || (v->stride_h % 16)) return FA_ERR_MISALIGNED;
  }
  if ((st = check_view(p->o)) != FA_OK) return st;
  if (p->lse == nullptr) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p->lse) & 3u) return FA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return p->o_dtype == FA_BF16 ? launch_fwd_fp8<true>(p, s) : launch_fwd_fp8<false>(p, s);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Sq, int Sk, int D,
               float scale, float q_descale, float k_descale, float v_descale, int causal, int o_dtype,
               fa_stream_t stream) {
  fa_fwd_fp8_params p;
  std::memset(&p, 0, sizeof(p));
  p.q = dense(q, Sq, H, D);
  p.k = dense(k, Sk, H, D);
  p.v = dense(v, Sk, H, D);
  p.o = dense(o, Sq, H, D);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.D = D;
  p.scale = scale;
  p.q_descale = q_descale;
  p.k_descale = k_descale;
  p.v_descale = v_descale;
  p.causal = causal;
  p.o_dtype = o_dtype;
  return fa_fwd_fp8_ex(&p, stream);
}

size_t fa_fwd_workspace_size_ex(int B, int H, int Sq, int Sk, int D, int causal, int split_ranks, int* n_split) {
  if (n_split != nullptr) *n_split = 0;
  if (check_common(B, H, Sq, Sk, D, 1.f, causal, FA_BF16) != FA_OK) return 0;
  const int Dk = D <= 64 ? 64 : 128;
  const int ns = plan_split(B, H, Sq, Sk, Dk, causal, split_ranks, sm_count()).ns;
  if (n_split != nullptr) *n_split = ns;
  return size_t(split_layout(B, H, ns, Dk).bytes);
}

int fa_fwd_split_plan(int B, int H, int Sq, int Sk, int D, int causal, int split_ranks, int sms, int* n_split,
                      unsigned char* order, int order_capacity) {
  if (n_split != nullptr) *n_split = 0;
  int st = check_common(B, H, Sq, Sk, D, 1.f, causal, FA_BF16);
  if (st != FA_OK) return st;
  if (sms < 0 || order_capacity < 0 || (order == nullptr && order_capacity > 0)) return FA_ERR_INVALID_ARG;
  if (sms == 0 && (sms = sm_count()) <= 0) return FA_ERR_CUDA;
  const SplitPlan plan = plan_split(B, H, Sq, Sk, D <= 64 ? 64 : 128, causal, split_ranks, sms);
  if (n_split != nullptr) *n_split = plan.ns;
  if (plan.ns == 0) return 0;
  if (order_capacity < plan.units) return FA_ERR_INVALID_ARG;
  std::memcpy(order, plan.order, size_t(plan.units));
  return plan.units;
}

size_t fa_fwd_workspace_size(int B, int H, int Sq, int Sk, int D, int causal) {
  return fa_fwd_workspace_size_ex(B, H, Sq, Sk, D, causal, 0, nullptr);
}

size_t fa_bwd_workspace_size(int B, int H, int Sq, int D) {
  if (B < 1 || H < 1 || Sq < 1 || D < 1) return 0;
  const uint64_t dpad = D <= 64 ? 64 : (D <= 128 ? 128 : uint64_t(D));  // kernel width
  const uint64_t rows = uint64_t(B) * H * ((uint64_t(Sq) + 127) / 128 * 128);
  const uint64_t bytes = rows * (dpad + 2) * 4;  // dq accumulator, Dvec, LSE * log2(e)
  if (bytes > (uint64_t(1) << 50)) return 0;
  return size_t(bytes);
}

size_t fa_bwd_workspace_size_ex(int B, int H, int Sq, int Sk, int D, int deterministic) {
  if (deterministic != 0 && deterministic != 1) return 0;
  if (Sk < 1) return 0;
  const size_t base = fa_bwd_workspace_size(B, H, Sq, D);
  if (base == 0 || !deterministic) return base;
  const uint64_t dpad = D <= 64 ? 64 : 128;
  const uint64_t slots = uint64_t(B) * H * ((uint64_t(Sq) + 127) / 128) * ((uint64_t(Sk) + 127) / 128);
  const uint64_t bytes = det_part_offset(B, H, Sq, D) + slots * 128 * dpad * 4;
  if (bytes > (uint64_t(1) << 50)) return 0;
  return size_t(bytes);
}

int fa_bwd_ex(const fa_bwd_params* p, fa_stream_t stream) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  int st = check_common(p->B, p->H, p->Sq, p->Sk, p->D, p->scale, p->causal, p->dtype);
  if (st != FA_OK) return st;
  const fa_tensor* views[8] = {&p->q, &p->k, &p->v, &p->o, &p->dO, &p->dq, &p->dk, &p->dv};
  for (const fa_tensor* v : views)
    if ((st = check_view(*v)) != FA_OK) return st;
  if (p->lse == nullptr) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p->lse) & 3u) return FA_ERR_MISALIGNED;
  if (p->deterministic != 0 && p->deterministic != 1) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size_ex(p->B, p->H, p->Sq, p->Sk, p->D, p->deterministic);
  if (p->workspace == nullptr || p->workspace_bytes < need || need == 0) return FA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(p->workspace) & 255u) return FA_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->D <= 64) return p->dtype == FA_BF16 ? launch_bwd<64, true>(p, s) : launch_bwd<64, false>(p, s);
  return p->dtype == FA_BF16 ? launch_bwd<128, true>(p, s) : launch_bwd<128, false>(p, s);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
           void* dk, void* dv, int B, int H, int Sq, int Sk, int D, float scale, int causal, int dtype,
           void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  fa_bwd_params p;
  std::memset(&p, 0, sizeof(p));
  p.q = dense(q, Sq, H, D);
  p.k = dense(k, Sk, H, D);
  p.v = dense(v, Sk, H, D);
  p.o = dense(o, Sq, H, D);
  p.dO = dense(dO, Sq, H, D);
  p.lse = lse;
  p.dq = dense(dq, Sq, H, D);
  p.dk = dense(dk, Sk, H, D);
  p.dv = dense(dv, Sk, H, D);
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.D = D;
  p.scale = scale;
  p.causal = causal;
  p.dtype = dtype;
  p.workspace = workspace;
  p.workspace_bytes = workspace_bytes;
  return fa_bwd_ex(&p, stream);
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, int B, int H, int Sq, int Sk, int D, float scale, int causal,
                   int dtype, fa_stream_t stream) {
  fa_bwd_params p;
  std::memset(&p, 0, sizeof(p));
  p.q = dense(q, Sq, H, D);
  p.k = dense(k, Sk, H, D);
  p.v = dense(v, Sk, H, D);
  p.o = dense(o, Sq, H, D);
  p.dO = dense(dO, Sq, H, D);
  p.lse = lse;
  p.dq = dense(dq, Sq, H, D);
  p.dk = dense(dk, Sk, H, D);
  p.dv = dense(dv, Sk, H, D);
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.D = D;
  p.scale = scale;
  p.causal = causal;
  p.dtype = dtype;
  // Every argument check comes before the first CUDA call.
  int st = check_common(B, H, Sq, Sk, D, scale, causal, dtype);
  if (st != FA_OK) return st;
  const fa_tensor* views[8] = {&p.q, &p.k, &p.v, &p.o, &p.dO, &p.dq, &p.dk, &p.dv};
  for (const fa_tensor* t : views)
    if ((st = check_view(*t)) != FA_OK) return st;
  if (lse == nullptr) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_MISALIGNED;
  const size_t need = fa_bwd_workspace_size(B, H, Sq, D);
  if (need == 0 || need > kNoAllocScratchBytes) return FA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != FA_OK) return st;
  p.workspace = scratch;
  p.workspace_bytes = kNoAllocScratchBytes;
  return fa_bwd_ex(&p, stream);
}

int fa_selftest_wait_timeout(unsigned int limit_us, fa_stream_t stream) {
  if (limit_us < 1 || limit_us > 4000000u) return FA_ERR_INVALID_ARG;
  fa::fa_selftest_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000u);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_last_device_status(int* detail) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(h, fa::g_status, sizeof(h)) != cudaSuccess) return FA_ERR_CUDA;
  const int zero[4] = {0, 0, 0, 0};
  if (cudaMemcpyToSymbol(fa::g_status, zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (detail) std::memcpy(detail, h, sizeof(h));
  return h[0];
}

}  // extern "C"
