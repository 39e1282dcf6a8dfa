// Host side of the C ABI declared in include/moe_b200.h: plan, workspace
// layout, TMA descriptors, launch sequence, error and profiling plumbing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "dispatch.cuh"
#include "expert_gemm.cuh"
#include "backward.cuh"
#include "expert_gemm2.cuh"
#include "quant.cuh"
#include "router.cuh"
#include "router_tc.cuh"

using namespace moe;

namespace {

constexpr int kNumKernels = 5;      // router, scan, scatter, expert GEMM, finalize
constexpr int kMaxProfiled = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  size_t err, sched, topk_idx, topk_w, rank, chunk_count, expert_count, expert_offset, block_start, num_padded,
      slot_token, slot_topk, l1_done, l2_done, group_start, pair_start, router_partial, router_counter, h, y_acc,
      x_stage, y_stage, x_q, s_x, h8, act_amax, act_scale, bwd_dg, bwd_du, bwd_aw, bwd_dw, bwd_dl, bwd_wgt,
      zero_row, task_log, bwd_xp, bwd_dyp, total;
};

class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev_);
    if (prev_ != dev) cudaSetDevice(dev);
    dev_ = dev;
  }
  ~DeviceGuard() {
    if (prev_ != dev_) cudaSetDevice(prev_);
  }

 private:
  int prev_ = 0, dev_ = 0;
};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 tensor map: `inner` contiguous elements per row, `rows` rows,
// row pitch `pitch_elems`, box {64, box_rows}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_elems,
              uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D FP8 (byte) tensor map of K-major codes: `inner` bytes per row, `rows`
// rows, box {128, 64} (one 128-byte swizzle row per box row), 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, 64};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Entry points that launch kernels first drop whatever error an earlier runtime
// call on this thread left pending (cudaGetLastError returns and clears it), so
// that the cudaGetLastError() after each launch below reports that launch only.
// A sticky error (a lost context) is not cleared by this and still fails the
// launches that follow.
void drop_stale_error() { (void)cudaGetLastError(); }

int block_m_rule(int T, int k, int E) {
  // n = T*k/E compared against 16, 32, 64 without rounding
  const long long tk = (long long)T * k;
  if (tk <= 16LL * E) return 16;
  if (tk <= 32LL * E) return 32;
  if (tk <= 64LL * E) return 64;
  return 128;
}

}  // namespace

static_assert(sizeof(moe_task_record) == sizeof(TaskRecord), "the public task record is the kernels' record");

struct moe_plan {
  int T_max, H, I, E, k, BM, device, num_sms;
  int S = 0;                                           // shared experts
  int BN2, N1, N2, pool, chunks_max, blocks_max;
  int group_min, group_max, max_groups, ring_blocks;   // expert-GEMM task groups and h ring
  bool cta_pairs = false;                              // run the expert GEMM on CTA pairs
  int task_order = -1;                                 // -1 automatic, 0 staggered, 1 interleaved
  bool half_tails = true;                              // pair kernel: lone last blocks as M = 128 pair MMAs
  int wide_l1 = -1;                                    // pair kernel, bf16, I % 256 == 0: 256-column L1 tasks
                                                       // (-1 automatic: when I <= 1024)
  int pair_clusters = 0;                               // co-resident clusters of the pair kernel
  int pgroup_min, pgroup_max, pmax_groups, ring_pairs; // the same in units of block pairs
  int per_expert;                                      // expected blocks per expert + 1
  int fp8_rows = 0;                                    // FP8 plans: activation rows of one block group
  bool backward = false;                               // workspace holds the backward's regions
  bool task_log = false;                               // workspace holds the expert GEMM's task log
  // pipelined host entry: its own copy streams, two staging buffers used in turn, and the events
  // that order each buffer's copy-in, forward and copy-out
  cudaStream_t cp_in = nullptr, cp_out = nullptr;
  cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {}, ev_mark = nullptr;
  int pipe_next = 0;
  bool pipe_used[2] = {false, false};
  Layout L;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  bool profile = false;
  std::vector<cudaEvent_t> ev;   // kMaxProfiled * (kNumKernels + 1)
  int ev_used = 0;
  int withhold = -1;
  uint64_t timeout_ns = 2000000000ull;
};

// CTA-pair mode: a task is a pair of consecutive blocks run by one cluster of
// two CTAs, so there are pair_clusters concurrent tasks (groups and ring in pairs).
// Wide L1 tasks measured 2.5 % faster on the skewed layer (I = 768: short first-GEMM tasks, whose
// per-task costs halve) and 1.5-3 % slower where I is large (fine-grained, mixtral: the wide
// variant's four 48 KB stages instead of six), so the automatic choice is I <= 1024.
static bool wide_l1_active(const moe_plan& p) {
  const bool want = p.wide_l1 > 0 || (p.wide_l1 < 0 && p.I <= 1024);
  return want && p.I % (2 * kL1TileN) == 0;
}

static void size_pair_groups(moe_plan* p) {
  const int pairs_max = p->blocks_max;   // each pair holds at least one block
  const int clusters = std::max(1, p->pair_clusters > 0 ? p->pair_clusters : p->num_sms / 2);
  // L1 tasks per pair: I/256 with the wide L1 tasks (sized for them also when they are switched
  // off later, which changes only the performance)
  const int n1 = wide_l1_active(*p) ? p->I / (2 * kL1TileN) : p->N1;
  p->pgroup_min = (2 * clusters + n1 - 1) / n1;
  p->pgroup_min = std::max(p->pgroup_min, (pairs_max + kMaxGroups - 3) / (kMaxGroups - 2));
  p->pgroup_max = std::max(2 * p->pgroup_min, (p->per_expert + 1) / 2);
  p->pmax_groups = pairs_max / p->pgroup_min + 2;
  p->ring_pairs = std::min(3 * p->pgroup_max, pairs_max);
}

// order_lag of the expert GEMM's parameters: -1 for the staggered task order;
// for the interleaved one, two waves of concurrent tasks (pairs run
// pair_clusters tasks at once, the single-CTA kernel num_sms), which is the
// head start the last L1 tasks of the previous group get before its L2 tasks
// are handed out.
static int order_lag(const moe_plan& p) {
  const bool inter = p.task_order == 1;   // automatic: staggered (measured 1-2 % faster on every workload)
  if (!inter) return -1;
  return 2 * (p.cta_pairs ? std::max(1, p.pair_clusters) : p.num_sms);
}

static bool backward_permuted(const moe_plan& p) { return p.backward && p.BM >= 64; }

// Records of the task log: every task of a launch (at most every block, or pair, times N1 + N2).
static int task_log_capacity(const moe_plan& p) { return p.blocks_max * (p.N1 + p.N2); }

static Layout make_layout(const moe_plan& p) {
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) {
    o = align_up(o, align);
    const size_t at = o;
    o += bytes;
    return at;
  };
  const size_t tk = (size_t)p.T_max * p.k;
  L.err = take(16 * 4, 256);
  L.zero_row = take((size_t)p.H * 2, 256);   // zeroed when bound, never written: padding slots' A rows
  L.sched = take(16 * 4, 256);
  L.topk_idx = take(tk * 4, 256);
  L.topk_w = take(tk * 4, 256);
  L.rank = take(tk * 4, 256);
  L.chunk_count = take((size_t)p.chunks_max * p.E * 4, 256);
  L.expert_count = take((size_t)p.E * 4, 256);
  L.expert_offset = take((size_t)(p.E + 1) * 4, 256);
  L.block_start = take((size_t)(p.E + p.S + 1) * 4, 256);
  L.num_padded = L.sched + 2 * 4;
  L.slot_token = take((size_t)p.pool * 4, 256);
  L.slot_topk = take((size_t)p.pool * 4, 256);
  L.l1_done = take((size_t)p.blocks_max * 4, 256);
  L.l2_done = take((size_t)p.blocks_max * 4, 256);
  L.group_start = take((size_t)(std::max(p.max_groups, p.pmax_groups) + 1) * 4, 256);
  L.pair_start = take((size_t)(p.E + p.S + 1) * 4, 256);
  // split-H router: per token tile (fewer tiles than SMs) a logits accumulator and an arrival counter
  L.router_partial = take((size_t)p.num_sms * kRouterTokens * 256 * 4, 256);
  L.router_counter = take((size_t)p.num_sms * 4, 256);
  L.h = take((size_t)std::max({p.ring_blocks * p.BM, 2 * p.ring_pairs * p.BM, p.fp8_rows}) * p.I * 2, 1024);
  L.y_acc = take((size_t)p.T_max * p.H * 4, 1024);
  L.x_stage = take(2 * (size_t)p.T_max * p.H * 2, 1024);   // two buffers each (the pipelined entry alternates)
  L.y_stage = take(2 * (size_t)p.T_max * p.H * 2, 1024);
  L.x_q = take((size_t)p.T_max * p.H, 1024);   // FP8 first GEMM: x codes and token scales
  L.s_x = take((size_t)p.T_max * 4, 256);
  // FP8 plans: the activation of every block (or pair) at once, its codes and row amax / scale
  L.h8 = take((size_t)p.fp8_rows * p.I, 1024);
  L.act_amax = take((size_t)p.fp8_rows * 4, 256);
  L.act_scale = take((size_t)p.fp8_rows * 4, 256);
  // backward plans: dg, du and w * activation per slot [pool, I] bf16, dw [T_max, k] fp32, the dense
  // gate-logit gradient [T_max, E rounded up to 64] bf16, Wg transposed [E, H] bf16 (the fp32 dx
  // accumulator is the forward's y accumulator)
  const size_t bp = p.backward ? (size_t)p.pool : 0;
  L.bwd_dg = take(bp * p.I * 2, 1024);
  L.bwd_du = take(bp * p.I * 2, 1024);
  L.bwd_aw = take(bp * p.I * 2, 1024);
  L.bwd_dw = take(p.backward ? (size_t)p.T_max * p.k * 4 : 0, 256);
  L.bwd_dl = take(p.backward ? (size_t)p.T_max * ((p.E + 63) / 64 * 64) * 2 : 0, 1024);
  L.bwd_wgt = take(p.backward ? (size_t)p.E * p.H * 2 : 0, 1024);
  // x and dy rows in slot order [pool, H] bf16 each, when BLOCK_M >= 64 (no 64-slot K block of the
  // weight gradients crosses an expert, so the rows can come by TMA); else the kernels gather them
  const size_t bperm = backward_permuted(p) ? (size_t)p.pool * p.H * 2 : 0;
  L.bwd_xp = take(bperm, 1024);
  L.bwd_dyp = take(bperm, 1024);
  L.task_log = take(p.task_log ? (size_t)task_log_capacity(p) * sizeof(TaskRecord) : 0, 256);
  L.total = align_up(o, 1024);
  return L;
}

// Number of H splits for the router: with fewer 64-token tiles than SMs,
// spread the gate GEMM over about two CTAs per SM (the largest divisor of
// H/64 up to kRouterMaxSplit and that target).
static int router_splits(int T, int H, int num_sms) {
  const int tiles = (T + kRouterTokens - 1) / kRouterTokens;
  if (tiles >= num_sms) return 1;
  const int want = (2 * num_sms + tiles - 1) / tiles;
  const int nk = H / kRouterKChunk;
  int s = 1;
  for (int d = 1; d <= kRouterMaxSplit && d <= nk && d <= want; ++d)
    if (nk % d == 0) s = d;
  return s;
}

template <int EP>
static cudaError_t launch_router(const RouterParams& rp, int T, int splits, cudaStream_t st) {
  const dim3 grid((T + kRouterTokens - 1) / kRouterTokens, splits);
  moe_router_kernel<EP><<<grid, kRouterThreads, RouterSmem<EP>::kBytes, st>>>(rp);
  return cudaGetLastError();
}

template <int EP>
static cudaError_t set_router_smem() {
  return cudaFuncSetAttribute(moe_router_kernel<EP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              RouterSmem<EP>::kBytes);
}

static int expert_pad(int E) {
  int ep = 16;
  while (ep < E) ep *= 2;
  return ep;
}

struct SharedWeights {
  const void* Ws1;   // [S, H, I]
  const void* Ws3;   // [S, H, I]
  const void* Ws2;   // [S, I, H]
};

// FP8 E4M3 expert GEMMs: K-major codes of W1 / W3 [E, I, H] and W2 [E, H, I]
// with their column scales [E, I] and [E, H].
struct Fp8Weights {
  const void* W1q;
  const float* s1;
  const void* W3q;
  const float* s3;
  const void* W2q;
  const float* s2;
};

static int enqueue(moe_plan* p, const void* x, const void* Wg, const float* bias, const void* W1, const void* W3,
                   const void* W2, const SharedWeights& sw, int T, void* y, cudaStream_t st, bool full,
                   const Fp8Weights* f8 = nullptr) {
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  if (T < 0 || T > p->T_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;   // nothing to do; empty tensors may carry null pointers
  if (x == nullptr || Wg == nullptr || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_INVALID_ARG;
  if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 3u)) return MOE_ERR_INVALID_ARG;
  if (f8 != nullptr) {   // the FP8 operands stand in for W1 / W3 / W2
    if (p->fp8_rows == 0) return MOE_ERR_INVALID_ARG;   // the plan's workspace has no FP8 regions
    if (p->S > 0 || f8->s1 == nullptr || f8->s3 == nullptr || f8->s2 == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(f8->s1) || !aligned16(f8->s3) || !aligned16(f8->s2)) return MOE_ERR_INVALID_ARG;
    W1 = f8->W1q;
    W3 = f8->W3q;
    W2 = f8->W2q;
  }
  if (full) {
    if (W1 == nullptr || W3 == nullptr || W2 == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    if (p->S > 0) {
      if (sw.Ws1 == nullptr || sw.Ws3 == nullptr || sw.Ws2 == nullptr) return MOE_ERR_INVALID_ARG;
      if (!aligned16(sw.Ws1) || !aligned16(sw.Ws3) || !aligned16(sw.Ws2)) return MOE_ERR_INVALID_ARG;
    }
  }
  DeviceGuard guard(p->device);
  drop_stale_error();
  uint8_t* ws = p->ws;
  const Layout& L = p->L;
  const bool prof = p->profile && p->ev_used < kMaxProfiled;
  cudaEvent_t* ev = prof ? &p->ev[(size_t)p->ev_used * (kNumKernels + 1)] : nullptr;
  auto mark = [&](int i) {
    if (prof) cudaEventRecord(ev[i], st);
  };
  cudaError_t ce;

  // 1. router (+ per-chunk histogram, + zero the output accumulator)
  RouterParams rp{};
  rp.x = static_cast<const bf16*>(x);
  rp.Wg = static_cast<const bf16*>(Wg);
  rp.bias = bias;
  rp.topk_idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  rp.topk_w = reinterpret_cast<float*>(ws + L.topk_w);
  rp.rank = reinterpret_cast<int32_t*>(ws + L.rank);
  rp.chunk_count = reinterpret_cast<int32_t*>(ws + L.chunk_count);
  rp.y_acc = reinterpret_cast<float*>(ws + L.y_acc);
  rp.partial = reinterpret_cast<float*>(ws + L.router_partial);
  rp.tile_counter = reinterpret_cast<int32_t*>(ws + L.router_counter);
  rp.T = T;
  rp.H = p->H;
  rp.E = p->E;
  rp.k = p->k;
  const int splits = router_splits(T, p->H, p->num_sms);
  mark(0);
  if (f8 != nullptr) {   // x codes and token scales for the FP8 first GEMM
    moe_quantize_x_kernel<<<(T + 7) / 8, 256, 0, st>>>(static_cast<const bf16*>(x), ws + L.x_q,
                                                       reinterpret_cast<float*>(ws + L.s_x), T, p->H);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (p->E % 64 == 0 && splits == 1) {
    // many tokens, E a multiple of 64: gate GEMM on tcgen05
    RouterTcParams tp;
    std::memset(&tp, 0, sizeof(tp));
    if (!make_map(&tp.tm_x, x, p->H, T, p->H, kRtcTokens) || !make_map(&tp.tm_wg, Wg, p->E, p->H, p->E, 64))
      return MOE_ERR_CUDA;
    tp.bias = bias;
    tp.topk_idx = rp.topk_idx;
    tp.topk_w = rp.topk_w;
    tp.rank = rp.rank;
    tp.chunk_count = rp.chunk_count;
    tp.y_acc = rp.y_acc;
    tp.err = reinterpret_cast<int32_t*>(ws + L.err);
    tp.T = T;
    tp.H = p->H;
    tp.E = p->E;
    tp.k = p->k;
    tp.timeout_ns = p->timeout_ns;
    moe_router_tc_kernel<<<(T + kRtcTokens - 1) / kRtcTokens, kRtcThreads, kRtcSmemBytes, st>>>(tp);
    ce = cudaGetLastError();
  } else {
    switch (expert_pad(p->E)) {
      case 16: ce = launch_router<16>(rp, T, splits, st); break;
      case 32: ce = launch_router<32>(rp, T, splits, st); break;
      case 64: ce = launch_router<64>(rp, T, splits, st); break;
      case 128: ce = launch_router<128>(rp, T, splits, st); break;
      default: ce = launch_router<256>(rp, T, splits, st); break;
    }
  }
  if (ce != cudaSuccess) return MOE_ERR_CUDA;

  // 2. dispatch scan, 3. dispatch scatter
  DispatchParams dp{};
  dp.topk_idx = rp.topk_idx;
  dp.rank = rp.rank;
  dp.chunk_count = rp.chunk_count;
  dp.expert_count = reinterpret_cast<int32_t*>(ws + L.expert_count);
  dp.expert_offset = reinterpret_cast<int32_t*>(ws + L.expert_offset);
  dp.block_start = reinterpret_cast<int32_t*>(ws + L.block_start);
  dp.slot_token = reinterpret_cast<int32_t*>(ws + L.slot_token);
  dp.slot_topk = reinterpret_cast<int32_t*>(ws + L.slot_topk);
  dp.l1_done = reinterpret_cast<int32_t*>(ws + L.l1_done);
  dp.sched = reinterpret_cast<int32_t*>(ws + L.sched);
  dp.err = reinterpret_cast<int32_t*>(ws + L.err);
  dp.T = T;
  dp.E = p->E;
  dp.S = p->S;
  dp.k = p->k;
  dp.BM = p->BM;
  dp.num_chunks = (T + kRouterTokens - 1) / kRouterTokens;
  dp.pool = p->pool;
  dp.group_start = reinterpret_cast<int32_t*>(ws + L.group_start);
  dp.l2_done = reinterpret_cast<int32_t*>(ws + L.l2_done);
  dp.pair_start = p->cta_pairs ? reinterpret_cast<int32_t*>(ws + L.pair_start) : nullptr;
  dp.group_min = p->cta_pairs ? p->pgroup_min : p->group_min;
  dp.group_max = p->cta_pairs ? p->pgroup_max : p->group_max;
  dp.max_groups = p->cta_pairs ? p->pmax_groups : p->max_groups;
  if (f8 != nullptr) {
    // FP8: groups of exactly the units whose activation the buffer holds, run one after another
    const int units = std::max(1, p->fp8_rows / (p->cta_pairs ? 2 * p->BM : p->BM));
    dp.group_min = dp.group_max = units;
    dp.max_groups = std::min(kMaxGroups, p->blocks_max / units + 2);
  }
  mark(1);
  moe_dispatch_scan_kernel<<<1, kScanThreads, 0, st>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  mark(2);
  moe_dispatch_scatter_kernel<<<(T * p->k + 255) / 256, 256, 0, st>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  mark(3);
  if (!full) {
    if (prof) {
      mark(4);
      mark(5);
      ++p->ev_used;
    }
    return MOE_OK;
  }

  // 4. persistent expert GEMM (L1 + SwiGLU, L2 + weighted scatter-add). With
  // FP8 operands the two GEMMs are two launches of the same kernel around the
  // activation quantizer (each activation row is quantized once, with the
  // scale of its full amax, which the first launch gathers).
  bf16* h = reinterpret_cast<bf16*>(ws + L.h);
  const int E = p->E, H = p->H, I = p->I;
  float* act_amax = reinterpret_cast<float*>(ws + L.act_amax);
  float* act_scale = reinterpret_cast<float*>(ws + L.act_scale);
  uint8_t* h8 = ws + L.h8;
  const int h8_rows = p->fp8_rows;
  // FP8: per block group (groups of fp8_units units, each the rows the buffer holds), the
  // first GEMM alone, the activation quantizer over the group's rows, the second GEMM alone;
  // the task counter restarts before each launch, the row amaxes before each group
  const int unit_rows = p->cta_pairs ? 2 * p->BM : p->BM;
  const int fp8_units = std::max(1, h8_rows / unit_rows);
  const int fp8_groups = (p->blocks_max + fp8_units - 1) / fp8_units;   // enough for any routing
  auto restart_counter = [&]() { return cudaMemsetAsync(dp.sched, 0, 4, st) == cudaSuccess; };
  auto quantize_group = [&](int g) -> bool {
    const int grid = p->num_sms * 8;
    moe_quantize_act_kernel<<<grid, 256, 0, st>>>(h, act_amax, h8, act_scale, dp.group_start, dp.sched + 3, g,
                                                  fp8_units, unit_rows, I);
    return cudaGetLastError() == cudaSuccess && restart_counter();
  };
  if (p->cta_pairs) {
    Gemm2Params gp;
    std::memset(&gp, 0, sizeof(gp));
    bool ok = f8 != nullptr ? make_map_u8(&gp.tm_w1, W1, H, (uint64_t)E * I) && make_map_u8(&gp.tm_w3, W3, H, (uint64_t)E * I)
                            : make_map(&gp.tm_w1, W1, I, (uint64_t)E * H, I, 64) &&
                                  make_map(&gp.tm_w3, W3, I, (uint64_t)E * H, I, 64);
    if (ok && p->S > 0)
      ok = make_map(&gp.tm_ws1, sw.Ws1, I, (uint64_t)p->S * H, I, 64) &&
           make_map(&gp.tm_ws3, sw.Ws3, I, (uint64_t)p->S * H, I, 64);
    if (!ok) return MOE_ERR_CUDA;
    gp.x = static_cast<const bf16*>(x);
    gp.phase_only = -1;
    if (f8 != nullptr) {
      gp.xq = ws + L.x_q;
      gp.sx = reinterpret_cast<const float*>(ws + L.s_x);
      gp.s1 = f8->s1;
      gp.s3 = f8->s3;
      gp.w2q = static_cast<const uint8_t*>(f8->W2q);
      gp.s2 = f8->s2;
      gp.act_amax = act_amax;
      gp.act_scale = act_scale;
      gp.h8 = h8;
      gp.phase_only = 0;
    }
    gp.w2 = f8 != nullptr ? nullptr : static_cast<const bf16*>(W2);
    gp.ws2 = static_cast<const bf16*>(sw.Ws2);
    gp.S = p->S;
    gp.slot_token = dp.slot_token;
    gp.slot_topk = dp.slot_topk;
    gp.topk_w = rp.topk_w;
    gp.block_start = dp.block_start;
    gp.pair_start = dp.pair_start;
    gp.group_start = dp.group_start;
    gp.num_groups = dp.sched + 3;
    gp.task_counter = dp.sched;
    gp.l1_done = dp.l1_done;
    gp.l2_done = dp.l2_done;
    gp.err = dp.err;
    gp.h = h;
    gp.y_acc = rp.y_acc;
    gp.T = T;
    gp.H = H;
    gp.I = I;
    gp.E = E;
    gp.k = p->k;
    gp.BM = p->BM;
    gp.BN2 = p->BN2;
    const bool wide = f8 == nullptr && wide_l1_active(*p);   // 256 columns of I per L1 task
    gp.N1 = wide ? I / (2 * kL1TileN) : p->N1;
    gp.N2 = p->N2;
    gp.ring_pairs = f8 != nullptr ? fp8_units : p->ring_pairs;   // FP8: a group's pairs, each its own rows
    gp.max_groups = p->pmax_groups;
    gp.order_lag = order_lag(*p);
    gp.half_tails = (p->half_tails && f8 == nullptr && p->BM == kTileM) ? 1 : 0;   // bf16, 128-row blocks
    gp.zero_row = ws + L.zero_row;
    if (p->task_log) {
      gp.task_log = reinterpret_cast<TaskRecord*>(ws + L.task_log);
      gp.task_log_cap = task_log_capacity(*p);
      if (cudaMemsetAsync(gp.task_log, 0xFF, (size_t)gp.task_log_cap * sizeof(TaskRecord), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    gp.timeout_ns = p->timeout_ns;
    gp.withhold_pair = p->withhold;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(2 * p->pair_clusters));
    cfg.blockDim = dim3(kGemm1Threads);
    cfg.dynamicSmemBytes = wide ? kGemm2SmemBytesW : kGemm2SmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void (*kfn)(Gemm2Params) = f8 != nullptr ? moe_expert_gemm2_kernel<true, false>
                               : wide       ? moe_expert_gemm2_kernel<false, true>
                                            : moe_expert_gemm2_kernel<false, false>;
    if (f8 == nullptr) {
      if (cudaLaunchKernelEx(&cfg, kfn, gp) != cudaSuccess) return MOE_ERR_CUDA;
    } else {
      for (int g = 0; g < fp8_groups; ++g) {   // groups past the routing's last exit at once
        gp.only_group = g;
        gp.phase_only = 0;
        if (cudaMemsetAsync(act_amax, 0, (size_t)h8_rows * 4, st) != cudaSuccess ||
            cudaLaunchKernelEx(&cfg, kfn, gp) != cudaSuccess || !restart_counter() || !quantize_group(g))
          return MOE_ERR_CUDA;
        gp.phase_only = 1;
        if (cudaLaunchKernelEx(&cfg, kfn, gp) != cudaSuccess || !restart_counter()) return MOE_ERR_CUDA;
      }
    }
  } else {
    GemmParams gp;
    std::memset(&gp, 0, sizeof(gp));
    bool ok = f8 != nullptr ? make_map_u8(&gp.tm_w1, W1, H, (uint64_t)E * I) &&
                                  make_map_u8(&gp.tm_w3, W3, H, (uint64_t)E * I) &&
                                  make_map_u8(&gp.tm_w2, W2, I, (uint64_t)E * H)
                            : make_map(&gp.tm_w1, W1, I, (uint64_t)E * H, I, 64) &&
                                  make_map(&gp.tm_w3, W3, I, (uint64_t)E * H, I, 64) &&
                                  make_map(&gp.tm_w2, W2, H, (uint64_t)E * I, H, 64);
    if (ok && p->S > 0)
      ok = make_map(&gp.tm_ws1, sw.Ws1, I, (uint64_t)p->S * H, I, 64) &&
           make_map(&gp.tm_ws3, sw.Ws3, I, (uint64_t)p->S * H, I, 64) &&
           make_map(&gp.tm_ws2, sw.Ws2, H, (uint64_t)p->S * I, H, 64);
    if (!ok) return MOE_ERR_CUDA;
    gp.S = p->S;
    gp.x = static_cast<const bf16*>(x);
    gp.phase_only = -1;
    if (f8 != nullptr) {
      gp.xq = ws + L.x_q;
      gp.sx = reinterpret_cast<const float*>(ws + L.s_x);
      gp.s1 = f8->s1;
      gp.s3 = f8->s3;
      gp.s2 = f8->s2;
      gp.act_amax = act_amax;
      gp.act_scale = act_scale;
      gp.h8 = h8;
      gp.phase_only = 0;
    }
    gp.slot_token = dp.slot_token;
    gp.slot_topk = dp.slot_topk;
    gp.topk_w = rp.topk_w;
    gp.block_start = dp.block_start;
    gp.group_start = dp.group_start;
    gp.num_groups = dp.sched + 3;
    gp.task_counter = dp.sched;
    gp.l1_done = dp.l1_done;
    gp.l2_done = dp.l2_done;
    gp.ring_blocks = f8 != nullptr ? fp8_units : p->ring_blocks;   // FP8: a group's blocks, each its own rows
    gp.max_groups = p->max_groups;
    gp.order_lag = order_lag(*p);
    gp.zero_row = ws + L.zero_row;
    if (p->task_log) {
      gp.task_log = reinterpret_cast<TaskRecord*>(ws + L.task_log);
      gp.task_log_cap = task_log_capacity(*p);
      if (cudaMemsetAsync(gp.task_log, 0xFF, (size_t)gp.task_log_cap * sizeof(TaskRecord), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    gp.err = dp.err;
    gp.h = h;
    gp.y_acc = rp.y_acc;
    gp.T = T;
    gp.H = H;
    gp.I = I;
    gp.E = E;
    gp.k = p->k;
    gp.BM = p->BM;
    gp.BN2 = p->BN2;
    gp.N1 = p->N1;
    gp.N2 = p->N2;
    gp.timeout_ns = p->timeout_ns;
    gp.withhold_block = p->withhold;
    void (*kfn)(GemmParams) = f8 != nullptr ? moe_expert_gemm_kernel<true> : moe_expert_gemm_kernel<false>;
    if (f8 == nullptr) {
      kfn<<<p->num_sms, kGemm1Threads, kGemmSmemBytes, st>>>(gp);
    } else {
      for (int g = 0; g < fp8_groups; ++g) {
        gp.only_group = g;
        gp.phase_only = 0;
        if (cudaMemsetAsync(act_amax, 0, (size_t)h8_rows * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
        kfn<<<p->num_sms, kGemm1Threads, kGemmSmemBytes, st>>>(gp);
        if (cudaGetLastError() != cudaSuccess || !restart_counter() || !quantize_group(g)) return MOE_ERR_CUDA;
        gp.phase_only = 1;
        kfn<<<p->num_sms, kGemm1Threads, kGemmSmemBytes, st>>>(gp);
        if (cudaGetLastError() != cudaSuccess || !restart_counter()) return MOE_ERR_CUDA;
      }
    }
  }
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  mark(4);

  // 5. y = bf16(y_acc)
  const size_t n4 = (size_t)T * H / 4;
  const int fgrid = (int)std::min<size_t>((n4 + 255) / 256, (size_t)p->num_sms * 16);
  moe_finalize_kernel<<<fgrid, 256, 0, st>>>(rp.y_acc, static_cast<bf16*>(y), n4);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  mark(5);
  if (prof) ++p->ev_used;
  return MOE_OK;
}

// One launch of the backward GEMM kernel of kind K on the plan's persistent grid.
template <int K>
static cudaError_t launch_bwd(const BwdParams& bp, int grid, cudaStream_t st) {
  moe_backward_gemm_kernel<K><<<grid, kBwdThreads, kBwdSmemBytes, st>>>(bp);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- routing with no allocation
// Scratch of moe_route_static(): the error word, the dispatch counters, the
// in-chunk ranks [T*k], the per-chunk expert counts [ceil(T/64)*E], the block
// starts [E+1] and the per-block counters the dispatch scan clears. It is a
// file-scope device array, so every GPU that loads this library holds these
// 1 MiB until the process exits, and every call on a device uses the same copy.
namespace {
constexpr int kStaticScratchInts = 1 << 18;
constexpr int kStaticMaxDevices = 64;
std::mutex g_static_mu;
int32_t* g_static_scratch[kStaticMaxDevices] = {};
}  // namespace

static __device__ __align__(256) int32_t g_route_scratch[kStaticScratchInts];

// Once per device, with that device current: resolve the array's device
// address (host code may not use the symbol itself as a pointer) and allow
// the routing-only router its dynamic shared memory.
static int static_scratch_for_current_device(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kStaticMaxDevices) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_scratch[dev] == nullptr) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED_DEVICE;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || ptr == nullptr) return MOE_ERR_CUDA;
    cudaError_t ce = cudaFuncSetAttribute(moe_router_kernel<16, false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, RouterSmem<16>::kBytes);
    if (ce == cudaSuccess)
      ce = cudaFuncSetAttribute(moe_router_kernel<32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                RouterSmem<32>::kBytes);
    if (ce == cudaSuccess)
      ce = cudaFuncSetAttribute(moe_router_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                RouterSmem<64>::kBytes);
    if (ce == cudaSuccess)
      ce = cudaFuncSetAttribute(moe_router_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                RouterSmem<128>::kBytes);
    if (ce == cudaSuccess)
      ce = cudaFuncSetAttribute(moe_router_kernel<256, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                RouterSmem<256>::kBytes);
    if (ce != cudaSuccess) return MOE_ERR_CUDA;
    g_static_scratch[dev] = static_cast<int32_t*>(ptr);
  }
  *out = g_static_scratch[dev];
  return MOE_OK;
}

extern "C" int moe_route_static(const void* x, const void* Wg, const float* gate_bias, int T, int H, int E, int k,
                                int block_m, int32_t* topk_idx, float* topk_w, int32_t* expert_count,
                                int32_t* expert_offset, int32_t* slot_token, int32_t* slot_topk, int pool_capacity,
                                int32_t* num_padded, int32_t* error_word, void* stream) {
  if (T < 0 || H < 128 || H % 128 || E < 8 || E > 256 || E % 8 || k < 1 || k > 8 || k > E)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (block_m != 0 && block_m != 16 && block_m != 32 && block_m != 64 && block_m != 128)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // far beyond the scratch limit below; refused here so that no size arithmetic can overflow
  if (T > kStaticScratchInts) return MOE_ERR_STATIC_SCRATCH_LIMIT;
  const int BM = block_m ? block_m : block_m_rule(T > 0 ? T : 1, k, E);
  const long long pool = ((long long)T * k + (long long)E * (BM - 1) + BM - 1) / BM * BM;
  const long long chunks = ((long long)T + kRouterTokens - 1) / kRouterTokens;
  // scratch regions, each rounded up to 64 ints (256 bytes)
  auto r64 = [](long long v) { return (v + 63) / 64 * 64; };
  const long long o_err = 0, o_sched = 64, o_rank = 128;
  const long long o_chunk = o_rank + r64((long long)T * k);
  const long long o_bs = o_chunk + r64(chunks * E);
  const long long o_l1 = o_bs + r64(E + 1);
  const long long need = o_l1 + r64(pool / BM);
  if (need > kStaticScratchInts) return MOE_ERR_STATIC_SCRATCH_LIMIT;
  if (T == 0) return MOE_OK;
  if (x == nullptr || Wg == nullptr || !aligned16(x) || !aligned16(Wg)) return MOE_ERR_INVALID_ARG;
  if (gate_bias != nullptr && (reinterpret_cast<uintptr_t>(gate_bias) & 3u)) return MOE_ERR_INVALID_ARG;
  if (topk_idx == nullptr || topk_w == nullptr || expert_count == nullptr || expert_offset == nullptr ||
      slot_token == nullptr || slot_topk == nullptr || num_padded == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (pool_capacity < pool) return MOE_ERR_INVALID_ARG;
  drop_stale_error();
  int32_t* scratch = nullptr;
  int rc = static_scratch_for_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // The error word must start at zero; everything else is fully written below.
  if (cudaMemsetAsync(scratch + o_err, 0, 2 * sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;

  RouterParams rp{};
  rp.x = static_cast<const bf16*>(x);
  rp.Wg = static_cast<const bf16*>(Wg);
  rp.bias = gate_bias;
  rp.topk_idx = topk_idx;
  rp.topk_w = topk_w;
  rp.rank = scratch + o_rank;
  rp.chunk_count = scratch + o_chunk;
  rp.y_acc = nullptr;
  rp.partial = nullptr;   // one CTA per token tile (no H split)
  rp.tile_counter = nullptr;
  rp.T = T;
  rp.H = H;
  rp.E = E;
  rp.k = k;
  const int grid = (int)chunks;
  switch (expert_pad(E)) {
    case 16: moe_router_kernel<16, false><<<grid, kRouterThreads, RouterSmem<16>::kBytes, st>>>(rp); break;
    case 32: moe_router_kernel<32, false><<<grid, kRouterThreads, RouterSmem<32>::kBytes, st>>>(rp); break;
    case 64: moe_router_kernel<64, false><<<grid, kRouterThreads, RouterSmem<64>::kBytes, st>>>(rp); break;
    case 128: moe_router_kernel<128, false><<<grid, kRouterThreads, RouterSmem<128>::kBytes, st>>>(rp); break;
    default: moe_router_kernel<256, false><<<grid, kRouterThreads, RouterSmem<256>::kBytes, st>>>(rp); break;
  }
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  DispatchParams dp{};
  dp.topk_idx = topk_idx;
  dp.rank = rp.rank;
  dp.chunk_count = rp.chunk_count;
  dp.expert_count = expert_count;
  dp.expert_offset = expert_offset;
  dp.block_start = scratch + o_bs;
  dp.slot_token = slot_token;
  dp.slot_topk = slot_topk;
  dp.l1_done = scratch + o_l1;
  dp.sched = scratch + o_sched;
  dp.err = scratch + o_err;
  dp.T = T;
  dp.E = E;
  dp.k = k;
  dp.BM = BM;
  dp.num_chunks = (int)chunks;
  dp.pool = (int)pool;
  dp.group_start = nullptr;   // routing only: no expert-GEMM task groups
  dp.l2_done = nullptr;
  dp.pair_start = nullptr;
  dp.group_min = dp.group_max = dp.max_groups = 0;
  moe_dispatch_scan_kernel<<<1, kScanThreads, 0, st>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  moe_dispatch_scatter_kernel<<<(T * k + 255) / 256, 256, 0, st>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  // slots in use (written by the scan) and the device error word, to the caller's buffers
  if (cudaMemcpyAsync(num_padded, scratch + o_sched + 2, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (error_word != nullptr &&
      cudaMemcpyAsync(error_word, scratch + o_err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

extern "C" {

int moe_plan_create(moe_plan_t* out, int T_max, int H, int I, int E, int k, int block_m, int device) {
  return moe_plan_create_shared(out, T_max, H, I, E, k, 0, block_m, device);
}

int moe_plan_create_shared(moe_plan_t* out, int T_max, int H, int I, int E, int k, int n_shared, int block_m,
                           int device) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (T_max < 1 || H < 128 || H % 128 || I < 128 || I % 128 || E < 8 || E > kMaxExperts || E % 8 || k < 1 ||
      k > 8 || k > E || n_shared < 0 || n_shared > kMaxShared)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (block_m != 0 && block_m != 16 && block_m != 32 && block_m != 64 && block_m != 128)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // int32 indexing of slots, h rows and T*k
  if ((long long)T_max * (k + n_shared) + (long long)(E + n_shared) * 127 > (1LL << 30))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return MOE_ERR_CUDA;
  if (device < 0 || device >= ndev) return MOE_ERR_INVALID_ARG;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED_DEVICE;
  if (tensor_map_encoder() == nullptr) return MOE_ERR_CUDA;

  moe_plan* p = new (std::nothrow) moe_plan();
  if (p == nullptr) return MOE_ERR_CUDA;
  p->T_max = T_max;
  p->H = H;
  p->I = I;
  p->E = E;
  p->k = k;
  p->BM = block_m ? block_m : block_m_rule(T_max, k, E);
  p->device = device;
  p->num_sms = prop.multiProcessorCount;
  p->BN2 = (H % 256 == 0) ? 256 : 128;
  p->N1 = I / kL1TileN;
  p->N2 = H / p->BN2;
  p->S = n_shared;
  p->pool = T_max * k + E * (p->BM - 1);
  p->pool = (p->pool + p->BM - 1) / p->BM * p->BM;
  p->pool += n_shared * ((T_max + p->BM - 1) / p->BM) * p->BM;   // shared experts: every token once each
  p->chunks_max = (T_max + kRouterTokens - 1) / kRouterTokens;
  p->blocks_max = p->pool / p->BM;
  // Task groups (see the expert GEMM's task order): an L1 segment of at least
  // two waves of tasks so the one-group lag hides L1 completion; groups up to
  // an expert's expected block count so weight slices stay shared; at most
  // kMaxGroups groups. The h ring holds 3 groups: the block that last used a
  // slot is then two segments back in the task order.
  p->group_min = (2 * p->num_sms + p->N1 - 1) / p->N1;
  p->group_min = std::max(p->group_min, (p->blocks_max + kMaxGroups - 3) / (kMaxGroups - 2));
  const int per_expert = (int)(((long long)T_max * k + (long long)E * p->BM - 1) / ((long long)E * p->BM)) + 1;
  p->group_max = std::max(2 * p->group_min, per_expert);
  p->max_groups = p->blocks_max / p->group_min + 2;
  p->ring_blocks = std::min(3 * p->group_max, p->blocks_max);
  p->per_expert = per_expert;
  size_pair_groups(p);
  p->L = make_layout(*p);

  DeviceGuard guard(device);
  // both instances of each expert-GEMM kernel: bf16 and FP8 operands
  cudaError_t ce = cudaFuncSetAttribute(moe_expert_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kGemmSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_expert_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kGemmSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_expert_gemm2_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kGemm2SmemBytesW);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_expert_gemm2_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kGemm2SmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_expert_gemm2_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kGemm2SmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtcSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_backward_gemm_kernel<kBwdDgrad1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kBwdSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_backward_gemm_kernel<kBwdDgrad2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kBwdSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_backward_gemm_kernel<kBwdWgrad13>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kBwdSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_backward_gemm_kernel<kBwdWgrad2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kBwdSmemBytes);
  if (ce == cudaSuccess)
    ce = cudaFuncSetAttribute(moe_backward_gemm_kernel<kBwdDwg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kBwdSmemBytes);
  if (ce == cudaSuccess) ce = set_router_smem<16>();
  if (ce == cudaSuccess) ce = set_router_smem<32>();
  if (ce == cudaSuccess) ce = set_router_smem<64>();
  if (ce == cudaSuccess) ce = set_router_smem<128>();
  if (ce == cudaSuccess) ce = set_router_smem<256>();
  if (ce != cudaSuccess) {
    delete p;
    return MOE_ERR_CUDA;
  }
  {
    // how many 2-CTA clusters of the pair kernel can be resident at once (a
    // cluster needs two free SMs of one GPC); the pair grid is sized to it
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(p->num_sms & ~1));
    cfg.blockDim = dim3(kGemm1Threads);
    cfg.dynamicSmemBytes = kGemm2SmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, moe_expert_gemm2_kernel<false, false>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      clusters = 0;
    }
    p->pair_clusters = clusters;
    size_pair_groups(p);   // with the real number of concurrent pair tasks
    p->L = make_layout(*p);
    // Full 128-row blocks run on CTA pairs (half the weight-tile traffic per
    // SM); smaller blocks keep the single-CTA kernel.
    p->cta_pairs = p->BM == 128 && clusters > 0;
  }
  *out = p;
  return MOE_OK;
}

size_t moe_plan_workspace_bytes(moe_plan_t p) { return p ? p->L.total : 0; }

int moe_plan_bind_workspace(moe_plan_t p, void* ws, size_t bytes) {
  if (p == nullptr || ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_INVALID_ARG;
  if (bytes < p->L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  p->ws = static_cast<uint8_t*>(ws);
  p->ws_bytes = bytes;
  DeviceGuard guard(p->device);
  // error word and scheduler counters start at zero, and the zero row is zero
  if (cudaMemset(p->ws + p->L.err, 0, 16 * 4) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(p->ws + p->L.zero_row, 0, (size_t)p->H * 2) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(p->ws + p->L.sched, 0, 16 * 4) != cudaSuccess) return MOE_ERR_CUDA;
  // split-H router state: accumulators and counters are zero between calls
  if (cudaMemset(p->ws + p->L.router_counter, 0, (size_t)p->num_sms * 4) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(p->ws + p->L.router_partial, 0, (size_t)p->num_sms * kRouterTokens * 256 * 4) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  p->pipe_used[0] = p->pipe_used[1] = false;   // a new workspace: no staging buffer is in flight
  p->pipe_next = 0;
  return MOE_OK;
}

int moe_plan_describe(moe_plan_t p, moe_plan_desc* d) {
  if (p == nullptr || d == nullptr) return MOE_ERR_INVALID_ARG;
  d->T_max = p->T_max;
  d->H = p->H;
  d->I = p->I;
  d->E = p->E;
  d->k = p->k;
  d->block_m = p->BM;
  d->pool_capacity = p->pool;
  d->num_sms = p->num_sms;
  d->pair_clusters = p->pair_clusters;
  d->n_shared = p->S;
  d->cta_pairs = p->cta_pairs ? 1 : 0;
  d->workspace_bytes = p->L.total;
  d->task_order = order_lag(*p) >= 0 ? 1 : 0;
  d->half_tails = (p->cta_pairs && p->half_tails && p->BM == kTileM) ? 1 : 0;
  d->wide_l1 = (p->cta_pairs && wide_l1_active(*p)) ? 1 : 0;
  return MOE_OK;
}

int moe_plan_get_routing(moe_plan_t p, moe_routing* r) {
  if (p == nullptr || r == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  r->topk_idx = reinterpret_cast<int32_t*>(p->ws + p->L.topk_idx);
  r->topk_w = reinterpret_cast<float*>(p->ws + p->L.topk_w);
  r->expert_count = reinterpret_cast<int32_t*>(p->ws + p->L.expert_count);
  r->expert_offset = reinterpret_cast<int32_t*>(p->ws + p->L.expert_offset);
  r->slot_token = reinterpret_cast<int32_t*>(p->ws + p->L.slot_token);
  r->slot_topk = reinterpret_cast<int32_t*>(p->ws + p->L.slot_topk);
  r->num_padded = reinterpret_cast<int32_t*>(p->ws + p->L.num_padded);
  r->block_m = p->BM;
  r->pool_capacity = p->pool;
  return MOE_OK;
}

int moe_forward(moe_plan_t p, const void* x, const void* Wg, const float* bias, const void* W1, const void* W3,
                const void* W2, int T, void* y, void* stream) {
  if (p == nullptr || p->S > 0) return MOE_ERR_INVALID_ARG;
  return enqueue(p, x, Wg, bias, W1, W3, W2, SharedWeights{}, T, y, static_cast<cudaStream_t>(stream), true);
}

int moe_forward_shared(moe_plan_t p, const void* x, const void* Wg, const float* bias, const void* W1,
                       const void* W3, const void* W2, const void* Ws1, const void* Ws3, const void* Ws2, int T,
                       void* y, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  return enqueue(p, x, Wg, bias, W1, W3, W2, SharedWeights{Ws1, Ws3, Ws2}, T, y, static_cast<cudaStream_t>(stream),
                 true);
}

int moe_route(moe_plan_t p, const void* x, const void* Wg, const float* bias, int T, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  return enqueue(p, x, Wg, bias, nullptr, nullptr, nullptr, SharedWeights{}, T, nullptr,
                 static_cast<cudaStream_t>(stream), false);
}

static int forward_host(moe_plan_t p, const void* x_host, const void* Wg, const float* bias, const void* W1,
                        const void* W3, const void* W2, const SharedWeights& sw, int T, void* y_host, void* stream,
                        const Fp8Weights* f8 = nullptr) {
  if (p == nullptr || x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  if (T < 0 || T > p->T_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  DeviceGuard guard(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)T * p->H * 2;
  void* xd = p->ws + p->L.x_stage;
  void* yd = p->ws + p->L.y_stage;
  if (cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
  const int rc = enqueue(p, xd, Wg, bias, W1, W3, W2, sw, T, yd, st, true, f8);
  if (rc != MOE_OK) return rc;
  if (cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// The pipelined host entry: x is copied in on the plan's copy-in stream, the forward runs on
// `stream`, y is copied out on the copy-out stream, each call using the other of two staging
// buffers, so one call's copies overlap the neighbouring calls' kernels. A buffer is refilled
// only after the forward that read it has finished, and reused for y only after its previous
// y has been copied out.
static int forward_host_pipelined(moe_plan_t p, const void* x_host, const void* Wg, const float* bias,
                                  const void* W1, const void* W3, const void* W2, int T, void* y_host, void* stream,
                                  const Fp8Weights* f8) {
  if (p == nullptr || x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  if (p->S > 0) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > p->T_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  DeviceGuard guard(p->device);
  if (p->cp_in == nullptr) {
    if (cudaStreamCreateWithFlags(&p->cp_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p->cp_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&p->ev_mark, cudaEventDisableTiming) != cudaSuccess)
      return MOE_ERR_CUDA;
    for (int b = 0; b < 2; ++b)
      if (cudaEventCreateWithFlags(&p->ev_in[b], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&p->ev_done[b], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&p->ev_out[b], cudaEventDisableTiming) != cudaSuccess)
        return MOE_ERR_CUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int b = p->pipe_next;
  const size_t stage = (size_t)p->T_max * p->H * 2;
  const size_t bytes = (size_t)T * p->H * 2;
  void* xd = p->ws + p->L.x_stage + b * stage;
  void* yd = p->ws + p->L.y_stage + b * stage;
  if (p->pipe_used[b] && cudaStreamWaitEvent(p->cp_in, p->ev_done[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, p->cp_in) != cudaSuccess ||
      cudaEventRecord(p->ev_in[b], p->cp_in) != cudaSuccess || cudaStreamWaitEvent(st, p->ev_in[b], 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (p->pipe_used[b] && cudaStreamWaitEvent(st, p->ev_out[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
  const int rc = enqueue(p, xd, Wg, bias, W1, W3, W2, SharedWeights{}, T, yd, st, true, f8);
  if (rc != MOE_OK) return rc;
  if (cudaEventRecord(p->ev_done[b], st) != cudaSuccess || cudaStreamWaitEvent(p->cp_out, p->ev_done[b], 0) != cudaSuccess ||
      cudaMemcpyAsync(y_host, yd, bytes, cudaMemcpyDeviceToHost, p->cp_out) != cudaSuccess ||
      cudaEventRecord(p->ev_out[b], p->cp_out) != cudaSuccess)
    return MOE_ERR_CUDA;
  p->pipe_used[b] = true;
  p->pipe_next = b ^ 1;
  return MOE_OK;
}

int moe_forward_host_pipelined(moe_plan_t p, const void* x_host, const void* Wg, const float* bias, const void* W1,
                               const void* W3, const void* W2, int T, void* y_host, void* stream) {
  return forward_host_pipelined(p, x_host, Wg, bias, W1, W3, W2, T, y_host, stream, nullptr);
}

int moe_forward_host_pipelined_fp8(moe_plan_t p, const void* x_host, const void* Wg, const float* bias,
                                   const void* W1q, const float* s1, const void* W3q, const float* s3,
                                   const void* W2q, const float* s2, int T, void* y_host, void* stream) {
  const Fp8Weights f8{W1q, s1, W3q, s3, W2q, s2};
  return forward_host_pipelined(p, x_host, Wg, bias, nullptr, nullptr, nullptr, T, y_host, stream, &f8);
}

int moe_host_pipeline_after(moe_plan_t p, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->cp_in == nullptr) return MOE_OK;   // nothing pipelined yet: the first call creates the streams
  DeviceGuard guard(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaEventRecord(p->ev_mark, st) != cudaSuccess || cudaStreamWaitEvent(p->cp_in, p->ev_mark, 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->cp_out, p->ev_mark, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_host_pipeline_join(moe_plan_t p, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(p->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int b = 0; b < 2; ++b)
    if (p->pipe_used[b] && cudaStreamWaitEvent(st, p->ev_out[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_forward_host(moe_plan_t p, const void* x_host, const void* Wg, const float* bias, const void* W1,
                     const void* W3, const void* W2, int T, void* y_host, void* stream) {
  if (p != nullptr && p->S > 0) return MOE_ERR_INVALID_ARG;
  return forward_host(p, x_host, Wg, bias, W1, W3, W2, SharedWeights{}, T, y_host, stream);
}

int moe_forward_host_shared(moe_plan_t p, const void* x_host, const void* Wg, const float* bias, const void* W1,
                            const void* W3, const void* W2, const void* Ws1, const void* Ws3, const void* Ws2, int T,
                            void* y_host, void* stream) {
  return forward_host(p, x_host, Wg, bias, W1, W3, W2, SharedWeights{Ws1, Ws3, Ws2}, T, y_host, stream);
}

int moe_forward_fp8(moe_plan_t p, const void* x, const void* Wg, const float* bias, const void* W1q, const float* s1,
                    const void* W3q, const float* s3, const void* W2q, const float* s2, int T, void* y, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  const Fp8Weights f8{W1q, s1, W3q, s3, W2q, s2};
  return enqueue(p, x, Wg, bias, nullptr, nullptr, nullptr, SharedWeights{}, T, y, static_cast<cudaStream_t>(stream),
                 true, &f8);
}

int moe_forward_host_fp8(moe_plan_t p, const void* x_host, const void* Wg, const float* bias, const void* W1q,
                         const float* s1, const void* W3q, const float* s3, const void* W2q, const float* s2, int T,
                         void* y_host, void* stream) {
  const Fp8Weights f8{W1q, s1, W3q, s3, W2q, s2};
  return forward_host(p, x_host, Wg, bias, nullptr, nullptr, nullptr, SharedWeights{}, T, y_host, stream, &f8);
}

int moe_quantize_x_fp8(const void* x, void* xq, float* sx, int T, int H, void* stream) {
  if (T < 0 || H < 8 || H % 8) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x == nullptr || xq == nullptr || sx == nullptr || !aligned16(x) || (reinterpret_cast<uintptr_t>(xq) & 7u) ||
      (reinterpret_cast<uintptr_t>(sx) & 3u))
    return MOE_ERR_INVALID_ARG;
  drop_stale_error();
  moe_quantize_x_kernel<<<(T + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const bf16*>(x), static_cast<uint8_t*>(xq), sx, T, H);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_quantize_weights_fp8(const void* W, void* Wq, float* scale, int E, int H, int I, void* stream) {
  if (E < 1 || H < 64 || H % 64 || I < 64 || I % 64) return MOE_ERR_INVALID_ARG;
  if (W == nullptr || Wq == nullptr || scale == nullptr || !aligned16(Wq) || (reinterpret_cast<uintptr_t>(W) & 1u) ||
      (reinterpret_cast<uintptr_t>(scale) & 3u))
    return MOE_ERR_INVALID_ARG;
  if (E > 65535 || (long long)E * H * I > (1LL << 40)) return MOE_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  drop_stale_error();
  moe_weight_scales_kernel<<<dim3((unsigned)(I / 32), (unsigned)E), 256, 0, st>>>(static_cast<const bf16*>(W), scale,
                                                                                 H, I);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  moe_weight_quant_kernel<<<dim3((unsigned)(I / 64), (unsigned)(H / 64), (unsigned)E), 256, 0, st>>>(
      static_cast<const bf16*>(W), scale, static_cast<uint8_t*>(Wq), H, I);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_check(moe_plan_t p, void* stream, int32_t* detail) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  DeviceGuard guard(p->device);
  drop_stale_error();
  // Everything on `stream` only: the read and the clearing of the error word are
  // ordered after the plan's kernels there, and no other stream of the device waits.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t e[2] = {0, 0};
  if (cudaMemcpyAsync(e, p->ws + p->L.err, sizeof(e), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (e[0] != 0 && (cudaMemsetAsync(p->ws + p->L.err, 0, sizeof(e), st) != cudaSuccess ||
                    cudaStreamSynchronize(st) != cudaSuccess))
    return MOE_ERR_CUDA;
  if (detail) *detail = e[1];
  switch (e[0]) {
    case kDevOk: return MOE_OK;
    case kDevTimeout: return MOE_ERR_DEVICE_TIMEOUT;
    default: return MOE_ERR_DEVICE_BOUNDS;
  }
}

int moe_plan_set_profiling(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(p->device);
  if (enable && p->ev.empty()) {
    p->ev.resize((size_t)kMaxProfiled * (kNumKernels + 1));
    for (auto& e : p->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
  }
  p->profile = enable != 0;
  p->ev_used = 0;
  return MOE_OK;
}

int moe_plan_profile_read(moe_plan_t p, float* ms, int* count) {
  if (p == nullptr || ms == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(p->device);
  for (int i = 0; i < kNumKernels; ++i) ms[i] = 0.f;
  const int n = p->ev_used;
  if (n > 0 && cudaEventSynchronize(p->ev[(size_t)(n - 1) * (kNumKernels + 1) + kNumKernels]) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int f = 0; f < n; ++f) {
    cudaEvent_t* ev = &p->ev[(size_t)f * (kNumKernels + 1)];
    for (int i = 0; i < kNumKernels; ++i) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, ev[i], ev[i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
      ms[i] += t;
    }
  }
  if (count) *count = n;
  p->ev_used = 0;
  return MOE_OK;
}

int moe_plan_set_debug(moe_plan_t p, int withhold_block, uint64_t timeout_ns) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  p->withhold = withhold_block;
  p->timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
  return MOE_OK;
}

int moe_plan_set_fp8(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (enable && p->S > 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  // The activation rows of one block group (bf16 and codes, I * 3 + 8 bytes a row): up to
  // 256 MB, at least two rows per concurrent task slot of either kernel (a pair: 2 * BLOCK_M
  // rows per cluster; one CTA: BLOCK_M), at most every block's (or pair's) rows, in whole pairs.
  const int pairs_cap = std::min(p->blocks_max, (p->blocks_max + p->E + 1) / 2);
  const long long all_rows = (long long)std::max(p->blocks_max, 2 * pairs_cap) * p->BM;
  const long long budget = (256LL << 20) / ((long long)p->I * 3 + 8);
  const long long floor_rows = 2LL * std::max(2 * std::max(p->pair_clusters, 1), p->num_sms) * p->BM;
  long long rows = std::min(all_rows, std::max(budget, floor_rows));
  rows = std::max(2LL * p->BM, rows / (2 * p->BM) * (2 * p->BM));
  p->fp8_rows = enable ? (int)rows : 0;
  p->L = make_layout(*p);
  p->ws = nullptr;   // the workspace size changed: bind again
  p->ws_bytes = 0;
  return MOE_OK;
}

int moe_plan_set_backward(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (enable && p->S > 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  p->backward = enable != 0;
  p->L = make_layout(*p);
  p->ws = nullptr;   // the workspace size changed: bind again
  p->ws_bytes = 0;
  return MOE_OK;
}

int moe_backward(moe_plan_t p, const void* x, const void* Wg, const float* bias, const void* W1, const void* W3,
                 const void* W2, const void* dy, int T, void* dx, float* dWg, float* dbias, void* dW1, void* dW3,
                 void* dW2, void* stream) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (!p->backward || p->S > 0) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  if (T < 0 || T > p->T_max) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const void* need16[] = {W1, W3, W2, dy, dx, dW1, dW3, dW2};
  for (const void* q : need16)
    if (q == nullptr || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (dWg == nullptr || (reinterpret_cast<uintptr_t>(dWg) & 3u)) return MOE_ERR_INVALID_ARG;
  if (dbias != nullptr && (reinterpret_cast<uintptr_t>(dbias) & 3u)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // routing of x (router, dispatch scan, scatter), as the forward computes it; the
  // router also zeroes the fp32 accumulator rows that collect dx
  int rc = enqueue(p, x, Wg, bias, nullptr, nullptr, nullptr, SharedWeights{}, T, nullptr, st, false);
  if (rc != MOE_OK) return rc;
  DeviceGuard guard(p->device);
  uint8_t* ws = p->ws;
  const Layout& L = p->L;
  const int E = p->E, H = p->H, I = p->I, k = p->k;
  const int NE = (E + 63) / 64 * 64;
  bf16* dg = reinterpret_cast<bf16*>(ws + L.bwd_dg);
  bf16* du = reinterpret_cast<bf16*>(ws + L.bwd_du);
  bf16* aw = reinterpret_cast<bf16*>(ws + L.bwd_aw);
  float* dw = reinterpret_cast<float*>(ws + L.bwd_dw);
  bf16* dl = reinterpret_cast<bf16*>(ws + L.bwd_dl);
  bf16* wgt = reinterpret_cast<bf16*>(ws + L.bwd_wgt);
  if (cudaMemsetAsync(dw, 0, (size_t)T * k * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (dbias != nullptr && cudaMemsetAsync(dbias, 0, (size_t)E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;

  BwdParams bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.slot_token = reinterpret_cast<const int32_t*>(ws + L.slot_token);
  bp.slot_topk = reinterpret_cast<const int32_t*>(ws + L.slot_topk);
  bp.topk_w = reinterpret_cast<const float*>(ws + L.topk_w);
  bp.block_start = reinterpret_cast<const int32_t*>(ws + L.block_start);
  bp.sched = reinterpret_cast<const int32_t*>(ws + L.sched) + 1;   // blocks in use (the scan writes it)
  bp.x = static_cast<const bf16*>(x);
  bp.dy = static_cast<const bf16*>(dy);
  bp.zero_row = reinterpret_cast<const bf16*>(ws + L.zero_row);
  bp.dg = dg;
  bp.du = du;
  bp.aw = aw;
  bp.dw = dw;
  bp.dx_acc = reinterpret_cast<float*>(ws + L.y_acc);
  bp.dW1 = static_cast<bf16*>(dW1);
  bp.dW3 = static_cast<bf16*>(dW3);
  bp.dW2 = static_cast<bf16*>(dW2);
  bp.dWg = dWg;
  bp.err = reinterpret_cast<int32_t*>(ws + L.err);
  bp.T = T;
  bp.H = H;
  bp.I = I;
  bp.E = E;
  bp.k = k;
  bp.BM = p->BM;
  bp.pool = p->pool;
  bp.BN = (H % 256 == 0) ? 256 : 128;
  bp.BNi = (I % 256 == 0) ? 256 : 128;
  bp.NE = NE;
  bp.timeout_ns = p->timeout_ns;
  const int grid = p->num_sms;
  bf16* xp = reinterpret_cast<bf16*>(ws + L.bwd_xp);
  bf16* dyp = reinterpret_cast<bf16*>(ws + L.bwd_dyp);
  bp.permuted = backward_permuted(*p) ? 1 : 0;
  if (bp.permuted) {
    // x and dy rows in slot order (their operands then come by TMA)
    moe_permute_rows_kernel<<<p->num_sms * 8, 256, 0, st>>>(static_cast<const bf16*>(x), static_cast<const bf16*>(dy),
                                                         bp.slot_token, bp.sched, xp, dyp, bp.err, T, H, p->BM, p->pool);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }

  // 1. dgrad-1: g|u recomputed, da = dy W2^T; dg, du, w*a per slot; dw
  BwdParams b1 = bp;
  if (!make_map(&b1.tm_w1, W1, I, (uint64_t)E * H, I, 64) || !make_map(&b1.tm_w3, W3, I, (uint64_t)E * H, I, 64) ||
      !make_map(&b1.tm_w2, W2, H, (uint64_t)E * I, H, 128))
    return MOE_ERR_CUDA;
  if (bp.permuted && (!make_map(&b1.tm_xp, xp, H, p->pool, H, 128) || !make_map(&b1.tm_dyp, dyp, H, p->pool, H, 128)))
    return MOE_ERR_CUDA;
  if (launch_bwd<kBwdDgrad1>(b1, grid, st) != cudaSuccess) return MOE_ERR_CUDA;
  // 2. dgrad-2: dx += [dg|du] [W1|W3]^T through the slot records
  BwdParams b2 = bp;
  if (!make_map(&b2.tm_a, dg, I, p->pool, I, 128) || !make_map(&b2.tm_a2, du, I, p->pool, I, 128) ||
      !make_map(&b2.tm_w1, W1, I, (uint64_t)E * H, I, bp.BN) || !make_map(&b2.tm_w3, W3, I, (uint64_t)E * H, I, bp.BN))
    return MOE_ERR_CUDA;
  if (launch_bwd<kBwdDgrad2>(b2, grid, st) != cudaSuccess) return MOE_ERR_CUDA;
  // 3. gate: dl from dw, dbias, dx = bf16(dx_acc + dl Wg^T), the dense dl for dWg
  moe_transpose_wg_kernel<<<dim3((unsigned)((H + 31) / 32), (unsigned)((E + 31) / 32)), 256, 0, st>>>(
      static_cast<const bf16*>(Wg), wgt, H, E);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  moe_gate_backward_kernel<<<(T * 32 + kGateThreads - 1) / kGateThreads, kGateThreads, 0, st>>>(
      reinterpret_cast<const int32_t*>(ws + L.topk_idx), bp.topk_w, dw, wgt, bp.dx_acc, static_cast<bf16*>(dx), dl,
      dbias, bp.err, T, H, E, k, NE);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  // 4. weight gradients: dW1 = x^T dg, dW3 = x^T du; dW2 = (w a)^T dy; dWg = x^T dl
  BwdParams b3 = bp;
  if (!make_map(&b3.tm_b, dg, I, p->pool, I, 64) || !make_map(&b3.tm_b2, du, I, p->pool, I, 64)) return MOE_ERR_CUDA;
  if (bp.permuted && !make_map(&b3.tm_xp, xp, H, p->pool, H, 64)) return MOE_ERR_CUDA;
  if (launch_bwd<kBwdWgrad13>(b3, grid, st) != cudaSuccess) return MOE_ERR_CUDA;
  BwdParams b4 = bp;
  if (!make_map(&b4.tm_b, aw, I, p->pool, I, 64)) return MOE_ERR_CUDA;
  if (bp.permuted && !make_map(&b4.tm_dyp, dyp, H, p->pool, H, 64)) return MOE_ERR_CUDA;
  if (launch_bwd<kBwdWgrad2>(b4, grid, st) != cudaSuccess) return MOE_ERR_CUDA;
  BwdParams b5 = bp;
  if (!make_map(&b5.tm_a, x, H, T, H, 64) || !make_map(&b5.tm_b, dl, NE, T, NE, 64)) return MOE_ERR_CUDA;
  if (launch_bwd<kBwdDwg>(b5, grid, st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_plan_set_cta_pairs(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  if (enable && p->pair_clusters < 1) return MOE_ERR_UNSUPPORTED_SHAPE;
  p->cta_pairs = enable != 0;
  return MOE_OK;
}

int moe_plan_set_task_order(moe_plan_t p, int mode) {
  if (p == nullptr || mode < -1 || mode > 1) return MOE_ERR_INVALID_ARG;
  p->task_order = mode;
  return MOE_OK;
}

int moe_plan_set_task_log(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  p->task_log = enable != 0;
  p->L = make_layout(*p);
  p->ws = nullptr;   // the workspace size changed: bind again
  p->ws_bytes = 0;
  return MOE_OK;
}

int moe_plan_get_task_log(moe_plan_t p, const moe_task_record** records, int* capacity) {
  if (p == nullptr || records == nullptr || capacity == nullptr) return MOE_ERR_INVALID_ARG;
  if (!p->task_log) return MOE_ERR_INVALID_ARG;
  if (p->ws == nullptr) return MOE_ERR_NO_WORKSPACE;
  *records = reinterpret_cast<const moe_task_record*>(p->ws + p->L.task_log);
  *capacity = task_log_capacity(*p);
  return MOE_OK;
}

int moe_plan_set_wide_l1(moe_plan_t p, int mode) {
  if (p == nullptr || mode < -1 || mode > 1) return MOE_ERR_INVALID_ARG;
  p->wide_l1 = mode;
  return MOE_OK;
}

int moe_plan_set_half_tails(moe_plan_t p, int enable) {
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  p->half_tails = enable != 0;
  return MOE_OK;
}

int moe_forward_kernel_count(void) { return kNumKernels; }

int moe_plan_forward_launches(moe_plan_t p, int fp8) {
  if (p == nullptr) return -1;
  if (fp8 == 0) return kNumKernels;
  if (p->fp8_rows == 0) return -1;
  // the x quantizer, then per block group the first GEMM, the activation quantizer and the second
  const int fp8_units = std::max(1, p->fp8_rows / (p->cta_pairs ? 2 * p->BM : p->BM));
  const int fp8_groups = (p->blocks_max + fp8_units - 1) / fp8_units;
  return kNumKernels - 1 + 1 + 3 * fp8_groups;
}

void moe_plan_destroy(moe_plan_t p) {
  if (p == nullptr) return;
  {
    DeviceGuard guard(p->device);
    for (auto& e : p->ev) cudaEventDestroy(e);
    if (p->cp_in != nullptr) {
      cudaStreamSynchronize(p->cp_in);
      cudaStreamSynchronize(p->cp_out);
      for (int b = 0; b < 2; ++b) {
        cudaEventDestroy(p->ev_in[b]);
        cudaEventDestroy(p->ev_done[b]);
        cudaEventDestroy(p->ev_out[b]);
      }
      cudaEventDestroy(p->ev_mark);
      cudaStreamDestroy(p->cp_in);
      cudaStreamDestroy(p->cp_out);
    }
  }
  delete p;
}

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_NO_WORKSPACE: return "no workspace bound";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "routing index out of range on the device";
    case MOE_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    case MOE_ERR_STATIC_SCRATCH_LIMIT: return "sizes exceed the fixed scratch of moe_route_static";
    default: return "unknown status";
  }
}

}  // extern "C"
