// Persistent grouped GEMM over the expert blocks: phase L1 (x W1, x W3 with a
// fused SwiGLU epilogue, bf16 h out) and phase L2 (h W2 with the combine's
// gate-weighted scatter-add fused into the epilogue).
//
// Prior art this follows, re-done for one B200:
// * "FlashMoE Kernel", section "架构": one persistent kernel whose blocks run
//   tile tasks t = (M, *, phi); the two FFN matmuls and the combine's Hadamard
//   weighting are fused device routines. Here a task is (phase, expert,
//   m-block, n-tile).
// * "MegaMoE 在 MoE 系统谱系中的位置", section 2.1: warp roles inside the CTA
//   (dispatch/activation loads, weight TMA, MMA issue, scheduler, epilogue).
//   Here warp 0 is the TMA producer of the weight tiles, warp 1 issues
//   tcgen05 MMAs, warps 2-5 drain TMEM in the epilogue, warps 6.. load the
//   A rows (routed x rows in L1, the block's h rows in L2), and the last
//   warp is the scheduler: it claims, decodes and prepares the next task.
// * Same page, section 2.7: tasks are claimed from a global atomic counter,
//   and an L2 task of pool block b waits on an in-kernel counter until the L1
//   tasks of block b are complete (bounded wait here).
// * Same page, section 2.4: the slot's (token, top-k) record gives the
//   combine's write address from the epilogue.
// * ScatterMoE idea on the same page, section 一: the token gather is fused
//   into the operand load, no permuted copy of x. The routed x rows are
//   fetched with 16-byte cp.async by the gather warps straight into the
//   128-byte-swizzled K-major tile (a 4-row TMA gather costs far more TMA
//   time than its 512 bytes are worth at this tile shape, and one warp of
//   cp.async cannot keep up either); the weight tiles use TMA.
//
// The kernel is a template over the operand type: bf16 (kind::f16), or FP8 E4M3
// (kind::f8f6f4: x, W1/W3, W2 and the activation as K-major codes, 128 K
// elements per stage in the same 128-byte swizzle; token, column and
// activation-row scales applied in the epilogues). The FP8 forward launches it
// twice, first GEMM only and then second GEMM only (see GemmParams).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace moe {

struct GemmParams {
  const bf16* x;       // [T, H]
  CUtensorMap tm_w1;   // W1 as [E*H, I], box {64, 64}; FP8: W1q as [E*I, H] bytes, box {128, 64}
  CUtensorMap tm_w3;   // W3 likewise
  CUtensorMap tm_w2;   // W2 as [E*I, H], box {64, 64}; FP8: W2q as [E*H, I] bytes, box {128, 64}
  CUtensorMap tm_ws1;  // shared experts' W1 as [S*H, I] (experts E .. E+S-1; unused when S = 0)
  CUtensorMap tm_ws3;  // shared experts' W3 as [S*H, I]
  CUtensorMap tm_ws2;  // shared experts' W2 as [S*I, H]
  const int32_t* slot_token;
  const int32_t* slot_topk;
  const float* topk_w;
  const int32_t* block_start;   // [E+S+1]
  const int32_t* group_start;   // [groups + 1] first block of each block group
  const int32_t* num_groups;    // [1]
  int32_t* task_counter;
  int32_t* l1_done;             // [blocks] 4 arrivals per L1 n-tile of the block
  int32_t* l2_done;             // [blocks] 1 arrival per L2 n-tile of the block
  int32_t* err;                 // [0] code, [1] detail
  bf16* h;                      // ring of ring_blocks blocks of BM rows x I
  float* y_acc;                 // [T, H]
  int T, H, I, E, k, BM, BN2, N1, N2;
  int S;                        // shared experts (0 .. kMaxShared)
  // FP8 E4M3 expert GEMMs (the kernel's FP8 instance): x codes [T, H] with per-token scales,
  // W1/W3 codes K-major [E, I, H] with column scales [E, I], W2 codes K-major
  // [E, H, I] with column scales [E, H] (tensor maps above). The two GEMMs run
  // as two launches per block group (phase_only 0, then 1) around the activation quantizer:
  // the first stores the bf16 activation in h and raises act_amax of its row
  // (zero before the launch) to the row's largest |h|; the quantizer writes
  // the row's codes to h8 and its scale to act_scale; the second reads them.
  const uint8_t* xq;
  const float* sx;
  const float* s1;
  const float* s3;
  const float* s2;
  float* act_amax;           // [h rows]
  const float* act_scale;    // [h rows]
  const uint8_t* h8;         // [h rows, I]
  int phase_only;            // -1: both phases in one launch; 0: first GEMM only; 1: second GEMM only
  int only_group;            // with phase_only >= 0: the block group whose tasks this launch runs
  int ring_blocks;              // block b uses ring slot b % ring_blocks
  int max_groups;
  int order_lag;                // task order (see locate_task): -1 staggered, >= 0 interleaved after this lag
  TaskRecord* task_log;         // one record per task of the launch, or null (no log)
  int task_log_cap;
  const uint8_t* zero_row;      // 2*H zero bytes: the A row of a padding slot
  unsigned long long timeout_ns;
  int withhold_block;           // test hook: never publish L1 completion of this block (-1: off)
};

struct Task {
  int phase;   // 0 = L1, 1 = L2, -1 = no more work
  int e, b, n;
  int id;      // task number (the claimed counter value)
};

struct GemmSmem {
  // L2 epilogue staging, per epilogue warp: 32 rows x 32 fp32 (rows padded to
  // 144 B so that row-wise and transposed 16-byte accesses are conflict-free),
  // and the token of each staged row.
  float out_stage[4][32][36];
  int out_tok[4][32];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t task_full[kTaskRing];
  uint64_t task_empty[kTaskRing];
  uint64_t mma_done;
  Task tasks[kTaskRing];
  uint32_t tmem_base;
  int abort;
  int taken;                     // tasks the producer has taken from the ring
  int num_groups;
  int rows[kTaskRing][kTileM];   // token row of each A-tile row, per task-ring slot (L1 tasks)
  int block_start[kMaxExpertsAll + 1];
  int group_start[kMaxGroups + 1];
};

static_assert(offsetof(GemmSmem, out_stage) % 16 == 0, "staging rows are read as float4");
static_assert((36 * 4) % 16 == 0, "staging rows must stay 16-byte aligned");

constexpr size_t kGemmSmemBytes = 1024 /*alignment slack*/ + (size_t)kStages * kStageBytes + sizeof(GemmSmem);

__device__ __forceinline__ void set_error(const GemmParams& p, GemmSmem& s, int code, int detail) {
  if (atomicCAS(p.err, 0, code) == 0) p.err[1] = detail;
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
}

// Bounded wait of a whole warp on an mbarrier phase. All lanes agree on the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const GemmParams& p, GemmSmem& s,
                                          int where) {
  bool ok = ptx::mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
      if (ptx::mbar_try_wait(bar, parity)) {
        ok = true;
        break;
      }
      if (*reinterpret_cast<volatile int*>(&s.abort)) break;
      if (ptx::globaltimer() - t0 > p.timeout_ns) {
        set_error(p, s, kDevTimeout, where);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Task order. Blocks are cut into groups (expert-aligned where possible) and
// the phases interleave with a lag of one group:
//   L1(0), L1(1), L2(0), L1(2), L2(1), ..., L1(G-1), L2(G-2), L2(G-1)
// so that L2 tasks of a group start once its L1 tasks have had a whole
// segment to finish, and the h ring only has to hold a few groups. Segment
// s: s = 0 is L1(0); s = 2g-1 is L1(g) and s = 2g is L2(g-1) for g = 1..G
// (L1(G) is empty). Inside a segment the order is (expert, n-tile, m-block)
// so that the m-blocks sharing a weight slice run side by side.
// Bounded wait (one thread) until *ctr >= need, with acquire semantics.
__device__ __forceinline__ bool wait_counter(const int* ctr, int need, const GemmParams& p, GemmSmem& s,
                                             int detail) {
  if (ptx::ld_acquire_gpu(ctr) >= need) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::ld_acquire_gpu(ctr) < need) {
    if (*reinterpret_cast<volatile int*>(&s.abort) || *reinterpret_cast<volatile int*>(p.err) != 0) return false;
    if (ptx::globaltimer() - t0 > p.timeout_ns) {
      set_error(p, s, kDevTimeout, detail);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}

// Where task t falls in the task order: its phase (0 = L1, 1 = L2), its group
// g and its index tl among that phase's tasks of group g. Group g holds the
// units (blocks, or block pairs) gs[g] .. gs[g+1]-1 and has (gs[g+1]-gs[g])*N1
// L1 tasks and (..)*N2 L2 tasks. The L2 tasks of a group always come after
// every L1 task of that group and before the L1 tasks of the group two later
// (whose h rows reuse its ring slots). Two orders:
//
// * staggered (lag < 0): L1(0), L1(1), L2(0), L1(2), L2(1), ..., L2(G-1);
// * interleaved (lag >= 0): L1(0), then for m = 1..G-1 one segment that
//   starts with `lag` L1 tasks of group m (so that the last L1 tasks of group
//   m-1 have finished) and then mixes the rest of L1(m) with L2(m-1) evenly
//   (Bresenham: L2 task c is the v-th of the mixed part when
//   floor(v*n2/R) = c < floor((v+1)*n2/R)), then L2(G-1). A CTA then
//   alternates long-K first-GEMM tasks with second-GEMM tasks whose
//   combine epilogue would otherwise outlast their short MMAs.
struct TaskPos {
  int phase, g, tl;
};

__device__ __forceinline__ TaskPos locate_task(int t, const int* gs, int G, int N1, int N2, int lag) {
  if (lag < 0) {
    // segment 0 = L1(0); odd 2g-1 = L1(g); even 2g = L2(g-1)
    auto start = [&](int seg) {
      if (seg == 0) return 0;
      const int g = (seg + 1) >> 1;
      if (seg & 1) return gs[g] * N1 + gs[g - 1] * N2;
      return gs[min(g + 1, G)] * N1 + gs[g - 1] * N2;
    };
    int lo = 0, hi = 2 * G;   // last segment whose start is <= t (empty segments share the next start)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start(mid) <= t) lo = mid;
      else hi = mid - 1;
    }
    const int seg = lo;
    if (seg == 0 || (seg & 1)) return TaskPos{0, (seg + 1) >> 1, t - start(seg)};
    return TaskPos{1, (seg >> 1) - 1, t - start(seg)};
  }
  // segment m >= 1 starts after every L1 task of groups < m and every L2 task of groups < m-1
  auto start = [&](int m) { return m == 0 ? 0 : gs[m] * N1 + gs[m - 1] * N2; };
  int lo = 0, hi = G;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start(mid) <= t) lo = mid;
    else hi = mid - 1;
  }
  const int m = lo;
  const int u = t - start(m);
  if (m == 0) return TaskPos{0, 0, u};
  const int n1 = m < G ? (gs[m + 1] - gs[m]) * N1 : 0;
  const int n2 = (gs[m] - gs[m - 1]) * N2;
  const int l = min(lag, n1);
  if (u < l) return TaskPos{0, m, u};
  const long long v = u - l, R = (long long)(n1 - l) + n2;
  const int c2 = (int)(v * n2 / R);
  const int c2_next = (int)((v + 1) * n2 / R);
  if (c2_next > c2) return TaskPos{1, m - 1, c2};
  return TaskPos{0, m, l + (int)v - c2};
}

__device__ __forceinline__ Task decode_task(int t, const GemmSmem& s, const GemmParams& p) {
  Task task{-1, 0, 0, 0, 0};
  const int G = s.num_groups;
  const int nb_total = s.block_start[p.E + p.S];
  // one-phase launches (a single block group): the second GEMM's tasks follow the first's
  TaskPos pos;
  if (p.phase_only >= 0) {
    // one GEMM of one block group (the FP8 forward's launches): its tasks in order
    const int g = p.only_group;
    if (g < 0 || g >= G) return task;
    const int NT = p.phase_only == 0 ? p.N1 : p.N2;
    if (t < 0 || t >= (s.group_start[g + 1] - s.group_start[g]) * NT) return task;
    pos = TaskPos{p.phase_only, g, t};
  } else {
    if (t < 0 || t >= nb_total * (p.N1 + p.N2) || G <= 0) return task;
    pos = locate_task(t, s.group_start, G, p.N1, p.N2, p.order_lag);
  }
  task.phase = pos.phase;
  const int g = pos.g, NT = pos.phase == 0 ? p.N1 : p.N2;
  const int gb0 = s.group_start[g], gb1 = s.group_start[g + 1];
  const int tl = pos.tl;
  // expert of the tl-th task: its blocks inside the group occupy consecutive NT-task runs
  const int vb = gb0 + tl / NT;
  int elo = 0, ehi = p.E + p.S - 1;
  while (elo < ehi) {
    const int mid = (elo + ehi + 1) >> 1;
    if (s.block_start[mid] <= vb) elo = mid;
    else ehi = mid - 1;
  }
  const int e = elo;
  const int eb0 = max(gb0, s.block_start[e]);
  const int eb1 = min(gb1, s.block_start[e + 1]);
  const int nb = eb1 - eb0;
  const int local = tl - (eb0 - gb0) * NT;
  task.e = e;
  task.n = local / nb;
  task.b = eb0 + (local - task.n * nb);
  task.id = t;
  return task;
}

__device__ __forceinline__ uint8_t* stage_ptr(uint8_t* tiles, int stage) { return tiles + stage * kStageBytes; }

// K blocks of an L1 task: 64 bf16 or 128 FP8 elements, one 128-byte swizzle row either way.
template <bool F8>
__device__ __forceinline__ int l1_ksteps(const GemmParams& p) { return F8 ? p.H / 128 : p.H / kBK; }
template <bool F8>
__device__ __forceinline__ int l2_ksteps(const GemmParams& p) { return F8 ? p.I / 128 : p.I / kBK; }

// ---------------------------------------------------------------- scheduler (last warp)
// Claims tasks from the global counter, decodes them, stages the routed row
// indices of L1 tasks in s.rows[q] and waits for the L1 tiles an L2 task
// reads, then publishes the task in ring slot q. Every global round trip of
// the task switch happens here, one task ahead of the producer, so the weight
// stream never pauses for it. It claims the next task only once the producer
// has taken the last one it published: at most one claimed task waits in the
// ring, which keeps the end of the kernel balanced across CTAs.
__device__ __forceinline__ int claim_task(const GemmParams& p, GemmSmem& s, int lane) {
  int t = 0x7fffffff;
  if (lane == 0) {
    const bool stop =
        *reinterpret_cast<volatile int*>(&s.abort) || *reinterpret_cast<volatile int*>(p.err) != 0;
    if (!stop) t = atomicAdd(p.task_counter, 1);
  }
  return __shfl_sync(0xffffffffu, t, 0);
}

// Bounded wait (one thread) until the producer has taken `n` tasks.
__device__ __forceinline__ bool wait_taken(int n, const GemmParams& p, GemmSmem& s) {
  if (*reinterpret_cast<volatile int*>(&s.taken) >= n) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (*reinterpret_cast<volatile int*>(&s.taken) < n) {
    if (*reinterpret_cast<volatile int*>(&s.abort)) return false;
    if (ptx::globaltimer() - t0 > p.timeout_ns) {
      set_error(p, s, kDevTimeout, 10);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

template <bool F8>
__device__ void gemm_scheduler(const GemmParams& p, GemmSmem& s) {
  const int lane = ptx::lane_id();
  int q = 0;
  uint32_t qphase = 0;
  int pushed = 0;
  while (true) {
    bool ok = true;
    if (lane == 0) ok = wait_taken(pushed, p, s);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    Task task{-1, 0, 0, 0, 0};
    if (ok) task = decode_task(claim_task(p, s, lane), s, p);
    if (!warp_wait(&s.task_empty[q], qphase ^ 1, p, s, 1)) break;
    if (task.phase == 0) {
      // all loads first (one round trip), then the checks
      constexpr int kPer = kTileM / 32;
      int tok[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int r = lane + 32 * i;
        tok[i] = r < p.BM ? p.slot_token[task.b * p.BM + r] : 0;
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int r = lane + 32 * i;
        if (r < p.BM) {
          if (tok[i] >= p.T) {
            set_error(p, s, kDevBounds, task.b);
            tok[i] = 0;
          }
          s.rows[q][r] = tok[i] < 0 ? -1 : tok[i];   // padding slot: the gather fills the row with zeros
        }
      }
    } else if (task.phase == 1) {
      // the L2 task of block b reads h rows written by all L1 n-tiles of block b
      // (one arrival per epilogue warp per n-tile)
      bool fine = true;
      if (lane == 0) fine = wait_counter(p.l1_done + task.b, 4 * p.N1, p, s, 0x10000 | task.b);
      if (__shfl_sync(0xffffffffu, fine ? 1 : 0, 0) == 0) task.phase = -1;
    }
    __syncwarp();
    if (lane == 0) {
      s.tasks[q] = task;
      ptx::mbar_arrive(&s.task_full[q]);
    }
    __syncwarp();
    ++pushed;
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;
  }
}

// ---------------------------------------------------------------- producer (warp 0)
// Weight-tile TMA (and the h tiles of L2 tasks) for the tasks the scheduler publishes.
template <bool F8>
__device__ void gemm_producer(const GemmParams& p, GemmSmem& s, uint8_t* tiles) {
  const int lane = ptx::lane_id();
  // Weight tiles are streamed: the few m-blocks sharing a slice read it at
  // nearly the same time, so mark it first to evict.
  const uint64_t pol = ptx::policy_evict_first();
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  uint32_t issued = 0, issued_parity = 0;   // per stage: ever issued, parity of the last issue
  bool ok = true;
  while (ok) {
    if (!warp_wait(&s.task_full[q], qphase, p, s, 11)) break;
    const Task task = s.tasks[q];
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive(&s.task_empty[q]);
      *reinterpret_cast<volatile int*>(&s.taken) = *reinterpret_cast<volatile int*>(&s.taken) + 1;
    }
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;

    const int nk = task.phase == 0 ? l1_ksteps<F8>(p) : l2_ksteps<F8>(p);
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait(&s.empty[stage], phase ^ 1, p, s, 2)) {
        ok = false;
        break;
      }
      const uint32_t a_addr = ptx::smem_u32(stage_ptr(tiles, stage));
      const uint32_t b_addr = a_addr + kTileABytes;
      if (task.phase == 0) {
        // B: 128 columns of W1 next to the same 128 of W3; A comes from the gather warps.
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&s.full[stage], 4 * kBoxBytes);
          const int n0 = task.n * kL1TileN;
          if (F8) {
            // K-major FP8 codes: 64 rows (columns of I) x 128 bytes (K) per box
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ptx::tma_load_2d(b_addr + j * kBoxBytes, j < 2 ? &p.tm_w1 : &p.tm_w3, &s.full[stage], kb * 128,
                               task.e * p.I + n0 + (j & 1) * 64, pol);
          } else {
            const bool sh = task.e >= p.E;   // shared expert: its own weight tensors
            const int wrow = (sh ? task.e - p.E : task.e) * p.H + kb * kBK;
            const CUtensorMap* m1 = sh ? &p.tm_ws1 : &p.tm_w1;
            const CUtensorMap* m3 = sh ? &p.tm_ws3 : &p.tm_w3;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ptx::tma_load_2d(b_addr + j * kBoxBytes, j < 2 ? m1 : m3, &s.full[stage], n0 + (j & 1) * 64, wrow,
                               pol);
          }
        }
      } else {
        // B: 256 (or 128) columns of W2; A (the block's h rows) comes from the gather warps.
        if (lane == 0 && F8) {   // K-major E4M3 codes: BN2 rows of 128 bytes, 64 per box
          const int nbox = p.BN2 / 64;
          ptx::mbar_arrive_expect_tx(&s.full[stage], nbox * kBoxBytes);
          for (int j = 0; j < nbox; ++j)
            ptx::tma_load_2d(b_addr + j * kBoxBytes, &p.tm_w2, &s.full[stage], kb * 128,
                             task.e * p.H + task.n * p.BN2 + j * 64, pol);
        } else if (lane == 0) {
          const int nbox = p.BN2 / 64;
          ptx::mbar_arrive_expect_tx(&s.full[stage], nbox * kBoxBytes);
          const bool sh = task.e >= p.E;
          const int wrow = (sh ? task.e - p.E : task.e) * p.I + kb * kBK;
          for (int j = 0; j < nbox; ++j)
            ptx::tma_load_2d(b_addr + j * kBoxBytes, sh ? &p.tm_ws2 : &p.tm_w2, &s.full[stage], task.n * p.BN2 + j * 64,
                             wrow, pol);
        }
      }
      __syncwarp();
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  // On an early exit, let every issued copy land before the CTA can retire.
  for (int st = 0; st < kStages; ++st)
    if (issued & (1u << st)) {
      const uint32_t par = (issued_parity >> st) & 1u;
      const uint64_t t0 = ptx::globaltimer();
      while (!ptx::mbar_try_wait(&s.full[st], par)) {
        if (ptx::globaltimer() - t0 > p.timeout_ns) break;
      }
    }
}

// ---------------------------------------------------------------- MMA issuer (warp 1)
template <bool F8>
__device__ void gemm_mma(const GemmParams& p, GemmSmem& s, uint8_t* tiles, uint32_t tmem_base) {
  const int lane = ptx::lane_id();
  const uint32_t idesc_l1 =
      F8 ? ptx::idesc_e4m3_f32(128, 2 * kL1TileN) : ptx::idesc_bf16_f32(128, 2 * kL1TileN, false, true);
  constexpr bool f8 = F8;
  const uint32_t idesc_l2 = F8 ? ptx::idesc_e4m3_f32(128, p.BN2) : ptx::idesc_bf16_f32(128, p.BN2, false, true);
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool issued_any = false;
  while (true) {
    if (!warp_wait(&s.task_full[q], qphase, p, s, 3)) break;
    const Task task = s.tasks[q];
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&s.task_empty[q]);
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;
    if (!warp_wait(&s.acc_empty[acc], acc_phase ^ 1, p, s, 4)) break;
    ptx::tc_fence_after();
    const uint32_t d_tmem = tmem_base + acc * 256;
    const uint32_t idesc = task.phase == 0 ? idesc_l1 : idesc_l2;
    const int nk = task.phase == 0 ? l1_ksteps<F8>(p) : l2_ksteps<F8>(p);
    bool ok = true;
    uint64_t t_first = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait(&s.full[stage], phase, p, s, 5)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      ptx::fence_proxy_async_shared();   // cp.async-written A rows -> tensor-core reads
      if (kb == 0) t_first = ptx::globaltimer();
      if (lane == 0) {
        const uint32_t a_addr = ptx::smem_u32(stage_ptr(tiles, stage));
        const uint32_t b_addr = a_addr + kTileABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // A: K-major, 128-byte rows, 8-row groups 1024 B apart; step 32 B along K
          // (16 bf16 or 32 FP8 elements per MMA).
          const uint64_t ad = ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          if (f8) {
            // B: K-major FP8 codes (W1 | W3, or W2), rows of 128 bytes
            const uint64_t bd = ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            ptx::mma_f8(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          } else {
            // B: MN-major, 64-column boxes 8 KB apart, 8-row K groups 1024 B apart; step 16 rows = 2 KB.
            const uint64_t bd = ptx::smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            ptx::mma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
        }
        ptx::mma_commit(&s.empty[stage]);
        issued_any = true;
      }
      __syncwarp();
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
    if (lane == 0) ptx::mma_commit(&s.acc_full[acc]);
    if (lane == 0 && p.task_log != nullptr && task.id < p.task_log_cap) {
      TaskRecord* r = p.task_log + task.id;
      r->task = task.id;
      r->unit = task.b;
      r->expert = task.e;
      r->phase_n = ((uint32_t)task.phase << 16) | (uint32_t)task.n;
      r->smid = smid_u32();
      r->cta = blockIdx.x;
      r->t_first_mma = t_first;
      r->t_last_mma = ptx::globaltimer();
    }
    __syncwarp();
    if (++acc == 2) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
  // Every MMA must have finished before TMEM is released.
  issued_any = __any_sync(0xffffffffu, issued_any);
  if (issued_any) {
    if (lane == 0) ptx::mma_commit(&s.mma_done);
    __syncwarp();
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(&s.mma_done, 0)) {
      if (ptx::globaltimer() - t0 > p.timeout_ns) break;
    }
  }
}

// ---------------------------------------------------------------- A-row warps (warps 6 .. 6+G-1)
// L1 tasks: the A tile is BM routed rows of x, 64 columns per stage. Warp
// instruction i (4 rows x 128 B, one 16-byte chunk per lane) is issued by
// gather warp i % G; chunk c of row r lands at chunk c ^ (r % 8) of the
// row's 128 bytes, the 128-byte swizzle the MMA descriptor expects. Every
// lane arrives on the stage's full barrier when its own copies have landed.
// L2 tasks: the same for the block's BM rows of h in the ring (a single
// 128-row TMA box per stage kept the tensor pipe waiting twice as long).
template <bool F8>
__device__ void gemm_gather(const GemmParams& p, GemmSmem& s, uint8_t* tiles, int g) {
  constexpr int kRowsPerLane = (kTileM / 4 + kGatherWarps - 1) / kGatherWarps;   // rows >= BM are skipped
  const int lane = ptx::lane_id();
  const int c = lane & 7;
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  while (true) {
    if (!warp_wait(&s.task_full[q], qphase, p, s, 8)) break;
    const Task task = s.tasks[q];
    const int q_task = q;
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;
    // smem offset and source row of each of this lane's rows: L1, the routed x
    // rows (indices staged by the scheduler); L2, the block's h rows in the ring
    // (byte addresses: a stage takes the next 128 bytes of every row, 64 bf16 or 128 FP8 codes)
    int nrows = 0;
    uint32_t soff[kRowsPerLane];
    const uint8_t* src[kRowsPerLane];
    const int* rows = s.rows[q_task];
    // activation rows: bf16, or FP8 codes (rows of I bytes); x rows: bf16, or FP8 codes
    const size_t hpitch = F8 ? (size_t)p.I : (size_t)p.I * 2;
    const int ring_row0 = (task.b % p.ring_blocks) * p.BM;
    const uint8_t* hblock = (F8 ? p.h8 : reinterpret_cast<const uint8_t*>(p.h)) + (size_t)ring_row0 * hpitch;
    const uint8_t* xrows = F8 ? p.xq : reinterpret_cast<const uint8_t*>(p.x);
    const size_t xpitch = F8 ? (size_t)p.H : (size_t)p.H * 2;
#pragma unroll
    for (int j = 0; j < kRowsPerLane; ++j) {
      const int r = (j * kGatherWarps + g) * 4 + (lane >> 3);
      soff[j] = r * 128 + ((c ^ (r & 7)) << 4);
      src[j] = xrows + c * 16;
      if (r < p.BM) {
        // L1 padding slots (row index -1) read the all-zero row: the tensor core
        // multiplies zeros and their h rows come out 0 for the L2 tasks
        const int xr = rows[r];
        src[j] = task.phase == 1 ? hblock + (size_t)r * hpitch + c * 16
                 : xr < 0        ? p.zero_row + c * 16
                                 : xrows + (size_t)xr * xpitch + c * 16;
        nrows = j + 1;
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&s.task_empty[q_task]);   // slot (and its rows) free
    const int nk = task.phase == 0 ? l1_ksteps<F8>(p) : l2_ksteps<F8>(p);
    bool ok = true;

    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait(&s.empty[stage], phase ^ 1, p, s, 9)) {
        ok = false;
        break;
      }
      const uint32_t a_addr = ptx::smem_u32(stage_ptr(tiles, stage));
#pragma unroll
      for (int j = 0; j < kRowsPerLane; ++j)
        if (j < nrows) ptx::cp_async_16(a_addr + soff[j], src[j] + (size_t)kb * 128);
      ptx::cp_async_mbar_arrive_noinc(&s.full[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
  }
  ptx::cp_async_wait_all();
}

// silu(g) * u = g / (1 + e^-g) * u. The division is the fast one (__fdividef, within 2 ulp; it
// returns 0 once 1 + e^-g passes 2^126, where silu(g) is 0 to fp32 precision): an IEEE division
// here made the first GEMM's epilogue the slowest role of the FP8 kernels.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// FP8 first GEMM: g[i] *= tscale * (column i's W1 scale), u[i] *= tscale * (W3 scale) for the
// 32 columns of a chunk; lane j holds column j's scales (sa, sb) and shuffles them to the warp.
__device__ __forceinline__ void fp8_scale_columns_shfl(uint32_t (&g)[32], uint32_t (&u)[32], float tscale, float sa,
                                                       float sb) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    g[i] = __float_as_uint(__uint_as_float(g[i]) * (tscale * __shfl_sync(0xffffffffu, sa, i)));
    u[i] = __float_as_uint(__uint_as_float(u[i]) * (tscale * __shfl_sync(0xffffffffu, sb, i)));
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// h[0..31] = bf16(silu(g) * u) for one row's 32 columns; amax = max(amax, |silu(g) * u|).
__device__ __forceinline__ void store_swiglu32(bf16* dst, const uint32_t (&g)[32], const uint32_t (&u)[32],
                                               float& amax) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[i] = silu_mul(__uint_as_float(g[8 * v + i]), __uint_as_float(u[8 * v + i]));
      amax = fmaxf(amax, fabsf(f[i]));
    }
    d4[v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                       pack_bf16x2(f[6], f[7]));
  }
}

// FP8: raise the row's activation amax (non-negative floats order as their bits) to `amax`,
// the largest |h| of this task's columns (bf16 rounding is monotonic: the rounded maximum
// is the maximum of the rounded values).
__device__ __forceinline__ void publish_act_amax(float* act_amax, int row, float amax) {
  atomicMax(reinterpret_cast<unsigned int*>(act_amax + row), __float_as_uint(__bfloat162float(__float2bfloat16_rn(amax))));
}

// Combine of one epilogue warp's 32 accumulator rows (TMEM lanes tbase..+31,
// columns 0..ncols-1, ncols a multiple of 64): y_acc[tok_r][c] += w_r *
// acc[r][c] for every row r with tok_r >= 0. Each lane holds row `lane`; per
// 32 columns the warp stages w*acc in shared memory (rows padded to 36 floats,
// conflict-free both ways) and reads it back transposed, so that 8 lanes
// cover one row's 128 contiguous bytes and every red.v4 instruction adds 4
// whole 128-byte row segments. The TMEM load of the next 32 columns is in
// flight while the current ones are staged and reduced, and `release()` runs
// as soon as the last TMEM load has landed, so the MMA warp can reuse the
// accumulator while the last reductions are still being issued.
__device__ __forceinline__ void combine_stage_and_reduce(const uint32_t (&v)[32], int c, float w, float* srow,
                                                         float (*stage)[36], float* const (&ybase)[8], int sub,
                                                         int cc, const float* cs, float csl) {
  // FP8 W2: scales of the lane's 4 transposed columns, from the lanes that hold them (lane j: column j)
  float4 m = make_float4(1.f, 1.f, 1.f, 1.f);
  if (cs != nullptr)
    m = make_float4(__shfl_sync(0xffffffffu, csl, cc), __shfl_sync(0xffffffffu, csl, cc + 1),
                    __shfl_sync(0xffffffffu, csl, cc + 2), __shfl_sync(0xffffffffu, csl, cc + 3));
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(srow)[i] =
        make_float4(w * __uint_as_float(v[4 * i + 0]), w * __uint_as_float(v[4 * i + 1]),
                    w * __uint_as_float(v[4 * i + 2]), w * __uint_as_float(v[4 * i + 3]));
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (ybase[i] != nullptr) {
      float4 a = *reinterpret_cast<const float4*>(&stage[i * 4 + sub][cc]);
      if (cs != nullptr) a = make_float4(a.x * m.x, a.y * m.y, a.z * m.z, a.w * m.w);
      ptx::red_add_v4_f32(ybase[i] + c * 32, a);
    }
  __syncwarp();
}

template <typename Release>
__device__ __forceinline__ void combine_rows(uint32_t tbase, int ncols, float w, int tok, float* y_acc, int H,
                                             int col0, float (*stage)[36], int* stage_tok, const float* cs,
                                             Release release) {
  const int lane = ptx::lane_id();
  stage_tok[lane] = tok;
  __syncwarp();
  const int sub = lane >> 3;
  const int cc = (lane & 7) * 4;
  float* ybase[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = stage_tok[i * 4 + sub];
    ybase[i] = t >= 0 ? y_acc + (size_t)t * H + col0 + cc : nullptr;
  }
  float* srow = stage[lane];
  // FP8 W2: this lane holds the scale of column 32c + lane of the two chunks in hand, and
  // loads those of the next two while they are reduced
  float csa = 1.f, csb = 1.f;
  if (cs != nullptr) {
    csa = __ldg(cs + lane);
    csb = __ldg(cs + 32 + lane);
  }
  uint32_t va[32], vb[32];
  ptx::tmem_ld32(tbase, va);
#pragma unroll 1
  for (int c = 0; c < ncols / 32; c += 2) {
    float nca = 1.f, ncb = 1.f;
    if (cs != nullptr && c + 2 < ncols / 32) {
      nca = __ldg(cs + (c + 2) * 32 + lane);
      ncb = __ldg(cs + (c + 3) * 32 + lane);
    }
    ptx::tmem_ld_wait();                                         // va holds columns 32c ..
    ptx::tmem_ld32(tbase + (c + 1) * 32, vb);
    combine_stage_and_reduce(va, c, w, srow, stage, ybase, sub, cc, cs, csa);
    ptx::tmem_ld_wait();                                         // vb holds columns 32(c+1) ..
    if (c + 2 < ncols / 32) ptx::tmem_ld32(tbase + (c + 2) * 32, va);
    else release();                                              // no TMEM reads left
    combine_stage_and_reduce(vb, c + 1, w, srow, stage, ybase, sub, cc, cs, csb);
    csa = nca;
    csb = ncb;
  }
}

// ---------------------------------------------------------------- epilogue (warps 2..5)
template <bool F8>
__device__ void gemm_epilogue(const GemmParams& p, GemmSmem& s, uint32_t tmem_base) {
  const int warp = threadIdx.x >> 5;
  const int lane = ptx::lane_id();
  const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
  const int r = quarter * 32 + lane;         // tile row of this thread
  int q = 0;
  uint32_t qphase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  while (true) {
    if (!warp_wait(&s.task_full[q], qphase, p, s, 6)) break;
    const Task task = s.tasks[q];
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&s.task_empty[q]);
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;
    // FP8: the task's scales, loaded before the accumulator wait (lane j: column 32c + j of chunk c)
    float tscale = 0.f, rscale = 1.f, sa[4] = {1.f, 1.f, 1.f, 1.f}, sb[4] = {1.f, 1.f, 1.f, 1.f};
    if (F8 && task.phase == 0) {
      const size_t col0 = (size_t)task.e * p.I + task.n * kL1TileN;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sa[c] = __ldg(p.s1 + col0 + c * 32 + lane);
        sb[c] = __ldg(p.s3 + col0 + c * 32 + lane);
      }
      if (r < p.BM) {   // the token's scale (padding rows: 0, so their activation is 0)
        const int tok = p.slot_token[task.b * p.BM + r];
        tscale = (tok >= 0 && tok < p.T) ? __ldg(p.sx + tok) : 0.f;
      }
    } else if (F8 && r < p.BM) {
      rscale = __ldcg(p.act_scale + (task.b % p.ring_blocks) * p.BM + r);   // the activation row's scale
    }
    if (!warp_wait(&s.acc_full[acc], acc_phase, p, s, 7)) break;
    ptx::tc_fence_after();
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 256;
    const bool valid = r < p.BM;
    const int slot = task.b * p.BM + r;
    if (task.phase == 0) {
      // Ring slot of block b; its previous user, block b - ring_blocks, must
      // have been read by all of its L2 n-tiles before it is overwritten.
      bool store = valid;
      if (task.b >= p.ring_blocks) {
        bool ok = true;
        if (lane == 0) ok = wait_counter(p.l2_done + (task.b - p.ring_blocks), p.N2, p, s, 0x40000 | task.b);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        store = store && ok;
      }
      const int ring_row = (task.b % p.ring_blocks) * p.BM + r;
      bf16* hrow = p.h + (size_t)ring_row * p.I + task.n * kL1TileN;
      float amax = 0.f;     // FP8: the row's largest |h| over this task's columns
#pragma unroll 1
      for (int c = 0; c < kL1TileN / 32; ++c) {
        uint32_t g[32], u[32];
        ptx::tmem_ld32(tbase + c * 32, g);
        ptx::tmem_ld32(tbase + kL1TileN + c * 32, u);
        ptx::tmem_ld_wait();
        if (F8)
          fp8_scale_columns_shfl(g, u, tscale, c == 0 ? sa[0] : c == 1 ? sa[1] : c == 2 ? sa[2] : sa[3],
                                 c == 0 ? sb[0] : c == 1 ? sb[1] : c == 2 ? sb[2] : sb[3]);
        if (store) store_swiglu32(hrow + c * 32, g, u, amax);
      }
      if (F8 && store) publish_act_amax(p.act_amax, ring_row, amax);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.acc_empty[acc]);
      // Publish per warp (no cross-warp barrier): this warp's 32 h rows of the
      // (block, n-tile) are written. Block b is complete at 4 * N1 arrivals.
      __threadfence();
      __syncwarp();
      if (lane == 0 && task.b != p.withhold_block) ptx::red_release_gpu_add(p.l1_done + task.b, 1);
    } else {
      // This task's MMAs are complete, so its h tiles have been read: one
      // arrival on the block's L2 counter frees the ring slot once all N2 land.
      if (quarter == 0 && lane == 0) ptx::red_release_gpu_add(p.l2_done + task.b, 1);
      int tok = -1;
      float w = 0.f;
      if (valid) {
        tok = p.slot_token[slot];
        if (tok >= p.T) {
          set_error(p, s, kDevBounds, 0x20000 | task.b);
          tok = -1;
        }
        if (tok >= 0) {
          const int j = p.slot_topk[slot];
          if (task.e >= p.E) {
            w = 1.f;   // shared expert: every token, weight 1
          } else if (j < 0 || j >= p.k) {
            set_error(p, s, kDevBounds, 0x30000 | task.b);
            tok = -1;
          } else {
            w = p.topk_w[(size_t)tok * p.k + j];
          }
        }
      }
      // FP8: o = acc * (activation scale of the row) * (W2 column scale)
      if (F8 && tok >= 0) w *= rscale;   // FP8: the activation row's scale
      // Combine: y_acc[token] += w * o, 128-byte row segments per red.v4 (the L2 does the fp32 adds).
      combine_rows(tbase, p.BN2, w, tok, p.y_acc, p.H, task.n * p.BN2, s.out_stage[quarter], s.out_tok[quarter],
                   F8 ? p.s2 + (size_t)task.e * p.H + task.n * p.BN2 : nullptr, [&]() {
                     ptx::tc_fence_before();
                     __syncwarp();
                     if (lane == 0) ptx::mbar_arrive(&s.acc_empty[acc]);
                   });
    }
    if (p.task_log != nullptr && quarter == 0 && lane == 0 && task.id < p.task_log_cap)
      p.task_log[task.id].t_done = ptx::globaltimer();
    if (++acc == 2) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
}

template <bool F8>
__global__ void __launch_bounds__(kGemm1Threads, 1) moe_expert_gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmem& s = *reinterpret_cast<GemmSmem*>(tiles + (size_t)kStages * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&s.full[i], 1 + 32 * kGatherWarps);   // producer + every gather lane
      ptx::mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.acc_full[i], 1);
      ptx::mbar_init(&s.acc_empty[i], 4);
    }
    for (int i = 0; i < kTaskRing; ++i) {
      ptx::mbar_init(&s.task_full[i], 1);
      ptx::mbar_init(&s.task_empty[i], 6 + kGatherWarps);   // producer, MMA, 4 epilogue warps, gather warps
    }
    ptx::mbar_init(&s.mma_done, 1);
    s.abort = 0;
    s.taken = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&p.tm_w1);
    ptx::prefetch_tmap(&p.tm_w3);
    ptx::prefetch_tmap(&p.tm_w2);
    if (p.S > 0) {
      ptx::prefetch_tmap(&p.tm_ws1);
      ptx::prefetch_tmap(&p.tm_ws3);
      ptx::prefetch_tmap(&p.tm_ws2);
    }
  }
  for (int e = threadIdx.x; e <= p.E + p.S; e += kGemm1Threads) s.block_start[e] = p.block_start[e];
  {
    const int ng = min(*p.num_groups, min(p.max_groups, kMaxGroups));
    if (threadIdx.x == 0) s.num_groups = ng;
    for (int g = threadIdx.x; g <= ng; g += kGemm1Threads) s.group_start[g] = p.group_start[g];
  }
  if (warp == 1) {
    ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  // Rows >= BLOCK_M of the A tiles are never loaded: keep them zero.
  if (p.BM < kTileM) {
    const int row_bytes = 128;
    for (int st = 0; st < kStages; ++st) {
      uint4* a = reinterpret_cast<uint4*>(stage_ptr(tiles, st) + p.BM * row_bytes);
      const int n = (kTileM - p.BM) * row_bytes / 16;
      for (int i = threadIdx.x; i < n; i += kGemm1Threads) a[i] = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_shared();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;

  if (warp == 0) gemm_producer<F8>(p, s, tiles);
  else if (warp == 1) gemm_mma<F8>(p, s, tiles, tmem_base);
  else if (warp < 6) gemm_epilogue<F8>(p, s, tmem_base);
  else if (warp < 6 + kGatherWarps) gemm_gather<F8>(p, s, tiles, warp - 6);
  else gemm_scheduler<F8>(p, s);

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace moe
