// Persistent grouped GEMM over the expert blocks on CTA pairs (tcgen05
// cta_group::2): the same tasks as expert_gemm.cuh (L1 = x W1, x W3 + SwiGLU
// into the h ring; L2 = h W2 + gate-weighted scatter-add combine), but every
// task covers a PAIR of consecutive blocks of one expert, 256 rows, computed
// by the two CTAs of a cluster together:
//
// * each CTA holds its own block's 128 A rows and HALF of the weight tile
//   (L1: CTA 0 the 128 W1 columns, CTA 1 the matching 128 W3 columns; L2:
//   each CTA 128 of the 256 W2 columns), so one weight tile load feeds 256
//   rows and a stage is 32 KB per CTA instead of 48 KB (6 stages fit);
// * the leader CTA (rank 0) claims and prepares tasks in its scheduler warp,
//   publishes them in both CTAs' task rings, issues the MMAs for both CTAs
//   and multicasts its commits to both CTAs' barriers; each CTA's
//   accumulator is its own 128 rows x 256 columns in its own TMEM;
// * L1 weight halves come by TMA; in L2 the A-row warps load both the h
//   rows and the CTA's W2 half with cp.async (with a 64x64 TMA box of W2
//   the L2 tasks ran at about half the tensor-pipe rate, with cp.async at
//   70-90 %);
// * each CTA's loads land on its own stage barrier; the follower's warp 1
//   relays the completion of each of its
//   stages to the leader's barrier with one remote arrival (counting the
//   follower's bytes on the leader's barrier directly, with the pair form of
//   the TMA load, measured 2.5x slower here).
//
// Prior art: "MegaMoE 在 MoE 系统谱系中的位置", section 2.1 (the MMA warp issues
// for the leader CTA only; warp roles with their own jobs) and section 2.7
// (atomic task queue, L2 waits for its L1 tiles). No TMA multicast is used.
//
// Like expert_gemm.cuh, a template over bf16 or FP8 E4M3 operands; in the FP8
// second GEMM the A-row warps copy the CTA's half of the K-major W2 codes.
//
// Half tasks (bf16, BLOCK_M = 128): when an expert has an odd number of
// blocks, its last block would leave the second CTA of its pair without
// rows, and an M = 256 MMA would still spend the time of two blocks on it.
// Instead that block runs as M = 128 pair MMAs (64 rows in each CTA: rows
// 0-63 of the block in CTA 0, rows 64-127 in CTA 1), which take half the
// tensor time. Their accumulator layout differs from M = 256: each CTA's D
// (64 rows x N) puts columns 0 .. N/2-1 (the CTA-0 half of the B tile) in
// TMEM lanes 0-63 and columns N/2 .. N-1 (the CTA-1 half) in lanes 64-127,
// both at TMEM columns 0 .. N/2-1. So in a half L1 task each CTA loads one
// 64-column box of W1 and the matching box of W3 (CTA 0 the first 64 of the
// task's 128 columns of I, CTA 1 the next 64), and epilogue warp q finds g
// and u of row 32*(q%2) + lane, columns 64*(q/2) + c, at TMEM columns c and
// 64 + c; in a half L2 task warp q combines columns 128*(q/2) .. +127.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

#include "common.cuh"
#include "expert_gemm.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kStages2 = 6;
constexpr int kTileB2Bytes = 2 * kBoxBytes;                 // 128 weight columns x 64 rows per CTA
constexpr int kStage2Bytes = kTileABytes + kTileB2Bytes;    // 32 KB

struct Gemm2Params {
  const bf16* x;       // [T, H]
  const bf16* w2;      // [E, I, H]
  const bf16* ws2;     // [S, I, H] shared experts (experts E .. E+S-1), or null when S = 0
  CUtensorMap tm_w1;   // W1 as [E*H, I], box {64, 64}
  CUtensorMap tm_w3;   // W3 as [E*H, I], box {64, 64}
  CUtensorMap tm_ws1;  // shared experts' W1 as [S*H, I] (unused when S = 0)
  CUtensorMap tm_ws3;  // shared experts' W3 as [S*H, I]
  const int32_t* slot_token;
  const int32_t* slot_topk;
  const float* topk_w;
  const int32_t* block_start;   // [E+1]
  const int32_t* pair_start;    // [E+1] pairs of consecutive blocks per expert
  const int32_t* group_start;   // [groups + 1] in pairs
  const int32_t* num_groups;
  int32_t* task_counter;
  int32_t* l1_done;             // [pairs] 8 arrivals per L1 n-tile (4 epilogue warps x 2 CTAs)
  int32_t* l2_done;             // [pairs] 1 arrival per L2 n-tile
  int32_t* err;
  bf16* h;
  float* y_acc;                 // [T, H]
  int T, H, I, E, k, BM, BN2, N1, N2;
  int S;                        // shared experts (0 .. kMaxShared)
  // FP8 E4M3 expert GEMMs (the kernel's FP8 instance; see GemmParams): x codes, token scales,
  // K-major W1/W3 codes in tm_w1 / tm_w3 (box {128, 64}), column scales
  const uint8_t* xq;
  const float* sx;
  const float* s1;
  const float* s3;
  const uint8_t* w2q;   // FP8: W2 codes K-major [E, H, I] (the A-row warps copy this CTA's half)
  const float* s2;      // FP8: W2 column scales [E, H]
  float* act_amax;         // FP8: [h rows] row amax of the bf16 activation (see GemmParams)
  const float* act_scale;  // FP8: [h rows] row scale written by the activation quantizer
  const uint8_t* h8;       // FP8: [h rows, I] activation codes
  int phase_only;          // -1: both phases; 0: first GEMM only; 1: second GEMM only
  int only_group;          // with phase_only >= 0: the block group whose tasks this launch runs
  int ring_pairs, max_groups;
  int order_lag;                // task order (locate_task in expert_gemm.cuh): -1 staggered, >= 0 interleaved
  int half_tails;               // 1: an expert's lone last block runs as an M = 128 pair MMA (bf16, BM = 128)
  const uint8_t* zero_row;      // 2*H zero bytes: the A row of a padding slot
  TaskRecord* task_log;         // one record per task of the launch (written by the leader), or null
  int task_log_cap;
  unsigned long long timeout_ns;
  int withhold_pair;            // test hook: never publish L1 completion of this pair (-1: off)
};

struct Task2 {
  int phase;    // 0 = L1, 1 = L2, -1 = no more work
  int e, p, n;  // expert, pair, n-tile
  int b0, b1;   // blocks of CTA 0 and CTA 1 (b1 = -1: the expert has an odd block count)
  int half;     // 1: the lone block b0 split over the pair, rows 0-63 in CTA 0 and 64-127 in CTA 1
  int id;       // task number (the claimed counter value)
};

struct Gemm2Smem {
  float out_stage[4][32][36];   // L2 epilogue staging (see combine_rows in expert_gemm.cuh)
  int out_tok[4][32];
  uint64_t full[kStages2];
  uint64_t empty[kStages2];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t task_full[kTaskRing];
  uint64_t task_empty[kTaskRing];
  uint64_t mma_done;
  Task2 tasks[kTaskRing];
  uint32_t tmem_base;
  int abort;
  int taken;   // tasks the leader's producer has taken from the ring
  int num_groups;
  int rows[kTaskRing][kTileM];
  int block_start[kMaxExpertsAll + 1];
  int pair_start[kMaxExpertsAll + 1];
  int group_start[kMaxGroups + 1];
};

static_assert(offsetof(Gemm2Smem, out_stage) % 16 == 0, "staging rows are read as float4");
static_assert(sizeof(Task2) == 32, "tasks are copied to the peer as 8 words");

constexpr size_t kGemm2SmemBytes = 1024 + (size_t)kStages2 * kStage2Bytes + sizeof(Gemm2Smem);

// Wide variant (bf16, I % 256 == 0): an L1 task covers 256 columns of I (two
// N = 256 MMAs per K block on the same A tile, into both TMEM accumulators),
// so the routed x rows are gathered once per 256 columns instead of per 128;
// a stage then holds 128 B-tile columns per CTA (48 KB), four stages.
constexpr int kStages2W = 4;
constexpr int kStage2BytesW = kTileABytes + 2 * kTileB2Bytes;   // 48 KB
constexpr size_t kGemm2SmemBytesW = 1024 + (size_t)kStages2W * kStage2BytesW + sizeof(Gemm2Smem);
static_assert(kGemm2SmemBytesW <= 232448, "wide pair kernel exceeds the shared memory of a CTA");
template <bool W>
__host__ __device__ constexpr int stages2() { return W ? kStages2W : kStages2; }
template <bool W>
__host__ __device__ constexpr int stage2_bytes() { return W ? kStage2BytesW : kStage2Bytes; }

__device__ __forceinline__ void set_error2(const Gemm2Params& p, Gemm2Smem& s, int code, int detail) {
  if (atomicCAS(p.err, 0, code) == 0) p.err[1] = detail;
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
}

// Bounded wait of a whole warp on a local barrier phase. Arrivals may come
// from the peer CTA; the per-stage barriers are waited on at CTA scope (the
// data they guard is TMA- or cp.async-written shared memory read by the
// tensor core), the task ring of the follower, whose task words and row
// indices the leader writes through the cluster window, at cluster scope.
// Gives up on timeout, on this CTA's abort flag, or (checked every few
// microseconds) on a recorded error.
template <bool kClusterAcquire = false>
__device__ __forceinline__ bool warp_wait2(uint64_t* bar, uint32_t parity, const Gemm2Params& p, Gemm2Smem& s,
                                           int where) {
  auto poll = [&]() {
    return kClusterAcquire ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
  };
  bool ok = poll();
  if (!ok) {
    const uint64_t t0 = ptx::globaltimer();
    uint64_t next_check = t0 + 4000;
    while (true) {
      if (poll()) {
        ok = true;
        break;
      }
      if (*reinterpret_cast<volatile int*>(&s.abort)) break;
      const uint64_t now = ptx::globaltimer();
      if (now > next_check) {
        if (*reinterpret_cast<volatile int*>(p.err) != 0) break;
        next_check = now + 4000;
      }
      if (now - t0 > p.timeout_ns) {
        set_error2(p, s, kDevTimeout, 0x100 | where);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool wait_counter2(const int* ctr, int need, const Gemm2Params& p, Gemm2Smem& s,
                                              int detail) {
  if (ptx::ld_acquire_gpu(ctr) >= need) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (ptx::ld_acquire_gpu(ctr) < need) {
    if (*reinterpret_cast<volatile int*>(&s.abort) || *reinterpret_cast<volatile int*>(p.err) != 0) return false;
    if (ptx::globaltimer() - t0 > p.timeout_ns) {
      set_error2(p, s, kDevTimeout, detail);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}

__device__ __forceinline__ int claim_task_any(int32_t* counter, const int32_t* err, const int* abort, int lane) {
  int t = 0x7fffffff;
  if (lane == 0) {
    const bool stop = *reinterpret_cast<const volatile int*>(abort) || *reinterpret_cast<const volatile int*>(err) != 0;
    if (!stop) t = atomicAdd(counter, 1);
  }
  return t;   // valid in lane 0 only
}

// Task order as in expert_gemm.cuh (locate_task), in units of block pairs.
__device__ __forceinline__ Task2 decode_task2(int t, const Gemm2Smem& s, const Gemm2Params& p) {
  Task2 task{-1, 0, 0, 0, -1, -1, 0, 0};
  const int G = s.num_groups;
  const int np_total = s.pair_start[p.E + p.S];
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
    if (t < 0 || t >= np_total * (p.N1 + p.N2) || G <= 0) return task;
    pos = locate_task(t, s.group_start, G, p.N1, p.N2, p.order_lag);
  }
  task.phase = pos.phase;
  const int g = pos.g, NT = pos.phase == 0 ? p.N1 : p.N2;
  const int gp0 = s.group_start[g], gp1 = s.group_start[g + 1];
  const int tl = pos.tl;
  const int vp = gp0 + tl / NT;
  int elo = 0, ehi = p.E + p.S - 1;
  while (elo < ehi) {
    const int mid = (elo + ehi + 1) >> 1;
    if (s.pair_start[mid] <= vp) elo = mid;
    else ehi = mid - 1;
  }
  const int e = elo;
  const int ep0 = max(gp0, s.pair_start[e]);
  const int ep1 = min(gp1, s.pair_start[e + 1]);
  const int np = ep1 - ep0;
  const int local = tl - (ep0 - gp0) * NT;
  task.e = e;
  task.n = local / np;
  task.p = ep0 + (local - task.n * np);
  task.b0 = s.block_start[e] + 2 * (task.p - s.pair_start[e]);
  task.b1 = task.b0 + 1 < s.block_start[e + 1] ? task.b0 + 1 : -1;
  task.half = (task.b1 < 0 && p.half_tails) ? 1 : 0;
  task.id = t;
  return task;
}

template <bool W>
__device__ __forceinline__ uint8_t* stage2_ptr(uint8_t* tiles, int stage) { return tiles + stage * stage2_bytes<W>(); }

// K blocks of an L1 task: 64 bf16 or 128 FP8 elements (one 128-byte swizzle row).
template <bool F8>
__device__ __forceinline__ int l1_ksteps2(const Gemm2Params& p) { return F8 ? p.H / 128 : p.H / kBK; }

template <bool F8>
__device__ __forceinline__ int l2_ksteps2(const Gemm2Params& p) { return F8 ? p.I / 128 : p.I / kBK; }

// ---------------------------------------------------------------- leader scheduler (last warp)
// Claims tasks, decodes them, stages the token rows of both CTAs' A tiles
// (L1) or waits for the L1 tiles of the pair (L2), and publishes each task in
// both CTAs' rings; as in expert_gemm.cuh it runs one task ahead of the
// leader's producer and never further.
__device__ __forceinline__ bool prepare_task2(Task2& task, int q, uint32_t qparity, const Gemm2Params& p,
                                              Gemm2Smem& s, int lane) {
  if (!warp_wait2(&s.task_empty[q], qparity, p, s, 1)) return false;
  if (task.phase == 0) {
    // token rows of both CTAs' A tiles: CTA 0 locally, CTA 1 through the cluster window
    // (all loads first, one round trip)
    constexpr int kPer = kTileM / 32;
    int tok0[kPer], tok1[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = lane + 32 * i;
      if (task.half) {   // rows 0-63 of block b0 in CTA 0, rows 64-127 in CTA 1
        tok0[i] = r < 64 ? p.slot_token[task.b0 * p.BM + r] : -1;
        tok1[i] = r < 64 ? p.slot_token[task.b0 * p.BM + 64 + r] : -1;
      } else {
        tok0[i] = r < p.BM ? p.slot_token[task.b0 * p.BM + r] : 0;
        tok1[i] = r < p.BM && task.b1 >= 0 ? p.slot_token[task.b1 * p.BM + r] : 0;
      }
    }
    const uint32_t peer_rows = ptx::mapa(ptx::smem_u32(&s.rows[q][0]), 1);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = lane + 32 * i;
      if (r < p.BM) {
        if (tok0[i] >= p.T || tok1[i] >= p.T) {
          set_error2(p, s, kDevBounds, task.p);
          tok0[i] = tok0[i] >= p.T ? 0 : tok0[i];
          tok1[i] = tok1[i] >= p.T ? 0 : tok1[i];
        }
        // padding slot (or no block): -1, the gather fills the row with zeros
        s.rows[q][r] = tok0[i] < 0 ? -1 : tok0[i];
        ptx::st_cluster_u32(peer_rows + 4 * r,
                            (tok1[i] < 0 || (task.b1 < 0 && !task.half)) ? 0xffffffffu : (uint32_t)tok1[i]);
      }
    }
  } else if (task.phase == 1) {
    // the L2 task of pair p reads h rows written by all L1 n-tiles of the pair
    // (one arrival per epilogue warp of both CTAs per n-tile)
    bool fine = true;
    if (lane == 0) fine = wait_counter2(p.l1_done + task.p, 8 * p.N1, p, s, 0x10000 | task.p);
    if (__shfl_sync(0xffffffffu, fine ? 1 : 0, 0) == 0) task.phase = -1;
  }
  __syncwarp();
  return true;
}

__device__ __forceinline__ void push_task2(const Task2& task, int q, Gemm2Smem& s, int lane) {
  if (lane < 8) {
    const uint32_t v = reinterpret_cast<const uint32_t*>(&task)[lane];
    reinterpret_cast<uint32_t*>(&s.tasks[q])[lane] = v;
    ptx::st_cluster_u32(ptx::mapa(ptx::smem_u32(&s.tasks[q]), 1) + 4 * lane, v);
  }
  // every lane's stores into the peer (task words here, row indices in
  // prepare_task2) are ordered before lane 0's releasing arrive
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
  __syncwarp();
  if (lane == 0) {
    ptx::mbar_arrive(&s.task_full[q]);
    ptx::mbar_arrive_remote(ptx::mapa(ptx::smem_u32(&s.task_full[q]), 1));   // releases the stores above
  }
  __syncwarp();
}

// Bounded wait (one thread) until the leader's producer has taken `n` tasks.
__device__ __forceinline__ bool wait_taken2(int n, const Gemm2Params& p, Gemm2Smem& s) {
  if (*reinterpret_cast<volatile int*>(&s.taken) >= n) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (*reinterpret_cast<volatile int*>(&s.taken) < n) {
    if (*reinterpret_cast<volatile int*>(&s.abort)) return false;
    if (ptx::globaltimer() - t0 > p.timeout_ns) {
      set_error2(p, s, kDevTimeout, 0x10a);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

template <bool F8, bool W>
__device__ void gemm2_scheduler(const Gemm2Params& p, Gemm2Smem& s) {
  const int lane = ptx::lane_id();
  int q = 0;
  uint32_t qphase = 0;
  int pushed = 0;
  while (true) {
    bool ok = true;
    if (lane == 0) ok = wait_taken2(pushed, p, s);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    Task2 task{-1, 0, 0, 0, -1, -1, 0, 0};
    if (ok) {
      const int t = __shfl_sync(0xffffffffu, claim_task_any(p.task_counter, p.err, &s.abort, lane), 0);
      task = decode_task2(t, s, p);
    }
    if (!prepare_task2(task, q, qphase ^ 1, p, s, lane)) break;
    push_task2(task, q, s, lane);
    ++pushed;
    if (++q == kTaskRing) {
      q = 0;
      qphase ^= 1;
    }
    if (task.phase < 0) break;
  }
}

// ---------------------------------------------------------------- leader warp 0: TMA
template <bool F8, bool W>
__device__ void gemm2_leader_producer(const Gemm2Params& p, Gemm2Smem& s, uint8_t* tiles) {
  const int lane = ptx::lane_id();
  // weight tiles: normal L2 priority, so that the other pairs of the expert that read the same
  // tile shortly after still find it (evict-first measured 1.5-3.5 % slower on CTA pairs)
  const uint64_t pol = ptx::policy_evict_normal();
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  uint32_t issued = 0, issued_parity = 0;
  bool ok = true;
  while (ok) {
    if (!warp_wait2(&s.task_full[q], qphase, p, s, 14)) break;
    const Task2 task = s.tasks[q];
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
    const int nk = task.phase == 0 ? l1_ksteps2<F8>(p) : l2_ksteps2<F8>(p);
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait2(&s.empty[stage], phase ^ 1, p, s, 2)) {
        ok = false;
        break;
      }
      const uint32_t a_addr = ptx::smem_u32(stage2_ptr<W>(tiles, stage));
      const uint32_t b_addr = a_addr + kTileABytes;
      if (lane == 0) {
        // this CTA's half only; the follower's half lands on the follower's own
        // barrier and reaches this one through its relay arrival
        if (W && task.phase == 0) {
          // 256 columns of I: W1 columns n0 .. n0+255 (the follower: W3), or in a half task
          // W1 and W3 columns n0 .. n0+63 and n0+128 .. n0+191 (the follower: the other 64s)
          ptx::mbar_arrive_expect_tx(&s.full[stage], 4 * kBoxBytes);
          const int n0 = task.n * 2 * kL1TileN;
          const bool sh = task.e >= p.E;
          const int wrow = (sh ? task.e - p.E : task.e) * p.H + kb * kBK;
          const CUtensorMap* m1 = sh ? &p.tm_ws1 : &p.tm_w1;
          const CUtensorMap* m3 = sh ? &p.tm_ws3 : &p.tm_w3;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const CUtensorMap* m = task.half ? ((j & 1) ? m3 : m1) : m1;
            const int col = task.half ? n0 + (j >> 1) * kL1TileN : n0 + j * 64;
            ptx::tma_load_2d(b_addr + j * kBoxBytes, m, &s.full[stage], col, wrow, pol);
          }
        } else if (task.phase == 0) {
          ptx::mbar_arrive_expect_tx(&s.full[stage], 2 * kBoxBytes);
          const int n0 = task.n * kL1TileN;
          if (F8) {   // K-major FP8 codes: 64 rows (columns of I) x 128 bytes per box
            ptx::tma_load_2d(b_addr, &p.tm_w1, &s.full[stage], kb * 128, task.e * p.I + n0, pol);
            ptx::tma_load_2d(b_addr + kBoxBytes, &p.tm_w1, &s.full[stage], kb * 128, task.e * p.I + n0 + 64, pol);
          } else {
            const bool sh = task.e >= p.E;   // shared expert: its own weight tensors
            const int wrow = (sh ? task.e - p.E : task.e) * p.H + kb * kBK;
            const CUtensorMap* m1 = sh ? &p.tm_ws1 : &p.tm_w1;
            if (task.half) {   // columns n0 .. n0+63 of W1 and of W3 (the follower takes the next 64)
              ptx::tma_load_2d(b_addr, m1, &s.full[stage], n0, wrow, pol);
              ptx::tma_load_2d(b_addr + kBoxBytes, sh ? &p.tm_ws3 : &p.tm_w3, &s.full[stage], n0, wrow, pol);
            } else {
              ptx::tma_load_2d(b_addr, m1, &s.full[stage], n0, wrow, pol);
              ptx::tma_load_2d(b_addr + kBoxBytes, m1, &s.full[stage], n0 + 64, wrow, pol);
            }
          }
        } else {
          // L2: both operands come from the A-row warps' cp.async (a TMA box of
          // W2 kept the tensor pipe waiting); only this arrival is the producer's
          ptx::mbar_arrive(&s.full[stage]);
        }
      }
      __syncwarp();
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == stages2<W>()) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  for (int st = 0; st < stages2<W>(); ++st)
    if (issued & (1u << st)) {
      const uint64_t t0 = ptx::globaltimer();
      while (!ptx::mbar_try_wait(&s.full[st], (issued_parity >> st) & 1u))
        if (ptx::globaltimer() - t0 > p.timeout_ns) break;
    }
}

// Pop the next task from this CTA's ring and release the slot to the leader.
__device__ __forceinline__ bool pop_task2(Task2& task, int& q, uint32_t& qphase, int* q_popped, bool is_leader,
                                          const Gemm2Params& p, Gemm2Smem& s, int where, bool release_now) {
  const int lane = ptx::lane_id();
  const bool got = is_leader ? warp_wait2(&s.task_full[q], qphase, p, s, where)
                             : warp_wait2<true>(&s.task_full[q], qphase, p, s, where);
  if (!got) return false;
  task = s.tasks[q];
  if (q_popped) *q_popped = q;
  if (release_now) {
    __syncwarp();
    if (lane == 0) {
      if (is_leader) ptx::mbar_arrive(&s.task_empty[q]);
      else ptx::mbar_arrive_remote(ptx::mapa(ptx::smem_u32(&s.task_empty[q]), 0));
    }
  }
  if (++q == kTaskRing) {
    q = 0;
    qphase ^= 1;
  }
  return true;
}

__device__ __forceinline__ void release_task_slot2(int q, bool is_leader, Gemm2Smem& s) {
  __syncwarp();
  if (ptx::lane_id() == 0) {
    if (is_leader) ptx::mbar_arrive(&s.task_empty[q]);
    else ptx::mbar_arrive_remote(ptx::mapa(ptx::smem_u32(&s.task_empty[q]), 0));
  }
}

// ---------------------------------------------------------------- follower warp 0: its TMA halves
template <bool F8, bool W>
__device__ void gemm2_follower_producer(const Gemm2Params& p, Gemm2Smem& s, uint8_t* tiles) {
  const int lane = ptx::lane_id();
  const uint64_t pol = ptx::policy_evict_normal();   // weight tiles (see the leader)
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  while (true) {
    Task2 task;
    if (!pop_task2(task, q, qphase, nullptr, false, p, s, 3, true)) break;
    if (task.phase < 0) break;
    const int nk = task.phase == 0 ? l1_ksteps2<F8>(p) : l2_ksteps2<F8>(p);
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait2(&s.empty[stage], phase ^ 1, p, s, 4)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const uint32_t a_addr = ptx::smem_u32(stage2_ptr<W>(tiles, stage));
        const uint32_t b_addr = a_addr + kTileABytes;
        if (W && task.phase == 0) {   // the leader's layout, with W3 (or the other 64 columns)
          ptx::mbar_arrive_expect_tx(&s.full[stage], 4 * kBoxBytes);
          const int n0 = task.n * 2 * kL1TileN;
          const bool sh = task.e >= p.E;
          const int wrow = (sh ? task.e - p.E : task.e) * p.H + kb * kBK;
          const CUtensorMap* m1 = sh ? &p.tm_ws1 : &p.tm_w1;
          const CUtensorMap* m3 = sh ? &p.tm_ws3 : &p.tm_w3;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const CUtensorMap* m = task.half ? ((j & 1) ? m3 : m1) : m3;
            const int col = task.half ? n0 + (j >> 1) * kL1TileN + 64 : n0 + j * 64;
            ptx::tma_load_2d(b_addr + j * kBoxBytes, m, &s.full[stage], col, wrow, pol);
          }
        } else if (task.phase == 0) {
          ptx::mbar_arrive_expect_tx(&s.full[stage], 2 * kBoxBytes);
          const int n0 = task.n * kL1TileN;
          if (F8) {
            ptx::tma_load_2d(b_addr, &p.tm_w3, &s.full[stage], kb * 128, task.e * p.I + n0, pol);
            ptx::tma_load_2d(b_addr + kBoxBytes, &p.tm_w3, &s.full[stage], kb * 128, task.e * p.I + n0 + 64, pol);
          } else {
            const bool sh = task.e >= p.E;
            const int wrow = (sh ? task.e - p.E : task.e) * p.H + kb * kBK;
            const CUtensorMap* m3 = sh ? &p.tm_ws3 : &p.tm_w3;
            if (task.half) {   // columns n0+64 .. n0+127 of W1 and of W3
              ptx::tma_load_2d(b_addr, sh ? &p.tm_ws1 : &p.tm_w1, &s.full[stage], n0 + 64, wrow, pol);
              ptx::tma_load_2d(b_addr + kBoxBytes, m3, &s.full[stage], n0 + 64, wrow, pol);
            } else {
              ptx::tma_load_2d(b_addr, m3, &s.full[stage], n0, wrow, pol);
              ptx::tma_load_2d(b_addr + kBoxBytes, m3, &s.full[stage], n0 + 64, wrow, pol);
            }
          }
        } else {
          ptx::mbar_arrive(&s.full[stage]);   // L2: operands by the A-row warps (see the leader)
        }
      }
      __syncwarp();
      if (++stage == stages2<W>()) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
  }
}

// ---------------------------------------------------------------- follower warp 1: stage relay
// The follower's TMA bytes and gather lanes land on its own stage barrier;
// once a stage is complete, one arrival on the leader's barrier of that stage.
template <bool F8, bool W>
__device__ void gemm2_follower_relay(const Gemm2Params& p, Gemm2Smem& s) {
  const int lane = ptx::lane_id();
  const uint32_t lead_full0 = ptx::mapa(ptx::smem_u32(&s.full[0]), 0);
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  while (true) {
    Task2 task;
    if (!pop_task2(task, q, qphase, nullptr, false, p, s, 5, true)) break;
    if (task.phase < 0) break;
    const int nk = task.phase == 0 ? l1_ksteps2<F8>(p) : l2_ksteps2<F8>(p);
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait2(&s.full[stage], phase, p, s, 6)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        ptx::fence_proxy_async_shared();   // cp.async-written rows -> the tensor core's reads
        ptx::mbar_arrive_peer(lead_full0 + 8 * stage);
      }
      __syncwarp();
      if (++stage == stages2<W>()) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
  }
}

// ---------------------------------------------------------------- leader warp 1: MMA issuer
template <bool F8, bool W>
__device__ void gemm2_mma(const Gemm2Params& p, Gemm2Smem& s, uint8_t* tiles, uint32_t tmem_base) {
  const int lane = ptx::lane_id();
  const uint32_t idesc_l1 =
      F8 ? ptx::idesc_e4m3_f32(256, 2 * kL1TileN) : ptx::idesc_bf16_f32(256, 2 * kL1TileN, false, true);
  constexpr bool f8 = F8;
  const uint32_t idesc_l2 = F8 ? ptx::idesc_e4m3_f32(256, p.BN2) : ptx::idesc_bf16_f32(256, p.BN2, false, true);
  // half tasks (bf16 only): 64 rows per CTA
  const uint32_t idesc_l1_half = ptx::idesc_bf16_f32(128, 2 * kL1TileN, false, true);
  const uint32_t idesc_l2_half = ptx::idesc_bf16_f32(128, p.BN2, false, true);
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool issued_any = false;
  while (true) {
    Task2 task;
    if (!pop_task2(task, q, qphase, nullptr, true, p, s, 7, true)) break;
    if (task.phase < 0) break;
    if (!warp_wait2(&s.acc_empty[acc], acc_phase ^ 1, p, s, 8)) break;
    // wide L1 task: both accumulators, this slot and the next one in turn
    const bool two = W && task.phase == 0;
    const int acc2 = acc ^ 1;
    const uint32_t acc2_phase = acc == 1 ? acc_phase ^ 1 : acc_phase;
    if (two && !warp_wait2(&s.acc_empty[acc2], acc2_phase ^ 1, p, s, 8)) break;
    ptx::tc_fence_after();
    const uint32_t d_tmem = tmem_base + acc * 256;
    const uint32_t d_tmem2 = tmem_base + acc2 * 256;
    const uint32_t idesc = task.half ? (task.phase == 0 ? idesc_l1_half : idesc_l2_half)
                                     : (task.phase == 0 ? idesc_l1 : idesc_l2);
    const int nk = task.phase == 0 ? l1_ksteps2<F8>(p) : l2_ksteps2<F8>(p);
    bool ok = true;
    uint64_t t_first = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait2(&s.full[stage], phase, p, s, 9)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      ptx::fence_proxy_async_shared();
      if (kb == 0) t_first = ptx::globaltimer();
      if (lane == 0) {
        const uint32_t a_addr = ptx::smem_u32(stage2_ptr<W>(tiles, stage));
        const uint32_t b_addr = a_addr + kTileABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          if (f8) {
            // B half: K-major FP8 codes (W1 | W3, or W2), rows of 128 bytes in each CTA
            const uint64_t bd = ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            ptx::mma_f8_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          } else {
            const uint64_t bd = ptx::smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            ptx::mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            if (two) {   // the next 128 columns of I: B boxes 2 and 3, the same A tile
              const uint64_t bd2 = ptx::smem_desc_sw128(b_addr + 2 * kBoxBytes + kk * 2048, kBoxBytes, 1024);
              ptx::mma_bf16_pair(d_tmem2, ad, bd2, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
        }
        ptx::mma_commit_pair_multicast(&s.empty[stage], 0x3);
        issued_any = true;
      }
      __syncwarp();
      if (++stage == stages2<W>()) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
    if (lane == 0) {
      ptx::mma_commit_pair_multicast(&s.acc_full[acc], 0x3);
      if (two) ptx::mma_commit_pair_multicast(&s.acc_full[acc2], 0x3);
    }
    if (lane == 0 && p.task_log != nullptr && task.id < p.task_log_cap) {
      TaskRecord* r = p.task_log + task.id;
      r->task = task.id;
      r->unit = task.p;
      r->expert = task.e;
      r->phase_n = ((uint32_t)task.phase << 16) | (uint32_t)task.n;
      r->smid = smid_u32();
      r->cta = blockIdx.x;
      r->t_first_mma = t_first;
      r->t_last_mma = ptx::globaltimer();
    }
    __syncwarp();
    for (int used = two ? 2 : 1; used > 0; --used)
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
  }
  issued_any = __any_sync(0xffffffffu, issued_any);
  if (issued_any) {
    if (lane == 0) ptx::mma_commit_pair_multicast(&s.mma_done, 0x1);
    __syncwarp();
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(&s.mma_done, 0)) {
      if (ptx::globaltimer() - t0 > p.timeout_ns) break;
    }
  }
}

// ---------------------------------------------------------------- epilogue (warps 2..5 of both CTAs)
template <bool F8, bool W>
__device__ void gemm2_epilogue(const Gemm2Params& p, Gemm2Smem& s, uint32_t tmem_base, uint32_t rank) {
  const int warp = threadIdx.x >> 5;
  const int lane = ptx::lane_id();
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const bool is_leader = rank == 0;
  const uint32_t lead_acc_empty0 = ptx::mapa(ptx::smem_u32(&s.acc_empty[0]), 0);
  int q = 0;
  uint32_t qphase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  while (true) {
    Task2 task;
    if (!pop_task2(task, q, qphase, nullptr, is_leader, p, s, 10, true)) break;
    if (task.phase < 0) break;
    // FP8: the task's scales, loaded before the accumulator wait (lane j: column 32c + j of chunk c)
    float tscale = 0.f, rscale = 1.f, sa[4] = {1.f, 1.f, 1.f, 1.f}, sb[4] = {1.f, 1.f, 1.f, 1.f};
    if (F8) {
      const int bo = rank == 0 ? task.b0 : task.b1;
      if (task.phase == 0) {
        const size_t col0 = (size_t)task.e * p.I + task.n * kL1TileN;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sa[c] = __ldg(p.s1 + col0 + c * 32 + lane);
          sb[c] = __ldg(p.s3 + col0 + c * 32 + lane);
        }
        if (r < p.BM && bo >= 0) {   // the token's scale (padding rows: 0, so their activation is 0)
          const int tok = p.slot_token[bo * p.BM + r];
          tscale = (tok >= 0 && tok < p.T) ? __ldg(p.sx + tok) : 0.f;
        }
      } else if (r < p.BM && bo >= 0) {   // the activation row's scale
        rscale = __ldcg(p.act_scale + ((task.p % p.ring_pairs) * 2 + (int)rank) * p.BM + r);
      }
    }
    auto next_acc = [&]() {
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    };
    auto release_acc = [&]() {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (is_leader) ptx::mbar_arrive(&s.acc_empty[acc]);
        else ptx::mbar_arrive_peer(lead_acc_empty0 + 8 * acc);
      }
    };
    if (W && !F8 && task.phase == 0) {
      // wide L1 task: 256 columns of I in two accumulators (this slot, then the next), each
      // released as soon as it is read, so the next task's MMAs start on the first one
      const bool hf = task.half != 0;
      const int hr = (quarter & 1) * 32 + lane, hc = quarter >> 1;   // half task: row and column half
      const int b_own = hf ? task.b0 : (rank == 0 ? task.b0 : task.b1);
      bool store = hf || (r < p.BM && b_own >= 0);
      if (task.p >= p.ring_pairs) {
        bool ok = true;
        if (lane == 0) ok = wait_counter2(p.l2_done + (task.p - p.ring_pairs), p.N2, p, s, 0x40000 | task.p);
        store = store && __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      const int ring_row = hf ? (task.p % p.ring_pairs) * 2 * p.BM + (int)rank * 64 + hr
                              : ((task.p % p.ring_pairs) * 2 + (int)rank) * p.BM + r;
      bool fine = true;
      for (int sub = 0; sub < 2; ++sub) {
        if (!warp_wait2(&s.acc_full[acc], acc_phase, p, s, 11)) {
          fine = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 256;
        const int n0 = task.n * 2 * kL1TileN + sub * kL1TileN;
        float amax = 0.f;
        if (hf) {   // g at TMEM columns 0..63, u at 64..127: columns 64*hc .. +63 of these 128
          bf16* hrow = p.h + (size_t)ring_row * p.I + n0 + hc * 64;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t g[32], u[32];
            ptx::tmem_ld32(tb + c * 32, g);
            ptx::tmem_ld32(tb + 64 + c * 32, u);
            ptx::tmem_ld_wait();
            if (store) store_swiglu32(hrow + c * 32, g, u, amax);
          }
        } else {
          bf16* hrow = p.h + (size_t)ring_row * p.I + n0;
#pragma unroll 1
          for (int c = 0; c < kL1TileN / 32; ++c) {
            uint32_t g[32], u[32];
            ptx::tmem_ld32(tb + c * 32, g);
            ptx::tmem_ld32(tb + kL1TileN + c * 32, u);
            ptx::tmem_ld_wait();
            if (store) store_swiglu32(hrow + c * 32, g, u, amax);
          }
        }
        release_acc();
        next_acc();
      }
      if (!fine) break;
      __threadfence();
      __syncwarp();
      if (lane == 0 && task.p != p.withhold_pair) ptx::red_release_gpu_add(p.l1_done + task.p, 1);
      if (p.task_log != nullptr && is_leader && quarter == 0 && lane == 0 && task.id < p.task_log_cap)
        p.task_log[task.id].t_done = ptx::globaltimer();
      continue;
    }
    if (!warp_wait2(&s.acc_full[acc], acc_phase, p, s, 11)) break;
    ptx::tc_fence_after();
    const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 256;
    if (!F8 && task.half) {
      // M = 128 pair accumulator: this warp's lanes hold row hr of this CTA's 64
      // rows (block row 64*rank + hr) and the column half hc of the tile
      const int hr = (quarter & 1) * 32 + lane, hc = quarter >> 1;
      const int brow = (int)rank * 64 + hr;
      if (task.phase == 0) {
        bool store = true;
        if (task.p >= p.ring_pairs) {
          bool ok = true;
          if (lane == 0) ok = wait_counter2(p.l2_done + (task.p - p.ring_pairs), p.N2, p, s, 0x40000 | task.p);
          store = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        // g at TMEM columns 0..63, u at 64..127: columns 64*hc .. +63 of the task's 128 of I
        bf16* hrow = p.h + ((size_t)(task.p % p.ring_pairs) * 2 * p.BM + brow) * p.I + task.n * kL1TileN + hc * 64;
        float amax = 0.f;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t g[32], u[32];
          ptx::tmem_ld32(tbase + c * 32, g);
          ptx::tmem_ld32(tbase + 64 + c * 32, u);
          ptx::tmem_ld_wait();
          if (store) store_swiglu32(hrow + c * 32, g, u, amax);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (is_leader) ptx::mbar_arrive(&s.acc_empty[acc]);
          else ptx::mbar_arrive_peer(lead_acc_empty0 + 8 * acc);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0 && task.p != p.withhold_pair) ptx::red_release_gpu_add(p.l1_done + task.p, 1);
      } else {
        if (is_leader && quarter == 0 && lane == 0) ptx::red_release_gpu_add(p.l2_done + task.p, 1);
        const int slot = task.b0 * p.BM + brow;
        int tok = p.slot_token[slot];
        float w = 0.f;
        if (tok >= p.T) {
          set_error2(p, s, kDevBounds, 0x20000 | task.p);
          tok = -1;
        }
        if (tok >= 0) {
          const int j = p.slot_topk[slot];
          if (task.e >= p.E) {
            w = 1.f;
          } else if (j < 0 || j >= p.k) {
            set_error2(p, s, kDevBounds, 0x30000 | task.p);
            tok = -1;
          } else {
            w = p.topk_w[(size_t)tok * p.k + j];
          }
        }
        combine_rows(tbase, p.BN2 / 2, w, tok, p.y_acc, p.H, task.n * p.BN2 + hc * (p.BN2 / 2), s.out_stage[quarter],
                     s.out_tok[quarter], nullptr, [&]() {
                       ptx::tc_fence_before();
                       __syncwarp();
                       if (lane == 0) {
                         if (is_leader) ptx::mbar_arrive(&s.acc_empty[acc]);
                         else ptx::mbar_arrive_peer(lead_acc_empty0 + 8 * acc);
                       }
                     });
      }
      if (p.task_log != nullptr && is_leader && quarter == 0 && lane == 0 && task.id < p.task_log_cap)
        p.task_log[task.id].t_done = ptx::globaltimer();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
      continue;
    }
    const int b_own = rank == 0 ? task.b0 : task.b1;
    const bool valid = r < p.BM && b_own >= 0;
    const int slot = (b_own < 0 ? 0 : b_own) * p.BM + r;
    if (task.phase == 0) {
      bool store = valid;
      if (task.p >= p.ring_pairs) {
        bool ok = true;
        if (lane == 0) ok = wait_counter2(p.l2_done + (task.p - p.ring_pairs), p.N2, p, s, 0x40000 | task.p);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        store = store && ok;
      }
      const int ring_row = ((task.p % p.ring_pairs) * 2 + (int)rank) * p.BM + r;
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
      if (lane == 0) {
        if (is_leader) ptx::mbar_arrive(&s.acc_empty[acc]);
        else ptx::mbar_arrive_peer(lead_acc_empty0 + 8 * acc);
      }
      __threadfence();
      __syncwarp();
      if (lane == 0 && task.p != p.withhold_pair) ptx::red_release_gpu_add(p.l1_done + task.p, 1);
    } else {
      if (is_leader && quarter == 0 && lane == 0) ptx::red_release_gpu_add(p.l2_done + task.p, 1);
      int tok = -1;
      float w = 0.f;
      if (valid) {
        tok = p.slot_token[slot];
        if (tok >= p.T) {
          set_error2(p, s, kDevBounds, 0x20000 | task.p);
          tok = -1;
        }
        if (tok >= 0) {
          const int j = p.slot_topk[slot];
          if (task.e >= p.E) {
            w = 1.f;   // shared expert: every token, weight 1
          } else if (j < 0 || j >= p.k) {
            set_error2(p, s, kDevBounds, 0x30000 | task.p);
            tok = -1;
          } else {
            w = p.topk_w[(size_t)tok * p.k + j];
          }
        }
      }
      if (F8 && tok >= 0) w *= rscale;   // FP8: the activation row's scale
      combine_rows(tbase, p.BN2, w, tok, p.y_acc, p.H, task.n * p.BN2, s.out_stage[quarter], s.out_tok[quarter],
                   F8 ? p.s2 + (size_t)task.e * p.H + task.n * p.BN2 : nullptr, [&]() {
                     ptx::tc_fence_before();
                     __syncwarp();
                     if (lane == 0) {
                       if (is_leader) ptx::mbar_arrive(&s.acc_empty[acc]);
                       else ptx::mbar_arrive_peer(lead_acc_empty0 + 8 * acc);
                     }
                   });
    }
    if (p.task_log != nullptr && is_leader && quarter == 0 && lane == 0 && task.id < p.task_log_cap)
      p.task_log[task.id].t_done = ptx::globaltimer();
    if (++acc == 2) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
}

// ---------------------------------------------------------------- gather warps (warps 6.. of both CTAs)
template <bool F8, bool W>
__device__ void gemm2_gather(const Gemm2Params& p, Gemm2Smem& s, uint8_t* tiles, int g, uint32_t rank) {
  constexpr int kRowsPerLane = (kTileM / 4 + kGatherWarps - 1) / kGatherWarps;
  const uint64_t wpol = ptx::policy_evict_normal();   // W2 halves (see the leader producer)
  const int lane = ptx::lane_id();
  const int c = lane & 7;
  const bool is_leader = rank == 0;
  int stage = 0;
  uint32_t phase = 0;
  int q = 0;
  uint32_t qphase = 0;
  while (true) {
    Task2 task;
    int q_task = 0;
    if (!pop_task2(task, q, qphase, &q_task, is_leader, p, s, 12, false)) break;
    if (task.phase < 0) break;
    // half task: both CTAs take block b0, 64 rows each (CTA 1 its rows 64-127)
    const int b_own = task.half ? task.b0 : (rank == 0 ? task.b0 : task.b1);
    const int rows_own = task.half ? 64 : p.BM;
    const int ring_row0 = task.half ? (task.p % p.ring_pairs) * 2 * p.BM + (int)rank * 64
                                    : ((task.p % p.ring_pairs) * 2 + (int)rank) * p.BM;
    int nrows = 0;
    uint32_t soff[kRowsPerLane];
    const uint8_t* src[kRowsPerLane];   // byte addresses; a stage takes the next 128 bytes of a row
    if (b_own >= 0) {
      // L1: the routed x rows (bf16, or FP8 codes) of this CTA's block; L2: its h rows in the ring
      // activation rows: bf16, or FP8 codes (rows of I bytes)
      const int* rows = s.rows[q_task];
      const size_t hpitch = F8 ? (size_t)p.I : (size_t)p.I * 2;
      const uint8_t* hblock = (F8 ? p.h8 : reinterpret_cast<const uint8_t*>(p.h)) + (size_t)ring_row0 * hpitch;
      const uint8_t* xrows = F8 ? p.xq : reinterpret_cast<const uint8_t*>(p.x);
      const size_t xpitch = F8 ? (size_t)p.H : (size_t)p.H * 2;
#pragma unroll
      for (int j = 0; j < kRowsPerLane; ++j) {
        const int rr = (j * kGatherWarps + g) * 4 + (lane >> 3);
        soff[j] = rr * 128 + ((c ^ (rr & 7)) << 4);
        src[j] = xrows + c * 16;
        if (rr < rows_own) {
          // L1 padding slot (-1): the all-zero row, so the tensor core multiplies zeros and
          // the slot's h row comes out 0
          const int xr = rows[rr];
          src[j] = task.phase == 1 ? hblock + (size_t)rr * hpitch + c * 16
                   : xr < 0        ? p.zero_row + c * 16
                                   : xrows + (size_t)xr * xpitch + c * 16;
          nrows = j + 1;
        }
      }
    }
    release_task_slot2(q_task, is_leader, s);   // rows read: the slot may be refilled
    // L2: this CTA's half of the W2 tile too (BN2/2 columns: one or two 64x64
    // boxes, each 64 K-rows of 128 bytes in the same 128-byte swizzle as TMA)
    const int nhalf = task.phase == 1 && !F8 ? p.BN2 / 128 : 0;
    const int nchunk8 = task.phase == 1 && F8 ? (p.BN2 / 2) * 8 / (32 * kGatherWarps) : 0;   // 8, or 4 (BN2 = 128)
    const uint8_t* w2row8 =
        F8 ? p.w2q + ((size_t)task.e * p.H + task.n * p.BN2 + (int)rank * (p.BN2 / 2)) * p.I : nullptr;
    const int tl = g * 32 + lane;
    const bf16* w2src = F8 ? nullptr
                              : (task.e >= p.E ? p.ws2 + (size_t)(task.e - p.E) * p.I * p.H
                                               : p.w2 + (size_t)task.e * p.I * p.H) +
                                    task.n * p.BN2 + (int)rank * (p.BN2 / 2) + c * 8;
    const int nk = task.phase == 0 ? l1_ksteps2<F8>(p) : l2_ksteps2<F8>(p);
    bool ok = true;

    for (int kb = 0; kb < nk; ++kb) {
      if (!warp_wait2(&s.empty[stage], phase ^ 1, p, s, 13)) {
        ok = false;
        break;
      }
      const uint32_t a_addr = ptx::smem_u32(stage2_ptr<W>(tiles, stage));
#pragma unroll
      for (int j = 0; j < kRowsPerLane; ++j)
        if (j < nrows) ptx::cp_async_16(a_addr + soff[j], src[j] + (size_t)kb * 128);
      for (int j = 0; j < nhalf; ++j) {
#pragma unroll
        for (int i = 0; i < 64 / 4 / kGatherWarps; ++i) {
          const int kr = (i * kGatherWarps + g) * 4 + (lane >> 3);
          ptx::cp_async_16_hint(a_addr + kTileABytes + j * kBoxBytes + kr * 128 + ((c ^ (kr & 7)) << 4),
                                w2src + (size_t)(kb * kBK + kr) * p.H + j * 64, wpol);
        }
      }
      // FP8 L2: this CTA's W2 codes, BN2/2 rows of 128 bytes (8 chunks per row), K-major
      for (int i = 0; i < nchunk8; ++i) {
        const int qc = i * 32 * kGatherWarps + tl;   // chunk: row qc / 8, 16 bytes (qc & 7)
        const int wr = qc >> 3, wc = qc & 7;
        ptx::cp_async_16_hint(a_addr + kTileABytes + wr * 128 + ((wc ^ (wr & 7)) << 4),
                              w2row8 + (size_t)wr * p.I + kb * 128 + wc * 16, wpol);
      }
      ptx::cp_async_mbar_arrive_noinc(&s.full[stage]);
      if (++stage == stages2<W>()) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
  }
  ptx::cp_async_wait_all();
}

template <bool F8, bool W>
__global__ void __launch_bounds__(kGemm1Threads, 1) moe_expert_gemm2_kernel(const __grid_constant__ Gemm2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Gemm2Smem& s = *reinterpret_cast<Gemm2Smem*>(tiles + (size_t)stages2<W>() * stage2_bytes<W>());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool is_leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages2<W>(); ++i) {
      // leader: its producer, its gather lanes and the follower's relay; follower: its producer
      // (with its TMA bytes) and its gather lanes
      ptx::mbar_init(&s.full[i], is_leader ? 1 + 32 * kGatherWarps + 1 : 1 + 32 * kGatherWarps);
      ptx::mbar_init(&s.empty[i], 1);   // the leader's MMA commit, multicast to both CTAs
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.acc_full[i], 1);
      ptx::mbar_init(&s.acc_empty[i], 8);   // 4 epilogue warps in each CTA (used in the leader)
    }
    for (int i = 0; i < kTaskRing; ++i) {
      ptx::mbar_init(&s.task_full[i], 1);
      // in the leader: its producer, MMA, 4 epilogue and gather warps, and the
      // follower's producer, relay, 4 epilogue and gather warps
      ptx::mbar_init(&s.task_empty[i], (2 + 4 + kGatherWarps) + (2 + 4 + kGatherWarps));
    }
    ptx::mbar_init(&s.mma_done, 1);
    s.abort = 0;
    s.taken = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&p.tm_w1);
    ptx::prefetch_tmap(&p.tm_w3);
    if (p.S > 0) {
      ptx::prefetch_tmap(&p.tm_ws1);
      ptx::prefetch_tmap(&p.tm_ws3);
    }
  }
  for (int e = threadIdx.x; e <= p.E + p.S; e += kGemm1Threads) {
    s.block_start[e] = p.block_start[e];
    s.pair_start[e] = p.pair_start[e];
  }
  {
    const int ng = min(*p.num_groups, min(p.max_groups, kMaxGroups));
    if (threadIdx.x == 0) s.num_groups = ng;
    for (int g = threadIdx.x; g <= ng; g += kGemm1Threads) s.group_start[g] = p.group_start[g];
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&s.tmem_base, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  if (p.BM < kTileM) {
    for (int st = 0; st < stages2<W>(); ++st) {
      uint4* a = reinterpret_cast<uint4*>(stage2_ptr<W>(tiles, st) + p.BM * 128);
      const int n = (kTileM - p.BM) * 128 / 16;
      for (int i = threadIdx.x; i < n; i += kGemm1Threads) a[i] = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_shared();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // both CTAs' barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem_base = s.tmem_base;

  if (warp == 0) {
    if (is_leader) gemm2_leader_producer<F8, W>(p, s, tiles);
    else gemm2_follower_producer<F8, W>(p, s, tiles);
  } else if (warp == 1) {
    if (is_leader) gemm2_mma<F8, W>(p, s, tiles, tmem_base);
    else gemm2_follower_relay<F8, W>(p, s);
  } else if (warp < 6) {
    gemm2_epilogue<F8, W>(p, s, tmem_base, rank);
  } else if (warp < 6 + kGatherWarps) {
    gemm2_gather<F8, W>(p, s, tiles, warp - 6, rank);
  } else if (is_leader) {
    gemm2_scheduler<F8, W>(p, s);
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // no peer still arrives on or stores into this CTA's shared memory
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace moe
