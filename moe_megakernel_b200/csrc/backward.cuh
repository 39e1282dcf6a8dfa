// Backward of the MoE layer on the 5th-generation tensor cores: the
// gradients of y = sum_j w[t,j] FFN_{e_j}(x[t]) (SwiGLU experts, gate
// softmax over the k kept logits) for an upstream dy, computed with the
// forward's routing records (per expert, blocks of BLOCK_M slots holding
// (token, top-k position)).
//
// "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", abstract: forward and backward MoE megakernels, the backward
// reducing the experts' weight gradients over their tokens. Reading taken:
// the chain-rule gradient of the layer as written; the choice of experts is
// piecewise constant (no gradient through it); the bf16 rounding of the
// SwiGLU activation is passed straight through, while dW2 and the combine
// weights' gradient use the rounded activation the forward multiplied.
//
// One persistent kernel template, five task kinds (each a separate launch,
// ordered on the stream), all M = 128 x N <= 256 tcgen05 MMAs with an fp32
// TMEM accumulator; per slot s of expert e with token t, top-k position j
// and weight w = topk_w[t,j]:
//
//   kDgrad1  (block, 128 columns n of I): da~ = dy_t W2[e]^T (K = H, first, into
//            one of two 128-column TMEM slots used in turn) and g|u =
//            x_t [W1|W3][e] (K = H, as the forward's first GEMM, into columns
//            0-255), so that a task's da~ loop overlaps the previous task's
//            epilogue; epilogue:
//            a = bf16(silu(g) u), da = w da~, dg = da u silu'(g),
//            du = da silu(g); stores dg, du and aw = bf16(w a) per slot, and
//            adds sum_i a_i da~_i (= dy_t . o) into dw[t,j];
//   kDgrad2  (block, 256 or 128 columns of H): dx_t += [dg|du]_s [W1|W3][e]^T
//            (K = 2I), added into the fp32 dx accumulator through the slot
//            record like the forward's combine (weight 1);
//   kWgrad13 (expert, 128 rows of H, 128 columns of I): dW1[e] = x^T dg,
//            dW3[e] = x^T du over the expert's slots (K = its padded slots);
//   kWgrad2  (expert, 128 rows of H, 256 or 128 columns of I):
//            dW2[e]^T = dy^T aw over the expert's slots (the transpose keeps
//            the gathered operand at 128 columns of dy and loads the wider
//            aw tile by TMA), stored transposed into dW2[e] [I, H];
//   kDwg     (128 rows of H): dWg = x^T dl over all tokens (dl dense [T, E],
//            written by the gate kernel).
//
// Operand layouts in shared memory (128-byte swizzle): K-major tiles are 128
// rows of 64 K elements (one 128-byte row each); MN-major tiles are boxes of
// 64 M (or N) elements x 64 K rows, 8 KB each. Gathered operands (token rows
// through the slot record: x and dy) are copied with cp.async by four gather
// warps, padding slots and slots past the expert's range from an all-zero
// row; the rest
// (weights, dg / du / aw rows, x and dl for dWg) by TMA. Warp roles: 0 TMA
// producer, 1 MMA issuer, 2-5 epilogue, 6-9 gather. Tasks are dealt round
// robin (task = CTA + i * grid), so every role walks the same task list
// without a queue; an expert with no tokens has K = 0 and its weight
// gradients are written as zeros. Every wait is bounded like the forward's.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "expert_gemm.cuh"
#include "ptx.cuh"

namespace moe {

enum BwdKind : int { kBwdDgrad1 = 0, kBwdDgrad2 = 1, kBwdWgrad13 = 2, kBwdWgrad2 = 3, kBwdDwg = 4 };

constexpr int kBwdStages = 4;
constexpr int kBwdABytes = 16384;                       // 128 x 64 bf16 (K-major) or 2 MN-major boxes
constexpr int kBwdBBytes = 32768;                       // 4 boxes of 8 KB, or 256 K-major rows
constexpr int kBwdStageBytes = kBwdABytes + kBwdBBytes;
constexpr int kBwdGatherWarps = 4;
constexpr int kBwdThreads = 64 + 128 + 32 * kBwdGatherWarps;   // producer, MMA, 4 epilogue, 4 gather warps

struct BwdParams {
  // routing records of the forward (the dispatch's outputs)
  const int32_t* slot_token;     // [pool]
  const int32_t* slot_topk;      // [pool]
  const float* topk_w;           // [T, k]
  const int32_t* block_start;    // [E + 1]
  const int32_t* sched;          // [1]: number of blocks
  const bf16* x;                 // [T, H]
  const bf16* dy;                // [T, H]
  const bf16* zero_row;          // [H] zeros: the gathered row of a padding slot or a slot past the expert
  int permuted;                  // 1: x and dy rows in slot order (tm_xp, tm_dyp) replace the gathers
  CUtensorMap tm_xp;             // x rows in slot order [pool, H]: dgrad1 box {64, 128} (K-major A),
  CUtensorMap tm_dyp;            // wgrad box {64, 64} (MN-major A); dy rows likewise
  // tensor maps (128-byte swizzle), per kind
  CUtensorMap tm_w1;   // dgrad1: W1 as [E*H, I], box {64, 64} (MN-major B); dgrad2: box {64, BNd} (K-major B)
  CUtensorMap tm_w3;   // the same for W3
  CUtensorMap tm_w2;   // dgrad1: W2 as [E*I, H], box {64, 128} (K-major B: rows i, K = h)
  CUtensorMap tm_a;    // dgrad2: dg as [pool, I] box {64, 128}; dwg: x [T, H] box {64, 64}
  CUtensorMap tm_a2;   // dgrad2: du as [pool, I], box {64, 128}
  CUtensorMap tm_b;    // wgrad13: dg as [pool, I] box {64, 64}; wgrad2: aw [pool, I] box {64, 64}; dwg: dl [T, NE]
  CUtensorMap tm_b2;   // wgrad13: du as [pool, I] box {64, 64}
  bf16* dg;            // [pool, I]
  bf16* du;            // [pool, I]
  bf16* aw;            // [pool, I]: w * bf16(activation)
  float* dw;           // [T, k]: dy . o accumulated over the n-tiles (zero before dgrad1)
  float* dx_acc;       // [T, H] fp32 (zero before dgrad2)
  bf16* dW1;           // [E, H, I]
  bf16* dW3;           // [E, H, I]
  bf16* dW2;           // [E, I, H]
  float* dWg;          // [H, E]
  int32_t* err;
  int T, H, I, E, k, BM;
  int pool;            // rows of dg / du / aw
  int BN;              // dgrad2: columns of H per task (256, or 128 when H % 256 != 0)
  int BNi;             // wgrad2: columns of I per task (256, or 128 when I % 256 != 0)
  int NE;              // dwg: columns of the dl tile, E rounded up to 64
  unsigned long long timeout_ns;
};

struct BwdSmem {
  float out_stage[4][32][36];   // dgrad2 combine staging (combine_rows)
  int out_tok[4][32];
  uint64_t full[kBwdStages];
  uint64_t empty[kBwdStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t da_empty[2];         // dgrad1: the two da slots (TMEM columns 256.., 384..) are free
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int nblocks;
  int block_start[kMaxExperts + 1];
};

constexpr size_t kBwdSmemBytes = 1024 + (size_t)kBwdStages * kBwdStageBytes + sizeof(BwdSmem);

struct BwdTask {
  int e;     // expert (dgrad, wgrad)
  int b;     // block (dgrad)
  int m, n;  // output tile: rows m * 128, columns n * (tile width)
  int nk;    // K blocks of 64
};

__device__ __forceinline__ void bwd_error(const BwdParams& p, BwdSmem& s, int code, int detail) {
  if (atomicCAS(p.err, 0, code) == 0) p.err[1] = detail;
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
}

// Bounded wait of a whole warp on a barrier phase (as in the forward kernels).
__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, const BwdParams& p, BwdSmem& s, int where) {
  bool ok = ptx::mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = ptx::globaltimer();
    uint64_t next_check = t0 + 4000;
    while (true) {
      if (ptx::mbar_try_wait(bar, parity)) {
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
        bwd_error(p, s, kDevTimeout, 0x200 | where);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

template <int Kind>
__device__ __forceinline__ int bwd_num_tasks(const BwdParams& p, const BwdSmem& s) {
  if (Kind == kBwdDgrad1) return s.nblocks * (p.I / 128);
  if (Kind == kBwdDgrad2) return s.nblocks * (p.H / p.BN);
  if (Kind == kBwdWgrad13) return p.E * (p.H / 128) * (p.I / 128);
  if (Kind == kBwdWgrad2) return p.E * (p.H / 128) * (p.I / p.BNi);
  return p.H / 128;
}

// Expert owning block b (block_start is non-decreasing).
__device__ __forceinline__ int bwd_expert_of_unit(const int* starts, int E, long long unit, int per) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)starts[mid] * per <= unit) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <int Kind>
__device__ __forceinline__ BwdTask bwd_decode(int t, const BwdParams& p, const BwdSmem& s) {
  BwdTask task{0, 0, 0, 0, 0};
  if (Kind == kBwdDgrad1 || Kind == kBwdDgrad2) {
    // an expert's tasks are its blocks x column tiles, column-tile major, so that
    // concurrent tasks share a weight tile
    const int NT = Kind == kBwdDgrad1 ? p.I / 128 : p.H / p.BN;
    const int e = bwd_expert_of_unit(s.block_start, p.E, t, NT);
    const int nb = s.block_start[e + 1] - s.block_start[e];
    const int local = t - s.block_start[e] * NT;
    task.e = e;
    task.n = local / nb;
    task.b = s.block_start[e] + local % nb;
    task.nk = Kind == kBwdDgrad1 ? 2 * (p.H / 64) : 2 * (p.I / 64);
  } else if (Kind == kBwdWgrad13 || Kind == kBwdWgrad2) {
    const int MT = p.H / 128;
    const int NT = Kind == kBwdWgrad13 ? p.I / 128 : p.I / p.BNi;
    task.e = t / (MT * NT);
    const int local = t - task.e * MT * NT;
    task.m = local / NT;
    task.n = local % NT;
    const int slots = (s.block_start[task.e + 1] - s.block_start[task.e]) * p.BM;
    task.nk = (slots + 63) / 64;
  } else {
    task.m = t;
    task.nk = (p.T + 63) / 64;
  }
  return task;
}

// ---------------------------------------------------------------- warp 0: TMA producer
template <int Kind>
__device__ void bwd_producer(const BwdParams& p, BwdSmem& s, uint8_t* tiles) {
  const int lane = ptx::lane_id();
  const uint64_t pol_w = ptx::policy_evict_first();
  const uint64_t pol_n = ptx::policy_evict_normal();
  const int ntasks = bwd_num_tasks<Kind>(p, s);
  int stage = 0;
  uint32_t phase = 0;
  uint32_t issued = 0, issued_parity = 0;
  bool ok = true;
  for (int t = blockIdx.x; t < ntasks && ok; t += gridDim.x) {
    const BwdTask task = bwd_decode<Kind>(t, p, s);
    for (int kb = 0; kb < task.nk; ++kb) {
      if (!bwd_wait(&s.empty[stage], phase ^ 1, p, s, 1)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const uint32_t a = ptx::smem_u32(tiles + stage * kBwdStageBytes);
        const uint32_t b = a + kBwdABytes;
        uint64_t* bar = &s.full[stage];
        if (Kind == kBwdDgrad1) {
          const int n0 = task.n * 128;
          const bool da_part = kb < p.H / 64;   // dy W2^T first, then x [W1 | W3]
          const int kh = (da_part ? kb : kb - p.H / 64) * 64;
          // one arrival with every byte of the stage: B, and A when it comes by TMA
          ptx::mbar_arrive_expect_tx(bar, (da_part ? 2 : 4) * kBoxBytes + (p.permuted ? kTileABytes : 0));
          if (p.permuted)   // the block's dy rows (first half of K) or x rows (second half)
            ptx::tma_load_2d(a, da_part ? &p.tm_dyp : &p.tm_xp, bar, kh, task.b * p.BM, pol_n);
          if (da_part) {   // W2 rows i = n0 .. n0+127, K = h (K-major)
            ptx::tma_load_2d(b, &p.tm_w2, bar, kh, task.e * p.I + n0, pol_w);
          } else {         // W1 | W3 columns n0 .. n0+127, rows h of this K block (MN-major)
            const int row = task.e * p.H + kh;
            ptx::tma_load_2d(b, &p.tm_w1, bar, n0, row, pol_w);
            ptx::tma_load_2d(b + kBoxBytes, &p.tm_w1, bar, n0 + 64, row, pol_w);
            ptx::tma_load_2d(b + 2 * kBoxBytes, &p.tm_w3, bar, n0, row, pol_w);
            ptx::tma_load_2d(b + 3 * kBoxBytes, &p.tm_w3, bar, n0 + 64, row, pol_w);
          }
        } else if (Kind == kBwdDgrad2) {
          const int ki = kb < p.I / 64 ? kb : kb - p.I / 64;
          const bool second = kb >= p.I / 64;   // du with W3 after dg with W1
          ptx::mbar_arrive_expect_tx(bar, kTileABytes + p.BN * 128);
          ptx::tma_load_2d(a, second ? &p.tm_a2 : &p.tm_a, bar, ki * 64, task.b * p.BM, pol_n);
          ptx::tma_load_2d(b, second ? &p.tm_w3 : &p.tm_w1, bar, ki * 64, task.e * p.H + task.n * p.BN, pol_w);
        } else if (Kind == kBwdWgrad13) {
          const int s0 = s.block_start[task.e] * p.BM + kb * 64, n0 = task.n * 128;
          ptx::mbar_arrive_expect_tx(bar, 4 * kBoxBytes + (p.permuted ? 2 * kBoxBytes : 0));
          if (p.permuted) {   // x^T: 128 columns of x (2 MN-major boxes) of the slots
            ptx::tma_load_2d(a, &p.tm_xp, bar, task.m * 128, s0, pol_n);
            ptx::tma_load_2d(a + kBoxBytes, &p.tm_xp, bar, task.m * 128 + 64, s0, pol_n);
          }
          ptx::tma_load_2d(b, &p.tm_b, bar, n0, s0, pol_n);
          ptx::tma_load_2d(b + kBoxBytes, &p.tm_b, bar, n0 + 64, s0, pol_n);
          ptx::tma_load_2d(b + 2 * kBoxBytes, &p.tm_b2, bar, n0, s0, pol_n);
          ptx::tma_load_2d(b + 3 * kBoxBytes, &p.tm_b2, bar, n0 + 64, s0, pol_n);
        } else if (Kind == kBwdWgrad2) {   // aw columns n0 .. n0+BNi-1 of the slots (MN-major B)
          const int s0 = s.block_start[task.e] * p.BM + kb * 64, n0 = task.n * p.BNi;
          ptx::mbar_arrive_expect_tx(bar, (p.BNi / 64) * kBoxBytes + (p.permuted ? 2 * kBoxBytes : 0));
          if (p.permuted) {   // dy^T: 128 columns of dy (2 MN-major boxes) of the slots
            ptx::tma_load_2d(a, &p.tm_dyp, bar, task.m * 128, s0, pol_n);
            ptx::tma_load_2d(a + kBoxBytes, &p.tm_dyp, bar, task.m * 128 + 64, s0, pol_n);
          }
          for (int j = 0; j < p.BNi / 64; ++j) ptx::tma_load_2d(b + j * kBoxBytes, &p.tm_b, bar, n0 + j * 64, s0, pol_n);
        } else {   // dwg: x^T (rows h) and dl (columns e), K = tokens
          const int m0 = task.m * 128;
          ptx::mbar_arrive_expect_tx(bar, 2 * kBoxBytes + (p.NE / 64) * kBoxBytes);
          ptx::tma_load_2d(a, &p.tm_a, bar, m0, kb * 64, pol_n);
          ptx::tma_load_2d(a + kBoxBytes, &p.tm_a, bar, m0 + 64, kb * 64, pol_n);
          for (int j = 0; j < p.NE / 64; ++j) ptx::tma_load_2d(b + j * kBoxBytes, &p.tm_b, bar, j * 64, kb * 64, pol_n);
        }
      }
      __syncwarp();
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == kBwdStages) {
        stage = 0;
        phase ^= 1;
      }
    }
  }
  // let every issued copy land before the CTA can exit
  for (int st = 0; st < kBwdStages; ++st)
    if (issued & (1u << st)) {
      const uint64_t t0 = ptx::globaltimer();
      while (!ptx::mbar_try_wait(&s.full[st], (issued_parity >> st) & 1u))
        if (ptx::globaltimer() - t0 > p.timeout_ns) break;
    }
}

// ---------------------------------------------------------------- warps 6..9: gathered operands
// dgrad1: the x rows (first H/64 K blocks) and the dy rows (the rest) of the
// block's slots, K-major like the forward's A tile; wgrad13: x^T, 64 slots x
// 128 columns of H as two MN-major boxes; wgrad2: dy^T as the B operand, 64
// slots x BN columns of H (BN/64 boxes). Rows of padding slots, and slots
// past the expert's range, are zeros.
template <int Kind>
__device__ void bwd_gather(const BwdParams& p, BwdSmem& s, uint8_t* tiles, int g) {
  const int lane = ptx::lane_id();
  const int tid = g * 32 + lane;   // 0 .. 127
  const int ntasks = bwd_num_tasks<Kind>(p, s);
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int t = blockIdx.x; t < ntasks && ok; t += gridDim.x) {
    const BwdTask task = bwd_decode<Kind>(t, p, s);
    if (Kind == kBwdDgrad1 && !p.permuted) {
      // this lane's 8 rows of the block and its 16-byte column c (as in the forward's gather)
      const int c = lane & 7;
      int tok[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = (j * kBwdGatherWarps + g) * 4 + (lane >> 3);
        tok[j] = r < p.BM ? p.slot_token[task.b * p.BM + r] : -1;
        if (tok[j] >= p.T) {
          bwd_error(p, s, kDevBounds, 0x1000 | task.b);
          tok[j] = -1;
        }
      }
      for (int kb = 0; kb < task.nk; ++kb) {
        if (!bwd_wait(&s.empty[stage], phase ^ 1, p, s, 2)) {
          ok = false;
          break;
        }
        const uint32_t a = ptx::smem_u32(tiles + stage * kBwdStageBytes);
        const bool da_part = kb < p.H / 64;   // dy rows first, then x rows
        const bf16* base = da_part ? p.dy : p.x;
        const int kc = (da_part ? kb : kb - p.H / 64) * 64 + c * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = (j * kBwdGatherWarps + g) * 4 + (lane >> 3);
          const bf16* src = (tok[j] < 0 ? p.zero_row : base + (size_t)tok[j] * p.H) + kc;
          ptx::cp_async_16(a + r * 128 + ((c ^ (r & 7)) << 4), src);
        }
        ptx::cp_async_mbar_arrive_noinc(&s.full[stage]);
        if (++stage == kBwdStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    } else if ((Kind == kBwdWgrad13 || Kind == kBwdWgrad2) && !p.permuted) {
      const int s_begin = s.block_start[task.e] * p.BM;
      const int s_end = s.block_start[task.e + 1] * p.BM;
      // the A operand, 64 slot rows x 16 chunks (128 columns of H) of x (wgrad13) or dy (wgrad2).
      // A thread's chunks of a stage lie on rows kr0 + rstep * i (i < per) at one chunk column:
      // thread tid takes chunk q = 128 i + tid, i.e. row q / cpr, column q % cpr.
      const int cpr = 16;   // 16-byte chunks per row
      const int col0 = task.m * 128;
      const bf16* base = Kind == kBwdWgrad13 ? p.x : p.dy;
      const int per = 64 * cpr / 128;   // chunks per thread per stage: 8
      const int kr0 = tid / cpr, rstep = 128 / cpr, cc = tid % cpr;
      const int box = cc >> 3, c = cc & 7;
      // the tokens of a stage's rows are loaded one stage ahead, so that their round trip
      // overlaps the wait for a free stage and the previous stage's copies
      auto load_tokens = [&](int kb, int (&tk)[16]) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          tk[i] = -1;
          const int slot = s_begin + kb * 64 + kr0 + rstep * i;
          if (i < per && kb < task.nk && slot < s_end) tk[i] = __ldg(p.slot_token + slot);
        }
      };
      int tk_cur[16], tk_next[16];
      load_tokens(0, tk_cur);
      for (int kb = 0; kb < task.nk; ++kb) {
        load_tokens(kb + 1, tk_next);
        if (!bwd_wait(&s.empty[stage], phase ^ 1, p, s, 3)) {
          ok = false;
          break;
        }
        const uint32_t dst0 = ptx::smem_u32(tiles + stage * kBwdStageBytes);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i < per) {
            const int kr = kr0 + rstep * i;
            int tk = tk_cur[i];
            if (tk >= p.T) {
              bwd_error(p, s, kDevBounds, 0x2000 | task.e);
              tk = -1;
            }
            const bf16* src = (tk < 0 ? p.zero_row : base + (size_t)tk * p.H) + col0 + cc * 8;
            ptx::cp_async_16(dst0 + box * kBoxBytes + kr * 128 + ((c ^ (kr & 7)) << 4), src);
          }
        }
        ptx::cp_async_mbar_arrive_noinc(&s.full[stage]);
#pragma unroll
        for (int i = 0; i < 16; ++i) tk_cur[i] = tk_next[i];
        if (++stage == kBwdStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    } else {
      // no gathered operand: one (copy-less) arrival per stage keeps the barrier counts uniform
      for (int kb = 0; kb < task.nk; ++kb) {
        if (!bwd_wait(&s.empty[stage], phase ^ 1, p, s, 4)) {
          ok = false;
          break;
        }
        ptx::cp_async_mbar_arrive_noinc(&s.full[stage]);
        if (++stage == kBwdStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }
  ptx::cp_async_wait_all();
}

// ---------------------------------------------------------------- warp 1: MMA issuer
template <int Kind>
__device__ void bwd_mma(const BwdParams& p, BwdSmem& s, uint8_t* tiles, uint32_t tmem_base) {
  const int lane = ptx::lane_id();
  const int ntasks = bwd_num_tasks<Kind>(p, s);
  constexpr int kAccs = Kind == kBwdDgrad1 ? 1 : 2;   // dgrad1 holds g|u and da: 384 columns
  // instruction descriptors: A K-major unless wgrad / dwg (x^T, aw^T are MN-major)
  const bool a_mn = Kind == kBwdWgrad13 || Kind == kBwdWgrad2 || Kind == kBwdDwg;
  const uint32_t id_main =
      Kind == kBwdDgrad1 ? ptx::idesc_bf16_f32(128, 256, false, true)
      : Kind == kBwdDgrad2 ? ptx::idesc_bf16_f32(128, p.BN, false, false)
      : Kind == kBwdWgrad13 ? ptx::idesc_bf16_f32(128, 256, true, true)
      : Kind == kBwdWgrad2 ? ptx::idesc_bf16_f32(128, p.BNi, true, true)
                           : ptx::idesc_bf16_f32(128, p.NE, true, true);
  const uint32_t id_da = ptx::idesc_bf16_f32(128, 128, false, false);   // dgrad1: dy W2^T, W2 rows K-major
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool issued_any = false;
  bool ok = true;
  int nt = 0;   // dgrad1: tasks of this CTA so far (da slot nt & 1; g|u columns shared)
  for (int t = blockIdx.x; t < ntasks && ok; t += gridDim.x) {
    const BwdTask task = bwd_decode<Kind>(t, p, s);
    if (task.nk == 0) continue;   // no K: the epilogue writes zeros without the accumulator
    uint32_t d = tmem_base + acc * 256, d_da = 0;
    if (Kind == kBwdDgrad1) {
      // da slot nt & 1 was last read by the epilogue of task nt - 2 (use (nt >> 1) of the slot)
      const int slot = nt & 1;
      if (!bwd_wait(&s.da_empty[slot], ((nt >> 1) & 1) ^ 1, p, s, 5)) break;
      d = tmem_base;
      d_da = tmem_base + 256 + 128 * slot;
    } else if (!bwd_wait(&s.acc_empty[acc], acc_phase ^ 1, p, s, 5)) {
      break;
    }
    ptx::tc_fence_after();
    for (int kb = 0; kb < task.nk; ++kb) {
      // dgrad1: the g|u columns were last read by the epilogue of task nt - 1
      if (Kind == kBwdDgrad1 && kb == p.H / 64) {
        if (!bwd_wait(&s.acc_empty[0], (nt & 1) ^ 1, p, s, 5)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
      }
      if (!bwd_wait(&s.full[stage], phase, p, s, 6)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      ptx::fence_proxy_async_shared();   // cp.async-written rows -> the tensor core's reads
      if (lane == 0) {
        const uint32_t a = ptx::smem_u32(tiles + stage * kBwdStageBytes);
        const uint32_t b = a + kBwdABytes;
        const bool da_part = Kind == kBwdDgrad1 && kb < p.H / 64;
        const int kfirst = Kind == kBwdDgrad1 && !da_part ? p.H / 64 : 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = a_mn ? ptx::smem_desc_sw128(a + kk * 2048, kBoxBytes, 1024)
                                   : ptx::smem_desc_sw128(a + kk * 32, 16, 1024);
          // B: MN-major boxes (weights of dgrad1's first part, dg / du, dy, dl) or K-major rows
          const bool b_kmajor = Kind == kBwdDgrad2 || da_part;
          const uint64_t bd = b_kmajor ? ptx::smem_desc_sw128(b + kk * 32, 16, 1024)
                                       : ptx::smem_desc_sw128(b + kk * 2048, kBoxBytes, 1024);
          const uint32_t acc_flag = (kb != kfirst || kk != 0) ? 1u : 0u;
          ptx::mma_bf16(da_part ? d_da : d, ad, bd, da_part ? id_da : id_main, acc_flag);
        }
        ptx::mma_commit(&s.empty[stage]);
        issued_any = true;
      }
      __syncwarp();
      if (++stage == kBwdStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (!ok) break;
    if (lane == 0) ptx::mma_commit(&s.acc_full[acc]);
    __syncwarp();
    ++nt;
    if (++acc == kAccs) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
  issued_any = __any_sync(0xffffffffu, issued_any);
  if (issued_any) {   // every MMA done before TMEM is freed
    if (lane == 0) ptx::mma_commit(&s.mma_done);
    __syncwarp();
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(&s.mma_done, 0))
      if (ptx::globaltimer() - t0 > p.timeout_ns) break;
  }
}

// 32 fp32 accumulator values -> 32 bf16 at dst (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_bf16x32(bf16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d4[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                       pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

// A warp's 32 rows x 32 columns of a bf16 output (lane = row, f = its 32 columns, base = row 0,
// column 0, pitch in elements), staged in shared memory (rows padded to 36 floats) so that each
// store instruction writes 8 rows x 64 contiguous bytes (4 lanes a row) instead of 32 rows x 16
// bytes: a quarter of the store transactions.
__device__ __forceinline__ void store_rows_bf16_staged(float (*stage)[36], const float (&f)[32], bf16* base,
                                                       size_t pitch) {
  const int lane = ptx::lane_id();
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(stage[lane])[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
  __syncwarp();
  const int cq = (lane & 3) * 8;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int rr = (lane >> 2) + 8 * j;
    const float4 a = *reinterpret_cast<const float4*>(&stage[rr][cq]);
    const float4 b = *reinterpret_cast<const float4*>(&stage[rr][cq + 4]);
    *reinterpret_cast<uint4*>(base + (size_t)rr * pitch + cq) =
        make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
  __syncwarp();
}

// ---------------------------------------------------------------- warps 2..5: epilogue
// With the operands by TMA (p.permuted), the four gather warps have nothing to copy; for
// dgrad-1 and dW1/dW3 they become a second set of epilogue warps: the warp of each TMEM lane
// quarter in warps 2-5 takes the first half of the accumulator's columns, the one in 6-9 the
// second half.
template <int Kind>
__device__ __forceinline__ bool bwd_helpers(const BwdParams& p) {
  return p.permuted && (Kind == kBwdDgrad1 || Kind == kBwdWgrad13);
}

template <int Kind>
__device__ void bwd_epilogue(const BwdParams& p, BwdSmem& s, uint32_t tmem_base, int half) {
  const int warp = threadIdx.x >> 5;
  const int lane = ptx::lane_id();
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;   // accumulator row (TMEM lane) of this thread
  const bool split = bwd_helpers<Kind>(p);   // columns split between this warp and its helper
  const int ntasks = bwd_num_tasks<Kind>(p, s);
  constexpr int kAccs = Kind == kBwdDgrad1 ? 1 : 2;
  int acc = 0;
  uint32_t acc_phase = 0;
  int nt_epi = 0;   // dgrad1: tasks of this CTA so far (their da slots alternate)
  for (int t = blockIdx.x; t < ntasks; t += gridDim.x) {
    const BwdTask task = bwd_decode<Kind>(t, p, s);
    const bool has_acc = task.nk > 0;
    if (has_acc) {
      if (!bwd_wait(&s.acc_full[acc], acc_phase, p, s, 7)) break;
      ptx::tc_fence_after();
    }
    const uint32_t tb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 256;
    auto release = [&]() {
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.acc_empty[acc]);
    };
    if (Kind == kBwdDgrad1) {
      const int dslot = nt_epi & 1;   // this task's da slot (TMEM columns 256 + 128 * dslot)
      const int slot = task.b * p.BM + r;
      int tok = r < p.BM ? p.slot_token[slot] : -1;
      int j = 0;
      float w = 0.f;
      if (tok >= p.T) {
        bwd_error(p, s, kDevBounds, 0x3000 | task.b);
        tok = -1;
      }
      if (tok >= 0) {
        j = p.slot_topk[slot];
        if (j < 0 || j >= p.k) {
          bwd_error(p, s, kDevBounds, 0x4000 | task.b);
          tok = -1;
        } else {
          w = p.topk_w[(size_t)tok * p.k + j];
        }
      }
      const int n0 = task.n * 128;
      float dwp = 0.f;   // sum over this warp's columns of a_i * da~_i
      const int c0 = split ? 2 * half : 0, c1 = split ? c0 + 2 : 4;
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        uint32_t g[32], u[32], v[32];
        ptx::tmem_ld32(tb + c * 32, g);
        ptx::tmem_ld32(tb + 128 + c * 32, u);
        ptx::tmem_ld32(tb + 256 + 128 * dslot + c * 32, v);
        ptx::tmem_ld_wait();
        float dg[32], du[32], aw[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float gg = __uint_as_float(g[i]), uu = __uint_as_float(u[i]), dat = __uint_as_float(v[i]);
          const float sg = 1.f / (1.f + __expf(-gg));   // sigmoid(g)
          const float si = gg * sg;                      // silu(g)
          const float a = __bfloat162float(__float2bfloat16_rn(si * uu));   // the forward's rounded activation
          const float da = w * dat;
          dg[i] = da * uu * sg * (1.f + gg * (1.f - sg));
          du[i] = da * si;
          aw[i] = w * a;
          dwp += a * dat;
        }
        if (tok >= 0) {   // padding slots: their rows stay as the dgrad2 / wgrad zeros need (never read)
          const size_t o = (size_t)slot * p.I + n0 + c * 32;
          store_bf16x32(p.dg + o, dg);
          store_bf16x32(p.du + o, du);
          store_bf16x32(p.aw + o, aw);
        } else if (r < p.BM) {   // padding slot of the block: zero rows (read by dgrad2 and the wgrads)
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = 0.f;
          const size_t o = (size_t)slot * p.I + n0 + c * 32;
          store_bf16x32(p.dg + o, z);
          store_bf16x32(p.du + o, z);
          store_bf16x32(p.aw + o, z);
        }
      }
      release();   // the g|u columns
      if (lane == 0) ptx::mbar_arrive(&s.da_empty[dslot]);
      ++nt_epi;
      if (tok >= 0) atomicAdd(p.dw + (size_t)tok * p.k + j, dwp);
    } else if (Kind == kBwdDgrad2) {
      int tok = r < p.BM ? p.slot_token[task.b * p.BM + r] : -1;
      if (tok >= p.T) {
        bwd_error(p, s, kDevBounds, 0x5000 | task.b);
        tok = -1;
      }
      combine_rows(tb, p.BN, 1.f, tok, p.dx_acc, p.H, task.n * p.BN, s.out_stage[quarter], s.out_tok[quarter],
                   nullptr, release);
    } else {
      // weight-gradient tiles: row r of the tile, ncols columns, bf16 (fp32 for dWg)
      const int ncols = Kind == kBwdWgrad13 ? 256 : Kind == kBwdWgrad2 ? p.BNi : p.NE;
      const int c0 = split ? half * (ncols / 64) : 0, c1 = split ? c0 + ncols / 64 : ncols / 32;
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        float f[32];
        if (has_acc) {
          uint32_t v[32];
          ptx::tmem_ld32(tb + c * 32, v);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = 0.f;
        }
        if (Kind == kBwdWgrad13) {   // columns 0..127: dW1, 128..255: dW3, of I columns n*128 ..
          bf16* out = c < 4 ? p.dW1 : p.dW3;
          if (split) {   // helper epilogue warps share the staging rows: one row per lane
            const size_t o = ((size_t)task.e * p.H + task.m * 128 + r) * p.I + task.n * 128 + (c & 3) * 32;
            store_bf16x32(out + o, f);
          } else {
            const size_t o = ((size_t)task.e * p.H + task.m * 128 + quarter * 32) * p.I + task.n * 128 + (c & 3) * 32;
            store_rows_bf16_staged(s.out_stage[quarter], f, out + o, p.I);
          }
        } else if (Kind == kBwdWgrad2) {
          // the tile is dW2[e]^T (rows h, columns i): each 32 x 32 block goes through the warp's
          // staging rows transposed (row ii = column i0 + 32c + ii of the tile), then 4 lanes write
          // 32 consecutive h (64 bytes) of each of 8 rows of dW2 per instruction
          float (*stg)[36] = s.out_stage[quarter];
#pragma unroll
          for (int i = 0; i < 32; ++i) stg[i][lane] = f[i];
          __syncwarp();
          const int hq = (lane & 3) * 8;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int ii = (lane >> 2) + 8 * j;
            const float4 a = *reinterpret_cast<const float4*>(&stg[ii][hq]);
            const float4 b = *reinterpret_cast<const float4*>(&stg[ii][hq + 4]);
            const size_t o = ((size_t)task.e * p.I + task.n * p.BNi + c * 32 + ii) * p.H + task.m * 128 + quarter * 32 + hq;
            *reinterpret_cast<uint4*>(p.dW2 + o) = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                             pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
          }
          __syncwarp();
        } else {
          float* out = p.dWg + (size_t)(task.m * 128 + r) * p.E;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i < p.E) out[c * 32 + i] = f[i];
        }
      }
      if (has_acc) release();
    }
    if (has_acc && ++acc == kAccs) {
      acc = 0;
      acc_phase ^= 1;
    }
  }
}

template <int Kind>
__global__ void __launch_bounds__(kBwdThreads, 1) moe_backward_gemm_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdSmem& s = *reinterpret_cast<BwdSmem*>(tiles + (size_t)kBwdStages * kBwdStageBytes);
  const int warp = threadIdx.x >> 5;
  const bool helpers = bwd_helpers<Kind>(p);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kBwdStages; ++i) {
      // producer + every gather lane (with helper epilogue warps: the producer alone)
      ptx::mbar_init(&s.full[i], helpers ? 1 : 1 + 32 * kBwdGatherWarps);
      ptx::mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.acc_full[i], 1);
      ptx::mbar_init(&s.acc_empty[i], helpers ? 8 : 4);   // every epilogue warp releases the accumulator
      ptx::mbar_init(&s.da_empty[i], helpers ? 8 : 4);
    }
    ptx::mbar_init(&s.mma_done, 1);
    s.abort = 0;
    const int nb = *p.sched;
    s.nblocks = nb;
    ptx::fence_mbar_init();
  }
  for (int e = threadIdx.x; e <= p.E; e += kBwdThreads) s.block_start[e] = p.block_start[e];
  if (warp == 0 && threadIdx.x == 0) {
    ptx::prefetch_tmap(&p.tm_w1);
    ptx::prefetch_tmap(&p.tm_w3);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&s.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // the block count comes from the dispatch: range-check it against the expert starts
  if (threadIdx.x == 0 && (s.nblocks != s.block_start[p.E] || s.nblocks < 0)) bwd_error(p, s, kDevBounds, 0x6000);
  __syncthreads();
  const uint32_t tmem_base = s.tmem_base;
  if (Kind == kBwdDgrad1 && blockIdx.x == 0) {
    // The weight-gradient kernels read K blocks of 64 slots; with BLOCK_M < 64 the last one of an
    // expert runs past its slots (those rows are multiplied by zeros there), and the pool's rows
    // past the last used slot hold nothing written: zero the 64 after it, so that no stale NaN
    // meets those zeros.
    const size_t r0 = (size_t)s.nblocks * p.BM, r1 = min((size_t)p.pool, r0 + 64);
    const size_t n16 = (r1 > r0 ? r1 - r0 : 0) * p.I / 8;   // 16-byte chunks per buffer
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (size_t i = threadIdx.x; i < n16; i += kBwdThreads) {
      reinterpret_cast<uint4*>(p.dg + r0 * p.I)[i] = z;
      reinterpret_cast<uint4*>(p.du + r0 * p.I)[i] = z;
      reinterpret_cast<uint4*>(p.aw + r0 * p.I)[i] = z;
    }
  }
  if (!*reinterpret_cast<volatile int*>(&s.abort)) {
    if (warp == 0) bwd_producer<Kind>(p, s, tiles);
    else if (warp == 1) bwd_mma<Kind>(p, s, tiles, tmem_base);
    else if (warp < 6) bwd_epilogue<Kind>(p, s, tmem_base, 0);
    else if (helpers) bwd_epilogue<Kind>(p, s, tmem_base, 1);
    else bwd_gather<Kind>(p, s, tiles, warp - 6);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------- gate backward (no tensor cores)
// One warp per token: dl[t,j] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]) (the
// softmax over the k kept logits), the dense row dl[t, :] (bf16, zeros
// except the k selected experts) for dWg = x^T dl, dbias[e] += dl[t,j]
// (summed per CTA in shared memory first), and
// dx[t] = bf16(dx_acc[t] + sum_j dl[t,j] Wg[:, e_j]) with Wg read through
// its transpose WgT [E, H] (rows contiguous).
constexpr int kGateThreads = 256;

__global__ void __launch_bounds__(kGateThreads) moe_gate_backward_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, const float* __restrict__ dw,
    const bf16* __restrict__ WgT, const float* __restrict__ dx_acc, bf16* __restrict__ dx, bf16* __restrict__ dl_dense,
    float* __restrict__ dbias, int32_t* err, int T, int H, int E, int k, int NE) {
  __shared__ float s_bias[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += kGateThreads) s_bias[e] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * kGateThreads + threadIdx.x) >> 5;
  if (t < T) {
    // lane j < k holds pair (t, j)
    int e = 0;
    float w = 0.f, d = 0.f;
    if (lane < k) {
      e = topk_idx[(size_t)t * k + lane];
      w = topk_w[(size_t)t * k + lane];
      d = dw[(size_t)t * k + lane];
      if (e < 0 || e >= E) {
        atomicCAS(err, 0, kDevBounds);
        e = 0;
        w = 0.f;
      }
    }
    float wd = w * d;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wd += __shfl_xor_sync(0xffffffffu, wd, off);
    const float dl = lane < k ? w * (d - wd) : 0.f;
    if (lane < k && dbias != nullptr) atomicAdd(&s_bias[e], dl);
    // dense dl row (bf16, NE >= E columns), zeros elsewhere
    for (int c = lane; c < NE; c += 32) {
      float v = 0.f;
      for (int j = 0; j < k; ++j) {
        const int ej = __shfl_sync(0xffffffffu, e, j);
        const float lj = __shfl_sync(0xffffffffu, dl, j);
        if (ej == c) v = lj;
      }
      dl_dense[(size_t)t * NE + c] = __float2bfloat16_rn(v);
    }
    // dx row: 8 columns per lane per step
    int ej[8];
    float lj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ej[j] = __shfl_sync(0xffffffffu, e, j);
      lj[j] = __shfl_sync(0xffffffffu, dl, j);
    }
    for (int h0 = lane * 8; h0 < H; h0 += 256) {
      const float4 a0 = *reinterpret_cast<const float4*>(dx_acc + (size_t)t * H + h0);
      const float4 a1 = *reinterpret_cast<const float4*>(dx_acc + (size_t)t * H + h0 + 4);
      float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      for (int j = 0; j < k; ++j) {
        const uint4 q = *reinterpret_cast<const uint4*>(WgT + (size_t)ej[j] * H + h0);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(b[i]);
          v[2 * i] += lj[j] * f.x;
          v[2 * i + 1] += lj[j] * f.y;
        }
      }
      *reinterpret_cast<uint4*>(dx + (size_t)t * H + h0) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
  }
  __syncthreads();
  if (dbias != nullptr)
    for (int e = threadIdx.x; e < E; e += kGateThreads)
      if (s_bias[e] != 0.f) atomicAdd(dbias + e, s_bias[e]);
}

// Rows of x and dy in slot order for the backward's TMA operands: xp[s] = x[t], dyp[s] = dy[t]
// for slot s with token t, zeros for padding slots and for the 64 rows after the last used
// slot (a weight-gradient K block of 64 slots may reach past the pool's last expert). One
// warp per row, up to four 16-byte loads of x and four of dy per lane in flight.
__global__ void __launch_bounds__(256) moe_permute_rows_kernel(const bf16* __restrict__ x, const bf16* __restrict__ dy,
                                                               const int32_t* __restrict__ slot_token,
                                                               const int32_t* __restrict__ nblocks, bf16* __restrict__ xp,
                                                               bf16* __restrict__ dyp, int32_t* err, int T, int H, int BM,
                                                               int pool) {
  const int rows = min(*nblocks * BM + 64, pool);
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int sl = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; sl < rows; sl += warps) {
    int t = sl < *nblocks * BM ? slot_token[sl] : -1;
    if (t >= T) {
      atomicCAS(err, 0, kDevBounds);
      t = -1;
    }
    const uint4* xs = reinterpret_cast<const uint4*>(x + (size_t)(t < 0 ? 0 : t) * H);
    const uint4* ds = reinterpret_cast<const uint4*>(dy + (size_t)(t < 0 ? 0 : t) * H);
    uint4* xo = reinterpret_cast<uint4*>(xp + (size_t)sl * H);
    uint4* dout = reinterpret_cast<uint4*>(dyp + (size_t)sl * H);
    const uint4 z = make_uint4(0, 0, 0, 0);
    const int n = H / 8;
    // four 16-byte pieces of each row in flight per lane before the stores
    for (int i0 = lane; i0 < n; i0 += 32 * 4) {
      uint4 a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + 32 * u;
        a[u] = (t < 0 || i >= n) ? z : __ldg(xs + i);
        b[u] = (t < 0 || i >= n) ? z : __ldg(ds + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + 32 * u;
        if (i < n) {
          xo[i] = a[u];
          dout[i] = b[u];
        }
      }
    }
  }
}

// WgT[e][h] = Wg[h][e] (32 x 32 tiles through shared memory).
__global__ void __launch_bounds__(256) moe_transpose_wg_kernel(const bf16* __restrict__ Wg, bf16* __restrict__ WgT,
                                                               int H, int E) {
  __shared__ bf16 tile[32][33];
  const int h0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  for (int i = threadIdx.x; i < 32 * 32; i += 256) {
    const int hh = i / 32, ee = i % 32;
    if (h0 + hh < H && e0 + ee < E) tile[hh][ee] = Wg[(size_t)(h0 + hh) * E + e0 + ee];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * 32; i += 256) {
    const int ee = i / 32, hh = i % 32;
    if (h0 + hh < H && e0 + ee < E) WgT[(size_t)(e0 + ee) * H + h0 + hh] = tile[hh][ee];
  }
}

}  // namespace moe
