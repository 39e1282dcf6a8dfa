// Shared definitions of the CUDA path: device error codes, tile constants.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace moe {

using bf16 = __nv_bfloat16;

// Sticky device error codes written to the workspace error word (first one wins).
enum DeviceError : int {
  kDevOk = 0,
  kDevTimeout = 1,   // a bounded wait ran out
  kDevBounds = 2,    // an index read from routing metadata was out of range
};

// Expert id a router writes for a token whose selection it gave up on (a
// bounded wait ran out); the dispatch scatter skips it and records a timeout.
constexpr int kAbortedExpert = -1;

// Router tile: tokens per CTA (one 16-row mma.sync tile per warp) and K chunk.
constexpr int kRouterTokens = 64;
constexpr int kRouterThreads = 128;
constexpr int kRouterKChunk = 64;
constexpr int kRouterMaxSplit = 64;     // at most this many H splits (only while tiles < SMs)

// Expert GEMM tile: M = 128 rows (one tcgen05 MMA), K block = 64 bf16 = one
// 128-byte swizzle row, N = 256 (L1: 128 columns of W1 next to the same 128 of
// W3; L2: 256 columns of W2, or 128 when H is not a multiple of 256).
constexpr int kTileM = 128;
constexpr int kBK = 64;
constexpr int kL1TileN = 128;          // columns of I per L1 task (per weight)
constexpr int kStages = 4;
constexpr int kTileABytes = kTileM * kBK * 2;      // 16 KB
constexpr int kBoxBytes = 64 * kBK * 2;            // one 64x64 bf16 box, 8 KB
constexpr int kTileBBytes = 4 * kBoxBytes;         // 32 KB
constexpr int kStageBytes = kTileABytes + kTileBBytes;
constexpr int kTaskRing = 4;
#ifndef MOE_GATHER_WARPS
#define MOE_GATHER_WARPS 4
#endif
constexpr int kGatherWarps = MOE_GATHER_WARPS;     // warps that gather routed x rows
// expert-GEMM CTA: producer, MMA (or relay), 4 epilogue warps, A-row warps, scheduler
constexpr int kGemm1Threads = 224 + 32 * kGatherWarps;
constexpr int kTmemCols = 512;                     // two 256-column fp32 accumulators
constexpr int kMaxGroups = 512;                    // block groups of the expert GEMM's task order
constexpr int kMaxExperts = 256;                   // routed experts per plan
constexpr int kMaxShared = 8;                      // shared experts per plan
constexpr int kMaxExpertsAll = kMaxExperts + kMaxShared;

// One record of the expert GEMM's task log (a plan option): written by the
// CTA (or CTA pair) that ran task number `task` of the launch. Timestamps are
// %globaltimer nanoseconds: the issue of the task's first MMA, the issue of
// its last one (the accumulator commit), and the end of its epilogue.
struct TaskRecord {
  uint32_t task;      // task number in the launch's task order
  uint32_t unit;      // block (single-CTA kernel) or block pair (CTA pairs)
  uint32_t expert;
  uint32_t phase_n;   // phase (0 = first GEMM, 1 = second GEMM) << 16 | n-tile
  uint32_t smid;      // SM of the CTA that issued the MMAs
  uint32_t cta;       // its blockIdx.x
  uint64_t t_first_mma;
  uint64_t t_last_mma;
  uint64_t t_done;
};
static_assert(sizeof(TaskRecord) == 48, "task records are 48 bytes");

__device__ __forceinline__ uint32_t smid_u32() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
  return r;
}

}  // namespace moe
