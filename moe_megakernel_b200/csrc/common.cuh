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

}  // namespace moe
