// Dispatch: exclusive scans of the router's per-chunk histograms, padding of
// every expert to a multiple of BLOCK_M, and the stable token -> slot
// permutation with its (token, top-k position) record per slot. Shared
// experts (same page, section 2.7: their two GEMM phases share the routed
// experts' task queue) follow the routed pool as experts E .. E+S-1 whose
// blocks hold every token once, in order, with the record (t, kSharedTopk).
//
// "MegaMoE 在 MoE 系统谱系中的位置", section 2.4 (TokenSrcMetadata: each pool
// slot records where its token came from, and the combine writes through that
// record), section 2.6 (dropless pool with at most BLOCK_M-1 padding rows per
// expert); "FlashMoE Kernel", section "通信" (padding to the tile happens only
// in place, for local compute).
#pragma once
#include <cstdint>

#include "common.cuh"

namespace moe {

struct DispatchParams {
  const int32_t* topk_idx;   // [T, k]
  const int32_t* rank;       // [T, k]
  int32_t* chunk_count;      // [num_chunks, E]: counts in, per-chunk bases out
  int32_t* expert_count;     // [E]
  int32_t* expert_offset;    // [E+1] slot offsets of the routed experts (multiples of BLOCK_M)
  int32_t* block_start;      // [E+S+1] first block of every expert, shared ones last
  int32_t* slot_token;       // [pool]
  int32_t* slot_topk;        // [pool]
  int32_t* l1_done;          // [pool / BLOCK_M] zeroed here
  int32_t* sched;            // [0] task counter, [1] blocks, [2] padded slots, [3] block groups
  int32_t* err;              // sticky device error word
  // Block groups of the expert GEMM's task order (nullptr: routing only, no groups).
  int32_t* group_start;      // [max_groups + 1] first block (or pair) of each group
  int32_t* l2_done;          // [pool / BLOCK_M] zeroed here
  // CTA-pair mode (nullptr: groups over blocks): pairs of consecutive blocks
  // of one expert, pair_start[e] = first pair of expert e; groups over pairs.
  int32_t* pair_start;       // [E+S+1]
  int T, E, S, k, BM, num_chunks, pool;
  int group_min, group_max, max_groups;
};

constexpr int kScanThreads = 1024;

// slot_topk of a shared expert's slot: combine weight 1, no top-k position.
constexpr int kSharedTopk = -2;

// One CTA. (1) Expert e's chunk counts are scanned by kScanThreads/E threads,
// each over a contiguous range of chunks; (2) warp 0 scans the padded block
// counts over the routed and shared experts with shuffles; (3) thread 0 forms
// the block groups while the other threads write offsets, padding and
// shared-expert records and counters.
__global__ void __launch_bounds__(kScanThreads) moe_dispatch_scan_kernel(const DispatchParams p) {
  constexpr int kPerLane = (kMaxExpertsAll + 31) / 32;
  if (p.E < 1 || p.E > kMaxExperts || p.S < 0 || p.S > kMaxShared) {   // the host validates; never trust it blindly
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kDevBounds);
    return;
  }
  __shared__ int32_t s_nb[kMaxExpertsAll + 1];
  __shared__ int32_t s_bs[kMaxExpertsAll + 1];
  __shared__ int32_t s_cnt[kMaxExperts];
  __shared__ int32_t s_part[kScanThreads];
  const int tid = threadIdx.x;
  // (1) per-expert scan over chunks: threads per expert tpe (a power of two), each a run of
  // chunks; neighbouring threads take neighbouring experts, so a warp's loads are contiguous
  int tpe = 1;
  while (tpe * 2 * p.E <= kScanThreads) tpe *= 2;
  const bool act = tid < tpe * p.E;
  const int e = act ? tid % p.E : p.E, sub = act ? tid / p.E : 0;
  const int per = (p.num_chunks + tpe - 1) / tpe;
  const int c0 = min(sub * per, p.num_chunks), c1 = min(c0 + per, p.num_chunks);
  int local = 0;
  if (e < p.E) {
    for (int c = c0; c < c1; ++c) local += p.chunk_count[(size_t)c * p.E + e];
    s_part[e * tpe + sub] = local;
  }
  __syncthreads();
  if (e < p.E) {
    int base = 0;
    for (int q = 0; q < sub; ++q) base += s_part[e * tpe + q];
    if (sub == tpe - 1) {
      const int run = base + local;
      s_cnt[e] = run;
      s_nb[e] = (run + p.BM - 1) / p.BM;
    }
    // counts -> per-chunk bases, 8 loads in flight before the 8 stores
    constexpr int U = 8;
    int c = c0;
    for (; c + U <= c1; c += U) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = p.chunk_count[(size_t)(c + u) * p.E + e];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        p.chunk_count[(size_t)(c + u) * p.E + e] = base;
        base += v[u];
      }
    }
    for (; c < c1; ++c) {
      const int v = p.chunk_count[(size_t)c * p.E + e];
      p.chunk_count[(size_t)c * p.E + e] = base;
      base += v;
    }
  }
  const int EA = p.E + p.S;   // routed + shared experts
  if (tid < p.S) s_nb[p.E + tid] = (p.T + p.BM - 1) / p.BM;   // a shared expert sees every token
  __syncthreads();
  // (2) exclusive scan of the block counts (E + S <= kMaxExpertsAll)
  if (tid < 32) {
    int v[kPerLane], sum = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int ee = tid * kPerLane + i;
      v[i] = ee < EA ? s_nb[ee] : 0;
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (tid >= off) incl += o;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int ee = tid * kPerLane + i;
      if (ee < EA) s_bs[ee] = run;
      run += v[i];
    }
    if (tid == 31) s_bs[EA] = incl;
  }
  __shared__ int32_t s_ps[kMaxExpertsAll + 1];
  if (p.pair_start != nullptr && tid < 32) {   // exclusive scan of ceil(blocks / 2) per expert
    int v[kPerLane], sum = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int ee = tid * kPerLane + i;
      v[i] = ee < EA ? (s_nb[ee] + 1) / 2 : 0;
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (tid >= off) incl += o;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int ee = tid * kPerLane + i;
      if (ee < EA) s_ps[ee] = run;
      run += v[i];
    }
    if (tid == 31) s_ps[EA] = incl;
  }
  __syncthreads();
  const int nblocks = s_bs[EA];
  if (tid == 0) {
    p.sched[0] = 0;
    p.sched[1] = nblocks;
    p.sched[2] = s_bs[p.E] * p.BM;   // routed slots (the routing result)
    if (p.group_start != nullptr) {
      // Consecutive blocks form groups of at most group_max blocks; a group is
      // closed at the first expert boundary at least group_min blocks after
      // its start, so small experts share a group and an expert's blocks
      // rarely straddle two. One binary search over the expert boundaries per
      // group (block starts are non-decreasing).
      const int32_t* units = p.pair_start != nullptr ? s_ps : s_bs;   // group over pairs or blocks
      const int total = units[EA];
      int ng = 0, start = 0;
      p.group_start[0] = 0;
      while (start < total && ng < p.max_groups) {
        const int target = start + p.group_min;
        int lo = 0, hi = EA;   // first e with units[e] >= target (EA if none)
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (units[mid] >= target) hi = mid;
          else lo = mid + 1;
        }
        const int boundary = units[lo] >= target ? units[lo] : total;
        start = min(min(boundary, start + p.group_max), total);
        p.group_start[++ng] = start;
      }
      if (start != total) atomicCAS(p.err, 0, kDevBounds);   // more groups than max_groups
      p.sched[3] = ng;
    }
    return;
  }
  // (3) everything else, on threads 1..
  for (int ee = tid - 1; ee <= EA; ee += kScanThreads - 1) {
    p.block_start[ee] = s_bs[ee];
    if (p.pair_start != nullptr) p.pair_start[ee] = s_ps[ee];
    if (ee <= p.E) p.expert_offset[ee] = s_bs[ee] * p.BM;
    if (ee < p.E) p.expert_count[ee] = s_cnt[ee];
  }
  // shared experts: slot (first slot of expert E+s) + t holds token t
  for (int i = tid - 1; i < p.S * s_nb[p.E] * p.BM; i += kScanThreads - 1) {
    const int per = s_nb[p.E] * p.BM;
    const int t = i % per;
    const int sl = s_bs[p.E] * p.BM + i;
    if (sl < p.pool) {
      p.slot_token[sl] = t < p.T ? t : -1;
      p.slot_topk[sl] = t < p.T ? kSharedTopk : -1;
    }
  }
  // padding slots of each expert's last block
  for (int ee = tid - 1; ee < p.E; ee += kScanThreads - 1) {
    const int beg = s_bs[ee] * p.BM + s_cnt[ee];
    const int end = (s_bs[ee] + s_nb[ee]) * p.BM;
    for (int sl = beg; sl < end && sl < p.pool; ++sl) {
      p.slot_token[sl] = -1;
      p.slot_topk[sl] = -1;
    }
  }
  for (int b = tid - 1; b < nblocks; b += kScanThreads - 1) p.l1_done[b] = 0;
  if (p.l2_done != nullptr)
    for (int b = tid - 1; b < nblocks; b += kScanThreads - 1) p.l2_done[b] = 0;
}

// One thread per routed pair (t, j): slot = offset[e] + chunk base + in-chunk rank.
__global__ void __launch_bounds__(256) moe_dispatch_scatter_kernel(const DispatchParams p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.T * p.k) return;
  const int t = i / p.k, j = i - t * p.k;
  const int e = p.topk_idx[i];
  if (e == kAbortedExpert) {   // the router gave up on this token (and recorded the timeout)
    atomicCAS(p.err, 0, kDevTimeout);
    return;
  }
  if (e < 0 || e >= p.E) {
    atomicCAS(p.err, 0, kDevBounds);
    return;
  }
  const int c = t / kRouterTokens;
  const int s = p.expert_offset[e] + p.chunk_count[(size_t)c * p.E + e] + p.rank[i];
  if (s < 0 || s >= p.pool) {
    atomicCAS(p.err, 0, kDevBounds);
    return;
  }
  p.slot_token[s] = t;
  p.slot_topk[s] = j;
}

// y = bf16(y_acc), round to nearest even; 4 elements per thread.
__global__ void __launch_bounds__(256) moe_finalize_kernel(const float* __restrict__ y_acc, bf16* __restrict__ y,
                                                           size_t n4) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(y_acc)[i];
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&a);
    o.y = *reinterpret_cast<const uint32_t*>(&b);
    reinterpret_cast<uint2*>(y)[i] = o;
  }
}

}  // namespace moe
