// Dispatch: exclusive scans of the router's per-chunk histograms, padding of
// every expert to a multiple of BLOCK_M, and the stable token -> slot
// permutation with its (token, top-k position) record per slot.
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
  int32_t* expert_offset;    // [E+1] slot offsets (multiples of BLOCK_M)
  int32_t* block_start;      // [E+1] the same in blocks
  int32_t* slot_token;       // [pool]
  int32_t* slot_topk;        // [pool]
  int32_t* l1_done;          // [pool / BLOCK_M] zeroed here
  int32_t* sched;            // [0] task counter, [1] blocks, [2] padded slots, [3] block groups
  int32_t* err;              // sticky device error word
  // Block groups of the expert GEMM's task order (nullptr: routing only, no groups).
  int32_t* group_start;      // [max_groups + 1] first block of each group
  int32_t* l2_done;          // [pool / BLOCK_M] zeroed here
  int T, E, k, BM, num_chunks, pool;
  int group_min, group_max, max_groups;
};

constexpr int kScanThreads = 1024;

// One CTA. Thread e scans expert e's chunk counts; thread 0 scans the padded
// block counts over experts (E <= 256 values).
__global__ void __launch_bounds__(kScanThreads) moe_dispatch_scan_kernel(const DispatchParams p) {
  __shared__ int32_t s_nb[257];
  __shared__ int32_t s_bs[257];
  __shared__ int32_t s_cnt[256];
  for (int e = threadIdx.x; e < p.E; e += kScanThreads) {
    int run = 0;
    int c = 0;
    constexpr int U = 8;
    for (; c + U <= p.num_chunks; c += U) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = p.chunk_count[(size_t)(c + u) * p.E + e];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        p.chunk_count[(size_t)(c + u) * p.E + e] = run;
        run += v[u];
      }
    }
    for (; c < p.num_chunks; ++c) {
      const int v = p.chunk_count[(size_t)c * p.E + e];
      p.chunk_count[(size_t)c * p.E + e] = run;
      run += v;
    }
    s_cnt[e] = run;
    s_nb[e] = (run + p.BM - 1) / p.BM;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      s_bs[e] = acc;
      acc += s_nb[e];
    }
    s_bs[p.E] = acc;
    p.sched[0] = 0;
    p.sched[1] = acc;
    p.sched[2] = acc * p.BM;
    if (p.group_start != nullptr) {
      // Consecutive blocks form groups of at most group_max blocks; a group is
      // closed at an expert boundary once it holds group_min blocks, so that
      // small experts share a group and an expert's blocks rarely straddle two.
      int ng = 0, cur = 0, start = 0;
      p.group_start[0] = 0;
      for (int e = 0; e < p.E; ++e) {
        int nb = s_nb[e];
        while (nb > 0) {
          const int take = min(nb, p.group_max - cur);
          cur += take;
          nb -= take;
          if (cur == p.group_max) {
            start += cur;
            cur = 0;
            if (ng < p.max_groups) p.group_start[++ng] = start;
          }
        }
        if (cur >= p.group_min) {
          start += cur;
          cur = 0;
          if (ng < p.max_groups) p.group_start[++ng] = start;
        }
      }
      if (cur > 0) {
        start += cur;
        if (ng < p.max_groups) p.group_start[++ng] = start;
      }
      if (start != acc) atomicCAS(p.err, 0, kDevBounds);   // more groups than max_groups
      p.sched[3] = ng;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= p.E; e += kScanThreads) {
    p.block_start[e] = s_bs[e];
    p.expert_offset[e] = s_bs[e] * p.BM;
    if (e < p.E) p.expert_count[e] = s_cnt[e];
  }
  // padding slots of each expert's last block
  for (int e = threadIdx.x; e < p.E; e += kScanThreads) {
    const int beg = s_bs[e] * p.BM + s_cnt[e];
    const int end = (s_bs[e] + s_nb[e]) * p.BM;
    for (int s = beg; s < end && s < p.pool; ++s) {
      p.slot_token[s] = -1;
      p.slot_topk[s] = -1;
    }
  }
  const int nblocks = s_bs[p.E];
  for (int b = threadIdx.x; b < nblocks; b += kScanThreads) p.l1_done[b] = 0;
  if (p.l2_done != nullptr)
    for (int b = threadIdx.x; b < nblocks; b += kScanThreads) p.l2_done[b] = 0;
}

// One thread per routed pair (t, j): slot = offset[e] + chunk base + in-chunk rank.
__global__ void __launch_bounds__(256) moe_dispatch_scatter_kernel(const DispatchParams p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.T * p.k) return;
  const int t = i / p.k, j = i - t * p.k;
  const int e = p.topk_idx[i];
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
