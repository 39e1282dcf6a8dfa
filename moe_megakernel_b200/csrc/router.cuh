// Router: gate GEMM logits = x Wg (+ b), warp-level top-k, softmax over the
// k selected logits, plus the per-chunk expert histogram and stable in-chunk
// ranks that the dispatch scan consumes.
//
// Gate definition: "FlashMoE Kernel", opening paragraph (gate is the first step
// of the fused layer); softmax top-k with weights renormalised over the k
// selected experts. Within a token the k experts are written in ascending
// expert id; ties in the selection go to the lower id.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

struct RouterParams {
  const bf16* x;        // [T, H]
  const bf16* Wg;       // [H, E]
  const float* bias;    // [E] or nullptr
  int32_t* topk_idx;    // [T, k]
  float* topk_w;        // [T, k]
  int32_t* rank;        // [T, k]  rank of (t, j) among this chunk's tokens routed to the same expert
  int32_t* chunk_count; // [num_chunks, E]
  float* y_acc;         // [T, H] zeroed here, accumulated by the expert GEMM
  // Split of H over gridDim.y CTAs (fewer token tiles than SMs): every split
  // adds its partial logits into the tile's accumulator [tiles][64][EP] fp32
  // and arrives on the tile's counter; the last CTA to arrive reads the sums,
  // and leaves accumulator and counter at zero for the next call.
  float* partial;
  int32_t* tile_counter;
  int T, H, E, k;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;   // zero-fill when out of range
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(s));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Per-chunk histogram and stable ranks for up to `nchunks` chunks of 64
// tokens whose selected experts are in sel[t * 8 + j] (t local to the CTA):
// every (t, j) sets bit t%64 of its expert's token mask; the count of an
// expert is the mask's popcount and the rank of (t, j) the popcount of the
// mask below bit t, i.e. the number of earlier tokens of the chunk routed to
// the same expert. `mask` holds nchunks * E 64-bit words of shared memory.
__device__ __forceinline__ void chunk_histogram(const int32_t* sel, unsigned long long* mask, int ntok,
                                                int nchunks, int chunk0, int t0, int E, int k, int32_t* rank,
                                                int32_t* chunk_count, int nthreads) {
  for (int i = threadIdx.x; i < nchunks * E; i += nthreads) mask[i] = 0ull;
  __syncthreads();
  // (an expert id outside [0, E) -- only possible after an aborted top-k --
  // is left out here; the dispatch scatter reports it as a bounds error)
  for (int i = threadIdx.x; i < ntok * k; i += nthreads) {
    const int t = i / k, j = i - t * k;
    const int e = sel[t * 8 + j];
    if (e >= 0 && e < E) atomicOr(&mask[(t >> 6) * E + e], 1ull << (t & 63));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ntok * k; i += nthreads) {
    const int t = i / k, j = i - t * k;
    const int e = sel[t * 8 + j];
    const unsigned long long m = (e >= 0 && e < E) ? mask[(t >> 6) * E + e] : 0ull;
    rank[(size_t)(t0 + t) * k + j] = __popcll(m & ((1ull << (t & 63)) - 1ull));
  }
  const int chunks_used = (ntok + 63) >> 6;
  for (int i = threadIdx.x; i < chunks_used * E; i += nthreads)
    chunk_count[(size_t)(chunk0 + i / E) * E + (i % E)] = __popcll(mask[i]);
}

// Shared memory of one router CTA, for EP padded experts.
template <int EP>
struct RouterSmem {
  static constexpr int kXStride = kRouterKChunk + 8;  // bf16 per x row (padding: no ldmatrix bank conflicts)
  static constexpr int kWStride = EP + 8;             // bf16 per Wg row
  static constexpr int kXBytes = kRouterTokens * kXStride * 2;
  static constexpr int kWBytes = kRouterKChunk * kWStride * 2;
  static constexpr int kStageBytes = kXBytes + kWBytes;
  static constexpr int kLogitStride = EP + 1;         // fp32 per logit row
  static constexpr int kTileBytes = 2 * kStageBytes;  // double-buffered; logits alias this after the K loop
  static constexpr int kSelBytes = kRouterTokens * 8 * 4;
  static constexpr int kMaskBytes = 256 * 8;           // one 64-token chunk, E <= 256
  static constexpr int kBytes = kTileBytes + kSelBytes + kMaskBytes;
  static_assert(kRouterTokens * kLogitStride * 4 <= kTileBytes, "logits must fit in the tile buffers");
};

// kZeroAcc: also zero this chunk's rows of the fp32 output accumulator (the
// full forward); routing-only callers without an accumulator pass false.
template <int EP, bool kZeroAcc = true>
__global__ void __launch_bounds__(kRouterThreads) moe_router_kernel(const RouterParams p) {
  using S = RouterSmem<EP>;
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NT = EP / 8;   // n-tiles of 8 experts
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRouterTokens;
  const int ntok = min(kRouterTokens, p.T - t0);

  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  auto load_chunk = [&](int stage, int kc) {
    bf16* xs = reinterpret_cast<bf16*>(smem + stage * S::kStageBytes);
    bf16* ws = reinterpret_cast<bf16*>(smem + stage * S::kStageBytes + S::kXBytes);
    const int h0 = kc * kRouterKChunk;
    // x: 64 rows x 8 chunks of 16 B
    for (int i = threadIdx.x; i < kRouterTokens * 8; i += kRouterThreads) {
      const int r = i >> 3, c = i & 7;
      const bool ok = r < ntok;
      const bf16* src = p.x + (size_t)(ok ? t0 + r : 0) * p.H + h0 + c * 8;
      cp_async16(xs + r * S::kXStride + c * 8, src, ok);
    }
    // Wg: 64 rows x EP/8 chunks of 16 B (columns >= E zero-filled)
    constexpr int CPR = EP / 8;
    for (int i = threadIdx.x; i < kRouterKChunk * CPR; i += kRouterThreads) {
      const int r = i / CPR, c = i % CPR;
      const bool ok = c * 8 < p.E;
      const bf16* src = p.Wg + (size_t)(h0 + r) * p.E + (ok ? c * 8 : 0);
      cp_async16(ws + r * S::kWStride + c * 8, src, ok);
    }
    cp_async_commit();
  };

  // this CTA's share of H: chunks [kc0, kc0 + nk)
  const int nk = p.H / kRouterKChunk / gridDim.y;
  const int kc0 = blockIdx.y * nk;
  load_chunk(0, kc0);
  for (int kc = 0; kc < nk; ++kc) {
    const int stage = kc & 1;
    if (kc + 1 < nk) {
      load_chunk(stage ^ 1, kc0 + kc + 1);
      cp_async_wait_1();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    const bf16* xs = reinterpret_cast<const bf16*>(smem + stage * S::kStageBytes);
    const bf16* ws = reinterpret_cast<const bf16*>(smem + stage * S::kStageBytes + S::kXBytes);
#pragma unroll
    for (int ks = 0; ks < kRouterKChunk / 16; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(a, xs + (warp * 16 + (lane & 15)) * S::kXStride + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b[4];
        const int q = lane >> 3, i = lane & 7;
        ldmatrix_x4_trans(b, ws + (ks * 16 + (q & 1) * 8 + i) * S::kWStride + np * 16 + (q >> 1) * 8);
        mma_16816(acc[2 * np], a, b[0], b[1]);
        mma_16816(acc[2 * np + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();
  }

  // Logits (+ bias) to shared memory; padded experts get -inf.
  float* logits = reinterpret_cast<float*>(smem);
  if (gridDim.y > 1) {
    // Split H: add this split's partial logits into the tile's accumulator
    // (fp32 vector reductions at L2; the summation order over splits varies
    // run to run, at fp32 rounding level); the last CTA of the tile to arrive
    // takes the sums.
    __shared__ int s_last;
    const int tile = blockIdx.x, nsplit = gridDim.y;
    float* tacc = p.partial + (size_t)tile * kRouterTokens * EP;
    const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int col = nt * 8 + 2 * (lane & 3);
      if (r0 < ntok) ptx::red_add_v2_f32(tacc + r0 * EP + col, acc[nt][0], acc[nt][1]);
      if (r0 + 8 < ntok) ptx::red_add_v2_f32(tacc + (r0 + 8) * EP + col, acc[nt][2], acc[nt][3]);
    }
    if constexpr (kZeroAcc) {
      // every split zeroes its share of the tile's output-accumulator rows
      const size_t n4 = (size_t)ntok * p.H / 4;
      const size_t per = (n4 + nsplit - 1) / nsplit;
      const size_t b0 = blockIdx.y * per, b1 = min(n4, b0 + per);
      float4* dst = reinterpret_cast<float4*>(p.y_acc + (size_t)t0 * p.H);
      for (size_t i = b0 + threadIdx.x; i < b1; i += kRouterThreads) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(p.tile_counter + tile, 1) == nsplit - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // read the sums (L2) and leave the accumulator at zero for the next call
    float4* all = reinterpret_cast<float4*>(tacc);
#pragma unroll 4
    for (int i = threadIdx.x; i < ntok * EP / 4; i += kRouterThreads) {
      const float4 v = __ldcg(all + i);
      __stcg(all + i, make_float4(0.f, 0.f, 0.f, 0.f));
      const int row = (4 * i) / EP, col = (4 * i) % EP;
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cj = col + j;
        const float b = (cj < p.E && p.bias != nullptr) ? p.bias[cj] : 0.f;
        logits[row * S::kLogitStride + cj] = cj < p.E ? vv[j] + b : -INFINITY;
      }
    }
    if (threadIdx.x == 0) p.tile_counter[tile] = 0;   // ready for the next call
    __syncthreads();
  } else {
    const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = nt * 8 + 2 * (lane & 3) + h;
        const float b = (col < p.E && p.bias != nullptr) ? p.bias[col] : 0.f;
        const float v0 = col < p.E ? acc[nt][h] + b : -INFINITY;
        const float v1 = col < p.E ? acc[nt][2 + h] + b : -INFINITY;
        logits[r0 * S::kLogitStride + col] = v0;
        logits[(r0 + 8) * S::kLogitStride + col] = v1;
      }
    }
  }
  __syncwarp();

  // Warp-level top-k over the logits in shared memory; rows are dealt to the
  // 4 warps round-robin so that a partly filled tile still uses all of them.
  __syncthreads();
  int32_t* sel = reinterpret_cast<int32_t*>(smem + S::kTileBytes);   // [64][8] ascending expert ids
  constexpr int VPL = (EP + 31) / 32;
  for (int rr = 0; rr < 16; ++rr) {
    const int row = rr * 4 + warp;
    if (row >= ntok) break;   // warp-uniform
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < EP ? logits[row * S::kLogitStride + e] : -INFINITY;
    }
    int chosen[8];
    float chosen_l[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      chosen[r] = 0x7fffffff;
      chosen_l[r] = -INFINITY;
      if (r < p.k) {
        float best = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int e = lane + 32 * i;
          if (e < p.E && (v[i] > best || (v[i] == best && e < bi))) {
            best = v[i];
            bi = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ob > best || (ob == best && oi < bi)) {
            best = ob;
            bi = oi;
          }
        }
        chosen[r] = bi;
        chosen_l[r] = best;
        // the chosen logit leaves the race (selects, not a store at the runtime index bi >> 5,
        // which would put v in local memory)
        const bool mine = (bi & 31) == lane;
#pragma unroll
        for (int i = 0; i < VPL; ++i) v[i] = (mine && i == (bi >> 5)) ? -INFINITY : v[i];
      }
    }
    // Softmax over the k selected; chosen_l[0] is their maximum.
    float denom = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (r < p.k) denom += expf(chosen_l[r] - chosen_l[0]);
    int me = 0x7fffffff;
    float ml = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      me = r == lane ? chosen[r] : me;
      ml = r == lane ? chosen_l[r] : ml;
    }
    if (lane < p.k) {
      int pos = 0;   // position in ascending expert order
#pragma unroll
      for (int r = 0; r < 8; ++r) pos += (r < p.k && chosen[r] < me) ? 1 : 0;
      const size_t o = (size_t)(t0 + row) * p.k + pos;
      p.topk_idx[o] = me;
      p.topk_w[o] = expf(ml - chosen_l[0]) / denom;
      sel[row * 8 + pos] = me;
    }
  }
  __syncthreads();

  // Per-chunk histogram and stable ranks (tokens in ascending order).
  chunk_histogram(sel, reinterpret_cast<unsigned long long*>(smem + S::kTileBytes + S::kSelBytes), ntok, 1,
                  blockIdx.x, t0, p.E, p.k, p.rank, p.chunk_count, kRouterThreads);

  // Zero this chunk's rows of the fp32 output accumulator (the splits did it already).
  if (kZeroAcc && gridDim.y == 1) {
    float4* dst = reinterpret_cast<float4*>(p.y_acc + (size_t)t0 * p.H);
    const size_t n4 = (size_t)ntok * p.H / 4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t i = threadIdx.x; i < n4; i += kRouterThreads) dst[i] = z;
  }
}

}  // namespace moe
