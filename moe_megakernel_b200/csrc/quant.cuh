// FP8 E4M3 operands of the expert GEMMs: per-token quantization of x, the
// one-time per-(expert, column) quantization of W1 / W3 / W2 into the K-major
// layout the tcgen05 kind::f8f6f4 MMA reads, and the bf16 -> E4M3 conversion
// the expert GEMM applies to the activation rows it loads.
//
// "MegaMoE 在 MoE 系统谱系中的位置", section 一 (the Mega MoE GEMMs take 8-bit
// operands with scale factors loaded beside them) and section 2.1 (amax and
// quantization in the epilogue). Scales here are powers of two, the smallest
// p with amax / p <= 448, so that dividing by them is exact and the only
// rounding is the E4M3 conversion (round to nearest even, saturating).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {

constexpr float kE4m3Max = 448.f;

// Exponent k of the scale 2**k for a row with largest magnitude amax: the
// smallest k with amax <= 448 * 2**k. Decided on amax itself, with no rounded
// quotient: amax = m * 2**e exactly (m in [0.5, 1)) and 448 = 0.875 * 2**9,
// so amax <= 0.875 * 2**(k+9) holds from k = e - 9 when m <= 0.875 and from
// k = e - 8 otherwise.
__device__ __forceinline__ int pow2_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int e;
  const float m = frexpf(amax, &e);
  return m <= 0.875f ? e - 9 : e - 8;
}

// Eight bf16 values (one uint4) times `inv` (an exact power of two) -> eight E4M3 codes, in order.
__device__ __forceinline__ uint2 bf16x8_to_e4m3(const uint4 v, float inv) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
  uint32_t w[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float2 f0 = __bfloat1622float2(b[2 * j]);
    const float2 f1 = __bfloat1622float2(b[2 * j + 1]);
    w[j] = (uint32_t)ptx::cvt_e4m3x2(f0.x * inv, f0.y * inv) | ((uint32_t)ptx::cvt_e4m3x2(f1.x * inv, f1.y * inv) << 16);
  }
  return make_uint2(w[0], w[1]);
}

// One warp per token: amax over the row, then codes xq = e4m3(x * 2**-k) and sx = 2**k.
__global__ void __launch_bounds__(256) moe_quantize_x_kernel(const bf16* __restrict__ x, uint8_t* __restrict__ xq,
                                                             float* __restrict__ sx, int T, int H) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)warp * H);   // 8 bf16 per uint4
  const int n8 = H / 8;
  float amax = 0.f;
  for (int i = lane; i < n8; i += 32) {
    const uint4 v = __ldg(row + i);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(b[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const int k = pow2_scale_exp(amax);
  const float inv = ldexpf(1.f, -k);
  if (lane == 0) sx[warp] = ldexpf(1.f, k);
  uint2* out = reinterpret_cast<uint2*>(xq + (size_t)warp * H);   // 8 codes per uint2
  for (int i = lane; i < n8; i += 32) out[i] = bf16x8_to_e4m3(__ldg(row + i), inv);
}

// Second-GEMM operand of the FP8 layer: every h row (bf16, I columns) to E4M3
// codes with the row's power-of-two scale, from the row amax the first GEMM's
// epilogues gathered. Rows: *units * unit_rows (blocks or block pairs of the
// dispatch); one warp per row, grid-stride. act_scale[row] = the scale 2**k.
__global__ void __launch_bounds__(256) moe_quantize_act_kernel(const bf16* __restrict__ h,
                                                               const float* __restrict__ act_amax,
                                                               uint8_t* __restrict__ h8, float* __restrict__ act_scale,
                                                               const int32_t* __restrict__ group_start,
                                                               const int32_t* __restrict__ num_groups, int group,
                                                               int ring_units, int unit_rows, int I) {
  // the rows of block group `group`: its units (blocks, or block pairs) u map to buffer slot u % ring_units
  if (group >= *num_groups) return;
  const int u0 = group_start[group], u1 = group_start[group + 1];
  if (u1 - u0 > ring_units) return;   // never: the host sizes the groups to the buffer
  const int nrows = (u1 - u0) * unit_rows;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < nrows; i += warps) {
    const int row = ((u0 + i / unit_rows) % ring_units) * unit_rows + i % unit_rows;
    const int k = pow2_scale_exp(__ldcg(act_amax + row));
    const float inv = ldexpf(1.f, -k);
    if (lane == 0) act_scale[row] = ldexpf(1.f, k);
    const uint4* in = reinterpret_cast<const uint4*>(h + (size_t)row * I);
    uint2* out = reinterpret_cast<uint2*>(h8 + (size_t)row * I);
    for (int i = lane; i < I / 8; i += 32) out[i] = bf16x8_to_e4m3(__ldcg(in + i), inv);
  }
}

// Column scales of W [E, H, I]: block (blockIdx.x = 32 columns, blockIdx.y = expert), 256 threads.
__global__ void __launch_bounds__(256) moe_weight_scales_kernel(const bf16* __restrict__ W, float* __restrict__ s,
                                                                int H, int I) {
  __shared__ float part[8][32];
  const int e = blockIdx.y, i = blockIdx.x * 32 + (threadIdx.x & 31), r0 = threadIdx.x >> 5;
  float amax = 0.f;
  if (i < I)
    for (int h = r0; h < H; h += 8) amax = fmaxf(amax, fabsf(__bfloat162float(W[((size_t)e * H + h) * I + i])));
  part[r0][threadIdx.x & 31] = amax;
  __syncthreads();
  if (threadIdx.x < 32 && i < I) {
    float m = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) m = fmaxf(m, part[r][threadIdx.x]);
    s[(size_t)e * I + i] = ldexpf(1.f, pow2_scale_exp(m));
  }
}

// Quantize and transpose W [E, H, I] -> Wq [E, I, H] with the column scales:
// one 64 (h) x 64 (i) tile per block of 256 threads.
__global__ void __launch_bounds__(256) moe_weight_quant_kernel(const bf16* __restrict__ W, const float* __restrict__ s,
                                                               uint8_t* __restrict__ Wq, int H, int I) {
  __shared__ float tile[64][65];
  const int e = blockIdx.z, h0 = blockIdx.y * 64, i0 = blockIdx.x * 64;
  for (int t = threadIdx.x; t < 64 * 64; t += 256) {
    const int r = t / 64, c = t % 64;   // r: h, c: i (coalesced along i)
    tile[r][c] = __bfloat162float(W[((size_t)e * H + h0 + r) * I + i0 + c]);
  }
  __syncthreads();
  const int i = threadIdx.x / 4, part = threadIdx.x % 4;   // output row i, 16 codes of h each
  const float inv = 1.f / s[(size_t)e * I + i0 + i];        // an exact power of two
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int h = part * 16 + q * 4;
    w[q] = (uint32_t)ptx::cvt_e4m3x2(tile[h][i] * inv, tile[h + 1][i] * inv) |
           ((uint32_t)ptx::cvt_e4m3x2(tile[h + 2][i] * inv, tile[h + 3][i] * inv) << 16);
  }
  *reinterpret_cast<uint4*>(Wq + ((size_t)e * I + i0 + i) * H + h0 + part * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace moe
