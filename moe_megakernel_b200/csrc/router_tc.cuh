// Router on the 5th-generation tensor cores, for many tokens and E a multiple
// of 64 (E <= 256): logits = x Wg (+ b) for 128 tokens per CTA with tcgen05
// MMAs (TMA-fed, fp32 accumulator in TMEM), then top-k and the softmax over
// the k kept logits, then the same per-64-token histogram and stable ranks as
// the warp-MMA router; the epilogue warps zero the tokens' output-accumulator
// rows while the MMAs run.
//
// Gate definition: "FlashMoE Kernel", opening paragraph (gate is the first step
// of the fused layer); softmax top-k renormalised over the k selected experts;
// within a token the experts are written in ascending id, ties in the
// selection go to the lower id. The TMEM accumulator puts one token's logits
// in one thread (lane = token row), so the top-k here is per thread: each of
// the 128 epilogue threads keeps a sorted list of its token's k best logits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"
#include "router.cuh"

namespace moe {

constexpr int kRtcTokens = 128;                  // tokens per CTA (one MMA M)
constexpr int kRtcStages = 4;
constexpr int kRtcThreads = 192;                 // producer, MMA, 4 epilogue warps
constexpr int kRtcABytes = kRtcTokens * kBK * 2; // 16 KB
constexpr int kRtcBMaxBytes = 4 * kBoxBytes;     // E <= 256: up to four 64-column boxes
constexpr int kRtcStageBytes = kRtcABytes + kRtcBMaxBytes;

struct RouterTcParams {
  CUtensorMap tm_x;    // x [T, H], box {64, 128}
  CUtensorMap tm_wg;   // Wg [H, E], box {64, 64}
  const float* bias;   // [E] or nullptr
  int32_t* topk_idx;   // [T, k]
  float* topk_w;       // [T, k]
  int32_t* rank;       // [T, k]
  int32_t* chunk_count;   // [ceil(T/64), E]
  float* y_acc;        // [T, H]
  int32_t* err;
  int T, H, E, k;
  unsigned long long timeout_ns;
};

struct RouterTcSmem {
  uint64_t full[kRtcStages];
  uint64_t empty[kRtcStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort;
  int sel[kRtcTokens][8];   // selected experts per token, ascending id
  float bias[256];          // the gate bias (when given)
  unsigned long long mask[2 * 256];   // per 64-token chunk and expert: token bitmask
};

constexpr size_t kRtcSmemBytes = 1024 + (size_t)kRtcStages * kRtcStageBytes + sizeof(RouterTcSmem);

__device__ __forceinline__ bool rtc_wait(uint64_t* bar, uint32_t parity, const RouterTcParams& p,
                                         RouterTcSmem& s, int where) {
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
        if (atomicCAS(p.err, 0, kDevTimeout) == 0) p.err[1] = 0x50000 | where;
        *reinterpret_cast<volatile int*>(&s.abort) = 1;
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kRtcThreads, 1) moe_router_tc_kernel(const __grid_constant__ RouterTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RouterTcSmem& s = *reinterpret_cast<RouterTcSmem*>(tiles + (size_t)kRtcStages * kRtcStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRtcTokens;
  const int ntok = min(kRtcTokens, p.T - t0);
  const int nk = p.H / kBK;
  const int nbox = p.E / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRtcStages; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], 1);
    }
    ptx::mbar_init(&s.acc_full, 1);
    s.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&s.tmem_base, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    const uint64_t pol = ptx::policy_evict_last();   // Wg is read by every CTA
    uint32_t issued = 0, issued_parity = 0;
    int stage = 0;
    uint32_t phase = 0;
    // CTAs start at different K offsets so that they do not all read the same
    // Wg tile at the same moment (the sum over K is order-independent up to
    // fp32 rounding).
    const int kstart = blockIdx.x % nk;
    for (int i = 0; i < nk; ++i) {
      const int kb = (kstart + i) % nk;
      if (!rtc_wait(&s.empty[stage], phase ^ 1, p, s, 1)) break;
      if (lane == 0) {
        const uint32_t a = ptx::smem_u32(tiles + stage * kRtcStageBytes);
        ptx::mbar_arrive_expect_tx(&s.full[stage], kRtcABytes + nbox * kBoxBytes);
        ptx::tma_load_2d(a, &p.tm_x, &s.full[stage], kb * kBK, t0, ptx::policy_evict_first());
        for (int j = 0; j < nbox; ++j)
          ptx::tma_load_2d(a + kRtcABytes + j * kBoxBytes, &p.tm_wg, &s.full[stage], j * 64, kb * kBK, pol);
      }
      __syncwarp();
      issued |= 1u << stage;
      issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
      if (++stage == kRtcStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    for (int st = 0; st < kRtcStages; ++st)   // let every issued copy land
      if (issued & (1u << st)) {
        const uint64_t tw = ptx::globaltimer();
        while (!ptx::mbar_try_wait(&s.full[st], (issued_parity >> st) & 1u))
          if (ptx::globaltimer() - tw > p.timeout_ns) break;
      }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    const uint32_t idesc = ptx::idesc_bf16_f32(128, p.E, false, true);
    int stage = 0;
    uint32_t phase = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (!rtc_wait(&s.full[stage], phase, p, s, 2)) break;
      ptx::tc_fence_after();
      if (lane == 0) {
        const uint32_t a = ptx::smem_u32(tiles + stage * kRtcStageBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(a + kk * 32, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(a + kRtcABytes + kk * 2048, kBoxBytes, 1024);
          ptx::mma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        ptx::mma_commit(&s.empty[stage]);
      }
      __syncwarp();
      if (++stage == kRtcStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (lane == 0) ptx::mma_commit(&s.acc_full);   // also orders every MMA before TMEM is read or freed
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: one token per thread
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    if (p.bias != nullptr)
      for (int e = r; e < p.E; e += 128) s.bias[e] = p.bias[e];
    asm volatile("bar.sync 1, 128;" ::: "memory");   // the four epilogue warps: bias staged
    {
      // while the MMAs run: zero these tokens' rows of the fp32 output accumulator
      float4* dst = reinterpret_cast<float4*>(p.y_acc + (size_t)t0 * p.H);
      const size_t n4 = (size_t)ntok * p.H / 4;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      for (size_t i = r; i < n4; i += 128) dst[i] = z;
    }
    // the MMA warp commits acc_full even after giving up on a stage, so the
    // accumulator is complete only if no role of this CTA aborted
    bool ok = rtc_wait(&s.acc_full, 0, p, s, 3);
    ok = ok && !*reinterpret_cast<volatile int*>(&s.abort);
    ptx::tc_fence_after();
    // best[0..k-1]: the k largest logits so far, descending; equal values keep
    // arrival order, and candidates arrive in ascending expert id, so a tie
    // goes to the lower id.
    float best[8];
    int bidx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      best[j] = -INFINITY;
      bidx[j] = 0x7fffffff;
    }
    float kth = -INFINITY;   // best[k-1]
    const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float* bias = p.bias != nullptr ? s.bias : nullptr;
    for (int c = 0; c < p.E / 32; ++c) {
      uint32_t v[32];
      ptx::tmem_ld32(tbase + c * 32, v);
      ptx::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int e = c * 32 + i;
        const float l = __uint_as_float(v[i]) + (bias != nullptr ? bias[e] : 0.f);
        if (l > kth) {
          // insert by one pass of compare-and-exchange down the list: the new
          // value moves past only strictly smaller ones (a tie keeps the earlier,
          // lower id), and the list stays in registers
          float x = l;
          int xi = e;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < p.k) {
              const bool sw = x > best[j];
              const float tb = best[j];
              const int ti = bidx[j];
              best[j] = sw ? x : tb;
              bidx[j] = sw ? xi : ti;
              x = sw ? tb : x;
              xi = sw ? ti : xi;
            }
          }
          // the k-th largest is the smallest of the k kept (a select by the runtime index k - 1
          // would become an indexed load and put the list in local memory)
          kth = best[0];
#pragma unroll
          for (int j = 1; j < 8; ++j)
            if (j < p.k) kth = fminf(kth, best[j]);
        }
      }
    }
    if (!ok && r < ntok) {
      // aborted (a bounded wait ran out): no selection. The token's rows get the
      // sentinel expert id -1 (weight 0), which the dispatch scatter skips as a
      // timeout instead of reading whatever the workspace held before.
      const size_t o = (size_t)(t0 + r) * p.k;
      for (int j = 0; j < p.k; ++j) {
        p.topk_idx[o + j] = kAbortedExpert;
        p.topk_w[o + j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) s.sel[r][j] = -1;
      if (r == 0) atomicCAS(p.err, 0, kDevTimeout);
    }
    if (ok && r < ntok) {
      // softmax over the k kept logits (best[0] is their maximum)
      float denom = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < p.k) denom += expf(best[j] - best[0]);
      const size_t o = (size_t)(t0 + r) * p.k;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < p.k) {
          int pos = 0;   // position in ascending expert order
#pragma unroll
          for (int i = 0; i < 8; ++i) pos += (i < p.k && bidx[i] < bidx[j]) ? 1 : 0;
          p.topk_idx[o + pos] = bidx[j];
          p.topk_w[o + pos] = expf(best[j] - best[0]) / denom;
          s.sel[r][pos] = bidx[j];
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) ptx::tmem_dealloc(tmem, 256);

  // Per 64-token chunk: histogram and stable ranks (tokens ascending).
  chunk_histogram(&s.sel[0][0], s.mask, ntok, 2, blockIdx.x * 2, t0, p.E, p.k, p.rank, p.chunk_count,
                  kRtcThreads);
}

}  // namespace moe
