/*
 * moe_b200.h - C ABI of the single-GPU MoE-layer forward for B200 (sm_100a).
 *
 * The library computes one dropless top-k mixture-of-experts layer forward on
 * one GPU:
 *
 *   gate      l = x Wg (+ b); keep the k largest logits per token; weights are
 *             the softmax over the k kept logits.
 *   dispatch  per-expert histogram, exclusive scan of the counts padded to
 *             BLOCK_M, stable token -> slot permutation with a (token, top-k
 *             position) record per slot.
 *   expert    h = bf16(silu(x W1[e]) * (x W3[e])) for every slot of expert e,
 *             then o = h W2[e].
 *   combine   y[t] = sum_j w[t,j] * o(t,j), scatter-added from the down
 *             projection's epilogue.
 *
 * Sources: "FlashMoE Kernel" (opening paragraph: the layer is gate -> dispatch
 * -> expert FFN -> combine; section "架构": the FFN matmuls and the combine's
 * weighting are fused tile tasks; section "通信": in-place padding to the tile);
 * "MegaMoE 在 MoE 系统谱系中的位置" (section 2.4: per-slot TokenSrcMetadata;
 * section 2.5: BLOCK_M from the expected tokens per expert; section 2.6:
 * dropless pool sized T*k + E*(BLOCK_M-1) on one rank; section 2.7: tasks
 * claimed from an atomic counter, L2 tasks wait for their block's L1 tasks;
 * section 五: the forward entry points take bf16 or fp8/fp4 tensors).
 *
 * Conventions for every entry point:
 *  - bf16 tensors are passed as `const void*` to 16-byte-aligned, contiguous,
 *    row-major device memory; fp32 and int32 likewise.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All GPU work
 *    is enqueued on it; nothing synchronises the host unless stated.
 *  - Every function returns a moe_status; no exception crosses the ABI.
 *  - Device-side failures (a bounded wait that ran out, a routing index out of
 *    range) are sticky in the workspace and are reported by moe_check().
 *  - The caller owns all device memory: inputs, weights, outputs and the
 *    workspace. A plan owns only host state (and, once a pipelined host-buffer
 *    call has run, its two copy streams and their events).
 *
 * Order of use: moe_plan_create (or _shared) -> [moe_plan_set_fp8] ->
 * moe_plan_workspace_bytes -> allocate -> moe_plan_bind_workspace ->
 * any number of moe_forward / moe_forward_shared / moe_forward_fp8 /
 * moe_forward_host* / moe_route calls -> moe_check -> moe_plan_destroy.
 * moe_route_static routes without a plan or workspace. FP8 weights come from
 * moe_quantize_weights_fp8, once per set of weights.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_plan* moe_plan_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, misaligned pointer, T out of range */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the supported set (see moe_plan_create) */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* bound workspace smaller than moe_plan_workspace_bytes() */
  MOE_ERR_NO_WORKSPACE = 4,        /* moe_forward before moe_plan_bind_workspace */
  MOE_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = 6,      /* a bounded device-side wait ran out (sticky, via moe_check) */
  MOE_ERR_DEVICE_BOUNDS = 7,       /* routing metadata held an out-of-range index (sticky) */
  MOE_ERR_UNSUPPORTED_DEVICE = 8,  /* the device is not sm_100 */
  MOE_ERR_STATIC_SCRATCH_LIMIT = 9 /* moe_route_static: sizes exceed its fixed scratch */
} moe_status;

/* Device views of the routing results inside the bound workspace. Valid after
 * a moe_forward()/moe_route() on the plan's stream has completed; overwritten
 * by the next call. Layouts:
 *   topk_idx      int32 [T, k]   selected experts of token t, ascending expert id
 *   topk_w        fp32  [T, k]   softmax weights over the k selected logits
 *   expert_count  int32 [E]      tokens routed to each expert
 *   expert_offset int32 [E+1]    first slot of each expert; multiples of block_m
 *   slot_token    int32 [pool]   token of each slot, -1 for padding
 *   slot_topk     int32 [pool]   top-k position j of each slot, -1 for padding
 *   num_padded    int32 [1]      slots in use by routed experts = expert_offset[E]
 * With shared experts (moe_plan_create_shared) the slots after the routed
 * ones hold every token once per shared expert, in token order, with
 * slot_topk = -2 (combine weight 1), padded to block_m with (-1, -1).
 * ("MegaMoE 在 MoE 系统谱系中的位置", section 2.4: the slot record; the rank
 * field of that record is dropped on one GPU.) */
typedef struct {
  int32_t* topk_idx;
  float* topk_w;
  int32_t* expert_count;
  int32_t* expert_offset;
  int32_t* slot_token;
  int32_t* slot_topk;
  int32_t* num_padded;
  int32_t block_m;
  int32_t pool_capacity;
} moe_routing;

/* One record of the expert GEMM's task log (moe_plan_set_task_log). Every
 * task of the persistent kernel (one column tile of one GEMM for one block,
 * or pair of blocks) is written by the CTA that ran it: its number in the
 * task order, its block (or pair), expert, phase (0: x W1 / x W3 + SwiGLU,
 * 1: h W2 + combine) and column tile, the SM and CTA that issued its MMAs,
 * and three %globaltimer stamps in nanoseconds: the issue of its first MMA,
 * of its last one, and the end of its epilogue. A record whose task is
 * 0xFFFFFFFF belongs to no task of the last launch. (Tracing of the task
 * queue; "MegaMoE 在 MoE 系统谱系中的位置", section 2.7, describes the queue,
 * and "FlashMoE Kernel", section 实测摘要, reports SM utilisation, which these
 * records measure.) */
typedef struct {
  uint32_t task;
  uint32_t unit;
  uint32_t expert;
  uint32_t phase_n;   /* phase << 16 | column tile */
  uint32_t smid;
  uint32_t cta;
  uint64_t t_first_mma;
  uint64_t t_last_mma;
  uint64_t t_done;
} moe_task_record;

/* Static description of a plan. */
typedef struct {
  int32_t T_max, H, I, E, k;
  int32_t block_m;         /* rows per expert block (16, 32, 64 or 128) */
  int32_t pool_capacity;   /* T_max*k + E*(block_m-1) slots rounded up to block_m, plus
                              n_shared * ceil(T_max/block_m) * block_m */
  int32_t num_sms;         /* persistent grid size */
  int32_t pair_clusters;   /* co-resident 2-CTA clusters of the CTA-pair expert GEMM */
  int32_t cta_pairs;       /* 1: the expert GEMM runs on CTA pairs (see moe_plan_set_cta_pairs) */
  int32_t n_shared;        /* shared experts (moe_plan_create_shared) */
  size_t workspace_bytes;
  int32_t task_order;      /* expert-GEMM task order in use: 0 staggered, 1 interleaved
                              (see moe_plan_set_task_order) */
  int32_t half_tails;      /* 1: bf16 forwards on CTA pairs run an expert's lone last block
                              as M = 128 pair MMAs (see moe_plan_set_half_tails) */
  int32_t wide_l1;         /* 1: bf16 forwards on CTA pairs run 256-column first-GEMM tasks
                              (see moe_plan_set_wide_l1) */
} moe_plan_desc;

/* Create a plan for up to T_max tokens of a layer with hidden size H, expert
 * intermediate size I, E experts and top-k routing, on CUDA device `device`.
 * block_m = 0 picks BLOCK_M from n = T_max*k/E: 16 if n <= 16, 32 if n <= 32,
 * 64 if n <= 64, else 128 (the candidate table of "MegaMoE 在 MoE 系统谱系中
 * 的位置", section 2.5, cut to the 128-row MMA tile); otherwise it must be one
 * of 16, 32, 64, 128.
 * Supported: T_max >= 1; H % 128 == 0; I % 128 == 0; E % 8 == 0, 8 <= E <= 256;
 * 1 <= k <= min(E, 8). Errors: MOE_ERR_INVALID_ARG (null plan pointer),
 * MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_UNSUPPORTED_DEVICE, MOE_ERR_CUDA.
 * Allocates no device memory. */
int moe_plan_create(moe_plan_t* plan, int T_max, int H, int I, int E, int k, int block_m, int device);

/* The same with n_shared (0 .. 8) shared experts ("MegaMoE 在 MoE 系统谱系中
 * 的位置", section 2.7: the shared experts' two GEMM phases are scheduled in
 * the routed experts' task queue). A shared expert is a SwiGLU FFN of the
 * same H and I applied to every token with weight 1; its output is added to
 * the routed combine: y[t] = sum_j w[t,j] FFN_{e_j}(x[t]) + sum_s FFNs_s(x[t]).
 * Routing and BLOCK_M do not depend on it. Such a plan runs with
 * moe_forward_shared / moe_forward_host_shared (moe_forward and
 * moe_forward_host return MOE_ERR_INVALID_ARG for it). Errors as for
 * moe_plan_create; n_shared outside 0..8 is MOE_ERR_UNSUPPORTED_SHAPE. */
int moe_plan_create_shared(moe_plan_t* plan, int T_max, int H, int I, int E, int k, int n_shared, int block_m,
                           int device);

/* Bytes of device workspace the plan needs (routing arrays, scheduler
 * counters, the bf16 intermediate h [pool, I], the fp32 output accumulator
 * [T_max, H] and bf16 staging for moe_forward_host). 0 for a null plan. */
size_t moe_plan_workspace_bytes(moe_plan_t plan);

/* Bind caller-allocated device memory (256-byte aligned, at least
 * moe_plan_workspace_bytes()) as the plan's workspace. The plan does not take
 * ownership. Errors: MOE_ERR_INVALID_ARG (null or misaligned),
 * MOE_ERR_WORKSPACE_TOO_SMALL. Calls sharing one workspace must not overlap in
 * time on the GPU. */
int moe_plan_bind_workspace(moe_plan_t plan, void* workspace, size_t bytes);

/* Fill `desc` with the plan's static description. */
int moe_plan_describe(moe_plan_t plan, moe_plan_desc* desc);

/* Fill `out` with device pointers to the routing results in the workspace. */
int moe_plan_get_routing(moe_plan_t plan, moe_routing* out);

/* The whole layer forward for T tokens (0 <= T <= T_max):
 *   x    bf16 [T, H]      device
 *   Wg   bf16 [H, E]      device
 *   gate_bias fp32 [E]    device, or NULL for no bias (added to the logits
 *                         before the top-k and the softmax)
 *   W1   bf16 [E, H, I]   device (gated branch, SiLU applied)
 *   W3   bf16 [E, H, I]   device (linear branch)
 *   W2   bf16 [E, I, H]   device (down projection)
 *   y    bf16 [T, H]      device, written
 * Enqueues router, dispatch scan, dispatch scatter, the persistent expert
 * GEMM and the bf16 cast of the output on `stream`; no host synchronisation
 * and no host read of routing. T = 0 enqueues nothing. Errors:
 * MOE_ERR_INVALID_ARG, MOE_ERR_NO_WORKSPACE, MOE_ERR_CUDA (launch failure). */
int moe_forward(moe_plan_t plan, const void* x, const void* Wg, const float* gate_bias, const void* W1,
                const void* W3, const void* W2, int T, void* y, void* stream);

/* moe_forward for a plan with shared experts (moe_plan_create_shared), which
 * run as more blocks of the same persistent expert GEMM:
 *   Ws1  bf16 [S, H, I]   device (shared experts' gated branch)
 *   Ws3  bf16 [S, H, I]   device (linear branch)
 *   Ws2  bf16 [S, I, H]   device (down projection)
 * With S = 0 the shared pointers are ignored and may be NULL. Errors as for
 * moe_forward; a NULL or misaligned shared pointer with S > 0 is
 * MOE_ERR_INVALID_ARG. */
int moe_forward_shared(moe_plan_t plan, const void* x, const void* Wg, const float* gate_bias, const void* W1,
                       const void* W3, const void* W2, const void* Ws1, const void* Ws3, const void* Ws2, int T,
                       void* y, void* stream);

/* moe_forward with x and y in HOST memory: copies x [T, H] into the
 * workspace's staging buffer, runs the layer, copies y [T, H] back, all
 * enqueued on `stream` (pinned host buffers make the copies asynchronous; the
 * caller synchronises the stream before reading y). Weights stay on the device. */
int moe_forward_host(moe_plan_t plan, const void* x_host, const void* Wg, const float* gate_bias, const void* W1,
                     const void* W3, const void* W2, int T, void* y_host, void* stream);

/* moe_forward_host for a plan with shared experts (see moe_forward_shared). */
int moe_forward_host_shared(moe_plan_t plan, const void* x_host, const void* Wg, const float* gate_bias,
                            const void* W1, const void* W3, const void* W2, const void* Ws1, const void* Ws3,
                            const void* Ws2, int T, void* y_host, void* stream);

/* ---- FP8 E4M3 expert GEMMs ("MegaMoE 在 MoE 系统谱系中的位置", section 一:
 * the expert GEMMs take 8-bit operands whose scale factors are loaded beside
 * them; section 2.1: the activation is quantized from its amax between the
 * two GEMMs). Scales are powers of two: for a row (or column) with largest
 * magnitude amax the scale is the smallest 2**k with amax / 2**k <= 448 (1
 * when amax == 0), so dividing by it is exact; a code is the E4M3 value
 * nearest to value / scale (ties to even, saturating at +-448). Both GEMMs
 * run on tcgen05 kind::f8f6f4 with fp32 accumulation: x per token, W1 / W3 /
 * W2 per (expert, output column), and the activation h = bf16(silu(g) * u)
 * per token over I (its amax is gathered by the first GEMM's epilogues, and
 * each row is quantized once before the second GEMM). Accumulators are
 * multiplied by the row and column scales in the epilogues. */

/* Codes and scales of a weight tensor, done once per set of weights:
 *   W     bf16 [E, K, N]  device (W1 or W3: K = H, N = I; W2: K = I, N = H,
 *                         as moe_forward takes them)
 *   Wq    u8   [E, N, K]  device, written: K-major E4M3 codes, 16-byte aligned
 *   scale fp32 [E, N]     device, written: per (expert, column) scale over K
 * K % 64 == 0 and N % 64 == 0 (the arguments H and I are K and N). Enqueued
 * on `stream`. Errors: MOE_ERR_INVALID_ARG (null, misaligned or bad sizes),
 * MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_CUDA. */
int moe_quantize_weights_fp8(const void* W, void* Wq, float* scale, int E, int H, int I, void* stream);

/* Codes and scales of activations, as moe_forward_fp8 forms them inside its
 * first kernel (exposed so the quantization can be checked on its own):
 *   x  bf16 [T, H] device (16-byte aligned), xq u8 [T, H] device (8-byte
 *   aligned) written, sx fp32 [T] device written (per-token scale over H).
 * H % 8 == 0. Errors: MOE_ERR_INVALID_ARG, MOE_ERR_CUDA. */
int moe_quantize_x_fp8(const void* x, void* xq, float* sx, int T, int H, void* stream);

/* Give the plan the workspace regions of the FP8 forward (enable = 1) or
 * drop them (0): the activation of all blocks at once (bf16 and E4M3 codes)
 * and its per-row amax and scale, so moe_plan_workspace_bytes grows. Unbinds
 * the workspace: call moe_plan_bind_workspace again afterwards. Plans with
 * shared experts: MOE_ERR_UNSUPPORTED_SHAPE. */
int moe_plan_set_fp8(moe_plan_t plan, int enable);

/* moe_forward with FP8 expert GEMMs (the plan needs moe_plan_set_fp8(plan, 1)). W1q / W3q, s1 / s3 (u8 [E, I, H], fp32
 * [E, I]) and W2q / s2 (u8 [E, H, I], fp32 [E, H]) come from
 * moe_quantize_weights_fp8; all 16-byte aligned. x is quantized per token on
 * the device at the start of each call (into the workspace); the gate and
 * routing are the bf16 layer's. The expert GEMM runs as two launches: the
 * first GEMM with the bf16 activation and its row amax, then (after the
 * activation rows are quantized once each) the second GEMM. A plan without
 * FP8 regions or with shared experts: MOE_ERR_INVALID_ARG. Other errors as
 * for moe_forward. */
int moe_forward_fp8(moe_plan_t plan, const void* x, const void* Wg, const float* gate_bias, const void* W1q,
                    const float* s1, const void* W3q, const float* s3, const void* W2q, const float* s2, int T,
                    void* y, void* stream);

/* moe_forward_fp8 with x and y in HOST memory (see moe_forward_host). */
int moe_forward_host_fp8(moe_plan_t plan, const void* x_host, const void* Wg, const float* gate_bias,
                         const void* W1q, const float* s1, const void* W3q, const float* s3, const void* W2q,
                         const float* s2, int T, void* y_host, void* stream);

/* ---- Pipelined host-buffer forward (serving loops). Like moe_forward_host,
 * but the copies run on two streams of the plan's own, so that the copy of
 * one call's x in and the previous call's y out overlap the neighbouring
 * calls' kernels (which run on `stream`, in call order). Calls use the two
 * halves of the plan's staging buffers in turn: a half is refilled only after
 * the forward that read it has finished and its y has been copied out. The
 * caller keeps x_host and y_host untouched until the call's copies are done:
 * moe_host_pipeline_join(plan, stream) makes `stream` wait for every copy
 * issued so far (synchronise `stream` after it before reading y_host).
 * Plans with shared experts: MOE_ERR_INVALID_ARG. Do not interleave with
 * moe_forward_host* calls on the same plan without a join in between.
 * Errors as for moe_forward_host (moe_forward_host_fp8 for the FP8 form). */
int moe_forward_host_pipelined(moe_plan_t plan, const void* x_host, const void* Wg, const float* gate_bias,
                               const void* W1, const void* W3, const void* W2, int T, void* y_host, void* stream);
int moe_forward_host_pipelined_fp8(moe_plan_t plan, const void* x_host, const void* Wg, const float* gate_bias,
                                   const void* W1q, const float* s1, const void* W3q, const float* s3,
                                   const void* W2q, const float* s2, int T, void* y_host, void* stream);

/* Order the pipeline's later copies after the work already enqueued on `stream`
 * (for instance a timing event). A no-op before the first pipelined call. */
int moe_host_pipeline_after(moe_plan_t plan, void* stream);

/* Make `stream` wait for every pipelined copy issued so far (enqueue only). */
int moe_host_pipeline_join(moe_plan_t plan, void* stream);

/* Gate and dispatch only (router, scan, scatter) for T tokens; fills the
 * routing results exactly as moe_forward does, without the expert FFN. */
int moe_route(moe_plan_t plan, const void* x, const void* Wg, const float* gate_bias, int T, void* stream);

/* Synchronise `stream`, return the sticky device error of the plan's
 * workspace (MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_BOUNDS) and
 * clear it; MOE_ERR_CUDA if the stream reports an error. If `detail` is not
 * NULL it receives the error's detail word (which wait or which block). */
int moe_check(moe_plan_t plan, void* stream, int32_t* detail);

/* Profiling: when enabled, moe_forward records CUDA events on its stream
 * around each of its five kernels (moe_forward_fp8: the router segment also
 * holds the x quantizer, the expert-GEMM segment both GEMM launches and the
 * activation quantizer between them). moe_plan_profile_read() synchronises on
 * the last recorded event, writes the summed milliseconds of each kernel
 * (router, scan, scatter, expert GEMM, finalize) over the forwards recorded
 * since the previous read into ms[0..4], the number of such forwards into
 * *count, and resets the sums. At most 256 forwards are kept between reads. */
int moe_plan_set_profiling(moe_plan_t plan, int enable);
int moe_plan_profile_read(moe_plan_t plan, float* ms, int* count);

/* Test hooks: the persistent kernel gives up any device-side wait after
 * timeout_ns nanoseconds (default 2e9) and records MOE_ERR_DEVICE_TIMEOUT;
 * withhold_block >= 0 makes the kernel never publish the completion of that
 * L1 block, so the L2 tasks waiting on it time out. -1 restores normal runs. */
int moe_plan_set_debug(moe_plan_t plan, int withhold_block, uint64_t timeout_ns);

/* Routing without any device allocation: the gate and the dispatch of
 * moe_route(), for callers that cannot allocate device memory - for example
 * code running inside an inference engine's enqueue-style callback where
 * allocation is not allowed, a process whose device memory is fully
 * reserved up front by a framework's pool so cudaMalloc would fail, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device-wide
 * synchronisation. It needs no plan and no workspace: its scratch (ranks,
 * per-chunk counts, counters, error word) lives in a fixed 1 MiB device array
 * inside this library, which every GPU that loads the library holds until the
 * process exits. The pages have no counterpart of this entry point.
 *
 * Runs on the calling thread's current device; x [T,H] and Wg [H,E] (bf16),
 * gate_bias [E] (fp32, or NULL) and every output are device pointers on it.
 * The caller passes the outputs, laid out as in moe_routing:
 *   topk_idx int32 [T,k], topk_w fp32 [T,k], expert_count int32 [E],
 *   expert_offset int32 [E+1], slot_token and slot_topk int32 [pool_capacity],
 *   num_padded int32 [1]; error_word int32 [1] or NULL receives the device
 *   error code of this call (0 = none, 2 = a routing index out of range).
 * block_m = 0 applies the same BLOCK_M rule as moe_plan_create. The slots in
 * use are at most pool = ceil((T*k + E*(BLOCK_M-1)) / BLOCK_M) * BLOCK_M;
 * pool_capacity must be at least that.
 * Limit: 128 + T*k + ceil(T/64)*E + (E+1) + pool/BLOCK_M int32 values (each
 * term rounded up to a multiple of 64) must fit in 262144; larger sizes return
 * MOE_ERR_STATIC_SCRATCH_LIMIT before anything is enqueued (T = 16384, k = 8,
 * E = 256 fits). Shape rules as moe_plan_create; T = 0 enqueues nothing.
 * The first call on each device resolves the array's device address and sets
 * kernel attributes (host-side set-up, no allocation); make that first call
 * before any stream capture. Every call shares the one array and clears its
 * error word itself, so calls whose GPU work overlaps in time (other streams,
 * other host threads) race on the scratch: serialise them. Allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library call). */
int moe_route_static(const void* x, const void* Wg, const float* gate_bias, int T, int H, int E, int k,
                     int block_m, int32_t* topk_idx, float* topk_w, int32_t* expert_count, int32_t* expert_offset,
                     int32_t* slot_token, int32_t* slot_topk, int pool_capacity, int32_t* num_padded,
                     int32_t* error_word, void* stream);

/* Expert-GEMM variant: enable != 0 runs the persistent expert GEMM on CTA
 * pairs (clusters of two CTAs on neighbouring SMs, tcgen05 cta_group::2):
 * each task covers two consecutive blocks of one expert (256 rows) and each
 * CTA loads half of the weight tile. enable = 0 runs one CTA per block. A new
 * plan uses pairs when BLOCK_M is 128 and the device can co-schedule 2-CTA
 * clusters, else one CTA per block. Results are the same up to fp32
 * summation order. Takes effect at the next moe_forward; the workspace size
 * does not depend on it. Errors: MOE_ERR_INVALID_ARG (null plan),
 * MOE_ERR_UNSUPPORTED_SHAPE (pairs requested where no 2-CTA cluster fits). */
int moe_plan_set_cta_pairs(moe_plan_t plan, int enable);

/* Order in which the persistent expert GEMM hands out its tasks (the same
 * tasks and results either way; "MegaMoE 在 MoE 系统谱系中的位置", section 2.7:
 * one queue holds the tasks of both GEMMs and an L2 task runs once the L1
 * tasks of its rows are done). Blocks (or block pairs) are cut into groups;
 *   0  staggered: L1 of group 0, L1 of group 1, L2 of group 0, L1 of group 2,
 *      L2 of group 1, ...;
 *   1  interleaved: after the L1 tasks of group 0, each segment hands out a
 *      lag of L1 tasks of group m and then mixes the rest of them evenly with
 *      the L2 tasks of group m-1, so that a CTA alternates the two kinds and
 *      a second-GEMM combine epilogue overlaps a first-GEMM MMA;
 *  -1  automatic (the default): staggered, which measured 1-2 % faster than
 *      interleaved on the fine-grained and skewed layers and as fast on the
 *      others.
 * FP8 forwards (one launch per GEMM) ignore it. Errors: MOE_ERR_INVALID_ARG
 * (null plan or another mode). */
int moe_plan_set_task_order(moe_plan_t plan, int mode);

/* Tile size of an expert's last block on CTA pairs, chosen from the expert's
 * load ("MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
 * Replication", abstract: the planner cuts each expert's tokens into
 * tile-aligned blocks; here on one GPU, without replication). A pair task
 * covers two 128-row blocks of one expert with M = 256 MMAs. When an expert
 * has an odd number of blocks (every cold expert with at most 128 tokens has
 * one), its last block alone would leave the second CTA of the pair without
 * rows while the M = 256 MMA still costs two blocks. With enable = 1 (the
 * default) that block runs as M = 128 pair MMAs, 64 of its rows in each CTA,
 * at half the tensor time; with 0 it runs as before. Applies to bf16
 * forwards with BLOCK_M = 128 on CTA pairs; results are the same either way
 * (up to the order of the fp32 combine additions). Errors: MOE_ERR_INVALID_ARG
 * (null plan). */
int moe_plan_set_half_tails(moe_plan_t plan, int enable);

/* Width of the first GEMM's tasks on CTA pairs (bf16, I % 256 == 0). With
 * mode = 1 an L1 task computes 256 columns of I (W1 and W3 both) for its 256
 * routed rows as two N = 256 MMAs per K block on the same gathered x tile,
 * filling both TMEM accumulators (four 48 KB pipeline stages instead of six
 * of 32 KB); with 0 it computes 128 columns; -1 (the default) picks 1 when
 * I <= 1024, where the first-GEMM tasks are short (measured: 2.5 % faster on
 * I = 768, 1.5-3 % slower on I = 2048 and 14336). Results are the same
 * either way. Errors: MOE_ERR_INVALID_ARG (null plan or another mode). */
int moe_plan_set_wide_l1(moe_plan_t plan, int mode);

/* Give the plan the workspace regions of moe_backward (enable = 1) or drop them
 * (0). The workspace size changes: query moe_plan_workspace_bytes and bind a
 * workspace again. Plans with shared experts have no backward.
 * Errors: MOE_ERR_INVALID_ARG (null plan), MOE_ERR_UNSUPPORTED_SHAPE (shared experts). */
int moe_plan_set_backward(moe_plan_t plan, int enable);

/* Backward of the layer for the upstream gradient dy: the chain-rule gradients
 * of y = sum_j w[t,j] FFN_{e_j}(x[t]) with respect to x, Wg, the gate bias and
 * the expert weights ("MegaFlux: Skew-Resilient MoE Megakernels via Pipelined
 * Expert Replication", abstract: a backward MoE megakernel that reduces the
 * experts' weight gradients; the pages do not define it further). Readings:
 * the choice of the k experts is piecewise constant (no gradient through it);
 * the softmax over the k kept logits is differentiated; the bf16 rounding of
 * the SwiGLU activation passes the gradient unchanged, while dW2 and the
 * gradient of the combine weights use the rounded activation the forward
 * multiplied. The routing is recomputed from x on the device (router and
 * dispatch, as in moe_forward), then: dgrad (x and dy rows gathered through
 * the slot records; g, u and dy W2^T on tcgen05; dg, du in the epilogue; dx
 * added through the slot records), the gate backward, and the weight
 * gradients as reductions over each expert's slots on tcgen05.
 *   x, Wg, gate_bias, W1, W3, W2: as for moe_forward (device)
 *   dy   bf16 [T, H]  device, the upstream gradient of y
 *   dx   bf16 [T, H]  device, out
 *   dWg  fp32 [H, E]  device, out
 *   dbias fp32 [E]    device, out, or NULL (not computed)
 *   dW1, dW3 bf16 [E, H, I], dW2 bf16 [E, I, H]  device, out (experts no token
 *        chose get zeros)
 * Outputs are overwritten, not accumulated into. The plan needs
 * moe_plan_set_backward(plan, 1) and a bound workspace; every pointer but
 * dbias non-NULL and 16-byte aligned (dWg and dbias 4-byte). Enqueued on
 * `stream` only. Intermediates: dg, du and w * activation per slot
 * ([pool, I] bf16 each) and the dense gate-logit gradient live in the
 * workspace. Errors: MOE_ERR_INVALID_ARG (no backward regions, shared
 * experts, bad pointers, T out of range), MOE_ERR_NO_WORKSPACE,
 * MOE_ERR_CUDA; device-side errors through moe_check. */
int moe_backward(moe_plan_t plan, const void* x, const void* Wg, const float* gate_bias, const void* W1,
                 const void* W3, const void* W2, const void* dy, int T, void* dx, float* dWg, float* dbias,
                 void* dW1, void* dW3, void* dW2, void* stream);

/* Give the plan a task log (enable = 1) or drop it (0): every expert-GEMM
 * launch then writes one moe_task_record per task into the workspace (48
 * bytes x every block, or pair, x the GEMMs' column tiles; the region is
 * reset before each launch, on the stream). The workspace size changes:
 * bind a workspace again. Costs one store per task. Errors:
 * MOE_ERR_INVALID_ARG (null plan). */
int moe_plan_set_task_log(moe_plan_t plan, int enable);

/* Device pointer to the task log of the last launch and its number of
 * records (read it after the forward's stream work has finished, e.g. after
 * moe_check). With FP8 forwards (two launches) it holds the second launch.
 * Errors: MOE_ERR_INVALID_ARG (null arguments, no task log),
 * MOE_ERR_NO_WORKSPACE. */
int moe_plan_get_task_log(moe_plan_t plan, const moe_task_record** records, int* capacity);

/* Number of kernels one moe_forward launches (for launch accounting). */
int moe_forward_kernel_count(void);

/* Number of kernels one forward of this plan launches: moe_forward_kernel_count()
 * for bf16 (fp8 = 0); for moe_forward_fp8 (fp8 = 1) the router, dispatch scan
 * and scatter and the finalize, the x quantizer, and per block group of the FP8
 * schedule the first GEMM, the activation quantizer and the second GEMM (groups
 * past the routing's last block exit at once but are still launched).
 * -1: null plan, or fp8 = 1 on a plan without FP8 regions. */
int moe_plan_forward_launches(moe_plan_t plan, int fp8);

void moe_plan_destroy(moe_plan_t plan);
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
