/*
 * moe_b200.h -- C ABI of libmoe_b200.so: the forward pass of one
 * Mixture-of-Experts FFN layer with FP8 (E4M3) activations and MXFP4 (E2M1 +
 * UE8M0) expert weights on one NVIDIA B200 (sm_100a).
 *
 * What the layer computes (page title, section):
 *   router scores, biased top-k selection, softmax gates over the unbiased
 *   scores of the selected experts     -- "전문가 혼합(Mixture of Experts; MoE)"
 *                                         lesson, "FFN 교체", "부하 분산 문제",
 *                                         "Step 1: 라우터";
 *   dispatch -> linear1 (FP8 x FP4) -> SwiGLU -> linear2 (FP8 x FP4) -> combine
 *                                       -- "DeepSeek Mega MoE / DeepGEMM mega
 *                                         kernel", "TL;DR" and the
 *                                         "Thông số kỹ thuật" table; "Mega MoE"
 *                                         wiki, "한 줄 정의";
 *   an always-on shared expert          -- MoE lesson, "공유 전문가".
 * On one device dispatch and combine are an in-memory permutation and gather.
 *
 * Conventions shared by every entry point
 *   - All arrays are row-major and contiguous.  Every array pointer is a DEVICE
 *     pointer on the device that was current when moe_set_workspace() ran,
 *     16-byte aligned; W1 and W2 must be 32-byte aligned.  The caller owns all
 *     memory (inputs, outputs, workspace) and the plan.  The library never
 *     allocates device memory.
 *   - Shapes: T tokens, hidden size H, expert intermediate size I, E routed
 *     experts, k experts per token, shared in {0,1}; n = E + shared; R = T*k.
 *     Constraints: T >= 1, H % 128 == 0, I % 128 == 0, 1 <= k <= min(E, 16),
 *     1 <= E <= 1024.  Violations return MOE_ERR_UNSUPPORTED_SHAPE.
 *   - x         bf16  [T, H]
 *     W_router  fp32  [E, H]            routed experts only
 *     bias      fp32  [E]               added to the scores for selection only
 *     W1        uint8 [n, 2I, H/2]      MXFP4 codes; rows 0..I-1 = gate,
 *                                       rows I..2I-1 = up; byte j of a row holds
 *                                       element 2j (low nibble), 2j+1 (high)
 *     W1_scales uint8 [n, 2I, H/32]     UE8M0, one per 32 consecutive K elements
 *     W2        uint8 [n, H, I/2]       MXFP4 codes
 *     W2_scales uint8 [n, H, I/32]      UE8M0
 *     out       bf16  [T, H]
 *     Expert index E is the shared expert when shared == 1.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All compute entry points are asynchronous and stream-ordered; they never
 *     synchronise the host.  Device-side failures (bounded waits that ran out)
 *     are recorded in the workspace and reported by moe_check_status().
 *   - Return codes are the MOE_* values below.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_plan_s* moe_plan_t;

enum moe_status_code {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,        /* NULL/misaligned pointer, bad option, plan state */
  MOE_ERR_UNSUPPORTED_SHAPE = -2,  /* shape outside the constraints above           */
  MOE_ERR_CUDA = -3,               /* a CUDA runtime/driver call or launch failed    */
  MOE_ERR_DEVICE_TIMEOUT = -4,     /* a device-side wait ran out (see check_status)  */
  MOE_ERR_WORKSPACE = -5,          /* workspace missing or too small                 */
  MOE_ERR_DEBUG_BOUNDS = -6        /* a device-side bounds check failed              */
};

enum moe_option {
  MOE_OPT_MAX_SMS = 1,         /* persistent GEMM grid size cap (0 = all SMs)            */
  MOE_OPT_TIMEOUT_NS = 2,      /* device wait limit in ns (default 2e9)                  */
  MOE_OPT_INJECT_FAULT = 3,    /* test hook: 1 = the linear1 TMA producer of one CTA never
                                  fills its first pipeline stage, so the MMA warp's
                                  bounded wait runs out and the call reports
                                  MOE_ERR_DEVICE_TIMEOUT                                  */
  MOE_OPT_ROUTER_TC = 4,       /* 1 (default): router logits on tensor cores when T >= 64
                                  and E % 16 == 0, as x (bf16) times W_router split into two
                                  bf16 parts (hi = bf16(W), lo = bf16(W - hi); |residual| <=
                                  2^-18 |W|) accumulated in fp32; 0: fp32 FMA on CUDA cores */
  MOE_OPT_PHASE_EVENTS = 5,    /* 1 = record a CUDA event after each kernel of moe_forward
                                  on its stream, read back with moe_phase_times()        */
  MOE_OPT_STATIC_WEIGHTS = 6,  /* 1 = the caller promises that W_router / W1_scales /
                                  W2_scales do not change between calls that pass the same
                                  pointers: moe_forward then reuses the tiled scale units
                                  and the split router weights built by the last
                                  moe_prepare_weights (or forward) from those pointers.
                                  0 (default): every forward rebuilds them.              */
  MOE_OPT_GRAPH = 7,           /* 1 = moe_forward records its launch sequence as a CUDA
                                  graph the first time it sees a set of argument pointers
                                  (up to 4 sets per plan) and replays it on later calls,
                                  removing per-kernel launch overhead.  Not used while the
                                  caller's stream is capturing or MOE_OPT_PHASE_EVENTS is
                                  1.  The CUDA runtime may reserve memory for the recorded
                                  graphs; changing any option drops them.  Default 0.    */
  MOE_OPT_SWAP_ROWS = 8,       /* grouped GEMM row tiles holding at most this many rows of
                                  their expert (0, 32 or 64; default 0) are computed
                                  transposed: 128 weight rows as the MMA's M side and the
                                  tile's tokens as N = 32 or 64.  Fewer multiply-adds, but
                                  twice the MMA instructions, each with a fixed cost, so
                                  it measured slower on B200; kept as an option.
                                  0 = always 128 token rows.  Single-CTA kernel only.     */
  MOE_OPT_PAIR_TILES = 9,      /* grouped GEMMs on CTA pairs (2-CTA clusters, one
                                  M = 256 MMA across the pair, each CTA loading half of
                                  the weight tile): 0 = never, 1 (default) = when the
                                  experts average >= 1024 rows (T*k >= 1024*E), 2 = always.
                                  Needs 128-row tiles.                                     */
  MOE_OPT_FUSED = 10,          /* 1 = moe_forward runs every step (router, top-k, dispatch
                                  scans, scatter + quantisation, linear1, linear2, combine)
                                  in ONE persistent cooperative kernel, one CTA per SM:
                                  grid-wide barriers after the router and after top-k and
                                  the scans; from there on readiness counters (bounded
                                  waits) -- the linear1 producers start once every CTA has
                                  scattered its share (done by the epilogue warps before
                                  their first tile), linear2 tiles once their expert's
                                  linear1 tiles are stored, the combine (epilogue warps,
                                  bulk copies into the idle operand buffers) once every
                                  linear2 tile is.  Weight preparation, when needed, runs
                                  before it.  Router: tensor cores when MOE_OPT_ROUTER_TC
                                  applies; with at most 16 tokens (E a multiple of 4, at
                                  most 256) a warp per (expert, K part) over all tokens;
                                  else CUDA cores as the separate launches.  With MOE_OPT_PHASE_EVENTS = 1 every CTA writes
                                  the global timer at each step into the "stamps" region
                                  and moe_phase_times splits the kernel's time by them.
                                  No CUDA graph is recorded.  Default 0.                  */
  MOE_OPT_DEPENDENT_LAUNCH = 11, /* 1: the kernels after the first of a moe_forward are
                                  launched as programmatic dependents (each waits on the
                                  device for its predecessor; the grouped GEMMs request
                                  their first weight tiles before that wait).  0 = plain
                                  stream order.  2 (default) = automatic: dependent
                                  launches for T <= 64 (short kernels, where launch latency
                                  counts), plain order above (there the GEMMs' early CTAs
                                  slowed the scatter).  Off while MOE_OPT_PHASE_EVENTS is
                                  1.  moe_plan_get_option reports 1 or 0.                  */
  MOE_OPT_L2_TILE_ROWS = 12,   /* linear2 weight rows per tile: 0 (default) = 224 when
                                  T <= 16 and H % 224 == 0, else 256; 224 = always when
                                  H % 224 == 0 (else MOE_ERR_UNSUPPORTED_SHAPE): the
                                  narrower tile leaves TMEM room for two accumulators, so
                                  one tile's epilogue overlaps the next tile's MMAs;
                                  256 = always.  CTA-pair GEMMs always use 256.            */
  MOE_OPT_CHAIN = 13,          /* 1 = with at most 16 tokens, linear1 and linear2 run as
                                  one cooperative launch: each linear2 tile's producer
                                  streams its weights at once and waits (bounded) only
                                  for the linear1 tiles of its own expert.  moe_phase_times
                                  reports both under linear1.  Measured slower inside a
                                  CUDA graph (the cooperative launch cannot start early
                                  as the dependent launches do).  0 (default) = two
                                  launches.                                                */
  MOE_OPT_TILE_ROWS = 14,      /* rows of the grouped GEMMs' row tiles: 0 (default) = 32
                                  when T <= 32 and the routed experts average at most 32
                                  rows (T*k <= 32*E) and neither transposed tiles nor
                                  forced CTA pairs are asked for, else 128; 32 or 128 =
                                  always.  32-row tiles run on a shared-memory layout with
                                  32-row A regions and 6 pipeline stages (more weight bytes
                                  in flight per SM); the MMA still spans 128 rows.  32 is
                                  incompatible with MOE_OPT_SWAP_ROWS != 0 and
                                  MOE_OPT_PAIR_TILES = 2 (MOE_ERR_INVALID_ARG).  The
                                  activation scale atoms (and moe_workspace_region's "xsf"
                                  and "hsf" regions) are laid out per row tile.            */
  MOE_OPT_ZERO_PAD = 15        /* on 128-row tiles, the A rows a tile does not fill are
                                  zeroed (a bulk copy from a zero buffer in the workspace)
                                  before the MMA, which spans all 128 rows, reads them:
                                  zero operands draw less power than stale rows of earlier
                                  tiles, which raises the clock where the power limit holds
                                  it down.  The results do not change.  0 (default) = when
                                  the routed experts average at most 32 rows (T*k <= 32*E)
                                  and the tiles have 128 rows; 1 = always (128-row tiles);
                                  2 = never.  moe_plan_get_option reports 1 (on) or 2.     */
};

/* Phases of moe_forward, in launch order (moe_phase_times). */
enum moe_phase {
  MOE_PHASE_ROUTER = 0, MOE_PHASE_TOPK, MOE_PHASE_SCAN, MOE_PHASE_SCATTER_QUANT,
  MOE_PHASE_PREPARE,     /* weight scale re-layout (zero when reused, MOE_OPT_STATIC_WEIGHTS) */
  MOE_PHASE_LINEAR1, MOE_PHASE_LINEAR2, MOE_PHASE_COMBINE, MOE_PHASE_COUNT_
};

/* Workspace regions (moe_workspace_region) -- for tests and debugging. */
enum moe_region {
  MOE_REGION_STATUS = 0,   /* uint32 [4]: code, where, block, detail                      */
  MOE_REGION_TOPK_IDS,     /* int32  [T, k]                                               */
  MOE_REGION_GATES,        /* fp32   [T, k]                                               */
  MOE_REGION_COUNTS,       /* int32  [n]                                                  */
  MOE_REGION_OFFSETS,      /* int32  [n + 1]                                              */
  MOE_REGION_PERM,         /* int32  [R]                                                  */
  MOE_REGION_SLOT_POS,     /* int32  [T, k]                                               */
  MOE_REGION_XQ,           /* uint8  [R + shared*T, H]   E4M3, dispatched row order       */
  MOE_REGION_XSF,          /* scale atoms of XQ: [row tile][H/128] x 512 B, see below    */
  MOE_REGION_HQ,           /* uint8  [R + shared*T, I]   E4M3 SwiGLU output               */
  MOE_REGION_HSF,          /* scale atoms of HQ: [row tile][I/128] x 512 B               */
  MOE_REGION_Y,            /* bf16   [R + shared*T, H]   expert output rows               */
  MOE_REGION_STAMPS,       /* uint64 [stamp point][1024]: global-timer ns at which each CTA of
                              the last MOE_OPT_FUSED forward run with MOE_OPT_PHASE_EVENTS = 1
                              passed each point of the kernel (debug; see moe_phase_times)  */
  MOE_REGION_COUNT_
};

/* Scale atoms.  Expert e's dispatched rows [offsets[e], offsets[e+1]) form
 * ceil(count/128) row tiles; row tile g = (sum of the row tiles of experts
 * before e) + rank/128 holds the row of rank `rank` inside the expert at
 * r = rank % 128.  Atom (g, kt) is 512 bytes; the row's UE8M0 code (p + 127)
 * for channels [128 kt, 128 kt + 128) sits in all four bytes at offset
 * (r % 32) * 16 + (r / 32) * 4.  Bytes of rows past the expert's count are
 * unspecified. */

/* Create a plan for one layer shape.  Host only; touches no device.
 * `out` receives a heap object the caller releases with moe_plan_destroy(). */
int moe_plan(int T, int H, int I, int E, int k, int shared, moe_plan_t* out);

/* Set a moe_option.  Returns MOE_ERR_INVALID_ARG for an unknown key/value. */
int moe_plan_set_option(moe_plan_t plan, int key, long long value);
/* The value an option has for this plan, resolved: MOE_OPT_TILE_ROWS and
 * MOE_OPT_L2_TILE_ROWS report the row-tile heights the next forward uses (32 or
 * 128; 224 or 256), every other key the value last set (or its default).
 * MOE_ERR_INVALID_ARG for an unknown key or a NULL pointer.  No device work. */
int moe_plan_get_option(moe_plan_t plan, int key, long long* value);

/* Bytes of device workspace the plan needs (0 for a NULL plan). */
size_t moe_workspace_bytes(moe_plan_t plan);

/* Bind caller-allocated device workspace (>= moe_workspace_bytes, 256-byte
 * aligned).  The device current at this call becomes the plan's device. */
int moe_set_workspace(moe_plan_t plan, void* workspace, size_t bytes);

/* Offset and size of a workspace region (moe_region) in bytes. */
int moe_workspace_region(moe_plan_t plan, int region, size_t* offset, size_t* bytes);

/* The whole layer: out = bf16( sum_j gate[t,j] * Expert_{id[t,j]}(x_t) + shared*Expert_E(x_t) ).
 * Requantisation points: x -> E4M3 (per token per 128 channels, power-of-two
 * scale), SwiGLU output -> E4M3 (same rule), expert rows -> bf16, out -> bf16. */
int moe_forward(moe_plan_t plan, const void* x_bf16, const float* W_router, const float* bias,
                const uint8_t* W1, const uint8_t* W1_scales,
                const uint8_t* W2, const uint8_t* W2_scales,
                void* out_bf16, void* stream);

/* Re-lay out the UE8M0 weight scales (canonical [n][rows][K/32]) into the
 * tiled units the GEMMs load, inside the workspace.  moe_forward does this
 * itself on every call unless MOE_OPT_STATIC_WEIGHTS is 1 and the pointers
 * match the last preparation.  Asynchronous on `stream`. */
int moe_prepare_weights(moe_plan_t plan, const uint8_t* W1_scales, const uint8_t* W2_scales, void* stream);

/* Routing only: topk_ids int32 [T,k] (descending biased score, lower id first
 * on ties) and gates fp32 [T,k] (softmax over the selected unbiased scores). */
int moe_debug_routing(moe_plan_t plan, const void* x_bf16, const float* W_router, const float* bias,
                      int32_t* topk_ids, float* gates, void* stream);

/* Routing without any device allocation.  The pages describe no counterpart:
 * this entry point exists for callers that cannot allocate device memory when
 * they need a routing decision -- e.g. code running while another component
 * owns the CUDA allocator (a serving loop with a fixed, pre-carved memory
 * pool), hooks that must not call back into an allocator, or runtimes that only
 * hand over raw stream and buffer pointers.  It needs no plan and no workspace.
 *
 * Computes exactly what moe_debug_routing computes with MOE_OPT_ROUTER_TC = 0
 * (same kernels: the fp32 CUDA-core router, then the same top-k): topk_ids
 * int32 [T,k] and gates fp32 [T,k] from x bf16 [T,H], W_router fp32 [E,H] and
 * bias fp32 [E], all device pointers supplied by the caller (x and W_router
 * 16-byte aligned).  Its intermediates live in one fixed scratch array of
 * MOE_ROUTE_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library's device memory;
 * every device that loads the library holds that array until the process
 * exits.  The call needs
 *     r(T*E*4) + r(T*k*4) + r(ceil(T/32)*E*4) + 256  bytes,  r(v) = v rounded up to 256,
 * and returns MOE_ERR_WORKSPACE (nothing launched) when that exceeds the array
 * -- about 15,000 tokens at E = 256, k = 8.  Shapes as for moe_plan
 * (MOE_ERR_UNSUPPORTED_SHAPE otherwise).  Calls no allocating routine.
 *
 * Every pointer must be device memory of the CURRENT device (the kernels run
 * there); MOE_ERR_INVALID_ARG otherwise (checked with cudaPointerGetAttributes,
 * before anything is launched).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it for the life of the process; make that first
 * call before any stream capture.  The cached address is not valid after the
 * device is reset (cudaDeviceReset): do not call this entry point again in a
 * process that reset a device it used.  All calls share the one array and
 * leave their intermediates in it:
 * calls whose kernels can overlap on the GPU (different streams without
 * ordering between them) race on it, so order them on one stream or by events.
 * Asynchronous on `stream`. */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (16u << 20)
int moe_route_noalloc(int T, int H, int E, int k, const void* x_bf16, const float* W_router, const float* bias,
                      int32_t* topk_ids, float* gates, void* stream);

/* Dispatch only, from given topk_ids int32 [T,k] (each id in [0,E), distinct
 * within a token): counts int32 [n], offsets int32 [n+1], perm int32 [R]
 * (entry t*k+j at the row token t's j-th copy occupies), slot_pos int32 [T,k].
 * Order: expert-major, ascending token id within an expert; shared rows last. */
int moe_debug_dispatch(moe_plan_t plan, const int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                       int32_t* perm, int32_t* slot_pos, void* stream);

/* Activation quantisation only, token order: xq uint8 [T,H] E4M3 codes and
 * xs fp32 [T,H/128] power-of-two scales (smallest 2^p with amax <= 448*2^p,
 * p >= -126; 1 for an all-zero block); x ~ decode(xq) * xs. */
int moe_debug_quant_x(moe_plan_t plan, const void* x_bf16, uint8_t* xq, float* xs, void* stream);

/* Kernel durations (ms) of the most recent moe_forward that ran with
 * MOE_OPT_PHASE_EVENTS = 1, one per moe_phase, measured with CUDA events on
 * that call's stream.  Waits for those events.  Returns the number of values
 * written (MOE_PHASE_COUNT_), or a negative MOE_* code. */
int moe_phase_times(moe_plan_t plan, float* ms, int capacity);

/* Synchronise `stream`, then return the device-side status recorded since the
 * last call (MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEBUG_BOUNDS) and clear it.
 * `detail` (may be NULL) receives the 4 status words. */
int moe_check_status(moe_plan_t plan, void* stream, uint32_t* detail);

/* One auxiliary-loss-free balancing step on the selection bias ("전문가 혼합(Mixture of
 * Experts; MoE)" lesson, "부하 분산 문제" item 3 and "Step 2: 100개 토큰 라우팅하기"):
 * using the routed experts' row counts of the most recent moe_forward on this plan,
 *   bias[e] += gamma   if counts[e] * E <  T * k   (used less than the mean load),
 *   bias[e] -= gamma   if counts[e] * E >  T * k   (used more),
 *   unchanged          otherwise,
 * one fp32 addition per expert.  bias: device fp32 [E], 4-byte aligned, updated in place;
 * the call is asynchronous on `stream` and must be ordered after the forward whose counts it
 * uses.  Returns MOE_OK, MOE_ERR_INVALID_ARG (NULL/misaligned bias, non-finite gamma),
 * MOE_ERR_WORKSPACE (no workspace bound) or MOE_ERR_CUDA.  The pages' design has this step
 * in training; it never runs inside moe_forward. */
int moe_update_bias(moe_plan_t plan, float* bias, float gamma, void* stream);

/* ---- Dense block-scaled GEMM (the grouped GEMM's linear2 kernel with one group) ----------
 *
 *   out[m][n] = bf16_rne( sum_k  A(m,k) * 2^(A_scales[m][k/128] - 127)
 *                               * E2M1(B, n, k) * 2^(B_scales[n][k/32] - 127) )
 *
 * The operand formats of the expert FFN ("DeepSeek Mega MoE / DeepGEMM mega kernel", "TL;DR":
 * FP8 activations x FP4 weights): A = E4M3 codes [M][K] with one UE8M0 (power-of-two) scale
 * per row per 128 K-channels, B = packed E2M1 [N][K/2] (low nibble = even element) with one
 * UE8M0 scale per row per 32 K, fp32 accumulation on the tensor cores, bf16 output [M][N],
 * all row-major.  Constraints: M >= 1, N % 128 == 0, K % 128 == 0, M*K < 2^31 and N*K < 2^32;
 * A, B and out 16-byte aligned, the scale arrays 4-byte aligned; all device pointers on the
 * current device.  Codes 0x7F/0xFF (E4M3 NaN) and scale 0xFF give NaN results. */

/* Device workspace moe_gemm_fp8_fp4 needs for an M x N x K product (scale atoms, bookkeeping
 * and 16 bytes of status). */
size_t moe_gemm_workspace_bytes(int M, int N, int K);

/* Asynchronous on `stream`; the caller owns every buffer.  `workspace` (256-byte aligned, at
 * least moe_gemm_workspace_bytes) holds the status words in its first 16 bytes: word 0 is
 * MOE_OK or MOE_ERR_DEVICE_TIMEOUT once the stream reaches the end of the call (a bounded wait
 * of the kernel ran out).  Returns MOE_OK, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_INVALID_ARG,
 * MOE_ERR_WORKSPACE or MOE_ERR_CUDA. */
int moe_gemm_fp8_fp4(int M, int N, int K, const uint8_t* A, const uint8_t* A_scales, const uint8_t* B,
                     const uint8_t* B_scales, void* out_bf16, void* workspace, size_t workspace_bytes,
                     void* stream);

/* Release a plan (NULL is a no-op).  Does not free the workspace. */
void moe_plan_destroy(moe_plan_t plan);

/* Static string for a return code. */
const char* moe_error_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
