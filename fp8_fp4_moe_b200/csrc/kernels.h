// Host-side launchers of the libmoe_b200 kernels (internal interface).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace moe {

// Programmatic dependent launch of the forward's kernels: while switched on (per host thread),
// the launchers below ask for it.  Every kernel they launch waits on the device for its
// predecessor before reading what earlier kernels wrote (griddep_wait in common.cuh).
void set_dependent_launch(bool on);
bool dependent_launch();
template <class... KArgs, class... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent_launch() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// 2-D tiled tensor map (cuTensorMapEncodeTiled through the runtime's driver entry point):
// dims {inner, outer}, row pitch in bytes, box {box_inner, box_outer}.  MOE_OK or MOE_ERR_CUDA.
// 3-D map over [outer2][outer][inner] with byte strides row_bytes (outer) and slab_bytes (outer2).
int encode_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t outer2, uint64_t row_bytes, uint64_t slab_bytes, uint32_t box_inner, uint32_t box_outer,
              uint32_t box_outer2);
int encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

// ---- grouped block-scaled GEMMs (gemm_sm100.cu) --------------------------------
constexpr int kGemmBM = 128;      // rows (tokens) per tile
// Row tiles of 32 rows: for layers whose experts get few rows each (decode), the GEMMs use a
// shared-memory layout with 32-row A regions and 6 pipeline stages (more weight bytes in
// flight per SM); the MMA still has M = 128, the rows past the tile are never stored.
constexpr int kGemmBMSmall = 32;
constexpr int kGemmBN = 256;      // accumulator columns per tile
constexpr int kGemmBK = 128;      // K per pipeline stage
constexpr int kGemmStages = 4;
// linear2 weight tiles of 224 rows (output columns) leave TMEM room for two accumulators, so
// the epilogue of one tile overlaps the MMAs of the next (single-CTA kernel, H a multiple of
// 224).  Otherwise 256-row tiles with one accumulator.
constexpr int kGemmBN2Double = 224;
constexpr int kGemmThreads = 320; // 10 warps: TMA, MMA, 8 x epilogue

// Scale-factor atoms (the unit the MMA's scale copy reads): 128 rows x 4 K-blocks
// of 32, row r at byte (r%32)*16 + (r/32)*4, K-block b at +b.
//   activations: [row tile g = mtile_start[e] + mt][K/128] atoms of 512 B, the
//                row's power-of-two code in all four bytes (row r < bm of the tile);
//   weights:     [expert][n-tile][K/128] units of 1024 B (two atoms: the tile's
//                B rows 0..127 and 128..255).
struct GemmArgs {
  int bm;              // rows per row tile: kGemmBM, or kGemmBMSmall (small-tile layout only)
  int K;               // reduction length (H for linear1, I for linear2)
  int N;               // linear1: I (SwiGLU width); linear2: H (output width)
  int rows_b;          // B rows per expert (2I or H)
  int n_experts;       // E + shared
  int rows_total;      // R + shared * T
  int n_tiles_n;       // linear1: I/128; linear2: ceil(H/bn)
  int bn;              // linear2: weight rows (output columns) per tile, 256 or kGemmBN2Double
  int swap_rows;       // tiles with at most this many expert rows run transposed (0, 32 or 64)
  const int32_t* counts;       // [n_experts]
  const int32_t* offsets;      // [n_experts + 1]
  const int32_t* mtile_start;  // [n_experts + 1] prefix sum of ceil(count/bm)
  const int32_t* ptile_start;  // [n_experts + 1] prefix sum of ceil(ceil(count/128)/2) (CTA pairs)
  // Row-tile table: entry g in [mtile_start[e], mtile_start[e + 1]) holds {e, mtile_start[e],
  // counts[e], offsets[e]}; the CTA-pair table the same over ptile_start with ptile_start[e]
  // in .y.  An expert's tiles are consecutive (banded row-tile order inside the expert), so
  // tile t belongs to the expert of entry t / n_tiles_n.
  const int4* tile_info;
  const int4* ptile_info;
  // Chained linear1 -> linear2 in one kernel: linear1's epilogue adds 1 to dep_signal[e] when a
  // tile of expert e is stored; linear2's producer loads a tile's A rows only once
  // dep_wait[e] >= ceil(count_e / bm) * dep_per_mtile.  Null outside the chained kernel.
  uint32_t* dep_signal;
  const uint32_t* dep_wait;
  int dep_per_mtile;
  // Single-kernel forward (null elsewhere): the producer loads no A rows or activation scales
  // before *rows_ready >= rows_ready_need (the grid's scatter is done); the epilogue adds 1 to
  // *tiles_done after each stored tile.
  const uint32_t* rows_ready;
  uint32_t rows_ready_need;
  uint32_t* tiles_done;
  // phase timing of the single-kernel forward (null unless asked for): the producer writes the
  // global timer into stamp_rows[cta] once the rows are ready
  unsigned long long* stamp_rows;
  const uint8_t* sfa;          // activation scale atoms
  const uint8_t* sfb;          // weight scale units
  uint8_t* hq;                 // linear1 out: [rows_total][I] E4M3
  uint32_t* hsf;               // linear1 out: activation scale atoms of hq (K = I)
  uint16_t* y;                 // linear2 out: [rows_total][H] bf16
  uint32_t* status;
  uint64_t timeout_ns;
  int inject_fault;
  // 16 KB of zeros (16-byte aligned): with 128-row A regions, the A rows past a tile's box are
  // zeroed from it (null = leave them as they are)
  const uint8_t* zeros;
};
constexpr size_t kGemmZeroBytes = 16384;

size_t gemm_smem_bytes();
cudaError_t gemm_prepare_device();   // sets the kernels' shared-memory attributes
// canonical UE8M0 weight scales [n][rows_b][K/32] -> weight scale units.  mode 1: linear1
// (128 gate + 128 up rows per tile); mode 2: linear2 with tiles of tile_rows weight rows (the
// unit's second atom covers tile rows 128..255; rows past the tile are never used).
cudaError_t launch_tile_weight_scales(const uint8_t* src, uint8_t* dst, int n_experts, int rows_b, int K,
                                      int n_tiles_n, int mode, int N, cudaStream_t s, int tile_rows = kGemmBN);
// A-operand tensor maps of one activation matrix with box heights 16, 32, 64, 128 rows
// (the producer picks the smallest box that covers the tile's rows of its expert).
struct AMaps {
  CUtensorMap m[4];
};
// small_tiles: args.bm == kGemmBMSmall, so the kernel uses the layout with 32-row A regions and
// 6 pipeline stages (no transposed tiles: args.swap_rows must be 0).
cudaError_t launch_gemm_linear1(const AMaps& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s, bool small_tiles = false);
cudaError_t launch_gemm_linear2(const AMaps& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s, bool small_tiles = false);
// linear1 + linear2 in one cooperative launch (small-tile layout, bm == kGemmBMSmall), a
// programmatic dependent of the kernel before it while dependent launches are on:
// g1.dep_signal == g2.dep_wait (n_experts counters, zero before the launch), g2.dep_per_mtile =
// g1.n_tiles_n; b2's box height = g2.bn.  grid <= the co-resident CTAs of the device.
cudaError_t launch_gemm_chain(const AMaps& a1, const AMaps& a2, const CUtensorMap& b1, const CUtensorMap& b2,
                              const GemmArgs& g1, const GemmArgs& g2, int grid, cudaStream_t s);
// CTA-pair variants: b with 128-row boxes (each CTA loads half of the 256 B rows), scale atoms
// and weight scale units as 2-D uint8 maps of 256-byte rows (boxes of 2 and 4 rows); grid =
// 2 x pairs.
cudaError_t launch_gemm_pair_linear1(const AMaps& a, const CUtensorMap& b, const CUtensorMap& sfa,
                                     const CUtensorMap& sfb, const GemmArgs& args, int pairs, cudaStream_t s);
cudaError_t launch_gemm_pair_linear2(const AMaps& a, const CUtensorMap& b, const CUtensorMap& sfa,
                                     const CUtensorMap& sfb, const GemmArgs& args, int pairs, cudaStream_t s);
int gemm_pair_max_clusters();        // co-resident CTA pairs on this device (after gemm_prepare_device)

// ---- router on tensor cores (gemm_sm100.cu) -------------------------------------
constexpr int kRouterThreads = 192;   // 6 warps: TMA, MMA, 4 x epilogue
struct RouterArgs {
  int T, H, E;
  int k_splits;                       // K split into this many equal parts (divides H / 64)
  float* logits;                      // [k_splits][T][E] fp32 partial sums
  uint32_t* status;
  uint64_t timeout_ns;
};
size_t router_tc_smem_bytes();
// K splits of the tensor-core router for a T x E problem: enough CTAs to cover a 148-SM part,
// each split a whole number of 64-wide K stages, at most 16 splits and 4 Mi partial floats.
int router_tc_splits(int T, int H, int E);
// x bf16 [T][H] and W_hi / W_lo bf16 [E][H] as 128-byte-swizzled TMA maps (box 64 x 128).
// Split s of the K range writes its partial logits to logits + s * T * E; top-k adds the
// k_splits parts in split order.
cudaError_t launch_router_tc(const CUtensorMap& x, const CUtensorMap& whi, const CUtensorMap& wlo,
                             const RouterArgs& args, cudaStream_t s);
// W fp32 [n] -> hi = bf16(W), lo = bf16(W - hi)
cudaError_t launch_split_router_weights(const float* W, uint16_t* hi, uint16_t* lo, long n, cudaStream_t s);

// ---- the single persistent forward (gemm_sm100.cu) -------------------------------
// Every step of the forward in one cooperative launch of one CTA per SM (kGemmThreads threads).
// Grid-wide barriers only where every CTA needs every other CTA's result: after the router, and
// after the top-k / dispatch scans (with more than 32 tokens also between top-k, the per-expert
// group scan and the expert scan).  From there on readiness counters replace barriers: the
// GEMM producers stream weights at once and load A rows when the grid's scatter (done by the
// epilogue warps before their first linear1 tile) is complete; linear2 tiles wait per expert for
// its linear1 tiles; the combine (epilogue warps after their last linear2 tile) waits for all
// linear2 tiles.
enum : int { kRouterSplitBlock = 0, kRouterWarp8 = 1, kRouterWarp2 = 2, kRouterTensor = 3, kRouterSplitK = 4 };
// kRouterSplitK: tokens per launch and 256-channel chunks per K part it handles
constexpr int kSplitKMaxT = 16, kSplitKMaxChunks = 8;
struct FusedArgs {
  int T, H, E, k, shared;
  int bm;                          // rows per row tile of the GEMMs
  int router_kind;                 // kRouter*
  int router_parts;                // partial logit arrays (tensor-core router K splits, split-K parts)
  const uint16_t* x;
  const float* W_router;
  const float* bias;
  float* logits;
  int32_t* topk_ids;
  float* gates;
  int32_t* local_rank;
  int32_t* group_counts;
  int32_t* group_base;
  int32_t* counts;
  int32_t* offsets;
  int32_t* mtile_start;
  int32_t* ptile_start;
  int4* tile_info;
  int4* ptile_info;
  int32_t* slot_pos;
  int32_t* perm;
  uint8_t* xq;
  uint8_t* xsf;
  const uint16_t* y;
  uint16_t* out;
  uint32_t* status;
  uint32_t* gridbar;               // [2] arrival count, generation (zeroed before each launch)
  // [0] scatter warps done, [1] linear2 tiles stored, [2 .. 2 + n) linear1 tiles stored per
  // expert: zeroed inside the kernel before the first grid barrier
  uint32_t* counters;
  // phase timing (MOE_OPT_PHASE_EVENTS; null otherwise): stamps[id * kStampMaxCtas + cta] = the
  // global timer (ns) when CTA cta passed point id (kStamp*)
  unsigned long long* stamps;
  uint64_t timeout_ns;
  RouterArgs ra;
  GemmArgs g1, g2;
};
enum : int {
  kStampStart = 0,     // TMEM allocated
  kStampRouted,        // past the grid barrier that follows the router
  kStampScanned,       // past the grid barrier that follows top-k and the dispatch scans
  kStampRowsReady,     // the linear1 producer saw every CTA's scatter done
  kStampLinear1,       // the CTA's linear1 tiles stored
  kStampCombine,       // every linear2 tile stored, combine starts (first epilogue warp)
  kStampEnd,           // the CTA's combine items written
  kStampRouterDone,    // the CTA's own router items done (before the barrier)
  kStampTopkDone,      // top-k of the CTA's token groups done (before the scans)
  kStampScanDone,      // the expert scan done (CTA 0)
  kStampScatterDone,   // the CTA's epilogue warps finished their scatter items
  kStampCount
};
constexpr int kStampMaxCtas = 1024;
// small_tiles: the 32-row, 6-stage GEMM layout (g1.bm == kGemmBMSmall); g2.bn = 224 or 256.
cudaError_t launch_fused_forward(const AMaps& a1, const AMaps& a2, const CUtensorMap& b1, const CUtensorMap& b2,
                                 const CUtensorMap& x, const CUtensorMap& whi, const CUtensorMap& wlo,
                                 const FusedArgs& args, int ctas, bool small_tiles, cudaStream_t s);
int fused_max_ctas();                // co-resident CTAs of the fused kernel (after gemm_prepare_device)

// ---- routing / dispatch / combine (path_kernels.cu) -----------------------------
cudaError_t launch_router_logits(const uint16_t* x, const float* W_r, float* logits, int T, int H, int E,
                                 cudaStream_t s);
// mode 0: select from logits (+bias), write ids/gates, then rank.  mode 1: rank given ids.
// mode 1 validates the given ids (range, distinct per token) and records MOE_ERR_DEBUG_BOUNDS in `status`.
// logits holds n_parts partial [T][E] arrays (consecutive); a score is their sum in part order
// (n_parts > 1 needs E <= kTopkMaxSplitE).
constexpr int kTopkMaxSplitE = 256;
cudaError_t launch_topk_rank(int mode, const float* logits, int n_parts, const float* bias, int32_t* topk_ids,
                             float* gates,
                             int32_t* local_rank, int32_t* group_counts, uint32_t* status, int T, int E, int k,
                             cudaStream_t s);
// The scatter step folded into the one-group kernel below (x == nullptr: not folded): the
// arguments launch_scatter_quant takes beyond the routing results.
struct FoldedScatter {
  const uint16_t* x;
  int32_t* slot_pos;
  int32_t* perm;
  uint8_t* xq;
  uint8_t* xsf;
  int H;
  uint32_t* zero;
  int n_zero;
};
// At most this many (token, 256-channel slice) items for the fold: the block's 32 warps take
// them one by one, which beats a separate launch only while they are few.
constexpr int kFoldScatterMaxItems = 128;
// T <= 32: launch_topk_rank followed by launch_dispatch_scan, as one single-block kernel; with
// fs.x set (T * slices <= kFoldScatterMaxItems), also launch_scatter_quant's work.
cudaError_t launch_topk_scan_one_group(int mode, const float* logits, int n_parts, const float* bias,
                                      int32_t* topk_ids, float* gates, int32_t* local_rank, int32_t* group_counts,
                                      uint32_t* status, int32_t* group_base, int32_t* counts, int32_t* offsets,
                                      int32_t* mtile_start, int32_t* ptile_start, int4* tile_info,
                                      int4* ptile_info, int T, int E, int k, int shared, int bm, FoldedScatter fs,
                                      cudaStream_t s);
// counts, offsets, mtile_start (bm-row tiles), ptile_start (pairs of 128-row tiles) (n + 1
// entries), the row-tile tables (see GemmArgs) and group_base[g][e] = rows of expert e in token
// groups < g (relative to offsets[e]).
cudaError_t launch_dispatch_scan(const int32_t* group_counts, int32_t* counts, int32_t* offsets,
                                 int32_t* group_base, int32_t* mtile_start, int32_t* ptile_start, int4* tile_info,
                                 int4* ptile_info, int T, int E, int k, int shared, int bm, cudaStream_t s);
// Writes slot_pos/perm and (if x != nullptr) the dispatched E4M3 rows + scale atoms (bm-row tiles);
// also zeroes zero[0 .. n_zero) (if given) for the kernels that follow.
cudaError_t launch_scatter_quant(const uint16_t* x, const int32_t* topk_ids, const int32_t* local_rank,
                                 const int32_t* group_base, const int32_t* offsets, const int32_t* mtile_start,
                                 int32_t* slot_pos, int32_t* perm, uint8_t* xq, uint8_t* xsf, int T, int H, int E,
                                 int k, int shared, int bm, cudaStream_t s, uint32_t* zero = nullptr,
                                 int n_zero = 0);
// Token-order quantisation (debug entry point).
cudaError_t launch_quant_tokens(const uint16_t* x, uint8_t* xq, float* xs, int T, int H, cudaStream_t s);
// Auxiliary-loss-free balancing step from the routed experts' loads.
cudaError_t launch_update_bias(float* bias, const int32_t* counts, int T, int k, int E, float gamma,
                               cudaStream_t s);
cudaError_t launch_combine(const uint16_t* y, const int32_t* slot_pos, const float* gates, uint16_t* out, int T,
                           int H, int k, int shared, cudaStream_t s);

}  // namespace moe
