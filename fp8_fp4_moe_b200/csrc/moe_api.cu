// Host side of libmoe_b200.so: plans, workspace layout, argument checks, TMA
// descriptors and the launch sequence of the layer forward.
//
// Launch sequence of moe_forward (one stream, no host synchronisation):
//   router_logits -> topk_rank -> dispatch_scan -> scatter_quant
//   -> grouped GEMM linear1 (+SwiGLU +E4M3 requant) -> grouped GEMM linear2 -> combine
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/moe_b200.h"
#include "kernels.h"

using namespace moe;

struct moe_plan_s {
  int T, H, I, E, k, shared, n;
  long long R, rows;
  int G;
  // options
  int max_sms = 0;
  uint64_t timeout_ns = 2000000000ull;
  int inject_fault = 0;
  int static_weights = 0;
  int router_tc = 1;
  int swap_rows = 0;
  int pair_mode = 1;                // MOE_OPT_PAIR_TILES
  int fused = 0;                    // MOE_OPT_FUSED
  int dep_launch = 2;               // MOE_OPT_DEPENDENT_LAUNCH (2 = automatic)
  int l2_tile_rows = 0;             // MOE_OPT_L2_TILE_ROWS
  int chain = 0;                    // MOE_OPT_CHAIN
  int tile_rows = 0;                // MOE_OPT_TILE_ROWS
  int zero_pad = 0;                 // MOE_OPT_ZERO_PAD
  int router_splits = 1;            // K splits of the tensor-core router (partial logit arrays)
  // workspace layout
  size_t region_off[MOE_REGION_COUNT_];
  size_t region_len[MOE_REGION_COUNT_];
  size_t off_logits, off_rank, off_gcounts, off_gbase, off_mtile, off_ptile, off_w1sf, off_w2sf, off_whi, off_wlo;
  size_t off_tinfo, off_ptinfo;     // row-tile tables of the grouped GEMMs (mt_cap int4 each)
  size_t off_dep;                   // per-expert linear1 tile counters of the chained GEMM kernel
  size_t off_gridbar;               // grid barrier words of the fused forward
  size_t off_zeros;                 // kGemmZeroBytes of zeros (A-region padding source)
  size_t off_counters;              // readiness counters of the fused forward (2 + n words)
  int fused_ctas_last = 0;          // CTAs of the last fused launch with stamps (0: none)
  int splitk_parts = 1;             // K parts of the fused forward's split-K router (few tokens)
  long long mt_cap;                 // bound on row tiles: ceil(rows/32) + n (any row-tile height)
  size_t total;
  // bound state
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  int device = -1;
  int num_sms = 0;
  alignas(64) AMaps amA1, amA2;
  alignas(64) CUtensorMap tmB1, tmB2, tmB2d, tmX, tmWhi, tmWlo;   // tmB2d: 224-row boxes
  alignas(64) CUtensorMap tmB1g;    // W1 as [experts x {gate, up}][I][H]: a tile's two halves in one box
  alignas(64) CUtensorMap tmB2p, tmSfa1, tmSfa2, tmSfb1, tmSfb2;   // CTA-pair GEMM operands
  const void* x_cached = nullptr;        // tmX encodes this x pointer
  const void* wr_prepared = nullptr;     // W_router the hi/lo split was made from
  const void* w1_cached = nullptr;
  const void* w2_cached = nullptr;
  const void* w1s_prepared = nullptr;   // weight scales the prepared units were built from
  const void* w2s_prepared = nullptr;
  int w2_tile_rows = 0;                // linear2 tile height the W2 scale units were laid out for
  // MOE_OPT_GRAPH: recorded launch sequences, keyed by the forward's pointers
  int use_graph = 0;
  struct GraphEntry {
    const void* key[8];
    cudaGraphExec_t exec;
  };
  std::vector<GraphEntry> graphs;
  cudaStream_t cap_stream = nullptr;
  // per-phase timing (MOE_OPT_PHASE_EVENTS)
  int phase_events = 0;
  bool events_ready = false;
  bool events_recorded = false;
  cudaEvent_t ev[MOE_PHASE_COUNT_ + 1];
};

namespace moe {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

int get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? MOE_OK : MOE_ERR_CUDA;
}
}  // namespace

int encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  if (get_encode() != MOE_OK) return MOE_ERR_CUDA;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

int encode_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t outer2, uint64_t row_bytes, uint64_t slab_bytes, uint32_t box_inner, uint32_t box_outer,
              uint32_t box_outer2) {
  if (get_encode() != MOE_OK) return MOE_ERR_CUDA;
  cuuint64_t dims[3] = {inner, outer, outer2};
  cuuint64_t strides[2] = {row_bytes, slab_bytes};
  cuuint32_t box[3] = {box_inner, box_outer, box_outer2};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe

namespace {

bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <class T>
T* at(moe_plan_t p, size_t off) {
  return reinterpret_cast<T*>(p->ws + off);
}
template <class T>
T* region(moe_plan_t p, int r) {
  return at<T>(p, p->region_off[r]);
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int check_bound(moe_plan_t p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!p->ws) return MOE_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev != p->device) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Rows per GEMM row tile: 32 (small-tile layout: 32-row A regions, 6 stages) when the routed
// experts average at most 32 rows -- decode, where each expert's weights stream past a handful
// of rows and the pipeline depth decides the bandwidth -- unless transposed tiles or forced CTA
// pairs are asked for; 128 otherwise.
// Experts average at most 32 routed rows (decode-shaped: every row tile is mostly padding).
bool decode_shaped(moe_plan_t p) { return (long long)p->T * p->k <= (long long)kGemmBMSmall * p->E; }

int plan_bm(moe_plan_t p) {
  if (p->tile_rows != 0) return p->tile_rows;
  if (p->swap_rows != 0 || p->pair_mode == 2) return kGemmBM;
  return decode_shaped(p) && p->T <= 32 ? kGemmBMSmall : kGemmBM;
}

// linear1 and linear2 as one cooperative launch (MOE_OPT_CHAIN; 32-row tiles, at most 16 tokens)
bool use_chain(moe_plan_t p) { return p->chain && plan_bm(p) == kGemmBMSmall && p->T <= 16; }

// Programmatic dependent launches: automatic for at most 64 tokens, where each kernel is short
// and launch latency and the GEMMs' early weight requests matter; with more tokens the GEMM's
// early-resident CTAs take the registers the scatter's blocks need, and the forward measured
// 1.5-2 % slower (T = 8192 and 32768).
bool plan_dep_launch(moe_plan_t p) {
  if (p->dep_launch != 2) return p->dep_launch != 0;
  return p->T <= 64;
}

// Zero padding of the A rows a 128-row tile leaves empty: automatic for decode-shaped layers with
// more than 32 tokens, where the MMAs of mostly-empty tiles and the weight stream together hold
// the part at its power limit (zero operands lower the power drawn and so raise the clock);
// measured slower where tiles are mostly full (the extra copies cost more than they save).
bool plan_zero_pad(moe_plan_t p) {
  if (p->zero_pad == 1) return true;
  if (p->zero_pad == 2) return false;
  return plan_bm(p) == kGemmBM && decode_shaped(p);
}

// CTA-pair GEMMs (M = 256 per pair, each CTA loading half of the weight tile) when the experts
// average at least 1024 rows, or when forced (128-row tiles only).  Measured in one process
// against single CTAs: T = 32768 (1024 rows per expert) 1.7 % faster; the Zipf-skewed T = 8192
// layer (256 on average, most experts far fewer) 7 % slower.
bool use_pairs(moe_plan_t p) {
  if (p->pair_mode == 0 || gemm_pair_max_clusters() < 1 || plan_bm(p) != kGemmBM) return false;
  return p->pair_mode == 2 || (long long)p->T * p->k >= 1024ll * p->E;
}

// linear2 weight rows per tile.  224 (double-buffered accumulator) needs H % 224 == 0 and the
// single-CTA kernel; automatic only for few tokens (T <= 16), where 224-row tiles spread the
// experts' weight tiles more evenly over the SMs (DSV3 T = 1: 288 tiles instead of 252) --
// with many tiles per SM the 14 % more tiles cost more than the overlap saves.
int linear2_bn(moe_plan_t p) {
  if (use_pairs(p) || p->H % kGemmBN2Double != 0 || p->l2_tile_rows == kGemmBN) return kGemmBN;
  if (p->l2_tile_rows == kGemmBN2Double) return kGemmBN2Double;
  return p->T <= 16 ? kGemmBN2Double : kGemmBN;
}

GemmArgs gemm_args(moe_plan_t p, int mode) {
  GemmArgs a{};
  a.bm = plan_bm(p);
  a.n_experts = p->n;
  a.rows_total = (int)p->rows;
  a.counts = region<int32_t>(p, MOE_REGION_COUNTS);
  a.offsets = region<int32_t>(p, MOE_REGION_OFFSETS);
  a.mtile_start = at<int32_t>(p, p->off_mtile);
  a.ptile_start = at<int32_t>(p, p->off_ptile);
  a.tile_info = at<int4>(p, p->off_tinfo);
  a.ptile_info = at<int4>(p, p->off_ptinfo);
  a.status = region<uint32_t>(p, MOE_REGION_STATUS);
  a.timeout_ns = p->timeout_ns;
  a.swap_rows = p->swap_rows;
  a.zeros = plan_zero_pad(p) ? at<uint8_t>(p, p->off_zeros) : nullptr;
  if (mode == 1) {
    a.K = p->H;
    a.N = p->I;
    a.rows_b = 2 * p->I;
    a.n_tiles_n = p->I / 128;
    a.bn = kGemmBN;
    a.sfa = region<uint8_t>(p, MOE_REGION_XSF);
    a.sfb = at<uint8_t>(p, p->off_w1sf);
    a.hq = region<uint8_t>(p, MOE_REGION_HQ);
    a.hsf = region<uint32_t>(p, MOE_REGION_HSF);
    a.inject_fault = p->inject_fault;
  } else {
    a.K = p->I;
    a.N = p->H;
    a.rows_b = p->H;
    a.bn = linear2_bn(p);
    a.n_tiles_n = (p->H + a.bn - 1) / a.bn;
    a.sfa = region<uint8_t>(p, MOE_REGION_HSF);
    a.sfb = at<uint8_t>(p, p->off_w2sf);
    a.y = region<uint16_t>(p, MOE_REGION_Y);
    a.inject_fault = 0;
  }
  return a;
}

int gemm_grid(moe_plan_t p, int n_tiles_n) {
  const int bm = plan_bm(p);
  const long long mt_bound = (p->rows + bm - 1) / bm + p->n;
  long long tiles = mt_bound * n_tiles_n;
  int sms = p->num_sms;
  if (p->max_sms > 0 && p->max_sms < sms) sms = p->max_sms;
  return (int)(tiles < sms ? tiles : sms);
}

int pair_grid(moe_plan_t p, int n_tiles_n) {
  const long long pt_bound = (p->rows + 2 * kGemmBM - 1) / (2 * kGemmBM) + p->n;
  long long tiles = pt_bound * n_tiles_n;
  int pairs = gemm_pair_max_clusters();
  if (p->max_sms > 0 && p->max_sms / 2 < pairs) pairs = p->max_sms / 2 > 0 ? p->max_sms / 2 : 1;
  return (int)(tiles < pairs ? tiles : pairs);
}

// Record the event that closes phase `i` (event 0 opens the forward).
void mark(moe_plan_t p, int i, cudaStream_t s) {
  if (p->phase_events && p->events_ready) cudaEventRecord(p->ev[i], s);
}

// Tensor-core router from 64 tokens on, for a multiple of 16 experts; CUDA cores otherwise.  (At
// 128 and 192 tokens of the DeepSeek-V3 shape the CUDA-core router took 1.35 ms of a 2.65 ms
// forward; the tensor-core one a few microseconds.  At 32 and 64 tokens the two are even.)
bool use_tc_router(moe_plan_t p) { return p->router_tc && p->T >= 64 && p->E >= 16 && p->E % 16 == 0; }

// logits [T][E] fp32 into the workspace
int run_router(moe_plan_t p, const uint16_t* x, const float* W_router, cudaStream_t s) {
  if (!use_tc_router(p))
    return cuda_rc(launch_router_logits(x, W_router, at<float>(p, p->off_logits), p->T, p->H, p->E, s));
  if (!p->static_weights || W_router != p->wr_prepared) {
    if (launch_split_router_weights(W_router, at<uint16_t>(p, p->off_whi), at<uint16_t>(p, p->off_wlo),
                                    (long)p->E * p->H, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    p->wr_prepared = W_router;
  }
  if (x != p->x_cached) {
    int rc = encode_2d(&p->tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, p->H, p->T, 2ull * p->H, 64, 128);
    if (rc != MOE_OK) return rc;
    p->x_cached = x;
  }
  RouterArgs ra{p->T, p->H, p->E, p->router_splits, at<float>(p, p->off_logits),
                region<uint32_t>(p, MOE_REGION_STATUS), p->timeout_ns};
  return cuda_rc(launch_router_tc(p->tmX, p->tmWhi, p->tmWlo, ra, s));
}

// K parts of the fused forward's split-K router: a warp per (expert, part) computes all T tokens,
// so with few tokens every warp of the grid streams a slice of W_router.  0 = not used (more
// than kSplitKMaxT tokens, or E beyond what the top-k adds up in parts).  Enough parts for
// about one item per warp of a 148-SM grid, each at most kSplitKMaxChunks chunks of 256 channels.
int splitk_parts(int T, int H, int E) {
  if (T > kSplitKMaxT || E > kTopkMaxSplitE || E % 4 != 0) return 0;
  const int C = (H + 255) / 256;
  int s = (148 * (kGemmThreads / 32) + E - 1) / E;
  const int s_min = (C + kSplitKMaxChunks - 1) / kSplitKMaxChunks;
  if (s < s_min) s = s_min;
  if (s > C) s = C;
  return s;
}

// partial logit arrays the router leaves for top-k
int logit_parts(moe_plan_t p) { return use_tc_router(p) ? p->router_splits : 1; }

// routing + dispatch + quantisation into the workspace
int run_front(moe_plan_t p, const uint16_t* x, const float* W_router, const float* bias, cudaStream_t s) {
  int32_t* ids = region<int32_t>(p, MOE_REGION_TOPK_IDS);
  float* gates = region<float>(p, MOE_REGION_GATES);
  cudaError_t e;
  mark(p, 0, s);
  int rc = run_router(p, x, W_router, s);
  if (rc != MOE_OK) return rc;
  mark(p, 1 + MOE_PHASE_ROUTER, s);
  // every later kernel of the forward may start before its predecessor ends (it waits for it
  // on the device); not between the per-phase events
  set_dependent_launch(plan_dep_launch(p) && !p->phase_events);
  // a few tokens: the scatter folds into the one-group kernel (one launch less on the path), while
  // each of the block's 32 warps has at most one (token, slice) item (interleaved on one box:
  // T = 1 78.0 -> 76.9 us; T = 4, 112 items, 193 -> 201 us, so not there)
  const bool fold = p->T <= 32 && (long)p->T * ((p->H + 255) / 256) <= 32;
  if (p->T <= 32) {
    // one token group: top-k, ranks and the scans in one block (reported under top-k)
    FoldedScatter fs{};
    if (fold)
      fs = FoldedScatter{x, region<int32_t>(p, MOE_REGION_SLOT_POS), region<int32_t>(p, MOE_REGION_PERM),
                         region<uint8_t>(p, MOE_REGION_XQ), region<uint8_t>(p, MOE_REGION_XSF), p->H,
                         use_chain(p) ? at<uint32_t>(p, p->off_dep) : nullptr, p->n};
    if ((e = launch_topk_scan_one_group(0, at<float>(p, p->off_logits), logit_parts(p), bias, ids, gates,
                                        at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gcounts),
                                        region<uint32_t>(p, MOE_REGION_STATUS), at<int32_t>(p, p->off_gbase),
                                        region<int32_t>(p, MOE_REGION_COUNTS), region<int32_t>(p, MOE_REGION_OFFSETS),
                                        at<int32_t>(p, p->off_mtile), at<int32_t>(p, p->off_ptile),
                                        at<int4>(p, p->off_tinfo), at<int4>(p, p->off_ptinfo), p->T, p->E, p->k,
                                        p->shared, plan_bm(p), fs, s)) != cudaSuccess)
      return cuda_rc(e);
    mark(p, 1 + MOE_PHASE_TOPK, s);
  } else {
    if ((e = launch_topk_rank(0, at<float>(p, p->off_logits), logit_parts(p), bias, ids, gates,
                              at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gcounts),
                              region<uint32_t>(p, MOE_REGION_STATUS), p->T, p->E, p->k, s)) != cudaSuccess)
      return cuda_rc(e);
    mark(p, 1 + MOE_PHASE_TOPK, s);
    if ((e = launch_dispatch_scan(at<int32_t>(p, p->off_gcounts), region<int32_t>(p, MOE_REGION_COUNTS),
                                  region<int32_t>(p, MOE_REGION_OFFSETS), at<int32_t>(p, p->off_gbase),
                                  at<int32_t>(p, p->off_mtile), at<int32_t>(p, p->off_ptile),
                                  at<int4>(p, p->off_tinfo), at<int4>(p, p->off_ptinfo), p->T, p->E, p->k,
                                  p->shared, plan_bm(p), s)) != cudaSuccess)
      return cuda_rc(e);
  }
  mark(p, 1 + MOE_PHASE_SCAN, s);
  if (fold) {
    mark(p, 1 + MOE_PHASE_SCATTER_QUANT, s);
    return MOE_OK;
  }
  e = launch_scatter_quant(x, ids, at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gbase),
                           region<int32_t>(p, MOE_REGION_OFFSETS), at<int32_t>(p, p->off_mtile),
                           region<int32_t>(p, MOE_REGION_SLOT_POS), region<int32_t>(p, MOE_REGION_PERM),
                           region<uint8_t>(p, MOE_REGION_XQ), region<uint8_t>(p, MOE_REGION_XSF), p->T, p->H,
                           p->E, p->k, p->shared, plan_bm(p), s,
                           use_chain(p) ? at<uint32_t>(p, p->off_dep) : nullptr, p->n);
  mark(p, 1 + MOE_PHASE_SCATTER_QUANT, s);
  return cuda_rc(e);
}

// Weight scale factors -> the tiled units the GEMMs bulk-load (both weights).
int prepare_weights(moe_plan_t p, const uint8_t* W1_scales, const uint8_t* W2_scales, cudaStream_t s) {
  cudaError_t e = launch_tile_weight_scales(W1_scales, at<uint8_t>(p, p->off_w1sf), p->n, 2 * p->I, p->H,
                                            p->I / 128, 1, p->I, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int bn2 = linear2_bn(p);
  e = launch_tile_weight_scales(W2_scales, at<uint8_t>(p, p->off_w2sf), p->n, p->H, p->I, (p->H + bn2 - 1) / bn2, 2,
                                p->H, s, bn2);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  p->w1s_prepared = W1_scales;
  p->w2s_prepared = W2_scales;
  p->w2_tile_rows = bn2;
  return MOE_OK;
}

// The prepared weight scale units are stale (new pointers, not promised static, or laid out
// for another linear2 tile height).
bool weights_need_prepare(moe_plan_t p, const uint8_t* W1_scales, const uint8_t* W2_scales) {
  return !p->static_weights || W1_scales != p->w1s_prepared || W2_scales != p->w2s_prepared ||
         p->w2_tile_rows != linear2_bn(p);
}

// MOE_OPT_FUSED: weight preparation when needed, then every step in one cooperative launch.
int launch_fused(moe_plan_t p, const uint16_t* x, const float* W_router, const float* bias,
                 const uint8_t* W1_scales, const uint8_t* W2_scales, void* out, cudaStream_t s) {
  const bool tc = use_tc_router(p);
  mark(p, 0, s);
  if (tc) {
    if (!p->static_weights || W_router != p->wr_prepared) {
      if (launch_split_router_weights(W_router, at<uint16_t>(p, p->off_whi), at<uint16_t>(p, p->off_wlo),
                                      (long)p->E * p->H, s) != cudaSuccess)
        return MOE_ERR_CUDA;
      p->wr_prepared = W_router;
    }
    if (x != p->x_cached) {
      int rc = encode_2d(&p->tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, p->H, p->T, 2ull * p->H, 64, 128);
      if (rc != MOE_OK) return rc;
      p->x_cached = x;
    }
  }
  if (weights_need_prepare(p, W1_scales, W2_scales)) {
    int rc = prepare_weights(p, W1_scales, W2_scales, s);
    if (rc != MOE_OK) return rc;
  }
  FusedArgs a{};
  a.T = p->T; a.H = p->H; a.E = p->E; a.k = p->k; a.shared = p->shared;
  a.bm = plan_bm(p);
  a.router_kind = tc ? kRouterTensor
                  : p->splitk_parts > 0 ? kRouterSplitK
                  : (long long)p->T * p->E <= 4096 ? kRouterSplitBlock : p->E <= 32 ? kRouterWarp8 : kRouterWarp2;
  a.router_parts = tc ? p->router_splits : p->splitk_parts > 0 ? p->splitk_parts : 1;
  a.x = x;
  a.W_router = W_router;
  a.bias = bias;
  a.logits = at<float>(p, p->off_logits);
  a.topk_ids = region<int32_t>(p, MOE_REGION_TOPK_IDS);
  a.gates = region<float>(p, MOE_REGION_GATES);
  a.local_rank = at<int32_t>(p, p->off_rank);
  a.group_counts = at<int32_t>(p, p->off_gcounts);
  a.group_base = at<int32_t>(p, p->off_gbase);
  a.counts = region<int32_t>(p, MOE_REGION_COUNTS);
  a.offsets = region<int32_t>(p, MOE_REGION_OFFSETS);
  a.mtile_start = at<int32_t>(p, p->off_mtile);
  a.ptile_start = at<int32_t>(p, p->off_ptile);
  a.tile_info = at<int4>(p, p->off_tinfo);
  a.ptile_info = at<int4>(p, p->off_ptinfo);
  a.slot_pos = region<int32_t>(p, MOE_REGION_SLOT_POS);
  a.perm = region<int32_t>(p, MOE_REGION_PERM);
  a.xq = region<uint8_t>(p, MOE_REGION_XQ);
  a.xsf = region<uint8_t>(p, MOE_REGION_XSF);
  a.y = region<uint16_t>(p, MOE_REGION_Y);
  a.out = static_cast<uint16_t*>(out);
  a.status = region<uint32_t>(p, MOE_REGION_STATUS);
  a.gridbar = at<uint32_t>(p, p->off_gridbar);
  a.counters = at<uint32_t>(p, p->off_counters);
  a.stamps = (p->phase_events && p->events_ready) ? region<unsigned long long>(p, MOE_REGION_STAMPS) : nullptr;
  a.timeout_ns = p->timeout_ns;
  a.ra = RouterArgs{p->T, p->H, p->E, a.router_parts, a.logits, a.status, p->timeout_ns};
  a.g1 = gemm_args(p, 1);
  a.g2 = gemm_args(p, 2);
  int ctas = fused_max_ctas();
  if (p->max_sms > 0 && p->max_sms < ctas) ctas = p->max_sms;
  if (ctas > kStampMaxCtas) ctas = kStampMaxCtas;
  p->fused_ctas_last = a.stamps != nullptr ? ctas : 0;
  // a launch that ran out of time may have left arrivals behind
  if (cudaMemsetAsync(a.gridbar, 0, 8, s) != cudaSuccess) return MOE_ERR_CUDA;
  const CUtensorMap& b2 = a.g2.bn == kGemmBN2Double ? p->tmB2d : p->tmB2;
  if (launch_fused_forward(p->amA1, p->amA2, p->tmB1g, b2, p->tmX, p->tmWhi, p->tmWlo, a, ctas,
                           plan_bm(p) == kGemmBMSmall, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // one kernel: its whole time is reported under the first phase
  for (int i = 1; i <= MOE_PHASE_COUNT_; ++i) mark(p, i, s);
  if (p->phase_events && p->events_ready) p->events_recorded = true;
  return MOE_OK;
}

// The forward's launch sequence on stream s (TMA maps already current).
// Plain stream order again when the forward's launch sequence ends, on every return path.
struct DependentLaunchOff {
  ~DependentLaunchOff() { set_dependent_launch(false); }
};

int launch_forward(moe_plan_t p, const uint16_t* x, const float* W_router, const float* bias,
                   const uint8_t* W1_scales, const uint8_t* W2_scales, void* out, cudaStream_t s) {
  if (p->fused) return launch_fused(p, x, W_router, bias, W1_scales, W2_scales, out, s);
  DependentLaunchOff restore;
  int rc = run_front(p, x, W_router, bias, s);
  if (rc != MOE_OK) return rc;
  if (weights_need_prepare(p, W1_scales, W2_scales)) {
    if ((rc = prepare_weights(p, W1_scales, W2_scales, s)) != MOE_OK) return rc;
  }
  mark(p, 1 + MOE_PHASE_PREPARE, s);
  GemmArgs a1 = gemm_args(p, 1);
  GemmArgs a2 = gemm_args(p, 2);
  if (use_pairs(p)) {
    if (launch_gemm_pair_linear1(p->amA1, p->tmB1, p->tmSfa1, p->tmSfb1, a1, pair_grid(p, a1.n_tiles_n), s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    mark(p, 1 + MOE_PHASE_LINEAR1, s);
    if (launch_gemm_pair_linear2(p->amA2, p->tmB2p, p->tmSfa2, p->tmSfb2, a2, pair_grid(p, a2.n_tiles_n), s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    mark(p, 1 + MOE_PHASE_LINEAR2, s);
  } else {
    const bool small_tiles = plan_bm(p) == kGemmBMSmall;
    const CUtensorMap& b2 = a2.bn == kGemmBN2Double ? p->tmB2d : p->tmB2;
    if (use_chain(p)) {
      // one cooperative launch: linear2 tiles start as soon as their expert's linear1 tiles are
      // stored (per-expert counters, zeroed by the scatter kernel); reported under linear1
      uint32_t* dep = at<uint32_t>(p, p->off_dep);
      a1.dep_signal = dep;
      a2.dep_wait = dep;
      a2.dep_per_mtile = a1.n_tiles_n;
      if (launch_gemm_chain(p->amA1, p->amA2, p->tmB1g, b2, a1, a2, gemm_grid(p, a1.n_tiles_n), s) != cudaSuccess)
        return MOE_ERR_CUDA;
      mark(p, 1 + MOE_PHASE_LINEAR1, s);
      mark(p, 1 + MOE_PHASE_LINEAR2, s);
    } else {
      if (launch_gemm_linear1(p->amA1, p->tmB1g, a1, gemm_grid(p, a1.n_tiles_n), s, small_tiles) != cudaSuccess)
        return MOE_ERR_CUDA;
      mark(p, 1 + MOE_PHASE_LINEAR1, s);
      if (launch_gemm_linear2(p->amA2, b2, a2, gemm_grid(p, a2.n_tiles_n), s, small_tiles) != cudaSuccess)
        return MOE_ERR_CUDA;
      mark(p, 1 + MOE_PHASE_LINEAR2, s);
    }
  }
  cudaError_t e = launch_combine(region<uint16_t>(p, MOE_REGION_Y), region<int32_t>(p, MOE_REGION_SLOT_POS),
                                 region<float>(p, MOE_REGION_GATES), static_cast<uint16_t*>(out), p->T, p->H, p->k,
                                 p->shared, s);
  mark(p, 1 + MOE_PHASE_COMBINE, s);
  if (p->phase_events && p->events_ready) p->events_recorded = true;
  return cuda_rc(e);
}

void drop_graphs(moe_plan_t p) {
  for (auto& g : p->graphs) cudaGraphExecDestroy(g.exec);
  p->graphs.clear();
}

// MOE_OPT_GRAPH: replay the launch sequence recorded for this exact argument set,
// recording it (on a private stream) the first time.
int forward_graph(moe_plan_t p, const void* x, const float* W_router, const float* bias, const uint8_t* W1,
                  const uint8_t* W1_scales, const uint8_t* W2, const uint8_t* W2_scales, void* out, cudaStream_t s) {
  const void* key[8] = {x, W_router, bias, W1, W1_scales, W2, W2_scales, out};
  for (auto& g : p->graphs)
    if (std::memcmp(g.key, key, sizeof(key)) == 0) return cuda_rc(cudaGraphLaunch(g.exec, s));
  if (!p->cap_stream && cudaStreamCreateWithFlags(&p->cap_stream, cudaStreamNonBlocking) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamBeginCapture(p->cap_stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return MOE_ERR_CUDA;
  int rc = launch_forward(p, static_cast<const uint16_t*>(x), W_router, bias, W1_scales, W2_scales, out,
                          p->cap_stream);
  cudaGraph_t graph = nullptr;
  cudaError_t e = cudaStreamEndCapture(p->cap_stream, &graph);
  if (rc != MOE_OK || e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return rc != MOE_OK ? rc : MOE_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (p->graphs.size() >= 4) {
    cudaGraphExecDestroy(p->graphs.front().exec);
    p->graphs.erase(p->graphs.begin());
  }
  moe_plan_s::GraphEntry ge;
  std::memcpy(ge.key, key, sizeof(key));
  ge.exec = exec;
  p->graphs.push_back(ge);
  return cuda_rc(cudaGraphLaunch(exec, s));
}

}  // namespace

extern "C" {

int moe_prepare_weights(moe_plan_t p, const uint8_t* W1_scales, const uint8_t* W2_scales, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(W1_scales, 4) || !aligned(W2_scales, 4)) return MOE_ERR_INVALID_ARG;
  return prepare_weights(p, W1_scales, W2_scales, static_cast<cudaStream_t>(stream));
}

int moe_plan(int T, int H, int I, int E, int k, int shared, moe_plan_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (T < 1 || H < 128 || I < 128 || H % 128 || I % 128 || E < 1 || E > 1024 || k < 1 || k > 16 || k > E ||
      (shared != 0 && shared != 1) || E + shared > 1024)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const long long R = (long long)T * k;
  const long long rows = R + (long long)shared * T;
  // 32-bit row indices and TMA coordinates
  if (rows * (long long)(H > I ? H : I) > (1ll << 40) || rows >= (1ll << 31) ||
      (long long)(E + shared) * 2 * I >= (1ll << 31) || (long long)(E + shared) * H >= (1ll << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_plan_t p = new (std::nothrow) moe_plan_s();
  if (!p) return MOE_ERR_INVALID_ARG;
  p->T = T; p->H = H; p->I = I; p->E = E; p->k = k; p->shared = shared; p->n = E + shared;
  p->R = R; p->rows = rows; p->G = (T + 31) / 32;
  size_t off = 0;
  auto add = [&](size_t bytes) {
    size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    return o;
  };
  auto reg = [&](int r, size_t bytes) {
    p->region_off[r] = add(bytes);
    p->region_len[r] = bytes;
  };
  const size_t Tk = (size_t)T * k;
  reg(MOE_REGION_STATUS, 16);
  reg(MOE_REGION_TOPK_IDS, Tk * 4);
  reg(MOE_REGION_GATES, Tk * 4);
  reg(MOE_REGION_COUNTS, (size_t)p->n * 4);
  reg(MOE_REGION_OFFSETS, (size_t)(p->n + 1) * 4);
  reg(MOE_REGION_PERM, (size_t)R * 4);
  reg(MOE_REGION_SLOT_POS, Tk * 4);
  reg(MOE_REGION_XQ, (size_t)rows * H);
  p->mt_cap = (rows + kGemmBMSmall - 1) / kGemmBMSmall + p->n;
  reg(MOE_REGION_XSF, (size_t)p->mt_cap * (H / 128) * 512);
  reg(MOE_REGION_HQ, (size_t)rows * I);
  reg(MOE_REGION_HSF, (size_t)p->mt_cap * (I / 128) * 512);
  reg(MOE_REGION_Y, (size_t)rows * H * 2);
  reg(MOE_REGION_STAMPS, (size_t)kStampCount * kStampMaxCtas * 8);
  // the tensor-core router's split count depends on the shape only, so results do not
  // depend on the device or on options
  p->router_splits = (E >= 16 && E % 16 == 0) ? router_tc_splits(T, H, E) : 1;
  p->splitk_parts = splitk_parts(T, H, E);
  const int parts = p->router_splits > p->splitk_parts ? p->router_splits : p->splitk_parts;
  p->off_logits = add((size_t)parts * T * E * 4);
  p->off_rank = add(Tk * 4);
  p->off_gcounts = add((size_t)p->G * E * 4);
  p->off_gbase = add((size_t)p->G * E * 4);
  p->off_mtile = add((size_t)(p->n + 1) * 4);
  p->off_ptile = add((size_t)(p->n + 1) * 4);
  p->off_tinfo = add((size_t)p->mt_cap * 16);
  p->off_ptinfo = add((size_t)p->mt_cap * 16);
  p->off_dep = add((size_t)p->n * 4);
  p->off_gridbar = add(8);
  p->off_zeros = add(kGemmZeroBytes);
  p->off_counters = add((size_t)(2 + p->n) * 4);
  p->off_w1sf = add((size_t)p->n * (I / 128) * (H / 128) * 1024);
  // linear2 weight scale units for the narrower of the two tile heights (more tiles)
  p->off_w2sf = add((size_t)p->n * ((H + kGemmBN2Double - 1) / kGemmBN2Double) * (I / 128) * 1024);
  p->off_whi = add((size_t)E * H * 2);
  p->off_wlo = add((size_t)E * H * 2);
  p->total = off;
  *out = p;
  return MOE_OK;
}

int moe_plan_set_option(moe_plan_t p, int key, long long value) {
  if (!p) return MOE_ERR_INVALID_ARG;
  drop_graphs(p);                       // recorded sequences depend on the options
  switch (key) {
    case MOE_OPT_GRAPH:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->use_graph = (int)value;
      return MOE_OK;
    case MOE_OPT_MAX_SMS:
      if (value < 0) return MOE_ERR_INVALID_ARG;
      p->max_sms = (int)value;
      return MOE_OK;
    case MOE_OPT_TIMEOUT_NS:
      if (value <= 0) return MOE_ERR_INVALID_ARG;
      p->timeout_ns = (uint64_t)value;
      return MOE_OK;
    case MOE_OPT_INJECT_FAULT:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->inject_fault = (int)value;
      return MOE_OK;
    case MOE_OPT_STATIC_WEIGHTS:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->static_weights = (int)value;
      return MOE_OK;
    case MOE_OPT_ROUTER_TC:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->router_tc = (int)value;
      return MOE_OK;
    case MOE_OPT_PHASE_EVENTS:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->phase_events = (int)value;
      return MOE_OK;
    case MOE_OPT_FUSED:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      if (value == 1 && p->ws && fused_max_ctas() < 1) return MOE_ERR_UNSUPPORTED_SHAPE;
      p->fused = (int)value;
      return MOE_OK;
    case MOE_OPT_CHAIN:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      p->chain = (int)value;
      return MOE_OK;
    case MOE_OPT_L2_TILE_ROWS:
      if (value != 0 && value != kGemmBN && value != kGemmBN2Double) return MOE_ERR_INVALID_ARG;
      if (value == kGemmBN2Double && p->H % kGemmBN2Double != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
      p->l2_tile_rows = (int)value;
      return MOE_OK;
    case MOE_OPT_DEPENDENT_LAUNCH:
      if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
      p->dep_launch = (int)value;
      return MOE_OK;
    case MOE_OPT_PAIR_TILES:
      if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
      if (value == 2 && p->tile_rows == kGemmBMSmall) return MOE_ERR_INVALID_ARG;
      p->pair_mode = (int)value;
      return MOE_OK;
    case MOE_OPT_SWAP_ROWS:
      if (value != 0 && value != 32 && value != 64) return MOE_ERR_INVALID_ARG;
      if (value != 0 && p->tile_rows == kGemmBMSmall) return MOE_ERR_INVALID_ARG;
      p->swap_rows = (int)value;
      return MOE_OK;
    case MOE_OPT_ZERO_PAD:
      if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
      p->zero_pad = (int)value;
      return MOE_OK;
    case MOE_OPT_TILE_ROWS:
      if (value != 0 && value != kGemmBMSmall && value != kGemmBM) return MOE_ERR_INVALID_ARG;
      if (value == kGemmBMSmall && (p->swap_rows != 0 || p->pair_mode == 2)) return MOE_ERR_INVALID_ARG;
      p->tile_rows = (int)value;
      return MOE_OK;
    default:
      return MOE_ERR_INVALID_ARG;
  }
}

int moe_plan_get_option(moe_plan_t p, int key, long long* value) {
  if (!p || !value) return MOE_ERR_INVALID_ARG;
  switch (key) {
    case MOE_OPT_GRAPH: *value = p->use_graph; return MOE_OK;
    case MOE_OPT_MAX_SMS: *value = p->max_sms; return MOE_OK;
    case MOE_OPT_TIMEOUT_NS: *value = (long long)p->timeout_ns; return MOE_OK;
    case MOE_OPT_INJECT_FAULT: *value = p->inject_fault; return MOE_OK;
    case MOE_OPT_STATIC_WEIGHTS: *value = p->static_weights; return MOE_OK;
    case MOE_OPT_ROUTER_TC: *value = p->router_tc; return MOE_OK;
    case MOE_OPT_PHASE_EVENTS: *value = p->phase_events; return MOE_OK;
    case MOE_OPT_FUSED: *value = p->fused; return MOE_OK;
    case MOE_OPT_CHAIN: *value = p->chain; return MOE_OK;
    case MOE_OPT_L2_TILE_ROWS: *value = linear2_bn(p); return MOE_OK;
    case MOE_OPT_DEPENDENT_LAUNCH: *value = plan_dep_launch(p) ? 1 : 0; return MOE_OK;
    case MOE_OPT_PAIR_TILES: *value = p->pair_mode; return MOE_OK;
    case MOE_OPT_SWAP_ROWS: *value = p->swap_rows; return MOE_OK;
    case MOE_OPT_TILE_ROWS: *value = plan_bm(p); return MOE_OK;
    case MOE_OPT_ZERO_PAD: *value = plan_zero_pad(p) ? 1 : 2; return MOE_OK;
    default: return MOE_ERR_INVALID_ARG;
  }
}

size_t moe_workspace_bytes(moe_plan_t p) { return p ? p->total : 0; }

int moe_workspace_region(moe_plan_t p, int r, size_t* offset, size_t* bytes) {
  if (!p || r < 0 || r >= MOE_REGION_COUNT_ || !offset || !bytes) return MOE_ERR_INVALID_ARG;
  *offset = p->region_off[r];
  *bytes = p->region_len[r];
  return MOE_OK;
}

int moe_set_workspace(moe_plan_t p, void* ws, size_t bytes) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (!ws || bytes < p->total || !aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_SHAPE;   // built for sm_100a only
  if (gemm_prepare_device() != cudaSuccess) return MOE_ERR_CUDA;
  drop_graphs(p);
  p->ws = static_cast<uint8_t*>(ws);
  p->ws_bytes = bytes;
  p->device = dev;
  p->num_sms = sms;
  p->w1_cached = p->w2_cached = nullptr;
  p->w1s_prepared = p->w2s_prepared = nullptr;
  p->x_cached = p->wr_prepared = nullptr;
  int rc = MOE_OK;
  for (int i = 0; i < 4 && rc == MOE_OK; ++i) {
    rc = encode_2d(&p->amA1.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, region<uint8_t>(p, MOE_REGION_XQ), p->H, p->rows,
                   p->H, 128, 16u << i);
    if (rc == MOE_OK)
      rc = encode_2d(&p->amA2.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, region<uint8_t>(p, MOE_REGION_HQ), p->I,
                     p->rows, p->I, 128, 16u << i);
  }
  if (rc == MOE_OK)
    rc = encode_2d(&p->tmWhi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, at<uint16_t>(p, p->off_whi), p->H, p->E,
                   2ull * p->H, 64, 128);
  if (rc == MOE_OK)
    rc = encode_2d(&p->tmWlo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, at<uint16_t>(p, p->off_wlo), p->H, p->E,
                   2ull * p->H, 64, 128);
  // scale atoms (512 B) and weight scale units (1024 B) as rows of 256 bytes, no swizzle
  struct SfMap {
    CUtensorMap* m;
    const void* base;
    size_t bytes;
    uint32_t box_rows;
  } sf[4] = {{&p->tmSfa1, region<uint8_t>(p, MOE_REGION_XSF), p->region_len[MOE_REGION_XSF], 2},
             {&p->tmSfa2, region<uint8_t>(p, MOE_REGION_HSF), p->region_len[MOE_REGION_HSF], 2},
             {&p->tmSfb1, at<uint8_t>(p, p->off_w1sf), (size_t)p->n * (p->I / 128) * (p->H / 128) * 1024, 4},
             {&p->tmSfb2, at<uint8_t>(p, p->off_w2sf),
              (size_t)p->n * ((p->H + kGemmBN - 1) / kGemmBN) * (p->I / 128) * 1024, 4}};
  for (int i = 0; i < 4 && rc == MOE_OK; ++i)
    rc = encode_2d(sf[i].m, CU_TENSOR_MAP_DATA_TYPE_UINT8, sf[i].base, 256, sf[i].bytes / 256, 256, 256,
                   sf[i].box_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != MOE_OK) {
    p->ws = nullptr;
    return rc;
  }
  if (cudaMemset(region<uint32_t>(p, MOE_REGION_STATUS), 0, 16) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(at<uint32_t>(p, p->off_gridbar), 0, 8) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(at<uint8_t>(p, p->off_zeros), 0, kGemmZeroBytes) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_forward(moe_plan_t p, const void* x, const float* W_router, const float* bias, const uint8_t* W1,
                const uint8_t* W1_scales, const uint8_t* W2, const uint8_t* W2_scales, void* out, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(x, 16) || !aligned(W_router, 16) || !aligned(bias, 4) || !aligned(W1, 32) ||
      !aligned(W1_scales, 4) || !aligned(W2, 32) || !aligned(W2_scales, 4) || !aligned(out, 16))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (W1 != p->w1_cached) {
    rc = encode_2d(&p->tmB1, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W1, p->H, (uint64_t)p->n * 2 * p->I, p->H / 2,
                   128, 128);
    if (rc == MOE_OK)
      rc = encode_3d(&p->tmB1g, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W1, p->H, p->I, (uint64_t)p->n * 2, p->H / 2,
                     (uint64_t)p->I * (p->H / 2), 128, 128, 2);
    if (rc != MOE_OK) return rc;
    p->w1_cached = W1;
  }
  if (W2 != p->w2_cached) {
    rc = encode_2d(&p->tmB2, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W2, p->I, (uint64_t)p->n * p->H, p->I / 2,
                   128, 256);
    if (rc == MOE_OK)
      rc = encode_2d(&p->tmB2d, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W2, p->I, (uint64_t)p->n * p->H, p->I / 2,
                     128, kGemmBN2Double);
    if (rc == MOE_OK)
      rc = encode_2d(&p->tmB2p, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, W2, p->I, (uint64_t)p->n * p->H, p->I / 2,
                     128, 128);
    if (rc != MOE_OK) return rc;
    p->w2_cached = W2;
  }
  if (p->phase_events && !p->events_ready) {
    for (int i = 0; i <= MOE_PHASE_COUNT_; ++i)
      if (cudaEventCreate(&p->ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
    p->events_ready = true;
  }
  if (p->use_graph && !p->phase_events && !p->fused) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) != cudaSuccess) return MOE_ERR_CUDA;
    if (st == cudaStreamCaptureStatusNone) return forward_graph(p, x, W_router, bias, W1, W1_scales, W2, W2_scales,
                                                                out, s);
  }
  return launch_forward(p, static_cast<const uint16_t*>(x), W_router, bias, W1_scales, W2_scales, out, s);
}

int moe_phase_times(moe_plan_t p, float* ms, int capacity) {
  if (!p || !ms || capacity < MOE_PHASE_COUNT_) return MOE_ERR_INVALID_ARG;
  if (!p->events_recorded) return MOE_ERR_INVALID_ARG;
  if (cudaEventSynchronize(p->ev[MOE_PHASE_COUNT_]) != cudaSuccess) return MOE_ERR_CUDA;
  for (int i = 0; i < MOE_PHASE_COUNT_; ++i)
    if (cudaEventElapsedTime(&ms[i], p->ev[i], p->ev[i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
  if (p->fused && p->fused_ctas_last > 0) {
    // one kernel: split its event time by the phase stamps (the latest CTA at each point; the
    // router phase runs from the earliest start)
    const int n = p->fused_ctas_last;
    std::vector<unsigned long long> h((size_t)kStampCount * n);
    for (int id = 0; id < kStampCount; ++id)
      if (cudaMemcpy(h.data() + (size_t)id * n, region<unsigned long long>(p, MOE_REGION_STAMPS) + (size_t)id * kStampMaxCtas,
                     n * 8, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    unsigned long long t[kStampCount];
    for (int id = 0; id < kStampCount; ++id) {
      unsigned long long v = id == kStampStart ? ~0ull : 0ull;
      for (int c = 0; c < n; ++c) {
        const unsigned long long s = h[(size_t)id * n + c];
        if (id == kStampCombine && s == 0) continue;            // CTAs without combine items skip it
        v = id == kStampStart ? (s < v ? s : v) : (s > v ? s : v);
      }
      t[id] = v;
    }
    if (t[kStampCombine] == 0) t[kStampCombine] = t[kStampLinear1];
    const float total = ms[MOE_PHASE_ROUTER];
    auto d = [&](int a, int b) { return t[b] > t[a] ? (float)((t[b] - t[a]) * 1e-6) : 0.f; };
    for (int i = 0; i < MOE_PHASE_COUNT_; ++i) ms[i] = 0.f;
    ms[MOE_PHASE_TOPK] = d(kStampRouted, kStampScanned);
    ms[MOE_PHASE_SCATTER_QUANT] = d(kStampScanned, kStampRowsReady);
    ms[MOE_PHASE_LINEAR1] = d(kStampRowsReady, kStampLinear1);
    ms[MOE_PHASE_LINEAR2] = d(kStampLinear1, kStampCombine);
    ms[MOE_PHASE_COMBINE] = d(kStampCombine, kStampEnd);
    // the router phase carries the launch and the rest of the event time
    float rest = total;
    for (int i = 1; i < MOE_PHASE_COUNT_; ++i) rest -= ms[i];
    ms[MOE_PHASE_ROUTER] = rest > 0.f ? rest : d(kStampStart, kStampRouted);
  }
  return MOE_PHASE_COUNT_;
}

int moe_debug_routing(moe_plan_t p, const void* x, const float* W_router, const float* bias, int32_t* topk_ids,
                      float* gates, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(x, 16) || !aligned(W_router, 16) || !aligned(bias, 4) || !aligned(topk_ids, 4) || !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = run_router(p, static_cast<const uint16_t*>(x), W_router, s);
  if (rc != MOE_OK) return rc;
  cudaError_t e = launch_topk_rank(0, at<float>(p, p->off_logits), logit_parts(p), bias, topk_ids, gates,
                                   at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gcounts),
                                   region<uint32_t>(p, MOE_REGION_STATUS), p->T, p->E, p->k, s);
  return cuda_rc(e);
}

int moe_update_bias(moe_plan_t p, float* bias, float gamma, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(bias, 4) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_update_bias(bias, region<int32_t>(p, MOE_REGION_COUNTS), p->T, p->k, p->E, gamma,
                                    static_cast<cudaStream_t>(stream)));
}

int moe_debug_dispatch(moe_plan_t p, const int32_t* topk_ids, int32_t* counts, int32_t* offsets, int32_t* perm,
                       int32_t* slot_pos, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(topk_ids, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm, 4) ||
      !aligned(slot_pos, 4))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_topk_rank(1, nullptr, 1, nullptr, const_cast<int32_t*>(topk_ids), nullptr,
                                   at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gcounts),
                                   region<uint32_t>(p, MOE_REGION_STATUS), p->T, p->E, p->k, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if ((e = launch_dispatch_scan(at<int32_t>(p, p->off_gcounts), counts, offsets, at<int32_t>(p, p->off_gbase),
                                at<int32_t>(p, p->off_mtile), at<int32_t>(p, p->off_ptile),
                                at<int4>(p, p->off_tinfo), at<int4>(p, p->off_ptinfo), p->T, p->E, p->k,
                                p->shared, plan_bm(p), s)) != cudaSuccess)
    return MOE_ERR_CUDA;
  // positions = offsets (written just above into the caller's buffer) + group base + rank
  e = launch_scatter_quant(nullptr, topk_ids, at<int32_t>(p, p->off_rank), at<int32_t>(p, p->off_gbase), offsets,
                           at<int32_t>(p, p->off_mtile), slot_pos, perm, nullptr, nullptr, p->T, p->H, p->E, p->k,
                           p->shared, plan_bm(p), s);
  return cuda_rc(e);
}

int moe_debug_quant_x(moe_plan_t p, const void* x, uint8_t* xq, float* xs, void* stream) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  if (!aligned(x, 16) || !aligned(xq, 8) || !aligned(xs, 4)) return MOE_ERR_INVALID_ARG;
  return cuda_rc(launch_quant_tokens(static_cast<const uint16_t*>(x), xq, xs, p->T, p->H,
                                     static_cast<cudaStream_t>(stream)));
}

int moe_check_status(moe_plan_t p, void* stream, uint32_t* detail) {
  int rc = check_bound(p);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t h[4] = {0, 0, 0, 0};
  uint32_t* d = region<uint32_t>(p, MOE_REGION_STATUS);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(d, 0, sizeof(h)) != cudaSuccess) return MOE_ERR_CUDA;
  if (detail) std::memcpy(detail, h, sizeof(h));
  return (int)(int32_t)h[0];
}

void moe_plan_destroy(moe_plan_t p) {
  if (!p) return;
  drop_graphs(p);
  if (p->cap_stream) cudaStreamDestroy(p->cap_stream);
  if (p->events_ready)
    for (int i = 0; i <= MOE_PHASE_COUNT_; ++i) cudaEventDestroy(p->ev[i]);
  delete p;
}

const char* moe_error_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or device";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_DEBUG_BOUNDS: return "device-side bounds check failed";
    default: return "unknown error";
  }
}

}  // extern "C"
