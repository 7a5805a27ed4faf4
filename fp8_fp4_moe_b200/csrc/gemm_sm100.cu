// Grouped block-scaled GEMMs of the expert FFN on sm_100a (tcgen05 + TMA).
//
//   linear1: for each expert e, acc[n_e, 2 x 128] = xq_e (E4M3, K = H) x W1_e^T
//            (E2M1, gate rows j and up rows I + j of one 128-channel block),
//            then h = silu(gate) * up and E4M3 requantisation of h with one
//            power-of-two scale per row per 128 channels;
//   linear2: for each expert e, rows[n_e, 256] = hq_e (E4M3, K = I) x W2_e^T
//            (E2M1), stored as bf16.
// The expert FFN is "linear1 (FP8 x FP4) -> SwiGLU -> linear2 (FP8 x FP4)"
// ("DeepSeek Mega MoE / DeepGEMM mega kernel", TL;DR and "Thông số kỹ thuật").
//
// Design (one CTA per SM, persistent, static round-robin over tiles):
//   warp 0      TMA producer.  Per 128-deep K stage: the A tile 128 x 128 B
//               (SW128), the B tile 256 x 128 FP4 elements loaded with the
//               16U4_ALIGN16B type (packed nibbles land in the padded
//               shared-memory form the f8f6f4 MMA reads: 128 bytes per 128
//               elements), and the two scale-factor atoms of the stage as
//               bulk copies (A: 512 B, B: 1024 B) from pre-tiled layouts;
//   warp 1      TMEM owner and single-thread MMA issuer:
//               tcgen05.cp of the scale atoms (32x128b.warpx4), then
//               tcgen05.mma.kind::mxf8f6f4.block_scale M=128 N=256 K=32 x4,
//               fp32 accumulator in TMEM columns [0, 256);
//   warps 2..9  epilogue, two warps per 32-lane TMEM quarter, each owning
//               half of the accumulator columns: tcgen05.ld, release the
//               accumulator, then SwiGLU + requant (linear1) or bf16 (linear2).
// Scale-factor atom (128 rows x 4 K-blocks of 32): row r at byte
// (r % 32) * 16 + (r / 32) * 4, block b at + b; copied to TMEM it gives row r
// its scale at lane r % 32 (all four sub-partitions), column r / 32, byte b.
// Tiles never cross experts: expert e owns rows [offsets[e], offsets[e+1]) of
// the dispatched activations, split into ceil(n_e/128) row tiles (global row
// tile index mtile_start[e] + mt); rows of a tile past n_e are computed on
// whatever the loads return and never stored.
// Every wait is bounded (WaitCtl); on a timeout the CTA records
// MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM, returns.
#include "common.cuh"
#include "kernels.h"
#include "path_phases.cuh"

namespace moe {

namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, S = kGemmStages;
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0, kSfaCol = 256, kSfbCol = 264;
constexpr uint32_t kATileBytes = BM * BK;            // 16 KB
constexpr uint32_t kBTileBytes = BN * BK;            // 32 KB in shared memory (unpacked FP4)
constexpr uint32_t kSfaBytes = 512, kSfbBytes = 1024;

// Shared memory of the single-CTA grouped GEMM: STAGES pipeline stages with an A region of
// A_BYTES each, and (STAGING) a 2 KB per-warp buffer the epilogue stores go through.  The
// linear1 epilogue exchanges per-row amax values for AMAX_ROWS accumulator rows (the rows a
// tile can hold; 128 also leaves room for the transposed-tile exchange).
template <int STAGES, uint32_t A_BYTES, bool STAGING, int AMAX_ROWS = 128>
struct GemmSmem {
  static constexpr int kStages = STAGES;
  static constexpr uint32_t kABytes = A_BYTES;
  static constexpr bool kStaging = STAGING;
  static constexpr int kAmaxRows = AMAX_ROWS;
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + STAGES * A_BYTES;
  static constexpr uint32_t sfa = b + STAGES * kBTileBytes;
  static constexpr uint32_t sfb = sfa + STAGES * kSfaBytes;
  static constexpr uint32_t amax = sfb + STAGES * kSfbBytes;      // [2 buffers][2 halves][AMAX_ROWS] fp32
  static constexpr uint32_t stage_out = amax + 2 * 2 * AMAX_ROWS * 4;   // [8 epilogue warps][32 rows][64 B]
  static constexpr uint32_t bars = stage_out + (STAGING ? 8 * 2048 : 0);
  // full[STAGES], empty[STAGES], accf[2], acce[2], drain
  static constexpr uint32_t n_bars = 2 * STAGES + 5;
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t total = misc + 16;
};
// Any number of rows per tile: 4 stages with 128-row A regions.
using SmemLayout = GemmSmem<S, kATileBytes, true>;
// 32-row row tiles (decode-sized experts): 32-row A regions leave room for 6 stages; the MMA
// still reads 128 A rows, the ones past the region are other stages' bytes and land in
// accumulator rows that are never stored.  Epilogue stores go straight to global memory.
using SmallSmem = GemmSmem<6, kGemmBMSmall * BK, false, kGemmBMSmall>;
static_assert(SmallSmem::total + 1024 <= 232448, "small-tile layout exceeds shared memory");

struct TileCoord {
  int e, mt, nt, count, row0, gmt;   // gmt = global row-tile index
  int rows;                          // rows of the expert in this tile (1..128)
};

// Order of an expert's (m, n) tiles, `local` in [0, m_count * n_count): bands of kBand row tiles,
// every column tile of a band before the next band, row tiles fastest inside a band.  While the
// grid works through one band, its rows (and the expert's weight tiles) stay in L2; with the plain
// n-major order an expert of many row tiles -- the shared expert of a large batch -- streamed all
// of its rows from DRAM once per column tile.  An expert of at most kBand row tiles is one band:
// n-major, m fastest.
constexpr int kBand = 8;
__device__ __forceinline__ void banded_mn(int local, int m_count, int n_count, int& m, int& n) {
  const int full = m_count / kBand;                 // complete bands
  const int in_full = full * kBand * n_count;
  if (local < in_full) {
    const int band = local / (kBand * n_count), rem = local - band * kBand * n_count;
    n = rem / kBand;
    m = band * kBand + (rem - n * kBand);
  } else {
    const int last = m_count - full * kBand;        // row tiles of the last, shorter band
    const int rem = local - in_full;
    n = rem / last;
    m = full * kBand + (rem - n * last);
  }
}

// The tiles of expert e are [mtile_start[e], mtile_start[e + 1]) x n_tiles_n, so tile / n_tiles_n
// is one of e's row tiles and its table entry names e: one load per tile instead of a search
// over the experts.  Each role loads the entry of its next tile while it works on the current
// one (tile_entry / TileCursor), so the load's latency is off the tile boundary.
__device__ __forceinline__ int4 tile_entry(const GemmArgs& p, int tile, int total_tiles) {
  return tile < total_tiles ? ld_cg_v4(p.tile_info + tile / p.n_tiles_n) : make_int4(0, 0, 0, 0);
}
// info = the table entry {e, mtile_start, count, offset} of `tile`
__device__ __forceinline__ TileCoord decode_tile_entry(const GemmArgs& p, int tile, int4 info) {
  const int bm = p.bm;
  TileCoord c;
  c.e = info.x;
  c.count = info.z;
  const int mtiles = (c.count + bm - 1) / bm;
  const int mstart = info.y;
  const int local = tile - mstart * p.n_tiles_n;
  banded_mn(local, mtiles, p.n_tiles_n, c.mt, c.nt);
  c.row0 = info.w + c.mt * bm;
  c.gmt = mstart + c.mt;
  c.rows = min(bm, c.count - c.mt * bm);
  return c;
}
// Walks tiles first, first + stride, ... with the next tile's table entry already requested.
struct TileCursor {
  int tile, stride, total;
  int4 next;
  __device__ __forceinline__ TileCursor(const GemmArgs& p, int first, int stride_, int total_)
      : tile(first), stride(stride_), total(total_), next(tile_entry(p, first, total_)) {}
  __device__ __forceinline__ bool more() const { return tile < total; }
  // coordinates of the current tile; requests the entry of the one after it
  __device__ __forceinline__ TileCoord take(const GemmArgs& p) {
    const TileCoord c = decode_tile_entry(p, tile, next);
    next = tile_entry(p, tile + stride, total);
    return c;
  }
  __device__ __forceinline__ void advance() { tile += stride; }
};

// Accumulator slots.  With 256-row weight tiles (every linear1, linear2 by default) the
// slots are TMEM columns [0, 128) and [128, 256) and the scale factors sit at 256..271: a
// tile with at most swap_rows rows of its expert is computed transposed (weights as the
// M = 128 operand, the tile's tokens as N = 32 or 64) into one slot, alternating between the
// two, and any other tile takes both slots (M = 128 tokens, N = 256).  With 224-row weight
// tiles (linear2, DOUBLE) the slots are [0, 224) and [256, 480), the scale factors sit at
// 224..239, and every tile takes one slot, alternating: the epilogue drains one tile while
// the MMAs of the next accumulate into the other.  The MMA issuer and the epilogue walk the
// same tile sequence and keep one use counter per slot, so both derive the same mbarrier
// parities.
struct SlotPlan {
  bool swap;
  int lo, hi;        // slots [lo, hi] this tile uses
  int nt_tok;        // swapped tiles: token columns (MMA N)
};
template <bool DOUBLE, bool SWAP_OK = true>
__device__ __forceinline__ SlotPlan plan_slots(const GemmArgs& p, const TileCoord& c, int& next_slot) {
  SlotPlan s;
  s.swap = SWAP_OK && c.rows <= p.swap_rows;
  s.nt_tok = c.rows <= 32 ? 32 : 64;
  if (s.swap || DOUBLE) {
    s.lo = s.hi = next_slot;
    next_slot ^= 1;
  } else {
    s.lo = 0;
    s.hi = 1;
  }
  return s;
}
// TMEM column layout for a weight-tile height NB (256, or 224 for double-buffered linear2).
template <int NB>
struct TmemMap {
  static constexpr bool kDouble = NB < 256;
  static constexpr uint32_t slot_stride = kDouble ? 256 : 128;
  static constexpr uint32_t sfa = kDouble ? 224 : 256;
  static constexpr uint32_t sfb = sfa + 8;              // two atoms: sfb, sfb + 4
  static_assert(NB % 32 == 0 && NB >= 160 && NB <= 256, "weight tile height");
};

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart.
  return smem_desc(saddr, 16, 1024, kLayoutSwizzle128B);
}
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  // 32 rows x 16 bytes, contiguous, no swizzle: 8-row core matrices 128 bytes apart.
  return smem_desc(saddr, 16, 128, kLayoutNoSwizzle);
}

// Named barrier over the epilogue warps (ids 1..; 0 is __syncthreads).
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
}
// Epilogue-wide AND of `ok` (a barrier too): every epilogue warp takes the same branch, so a
// wait that timed out in one warp cannot leave the others blocked in a later epi_bar.
__device__ __forceinline__ bool epi_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(kEpiWarps * 32)
      : "memory");
  return r != 0;
}

// Store 64 bytes of each of the warp's 32 rows (lane l holds row l's bytes in v[0..3]) so that
// every global store instruction writes whole 32-byte sectors: the chunk goes through a
// 2 KB per-warp shared buffer (16-byte pieces XOR-swizzled against bank conflicts) and
// comes back with 4 lanes per row.  dst0 = address of lane 0's row, row_stride in bytes;
// only rows with row_ok set (in the owning lane) are written.
__device__ __forceinline__ void store_rows_64b(uint8_t* buf, const uint4 (&v)[4], uint8_t* dst0, long row_stride,
                                               bool row_ok, int lane) {
  if (buf == nullptr) {                // no staging buffer (few rows): each lane writes its row
    if (row_ok) {
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(dst0 + lane * row_stride + c * 16) = v[c];
    }
    return;
  }
  const uint32_t okmask = __ballot_sync(0xffffffffu, row_ok);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16)) = v[c];
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = it * 8 + (lane >> 2);
    const int c = lane & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(buf + r * 64 + ((c ^ ((r >> 1) & 3)) * 16));
    if (okmask & (1u << r)) *reinterpret_cast<uint4*>(dst0 + r * row_stride + c * 16) = w;
  }
  __syncwarp();
}

// Release the accumulator: both slots of this CTA (NB = 256), the tile's own slot (acce
// points at it; NB < 256), or (CTA pairs) the rank-0 CTA's barrier through its cluster-window
// address.
template <int NB>
__device__ __forceinline__ void release_acc(uint64_t* acce, uint32_t acce_remote) {
  if (acce_remote != 0) {
    mbar_arrive_cluster(acce_remote);
  } else if (NB < 256) {
    mbar_arrive(acce);
  } else {
    mbar_arrive(&acce[0]);
    mbar_arrive(&acce[1]);
  }
}

// One tile's epilogue; `acc` = TMEM address (lane 0) of the tile's accumulator.  AR: rows of
// the amax exchange buffer (>= the tile's rows; accumulator rows past them are never stored).
template <int MODE, int NB = 256, int AR = 128>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& p, const TileCoord& c, uint32_t acc, int q,
                                              int half, int lane, uint64_t* acce, uint32_t acce_remote,
                                              float* amax_s, int buf, uint8_t* obuf) {
  const int m = q * 32 + lane;                         // accumulator row = TMEM lane
  const uint32_t t_row = acc + ((uint32_t)(q * 32) << 16);
  const bool valid = m < c.rows;                       // rows of this tile of the expert
  if constexpr (MODE == 1) {
    // this warp: h channels [64*half, 64*half + 64) of the tile's 128
    uint32_t g[64], u[64];
    static_assert(NB == 256, "linear1 tiles hold 128 gate and 128 up rows");
    tmem_ld_32x32b_x32(t_row + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&g[0]));
    tmem_ld_32x32b_x32(t_row + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&g[32]));
    tmem_ld_32x32b_x32(t_row + 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
    tmem_ld_32x32b_x32(t_row + 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) release_acc<NB>(acce, acce_remote);     // accumulator may be overwritten now
    float h[64];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const float gv = __uint_as_float(g[i]);
      const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * __uint_as_float(u[i]);   // silu(gate) * up
      h[i] = hv;
      amax = fmaxf(amax, fabsf(hv));
    }
    // the 128-channel block's amax spans both halves: exchange through shared memory
    float* slot = amax_s + buf * 2 * AR;
    if (m < AR) slot[half * AR + m] = amax;
    epi_bar();
    if (m < AR) amax = fmaxf(amax, slot[(half ^ 1) * AR + m]);
    const int pexp = pow2_exp_e4m3(amax);
    const float sc = exp2_neg(pexp);
    uint4 w[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      w[v].x = pack_e4m3x4(h[v * 16 + 0] * sc, h[v * 16 + 1] * sc, h[v * 16 + 2] * sc, h[v * 16 + 3] * sc);
      w[v].y = pack_e4m3x4(h[v * 16 + 4] * sc, h[v * 16 + 5] * sc, h[v * 16 + 6] * sc, h[v * 16 + 7] * sc);
      w[v].z = pack_e4m3x4(h[v * 16 + 8] * sc, h[v * 16 + 9] * sc, h[v * 16 + 10] * sc, h[v * 16 + 11] * sc);
      w[v].w = pack_e4m3x4(h[v * 16 + 12] * sc, h[v * 16 + 13] * sc, h[v * 16 + 14] * sc, h[v * 16 + 15] * sc);
    }
    store_rows_64b(obuf, w, p.hq + (long)(c.row0 + q * 32) * p.N + (long)c.nt * 128 + half * 64, p.N, valid, lane);
    if (valid) {
      if (half == 0) {
        // scale word of (row tile gmt, K-tile nt of linear2) in the tiled atom layout
        uint8_t* atom = reinterpret_cast<uint8_t*>(p.hsf) + ((long)c.gmt * (p.N / 128) + c.nt) * 512;
        *reinterpret_cast<uint32_t*>(atom + (m % 32) * 16 + (m / 32) * 4) = (uint32_t)(pexp + 127) * 0x01010101u;
      }
    }
  } else {
    // this warp: output columns [128*half, min(128*half + 128, NB)) of the tile
    const int nch = half == 0 ? 4 : (NB - 128) / 32;   // 32-column chunks (warp-uniform)
    uint32_t packed[64];
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      if (ch < nch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + half * 128 + ch * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          packed[ch * 16 + i] = *reinterpret_cast<uint32_t*>(&b2);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) release_acc<NB>(acce, acce_remote);
    const int col0 = c.nt * NB + half * 128;
    uint8_t* dst0 = reinterpret_cast<uint8_t*>(p.y + (long)(c.row0 + q * 32) * p.N + col0);
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      if (ch < nch && col0 + ch * 32 < p.N) {          // warp-uniform column tail
        uint4 w[4];
#pragma unroll
        for (int v = 0; v < 4; ++v)
          w[v] = make_uint4(packed[ch * 16 + v * 4 + 0], packed[ch * 16 + v * 4 + 1], packed[ch * 16 + v * 4 + 2],
                            packed[ch * 16 + v * 4 + 3]);
        store_rows_64b(obuf, w, dst0 + ch * 64, (long)p.N * 2, valid, lane);
      }
    }
  }
}

// Lane l ends with the maximum over the warp's 32 lanes of a[l % TW] (TW = 16 or 32):
// each step keeps half of the values and folds in the partner's copy of the other half.
template <int TW>
__device__ __forceinline__ float warp_transpose_max(float (&a)[TW], int lane) {
  if constexpr (TW == 16) {
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = fmaxf(a[i], __shfl_xor_sync(0xffffffffu, a[i], 16));
  }
#pragma unroll
  for (int s = TW / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? a[i] : a[i + s];
      const float keep = upper ? a[i + s] : a[i];
      a[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, s));
    }
  }
  return a[0];
}

// Epilogue of a transposed tile: TMEM lane = weight row (channel), column = token.
//   linear1: gate accumulator in slot columns [0, NT), up in [64, 64 + NT); warp (q, half)
//            owns channels q*32 + lane of the tile's 128 and tokens [half*NT/2, half*NT/2 + NT/2);
//            the per-token amax over the 128 channels goes through shared memory.
//   linear2: rows 0..127 of the NB-row weight tile in slot columns [0, NT), rows 128..NB-1 in
//            [64, 64 + NT) (the MMA also covers rows NB..255 of the stage, which are dropped);
//            warp (q, half) owns output channels half*128 + q*32 + lane, all tokens.
// Per token, a warp's 32 channels are consecutive in the output row: one store instruction
// covers 32 bytes (linear1) or 64 bytes (linear2).
template <int MODE, int NT, int NB = 256>
__device__ __forceinline__ void epilogue_swap(const GemmArgs& p, const TileCoord& c, uint32_t acc, int q, int half,
                                              int lane, uint64_t* acce_slot, float* amax_s, int buf) {
  const uint32_t t_lane = acc + ((uint32_t)(q * 32) << 16);
  if constexpr (MODE == 1) {
    constexpr int TW = NT / 2;
    uint32_t g[TW], u[TW];
    if constexpr (TW == 16) {
      tmem_ld_32x32b_x16(t_lane + half * TW, g);
      tmem_ld_32x32b_x16(t_lane + 64 + half * TW, u);
    } else {
      tmem_ld_32x32b_x32(t_lane + half * TW, g);
      tmem_ld_32x32b_x32(t_lane + 64 + half * TW, u);
    }
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_slot);
    float h[TW], a[TW];
#pragma unroll
    for (int j = 0; j < TW; ++j) {
      const float gv = __uint_as_float(g[j]);
      h[j] = __fdividef(gv, 1.0f + __expf(-gv)) * __uint_as_float(u[j]);   // silu(gate) * up
      a[j] = fabsf(h[j]);
    }
    const int tl = lane % TW;                    // this lane's token within the warp's range
    const int tok = half * TW + tl;              // token row within the tile
    float* slot = amax_s + buf * 256;            // [quarter][64 tokens]
    const float am_q = warp_transpose_max<TW>(a, lane);
    if (lane < TW) slot[q * 64 + tok] = am_q;
    epi_bar();
    const float am = fmaxf(fmaxf(slot[tok], slot[64 + tok]), fmaxf(slot[128 + tok], slot[192 + tok]));
    const int pexp = pow2_exp_e4m3(am);
    const float sc = exp2_neg(pexp);
    if (q == 0 && lane < TW && tok < c.rows) {
      uint8_t* atom = reinterpret_cast<uint8_t*>(p.hsf) + ((long)c.gmt * (p.N / 128) + c.nt) * 512;
      *reinterpret_cast<uint32_t*>(atom + (tok % 32) * 16 + (tok / 32) * 4) = (uint32_t)(pexp + 127) * 0x01010101u;
    }
    uint8_t* dst = p.hq + (long)(c.row0 + half * TW) * p.N + (long)c.nt * 128 + q * 32 + lane;
#pragma unroll
    for (int j = 0; j < TW; ++j) {
      const float sj = __shfl_sync(0xffffffffu, sc, j);
      const uint8_t b = (uint8_t)(cvt_e4m3x2(h[j] * sj, 0.f) & 0xFF);
      if (half * TW + j < c.rows) dst[(long)j * p.N] = b;
    }
  } else {
    uint32_t r[NT];
    tmem_ld_32x32b_x32(t_lane + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    if constexpr (NT == 64) tmem_ld_32x32b_x32(t_lane + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce_slot);
    const int local = half * 128 + q * 32 + lane;     // weight row within the tile
    const int col = c.nt * NB + local;
    if (local < NB && col < p.N) {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + (long)c.row0 * p.N + col;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        if (j < c.rows) dst[(long)j * p.N] = __float2bfloat16_rn(__uint_as_float(r[j]));
    }
  }
}

// Bounded wait until *ctr >= need, then a gpu-scope acquire.  Polls with relaxed loads and a
// growing pause (one thread per waiter: callers elect it).  On expiry records
// MOE_ERR_DEVICE_TIMEOUT at `where` and returns false; returns false at once when `abort_flag`
// (if given) is raised.
__device__ __forceinline__ bool wait_counter(const uint32_t* ctr, uint32_t need, uint32_t* status,
                                             uint64_t timeout_ns, uint32_t where, volatile int* abort_flag) {
  if (ld_acquire_gpu(ctr) >= need) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t pause = 32;
  while (ld_relaxed_gpu(ctr) < need) {
    if (abort_flag != nullptr && *abort_flag) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      report_status(status, kStatusTimeout, where, need);
      return false;
    }
    poll_pause(pause);
  }
  fence_acq_rel_gpu();
  return true;
}

// Work an epilogue warp does before its first tile or after its last one (the single-kernel
// forward's scatter and combine); called with the warp's index among all epilogue warps of the
// grid, their number, whether the GEMM ran without a device-side failure, and the CTA's
// (1024-aligned) dynamic shared memory.
struct NoEpilogueWork {
  __device__ __forceinline__ void operator()(int, int, bool, uint8_t*) const {}
};

// One grouped GEMM over tiles cta, cta + n_ctas, ... by all kGemmThreads threads of the CTA,
// with `tmem_base` holding 512 allocated TMEM columns and `smem` the 1024-aligned dynamic
// shared memory.  Initialises its barriers on entry and invalidates them on exit, so the
// same CTA may run it again (the single persistent forward runs linear1, then linear2).
// NB: weight rows per tile (linear2 may use 224, whose accumulator is double-buffered; tmB's
// box must then be 224 rows high and the weight scale units laid out for 224-row tiles).
// Readiness (single-kernel forward): with p.rows_ready set, the producer loads no A rows or
// activation scales before *p.rows_ready >= p.rows_ready_need (weights stream before that); with
// p.tiles_done set, the epilogue adds 1 to it after each stored tile.  `pre` / `post`: work of
// the epilogue warps around their tiles (NoEpilogueWork elsewhere).
template <int MODE, class L = SmemLayout, int NB = 256, class Pre = NoEpilogueWork, class Post = NoEpilogueWork>
__device__ __forceinline__ void gemm_body(const AMaps& tmA, const CUtensorMap& tmB, const GemmArgs& p,
                                          uint8_t* smem, uint32_t tmem_base, int cta, int n_ctas,
                                          const Pre& pre = Pre(), const Post& post = Post()) {
  static_assert(MODE == 2 || NB == 256, "linear1 tiles are 256 weight rows");
  using TM = TmemMap<NB>;
  constexpr int S = L::kStages;
  constexpr uint32_t kATileBytes = L::kABytes;
  // bytes one stage's copies bring: A rows (box height set per tile), weights, scale factors
  constexpr uint32_t kStageTxNoA = NB * BK / 2 + kSfaBytes + kSfbBytes;
  uint8_t* a_s = smem + L::a;
  uint8_t* b_s = smem + L::b;
  uint8_t* sfa_s = smem + L::sfa;
  uint8_t* sfb_s = smem + L::sfb;
  float* amax_s = reinterpret_cast<float*>(smem + L::amax);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* accf = bars + 2 * S;      // [2] accumulator slot full
  uint64_t* acce = accf + 2;          // [2] accumulator slot empty
  uint64_t* drain = accf + 4;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf[i], 1);
      mbar_init(&acce[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&tmA.m[i]);
    tma_prefetch_desc(&tmB);
  }
  __syncthreads();
  tc_fence_after();

  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total_tiles = ld_cg(p.mtile_start + p.n_experts) * p.n_tiles_n;
  const int KT = p.K / BK;
  // the transposed-tile epilogue needs the full amax exchange buffer
  constexpr bool kSwapOk = L::kAmaxRows >= 128;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t fills[S];
      // Rows of each stage's A region that may hold data of an earlier tile (all of them at the
      // start).  With p.zeros set (128-row regions only) the rows a tile's box does not cover are
      // zeroed by a bulk copy from that buffer before the MMA reads them: the MMA computes all 128
      // rows whatever the tile holds, and zero operands draw less power than stale rows.
      constexpr uint32_t kARows = kATileBytes / BK;
      const bool zero_pad = p.zeros != nullptr && kARows == BM;
      uint32_t dirty[S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        fills[s] = 0;
        dirty[s] = kARows;
      }
      // bytes of the zero copy stage st needs before a box of a_box rows lands (0 if none)
      auto zero_bytes = [&](int st, uint32_t a_box) -> uint32_t {
        return zero_pad && dirty[st] > a_box ? (dirty[st] - a_box) * BK : 0u;
      };
      auto zero_fill = [&](int st, uint32_t a_box, uint32_t zb) {
        if (zb != 0) bulk_load(a_s + st * kATileBytes + a_box * BK, p.zeros, zb, &full[st]);
        dirty[st] = a_box;
      };
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool withhold = p.inject_fault != 0 && cta == 0;
      // A rows of a tile that belong to its expert decide the A box height (16, 32, 64 or 128
      // rows; never more than the A region, which holds the host-chosen bm rows); the MMA still
      // reads 128 rows, the rest are leftovers whose accumulator rows are dropped.
      auto a_box_of = [&](const TileCoord& c) {
        return c.rows <= 16 ? 0 : c.rows <= 32 ? 1 : c.rows <= 64 ? 2 : 3;
      };
      auto load_b = [&](const TileCoord& c, int st, int kt) {
        if constexpr (MODE == 1) {
          // the tile's 128 gate rows and the matching 128 up rows (I rows further on) in one box
          // of the 3-D map [experts x {gate, up}][I][H]: gate half first, up half behind it
          tma_load_3d(b_s + st * kBTileBytes, &tmB, kt * BK, c.nt * 128, c.e * 2, &full[st]);
        } else {
          const int brow = c.e * p.rows_b + c.nt * NB;
          tma_load_2d(b_s + st * kBTileBytes, &tmB, kt * BK, brow, &full[st]);
        }
      };
      // The weights and the tile table were written before the previous kernel started, so
      // the first tile's first stages request their weight tiles before waiting for it; the
      // A rows and all scale factors follow the wait.  (Not with the withheld-stage test hook,
      // whose stage must stay empty.)
      int npre = 0;
      TileCursor cur(p, cta, n_ctas, total_tiles);
      if (cur.more() && !withhold) {
        const TileCoord c0 = decode_tile_entry(p, cta, cur.next);
        const uint32_t a_box = 16u << a_box_of(c0);
        npre = min(S, KT);
        for (int kt = 0; kt < npre; ++kt) {       // first use of these stages: nothing to wait for
          const uint32_t zb = zero_bytes(kt, a_box);
          mbar_arrive_expect_tx(&full[kt], kStageTxNoA + a_box * BK + zb);
          load_b(c0, kt, kt);
          zero_fill(kt, a_box, zb);
        }
      }
      griddep_wait();
      griddep_launch_dependents();
      // single-kernel forward: the A rows of every tile exist once the grid's scatter is done
      bool rows_ok = true;
      if (p.rows_ready != nullptr) {
        rows_ok = wait_counter(p.rows_ready, p.rows_ready_need, ctl.status, ctl.timeout_ns, kWhereGemmDependency,
                               ctl.abort_flag);
        if (!rows_ok) *ctl.abort_flag = 1;
        fence_proxy_async_global();          // the acquired rows before this thread's TMA reads
        if (p.stamp_rows != nullptr) p.stamp_rows[cta] = globaltimer_ns();
      }
      for (; cur.more() && ok; cur.advance()) {
        const int tile = cur.tile;
        const TileCoord c = cur.take(p);
        const uint8_t* sfa_tile = p.sfa + (long)c.gmt * KT * kSfaBytes;
        const uint8_t* sfb_tile = p.sfb + ((long)c.e * p.n_tiles_n + c.nt) * KT * kSfbBytes;
        const int a_sel = a_box_of(c);
        const uint32_t a_box = 16u << a_sel;
        // chained kernel: this tile's A rows exist once every linear1 tile of its expert is
        // stored (bounded wait; on expiry the stages already requested are still completed, so
        // that the drain below finds every copy accounted for, and nothing further is loaded)
        bool dep_ok = rows_ok;
        if (dep_ok && p.dep_wait != nullptr) {
          const uint32_t need = (uint32_t)(((c.count + p.bm - 1) / p.bm) * p.dep_per_mtile);
          dep_ok = wait_counter(p.dep_wait + c.e, need, ctl.status, ctl.timeout_ns, kWhereGemmDependency,
                                ctl.abort_flag);
          if (!dep_ok) *ctl.abort_flag = 1;
          fence_proxy_async_global();      // the acquired rows before this thread's TMA reads
        }
        for (int kt = 0; kt < KT; ++kt) {
          const bool pre = tile == cta && kt < npre;   // weight tile already requested
          if (!dep_ok && !pre) { ok = false; break; }
          if (!pre && !mbar_wait(&empty[stage], phase ^ 1, ctl, kWhereGemmProducer)) { ok = false; break; }
          if (withhold) {
            withhold = false;            // test hook: this stage never fills
          } else {
            if (!pre) {
              const uint32_t zb = zero_bytes(stage, a_box);
              mbar_arrive_expect_tx(&full[stage], kStageTxNoA + a_box * BK + zb);
              load_b(c, stage, kt);
              zero_fill(stage, a_box, zb);
            }
            tma_load_2d(a_s + stage * kATileBytes, &tmA.m[a_sel], kt * BK, c.row0, &full[stage]);
            bulk_load(sfa_s + stage * kSfaBytes, sfa_tile + kt * kSfaBytes, kSfaBytes, &full[stage]);
            bulk_load(sfb_s + stage * kSfbBytes, sfb_tile + kt * kSfbBytes, kSfbBytes, &full[stage]);
            fills[stage] += 1;
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      // wait for our own bulk copies before the CTA may exit (abort path)
#pragma unroll
      for (int s = 0; s < S; ++s) {
        if (fills[s] > 0 && !mbar_wait_drain(&full[s], (fills[s] - 1) & 1, p.timeout_ns)) {
          report_status(p.status, kStatusTimeout, kWhereGemmDrain, s);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t uses0 = 0, uses1 = 0;      // completed uses of each accumulator slot
      int next_slot = 0;
      bool ok = true;
      for (TileCursor cur(p, cta, n_ctas, total_tiles); cur.more() && ok; cur.advance()) {
        const TileCoord c = cur.take(p);
        const SlotPlan sp = plan_slots<TM::kDouble, kSwapOk>(p, c, next_slot);
        for (int sl = sp.lo; sl <= sp.hi && ok; ++sl)
          ok = mbar_wait(&acce[sl], ((sl ? uses1 : uses0) & 1) ^ 1, ctl, kWhereGemmMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem_base + kAccCol + sp.lo * TM::slot_stride;
        const uint32_t sfa_t = tmem_base + TM::sfa, sfb_t = tmem_base + TM::sfb;
        const uint32_t id_swap0 = idesc_mxf8f6f4(BM, sp.nt_tok, 0, 0, kFmtE2M1, kFmtE4M3);
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, ctl, kWhereGemmMma + 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_addr = smem_u32(sfa_s + stage * kSfaBytes);
          const uint32_t sfb_addr = smem_u32(sfb_s + stage * kSfbBytes);
          tc_cp_32x128b_warpx4(sfa_t, sf_desc(sfa_addr));
          tc_cp_32x128b_warpx4(sfb_t, sf_desc(sfb_addr));
          tc_cp_32x128b_warpx4(sfb_t + 4, sf_desc(sfb_addr + 512));
          const uint32_t a_addr = smem_u32(a_s + stage * kATileBytes);
          const uint32_t b_addr = smem_u32(b_s + stage * kBTileBytes);
          if (sp.swap) {
            // weights (E2M1, rows 0..127 and 128..255 of the B stage) as A, tokens (E4M3) as B;
            // the weight scale atoms are the A scales, the token atom the B scales
#pragma unroll
            for (int kb = 0; kb < BK / 32; ++kb) {
              const uint32_t id = id_swap0 | ((uint32_t)kb << 4) | ((uint32_t)kb << 29);
              tc_mma_mxf8f6f4(acc, sw128_desc(b_addr + kb * 32), sw128_desc(a_addr + kb * 32), id, sfb_t, sfa_t,
                              (kt | kb) != 0);
              tc_mma_mxf8f6f4(acc + 64, sw128_desc(b_addr + kBTileBytes / 2 + kb * 32),
                              sw128_desc(a_addr + kb * 32), id, sfb_t + 4, sfa_t, (kt | kb) != 0);
            }
          } else {
#pragma unroll
            for (int kb = 0; kb < BK / 32; ++kb) {
              tc_mma_mxf8f6f4(acc, sw128_desc(a_addr + kb * 32), sw128_desc(b_addr + kb * 32),
                              idesc_mxf8f6f4(BM, NB, kb, kb), sfa_t, sfb_t, (kt | kb) != 0);
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        for (int sl = sp.lo; sl <= sp.hi; ++sl) tc_commit(&accf[sl]);
        uses0 += sp.lo == 0;
        uses1 += sp.hi == 1;
      }
      // all MMAs this thread issued have finished once `drain` completes
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0, p.timeout_ns)) report_status(p.status, kStatusTimeout, kWhereGemmDrain, 9);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;      // which half of the accumulator columns
    uint8_t* obuf = L::kStaging ? smem + L::stage_out + (warp - 2) * 2048 : nullptr;
    const int epi_id = cta * kEpiWarps + (warp - 2), n_epi = n_ctas * kEpiWarps;
    pre(epi_id, n_epi, true, smem);
    uint32_t uses0 = 0, uses1 = 0;
    int next_slot = 0;
    int buf = 0;
    bool all_ok = true;
    for (TileCursor cur(p, cta, n_ctas, total_tiles); cur.more(); cur.advance()) {
      const TileCoord c = cur.take(p);
      const SlotPlan sp = plan_slots<TM::kDouble, kSwapOk>(p, c, next_slot);
      bool ok = true;
      for (int sl = sp.lo; sl <= sp.hi && ok; ++sl)
        ok = mbar_wait(&accf[sl], (sl ? uses1 : uses0) & 1, ctl, kWhereGemmEpilogue);
      // epilogue-uniform decision: tcgen05.ld below is .sync.aligned and the epilogue syncs
      if (!epi_all(ok)) {
        all_ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem_base + kAccCol + sp.lo * TM::slot_stride;
      if (kSwapOk && sp.swap) {
        if (sp.nt_tok == 32)
          epilogue_swap<MODE, 32, NB>(p, c, acc, q, half, lane, &acce[sp.lo], amax_s, buf);
        else
          epilogue_swap<MODE, 64, NB>(p, c, acc, q, half, lane, &acce[sp.lo], amax_s, buf);
      } else {
        epilogue_tile<MODE, NB, L::kAmaxRows>(p, c, acc, q, half, lane, TM::kDouble ? &acce[sp.lo] : acce, 0u,
                                              amax_s, buf, obuf);
      }
      if (p.dep_signal != nullptr || p.tiles_done != nullptr) {
        // chained kernel / single-kernel forward: publish this tile's rows (h and its scale words
        // to the linear2 producers; bf16 rows to the combine): generic stores -> other CTAs'
        // TMA or generic reads: proxy fence, CTA barrier, gpu-scope release
        fence_proxy_async_global();
        epi_bar();
        if (threadIdx.x == 2 * 32) {
          __threadfence();
          if (p.dep_signal != nullptr) atomicAdd(p.dep_signal + c.e, 1u);
          if (p.tiles_done != nullptr) atomicAdd(p.tiles_done, 1u);
        }
      }
      uses0 += sp.lo == 0;
      uses1 += sp.hi == 1;
      buf ^= 1;
    }
    post(epi_id, n_epi, all_ok && !*abort_flag, smem);
  }

  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < (int)L::n_bars; ++i) mbar_inval(bars + i);
  }
  __syncthreads();
}

template <int MODE, class L, int NB = 256>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc);
  const int warp = threadIdx.x / 32;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  gemm_body<MODE, L, NB>(tmA, tmB, p, smem, tmem_base, blockIdx.x, gridDim.x);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// linear1 then linear2 in one cooperative launch for few tokens (the few-row layout): each CTA
// runs its linear1 tiles, then its linear2 tiles, in one TMEM allocation.  linear2's producer
// requests its first weight stages as soon as the CTA's linear1 work is done and waits, per
// tile, only for the linear1 tiles of that tile's expert (g1.dep_signal == g2.dep_wait, zeroed
// before the launch) -- no grid-wide barrier and no second launch.  Co-residency of all CTAs
// (cooperative launch) guarantees that every awaited linear1 tile is being worked on.
template <int NB2>
__global__ void __launch_bounds__(kGemmThreads, 1)
    chained_gemm_kernel(const __grid_constant__ AMaps tmA1, const __grid_constant__ AMaps tmA2,
                        const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                        const GemmArgs g1, const GemmArgs g2) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmallSmem::misc);
  const int warp = threadIdx.x / 32;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  gemm_body<1, SmallSmem>(tmA1, tmB1, g1, smem, tmem_base, blockIdx.x, gridDim.x);
  gemm_body<2, SmallSmem, NB2>(tmA2, tmB2, g2, smem, tmem_base, blockIdx.x, gridDim.x);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ CTA-pair grouped GEMM
// Same tiles as above with two row tiles per CTA pair: rank r of a 2-CTA cluster holds row
// tile 2*pm + r of its expert (A, 128 rows) and half of the 256 B rows (linear1: rank 0 the
// gate rows, rank 1 the up rows; linear2: rows 128*r.. of the 256-row tile), and one
// tcgen05.mma.cta_group::2 (M = 256, N = 256) per 32-deep K step, issued by rank 0, writes
// each CTA's 128 x 256 accumulator into its own TMEM.  Each CTA loads its own scale atom and
// the full 256-row weight scale unit (both 2-D TMA), every copy completing on rank 0's stage
// barrier; rank 0's MMA commits multicast to both CTAs' empty / accumulator barriers; the
// epilogue warps of both CTAs release the accumulator on rank 0's barrier.  Half the B bytes
// per CTA leave room for 6 stages.
constexpr int SP = 6;
constexpr uint32_t kBHalfBytes = 128 * BK;               // 16 KB of shared memory (unpacked E2M1)
constexpr uint32_t kPairTxBytesNoA = 128 * BK / 2 + kSfaBytes + kSfbBytes;   // per CTA, without A

struct PairSmem {
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + SP * kATileBytes;
  static constexpr uint32_t sfa = b + SP * kBHalfBytes;
  static constexpr uint32_t sfb = sfa + SP * kSfaBytes;
  static constexpr uint32_t amax = sfb + SP * kSfbBytes;
  static constexpr uint32_t stage_out = amax + 2 * 2 * 128 * 4;
  static constexpr uint32_t bars = stage_out + 8 * 2048;
  // full[SP], empty[SP], accf, acce, drain
  static constexpr uint32_t n_bars = 2 * SP + 3;
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t total = misc + 16;
};

// Tile `tile` of the pair grid as seen by CTA `rank`: row tile 2*pm + rank of the expert (its
// rows can be 0 for rank 1 on an expert with an odd number of row tiles).
// The expert comes from the pair-tile table entry tile / n_tiles_n (as in decode_tile).
__device__ __forceinline__ TileCoord decode_pair_tile(const GemmArgs& p, int tile, int rank) {
  const int4 info = ld_cg_v4(p.ptile_info + tile / p.n_tiles_n);   // {e, ptile_start, count, offset}
  TileCoord c;
  c.e = info.x;
  c.count = info.z;
  const int mtiles = (c.count + BM - 1) / BM;
  const int ptiles = (mtiles + 1) / 2;
  const int local = tile - info.y * p.n_tiles_n;
  int pm;
  banded_mn(local, ptiles, p.n_tiles_n, pm, c.nt);
  c.mt = 2 * pm + rank;
  c.row0 = info.w + c.mt * BM;
  c.gmt = ld_cg(p.mtile_start + c.e) + c.mt;
  c.rows = max(0, min(BM, c.count - c.mt * BM));
  return c;
}

__device__ __forceinline__ int a_box_sel(int rows) { return rows <= 16 ? 0 : rows <= 32 ? 1 : rows <= 64 ? 2 : 3; }

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ AMaps tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmSfa, const __grid_constant__ CUtensorMap tmSfb,
                             const GemmArgs p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem + PairSmem::a;
  uint8_t* b_s = smem + PairSmem::b;
  uint8_t* sfa_s = smem + PairSmem::sfa;
  uint8_t* sfb_s = smem + PairSmem::sfb;
  float* amax_s = reinterpret_cast<float*>(smem + PairSmem::amax);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PairSmem::bars);
  uint64_t* full = bars;
  uint64_t* empty = bars + SP;
  uint64_t* accf = bars + 2 * SP;
  uint64_t* acce = accf + 1;
  uint64_t* drain = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PairSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PairSmem::misc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SP; ++s) {
      mbar_init(&full[s], 1);          // rank 0's: its producer's arrive + both CTAs' bytes
      mbar_init(&empty[s], 1);         // each CTA's: rank 0's multicast commit
    }
    mbar_init(accf, 1);                // each CTA's: rank 0's multicast commit
    mbar_init(acce, 2 * kEpiWarps);    // rank 0's: the epilogue warps of both CTAs
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) tma_prefetch_desc(&tmA.m[i]);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSfa);
    tma_prefetch_desc(&tmSfb);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync();                      // the peer's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total_tiles = ld_cg(p.ptile_start + p.n_experts) * p.n_tiles_n;
  const int KT = p.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t fills[SP];
#pragma unroll
      for (int s = 0; s < SP; ++s) fills[s] = 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        const TileCoord c = decode_pair_tile(p, tile, rank);
        const int a_sel = a_box_sel(c.rows);
        // rank 0 expects the bytes of both CTAs: the peer's A box follows from its rows
        const int peer_rows = max(0, min(BM, c.count - (c.mt + 1) * BM));
        const uint32_t tx = 2 * kPairTxBytesNoA + ((16u << a_sel) + (16u << a_box_sel(peer_rows))) * BK;
        const int brow = MODE == 1 ? c.e * p.rows_b + rank * p.N + c.nt * 128 : c.e * p.rows_b + c.nt * BN + rank * 128;
        const int sfa_row = (c.gmt * KT) * 2;
        const int sfb_row = ((c.e * p.n_tiles_n + c.nt) * KT) * 4;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctl, kWhereGemmProducer)) { ok = false; break; }
          const uint32_t fb = mapa_shared(&full[stage], 0);
          if (rank == 0) {
            mbar_arrive_expect_tx(&full[stage], tx);
            fills[stage] += 1;
          }
          tma_load_2d_pair(a_s + stage * kATileBytes, &tmA.m[a_sel], kt * BK, c.row0, fb);
          tma_load_2d_pair(b_s + stage * kBHalfBytes, &tmB, kt * BK, brow, fb);
          tma_load_2d_pair(sfa_s + stage * kSfaBytes, &tmSfa, 0, sfa_row + kt * 2, fb);
          tma_load_2d_pair(sfb_s + stage * kSfbBytes, &tmSfb, 0, sfb_row + kt * 4, fb);
          if (++stage == SP) { stage = 0; phase ^= 1; }
        }
      }
      // rank 0's stage barriers count both CTAs' copies: waiting for them covers the peer too
#pragma unroll
      for (int s = 0; s < SP; ++s) {
        if (fills[s] > 0 && !mbar_wait_drain(&full[s], (fills[s] - 1) & 1, p.timeout_ns)) {
          report_status(p.status, kStatusTimeout, kWhereGemmDrain, s);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        if (!mbar_wait(acce, acc_phase ^ 1, ctl, kWhereGemmMma)) break;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, ctl, kWhereGemmMma + 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_addr = smem_u32(sfa_s + stage * kSfaBytes);
          const uint32_t sfb_addr = smem_u32(sfb_s + stage * kSfbBytes);
          tc_cp_32x128b_warpx4_pair(tmem_base + kSfaCol, sf_desc(sfa_addr));
          tc_cp_32x128b_warpx4_pair(tmem_base + kSfbCol, sf_desc(sfb_addr));
          tc_cp_32x128b_warpx4_pair(tmem_base + kSfbCol + 4, sf_desc(sfb_addr + 512));
          const uint32_t a_addr = smem_u32(a_s + stage * kATileBytes);
          const uint32_t b_addr = smem_u32(b_s + stage * kBHalfBytes);
#pragma unroll
          for (int kb = 0; kb < BK / 32; ++kb) {
            tc_mma_mxf8f6f4_pair(tmem_base + kAccCol, sw128_desc(a_addr + kb * 32), sw128_desc(b_addr + kb * 32),
                                 idesc_mxf8f6f4(2 * BM, BN, kb, kb), tmem_base + kSfaCol, tmem_base + kSfbCol,
                                 (kt | kb) != 0);
          }
          tc_commit_pair(&empty[stage], 0x3);
          if (++stage == SP) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit_pair(accf, 0x3);
        acc_phase ^= 1;
      }
      tc_commit_pair(drain, 0x1);
      if (!mbar_wait_drain(drain, 0, p.timeout_ns)) report_status(p.status, kStatusTimeout, kWhereGemmDrain, 9);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9, both CTAs)
    const int q = warp & 3;
    const int half = (warp - 2) / 4;
    uint8_t* obuf = smem + PairSmem::stage_out + (warp - 2) * 2048;
    const uint32_t acce0 = mapa_shared(acce, 0);
    uint32_t acc_phase = 0;
    int buf = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const TileCoord c = decode_pair_tile(p, tile, rank);
      const bool ok = mbar_wait(accf, acc_phase, ctl, kWhereGemmEpilogue);
      if (!epi_all(ok)) break;
      tc_fence_after();
      epilogue_tile<MODE>(p, c, tmem_base, q, half, lane, acce, acce0, amax_s, buf, obuf);
      acc_phase ^= 1;
      buf ^= 1;
    }
  }

  __syncthreads();
  cluster_sync();                      // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Weight scale factors, canonical [n][rows_b][K/32] UE8M0 -> tiled atoms.
// Block per (expert, 128-row group): the group's K/32-byte rows are staged in
// shared memory, then written as K/128 atoms of 512 bytes (row r at byte
// (r%32)*16 + (r/32)*4, its 4 K-blocks at +0..3).  linear1 groups pair gate
// rows j.. and up rows I + j.. of one 128-channel block into a 1024-byte unit;
// linear2 groups pair row blocks 2t and 2t+1 of a 256-row tile.
__global__ void __launch_bounds__(256) tile_weight_scales_kernel(const uint8_t* __restrict__ src,
                                                                 uint8_t* __restrict__ dst, int rows_b, int K,
                                                                 int n_tiles_n, int mode, int N, int tile_rows) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ uint32_t sm[];                // [128 rows][K/128 words]
  const int kw = K / 128;
  const int e = blockIdx.y;
  const int grp = blockIdx.x;                     // 128-row group within the expert's B rows
  // which (n-tile, half) this group fills
  int nt, hf, row_first;
  if (mode == 1) {                                // rows_b = 2N: groups 0..N/128-1 gate, N/128.. up
    const int ng = N / 128;
    hf = grp >= ng;
    nt = grp - hf * ng;
    row_first = grp * 128;
  } else {                                        // rows_b = H (=N): tile_rows-row tiles, 2 halves
    nt = grp / 2;
    hf = grp % 2;
    row_first = nt * tile_rows + hf * 128;
  }
  const uint32_t* s32 = reinterpret_cast<const uint32_t*>(src);
  for (int i = threadIdx.x; i < 128 * kw; i += blockDim.x) {
    const int r = i / kw, w = i % kw;
    const int row = row_first + r;
    sm[i] = row < rows_b ? s32[((long)e * rows_b + row) * kw + w] : 0x7F7F7F7Fu;
  }
  __syncthreads();
  uint8_t* out = dst + ((long)e * n_tiles_n + nt) * kw * 1024 + hf * 512;
  for (int i = threadIdx.x; i < 32 * kw; i += blockDim.x) {
    const int kt = i / 32, r0 = i % 32;           // 16-byte chunk r0 of atom kt
    uint4 v;
    v.x = sm[(r0 + 0) * kw + kt];
    v.y = sm[(r0 + 32) * kw + kt];
    v.z = sm[(r0 + 64) * kw + kt];
    v.w = sm[(r0 + 96) * kw + kt];
    *reinterpret_cast<uint4*>(out + (long)kt * 1024 + r0 * 16) = v;
  }
}

// ------------------------------------------------------------------ router on tensor cores
// logits[t][e] = sum_h x[t][h] * (W_hi[e][h] + W_lo[e][h]) with W = W_hi + W_lo + r, W_hi and W_lo
// bf16 (|r| <= 2^-18 |W|): two bf16 MMAs per K slice into one fp32 accumulator.
// One CTA per (128-token, 128-expert) tile: warp 0 TMA, warp 1 MMA (+TMEM), warps 2..5 epilogue.
constexpr int RBK = 64;                                 // bf16 elements per stage = 128 bytes
constexpr int RBN = 128;
constexpr int RS = 4;
constexpr uint32_t kRTile = 128 * 128;                  // bytes of one 128-row x 128-byte tile

struct RouterSmem {
  static constexpr uint32_t a = 0;
  static constexpr uint32_t bh = a + RS * kRTile;
  static constexpr uint32_t bl = bh + RS * kRTile;
  static constexpr uint32_t bars = bl + RS * kRTile;    // full[RS], empty[RS], accf, drain
  static constexpr uint32_t misc = bars + (2 * RS + 2) * 8;
  static constexpr uint32_t total = misc + 16;
};

// One router tile (128 tokens from m0, 128 experts from n0, K split `split` of `n_splits`)
// by all threads of the CTA; warps 0..5 work (TMA, MMA, 4 x epilogue), any others only join
// the CTA barriers.  TMEM columns [tmem_base, tmem_base + 128) are the accumulator.
// Initialises its barriers on entry and invalidates them on exit.
__device__ __forceinline__ void router_tc_item(const CUtensorMap& tmX, const CUtensorMap& tmWhi,
                                               const CUtensorMap& tmWlo, const RouterArgs& p, uint8_t* smem,
                                               uint32_t tmem_base, int m0, int n0, int split, int n_splits) {
  uint8_t* a_s = smem + RouterSmem::a;
  uint8_t* bh_s = smem + RouterSmem::bh;
  uint8_t* bl_s = smem + RouterSmem::bl;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RouterSmem::bars);
  uint64_t* empty = full + RS;
  uint64_t* accf = full + 2 * RS;
  uint64_t* drain = accf + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + RouterSmem::misc + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // stages [kt0, kt0 + KT) of this split; partial logits in slice `split`
  const int KT = p.H / RBK / n_splits;
  const int kt0 = split * KT;
  float* const logits = p.logits + (long)split * p.T * p.E;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  tc_fence_after();
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  if (warp == 0) {
    if (lane == 0) {
      uint32_t fills[RS];
#pragma unroll
      for (int s = 0; s < RS; ++s) fills[s] = 0;
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1, ctl, kWhereRouterProducer)) break;
        mbar_arrive_expect_tx(&full[stage], 3 * kRTile);
        const int kx = (kt0 + kt) * RBK;
        tma_load_2d(a_s + stage * kRTile, &tmX, kx, m0, &full[stage]);
        tma_load_2d(bh_s + stage * kRTile, &tmWhi, kx, n0, &full[stage]);
        tma_load_2d(bl_s + stage * kRTile, &tmWlo, kx, n0, &full[stage]);
        fills[stage] += 1;
        if (++stage == RS) { stage = 0; phase ^= 1; }
      }
#pragma unroll
      for (int s = 0; s < RS; ++s)
        if (fills[s] > 0 && !mbar_wait_drain(&full[s], (fills[s] - 1) & 1, p.timeout_ns))
          report_status(p.status, kStatusTimeout, kWhereGemmDrain, 0x20 + s);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      constexpr uint32_t idesc = idesc_bf16(128, RBN);
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait(&full[stage], phase, ctl, kWhereRouterMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(a_s + stage * kRTile);
        const uint32_t bh_addr = smem_u32(bh_s + stage * kRTile);
        const uint32_t bl_addr = smem_u32(bl_s + stage * kRTile);
#pragma unroll
        for (int kb = 0; kb < RBK / 16; ++kb)
          tc_mma_bf16(tmem_base, sw128_desc(a_addr + kb * 32), sw128_desc(bh_addr + kb * 32), idesc, (kt | kb) != 0);
#pragma unroll
        for (int kb = 0; kb < RBK / 16; ++kb)
          tc_mma_bf16(tmem_base, sw128_desc(a_addr + kb * 32), sw128_desc(bl_addr + kb * 32), idesc, 1);
        tc_commit(&empty[stage]);
        if (++stage == RS) { stage = 0; phase ^= 1; }
      }
      if (ok) tc_commit(accf);
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0, p.timeout_ns)) report_status(p.status, kStatusTimeout, kWhereGemmDrain, 0x29);
    }
  } else if (warp < kRouterThreads / 32) {
    const int q = warp & 3;
    const bool ok = mbar_wait(accf, 0, ctl, kWhereRouterEpilogue);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int t = m0 + q * 32 + lane;
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
#pragma unroll
      for (int ch = 0; ch < RBN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + ch * 32, r);
        tmem_ld_wait();
        const int e0 = n0 + ch * 32;
        if (t < p.T) {
          float* dst = logits + (long)t * p.E + e0;
          if (e0 + 32 <= p.E) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              *reinterpret_cast<float4*>(dst + 4 * v) =
                  make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                              __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (e0 + i < p.E) dst[i] = __uint_as_float(r[i]);
          }
        }
      }
      tc_fence_before();
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * RS + 2; ++i) mbar_inval(full + i);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWhi,
                     const __grid_constant__ CUtensorMap tmWlo, const RouterArgs p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + RouterSmem::misc);
  const int warp = threadIdx.x / 32;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  router_tc_item(tmX, tmWhi, tmWlo, p, smem, tmem_base, blockIdx.y * 128, blockIdx.x * RBN, blockIdx.z, gridDim.z);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

// W fp32 -> (hi, lo) bf16 with hi = bf16(W), lo = bf16(W - hi) (W - hi is exact in fp32).
__global__ void split_router_weights_kernel(const float* __restrict__ W, __nv_bfloat16* __restrict__ hi,
                                            __nv_bfloat16* __restrict__ lo, long n) {
  griddep_wait();
  griddep_launch_dependents();
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const float w = W[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(w);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(w - __bfloat162float(h));
  }
}

// ------------------------------------------------------------------ the single persistent forward
// Shared memory of the fused kernel: the largest step layout, then the kernel-lifetime words.
template <class L>
struct FusedSmem {
  static constexpr uint32_t misc = (L::total + 15) & ~15u;
  static constexpr uint32_t bytes = misc + 16 + 1024;
  static_assert(misc >= RouterSmem::total && misc >= sizeof(TopkSmem) + 3 * 32 * 4,
                "every step's shared memory must fit below the fused kernel's own words");
  static_assert(bytes <= 232448, "fused kernel exceeds shared memory");
};
// Grid-wide barrier for a cooperative launch: bar[0] counts arrivals, bar[1] is the
// generation the last arrival advances.  The wait is bounded; on expiry the CTA records
// MOE_ERR_DEVICE_TIMEOUT and the barrier reports false.  All threads call it.
__device__ __forceinline__ bool grid_sync(uint32_t* bar, uint32_t n_ctas, uint32_t* status, uint64_t timeout_ns,
                                          volatile int* ok_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    // the CTA's writes are ordered before its release-add; the last arrival acquires them all
    // and releases the next generation, which every waiting CTA acquires
    const uint32_t gen = ld_acquire_gpu(&bar[1]);
    if (atom_add_acq_rel_gpu(&bar[0], 1u) == n_ctas - 1) {
      bar[0] = 0u;
      st_release_gpu(&bar[1], gen + 1);
    } else {
      const uint64_t t0 = globaltimer_ns();
      uint32_t pause = 32;
      while (ld_relaxed_gpu(&bar[1]) == gen) {
        if (globaltimer_ns() - t0 > timeout_ns) {
          report_status(status, kStatusTimeout, kWhereGridBarrier, gen);
          ok = false;
          break;
        }
        poll_pause(pause);
      }
      fence_acq_rel_gpu();
    }
    *ok_smem = ok && ld_acquire_gpu(status) == 0u;
  }
  __syncthreads();
  return *ok_smem != 0;
}

constexpr int kScatterBulkSlices = 8;

// Before its first linear1 tile, each epilogue warp of the grid scatters (and quantises) its
// share of the (token, channel group) items; once all eight of a CTA's have, one thread adds 1 to
// the scatter counter (one atomic per CTA, not per warp); the producers load A rows only once
// every CTA has done so.
template <class L>
struct ScatterWork {
  const FusedArgs* a;
  __device__ __forceinline__ void operator()(int epi_id, int n_epi, bool, uint8_t* smem) const {
    const FusedArgs& f = *a;
    const int slices = (f.H + 255) / 256;
    bool pending = false;
    if (L::kStaging && (long)f.T * slices >= 32768) {
      // many items: eight slices per item through the warp's 2 KB of staging memory
      uint8_t* stage = smem + L::stage_out + (epi_id % kEpiWarps) * 2048;
      const long items = (long)f.T * ((slices + kScatterBulkSlices - 1) / kScatterBulkSlices);
      for (long it = epi_id; it < items; it += n_epi)
        scatter_items_bulk<kScatterBulkSlices>(it, f.x, f.topk_ids, f.local_rank, f.group_base, f.offsets,
                                               f.mtile_start, f.slot_pos, f.perm, f.xq, f.xsf, f.T, f.H, f.E, f.k,
                                               f.shared, f.bm, stage, pending);
    } else {
      const long items = (long)f.T * slices;
      for (long it = epi_id; it < items; it += n_epi)
        scatter_item(it, f.x, f.topk_ids, f.local_rank, f.group_base, f.offsets, f.mtile_start, f.slot_pos, f.perm,
                     f.xq, f.xsf, f.T, f.H, f.E, f.k, f.shared, f.bm);
    }
    // bulk copies complete (their writes performed), generic stores -> other CTAs' TMA reads:
    // proxy fence, CTA barrier, gpu-scope release
    scatter_bulk_drain(pending, f.k, f.shared);
    fence_proxy_async_global();
    epi_bar();
    if (threadIdx.x == 2 * 32) {
      if (f.stamps != nullptr) f.stamps[kStampScatterDone * kStampMaxCtas + blockIdx.x] = globaltimer_ns();
      __threadfence();
      atomicAdd(f.counters + 0, 1u);
    }
  }
};

// After its last linear2 tile, each epilogue warp waits (bounded) until every linear2 tile of
// the grid is stored, then combines its share of the (token, channel chunk) items.  With one CTA
// per SM only eight warps per SM do this, so they gather with bulk copies into the operand stage
// buffers (idle once the CTA's last linear2 tile is done): per item, lane j < k + shared copies
// expert row j's chunk (1024 channels, 2 KB; 512 when k + shared > 12 rows would not fit) into
// the warp's slice of that memory, completing on one mbarrier of the warp (in the amax area,
// which linear2 does not use); the lanes then sum the rows from shared memory in slot order,
// gate-weighted, add the shared row and store bf16.
template <class L>
struct CombineWork {
  static constexpr uint32_t kSlice = ((L::sfa - L::a) / kEpiWarps) & ~1023u;   // per warp
  static_assert(kSlice >= 12 * 2048 && kSlice >= 17 * 1024, "a warp's slice holds one item");
  static_assert(L::stage_out - L::amax >= kEpiWarps * 8, "the amax area holds the combine barriers");
  const FusedArgs* a;
  uint32_t tiles2;                 // linear2 tiles of the forward

  template <int CW>
  __device__ __forceinline__ bool run(int epi_id, int n_epi, uint8_t* buf, uint64_t* bar) const {
    const FusedArgs& f = *a;
    const int lane = threadIdx.x % 32;
    const int R = f.k + f.shared;                        // rows per item
    const int chunks = (f.H + CW - 1) / CW;
    const long items = (long)f.T * chunks;
    const long Rk = (long)f.T * f.k;
    uint32_t parity = 0;
    for (long it = epi_id; it < items; it += n_epi) {
      const int t = (int)(it / chunks);
      const int c0 = (int)(it % chunks) * CW;
      const int w_ch = min(CW, f.H - c0);                // channels of this chunk (a multiple of 128)
      long row = 0;
      float g = 0.f;
      if (lane < f.k) {
        row = ld_cg(f.slot_pos + (long)t * f.k + lane);
        g = f.gates[(long)t * f.k + lane];
      } else if (lane < R) {
        row = Rk + t;                                    // the shared expert's row
        g = 1.f;
      }
      if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(R * w_ch * 2));
      __syncwarp();
      if (lane < R) bulk_load(buf + lane * (CW * 2), f.y + row * f.H + c0, (uint32_t)w_ch * 2, bar);
      if (!__all_sync(0xffffffffu, mbar_wait_drain(bar, parity, f.timeout_ns))) {
        if (lane == 0) report_status(f.status, kStatusTimeout, kWhereGemmDrain + 2, (uint32_t)it);
        return false;                  // (the barrier stays valid; nothing else uses this memory)
      }
      parity ^= 1;
      // lane: 8 channels in each 256-channel group of the chunk
#pragma unroll
      for (int q4 = 0; q4 < CW / 256; ++q4) {
        const int ch = q4 * 256 + lane * 8;
        const bool live = ch < w_ch;                     // warp-uniform per half-warp (128-channel steps)
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int r = 0; r < R; ++r) {
          const float gr = __shfl_sync(0xffffffffu, g, r);             // every lane takes part
          if (!live) continue;
          const uint4 v = *reinterpret_cast<const uint4*>(buf + r * (CW * 2) + ch * 2);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          if (r < f.k) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[2 * q] = fmaf(gr, __uint_as_float(wv[q] << 16), acc[2 * q]);
              acc[2 * q + 1] = fmaf(gr, __uint_as_float(wv[q] & 0xFFFF0000u), acc[2 * q + 1]);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[2 * q] += __uint_as_float(wv[q] << 16);
              acc[2 * q + 1] += __uint_as_float(wv[q] & 0xFFFF0000u);
            }
          }
        }
        uint4 o;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[0], acc[1]);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[2], acc[3]);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[4], acc[5]);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(acc[6], acc[7]);
        o.x = *reinterpret_cast<uint32_t*>(&b0);
        o.y = *reinterpret_cast<uint32_t*>(&b1);
        o.z = *reinterpret_cast<uint32_t*>(&b2);
        o.w = *reinterpret_cast<uint32_t*>(&b3);
        if (live) *reinterpret_cast<uint4*>(f.out + (long)t * f.H + c0 + ch) = o;
      }
      __syncwarp();                    // every lane has read the item before the next copies land
    }
    return true;
  }

  __device__ __forceinline__ void operator()(int epi_id, int n_epi, bool ok, uint8_t* smem) const {
    const FusedArgs& f = *a;
    if (!__all_sync(0xffffffffu, ok)) return;             // warp-uniform from here on
    const int lane = threadIdx.x % 32;
    // lane 0 polls for the warp
    bool ready = true;
    if (lane == 0)
      ready = wait_counter(f.counters + 1, tiles2, f.status, f.timeout_ns, kWhereGemmDependency + 1, nullptr);
    ready = __shfl_sync(0xffffffffu, ready, 0);
    if (!ready) return;
    __syncwarp();
    fence_proxy_async_global();            // the acquired rows, before this lane's bulk copies
    if (f.stamps != nullptr && threadIdx.x == 2 * 32) f.stamps[kStampCombine * kStampMaxCtas + blockIdx.x] = globaltimer_ns();
    const int w = epi_id % kEpiWarps;
    uint8_t* buf = smem + L::a + w * kSlice;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::amax) + w;
    if (lane == 0) {
      mbar_init(bar, 1);
      fence_mbarrier_init();
    }
    __syncwarp();
    const bool done = f.k + f.shared <= 12 ? run<1024>(epi_id, n_epi, buf, bar) : run<512>(epi_id, n_epi, buf, bar);
    if (done && lane == 0) mbar_inval(bar);
  }
};

template <class L, int NB2>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fused_forward_kernel(const __grid_constant__ AMaps amA1, const __grid_constant__ AMaps amA2,
                         const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                         const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWhi,
                         const __grid_constant__ CUtensorMap tmWlo, const FusedArgs a) {
  using FS = FusedSmem<L>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // kernel-lifetime words past every step's own layout
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + FS::misc);
  volatile int* ok_smem = reinterpret_cast<volatile int*>(smem + FS::misc + 8);
  const int warp = threadIdx.x / 32;
  constexpr int NW = kGemmThreads / 32;
  const int cta = blockIdx.x, n_ctas = gridDim.x;
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  // the readiness counters start at zero (visible to every CTA after the first grid barrier)
  if (cta == 0)
    for (int i = threadIdx.x; i < 2 + a.E + a.shared; i += blockDim.x) a.counters[i] = 0u;
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long wstride = (long)n_ctas * NW, wfirst = (long)cta * NW + warp;
  const int G = (a.T + 31) / 32;
  auto stamp = [&](int id) {
    if (a.stamps != nullptr && threadIdx.x == 0) a.stamps[id * kStampMaxCtas + cta] = globaltimer_ns();
  };
  stamp(kStampStart);

  bool ok = true;
  // S1 router
  if (a.router_kind == kRouterTensor) {
    const int mt = (a.T + 127) / 128, nt = (a.E + RBN - 1) / RBN;
    for (int it = cta; it < mt * nt * a.router_parts; it += n_ctas) {
      const int split = it % a.router_parts, tile = it / a.router_parts;
      router_tc_item(tmX, tmWhi, tmWlo, a.ra, smem, tmem_base, (tile / nt) * 128, (tile % nt) * RBN, split,
                     a.router_parts);
    }
  } else if (a.router_kind == kRouterSplitK) {
    router_splitk_items<kSplitKMaxT, kSplitKMaxChunks>(a.x, a.W_router, a.logits, a.T, a.H, a.E, a.router_parts,
                                                       wfirst, wstride);
  } else if (a.router_kind == kRouterSplitBlock) {
    float* part = reinterpret_cast<float*>(smem);
    for (int it = cta; it < a.E * a.T; it += n_ctas)
      router_split_block<kGemmThreads>(a.x, a.W_router, a.logits, a.T, a.H, a.E, it % a.E, it / a.E, part);
  } else if (a.router_kind == kRouterWarp8) {
    router_warp_items<8>(a.x, a.W_router, a.logits, a.T, a.H, a.E, wfirst, wstride);
  } else {
    router_warp_items<2>(a.x, a.W_router, a.logits, a.T, a.H, a.E, wfirst, wstride);
  }
  if (a.stamps != nullptr) {
    __syncthreads();
    stamp(kStampRouterDone);
  }
  ok = grid_sync(a.gridbar, n_ctas, a.status, a.timeout_ns, ok_smem);
  stamp(kStampRouted);
  // S2 + dispatch scans
  if (G == 1) {
    // one token group: top-k, ranks, counts and the expert scan in CTA 0 (the group's per-expert
    // masks stay in shared memory)
    if (ok && cta == 0) {
      TopkSmem& tsm = *reinterpret_cast<TopkSmem*>(smem);
      int32_t(*wsum)[32] = reinterpret_cast<int32_t(*)[32]>(smem + sizeof(TopkSmem));
      topk_rank_group<kGemmThreads>(0, 0, a.logits, a.router_parts, a.bias, a.topk_ids, a.gates, a.local_rank,
                                    a.group_counts, a.status, a.T, a.E, a.k, tsm);
      stamp(kStampTopkDone);
      // topk_rank_group leaves the masks in place (its last barrier follows the count writes)
      int32_t* cnt_s = reinterpret_cast<int32_t*>(tsm.mask);
      for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        const int c = __popc(tsm.mask[e]);
        cnt_s[e] = c;
        a.counts[e] = c;
        a.group_base[e] = 0;
      }
      __syncthreads();
      expert_scan_block<kGemmThreads>(a.counts, a.offsets, a.mtile_start, a.ptile_start, a.tile_info, a.ptile_info,
                                      a.T, a.E, a.shared, a.bm, wsum, cnt_s);
      stamp(kStampScanDone);
    }
  } else {
    if (ok) {
      TopkSmem& tsm = *reinterpret_cast<TopkSmem*>(smem);
      for (int g = cta; g < G; g += n_ctas)
        topk_rank_group<kGemmThreads>(g, 0, a.logits, a.router_parts, a.bias, a.topk_ids, a.gates, a.local_rank,
                                      a.group_counts, a.status, a.T, a.E, a.k, tsm);
      stamp(kStampTopkDone);
    }
    ok = grid_sync(a.gridbar, n_ctas, a.status, a.timeout_ns, ok_smem) && ok;
    if (ok)
      for (long e = wfirst; e < a.E; e += wstride)
        column_scan_warp((int)e, a.group_counts, a.group_base, a.counts, G, a.E);
    ok = grid_sync(a.gridbar, n_ctas, a.status, a.timeout_ns, ok_smem) && ok;
    if (ok && cta == 0) {
      expert_scan_block<kGemmThreads>(a.counts, a.offsets, a.mtile_start, a.ptile_start, a.tile_info, a.ptile_info,
                                      a.T, a.E, a.shared, a.bm, reinterpret_cast<int32_t(*)[32]>(smem));
      stamp(kStampScanDone);
    }
  }
  ok = grid_sync(a.gridbar, n_ctas, a.status, a.timeout_ns, ok_smem) && ok;
  stamp(kStampScanned);
  // S3 scatter (epilogue warps, before their first linear1 tile) + S4 linear1: the producers
  // stream weights at once and load A rows once every epilogue warp of the grid has scattered
  if (ok) {
    GemmArgs g1 = a.g1;
    g1.rows_ready = a.counters + 0;
    g1.rows_ready_need = (uint32_t)n_ctas;
    g1.dep_signal = a.counters + 2;
    g1.stamp_rows = a.stamps != nullptr ? a.stamps + kStampRowsReady * kStampMaxCtas : nullptr;
    gemm_body<1, L, 256, ScatterWork<L>>(amA1, tmB1, g1, smem, tmem_base, cta, n_ctas, ScatterWork<L>{&a});
    stamp(kStampLinear1);
    // S5 linear2: each tile's producer waits only for its expert's linear1 tiles; S6 combine by
    // the epilogue warps once every linear2 tile is stored
    GemmArgs g2 = a.g2;
    g2.dep_wait = a.counters + 2;
    g2.dep_per_mtile = a.g1.n_tiles_n;
    g2.tiles_done = a.counters + 1;
    const uint32_t tiles2 = (uint32_t)(ld_cg(a.mtile_start + a.E + a.shared) * a.g2.n_tiles_n);
    gemm_body<2, L, NB2, NoEpilogueWork, CombineWork<L>>(amA2, tmB2, g2, smem, tmem_base, cta, n_ctas,
                                                         NoEpilogueWork(), CombineWork<L>{&a, tiles2});
    stamp(kStampEnd);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

size_t router_tc_smem_bytes() { return RouterSmem::total + 1024; }

int router_tc_splits(int T, int H, int E) {
  if (E > kTopkMaxSplitE) return 1;
  const long tiles = (long)((T + 127) / 128) * ((E + RBN - 1) / RBN);
  const int kt = H / RBK;
  int best = 1;
  for (int s = 2; s <= 16; ++s)
    if (kt % s == 0 && tiles * s <= 148 && (long)s * T * E <= (4l << 20)) best = s;
  return best;
}

cudaError_t launch_router_tc(const CUtensorMap& x, const CUtensorMap& whi, const CUtensorMap& wlo,
                             const RouterArgs& args, cudaStream_t s) {
  if (args.k_splits < 1 || (args.H / RBK) % args.k_splits != 0) return cudaErrorInvalidValue;
  dim3 grid((args.E + RBN - 1) / RBN, (args.T + 127) / 128, args.k_splits);
  router_tc_kernel<<<grid, kRouterThreads, router_tc_smem_bytes(), s>>>(x, whi, wlo, args);
  return cudaGetLastError();
}

cudaError_t launch_split_router_weights(const float* W, uint16_t* hi, uint16_t* lo, long n, cudaStream_t s) {
  split_router_weights_kernel<<<296, 256, 0, s>>>(W, reinterpret_cast<__nv_bfloat16*>(hi),
                                                  reinterpret_cast<__nv_bfloat16*>(lo), n);
  return cudaGetLastError();
}

size_t gemm_smem_bytes() { return SmemLayout::total + 1024; }
size_t gemm_small_smem_bytes() { return SmallSmem::total + 1024; }
size_t gemm_pair_smem_bytes() { return PairSmem::total + 1024; }
int g_fused_ctas[64] = {};
struct FusedVariant {
  const void* fn;
  size_t smem;
};
int g_pair_clusters[64] = {};

cudaError_t gemm_prepare_device() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<1, SmemLayout>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<1, SmallSmem>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_small_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<2, SmallSmem>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_small_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<2, SmallSmem, kGemmBN2Double>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_small_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<2, SmemLayout, kGemmBN2Double>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(chained_gemm_kernel<kGemmBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_small_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(chained_gemm_kernel<kGemmBN2Double>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_small_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tile_weight_scales_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)router_tc_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<2, SmemLayout>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes());
  if (e != cudaSuccess) return e;
  for (int mode = 1; mode <= 2; ++mode) {
    const void* fn = mode == 1 ? (const void*)grouped_gemm_pair_kernel<1> : (const void*)grouped_gemm_pair_kernel<2>;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gemm_pair_smem_bytes());
    if (e != cudaSuccess) return e;
  }
  // co-resident pairs: a persistent grid of more clusters than fit would run in two waves
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 148, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = gemm_pair_smem_bytes();
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, (const void*)grouped_gemm_pair_kernel<1>, &cfg);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) g_pair_clusters[dev] = clusters;
  // the fused forward: one CTA per SM, all co-resident (cooperative launch); every variant has the
  // same block shape and (nearly) all of shared memory, so the smallest co-resident count counts
  int per_sm_min = 1 << 30, sms = 0, coop = 0;
  const FusedVariant variants[] = {
      {(const void*)fused_forward_kernel<SmemLayout, kGemmBN>, FusedSmem<SmemLayout>::bytes},
      {(const void*)fused_forward_kernel<SmemLayout, kGemmBN2Double>, FusedSmem<SmemLayout>::bytes},
      {(const void*)fused_forward_kernel<SmallSmem, kGemmBN>, FusedSmem<SmallSmem>::bytes},
      {(const void*)fused_forward_kernel<SmallSmem, kGemmBN2Double>, FusedSmem<SmallSmem>::bytes}};
  for (const FusedVariant& v : variants) {
    e = cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)v.smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, kGemmThreads, v.smem)) != cudaSuccess)
      return e;
    per_sm_min = per_sm < per_sm_min ? per_sm : per_sm_min;
  }
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) g_fused_ctas[dev] = coop ? per_sm_min * sms : 0;
  return cudaSuccess;
}

int fused_max_ctas() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  return g_fused_ctas[dev];
}

cudaError_t launch_fused_forward(const AMaps& a1, const AMaps& a2, const CUtensorMap& b1, const CUtensorMap& b2,
                                 const CUtensorMap& x, const CUtensorMap& whi, const CUtensorMap& wlo,
                                 const FusedArgs& args, int ctas, bool small_tiles, cudaStream_t s) {
  if (ctas < 1 || ctas > fused_max_ctas()) return cudaErrorInvalidValue;
  if (args.g2.bn != kGemmBN && args.g2.bn != kGemmBN2Double) return cudaErrorInvalidValue;
  if (small_tiles && (args.bm != kGemmBMSmall || args.g1.swap_rows != 0 || args.g2.swap_rows != 0))
    return cudaErrorInvalidValue;
  if (args.router_kind == kRouterSplitK &&
      (args.T > kSplitKMaxT || args.router_parts < 1 ||
       ((args.H + 255) / 256 + args.router_parts - 1) / args.router_parts > kSplitKMaxChunks))
    return cudaErrorInvalidValue;
  void* params[] = {const_cast<AMaps*>(&a1), const_cast<AMaps*>(&a2), const_cast<CUtensorMap*>(&b1),
                    const_cast<CUtensorMap*>(&b2), const_cast<CUtensorMap*>(&x), const_cast<CUtensorMap*>(&whi),
                    const_cast<CUtensorMap*>(&wlo), const_cast<FusedArgs*>(&args)};
  const bool d = args.g2.bn == kGemmBN2Double;
  const void* fn = small_tiles ? (d ? (const void*)fused_forward_kernel<SmallSmem, kGemmBN2Double>
                                    : (const void*)fused_forward_kernel<SmallSmem, kGemmBN>)
                               : (d ? (const void*)fused_forward_kernel<SmemLayout, kGemmBN2Double>
                                    : (const void*)fused_forward_kernel<SmemLayout, kGemmBN>);
  const size_t smem = small_tiles ? FusedSmem<SmallSmem>::bytes : FusedSmem<SmemLayout>::bytes;
  return cudaLaunchCooperativeKernel(fn, dim3(ctas), dim3(kGemmThreads), params, smem, s);
}

int gemm_pair_max_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  return g_pair_clusters[dev];
}

cudaError_t launch_gemm_pair_linear1(const AMaps& a, const CUtensorMap& b, const CUtensorMap& sfa,
                                     const CUtensorMap& sfb, const GemmArgs& args, int pairs, cudaStream_t s) {
  if (args.bm != kGemmBM) return cudaErrorInvalidValue;
  return launch_kernel(grouped_gemm_pair_kernel<1>, 2 * pairs, kGemmThreads, gemm_pair_smem_bytes(), s, a, b, sfa,
                       sfb, args);
}

cudaError_t launch_gemm_pair_linear2(const AMaps& a, const CUtensorMap& b, const CUtensorMap& sfa,
                                     const CUtensorMap& sfb, const GemmArgs& args, int pairs, cudaStream_t s) {
  if (args.bm != kGemmBM) return cudaErrorInvalidValue;
  return launch_kernel(grouped_gemm_pair_kernel<2>, 2 * pairs, kGemmThreads, gemm_pair_smem_bytes(), s, a, b, sfa,
                       sfb, args);
}

cudaError_t launch_gemm_linear1(const AMaps& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s, bool small_tiles) {
  if (small_tiles && (args.bm > kGemmBMSmall || args.swap_rows != 0)) return cudaErrorInvalidValue;
  if (small_tiles)
    return launch_kernel(grouped_gemm_kernel<1, SmallSmem>, grid, kGemmThreads, gemm_small_smem_bytes(), s, a, b, args);
  return launch_kernel(grouped_gemm_kernel<1, SmemLayout>, grid, kGemmThreads, gemm_smem_bytes(), s, a, b, args);
}

cudaError_t launch_gemm_linear2(const AMaps& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s, bool small_tiles) {
  constexpr int D = kGemmBN2Double;
  if (args.bn != kGemmBN && args.bn != D) return cudaErrorInvalidValue;
  if (small_tiles && (args.bm > kGemmBMSmall || args.swap_rows != 0)) return cudaErrorInvalidValue;
  if (small_tiles)
    return args.bn == D ? launch_kernel(grouped_gemm_kernel<2, SmallSmem, D>, grid, kGemmThreads,
                                        gemm_small_smem_bytes(), s, a, b, args)
                        : launch_kernel(grouped_gemm_kernel<2, SmallSmem>, grid, kGemmThreads,
                                        gemm_small_smem_bytes(), s, a, b, args);
  return args.bn == D ? launch_kernel(grouped_gemm_kernel<2, SmemLayout, D>, grid, kGemmThreads, gemm_smem_bytes(),
                                      s, a, b, args)
                      : launch_kernel(grouped_gemm_kernel<2, SmemLayout>, grid, kGemmThreads, gemm_smem_bytes(), s,
                                      a, b, args);
}

cudaError_t launch_gemm_chain(const AMaps& a1, const AMaps& a2, const CUtensorMap& b1, const CUtensorMap& b2,
                              const GemmArgs& g1, const GemmArgs& g2, int grid, cudaStream_t s) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const void* k = g2.bn == kGemmBN2Double ? reinterpret_cast<const void*>(chained_gemm_kernel<kGemmBN2Double>)
                                          : reinterpret_cast<const void*>(chained_gemm_kernel<kGemmBN>);
  if (g2.bn != kGemmBN && g2.bn != kGemmBN2Double) return cudaErrorInvalidValue;
  if (g1.bm > kGemmBMSmall || g2.bm > kGemmBMSmall || g1.swap_rows != 0 || g2.swap_rows != 0)
    return cudaErrorInvalidValue;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kGemmThreads, gemm_small_smem_bytes())) !=
      cudaSuccess)
    return e;
  if (grid < 1 || grid > per_sm * sms) return cudaErrorInvalidValue;   // every CTA co-resident
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = gemm_small_smem_bytes();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;      // co-resident CTAs (also when recorded in a graph)
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent_launch() ? 2 : 1;
  if (g2.bn == kGemmBN2Double) return cudaLaunchKernelEx(&cfg, chained_gemm_kernel<kGemmBN2Double>, a1, a2, b1, b2, g1, g2);
  return cudaLaunchKernelEx(&cfg, chained_gemm_kernel<kGemmBN>, a1, a2, b1, b2, g1, g2);
}

cudaError_t launch_tile_weight_scales(const uint8_t* src, uint8_t* dst, int n_experts, int rows_b, int K,
                                      int n_tiles_n, int mode, int N, cudaStream_t s, int tile_rows) {
  const int groups = mode == 1 ? rows_b / 128 : n_tiles_n * 2;
  const size_t smem = (size_t)128 * (K / 128) * 4;
  if (smem > 128 * 1024) return cudaErrorInvalidValue;
  dim3 grid(groups, n_experts);
  return launch_kernel(tile_weight_scales_kernel, grid, 256, smem, s, src, dst, rows_b, K, n_tiles_n, mode, N,
                       tile_rows);
}

}  // namespace moe
