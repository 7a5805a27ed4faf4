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
//   warp 0      TMA producer: A tile 128 x 128 B (SW128) and B tile
//               256 x 128 FP4 elements, loaded with the 16U4_ALIGN16B type so
//               the packed nibbles land in the padded shared-memory form the
//               f8f6f4 MMA reads (128 bytes of shared memory per 128 elements);
//   warp 1      TMEM owner and single-thread MMA issuer:
//               tcgen05.mma.kind::mxf8f6f4.block_scale, M=128, N=256, K=32,
//               fp32 accumulator in TMEM columns [0, 256);
//   warp 2      scale-factor loader: cp.async of the UE8M0 scale words into
//               the 128-row x 4-block atom layout (row r at byte
//               (r%32)*16 + (r/32)*4, block b at +b), copied to TMEM by the
//               MMA thread with tcgen05.cp 32x128b.warpx4;
//   warps 3..6  epilogue: tcgen05.ld of their 32-lane quarter, release the
//               accumulator, then SwiGLU + requant (linear1) or bf16 (linear2)
//               and stores.
// Tiles never cross experts: expert e owns rows [offsets[e], offsets[e+1]) of
// the dispatched activations, split into ceil(n_e/128) row tiles; rows of a
// tile past n_e are computed on whatever the loads return and never stored.
// Every wait is bounded (WaitCtl); on a timeout the CTA records
// MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM, returns.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK, S = kGemmStages;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0, kSfaCol = 256, kSfbCol = 264;
constexpr uint32_t kATileBytes = BM * BK;            // 16 KB
constexpr uint32_t kBTileBytes = BN * BK;            // 32 KB in shared memory (unpacked FP4)
constexpr uint32_t kSfaBytes = 512, kSfbBytes = 1024;
// Transaction bytes per stage: A 16 KB + B counted at 4 bits per element (16 KB).
constexpr uint32_t kStageTxBytes = BM * BK + BN * BK / 2;

struct SmemLayout {
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + S * kATileBytes;
  static constexpr uint32_t sfa = b + S * kBTileBytes;
  static constexpr uint32_t sfb = sfa + S * kSfaBytes;
  static constexpr uint32_t bars = sfb + S * kSfbBytes;
  // full_tma[S], full_sf[S], empty[S], accf, acce, drain
  static constexpr uint32_t n_bars = 3 * S + 3;
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t total = misc + 16;
};

struct TileCoord {
  int e, mt, nt, count, row0;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmArgs& p, int tile) {
  // largest e with mtile_start[e] * n_tiles_n <= tile
  int lo = 0, hi = p.n_experts;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(p.mtile_start + mid) * p.n_tiles_n <= tile) lo = mid; else hi = mid;
  }
  TileCoord c;
  c.e = lo;
  c.count = __ldg(p.counts + lo);
  const int mtiles = (c.count + BM - 1) / BM;
  const int local = tile - __ldg(p.mtile_start + lo) * p.n_tiles_n;
  c.nt = local / mtiles;             // tiles of one expert: n-major, m fastest
  c.mt = local - c.nt * mtiles;
  c.row0 = __ldg(p.offsets + lo) + c.mt * BM;
  return c;
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart.
  return smem_desc(saddr, 16, 1024, kLayoutSwizzle128B);
}
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  // 32 rows x 16 bytes, contiguous, no swizzle: 8-row core matrices 128 bytes apart.
  return smem_desc(saddr, 16, 128, kLayoutNoSwizzle);
}

template <int MODE>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& p, const TileCoord& c, uint32_t tmem_base, int q,
                                              int lane, uint64_t* acce) {
  const int m = q * 32 + lane;                         // accumulator row = TMEM lane
  const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
  const bool valid = c.mt * BM + m < c.count;
  const long grow = (long)c.row0 + m;
  if constexpr (MODE == 1) {
    float h[128];
    float amax = 0.f;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t g[32], u[32];
      tmem_ld_32x32b_x32(t_row + kAccCol + ch * 32, g);
      tmem_ld_32x32b_x32(t_row + kAccCol + 128 + ch * 32, u);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float gv = __uint_as_float(g[i]);
        const float uv = __uint_as_float(u[i]);
        const float hv = gv / (1.0f + expf(-gv)) * uv;   // silu(gate) * up
        h[ch * 32 + i] = hv;
        amax = fmaxf(amax, fabsf(hv));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce);
    if (valid) {
      const int pexp = pow2_exp_e4m3(amax);
      const float sc = exp2_neg(pexp);
      uint8_t* dst = p.hq + grow * p.N + (long)c.nt * 128;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        uint4 w;
        w.x = pack_e4m3x4(h[v * 16 + 0] * sc, h[v * 16 + 1] * sc, h[v * 16 + 2] * sc, h[v * 16 + 3] * sc);
        w.y = pack_e4m3x4(h[v * 16 + 4] * sc, h[v * 16 + 5] * sc, h[v * 16 + 6] * sc, h[v * 16 + 7] * sc);
        w.z = pack_e4m3x4(h[v * 16 + 8] * sc, h[v * 16 + 9] * sc, h[v * 16 + 10] * sc, h[v * 16 + 11] * sc);
        w.w = pack_e4m3x4(h[v * 16 + 12] * sc, h[v * 16 + 13] * sc, h[v * 16 + 14] * sc, h[v * 16 + 15] * sc);
        *reinterpret_cast<uint4*>(dst + v * 16) = w;
      }
      p.hsf[grow * (p.N / 128) + c.nt] = (uint32_t)(pexp + 127) * 0x01010101u;
    }
  } else {
    uint32_t packed[128];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + kAccCol + ch * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        packed[ch * 16 + i] = *reinterpret_cast<uint32_t*>(&b2);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acce);
    if (valid) {
      const int col0 = c.nt * BN;
      uint16_t* dst = p.y + grow * p.N + col0;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        if (col0 + ch * 32 < p.N) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w = make_uint4(packed[ch * 16 + v * 4 + 0], packed[ch * 16 + v * 4 + 1],
                                 packed[ch * 16 + v * 4 + 2], packed[ch * 16 + v * 4 + 3]);
            *reinterpret_cast<uint4*>(dst + ch * 32 + v * 8) = w;
          }
        }
      }
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_s = smem + SmemLayout::a;
  uint8_t* b_s = smem + SmemLayout::b;
  uint8_t* sfa_s = smem + SmemLayout::sfa;
  uint8_t* sfb_s = smem + SmemLayout::sfb;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars);
  uint64_t* full_tma = bars;
  uint64_t* full_sf = bars + S;
  uint64_t* empty = bars + 2 * S;
  uint64_t* accf = bars + 3 * S;
  uint64_t* acce = accf + 1;
  uint64_t* drain = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_sf[s], 32);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int total_tiles = __ldg(p.mtile_start + p.n_experts) * p.n_tiles_n;
  const int KT = p.K / BK;

  // per-stage fill counters of the TMA producer (for draining on abort)
  uint32_t fills[S];
#pragma unroll
  for (int s = 0; s < S; ++s) fills[s] = 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const TileCoord c = decode_tile(p, tile);
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctl, kWhereGemmProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_tma[stage], kStageTxBytes);
          tma_load_2d(a_s + stage * kATileBytes, &tmA, kt * BK, c.row0, &full_tma[stage]);
          if constexpr (MODE == 1) {
            const int brow = c.e * p.rows_b + c.nt * 128;
            tma_load_2d(b_s + stage * kBTileBytes, &tmB, kt * BK, brow, &full_tma[stage]);
            tma_load_2d(b_s + stage * kBTileBytes + kBTileBytes / 2, &tmB, kt * BK, brow + p.N, &full_tma[stage]);
          } else {
            const int brow = c.e * p.rows_b + c.nt * BN;
            tma_load_2d(b_s + stage * kBTileBytes, &tmB, kt * BK, brow, &full_tma[stage]);
          }
          fills[stage] += 1;
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      // wait for our own bulk copies before the CTA may exit (abort path)
#pragma unroll
      for (int s = 0; s < S; ++s) {
        if (fills[s] > 0 && !mbar_wait_drain(&full_tma[s], (fills[s] - 1) & 1, p.timeout_ns)) {
          report_status(p.status, kStatusTimeout, kWhereGemmDrain, s);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(acce, acc_phase ^ 1, ctl, kWhereGemmMma)) break;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full_tma[stage], phase, ctl, kWhereGemmMma + 1) ||
              !mbar_wait(&full_sf[stage], phase, ctl, kWhereGemmMma + 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          fence_proxy_async_smem();
          const uint32_t sfa_addr = smem_u32(sfa_s + stage * kSfaBytes);
          const uint32_t sfb_addr = smem_u32(sfb_s + stage * kSfbBytes);
          tc_cp_32x128b_warpx4(tmem_base + kSfaCol, sf_desc(sfa_addr));
          tc_cp_32x128b_warpx4(tmem_base + kSfbCol, sf_desc(sfb_addr));
          tc_cp_32x128b_warpx4(tmem_base + kSfbCol + 4, sf_desc(sfb_addr + 512));
          const uint32_t a_addr = smem_u32(a_s + stage * kATileBytes);
          const uint32_t b_addr = smem_u32(b_s + stage * kBTileBytes);
#pragma unroll
          for (int kb = 0; kb < BK / 32; ++kb) {
            tc_mma_mxf8f6f4(tmem_base + kAccCol, sw128_desc(a_addr + kb * 32), sw128_desc(b_addr + kb * 32),
                            idesc_mxf8f6f4(BM, BN, kb, kb), tmem_base + kSfaCol, tmem_base + kSfbCol,
                            (kt | kb) != 0);
          }
          tc_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(accf);
        acc_phase ^= 1;
      }
      // all MMAs this thread issued have finished once `drain` completes
      tc_commit(drain);
      if (!mbar_wait_drain(drain, 0, p.timeout_ns)) report_status(p.status, kStatusTimeout, kWhereGemmDrain, 9);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale-factor loader
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    bool withhold = p.inject_fault != 0 && blockIdx.x == 0;
    const int kw_a = p.K / 128;     // u32 words per activation row
    const int kb_b = p.K / 32;      // bytes per weight scale row
    const long wrow_max = (long)p.n_experts * p.rows_b - 1;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const TileCoord c = decode_tile(p, tile);
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1, ctl, kWhereGemmSfLoader)) { ok = false; break; }
        if (withhold) {
          // test hook: this stage's scale factors never arrive
          withhold = false;
        } else {
          uint8_t* da = sfa_s + stage * kSfaBytes + lane * 16;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = lane + 32 * i;
            long grow = (long)c.row0 + r;
            if (grow > p.rows_total - 1) grow = p.rows_total - 1;
            cp_async_4(da + i * 4, p.sfa + grow * kw_a + kt);
          }
          uint8_t* db = sfb_s + stage * kSfbBytes + lane * 16;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int n = lane + 32 * i;
            long wrow;
            if constexpr (MODE == 1) {
              wrow = (long)c.e * p.rows_b + (n < 128 ? c.nt * 128 + n : p.N + c.nt * 128 + (n - 128));
            } else {
              wrow = (long)c.e * p.rows_b + (long)c.nt * BN + n;
            }
            if (wrow > wrow_max) wrow = wrow_max;
            cp_async_4(db + (i / 4) * 512 + (i % 4) * 4, p.sfb + wrow * kb_b + kt * 4);
          }
          cp_async_arrive_noinc(&full_sf[stage]);
        }
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ epilogue (warps 3..6)
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(p, tile);
      // warp-uniform decision: tcgen05.ld below is .sync.aligned
      const bool ok = mbar_wait(accf, acc_phase, ctl, kWhereGemmEpilogue);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      epilogue_tile<MODE>(p, c, tmem_base, q, lane, acce);
      acc_phase ^= 1;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

size_t gemm_smem_bytes() { return SmemLayout::total + 1024; }

cudaError_t gemm_prepare_device() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm_smem_bytes());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)gemm_smem_bytes());
}

cudaError_t launch_gemm_linear1(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s) {
  grouped_gemm_kernel<1><<<grid, kGemmThreads, gemm_smem_bytes(), s>>>(a, b, args);
  return cudaGetLastError();
}

cudaError_t launch_gemm_linear2(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, int grid,
                                cudaStream_t s) {
  grouped_gemm_kernel<2><<<grid, kGemmThreads, gemm_smem_bytes(), s>>>(a, b, args);
  return cudaGetLastError();
}

}  // namespace moe
