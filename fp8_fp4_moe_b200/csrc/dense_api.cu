// Dense block-scaled FP8 x FP4 GEMM: the grouped GEMM kernel in its linear2 form (bf16 rows out)
// run over a single group of M rows.  The operand formats are the expert FFN's ("DeepSeek Mega
// MoE / DeepGEMM mega kernel", "TL;DR": FP8 activations x FP4 weights).  The caller's UE8M0
// activation scales [M][K/128] become the kernel's scale atoms and the weight scales [N][K/32]
// its scale units, both in the caller's workspace; the library allocates nothing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/moe_b200.h"
#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

struct DenseLayout {
  size_t status, counts, offsets, mtile, ptile, tinfo, atoms, units, total;
};

size_t r256(size_t b) { return (b + 255) & ~size_t(255); }

DenseLayout dense_layout(int M, int N, int K) {
  DenseLayout L;
  size_t off = 0;
  L.status = off;  off += r256(16);
  L.counts = off;  off += r256(4);
  L.offsets = off; off += r256(8);
  L.mtile = off;   off += r256(8);
  L.ptile = off;   off += r256(8);
  const size_t mt = ((size_t)M + 127) / 128, kt = (size_t)K / 128, nt = ((size_t)N + 255) / 256;
  L.tinfo = off;   off += r256(mt * 16);
  L.atoms = off;   off += r256(mt * kt * 512);
  L.units = off;   off += r256(nt * kt * 1024);
  L.total = off;
  return L;
}

bool shape_ok(int M, int N, int K) {
  return M >= 1 && N >= 128 && K >= 128 && N % 128 == 0 && K % 128 == 0 && (long long)M * K < (1ll << 31) &&
         (long long)N * K < (1ll << 32);
}

bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The single group's bookkeeping (row-tile table entries {0, 0, M, 0}) and the activation scale
// atoms: atom (row tile g, K-block kb)
// holds row 128 g + r's code at bytes (r % 32) * 16 + (r / 32) * 4 .. + 3 (one per 32-K block of
// the 128).  Rows past M get code 127 (x1); their accumulator rows are never stored.
__global__ void __launch_bounds__(256) dense_setup_kernel(const uint8_t* __restrict__ A_scales, int M, int K,
                                                          int32_t* counts, int32_t* offsets, int32_t* mtile,
                                                          int32_t* ptile, int4* tinfo, uint8_t* atoms) {
  const int kw = K / 128, mt = (M + 127) / 128;
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < mt; g += gridDim.x * blockDim.x)
    tinfo[g] = make_int4(0, 0, M, 0);
  const long n = (long)mt * 128 * kw;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int row = (int)(i / kw), kb = (int)(i % kw);
    const uint32_t code = row < M ? A_scales[(long)row * kw + kb] : 127u;
    const int g = row / 128, r = row % 128;
    *reinterpret_cast<uint32_t*>(atoms + ((long)g * kw + kb) * 512 + (r % 32) * 16 + (r / 32) * 4) =
        code * 0x01010101u;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    counts[0] = M;
    offsets[0] = 0;
    offsets[1] = M;
    mtile[0] = 0;
    mtile[1] = mt;
    ptile[0] = 0;
    ptile[1] = (mt + 1) / 2;
  }
}

bool g_prepared[64] = {};

}  // namespace

extern "C" {

size_t moe_gemm_workspace_bytes(int M, int N, int K) {
  return shape_ok(M, N, K) ? dense_layout(M, N, K).total : 0;
}

int moe_gemm_fp8_fp4(int M, int N, int K, const uint8_t* A, const uint8_t* A_scales, const uint8_t* B,
                     const uint8_t* B_scales, void* out_bf16, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (!shape_ok(M, N, K)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(out_bf16, 16) || !aligned(A_scales, 1) ||
      !aligned(B_scales, 4))
    return MOE_ERR_INVALID_ARG;
  const DenseLayout L = dense_layout(M, N, K);
  if (!aligned(workspace, 256) || workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
  int dev = -1, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MOE_ERR_CUDA;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_SHAPE;   // built for sm_100a only
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev >= 64 || !g_prepared[dev]) {
    if (gemm_prepare_device() != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 64) g_prepared[dev] = true;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AMaps am;
  for (int i = 0; i < 4; ++i)
    if (encode_2d(&am.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, 128, 16u << i) != MOE_OK)
      return MOE_ERR_CUDA;
  CUtensorMap tb;
  if (encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, B, K, N, K / 2, 128, 256) != MOE_OK)
    return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws + L.status, 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
  const int mt = (M + 127) / 128, nt = (N + 255) / 256;
  const long setup_items = (long)mt * 128 * (K / 128);
  const int setup_grid = (int)((setup_items + 255) / 256 < 4 * sms ? (setup_items + 255) / 256 : 4 * sms);
  dense_setup_kernel<<<setup_grid, 256, 0, s>>>(A_scales, M, K, reinterpret_cast<int32_t*>(ws + L.counts),
                                                reinterpret_cast<int32_t*>(ws + L.offsets),
                                                reinterpret_cast<int32_t*>(ws + L.mtile),
                                                reinterpret_cast<int32_t*>(ws + L.ptile),
                                                reinterpret_cast<int4*>(ws + L.tinfo), ws + L.atoms);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_tile_weight_scales(B_scales, ws + L.units, 1, N, K, nt, 2, N, s) != cudaSuccess) return MOE_ERR_CUDA;
  GemmArgs a{};
  a.bm = kGemmBM;
  a.K = K;
  a.N = N;
  a.rows_b = N;
  a.n_experts = 1;
  a.rows_total = M;
  a.n_tiles_n = nt;
  a.bn = kGemmBN;
  a.swap_rows = 0;
  a.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  a.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  a.mtile_start = reinterpret_cast<const int32_t*>(ws + L.mtile);
  a.ptile_start = reinterpret_cast<const int32_t*>(ws + L.ptile);
  a.tile_info = reinterpret_cast<const int4*>(ws + L.tinfo);
  a.ptile_info = nullptr;                // the dense product never runs on CTA pairs
  a.sfa = ws + L.atoms;
  a.sfb = ws + L.units;
  a.y = static_cast<uint16_t*>(out_bf16);
  a.status = reinterpret_cast<uint32_t*>(ws + L.status);
  a.timeout_ns = 2000000000ull;
  a.inject_fault = 0;
  const long tiles = (long)mt * nt;
  const int grid = (int)(tiles < sms ? tiles : sms);
  return launch_gemm_linear2(am, tb, a, grid, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
