// Routing, dispatch (+ activation quantisation) and combine kernels: stand-alone launches of
// the bodies in path_phases.cuh, plus the tiled and shared-memory routers.
//
// Router and gates: "전문가 혼합(Mixture of Experts; MoE)" lesson, "FFN 교체"
// (the router is one linear layer giving a score per expert) and "Step 1: 라우터"
// (selection by descending score + bias, gates = softmax over the selected
// experts' original scores); the bias steers selection only ("부하 분산 문제").
// Dispatch/combine: "Mega MoE" wiki, "한 줄 정의" -- on one device an in-HBM
// permutation of token copies into expert-major order and a gather back.
#include "common.cuh"
#include "kernels.h"
#include "path_phases.cuh"

namespace moe {

namespace {

// --------------------------------------------------------------------------- router
// logits[t][e] = sum_h x[t][h] * W_r[e][h], fp32 FMA on CUDA cores.
// Block tile: 64 tokens x ET experts, K chunks of 32 staged in shared memory.
template <int ET>
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ W, float* __restrict__ logits,
                                                            int T, int H, int E) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int TT = 64, KC = 32;
  constexpr int EPT = ET / 16;           // experts per thread
  __shared__ float xs[KC][TT + 1];
  __shared__ float ws[KC][ET + 1];
  const int t0 = blockIdx.x * TT;
  const int e0 = blockIdx.y * ET;
  const int tx = threadIdx.x % 16;       // expert lane
  const int ty = threadIdx.x / 16;       // token group of 4
  float acc[4][EPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < EPT; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < H; k0 += KC) {
    for (int idx = threadIdx.x; idx < TT * KC; idx += 256) {
      const int tt = idx / KC, kk = idx % KC;
      const int t = t0 + tt;
      float v = 0.f;
      if (t < T) v = __uint_as_float((uint32_t)x[(long)t * H + k0 + kk] << 16);
      xs[kk][tt] = v;
    }
    for (int idx = threadIdx.x; idx < ET * KC; idx += 256) {
      const int ee = idx / KC, kk = idx % KC;
      const int e = e0 + ee;
      ws[kk][ee] = (e < E) ? W[(long)e * H + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < KC; ++kk) {
      float xv[4], wv[EPT];
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < EPT; ++j) wv[j] = ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      const int e = e0 + tx + 16 * j;
      if (e < E) logits[(long)t * E + e] = acc[i][j];
    }
  }
}

template <int EC>
__global__ void __launch_bounds__(256) router_logits_warp_kernel(const uint16_t* __restrict__ x,
                                                                 const float* __restrict__ W,
                                                                 float* __restrict__ logits, int T, int H, int E) {
  griddep_wait();
  griddep_launch_dependents();
  router_warp_items<EC>(x, W, logits, T, H, E, (long)blockIdx.x * 8 + threadIdx.x / 32, (long)gridDim.x * 8);
}

__global__ void __launch_bounds__(256) router_logits_split_kernel(const uint16_t* __restrict__ x,
                                                                  const float* __restrict__ W,
                                                                  float* __restrict__ logits, int T, int H, int E) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float part[8];
  router_split_block<256>(x, W, logits, T, H, E, blockIdx.x, blockIdx.y, part);
}

// Few experts (E <= 8) with W_router small enough for shared memory: stage it
// once per block, then each warp takes 4 tokens at a time so every W value read
// from shared memory feeds 4 FMAs.  The x rows are read four 256-channel chunks
// at a time (all loads issued before any is used: one block per SM leaves few
// warps to hide the latency); each lane still adds its channels chunk by chunk.
constexpr int kSmemRouterMaxBytes = 200 * 1024;

__global__ void __launch_bounds__(256) router_logits_smem_kernel(const uint16_t* __restrict__ x,
                                                                 const float* __restrict__ W,
                                                                 float* __restrict__ logits, int T, int H, int E) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float4 w_s4[];
  const float* w_s = reinterpret_cast<const float*>(w_s4);
  const int n4 = E * H / 4;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) w_s4[i] = __ldg(reinterpret_cast<const float4*>(W) + i);
  __syncthreads();
  const int lane = threadIdx.x % 32;
  const int groups = (T + 3) / 4;
  for (int grp = blockIdx.x * 8 + threadIdx.x / 32; grp < groups; grp += gridDim.x * 8) {
    const int t0 = grp * 4;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int cb4 = 0; cb4 < H; cb4 += 1024) {
      uint4 raw[4][4];                          // [chunk][token]
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c0 = cb4 + u * 256 + lane * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          raw[u][i] = make_uint4(0, 0, 0, 0);
          if (c0 < H && t0 + i < T) raw[u][i] = __ldg(reinterpret_cast<const uint4*>(x + (long)(t0 + i) * H + c0));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c0 = cb4 + u * 256 + lane * 8;
        if (c0 < H) {                           // H % 8 == 0: a lane's 8 channels are all in or all out
          float xv[4][8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 r = raw[u][i];
            xv[i][0] = __uint_as_float(r.x << 16); xv[i][1] = __uint_as_float(r.x & 0xFFFF0000u);
            xv[i][2] = __uint_as_float(r.y << 16); xv[i][3] = __uint_as_float(r.y & 0xFFFF0000u);
            xv[i][4] = __uint_as_float(r.z << 16); xv[i][5] = __uint_as_float(r.z & 0xFFFF0000u);
            xv[i][6] = __uint_as_float(r.w << 16); xv[i][7] = __uint_as_float(r.w & 0xFFFF0000u);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < E) {
              const float4 w0 = *reinterpret_cast<const float4*>(w_s + (long)j * H + c0);
              const float4 w1 = *reinterpret_cast<const float4*>(w_s + (long)j * H + c0 + 4);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                float a = acc[i][j];
                a = fmaf(xv[i][0], w0.x, a); a = fmaf(xv[i][1], w0.y, a); a = fmaf(xv[i][2], w0.z, a);
                a = fmaf(xv[i][3], w0.w, a); a = fmaf(xv[i][4], w1.x, a); a = fmaf(xv[i][5], w1.y, a);
                a = fmaf(xv[i][6], w1.z, a); a = fmaf(xv[i][7], w1.w, a);
                acc[i][j] = a;
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = acc[i][j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && j < E && t0 + i < T) logits[(long)(t0 + i) * E + j] = v;
      }
  }
}

// --------------------------------------------------------------------------- top-k + rank
__global__ void __launch_bounds__(1024) topk_rank_kernel(int mode, const float* __restrict__ logits, int n_parts,
                                                         const float* __restrict__ bias, int32_t* topk_ids,
                                                         float* gates, int32_t* __restrict__ local_rank,
                                                         int32_t* __restrict__ group_counts, uint32_t* status,
                                                         int T, int E, int k) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ TopkSmem sm;
  topk_rank_group<1024>(blockIdx.x, mode, logits, n_parts, bias, topk_ids, gates, local_rank, group_counts, status,
                        T, E, k, sm);
}

// T <= 32 (a single token group): top-k, ranks and both dispatch scans in one block; the
// group's counts are the experts' counts and every group base is 0.
__global__ void __launch_bounds__(1024) topk_scan_one_group_kernel(
    int mode, const float* __restrict__ logits, int n_parts, const float* __restrict__ bias, int32_t* topk_ids,
    float* gates, int32_t* __restrict__ local_rank, int32_t* __restrict__ group_counts, uint32_t* status,
    int32_t* group_base, int32_t* counts, int32_t* offsets, int32_t* mtile_start, int32_t* ptile_start,
    int4* tile_info, int4* ptile_info, int T, int E, int k, int shared, int bm, FoldedScatter fs) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ TopkSmem sm;
  __shared__ int32_t wsum[3][32];
  topk_rank_group<1024>(0, mode, logits, n_parts, bias, topk_ids, gates, local_rank, group_counts, status, T, E, k,
                        sm);
  // the group's per-expert masks are still in shared memory: counts without a global round trip
  int32_t* cnt_s = reinterpret_cast<int32_t*>(sm.mask);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = __popc(sm.mask[e]);
    cnt_s[e] = c;
    counts[e] = c;
    group_base[e] = 0;
  }
  __syncthreads();
  expert_scan_block<1024>(counts, offsets, mtile_start, ptile_start, tile_info, ptile_info, T, E, shared, bm, wsum,
                          cnt_s);
  if (fs.x != nullptr) {
    // the scatter of a few tokens, here instead of in a kernel of its own: the positions and the
    // tile starts this block wrote are visible to all of its threads after the barrier
    if (fs.zero != nullptr)
      for (int i = threadIdx.x; i < fs.n_zero; i += blockDim.x) fs.zero[i] = 0u;
    __syncthreads();
    const long items = (long)T * ((fs.H + 255) / 256);
    for (long it = threadIdx.x / 32; it < items; it += blockDim.x / 32)
      scatter_item(it, fs.x, topk_ids, local_rank, group_base, offsets, mtile_start, fs.slot_pos, fs.perm, fs.xq,
                   fs.xsf, T, fs.H, E, k, shared, bm);
  }
}

// --------------------------------------------------------------------------- scan
__global__ void __launch_bounds__(256) column_scan_kernel(const int32_t* __restrict__ group_counts,
                                                          int32_t* __restrict__ group_base, int32_t* counts, int G,
                                                          int E) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x * 8 + threadIdx.x / 32;
  if (e < E) column_scan_warp(e, group_counts, group_base, counts, G, E);
}

__global__ void __launch_bounds__(1024) expert_scan_kernel(int32_t* counts, int32_t* offsets, int32_t* mtile_start,
                                                           int32_t* ptile_start, int4* tile_info, int4* ptile_info,
                                                           int T, int E, int shared, int bm) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int32_t wsum[3][32];
  expert_scan_block<1024>(counts, offsets, mtile_start, ptile_start, tile_info, ptile_info, T, E, shared, bm, wsum);
}

// --------------------------------------------------------------------------- scatter + quant
// SL 256-channel slices per warp (one position lookup for all of them): 4 when there are
// enough (token, slice) items to fill the GPU with warps anyway, else 1.
template <int SL>
__global__ void __launch_bounds__(256) scatter_quant_kernel(const uint16_t* __restrict__ x,
                                                            const int32_t* __restrict__ topk_ids,
                                                            const int32_t* __restrict__ local_rank,
                                                            const int32_t* __restrict__ group_base,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ mtile_start,
                                                            int32_t* slot_pos, int32_t* perm, uint8_t* xq,
                                                            uint8_t* xsf, int T, int H, int E, int k, int shared,
                                                            int bm, uint32_t* zero, int n_zero) {
  griddep_wait();
  griddep_launch_dependents();
  // counters the next kernel starts from (the chained GEMM's per-expert linear1 counts): zeroed
  // here, once every kernel before this one has finished, so no memset sits between the launches
  if (zero != nullptr && blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_zero; i += blockDim.x) zero[i] = 0u;
  scatter_items<SL>((long)blockIdx.x * 8 + threadIdx.x / 32, x, topk_ids, local_rank, group_base, offsets,
                    mtile_start, slot_pos, perm, xq, xsf, T, H, E, k, shared, bm);
}

// Token-order quantisation for the debug entry point: xq[t][H], xs[t][H/128] = 2^p.
__global__ void __launch_bounds__(256) quant_tokens_kernel(const uint16_t* __restrict__ x, uint8_t* xq, float* xs,
                                                           int T, int H) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  const uint16_t* xr = x + (long)t * H;
  for (int cb = 0; cb < H; cb += 256) {
    const int c0 = cb + lane * 8;
    const bool active = c0 < H;
    const uint4 raw = active ? *reinterpret_cast<const uint4*>(xr + c0) : make_uint4(0, 0, 0, 0);
    float v[8];
    v[0] = __uint_as_float(raw.x << 16); v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    v[2] = __uint_as_float(raw.y << 16); v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    v[4] = __uint_as_float(raw.z << 16); v[5] = __uint_as_float(raw.z & 0xFFFF0000u);
    v[6] = __uint_as_float(raw.w << 16); v[7] = __uint_as_float(raw.w & 0xFFFF0000u);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const int p = pow2_exp_e4m3(amax);
    const float sc = exp2_neg(p);
    uint2 q;
    q.x = pack_e4m3x4(v[0] * sc, v[1] * sc, v[2] * sc, v[3] * sc);
    q.y = pack_e4m3x4(v[4] * sc, v[5] * sc, v[6] * sc, v[7] * sc);
    if (active) {
      *reinterpret_cast<uint2*>(xq + (long)t * H + c0) = q;
      if ((lane & 15) == 0) xs[(long)t * (H / 128) + c0 / 128] = exp2_neg(-p);
    }
  }
}

// --------------------------------------------------------------------------- combine
template <int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y,
                                                      const int32_t* __restrict__ slot_pos,
                                                      const float* __restrict__ gates, uint16_t* __restrict__ out,
                                                      int T, int H, int k, int shared) {
  griddep_wait();
  griddep_launch_dependents();
  combine_item<KMAX>((long)blockIdx.x * 8 + threadIdx.x / 32, y, slot_pos, gates, out, T, H, k, shared);
}

// --------------------------------------------------------------------------- bias update
// bias[e] += gamma * sign(T*k - counts[e]*E): an over-used expert (more rows than the mean
// load T*k/E) loses gamma, an under-used one gains it, one at the mean keeps its bias.
__global__ void __launch_bounds__(256) update_bias_kernel(float* bias, const int32_t* __restrict__ counts, int T,
                                                          int k, int E, float gamma) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    const long long diff = (long long)T * k - (long long)counts[e] * E;
    const float step = diff > 0 ? gamma : diff < 0 ? -gamma : 0.f;
    bias[e] = __fadd_rn(bias[e], step);
  }
}

thread_local bool g_dependent_launch = false;

}  // namespace

void set_dependent_launch(bool on) { g_dependent_launch = on; }
bool dependent_launch() { return g_dependent_launch; }

cudaError_t launch_update_bias(float* bias, const int32_t* counts, int T, int k, int E, float gamma,
                               cudaStream_t s) {
  update_bias_kernel<<<(E + 255) / 256, 256, 0, s>>>(bias, counts, T, k, E, gamma);
  return cudaGetLastError();
}

cudaError_t launch_router_logits(const uint16_t* x, const float* W_r, float* logits, int T, int H, int E,
                                 cudaStream_t s) {
  if (E <= 8 && (size_t)E * H * 4 <= kSmemRouterMaxBytes && T >= 64) {
    static bool attr_set[64] = {};      // the shared-memory opt-in, once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(router_logits_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSmemRouterMaxBytes);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const int groups = (T + 3) / 4;
    int grid = (groups + 7) / 8;
    if (grid > 148) grid = 148;
    router_logits_smem_kernel<<<grid, 256, (size_t)E * H * 4, s>>>(x, W_r, logits, T, H, E);
  } else if ((long)T * E <= 4096) {
    router_logits_split_kernel<<<dim3(E, T), 256, 0, s>>>(x, W_r, logits, T, H, E);
  } else if (E <= 32 || (long)T * E <= 16384 || (long)((T + 63) / 64) * ((E + 63) / 64) < 148) {
    // (also whenever the tiled router would have fewer blocks than SMs: with 64 x 64 (token,
    // expert) tiles over all of H, a handful of blocks takes milliseconds at H = 7168)
    // warp per (token, expert chunk)
    const int ec = (E <= 32) ? 8 : 2;
    const long items = (long)T * ((E + ec - 1) / ec);
    const long blocks = (items + 7) / 8;
    const int grid = (int)(blocks < 148 * 16 ? blocks : 148 * 16);
    if (ec == 8) router_logits_warp_kernel<8><<<grid, 256, 0, s>>>(x, W_r, logits, T, H, E);
    else router_logits_warp_kernel<2><<<grid, 256, 0, s>>>(x, W_r, logits, T, H, E);
  } else {
    // more than 32 experts and T * E > 16384 (E <= 32 took the warp kernel above)
    dim3 grid((T + 63) / 64, (E + 63) / 64);
    router_logits_kernel<64><<<grid, 256, 0, s>>>(x, W_r, logits, T, H, E);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk_rank(int mode, const float* logits, int n_parts, const float* bias, int32_t* topk_ids,
                             float* gates, int32_t* local_rank, int32_t* group_counts, uint32_t* status, int T, int E,
                             int k, cudaStream_t s) {
  if (n_parts < 1 || (n_parts > 1 && E > kTopkMaxSplitE)) return cudaErrorInvalidValue;
  const int G = (T + 31) / 32;
  return launch_kernel(topk_rank_kernel, G, 1024, 0, s, mode, logits, n_parts, bias, topk_ids, gates, local_rank,
                       group_counts, status, T, E, k);
}

cudaError_t launch_topk_scan_one_group(int mode, const float* logits, int n_parts, const float* bias,
                                      int32_t* topk_ids, float* gates, int32_t* local_rank, int32_t* group_counts,
                                      uint32_t* status, int32_t* group_base, int32_t* counts, int32_t* offsets,
                                      int32_t* mtile_start, int32_t* ptile_start, int4* tile_info,
                                      int4* ptile_info, int T, int E, int k, int shared, int bm, FoldedScatter fs,
                                      cudaStream_t s) {
  if (T > 32 || n_parts < 1 || (n_parts > 1 && E > kTopkMaxSplitE)) return cudaErrorInvalidValue;
  if (fs.x != nullptr && (long)T * ((fs.H + 255) / 256) > kFoldScatterMaxItems) return cudaErrorInvalidValue;
  return launch_kernel(topk_scan_one_group_kernel, 1, 1024, 0, s, mode, logits, n_parts, bias, topk_ids, gates,
                       local_rank, group_counts, status, group_base, counts, offsets, mtile_start, ptile_start,
                       tile_info, ptile_info, T, E, k, shared, bm, fs);
}

cudaError_t launch_dispatch_scan(const int32_t* group_counts, int32_t* counts, int32_t* offsets,
                                 int32_t* group_base, int32_t* mtile_start, int32_t* ptile_start, int4* tile_info,
                                 int4* ptile_info, int T, int E, int k, int shared, int bm, cudaStream_t s) {
  const int G = (T + 31) / 32;
  cudaError_t e = launch_kernel(column_scan_kernel, (E + 7) / 8, 256, 0, s, group_counts, group_base, counts, G, E);
  if (e != cudaSuccess) return e;
  return launch_kernel(expert_scan_kernel, 1, 1024, 0, s, counts, offsets, mtile_start, ptile_start, tile_info,
                       ptile_info, T, E, shared, bm);
}

cudaError_t launch_scatter_quant(const uint16_t* x, const int32_t* topk_ids, const int32_t* local_rank,
                                 const int32_t* group_base, const int32_t* offsets, const int32_t* mtile_start,
                                 int32_t* slot_pos, int32_t* perm, uint8_t* xq, uint8_t* xsf, int T, int H, int E,
                                 int k, int shared, int bm, cudaStream_t s, uint32_t* zero, int n_zero) {
  const long slices = (long)T * (x == nullptr ? 1 : (H + 255) / 256);
  // Mixtral T = 4096 (65,536 slices): 4 per warp, the scatter 26 -> 19 us; DSV3 T = 512
  // (14,336) and T = 1 (28) keep one per warp, four would leave too few warps in flight
  if (x != nullptr && slices >= 32768) {
    const long items = (long)T * (((H + 255) / 256 + 3) / 4);
    return launch_kernel(scatter_quant_kernel<4>, (unsigned)((items + 7) / 8), 256, 0, s, x, topk_ids, local_rank,
                         group_base, offsets, mtile_start, slot_pos, perm, xq, xsf, T, H, E, k, shared, bm, zero,
                         n_zero);
  }
  return launch_kernel(scatter_quant_kernel<1>, (unsigned)((slices + 7) / 8), 256, 0, s, x, topk_ids, local_rank,
                       group_base, offsets, mtile_start, slot_pos, perm, xq, xsf, T, H, E, k, shared, bm, zero,
                       n_zero);
}

cudaError_t launch_quant_tokens(const uint16_t* x, uint8_t* xq, float* xs, int T, int H, cudaStream_t s) {
  quant_tokens_kernel<<<(T + 7) / 8, 256, 0, s>>>(x, xq, xs, T, H);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* y, const int32_t* slot_pos, const float* gates, uint16_t* out, int T,
                           int H, int k, int shared, cudaStream_t s) {
  const long items = (long)T * ((H + 255) / 256);
  const unsigned grid = (unsigned)((items + 7) / 8);
  auto kern = k <= 2 ? combine_kernel<2> : k <= 4 ? combine_kernel<4> : k <= 8 ? combine_kernel<8> : combine_kernel<16>;
  return launch_kernel(kern, grid, 256, 0, s, y, slot_pos, gates, out, T, H, k, shared);
}

}  // namespace moe
