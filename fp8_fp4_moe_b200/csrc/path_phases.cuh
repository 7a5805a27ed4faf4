// Device-side bodies of the routing, dispatch and combine steps, shared by the stand-alone
// kernels (path_kernels.cu) and the single persistent forward kernel (gemm_sm100.cu).  Each
// body states who calls it: a whole warp for one work item, or all threads of a block.
//
// Router and gates: "전문가 혼합(Mixture of Experts; MoE)" lesson, "FFN 교체"
// (the router is one linear layer giving a score per expert) and "Step 1: 라우터"
// (selection by descending score + bias, gates = softmax over the selected
// experts' original scores); the bias steers selection only ("부하 분산 문제").
// Dispatch/combine: "Mega MoE" wiki, "한 줄 정의" -- on one device an in-HBM
// permutation of token copies into expert-major order and a gather back.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// --------------------------------------------------------------------------- router
// Warp per (token, chunk of EC experts): for few experts or few tokens, where
// the tiled kernel above has too little parallelism.  Lane l covers channels
// [c + 8l, c + 8l + 8) of every 256-channel slice; W rows stream through L1/L2.
// Called by whole warps: items first, first + stride, ...
template <int EC>
__device__ __forceinline__ void router_warp_items(const uint16_t* __restrict__ x, const float* __restrict__ W,
                                                  float* __restrict__ logits, int T, int H, int E, long first,
                                                  long stride) {
  const int lane = threadIdx.x % 32;
  const int n_chunks = (E + EC - 1) / EC;
  const long n_items = (long)T * n_chunks;
  for (long item = first; item < n_items; item += stride) {
    const int t = (int)(item / n_chunks);
    const int e0 = (int)(item % n_chunks) * EC;
    float acc[EC];
#pragma unroll
    for (int j = 0; j < EC; ++j) acc[j] = 0.f;
    const uint16_t* xr = x + (long)t * H;
    for (int cb = 0; cb < H; cb += 256) {
      const int c0 = cb + lane * 8;
      if (c0 >= H) break;                       // no shuffles inside this loop
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xr + c0));
      float xv[8];
      xv[0] = __uint_as_float(raw.x << 16); xv[1] = __uint_as_float(raw.x & 0xFFFF0000u);
      xv[2] = __uint_as_float(raw.y << 16); xv[3] = __uint_as_float(raw.y & 0xFFFF0000u);
      xv[4] = __uint_as_float(raw.z << 16); xv[5] = __uint_as_float(raw.z & 0xFFFF0000u);
      xv[6] = __uint_as_float(raw.w << 16); xv[7] = __uint_as_float(raw.w & 0xFFFF0000u);
#pragma unroll
      for (int j = 0; j < EC; ++j) {
        if (e0 + j < E) {
          const float4* wr = reinterpret_cast<const float4*>(W + (long)(e0 + j) * H + c0);
          const float4 w0 = __ldg(wr), w1 = __ldg(wr + 1);
          float a = acc[j];
          a = fmaf(xv[0], w0.x, a); a = fmaf(xv[1], w0.y, a); a = fmaf(xv[2], w0.z, a); a = fmaf(xv[3], w0.w, a);
          a = fmaf(xv[4], w1.x, a); a = fmaf(xv[5], w1.y, a); a = fmaf(xv[6], w1.z, a); a = fmaf(xv[7], w1.w, a);
          acc[j] = a;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < EC; ++j) {
      float v = acc[j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0 && e0 + j < E) logits[(long)t * E + e0 + j] = v;
    }
  }
}

// Few tokens: one block of NT threads per (expert, token) so that all SMs stream W_router.
// Thread i covers channels [8i, 8i + 8) of every 8*NT-channel pass; four passes are loaded
// before any is used.  The warps' partial sums are added in warp order (deterministic).
// Called by all NT threads of the block (it synchronises them); part: NT/32 floats.
template <int NT>
__device__ __forceinline__ void router_split_block(const uint16_t* __restrict__ x, const float* __restrict__ W,
                                                   float* __restrict__ logits, int T, int H, int E, int e, int t,
                                                   float* part) {
  constexpr int kPass = 8 * NT;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const uint16_t* xr = x + (long)t * H;
  const float* wr = W + (long)e * H;
  float acc = 0.f;
  for (int base = threadIdx.x * 8; base < H; base += 4 * kPass) {
    uint4 xv[4];
    float4 w0[4], w1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = base + u * kPass;
      if (c < H) {
        xv[u] = __ldg(reinterpret_cast<const uint4*>(xr + c));
        w0[u] = __ldg(reinterpret_cast<const float4*>(wr + c));
        w1[u] = __ldg(reinterpret_cast<const float4*>(wr + c) + 1);
      } else {
        xv[u] = make_uint4(0, 0, 0, 0);
        w0[u] = w1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc = fmaf(__uint_as_float(xv[u].x << 16), w0[u].x, acc);
      acc = fmaf(__uint_as_float(xv[u].x & 0xFFFF0000u), w0[u].y, acc);
      acc = fmaf(__uint_as_float(xv[u].y << 16), w0[u].z, acc);
      acc = fmaf(__uint_as_float(xv[u].y & 0xFFFF0000u), w0[u].w, acc);
      acc = fmaf(__uint_as_float(xv[u].z << 16), w1[u].x, acc);
      acc = fmaf(__uint_as_float(xv[u].z & 0xFFFF0000u), w1[u].y, acc);
      acc = fmaf(__uint_as_float(xv[u].w << 16), w1[u].z, acc);
      acc = fmaf(__uint_as_float(xv[u].w & 0xFFFF0000u), w1[u].w, acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) part[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = part[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) v += part[w];
    logits[(long)t * E + e] = v;
  }
  __syncthreads();                     // part[] is free again
}
// Few tokens inside a persistent kernel: a warp per (expert e, K part s) computes the partial
// logits of ALL T <= TMAX tokens over its part of the channels, so every warp streams a slice of
// W_router once (the whole grid reads it at HBM speed) instead of one block per (expert, token).
// Part s covers the 256-channel chunks [s*C/S, (s+1)*C/S) (C = ceil(H/256)); lane l owns channels
// [c + 8l, c + 8l + 8) of each chunk, all W loads of the part are issued before the FMAs.  Writes
// logits[s][t][e]; the top-k adds the S parts in part order (deterministic).
// Called by whole warps: items first, first + stride, ... over E * S items.
template <int TMAX, int CMAX>
__device__ __forceinline__ void router_splitk_items(const uint16_t* __restrict__ x, const float* __restrict__ W,
                                                   float* __restrict__ logits, int T, int H, int E, int S,
                                                   long first, long stride) {
  const int lane = threadIdx.x % 32;
  const int C = (H + 255) / 256;
  for (long item = first; item < (long)E * S; item += stride) {
    const int e = (int)(item / S), s = (int)(item % S);
    const int c_lo = s * C / S, c_hi = (s + 1) * C / S;       // at most CMAX chunks (host-chosen S)
    float4 w[CMAX][2];
#pragma unroll
    for (int i = 0; i < CMAX; ++i) {
      const int c0 = (c_lo + i) * 256 + lane * 8;
      if (c_lo + i < c_hi && c0 < H) {
        const float4* wr = reinterpret_cast<const float4*>(W + (long)e * H + c0);
        w[i][0] = __ldg(wr);
        w[i][1] = __ldg(wr + 1);
      } else {
        w[i][0] = w[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) acc[t] = 0.f;
#pragma unroll
    for (int i = 0; i < CMAX; ++i) {
      const int c0 = (c_lo + i) * 256 + lane * 8;
      if (c_lo + i < c_hi && c0 < H) {                          // lane-uniform per chunk except the H tail
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          if (t < T) {
            const uint4 r = __ldg(reinterpret_cast<const uint4*>(x + (long)t * H + c0));
            float a = acc[t];
            a = fmaf(__uint_as_float(r.x << 16), w[i][0].x, a);
            a = fmaf(__uint_as_float(r.x & 0xFFFF0000u), w[i][0].y, a);
            a = fmaf(__uint_as_float(r.y << 16), w[i][0].z, a);
            a = fmaf(__uint_as_float(r.y & 0xFFFF0000u), w[i][0].w, a);
            a = fmaf(__uint_as_float(r.z << 16), w[i][1].x, a);
            a = fmaf(__uint_as_float(r.z & 0xFFFF0000u), w[i][1].y, a);
            a = fmaf(__uint_as_float(r.w << 16), w[i][1].z, a);
            a = fmaf(__uint_as_float(r.w & 0xFFFF0000u), w[i][1].w, a);
            acc[t] = a;
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      if (t < T) {
        float v = acc[t];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) logits[((long)s * T + t) * E + e] = v;
      }
    }
  }
}

// --------------------------------------------------------------------------- top-k + rank
// One block of NT threads per group of 32 tokens; warp w selects for tokens 32*g + w,
// 32*g + w + NT/32, ...  Then warp 0 ranks the group's copies: lane = token, and each
// expert keeps a 32-bit mask of the group's tokens that chose it.  A copy's rank inside
// its expert is the number of lower lanes in that mask (ascending token order).
// Called by all NT threads of the block (it synchronises them).
struct TopkSmem {
  int32_t ids[32][16];
  uint32_t mask[1024];
  float sum[32 * kTopkMaxSplitE];      // the group's summed logits when n_parts > 1
};
template <int NT>
__device__ __forceinline__ void topk_rank_group(int g, int mode, const float* __restrict__ logits, int n_parts,
                                                const float* __restrict__ bias, int32_t* topk_ids, float* gates,
                                                int32_t* __restrict__ local_rank, int32_t* __restrict__ group_counts,
                                                uint32_t* status, int T, int E, int k, TopkSmem& sm) {
  auto& ids_s = sm.ids;
  uint32_t* mask_s = sm.mask;
  float* sum_s = sm.sum;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int e = threadIdx.x; e < E; e += NT) mask_s[e] = 0u;
  if (mode == 0 && n_parts > 1) {
    // the whole block adds the parts of the group's 32 x E logits, each in part order
    // (E % 4 == 0 here: the parts come from the tensor-core router, E % 16 == 0)
    const long stride4 = (long)T * E / 4;
    const int n4 = min(32, T - g * 32) * E / 4;
    const float4* base = reinterpret_cast<const float4*>(logits + (long)g * 32 * E);
    for (int i = threadIdx.x; i < n4; i += NT) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < n_parts; s0 += 8) {
        float4 part[8];                // eight parts in flight, then added in part order
#pragma unroll
        for (int s = 0; s < 8; ++s)
          if (s0 + s < n_parts) part[s] = base[(s0 + s) * stride4 + i];   // written earlier, not read-only
#pragma unroll
        for (int s = 0; s < 8; ++s)
          if (s0 + s < n_parts) {
            if (s0 + s == 0) v = part[s];
            else { v.x += part[s].x; v.y += part[s].y; v.z += part[s].z; v.w += part[s].w; }
          }
      }
      reinterpret_cast<float4*>(sum_s)[i] = v;
    }
  }
  __syncthreads();
  for (int tw = warp; tw < 32; tw += NT / 32) {
    const int t = g * 32 + tw;
    if (t < T) {
      if (mode == 0) {
        const float* row = n_parts > 1 ? sum_s + tw * E : logits + (long)t * E;
        auto score = [&](int e) { return row[e]; };
        // k rounds of a warp arg-max over (score + bias), lower id on ties
        float chosen_score = 0.f;   // unbiased score of this lane's slot (lane < k)
        int chosen_id = -1;
        uint32_t taken = 0u;        // bit i: expert lane + 32*i already selected (E <= 1024)
        float cached[8];            // E <= 256: this lane's biased scores, read once
        float raw[8];               // ... and the unbiased ones
        const bool use_cache = E <= 256;
        if (use_cache) {
  #pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            raw[i] = (e < E) ? score(e) : 0.f;
            cached[i] = (e < E) ? raw[i] + bias[e] : 0.f;
          }
        }
        for (int j = 0; j < k; ++j) {
          float best = -INFINITY;
          int best_id = 0x7FFFFFFF;
          int free_id = 0x7FFFFFFF;   // lowest unselected id (fallback when every score is NaN)
          if (use_cache) {
            // lane-local best (ids ascend with i, so a strict > keeps the lowest id), then two
            // warp reductions: the largest order-preserving key of (score + 0), then the lowest
            // id holding it.  Key 0 = no selectable score in this lane (NaN, -inf or taken).
            int bi = -1;
  #pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int e = lane + 32 * i;
              if (e >= E || (taken & (1u << i))) continue;
              if (free_id == 0x7FFFFFFF) free_id = e;
              if (cached[i] > best) { best = cached[i]; bi = i; }
            }
            uint32_t key = 0u;
            if (bi >= 0) {
              const uint32_t u = __float_as_uint(best + 0.0f);       // -0 and +0 compare equal
              key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
            }
            const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
            best_id = __reduce_min_sync(0xffffffffu, (key == kmax && bi >= 0) ? lane + 32 * bi : 0x7FFFFFFF);
            if (kmax == 0u) best_id = __reduce_min_sync(0xffffffffu, free_id);
          } else {
            for (int i = 0, e = lane; e < E; ++i, e += 32) {
              if (taken & (1u << i)) continue;
              if (free_id == 0x7FFFFFFF) free_id = e;
              const float b = score(e) + bias[e];
              if (b > best || (b == best && e < best_id)) { best = b; best_id = e; }
            }
          }
          if (!use_cache) {
  #pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              const float ob = __shfl_xor_sync(0xffffffffu, best, off);
              const int oid = __shfl_xor_sync(0xffffffffu, best_id, off);
              if (ob > best || (ob == best && oid < best_id)) { best = ob; best_id = oid; }
              free_id = min(free_id, __shfl_xor_sync(0xffffffffu, free_id, off));
            }
            if (best_id == 0x7FFFFFFF) best_id = free_id;   // k <= E guarantees free_id < E
          }
          if ((best_id & 31) == lane) taken |= 1u << (best_id >> 5);
          float s_best;
          if (use_cache) {               // the owner lane holds the unbiased score in registers
            float mine = 0.f;
  #pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i == (best_id >> 5)) mine = raw[i];
            s_best = __shfl_sync(0xffffffffu, mine, best_id & 31);
          } else {
            s_best = score(best_id);
          }
          if (lane == j) { chosen_id = best_id; chosen_score = s_best; }
        }
        // softmax over the unbiased scores of the selected experts
        float m = (lane < k) ? chosen_score : -INFINITY;
  #pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float ex = (lane < k) ? expf(chosen_score - m) : 0.f;
        float sum = ex;
  #pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < k) {
          topk_ids[(long)t * k + lane] = chosen_id;
          gates[(long)t * k + lane] = ex / sum;
          ids_s[tw][lane] = chosen_id;
        }
      } else {
        int id = (lane < k) ? topk_ids[(long)t * k + lane] : -1;
        bool bad = lane < k && (id < 0 || id >= E);
        for (int j = 0; j < k; ++j) {
          const int other = __shfl_sync(0xffffffffu, id, j);
          if (lane < k && j != lane && other == id) bad = true;
        }
        if (__any_sync(0xffffffffu, bad)) {
          if (lane == 0) report_status(status, kStatusBounds, 0x10, (uint32_t)t);
          id = (lane < E) ? lane : 0;        // keep every index in range; results are void
        }
        if (lane < k) ids_s[tw][lane] = id;
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int tt = g * 32 + lane;
    if (tt < T)
      for (int j = 0; j < k; ++j) atomicOr(&mask_s[ids_s[lane][j]], 1u << lane);
    __syncwarp();
    if (tt < T)
      for (int j = 0; j < k; ++j)
        local_rank[(long)tt * k + j] = __popc(mask_s[ids_s[lane][j]] & ((1u << lane) - 1u));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += NT) group_counts[(long)g * E + e] = __popc(mask_s[e]);
  __syncthreads();                     // shared memory is free again
}

// --------------------------------------------------------------------------- scan
// Two steps.  Per routed expert e (one warp): counts[e] = sum over groups and the relative
// group base group_base[g][e] = rows of e in groups < g (warp scan over the groups, 32 at a
// time).  Then one block: exclusive scans over the n = E + shared experts (shared expert
// last, T rows) of counts -> offsets, of ceil(count/bm) -> mtile_start (bm-row tiles of the
// GEMMs) and of ceil(ceil(count/128)/2) -> ptile_start (128-row tile pairs of the CTA-pair GEMM).
__device__ __forceinline__ void column_scan_warp(int e, const int32_t* __restrict__ group_counts,
                                                 int32_t* __restrict__ group_base, int32_t* __restrict__ counts,
                                                 int G, int E) {
  const int lane = threadIdx.x % 32;
  int run = 0;
  for (int g0 = 0; g0 < G; g0 += 32) {
    const int g = g0 + lane;
    const int v = g < G ? group_counts[(long)g * E + e] : 0;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    if (g < G) group_base[(long)g * E + e] = run + inc - v;
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) counts[e] = run;
}

// Called by all NT threads of one block (it synchronises them); n = E + shared <= 1024.
// Also fills the row-tile tables the grouped GEMMs decode their tiles with (one entry per
// 128-row tile, or per pair of them, of every expert).  The routed experts' counts are read
// from cnt_src (the counts array itself, or a copy in shared memory).
template <int NT>
__device__ __forceinline__ void expert_scan_block(int32_t* counts, int32_t* offsets, int32_t* mtile_start,
                                                  int32_t* ptile_start, int4* tile_info, int4* ptile_info, int T,
                                                  int E, int shared, int bm, int32_t (*wsum)[32],
                                                  const int32_t* cnt_src = nullptr) {
  if (cnt_src == nullptr) cnt_src = counts;
  constexpr int PER = (1024 + NT - 1) / NT;   // consecutive experts per thread
  constexpr int NW = NT / 32;
  const int n = E + shared;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int c[PER];
  int tc = 0, tm = 0, tp = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = threadIdx.x * PER + j;
    c[j] = e < E ? cnt_src[e] : (e == E && shared ? T : 0);
    tc += c[j];
    tm += (c[j] + bm - 1) / bm;
    tp += ((c[j] + kGemmBM - 1) / kGemmBM + 1) / 2;
  }
  int ic = tc, im = tm, ip = tp;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ic, off);
    const int b = __shfl_up_sync(0xffffffffu, im, off);
    const int d = __shfl_up_sync(0xffffffffu, ip, off);
    if (lane >= off) { ic += a; im += b; ip += d; }
  }
  if (lane == 31) { wsum[0][warp] = ic; wsum[1][warp] = im; wsum[2][warp] = ip; }
  __syncthreads();
  if (warp == 0) {
    int a = lane < NW ? wsum[0][lane] : 0, b = lane < NW ? wsum[1][lane] : 0, d = lane < NW ? wsum[2][lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a2 = __shfl_up_sync(0xffffffffu, a, off);
      const int b2 = __shfl_up_sync(0xffffffffu, b, off);
      const int d2 = __shfl_up_sync(0xffffffffu, d, off);
      if (lane >= off) { a += a2; b += b2; d += d2; }
    }
    if (lane < NW) { wsum[0][lane] = a; wsum[1][lane] = b; wsum[2][lane] = d; }
  }
  __syncthreads();
  int bc = (warp > 0 ? wsum[0][warp - 1] : 0) + ic - tc;
  int bt = (warp > 0 ? wsum[1][warp - 1] : 0) + im - tm;
  int bp = (warp > 0 ? wsum[2][warp - 1] : 0) + ip - tp;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = threadIdx.x * PER + j;
    const int mt = (c[j] + bm - 1) / bm;
    const int pt = ((c[j] + kGemmBM - 1) / kGemmBM + 1) / 2;
    if (e < n) {
      if (e >= E) counts[e] = c[j];
      offsets[e] = bc;
      mtile_start[e] = bt;
      ptile_start[e] = bp;
      for (int g = 0; g < mt; ++g) tile_info[bt + g] = make_int4(e, bt, c[j], bc);
      for (int g = 0; g < pt; ++g) ptile_info[bp + g] = make_int4(e, bp, c[j], bc);
    }
    bc += c[j];
    bt += mt;
    bp += pt;
    if (e == n - 1) {
      offsets[n] = bc;
      mtile_start[n] = bt;
      ptile_start[n] = bp;
    }
  }
  __syncthreads();                     // wsum is free again
}

// --------------------------------------------------------------------------- scatter + quant
// One warp per (token, 256-channel slice).  Positions: slot_pos[t][j] = offsets[e] +
// group_base[g][e] + rank (group_base relative to the expert's first row); a row's scale
// word goes to the atom of its bm-row tile;
// the shared expert's row for token t is R + t.  Quantisation: per 128-channel
// block, smallest 2^p with amax <= 448 * 2^p (p >= -126; p = 0 if all zero),
// codes = E4M3 round-to-nearest-even of x * 2^-p (exact scaling), written once
// per destination row together with the block's UE8M0 code word.
// Called by a whole warp for one item = (token, SL consecutive slices): the destination rows
// are looked up once for the SL slices, whose x loads are all issued first; the warp of the
// token's first slices also records the positions.  scatter_item: one slice per item.
template <int SL>
__device__ __forceinline__ void scatter_items(long item, const uint16_t* __restrict__ x,
                                              const int32_t* __restrict__ topk_ids,
                                              const int32_t* __restrict__ local_rank,
                                              const int32_t* __restrict__ group_base,
                                              const int32_t* __restrict__ offsets,
                                              const int32_t* __restrict__ mtile_start, int32_t* slot_pos,
                                              int32_t* perm, uint8_t* xq, uint8_t* xsf, int T, int H, int E, int k,
                                              int shared, int bm) {
  const int lane = threadIdx.x % 32;
  const int n_slices = (x == nullptr) ? 1 : (H + 255) / 256;
  const int n_grp = (n_slices + SL - 1) / SL;
  if (item >= (long)T * n_grp) return;
  const int t = (int)(item / n_grp);
  const int grp = (int)(item % n_grp);
  const int g = t / 32;
  const long R = (long)T * k;
  const int kw = H / 128;
  // the token's 8 channels of this lane in each slice, loaded before the position lookups they
  // do not depend on
  uint4 raw[SL];
#pragma unroll
  for (int s = 0; s < SL; ++s) {
    const int c0 = (grp * SL + s) * 256 + lane * 8;
    raw[s] = x != nullptr && c0 < H ? *reinterpret_cast<const uint4*>(x + (long)t * H + c0) : make_uint4(0, 0, 0, 0);
  }
  int row = -1;                          // lane j < k holds the row of slot j; lane k the shared row
  int e = -1;
  if (lane < k) {
    e = topk_ids[(long)t * k + lane];
    row = offsets[e] + group_base[(long)g * E + e] + local_rank[(long)t * k + lane];
    if (grp == 0) {
      slot_pos[(long)t * k + lane] = row;
      perm[row] = t * k + lane;
    }
  } else if (lane == k && shared) {
    e = E;
    row = (int)(R + t);
  }
  if (x == nullptr) return;
  // this destination row's word inside its row tile's scale atoms
  long sf_off = 0;
  if (e >= 0) {
    const int rank = row - offsets[e];
    const int r = rank % bm;
    sf_off = ((long)(mtile_start[e] + rank / bm) * kw) * 512 + (r % 32) * 16 + (r / 32) * 4;
  }
  const int ndst = k + shared;
#pragma unroll
  for (int s = 0; s < SL; ++s) {
    if ((grp * SL + s) * 256 >= H) break;        // warp-uniform: the slice starts past H
    const int c0 = (grp * SL + s) * 256 + lane * 8;
    const bool active = c0 < H;                  // H % 128 == 0: whole half-warps
    // 8 channels per lane; a 128-channel block spans 16 lanes.  Every lane runs
    // the shuffles (full mask); a half-warp past H idles.
    const uint4 rw = raw[s];
    float v[8];
    v[0] = __uint_as_float(rw.x << 16); v[1] = __uint_as_float(rw.x & 0xFFFF0000u);
    v[2] = __uint_as_float(rw.y << 16); v[3] = __uint_as_float(rw.y & 0xFFFF0000u);
    v[4] = __uint_as_float(rw.z << 16); v[5] = __uint_as_float(rw.z & 0xFFFF0000u);
    v[6] = __uint_as_float(rw.w << 16); v[7] = __uint_as_float(rw.w & 0xFFFF0000u);
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
    const uint32_t code = (uint32_t)(p + 127) * 0x01010101u;
    const int blk = c0 / 128;
    for (int d = 0; d < ndst; ++d) {
      const long r = __shfl_sync(0xffffffffu, row, d);
      const long so = __shfl_sync(0xffffffffu, sf_off, d);
      if (active) {
        *reinterpret_cast<uint2*>(xq + r * H + c0) = q;
        if ((lane & 15) == 0) *reinterpret_cast<uint32_t*>(xsf + so + (long)blk * 512) = code;
      }
    }
  }
}
// Many items: the same as scatter_items for one item of SL slices (SL * 256 <= 2048 channels),
// except that the E4M3 bytes are staged in the warp's 2 KB of shared memory `stage` and sent to
// each destination row with one bulk copy, in place of SL x 32 eight-byte stores per row; the
// scale bytes and positions are plain stores.  `pending` (carried from item to item): the warp has
// bulk copies that may still read `stage`; scatter_bulk_drain waits for all of them to complete.
template <int SL>
__device__ __forceinline__ void scatter_items_bulk(long item, const uint16_t* __restrict__ x,
                                                   const int32_t* __restrict__ topk_ids,
                                                   const int32_t* __restrict__ local_rank,
                                                   const int32_t* __restrict__ group_base,
                                                   const int32_t* __restrict__ offsets,
                                                   const int32_t* __restrict__ mtile_start, int32_t* slot_pos,
                                                   int32_t* perm, uint8_t* xq, uint8_t* xsf, int T, int H, int E,
                                                   int k, int shared, int bm, uint8_t* stage, bool& pending) {
  static_assert(SL * 256 <= 2048, "one item's codes fit the warp's 2 KB of staging memory");
  const int lane = threadIdx.x % 32;
  const int n_slices = (H + 255) / 256;
  const int n_grp = (n_slices + SL - 1) / SL;
  const int t = (int)(item / n_grp);
  const int grp = (int)(item % n_grp);
  const int g = t / 32;
  const long R = (long)T * k;
  const int kw = H / 128;
  // the token's 8 channels of this lane in each slice, loaded before the position lookups
  uint4 raw[SL];
#pragma unroll
  for (int s = 0; s < SL; ++s) {
    const int c0 = (grp * SL + s) * 256 + lane * 8;
    raw[s] = c0 < H ? *reinterpret_cast<const uint4*>(x + (long)t * H + c0) : make_uint4(0, 0, 0, 0);
  }
  int row = -1;                          // lane j < k holds the row of slot j; lane k the shared row
  int e = -1;
  if (lane < k) {
    e = topk_ids[(long)t * k + lane];
    row = offsets[e] + group_base[(long)g * E + e] + local_rank[(long)t * k + lane];
    if (grp == 0) {
      slot_pos[(long)t * k + lane] = row;
      perm[row] = t * k + lane;
    }
  } else if (lane == k && shared) {
    e = E;
    row = (int)(R + t);
  }
  long sf_off = 0;                       // this destination row's word inside its tile's scale atoms
  if (e >= 0) {
    const int rank = row - offsets[e];
    const int r = rank % bm;
    sf_off = ((long)(mtile_start[e] + rank / bm) * kw) * 512 + (r % 32) * 16 + (r / 32) * 4;
  }
  const int ndst = k + shared;
  // the previous item's copies must have read the staging bytes before they are overwritten
  if (pending && lane < ndst) bulk_wait_read<0>();
  __syncwarp();
#pragma unroll
  for (int s = 0; s < SL; ++s) {
    if ((grp * SL + s) * 256 >= H) break;        // warp-uniform: the slice starts past H
    const int c0 = (grp * SL + s) * 256 + lane * 8;
    const bool active = c0 < H;                  // H % 128 == 0: whole half-warps
    const uint4 rw = raw[s];
    float v[8];
    v[0] = __uint_as_float(rw.x << 16); v[1] = __uint_as_float(rw.x & 0xFFFF0000u);
    v[2] = __uint_as_float(rw.y << 16); v[3] = __uint_as_float(rw.y & 0xFFFF0000u);
    v[4] = __uint_as_float(rw.z << 16); v[5] = __uint_as_float(rw.z & 0xFFFF0000u);
    v[6] = __uint_as_float(rw.w << 16); v[7] = __uint_as_float(rw.w & 0xFFFF0000u);
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
    if (active) *reinterpret_cast<uint2*>(stage + s * 256 + lane * 8) = q;
    const uint32_t code = (uint32_t)(p + 127) * 0x01010101u;
    const int blk = c0 / 128;
    for (int d = 0; d < ndst; ++d) {
      const long so = __shfl_sync(0xffffffffu, sf_off, d);
      if (active && (lane & 15) == 0) *reinterpret_cast<uint32_t*>(xsf + so + (long)blk * 512) = code;
    }
  }
  fence_proxy_async_smem();              // this lane's staging bytes, before the copies read them
  __syncwarp();
  if (lane < ndst) {
    const int c_base = grp * SL * 256;
    const uint32_t bytes = (uint32_t)min(SL * 256, H - c_base);   // E4M3: one byte a channel
    bulk_store(xq + (long)row * H + c_base, stage, bytes);
    bulk_commit();
  }
  pending = true;
}
// Waits until the warp's scatter bulk copies are complete (their writes performed).
__device__ __forceinline__ void scatter_bulk_drain(bool pending, int k, int shared) {
  if (pending && (threadIdx.x % 32) < k + shared) bulk_wait<0>();
  __syncwarp();
}
__device__ __forceinline__ void scatter_item(long item, const uint16_t* __restrict__ x,
                                             const int32_t* __restrict__ topk_ids,
                                             const int32_t* __restrict__ local_rank,
                                             const int32_t* __restrict__ group_base,
                                             const int32_t* __restrict__ offsets,
                                             const int32_t* __restrict__ mtile_start, int32_t* slot_pos,
                                             int32_t* perm, uint8_t* xq, uint8_t* xsf, int T, int H, int E, int k,
                                             int shared, int bm) {
  scatter_items<1>(item, x, topk_ids, local_rank, group_base, offsets, mtile_start, slot_pos, perm, xq, xsf, T, H,
                   E, k, shared, bm);
}

// --------------------------------------------------------------------------- combine
// out[t] = bf16( sum_{j<k} gate[t][j] * row[slot_pos[t][j]] + shared * row[R + t] ),
// fp32 accumulation in exactly that order (deterministic, no atomics).  KMAX >= k bounds
// the rows a lane holds in registers (all loaded before the first is used).
// Called by a whole warp for U (token, 256-channel slice) items (indices past T * slices are
// skipped).
template <int KMAX, int U>
__device__ __forceinline__ void combine_items(const long (&items)[U], const uint16_t* __restrict__ y,
                                              const int32_t* __restrict__ slot_pos, const float* __restrict__ gates,
                                              uint16_t* __restrict__ out, int T, int H, int k, int shared) {
  const int lane = threadIdx.x % 32;
  const int n_slices = (H + 255) / 256;
  const long R = (long)T * k;
  // every load of the U items is issued before the first is used; each sum keeps slot order
  int t[U], c0[U];
  bool valid[U], active[U];
  int my_row[U];
  float my_gate[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    valid[u] = items[u] < (long)T * n_slices;          // warp-uniform
    t[u] = valid[u] ? (int)(items[u] / n_slices) : 0;
    c0[u] = (valid[u] ? (int)(items[u] % n_slices) : 0) * 256 + lane * 8;
    active[u] = valid[u] && c0[u] < H;
    my_row[u] = 0;
    my_gate[u] = 0.f;
    if (valid[u] && lane < k) {
      my_row[u] = slot_pos[(long)t[u] * k + lane];
      my_gate[u] = gates[(long)t[u] * k + lane];
    }
  }
  uint4 raw[U][KMAX];
  float g[U][KMAX];
  uint4 raw_s[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const long r = __shfl_sync(0xffffffffu, my_row[u], j);
      g[u][j] = __shfl_sync(0xffffffffu, my_gate[u], j);
      if (j < k && active[u]) raw[u][j] = *reinterpret_cast<const uint4*>(y + r * H + c0[u]);
    }
    raw_s[u] = make_uint4(0, 0, 0, 0);
    if (shared && active[u]) raw_s[u] = *reinterpret_cast<const uint4*>(y + (R + t[u]) * H + c0[u]);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    if (!active[u]) continue;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        const uint32_t w[4] = {raw[u][j].x, raw[u][j].y, raw[u][j].z, raw[u][j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(g[u][j], __uint_as_float(w[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(g[u][j], __uint_as_float(w[i] & 0xFFFF0000u), acc[2 * i + 1]);
        }
      }
    }
    if (shared) {
      const uint32_t w[4] = {raw_s[u].x, raw_s[u].y, raw_s[u].z, raw_s[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
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
    *reinterpret_cast<uint4*>(out + (long)t[u] * H + c0[u]) = o;
  }
}

template <int KMAX>
__device__ __forceinline__ void combine_item(long item, const uint16_t* __restrict__ y,
                                             const int32_t* __restrict__ slot_pos, const float* __restrict__ gates,
                                             uint16_t* __restrict__ out, int T, int H, int k, int shared) {
  const long items[1] = {item};
  combine_items<KMAX, 1>(items, y, slot_pos, gates, out, T, H, k, shared);
}

}  // namespace
}  // namespace moe
