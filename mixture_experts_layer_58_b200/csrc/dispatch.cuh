// Memory-bound kernels around the expert GEMMs: dispatch (permute), the
// gate-weighted combine, the bias update and the w13 packing helper.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kPermChunk = 128;   // tokens per dispatch chunk
constexpr int kMaxTopK = 8;

// ---------------------------------------------------------------- permute
// Pass 1: per chunk of 128 tokens, how many of its (token, slot) pairs go to
// each expert. hist is [n_chunks, n_routed] int32 (workspace).
__global__ void __launch_bounds__(256)
permute_hist_kernel(const int32_t* __restrict__ idx, int T, int K, int n_routed,
                    int32_t* __restrict__ hist) {
  __shared__ int h[256];
  for (int e = threadIdx.x; e < 256; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kPermChunk;
  const int n = min(kPermChunk, T - t0) * K;
  const int32_t* src = idx + static_cast<size_t>(t0) * K;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = src[i];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(n_routed)) atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x)
    hist[static_cast<size_t>(blockIdx.x) * n_routed + e] = h[e];
}

// Pass 2: expert offsets (exclusive scan of the counts), then for this chunk
// the row of every (token, slot) pair, handed out per expert in pair order
// (token-major, so the order inside an expert is stable). The chunk's pairs
// go in rounds of 256, one per thread: within a warp, __match_any_sync ranks
// the lanes that share an expert; per-warp counts are scanned across the 8
// warps in shared memory; a running per-expert row carries from round to
// round, and the chunk's first row per expert comes from the earlier chunks'
// histograms. Pairs whose expert is outside [0, n_routed) get pos = -1.
__global__ void __launch_bounds__(256)
permute_index_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                     const int32_t* __restrict__ hist, int T, int K, int n_routed,
                     int32_t* __restrict__ offsets, int32_t* __restrict__ pos,
                     int32_t* __restrict__ src_token) {
  __shared__ int s_scan[256];
  __shared__ int s_next[256];          // next row of each expert
  __shared__ int s_wcnt[8][256];       // this batch of 256 pairs: rows per (warp, expert), then their first row
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int chunk = blockIdx.x;
  const int t0 = chunk * kPermChunk;
  const int n = min(kPermChunk, T - t0) * K;
  const long long total = static_cast<long long>(T) * K;

  const int c = tid < n_routed ? counts[tid] : 0;
  s_scan[tid] = c;
  __syncthreads();
  for (int o = 1; o < 256; o <<= 1) {
    const int v = tid >= o ? s_scan[tid - o] : 0;
    __syncthreads();
    s_scan[tid] += v;
    __syncthreads();
  }
  const int excl = s_scan[tid] - c;
  if (chunk == 0 && tid < n_routed) {
    offsets[tid] = excl;
    if (tid == n_routed - 1) offsets[n_routed] = s_scan[tid];
  }
  if (tid < n_routed) {
    // the histogram loads are independent: keep eight in flight
    int base = excl;
    int cc = 0;
    for (; cc + 8 <= chunk; cc += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = hist[static_cast<size_t>(cc + j) * n_routed + tid];
#pragma unroll
      for (int j = 0; j < 8; ++j) base += v[j];
    }
    for (; cc < chunk; ++cc) base += hist[static_cast<size_t>(cc) * n_routed + tid];
    s_next[tid] = base;
  }

  const int32_t* idx_c = idx + static_cast<size_t>(t0) * K;
  int32_t* pos_c = pos + static_cast<size_t>(t0) * K;
  const unsigned lanes_below = (1u << lane) - 1u;
  for (int r0 = 0; r0 < n; r0 += 256) {          // same trip count in every thread
    for (int j = tid; j < 8 * 256; j += 256) (&s_wcnt[0][0])[j] = 0;
    __syncthreads();
    const int i = r0 + tid;
    int e = -1;
    if (i < n) {
      e = idx_c[i];
      if (static_cast<unsigned>(e) >= static_cast<unsigned>(n_routed)) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int before = __popc(peers & lanes_below);
    if (e >= 0 && before == 0) s_wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (tid < n_routed) {
      int run = s_next[tid];
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const int v = s_wcnt[w][tid];
        s_wcnt[w][tid] = run;
        run += v;
      }
      s_next[tid] = run;
    }
    __syncthreads();
    if (i < n) {
      int p = -1;
      if (e >= 0) {
        const int row = s_wcnt[warp][e] + before;
        if (row >= 0 && row < total) {
          p = row;
          src_token[row] = t0 + i / K;
        }
      }
      pos_c[i] = p;
    }
    __syncthreads();                              // s_wcnt is cleared for the next batch
  }
}

// Pass 3: one warp per token reads its row once (16-byte vectors) and writes
// it to each of its K rows of x_perm; TAIL: also to row T*K + t (the rows of
// the shared expert when it runs as the last group of the routed GEMMs).
template <bool TAIL>
__device__ __forceinline__ void permute_copy_rows(const __nv_bfloat16* __restrict__ u,
                                                  const int32_t* __restrict__ pos, int T, int d,
                                                  int K, __nv_bfloat16* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const long long total = static_cast<long long>(T) * K;
  const int nvec = d >> 3;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const int my = lane < K ? pos[static_cast<size_t>(t) * K + lane] : -1;
    int p[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      p[k] = __shfl_sync(0xffffffffu, my, k);
      if (k >= K || p[k] < 0 || p[k] >= total) p[k] = -1;
    }
    const uint4* srow = reinterpret_cast<const uint4*>(u + static_cast<size_t>(t) * d);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = v0 + 32 * j;
        if (v < nvec) x[j] = __ldg(srow + v);
      }
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k) {
        if (p[k] < 0) continue;
        uint4* drow = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(p[k]) * d);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = v0 + 32 * j;
          if (v < nvec) drow[v] = x[j];
        }
      }
      if constexpr (TAIL) {
        uint4* drow = reinterpret_cast<uint4*>(x_perm + (total + t) * d);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = v0 + 32 * j;
          if (v < nvec) drow[v] = x[j];
        }
      }
    }
  }
}

__global__ void __launch_bounds__(256)
permute_copy_kernel(const __nv_bfloat16* __restrict__ u, const int32_t* __restrict__ pos, int T,
                    int d, int K, __nv_bfloat16* __restrict__ x_perm) {
  permute_copy_rows<false>(u, pos, T, d, K, x_perm);
}

// The copy with the shared expert's rows appended, and the end of its group:
// expert_offsets[n_routed + 1] = T*K + T. The shared group starts where the
// routed rows end (expert_offsets[n_routed], T*K unless routed slots were
// skipped; rows in between are computed and never read).
__global__ void __launch_bounds__(256)
permute_copy_tail_kernel(const __nv_bfloat16* __restrict__ u, const int32_t* __restrict__ pos,
                         int T, int d, int K, __nv_bfloat16* __restrict__ x_perm,
                         int32_t* __restrict__ expert_offsets, int n_routed) {
  if (blockIdx.x == 0 && threadIdx.x == 0)
    expert_offsets[n_routed + 1] = static_cast<int32_t>(static_cast<long long>(T) * K + T);
  permute_copy_rows<true>(u, pos, T, d, K, x_perm);
}

// ---------------------------------------------------------------- combine
__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v, float w) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    a[2 * i] = fmaf(w, f.x, a[2 * i]);
    a[2 * i + 1] = fmaf(w, f.y, a[2 * i + 1]);
  }
}

__device__ __forceinline__ void add_bf16x8(float (&a)[8], const uint4& v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    a[2 * i] += f.x;
    a[2 * i + 1] += f.y;
  }
}

// out_t = residual_t + shared_t + sum_k g[t,k] * y_perm[pos[t,k]]; one warp
// per token, fp32 sums in a fixed order, one bf16 rounding.
// SLOTS (the fused-scatter mode): the routed rows already carry their gate
// and sit in slot order, y[t*K + k]; slot k counts when pos[t,k] >= 0.
template <bool SLOTS>
__global__ void __launch_bounds__(256, 2)   // two blocks per SM: 16 warps of loads in flight
combine_kernel(const __nv_bfloat16* __restrict__ y_perm, const int32_t* __restrict__ pos,
               const float* __restrict__ gate, const __nv_bfloat16* __restrict__ shared_out,
               const __nv_bfloat16* residual, int T, int d, int K,
               __nv_bfloat16* out) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const long long total = static_cast<long long>(T) * K;
  const int nvec = d >> 3;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const int myp = lane < K ? pos[static_cast<size_t>(t) * K + lane] : -1;
    const float myg = (!SLOTS && lane < K) ? gate[static_cast<size_t>(t) * K + lane] : 1.0f;
    int p[kMaxTopK];
    float g[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      p[k] = __shfl_sync(0xffffffffu, myp, k);
      g[k] = __shfl_sync(0xffffffffu, myg, k);
      if (k >= K || p[k] < 0 || p[k] >= total) p[k] = -1;
      else if (SLOTS) p[k] = t * K + k;
    }
    const size_t row = static_cast<size_t>(t) * d;
    for (int v0 = lane; v0 < nvec; v0 += 64) {
      float a[2][8];
      uint4 yv[2][kMaxTopK];
      uint4 rv[2], sv[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int v = v0 + 32 * j;
        if (v < nvec) {
          if (residual) rv[j] = *(reinterpret_cast<const uint4*>(residual + row) + v);
          if (shared_out) sv[j] = __ldg(reinterpret_cast<const uint4*>(shared_out + row) + v);
#pragma unroll
          for (int k = 0; k < kMaxTopK; ++k)
            if (p[k] >= 0)
              yv[j][k] = __ldg(reinterpret_cast<const uint4*>(
                                   y_perm + static_cast<size_t>(p[k]) * d) + v);
        }
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int v = v0 + 32 * j;
        if (v >= nvec) continue;
#pragma unroll
        for (int i = 0; i < 8; ++i) a[j][i] = 0.0f;
        if (residual) add_bf16x8(a[j], rv[j]);
        if (shared_out) add_bf16x8(a[j], sv[j]);
#pragma unroll
        for (int k = 0; k < kMaxTopK; ++k) {
          if (p[k] < 0) continue;
          if (SLOTS) add_bf16x8(a[j], yv[j][k]);
          else acc_bf16x8(a[j], yv[j][k], g[k]);
        }
        uint4 o;
        o.x = pack_bf16x2(a[j][0], a[j][1]);
        o.y = pack_bf16x2(a[j][2], a[j][3]);
        o.z = pack_bf16x2(a[j][4], a[j][5]);
        o.w = pack_bf16x2(a[j][6], a[j][7]);
        *(reinterpret_cast<uint4*>(out + row) + v) = o;
      }
    }
  }
}

// dst_slot[pos[s]] = s for every (token, slot) pair s = t*K + k that has a
// row in [0, rows); the caller sets dst_slot to -1 first, so rows no pair
// maps to stay -1. The inverse of the dispatch's pos.
__global__ void __launch_bounds__(256)
slot_index_kernel(const int32_t* __restrict__ pos, long long n_pairs, int rows,
                  int32_t* __restrict__ dst_slot) {
  for (long long s = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; s < n_pairs;
       s += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = pos[s];
    if (p >= 0 && p < rows) dst_slot[p] = static_cast<int32_t>(s);
  }
}

// ---------------------------------------------------------------- bias update
__global__ void bias_update_kernel(const int32_t* __restrict__ counts, float* __restrict__ bias,
                                   int n_routed, long long tk, float gamma) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_routed) {
    const long long load = static_cast<long long>(n_routed) * counts[i];
    const float b = bias[i];
    if (load > tk) bias[i] = __fsub_rn(b, gamma);
    else if (load < tk) bias[i] = __fadd_rn(b, gamma);
  }
}

// ---------------------------------------------------------------- w13 packing
// w13[g][32*c + r]      = w1[g][16*c + r]   (r < 16)
// w13[g][32*c + 16 + r] = w3[g][16*c + r]
// 16-row chunks: a 32-column slice of a GEMM accumulator then holds the gate
// and up products of the same 16 h columns, and so do the 32 TMEM lanes of one
// warp when the weights are the MMA's M side.
__global__ void pack_w13_kernel(const __nv_bfloat16* __restrict__ w1,
                                const __nv_bfloat16* __restrict__ w3, int G, int inter, int d,
                                __nv_bfloat16* __restrict__ w13) {
  const size_t nvec_row = static_cast<size_t>(d) >> 3;
  const size_t total = static_cast<size_t>(G) * 2 * inter * nvec_row;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t v = i % nvec_row;
    const size_t r = i / nvec_row;
    const size_t g = r / (2 * static_cast<size_t>(inter));
    const int row13 = static_cast<int>(r - g * 2 * inter);
    const int c = row13 >> 5;
    const int within = row13 & 31;
    const __nv_bfloat16* srcm = within < 16 ? w1 : w3;
    const size_t srow = g * inter + c * 16 + (within & 15);
    reinterpret_cast<uint4*>(w13)[i] = __ldg(reinterpret_cast<const uint4*>(srcm + srow * d) + v);
  }
}

}  // namespace moe
