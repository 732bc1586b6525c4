// Backward of the routing, gating and combine steps of the DeepSeekMoE layer
// (the gradient of the forward layer of "DeepSeek-V3 technical report",
// Method §2; the pages print no backward equations, these are its exact
// derivative with the top-K selection held fixed). All HBM-bound: one warp
// per token, 16-byte vectors along d, fp32 accumulation, bf16 results.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "dispatch.cuh"

namespace moe {

constexpr int kBwdTokensPerBlock = 8;   // warps per block

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& q, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float (&f)[8]) {
  uint4 q;
  uint32_t* w = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 v = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&v);
  }
  return q;
}

// dgate[t,k] = dout_t . y_perm[pos[t,k]]   (the routed term g_k y_k of h'_t)
// dy_perm[pos[t,k]] = gate[t,k] dout_t
template <int TOPK>
__global__ void __launch_bounds__(32 * kBwdTokensPerBlock)
combine_backward_kernel(const __nv_bfloat16* __restrict__ dout,
                        const __nv_bfloat16* __restrict__ y_perm, const int32_t* __restrict__ pos,
                        const float* __restrict__ gate, int T, int d,
                        __nv_bfloat16* __restrict__ dy_perm, float* __restrict__ dgate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdTokensPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  int r[TOPK];
  float g[TOPK], dot[TOPK];
#pragma unroll
  for (int k = 0; k < TOPK; ++k) {
    r[k] = __ldg(pos + static_cast<size_t>(t) * TOPK + k);
    g[k] = __ldg(gate + static_cast<size_t>(t) * TOPK + k);
    dot[k] = 0.f;
  }
  const uint4* src = reinterpret_cast<const uint4*>(dout + static_cast<size_t>(t) * d);
  for (int v = lane; v < d / 8; v += 32) {
    float o[8];
    bf16x8_to_f32(__ldg(src + v), o);
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      float y[8], s[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(y_perm + static_cast<size_t>(r[k]) * d) + v), y);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dot[k] = fmaf(o[i], y[i], dot[k]);
        s[i] = g[k] * o[i];
      }
      reinterpret_cast<uint4*>(dy_perm + static_cast<size_t>(r[k]) * d)[v] = f32_to_bf16x8(s);
    }
  }
#pragma unroll
  for (int k = 0; k < TOPK; ++k) {
    const float s = warp_sum(dot[k]);
    if (lane == 0) dgate[static_cast<size_t>(t) * TOPK + k] = s;
  }
}

// dz[t,k] = dL/dz of the selected logits from dgate (KIND 0: sigmoid gate
// g_k = S s_k / sum_j s_j with s = sigmoid(u_t . e_k), recomputed here;
// KIND 1: g = S softmax of the selected logits). dz_perm[pos[t,k]] = dz[t,k].
template <int TOPK, int KIND>
__global__ void __launch_bounds__(32 * kBwdTokensPerBlock)
gate_backward_kernel(const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ e,
                     const int32_t* __restrict__ idx, const float* __restrict__ gate,
                     const float* __restrict__ dgate, const int32_t* __restrict__ pos, int T,
                     int d, float routed_scale, float* __restrict__ dz,
                     float* __restrict__ dz_perm) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdTokensPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  float dg[TOPK], out[TOPK];
#pragma unroll
  for (int k = 0; k < TOPK; ++k) dg[k] = __ldg(dgate + static_cast<size_t>(t) * TOPK + k);
  if constexpr (KIND == 0) {
    int ex[TOPK];
    float z[TOPK];
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      ex[k] = __ldg(idx + static_cast<size_t>(t) * TOPK + k);
      z[k] = 0.f;
    }
    const uint4* ur = reinterpret_cast<const uint4*>(u + static_cast<size_t>(t) * d);
    for (int v = lane; v < d / 8; v += 32) {
      float x[8];
      bf16x8_to_f32(__ldg(ur + v), x);
#pragma unroll
      for (int k = 0; k < TOPK; ++k) {
        float w[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(e + static_cast<size_t>(ex[k]) * d) + v), w);
#pragma unroll
        for (int i = 0; i < 8; ++i) z[k] = fmaf(x[i], w[i], z[k]);
      }
    }
    float s[TOPK], tot = 0.f, dgs = 0.f;
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      s[k] = 1.0f / (1.0f + __expf(-warp_sum(z[k])));
      tot += s[k];
      dgs = fmaf(dg[k], s[k], dgs);
    }
    const float inv = 1.0f / tot;
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      const float ds = routed_scale * inv * (dg[k] - dgs * inv);
      out[k] = ds * s[k] * (1.0f - s[k]);
    }
  } else {
    // p_k = g_k / S; dz_k = g_k (dg_k - sum_j p_j dg_j)
    float gk[TOPK], pdg = 0.f;
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      gk[k] = __ldg(gate + static_cast<size_t>(t) * TOPK + k);
      pdg = fmaf(gk[k] / routed_scale, dg[k], pdg);
    }
#pragma unroll
    for (int k = 0; k < TOPK; ++k) out[k] = gk[k] * (dg[k] - pdg);
  }
  if (lane < TOPK) {
    float v = out[0];
#pragma unroll
    for (int k = 1; k < TOPK; ++k)
      if (lane == k) v = out[k];
    dz[static_cast<size_t>(t) * TOPK + lane] = v;
    dz_perm[__ldg(pos + static_cast<size_t>(t) * TOPK + lane)] = v;
  }
}

// du_t = [dout_t] + [dx_shared_t] + sum_k dx_perm[pos[t,k]] + sum_k dz[t,k] e_{idx[t,k]}
template <int TOPK>
__global__ void __launch_bounds__(32 * kBwdTokensPerBlock)
combine_dx_kernel(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ dx_perm,
                  const int32_t* __restrict__ pos, const __nv_bfloat16* __restrict__ dx_shared,
                  const float* __restrict__ dz, const int32_t* __restrict__ idx,
                  const __nv_bfloat16* __restrict__ e, int T, int d,
                  __nv_bfloat16* __restrict__ du) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kBwdTokensPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  int r[TOPK], ex[TOPK];
  float z[TOPK];
#pragma unroll
  for (int k = 0; k < TOPK; ++k) {
    r[k] = __ldg(pos + static_cast<size_t>(t) * TOPK + k);
    ex[k] = __ldg(idx + static_cast<size_t>(t) * TOPK + k);
    z[k] = __ldg(dz + static_cast<size_t>(t) * TOPK + k);
  }
  for (int v = lane; v < d / 8; v += 32) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float x[8];
    if (dout) {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(dout + static_cast<size_t>(t) * d) + v), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += x[i];
    }
    if (dx_shared) {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(dx_shared + static_cast<size_t>(t) * d) + v), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += x[i];
    }
#pragma unroll
    for (int k = 0; k < TOPK; ++k) {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(dx_perm + static_cast<size_t>(r[k]) * d) + v), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += x[i];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(e + static_cast<size_t>(ex[k]) * d) + v), x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(z[k], x[i], acc[i]);
    }
    reinterpret_cast<uint4*>(du + static_cast<size_t>(t) * d)[v] = f32_to_bf16x8(acc);
  }
}

// de_i = sum over the rows r of group i of dz_perm[r] x_perm[r], in two
// passes so that a hot expert's rows are spread over many blocks and the sum
// keeps a fixed order (no atomics: reproducible):
//   table:  one block cuts every expert's rows into chunks of kCentroidChunk
//           rows (expert-major) and writes each chunk's row range;
//   pass 1: block (chunk, 256 columns) sums its <= 128 rows (warp w rows
//           w, w+8, ...; each lane 8 columns, four rows in flight), the 8 warp
//           partials added in order through shared memory, fp32 to workspace;
//   pass 2: block (expert, 256 columns) adds its chunks' partials in chunk
//           order and rounds once to bf16.
// Offsets are clamped into [0, rows] and made non-decreasing first, so x_perm
// is never read outside its rows.
constexpr int kCentroidCols = 256;
constexpr int kCentroidWarps = 8;
constexpr int kCentroidChunk = 128;
constexpr int kCentroidMaxExperts = 1024;

// Workspace: chunk_start [n + 1] int32 (first chunk of each expert, then the
// total), chunk_rows [max_chunks] int2 (row range), partials [max_chunks, d] fp32.
__host__ __device__ inline long long centroid_max_chunks(long long rows, int n) {
  return (rows + kCentroidChunk - 1) / kCentroidChunk + n;
}

__global__ void __launch_bounds__(1024)
centroid_chunk_table_kernel(const int32_t* __restrict__ offsets, int n, int rows,
                            int32_t* __restrict__ chunk_start, int2* __restrict__ chunk_rows) {
  __shared__ int s_lo[kCentroidMaxExperts + 1];
  __shared__ int s_scan[kCentroidMaxExperts];
  const int e = threadIdx.x;
  // clamped, non-decreasing offsets: running maximum of the clamped entries
  if (e <= n) s_lo[e] = min(max(__ldg(offsets + e), 0), rows);
  __syncthreads();
  for (int o = 1; o <= n; o <<= 1) {
    const int v = (e <= n && e >= o) ? s_lo[e - o] : 0;
    __syncthreads();
    if (e <= n && e >= o) s_lo[e] = max(s_lo[e], v);
    __syncthreads();
  }
  const int r0 = e < n ? s_lo[e] : 0;
  const int r1 = e < n ? s_lo[e + 1] : 0;
  const int nch = (r1 - r0 + kCentroidChunk - 1) / kCentroidChunk;
  if (e < kCentroidMaxExperts) s_scan[e] = nch;
  __syncthreads();
  for (int o = 1; o < kCentroidMaxExperts; o <<= 1) {
    const int v = (e < kCentroidMaxExperts && e >= o) ? s_scan[e - o] : 0;
    __syncthreads();
    if (e < kCentroidMaxExperts) s_scan[e] += v;
    __syncthreads();
  }
  if (e < n) {
    const int first = s_scan[e] - nch;
    chunk_start[e] = first;
    for (int j = 0; j < nch; ++j) {
      const int a = r0 + j * kCentroidChunk;
      chunk_rows[first + j] = make_int2(a, min(a + kCentroidChunk, r1));
    }
    if (e == n - 1) chunk_start[n] = s_scan[e];
  }
}

__global__ void __launch_bounds__(32 * kCentroidWarps)
centroid_partial_kernel(const __nv_bfloat16* __restrict__ x_perm,
                        const float* __restrict__ dz_perm, const int32_t* __restrict__ chunk_start,
                        const int2* __restrict__ chunk_rows, int n, int d,
                        float* __restrict__ partials) {
  __shared__ float part[kCentroidWarps][kCentroidCols + 4];
  const int c = blockIdx.x;
  if (c >= __ldg(chunk_start + n)) return;          // past the last chunk
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int col = blockIdx.y * kCentroidCols + lane * 8;
  const int2 rr = chunk_rows[c];
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (col < d) {
    int r = rr.x + warp;
    for (; r + 3 * kCentroidWarps < rr.y; r += 4 * kCentroidWarps) {
      uint4 q[4];
      float w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int rj = r + j * kCentroidWarps;
        q[j] = __ldg(reinterpret_cast<const uint4*>(x_perm + static_cast<size_t>(rj) * d + col));
        w[j] = __ldg(dz_perm + rj);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x[8];
        bf16x8_to_f32(q[j], x);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = fmaf(w[j], x[k], acc[k]);
      }
    }
    for (; r < rr.y; r += kCentroidWarps) {
      float x[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(x_perm + static_cast<size_t>(r) * d + col)), x);
      const float w = __ldg(dz_perm + r);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = fmaf(w, x[k], acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) part[warp][lane * 8 + k] = acc[k];
  __syncthreads();
  const int cc = blockIdx.y * kCentroidCols + threadIdx.x;
  if (threadIdx.x < kCentroidCols && cc < d) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kCentroidWarps; ++w) s += part[w][threadIdx.x];
    partials[static_cast<size_t>(c) * d + cc] = s;
  }
}

__global__ void __launch_bounds__(kCentroidCols)
centroid_reduce_kernel(const int32_t* __restrict__ chunk_start, const float* __restrict__ partials,
                       int d, __nv_bfloat16* __restrict__ de) {
  const int e = blockIdx.x;
  const int col = blockIdx.y * kCentroidCols + threadIdx.x;
  if (col >= d) return;
  const int c0 = __ldg(chunk_start + e), c1 = __ldg(chunk_start + e + 1);
  float s = 0.f;
  for (int c = c0; c < c1; ++c) s += __ldg(partials + static_cast<size_t>(c) * d + col);
  de[static_cast<size_t>(e) * d + col] = __float2bfloat16_rn(s);
}

}  // namespace moe
