// FP8 E4M3 quantisation and dispatch kernels.
//
// DeepSeek-V3 technical report summary (xyznot.com), "Main ideas", FP8 bullet:
// E4M3 everywhere, tile-wise 1x128 activation scaling, block-wise 128x128
// weight scaling; "DeepSeek model architecture explained" (deepseekmodel.com),
// block-quantisation pseudocode: scale = max|x| / 448 (448 = largest E4M3).
// Codes are decided in fp32: scale = amax / 448 and the quotient x / scale
// are IEEE-rounded fp32 divisions, the quotient goes to E4M3 with
// round-to-nearest-even, saturating at +-448; an all-zero tile gets scale 1.
#pragma once
#include <cuda_fp8.h>
#include "dispatch.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kQBlock = 128;

__device__ __forceinline__ float fp8_scale_of(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

__device__ __forceinline__ uint8_t to_e4m3(float q) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t to_e4m3x4(float a, float b, float c, float d) {
  return static_cast<uint32_t>(to_e4m3(a)) | (static_cast<uint32_t>(to_e4m3(b)) << 8) |
         (static_cast<uint32_t>(to_e4m3(c)) << 16) | (static_cast<uint32_t>(to_e4m3(d)) << 24);
}

// ---------------------------------------------------------------- activations
// One warp per row, two 128-wide tiles per iteration: lanes 0-15 own tile 2i,
// lanes 16-31 tile 2i+1, 8 elements (one 16-byte vector) each.
__global__ void __launch_bounds__(256)
quant_act_fp8_kernel(const __nv_bfloat16* __restrict__ x, int rows, int cols,
                     uint8_t* __restrict__ q, float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int tiles = cols / kQBlock;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    const __nv_bfloat16* xr = x + static_cast<size_t>(r) * cols;
    for (int t0 = 0; t0 < tiles; t0 += 2) {
      const int tile = t0 + (lane >> 4);
      const bool active = tile < tiles;
      float v[8];
      float m = 0.0f;
      if (active) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xr + tile * kQBlock) + (lane & 15));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (active) {
        const float s = fp8_scale_of(m);
        uint2 out;
        out.x = to_e4m3x4(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s), __fdiv_rn(v[2], s),
                          __fdiv_rn(v[3], s));
        out.y = to_e4m3x4(__fdiv_rn(v[4], s), __fdiv_rn(v[5], s), __fdiv_rn(v[6], s),
                          __fdiv_rn(v[7], s));
        reinterpret_cast<uint2*>(q + static_cast<size_t>(r) * cols + tile * kQBlock)[lane & 15] =
            out;
        if ((lane & 15) == 0) scales[static_cast<size_t>(r) * tiles + tile] = s;
      }
    }
  }
}

// ---------------------------------------------------------------- weights
// One CTA per 128x128 block of one group's [R, C] matrix; thread t owns row
// t/2, columns (t%2)*64 .. +64 of the block.
__global__ void __launch_bounds__(256)
quant_weight_fp8_kernel(const __nv_bfloat16* __restrict__ w, int R, int C,
                        uint8_t* __restrict__ q, float* __restrict__ scales) {
  __shared__ float red[8];
  const int cb = blockIdx.x, rb = blockIdx.y, g = blockIdx.z;
  const int nrb = R / kQBlock, ncb = C / kQBlock;
  const int row = rb * kQBlock + (threadIdx.x >> 1);
  const int col = cb * kQBlock + (threadIdx.x & 1) * 64;
  const size_t base = (static_cast<size_t>(g) * R + row) * C + col;
  float v[64];
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(w + base) + j);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[8 * j + 2 * i] = f.x;
      v[8 * j + 2 * i + 1] = f.y;
    }
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
  const float s = fp8_scale_of(m);
  uint4* dst = reinterpret_cast<uint4*>(q + base);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 o;
    o.x = to_e4m3x4(__fdiv_rn(v[16 * j + 0], s), __fdiv_rn(v[16 * j + 1], s),
                    __fdiv_rn(v[16 * j + 2], s), __fdiv_rn(v[16 * j + 3], s));
    o.y = to_e4m3x4(__fdiv_rn(v[16 * j + 4], s), __fdiv_rn(v[16 * j + 5], s),
                    __fdiv_rn(v[16 * j + 6], s), __fdiv_rn(v[16 * j + 7], s));
    o.z = to_e4m3x4(__fdiv_rn(v[16 * j + 8], s), __fdiv_rn(v[16 * j + 9], s),
                    __fdiv_rn(v[16 * j + 10], s), __fdiv_rn(v[16 * j + 11], s));
    o.w = to_e4m3x4(__fdiv_rn(v[16 * j + 12], s), __fdiv_rn(v[16 * j + 13], s),
                    __fdiv_rn(v[16 * j + 14], s), __fdiv_rn(v[16 * j + 15], s));
    dst[j] = o;
  }
  if (threadIdx.x == 0) scales[(static_cast<size_t>(g) * nrb + rb) * ncb + cb] = s;
}

// ---------------------------------------------------------------- dispatch
// FP8 dispatch with the activation quantisation fused in: one warp per token
// reads its bf16 row once, quantises every 1x128 tile by the rule of
// quant_act_fp8_kernel (lanes 0-15 tile 2i, lanes 16-31 tile 2i+1) and writes
// the codes and the tile's scale to each of the token's K rows of x8 / xs;
// with u8 given, also to the token's own row of u8 / us (the shared expert's
// input). Each token is quantised once, however many experts it goes to.
__global__ void __launch_bounds__(256)
permute_quant_fp8_kernel(const __nv_bfloat16* __restrict__ u, const int32_t* __restrict__ pos,
                         int T, int d, int K, uint8_t* __restrict__ x8, float* __restrict__ xs,
                         uint8_t* __restrict__ u8, float* __restrict__ us) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const long long total = static_cast<long long>(T) * K;
  const int tiles = d / kQBlock;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const int my = lane < K ? pos[static_cast<size_t>(t) * K + lane] : -1;
    int p[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      p[k] = __shfl_sync(0xffffffffu, my, k);
      if (k >= K || p[k] < 0 || p[k] >= total) p[k] = -1;
    }
    const __nv_bfloat16* ur = u + static_cast<size_t>(t) * d;
    for (int t0 = 0; t0 < tiles; t0 += 2) {
      const int tile = t0 + (lane >> 4);
      const bool active = tile < tiles;
      float v[8];
      float m = 0.0f;
      if (active) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(ur + tile * kQBlock) + (lane & 15));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (!active) continue;
      const float s = fp8_scale_of(m);
      uint2 q;
      q.x = to_e4m3x4(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s), __fdiv_rn(v[2], s),
                      __fdiv_rn(v[3], s));
      q.y = to_e4m3x4(__fdiv_rn(v[4], s), __fdiv_rn(v[5], s), __fdiv_rn(v[6], s),
                      __fdiv_rn(v[7], s));
      const size_t col = static_cast<size_t>(tile) * kQBlock;
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k) {
        if (p[k] < 0) continue;
        reinterpret_cast<uint2*>(x8 + static_cast<size_t>(p[k]) * d + col)[lane & 15] = q;
        if ((lane & 15) == 0) xs[static_cast<size_t>(p[k]) * tiles + tile] = s;
      }
      if (u8) {
        reinterpret_cast<uint2*>(u8 + static_cast<size_t>(t) * d + col)[lane & 15] = q;
        if ((lane & 15) == 0) us[static_cast<size_t>(t) * tiles + tile] = s;
      }
    }
  }
}

// ---------------------------------------------------------------- w13 packing (E4M3)
// Codes of W1 and W3 stacked as [G, 2, inter, d] -> [G, 2*inter, d] with 64-row
// chunks interleaved: rows [128c, 128c+64) = W1 rows [64c, 64c+64), rows
// [128c+64, 128c+128) = W3 rows [64c, 64c+64). A 128-row tile of the result
// then holds the gate and up rows of the same 64 h columns.
__global__ void pack_w13_fp8_kernel(const uint8_t* __restrict__ stacked, int G, int inter, int d,
                                    uint8_t* __restrict__ w13) {
  const size_t nvec_row = static_cast<size_t>(d) >> 4;
  const size_t total = static_cast<size_t>(G) * 2 * inter * nvec_row;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t v = i % nvec_row;
    const size_t r = i / nvec_row;
    const size_t g = r / (2 * static_cast<size_t>(inter));
    const int row13 = static_cast<int>(r - g * 2 * inter);
    const int c = row13 >> 7;
    const int within = row13 & 127;
    const int which = within >> 6;                     // 0 = W1, 1 = W3
    const size_t srow = (g * 2 + which) * inter + c * 64 + (within & 63);
    reinterpret_cast<uint4*>(w13)[i] = __ldg(reinterpret_cast<const uint4*>(stacked + srow * d) + v);
  }
}

}  // namespace moe
