// Backward GEMMs of the grouped SwiGLU expert FFNs on tcgen05 (bf16 operands,
// fp32 accumulation in TMEM, bf16 results).
//
// Data gradient (dgrad), per group g:  D = A[rows of g] * W_g, where A is a
// K-major [rows, K] operand (the incoming gradient) and W_g a [K, N] weight
// block stored row-major, i.e. the MMA's B operand read MN-major: TMA boxes
// of 64 N-columns x 64 K-rows land as 128B-swizzled atoms of 8 K-rows, and
// the descriptor steps 2 KB per K = 16. Used for dh = dy W2 (with the SwiGLU
// backward fused into the epilogue) and dx = [da|dc] W13.
//
// Weight gradient (wgrad), per group g:  dW_g = A_g^T B_g, the contraction
// over the group's token rows: A [rows, M] and B [rows, N] are both read
// MN-major (64-row K blocks). A group's last K block usually runs past its
// rows into the next group's; the MMA warp zeroes those rows of the A tile in
// shared memory (generic-proxy stores, then fence.proxy.async) before the MMA
// reads it, so they add nothing. Used for dW2 = dy^T h and dW13 = [da|dc]^T x.
//
// Both kernels keep the forward kernel's shape: one persistent CTA per SM,
// warp 0 TMA producer, warp 1 MMA issuer, warps 2-5 epilogue, a 4-stage ring
// of 48 KB and a double-buffered 2 x 256-column TMEM accumulator; tiles in
// index order from a global counter (tileq.cuh); all waits bounded, no TMA
// multicast.
#pragma once
#include "gemm.cuh"
#include "tileq.cuh"

namespace moe {

enum { EPI_DG_STORE = 0, EPI_DG_SWIGLU_BWD = 1 };

struct BwdCfg {
  static constexpr int kBN = 256;
  static constexpr int kBoxBytes = 64 * kBK * 2;        // 64 x 64 bf16 = 8 KB
  static constexpr int kABytes = kBM * kBK * 2;         // 16 KB
  static constexpr int kBBytes = 4 * kBoxBytes;         // 32 KB: 256 N x 64 K
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarBytes = 256;
  // wgrad: its own ring depth, and per epilogue warp kWgOutBufs 32 x 32 bf16
  // buffers for TMA stores (a chunk waits only for the store issued
  // kWgOutBufs chunks before it to have read its buffer)
  static constexpr int kWgStages = 4;
  static constexpr int kWgOutBufs = 2;
  static constexpr int kWgEpiWarps = 4;   // in groups of 4 (one per TMEM lane quarter)
  static constexpr int kWgThreads = 64 + 32 * kWgEpiWarps;
  static constexpr int kOutBufBytes = 32 * 32 * 2;
  static constexpr int kOutBytes = kWgEpiWarps * kWgOutBufs * kOutBufBytes;
  static size_t wgrad_smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kWgStages) * kStageBytes + kOutBytes + kBarBytes +
           2 * static_cast<size_t>(G + 1) * sizeof(int);
  }
  static size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kStages) * kStageBytes + kBarBytes +
           3 * static_cast<size_t>(G + 1) * sizeof(int);
  }
};

__device__ __forceinline__ float sigmoid_f32(float a) { return 1.0f / (1.0f + __expf(-a)); }

// ---------------------------------------------------------------------------
// dgrad: out[rows of g, n] = sum_k A[row, k] W_g[k, n]; K = w_rows per group.
// EPI_DG_SWIGLU_BWD: n indexes h columns (N = inter); with ac [rows, 2*inter]
// the saved forward pre-activations (a, c interleaved in 16-column chunks like
// the packed W13 rows), the epilogue writes dac [rows, 2*inter] in the same
// layout: da = dh c silu'(a), dc = dh silu(a).
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_dgrad_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmW,
                          const int32_t* __restrict__ offsets, int G, int K, int N, int rows,
                          __nv_bfloat16* __restrict__ out, int ldo,
                          const __nv_bfloat16* __restrict__ ac, int* tile_counter,
                          unsigned int* status) {
  using C = BwdCfg;
  constexpr int BN = C::kBN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * C::kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* tq_full = mma_done + 1;
  uint64_t* tq_empty = tq_full + kCtaTileQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_empty + kCtaTileQ);
  int* tq = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_tstart = s_off + (G + 1);
  int* s_end = s_tstart + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks_n = (N + BN - 1) / BN;   // N % 128 == 0: the last block may be half
  const int num_kb = K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], 128);
      }
      mbar_init(mma_done, 1);
      for (int j = 0; j < kCtaTileQ; ++j) {
        mbar_init(&tq_full[j], 1);
        mbar_init(&tq_empty[j], 5);   // MMA role + 4 epilogue warps
      }
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmW);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  } else if (warp == 1) {
    build_group_table(offsets, G, rows, kBM, n_blocks_n, s_off, s_end, s_tstart, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_tstart[G];

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    bool ok = true;
    int t_next = atomicAdd(tile_counter, 1);
    for (int i = 0; ok; ++i) {
      const int t = min(t_next, total_tiles);
      if (!cta_tile_push(i, t, tq, tq_full, tq_empty, status) || t >= total_tiles) break;
      t_next = atomicAdd(tile_counter, 1);
      int g, m_blk, n_blk;
      decode_tile(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int a_row = s_off[g] + m_blk * kBM;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
        tma_load_2d(sA + stage * C::kABytes, &tmA, &full[stage], kb * kBK, a_row);
        uint8_t* b = sB + stage * C::kBBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d(b + j * C::kBoxBytes, &tmW, &full[stage], n_blk * BN + 64 * j,
                      g * K + kb * kBK);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    for (int s = 0; s < kStages; ++s)
      if (issued & (1u << s))
        mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32_mn(kBM, BN, false, true);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int local = 0; ok; ++local) {
      int t;
      if (!cta_tile_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutMma) ||
          t >= total_tiles)
        break;
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(&tempty[acc], acc_par ^ 1u, status, kStatusTimeoutMma)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, status, kStatusTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * C::kABytes));
        const uint64_t bdesc =
            sw128_mnmajor_desc(smem_u32(sB + stage * C::kBBytes), C::kBoxBytes);
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k)
          umma_bf16(d_tmem, adesc + 2u * k, bdesc + 128u * k, idesc, (kb | k) != 0);
        umma_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) umma_commit(&tfull[acc]);
    }
    umma_commit(mma_done);
    mbar_wait(mma_done, 0, status, kStatusTimeoutMma);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    for (int local = 0;; ++local) {
      int t = total_tiles;
      bool got = true;
      if (lane == 0)
        got = cta_tile_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutEpilogue);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!got || t >= total_tiles) break;
      int g, m_blk, n_blk;
      decode_tile(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      const int grow = s_off[g] + m_blk * kBM + row_in_tile;
      const bool valid = grow < min(s_end[g], rows);
      const int ncols = min(BN, N - n_blk * BN);
      // SwiGLU backward: the saved [a|c] of this row, one 128-byte piece per
      // 32 h columns, loaded a chunk ahead (the first while the MMAs of the
      // tile still run) so its latency overlaps the work
      const uint4* ac_row = nullptr;
      uint4 in_next[8];
      if constexpr (EPI == EPI_DG_SWIGLU_BWD) {
        ac_row = reinterpret_cast<const uint4*>(ac + static_cast<size_t>(valid ? grow : 0) * ldo +
                                                2 * (n_blk * BN));
        if (valid) {
#pragma unroll
          for (int v = 0; v < 8; ++v) in_next[v] = __ldg(ac_row + v);
        }
      }
      if (!mbar_wait(&tfull[acc], acc_par, status, kStatusTimeoutEpilogue)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * BN + lane_addr;
#pragma unroll 1
      for (int c = 0; c < ncols; c += 32) {
        uint32_t r[32];
        uint4 in[8];
        if constexpr (EPI == EPI_DG_SWIGLU_BWD) {
#pragma unroll
          for (int v = 0; v < 8; ++v) in[v] = in_next[v];
          if (valid && c + 32 < ncols) {
#pragma unroll
            for (int v = 0; v < 8; ++v) in_next[v] = __ldg(ac_row + (c + 32) / 4 + v);
          }
        }
        tmem_ld_32cols(taddr + c, r);
        tmem_ld_wait();
        if (!valid) continue;
        if constexpr (EPI == EPI_DG_STORE) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * ldo +
                                                n_blk * BN + c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        } else {
          // h columns j0 + [0, 32) <-> ac / dac columns 2*j0 + [0, 64):
          // [a 0..15 | c 0..15 | a 16..31 | c 16..31]
          const int j0 = n_blk * BN + c;
          const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(in);
          uint32_t pk[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              float da[2], dc[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const float a = __bfloat162float(x[32 * half + i + e]);
                const float cc = __bfloat162float(x[32 * half + 16 + i + e]);
                const float dh = __uint_as_float(r[16 * half + i + e]);
                const float sg = sigmoid_f32(a);
                dc[e] = dh * (a * sg);
                da[e] = dh * cc * (sg * (1.0f + a * (1.0f - sg)));
              }
              pk[16 * half + i / 2] = pack_bf16x2(da[0], da[1]);
              pk[16 * half + 8 + i / 2] = pack_bf16x2(dc[0], dc[1]);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * ldo + 2 * j0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

// ---------------------------------------------------------------------------
// wgrad: dW[g][m][n] = sum over the rows r of group g of A[r, m] B[r, n];
// A [rows, M], B [rows, N], dW [G, M, N] bf16. Tiles (g, 128-row m block,
// 256-column n block), m blocks fastest; a group without rows writes zeros.
__global__ void __launch_bounds__(BwdCfg::kWgThreads, 1)
grouped_wgrad_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmD,
                          const int32_t* __restrict__ offsets, int G, int M, int N, int rows,
                          int* tile_counter, unsigned int* status) {
  using C = BwdCfg;
  constexpr int BN = C::kBN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kWgStages * C::kABytes;
  uint8_t* sOut = sB + C::kWgStages * C::kBBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::kOutBytes);
  uint64_t* empty = full + C::kWgStages;
  uint64_t* tfull = empty + C::kWgStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* tq_full = mma_done + 1;
  uint64_t* tq_empty = tq_full + kCtaTileQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_empty + kCtaTileQ);
  int* tq = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_end = s_off + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mb = M / kBM;
  const int nb = (N + BN - 1) / BN;   // N % 128 == 0: the last block may be half
  const int per_group = mb * nb;
  const int total_tiles = G * per_group;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < C::kWgStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], 32 * C::kWgEpiWarps);
      }
      mbar_init(mma_done, 1);
      for (int j = 0; j < kCtaTileQ; ++j) {
        mbar_init(&tq_full[j], 1);
        mbar_init(&tq_empty[j], 1 + C::kWgEpiWarps);   // MMA role + the epilogue warps
      }
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      tma_prefetch_desc(&tmD);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  } else if (warp == 1) {
    build_group_table(offsets, G, rows, kBM, 0, s_off, s_end, nullptr, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    bool ok = true;
    int t_next = atomicAdd(tile_counter, 1);
    for (int i = 0; ok; ++i) {
      const int t = min(t_next, total_tiles);
      if (!cta_tile_push(i, t, tq, tq_full, tq_empty, status) || t >= total_tiles) break;
      t_next = atomicAdd(tile_counter, 1);
      const int g = t / per_group;
      const int rem = t - g * per_group;
      const int n_blk = rem / mb;
      const int m_blk = rem - n_blk * mb;
      const int r0 = s_off[g];
      const int nkb = (s_end[g] - r0 + kBK - 1) / kBK;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
        uint8_t* a = sA + stage * C::kABytes;
        uint8_t* b = sB + stage * C::kBBytes;
        const int y = r0 + kb * kBK;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          tma_load_2d(a + j * C::kBoxBytes, &tmA, &full[stage], m_blk * kBM + 64 * j, y);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tma_load_2d(b + j * C::kBoxBytes, &tmB, &full[stage], n_blk * BN + 64 * j, y);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kWgStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    for (int s = 0; s < C::kWgStages; ++s)
      if (issued & (1u << s))
        mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA warp
    // Lane 0 issues the MMAs; the whole warp zeroes the A rows past a group's
    // end in its last K block.
    constexpr uint32_t idesc = idesc_bf16_f32_mn(kBM, BN, true, true);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int local = 0; ok; ++local) {
      int t = total_tiles;
      bool popped = true;
      if (lane == 0)
        popped = cta_tile_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutMma);
      popped = __shfl_sync(0xffffffffu, popped ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!popped || t >= total_tiles) break;
      const int g = t / per_group;
      const int r0 = s_off[g];
      const int m_rows = s_end[g] - r0;
      const int nkb = (m_rows + kBK - 1) / kBK;
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      // every lane waits (acquire); lane 0's outcome decides for the warp
      bool got = mbar_wait(&tempty[acc], acc_par ^ 1u, status, kStatusTimeoutMma);
      if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < nkb; ++kb) {
        got = mbar_wait(&full[stage], phase, status, kStatusTimeoutMma);
        if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0) {
          ok = false;
          break;
        }
        const int valid = m_rows - kb * kBK;   // rows of this K block inside the group
        if (valid < kBK) {
          uint4* a = reinterpret_cast<uint4*>(sA + stage * C::kABytes);
          // each 64-column box: row r = bytes [128 r, 128 r + 128)
          for (int q = valid * 8 + lane; q < 64 * 8; q += 32) {
            a[q] = make_uint4(0u, 0u, 0u, 0u);
            a[q + C::kBoxBytes / 16] = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint64_t adesc =
              sw128_mnmajor_desc(smem_u32(sA + stage * C::kABytes), C::kBoxBytes);
          const uint64_t bdesc =
              sw128_mnmajor_desc(smem_u32(sB + stage * C::kBBytes), C::kBoxBytes);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            umma_bf16(d_tmem, adesc + 128u * k, bdesc + 128u * k, idesc, (kb | k) != 0);
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::kWgStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && lane == 0) umma_commit(&tfull[acc]);
      __syncwarp();
    }
    if (lane == 0) {
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, status, kStatusTimeoutMma);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // Each warp owns TMEM lanes (= dW rows) quarter*32..+32. Per 32 columns
    // it writes its 32 x 32 bf16 block into one of two shared buffers and a
    // single lane stores the block with TMA (dW tiles are whole, and the
    // tensor map clips a last half block at N), so the global writes are
    // full rows of 64 B instead of one 16-B piece per row per instruction.
    // The buffer uses the 64-byte swizzle of the tensor map: 16-B chunk q of
    // row r sits at chunk q ^ ((r >> 1) & 3), so the 8 rows one phase of a
    // 16-B shared store touches fall in 8 different bank groups.
    const int quarter = warp & 3;
    const int eg = (warp - 2) >> 2;   // group eg drains columns [eg * BN / groups, +BN / groups)
    constexpr int kGroups = C::kWgEpiWarps / 4;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* obuf = sOut + (warp - 2) * C::kWgOutBufs * C::kOutBufBytes;
    const int sw = (lane >> 1) & 3;
    int chunk = 0;
    for (int local = 0;; ++local) {
      int t = total_tiles;
      bool got = true;
      if (lane == 0)
        got = cta_tile_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutEpilogue);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!got || t >= total_tiles) break;
      const int g = t / per_group;
      const int rem = t - g * per_group;
      const int n_blk = rem / mb;
      const int m_blk = rem - n_blk * mb;
      const bool empty_group = s_end[g] <= s_off[g];
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_par, status, kStatusTimeoutEpilogue)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + acc * BN + lane_addr;
      const int y = g * M + m_blk * kBM + quarter * 32;
      const int ncols = min(BN, N - n_blk * BN);   // 128 or 256
#pragma unroll 1
      for (int c = eg * (BN / kGroups); c < min(ncols, (eg + 1) * (BN / kGroups)); c += 64) {
        uint32_t r[2][32];
        tmem_ld_32cols(taddr + c, r[0]);
        tmem_ld_32cols(taddr + c + 32, r[1]);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h, ++chunk) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = empty_group ? 0u
                                : pack_bf16x2(__uint_as_float(r[h][2 * i]),
                                              __uint_as_float(r[h][2 * i + 1]));
          uint8_t* buf = obuf + (chunk % C::kWgOutBufs) * C::kOutBufBytes;
          // the store issued from this buffer kWgOutBufs chunks ago must have read it
          if (lane == 0) bulk_wait_group_read<C::kWgOutBufs - 1>();
          __syncwarp();
          uint4* row = reinterpret_cast<uint4*>(buf + lane * 64);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            row[v ^ sw] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmD, buf, n_blk * BN + c + 32 * h, y);
            bulk_commit_group();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    // shared memory stays valid until every store has read it
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

}  // namespace moe
