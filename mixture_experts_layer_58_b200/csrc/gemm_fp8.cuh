// Grouped FP8 (E4M3) GEMM with FP32 promotion every 128 K, on tcgen05.
//
// DeepSeek-V3 technical report summary (xyznot.com), "Main ideas", FP8 bullet:
// E4M3 operands with 1x128 activation tiles and 128x128 weight blocks, and the
// accumulation moved to FP32 on CUDA cores every N_c = 128 steps of K
// ("Problem setting": FP8 tensor cores accumulate with limited precision).
//
// For every 128-wide K block kb the tensor cores form the block's product
//   P_kb[m, n] = sum_{k in kb} qa[m, k] * qw[n, k]
// from a fresh start (tcgen05.mma kind::f8f6f4, 4 x K=32) into one of two
// 128-column TMEM buffers, and the epilogue warps fold it into fp32 registers:
//   acc[m, n] += P_kb[m, n] * s_a[m, kb] * s_w[block of n, kb].
// The scales are the pages' arbitrary fp32 values (max|x| / 448), which the
// hardware's block-scaled MMA (power-of-two, 32-element scale blocks) cannot
// express; promotion on the CUDA cores keeps them exact.
//
// 10 warps, one persistent CTA per SM, 128 x 128 tiles:
//   warp 0      TMA producer: A [128 rows x 128 B] + B [128 rows x 128 B] per stage,
//               6 stages; takes the tiles in index order from a global counter
//               and hands each index to the other roles (tileq.cuh).
//   warp 1      MMA issuer: one K block (4 x K=32) per P buffer, four buffers of
//               128 TMEM columns (the MMA runs up to three blocks ahead of the
//               promotion).
//   warps 2-9   promotion + epilogue. Warp w reads TMEM lane quarter w % 4;
//               half = (w - 2) / 4 picks its 64 columns: for the up-projection
//               the gate columns [32*half, +32) and the up columns
//               [64 + 32*half, +32) of the same 32 h columns (B is W1/W3
//               interleaved in 64-row chunks), for the down-projection the
//               columns [64*half, +64). 64 fp32 accumulators per thread.
// Epilogues: EPI8_SWIGLU_Q — h = silu(a) * b quantised in the epilogue,
// straight from its fp32 value, to E4M3 codes with one fp32 scale per 1x128
// tile of h (the activation rule: scale = max|h| / 448, codes decided in
// fp32), so h never goes to memory in a wider type; EPI8_STORE — bf16 output.
// A 1x128 tile of h spans two 128-column tiles of the up-projection (64 h
// columns each), so EPI8_SWIGLU_Q gives each CTA tile two column sub-tiles
// of the same token rows, one after the other: a thread keeps its 32 h values
// of the first in registers, and the two warps that hold the other 64 columns
// of its row exchange their partial maxima through shared memory.
#pragma once
#include "fp8.cuh"
#include "gemm.cuh"
#include "tileq.cuh"

namespace moe {

constexpr int kF8BK = 128;        // K elements (= bytes) per stage = one scale block
constexpr int kF8UmmaK = 32;      // K of one tcgen05.mma kind::f8f6f4
constexpr int kF8BN = 128;
constexpr int kF8Stages = 6;
constexpr int kF8Threads = 320;
constexpr int kF8EpiThreads = 256;

enum { EPI8_STORE = 0, EPI8_SWIGLU_Q = 2 };

// column sub-tiles per CTA tile
template <int EPI>
__host__ __device__ constexpr int f8_subtiles() { return EPI == EPI8_SWIGLU_Q ? 2 : 1; }

struct GemmF8Cfg {
  static constexpr int kABytes = kBM * kF8BK;
  static constexpr int kBBytes = kF8BN * kF8BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kPBufs = 4;                // P buffers of 128 TMEM columns
  static constexpr int kTmemCols = kPBufs * kF8BN;
  static constexpr int kBarBytes = 512;
  static constexpr int kRedBytes = 2 * 128 * 2 * 4;   // [2 tiles][128 rows][2 halves] fp32
  static size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kF8Stages) * kStageBytes + kRedBytes + kBarBytes +
           3 * static_cast<size_t>(G + 1) * sizeof(int);
  }
};

// Instruction descriptor of tcgen05.mma kind::f8f6f4: E4M3 A and B (format
// code 0, K-major), fp32 accumulator, shape M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The 8 epilogue warps meet between writing and reading a reduction buffer:
// lane 0 of each arrives once its warp's writes are done, every lane waits
// (bounded).
__device__ __forceinline__ bool xfer_sync_f8(uint64_t* bar, uint32_t parity, int lane,
                                             unsigned int* status) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  return mbar_wait(bar, parity, status, kStatusTimeoutEpilogue);
}

template <int EPI>
__global__ void __launch_bounds__(kF8Threads, 1)
grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const float* __restrict__ a_scales, const float* __restrict__ b_scales,
                        const int32_t* __restrict__ offsets, int G, int K, int n_per_group,
                        int rows, __nv_bfloat16* __restrict__ out, int ldo,
                        uint8_t* __restrict__ qout, float* __restrict__ qscales,
                        int* tile_counter, unsigned int* status) {
  using C = GemmF8Cfg;
  constexpr int SUB = f8_subtiles<EPI>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kF8Stages * C::kABytes;
  float* s_red = reinterpret_cast<float*>(sB + kF8Stages * C::kBBytes);   // [2][128][2]
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s_red) + C::kRedBytes);
  uint64_t* empty = full + kF8Stages;
  uint64_t* pfull = empty + kF8Stages;
  uint64_t* pempty = pfull + C::kPBufs;
  uint64_t* mma_done = pempty + C::kPBufs;
  uint64_t* tq_full = mma_done + 1;
  uint64_t* tq_empty = tq_full + kCtaTileQ;
  uint64_t* red_bar = tq_empty + kCtaTileQ;   // [2]: the 8 epilogue warps wrote s_red[i]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 2);
  int* tq = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_tstart = s_off + (G + 1);
  int* s_end = s_tstart + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks_n = n_per_group / (kF8BN * SUB);   // column tiles (of SUB sub-tiles)
  const int num_kb = K / kF8BK;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kF8Stages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int b = 0; b < C::kPBufs; ++b) {
        mbar_init(&pfull[b], 1);
        mbar_init(&pempty[b], kF8EpiThreads);
      }
      mbar_init(mma_done, 1);
      for (int j = 0; j < kCtaTileQ; ++j) {
        mbar_init(&tq_full[j], 1);
        mbar_init(&tq_empty[j], 1 + kF8EpiThreads / 32);   // MMA thread + epilogue warps
      }
      mbar_init(&red_bar[0], kF8EpiThreads / 32);
      mbar_init(&red_bar[1], kF8EpiThreads / 32);
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, C::kTmemCols);
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
      for (int sub = 0; sub < SUB && ok; ++sub) {
        const int b_row = g * n_per_group + (n_blk * SUB + sub) * kF8BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_2d(sA + stage * C::kABytes, &tmA, &full[stage], kb * kF8BK, a_row);
          tma_load_2d(sB + stage * C::kBBytes, &tmB, &full[stage], kb * kF8BK, b_row);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kF8Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    for (int s = 0; s < kF8Stages; ++s)
      if (issued & (1u << s))
        mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_e4m3_f32(kBM, kF8BN);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t kcount = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      int t;
      if (!cta_tile_pop(i, tq, tq_full, tq_empty, t, status, kStatusTimeoutMma) ||
          t >= total_tiles)
        break;
      for (int kb = 0; kb < SUB * num_kb; ++kb, ++kcount) {
        const uint32_t pb = kcount % C::kPBufs;
        const uint32_t ppar = (kcount / C::kPBufs) & 1u;
        if (!mbar_wait(&pempty[pb], ppar ^ 1u, status, kStatusTimeoutMma) ||
            !mbar_wait(&full[stage], phase, status, kStatusTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * C::kABytes));
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * C::kBBytes));
        const uint32_t d_tmem = tmem_base + pb * kF8BN;
#pragma unroll
        for (int k = 0; k < kF8BK / kF8UmmaK; ++k)   // 32 bytes of K per MMA
          umma_e4m3(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, k != 0);
        umma_commit(&empty[stage]);
        umma_commit(&pfull[pb]);
        if (++stage == kF8Stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    umma_commit(mma_done);
    mbar_wait(mma_done, 0, status, kStatusTimeoutMma);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ promotion + epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    // the thread's two runs of 32 columns
    constexpr bool kSwiglu = EPI == EPI8_SWIGLU_Q;
    const int col0 = kSwiglu ? 32 * half : 64 * half;
    const int col1 = kSwiglu ? 64 + 32 * half : 64 * half + 32;
    const int ksb = num_kb;                   // scale blocks along K
    uint32_t kcount = 0;
    bool broken = false;
    for (int it = 0;; ++it) {
      int t = total_tiles;
      bool got = true;
      if (lane == 0)
        got = cta_tile_pop(it, tq, tq_full, tq_empty, t, status, kStatusTimeoutEpilogue);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!got || t >= total_tiles) break;
      int g, m_blk, n_blk;
      decode_tile(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int row0 = s_off[g] + m_blk * kBM;
      const int row_end = min(s_end[g], rows);
      const int grow = row0 + row_in_tile;
      const bool valid = grow >= 0 && grow < row_end;
      const float* sa_row = a_scales + static_cast<size_t>(valid ? grow : 0) * ksb;
      float hkeep[32];                        // EPI8_SWIGLU_Q: h of the first sub-tile
#pragma unroll 1
      for (int sub = 0; sub < SUB; ++sub) {
        const int nb_col = n_blk * SUB + sub;   // 128-column tile of the B rows
        // weight scale rows of the two column runs
        const float* sw0;
        const float* sw1;
        if constexpr (kSwiglu) {
          // b_scales [G, 2, inter/128, K/128]: W1 blocks, then W3 blocks
          const int nb = n_per_group / 2 / kQBlock;
          const int hb = (nb_col * 64) / kQBlock;
          sw0 = b_scales + ((static_cast<size_t>(g) * 2 + 0) * nb + hb) * ksb;
          sw1 = b_scales + ((static_cast<size_t>(g) * 2 + 1) * nb + hb) * ksb;
        } else {
          // b_scales [G, N/128, K/128]
          const int nb = n_per_group / kQBlock;
          sw0 = b_scales + (static_cast<size_t>(g) * nb + nb_col) * ksb;
          sw1 = sw0;
        }
        float acc0[32], acc1[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          acc0[j] = 0.0f;
          acc1[j] = 0.0f;
        }
        float sa_n = valid ? __ldg(sa_row) : 0.0f;
        float w0_n = __ldg(sw0), w1_n = __ldg(sw1);
#pragma unroll 1
        for (int kb = 0; kb < num_kb; ++kb, ++kcount) {
          const float s0 = sa_n * w0_n;
          const float s1 = sa_n * w1_n;
          if (kb + 1 < num_kb) {
            sa_n = valid ? __ldg(sa_row + kb + 1) : 0.0f;
            w0_n = __ldg(sw0 + kb + 1);
            w1_n = __ldg(sw1 + kb + 1);
          }
          const uint32_t pb = kcount % C::kPBufs;
          const uint32_t ppar = (kcount / C::kPBufs) & 1u;
          if (!broken && !mbar_wait(&pfull[pb], ppar, status, kStatusTimeoutEpilogue))
            broken = true;
          tc_fence_after();
          const uint32_t taddr = tmem_base + pb * kF8BN + lane_addr;
          uint32_t r0[32], r1[32];
          tmem_ld_32cols(taddr + col0, r0);
          tmem_ld_32cols(taddr + col1, r1);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&pempty[pb]);
          // packed fp32 FMAs (two lanes of fp32 per instruction, each
          // rounded as a scalar fmaf): the promotion warps are bound by the
          // instructions they issue per 128-K block, and this halves its FMAs
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 q0 =
                __ffma2_rn(make_float2(__uint_as_float(r0[i]), __uint_as_float(r0[i + 1])),
                           make_float2(s0, s0), make_float2(acc0[i], acc0[i + 1]));
            const float2 q1 =
                __ffma2_rn(make_float2(__uint_as_float(r1[i]), __uint_as_float(r1[i + 1])),
                           make_float2(s1, s1), make_float2(acc1[i], acc1[i + 1]));
            acc0[i] = q0.x;
            acc0[i + 1] = q0.y;
            acc1[i] = q1.x;
            acc1[i + 1] = q1.y;
          }
        }
        if constexpr (EPI == EPI8_SWIGLU_Q) {
          if (sub == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) hkeep[i] = silu_f32(acc0[i]) * acc1[i];
            continue;
          }
          // sub-tile 1: this thread holds h columns [32*half, +32) (hkeep) and
          // [64 + 32*half, +32) (below) of the row's 1x128 tile n_blk; the
          // warp of the other half holds the rest
          float h1[32];
          float m = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            h1[i] = silu_f32(acc0[i]) * acc1[i];
            m = fmaxf(m, fmaxf(fabsf(hkeep[i]), fabsf(h1[i])));
          }
          const int rb = it & 1;
          float* red = s_red + rb * 256;
          red[row_in_tile * 2 + half] = m;
          if (!xfer_sync_f8(&red_bar[rb], (it >> 1) & 1, lane, status)) {
            broken = true;
            break;
          }
          const float amax = fmaxf(red[row_in_tile * 2], red[row_in_tile * 2 + 1]);
          if (valid) {
            const float sc = fp8_scale_of(amax);
            uint8_t* qrow = qout + static_cast<size_t>(grow) * ldo + n_blk * kQBlock;
            uint4 c0[2], c1[2];
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              c0[v] = make_uint4(
                  to_e4m3x4(__fdiv_rn(hkeep[16 * v + 0], sc), __fdiv_rn(hkeep[16 * v + 1], sc),
                            __fdiv_rn(hkeep[16 * v + 2], sc), __fdiv_rn(hkeep[16 * v + 3], sc)),
                  to_e4m3x4(__fdiv_rn(hkeep[16 * v + 4], sc), __fdiv_rn(hkeep[16 * v + 5], sc),
                            __fdiv_rn(hkeep[16 * v + 6], sc), __fdiv_rn(hkeep[16 * v + 7], sc)),
                  to_e4m3x4(__fdiv_rn(hkeep[16 * v + 8], sc), __fdiv_rn(hkeep[16 * v + 9], sc),
                            __fdiv_rn(hkeep[16 * v + 10], sc), __fdiv_rn(hkeep[16 * v + 11], sc)),
                  to_e4m3x4(__fdiv_rn(hkeep[16 * v + 12], sc), __fdiv_rn(hkeep[16 * v + 13], sc),
                            __fdiv_rn(hkeep[16 * v + 14], sc), __fdiv_rn(hkeep[16 * v + 15], sc)));
              c1[v] = make_uint4(
                  to_e4m3x4(__fdiv_rn(h1[16 * v + 0], sc), __fdiv_rn(h1[16 * v + 1], sc),
                            __fdiv_rn(h1[16 * v + 2], sc), __fdiv_rn(h1[16 * v + 3], sc)),
                  to_e4m3x4(__fdiv_rn(h1[16 * v + 4], sc), __fdiv_rn(h1[16 * v + 5], sc),
                            __fdiv_rn(h1[16 * v + 6], sc), __fdiv_rn(h1[16 * v + 7], sc)),
                  to_e4m3x4(__fdiv_rn(h1[16 * v + 8], sc), __fdiv_rn(h1[16 * v + 9], sc),
                            __fdiv_rn(h1[16 * v + 10], sc), __fdiv_rn(h1[16 * v + 11], sc)),
                  to_e4m3x4(__fdiv_rn(h1[16 * v + 12], sc), __fdiv_rn(h1[16 * v + 13], sc),
                            __fdiv_rn(h1[16 * v + 14], sc), __fdiv_rn(h1[16 * v + 15], sc)));
            }
            uint4* d0 = reinterpret_cast<uint4*>(qrow + 32 * half);
            uint4* d1 = reinterpret_cast<uint4*>(qrow + 64 + 32 * half);
            d0[0] = c0[0];
            d0[1] = c0[1];
            d1[0] = c1[0];
            d1[1] = c1[1];
            if (half == 0) qscales[static_cast<size_t>(grow) * (ldo / kQBlock) + n_blk] = sc;
          }
        } else if (valid) {
          __nv_bfloat16* yrow = out + static_cast<size_t>(grow) * ldo;
          {
            uint4* d0 = reinterpret_cast<uint4*>(yrow + nb_col * kF8BN + col0);
            uint4* d1 = reinterpret_cast<uint4*>(yrow + nb_col * kF8BN + col1);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              d0[v] = make_uint4(pack_bf16x2(acc0[8 * v], acc0[8 * v + 1]),
                                 pack_bf16x2(acc0[8 * v + 2], acc0[8 * v + 3]),
                                 pack_bf16x2(acc0[8 * v + 4], acc0[8 * v + 5]),
                                 pack_bf16x2(acc0[8 * v + 6], acc0[8 * v + 7]));
              d1[v] = make_uint4(pack_bf16x2(acc1[8 * v], acc1[8 * v + 1]),
                                 pack_bf16x2(acc1[8 * v + 2], acc1[8 * v + 3]),
                                 pack_bf16x2(acc1[8 * v + 4], acc1[8 * v + 5]),
                                 pack_bf16x2(acc1[8 * v + 6], acc1[8 * v + 7]));
            }
          }
        }
      }
      if (broken && EPI == EPI8_SWIGLU_Q) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace moe
