// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA)
// for the expert FFNs: per group g, D_g = A[rows of g] * B_g^T, both operands
// K-major. Epilogues: plain bf16 store, or SwiGLU over interleaved W1/W3 column
// pairs (h = silu(a) * b).
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer (one elected lane): A and B tiles into a
//               4-stage shared-memory ring (128B-swizzled, K block 64).
//   warp 1      MMA issuer (one elected lane): tcgen05.mma M=128, N=BN, K=16
//               into one of two TMEM accumulators (2 x BN fp32 columns).
//   warps 2-5   epilogue: tcgen05.ld of the finished accumulator (one TMEM
//               lane = one output row per thread), convert, store to global;
//               runs while the MMA warp fills the other accumulator.
// Tiles are (group, m-block of 128 rows, n-block of BN columns); within a
// group the m-blocks of one n-block are consecutive so the CTAs running at
// the same time share the weight tile through L2. The tile list is rebuilt
// on the device from group_offsets: no host round trip for the group sizes.
#pragma once
#include "dispatch.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kBM = 128;        // rows per tile (UMMA M)
constexpr int kBK = 64;         // bf16 K elements per stage = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kUmmaK = 16;      // K of one tcgen05.mma kind::f16
constexpr int kGemmThreads = 192;
constexpr int kMaxGroups = 1024;

enum { EPI_STORE = 0, EPI_SWIGLU = 1, EPI_SCATTER = 2 };

// EPI_SCATTER (the down-projection of the fused-scatter mode): output row r
// of a group goes to row slot[r] of the output, a (token, slot) row of a
// [T*K, d] buffer, multiplied by scale[slot[r]] (the token's gate for that
// expert) in fp32 before its bf16 rounding. Rows whose slot lies outside
// [0, n_slots) are not stored.
struct ScatterOut {
  const int32_t* slot;
  const float* scale;
  int n_slots;
  // Fused combine (cnt != nullptr): cnt [T, n_fb] counts, per token and
  // 128-feature block, the slot rows stored so far (zeroed before the
  // launch). The store that completes a block's top_k rows adds them in slot
  // order to residual and shared (either may be null) in fp32, rounds once
  // and writes the token's output row: the combine's arithmetic, in the
  // down-projection's epilogue.
  int32_t* cnt;
  const __nv_bfloat16* shared;
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int top_k;
  int n_fb;
};

// out[t, c .. c+8) of one token whose top_k slot rows are all stored: the
// combine's order (residual, shared, then the slots), one bf16 rounding. The
// slot rows come from other SMs: read through L2 (ld.global.cg).
__device__ __forceinline__ void combine_slots_8(const ScatterOut& sc, const __nv_bfloat16* y,
                                                int ldo, int t, int c) {
  const size_t orow = static_cast<size_t>(t) * ldo + c;
  uint4 yv[kMaxTopK];
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k)
    if (k < sc.top_k)
      yv[k] = __ldcg(reinterpret_cast<const uint4*>(
          y + (static_cast<size_t>(t) * sc.top_k + k) * ldo + c));
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = 0.0f;
  if (sc.residual) add_bf16x8(a, __ldcg(reinterpret_cast<const uint4*>(sc.residual + orow)));
  if (sc.shared) add_bf16x8(a, __ldcg(reinterpret_cast<const uint4*>(sc.shared + orow)));
#pragma unroll
  for (int k = 0; k < kMaxTopK; ++k)
    if (k < sc.top_k) add_bf16x8(a, yv[k]);
  *reinterpret_cast<uint4*>(sc.out + orow) =
      make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                 pack_bf16x2(a[6], a[7]));
}

// Fused combine after one thread stored the features [c0, c0 + 8 * nvec) of
// slot row drow (-1: nothing stored), counter block fb. Called by every lane
// of the warp. The store is made visible device-wide before the count, and
// the completing thread reads the other rows only after its count.
__device__ __forceinline__ void scatter_combine_thread(const ScatterOut& sc,
                                                       const __nv_bfloat16* y, int ldo,
                                                       int drow, int c0, int nvec, int fb) {
  __threadfence();
  bool last = false;
  if (drow >= 0) {
    const int t = drow / sc.top_k;
    last = atomicAdd(sc.cnt + static_cast<size_t>(t) * sc.n_fb + fb, 1) == sc.top_k - 1;
  }
  if (!last) return;
  __threadfence();
  const int t = drow / sc.top_k;
#pragma unroll 1
  for (int v = 0; v < nvec; ++v) combine_slots_8(sc, y, ldo, t, c0 + 8 * v);
}

template <int BN>
struct GemmCfg {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;   // double-buffered accumulator
  static constexpr int kBarBytes = 256;
  static size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kStages) * kStageBytes + kBarBytes +
           3 * static_cast<size_t>(G + 1) * sizeof(int);
  }
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// tile index -> (group, m block, n block); m blocks fastest inside a group.
// Group g covers rows [s_off[g], s_end[g]).
__device__ __forceinline__ void decode_tile(int t, const int* s_tstart, const int* s_off,
                                            const int* s_end, int G, int& g, int& m_blk,
                                            int& n_blk) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int local = t - s_tstart[g];
  const int mt = (s_end[g] - s_off[g] + kBM - 1) / kBM;
  n_blk = local / mt;
  m_blk = local - n_blk * mt;
}

// Group table of a grouped GEMM, built by one warp from the caller's device
// array offsets[0..G]. The offsets are not trusted: each is clamped into
// [0, rows] and raised to the running maximum of the ones before it, so the
// groups [s_off[g], s_end[g]) are disjoint, in order and inside the rows of
// the operands whatever the array holds (a valid array passes unchanged).
// With s_tstart, also the first tile of every group (tile_rows-row blocks
// times tiles_per_mblk column blocks) and the total in s_tstart[G].
__device__ __forceinline__ void build_group_table(const int32_t* __restrict__ offsets, int G,
                                                  int rows, int tile_rows, int tiles_per_mblk,
                                                  int* s_off, int* s_end, int* s_tstart,
                                                  int lane) {
  int run = 0;                                   // running maximum of the clamped offsets
  for (int base = 0; base <= G; base += 32) {
    const int j = base + lane;
    int v = 0;
    if (j <= G) v = min(max(__ldg(offsets + j), 0), rows);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v = max(v, n);
    }
    v = max(v, run);
    if (j <= G) s_off[j] = v;
    run = __shfl_sync(0xffffffffu, v, 31);
  }
  __syncwarp();
  int carry = 0;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    int nt = 0;
    if (g < G) {
      const int o0 = s_off[g], o1 = s_off[g + 1];
      s_end[g] = o1;
      nt = (o1 - o0 + tile_rows - 1) / tile_rows * tiles_per_mblk;
    }
    if (s_tstart) {
      int v = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (g < G) s_tstart[g] = carry + v - nt;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  if (lane == 0) {
    s_end[G] = s_off[G];
    if (s_tstart) s_tstart[G] = carry;
  }
  __syncwarp();
}

__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + __expf(-a)); }

template <int BN, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const int32_t* __restrict__ offsets, int G, int K, int n_per_group,
                         int rows, __nv_bfloat16* __restrict__ out, int ldo,
                         __nv_bfloat16* __restrict__ ac, unsigned int* status,
                         ScatterOut sc) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * C::kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_tstart = s_off + (G + 1);
  int* s_end = s_tstart + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks_n = n_per_group / BN;
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
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  } else if (warp == 1) {
    // Group table: row offsets and the first tile of every group (warp scan).
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
    uint32_t issued = 0, issued_par = 0;   // per stage: ever filled / parity of last fill
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      int g, m_blk, n_blk;
      decode_tile(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int a_row = s_off[g] + m_blk * kBM;
      const int b_row = g * n_per_group + n_blk * BN;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
        tma_load_2d(sA + stage * C::kABytes, &tmA, &full[stage], kb * kBK, a_row);
        tma_load_2d(sB + stage * C::kBBytes, &tmB, &full[stage], kb * kBK, b_row);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Never leave with a TMA write into shared memory still in flight.
    for (int s = 0; s < kStages; ++s)
      if (issued & (1u << s))
        mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int local = 0;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++local) {
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
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * C::kBBytes));
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k) {
          // advance 16 bf16 = 32 bytes along K inside the swizzle row
          umma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
        }
        umma_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) umma_commit(&tfull[acc]);
    }
    // Every issued MMA has finished before TMEM is released.
    umma_commit(mma_done);
    mbar_wait(mma_done, 0, status, kStatusTimeoutMma);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;               // TMEM lanes this warp may read
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++local) {
      int g, m_blk, n_blk;
      decode_tile(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_par, status, kStatusTimeoutEpilogue)) break;
      tc_fence_after();
      const int grow = s_off[g] + m_blk * kBM + row_in_tile;
      const int row_end = min(s_end[g], rows);
      const bool valid = grow < row_end;
      const uint32_t taddr = tmem_base + acc * BN + lane_addr;
      if constexpr (EPI == EPI_SWIGLU) {
        // W1/W3 rows interleaved in 16-row chunks: accumulator columns
        // [32q, 32q+16) = x.W1 and [32q+16, 32q+32) = x.W3 of h columns
        // n_blk*128 + 16q + [0, 16)
        static_assert(BN == 256, "SwiGLU epilogue: 256 accumulator columns -> 128 h columns");
        __nv_bfloat16* dst_row = out + static_cast<size_t>(grow) * ldo + n_blk * 128;
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
          uint32_t x0[32], x1[32];
          tmem_ld_32cols(taddr + c, x0);
          tmem_ld_32cols(taddr + c + 32, x1);
          tmem_ld_wait();
          if (valid && ac != nullptr) {
            // training: keep the 64 pre-activations [rows, 2 * ldo], packed W13 order
            uint32_t raw[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              raw[i] = pack_bf16x2(__uint_as_float(x0[2 * i]), __uint_as_float(x0[2 * i + 1]));
              raw[16 + i] =
                  pack_bf16x2(__uint_as_float(x1[2 * i]), __uint_as_float(x1[2 * i + 1]));
            }
            uint4* dst = reinterpret_cast<uint4*>(ac + static_cast<size_t>(grow) * (2 * ldo) +
                                                  n_blk * BN + c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_uint4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
          }
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              pk[i] = pack_bf16x2(
                  silu_f32(__uint_as_float(x0[2 * i])) * __uint_as_float(x0[16 + 2 * i]),
                  silu_f32(__uint_as_float(x0[2 * i + 1])) * __uint_as_float(x0[17 + 2 * i]));
              pk[8 + i] = pack_bf16x2(
                  silu_f32(__uint_as_float(x1[2 * i])) * __uint_as_float(x1[16 + 2 * i]),
                  silu_f32(__uint_as_float(x1[2 * i + 1])) * __uint_as_float(x1[17 + 2 * i]));
            }
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c / 2);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        int drow = grow;
        bool store = valid;
        float scale = 1.0f;
        if constexpr (EPI == EPI_SCATTER) {
          drow = valid ? __ldg(sc.slot + grow) : -1;
          store = valid && drow >= 0 && drow < sc.n_slots;
          scale = store ? __ldg(sc.scale + drow) : 0.0f;
        }
        __nv_bfloat16* dst_row = out + static_cast<size_t>(store ? drow : 0) * ldo + n_blk * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32cols(taddr + c, r);
          tmem_ld_wait();
          if (store) {
            uint32_t pk[16];
            if constexpr (EPI == EPI_SCATTER) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(scale * __uint_as_float(r[2 * i]),
                                    scale * __uint_as_float(r[2 * i + 1]));
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            }
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if constexpr (EPI == EPI_SCATTER) {
          // this thread stored the 256 features of one slot row: counter
          // block 2 * n_blk of its token stands for both 128-feature halves
          if (sc.cnt != nullptr)
            scatter_combine_thread(sc, out, ldo, store ? drow : -1, n_blk * BN, BN / 8,
                                   2 * n_blk);
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
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace moe
