// Grouped bf16 GEMM on CTA pairs: tcgen05.mma.cta_group::2, 256 x 256 tiles.
//
// The 1-CTA kernel (gemm.cuh) moves 48 KB from L2 into one SM per 128 x 256 x 64
// step, and the L2->SM crossbar, not the tensor cores, sets its speed. Here two
// CTAs of a cluster share one M = 256, N = 256 MMA: CTA r (r = 0 leader, 1 peer)
// loads rows [128r, 128r+128) of the A tile and rows [128r, 128r+128) of the
// B (weight) tile into its own shared memory, the leader issues the MMA, and
// the hardware reads A and B halves from both CTAs. Each SM so loads 32 KB per
// step for the same flops (a third less crossbar traffic) and the ring holds
// 6 stages. Each CTA's TMEM receives its own 128 rows x 256 columns of the
// accumulator (double-buffered: 2 x 256 columns).
//
// Synchronisation (all waits bounded; no TMA multicast):
//   full[s]   leader only. Expects 64 KB per phase: the leader's arrive.expect_tx
//             plus both CTAs' TMA loads, which complete on the leader's barrier.
//   empty[s]  both CTAs; the leader's MMA commit arrives on its own and on the
//             peer's (mapa address) when the stage has been read.
//   tfull[a]  both CTAs; committed like empty at the end of a tile.
//   tempty[a] leader only; lane 0 of each of the 8 epilogue warps (both CTAs)
//             arrives once it has drained its TMEM rows (release.cluster).
// Tiles are (group, 256-row block, 256-column block); a group's last block
// may hold fewer than 256 valid rows (stores are masked).
#pragma once
#include "gemm.cuh"

namespace moe {

constexpr int kStages2 = 6;
constexpr int kBM2 = 256;        // rows per CTA-pair tile (128 per CTA)

struct Gemm2smCfg {
  static constexpr int kABytes = 128 * kBK * 2;   // this CTA's 128 rows of A
  static constexpr int kBBytes = 128 * kBK * 2;   // this CTA's 128 rows of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarBytes = 256;
  static size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kStages2) * kStageBytes + kBarBytes +
           3 * static_cast<size_t>(G + 1) * sizeof(int);
  }
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void tmem_alloc_2sm(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_2sm() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// the leader CTA's barrier (`bar_cluster` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

// Four rows (r0..r3) of a tensor map whose box is one row high, 64 bf16 wide,
// into four consecutive 128-byte rows of this CTA's shared memory; completion
// counted on the leader's barrier.
__device__ __forceinline__ void tma_gather4_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int x, int r0, int r1,
                                                 int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4"
      ".mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3)
      : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at shared::cluster address `bar_cluster` (this
// CTA's or the peer's) when the pair MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar_cluster)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  unsigned int* status, unsigned int code) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, code);
      return false;
    }
  }
}

// tile index -> (group, 256-row block, n block); row blocks fastest in a group.
__device__ __forceinline__ void decode_tile_pair(int t, const int* s_tstart, const int* s_off,
                                                 const int* s_end, int G, int& g, int& m_blk,
                                                 int& n_blk) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int local = t - s_tstart[g];
  const int mt = (s_end[g] - s_off[g] + kBM2 - 1) / kBM2;
  n_blk = local / mt;
  m_blk = local - n_blk * mt;
}

// GATHER: the A rows of a tile are not contiguous; logical row r of A is row
// src_rows[r] of the tensor behind tmA (the token rows of u, read in place
// of an expert-contiguous copy), fetched four at a time with tile::gather4.
template <int EPI, bool GATHER>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
grouped_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB,
                              const int32_t* __restrict__ offsets, int G, int K, int n_per_group,
                              int rows, __nv_bfloat16* __restrict__ out, int ldo,
                              const int32_t* __restrict__ src_rows, unsigned int* status) {
  constexpr int BN = 256;
  using C = Gemm2smCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages2 * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages2 * C::kBBytes);
  uint64_t* empty = full + kStages2;
  uint64_t* tfull = empty + kStages2;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_tstart = s_off + (G + 1);
  int* s_end = s_tstart + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int n_blocks_n = n_per_group / BN;
  const int num_kb = K / kBK;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages2; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], 8);
      }
      mbar_init(mma_done, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    __syncwarp();
    tmem_alloc_2sm(tmem_slot, 512);
    tmem_relinquish_2sm();
  } else if (warp == 1) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int nt = 0;
      if (g < G) {
        const int o0 = offsets[g];
        const int o1 = offsets[g + 1];
        s_off[g] = o0;
        s_end[g] = o1 > o0 ? o1 : o0;
        nt = (o1 > o0 ? (o1 - o0 + kBM2 - 1) / kBM2 : 0) * n_blocks_n;
      }
      int v = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (g < G) s_tstart[g] = carry + v - nt;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) {
      s_tstart[G] = carry;
      s_off[G] = offsets[G];
      s_end[G] = offsets[G];
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_tstart[G];

  if (warp == 0 && (GATHER || lane == 0)) {
    // ------------------------------------------------------------ producer (both CTAs)
    // Gather form: the whole warp issues loads, lane i the four A rows
    // 4i..4i+3 of this CTA's 128; lane 0 waits and signals.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    bool ok = true;
    for (int t = pair; t < total_tiles && ok; t += npairs) {
      int g, m_blk, n_blk;
      decode_tile_pair(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int a_row = s_off[g] + m_blk * kBM2 + static_cast<int>(rank) * 128;
      const int b_row = g * n_per_group + n_blk * BN + static_cast<int>(rank) * 128;
      int src[4] = {0, 0, 0, 0};
      if constexpr (GATHER) {
        // rows past the group's end load any row of the group (masked later)
        const int first = (s_off[g] >= 0 && s_off[g] < rows) ? s_off[g] : 0;
        const int end = min(s_end[g], rows);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = a_row + 4 * lane + j;
          src[j] = __ldg(src_rows + (r >= 0 && r < end ? r : first));
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        bool got = true;
        if (lane == 0) got = mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer);
        if constexpr (GATHER) got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
        if (!got) {
          ok = false;
          break;
        }
        if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
        if constexpr (GATHER) {
          tma_gather4_pair(sA + stage * C::kABytes + lane * 4 * 128, &tmA, bar, kb * kBK, src[0],
                           src[1], src[2], src[3]);
        } else {
          tma_load_2d_pair(sA + stage * C::kABytes, &tmA, bar, kb * kBK, a_row);
        }
        if (lane == 0) tma_load_2d_pair(sB + stage * C::kBBytes, &tmB, bar, kb * kBK, b_row);
        issued |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages2) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // The leader's full barriers count both CTAs' bytes: once they have all
    // completed no TMA write into either CTA's shared memory is in flight.
    if (rank == 0 && lane == 0)
      for (int s = 0; s < kStages2; ++s)
        if (issued & (1u << s))
          mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (leader)
    constexpr uint32_t idesc = idesc_bf16_f32(kBM2, BN);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int local = 0;
    for (int t = pair; t < total_tiles && ok; t += npairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait_cluster(&tempty[acc], acc_par ^ 1u, status, kStatusTimeoutMma)) break;
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
        for (int k = 0; k < kBK / kUmmaK; ++k)
          umma_bf16_pair(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
        const uint32_t e = smem_u32(&empty[stage]);
        umma_commit_pair(mapa_shared(e, 0));
        umma_commit_pair(mapa_shared(e, 1));
        if (++stage == kStages2) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        const uint32_t f = smem_u32(&tfull[acc]);
        umma_commit_pair(mapa_shared(f, 0));
        umma_commit_pair(mapa_shared(f, 1));
      }
    }
    umma_commit_pair(mapa_shared(smem_u32(mma_done), 0));
    mbar_wait(mma_done, 0, status, kStatusTimeoutMma);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int row_in_half = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int local = 0;
    for (int t = pair; t < total_tiles; t += npairs, ++local) {
      int g, m_blk, n_blk;
      decode_tile_pair(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_par, status, kStatusTimeoutEpilogue)) break;
      tc_fence_after();
      const int grow = s_off[g] + m_blk * kBM2 + static_cast<int>(rank) * 128 + row_in_half;
      const int row_end = min(s_end[g], rows);
      const bool valid = grow >= 0 && grow < row_end;
      const uint32_t taddr = tmem_base + acc * BN + lane_addr;
      if constexpr (EPI == EPI_SWIGLU) {
        __nv_bfloat16* dst_row = out + static_cast<size_t>(grow) * ldo + n_blk * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t ga[32], up[32];
          tmem_ld_32cols(taddr + c, ga);
          tmem_ld_32cols(taddr + 128 + c, up);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_f32(__uint_as_float(ga[2 * i])) * __uint_as_float(up[2 * i]);
              const float h1 =
                  silu_f32(__uint_as_float(ga[2 * i + 1])) * __uint_as_float(up[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      } else {
        __nv_bfloat16* dst_row = out + static_cast<size_t>(grow) * ldo + n_blk * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32cols(taddr + c, r);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // neither CTA leaves while the pair may still signal it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, 512);
  }
}

}  // namespace moe
