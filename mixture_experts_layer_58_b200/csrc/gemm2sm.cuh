// Grouped bf16 GEMM on CTA pairs: tcgen05.mma.cta_group::2 with the weights as
// the MMA's M side (256 weight rows) and a group's token rows as its N side.
//
// The 1-CTA kernel (gemm.cuh) moves 48 KB from L2 into one SM per 128 x 256 x 64
// step, and the L2->SM crossbar, not the tensor cores, sets its speed. Here two
// CTAs of a cluster share one M = 256 MMA: CTA r (r = 0 leader, 1 peer) loads
// weight rows [128r, 128r+128) of the tile's 256 and half of its token rows
// into its own shared memory, the leader issues the MMA, and the hardware reads
// both halves from both CTAs. Each SM so loads 32 KB per 64 of K for the flops
// of a 128 x 256 x 64 step (a third less crossbar traffic). A ring stage holds
// two such K atoms (64 KB per CTA, 3 stages): one barrier round trip between
// the producer and the MMA thread per 128 of K, which measured far cheaper
// than one per 64 (the MMA thread waits, fences and commits per stage).
//
// Why weights as M: a group's rows come in tiles of 256, and its last tile
// holds 1..256 of them. With tokens as N that tile's MMA is N = its row count
// rounded up to 32, and a narrow MMA costs less tensor time than a full one
// (measured: about 107 clocks at N = 128 against 171 at N = 256 per K = 16
// step and SM), so a ragged tail no longer costs a full 256-row tile.
//
// TMEM: each CTA receives its 128 weight rows (lanes) x N token columns of the
// accumulator, double-buffered (2 x 256 columns). The epilogue transposes
// through shared memory: 32 token columns at a time, each warp's 32 lanes are
// written into a [32 tokens][features] bf16 tile, then the group of 4
// epilogue warps (one per TMEM lane quarter) that owns the chunk stores whole
// token rows with 16-byte vectors. With W1/W3 interleaved in
// 16-row chunks, lanes l and l+16 of a warp hold the gate and up products of
// the same h column, paired with one shuffle.
//
// Synchronisation (all waits bounded; no TMA multicast):
//   full[s]   leader only. Expects 64 KB per phase: the leader's arrive.expect_tx
//             plus both CTAs' TMA loads, which complete on the leader's barrier.
//   empty[s]  both CTAs; the leader's MMA commit arrives on its own and on the
//             peer's (mapa address) when the stage has been read.
//   tfull[a]  both CTAs; committed like empty at the end of a tile.
//   tempty[a] leader only; lane 0 of each epilogue warp of both CTAs arrives
//             once it has drained its TMEM columns (release.cluster).
// Tiles are (group, 256-token block, 256-weight-row block); token columns past
// the group's end are computed on whatever rows the loads fetched and never
// stored.
#pragma once
#include "gemm.cuh"

namespace moe {

// A ring stage holds kAtoms2 K-atoms of 64 (one 128-byte swizzle row each):
// the MMA thread issues 4 * kAtoms2 MMAs per full-barrier wait and per
// commit, so the barrier round trip, not the MMA, is paid once per 128 of K.
constexpr int kAtoms2 = 2;
constexpr int kStages2 = 3;
constexpr int kBM2 = 256;        // rows per CTA-pair tile (128 per CTA)
// Epilogue warps per CTA, in groups of 4 (one warp per TMEM lane quarter);
// group e drains the 32-column chunks e, e + groups, ... of each tile through
// its own double-buffered transpose tile.
constexpr int kPairEpiWarps = 4;
constexpr int kPairEpiGroups = kPairEpiWarps / 4;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;

struct Gemm2smCfg {
  static constexpr int kAtomBytes = 128 * kBK * 2;   // 128 rows x one 64-wide K atom
  static constexpr int kABytes = kAtoms2 * kAtomBytes;   // token rows (up to 128, this CTA's half)
  static constexpr int kBBytes = kAtoms2 * kAtomBytes;   // this CTA's 128 weight rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kXBytes = kPairEpiGroups * 2 * 32 * 128 * 2;   // per group, double-buffered
  static constexpr int kBarBytes = 256;
  static size_t smem_bytes(int G) {
    return 1024 + static_cast<size_t>(kStages2) * kStageBytes + kXBytes + kBarBytes +
           3 * static_cast<size_t>(G + 1) * sizeof(int);
  }
};

// Token columns of a pair tile whose first row leaves `rows_left` (> 0) rows
// in its group: at most 256, rounded up to a multiple of 32 (the MMA's N; each
// CTA supplies half).
__device__ __forceinline__ int pair_tile_cols(int rows_left) {
  const int n = rows_left < kBM2 ? rows_left : kBM2;
  return (n + 31) & ~31;
}

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

// Dynamic tile order. The leader's producer takes the next tile index from a
// global counter (zeroed before the launch) and publishes it, through a ring
// of kTileQ slots, to the other roles that walk the same tiles: the peer's
// producer, the leader's MMA thread and the epilogue warps of each CTA.
// Tiles cost different amounts (a group's last tile is a narrower MMA), so a
// fixed round-robin split would leave some pairs idle while others still work
// through full tiles; taking tiles in index order also keeps the pairs that
// share a weight tile close together in time, while it is still in L2.
constexpr int kTileQ = 4;
constexpr int kTileQConsumers = 2 + 2 * kPairEpiWarps;

__device__ __forceinline__ void st_shared_cluster_s32(uint32_t addr, int v) {
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Leader producer: wait until slot i % kTileQ is free, then publish t in both CTAs.
__device__ __forceinline__ bool tile_q_push(int i, int t, int* tq, uint64_t* tq_full,
                                            uint64_t* tq_empty, unsigned int* status) {
  const int j = i & (kTileQ - 1);
  if (!mbar_wait_cluster(&tq_empty[j], ((i / kTileQ) & 1) ^ 1u, status, kStatusTimeoutProducer))
    return false;
  tq[j] = t;
  st_shared_cluster_s32(mapa_shared(smem_u32(&tq[j]), 1), t);
  mbar_arrive(&tq_full[j]);
  mbar_arrive_cluster(mapa_shared(smem_u32(&tq_full[j]), 1));
  return true;
}

// Any other role (one thread): the i-th published tile index of this CTA's ring.
__device__ __forceinline__ bool tile_q_pop(int i, const int* tq, uint64_t* tq_full,
                                           uint64_t* tq_empty, int& t, unsigned int* status,
                                           unsigned int code) {
  const int j = i & (kTileQ - 1);
  if (!mbar_wait_cluster(&tq_full[j], (i / kTileQ) & 1, status, code)) return false;
  t = *reinterpret_cast<const volatile int*>(&tq[j]);
  mbar_arrive_cluster(mapa_shared(smem_u32(&tq_empty[j]), 0));
  return true;
}

// A group of 4 epilogue warps meets between writing and reading a transpose
// buffer: lane 0 of each arrives once its warp's writes are done (the
// mbarrier's release/acquire orders them), and every lane waits, bounded.
__device__ __forceinline__ bool xfer_sync(uint64_t* bar, uint32_t parity, int lane,
                                          unsigned int* status) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  return mbar_wait(bar, parity, status, kStatusTimeoutEpilogue);
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
grouped_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmA32,
                              const __grid_constant__ CUtensorMap tmB,
                              const int32_t* __restrict__ offsets, int G, int K, int n_per_group,
                              int rows, __nv_bfloat16* __restrict__ out, int ldo,
                              __nv_bfloat16* __restrict__ ac,
                              const int32_t* __restrict__ src_rows, int* tile_counter,
                              unsigned int* status, ScatterOut sc) {
  constexpr int BN = 256;
  using C = Gemm2smCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages2 * C::kABytes;
  __nv_bfloat16* sX = reinterpret_cast<__nv_bfloat16*>(sB + kStages2 * C::kBBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sX) + C::kXBytes);
  uint64_t* empty = full + kStages2;
  uint64_t* tfull = empty + kStages2;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* xready = mma_done + 1;   // [2 per group]: the group's 4 warps filled its sX half i
  uint64_t* tq_full = xready + 2 * kPairEpiGroups;   // [kTileQ]
  uint64_t* tq_empty = tq_full + kTileQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_empty + kTileQ);
  int* tq = reinterpret_cast<int*>(tmem_slot + 1);   // [kTileQ] tile indices
  int* s_off = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + C::kBarBytes);
  int* s_tstart = s_off + (G + 1);
  int* s_end = s_tstart + (G + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int n_blocks_n = n_per_group / BN;
  const int num_kb = K / (kBK * kAtoms2);   // ring stages per tile

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages2; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&tfull[a], 1);
        mbar_init(&tempty[a], 2 * kPairEpiWarps);
      }
      mbar_init(mma_done, 1);
      for (int j = 0; j < 2 * kPairEpiGroups; ++j) mbar_init(&xready[j], 4);
      for (int j = 0; j < kTileQ; ++j) {
        mbar_init(&tq_full[j], 1);
        mbar_init(&tq_empty[j], kTileQConsumers);
      }
      fence_mbar_init();
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmA32);
      tma_prefetch_desc(&tmB);
    }
    __syncwarp();
    tmem_alloc_2sm(tmem_slot, 512);
    tmem_relinquish_2sm();
  } else if (warp == 1) {
    build_group_table(offsets, G, rows, kBM2, n_blocks_n, s_off, s_end, s_tstart, lane);
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
    int t_next = 0;
    if (rank == 0 && lane == 0) t_next = atomicAdd(tile_counter, 1);
    for (int i = 0; ok; ++i) {
      int t = total_tiles;
      if (lane == 0) {
        if (rank == 0) {
          t = min(t_next, total_tiles);
          ok = tile_q_push(i, t, tq, tq_full, tq_empty, status);
          if (ok && t < total_tiles) t_next = atomicAdd(tile_counter, 1);
        } else {
          ok = tile_q_pop(i, tq, tq_full, tq_empty, t, status, kStatusTimeoutProducer);
        }
      }
      if constexpr (GATHER) {
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        t = __shfl_sync(0xffffffffu, t, 0);
      }
      if (!ok || t >= total_tiles) break;
      int g, m_blk, n_blk;
      decode_tile_pair(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int row0 = s_off[g] + m_blk * kBM2;
      const int ncols = pair_tile_cols(s_end[g] - row0);
      const int a_row = row0 + static_cast<int>(rank) * (ncols >> 1);
      const int b_row = g * n_per_group + n_blk * BN + static_cast<int>(rank) * 128;
      // bytes landing on the leader's barrier per stage, from both CTAs: the
      // weight half-tiles, and the token rows (a full tile or the gather form:
      // 128 rows in one box or 32 gathers; a ragged tail tile: its ncols/2
      // rows rounded up to boxes of 32, not a full 128-row box per K step)
      const int nbox = GATHER ? 4 : ((ncols >> 1) + 31) >> 5;
      const uint32_t stage_tx =
          2u * kAtoms2 * static_cast<uint32_t>(C::kAtomBytes + nbox * 32 * 128);
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
        if (rank == 0 && lane == 0) mbar_arrive_expect_tx(&full[stage], stage_tx);
        const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
#pragma unroll
        for (int at = 0; at < kAtoms2; ++at) {
          const int x = (kb * kAtoms2 + at) * kBK;
          uint8_t* a_dst = sA + stage * C::kABytes + at * C::kAtomBytes;
          if constexpr (GATHER) {
            tma_gather4_pair(a_dst + lane * 4 * 128, &tmA, bar, x, src[0], src[1], src[2],
                             src[3]);
          } else if (nbox == 4) {
            tma_load_2d_pair(a_dst, &tmA, bar, x, a_row);
          } else {
            // a ragged tail tile: only the token rows it uses, in boxes of 32
            for (int j = 0; j < nbox; ++j)
              tma_load_2d_pair(a_dst + j * (32 * 128), &tmA32, bar, x, a_row + 32 * j);
          }
          if (lane == 0)
            tma_load_2d_pair(sB + stage * C::kBBytes + at * C::kAtomBytes, &tmB, bar, x, b_row);
        }
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
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int local = 0; ok; ++local) {
      int t;
      if (!tile_q_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutMma) ||
          t >= total_tiles)
        break;
      int g, m_blk, n_blk;
      decode_tile_pair(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int ncols = pair_tile_cols(s_end[g] - (s_off[g] + m_blk * kBM2));
      const uint32_t idesc = idesc_bf16_f32(kBM2, ncols);
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
        // MMA A operand = the weight rows (sB), B operand = the token rows (sA)
#pragma unroll
        for (int at = 0; at < kAtoms2; ++at) {
          const uint64_t wdesc =
              sw128_kmajor_desc(smem_u32(sB + stage * C::kBBytes + at * C::kAtomBytes));
          const uint64_t xdesc =
              sw128_kmajor_desc(smem_u32(sA + stage * C::kABytes + at * C::kAtomBytes));
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            umma_bf16_pair(d_tmem, wdesc + 2u * k, xdesc + 2u * k, idesc, (kb | at | k) != 0);
        }
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
    const int eg = (warp - 2) >> 2;                 // epilogue group
    const int et = ((warp - 2) & 3) * 32 + lane;    // 0..127 across the group's 4 warps
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint64_t* gready = xready + 2 * eg;
    __nv_bfloat16* gX = sX + eg * (2 * 32 * 128);
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int chunk = 0;   // running count of this group's 32-column chunks: selects its sX half
    for (int local = 0;; ++local) {
      int t = total_tiles;
      bool got = true;
      if (lane == 0)
        got = tile_q_pop(local, tq, tq_full, tq_empty, t, status, kStatusTimeoutEpilogue);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!got || t >= total_tiles) break;
      int g, m_blk, n_blk;
      decode_tile_pair(t, s_tstart, s_off, s_end, G, g, m_blk, n_blk);
      const int row0 = s_off[g] + m_blk * kBM2;
      const int ncols = pair_tile_cols(s_end[g] - row0);
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_par, status, kStatusTimeoutEpilogue)) break;
      tc_fence_after();
      const int row_end = min(s_end[g], rows);
      const uint32_t taddr = tmem_base + acc * BN + lane_addr;
      bool ok = true;
#pragma unroll 1
      for (int j0 = 32 * eg; j0 < ncols; j0 += 32 * kPairEpiGroups, ++chunk) {
        ok = false;
        uint32_t v[32];
        tmem_ld_32cols(taddr + j0, v);
        tmem_ld_wait();
        __nv_bfloat16* X = gX + (chunk & 1) * (32 * 128);
        if constexpr (EPI == EPI_SWIGLU) {
          // lane l < 16: gate product of h column (l & 15) of this warp's 16;
          // lane l + 16: its up product. Lanes < 16 finish tokens 0..15 of the
          // chunk, lanes >= 16 tokens 16..31. X = [32 tokens][64 h columns].
          if (ac != nullptr) {
            // training: keep the pre-activations, [rows, 2 * ldo] in the
            // packed W13 column order (this lane's weight row = its column)
            __nv_bfloat16* acol =
                ac + n_blk * BN + static_cast<int>(rank) * 128 + quarter * 32 + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int grow = row0 + j0 + i;
              if (grow < row_end)
                acol[static_cast<size_t>(grow) * (2 * ldo)] =
                    __float2bfloat16_rn(__uint_as_float(v[i]));
            }
          }
          const bool lo = lane < 16;
          const int hc = quarter * 16 + (lane & 15);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t own = lo ? v[i] : v[i + 16];
            const uint32_t send = lo ? v[i + 16] : v[i];
            const uint32_t other = __shfl_xor_sync(0xffffffffu, send, 16);
            const float a = __uint_as_float(lo ? own : other);
            const float b = __uint_as_float(lo ? other : own);
            X[(i + (lo ? 0 : 16)) * 64 + hc] = __float2bfloat16_rn(silu_f32(a) * b);
          }
          if (!xfer_sync(&gready[chunk & 1], (chunk >> 1) & 1, lane, status)) break;
          __nv_bfloat16* dst0 = out + n_blk * 128 + static_cast<int>(rank) * 64;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int idx = et + 128 * k;
            const int r = idx >> 3, seg = idx & 7;
            const int grow = row0 + j0 + r;
            if (grow < row_end)
              *reinterpret_cast<uint4*>(dst0 + static_cast<size_t>(grow) * ldo + seg * 8) =
                  *reinterpret_cast<const uint4*>(X + r * 64 + seg * 8);
          }
        } else {
          // X = [32 tokens][128 output features of this CTA]
          if constexpr (EPI == EPI_SCATTER) {
            // lane i holds the gate of the chunk's token i (0 past the group)
            const int gr = row0 + j0 + lane;
            const int sl = gr < row_end ? __ldg(sc.slot + gr) : -1;
            const float gl = (sl >= 0 && sl < sc.n_slots) ? __ldg(sc.scale + sl) : 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              X[i * 128 + quarter * 32 + lane] =
                  __float2bfloat16_rn(__shfl_sync(0xffffffffu, gl, i) * __uint_as_float(v[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              X[i * 128 + quarter * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
          }
          if (!xfer_sync(&gready[chunk & 1], (chunk >> 1) & 1, lane, status)) break;
          const int fcol = n_blk * BN + static_cast<int>(rank) * 128;
          __nv_bfloat16* dst0 = out + fcol;
          int dr[4];   // slot row this lane stored in step k (-1: none)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int idx = et + 128 * k;
            const int r = idx >> 4, seg = idx & 15;
            const int grow = row0 + j0 + r;
            dr[k] = -1;
            if (grow < row_end) {
              int drow = grow;
              if constexpr (EPI == EPI_SCATTER) {
                drow = __ldg(sc.slot + grow);
                if (drow < 0 || drow >= sc.n_slots) continue;
              }
              *reinterpret_cast<uint4*>(dst0 + static_cast<size_t>(drow) * ldo + seg * 8) =
                  *reinterpret_cast<const uint4*>(X + r * 128 + seg * 8);
              dr[k] = drow;
            }
          }
          if constexpr (EPI == EPI_SCATTER) {
            // Fused combine: the 16 lanes of a half-warp stored one row's 128
            // features (this CTA's block 2 * n_blk + rank) in each step k;
            // lane 16h + k counts that row, and the half-warp that completes
            // a token's block writes its output features.
            if (sc.cnt != nullptr) {
              __threadfence();
              __syncwarp();
              const int kk = lane & 15;
              int mine = -1;
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (kk == k) mine = dr[k];
              bool last = false;
              if (mine >= 0)
                last = atomicAdd(sc.cnt + static_cast<size_t>(mine / sc.top_k) * sc.n_fb +
                                     fcol / 128,
                                 1) == sc.top_k - 1;
              const unsigned lm = __ballot_sync(0xffffffffu, last);
              if (lm != 0) {
                __threadfence();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  if ((lm >> ((lane & 16) + k)) & 1u)
                    combine_slots_8(sc, out, ldo, dr[k] / sc.top_k, fcol + (lane & 15) * 8);
              }
            }
          }
        }
        ok = true;
      }
      if (!ok) break;
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
