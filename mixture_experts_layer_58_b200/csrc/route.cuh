// Routing kernel: gate GEMM on tcgen05 + affinity + bias-adjusted top-K +
// gate normalisation + per-expert load histogram, fused in one launch.
//
// Each CTA owns 128 tokens. The logits z = u . e_i of all (<= 256) experts of
// those tokens accumulate in TMEM ([128 lanes] x [n_pad fp32 columns]), fed by
// a TMA ring exactly like the expert GEMM. The epilogue then gives every
// thread one token: TMEM lane = token row, so the whole top-K runs in that
// thread's registers as a sorted insertion over the experts in ascending
// index (strictly-greater insertion = lower index wins a tie), with no
// cross-thread merge. The histogram is a shared-memory count per expert,
// flushed with one global atomic per expert per CTA.
//
// Sources: DeepSeek-V3 technical report summary (xyznot.com), Method §2 —
// s_{i,t} = Sigmoid(u_t . e_i); g'_{i,t} = s_{i,t} if s_{i,t} + b_i is in the
// top K_r of the biased keys; g = g' normalised (times the routed scale).
// Softmax form: "DeepSeek model architecture explained" (deepseekmodel.com),
// DeepSeekMoE forward listing — top-k of the raw logits, softmax over them.
#pragma once
#include "gemm.cuh"
#include "gemm2sm.cuh"

namespace moe {

constexpr int kRouteMaxExperts = 256;

struct RouteSmem {
  static size_t bytes(int n_pad) {
    return 1024 + static_cast<size_t>(kStages) * (kBM * kBK * 2 + n_pad * kBK * 2) + 256 +
           2 * kRouteMaxExperts * sizeof(float);
  }
};

// One token's selection, shared by the fused kernel and the split-K form:
// fold logit z of expert j into the running top-K (keys in descending order;
// strictly-greater insertion over ascending j = the lower index wins a tie).
template <int TOPK, int KIND>
__device__ __forceinline__ void route_insert(float z, int j, float bias_j, float (&kv)[TOPK],
                                             float (&sv)[TOPK], int (&ki)[TOPK]) {
  float s, key;
  if constexpr (KIND == 0) {
    s = 1.0f / (1.0f + expf(-z));
    key = s + bias_j;
  } else {
    s = z;
    key = z;
  }
  if (key > kv[TOPK - 1]) {
#pragma unroll
    for (int p = TOPK - 1; p >= 0; --p) {
      const bool above_prev = (p > 0) && (key > kv[p > 0 ? p - 1 : 0]);
      if (key > kv[p]) {
        if (above_prev) {
          kv[p] = kv[p - 1];
          sv[p] = sv[p - 1];
          ki[p] = ki[p - 1];
        } else {
          kv[p] = key;
          sv[p] = s;
          ki[p] = j;
        }
      }
    }
  }
}

// Gates of one token's selection (sigmoid: S s_k / sum; softmax: S softmax
// of the selected logits), its row of topk_idx / topk_gate, and its loads
// added to the block's shared-memory histogram.
template <int TOPK, int KIND>
__device__ __forceinline__ void route_emit(const float (&sv)[TOPK], const int (&ki)[TOPK],
                                           float routed_scale, int t, int32_t* topk_idx,
                                           float* topk_gate, int* s_hist) {
  float g[TOPK];
  float sum = 0.0f;
  if constexpr (KIND == 0) {
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
      g[p] = sv[p];
      sum += sv[p];
    }
  } else {
    const float m = sv[0];
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
      g[p] = expf(sv[p] - m);
      sum += g[p];
    }
  }
#pragma unroll
  for (int p = 0; p < TOPK; ++p) {
    topk_idx[static_cast<size_t>(t) * TOPK + p] = ki[p];
    topk_gate[static_cast<size_t>(t) * TOPK + p] = (routed_scale * g[p]) / sum;
    if (ki[p] >= 0) atomicAdd(&s_hist[ki[p]], 1);   // -1 only for non-finite logits
  }
}

// PARTIAL (the split-K form for small batches): CTA (b, y) accumulates the
// logits of token block b over K blocks [y*kb_per_split, +kb_per_split) only
// and writes them, fp32, to partial[y][t][n_pad]; route_select_kernel adds
// the splits and selects.
template <int TOPK, int KIND, bool PARTIAL>
__global__ void __launch_bounds__(kGemmThreads, 1)
route_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
             const float* __restrict__ bias, int T, int d, int n_routed, int n_pad,
             uint32_t tmem_cols, float routed_scale, int32_t* __restrict__ topk_idx,
             float* __restrict__ topk_gate, int32_t* __restrict__ counts,
             float* __restrict__ partial, int kb_per_split, unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int a_bytes = kBM * kBK * 2;
  const int b_bytes = n_pad * kBK * 2;
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * a_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * b_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  float* s_bias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);
  int* s_hist = reinterpret_cast<int*>(s_bias + kRouteMaxExperts);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kb0 = PARTIAL ? static_cast<int>(blockIdx.y) * kb_per_split : 0;
  const int kb1 = PARTIAL ? min(kb0 + kb_per_split, d / kBK) : d / kBK;
  const int row0 = blockIdx.x * kBM;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      mbar_init(tfull, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmU);
      tma_prefetch_desc(&tmE);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  } else if (warp >= 2) {
    for (int e = threadIdx.x - 64; e < kRouteMaxExperts; e += 128) {
      s_bias[e] = (KIND == 0 && bias != nullptr && e < n_routed) ? bias[e] : 0.0f;
      s_hist[e] = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) break;
      mbar_arrive_expect_tx(&full[stage], a_bytes + b_bytes);
      tma_load_2d(sA + stage * a_bytes, &tmU, &full[stage], kb * kBK, row0);
      tma_load_2d(sB + stage * b_bytes, &tmE, &full[stage], kb * kBK, 0);
      issued |= 1u << stage;
      issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    for (int s = 0; s < kStages; ++s)
      if (issued & (1u << s))
        mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16_f32(kBM, n_pad);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&full[stage], phase, status, kStatusTimeoutMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * a_bytes));
      const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * b_bytes));
#pragma unroll
      for (int k = 0; k < kBK / kUmmaK; ++k)
        umma_bf16(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, ((kb - kb0) | k) != 0);
      umma_commit(&empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    (void)ok;
    // tfull fires when every MMA above has completed (also on the error path,
    // so TMEM is never released under a running MMA).
    umma_commit(tfull);
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int t = row0 + r;
    const bool have = mbar_wait(tfull, 0, status, kStatusTimeoutEpilogue);
    tc_fence_after();
    float kv[TOPK], sv[TOPK];
    int ki[TOPK];
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
      kv[p] = -INFINITY;
      sv[p] = 0.0f;
      ki[p] = -1;
    }
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    if constexpr (PARTIAL) {
      // this split's logits of the thread's token, fp32, to the workspace.
      // tcgen05.ld is a warp-wide instruction: every lane of the warp runs
      // it (under the warp-uniform `have`); only the stores check t < T.
      if (have) {
        float* prow = partial + (static_cast<size_t>(blockIdx.y) * T + t) * n_pad;
        for (int c = 0; c < n_pad; c += 32) {
          uint32_t zr[32];
          tmem_ld_32cols(taddr + c, zr);
          tmem_ld_wait();
          if (t < T) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              if (c + i < n_pad)
                *reinterpret_cast<float4*>(prow + c + i) =
                    make_float4(__uint_as_float(zr[i]), __uint_as_float(zr[i + 1]),
                                __uint_as_float(zr[i + 2]), __uint_as_float(zr[i + 3]));
          }
        }
      }
    } else if (have) {
      for (int c = 0; c < n_pad; c += 32) {
        uint32_t zr[32];
        tmem_ld_32cols(taddr + c, zr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = c + i;
          if (j < n_routed)
            route_insert<TOPK, KIND>(__uint_as_float(zr[i]), j, s_bias[j], kv, sv, ki);
        }
      }
    }
    tc_fence_before();
    if constexpr (!PARTIAL) {
      if (have && t < T)
        route_emit<TOPK, KIND>(sv, ki, routed_scale, t, topk_idx, topk_gate, s_hist);
      named_bar_sync(1, 128);
      for (int e = threadIdx.x - 64; e < n_routed; e += 128) {
        const int c = s_hist[e];
        if (c) atomicAdd(&counts[e], c);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// CTA-pair form for large batches: a cluster of 2 CTAs takes 256 tokens, CTA
// r its 128 token rows (the MMA's M side) and centroid rows [r*N_pad/2,
// +N_pad/2) (half of its N side); the leader issues tcgen05.mma.cta_group::2
// M = 256, N = N_pad over a 3-stage ring of two 64-wide K atoms per stage, and
// each CTA's TMEM receives its 128 tokens x all N_pad logits, so the epilogue
// is the one-CTA kernel's. Half the centroid bytes per SM and one barrier round
// trip per eight MMAs. Synchronisation as the pair GEMM (gemm2sm.cuh): full[s]
// on the leader counts both CTAs' TMA bytes, empty[s] and tfull in both CTAs
// are committed by the leader; all waits bounded; no TMA multicast.
constexpr int kRouteAtoms = 2;
constexpr int kRouteStages2 = 3;

struct RoutePairSmem {
  static size_t bytes(int n_pad) {
    return 1024 + static_cast<size_t>(kRouteStages2) * kRouteAtoms *
                      (128 * kBK * 2 + (n_pad / 2) * kBK * 2) +
           256 + 2 * kRouteMaxExperts * sizeof(float);
  }
};

template <int TOPK, int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
route_pair_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
                  const float* __restrict__ bias, int T, int d, int n_routed, int n_pad,
                  uint32_t tmem_cols, float routed_scale, int32_t* __restrict__ topk_idx,
                  float* __restrict__ topk_gate, int32_t* __restrict__ counts,
                  unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int a_atom = 128 * kBK * 2;              // this CTA's 128 token rows, one K atom
  const int b_atom = (n_pad / 2) * kBK * 2;      // this CTA's half of the centroids
  const int a_stage = kRouteAtoms * a_atom;
  const int b_stage = kRouteAtoms * b_atom;
  uint8_t* sA = smem;
  uint8_t* sB = smem + kRouteStages2 * a_stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kRouteStages2 * b_stage);
  uint64_t* empty = full + kRouteStages2;
  uint64_t* tfull = empty + kRouteStages2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  float* s_bias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);
  int* s_hist = reinterpret_cast<int*>(s_bias + kRouteMaxExperts);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int num_st = d / (kBK * kRouteAtoms);    // d % 256 == 0
  const int row0 = static_cast<int>(blockIdx.x >> 1) * (2 * kBM) + static_cast<int>(rank) * kBM;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kRouteStages2; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      mbar_init(tfull, 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmU);
      tma_prefetch_desc(&tmE);
    }
    __syncwarp();
    tmem_alloc_2sm(tmem_slot, tmem_cols);
    tmem_relinquish_2sm();
  } else if (warp >= 2) {
    for (int e = threadIdx.x - 64; e < kRouteMaxExperts; e += 128) {
      s_bias[e] = (KIND == 0 && bias != nullptr && e < n_routed) ? bias[e] : 0.0f;
      s_hist[e] = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_par = 0;
    const uint32_t stage_tx = 2u * kRouteAtoms * static_cast<uint32_t>(a_atom + b_atom);
    for (int st = 0; st < num_st; ++st) {
      if (!mbar_wait(&empty[stage], phase ^ 1u, status, kStatusTimeoutProducer)) break;
      if (rank == 0) mbar_arrive_expect_tx(&full[stage], stage_tx);
      const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
#pragma unroll
      for (int at = 0; at < kRouteAtoms; ++at) {
        const int x = (st * kRouteAtoms + at) * kBK;
        tma_load_2d_pair(sA + stage * a_stage + at * a_atom, &tmU, bar, x, row0);
        tma_load_2d_pair(sB + stage * b_stage + at * b_atom, &tmE, bar, x,
                         static_cast<int>(rank) * (n_pad / 2));
      }
      issued |= 1u << stage;
      issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
      if (++stage == kRouteStages2) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // the leader's full barriers count both CTAs' bytes: once they have
    // completed no TMA write into either CTA's shared memory is in flight
    if (rank == 0)
      for (int s = 0; s < kRouteStages2; ++s)
        if (issued & (1u << s))
          mbar_wait(&full[s], (issued_par >> s) & 1u, status, kStatusTimeoutProducer);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (leader)
    const uint32_t idesc = idesc_bf16_f32(2 * kBM, n_pad);
    int stage = 0;
    uint32_t phase = 0;
    for (int st = 0; st < num_st; ++st) {
      if (!mbar_wait(&full[stage], phase, status, kStatusTimeoutMma)) break;
      tc_fence_after();
#pragma unroll
      for (int at = 0; at < kRouteAtoms; ++at) {
        const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * a_stage + at * a_atom));
        const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * b_stage + at * b_atom));
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k)
          umma_bf16_pair(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (st | at | k) != 0);
      }
      const uint32_t e = smem_u32(&empty[stage]);
      umma_commit_pair(mapa_shared(e, 0));
      umma_commit_pair(mapa_shared(e, 1));
      if (++stage == kRouteStages2) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // tfull of both CTAs fires when every MMA above has completed (also on the
    // error path, so TMEM is never released under a running MMA)
    const uint32_t f = smem_u32(tfull);
    umma_commit_pair(mapa_shared(f, 0));
    umma_commit_pair(mapa_shared(f, 1));
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int t = row0 + quarter * 32 + lane;
    const bool have = mbar_wait(tfull, 0, status, kStatusTimeoutEpilogue);
    tc_fence_after();
    float kv[TOPK], sv[TOPK];
    int ki[TOPK];
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
      kv[p] = -INFINITY;
      sv[p] = 0.0f;
      ki[p] = -1;
    }
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    if (have) {
      for (int c = 0; c < n_pad; c += 32) {
        uint32_t zr[32];
        tmem_ld_32cols(taddr + c, zr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = c + i;
          if (j < n_routed)
            route_insert<TOPK, KIND>(__uint_as_float(zr[i]), j, s_bias[j], kv, sv, ki);
        }
      }
    }
    tc_fence_before();
    if (have && t < T)
      route_emit<TOPK, KIND>(sv, ki, routed_scale, t, topk_idx, topk_gate, s_hist);
    named_bar_sync(1, 128);
    for (int e = threadIdx.x - 64; e < n_routed; e += 128) {
      const int c = s_hist[e];
      if (c) atomicAdd(&counts[e], c);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // neither CTA leaves while the pair may still signal it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem_base, tmem_cols);
  }
}

// Split-K second pass: one warp per token adds its logits over the splits
// (fixed order, fp32; lane l holds experts l, l+32, ...), then selects the
// top-K with warp shuffles: K rounds of a warp-wide maximum of (key, lower
// expert index on equal keys), the winner leaving the candidates -- the same
// selection and order as route_insert. Gates, idx and the histogram as the
// fused kernel. Keys that are not finite numbers are never selected.
constexpr int kSelectWarps = 4;
template <int TOPK, int KIND>
__global__ void __launch_bounds__(32 * kSelectWarps)
route_select_kernel(const float* __restrict__ partial, int splits, const float* __restrict__ bias,
                    int T, int n_routed, int n_pad, float routed_scale,
                    int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                    int32_t* __restrict__ counts) {
  __shared__ int s_hist[kRouteMaxExperts];
  for (int e = threadIdx.x; e < kRouteMaxExperts; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelectWarps + (threadIdx.x >> 5);
  constexpr int kPer = kRouteMaxExperts / 32;
  if (t < T) {
    // z_j = sum over the splits in ascending order; the loads of four splits
    // are issued before their adds so that 4 x kPer of them are in flight
    float zs[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) zs[i] = 0.0f;
    const float* base = partial + static_cast<size_t>(t) * n_pad + lane;
    const size_t stride = static_cast<size_t>(T) * n_pad;
    int y = 0;
    for (; y + 4 <= splits; y += 4) {
      float v[4][kPer];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kPer; ++i)
          v[q][i] = (lane + 32 * i < n_routed) ? __ldg(base + (y + q) * stride + 32 * i) : 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int i = 0; i < kPer; ++i) zs[i] += v[q][i];
    }
    for (; y < splits; ++y)
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i < n_routed) zs[i] += __ldg(base + y * stride + 32 * i);
    float key[kPer], sval[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int j = lane + 32 * i;
      key[i] = -INFINITY;
      sval[i] = 0.0f;
      if (j < n_routed) {
        const float z = zs[i];
        float sv, kv;
        if constexpr (KIND == 0) {
          sv = 1.0f / (1.0f + expf(-z));
          kv = sv + (bias != nullptr ? __ldg(bias + j) : 0.0f);
        } else {
          sv = z;
          kv = z;
        }
        if (kv == kv) {                                  // NaN keys are never selected
          key[i] = kv;
          sval[i] = sv;
        }
      }
    }
    float sel_s[TOPK];
    int sel_j[TOPK];
#pragma unroll
    for (int p = 0; p < TOPK; ++p) {
      // this lane's best remaining candidate (ascending j on equal keys)
      float bk = -INFINITY;
      int bj = 0x7fffffff, bi = -1;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (key[i] > bk) {
          bk = key[i];
          bj = lane + 32 * i;
          bi = i;
        }
      // warp maximum of (key, then the lower index)
      float wk = bk;
      int wj = bi >= 0 ? bj : 0x7fffffff;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, wk, o);
        const int oj = __shfl_xor_sync(0xffffffffu, wj, o);
        if (ok > wk || (ok == wk && oj < wj)) {
          wk = ok;
          wj = oj;
        }
      }
      const bool found = wk > -INFINITY;
      float ws = 0.0f;
      if (found && bi >= 0 && bj == wj) {
#pragma unroll
        for (int i = 0; i < kPer; ++i)                    // (static indexes: registers)
          if (i == bi) {
            ws = sval[i];
            key[i] = -INFINITY;                           // leaves the candidates
          }
      }
      // the winner's s value from its lane
      ws = __shfl_sync(0xffffffffu, ws, found ? (wj & 31) : 0);
      sel_s[p] = found ? ws : 0.0f;
      sel_j[p] = found ? wj : -1;
    }
    if (lane == 0)
      route_emit<TOPK, KIND>(sel_s, sel_j, routed_scale, t, topk_idx, topk_gate, s_hist);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_routed; e += blockDim.x) {
    const int c = s_hist[e];
    if (c) atomicAdd(&counts[e], c);
  }
}

}  // namespace moe
