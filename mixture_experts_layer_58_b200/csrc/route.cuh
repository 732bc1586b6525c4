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

namespace moe {

constexpr int kRouteMaxExperts = 256;

struct RouteSmem {
  static size_t bytes(int n_pad) {
    return 1024 + static_cast<size_t>(kStages) * (kBM * kBK * 2 + n_pad * kBK * 2) + 256 +
           2 * kRouteMaxExperts * sizeof(float);
  }
};

template <int TOPK, int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1)
route_kernel(const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmE,
             const float* __restrict__ bias, int T, int d, int n_routed, int n_pad,
             uint32_t tmem_cols, float routed_scale, int32_t* __restrict__ topk_idx,
             float* __restrict__ topk_gate, int32_t* __restrict__ counts,
             unsigned int* status) {
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
  const int num_kb = d / kBK;
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
    for (int kb = 0; kb < num_kb; ++kb) {
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
    for (int kb = 0; kb < num_kb; ++kb) {
      if (!mbar_wait(&full[stage], phase, status, kStatusTimeoutMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t adesc = sw128_kmajor_desc(smem_u32(sA + stage * a_bytes));
      const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sB + stage * b_bytes));
#pragma unroll
      for (int k = 0; k < kBK / kUmmaK; ++k)
        umma_bf16(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0);
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
    if (have) {
      for (int c = 0; c < n_pad; c += 32) {
        uint32_t zr[32];
        tmem_ld_32cols(taddr + c, zr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = c + i;
          if (j < n_routed) {
            const float z = __uint_as_float(zr[i]);
            float s, key;
            if constexpr (KIND == 0) {
              s = 1.0f / (1.0f + expf(-z));
              key = s + s_bias[j];
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
        }
      }
    }
    tc_fence_before();
    if (have && t < T) {
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
    named_bar_sync(1, 128);
    for (int e = threadIdx.x - 64; e < n_routed; e += 128) {
      const int c = s_hist[e];
      if (c) atomicAdd(&counts[e], c);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace moe
