// Expert parallelism: the routed experts are split evenly over W ranks
// (rank p holds experts [p*n_local, (p+1)*n_local)), and the token rows
// travel by all-to-all exchanges: the dispatch sends every row of the
// expert-contiguous copy to the rank holding its expert, the experts run on
// the rows they received, and the return exchange brings each result back to
// the rank that owns the token. (DeepSeek-V3 technical report summary:
// "Problem setting and motivation", the all-to-all cost of fine-grained
// routing; "Main ideas", the DualPipe bullet; "Limitations", the SMs given
// to the all-to-all.)
//
// This header holds the two pieces that are not a collective:
//  - ep_plan_host: the host-side plan of one exchange (split sizes, the
//    expert-major grouping of the received rows and its inverse);
//  - gather_rows_kernel: dst[i] = src[index[i]], which puts the expert-major
//    down-projection output back in the order it was received, so that the
//    return exchange can send one contiguous block per rank.
#pragma once
#include "dispatch.cuh"

namespace moe {

// One warp per output row, 16-byte vectors, four in flight per lane. An index
// outside [0, n_src) writes a zero row and never reads src.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const __nv_bfloat16* __restrict__ src, int n_src,
                   const int32_t* __restrict__ index, int n, int d,
                   __nv_bfloat16* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nvec = d >> 3;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += warps) {
    const int r = index[i];
    const bool ok = static_cast<unsigned>(r) < static_cast<unsigned>(n_src);
    const uint4* srow = reinterpret_cast<const uint4*>(src + static_cast<size_t>(ok ? r : 0) * d);
    uint4* drow = reinterpret_cast<uint4*>(dst + static_cast<size_t>(i) * d);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = v0 + 32 * j;
        x[j] = make_uint4(0u, 0u, 0u, 0u);
        if (ok && v < nvec) x[j] = __ldg(srow + v);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = v0 + 32 * j;
        if (v < nvec) drow[v] = x[j];
      }
    }
  }
}

// Host plan of one exchange, seen from one rank.
//   local_counts [world * n_local]: rows this rank routes to each expert
//     (its route's load histogram; its expert-contiguous copy holds them in
//     expert order, so the rows for rank p form one contiguous block);
//   recv_counts [world, n_local]: rows rank q routes to this rank's local
//     expert e (the counts exchange's result).
// Received rows arrive source-major: rank q's block, inside it expert e's
// rows in q's token order. The experts read them expert-major: expert e's
// rows from rank 0, then from rank 1, ... (so that, for every expert, the
// rows keep the global token order of the ranks' batches laid end to end).
// regroup[j] = received row of expert-major row j; ungroup is its inverse.
// Returns the number of received rows, or -1 (a negative count) / -2 (more
// than 2^31 - 1 rows, or more than recv_capacity when regroup is given).
inline long long ep_plan_host(const int32_t* local_counts, const int32_t* recv_counts, int world,
                              int n_local, long long recv_capacity, long long* send_splits,
                              long long* recv_splits, int32_t* group_offsets, int32_t* regroup,
                              int32_t* ungroup) {
  long long total = 0;
  for (int q = 0; q < world; ++q)
    for (int e = 0; e < n_local; ++e) {
      const int32_t c = recv_counts[static_cast<size_t>(q) * n_local + e];
      const int32_t s = local_counts[static_cast<size_t>(q) * n_local + e];
      if (c < 0 || s < 0) return -1;
      total += c;
    }
  if (total > 0x7fffffffLL) return -2;
  if ((regroup || ungroup) && total > recv_capacity) return -2;
  for (int p = 0; p < world; ++p) {
    long long s = 0, r = 0;
    for (int e = 0; e < n_local; ++e) {
      s += local_counts[static_cast<size_t>(p) * n_local + e];
      r += recv_counts[static_cast<size_t>(p) * n_local + e];
    }
    send_splits[p] = s;
    recv_splits[p] = r;
  }
  long long j = 0;
  for (int e = 0; e < n_local; ++e) {
    group_offsets[e] = static_cast<int32_t>(j);
    long long base = 0;  // start of rank q's block in the received buffer
    for (int q = 0; q < world; ++q) {
      long long within = 0;  // expert e's first row inside rank q's block
      for (int e2 = 0; e2 < e; ++e2) within += recv_counts[static_cast<size_t>(q) * n_local + e2];
      const int32_t c = recv_counts[static_cast<size_t>(q) * n_local + e];
      for (int32_t r = 0; r < c; ++r, ++j) {
        const long long row = base + within + r;
        if (regroup) regroup[j] = static_cast<int32_t>(row);
        if (ungroup) ungroup[row] = static_cast<int32_t>(j);
      }
      base += recv_splits[q];
    }
  }
  group_offsets[n_local] = static_cast<int32_t>(j);
  return total;
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// Expert parallelism over peer memory (no host round trip, no all-to-all
// collective for the rows). Every rank all-gathers the per-expert loads of
// every rank, all_counts [W, N_r]; from it each rank computes, on the device,
// where its rows land in every owner's receive buffer, and its own dispatch
// kernel stores them there (NVLink peer stores; on one GPU a local buffer).
// The owner's receive buffer is expert-major: expert e's rows from rank 0,
// then from rank 1, ..., each rank's rows in its own token order -- the order
// a single GPU's stable dispatch gives the ranks' batches laid end to end.
//   row(E, p, i) = recv_off[E] + sum_{p' < p} all_counts[p', E] + i
//   recv_off[E]  = sum over the owner's experts E' < E of sum_p all_counts[p, E']
// The combine reads each token's K expert outputs back from the owners'
// output buffers at the same rows.

// One block of n_routed (<= 256) threads. dest_row[E]: first row of this
// rank's rows for expert E in its owner's receive buffer; group_offsets
// [n_local + 1]: the expert-major offsets of this rank's own receive buffer;
// global_counts[E]: the load of expert E summed over the ranks. A receive
// buffer needing more than `capacity` rows sets kStatusEpOverflow (the
// dispatch then drops the rows past the capacity: never a silent result,
// the status word reports it).
// add_counts (may be NULL) is added to global_counts: the loads of an
// earlier micro-batch of the same step, so the bias update sees the step's.
__global__ void __launch_bounds__(256)
ep_plan_device_kernel(const int32_t* __restrict__ all_counts, int world, int n_local, int rank,
                      long long capacity, const int32_t* __restrict__ add_counts,
                      int32_t* __restrict__ dest_row, int32_t* __restrict__ group_offsets,
                      int32_t* __restrict__ global_counts, unsigned int* status) {
  __shared__ long long s_scan[256];
  const int n_routed = world * n_local;
  const int E = threadIdx.x;
  long long tot = 0, before = 0;
  if (E < n_routed) {
    for (int p = 0; p < world; ++p) {
      const long long c = all_counts[static_cast<size_t>(p) * n_routed + E];
      tot += c;
      if (p < rank) before += c;
    }
  }
  s_scan[E] = tot;
  __syncthreads();
  for (int o = 1; o < 256; o <<= 1) {
    const long long v = E >= o ? s_scan[E - o] : 0;
    __syncthreads();
    s_scan[E] += v;
    __syncthreads();
  }
  if (E < n_routed) {
    const int owner0 = (E / n_local) * n_local;            // the owner's first expert
    const long long base = owner0 > 0 ? s_scan[owner0 - 1] : 0;
    const long long recv_off = s_scan[E] - tot - base;     // exclusive, within the owner
    dest_row[E] = static_cast<int32_t>(recv_off + before);
    global_counts[E] = static_cast<int32_t>(tot + (add_counts ? add_counts[E] : 0));
    if (E / n_local == rank) {
      const int e = E - owner0;
      group_offsets[e] = static_cast<int32_t>(recv_off);
      if (e == n_local - 1) {
        const long long n_recv = recv_off + tot;
        group_offsets[n_local] = static_cast<int32_t>(n_recv);
        if (n_recv > capacity) atomicOr(status, kStatusEpOverflow);
      }
    }
  }
}

// Row of (token t, slot k) in its expert's owner's receive buffer, and the
// owner, from this rank's dispatch (pos, expert_offsets) and the plan; -1 if
// the pair has no row or the row lies past the capacity.
__device__ __forceinline__ long long ep_p2p_row(int e, int p, const int32_t* offsets,
                                                const int32_t* dest_row, int n_routed,
                                                long long total, long long capacity) {
  if (static_cast<unsigned>(e) >= static_cast<unsigned>(n_routed) || p < 0 || p >= total)
    return -1;
  const long long row = static_cast<long long>(__ldg(dest_row + e)) + p - __ldg(offsets + e);
  return (row >= 0 && row < capacity) ? row : -1;
}

// One warp per token: reads its row of u once (16-byte vectors) and stores
// it into the receive buffer of each of its K experts' owners (peer_x[q] is
// rank q's buffer as seen from this GPU). Ends with a system-scope fence so
// the stores are visible to the peers before whatever this rank does next.
__global__ void __launch_bounds__(256)
ep_dispatch_p2p_kernel(const __nv_bfloat16* __restrict__ u, const int32_t* __restrict__ idx,
                       const int32_t* __restrict__ pos, const int32_t* __restrict__ offsets,
                       const int32_t* __restrict__ dest_row, int T, int d, int K, int n_routed,
                       int n_local, __nv_bfloat16* const* __restrict__ peer_x,
                       long long capacity) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const long long total = static_cast<long long>(T) * K;
  const int nvec = d >> 3;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    long long myrow = -1;
    int myq = 0;
    if (lane < K) {
      const int e = idx[static_cast<size_t>(t) * K + lane];
      const int p = pos[static_cast<size_t>(t) * K + lane];
      myrow = ep_p2p_row(e, p, offsets, dest_row, n_routed, total, capacity);
      myq = myrow >= 0 ? e / n_local : 0;
    }
    uint4* dst[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      const long long row = __shfl_sync(0xffffffffu, myrow, k);
      const int q = __shfl_sync(0xffffffffu, myq, k);
      dst[k] = (k < K && row >= 0)
                   ? reinterpret_cast<uint4*>(peer_x[q] + static_cast<size_t>(row) * d)
                   : nullptr;
    }
    const uint4* srow = reinterpret_cast<const uint4*>(u + static_cast<size_t>(t) * d);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (v0 + 32 * j < nvec) x[j] = __ldg(srow + v0 + 32 * j);
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k) {
        if (!dst[k]) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (v0 + 32 * j < nvec) dst[k][v0 + 32 * j] = x[j];
      }
    }
  }
  __threadfence_system();
}

// out_t = residual_t + shared_t + sum_k g[t,k] * y_q[row(t,k)]: the combine of
// one GPU, its routed rows read from the owners' output buffers (peer_y[q]).
// One warp per token, fp32 sums in slot order, one bf16 rounding.
__global__ void __launch_bounds__(256)
ep_combine_p2p_kernel(const __nv_bfloat16* const* __restrict__ peer_y,
                      const int32_t* __restrict__ idx, const int32_t* __restrict__ pos,
                      const int32_t* __restrict__ offsets, const int32_t* __restrict__ dest_row,
                      const float* __restrict__ gate, const __nv_bfloat16* __restrict__ shared_out,
                      const __nv_bfloat16* residual, int T, int d, int K, int n_routed,
                      int n_local, long long capacity, __nv_bfloat16* out) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const long long total = static_cast<long long>(T) * K;
  const int nvec = d >> 3;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    long long myrow = -1;
    int myq = 0;
    float myg = 0.0f;
    if (lane < K) {
      const int e = idx[static_cast<size_t>(t) * K + lane];
      const int p = pos[static_cast<size_t>(t) * K + lane];
      myrow = ep_p2p_row(e, p, offsets, dest_row, n_routed, total, capacity);
      myq = myrow >= 0 ? e / n_local : 0;
      myg = gate[static_cast<size_t>(t) * K + lane];
    }
    const uint4* src[kMaxTopK];
    float g[kMaxTopK];
#pragma unroll
    for (int k = 0; k < kMaxTopK; ++k) {
      const long long row = __shfl_sync(0xffffffffu, myrow, k);
      const int q = __shfl_sync(0xffffffffu, myq, k);
      g[k] = __shfl_sync(0xffffffffu, myg, k);
      src[k] = (k < K && row >= 0)
                   ? reinterpret_cast<const uint4*>(peer_y[q] + static_cast<size_t>(row) * d)
                   : nullptr;
    }
    const size_t row = static_cast<size_t>(t) * d;
    for (int v = lane; v < nvec; v += 32) {
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = 0.0f;
      uint4 yv[kMaxTopK];
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k)
        if (src[k]) yv[k] = src[k][v];
      if (residual) add_bf16x8(a, *(reinterpret_cast<const uint4*>(residual + row) + v));
      if (shared_out) add_bf16x8(a, __ldg(reinterpret_cast<const uint4*>(shared_out + row) + v));
#pragma unroll
      for (int k = 0; k < kMaxTopK; ++k)
        if (src[k]) acc_bf16x8(a, yv[k], g[k]);
      uint4 o;
      o.x = pack_bf16x2(a[0], a[1]);
      o.y = pack_bf16x2(a[2], a[3]);
      o.z = pack_bf16x2(a[4], a[5]);
      o.w = pack_bf16x2(a[6], a[7]);
      *(reinterpret_cast<uint4*>(out + row) + v) = o;
    }
  }
}

}  // namespace moe
