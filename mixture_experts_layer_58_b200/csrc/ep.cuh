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
#include "ptx.cuh"

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
