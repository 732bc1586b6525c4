// C-ABI entry points of libmoe.so (declared in include/moe.h): host-side
// validation, TMA tensor-map construction and kernel launches. Every entry
// point checks its arguments before touching the GPU and returns a status
// code; nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <unordered_map>

#include "moe.h"
#include "dispatch.cuh"
#include "fp8.cuh"
#include "gemm.cuh"
#include "gemm2sm.cuh"
#include "gemm_fp8.cuh"
#include "route.cuh"
#include "bwd.cuh"
#include "gemm_bwd.cuh"
#include "ep.cuh"

namespace {

using namespace moe;

__device__ unsigned int g_status;   // per-device status word (see moe_get_device_status)

// Tile counters of the CTA-pair GEMM's dynamic schedule; each launch takes the
// next slot (round robin) and zeroes it on its stream first.
constexpr int kTileCounters = 256;
__device__ int g_tile_counters[kTileCounters];

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  // set (release) after the fields below; read (acquire) before using them
  std::atomic<bool> ready{false};
  int num_sms = 0;
  unsigned int* status = nullptr;
  int* tile_counters = nullptr;
  std::atomic<unsigned> next_counter{0};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

inline int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return MOE_ERR_CUDA;
}

#define MOE_CUDA(call)                        \
  do {                                        \
    cudaError_t _e = (call);                  \
    if (_e != cudaSuccess) return cuda_fail(_e); \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device constants, looked up once.
int device_info(DeviceInfo** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_INVALID_ARG;
  DeviceInfo& di = g_dev[dev];
  if (!di.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!di.ready.load(std::memory_order_relaxed)) {
      MOE_CUDA(cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev));
      void* p = nullptr;
      MOE_CUDA(cudaGetSymbolAddress(&p, g_status));
      di.status = static_cast<unsigned int*>(p);
      MOE_CUDA(cudaGetSymbolAddress(&p, g_tile_counters));
      di.tile_counters = static_cast<int*>(p);
      di.ready.store(true, std::memory_order_release);
    }
  }
  *out = &di;
  return MOE_OK;
}

int get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    t_last_cuda_error = static_cast<int>(cudaErrorNotSupported);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, box
// [box_rows, 64 columns], 128-byte swizzle, zero fill out of bounds.
int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                   uint32_t box_rows) {
  int rc = get_encoder();
  if (rc != MOE_OK) return rc;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// 2-D bf16 tensor map for TMA stores of 32 x 32 blocks into a row-major
// [rows, cols] matrix; the shared-memory block uses the 64-byte swizzle.
int make_tmap_bf16_store32(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
  int rc = get_encoder();
  if (rc != MOE_OK) return rc;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

template <typename K>
int set_smem(K kernel, size_t bytes) {
  // The attribute is per-process state of the kernel: set it when a launch
  // needs more than any launch before (not per launch), so that launches
  // recorded into a CUDA graph after a first eager call make no such call.
  static std::mutex mu;
  static std::unordered_map<const void*, size_t> set;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = set[reinterpret_cast<const void*>(kernel)];
  if (bytes > cur) {
    MOE_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(bytes)));
    cur = bytes;
  }
  return MOE_OK;
}

inline cudaStream_t as_stream(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// ------------------------------------------------------------------ GEMM launch
template <int BN, int EPI>
int launch_grouped_gemm(const void* A, int rows, int K, const void* B, int G, int n_per_group,
                        const int32_t* offsets, void* out, int ldo, cudaStream_t st,
                        void* ac = nullptr, ScatterOut sc = ScatterOut{nullptr, nullptr, 0}) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  CUtensorMap tmA, tmB;
  if ((rc = make_tmap_bf16(&tmA, A, K, rows, kBM)) != MOE_OK) return rc;
  if ((rc = make_tmap_bf16(&tmB, B, K, static_cast<uint64_t>(G) * n_per_group, BN)) != MOE_OK)
    return rc;
  const size_t smem = GemmCfg<BN>::smem_bytes(G);
  auto kern = grouped_gemm_bf16_kernel<BN, EPI>;
  if ((rc = set_smem(kern, smem)) != MOE_OK) return rc;
  const long long max_tiles =
      (static_cast<long long>(rows) / kBM + G) * static_cast<long long>(n_per_group / BN);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(di->num_sms, max_tiles)));
  kern<<<grid, kGemmThreads, smem, st>>>(tmA, tmB, offsets, G, K, n_per_group, rows,
                                         static_cast<__nv_bfloat16*>(out), ldo,
                                         static_cast<__nv_bfloat16*>(ac), di->status, sc);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// 2-D E4M3 (byte) tensor map over a row-major [rows, cols] matrix, box
// [box_rows, 128 columns], 128-byte swizzle, zero fill out of bounds.
int make_tmap_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                 uint32_t box_rows) {
  int rc = get_encoder();
  if (rc != MOE_OK) return rc;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kF8BK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

template <int EPI>
int launch_grouped_gemm_fp8(const void* A, const float* a_scales, int rows, int K, const void* B,
                            const float* b_scales, int G, int n_per_group,
                            const int32_t* offsets, void* out, int ldo, cudaStream_t st,
                            void* qout = nullptr, float* qscales = nullptr) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  CUtensorMap tmA, tmB;
  if ((rc = make_tmap_u8(&tmA, A, K, rows, kBM)) != MOE_OK) return rc;
  if ((rc = make_tmap_u8(&tmB, B, K, static_cast<uint64_t>(G) * n_per_group, kF8BN)) != MOE_OK)
    return rc;
  const size_t smem = GemmF8Cfg::smem_bytes(G);
  auto kern = grouped_gemm_fp8_kernel<EPI>;
  if ((rc = set_smem(kern, smem)) != MOE_OK) return rc;
  const long long max_tiles = (static_cast<long long>(rows) / kBM + G) *
                              static_cast<long long>(n_per_group / (kF8BN * f8_subtiles<EPI>()));
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(di->num_sms, max_tiles)));
  int* counter = di->tile_counters + (di->next_counter.fetch_add(1) % kTileCounters);
  MOE_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  kern<<<grid, kF8Threads, smem, st>>>(tmA, tmB, a_scales, b_scales, offsets, G, K, n_per_group,
                                       rows, static_cast<__nv_bfloat16*>(out), ldo,
                                       static_cast<uint8_t*>(qout), qscales, counter,
                                       di->status);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// CTA-pair form of the grouped GEMM (256-row tiles, tcgen05 cta_group::2).
// With src_rows, logical A row r is row src_rows[r] of A ([a_rows, K]),
// gathered by the kernel (box one row high).
template <int EPI>
int launch_grouped_gemm_pair(const void* A, int rows, int K, const void* B, int G,
                             int n_per_group, const int32_t* offsets, void* out, int ldo,
                             cudaStream_t st, const int32_t* src_rows = nullptr,
                             int a_rows = 0, void* ac = nullptr,
                             ScatterOut sc = ScatterOut{nullptr, nullptr, 0}) {
  if (K % (kBK * kAtoms2) != 0) return MOE_ERR_UNSUPPORTED_SHAPE;   // whole ring stages
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  CUtensorMap tmA, tmA32, tmB;
  if (src_rows) {
    if ((rc = make_tmap_bf16(&tmA, A, K, a_rows, 1)) != MOE_OK) return rc;
    tmA32 = tmA;
  } else {
    // token rows: 128 per box for full tiles, 32 per box for ragged tails
    if ((rc = make_tmap_bf16(&tmA, A, K, rows, 128)) != MOE_OK) return rc;
    if ((rc = make_tmap_bf16(&tmA32, A, K, rows, 32)) != MOE_OK) return rc;
  }
  if ((rc = make_tmap_bf16(&tmB, B, K, static_cast<uint64_t>(G) * n_per_group, 128)) != MOE_OK)
    return rc;
  const size_t smem = Gemm2smCfg::smem_bytes(G);
  const long long max_tiles =
      (static_cast<long long>(rows) / kBM2 + G) * static_cast<long long>(n_per_group / 256);
  const int pairs = static_cast<int>(std::max(1LL, std::min<long long>(di->num_sms / 2, max_tiles)));
  int* counter = di->tile_counters + (di->next_counter.fetch_add(1) % kTileCounters);
  MOE_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  if (src_rows) {
    auto kern = grouped_gemm_bf16_pair_kernel<EPI, true>;
    if ((rc = set_smem(kern, smem)) != MOE_OK) return rc;
    kern<<<2 * pairs, kPairThreads, smem, st>>>(tmA, tmA32, tmB, offsets, G, K, n_per_group, rows,
                                                 static_cast<__nv_bfloat16*>(out), ldo,
                                                 static_cast<__nv_bfloat16*>(ac), src_rows,
                                                 counter, di->status, sc);
  } else {
    auto kern = grouped_gemm_bf16_pair_kernel<EPI, false>;
    if ((rc = set_smem(kern, smem)) != MOE_OK) return rc;
    kern<<<2 * pairs, kPairThreads, smem, st>>>(tmA, tmA32, tmB, offsets, G, K, n_per_group, rows,
                                                 static_cast<__nv_bfloat16*>(out), ldo,
                                                 static_cast<__nv_bfloat16*>(ac), nullptr,
                                                 counter, di->status, sc);
  }
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// dgrad: out[rows of g] = A[rows of g] (K-major, [rows, K]) * W_g ([K, N] row-major).
template <int EPI>
int launch_dgrad(const void* A, int rows, int K, const void* W, int G, int N,
                 const int32_t* offsets, void* out, int ldo, const void* ac, cudaStream_t st) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  CUtensorMap tmA, tmW;
  if ((rc = make_tmap_bf16(&tmA, A, K, rows, kBM)) != MOE_OK) return rc;
  if ((rc = make_tmap_bf16(&tmW, W, N, static_cast<uint64_t>(G) * K, 64)) != MOE_OK) return rc;
  const size_t smem = BwdCfg::smem_bytes(G);
  auto kern = grouped_dgrad_bf16_kernel<EPI>;
  if ((rc = set_smem(kern, smem)) != MOE_OK) return rc;
  const long long max_tiles = (static_cast<long long>(rows) / kBM + G) *
                              static_cast<long long>((N + BwdCfg::kBN - 1) / BwdCfg::kBN);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(di->num_sms, max_tiles)));
  int* counter = di->tile_counters + (di->next_counter.fetch_add(1) % kTileCounters);
  MOE_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  kern<<<grid, kGemmThreads, smem, st>>>(tmA, tmW, offsets, G, K, N, rows,
                                         static_cast<__nv_bfloat16*>(out), ldo,
                                         static_cast<const __nv_bfloat16*>(ac), counter,
                                         di->status);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// wgrad: dw[g] = A[rows of g]^T B[rows of g]; A [rows, M], B [rows, N], dw [G, M, N].
int launch_wgrad(const void* A, const void* B, int rows, int M, int N, int G,
                 const int32_t* offsets, void* dw, cudaStream_t st) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  CUtensorMap tmA, tmB, tmD;
  if ((rc = make_tmap_bf16(&tmA, A, M, rows, 64)) != MOE_OK) return rc;
  if ((rc = make_tmap_bf16(&tmB, B, N, rows, 64)) != MOE_OK) return rc;
  if ((rc = make_tmap_bf16_store32(&tmD, dw, N, static_cast<uint64_t>(G) * M)) != MOE_OK)
    return rc;
  int* counter = di->tile_counters + (di->next_counter.fetch_add(1) % kTileCounters);
  MOE_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  const size_t smem = BwdCfg::wgrad_smem_bytes(G);
  if ((rc = set_smem(grouped_wgrad_bf16_kernel, smem)) != MOE_OK) return rc;
  const long long tiles = static_cast<long long>(G) * (M / kBM) *
                          ((N + BwdCfg::kBN - 1) / BwdCfg::kBN);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(di->num_sms, tiles)));
  grouped_wgrad_bf16_kernel<<<grid, BwdCfg::kWgThreads, smem, st>>>(tmA, tmB, tmD, offsets, G, M, N,
                                                               rows, counter, di->status);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// Tile shape of the bf16 expert GEMMs, chosen per call from the average
// group size: CTA-pair 256-row tiles move less data per flop, but a group of a
// few rows (decode) would fill a 256-row tile with padding, so groups that
// average fewer than 256 rows run on single-CTA 128-row tiles.
inline bool use_pair_tiles(int rows, int G) {
  return static_cast<long long>(rows) >= 256LL * G;
}

int check_ffn_shape(int G, int rows, int d, int inter) {
  if (G < 1 || rows < 0 || d <= 0 || inter <= 0) return MOE_ERR_INVALID_ARG;
  if (G > kMaxGroups || d % 256 != 0 || inter % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(G) * 2 * inter > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// Split-K form of the gate GEMM for small batches: splits chosen from the
// shapes alone (so the workspace size needs no device query) -- K blocks of
// at least 4 stages per CTA and at most ~128 CTAs over all token blocks.
inline int route_splits(int T, int d) {
  const int blocks = (T + kBM - 1) / kBM;
  const int num_kb = d / kBK;
  int splits = std::max(1, std::min((num_kb + 3) / 4, 128 / std::max(1, blocks)));
  const int per = (num_kb + splits - 1) / splits;
  return (num_kb + per - 1) / per;
}

// CTA-pair route (one cluster per 256 tokens): tmE2 boxes half of the
// centroid rows (n_pad2 / 2, n_pad2 a multiple of 32).
template <int TOPK>
int launch_route_pair(int kind, const CUtensorMap& tmU, const CUtensorMap& tmE2, const float* bias,
                      int T, int d, int n_routed, int n_pad2, uint32_t tcols, float scale,
                      int32_t* idx, float* gate, int32_t* counts, unsigned int* status,
                      cudaStream_t st) {
  const size_t smem = RoutePairSmem::bytes(n_pad2);
  const int ctas = 2 * ((T + 2 * kBM - 1) / (2 * kBM));
  int rc;
  if (kind == MOE_GATE_SIGMOID_BIAS) {
    auto k = route_pair_kernel<TOPK, 0>;
    if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
    k<<<ctas, kGemmThreads, smem, st>>>(tmU, tmE2, bias, T, d, n_routed, n_pad2, tcols, scale, idx,
                                        gate, counts, status);
  } else {
    auto k = route_pair_kernel<TOPK, 1>;
    if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
    k<<<ctas, kGemmThreads, smem, st>>>(tmU, tmE2, bias, T, d, n_routed, n_pad2, tcols, scale, idx,
                                        gate, counts, status);
  }
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

template <int TOPK>
int launch_route_k(int kind, const CUtensorMap& tmU, const CUtensorMap& tmE, const float* bias,
                   int T, int d, int n_routed, int n_pad, uint32_t tcols, float scale,
                   int32_t* idx, float* gate, int32_t* counts, float* partial, int splits,
                   unsigned int* status, cudaStream_t st) {
  const size_t smem = RouteSmem::bytes(n_pad);
  const int blocks = (T + kBM - 1) / kBM;
  const int num_kb = d / kBK;
  int rc;
  if (partial == nullptr) {
    if (kind == MOE_GATE_SIGMOID_BIAS) {
      auto k = route_kernel<TOPK, 0, false>;
      if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
      k<<<blocks, kGemmThreads, smem, st>>>(tmU, tmE, bias, T, d, n_routed, n_pad, tcols, scale,
                                            idx, gate, counts, nullptr, num_kb, status);
    } else {
      auto k = route_kernel<TOPK, 1, false>;
      if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
      k<<<blocks, kGemmThreads, smem, st>>>(tmU, tmE, bias, T, d, n_routed, n_pad, tcols, scale,
                                            idx, gate, counts, nullptr, num_kb, status);
    }
    MOE_CUDA(cudaGetLastError());
    return MOE_OK;
  }
  const int per = (num_kb + splits - 1) / splits;
  const dim3 grid(blocks, splits);
  const int sel_blocks = (T + kSelectWarps - 1) / kSelectWarps;
  if (kind == MOE_GATE_SIGMOID_BIAS) {
    auto k = route_kernel<TOPK, 0, true>;
    if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
    k<<<grid, kGemmThreads, smem, st>>>(tmU, tmE, bias, T, d, n_routed, n_pad, tcols, scale, idx,
                                        gate, counts, partial, per, status);
    MOE_CUDA(cudaGetLastError());
    route_select_kernel<TOPK, 0><<<sel_blocks, 32 * kSelectWarps, 0, st>>>(
        partial, splits, bias, T, n_routed, n_pad, scale, idx, gate, counts);
  } else {
    auto k = route_kernel<TOPK, 1, true>;
    if ((rc = set_smem(k, smem)) != MOE_OK) return rc;
    k<<<grid, kGemmThreads, smem, st>>>(tmU, tmE, bias, T, d, n_routed, n_pad, tcols, scale, idx,
                                        gate, counts, partial, per, status);
    MOE_CUDA(cudaGetLastError());
    route_select_kernel<TOPK, 1><<<sel_blocks, 32 * kSelectWarps, 0, st>>>(
        partial, splits, nullptr, T, n_routed, n_pad, scale, idx, gate, counts);
  }
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// Diagnostic: one thread waits on an mbarrier that nothing arrives on, for at
// most limit_ns, then records kStatusTimeoutSelfTest in the status word, the
// way every pipeline wait of the library gives up.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicOr(status, kStatusTimeoutSelfTest);
        break;
      }
    }
  }
}

}  // namespace

extern "C" {

int moe_version(void) { return 300; }

int moe_selftest_wait_timeout(int limit_ms, moe_stream_t stream) {
  if (limit_ms <= 0 || limit_ms > 10000) return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(
      static_cast<unsigned long long>(limit_ms) * 1000000ull, di->status);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

const char* moe_strerror(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer, bad size or enum)";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error (see moe_last_cuda_error)";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out, or a device-side limit was hit";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int moe_last_cuda_error(void) { return t_last_cuda_error; }

int moe_get_device_status(unsigned int* status, int clear) {
  if (!status) return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  MOE_CUDA(cudaDeviceSynchronize());
  unsigned int v = 0;
  MOE_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof(v)));
  if (clear && v) {
    const unsigned int zero = 0;
    MOE_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)));
  }
  *status = v;
  return v ? MOE_ERR_DEVICE_TIMEOUT : MOE_OK;
}

// ------------------------------------------------------------------ route
namespace {
int route_impl(const void* u, const void* centroids, const float* bias, int T, int d,
               int n_routed, int top_k, moe_gate_kind kind, float routed_scale,
               int32_t* topk_idx, float* topk_gate, int32_t* expert_counts, float* partial,
               cudaStream_t st) {
  MOE_CUDA(cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * n_routed, st));
  if (T == 0) return MOE_OK;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int n_pad = std::max(16, (n_routed + 15) / 16 * 16);
  uint32_t tcols = 32;
  while (tcols < static_cast<uint32_t>(n_pad)) tcols <<= 1;
  CUtensorMap tmU, tmE;
  if ((rc = make_tmap_bf16(&tmU, u, d, T, kBM)) != MOE_OK) return rc;
  if ((rc = make_tmap_bf16(&tmE, centroids, d, n_routed, n_pad)) != MOE_OK) return rc;
  const float* b = (kind == MOE_GATE_SIGMOID_BIAS) ? bias : nullptr;
  const int splits = partial ? route_splits(T, d) : 1;
  // one pass over K with at least one full pair of 128-token blocks: the
  // CTA-pair kernel (N = N_r padded to 32, half of it per CTA)
  const bool pair = partial == nullptr && T >= 2 * kBM;
  const int n_pad2 = std::max(32, (n_routed + 31) / 32 * 32);
  uint32_t tcols2 = 32;
  while (tcols2 < static_cast<uint32_t>(n_pad2)) tcols2 <<= 1;
  CUtensorMap tmE2;
  if (pair && (rc = make_tmap_bf16(&tmE2, centroids, d, n_routed, n_pad2 / 2)) != MOE_OK)
    return rc;
#define MOE_ROUTE_PAIR_CASE(KK)                                                                \
  case KK:                                                                                     \
    return launch_route_pair<KK>(kind, tmU, tmE2, b, T, d, n_routed, n_pad2, tcols2,           \
                                 routed_scale, topk_idx, topk_gate, expert_counts, di->status, \
                                 st);
  if (pair) {
    switch (top_k) {
      MOE_ROUTE_PAIR_CASE(1)
      MOE_ROUTE_PAIR_CASE(2)
      MOE_ROUTE_PAIR_CASE(3)
      MOE_ROUTE_PAIR_CASE(4)
      MOE_ROUTE_PAIR_CASE(5)
      MOE_ROUTE_PAIR_CASE(6)
      MOE_ROUTE_PAIR_CASE(7)
      MOE_ROUTE_PAIR_CASE(8)
      default: return MOE_ERR_UNSUPPORTED_SHAPE;
    }
  }
#undef MOE_ROUTE_PAIR_CASE
#define MOE_ROUTE_CASE(KK)                                                                   \
  case KK:                                                                                   \
    return launch_route_k<KK>(kind, tmU, tmE, b, T, d, n_routed, n_pad, tcols, routed_scale, \
                              topk_idx, topk_gate, expert_counts, partial, splits, di->status, \
                              st);
  switch (top_k) {
    MOE_ROUTE_CASE(1)
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(3)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(5)
    MOE_ROUTE_CASE(6)
    MOE_ROUTE_CASE(7)
    MOE_ROUTE_CASE(8)
    default: return MOE_ERR_UNSUPPORTED_SHAPE;
  }
#undef MOE_ROUTE_CASE
}

int route_check(const void* u, const void* centroids, int T, int d, int n_routed, int top_k,
                moe_gate_kind kind, float routed_scale, int32_t* topk_idx, float* topk_gate,
                int32_t* expert_counts) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (kind != MOE_GATE_SIGMOID_BIAS && kind != MOE_GATE_SOFTMAX_TOPK) return MOE_ERR_INVALID_ARG;
  if (!expert_counts || !centroids || !aligned16(centroids)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!u || !topk_idx || !topk_gate || !aligned16(u))) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 256 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!(routed_scale == routed_scale)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace

int moe_route(const void* u, const void* centroids, const float* bias, int T, int d, int n_routed,
              int top_k, moe_gate_kind kind, float routed_scale, int32_t* topk_idx,
              float* topk_gate, int32_t* expert_counts, moe_stream_t stream) {
  const int rc = route_check(u, centroids, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
                             topk_gate, expert_counts);
  if (rc != MOE_OK) return rc;
  return route_impl(u, centroids, bias, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
                    topk_gate, expert_counts, nullptr, as_stream(stream));
}

size_t moe_route_splitk_workspace_size(int T, int d, int n_routed) {
  if (T <= 0 || d <= 0 || d % 256 != 0 || n_routed <= 0 || n_routed > kRouteMaxExperts)
    return 16;
  const size_t n_pad = std::max(16, (n_routed + 15) / 16 * 16);
  const size_t bytes = static_cast<size_t>(route_splits(T, d)) * T * n_pad * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

int moe_route_splitk(const void* u, const void* centroids, const float* bias, int T, int d,
                     int n_routed, int top_k, moe_gate_kind kind, float routed_scale,
                     int32_t* topk_idx, float* topk_gate, int32_t* expert_counts,
                     void* workspace, size_t ws_bytes, moe_stream_t stream) {
  const int rc = route_check(u, centroids, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
                             topk_gate, expert_counts);
  if (rc != MOE_OK) return rc;
  if (T > 0 && (!workspace || !aligned16(workspace) ||
                ws_bytes < moe_route_splitk_workspace_size(T, d, n_routed)))
    return MOE_ERR_WORKSPACE;
  return route_impl(u, centroids, bias, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
                    topk_gate, expert_counts, static_cast<float*>(workspace), as_stream(stream));
}

// ------------------------------------------------------------------ permute
size_t moe_permute_workspace_size(int T, int n_routed) {
  if (T <= 0 || n_routed <= 0) return 16;
  const size_t chunks = (static_cast<size_t>(T) + kPermChunk - 1) / kPermChunk;
  return (chunks * n_routed * sizeof(int32_t) + 255) / 256 * 256;
}

namespace {
// moe_permute, and with `tail` the shared expert's rows appended after the
// routed ones (moe_permute_shared).
int permute_impl(const void* u, const int32_t* topk_idx, const int32_t* expert_counts, int T,
                 int d, int n_routed, int top_k, void* x_perm, int32_t* expert_offsets,
                 int32_t* pos, int32_t* src_token, void* workspace, size_t ws_bytes,
                 cudaStream_t st, bool tail) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 256 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * (top_k + (tail ? 1 : 0)) > INT32_MAX)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (n_routed + (tail ? 2 : 1)),
                             st));
    return MOE_OK;
  }
  if (!u || !topk_idx || !x_perm || !pos || !src_token || !aligned16(u) || !aligned16(x_perm))
    return MOE_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < moe_permute_workspace_size(T, n_routed) || !aligned16(workspace))
    return MOE_ERR_WORKSPACE;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int chunks = (T + kPermChunk - 1) / kPermChunk;
  int32_t* hist = static_cast<int32_t*>(workspace);
  permute_hist_kernel<<<chunks, 256, 0, st>>>(topk_idx, T, top_k, n_routed, hist);
  MOE_CUDA(cudaGetLastError());
  permute_index_kernel<<<chunks, 256, 0, st>>>(topk_idx, expert_counts, hist, T, top_k, n_routed,
                                               expert_offsets, pos, src_token);
  MOE_CUDA(cudaGetLastError());
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  if (tail)
    permute_copy_tail_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(u), pos, T,
                                                     d, top_k, static_cast<__nv_bfloat16*>(x_perm),
                                                     expert_offsets, n_routed);
  else
    permute_copy_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(u), pos, T, d,
                                                top_k, static_cast<__nv_bfloat16*>(x_perm));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}
}  // namespace

int moe_permute(const void* u, const int32_t* topk_idx, const int32_t* expert_counts, int T, int d,
                int n_routed, int top_k, void* x_perm, int32_t* expert_offsets, int32_t* pos,
                int32_t* src_token, void* workspace, size_t ws_bytes, moe_stream_t stream) {
  return permute_impl(u, topk_idx, expert_counts, T, d, n_routed, top_k, x_perm, expert_offsets,
                      pos, src_token, workspace, ws_bytes, as_stream(stream), false);
}

int moe_permute_shared(const void* u, const int32_t* topk_idx, const int32_t* expert_counts,
                       int T, int d, int n_routed, int top_k, void* x_perm,
                       int32_t* expert_offsets, int32_t* pos, int32_t* src_token,
                       void* workspace, size_t ws_bytes, moe_stream_t stream) {
  return permute_impl(u, topk_idx, expert_counts, T, d, n_routed, top_k, x_perm, expert_offsets,
                      pos, src_token, workspace, ws_bytes, as_stream(stream), true);
}

int moe_permute_index(const int32_t* topk_idx, const int32_t* expert_counts, int T,
                      int n_routed, int top_k, int32_t* expert_offsets, int32_t* pos,
                      int32_t* src_token, void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = as_stream(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (n_routed + 1), st));
    return MOE_OK;
  }
  if (!topk_idx || !pos || !src_token) return MOE_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < moe_permute_workspace_size(T, n_routed) || !aligned16(workspace))
    return MOE_ERR_WORKSPACE;
  const int chunks = (T + kPermChunk - 1) / kPermChunk;
  int32_t* hist = static_cast<int32_t*>(workspace);
  permute_hist_kernel<<<chunks, 256, 0, st>>>(topk_idx, T, top_k, n_routed, hist);
  MOE_CUDA(cudaGetLastError());
  permute_index_kernel<<<chunks, 256, 0, st>>>(topk_idx, expert_counts, hist, T, top_k, n_routed,
                                               expert_offsets, pos, src_token);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ expert FFN
size_t moe_grouped_ffn_workspace_size(int rows, int inter, moe_dtype dtype) {
  if (rows <= 0 || inter <= 0) return 256;
  if (dtype == MOE_FP8_E4M3) {
    const size_t codes = (static_cast<size_t>(rows) * inter + 255) / 256 * 256;
    const size_t scales = (static_cast<size_t>(rows) * (inter / 128) * 4 + 255) / 256 * 256;
    return codes + scales;
  }
  return (static_cast<size_t>(rows) * inter * 2 + 255) / 256 * 256;
}

size_t moe_workspace_size(int T, int d, int n_routed, int top_k, int inter, int shared_inter,
                          moe_dtype dtype) {
  (void)d;
  if (T <= 0 || n_routed <= 0 || top_k <= 0 || inter <= 0) return 256;
  const long long rows = static_cast<long long>(T) * top_k;
  size_t ws = moe_permute_workspace_size(T, n_routed);
  if (rows <= INT32_MAX)
    ws = std::max(ws, moe_grouped_ffn_workspace_size(static_cast<int>(rows), inter, dtype));
  if (shared_inter > 0) ws = std::max(ws, moe_grouped_ffn_workspace_size(T, shared_inter, dtype));
  return ws;
}

int moe_expert_up_swiglu(const void* x, const int32_t* group_offsets, int G, int rows, int d,
                         int inter, const void* w13, void* h, moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!x || !group_offsets || !w13 || !h || !aligned16(x) || !aligned16(w13) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  if (use_pair_tiles(rows, G))
    return launch_grouped_gemm_pair<EPI_SWIGLU>(x, rows, d, w13, G, 2 * inter, group_offsets, h,
                                                inter, as_stream(stream));
  return launch_grouped_gemm<256, EPI_SWIGLU>(x, rows, d, w13, G, 2 * inter, group_offsets, h,
                                              inter, as_stream(stream));
}

int moe_expert_up_swiglu_gather(const void* u, int T, const int32_t* src_token,
                                const int32_t* group_offsets, int G, int rows, int d, int inter,
                                const void* w13, void* h, moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (T == 0 || !u || !src_token || !group_offsets || !w13 || !h || !aligned16(u) ||
      !aligned16(w13) || !aligned16(h))
    return MOE_ERR_INVALID_ARG;
  return launch_grouped_gemm_pair<EPI_SWIGLU>(u, rows, d, w13, G, 2 * inter, group_offsets, h,
                                              inter, as_stream(stream), src_token, T);
}

int moe_expert_down(const void* h, const int32_t* group_offsets, int G, int rows, int inter, int d,
                    const void* w2, void* y, moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!h || !group_offsets || !w2 || !y || !aligned16(h) || !aligned16(w2) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (use_pair_tiles(rows, G))
    return launch_grouped_gemm_pair<EPI_STORE>(h, rows, inter, w2, G, d, group_offsets, y, d,
                                               as_stream(stream));
  return launch_grouped_gemm<256, EPI_STORE>(h, rows, inter, w2, G, d, group_offsets, y, d,
                                             as_stream(stream));
}

int moe_grouped_ffn(const void* x, const float* x_scales, const int32_t* group_offsets, int G,
                    int rows, int d, int inter, const void* w13, const float* w13_scales,
                    const void* w2, const float* w2_scales, moe_dtype dtype, void* y,
                    void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (dtype != MOE_BF16 && dtype != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!workspace || ws_bytes < moe_grouped_ffn_workspace_size(rows, inter, dtype) ||
      !aligned16(workspace))
    return MOE_ERR_WORKSPACE;
  if (dtype == MOE_FP8_E4M3) {
    uint8_t* h8 = static_cast<uint8_t*>(workspace);
    float* hs = reinterpret_cast<float*>(h8 + (static_cast<size_t>(rows) * inter + 255) / 256 * 256);
    rc = moe_expert_up_swiglu_fp8(x, x_scales, group_offsets, G, rows, d, inter, w13, w13_scales,
                                  h8, hs, stream);
    if (rc != MOE_OK) return rc;
    return moe_expert_down_fp8(h8, hs, group_offsets, G, rows, inter, d, w2, w2_scales, y, stream);
  }
  rc = moe_expert_up_swiglu(x, group_offsets, G, rows, d, inter, w13, workspace, stream);
  if (rc != MOE_OK) return rc;
  return moe_expert_down(workspace, group_offsets, G, rows, inter, d, w2, y, stream);
}

// ------------------------------------------------------------------ FP8 variant
int moe_quant_act_fp8(const void* x, int rows, int cols, void* q, float* scales,
                      moe_stream_t stream) {
  if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || !aligned4(scales))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((rows + 7) / 8, di->num_sms * 8));
  quant_act_fp8_kernel<<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, static_cast<uint8_t*>(q), scales);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_quant_weights_fp8(const void* w, int G, int R, int C, void* q, float* scales,
                          moe_stream_t stream) {
  if (G <= 0 || R <= 0 || C <= 0) return MOE_ERR_INVALID_ARG;
  if (R % 128 != 0 || C % 128 != 0 || G > 65535 || R / 128 > 65535)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!w || !q || !scales || !aligned16(w) || !aligned16(q) || !aligned4(scales))
    return MOE_ERR_INVALID_ARG;
  quant_weight_fp8_kernel<<<dim3(C / 128, R / 128, G), 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), R, C, static_cast<uint8_t*>(q), scales);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_permute_fp8(const void* u, const int32_t* topk_idx, const int32_t* expert_counts, int T,
                    int d, int n_routed, int top_k, void* x8, float* x_scales, void* u8,
                    float* u_scales, int32_t* expert_offsets, int32_t* pos, int32_t* src_token,
                    void* workspace, size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 256 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = as_stream(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (n_routed + 1), st));
    return MOE_OK;
  }
  if (!u || !topk_idx || !x8 || !x_scales || !pos || !src_token || !aligned16(u) ||
      !aligned16(x8) || !aligned4(x_scales))
    return MOE_ERR_INVALID_ARG;
  if ((u8 == nullptr) != (u_scales == nullptr) || (u8 && (!aligned16(u8) || !aligned4(u_scales))))
    return MOE_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < moe_permute_workspace_size(T, n_routed) || !aligned16(workspace))
    return MOE_ERR_WORKSPACE;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int chunks = (T + kPermChunk - 1) / kPermChunk;
  int32_t* hist = static_cast<int32_t*>(workspace);
  permute_hist_kernel<<<chunks, 256, 0, st>>>(topk_idx, T, top_k, n_routed, hist);
  MOE_CUDA(cudaGetLastError());
  permute_index_kernel<<<chunks, 256, 0, st>>>(topk_idx, expert_counts, hist, T, top_k, n_routed,
                                               expert_offsets, pos, src_token);
  MOE_CUDA(cudaGetLastError());
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  permute_quant_fp8_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(u), pos, T,
                                                   d, top_k, static_cast<uint8_t*>(x8), x_scales,
                                                   static_cast<uint8_t*>(u8), u_scales);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_expert_up_swiglu_fp8(const void* x8, const float* x_scales, const int32_t* group_offsets,
                             int G, int rows, int d, int inter, const void* w13,
                             const float* w13_scales, void* h8, float* h_scales,
                             moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!x8 || !x_scales || !group_offsets || !w13 || !w13_scales || !h8 || !h_scales ||
      !aligned16(x8) || !aligned16(w13) || !aligned16(h8) || !aligned4(x_scales) ||
      !aligned4(w13_scales) || !aligned4(h_scales))
    return MOE_ERR_INVALID_ARG;
  return launch_grouped_gemm_fp8<EPI8_SWIGLU_Q>(x8, x_scales, rows, d, w13, w13_scales, G,
                                                2 * inter, group_offsets, nullptr, inter,
                                                as_stream(stream), h8, h_scales);
}

int moe_pack_w13_fp8(const void* w13_stacked, int G, int inter, int d, void* w13,
                     moe_stream_t stream) {
  if (G <= 0 || inter <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (inter % 64 != 0 || d % 16 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!w13_stacked || !w13 || !aligned16(w13_stacked) || !aligned16(w13))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  pack_w13_fp8_kernel<<<di->num_sms * 4, 256, 0, as_stream(stream)>>>(
      static_cast<const uint8_t*>(w13_stacked), G, inter, d, static_cast<uint8_t*>(w13));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_expert_down_fp8(const void* h8, const float* h_scales, const int32_t* group_offsets, int G,
                        int rows, int inter, int d, const void* w2, const float* w2_scales, void* y,
                        moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!h8 || !h_scales || !group_offsets || !w2 || !w2_scales || !y || !aligned16(h8) ||
      !aligned16(w2) || !aligned16(y) || !aligned4(h_scales) || !aligned4(w2_scales))
    return MOE_ERR_INVALID_ARG;
  return launch_grouped_gemm_fp8<EPI8_STORE>(h8, h_scales, rows, inter, w2, w2_scales, G, d,
                                             group_offsets, y, d, as_stream(stream));
}

// ------------------------------------------------------------------ combine
int moe_combine(const void* y_perm, const int32_t* pos, const float* topk_gate,
                const void* shared_out, const void* residual, int T, int d, int top_k, void* out,
                moe_stream_t stream) {
  if (T < 0 || d <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!y_perm || !pos || !topk_gate || !out || !aligned16(y_perm) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if ((shared_out && !aligned16(shared_out)) || (residual && !aligned16(residual)))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  combine_kernel<false><<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(y_perm), pos, topk_gate,
      static_cast<const __nv_bfloat16*>(shared_out), static_cast<const __nv_bfloat16*>(residual),
      T, d, top_k, static_cast<__nv_bfloat16*>(out));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ fused scatter
int moe_slot_index(const int32_t* pos, int T, int top_k, int rows, int32_t* dst_slot,
                   moe_stream_t stream) {
  if (T < 0 || top_k <= 0 || rows < 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!dst_slot || (T > 0 && !pos)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  MOE_CUDA(cudaMemsetAsync(dst_slot, 0xFF, sizeof(int32_t) * rows, st));
  if (T == 0) return MOE_OK;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const long long pairs = static_cast<long long>(T) * top_k;
  const int blocks =
      static_cast<int>(std::max(1LL, std::min<long long>((pairs + 255) / 256, di->num_sms * 8)));
  slot_index_kernel<<<blocks, 256, 0, st>>>(pos, pairs, rows, dst_slot);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_expert_down_scatter(const void* h, const int32_t* group_offsets, int G, int rows,
                            int inter, int d, const void* w2, const int32_t* dst_slot,
                            const float* topk_gate, int T, int top_k, void* y_slots,
                            moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (T < 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!h || !group_offsets || !w2 || !dst_slot || !topk_gate || !y_slots || !aligned16(h) ||
      !aligned16(w2) || !aligned16(y_slots))
    return MOE_ERR_INVALID_ARG;
  const ScatterOut sc{dst_slot, topk_gate, T * top_k};
  if (use_pair_tiles(rows, G))
    return launch_grouped_gemm_pair<EPI_SCATTER>(h, rows, inter, w2, G, d, group_offsets,
                                                 y_slots, d, as_stream(stream), nullptr, 0,
                                                 nullptr, sc);
  return launch_grouped_gemm<256, EPI_SCATTER>(h, rows, inter, w2, G, d, group_offsets, y_slots,
                                               d, as_stream(stream), nullptr, sc);
}

size_t moe_expert_down_scatter_combine_workspace_size(int T, int d) {
  if (T <= 0 || d <= 0) return 16;
  const size_t bytes = static_cast<size_t>(T) * ((d + 127) / 128) * sizeof(int32_t);
  return (bytes + 255) / 256 * 256;
}

int moe_expert_down_scatter_combine(const void* h, const int32_t* group_offsets, int G, int rows,
                                    int inter, int d, const void* w2, const int32_t* dst_slot,
                                    const float* topk_gate, int T, int top_k, void* y_slots,
                                    const void* shared_out, const void* residual, void* out,
                                    void* workspace, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (T < 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || T == 0) return MOE_OK;
  if (!h || !group_offsets || !w2 || !dst_slot || !topk_gate || !y_slots || !out ||
      !aligned16(h) || !aligned16(w2) || !aligned16(y_slots) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if ((shared_out && !aligned16(shared_out)) || (residual && !aligned16(residual)))
    return MOE_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      ws_bytes < moe_expert_down_scatter_combine_workspace_size(T, d))
    return MOE_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  const int n_fb = d / 128;
  int32_t* cnt = static_cast<int32_t*>(workspace);
  MOE_CUDA(cudaMemsetAsync(cnt, 0, static_cast<size_t>(T) * n_fb * sizeof(int32_t), st));
  const ScatterOut sc{dst_slot,
                      topk_gate,
                      T * top_k,
                      cnt,
                      static_cast<const __nv_bfloat16*>(shared_out),
                      static_cast<const __nv_bfloat16*>(residual),
                      static_cast<__nv_bfloat16*>(out),
                      top_k,
                      n_fb};
  if (use_pair_tiles(rows, G))
    return launch_grouped_gemm_pair<EPI_SCATTER>(h, rows, inter, w2, G, d, group_offsets,
                                                 y_slots, d, st, nullptr, 0, nullptr, sc);
  return launch_grouped_gemm<256, EPI_SCATTER>(h, rows, inter, w2, G, d, group_offsets, y_slots,
                                               d, st, nullptr, sc);
}

int moe_combine_slots(const void* y_slots, const int32_t* pos, const void* shared_out,
                      const void* residual, int T, int d, int top_k, void* out,
                      moe_stream_t stream) {
  if (T < 0 || d <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!y_slots || !pos || !out || !aligned16(y_slots) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if ((shared_out && !aligned16(shared_out)) || (residual && !aligned16(residual)))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  combine_kernel<true><<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(y_slots), pos, nullptr,
      static_cast<const __nv_bfloat16*>(shared_out), static_cast<const __nv_bfloat16*>(residual),
      T, d, top_k, static_cast<__nv_bfloat16*>(out));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ expert parallelism
int moe_ep_plan(const int32_t* local_counts, const int32_t* recv_counts, int world, int n_local,
                long long recv_capacity, long long* send_splits, long long* recv_splits,
                int32_t* group_offsets, int32_t* regroup, int32_t* ungroup, long long* n_recv) {
  if (!local_counts || !recv_counts || !send_splits || !recv_splits || !group_offsets || !n_recv)
    return MOE_ERR_INVALID_ARG;
  if (world < 1 || n_local < 1 || static_cast<long long>(world) * n_local > (1LL << 24))
    return MOE_ERR_INVALID_ARG;
  if ((regroup || ungroup) && recv_capacity < 0) return MOE_ERR_INVALID_ARG;
  // validate and size first, so that nothing is written on error
  long long total = 0;
  for (long long i = 0; i < static_cast<long long>(world) * n_local; ++i) {
    if (recv_counts[i] < 0 || local_counts[i] < 0) return MOE_ERR_INVALID_ARG;
    total += recv_counts[i];
  }
  if (total > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((regroup || ungroup) && total > recv_capacity) return MOE_ERR_INVALID_ARG;
  const long long r = ep_plan_host(local_counts, recv_counts, world, n_local, recv_capacity,
                                   send_splits, recv_splits, group_offsets, regroup, ungroup);
  if (r < 0) return MOE_ERR_INVALID_ARG;
  *n_recv = r;
  return MOE_OK;
}

// ------------------------------------------------------------------ expert parallelism over peer memory
int moe_ep_plan_device(const int32_t* all_counts, int world, int n_local, int rank,
                       long long recv_capacity, const int32_t* add_counts, int32_t* dest_row,
                       int32_t* group_offsets, int32_t* global_counts, moe_stream_t stream) {
  if (world < 1 || n_local < 1 || rank < 0 || rank >= world || recv_capacity < 0)
    return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(world) * n_local > kRouteMaxExperts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!all_counts || !dest_row || !group_offsets || !global_counts) return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  ep_plan_device_kernel<<<1, 256, 0, as_stream(stream)>>>(all_counts, world, n_local, rank,
                                                          recv_capacity, add_counts, dest_row,
                                                          group_offsets, global_counts,
                                                          di->status);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_ep_dispatch_p2p(const void* u, const int32_t* topk_idx, const int32_t* pos,
                        const int32_t* expert_offsets, const int32_t* dest_row, int T, int d,
                        int n_routed, int top_k, int world, void* const* peer_x,
                        long long recv_capacity, moe_stream_t stream) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0 || world < 1 || recv_capacity < 0)
    return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 8 != 0 ||
      n_routed % world != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!u || !topk_idx || !pos || !expert_offsets || !dest_row || !peer_x || !aligned16(u))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  ep_dispatch_p2p_kernel<<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(u), topk_idx, pos, expert_offsets, dest_row, T, d, top_k,
      n_routed, n_routed / world, reinterpret_cast<__nv_bfloat16* const*>(peer_x),
      recv_capacity);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_ep_combine_p2p(const void* const* peer_y, const int32_t* topk_idx, const int32_t* pos,
                       const int32_t* expert_offsets, const int32_t* dest_row,
                       const float* topk_gate, const void* shared_out, const void* residual,
                       int T, int d, int n_routed, int top_k, int world, long long recv_capacity,
                       void* out, moe_stream_t stream) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0 || world < 1 || recv_capacity < 0)
    return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 8 != 0 ||
      n_routed % world != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!peer_y || !topk_idx || !pos || !expert_offsets || !dest_row || !topk_gate || !out ||
      !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if ((shared_out && !aligned16(shared_out)) || (residual && !aligned16(residual)))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  ep_combine_p2p_kernel<<<blocks, 256, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16* const*>(peer_y), topk_idx, pos, expert_offsets,
      dest_row, topk_gate, static_cast<const __nv_bfloat16*>(shared_out),
      static_cast<const __nv_bfloat16*>(residual), T, d, top_k, n_routed, n_routed / world,
      recv_capacity, static_cast<__nv_bfloat16*>(out));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_ipc_get_handle(const void* dev_ptr, void* handle, long long* offset) {
  if (!dev_ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
  static PFN_cuMemGetAddressRange_v3020 range = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  });
  if (!range) return cuda_fail(cudaErrorNotSupported);
  CUdeviceptr base = 0;
  size_t size = 0;
  const CUresult r = range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr));
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return MOE_ERR_CUDA;
  }
  cudaIpcMemHandle_t h;
  MOE_CUDA(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)));
  std::memcpy(handle, &h, sizeof(h));
  *offset = static_cast<long long>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return MOE_OK;
}

int moe_ipc_open_handle(const void* handle, void** base) {
  if (!handle || !base) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  MOE_CUDA(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess));
  return MOE_OK;
}

int moe_ipc_close_handle(void* base) {
  if (!base) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(cudaIpcCloseMemHandle(base));
  return MOE_OK;
}

int moe_gather_rows(const void* src, int n_src, const int32_t* index, int n, int d, void* dst,
                    moe_stream_t stream) {
  if (n < 0 || n_src < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (n == 0) return MOE_OK;
  if (!src || !index || !dst || !aligned16(src) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  const int blocks = std::max(1, std::min((n + 7) / 8, di->num_sms * 8));
  gather_rows_kernel<<<blocks, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(src), n_src, index, n, d,
      static_cast<__nv_bfloat16*>(dst));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ bias update
int moe_bias_update(const int32_t* expert_counts, float* bias, int n_routed, long long T,
                    int top_k, float gamma, moe_stream_t stream) {
  if (!expert_counts || !bias || n_routed <= 0 || T < 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (!(gamma == gamma)) return MOE_ERR_INVALID_ARG;
  bias_update_kernel<<<(n_routed + 255) / 256, 256, 0, as_stream(stream)>>>(
      expert_counts, bias, n_routed, T * top_k, gamma);
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ backward
int moe_expert_up_swiglu_train(const void* x, const int32_t* group_offsets, int G, int rows,
                               int d, int inter, const void* w13, void* h, void* ac,
                               moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!x || !group_offsets || !w13 || !h || !ac || !aligned16(x) || !aligned16(w13) ||
      !aligned16(h) || !aligned16(ac))
    return MOE_ERR_INVALID_ARG;
  if (use_pair_tiles(rows, G))
    return launch_grouped_gemm_pair<EPI_SWIGLU>(x, rows, d, w13, G, 2 * inter, group_offsets, h,
                                                inter, as_stream(stream), nullptr, 0, ac);
  return launch_grouped_gemm<256, EPI_SWIGLU>(x, rows, d, w13, G, 2 * inter, group_offsets, h,
                                              inter, as_stream(stream), ac);
}

int moe_combine_backward(const void* dout, const void* y_perm, const int32_t* pos,
                         const float* topk_gate, int T, int d, int top_k, void* dy_perm,
                         float* dgate, moe_stream_t stream) {
  if (T < 0 || d <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!dout || !y_perm || !pos || !topk_gate || !dy_perm || !dgate || !aligned16(dout) ||
      !aligned16(y_perm) || !aligned16(dy_perm))
    return MOE_ERR_INVALID_ARG;
  const int blocks = (T + kBwdTokensPerBlock - 1) / kBwdTokensPerBlock;
  const auto* o = static_cast<const __nv_bfloat16*>(dout);
  const auto* y = static_cast<const __nv_bfloat16*>(y_perm);
  auto* dy = static_cast<__nv_bfloat16*>(dy_perm);
  cudaStream_t st = as_stream(stream);
#define MOE_CB_CASE(KK)                                                                       \
  case KK:                                                                                    \
    combine_backward_kernel<KK><<<blocks, 32 * kBwdTokensPerBlock, 0, st>>>(o, y, pos,        \
                                                                           topk_gate, T, d,   \
                                                                           dy, dgate);        \
    break;
  switch (top_k) {
    MOE_CB_CASE(1) MOE_CB_CASE(2) MOE_CB_CASE(3) MOE_CB_CASE(4)
    MOE_CB_CASE(5) MOE_CB_CASE(6) MOE_CB_CASE(7) MOE_CB_CASE(8)
    default: return MOE_ERR_UNSUPPORTED_SHAPE;
  }
#undef MOE_CB_CASE
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_expert_down_backward(const void* dy, const void* ac, const int32_t* group_offsets, int G,
                             int rows, int d, int inter, const void* w2, void* dac,
                             moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!dy || !ac || !group_offsets || !w2 || !dac || !aligned16(dy) || !aligned16(ac) ||
      !aligned16(w2) || !aligned16(dac))
    return MOE_ERR_INVALID_ARG;
  return launch_dgrad<EPI_DG_SWIGLU_BWD>(dy, rows, d, w2, G, inter, group_offsets, dac,
                                         2 * inter, ac, as_stream(stream));
}

int moe_expert_up_backward(const void* dac, const int32_t* group_offsets, int G, int rows, int d,
                           int inter, const void* w13, void* dx, moe_stream_t stream) {
  int rc = check_ffn_shape(G, rows, d, inter);
  if (rc != MOE_OK) return rc;
  if (rows == 0) return MOE_OK;
  if (!dac || !group_offsets || !w13 || !dx || !aligned16(dac) || !aligned16(w13) ||
      !aligned16(dx))
    return MOE_ERR_INVALID_ARG;
  return launch_dgrad<EPI_DG_STORE>(dac, rows, 2 * inter, w13, G, d, group_offsets, dx, d,
                                    nullptr, as_stream(stream));
}

int moe_expert_wgrad(const void* a, const void* b, const int32_t* group_offsets, int G, int rows,
                     int m, int n, void* dw, moe_stream_t stream) {
  if (G < 1 || rows < 0 || m <= 0 || n <= 0) return MOE_ERR_INVALID_ARG;
  if (G > kMaxGroups || m % 128 != 0 || n % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!group_offsets || !dw || !aligned16(dw)) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && (!a || !b || !aligned16(a) || !aligned16(b))) return MOE_ERR_INVALID_ARG;
  if (rows == 0) {
    MOE_CUDA(cudaMemsetAsync(dw, 0, static_cast<size_t>(G) * m * n * 2, as_stream(stream)));
    return MOE_OK;
  }
  return launch_wgrad(a, b, rows, m, n, G, group_offsets, dw, as_stream(stream));
}

int moe_gate_backward(const void* u, const void* centroids, const int32_t* topk_idx,
                      const float* topk_gate, const float* dgate, const int32_t* pos, int T,
                      int d, int n_routed, int top_k, moe_gate_kind kind, float routed_scale,
                      float* dz, float* dz_perm, moe_stream_t stream) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (kind != MOE_GATE_SIGMOID_BIAS && kind != MOE_GATE_SOFTMAX_TOPK) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!(routed_scale == routed_scale) || routed_scale == 0.0f) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!u || !centroids || !topk_idx || !topk_gate || !dgate || !pos || !dz || !dz_perm ||
      !aligned16(u) || !aligned16(centroids))
    return MOE_ERR_INVALID_ARG;
  const int blocks = (T + kBwdTokensPerBlock - 1) / kBwdTokensPerBlock;
  const auto* uu = static_cast<const __nv_bfloat16*>(u);
  const auto* ee = static_cast<const __nv_bfloat16*>(centroids);
  cudaStream_t st = as_stream(stream);
#define MOE_GB_CASE(KK)                                                                        \
  case KK:                                                                                     \
    if (kind == MOE_GATE_SIGMOID_BIAS)                                                         \
      gate_backward_kernel<KK, 0><<<blocks, 32 * kBwdTokensPerBlock, 0, st>>>(                 \
          uu, ee, topk_idx, topk_gate, dgate, pos, T, d, routed_scale, dz, dz_perm);           \
    else                                                                                       \
      gate_backward_kernel<KK, 1><<<blocks, 32 * kBwdTokensPerBlock, 0, st>>>(                 \
          uu, ee, topk_idx, topk_gate, dgate, pos, T, d, routed_scale, dz, dz_perm);           \
    break;
  switch (top_k) {
    MOE_GB_CASE(1) MOE_GB_CASE(2) MOE_GB_CASE(3) MOE_GB_CASE(4)
    MOE_GB_CASE(5) MOE_GB_CASE(6) MOE_GB_CASE(7) MOE_GB_CASE(8)
    default: return MOE_ERR_UNSUPPORTED_SHAPE;
  }
#undef MOE_GB_CASE
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

int moe_combine_dx(const void* dout, const void* dx_perm, const int32_t* pos,
                   const void* dx_shared, const float* dz, const int32_t* topk_idx,
                   const void* centroids, int T, int d, int top_k, void* du,
                   moe_stream_t stream) {
  if (T < 0 || d <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return MOE_OK;
  if (!dx_perm || !pos || !dz || !topk_idx || !centroids || !du || !aligned16(dx_perm) ||
      !aligned16(centroids) || !aligned16(du))
    return MOE_ERR_INVALID_ARG;
  if ((dout && !aligned16(dout)) || (dx_shared && !aligned16(dx_shared)))
    return MOE_ERR_INVALID_ARG;
  const int blocks = (T + kBwdTokensPerBlock - 1) / kBwdTokensPerBlock;
  const auto* o = static_cast<const __nv_bfloat16*>(dout);
  const auto* dxp = static_cast<const __nv_bfloat16*>(dx_perm);
  const auto* dxs = static_cast<const __nv_bfloat16*>(dx_shared);
  const auto* ee = static_cast<const __nv_bfloat16*>(centroids);
  auto* out = static_cast<__nv_bfloat16*>(du);
  cudaStream_t st = as_stream(stream);
#define MOE_DX_CASE(KK)                                                                        \
  case KK:                                                                                     \
    combine_dx_kernel<KK><<<blocks, 32 * kBwdTokensPerBlock, 0, st>>>(o, dxp, pos, dxs, dz,    \
                                                                      topk_idx, ee, T, d, out); \
    break;
  switch (top_k) {
    MOE_DX_CASE(1) MOE_DX_CASE(2) MOE_DX_CASE(3) MOE_DX_CASE(4)
    MOE_DX_CASE(5) MOE_DX_CASE(6) MOE_DX_CASE(7) MOE_DX_CASE(8)
    default: return MOE_ERR_UNSUPPORTED_SHAPE;
  }
#undef MOE_DX_CASE
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

size_t moe_centroid_grad_workspace_size(int rows, int n_routed, int d) {
  if (rows < 0 || n_routed <= 0 || d <= 0) return 256;
  const long long chunks = centroid_max_chunks(rows, n_routed);
  const size_t a = (static_cast<size_t>(n_routed + 1) * 4 + 15) / 16 * 16;
  const size_t b = (static_cast<size_t>(chunks) * 8 + 15) / 16 * 16;
  return a + b + static_cast<size_t>(chunks) * d * 4;
}

int moe_centroid_grad(const void* x_perm, const float* dz_perm, const int32_t* expert_offsets,
                      int n_routed, int rows, int d, void* de, void* workspace, size_t ws_bytes,
                      moe_stream_t stream) {
  if (n_routed <= 0 || rows < 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0 || n_routed >= kCentroidMaxExperts || (d + kCentroidCols - 1) / kCentroidCols > 65535)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!expert_offsets || !de || !aligned16(de)) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && (!x_perm || !dz_perm || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < moe_centroid_grad_workspace_size(rows, n_routed, d) ||
      !aligned16(workspace))
    return MOE_ERR_WORKSPACE;
  const long long chunks = centroid_max_chunks(rows, n_routed);
  if (chunks > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* chunk_start = reinterpret_cast<int32_t*>(ws);
  int2* chunk_rows =
      reinterpret_cast<int2*>(ws + (static_cast<size_t>(n_routed + 1) * 4 + 15) / 16 * 16);
  float* partials = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(chunk_rows) +
                                             (static_cast<size_t>(chunks) * 8 + 15) / 16 * 16);
  cudaStream_t st = as_stream(stream);
  const int ncb = (d + kCentroidCols - 1) / kCentroidCols;
  centroid_chunk_table_kernel<<<1, kCentroidMaxExperts, 0, st>>>(expert_offsets, n_routed, rows,
                                                                  chunk_start, chunk_rows);
  MOE_CUDA(cudaGetLastError());
  centroid_partial_kernel<<<dim3(static_cast<unsigned>(chunks), ncb), 32 * kCentroidWarps, 0,
                            st>>>(static_cast<const __nv_bfloat16*>(x_perm), dz_perm, chunk_start,
                                  chunk_rows, n_routed, d, partials);
  MOE_CUDA(cudaGetLastError());
  centroid_reduce_kernel<<<dim3(n_routed, ncb), kCentroidCols, 0, st>>>(
      chunk_start, partials, d, static_cast<__nv_bfloat16*>(de));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

// ------------------------------------------------------------------ helpers
int moe_pack_w13(const void* w1, const void* w3, int G, int inter, int d, void* w13,
                 moe_stream_t stream) {
  if (G <= 0 || inter <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (inter % 128 != 0 || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!w1 || !w3 || !w13 || !aligned16(w1) || !aligned16(w3) || !aligned16(w13))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc != MOE_OK) return rc;
  pack_w13_kernel<<<di->num_sms * 4, 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(w1), static_cast<const __nv_bfloat16*>(w3), G, inter, d,
      static_cast<__nv_bfloat16*>(w13));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ permute, allocation-free
// moe_permute without a workspace argument, for callers that cannot allocate
// device memory at the call site. Its scratch (the per-chunk expert
// histograms of the dispatch's first pass) lives in this file-scope device
// array instead: every GPU that loads the library holds it until the process
// exits, and every call shares it.
namespace {

constexpr int kNoAllocScratchInts = 65536;   // 256 KiB: ceil(T/128) * n_routed <= 65536
__device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

// device address of the array, per device; published with release order
// after the lookup, read with acquire order
std::atomic<int32_t*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_permute_scratch on the current device. In host code the
// array's name is only a stand-in for the symbol, never a device address: the
// address is looked up once per device with that device current.
int scratch_address(int32_t** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_INVALID_ARG;
  int32_t* ptr = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ptr = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!ptr) {
      void* p = nullptr;
      MOE_CUDA(cudaGetSymbolAddress(&p, g_permute_scratch));
      ptr = static_cast<int32_t*>(p);
      g_scratch_ptr[dev].store(ptr, std::memory_order_release);
    }
  }
  *out = ptr;
  return MOE_OK;
}

}  // namespace

extern "C" int moe_permute_noalloc(const void* u, const int32_t* topk_idx,
                                   const int32_t* expert_counts, int T, int d, int n_routed,
                                   int top_k, void* x_perm, int32_t* expert_offsets,
                                   int32_t* pos, int32_t* src_token, moe_stream_t stream) {
  if (T < 0 || d <= 0 || n_routed <= 0 || top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
  if (top_k > kMaxTopK || top_k > n_routed || n_routed > kRouteMaxExperts || d % 256 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(T) * top_k > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  const long long chunks = (static_cast<long long>(T) + kPermChunk - 1) / kPermChunk;
  if (chunks * n_routed > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T > 0 && (!u || !topk_idx || !x_perm || !pos || !src_token || !aligned16(u) ||
                !aligned16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  int32_t* hist = nullptr;
  int rc = scratch_address(&hist);
  if (rc != MOE_OK) return rc;
  cudaStream_t st = as_stream(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (n_routed + 1), st));
    return MOE_OK;
  }
  DeviceInfo* di;
  if ((rc = device_info(&di)) != MOE_OK) return rc;
  // Pass 1 overwrites every histogram entry pass 2 reads, so the array needs
  // no clearing between calls.
  const int nch = static_cast<int>(chunks);
  permute_hist_kernel<<<nch, 256, 0, st>>>(topk_idx, T, top_k, n_routed, hist);
  MOE_CUDA(cudaGetLastError());
  permute_index_kernel<<<nch, 256, 0, st>>>(topk_idx, expert_counts, hist, T, top_k, n_routed,
                                            expert_offsets, pos, src_token);
  MOE_CUDA(cudaGetLastError());
  const int blocks = std::max(1, std::min((T + 7) / 8, di->num_sms * 8));
  permute_copy_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(u), pos, T, d,
                                              top_k, static_cast<__nv_bfloat16*>(x_perm));
  MOE_CUDA(cudaGetLastError());
  return MOE_OK;
}
