// Dynamic tile order inside one CTA: the producer takes the next tile index
// from a global counter (zeroed before the launch) and publishes it through a
// ring of kCtaTileQ slots in shared memory to the CTA's other roles (the MMA
// thread and the epilogue warps), which walk the same tiles in the same
// order. Persistent CTAs then take tiles in index order, so CTAs that share
// an operand tile stay close in time (it is still in L2), and tiles of
// different cost do not pile up on some CTAs. All waits bounded.
#pragma once
#include "ptx.cuh"

namespace moe {

constexpr int kCtaTileQ = 4;

// Producer: wait until slot i % kCtaTileQ is free, then publish t.
__device__ __forceinline__ bool cta_tile_push(int i, int t, int* tq, uint64_t* tq_full,
                                              uint64_t* tq_empty, unsigned int* status) {
  const int j = i & (kCtaTileQ - 1);
  if (!mbar_wait(&tq_empty[j], ((i / kCtaTileQ) & 1) ^ 1u, status, kStatusTimeoutProducer))
    return false;
  *reinterpret_cast<volatile int*>(&tq[j]) = t;
  mbar_arrive(&tq_full[j]);
  return true;
}

// Consumer (one thread): the i-th published tile index.
__device__ __forceinline__ bool cta_tile_pop(int i, const int* tq, uint64_t* tq_full,
                                             uint64_t* tq_empty, int& t, unsigned int* status,
                                             unsigned int code) {
  const int j = i & (kCtaTileQ - 1);
  if (!mbar_wait(&tq_full[j], (i / kCtaTileQ) & 1, status, code)) return false;
  t = *reinterpret_cast<const volatile int*>(&tq[j]);
  mbar_arrive(&tq_empty[j]);
  return true;
}

}  // namespace moe
