// la_tc_sync.cuh -- the pieces the warp-specialised tensor-core kernels share:
// bounded mbarrier waits that record a timeout in a device error word instead
// of hanging, and the bf16 pack / unpack and exponential helpers of their
// CUDA-core steps.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "la_sm100.cuh"

namespace la {
namespace tcsync {

constexpr long long kTimeoutCycles = 4000000000LL;  // about two seconds
constexpr uint32_t kSuspendHintNs = 20000;

// The CTA's barriers, its abort flag (shared memory) and the kernel's device
// error words: err receives 1 when a wait timed out and 2 when draining did;
// where keeps the first failure as 0x80000000 | chunk << 8 | barrier index.
struct Sync {
  uint64_t *bar;
  volatile int *abort;
  unsigned int *err;
  unsigned int *where;
};

// Waiting threads sleep in the barrier (suspend hint) instead of polling, so
// they leave issue slots to the warps that share their SM sub-partition.
__device__ __forceinline__ bool wait_bar(const Sync &sy, int idx, uint32_t parity, int chunk = 0) {
  uint64_t *b = sy.bar + idx;
  if (sm100::mbar_test(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (sm100::mbar_wait_hint(b, parity, kSuspendHintNs)) return true;
    if (*sy.abort) return false;
    if (clock64() - t0 > kTimeoutCycles) {
      *sy.abort = 1;
      atomicOr(sy.err, 1u);
      atomicCAS(sy.where, 0u, 0x80000000u | ((uint32_t)(chunk & 0x7FFFFF) << 8) | (uint32_t)idx);
      return false;
    }
  }
}

// Warp-uniform wait for warps that go on to execute warp-collective or
// .sync.aligned instructions: every lane takes the same path even on abort.
__device__ __forceinline__ bool wait_bar_warp(const Sync &sy, int idx, uint32_t parity, int chunk = 0) {
  return __all_sync(0xffffffffu, wait_bar(sy, idx, parity, chunk));
}

// Wait that ignores the abort flag (used to drain asynchronous arrivals).
__device__ __forceinline__ void drain_bar(const Sync &sy, int idx, uint32_t parity) {
  uint64_t *b = sy.bar + idx;
  const long long t0 = clock64();
  while (!sm100::mbar_test(b, parity)) {
    if (clock64() - t0 > kTimeoutCycles) {
      atomicOr(sy.err, 2u);
      return;
    }
  }
}

// e^x on the PTX ex2.approx.ftz instruction (2^(x log2 e)): one multiply and
// one special-function op, relative error ~2^-22, far below the bf16 rounding
// the factors meet next.  Used for decay factors (x <= 0).
__device__ __forceinline__ float exp_fast(float x) {
  constexpr float kLog2e = 1.4426950408889634f;
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x * kLog2e));
  return e;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

}  // namespace tcsync
}  // namespace la
