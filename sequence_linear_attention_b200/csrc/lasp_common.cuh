// Device-side helpers shared by every kernel of the library: the device status
// word, bounded waits, decay powers and element conversion.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lasp.h"
#include "kernels.h"

namespace lasp {

// The library is compiled as one translation unit (lasp_lib.cu), so these
// per-device variables are defined here, once.
// First error seen by any kernel on this device: (code << 16) | site.
// lasp_check_device_status() reads and clears it.
__device__ unsigned int g_device_status = 0;
// Wall-clock limit, in nanoseconds, for any spin-wait inside a kernel.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

// Error sites recorded with the status code (low 16 bits of the status word).
enum Site : unsigned int {
  SITE_NONE = 0,
  SITE_DECAY = 1,        // a decay value outside (0, 1]
  SITE_PROBE = 2,        // the wait-timeout probe kernel
  SITE_STATES_TMA = 10,  // chunk-state kernel, waiting for a TMA tile
  SITE_STATES_MMA = 11,  // chunk-state kernel, waiting for the MMA
  SITE_OUT_TMA = 20,
  SITE_OUT_MMA = 21,
  SITE_BWD_TMA = 30,
  SITE_BWD_MMA = 31,
  SITE_GATE_RANGE = 40,  // gated form: a chunk's log-gates span more than the factorized form takes
};

__device__ __forceinline__ void record_error(int code, unsigned int site) {
  atomicCAS(&g_device_status, 0u, ((unsigned int)code << 16) | (site & 0xFFFFu));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// lambda_h in (0, 1]; NULL means 1. An invalid value is recorded and replaced
// by 1 so that the kernel still terminates normally.
__device__ __forceinline__ float load_decay(const float* decay, int h) {
  if (decay == nullptr) return 1.0f;
  float l = decay[h];
  if (!(l > 0.0f && l <= 1.0f)) {
    record_error(LASP_ERR_INVALID_ARG, SITE_DECAY);
    return 1.0f;
  }
  return l;
}

// lambda^n as exp2(n * log2(lambda)); exact 1 for lambda = 1 and for n = 0.
__device__ __forceinline__ float decay_pow(float log2_lambda, float n) {
  return exp2f(n * log2_lambda);
}

// Whether a kernel given `c` (kernels.h) does its work.
__device__ __forceinline__ bool runs(RunIf c) {
  return c.flag == nullptr || ((*reinterpret_cast<const volatile int*>(c.flag) != 0) == (c.want != 0));
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

}  // namespace lasp
