// common.cuh -- device helpers shared by the CSA2 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa2.h"

namespace csa2 {

constexpr int kBlockEntries = 64;   // entries sharing one E4M3 scale per channel
constexpr int kHeadDim = 512;       // main-KV head dimension the attention kernels are built for

// Record the first device-side data error; later errors leave it unchanged.
__device__ __forceinline__ void record_error(int* err, int code) {
  if (err != nullptr && *(volatile int*)err == 0) atomicCAS(err, 0, code);
}

// Two E4M3 bytes (low byte = first value) -> two halves, exact.
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint16_t v) {
  __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  return *reinterpret_cast<__half2*>(&r);
}

// Two E2M1 nibbles (low nibble = first value) -> two halves, exact.
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint8_t v) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)v, __NV_E2M1);
  return *reinterpret_cast<__half2*>(&r);
}

// Order-preserving key: larger score -> larger key; -0 maps like +0. NaN is
// reported through `nan` and ranked below every number.
__device__ __forceinline__ uint32_t rank_key(float f, bool& nan) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) { nan = true; return 0u; }
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch: a kernel launched with the programmatic stream
// serialisation attribute may start while the previous kernel of the stream is
// still running. It waits here before touching global memory that kernel may
// write or read, then lets its own dependents start (which therefore never
// overlap the kernel before it). Without the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait_and_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace csa2
