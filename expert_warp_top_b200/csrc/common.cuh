// common.cuh -- shared device helpers of the MoE layer library (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace moe {

// Bits of the device error flag.
constexpr unsigned kErrIndex = 1u;    // an index was out of range
constexpr unsigned kErrTimeout = 2u;  // a bounded wait expired

// The flag itself lives in api.cu; kernels receive its address.
struct DevErr {
  unsigned* flag;
};

__device__ __forceinline__ void raise_error(unsigned* flag, unsigned bits) {
  atomicOr(flag, bits);
}

template <typename T>
struct DType;
template <>
struct DType<__nv_bfloat16> {
  static constexpr int bytes = 2;
};
template <>
struct DType<float> {
  static constexpr int bytes = 4;
};

// ---------------------------------------------------------------------------
// 16-byte vector helpers: 8 bf16 or 4 f32 values <-> fp32 lanes.
// ---------------------------------------------------------------------------
template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p = __bfloat1622float2(h[i]);
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  __device__ __forceinline__ static uint4 from_f32(const float* f) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
  }
};

template <>
struct Vec16<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void to_f32(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 from_f32(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  *reinterpret_cast<uint4*>(p) = v;
}

__device__ __forceinline__ unsigned lane_id() { return threadIdx.x & 31u; }

// Programmatic dependent launch.  Every kernel of the library is launched so
// that the next kernel on the stream may be scheduled before this one ends;
// each kernel therefore waits for its predecessors (and for their memory
// operations to be visible) before it touches global memory, and then lets
// its own dependents be scheduled.  Both are no-ops without the launch
// attribute.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

}  // namespace moe
