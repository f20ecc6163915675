// Pieces shared by the bf16 tensor-core kernels: RoPE angles, host-side TMA
// descriptor encoding.
#pragma once
#include <cudaTypedefs.h>

#include <cstdint>

#include <cuda_runtime.h>

namespace la {

constexpr float kLog2e = 1.4426950408889634f;

constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }

// RoPE frequencies theta_i = base^(-2i/d), formed in fp64 on the host
struct RopeTheta {
  double theta[64];
  float thetaf[64];   // the same, rounded to fp32 (small in-tile angles)
};

// (cos, sin) of t * theta, the angle formed and reduced modulo 2 pi in fp64
__device__ __forceinline__ float2 rope_cs_exact(int64_t t, double theta) {
  const double two_pi = 6.283185307179586476925286766559;
  const double ang = (double)t * theta;
  const float red = (float)fma(-two_pi, rint(ang * 0.15915494309189533577), ang);
  float s, c;
  sincosf(red, &s, &c);
  return make_float2(c, s);
}

// (cos, sin) of a small angle (|ang| < ~200 rad): Cody-Waite reduction with a
// two-constant split of 2 pi, then the SFU (about 2^-21 absolute on [-pi, pi])
__device__ __forceinline__ float2 sincos_small(float ang) {
  const float k = rintf(ang * 0.15915494309189535f);
  float red = fmaf(-k, 6.28318548202514648f, ang);
  red = fmaf(-k, -1.7484556000744083e-07f, red);
  float s, c;
  __sincosf(red, &s, &c);
  return make_float2(c, s);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda)
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// the TMA swizzle whose span equals a box row of row_bytes (32, 64 or >= 128)
inline CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

}  // namespace la
