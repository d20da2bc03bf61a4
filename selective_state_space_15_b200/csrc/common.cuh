// Device helpers shared by the selective-scan kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// MUFU approximations (PTX ISA: ex2/lg2/rcp .approx).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(x) = log(1 + e^x).
// Precise form (float32 inputs): CUDA's expf/log1pf; x > 20 returns x (the remainder
// log1p(e^-x) < 2.1e-9 is below float32 resolution relative to x).
__device__ __forceinline__ float softplus_precise(float x) {
  return x > 20.f ? x : log1pf(expf(x));
}
// Fast form (bf16 inputs): w = e^x through ex2; log1p(w) from the alternating series
// w - w^2/2 + ... + w^7/7 when w < 1/8 (truncation error below w^8/8, i.e. relative
// error < 3e-7), else ln2 * log2(1 + w) through lg2, whose absolute error (~1e-7) is small
// against a result of at least log(1.125) = 0.118 there.
__device__ __forceinline__ float softplus_fast(float x) {
  if (x > 15.f) return x;
  const float w = ex2_approx(x * kLog2e);
  if (w < 0.125f) {
    float p = fmaf(w, -1.f / 7.f, 1.f / 6.f);
    p = fmaf(w, p, -1.f / 5.f);
    p = fmaf(w, p, 1.f / 4.f);
    p = fmaf(w, p, -1.f / 3.f);
    p = fmaf(w, p, 1.f / 2.f);
    // log1p(w) = w - w^2 (1/2 - w/3 + w^2/4 - ...) = w * (1 - w * p)
    p = fmaf(-w, p, 1.f);
    return w * p;
  }
  return kLn2 * lg2_approx(1.f + w);
}

// silu(z) = z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu_precise(float z) { return z / (1.f + expf(-z)); }
__device__ __forceinline__ float silu_fast(float z) { return z * rcp_approx(1.f + ex2_approx(-z * kLog2e)); }

template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static float to_f32(float v) { return v; }
  __device__ __forceinline__ static float from_f32(float v) { return v; }
  static constexpr bool kFast = false;
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
  static constexpr bool kFast = true;
};

template <bool kFast> __device__ __forceinline__ float softplus_t(float x) {
  return kFast ? softplus_fast(x) : softplus_precise(x);
}
template <bool kFast> __device__ __forceinline__ float silu_t(float z) {
  return kFast ? silu_fast(z) : silu_precise(z);
}

// 16-byte global->shared asynchronous copy; `src_bytes` < 16 zero-fills the remainder
// (src_bytes == 0 reads nothing).
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gmem_src, int src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Device status word (read and cleared by ssm_get_device_status on the host).  The library
// is a single translation unit, so this is the only definition.
__device__ int g_status = 0;
__device__ __forceinline__ void report_status(int code) { atomicCAS(&g_status, 0, code); }

}  // namespace ssm
