// ssm_common.cuh -- device helpers shared by the scan, SS2D and decode kernels.
//
// Transcendentals go to the SFU through the PTX approximate instructions
// (ex2 / lg2 / rcp); everything the method adds on top of them (the softplus
// of delta, the SiLU gate) is written here from its definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------- SFU calls
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

// -------------------------------------------------------------- softplus
// delta = softplus(x) with torch's threshold: x for x > 20, else
// log(1 + e^x).  With e = 2^(x log2 e):
//   e <  1/16 : log1p(e) by its alternating series to e^5 (truncation
//               below e^6/6, i.e. < 2e-7 of the result);
//   e >= 1/16 : ln2 * log2(1 + e) on the SFU (1 + e is then far enough
//               from 1 that its rounding costs < 1e-6 relative).
__device__ __forceinline__ float softplus_f32(float x) {
  const float e = ex2_approx(x * kLog2e);
  const float series =
      e * fmaf(e, fmaf(e, fmaf(e, fmaf(e, 0.2f, -0.25f), 1.0f / 3.0f), -0.5f), 1.0f);
  const float via_log = kLn2 * lg2_approx(1.0f + e);
  const float r = e < 0.0625f ? series : via_log;
  return x > 20.0f ? x : r;
}

// SiLU gate: z * sigmoid(z) = z / (1 + e^-z).
__device__ __forceinline__ float silu_f32(float z) {
  return z * rcp_approx(1.0f + ex2_approx(-z * kLog2e));
}

// ------------------------------------------------------- element access
template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ __forceinline__ static float load(const float *p, int64_t i) { return p[i]; }
  __device__ __forceinline__ static void store(float *p, int64_t i, float v) { p[i] = v; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ __forceinline__ static float load(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16 *p, int64_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
  }
};

// bf16 pair packed in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// --------------------------------------------------------- async copies
// 16-byte global -> shared copy; src_bytes < 16 zero-fills the rest.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace ssm
