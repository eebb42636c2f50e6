// ssm_common.cuh -- device helpers shared by the scan, SS2D and decode kernels.
//
// Transcendentals go to the SFU through the PTX approximate instructions
// (ex2 / lg2 / rcp); everything the method adds on top of them (the softplus
// of delta, the SiLU gate) is written here from its definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#ifdef SSM_DEBUG_BOUNDS
// Error word of the debug-bounds build: every checked global access whose
// index falls outside its buffer ORs its buffer-kind bit in here (and is
// skipped); read and cleared by ssm_check_device_errors.
__device__ unsigned int g_ssm_bounds_word = 0;
#endif

namespace ssm {

// Buffer kinds of the debug-bounds checks (bits of the error word).
enum BoundsKind : unsigned {
  kBndAct = 1u << 0,      // (b, L, d_in) / (b, d_in) activations and their gradients
  kBndBC = 1u << 1,       // B, C and their gradients
  kBndParam = 1u << 2,    // A, D, dt_bias (and dA, dD, ddt_bias)
  kBndState = 1u << 3,    // h0, h_last, the decode state, dh_last, dh0
  kBndChunk = 1u << 4,    // saved chunk states, split-scan block maps
  kBndWork = 1u << 5,     // SS2D accumulator workspace, conv window
  kBndSelfTest = 1u << 31 // the library's own check of the mechanism
};

// True when 0 <= i < n.  The debug-bounds build (SSM_DEBUG_BOUNDS) checks
// and records a miss in the error word; other builds compile this to true.
__device__ __forceinline__ bool in_bounds(int64_t i, int64_t n, unsigned kind) {
#ifdef SSM_DEBUG_BOUNDS
  if (i >= 0 && i < n) return true;
  atomicOr(&g_ssm_bounds_word, kind);
  return false;
#else
  (void)i; (void)n; (void)kind;
  return true;
#endif
}

constexpr float kLog2e = 1.4426950408889634f;
// Steps between the saved chunk-start states the backward scan works from.
constexpr int kStateChunk = 16;
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

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// -------------------------------------------------------------- softplus
// delta = softplus(x) = max(x, 0) + log1p(e) with e = exp(-|x|) in (0, 1]:
// one SFU exp2, then log1p(e) = e s(e) with s the degree-7 minimax fit of
// log1p(e) / e on [0, 1] made by fit_polys.py (relative error 2.2e-7), so
// the result keeps its relative accuracy where softplus(x) ~ e^x.  For
// x > 20 this returns x exactly (e s(e) < 2.1e-9 vanishes in the sum), which
// is torch's thresholded softplus.
constexpr float kLog1pS0 = 9.999998212e-01f;
constexpr float kLog1pS1 = -4.999740422e-01f;
constexpr float kLog1pS2 = 3.327547908e-01f;
constexpr float kLog1pS3 = -2.449546307e-01f;
constexpr float kLog1pS4 = 1.774524003e-01f;
constexpr float kLog1pS5 = -1.076816991e-01f;
constexpr float kLog1pS6 = 4.408961907e-02f;
constexpr float kLog1pS7 = -8.539204486e-03f;

__device__ __forceinline__ float softplus_f32(float x) {
  const float e = ex2_approx(-fabsf(x) * kLog2e);
  float s = fmaf(kLog1pS7, e, kLog1pS6);
  s = fmaf(s, e, kLog1pS5);
  s = fmaf(s, e, kLog1pS4);
  s = fmaf(s, e, kLog1pS3);
  s = fmaf(s, e, kLog1pS2);
  s = fmaf(s, e, kLog1pS1);
  s = fmaf(s, e, kLog1pS0);
  return fmaf(e, s, fmaxf(x, 0.0f));
}

// softplus of two values with packed fp32 arithmetic (same formula as above).
__device__ __forceinline__ float2 softplus2_f32(float2 x) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 e2 = __fmul2_rn(ax, make_float2(-kLog2e, -kLog2e));
  const float2 e = make_float2(ex2_approx(e2.x), ex2_approx(e2.y));
  float2 s = __ffma2_rn(make_float2(kLog1pS7, kLog1pS7), e, make_float2(kLog1pS6, kLog1pS6));
  s = __ffma2_rn(s, e, make_float2(kLog1pS5, kLog1pS5));
  s = __ffma2_rn(s, e, make_float2(kLog1pS4, kLog1pS4));
  s = __ffma2_rn(s, e, make_float2(kLog1pS3, kLog1pS3));
  s = __ffma2_rn(s, e, make_float2(kLog1pS2, kLog1pS2));
  s = __ffma2_rn(s, e, make_float2(kLog1pS1, kLog1pS1));
  s = __ffma2_rn(s, e, make_float2(kLog1pS0, kLog1pS0));
  return __ffma2_rn(e, s, make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)));
}

// SiLU gate: z * sigmoid(z) = z / (1 + e^-z) (SFU exp2 + reciprocal).
__device__ __forceinline__ float silu_f32(float z) {
  return z * rcp_approx(1.0f + ex2_approx(-z * kLog2e));
}

// SiLU through sigmoid(z) = (1 + tanh(z / 2)) / 2: one SFU op.  tanh.approx
// has a relative error near 2^-11, below the 2^-9 rounding of a bf16
// output, so bf16 paths use this form and fp32 paths the one above.
__device__ __forceinline__ float silu_fast(float z) {
  return z * fmaf(0.5f, tanh_approx(0.5f * z), 0.5f);
}

template <typename T> __device__ __forceinline__ float silu_for(float z) {
  if constexpr (sizeof(T) == 2)
    return silu_fast(z);
  else
    return silu_f32(z);
}

// ------------------------------------------------- exp2 on the FMA pipe
// 2^x for two values at once, on the FP32 pipe instead of the SFU, so a
// kernel can split its exponentials between the two units.
// Range reduction: j = rint(x) (adding 1.5 * 2^23 rounds to an integer),
// r = x - j in [-1/2, 1/2]; 2^r = 1 + r q(r) with q the degree-4 minimax
// fit of (2^r - 1) / r made by fit_polys.py (relative error of 2^r
// below 1.7e-7 and of 2^r - 1 below 4.7e-7); 2^j is added to the exponent
// field.  x is clamped to [-126, 126] so the exponent stays a normal number.
constexpr float kExp2Q0 = 6.931471229e-01f;
constexpr float kExp2Q1 = 2.402235121e-01f;
constexpr float kExp2Q2 = 5.550500378e-02f;
constexpr float kExp2Q3 = 9.666245431e-03f;
constexpr float kExp2Q4 = 1.333353808e-03f;

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fminf(fmaxf(x.x, -126.0f), 126.0f);
  x.y = fminf(fmaxf(x.y, -126.0f), 126.0f);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 t = __fadd2_rn(x, magic);                          // low bits hold rint(x)
  const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 r = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);   // x - j, exact
  float2 q = __ffma2_rn(make_float2(kExp2Q4, kExp2Q4), r, make_float2(kExp2Q3, kExp2Q3));
  q = __ffma2_rn(q, r, make_float2(kExp2Q2, kExp2Q2));
  q = __ffma2_rn(q, r, make_float2(kExp2Q1, kExp2Q1));
  q = __ffma2_rn(q, r, make_float2(kExp2Q0, kExp2Q0));
  const float2 p = __ffma2_rn(q, r, make_float2(1.0f, 1.0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

__device__ __forceinline__ float2 exp2_sfu2(float2 x) {
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// 32-byte vector accesses (sm_100 and later); the address must be 32-byte
// aligned.  The streaming load is volatile so it stays ordered before the
// (volatile) store that writes the same state back.
__device__ __forceinline__ void ld8_stream(const float *q, float *v) {
  asm volatile("ld.global.cs.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]),
                 "=f"(v[6]), "=f"(v[7])
               : "l"(q));
}
__device__ __forceinline__ void st8_stream(float *q, const float *v) {
  asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(q), "f"(v[0]),
               "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}
// read-only data (not written while the kernel runs)
__device__ __forceinline__ void ld8_ro(const void *q, uint32_t *w) {
  asm("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
        "=r"(w[7])
      : "l"(q));
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

// ------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while
// the kernel before it in the stream still runs: the earlier one lets it
// launch (grid_dependents_launch), and it waits for the earlier grids to
// finish with their writes visible (grid_dependency_wait) before reading
// what they produce.  Without such a launch the wait returns at once.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace ssm
