// state_update.cuh -- one-token selective state update (decode).
//
// "代码连连看——mamba", Mamba.step(), the SSM step without
// selective_state_update:  dt = softplus(dt + dt_proj.bias),
// dA = exp(einsum('bd,dn->bdn', dt, A)), dB = einsum('bd,bn->bdn', dt, B),
// state = state * dA + x * dB (in place), y = einsum('bdn,bn->bd', state, C)
// + D x, y = y * act(z).
//
// The step is a streaming read-modify-write of the fp32 state: 8 bytes per
// (batch, channel, state) plus a few bytes per channel.  G = N / 4 threads
// share a channel, each moving 4 states as one 16-byte vector; the partial
// C.state sums meet in a G-lane shuffle.
#pragma once

#include "ssm_common.cuh"

namespace ssm {

struct StepParams {
  float *state;
  const void *x, *dt;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *dt_bias;
  void *y;
  int64_t b, d_in;
  int dt_softplus;
  // fused causal-conv1d step in front of the SSM step (conv_state == nullptr: none)
  void *conv_state;             // (b, d_in, d_conv), activation dtype, in place
  const float *conv_w, *conv_b; // (d_in, d_conv), (d_in) nullable
  int d_conv;
};

// The conv step of Mamba.step() ("代码连连看——mamba"): the window is rolled
// left with x appended, dotted with the depthwise weight, plus the bias.
// The G lanes of a channel split the taps (lane g owns taps g, g + G, ...),
// so a warp reads and writes its channels' windows and weights as contiguous
// runs; conv_partial returns this lane's share of the sum and fills the new
// window entries it owns into nw.  Every value in the window is an input of
// the activation dtype, so storing it back is exact.
constexpr int kMaxConv = 8;

// CTAs of 256 threads the decode kernels are compiled to fit per SM.
#ifndef SSM_STEP_MIN_CTAS
#define SSM_STEP_MIN_CTAS 8
#endif
template <int G> constexpr int conv_taps_per_lane() { return (kMaxConv + G - 1) / G; }

// This lane's taps of the old window (the tap that takes x is left for
// conv_partial) and of the weight; loaded ahead of the arithmetic.
template <int G>
struct ConvTaps {
  float v[conv_taps_per_lane<G>()], w[conv_taps_per_lane<G>()], bias;
};

template <typename T, int G>
__device__ __forceinline__ void conv_load(const StepParams &p, int64_t bd, int64_t d, int g,
                                          ConvTaps<G> &c) {
  const T *cs = static_cast<const T *>(p.conv_state) + bd * p.d_conv;
  const float *w = p.conv_w + d * p.d_conv;
  const int K = p.d_conv;
  c.bias = (g == 0 && p.conv_b) ? p.conv_b[d] : 0.0f;
#pragma unroll
  for (int i = 0; i < conv_taps_per_lane<G>(); ++i) {
    const int j = g + i * G;
    c.v[i] = (j + 1 < K) ? Elem<T>::load(cs, j + 1) : 0.0f;
    c.w[i] = (j < K) ? w[j] : 0.0f;
  }
}

// This lane's share of the conv sum; fills the new window entries it owns
// into nw (x goes into the last tap).
template <int G>
__device__ __forceinline__ float conv_partial(const ConvTaps<G> &c, int K, int g, float xraw,
                                              float (&nw)[conv_taps_per_lane<G>()]) {
  float acc = c.bias;
#pragma unroll
  for (int i = 0; i < conv_taps_per_lane<G>(); ++i) {
    const int j = g + i * G;
    const float v = (j + 1 < K) ? c.v[i] : xraw;
    nw[i] = v;
    if (j < K) acc = fmaf(v, c.w[i], acc);
  }
  return acc;
}

template <typename T, int G>
__device__ __forceinline__ void conv_store(const StepParams &p, int64_t bd, int g,
                                           const float (&nw)[conv_taps_per_lane<G>()]) {
  T *cs = static_cast<T *>(p.conv_state) + bd * p.d_conv;
#pragma unroll
  for (int i = 0; i < conv_taps_per_lane<G>(); ++i) {
    const int j = g + i * G;
    if (j < p.d_conv) Elem<T>::store(cs, j, nw[i]);
  }
}

// NPT states per thread (4, or N when N < 4); G = N / NPT threads per channel.
template <typename T, int N, int NPT, bool CONV>
__global__ void __launch_bounds__(256) state_update_kernel(StepParams p) {
  constexpr int G = N / NPT;
  static_assert(G >= 1 && G <= 32 && (32 % G) == 0, "bad N");
  const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t bd = gid / G;
  const int g = (int)(gid - bd * G);
  const bool active =
      bd < p.b * p.d_in && in_bounds(bd * N + g * NPT + NPT - 1, p.b * p.d_in * N, kBndState) &&
      (!CONV || in_bounds(bd * p.d_conv + p.d_conv - 1, p.b * p.d_in * p.d_conv, kBndWork));
  const int64_t ib = active ? bd / p.d_in : 0;
  const int64_t d = active ? bd - ib * p.d_in : 0;
  const T *xs = static_cast<const T *>(p.x);
  const T *dts = static_cast<const T *>(p.dt);
  const T *Bs = static_cast<const T *>(p.B);
  const T *Cs = static_cast<const T *>(p.C);
  const T *zs = static_cast<const T *>(p.z);

  float acc = 0.0f, xv = 0.0f;
  float nw[conv_taps_per_lane<G>()];
  if (active) xv = Elem<T>::load(xs, bd);
  if constexpr (CONV) {
    ConvTaps<G> taps;
    if (active) conv_load<T, G>(p, bd, d, g, taps);
    float c = active ? conv_partial<G>(taps, p.d_conv, g, xv, nw) : 0.0f;
#pragma unroll
    for (int m = 1; m < G; m <<= 1) c += __shfl_xor_sync(0xffffffffu, c, m);
    xv = silu_f32(c);
  }
  if (active) {
    float delta = Elem<T>::load(dts, bd) + (p.dt_bias ? p.dt_bias[d] : 0.0f);
    if (p.dt_softplus) delta = softplus_f32(delta);
    const float dx = delta * xv;
    float *sp = p.state + bd * N + g * NPT;
    float s[NPT];
    if constexpr (NPT == 4) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(sp));
      s[0] = v.x; s[1] = v.y; s[2] = v.z; s[3] = v.w;
    } else {
#pragma unroll
      for (int j = 0; j < NPT; ++j) s[j] = sp[j];
    }
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
      const int n = g * NPT + j;
      const float a = ex2_approx(delta * (p.A[d * N + n] * kLog2e));
      s[j] = fmaf(s[j], a, dx * Elem<T>::load(Bs, ib * N + n));
      acc = fmaf(s[j], Elem<T>::load(Cs, ib * N + n), acc);
    }
    if constexpr (NPT == 4) {
      __stcs(reinterpret_cast<float4 *>(sp), make_float4(s[0], s[1], s[2], s[3]));
    } else {
#pragma unroll
      for (int j = 0; j < NPT; ++j) sp[j] = s[j];
    }
  }
#pragma unroll
  for (int m = 1; m < G; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if constexpr (CONV) {
    __syncwarp();  // every lane of the channel has read the old window
    if (active) conv_store<T, G>(p, bd, g, nw);
  }
  if (active && g == 0) {
    float yv = fmaf(p.D ? p.D[d] : 0.0f, xv, acc);
    if (zs) yv *= silu_f32(Elem<T>::load(zs, bd));
    Elem<T>::store(static_cast<T *>(p.y), bd, yv);
  }
}

// Vector kernel (N a multiple of 4, state and A 16-byte aligned, B and C
// 8-byte aligned): thread g of a channel owns states 4g .. 4g + 3 and each
// thread handles CPT channels spaced total / CPT apart, so CPT independent
// 16-byte state loads are in flight per thread and every warp instruction
// still touches one contiguous 512-byte span of the state.
template <typename T, int N, int CPT, bool CONV>
__global__ void __launch_bounds__(256, SSM_STEP_MIN_CTAS) state_update_vec_kernel(StepParams p) {
  constexpr int G = N / 4;
  static_assert(N % 4 == 0 && G <= 32 && 32 % G == 0, "bad N");
  const int64_t total = p.b * p.d_in;                 // channels
  const int64_t per = (total + CPT - 1) / CPT;        // channel stride between a thread's channels
  const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t base = gid / G;
  const int g = (int)(gid - base * G);
  const T *xs = static_cast<const T *>(p.x);
  const T *dts = static_cast<const T *>(p.dt);
  const T *zs = static_cast<const T *>(p.z);

  float4 st[CPT];
  int64_t bd[CPT], ibs[CPT], ds[CPT];
  bool on[CPT];
  ConvTaps<G> taps[CPT];
  const bool narrow = total <= 0xffffffffll;  // 32-bit division suffices
#pragma unroll
  for (int i = 0; i < CPT; ++i) {  // issue every state (and conv window) load first
    bd[i] = base + i * per;
    on[i] = base < per && bd[i] < total &&
            in_bounds(bd[i] * N + 4 * g + 3, total * N, kBndState) &&
            (!CONV || in_bounds(bd[i] * p.d_conv + p.d_conv - 1, total * p.d_conv, kBndWork));
    st[i] = on[i] ? __ldcs(reinterpret_cast<const float4 *>(p.state + bd[i] * N + 4 * g))
                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const int64_t c = on[i] ? bd[i] : 0;
    ibs[i] = narrow ? (int64_t)((uint32_t)c / (uint32_t)p.d_in) : c / p.d_in;
    ds[i] = c - ibs[i] * p.d_in;
    if constexpr (CONV) {
      if (on[i]) conv_load<T, G>(p, bd[i], ds[i], g, taps[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int64_t ib = ibs[i];
    const int64_t d = ds[i];
    float acc = 0.0f, xv = 0.0f;
    float nw[conv_taps_per_lane<G>()];
    if (on[i]) xv = Elem<T>::load(xs, bd[i]);
    if constexpr (CONV) {  // the G lanes of a channel are all on or all off
      float c = on[i] ? conv_partial<G>(taps[i], p.d_conv, g, xv, nw) : 0.0f;
#pragma unroll
      for (int m = 1; m < G; m <<= 1) c += __shfl_xor_sync(0xffffffffu, c, m);
      xv = silu_f32(c);
    }
    if (on[i]) {
      float delta = Elem<T>::load(dts, bd[i]) + (p.dt_bias ? p.dt_bias[d] : 0.0f);
      if (p.dt_softplus) delta = softplus_f32(delta);
      const float4 a4 = *reinterpret_cast<const float4 *>(p.A + d * N + 4 * g);
      float4 b4, c4;
      if constexpr (sizeof(T) == 2) {
        const uint2 wb = *reinterpret_cast<const uint2 *>(static_cast<const T *>(p.B) + ib * N + 4 * g);
        const uint2 wc = *reinterpret_cast<const uint2 *>(static_cast<const T *>(p.C) + ib * N + 4 * g);
        b4 = make_float4(bf16lo(wb.x), bf16hi(wb.x), bf16lo(wb.y), bf16hi(wb.y));
        c4 = make_float4(bf16lo(wc.x), bf16hi(wc.x), bf16lo(wc.y), bf16hi(wc.y));
      } else {
        b4 = *reinterpret_cast<const float4 *>(static_cast<const T *>(p.B) + ib * N + 4 * g);
        c4 = *reinterpret_cast<const float4 *>(static_cast<const T *>(p.C) + ib * N + 4 * g);
      }
      const float dx = delta * xv;
      const float dl = delta * kLog2e;
      float4 s4 = st[i];
      s4.x = fmaf(s4.x, ex2_approx(dl * a4.x), dx * b4.x);
      s4.y = fmaf(s4.y, ex2_approx(dl * a4.y), dx * b4.y);
      s4.z = fmaf(s4.z, ex2_approx(dl * a4.z), dx * b4.z);
      s4.w = fmaf(s4.w, ex2_approx(dl * a4.w), dx * b4.w);
      __stcs(reinterpret_cast<float4 *>(p.state + bd[i] * N + 4 * g), s4);
      acc = fmaf(s4.x, c4.x, fmaf(s4.y, c4.y, fmaf(s4.z, c4.z, s4.w * c4.w)));
    }
#pragma unroll
    for (int m = 1; m < G; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if constexpr (CONV) {
      __syncwarp();  // every lane of the channel has read the old window
      if (on[i]) conv_store<T, G>(p, bd[i], g, nw);
    }
    if (on[i] && g == 0) {
      float yv = fmaf(p.D ? p.D[d] : 0.0f, xv, acc);
      if (zs) yv *= silu_for<T>(Elem<T>::load(zs, bd[i]));
      Elem<T>::store(static_cast<T *>(p.y), bd[i], yv);
    }
  }
}

}  // namespace ssm
