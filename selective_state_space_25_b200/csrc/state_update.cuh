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
};

// NPT states per thread (4, or N when N < 4); G = N / NPT threads per channel.
template <typename T, int N, int NPT>
__global__ void __launch_bounds__(256) state_update_kernel(StepParams p) {
  constexpr int G = N / NPT;
  static_assert(G >= 1 && G <= 32 && (32 % G) == 0, "bad N");
  const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t bd = gid / G;
  const int g = (int)(gid - bd * G);
  const bool active = bd < p.b * p.d_in;
  const int64_t ib = active ? bd / p.d_in : 0;
  const int64_t d = active ? bd - ib * p.d_in : 0;
  const T *xs = static_cast<const T *>(p.x);
  const T *dts = static_cast<const T *>(p.dt);
  const T *Bs = static_cast<const T *>(p.B);
  const T *Cs = static_cast<const T *>(p.C);
  const T *zs = static_cast<const T *>(p.z);

  float acc = 0.0f, xv = 0.0f;
  if (active) {
    float delta = Elem<T>::load(dts, bd) + (p.dt_bias ? p.dt_bias[d] : 0.0f);
    if (p.dt_softplus) delta = softplus_f32(delta);
    xv = Elem<T>::load(xs, bd);
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
template <typename T, int N, int CPT>
__global__ void __launch_bounds__(256) state_update_vec_kernel(StepParams p) {
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
  int64_t bd[CPT];
  bool on[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) {  // issue every state load first
    bd[i] = base + i * per;
    on[i] = base < per && bd[i] < total;
    st[i] = on[i] ? __ldcs(reinterpret_cast<const float4 *>(p.state + bd[i] * N + 4 * g))
                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int64_t ib = on[i] ? bd[i] / p.d_in : 0;
    const int64_t d = on[i] ? bd[i] - ib * p.d_in : 0;
    float acc = 0.0f, xv = 0.0f;
    if (on[i]) {
      float delta = Elem<T>::load(dts, bd[i]) + (p.dt_bias ? p.dt_bias[d] : 0.0f);
      if (p.dt_softplus) delta = softplus_f32(delta);
      xv = Elem<T>::load(xs, bd[i]);
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
    if (on[i] && g == 0) {
      float yv = fmaf(p.D ? p.D[d] : 0.0f, xv, acc);
      if (zs) yv *= silu_for<T>(Elem<T>::load(zs, bd[i]));
      Elem<T>::store(static_cast<T *>(p.y), bd[i], yv);
    }
  }
}

}  // namespace ssm
