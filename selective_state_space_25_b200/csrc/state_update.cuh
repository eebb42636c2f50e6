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

}  // namespace ssm
