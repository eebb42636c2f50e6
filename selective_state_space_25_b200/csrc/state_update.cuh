// state_update.cuh -- one-token selective state update (decode).
//
// "代码连连看——mamba", Mamba.step(), the SSM step without
// selective_state_update:  dt = softplus(dt + dt_proj.bias),
// dA = exp(einsum('bd,dn->bdn', dt, A)), dB = einsum('bd,bn->bdn', dt, B),
// state = state * dA + x * dB (in place), y = einsum('bdn,bn->bd', state, C)
// + D x, y = y * act(z).
//
// The step is a streaming read-modify-write of the fp32 state: 8 bytes per
// (batch, channel, state) plus a few bytes per channel.  For N = 4, 8, 16 one
// thread owns a channel and moves its states as 32-byte vectors
// (state_update_lane_kernel); for N = 32, 64 G = N / 4 threads share a
// channel, each moving 4 states as one 16-byte vector, and the partial
// C.state sums meet in a G-lane shuffle (state_update_vec_kernel).
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

// A whole B or C row (N entries of the activation dtype) as packed words.
template <typename T, int N> struct RowWords {
  static constexpr int W = N * (int)sizeof(T) / 4;  // 32-bit words
  uint32_t w[W];
  __device__ __forceinline__ void load(const T *row) {
    if constexpr (W % 8 == 0) {  // 32-byte rows: one 32-byte load each
#pragma unroll
      for (int i = 0; i < W; i += 8) ld8_ro(reinterpret_cast<const uint32_t *>(row) + i, w + i);
    } else if constexpr (W % 4 == 0) {
#pragma unroll
      for (int i = 0; i < W; i += 4) {
        const uint4 q = __ldg(reinterpret_cast<const uint4 *>(row) + i / 4);
        w[i] = q.x; w[i + 1] = q.y; w[i + 2] = q.z; w[i + 3] = q.w;
      }
    } else {
      static_assert(W == 2, "row of 8 bytes");
      const uint2 q = __ldg(reinterpret_cast<const uint2 *>(row));
      w[0] = q.x; w[1] = q.y;
    }
  }
  // entries 2k, 2k + 1 as an fp32 pair
  __device__ __forceinline__ float2 pair(int k) const {
    if constexpr (sizeof(T) == 2)
      return make_float2(bf16lo(w[k]), bf16hi(w[k]));
    else
      return make_float2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1]));
  }
};

#ifndef SSM_LANE_MIN_CTAS
#define SSM_LANE_MIN_CTAS 3
#endif

// One thread per (batch, channel) (N = 4, 8 or 16; state, A, B and C 32-byte
// aligned, 16 for N = 4): the channel's N states are 32-byte vectors (one
// 16-byte vector for N = 4), issued with its A row and the batch's B / C
// rows before any arithmetic, so every per-channel term (the division that
// splits the channel index, softplus, the conv step, the gate, y) is formed
// once per channel rather than on each of G lanes of a channel.  Each lane
// moves whole 32-byte sectors: a warp's state loads cover one contiguous
// 32 N-float span in N / 8 instructions.
template <typename T, int N, bool CONV>
__global__ void __launch_bounds__(256, SSM_LANE_MIN_CTAS) state_update_lane_kernel(StepParams p) {
  static_assert(N == 4 || N == 8 || N == 16, "one thread per channel for N = 4, 8, 16");
  const int64_t total = p.b * p.d_in;
  const int64_t bd = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (bd >= total || !in_bounds(bd * N + N - 1, total * N, kBndState) ||
      (CONV && !in_bounds(bd * p.d_conv + p.d_conv - 1, total * p.d_conv, kBndWork)))
    return;  // nothing below synchronises, so idle threads may leave
  const int64_t ib = total <= 0xffffffffll ? (int64_t)((uint32_t)bd / (uint32_t)p.d_in)
                                           : bd / p.d_in;
  const int64_t d = bd - ib * p.d_in;
  if (!in_bounds(d * N + N - 1, p.d_in * N, kBndParam)) return;

  float sv[N], av[N];
  float *sp = p.state + bd * N;
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int v = 0; v < N; v += 8) ld8_stream(sp + v, sv + v);
#pragma unroll
    for (int v = 0; v < N; v += 8) ld8_ro(p.A + d * N + v, reinterpret_cast<uint32_t *>(av + v));
  } else {
    const float4 s4 = __ldcs(reinterpret_cast<const float4 *>(sp));
    const float4 a4 = __ldg(reinterpret_cast<const float4 *>(p.A + d * N));
    sv[0] = s4.x; sv[1] = s4.y; sv[2] = s4.z; sv[3] = s4.w;
    av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
  }
  RowWords<T, N> brow, crow;
  brow.load(static_cast<const T *>(p.B) + ib * N);
  crow.load(static_cast<const T *>(p.C) + ib * N);
  float xv = Elem<T>::load(static_cast<const T *>(p.x), bd);
  const float dtv = Elem<T>::load(static_cast<const T *>(p.dt), bd);
  const T *zs = static_cast<const T *>(p.z);
  const float zv = zs ? Elem<T>::load(zs, bd) : 0.0f;
  const float bias = p.dt_bias ? p.dt_bias[d] : 0.0f;
  const float Dv = p.D ? p.D[d] : 0.0f;

  if constexpr (CONV) {  // the window rolled left with x appended, dotted with the weight
    T *cs = static_cast<T *>(p.conv_state) + bd * p.d_conv;
    const float *w = p.conv_w + d * p.d_conv;
    const int K = p.d_conv;
    float acc = p.conv_b ? p.conv_b[d] : 0.0f;
    if (K == 4 && (reinterpret_cast<uintptr_t>(cs) & (4 * sizeof(T) - 1)) == 0 &&
        (reinterpret_cast<uintptr_t>(w) & 15) == 0) {
      // the common width: window and weight as one vector each
      const float4 w4 = __ldg(reinterpret_cast<const float4 *>(w));
      if constexpr (sizeof(T) == 2) {
        const uint2 q = *reinterpret_cast<const uint2 *>(cs);  // taps 0, 1 | 2, 3
        acc = fmaf(bf16hi(q.x), w4.x, acc);
        acc = fmaf(bf16lo(q.y), w4.y, acc);
        acc = fmaf(bf16hi(q.y), w4.z, acc);
        acc = fmaf(xv, w4.w, acc);
        // rolled window: taps 1, 2 | 3, x (x is a widened bf16, so its top
        // half is its exact bit pattern)
        const uint32_t xb = __float_as_uint(xv) >> 16;
        *reinterpret_cast<uint2 *>(cs) =
            make_uint2(__byte_perm(q.x, q.y, 0x5432), __byte_perm(q.y, xb, 0x5432));
      } else {
        const float4 q = *reinterpret_cast<const float4 *>(cs);
        acc = fmaf(q.y, w4.x, acc);
        acc = fmaf(q.z, w4.y, acc);
        acc = fmaf(q.w, w4.z, acc);
        acc = fmaf(xv, w4.w, acc);
        *reinterpret_cast<float4 *>(cs) = make_float4(q.y, q.z, q.w, xv);
      }
    } else {
      float win[kMaxConv];
#pragma unroll
      for (int j = 0; j < kMaxConv; ++j) {
        if (j < K) {
          win[j] = j + 1 < K ? Elem<T>::load(cs, j + 1) : xv;
          acc = fmaf(win[j], w[j], acc);
        }
      }
#pragma unroll
      for (int j = 0; j < kMaxConv; ++j)
        if (j < K) Elem<T>::store(cs, j, win[j]);
    }
    xv = silu_f32(acc);
  }

  float delta = dtv + bias;
  if (p.dt_softplus) delta = softplus_f32(delta);
  const float2 dl2 = make_float2(delta * kLog2e, delta * kLog2e);
  const float2 dx2 = make_float2(delta * xv, delta * xv);
  float2 yacc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int k = 0; k < N / 2; ++k) {
    float2 s2 = make_float2(sv[2 * k], sv[2 * k + 1]);
    const float2 a2 = exp2_sfu2(__fmul2_rn(dl2, make_float2(av[2 * k], av[2 * k + 1])));
    s2 = __ffma2_rn(s2, a2, __fmul2_rn(dx2, brow.pair(k)));
    sv[2 * k] = s2.x;
    sv[2 * k + 1] = s2.y;
    yacc = __ffma2_rn(s2, crow.pair(k), yacc);
  }
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int v = 0; v < N; v += 8) st8_stream(sp + v, sv + v);
  } else {
    __stcs(reinterpret_cast<float4 *>(sp), make_float4(sv[0], sv[1], sv[2], sv[3]));
  }
  float yv = fmaf(Dv, xv, yacc.x + yacc.y);
  if (zs) yv *= silu_for<T>(zv);
  Elem<T>::store(static_cast<T *>(p.y), bd, yv);
}

}  // namespace ssm
