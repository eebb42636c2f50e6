// scan_fwd.cuh -- selective scan forward kernels.
//
// The operation ("手把手拆解Mamba-minimal中的selective_scan实现" §3-§5, with
// the softplus of delta and the SiLU gate of "代码连连看——mamba"'s
// Mamba.step()): per (batch i, channel d, state n)
//     delta = softplus(dt + dt_bias),  dA = exp(delta A),  dBu = delta B u,
//     h = dA h + dBu,  y = sum_n C h + D u,  y *= silu(z).
// dA and dBu, (b, L, d_in, N) tensors in the pages' loop, are never stored:
// they are formed in registers one step at a time.
#pragma once

#include "ssm_common.cuh"

namespace ssm {

struct ScanParams {
  const void *u, *delta;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *dt_bias, *h0;
  float *h_last;
  void *y;
  int64_t b, L, d_in;
  int delta_softplus;
};

// ---------------------------------------------------------------------------
// Generic kernel: one thread per (batch, channel), all N states in registers,
// sequential over t.  Any d_in, any alignment of the element type; used when
// the staged kernel's alignment conditions do not hold and for N < 8.
// ---------------------------------------------------------------------------
template <typename T, int N>
__global__ void __launch_bounds__(128) scan_generic_kernel(ScanParams p) {
  const int64_t bd = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (bd >= p.b * p.d_in) return;
  const int64_t ib = bd / p.d_in;
  const int64_t d = bd - ib * p.d_in;
  const T *u = static_cast<const T *>(p.u);
  const T *dt = static_cast<const T *>(p.delta);
  const T *Bm = static_cast<const T *>(p.B);
  const T *Cm = static_cast<const T *>(p.C);
  const T *z = static_cast<const T *>(p.z);
  T *y = static_cast<T *>(p.y);

  float h[N], A2[N];
#pragma unroll
  for (int n = 0; n < N; ++n) {
    A2[n] = p.A[d * N + n] * kLog2e;
    h[n] = p.h0 ? p.h0[bd * N + n] : 0.0f;
  }
  const float bias = p.dt_bias ? p.dt_bias[d] : 0.0f;
  const float Dd = p.D ? p.D[d] : 0.0f;

  for (int64_t t = 0; t < p.L; ++t) {
    const int64_t row = ib * p.L + t;
    const int64_t i = row * p.d_in + d;
    float delta = Elem<T>::load(dt, i) + bias;
    if (p.delta_softplus) delta = softplus_f32(delta);
    const float ut = Elem<T>::load(u, i);
    const float du = delta * ut;
    float acc = 0.0f;
#pragma unroll
    for (int n = 0; n < N; ++n) {
      const float a = ex2_approx(delta * A2[n]);
      h[n] = fmaf(a, h[n], du * Elem<T>::load(Bm, row * N + n));
      acc = fmaf(h[n], Elem<T>::load(Cm, row * N + n), acc);
    }
    float yt = fmaf(Dd, ut, acc);
    if (z) yt *= silu_f32(Elem<T>::load(z, i));
    Elem<T>::store(y, i, yt);
  }
  if (p.h_last) {
#pragma unroll
    for (int n = 0; n < N; ++n) p.h_last[bd * N + n] = h[n];
  }
}

// ---------------------------------------------------------------------------
// Staged kernel.  A CTA owns (batch i, a tile of DT channels) for the whole
// sequence and walks it in chunks of TC steps:
//   1. the chunk's u / delta / z tile [TC x DT] and B / C rows [TC x N] are
//      copied global -> shared with 16-byte cp.async (issued one chunk ahead,
//      overlapping the previous chunk's scan);
//   2. pre-pass, one thread per (t, d): delta' = softplus(dt + bias),
//      delta' u, u and silu(z) go to shared memory as fp32; B, C rows are
//      widened to fp32 once for all channels;
//   3. scan: G = N / 4 threads share a channel, each owning 4 states in
//      registers; per step 4 x (exp2, FMUL, 2 FFMA) and a G-lane shuffle sum
//      of the partial C.h;
//   4. post-pass, one thread per (t, d): y = (C.h + D u) * silu(z), rounded
//      once and stored coalesced.
// Requires: N in {8, 16, 32, 64}; d_in * sizeof(T) a multiple of 16; u,
// delta, z, B, C 16-byte aligned.
// ---------------------------------------------------------------------------
template <typename T, int N, int DT, int TC>
struct StagedScan {
  static constexpr int NPT = 4;                 // states per thread
  static constexpr int G = N / NPT;             // threads per channel
  static constexpr int THREADS = DT * G;
  static constexpr int ESZ = sizeof(T);
  static constexpr int VEC = 16 / ESZ;          // elements per 16-byte granule
  static constexpr int ROW_GRAN = DT / VEC;     // granules per tile row
  static constexpr int TILE_BYTES = TC * DT * ESZ;
  static constexpr int BC_GRAN = N / VEC;       // granules per B / C row
  static constexpr int BC_BYTES = TC * N * ESZ;
  // shared-memory carve-up (bytes)
  static constexpr int OFF_U = 0;
  static constexpr int OFF_DT = OFF_U + TILE_BYTES;
  static constexpr int OFF_Z = OFF_DT + TILE_BYTES;
  static constexpr int OFF_B = OFF_Z + TILE_BYTES;
  static constexpr int OFF_C = OFF_B + BC_BYTES;
  static constexpr int OFF_DTU = OFF_C + BC_BYTES;                   // float2 [TC][DT]
  static constexpr int OFF_UG = OFF_DTU + TC * DT * 8;                // float2 [TC][DT]
  static constexpr int OFF_BF = OFF_UG + TC * DT * 8;                 // float [TC][N]
  static constexpr int OFF_CF = OFF_BF + TC * N * 4;                  // float [TC][N]
  static constexpr int OFF_YS = OFF_CF + TC * N * 4;                  // float [TC][DT]
  static constexpr int SMEM = OFF_YS + TC * DT * 4;
  static_assert(N % NPT == 0 && G <= 32 && (32 % G) == 0, "bad N");
  static_assert(DT % VEC == 0 && N % VEC == 0, "tile rows must be whole granules");
  static_assert(THREADS % 32 == 0, "whole warps");
};

template <typename T, int N, int DT, int TC, bool HAS_Z>
__global__ void __launch_bounds__(StagedScan<T, N, DT, TC>::THREADS)
    scan_staged_kernel(ScanParams p) {
  using S = StagedScan<T, N, DT, TC>;
  extern __shared__ __align__(16) unsigned char smem[];
  const int tid = threadIdx.x;
  const int64_t ib = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * DT;
  const int64_t L = p.L, d_in = p.d_in;

  const T *gu = static_cast<const T *>(p.u);
  const T *gdt = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);

  T *su = reinterpret_cast<T *>(smem + S::OFF_U);
  T *sdt = reinterpret_cast<T *>(smem + S::OFF_DT);
  T *sz = reinterpret_cast<T *>(smem + S::OFF_Z);
  T *sB = reinterpret_cast<T *>(smem + S::OFF_B);
  T *sC = reinterpret_cast<T *>(smem + S::OFF_C);
  float2 *sdtu = reinterpret_cast<float2 *>(smem + S::OFF_DTU);
  float2 *sug = reinterpret_cast<float2 *>(smem + S::OFF_UG);
  float *sBf = reinterpret_cast<float *>(smem + S::OFF_BF);
  float *sCf = reinterpret_cast<float *>(smem + S::OFF_CF);
  float *sys = reinterpret_cast<float *>(smem + S::OFF_YS);

  // ---- copy chunk [t0, t0 + TC) of this CTA's tiles into shared memory
  auto prefetch = [&](int64_t t0) {
    for (int q = tid; q < TC * S::ROW_GRAN; q += S::THREADS) {
      const int t = q / S::ROW_GRAN, gq = q - t * S::ROW_GRAN;
      const int64_t dd = d0 + gq * S::VEC;
      const bool ok = (t0 + t < L) && (dd < d_in);
      const int64_t off = ok ? ((ib * L + t0 + t) * d_in + dd) : 0;
      const int so = t * DT + gq * S::VEC;
      cp_async16(su + so, gu + off, ok ? 16 : 0);
      cp_async16(sdt + so, gdt + off, ok ? 16 : 0);
      if (HAS_Z) cp_async16(sz + so, gz + off, ok ? 16 : 0);
    }
    for (int q = tid; q < TC * S::BC_GRAN; q += S::THREADS) {
      const int t = q / S::BC_GRAN, gq = q - t * S::BC_GRAN;
      const bool ok = (t0 + t < L);
      const int64_t off = ok ? ((ib * L + t0 + t) * N + gq * S::VEC) : 0;
      const int so = t * N + gq * S::VEC;
      cp_async16(sB + so, gB + off, ok ? 16 : 0);
      cp_async16(sC + so, gC + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // ---- per-thread scan state: channel dl, state group g
  const int dl = tid / S::G;
  const int g = tid - dl * S::G;
  const int64_t d = d0 + dl;
  const bool d_ok = d < d_in;
  float A2[S::NPT], h[S::NPT];
#pragma unroll
  for (int j = 0; j < S::NPT; ++j) {
    const int n = g * S::NPT + j;
    A2[j] = d_ok ? p.A[d * N + n] * kLog2e : 0.0f;
    h[j] = (d_ok && p.h0) ? p.h0[(ib * d_in + d) * N + n] : 0.0f;
  }

  const int64_t nchunks = (L + TC - 1) / TC;
  prefetch(0);
  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t t0 = c * TC;
    const int tc = (int)((L - t0) < (int64_t)TC ? (L - t0) : (int64_t)TC);
    cp_async_wait<0>();
    __syncthreads();  // tiles of chunk c visible; previous post-pass done

    // ---- pre-pass: per (t, d) and per (t, n)
    for (int q = tid; q < TC * DT; q += S::THREADS) {
      const int t = q / DT, c_ = q - t * DT;
      const int64_t dd = d0 + c_;
      const float bias = (p.dt_bias && dd < d_in) ? p.dt_bias[dd] : 0.0f;
      float delta = Elem<T>::load(sdt, q) + bias;
      if (p.delta_softplus) delta = softplus_f32(delta);
      const float ut = Elem<T>::load(su, q);
      sdtu[q] = make_float2(delta, delta * ut);
      const float gate = HAS_Z ? silu_f32(Elem<T>::load(sz, q)) : 1.0f;
      sug[q] = make_float2(ut, gate);
    }
    for (int q = tid; q < TC * N; q += S::THREADS) {
      sBf[q] = Elem<T>::load(sB, q);
      sCf[q] = Elem<T>::load(sC, q);
    }
    __syncthreads();  // raw tiles consumed

    if (c + 1 < nchunks) prefetch(t0 + TC);  // overlaps the scan below

    // ---- scan over the chunk
    for (int t = 0; t < tc; ++t) {
      const float2 q = sdtu[t * DT + dl];
      const float4 bv = *reinterpret_cast<const float4 *>(sBf + t * N + g * S::NPT);
      const float4 cv = *reinterpret_cast<const float4 *>(sCf + t * N + g * S::NPT);
      const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
      const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < S::NPT; ++j) {
        const float a = ex2_approx(q.x * A2[j]);
        h[j] = fmaf(a, h[j], q.y * bb[j]);
        acc = fmaf(h[j], cc[j], acc);
      }
#pragma unroll
      for (int m = 1; m < S::G; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
      if (g == 0) sys[t * DT + dl] = acc;
    }
    __syncthreads();

    // ---- post-pass: D skip, gate, one rounding, coalesced store
    for (int q = tid; q < tc * DT; q += S::THREADS) {
      const int t = q / DT, c_ = q - t * DT;
      const int64_t dd = d0 + c_;
      if (dd >= d_in) continue;
      const float2 ug = sug[q];
      const float Dd = p.D ? p.D[dd] : 0.0f;
      const float yt = fmaf(Dd, ug.x, sys[q]) * ug.y;
      Elem<T>::store(gy, (ib * L + t0 + t) * d_in + dd, yt);
    }
  }

  if (p.h_last && d_ok) {
#pragma unroll
    for (int j = 0; j < S::NPT; ++j) p.h_last[(ib * d_in + d) * N + g * S::NPT + j] = h[j];
  }
}

}  // namespace ssm
