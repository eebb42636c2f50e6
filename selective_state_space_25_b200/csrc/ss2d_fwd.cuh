// ss2d_fwd.cuh -- VMamba SS2D forward: CrossScan, selective scan per
// direction, CrossMerge ("关于代码SS2D中的d_state设置", VMamba issue 206:
// the four scan orders only arrange the sequence; d_state = 1 for
// throughput).
//
// Direction k visits pixel p_k(l) at step l (pixels row-major, p = h W + w):
//   k0 row-major p = l; k1 column-major l = w H + h; k2 = k0 reversed;
//   k3 = k1 reversed.
// The orders are index arithmetic: u is gathered at p_k(l) when it is read
// and each output lands at p_k(l) when it is produced; no permuted copy and
// no per-direction output exists in memory.
#pragma once

#include "ssm_common.cuh"

namespace ssm {

__device__ __forceinline__ int64_t ss2d_pixel(int k, int64_t l, int64_t H, int64_t W) {
  const int64_t L = H * W;
  if (k >= 2) l = L - 1 - l;
  if ((k & 1) == 0) return l;
  const int64_t w = l / H;
  const int64_t h = l - w * H;
  return h * W + w;
}

struct Ss2dParams {
  const void *u, *delta;
  const float *A;
  const void *B, *C;
  const float *D, *dt_bias;
  void *y;
  float *acc_global;  // (b, L, d_in) fp32 accumulator when shared memory is too small
  int64_t b, H, W, d_in;
  int delta_softplus;
};

// Affine map h -> A h + B of a run of steps; compose(first, then).
struct Aff {
  float a, b;
};
__device__ __forceinline__ Aff aff_then(Aff first, Aff then) {
  return Aff{then.a * first.a, fmaf(then.a, first.b, then.b)};
}

// ---------------------------------------------------------------------------
// d_state = 1 kernel.  CTA = (batch, DT channels), all four directions in
// turn.  Within a direction the sequence is walked in chunks of
// S * TS steps: thread (segment s, channel c) takes TS consecutive steps,
// forms dA, delta B u in registers and their composed affine map; a
// shuffle scan over the warp's segments and a shared-memory pass over the
// warps give each segment its incoming state (the carry of the previous
// chunk included); the segment then replays its steps and adds y into the
// fp32 accumulator at the pixel each step visits.  Summation order per pixel
// is k0 + k1 + k2 + k3, deterministic, rounded once at the end.
// ---------------------------------------------------------------------------
template <int DT, int TS, int WARPS>
struct Ss2dCfg {
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int SPW = 32 / DT;       // segments per warp
  static constexpr int S = SPW * WARPS;     // segments per chunk
  static constexpr int LC = S * TS;         // steps per chunk
  static_assert(32 % DT == 0, "DT divides 32");
  // shared memory besides the accumulator
  static constexpr int AUX_BYTES = WARPS * DT * (int)sizeof(Aff) + DT * (int)sizeof(float);
};

template <typename T, int DT, int TS, int WARPS, bool ACC_SMEM>
__global__ void __launch_bounds__(Ss2dCfg<DT, TS, WARPS>::THREADS)
    ss2d_n1_kernel(Ss2dParams p) {
  using Cfg = Ss2dCfg<DT, TS, WARPS>;
  extern __shared__ __align__(16) unsigned char smem[];
  Aff *agg = reinterpret_cast<Aff *>(smem);                        // [WARPS][DT]
  float *carry = reinterpret_cast<float *>(smem + WARPS * DT * sizeof(Aff));  // [DT]
  float *acc_s = reinterpret_cast<float *>(smem + Cfg::AUX_BYTES);  // [L][DT]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int ch = lane % DT;
  const int sl = lane / DT;
  const int seg = warp * Cfg::SPW + sl;
  const int64_t ib = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * DT;
  const int64_t d = d0 + ch;
  const bool d_ok = d < p.d_in;
  const int64_t H = p.H, W = p.W, L = H * W, d_in = p.d_in;

  const T *gu = static_cast<const T *>(p.u);
  const T *gdt = static_cast<const T *>(p.delta);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);

  // accumulator addressing: shared [L][DT] or global (b, L, d_in)
  float *acc_base = ACC_SMEM ? acc_s : p.acc_global + ib * L * d_in + d0;
  const int64_t acc_stride = ACC_SMEM ? DT : d_in;

  const int64_t nchunks = (L + Cfg::LC - 1) / Cfg::LC;

  for (int k = 0; k < 4; ++k) {
    const int64_t pk = k * d_in + d;  // parameter row of (direction, channel)
    const float A2 = d_ok ? p.A[pk] * kLog2e : 0.0f;
    const float bias = (d_ok && p.dt_bias) ? p.dt_bias[pk] : 0.0f;
    const float Dd = (d_ok && p.D) ? p.D[pk] : 0.0f;
    const int64_t seq = ib * 4 + k;  // row block of (batch, direction) in delta / B / C
    if (tid < DT) carry[tid] = 0.0f;
    __syncthreads();

    for (int64_t c = 0; c < nchunks; ++c) {
      const int64_t l_begin = c * Cfg::LC + (int64_t)seg * TS;
      float a[TS], bu[TS], cc[TS], du[TS];
      Aff mine{1.0f, 0.0f};
#pragma unroll
      for (int j = 0; j < TS; ++j) {
        const int64_t l = l_begin + j;
        a[j] = 1.0f;
        bu[j] = 0.0f;
        cc[j] = 0.0f;
        du[j] = 0.0f;
        if (l < L && d_ok) {
          float delta = Elem<T>::load(gdt, (seq * L + l) * d_in + d) + bias;
          if (p.delta_softplus) delta = softplus_f32(delta);
          const float ut = Elem<T>::load(gu, (ib * L + ss2d_pixel(k, l, H, W)) * d_in + d);
          a[j] = ex2_approx(delta * A2);
          bu[j] = delta * ut * Elem<T>::load(gB, seq * L + l);
          cc[j] = Elem<T>::load(gC, seq * L + l);
          du[j] = Dd * ut;
        }
        mine = aff_then(mine, Aff{a[j], bu[j]});
      }
      // inclusive scan over the warp's segments of this channel (lanes ch, ch+DT, ...)
      Aff inc = mine;
#pragma unroll
      for (int off = 1; off < Cfg::SPW; off <<= 1) {
        const float pa = __shfl_up_sync(0xffffffffu, inc.a, off * DT);
        const float pb = __shfl_up_sync(0xffffffffu, inc.b, off * DT);
        if (sl >= off) inc = aff_then(Aff{pa, pb}, inc);
      }
      // exclusive prefix inside the warp
      Aff exc{__shfl_up_sync(0xffffffffu, inc.a, DT), __shfl_up_sync(0xffffffffu, inc.b, DT)};
      if (sl == 0) exc = Aff{1.0f, 0.0f};
      if (sl == Cfg::SPW - 1) agg[warp * DT + ch] = inc;
      __syncthreads();

      float h = carry[ch];
      for (int w = 0; w < warp; ++w) {
        const Aff q = agg[w * DT + ch];
        h = fmaf(q.a, h, q.b);
      }
      h = fmaf(exc.a, h, exc.b);

#pragma unroll
      for (int j = 0; j < TS; ++j) {
        const int64_t l = l_begin + j;
        h = fmaf(a[j], h, bu[j]);
        if (l < L && d_ok) {
          const float yt = fmaf(cc[j], h, du[j]);
          float *dst = acc_base + ss2d_pixel(k, l, H, W) * acc_stride + (ACC_SMEM ? ch : ch);
          if (k == 0)
            *dst = yt;
          else
            *dst += yt;
        }
      }
      __syncthreads();
      if (warp == WARPS - 1 && sl == Cfg::SPW - 1) carry[ch] = h;
      // the next chunk reads carry only after its first barrier
    }
    __syncthreads();
  }

  // round once and store, channel-fastest
  for (int64_t q = tid; q < L * DT; q += Cfg::THREADS) {
    const int64_t pix = q / DT;
    const int c_ = (int)(q - pix * DT);
    if (d0 + c_ < d_in)
      Elem<T>::store(gy, (ib * L + pix) * d_in + d0 + c_, acc_base[pix * acc_stride + c_]);
  }
}

// ---------------------------------------------------------------------------
// CrossScan / CrossMerge as stored permutations (for checking the index
// arithmetic above bit-exactly).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void cross_scan_kernel(const T *u, T *xs, int64_t b, int64_t H, int64_t W,
                                  int64_t d_in) {
  const int64_t L = H * W;
  const int64_t total = b * 4 * L * d_in;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = i % d_in;
    const int64_t l = (i / d_in) % L;
    const int k = (int)((i / (d_in * L)) % 4);
    const int64_t ib = i / (d_in * L * 4);
    xs[i] = u[(ib * L + ss2d_pixel(k, l, H, W)) * d_in + d];
  }
}

template <typename T>
__global__ void cross_merge_kernel(const T *ys, T *y, int64_t b, int64_t H, int64_t W,
                                   int64_t d_in) {
  const int64_t L = H * W;
  const int64_t total = b * L * d_in;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = i % d_in;
    const int64_t pix = (i / d_in) % L;
    const int64_t ib = i / (d_in * L);
    // l_k(p): inverse of p_k.  Row-major index and column-major index of p.
    const int64_t hh = pix / W, ww = pix - (pix / W) * W;
    const int64_t l_rm = pix, l_cm = ww * H + hh;
    const int64_t l_of[4] = {l_rm, l_cm, L - 1 - l_rm, L - 1 - l_cm};
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      s += Elem<T>::load(ys, ((ib * 4 + k) * L + l_of[k]) * d_in + d);
    Elem<T>::store(y, i, s);
  }
}

}  // namespace ssm
