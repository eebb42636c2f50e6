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

#include <type_traits>

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
  // optional: the state at the start of every kStateChunk-step chunk,
  // (b, ceil(L / kStateChunk), d_in, N) fp32 (the backward scan's workspace)
  float *chunk_h = nullptr;
  // Sequence blocks of the split scan (scan_ws.cuh): grid z-index k covers
  // steps [k Lb, min(L, (k + 1) Lb)); Lb = 0 means one block.  blk_decay and
  // blk_state are (b, nblk, d_in, N) fp32: the summary pass leaves each
  // block's decay product and its end state from zero there, and the carry
  // pass overwrites blk_decay[k] with the state block k + 1 starts from.
  int64_t Lb = 0;
  float *blk_decay = nullptr;
  float *blk_state = nullptr;
};

// ---------------------------------------------------------------------------
// Generic kernel: one thread per (batch, channel), all N states in registers,
// sequential over t.  Any d_in, any alignment of the element type; used when
// the staged kernel's alignment conditions do not hold and for N < 8.
// ---------------------------------------------------------------------------
template <typename T, int N>
__global__ void __launch_bounds__(128) scan_generic_kernel(ScanParams p) {
  const int64_t bd = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (bd >= p.b * p.d_in || !in_bounds(bd * N + N - 1, p.b * p.d_in * N, kBndState)) return;
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

  const int64_t n_chunks = (p.L + kStateChunk - 1) / kStateChunk;
  for (int64_t t = 0; t < p.L; ++t) {
    if (p.chunk_h && t % kStateChunk == 0 &&
        in_bounds(((ib * n_chunks + t / kStateChunk) * p.d_in + d) * N + N - 1,
                  p.b * n_chunks * p.d_in * N, kBndChunk)) {
      float *dst = p.chunk_h + ((ib * n_chunks + t / kStateChunk) * p.d_in + d) * N;
#pragma unroll
      for (int n = 0; n < N; ++n) dst[n] = h[n];
    }
    const int64_t row = ib * p.L + t;
    const int64_t i = row * p.d_in + d;
    if (!in_bounds(i, p.b * p.L * p.d_in, kBndAct) || !in_bounds(row * N + N - 1, p.b * p.L * N, kBndBC))
      break;
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
// Fast kernel (d_state 64; d_state 8 to 32 take the warp-specialised kernel of
// scan_ws.cuh).  A CTA owns (batch i, a tile of DT channels) for the whole
// sequence and walks it in chunks of TC steps:
//   1. the chunk's u / delta / z tile [TC x DT] and B / C rows [TC x N] are
//      copied global -> shared with 16-byte cp.async, issued as soon as the
//      previous chunk's u / delta / z tile has been consumed (B / C rows,
//      which the scan reads, are double-buffered), so the copy overlaps that
//      chunk's scan;
//   2. pre-pass, one thread per (channel, 4 steps): delta = softplus(dt +
//      bias), delta u, u and silu(z) are formed once per (t, d) (not once per
//      state) and stored channel-major ([d][t], rows padded against bank
//      conflicts) so the scan reads 4 steps of a channel in one 16-byte
//      load.  Steps past the end of the sequence get delta = 0, which makes
//      them identity steps;
//   3. scan: the G = N / NPT threads of a channel split its states, NPT each,
//      and walk the chunk 4 steps per pass: first the pass's shared-memory
//      loads and its exponentials (which do not depend on the state), then
//      the recurrence h = dA h + delta u B and the C.h partial sums.  B and C
//      rows are read straight from the copied tile (bf16 words widened in
//      registers).  Per step and state
//      pair: a packed delta A log2 e, two exp2 (SFU, or the FMA-pipe
//      polynomial for the last NPOLY pairs), packed delta u * B, the packed
//      recurrence FMA and the packed C.h FMA.  Each thread writes its 4
//      partial C.h sums of a pass as one 16-byte store, one plane per state
//      group, so no cross-lane traffic sits on the recurrence's path;
//   4. post-pass, one thread per (channel, 4 steps): y = (sum of the G
//      partials + D u) silu(z), rounded once and stored (a warp writes whole
//      channel rows).
// Requires N % NPT == 0, TC % 8 == 0, d_in * sizeof(T) a multiple of 16 and
// u, delta, z, B, C, y 16-byte aligned (checked by the launcher).
// ---------------------------------------------------------------------------
// BCF: B and C rows widened to fp32 once per CTA in the pre-pass (instead of
// by every thread in the scan); the raw tile is then single-buffered.
template <typename T, int N, int NPT, int DT, int TC, bool BCF = false>
struct FastScan {
  static constexpr int G = N / NPT;             // threads per channel
  static constexpr int U = 4;                   // steps per scan pass
  static constexpr int THREADS = DT * G;
  static constexpr int ESZ = sizeof(T);
  static constexpr int VEC = 16 / ESZ;          // elements per 16-byte granule
  static constexpr int ROW_GRAN = DT / VEC;     // granules per tile row
  static constexpr int BC_GRAN = N / VEC;       // granules per B / C row
  static constexpr int TCP = TC + 4;            // padded channel-major row (floats)
  static constexpr int TILE = TC * DT * ESZ;
  static constexpr int BCT = TC * N * ESZ;
  static constexpr int OFF_U = 0;
  static constexpr int OFF_DT = OFF_U + TILE;
  static constexpr int OFF_Z = OFF_DT + TILE;
  static constexpr int OFF_B = OFF_Z + TILE;
  static constexpr int STAGES = BCF ? 1 : 2;            // raw B / C stages
  static constexpr int OFF_C = OFF_B + STAGES * BCT;
  static constexpr int OFF_BF = OFF_C + STAGES * BCT;    // float [TC][N] B, then C (BCF)
  static constexpr int BF_BYTES = BCF ? 2 * TC * N * 4 : 0;
  static constexpr int OFF_DLT = (OFF_BF + BF_BYTES + 15) / 16 * 16;  // float [DT][TCP]: delta
  static constexpr int OFF_DU = OFF_DLT + DT * TCP * 4;  // float [DT][TCP]: delta u
  static constexpr int OFF_UF = OFF_DU + DT * TCP * 4;   // float [DT][TCP]: u
  static constexpr int OFF_GT = OFF_UF + DT * TCP * 4;   // float [DT][TCP]: silu(z)
  // C.h partial sums, one plane per state group g: [g][DT][TCP].  Planes
  // are skewed so a quarter-warp's 16-byte accesses land in 8 distinct bank
  // groups both when the scan writes and when the post-pass reads.
  static constexpr int PADG = G >= 8 ? 4 : 32 / G;
  static constexpr int PLANE = DT * TCP + PADG;
  static constexpr int OFF_YS = OFF_GT + DT * TCP * 4;
  static constexpr int SMEM = OFF_YS + G * PLANE * 4;
  static_assert(NPT % 2 == 0 && N % NPT == 0 && G <= 32 && (32 % G) == 0, "bad NPT");
  static_assert(DT % VEC == 0 && N % VEC == 0, "tile rows must be whole granules");
  static_assert(THREADS % 32 == 0 && THREADS % DT == 0, "thread count");
  static_assert(TC % 8 == 0, "chunk length");
  static_assert(OFF_DLT % 16 == 0 && (PLANE * 4) % 16 == 0, "alignment");
};

// Raw words of NPT consecutive B / C entries (bf16 pairs, or fp32 values).
template <typename T, int NPT> struct StateWords {
  static constexpr int W = sizeof(T) == 2 ? NPT / 2 : NPT;
  uint32_t w[W];
  __device__ __forceinline__ void load(const T *row) {
    if constexpr (W == 1) {
      w[0] = *reinterpret_cast<const uint32_t *>(row);
    } else if constexpr (W == 2) {
      const uint2 q = *reinterpret_cast<const uint2 *>(row);
      w[0] = q.x; w[1] = q.y;
    } else {
#pragma unroll
      for (int i = 0; i < W; i += 4) {
        const uint4 q = *reinterpret_cast<const uint4 *>(row + i * 4 / sizeof(T));
        w[i] = q.x; w[i + 1] = q.y; w[i + 2] = q.z; w[i + 3] = q.w;
      }
    }
  }
  // entries 2k, 2k + 1 as a packed fp32 pair
  __device__ __forceinline__ float2 pair(int k) const {
    if constexpr (sizeof(T) == 2)
      return make_float2(bf16lo(w[k]), bf16hi(w[k]));
    else
      return make_float2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1]));
  }
};

// Everything stage 2 of a scan pass needs, produced by stage 1.
template <typename T, int NPT> struct PassBuf {
  float du[4];                      // delta u of the 4 steps
  float2 a[4][NPT / 2];             // exp2(delta A log2 e) per step and state pair
  StateWords<T, NPT> B[4], C[4];    // B, C entries of this thread's states
};

// SAVE: also store the state at every kStateChunk-step chunk start (p.chunk_h).
template <typename T, int N, int NPT, int DT, int TC, bool HAS_Z, int NPOLY, bool BCF, bool SAVE>
__global__ void __launch_bounds__(FastScan<T, N, NPT, DT, TC, BCF>::THREADS)
    scan_fast_kernel(ScanParams p) {
  using S = FastScan<T, N, NPT, DT, TC, BCF>;
  using TB = typename std::conditional<BCF, float, T>::type;  // element type the scan reads B / C in
  constexpr int G = S::G, THREADS = S::THREADS, NP2 = NPT / 2, TCP = S::TCP;
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
  float *sdl = reinterpret_cast<float *>(smem + S::OFF_DLT);
  float *sdu = reinterpret_cast<float *>(smem + S::OFF_DU);
  float *suf = reinterpret_cast<float *>(smem + S::OFF_UF);
  float *sgt = reinterpret_cast<float *>(smem + S::OFF_GT);
  float *sys = reinterpret_cast<float *>(smem + S::OFF_YS);
  float *sBf = reinterpret_cast<float *>(smem + S::OFF_BF);
  float *sCf = sBf + TC * N;

  auto prefetch = [&](int64_t t0, int stage) {
    for (int q = tid; q < TC * S::ROW_GRAN; q += THREADS) {
      const int t = q / S::ROW_GRAN, gq = q - t * S::ROW_GRAN;
      const int64_t dd = d0 + gq * S::VEC;
      const bool ok = (t0 + t < L) && (dd < d_in) &&
                      in_bounds((ib * L + t0 + t) * d_in + dd + S::VEC - 1, p.b * L * d_in, kBndAct);
      const int64_t off = ok ? ((ib * L + t0 + t) * d_in + dd) : 0;
      const int so = t * DT + gq * S::VEC;
      cp_async16(su + so, gu + off, ok ? 16 : 0);
      cp_async16(sdt + so, gdt + off, ok ? 16 : 0);
      if (HAS_Z) cp_async16(sz + so, gz + off, ok ? 16 : 0);
    }
    for (int q = tid; q < TC * S::BC_GRAN; q += THREADS) {
      const int t = q / S::BC_GRAN, gq = q - t * S::BC_GRAN;
      const bool ok =
          (t0 + t < L) && in_bounds((ib * L + t0 + t) * N + gq * S::VEC + S::VEC - 1, p.b * L * N, kBndBC);
      const int64_t off = ok ? ((ib * L + t0 + t) * N + gq * S::VEC) : 0;
      const int so = stage * TC * N + t * N + gq * S::VEC;
      cp_async16(sB + so, gB + off, ok ? 16 : 0);
      cp_async16(sC + so, gC + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // ---- pre/post-pass role: channel c (fixed per thread), 4-step groups
  const int c = tid % DT;
  const int sg0 = tid / DT;
  constexpr int SG_STRIDE = THREADS / DT;
  const int64_t dc = d0 + c;
  const bool c_ok = dc < d_in;
  const float bias = (c_ok && p.dt_bias) ? p.dt_bias[dc] : 0.0f;
  const float Dc = (c_ok && p.D) ? p.D[dc] : 0.0f;

  // ---- scan role: channel dl, states g*NPT .. g*NPT + NPT - 1
  const int dl = tid / G;
  const int g = tid - dl * G;
  const int64_t d = d0 + dl;
  const bool d_ok = d < d_in;
  float2 A2[NP2], h[NP2];
#pragma unroll
  for (int k = 0; k < NP2; ++k) {
    const int n = g * NPT + 2 * k;
    A2[k] = d_ok ? make_float2(p.A[d * N + n] * kLog2e, p.A[d * N + n + 1] * kLog2e)
                 : make_float2(0.0f, 0.0f);
    const float *h0 = p.h0 + (ib * d_in + d) * N + n;
    h[k] = (d_ok && p.h0) ? make_float2(h0[0], h0[1]) : make_float2(0.0f, 0.0f);
  }
  const float *rdl = sdl + dl * TCP;
  const float *rdu = sdu + dl * TCP;
  float *ys_own = sys + g * S::PLANE + dl * TCP;

  // stage 1 of a pass: loads and exponentials (independent of the state)
  auto stage1 = [&](int t, const TB *cB, const TB *cC, PassBuf<TB, NPT> &pb) {
    const float4 dv = *reinterpret_cast<const float4 *>(rdl + t);
    const float4 uv = *reinterpret_cast<const float4 *>(rdu + t);
    const float dd[4] = {dv.x, dv.y, dv.z, dv.w};
    pb.du[0] = uv.x; pb.du[1] = uv.y; pb.du[2] = uv.z; pb.du[3] = uv.w;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      pb.B[s].load(cB + (t + s) * N + g * NPT);
      pb.C[s].load(cC + (t + s) * N + g * NPT);
      const float2 d2 = make_float2(dd[s], dd[s]);
#pragma unroll
      for (int k = 0; k < NP2; ++k) {
        const float2 x = __fmul2_rn(d2, A2[k]);
        pb.a[s][k] = (k >= NP2 - NPOLY) ? exp2_poly2(x) : exp2_sfu2(x);
      }
    }
  };
  // stage 2 of a pass: the recurrence and the partial C.h sums
  auto stage2 = [&](int t, const PassBuf<TB, NPT> &pb) {
    float ys[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float2 u2 = make_float2(pb.du[s], pb.du[s]);
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int k = 0; k < NP2; ++k) {
        h[k] = __ffma2_rn(pb.a[s][k], h[k], __fmul2_rn(u2, pb.B[s].pair(k)));
        acc = __ffma2_rn(h[k], pb.C[s].pair(k), acc);
      }
      ys[s] = acc.x + acc.y;
    }
    *reinterpret_cast<float4 *>(ys_own + t) = make_float4(ys[0], ys[1], ys[2], ys[3]);
  };

  const int64_t nchunks = (L + TC - 1) / TC;
  const int64_t n_saved = (L + kStateChunk - 1) / kStateChunk;
  static_assert(TC % kStateChunk == 0, "saved chunk starts fall on pass boundaries");
  prefetch(0, 0);
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int stage = S::STAGES == 2 ? (int)(ch & 1) : 0;
    const T *rB = sB + stage * TC * N;  // raw (copied) B / C rows of this chunk
    const T *rC = sC + stage * TC * N;
    const TB *cB, *cC;                  // the rows the scan reads
    if constexpr (BCF) {
      cB = sBf;
      cC = sCf;
    } else {
      cB = rB;
      cC = rC;
    }
    const int64_t t0 = ch * TC;
    const int tc = (int)((L - t0) < (int64_t)TC ? (L - t0) : (int64_t)TC);
    cp_async_wait<0>();
    __syncthreads();  // raw tiles of this chunk visible; previous post-pass done

    // ---- pre-pass: per (channel, 4 steps)
    for (int sg = sg0; sg < TC / 4; sg += SG_STRIDE) {
      float dv[4], duv[4], uv[4], gv[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int t = sg * 4 + s;
        const float ut = Elem<T>::load(su, t * DT + c);
        float e = Elem<T>::load(sdt, t * DT + c) + bias;
        if (p.delta_softplus) e = softplus_f32(e);
        e = t < tc ? e : 0.0f;  // identity step past the end
        dv[s] = e;
        duv[s] = e * ut;
        uv[s] = ut;
        gv[s] = HAS_Z ? silu_for<T>(Elem<T>::load(sz, t * DT + c)) : 1.0f;
      }
      const int o = c * TCP + sg * 4;
      *reinterpret_cast<float4 *>(sdl + o) = make_float4(dv[0], dv[1], dv[2], dv[3]);
      *reinterpret_cast<float4 *>(sdu + o) = make_float4(duv[0], duv[1], duv[2], duv[3]);
      *reinterpret_cast<float4 *>(suf + o) = make_float4(uv[0], uv[1], uv[2], uv[3]);
      *reinterpret_cast<float4 *>(sgt + o) = make_float4(gv[0], gv[1], gv[2], gv[3]);
    }
    if constexpr (BCF) {
      for (int q = tid; q < TC * N / 2; q += THREADS) {
        const uint32_t wb = reinterpret_cast<const uint32_t *>(rB)[q];
        const uint32_t wc = reinterpret_cast<const uint32_t *>(rC)[q];
        reinterpret_cast<float2 *>(sBf)[q] = make_float2(bf16lo(wb), bf16hi(wb));
        reinterpret_cast<float2 *>(sCf)[q] = make_float2(bf16lo(wc), bf16hi(wc));
      }
    }
    __syncthreads();  // delta, delta u, u, gate (and fp32 B / C) ready; raw tiles consumed

    if (ch + 1 < nchunks) prefetch(t0 + TC, S::STAGES == 2 ? stage ^ 1 : 0);  // overlaps the scan

    // ---- scan over the chunk, 4 steps per pass
    const int tcr = (tc + 3) / 4 * 4;
    for (int t = 0; t < tcr; t += 4) {
      if (SAVE && (t % kStateChunk) == 0 && t < tc && d_ok &&
          in_bounds(((ib * n_saved + (t0 + t) / kStateChunk) * d_in + d) * N + g * NPT + NPT - 1,
                    p.b * n_saved * d_in * N, kBndChunk)) {  // a saved chunk start
        float2 *dst = reinterpret_cast<float2 *>(
            p.chunk_h + ((ib * n_saved + (t0 + t) / kStateChunk) * d_in + d) * N + g * NPT);
#pragma unroll
        for (int k = 0; k < NP2; ++k) dst[k] = h[k];
      }
      PassBuf<TB, NPT> pb;
      stage1(t, cB, cC, pb);
      stage2(t, pb);
    }
    __syncthreads();  // partial sums of the chunk complete

    // ---- post-pass: sum of the partials, D skip, gate, one rounding
    if (c_ok) {
      for (int sg = sg0; sg * 4 < tc; sg += SG_STRIDE) {
        const int o = c * TCP + sg * 4;
        const float4 u4 = *reinterpret_cast<const float4 *>(suf + o);
        const float4 g4 = *reinterpret_cast<const float4 *>(sgt + o);
        float4 y4 = *reinterpret_cast<const float4 *>(sys + o);
#pragma unroll
        for (int q = 1; q < G; ++q) {
          const float4 v = *reinterpret_cast<const float4 *>(sys + q * S::PLANE + o);
          y4.x += v.x; y4.y += v.y; y4.z += v.z; y4.w += v.w;
        }
        const float uu[4] = {u4.x, u4.y, u4.z, u4.w}, gg[4] = {g4.x, g4.y, g4.z, g4.w};
        const float yy[4] = {y4.x, y4.y, y4.z, y4.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int t = sg * 4 + s;
          if (t < tc && in_bounds((ib * L + t0 + t) * d_in + dc, p.b * L * d_in, kBndAct))
            Elem<T>::store(gy, (ib * L + t0 + t) * d_in + dc, fmaf(Dc, uu[s], yy[s]) * gg[s]);
        }
      }
    }
  }

  if (p.h_last && d_ok && in_bounds((ib * d_in + d) * N + g * NPT + NPT - 1, p.b * d_in * N, kBndState)) {
    float *hl = p.h_last + (ib * d_in + d) * N + g * NPT;
#pragma unroll
    for (int k = 0; k < NP2; ++k) {
      hl[2 * k] = h[k].x;
      hl[2 * k + 1] = h[k].y;
    }
  }
}

}  // namespace ssm
