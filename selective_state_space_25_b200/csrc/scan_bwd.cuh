// scan_bwd.cuh -- backward of the selective scan: the reverse-time adjoint
// of the recurrence of "手把手拆解Mamba-minimal中的selective_scan实现" §3-§5
// with the gate of "代码连连看——mamba" (Mamba.step()); the fast backward
// the VMamba discussion ("关于代码SS2D中的d_state设置") asks of a scan kernel.
//
// For one (batch, channel), with delta_t = softplus(dt_t + bias),
// a_t = exp(delta_t A) and h_t the state after step t:
//     lam   <- lam + g_t C_t                   g_t = dout_t silu(z_t)
//     dC_t  += g_t h_t          dD += g_t u_t   dz_t = dout_t yp_t silu'(z_t)
//     ddelta_t = softplus'(.) (sum_n A lam a_t h_{t-1} + u_t sum_n lam B_t)
//     dA    += lam delta_t a_t h_{t-1}
//     dB_t  += lam delta_t u_t  du_t = g_t D + delta_t sum_n lam B_t
//     lam   <- lam a_t                          (dh0 = lam at the end)
//
// One CTA owns DT channels of one batch for the whole sequence; G = N / NPT
// threads share a channel, NPT states each.
//   pass 1  walks the sequence forwards and saves the state at the start of
//           every TT-step chunk in the caller's workspace (skipped when the
//           forward already saved them there: states_saved);
//   pass 2  walks the chunks backwards.  Per chunk: recompute the states
//           from the saved start into registers, writing each thread's
//           partial C.h and its terms g_t h_t of dC_t as shared rows;
//           dC_t = the sum of those rows over the channels (a column pass);
//           the adjoint, taking h_{t-1} from registers, which writes the
//           terms lam_t delta_t u_t of dB_t into the rows and leaves each
//           thread's partial sums of lam B and A lam a h_{t-1}; dB_t as a
//           second column sum; and a pass per (step, channel) that adds the
//           G partials and writes du, ddelta and dz.
// A chunk's inputs are copied into shared memory one chunk ahead (cp.async)
// when they are 16-byte aligned.  Nothing in the per-step loops crosses
// lanes, so each step's critical
// path is the adjoint's own FMA chain.  dB and dC rows of the chunk go to
// the fp32 outputs with (vector) global atomics, one per CTA and row;
// dA, dD and ddt_bias are added once per CTA at the end.
#pragma once

#include "ssm_common.cuh"

namespace ssm {

struct BwdParams {
  const void *u, *delta;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *dt_bias;
  const float *h0;
  const void *dout;
  const float *dh_last;
  void *du, *ddelta, *dz;
  float *dA, *dB, *dC, *dD, *ddt_bias, *dh0;
  float *chunk_h;  // workspace (b, n_chunks, d_in, N) fp32
  int64_t b, L, d_in;
  int softplus;
  int vec_atomics;   // dB and dC 16-byte aligned: float4 atomics
  int states_saved;  // chunk_h already holds the chunk-start states (saved by the forward)
  // Split backward (few channels): grid z-index k walks chunks
  // [k Cb, min(nC, (k + 1) Cb)) from the adjoint lam_in holds for it
  // (scan_bwd_adjoint_kernel + scan_carry_kernel); Cb = 0 means one block.
  // Needs states_saved.
  int64_t Cb = 0;
  const float *lam_in = nullptr;  // (b, nblk, d_in, N): block k's start at slot nblk - 2 - k
};

template <typename T, int N, int NPT_>
struct BwdCfg {
  static constexpr int NPT = NPT_;           // states per thread
  static constexpr int G = N / NPT;          // threads per channel
  static constexpr int THREADS = 128;
  static constexpr int DT = THREADS / G;     // channels per CTA
  static constexpr int TT = kStateChunk;     // steps per chunk
  static constexpr int PROW = DT + 1;        // plane row (padded: column reads hit distinct banks)
  static constexpr int PL = TT * PROW;       // one (step, channel) plane
  // state row, padded so the column passes' vector reads of 4 (NPT 2) or 2
  // (NPT 4) step rows per wavefront fall in distinct banks
  static constexpr int HROW = THREADS * NPT + (NPT == 1 ? 1 : 16);
  // raw input tiles of one chunk (cp.async targets): u, delta, z, dout
  // [TT][DT] and B, C [TT][N] in the activation dtype; two of them
  static constexpr int RAW_ACT = TT * DT, RAW_BC = TT * N;
  static constexpr int RAW_BYTES = ((4 * RAW_ACT + 2 * RAW_BC) * (int)sizeof(T) + 15) / 16 * 16;
  static constexpr int OFF_F = 2 * RAW_BYTES / 4;  // first float after the raw tiles
  // planes: {delta, delta u, g, u} as one 16-byte entry, then the dz factor
  // and softplus' (one float each)
  static constexpr int OFF_Q = OFF_F;
  static constexpr int OFF_DZF = OFF_Q + 4 * PL;
  static constexpr int OFF_SPG = OFF_DZF + PL;
  static constexpr int OFF_BC = (OFF_SPG + PL + 3) / 4 * 4;  // {B, C} pairs [t][n]
  static constexpr int OFF_P1 = OFF_BC + 2 * TT * N;     // partial sum_n lam B      [t][thread]
  static constexpr int OFF_P2 = OFF_P1 + TT * THREADS;  // partial sum_n A lam a h [t][thread]
  static constexpr int OFF_PY = OFF_P2 + TT * THREADS;  // partial C.h             [t][thread]
  static constexpr int OFF_H = (OFF_PY + TT * THREADS + 3) / 4 * 4;  // states, then adjoints
  static constexpr int FLOATS = OFF_H + TT * HROW;
  static constexpr size_t SMEM = FLOATS * sizeof(float);
  static_assert(N % NPT == 0 && (NPT == 1 || NPT == 2 || NPT == 4), "bad NPT");
  static_assert(G >= 1 && G <= 32 && 32 % G == 0 && THREADS % DT == 0, "bad N / NPT");
};

// The cp.async staging copies whole 16-byte groups of a CTA's channel run
// and of a B / C row.
template <typename T, int N, int NPT>
__host__ __device__ constexpr bool bwd_async_ok() {
  return BwdCfg<T, N, NPT>::DT % (16 / (int)sizeof(T)) == 0 && N % (16 / (int)sizeof(T)) == 0;
}

template <int NPT>
__device__ __forceinline__ void load_vec(const float *s, float (&v)[NPT]) {
  if constexpr (NPT == 4) {
    const float4 w = *reinterpret_cast<const float4 *>(s);
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
  } else if constexpr (NPT == 2) {
    const float2 w = *reinterpret_cast<const float2 *>(s);
    v[0] = w.x; v[1] = w.y;
  } else {
#pragma unroll
    for (int j = 0; j < NPT; ++j) v[j] = s[j];
  }
}

template <int NPT>
__device__ __forceinline__ void store_vec(float *s, const float (&v)[NPT]) {
  if constexpr (NPT == 4) {
    *reinterpret_cast<float4 *>(s) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (NPT == 2) {
    *reinterpret_cast<float2 *>(s) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int j = 0; j < NPT; ++j) s[j] = v[j];
  }
}

// B and C of NPT consecutive states from {B, C} pairs.
template <int NPT>
__device__ __forceinline__ void load_bc(const float *s, float (&b)[NPT], float (&c)[NPT]) {
  if constexpr (NPT == 1) {
    const float2 w = *reinterpret_cast<const float2 *>(s);
    b[0] = w.x; c[0] = w.y;
  } else {
#pragma unroll
    for (int k = 0; k < NPT; k += 2) {
      const float4 w = *reinterpret_cast<const float4 *>(s + 2 * k);
      b[k] = w.x; c[k] = w.y; b[k + 1] = w.z; c[k + 1] = w.w;
    }
  }
}

// Sum of the G consecutive partials starting at s, read by the lane of
// channel pch.  With more than one 16-byte group per lane the lanes start at
// rotated groups, so the eight lanes of a quarter warp (G floats apart) hit
// eight different bank groups.
template <int G>
__device__ __forceinline__ float sum_partials(const float *s, int pch) {
  float acc = 0.0f;
  if constexpr (G % 4 == 0) {
    constexpr int M = G / 4;  // 16-byte groups per lane
    const int rot = M > 1 ? (pch >> (M >= 8 ? 0 : (M == 4 ? 1 : 2))) & (M - 1) : 0;
#pragma unroll
    for (int k = 0; k < M; ++k) {
      const float4 w = *reinterpret_cast<const float4 *>(s + 4 * ((k + rot) & (M - 1)));
      acc += (w.x + w.y) + (w.z + w.w);
    }
  } else if constexpr (G == 2) {
    const float2 w = *reinterpret_cast<const float2 *>(s);
    acc = w.x + w.y;
  } else {
    acc = s[0];
  }
  return acc;
}

template <typename T, int N, int NPT_, bool ASYNC>
__global__ void __launch_bounds__(128, 3) scan_bwd_kernel(BwdParams p) {
  using Cfg = BwdCfg<T, N, NPT_>;
  constexpr int NPT = Cfg::NPT, G = Cfg::G, DT = Cfg::DT, TT = Cfg::TT, NT = Cfg::THREADS;
  constexpr int PROW = Cfg::PROW, HROW = Cfg::HROW;
  static_assert(!ASYNC || bwd_async_ok<T, N, NPT_>(), "raw tiles need whole 16-byte groups");
  extern __shared__ float4 bwd_smem4[];
  float *sm = reinterpret_cast<float *>(bwd_smem4);
  float4 *sQ = reinterpret_cast<float4 *>(sm + Cfg::OFF_Q);
  float *sDzf = sm + Cfg::OFF_DZF, *sSpg = sm + Cfg::OFF_SPG;
  float *sBC = sm + Cfg::OFF_BC;
  float *sP1 = sm + Cfg::OFF_P1, *sP2 = sm + Cfg::OFF_P2, *sPy = sm + Cfg::OFF_PY;
  float *sH = sm + Cfg::OFF_H;

  const int tid = threadIdx.x;
  const int ch = tid / G, g = tid - (tid / G) * G;
  const int64_t ib = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * DT;
  const int64_t d = d0 + ch;
  const bool active = d < p.d_in;
  const int64_t L = p.L, d_in = p.d_in;
  const int nC = (int)((L + TT - 1) / TT);
  // this CTA's chunks [c_begin, c_end) (all of them without the split)
  const int blk = (int)blockIdx.z;
  const int nblk = p.Cb > 0 ? (int)((nC + p.Cb - 1) / p.Cb) : 1;
  const int c_begin = p.Cb > 0 ? blk * (int)p.Cb : 0;
  const int c_end = p.Cb > 0 && c_begin + p.Cb < nC ? c_begin + (int)p.Cb : nC;
  const T *gu = static_cast<const T *>(p.u);
  const T *gdelta = static_cast<const T *>(p.delta);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  const T *gz = static_cast<const T *>(p.z);
  const T *gdout = static_cast<const T *>(p.dout);

  float Av[NPT], A2[NPT];
#pragma unroll
  for (int j = 0; j < NPT; ++j) {
    Av[j] = active ? p.A[d * N + g * NPT + j] : 0.0f;
    A2[j] = Av[j] * kLog2e;
  }

  // staging keeps one channel per thread (NT is a multiple of DT)
  const float sbias = (p.dt_bias && d0 + tid % DT < d_in) ? p.dt_bias[d0 + tid % DT] : 0.0f;

  auto rows_of = [&](int c) { return (int)(L - (int64_t)c * TT < TT ? L - (int64_t)c * TT : TT); };

  // --- raw tiles (ASYNC): chunk c's inputs copied as they are, 16 bytes at
  // a time; rows past the sequence and channels past d_in are zero-filled.
  auto raw_base = [&](int buf) {
    return reinterpret_cast<T *>(reinterpret_cast<char *>(bwd_smem4) + buf * Cfg::RAW_BYTES);
  };
  auto issue = [&](int c, bool full, int buf) {
    constexpr int EPG = 16 / (int)sizeof(T);  // elements per 16-byte group
    // groups per activation row and per B / C row (>= 1 so instantiations
    // that never stage asynchronously still compile cleanly)
    constexpr int GA = DT / EPG > 0 ? DT / EPG : 1;
    constexpr int GB = N / EPG > 0 ? N / EPG : 1;
    T *raw = raw_base(buf);
    const int64_t t0 = (int64_t)c * TT;
    const int nT = rows_of(c);
    const int ntens = full ? 4 : 2;  // u, delta [, z, dout]
    for (int i = tid; i < ntens * TT * GA; i += NT) {
      const int k = i / (TT * GA), r = (i / GA) % TT, q = i % GA;
      const T *src = k == 0 ? gu : k == 1 ? gdelta : k == 2 ? (gz ? gz : gdout) : gdout;
      const int64_t col = d0 + q * EPG;
      const bool ok = r < nT && col < d_in && (k != 2 || gz) &&
                      in_bounds((ib * L + t0 + r) * d_in + col + EPG - 1, p.b * L * d_in, kBndAct);
      const T *gp = ok ? src + (ib * L + t0 + r) * d_in + col : src;
      cp_async16(raw + k * Cfg::RAW_ACT + r * DT + q * EPG, gp, ok ? 16 : 0);
    }
    for (int i = tid; i < (full ? 2 : 1) * TT * GB; i += NT) {
      const int k = i / (TT * GB), r = (i / GB) % TT, q = i % GB;
      const T *src = k == 0 ? gB : gC;
      const bool ok =
          r < nT && in_bounds((ib * L + t0 + r) * N + q * EPG + EPG - 1, p.b * L * N, kBndBC);
      const T *gp = ok ? src + (ib * L + t0 + r) * N + q * EPG : src;
      cp_async16(raw + 4 * Cfg::RAW_ACT + k * Cfg::RAW_BC + r * N + q * EPG, gp, ok ? 16 : 0);
    }
  };

  // Chunk c's (step, channel) inputs into the planes; with `full` also the
  // gate terms and C.  Rows past the sequence and channels past d_in are 0.
  // ASYNC reads the raw tile in smem buffer `buf`, else global memory.
  auto stage = [&](int c, bool full, int buf) {
    const int64_t t0 = (int64_t)c * TT;
    const int nT = rows_of(c);
    const T *raw = raw_base(buf);
    for (int i = tid; i < TT * DT; i += NT) {
      const int t = i / DT, cc = i - t * DT;
      const int64_t dd = d0 + cc;
      float dl = 0.0f, uu = 0.0f, gg = 0.0f, dzf = 0.0f, spg = 0.0f;
      if (t < nT && dd < d_in && in_bounds((ib * L + t0 + t) * d_in + dd, p.b * L * d_in, kBndAct)) {
        const int64_t at = (ib * L + t0 + t) * d_in + dd;
        const int ra = t * DT + cc;
        const float pre =
            (ASYNC ? Elem<T>::load(raw + Cfg::RAW_ACT, ra) : Elem<T>::load(gdelta, at)) + sbias;
        uu = ASYNC ? Elem<T>::load(raw, ra) : Elem<T>::load(gu, at);
        if (p.softplus) {
          dl = softplus_f32(pre);
          if (full) spg = pre > 20.0f ? 1.0f : rcp_approx(1.0f + ex2_approx(-pre * kLog2e));
        } else {
          dl = pre;
          spg = 1.0f;
        }
        if (full) {
          const float go =
              ASYNC ? Elem<T>::load(raw + 3 * Cfg::RAW_ACT, ra) : Elem<T>::load(gdout, at);
          if (gz) {
            const float zz =
                ASYNC ? Elem<T>::load(raw + 2 * Cfg::RAW_ACT, ra) : Elem<T>::load(gz, at);
            const float sg = rcp_approx(1.0f + ex2_approx(-zz * kLog2e));
            gg = go * zz * sg;
            dzf = go * sg * fmaf(zz, 1.0f - sg, 1.0f);
          } else {
            gg = go;
          }
        }
      }
      const int s = t * PROW + cc;
      sQ[s] = make_float4(dl, dl * uu, gg, uu);
      if (full) {
        sDzf[s] = dzf;
        sSpg[s] = spg;
      }
    }
    for (int i = tid; i < TT * N; i += NT) {
      const int t = i / N;
      const int64_t row = (ib * L + t0 + t) * N + (i - t * N);
      float bb, cc = 0.0f;
      if constexpr (ASYNC) {  // zero-filled past the sequence already
        bb = Elem<T>::load(raw + 4 * Cfg::RAW_ACT, i);
        if (full) cc = Elem<T>::load(raw + 4 * Cfg::RAW_ACT + Cfg::RAW_BC, i);
      } else {
        bb = t < nT ? Elem<T>::load(gB, row) : 0.0f;
        if (full) cc = t < nT ? Elem<T>::load(gC, row) : 0.0f;
      }
      *reinterpret_cast<float2 *>(sBC + 2 * i) = make_float2(bb, cc);
    }
    return nT;
  };

  float *my_chunk_h = p.chunk_h + ((ib * nC) * d_in + d) * N + g * NPT;  // + c * d_in * N
  // chunk c's saved state of this thread lies inside the workspace
  auto chunk_ok = [&](int64_t c) {
    return in_bounds(((ib * nC + c) * d_in + d) * N + g * NPT + NPT - 1, p.b * nC * d_in * N,
                     kBndChunk);
  };
  float h[NPT];

  // one forward step of this thread's states (pass 1 and the recompute)
  auto fwd_step = [&](int t) -> float {
    const float4 q = sQ[t * PROW + ch];
    const float dl = q.x, du = q.y;
    float bv[NPT], cv[NPT];
    load_bc<NPT>(sBC + 2 * (t * N + g * NPT), bv, cv);
    float yp = 0.0f;
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
      h[j] = fmaf(ex2_approx(dl * A2[j]), h[j], du * bv[j]);
      yp = fmaf(h[j], cv[j], yp);
    }
    return yp;
  };

  // the same, also handing back g_t of this thread's channel
  auto fwd_step_g = [&](int t, float &gt) -> float {
    const float4 q = sQ[t * PROW + ch];
    const float dl = q.x, du = q.y;
    gt = q.z;
    float bv[NPT], cv[NPT];
    load_bc<NPT>(sBC + 2 * (t * N + g * NPT), bv, cv);
    float yp = 0.0f;
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
      h[j] = fmaf(ex2_approx(dl * A2[j]), h[j], du * bv[j]);
      yp = fmaf(h[j], cv[j], yp);
    }
    return yp;
  };

  // ---------------- pass 1: chunk-start states, forwards (unless saved)
  const int n_pass1 = p.states_saved ? 0 : nC;
#pragma unroll
  for (int j = 0; j < NPT; ++j)
    h[j] = (active && p.h0) ? p.h0[(ib * d_in + d) * N + g * NPT + j] : 0.0f;
  if constexpr (ASYNC) {
    // chunks 0 .. nC-2 (partial input), then the first chunk of pass 2 (full)
    if (n_pass1 >= 2) issue(0, false, 0); else issue(c_end - 1, true, (c_end - 1) & 1);
    cp_async_commit();
  }
  for (int c = 0; c < n_pass1; ++c) {
    if (active && chunk_ok(c)) store_vec<NPT>(my_chunk_h + (int64_t)c * d_in * N, h);
    if (c == nC - 1) break;  // the last chunk's end state is not needed
    if constexpr (ASYNC) {
      if (c + 1 <= nC - 2) issue(c + 1, false, (c + 1) & 1);
      else issue(nC - 1, true, (nC - 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
    }
    __syncthreads();
    stage(c, false, c & 1);  // a chunk before the last is full
    __syncthreads();
#pragma unroll
    for (int t = 0; t < TT; ++t) (void)fwd_step(t);
  }

  // ---------------- pass 2: adjoint, chunks backwards
  float lam[NPT], dAacc[NPT];
#pragma unroll
  for (int j = 0; j < NPT; ++j) {
    if (blk == nblk - 1) {  // the last block starts from dh_last
      lam[j] = (active && p.dh_last) ? p.dh_last[(ib * d_in + d) * N + g * NPT + j] : 0.0f;
    } else {  // an earlier one from the adjoint its right-hand blocks leave
      const int64_t i = ((ib * nblk + (nblk - 2 - blk)) * d_in + d) * N + g * NPT + j;
      lam[j] = active && in_bounds(i, p.b * nblk * d_in * N, kBndChunk) ? p.lam_in[i] : 0.0f;
    }
    dAacc[j] = 0.0f;
  }
  // the per-(step, channel) pass keeps one channel per thread
  const int pch = tid % DT;
  const float pD = (d0 + pch < d_in && p.D) ? p.D[d0 + pch] : 0.0f;
  float Dacc = 0.0f, bias_acc = 0.0f;

  // one adjoint step; hp = h_{t-1} (this thread's states before step t).
  // The chunk's row t receives lam_t delta_t u_t, this channel's terms of dB_t.
  auto adj_step_h = [&](int t, const float (&hp)[NPT]) {
    const float4 qv = sQ[t * PROW + ch];
    const float gt = qv.z, dl = qv.x, du = qv.y;
    float bv[NPT], cv[NPT], lt[NPT];
    load_bc<NPT>(sBC + 2 * (t * N + g * NPT), bv, cv);
    float S1 = 0.0f, S2 = 0.0f;
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
      lam[j] = fmaf(gt, cv[j], lam[j]);
      lt[j] = lam[j] * du;
      const float la = lam[j] * ex2_approx(dl * A2[j]);
      const float q = la * hp[j];
      S2 = fmaf(Av[j], q, S2);
      S1 = fmaf(lam[j], bv[j], S1);
      dAacc[j] = fmaf(q, dl, dAacc[j]);
      lam[j] = la;
    }
    store_vec<NPT>(sH + t * HROW + tid * NPT, lt);
    sP1[t * NT + tid] = S1;
    sP2[t * NT + tid] = S2;
  };
  // sum over the CTA's channels of the chunk's rows X[t][ch][n] for every
  // (t, n); added to out (b, L, N) rows t0 .. t0+nT-1
  auto column_pass = [&](float *out, int64_t t0, int nT) {
    for (int o = tid; o < TT * G; o += NT) {
      const int t = o / G, gi = o - (o / G) * G;
      float acc[NPT];
#pragma unroll
      for (int j = 0; j < NPT; ++j) acc[j] = 0.0f;
      const float *xs = sH + t * HROW + gi * NPT;
#pragma unroll 8
      for (int cc = 0; cc < DT; ++cc) {
        float x[NPT];
        load_vec<NPT>(xs + cc * G * NPT, x);
#pragma unroll
        for (int j = 0; j < NPT; ++j) acc[j] += x[j];
      }
      if (t < nT && in_bounds((ib * L + t0 + t) * N + gi * NPT + NPT - 1, p.b * L * N, kBndBC)) {
        float *dst = out + (ib * L + t0 + t) * N + gi * NPT;
        if (p.vec_atomics) {
          if constexpr (NPT == 4) {
            atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(acc[0], acc[1], acc[2], acc[3]));
            continue;
          } else if constexpr (NPT == 2) {
            atomicAdd(reinterpret_cast<float2 *>(dst), make_float2(acc[0], acc[1]));
            continue;
          }
        }
#pragma unroll
        for (int j = 0; j < NPT; ++j) atomicAdd(dst + j, acc[j]);
      }
    }
  };

  float hs_next[NPT];
  if (active && chunk_ok(c_end - 1))
    load_vec<NPT>(my_chunk_h + (int64_t)(c_end - 1) * d_in * N, hs_next);
  for (int c = c_end - 1; c >= c_begin; --c) {
    float hs[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) hs[j] = active ? hs_next[j] : 0.0f;
    if (c > c_begin && active && chunk_ok(c - 1))
      load_vec<NPT>(my_chunk_h + (int64_t)(c - 1) * d_in * N, hs_next);
    if constexpr (ASYNC) {
      if (c > c_begin) issue(c - 1, true, (c - 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
    }
    __syncthreads();  // the previous chunk's planes have been read; this chunk's tile landed
    const int nT = stage(c, true, c & 1);
    const int64_t t0 = (int64_t)c * TT;
    __syncthreads();

    // recompute the chunk's states (kept in registers for the adjoint) and
    // the partial pre-gate outputs; row t of the chunk receives g_t h_t, this
    // channel's terms of dC_t.  A chunk past the end of the sequence runs
    // identity steps there (delta, delta u and g are staged as 0), so every
    // chunk takes the same unrolled path; outputs stop at nT.
    float hreg[TT][NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) h[j] = hs[j];
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      float gt;
      sPy[t * NT + tid] = fwd_step_g(t, gt);
      float pc[NPT];
#pragma unroll
      for (int j = 0; j < NPT; ++j) {
        hreg[t][j] = h[j];
        pc[j] = gt * h[j];
      }
      store_vec<NPT>(sH + t * HROW + tid * NPT, pc);
    }
    __syncthreads();
    column_pass(p.dC, t0, nT);  // dC_t = sum_ch g_t h_t
    __syncthreads();

    // the adjoint through the chunk (rows become lam_t delta_t u_t)
#pragma unroll
    for (int t = TT - 1; t >= 1; --t) adj_step_h(t, hreg[t - 1]);
    adj_step_h(0, hs);
    __syncthreads();
    column_pass(p.dB, t0, nT);  // dB_t = sum_ch lam_t delta_t u_t

    // per (step, channel): add the partials, write du, ddelta, dz
    for (int i = tid; i < TT * DT; i += NT) {
      const int t = i / DT;  // i % DT == pch
      const int64_t dd = d0 + pch;
      const int s = t * PROW + pch;
      const float S1 = sum_partials<G>(sP1 + t * NT + pch * G, pch);
      const float S2 = sum_partials<G>(sP2 + t * NT + pch * G, pch);
      const float yp = sum_partials<G>(sPy + t * NT + pch * G, pch);
      const float4 qv = sQ[s];
      const float gt = qv.z, dl = qv.x, uu = qv.w;
      const float ddt = fmaf(uu, S1, S2) * sSpg[s];
      if (t < nT && dd < d_in && in_bounds((ib * L + t0 + t) * d_in + dd, p.b * L * d_in, kBndAct)) {
        const int64_t at = (ib * L + t0 + t) * d_in + dd;
        Elem<T>::store(static_cast<T *>(p.du), at, fmaf(gt, pD, dl * S1));
        Elem<T>::store(static_cast<T *>(p.ddelta), at, ddt);
        if (gz && p.dz) Elem<T>::store(static_cast<T *>(p.dz), at, sDzf[s] * fmaf(pD, uu, yp));
        bias_acc += ddt;
        Dacc = fmaf(gt, uu, Dacc);
      }
    }
  }
  if constexpr (ASYNC) cp_async_wait<0>();  // nothing may be in flight at exit

  if (active && in_bounds(d * N + g * NPT + NPT - 1, d_in * N, kBndParam) &&
      in_bounds((ib * d_in + d) * N + g * NPT + NPT - 1, p.b * d_in * N, kBndState)) {
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
      atomicAdd(p.dA + d * N + g * NPT + j, dAacc[j]);
      if (p.dh0 && blk == 0) p.dh0[(ib * d_in + d) * N + g * NPT + j] = lam[j];
    }
  }
  if (d0 + pch < d_in) {
    if (p.dD) atomicAdd(p.dD + d0 + pch, Dacc);
    if (p.ddt_bias) atomicAdd(p.ddt_bias + d0 + pch, bias_acc);
  }
}

// Adjoint summary of the split backward.  Block k >= 1 of the sequence
// (chunks [k Cb, min(nC, (k + 1) Cb))) maps the adjoint arriving at its last
// step, lam_in, to the one leaving its first step: lam_out = M_k lam_in + R_k
// (per (batch, channel, state)), with M_k = prod_t exp(delta_t A) and R_k the
// adjoint walked backwards through the block from zero, lam <- (lam + g_t C_t)
// exp(delta_t A) -- scan_bwd_kernel's adjoint step, g_t = dout_t silu(z_t).
// M_k and R_k go to slot nblk - 1 - k of (b, nblk, d_in, N) arrays, the order
// in which scan_carry_kernel composes them from dh_last; the carry then leaves
// in slot nblk - 2 - k the adjoint block k starts from.
// kAdjG threads per (batch, block, channel), N / kAdjG states each, so a CTA
// of 128 threads covers kAdjChannels channels.  The walk is one dependent
// chain per state and needs only the step's inputs, so they are staged in
// shared memory by chunk (delta, dout, z rows of the CTA's channels and the
// C row), two chunks ahead in a three-slot ring: with ASYNC by cp.async (the
// rows are whole 16-byte groups: d_in times the element size a multiple of
// 16 and 16-byte aligned inputs), else by plain loads before each chunk.
constexpr int kAdjG = 4, kAdjChannels = 128 / kAdjG;
template <typename T, int N, bool ASYNC>
__global__ void __launch_bounds__(128) scan_bwd_adjoint_kernel(BwdParams p, float *adj_decay,
                                                               float *adj_state) {
  constexpr int NA = N / kAdjG, CH = kAdjChannels, TT = kStateChunk, R = 3;
  constexpr int VEC = 16 / (int)sizeof(T);          // elements per 16-byte group
  constexpr int ROW_G = CH / VEC, C_G = N / VEC;    // groups per channel row, per C row
  static_assert(N % kAdjG == 0 && NA >= 1, "states per thread");
  static_assert(CH % VEC == 0 && N % VEC == 0, "whole 16-byte groups");
  __shared__ __align__(16) T sD[R][TT][CH], sG[R][TT][CH], sZ[R][TT][CH], sC[R][TT][N];
  const int64_t L = p.L, d_in = p.d_in;
  const int64_t nC = (L + TT - 1) / TT;
  const int64_t nblk = (nC + p.Cb - 1) / p.Cb;
  const int64_t blk = (int64_t)blockIdx.y + 1;  // blocks 1 .. nblk - 1
  if (blk >= nblk) return;                        // the whole CTA
  const int64_t ib = blockIdx.z;
  const int tid = threadIdx.x, j = tid % kAdjG, cc = tid / kAdjG;
  const int64_t d0 = (int64_t)blockIdx.x * CH, d = d0 + cc;
  const bool active = d < d_in;
  const int64_t c_begin = blk * p.Cb, c_end = c_begin + p.Cb < nC ? c_begin + p.Cb : nC;
  const int nch = (int)(c_end - c_begin);
  const T *gdelta = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gdout = static_cast<const T *>(p.dout);
  const T *gC = static_cast<const T *>(p.C);
  const int64_t n_act = p.b * L * d_in, n_bc = p.b * L * N;

  // stage chunk c into ring slot `slot` (rows past L and channels past d_in
  // are zero)
  auto stage = [&](int64_t c, int slot) {
    const int64_t t0 = c * TT;
    if constexpr (ASYNC) {
      for (int q = tid; q < 3 * TT * ROW_G; q += 128) {
        const int which = q / (TT * ROW_G), rem = q - which * TT * ROW_G;
        const int i = rem / ROW_G, g = rem - i * ROW_G;
        const int64_t at = (ib * L + t0 + i) * d_in + d0 + g * VEC;
        const bool ok = (which != 2 || gz) && t0 + i < L && d0 + g * VEC < d_in &&
                        in_bounds(at + VEC - 1, n_act, kBndAct);
        const T *src = which == 0 ? gdelta : which == 1 ? gdout : (gz ? gz : gdelta);
        T *dst = which == 0 ? &sD[slot][i][g * VEC] : which == 1 ? &sG[slot][i][g * VEC]
                                                               : &sZ[slot][i][g * VEC];
        cp_async16(dst, src + (ok ? at : 0), ok ? 16 : 0);
      }
      for (int q = tid; q < TT * C_G; q += 128) {
        const int i = q / C_G, g = q - i * C_G;
        const int64_t ct = (ib * L + t0 + i) * N + g * VEC;
        const bool ok = t0 + i < L && in_bounds(ct + VEC - 1, n_bc, kBndBC);
        cp_async16(&sC[slot][i][g * VEC], gC + (ok ? ct : 0), ok ? 16 : 0);
      }
      cp_async_commit();
    } else {
      for (int q = tid; q < 3 * TT * CH; q += 128) {
        const int which = q / (TT * CH), rem = q - which * TT * CH;
        const int i = rem / CH, e = rem - i * CH;
        const int64_t at = (ib * L + t0 + i) * d_in + d0 + e;
        const T *src = which == 0 ? gdelta : which == 1 ? gdout : gz;
        const bool ok = src && t0 + i < L && d0 + e < d_in && in_bounds(at, n_act, kBndAct);
        T *dst = which == 0 ? &sD[slot][i][e] : which == 1 ? &sG[slot][i][e] : &sZ[slot][i][e];
        *dst = ok ? src[at] : T(0.0f);
      }
      for (int q = tid; q < TT * N; q += 128) {
        const int i = q / N, n = q - i * N;
        const int64_t ct = (ib * L + t0 + i) * N + n;
        const bool ok = t0 + i < L && in_bounds(ct, n_bc, kBndBC);
        sC[slot][i][n] = ok ? gC[ct] : T(0.0f);
      }
    }
  };

  float A2[NA], lam[NA];
#pragma unroll
  for (int k = 0; k < NA; ++k) {
    const int64_t n = j * NA + k;
    A2[k] = active && in_bounds(d * N + n, d_in * N, kBndParam) ? p.A[d * N + n] * kLog2e : 0.0f;
    lam[k] = 0.0f;
  }
  const float bias = active && p.dt_bias ? p.dt_bias[d] : 0.0f;
  float dsum = 0.0f;

  // chunks from the block's last backwards: chunk c_end - 1 - i in slot i % R
  if constexpr (ASYNC) {
    stage(c_end - 1, 0);
    if (nch > 1) stage(c_end - 2, 1);
    else cp_async_commit();
  }
  for (int i = 0; i < nch; ++i) {
    const int64_t c = c_end - 1 - i;
    const int slot = i % R;
    if constexpr (ASYNC) {
      if (i + 2 < nch) stage(c - 2, (i + 2) % R);
      else cp_async_commit();
      cp_async_wait<2>();  // chunk c has landed (this thread's copies)
    } else {
      stage(c, slot);
    }
    __syncthreads();  // every thread's copies of chunk c are visible
    if (active) {
      const int64_t t0 = c * TT;
      const int tc = (int)(L - t0 < TT ? L - t0 : TT);
      for (int s = tc - 1; s >= 0; --s) {
        const float pre = Elem<T>::load(&sD[slot][s][0], cc) + bias;
        const float dl = p.softplus ? softplus_f32(pre) : pre;
        const float go = Elem<T>::load(&sG[slot][s][0], cc);
        float gt = go;
        if (gz) {
          const float zz = Elem<T>::load(&sZ[slot][s][0], cc);
          gt = go * zz * rcp_approx(1.0f + ex2_approx(-zz * kLog2e));
        }
        dsum += dl;
#pragma unroll
        for (int k = 0; k < NA; ++k)
          lam[k] = fmaf(gt, Elem<T>::load(&sC[slot][s][0], j * NA + k), lam[k]) *
                   ex2_approx(dl * A2[k]);
      }
    }
    __syncthreads();  // slot i % R is refilled at iteration i + 1
  }
  if constexpr (ASYNC) cp_async_wait<0>();  // only empty groups can remain

  const int64_t row = ((ib * nblk + (nblk - 1 - blk)) * d_in + d) * N + j * NA;
  if (!active || !in_bounds(row + NA - 1, p.b * nblk * d_in * N, kBndChunk)) return;
#pragma unroll
  for (int k = 0; k < NA; ++k) {
    adj_state[row + k] = lam[k];
    adj_decay[row + k] = ex2_approx(dsum * A2[k]);
  }
}

}  // namespace ssm
