// scan_ws.cuh -- selective scan forward with warp-specialised staging.
//
// The operation is the one of scan_fwd.cuh ("手把手拆解Mamba-minimal中的
// selective_scan实现" §3-§5; softplus of delta and the SiLU gate of
// "代码连连看——mamba"'s Mamba.step()): per (batch i, channel d, state n)
//     delta = softplus(dt + dt_bias),  dA = exp(delta A),  dBu = delta B u,
//     h = dA h + dBu,  y = sum_n C h + D u,  y *= silu(z).
//
// A CTA owns (batch i, DT = 32 channels) for the whole sequence and walks it
// in chunks of TC steps with two kinds of warps:
//   - G = N / NS scan warps, one channel per lane (every lane of a warp reads
//     the same B / C entries: one warp-uniform shared load serves 32
//     channels), NS states per thread in fp32 registers; per step
//     h = exp2(delta A log2 e) h + (delta u) B and the partial C.h of the
//     thread's states, left in a per-group plane.  The exponentials and
//     delta u B of the next 4-step group are formed while this group's
//     recurrence runs, so the SFU is fed continuously;
//   - H helper warps that keep the scan fed: they copy the chunk P + 1 ahead
//     global -> shared (16-byte cp.async into a ring of R = P + 2 slots), run
//     the pre-pass of the next chunk (delta = softplus(dt + bias), delta u,
//     D u and silu(z) once per (t, d), fp32, channel-major; steps past the end
//     get delta = 0, identity steps) and the post-pass of the previous one
//     (y = (sum of the G partials + D u) silu(z), rounded once, stored).
// The two run concurrently between one CTA barrier per chunk: the pre-pass
// outputs and the partial planes are double-buffered, so the scan of chunk
// i overlaps the copy of chunk i + P + 1, the pre-pass of i + 1 and the
// post-pass of i - 1.  dA and dBu ((b, L, d_in, N) tensors in the pages'
// loop) are never stored.
#pragma once

#include "scan_fwd.cuh"

namespace ssm {

template <typename T, int N, int NS, int TC, int H, int P, int DT_ = 32>
struct WsScan {
  // channels per CTA: one per lane; with DT < 32 a warp holds 32 / DT state
  // groups of DT channels (each quarter- or half-warp reads one B / C address)
  static constexpr int DT = DT_;
  static constexpr int G = N / NS;              // state groups = scan warps
  static constexpr int NP2 = NS / 2;            // state pairs per scan thread
  static constexpr int R = P + 2;               // ring slots
  static constexpr int SCAN_THREADS = DT * G;
  static constexpr int HELP_THREADS = 32 * H;
  static constexpr int THREADS = SCAN_THREADS + HELP_THREADS;
  static constexpr int TCP = TC + 4;            // padded channel-major row (floats)
  static constexpr int ESZ = sizeof(T);
  static constexpr int VEC = 16 / ESZ;          // elements per 16-byte granule
  static constexpr int ROW_GRAN = DT / VEC;     // granules per raw tile row
  static constexpr int RAWROW = DT * ESZ + 16;  // padded raw tile row (bytes)
  static constexpr int BC_GRAN = N / VEC;       // granules per B / C row
  static constexpr int RAW_TILE = TC * RAWROW;  // one tensor, one slot
  static constexpr int BC_TILE = TC * N * ESZ;
  static constexpr int CPS = DT / 2;            // channel pairs (pre/post items per step group)
  static constexpr int ARR = DT * TCP * 4;      // one [DT][TCP] fp32 array
  static constexpr int OFF_RAW = 0;                             // [R][3][TC] rows: u, dt, z
  static constexpr int OFF_BC = OFF_RAW + R * 3 * RAW_TILE;     // [R][2][TC][N] T: B, C
  static constexpr int OFF_DL = OFF_BC + R * 2 * BC_TILE;       // [2] delta
  static constexpr int OFF_DU = OFF_DL + 2 * ARR;               // [2] delta u
  static constexpr int OFF_DZ = OFF_DU + 2 * ARR;               // [2] D u
  static constexpr int OFF_GT = OFF_DZ + 2 * ARR;               // [2] silu(z)
  static constexpr int SMEM = OFF_GT + 2 * ARR;                 // dynamic part
  // The partial C.h planes [2][G][DT][TCP] are a separate static array, so
  // the compiler sees that the scan's stores to them never alias the staged
  // rows it reads, and may issue later steps' loads and exponentials early.
  static constexpr int PL_FLOATS = 2 * G * DT * TCP;
  static_assert(N % NS == 0 && NS % 2 == 0 && NS >= 2, "states per thread");
  static_assert(TC % 4 == 0 && TC % kStateChunk == 0, "chunk length");
  static_assert(DT % VEC == 0 && N % VEC == 0, "whole granules");
  static_assert(HELP_THREADS % CPS == 0 && P >= 1, "helper layout");
  static_assert((DT == 8 || DT == 16 || DT == 32) && SCAN_THREADS % 32 == 0, "channel tile");
  static_assert(RAWROW % 16 == 0 && OFF_BC % 16 == 0 && OFF_DL % 16 == 0, "alignment");
  static_assert(PL_FLOATS * 4 <= 48 * 1024, "static shared memory");
  static_assert(SMEM + PL_FLOATS * 4 <= 227 * 1024, "shared memory");
};

// Barrier 1 joins the helper warps only (barrier 0 is __syncthreads).
__device__ __forceinline__ void helper_barrier(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

template <typename T, int N, int NS, int TC, int H, int P, bool HAS_Z, bool SAVE, bool SUMMARY,
          int DT_ = 32>
__global__ void __launch_bounds__(WsScan<T, N, NS, TC, H, P, DT_>::THREADS)
    scan_ws_kernel(ScanParams p) {
  // SUMMARY && SAVE is the states pass of the backward: one block from h0,
  // no outputs, the chunk-start states saved; a plain SUMMARY is the split
  // scan's summary of each block from h = 0.
  using K = WsScan<T, N, NS, TC, H, P, DT_>;
  constexpr int DT = K::DT, G = K::G, NP2 = K::NP2, R = K::R, TCP = K::TCP;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(16) float s_planes[K::PL_FLOATS];
  const int tid = threadIdx.x;
  const int64_t ib = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * DT;
  const int64_t L = p.L, d_in = p.d_in;
  // this CTA's block of the sequence: [t_begin, t_end)
  // (the summary pass runs the first nblk - 1 blocks only: nblk comes from Lb)
  const int64_t blk = blockIdx.z, nblk = p.Lb > 0 ? (L + p.Lb - 1) / p.Lb : 1;
  const int64_t t_begin = blk * p.Lb;
  const int64_t t_end = p.Lb > 0 && t_begin + p.Lb < L ? t_begin + p.Lb : L;
  const int64_t nchunks = (t_end - t_begin + TC - 1) / TC;
  const int64_t blk_row = (ib * nblk + blk) * d_in;  // row of (batch, block) in blk_decay / blk_state
  // buffer sizes (elements) for the debug-bounds checks
  const int64_t n_act = p.b * L * d_in, n_bc = p.b * L * N, n_state = p.b * d_in * N;
  const int64_t n_blk = p.b * nblk * d_in * N, n_par = d_in * N;
  auto arr = [&](int off, int buf) {
    return reinterpret_cast<float *>(smem + off + buf * K::ARR);
  };
  auto raw = [&](int slot, int tensor) {  // tensor 0 u, 1 dt, 2 z
    return smem + K::OFF_RAW + (slot * 3 + tensor) * K::RAW_TILE;
  };
  auto rawbc = [&](int slot, int which) {  // which 0 B, 1 C
    return reinterpret_cast<T *>(smem + K::OFF_BC + (slot * 2 + which) * K::BC_TILE);
  };

  if (tid < K::SCAN_THREADS) {
    // =================================================== scan warps
    // the split scan's last pass is launched while the carry pass finishes:
    // the helpers stage inputs meanwhile, the scan warps wait for the block
    // start states
    grid_dependency_wait();
    const int c = tid % DT;  // channel
    const int g = tid / DT;  // state group
    const int64_t d = d0 + c;
    const bool d_ok = d < d_in;
    float2 A2[NP2], h[NP2];
#pragma unroll
    for (int k = 0; k < NP2; ++k) {
      const int n = g * NS + 2 * k;
      A2[k] = d_ok && in_bounds(d * N + n + 1, n_par, kBndParam)
                  ? make_float2(p.A[d * N + n] * kLog2e, p.A[d * N + n + 1] * kLog2e)
                  : make_float2(0.0f, 0.0f);
      // the summary starts every block from zero; the scan (and the states
      // pass) starts block 0 from h0 and block k > 0 from the state the
      // carry pass left in blk_decay[k - 1]
      const float *h0 = blk == 0 ? p.h0 + (ib * d_in + d) * N + n
                                 : p.blk_decay + (blk_row - d_in + d) * N + n;
      const bool from = d_ok && (!SUMMARY || SAVE) && (blk > 0 || p.h0) &&
                        (blk == 0 ? in_bounds((ib * d_in + d) * N + n + 1, n_state, kBndState)
                                  : in_bounds((blk_row - d_in + d) * N + n + 1, n_blk, kBndChunk));
      h[k] = from ? make_float2(h0[0], h0[1]) : make_float2(0.0f, 0.0f);
    }
    float dsum = 0.0f;  // sum of delta over the block (summary pass)
    const int64_t n_saved = (L + kStateChunk - 1) / kStateChunk;
    __syncthreads();  // the first chunk's pre-pass is done
    int slot = 0;     // ch % R
    for (int64_t ch = 0; ch < nchunks; ++ch) {
      const int buf = (int)(ch & 1);
      const int64_t t0 = t_begin + ch * TC;
      const float *rdl = arr(K::OFF_DL, buf) + c * TCP;
      const float *rdu = arr(K::OFF_DU, buf) + c * TCP;
      float *pl_own = s_planes + ((buf * G + g) * DT + c) * TCP;
      const T *rB = rawbc(slot, 0), *rC = rawbc(slot, 1);
      // the exponentials and delta u B of the next 4-step group are formed
      // one step at a time between this group's recurrence steps, so the SFU
      // sees a steady stream instead of bursts of 4 * NP2 requests
      struct Grp {
        float2 a[4][NP2], b[4][NP2];
        StateWords<T, NS> C[4];
      };
      auto stage1_step = [&](int t, int jj, float dl, float du, Grp &q) {
        StateWords<T, NS> Bw;
        Bw.load(rB + t * N + g * NS);
        if constexpr (SUMMARY) dsum += dl;
        else q.C[jj].load(rC + t * N + g * NS);
        const float2 d2 = make_float2(dl, dl);
        const float2 u2 = make_float2(du, du);
#pragma unroll
        for (int k = 0; k < NP2; ++k) {
          q.a[jj][k] = exp2_sfu2(__fmul2_rn(d2, A2[k]));
          q.b[jj][k] = __fmul2_rn(u2, Bw.pair(k));
        }
      };
      Grp cur, nxt;
      {
        const float4 dv = *reinterpret_cast<const float4 *>(rdl);
        const float4 uv = *reinterpret_cast<const float4 *>(rdu);
        stage1_step(0, 0, dv.x, uv.x, cur);
        stage1_step(1, 1, dv.y, uv.y, cur);
        stage1_step(2, 2, dv.z, uv.z, cur);
        stage1_step(3, 3, dv.w, uv.w, cur);
      }
#pragma unroll
      for (int j4 = 0; j4 < TC / 4; ++j4) {
        const bool ahead = j4 + 1 < TC / 4;
        float4 ndv = make_float4(0.0f, 0.0f, 0.0f, 0.0f), nuv = ndv;
        if (ahead) {
          ndv = *reinterpret_cast<const float4 *>(rdl + 4 * (j4 + 1));
          nuv = *reinterpret_cast<const float4 *>(rdu + 4 * (j4 + 1));
        }
        const float nds[4] = {ndv.x, ndv.y, ndv.z, ndv.w};
        const float nus[4] = {nuv.x, nuv.y, nuv.z, nuv.w};
        float ys[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int t = 4 * j4 + jj;
          if (ahead) stage1_step(t + 4, jj, nds[jj], nus[jj], nxt);
          if (SAVE && t % kStateChunk == 0 && d_ok && t0 + t < L &&
              in_bounds(((ib * n_saved + (t0 + t) / kStateChunk) * d_in + d) * N + g * NS + NS - 1,
                        p.b * n_saved * d_in * N, kBndChunk)) {  // the state before step t
            float2 *dst = reinterpret_cast<float2 *>(
                p.chunk_h + ((ib * n_saved + (t0 + t) / kStateChunk) * d_in + d) * N + g * NS);
#pragma unroll
            for (int k = 0; k < NP2; ++k) dst[k] = h[k];
          }
          float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int k = 0; k < NP2; ++k) {
            h[k] = __ffma2_rn(cur.a[jj][k], h[k], cur.b[jj][k]);
            if constexpr (!SUMMARY) acc = __ffma2_rn(h[k], cur.C[jj].pair(k), acc);
          }
          ys[jj] = acc.x + acc.y;
        }
        if constexpr (!SUMMARY)
          *reinterpret_cast<float4 *>(pl_own + 4 * j4) = make_float4(ys[0], ys[1], ys[2], ys[3]);
        if (ahead) cur = nxt;
      }
      slot = slot == R - 1 ? 0 : slot + 1;
      __syncthreads();  // partials of this chunk written; next chunk's pre-pass done
    }
    if constexpr (SUMMARY && SAVE) {
      // the states pass keeps nothing but the saved states
    } else if constexpr (SUMMARY) {  // the block's map h -> P h + Q
      if (d_ok && in_bounds((blk_row + d) * N + g * NS + NS - 1, n_blk, kBndChunk)) {
        float *q = p.blk_state + (blk_row + d) * N + g * NS;
        float *pd = p.blk_decay + (blk_row + d) * N + g * NS;
#pragma unroll
        for (int k = 0; k < NP2; ++k) {
          q[2 * k] = h[k].x;
          q[2 * k + 1] = h[k].y;
          const float2 e = exp2_sfu2(__fmul2_rn(make_float2(dsum, dsum), A2[k]));
          pd[2 * k] = e.x;
          pd[2 * k + 1] = e.y;
        }
      }
    } else if (p.h_last && d_ok && blk == nblk - 1 &&
               in_bounds((ib * d_in + d) * N + g * NS + NS - 1, n_state, kBndState)) {
      float *hl = p.h_last + (ib * d_in + d) * N + g * NS;
#pragma unroll
      for (int k = 0; k < NP2; ++k) {
        hl[2 * k] = h[k].x;
        hl[2 * k + 1] = h[k].y;
      }
    }
    return;
  }

  // ===================================================== helper warps
  const int hid = tid - K::SCAN_THREADS;
  const T *gu = static_cast<const T *>(p.u);
  const T *gdt = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);

  // copy chunk ch into ring slot `slot` (one cp.async group per call)
  auto prefetch = [&](int64_t ch, int slot) {
    const int64_t t0 = t_begin + ch * TC;
    for (int q = hid; q < TC * K::ROW_GRAN; q += K::HELP_THREADS) {
      const int t = q / K::ROW_GRAN, gq = q - t * K::ROW_GRAN;
      const int64_t dd = d0 + gq * K::VEC;
      const bool ok = (t0 + t < t_end) && (dd < d_in) &&
                      in_bounds((ib * L + t0 + t) * d_in + dd + K::VEC - 1, n_act, kBndAct);
      const int64_t off = ok ? ((ib * L + t0 + t) * d_in + dd) : 0;
      const int so = t * K::RAWROW + gq * 16;
      cp_async16(raw(slot, 0) + so, gu + off, ok ? 16 : 0);
      cp_async16(raw(slot, 1) + so, gdt + off, ok ? 16 : 0);
      if (HAS_Z && !SUMMARY) cp_async16(raw(slot, 2) + so, gz + off, ok ? 16 : 0);
    }
    for (int q = hid; q < TC * K::BC_GRAN; q += K::HELP_THREADS) {
      const int t = q / K::BC_GRAN, gq = q - t * K::BC_GRAN;
      const bool ok = t0 + t < t_end &&
                      in_bounds((ib * L + t0 + t) * N + gq * K::VEC + K::VEC - 1, n_bc, kBndBC);
      const int64_t off = ok ? ((ib * L + t0 + t) * N + gq * K::VEC) : 0;
      const int so = t * N + gq * K::VEC;
      cp_async16(rawbc(slot, 0) + so, gB + off, ok ? 16 : 0);
      if (!SUMMARY) cp_async16(rawbc(slot, 1) + so, gC + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // pre/post items: channel pair cp (fixed), 4-step groups sg
  constexpr int SG_STRIDE = K::HELP_THREADS / K::CPS;
  const int cp = hid % K::CPS;
  const int sg0 = hid / K::CPS;
  const int64_t dp = d0 + 2 * cp;
  const bool p_ok = dp < d_in;  // d_in is a multiple of VEC >= 4, so dp + 1 < d_in too
  const bool par_ok = p_ok && in_bounds(dp + 1, d_in, kBndParam);
  const float2 bias2 = (par_ok && p.dt_bias) ? make_float2(p.dt_bias[dp], p.dt_bias[dp + 1])
                                             : make_float2(0.0f, 0.0f);
  const float2 D2 = (par_ok && p.D) ? make_float2(p.D[dp], p.D[dp + 1]) : make_float2(0.0f, 0.0f);
  // Every other group of four pairs visits its two channel rows in swapped
  // order, so a quarter-warp's 16-byte accesses hit distinct banks.  Rows are
  // chosen by register selects: a runtime index into the per-thread arrays
  // below would move them to local memory.
  const int swp = (cp >> 2) & 1;
  const int row_a = 2 * cp + swp, row_b = 2 * cp + 1 - swp;

  // post-pass of chunk ch (buffer buf, tc valid steps).  A helper thread reads
  // the D u / gate entries of exactly the items its own pre-pass writes, so
  // the pre-pass of chunk ch + 2 may reuse the buffer right after.
  auto post = [&](int64_t ch, int tc, int buf) {
    if (SUMMARY || !p_ok) return;
    const int64_t t0 = t_begin + ch * TC;
    const float *pdz = arr(K::OFF_DZ, buf), *pgt = arr(K::OFF_GT, buf);
    const float *ppl = s_planes + buf * G * DT * TCP;
    for (int sg = sg0; sg * 4 < tc; sg += SG_STRIDE) {
      float4 ya, yb;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int o = (e ? row_b : row_a) * TCP + sg * 4;
        float4 acc = *reinterpret_cast<const float4 *>(pdz + o);
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const float4 v = *reinterpret_cast<const float4 *>(ppl + q * DT * TCP + o);
          acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        if (HAS_Z) {
          const float4 g4 = *reinterpret_cast<const float4 *>(pgt + o);
          acc.x *= g4.x; acc.y *= g4.y; acc.z *= g4.z; acc.w *= g4.w;
        }
        if (e == 0) ya = acc; else yb = acc;
      }
      const float4 c0 = swp ? yb : ya, c1 = swp ? ya : yb;  // channels 2 cp, 2 cp + 1
      const float y0[4] = {c0.x, c0.y, c0.z, c0.w};
      const float y1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int t = sg * 4 + jj;
        const int64_t o = (ib * L + t0 + t) * d_in + dp;
        if (t < tc && in_bounds(o + 1, n_act, kBndAct)) {
          if constexpr (sizeof(T) == 2)
            *reinterpret_cast<uint32_t *>(gy + o) = pack_bf16x2(y0[jj], y1[jj]);
          else
            *reinterpret_cast<float2 *>(gy + o) = make_float2(y0[jj], y1[jj]);
        }
      }
    }
  };

  // pre-pass of the chunk staged in ring slot `slot` (tc valid steps) into buffer buf
  auto pre = [&](int slot, int tc, int buf) {
    float *pdl = arr(K::OFF_DL, buf), *pdu = arr(K::OFF_DU, buf);
    float *pdz = arr(K::OFF_DZ, buf), *pgt = arr(K::OFF_GT, buf);
    const unsigned char *ru = raw(slot, 0) + 2 * cp * K::ESZ;
    const unsigned char *rd = raw(slot, 1) + 2 * cp * K::ESZ;
    const unsigned char *rz = raw(slot, 2) + 2 * cp * K::ESZ;
    for (int sg = sg0; sg < TC / 4; sg += SG_STRIDE) {
      float dl[2][4], dlu[2][4], dd[2][4], gg[2][4] = {};
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int t = sg * 4 + jj;
        float2 u2, e2, z2 = make_float2(0.0f, 0.0f);
        if constexpr (sizeof(T) == 2) {
          const uint32_t wu = *reinterpret_cast<const uint32_t *>(ru + t * K::RAWROW);
          const uint32_t wd = *reinterpret_cast<const uint32_t *>(rd + t * K::RAWROW);
          u2 = make_float2(bf16lo(wu), bf16hi(wu));
          e2 = make_float2(bf16lo(wd), bf16hi(wd));
          if (HAS_Z && !SUMMARY) {
            const uint32_t wz = *reinterpret_cast<const uint32_t *>(rz + t * K::RAWROW);
            z2 = make_float2(bf16lo(wz), bf16hi(wz));
          }
        } else {
          u2 = *reinterpret_cast<const float2 *>(ru + t * K::RAWROW);
          e2 = *reinterpret_cast<const float2 *>(rd + t * K::RAWROW);
          if (HAS_Z && !SUMMARY) z2 = *reinterpret_cast<const float2 *>(rz + t * K::RAWROW);
        }
        e2 = __fadd2_rn(e2, bias2);
        if (p.delta_softplus) e2 = softplus2_f32(e2);
        if (t >= tc) e2 = make_float2(0.0f, 0.0f);  // identity step past the end
        const float2 eu = __fmul2_rn(e2, u2);
        const float2 du2 = __fmul2_rn(D2, u2);
        dl[0][jj] = e2.x; dl[1][jj] = e2.y;
        dlu[0][jj] = eu.x; dlu[1][jj] = eu.y;
        dd[0][jj] = du2.x; dd[1][jj] = du2.y;
        if (HAS_Z && !SUMMARY) {
          gg[0][jj] = silu_for<T>(z2.x);
          gg[1][jj] = silu_for<T>(z2.y);
        }
      }
      const float4 l0 = make_float4(dl[0][0], dl[0][1], dl[0][2], dl[0][3]);
      const float4 l1 = make_float4(dl[1][0], dl[1][1], dl[1][2], dl[1][3]);
      const float4 u0 = make_float4(dlu[0][0], dlu[0][1], dlu[0][2], dlu[0][3]);
      const float4 u1 = make_float4(dlu[1][0], dlu[1][1], dlu[1][2], dlu[1][3]);
      const float4 z0 = make_float4(dd[0][0], dd[0][1], dd[0][2], dd[0][3]);
      const float4 z1 = make_float4(dd[1][0], dd[1][1], dd[1][2], dd[1][3]);
      const int ia = row_a * TCP + sg * 4, ibb = row_b * TCP + sg * 4;
      *reinterpret_cast<float4 *>(pdl + ia) = swp ? l1 : l0;
      *reinterpret_cast<float4 *>(pdl + ibb) = swp ? l0 : l1;
      *reinterpret_cast<float4 *>(pdu + ia) = swp ? u1 : u0;
      *reinterpret_cast<float4 *>(pdu + ibb) = swp ? u0 : u1;
      if (SUMMARY) continue;  // the summary needs delta and delta u only
      *reinterpret_cast<float4 *>(pdz + ia) = swp ? z1 : z0;
      *reinterpret_cast<float4 *>(pdz + ibb) = swp ? z0 : z1;
      if (HAS_Z) {
        const float4 g0 = make_float4(gg[0][0], gg[0][1], gg[0][2], gg[0][3]);
        const float4 g1 = make_float4(gg[1][0], gg[1][1], gg[1][2], gg[1][3]);
        *reinterpret_cast<float4 *>(pgt + ia) = swp ? g1 : g0;
        *reinterpret_cast<float4 *>(pgt + ibb) = swp ? g0 : g1;
      }
    }
  };

  auto tc_of = [&](int64_t ch) {
    const int64_t rem = t_end - t_begin - ch * TC;
    return (int)(rem < (int64_t)TC ? rem : (int64_t)TC);
  };

  // prologue: chunks 0 .. P in flight (one group each, empty past the end),
  // then the pre-pass of chunk 0
#pragma unroll
  for (int c0 = 0; c0 <= P; ++c0) {
    if (c0 < nchunks) prefetch(c0, c0);
    else cp_async_commit();
  }
  cp_async_wait<P>();
  helper_barrier(K::HELP_THREADS);
  pre(0, tc_of(0), 0);
  __syncthreads();

  // Chunk c lives in ring slot c % R and in group c of this thread's
  // cp.async groups; at iteration ch, with ch + P + 2 groups committed,
  // waiting until P are pending means chunk ch + 1 has landed.  The slot
  // refilled at iteration ch held chunk ch - 1, whose scan is finished.
  int nslot = 1;            // (ch + 1) % R
  int islot = (P + 1) % R;  // (ch + P + 1) % R
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    if (ch + P + 1 < nchunks) prefetch(ch + P + 1, islot);
    else cp_async_commit();
    cp_async_wait<P>();
    helper_barrier(K::HELP_THREADS);  // chunk ch + 1's tiles visible to every helper
    if (ch > 0) post(ch - 1, TC, (int)((ch - 1) & 1));
    if (ch + 1 < nchunks) pre(nslot, tc_of(ch + 1), (int)((ch + 1) & 1));
    nslot = nslot == R - 1 ? 0 : nslot + 1;
    islot = islot == R - 1 ? 0 : islot + 1;
    __syncthreads();  // matches the scan warps' barrier of chunk ch
  }
  if (nchunks > 0) post(nchunks - 1, tc_of(nchunks - 1), (int)((nchunks - 1) & 1));
  cp_async_wait<0>();  // only empty groups can remain
}

// Carry pass of the split scan, a parallel scan over the blocks.  Chain
// (batch i, column r = channel N + state) has the block maps
// h -> P_k h + Q_k (P_k = blk_decay[k], Q_k = blk_state[k], k < nblk - 1);
// composed in order with (a, b) o (a', b') = (a a', a' b + b'), (a, b) the
// earlier map, and applied to h0, they give the state each block starts from.  A CTA owns 32 chains;
// 32-block tiles of P and Q are read row by row (coalesced) into shared
// memory, each warp scans 4 chains across the tile with shuffles (lane =
// block), and the state leaving a tile carries into the next.  The state
// block k + 1 starts from overwrites P_k, which the tile has already read.
constexpr int kCarryThreads = 256;
__global__ void __launch_bounds__(kCarryThreads) scan_carry_kernel(const float *h0, float *blk_decay,
                                                                   const float *blk_state, int64_t b,
                                                                   int64_t nblk, int64_t d_in, int N) {
  constexpr int TILE = 32, WARPS = kCarryThreads / 32, CPW = TILE / WARPS;  // chains per warp
  __shared__ float sP[TILE][TILE + 1], sQ[TILE][TILE + 1];
  const int64_t per = d_in * N, nmaps = nblk - 1;
  const int64_t ib = blockIdx.y, r0 = (int64_t)blockIdx.x * TILE;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t col = r0 + lane;  // this lane's chain in the row loads and stores
  grid_dependents_launch();       // the scan pass may start staging its inputs
  grid_dependency_wait();         // the summary pass's maps are written
  float carry[CPW];               // state entering the tile, chains warp CPW + c
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    const int64_t r = r0 + warp * CPW + c;
    carry[c] = (h0 && r < per && in_bounds(ib * per + r, b * per, kBndState)) ? h0[ib * per + r]
                                                                              : 0.0f;
  }
  for (int64_t k0 = 0; k0 < nmaps; k0 += TILE) {
    __syncthreads();  // the previous tile's results are stored
    for (int rr = warp; rr < TILE; rr += WARPS) {
      const int64_t k = k0 + rr, i = (ib * nblk + k) * per + col;
      const bool ok = k < nmaps && col < per && in_bounds(i, b * nblk * per, kBndChunk);
      sP[rr][lane] = ok ? blk_decay[i] : 1.0f;  // identity maps past the last block
      sQ[rr][lane] = ok ? blk_state[i] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
      const int cc = warp * CPW + c;
      float a = sP[lane][cc], q = sQ[lane][cc];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {  // inclusive: maps k0 .. k0 + lane
        // (pa, pq) composes the off earlier maps; (a, q) this lane's so far
        const float pa = __shfl_up_sync(0xffffffffu, a, off);
        const float pq = __shfl_up_sync(0xffffffffu, q, off);
        if (lane >= off) {
          q = fmaf(a, pq, q);
          a *= pa;
        }
      }
      const float h = fmaf(a, carry[c], q);  // the state after block k0 + lane
      carry[c] = __shfl_sync(0xffffffffu, h, 31);
      sP[lane][cc] = h;
    }
    __syncthreads();
    for (int rr = warp; rr < TILE; rr += WARPS) {
      const int64_t k = k0 + rr, i = (ib * nblk + k) * per + col;
      if (k < nmaps && col < per && in_bounds(i, b * nblk * per, kBndChunk))
        blk_decay[i] = sP[rr][lane];
    }
  }
}

}  // namespace ssm
