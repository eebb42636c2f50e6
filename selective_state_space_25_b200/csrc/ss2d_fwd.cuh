// ss2d_fwd.cuh -- VMamba SS2D forward: CrossScan, selective scan per
// direction, CrossMerge ("关于代码SS2D中的d_state设置", VMamba issue 206:
// the four scan orders only arrange the sequence; d_state = 1 for
// throughput).
//
// Direction k visits pixel p_k(l) at step l (pixels row-major, p = h W + w):
//   k0 row-major p = l; k1 column-major l = w H + h; k2 = k0 reversed;
//   k3 = k1 reversed.
// The orders are index arithmetic: u is gathered at p_k(l) when it is read
// and each output lands at p_k(l) when it is produced; no permuted copy
// exists in memory, and per-direction outputs only in the direction split
// (DSPLIT below), as fp32 slices of the caller's workspace.
#pragma once

#include <type_traits>

#include "ssm_common.cuh"

namespace ssm {

// Scan orders.  Cross (VMamba's CrossScan): k0 row-major, k1 column-major,
// k2 / k3 their reverses.  Snake (the snake scan of the same thread): as
// cross, but odd rows of k0 run right to left and odd columns of k1 bottom
// to top, so consecutive steps stay neighbours.
enum Ss2dOrder { kOrderCross = 0, kOrderSnake = 1 };

template <int ORDER>
__device__ __forceinline__ int64_t ss2d_pixel(int k, int64_t l, int64_t H, int64_t W) {
  const int64_t L = H * W;
  if (k >= 2) l = L - 1 - l;
  if ((k & 1) == 0) {
    if constexpr (ORDER == kOrderCross) return l;
    const int64_t h = l / W, r = l - h * W;
    return h * W + ((h & 1) ? W - 1 - r : r);
  }
  const int64_t w = l / H;
  const int64_t r = l - w * H;
  const int64_t h = (ORDER == kOrderSnake && (w & 1)) ? H - 1 - r : r;
  return h * W + w;
}

// Step index at which direction k visits pixel (h, w): the inverse of ss2d_pixel.
template <int ORDER>
__device__ __forceinline__ int64_t ss2d_step_of(int k, int64_t h, int64_t w, int64_t H,
                                                int64_t W) {
  int64_t l;
  if ((k & 1) == 0)
    l = h * W + ((ORDER == kOrderSnake && (h & 1)) ? W - 1 - w : w);
  else
    l = w * H + ((ORDER == kOrderSnake && (w & 1)) ? H - 1 - h : h);
  return k >= 2 ? H * W - 1 - l : l;
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

// ---------------------------------------------------------------------------
// d_state = 1 kernel.  A CTA owns (batch i, 8 channels) and runs the four
// directions in turn, summing their outputs per pixel in an fp32
// accumulator of the whole image (k0 + k1 + k2 + k3, one rounding at the
// end, deterministic).  Within a direction the sequence is walked in chunks
// of LC = 8 WARPS TS steps:
//   1. the chunk's delta rows and the u rows of the pixels it visits (16
//      bytes = 8 bf16 channels each) are copied global -> shared with
//      cp.async, one chunk ahead, each warp the rows of its own segments,
//      and the accumulator row each step lands on is worked out once per
//      step for all channels; B / C values likewise when they are 16-byte
//      aligned, else read directly;
//   2. thread (segment s, channel pair cp) takes TS consecutive steps of its
//      two channels: delta = softplus(dt + bias), dA = exp2(delta A log2 e)
//      (FMA-pipe polynomial or SFU), delta u B, C and D u go to registers,
//      and the segment's composed affine map h -> P h + Q is formed;
//   3. a shuffle scan over the warp's 8 segments and a pass over the warps'
//      totals give each segment its incoming state, the carry of the previous
//      chunk included (the operator is (a, b) o (a', b') = (a a', a' b + b'));
//      the exchange of the warps' totals is the chunk's one CTA barrier: the
//      staged rows are warp-private, and the barrier also orders every
//      accumulator update of a chunk before those of the next;
//   4. the segment replays its steps, h = dA h + delta u B, and adds
//      y = C h + D u into the accumulator at the pixel each step visits.
// TS is odd so the 8 segments of a warp hit distinct bank groups in the
// staged rows; the accumulator row of pixel (h, w) is h RS + w with the
// row stride RS = W rounded up to odd, so both row- and column-major runs
// spread over the banks.
// ---------------------------------------------------------------------------
template <typename T, int TS, int WARPS, bool ACC_SMEM = true>
struct Ss2dCfg {
  static constexpr int DT = 8, PAIRS = 4, SPW = 8;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int S = SPW * WARPS;       // segments per chunk
  static constexpr int RW = SPW * TS;         // steps (staged rows) per warp
  static constexpr int LC = S * TS;           // steps per chunk
  // accumulator row of a step: 16-bit in shared memory (H RS <= 6272), else
  // the pixel index
  using RowT = typename std::conditional<ACC_SMEM, unsigned short, int>::type;
  static constexpr int ESZ = sizeof(T);
  static constexpr int ROWB = DT * ESZ;       // bytes of one staged row (8 channels)
  static constexpr int GRAN_PER_ROW = ROWB / 16;
  static constexpr int BC_VEC = 16 / ESZ;
  static constexpr int BC_PAD = BC_VEC;       // room for the unaligned B / C fallback
  static constexpr int OFF_D = 0;
  static constexpr int OFF_U = OFF_D + LC * ROWB;
  static constexpr int OFF_B = OFF_U + LC * ROWB;
  static constexpr int OFF_C = OFF_B + (LC + BC_PAD) * ESZ;
  static constexpr int OFF_AGG = (OFF_C + (LC + BC_PAD) * ESZ + 15) / 16 * 16;  // float4 [2][WARPS][PAIRS]
  static constexpr int OFF_CARRY = OFF_AGG + 2 * WARPS * PAIRS * 16;          // float [2][8]
  static constexpr int OFF_ROW = OFF_CARRY + 64;   // RowT [LC]: accumulator row of each step
  static constexpr int OFF_ACC = (OFF_ROW + LC * (int)sizeof(RowT) + 15) / 16 * 16;  // float [L][8]
  static constexpr int AUX_BYTES = OFF_ACC;
  static_assert(TS % 2 == 1, "TS odd keeps the warp's segments on distinct bank groups");
  static_assert(ROWB % 16 == 0 && (RW * ESZ) % 16 == 0, "16-byte staging of a warp's rows");
  static_assert(RW % BC_VEC == 0, "a warp's B / C rows are whole 16-byte granules");
};

struct Aff2 {
  float2 a, b;  // two channels' h -> a h + b
};
__device__ __forceinline__ Aff2 aff2_then(Aff2 first, Aff2 then) {
  return Aff2{__fmul2_rn(then.a, first.a), __ffma2_rn(then.a, first.b, then.b)};
}

// a / b for 0 <= a < 2^24, 0 < b, from a float reciprocal and one correction
// (the float quotient is within one of the integer one there).
__device__ __forceinline__ int div_small(int a, int b, float inv_b) {
  int q = (int)((float)a * inv_b);
  const int r = a - q * b;
  q += (r >= b) - (r < 0);
  return q;
}

// Row stride (pixels) of the shared accumulator: W rounded up to odd, so
// runs TS (odd) steps apart in row- or column-major order fall on distinct
// 32-byte bank groups.
__host__ __device__ __forceinline__ int ss2d_acc_stride(int W) { return W | 1; }

// Image position (h, w) that direction k visits at step l (32-bit, one
// division).
template <int ORDER>
__device__ __forceinline__ void ss2d_pos(int k, int l, int H, int W, float invH, float invW,
                                         int &h, int &w) {
  const int ll = k >= 2 ? H * W - 1 - l : l;
  if ((k & 1) == 0) {
    h = div_small(ll, W, invW);
    const int r = ll - h * W;
    w = (ORDER == kOrderSnake && (h & 1)) ? W - 1 - r : r;
  } else {
    w = div_small(ll, H, invH);
    const int r = ll - w * H;
    h = (ORDER == kOrderSnake && (w & 1)) ? H - 1 - r : r;
  }
}

// ROW_ASYNC: delta / u rows staged with cp.async (needs d_in a multiple of 8
// and 16-byte aligned u, delta); otherwise with plain bounds-checked loads.
// BC_ASYNC: B / C staged with cp.async (needs H W a multiple of 16 / sizeof(T)
// and 16-byte aligned B, C); otherwise read from global memory per step.
// DSPLIT: the CTA runs direction blockIdx.z alone and leaves that
// direction's fp32 outputs, pixel-major, in slice z of the caller's
// workspace (4, b, H W, d_in) -- from its shared accumulator at the end, or
// directly when the accumulator lives in the workspace; ss2d_merge4_kernel
// then sums the four slices k0 + k1 + k2 + k3 and rounds once -- the fused
// kernel's operations in its order, for grids too small to fill the GPU one
// CTA per tile.
template <typename T, int TS, int WARPS, bool ACC_SMEM, bool A_POLY, bool ROW_ASYNC,
          bool BC_ASYNC, int ORDER, bool DSPLIT = false>
__global__ void __launch_bounds__(Ss2dCfg<T, TS, WARPS>::THREADS)
    ss2d_n1_kernel(Ss2dParams p) {
  using Cfg = Ss2dCfg<T, TS, WARPS, ACC_SMEM>;
  constexpr int THREADS = Cfg::THREADS, LC = Cfg::LC, DT = Cfg::DT, RW = Cfg::RW;
  using RowT = typename Cfg::RowT;
  extern __shared__ __align__(16) unsigned char smem[];
  T *tD = reinterpret_cast<T *>(smem + Cfg::OFF_D);
  T *tU = reinterpret_cast<T *>(smem + Cfg::OFF_U);
  T *tB = reinterpret_cast<T *>(smem + Cfg::OFF_B);
  T *tC = reinterpret_cast<T *>(smem + Cfg::OFF_C);
  float4 *agg = reinterpret_cast<float4 *>(smem + Cfg::OFF_AGG);
  float *carry = reinterpret_cast<float *>(smem + Cfg::OFF_CARRY);
  RowT *tR = reinterpret_cast<RowT *>(smem + Cfg::OFF_ROW);
  float *acc_s = reinterpret_cast<float *>(smem + Cfg::OFF_ACC);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int cp = lane & 3;           // channel pair
  const int sl = lane >> 2;          // segment within the warp
  const int seg = warp * Cfg::SPW + sl;
  const int64_t ib = blockIdx.y;
  const int64_t d0 = (int64_t)blockIdx.x * DT;
  const int64_t H = p.H, W = p.W, L = H * W, d_in = p.d_in;
  // H W < 2^22 and H W d_in < 2^31 (checked by the launcher): per-image
  // offsets fit 32-bit integers; only the per-(batch, direction) bases are 64-bit
  const int Hi = (int)H, Wi = (int)W, Li = (int)L, di = (int)d_in;
  const float invH = 1.0f / (float)Hi, invW = 1.0f / (float)Wi;
  const int RS = ss2d_acc_stride(Wi);
  const int64_t dA = d0 + 2 * cp;    // first channel of the pair
  const bool ok0 = dA < d_in, ok1 = dA + 1 < d_in;

  const T *gu = static_cast<const T *>(p.u) + ib * L * d_in + d0;    // this image, channel d0
  const T *gdt = static_cast<const T *>(p.delta) + ib * 4 * L * d_in + d0;
  const T *gB = static_cast<const T *>(p.B) + ib * 4 * L;
  const T *gC = static_cast<const T *>(p.C) + ib * 4 * L;
  T *gy = static_cast<T *>(p.y) + ib * L * d_in + d0;

  // this image, channel d0 (with DSPLIT in the slice of direction blockIdx.z)
  float *acc_g = p.acc_global + ((DSPLIT ? (int64_t)blockIdx.z * p.b : 0) + ib) * L * d_in + d0;
  // a channel pair is one 8-byte access: always in shared memory; in the
  // caller's workspace only for even d_in and an 8-byte aligned workspace
  const bool acc_pairs =
      ACC_SMEM || ((d_in & 1) == 0 && (reinterpret_cast<uintptr_t>(p.acc_global) & 7) == 0);
  // every channel of the tile exists and is accumulated as pairs (CTA-uniform)
  const bool whole_tile = d0 + DT <= d_in && acc_pairs;

  const int nchunks = (Li + LC - 1) / LC;
  const int kz = DSPLIT ? (int)blockIdx.z : 0;  // the direction (DSPLIT), else the first one

  // stage the delta / u rows (and B / C) of this warp's steps of chunk c of
  // direction k: rows w0 .. w0 + RW - 1
  const int w0 = warp * RW;
  constexpr int NRI = (RW + 31) / 32;  // rows per lane
  int pq[NRI], pr[NRI], dq = 0, dr = 0;
  auto prefetch = [&](int k, int c) {
    const int l0 = c * LC;
    const T *dk = gdt + (int64_t)k * L * d_in;  // delta rows of direction k
    if constexpr (ROW_ASYNC) {
      // lane rows w0 + lane + 32 i; their image positions are kept as
      // (q, r) = divmod(ll, D) and moved by LC steps per chunk, so only a
      // direction's first chunk divides
      const bool odd = (k & 1) != 0, rev = k >= 2;
      const int D = odd ? Hi : Wi;
      if (c == 0) {
        dq = div_small(LC, D, odd ? invH : invW);
        dr = LC - dq * D;
      }
#pragma unroll
      for (int i = 0; i < NRI; ++i) {
        const int rl = lane + 32 * i;
        if (rl >= RW) break;
        const int row = w0 + rl;
        const int l = l0 + row;
        if (c == 0) {  // rows past the end keep meaningless (q, r): they stay past it
          const int ll = rev ? Li - 1 - l : l;
          pq[i] = div_small(ll, D, odd ? invH : invW);
          pr[i] = ll - pq[i] * D;
        } else if (!rev) {
          pr[i] += dr;
          pq[i] += dq;
          if (pr[i] >= D) { pr[i] -= D; ++pq[i]; }
        } else {
          pr[i] -= dr;
          pq[i] -= dq;
          if (pr[i] < 0) { pr[i] += D; --pq[i]; }
        }
        const int q = pq[i], rr = pr[i];
        const bool flip = ORDER == kOrderSnake && (q & 1);
        const int hh = odd ? (flip ? Hi - 1 - rr : rr) : q;
        const int ww = odd ? q : (flip ? Wi - 1 - rr : rr);
        const int pix0 = hh * Wi + ww;
        const bool ok =
            l < Li &&
            in_bounds((ib * L + pix0) * d_in + d0 + DT - 1, p.b * L * d_in, kBndAct) &&
            in_bounds(((ib * 4 + k) * L + l) * d_in + d0 + DT - 1, p.b * 4 * L * d_in, kBndAct);
        const int pix = ok ? pix0 : 0;
        tR[row] = (RowT)(ACC_SMEM ? (ok ? hh * RS + ww : 0) : pix);
#pragma unroll
        for (int part = 0; part < Cfg::GRAN_PER_ROW; ++part) {
          const int po = part * (16 / Cfg::ESZ);
          cp_async16(tD + row * DT + po, dk + (ok ? l * di : 0) + po, ok ? 16 : 0);
          cp_async16(tU + row * DT + po, gu + pix * di + po, ok ? 16 : 0);
        }
      }
    } else {
      for (int r = w0 * DT + lane; r < (w0 + RW) * DT; r += 32) {
        const int row = r / DT, ch = r - row * DT;
        const int l = l0 + row;
        int hh = 0, ww = 0;
        if (l < Li) ss2d_pos<ORDER>(k, l, Hi, Wi, invH, invW, hh, ww);
        const int pix0 = hh * Wi + ww;
        const bool ok = l < Li && d0 + ch < d_in &&
                        in_bounds((ib * L + pix0) * d_in + d0 + ch, p.b * L * d_in, kBndAct) &&
                        in_bounds(((ib * 4 + k) * L + l) * d_in + d0 + ch, p.b * 4 * L * d_in, kBndAct);
        const int pix = ok ? pix0 : 0;
        if (ch == 0) tR[row] = (RowT)(ACC_SMEM ? (ok ? hh * RS + ww : 0) : pix);
        tD[r] = ok ? dk[l * di + ch] : T(0.0f);
        tU[r] = ok ? gu[pix * di + ch] : T(0.0f);
      }
    }
    if constexpr (BC_ASYNC) {
      for (int r = w0 / Cfg::BC_VEC + lane; r < (w0 + RW) / Cfg::BC_VEC; r += 32) {
        const int l = l0 + r * Cfg::BC_VEC;
        const int rem = Li - l;
        int bytes = rem <= 0 ? 0 : (rem >= Cfg::BC_VEC ? 16 : rem * Cfg::ESZ);
        if (bytes && !in_bounds((ib * 4 + k) * L + l + bytes / Cfg::ESZ - 1, p.b * 4 * L, kBndBC))
          bytes = 0;
        const int64_t off = bytes ? (int64_t)k * L + l : 0;
        cp_async16(tB + r * Cfg::BC_VEC, gB + off, bytes);
        cp_async16(tC + r * Cfg::BC_VEC, gC + off, bytes);
      }
    }
    cp_async_commit();
  };

  // the first direction starts from h = 0: buffer 0, or with DSPLIT buffer
  // (kz nchunks) & 1, so both are cleared
  if (tid < 2 * DT) carry[tid] = 0.0f;
  prefetch(kz, 0);
  float2 A2 = make_float2(0.0f, 0.0f), bias = A2;
  // the skip term of all four directions, (sum_k D_k) u, is added once, with
  // direction 0's outputs
  float2 Dsum = A2;
  if (p.D) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (ok0) Dsum.x += p.D[k * d_in + dA];
      if (ok1) Dsum.y += p.D[k * d_in + dA + 1];
    }
  }

  // one chunk of direction K (index arithmetic specialised per direction).
  // Chunk q = k nchunks + c reads the carry and the warp totals in buffer
  // q & 1 and leaves the next carry in the other buffer.  Its one CTA barrier
  // (after the warp totals) also orders every accumulator update of the
  // previous chunk before its own, the next direction's first chunk included.
  auto chunk = [&](auto kc, int c) {
    constexpr int K = decltype(kc)::value;
    constexpr bool FIRST = K == 0 || DSPLIT;  // this CTA's first direction stores, later ones add
    const int l0 = c * LC;
    const int cq = (K * nchunks + c) & 1;
    [[maybe_unused]] const T *Bk = gB + (int64_t)K * L;
    [[maybe_unused]] const T *Ck = gC + (int64_t)K * L;
    cp_async_wait<0>();
    __syncwarp();  // this warp's staged rows visible to all its lanes

    // ---- 1. this segment's steps into registers
    const int lb = l0 + seg * TS;
    // the segment run from h = 0: Q its state, P the product of its decays,
    // so step j's true output is C_j (P_j h_in + Q_j) = gg_j h_in + yl_j
    float2 yl[TS], gg[TS];
    int rows[TS];  // accumulator row (or pixel) each step lands on
    float2 P = make_float2(1.0f, 1.0f), Q = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < TS; ++j) {
      const int row = seg * TS + j;
      rows[j] = tR[row];
      float2 dv, uv, bc;
      if constexpr (sizeof(T) == 2) {
        const uint32_t wd = *reinterpret_cast<const uint32_t *>(tD + row * DT + 2 * cp);
        const uint32_t wu = *reinterpret_cast<const uint32_t *>(tU + row * DT + 2 * cp);
        dv = make_float2(bf16lo(wd), bf16hi(wd));
        uv = make_float2(bf16lo(wu), bf16hi(wu));
      } else {
        dv = *reinterpret_cast<const float2 *>(tD + row * DT + 2 * cp);
        uv = *reinterpret_cast<const float2 *>(tU + row * DT + 2 * cp);
      }
      if constexpr (BC_ASYNC) {
        bc = make_float2(Elem<T>::load(tB, row), Elem<T>::load(tC, row));
      } else {
        bc = lb + j < Li ? make_float2(Elem<T>::load(Bk, lb + j), Elem<T>::load(Ck, lb + j))
                         : make_float2(0.0f, 0.0f);
      }
      // Steps past the end (last chunk only) run on zero-filled rows; they
      // come after every real step, so they reach no stored output: the scan
      // is causal and the carry out of a direction's last chunk is dropped.
      float2 e = __fadd2_rn(dv, bias);
      if (p.delta_softplus) e = softplus2_f32(e);
      const float2 x = __fmul2_rn(e, A2);
      const float2 a = A_POLY ? exp2_poly2(x) : exp2_sfu2(x);
      Q = __ffma2_rn(a, Q, __fmul2_rn(__fmul2_rn(e, uv), make_float2(bc.x, bc.x)));
      P = __fmul2_rn(a, P);
      const float2 c2 = make_float2(bc.y, bc.y);
      yl[j] = K == 0 ? __ffma2_rn(c2, Q, __fmul2_rn(Dsum, uv)) : __fmul2_rn(c2, Q);
      gg[j] = __fmul2_rn(c2, P);
    }
    const Aff2 mine{P, Q};

    // ---- 2. inclusive scan over the warp's segments (lanes cp, cp + 4, ...)
    Aff2 inc = mine;
#pragma unroll
    for (int off = 1; off < Cfg::SPW; off <<= 1) {
      Aff2 prev;
      prev.a.x = __shfl_up_sync(0xffffffffu, inc.a.x, off * 4);
      prev.a.y = __shfl_up_sync(0xffffffffu, inc.a.y, off * 4);
      prev.b.x = __shfl_up_sync(0xffffffffu, inc.b.x, off * 4);
      prev.b.y = __shfl_up_sync(0xffffffffu, inc.b.y, off * 4);
      if (sl >= off) inc = aff2_then(prev, inc);
    }
    Aff2 exc;
    exc.a.x = __shfl_up_sync(0xffffffffu, inc.a.x, 4);
    exc.a.y = __shfl_up_sync(0xffffffffu, inc.a.y, 4);
    exc.b.x = __shfl_up_sync(0xffffffffu, inc.b.x, 4);
    exc.b.y = __shfl_up_sync(0xffffffffu, inc.b.y, 4);
    if (sl == 0) exc = Aff2{make_float2(1.0f, 1.0f), make_float2(0.0f, 0.0f)};
    if (sl == Cfg::SPW - 1)
      agg[(cq * WARPS + warp) * Cfg::PAIRS + cp] = make_float4(inc.a.x, inc.a.y, inc.b.x, inc.b.y);
    // the warp is done with its staged rows (the scan above took every lane's
    // steps): stage its rows of the next chunk
    if (c + 1 < nchunks) prefetch(K, c + 1);
    else if (!DSPLIT && K < 3) prefetch(K + 1, 0);
    __syncthreads();  // warp totals visible

    // ---- 3. incoming state: previous chunk's carry, earlier warps, earlier segments
    float2 h = make_float2(carry[cq * DT + 2 * cp], carry[cq * DT + 2 * cp + 1]);
    {  // all warp totals are loaded at once; earlier warps' maps applied in order
      float4 g4[WARPS - 1];
#pragma unroll
      for (int w = 0; w < WARPS - 1; ++w) g4[w] = agg[(cq * WARPS + w) * Cfg::PAIRS + cp];
#pragma unroll
      for (int w = 0; w < WARPS - 1; ++w)
        if (w < warp) h = __ffma2_rn(make_float2(g4[w].x, g4[w].y), h, make_float2(g4[w].z, g4[w].w));
    }
    h = __ffma2_rn(exc.a, h, exc.b);

    // ---- 4. replay, accumulate y at the visited pixels.  A whole chunk of a
    // whole channel tile (all but a direction's last chunk, all but a ragged
    // last tile) needs no per-step checks.
    if (whole_tile && l0 + LC <= Li) {
#pragma unroll
      for (int j = 0; j < TS; ++j) {
        if (!(ACC_SMEM ? in_bounds(rows[j] * DT + 2 * cp + 1, (int64_t)Hi * RS * DT, kBndWork)
                       : in_bounds((ib * L + rows[j]) * d_in + d0 + 2 * cp + 1, p.b * L * d_in,
                                   kBndWork)))
          continue;
        const float2 yv = __ffma2_rn(gg[j], h, yl[j]);
        float2 *d2 = reinterpret_cast<float2 *>(ACC_SMEM ? acc_s + rows[j] * DT + 2 * cp
                                                         : acc_g + rows[j] * di + 2 * cp);
        if constexpr (FIRST)
          *d2 = yv;
        else
          *d2 = __fadd2_rn(*d2, yv);
      }
    } else {
#pragma unroll
      for (int j = 0; j < TS; ++j) {
        if (ok0 && lb + j < Li &&
            (ACC_SMEM ? in_bounds(rows[j] * DT + 2 * cp + 1, (int64_t)Hi * RS * DT, kBndWork)
                      : in_bounds((ib * L + rows[j]) * d_in + d0 + 2 * cp + (ok1 ? 1 : 0),
                                  p.b * L * d_in, kBndWork))) {
          const float2 yv = __ffma2_rn(gg[j], h, yl[j]);
          float *dst = ACC_SMEM ? acc_s + rows[j] * DT + 2 * cp : acc_g + rows[j] * di + 2 * cp;
          if (ok1 && acc_pairs) {
            float2 *d2 = reinterpret_cast<float2 *>(dst);
            if constexpr (FIRST)
              *d2 = yv;
            else
              *d2 = __fadd2_rn(*d2, yv);
          } else {
            dst[0] = FIRST ? yv.x : dst[0] + yv.x;
            if (ok1) dst[1] = FIRST ? yv.y : dst[1] + yv.y;
          }
        }
      }
    }
    const bool last = c == nchunks - 1;
    if (warp == WARPS - 1 && sl == Cfg::SPW - 1) {  // the next direction starts from h = 0
      const float2 hend = __ffma2_rn(P, h, Q);  // the state after the chunk
      carry[(cq ^ 1) * DT + 2 * cp] = last ? 0.0f : hend.x;
      carry[(cq ^ 1) * DT + 2 * cp + 1] = last ? 0.0f : hend.y;
    }
  };

  for (int k = kz; k < (DSPLIT ? kz + 1 : 4); ++k) {
    const int64_t pk0 = k * d_in + dA;  // parameter rows of (direction, channel pair)
    A2 = make_float2(ok0 ? p.A[pk0] * kLog2e : 0.0f, ok1 ? p.A[pk0 + 1] * kLog2e : 0.0f);
    bias = make_float2((ok0 && p.dt_bias) ? p.dt_bias[pk0] : 0.0f,
                       (ok1 && p.dt_bias) ? p.dt_bias[pk0 + 1] : 0.0f);
    for (int c = 0; c < nchunks; ++c) {
      switch (k) {
        case 0: chunk(std::integral_constant<int, 0>{}, c); break;
        case 1: chunk(std::integral_constant<int, 1>{}, c); break;
        case 2: chunk(std::integral_constant<int, 2>{}, c); break;
        default: chunk(std::integral_constant<int, 3>{}, c); break;
      }
    }
  }
  __syncthreads();

  if constexpr (DSPLIT && !ACC_SMEM) {
    return;  // the replay wrote this direction's slice
  } else if constexpr (DSPLIT) {
    // ---- this direction's fp32 outputs, pixel-major, into workspace slice kz
    float *part = p.acc_global + ((int64_t)kz * p.b + ib) * L * d_in + d0;
    const int64_t n_part = 4 * p.b * L * d_in;
    if (d0 + DT <= d_in && (d_in & 3) == 0 && (reinterpret_cast<uintptr_t>(p.acc_global) & 15) == 0) {
      for (int pix = tid; pix < Li; pix += THREADS) {
        const int hh = div_small(pix, Wi, invW), w = pix - hh * Wi;
        if (!in_bounds(((int64_t)kz * p.b + ib) * L * d_in + (int64_t)pix * d_in + d0 + DT - 1,
                       n_part, kBndWork) ||
            !in_bounds((int64_t)(hh * RS + w) * DT + DT - 1, (int64_t)Hi * RS * DT, kBndWork))
          continue;
        const float4 *a4 = reinterpret_cast<const float4 *>(acc_s + (hh * RS + w) * DT);
        float4 *o = reinterpret_cast<float4 *>(part + (int64_t)pix * di);
        o[0] = a4[0];
        o[1] = a4[1];
      }
    } else {
      const int ch = tid & (DT - 1);
      if (d0 + ch < d_in) {
        for (int hh = 0; hh < Hi; ++hh) {
          for (int w = tid / DT; w < Wi; w += THREADS / DT) {
            const int pix = hh * Wi + w;
            if (!in_bounds(((int64_t)kz * p.b + ib) * L * d_in + (int64_t)pix * d_in + d0 + ch,
                           n_part, kBndWork))
              continue;
            part[(int64_t)pix * di + ch] = acc_s[(hh * RS + w) * DT + ch];
          }
        }
      }
    }
    return;
  }

  // ---- round once and store.  Shared accumulator, whole 8-channel tile and
  // 16-byte aligned rows: one pixel per thread, its 8 channels as one vector;
  // otherwise image row by image row, a channel per thread.
  if (ACC_SMEM && d0 + DT <= d_in && (d_in * Cfg::ESZ) % 16 == 0 &&
      (reinterpret_cast<uintptr_t>(p.y) & 15) == 0) {
    for (int pix = tid; pix < Li; pix += THREADS) {
      const int hh = div_small(pix, Wi, invW), w = pix - hh * Wi;
      if (!in_bounds((ib * L + pix) * d_in + d0 + DT - 1, p.b * L * d_in, kBndAct) ||
          !in_bounds((int64_t)(hh * RS + w) * DT + DT - 1, (int64_t)Hi * RS * DT, kBndWork))
        continue;
      const float4 *a4 = reinterpret_cast<const float4 *>(acc_s + (hh * RS + w) * DT);
      const float4 v0 = a4[0], v1 = a4[1];
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint4 *>(gy + pix * di) =
            make_uint4(pack_bf16x2(v0.x, v0.y), pack_bf16x2(v0.z, v0.w), pack_bf16x2(v1.x, v1.y),
                       pack_bf16x2(v1.z, v1.w));
      } else {
        float4 *o = reinterpret_cast<float4 *>(gy + pix * di);
        o[0] = v0;
        o[1] = v1;
      }
    }
  } else {
    const int ch = tid & (DT - 1);
    if (d0 + ch < d_in) {
      for (int hh = 0; hh < Hi; ++hh) {
        for (int w = tid / DT; w < Wi; w += THREADS / DT) {
          const int pix = hh * Wi + w;
          if (!in_bounds((ib * L + pix) * d_in + d0 + ch, p.b * L * d_in, kBndAct)) continue;
          const float v = ACC_SMEM ? acc_s[(hh * RS + w) * DT + ch] : acc_g[pix * di + ch];
          Elem<T>::store(gy, pix * di + ch, v);
        }
      }
    }
  }
}

// The direction split's merge: y = ((p0 + p1) + p2) + p3 over the four fp32
// slices (4, n) the DSPLIT kernel stored, rounded once to the activation
// dtype.  Four elements per thread when n is a multiple of 4 and parts and y
// are 16- and 8-byte aligned (VEC4).
template <typename T, bool VEC4>
__global__ void ss2d_merge4_kernel(const float *parts, T *y, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if constexpr (VEC4) {
    const float4 *p4 = reinterpret_cast<const float4 *>(parts);
    const int64_t n4 = n / 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += stride) {
      if (!in_bounds(3 * n4 + i, 4 * n4, kBndWork) || !in_bounds(4 * i + 3, n, kBndAct)) continue;
      float4 s = p4[i];
#pragma unroll
      for (int k = 1; k < 4; ++k) {
        const float4 v = p4[k * n4 + i];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint2 *>(y + 4 * i) = make_uint2(pack_bf16x2(s.x, s.y), pack_bf16x2(s.z, s.w));
      } else {
        *reinterpret_cast<float4 *>(y + 4 * i) = s;
      }
    }
  } else {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride) {
      if (!in_bounds(3 * n + i, 4 * n, kBndWork) || !in_bounds(i, n, kBndAct)) continue;
      float s = parts[i];
      s += parts[n + i];
      s += parts[2 * n + i];
      s += parts[3 * n + i];
      Elem<T>::store(y, i, s);
    }
  }
}

// ---------------------------------------------------------------------------
// CrossScan / CrossMerge as stored permutations (for checking the index
// arithmetic above bit-exactly).
// ---------------------------------------------------------------------------
template <typename T, int ORDER>
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
    const int64_t src = (ib * L + ss2d_pixel<ORDER>(k, l, H, W)) * d_in + d;
    if (in_bounds(src, b * L * d_in, kBndAct)) xs[i] = u[src];
  }
}

template <typename T, int ORDER>
__global__ void cross_merge_kernel(const T *ys, T *y, int64_t b, int64_t H, int64_t W,
                                   int64_t d_in) {
  const int64_t L = H * W;
  const int64_t total = b * L * d_in;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = i % d_in;
    const int64_t pix = (i / d_in) % L;
    const int64_t ib = i / (d_in * L);
    const int64_t hh = pix / W, ww = pix - hh * W;
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {  // summed k0 + k1 + k2 + k3, rounded once
      const int64_t src = ((ib * 4 + k) * L + ss2d_step_of<ORDER>(k, hh, ww, H, W)) * d_in + d;
      if (in_bounds(src, b * 4 * L * d_in, kBndAct)) s += Elem<T>::load(ys, src);
    }
    Elem<T>::store(y, i, s);
  }
}

}  // namespace ssm
