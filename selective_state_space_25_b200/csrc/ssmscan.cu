// ssmscan.cu -- the C ABI of libssmscan.so (include/ssmscan.h): argument
// validation, kernel selection and launch.  Every entry point validates all
// arguments before it touches CUDA, never allocates, never synchronises
// (except ssm_check_device_errors) and reports failures as ssm_status with a
// per-thread message.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>
#include <type_traits>

#include "ssmscan.h"
#include "scan_bwd.cuh"
#include "scan_fwd.cuh"
#include "scan_ws.cuh"
#include "ss2d_fwd.cuh"
#include "state_update.cuh"

namespace {

thread_local std::string g_last_error;

ssm_status fail(ssm_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

ssm_status ok() { return SSM_OK; }

bool mul_ok(int64_t a, int64_t b, int64_t *out) { return !__builtin_mul_overflow(a, b, out); }

bool supported_state(int64_t n) {
  return n == 1 || n == 2 || n == 4 || n == 8 || n == 16 || n == 32 || n == 64;
}

size_t esize(ssm_dtype t) { return t == SSM_BF16 ? 2 : 4; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A named byte range of one argument; NULL or empty ranges overlap nothing.
struct Span {
  const char *name;
  const void *p;
  int64_t bytes;
};

bool overlap(const Span &a, const Span &b) {
  if (!a.p || !b.p || a.bytes <= 0 || b.bytes <= 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
  return a0 < b0 + (uintptr_t)b.bytes && b0 < a0 + (uintptr_t)a.bytes;
}

// Outputs (and in-place buffers) must not overlap an input or each other.
// same_out / same_in name one output allowed to be exactly the given input
// (the same address: h_last == h0); any other overlap is an error.
ssm_status check_disjoint(const char *what, std::initializer_list<Span> outs,
                          std::initializer_list<Span> ins, const void *same_out = nullptr,
                          const void *same_in = nullptr) {
  for (const Span &o : outs) {
    for (const Span &i : ins) {
      if (same_out && o.p == same_out && i.p == same_in && o.p == i.p && o.bytes == i.bytes) continue;
      if (overlap(o, i))
        return fail(SSM_ERR_INVALID_ARG, "%s: %s overlaps the input %s", what, o.name, i.name);
    }
    for (const Span &o2 : outs)
      if (&o2 != &o && overlap(o, o2))
        return fail(SSM_ERR_INVALID_ARG, "%s: outputs %s and %s overlap", what, o.name, o2.name);
  }
  return SSM_OK;
}

ssm_status check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return ok();
}

// Launch with programmatic stream serialization: the kernel may start once
// every block of the previous kernel in the stream has called
// grid_dependents_launch (or exited), and calls grid_dependency_wait before
// it reads that kernel's results.
template <typename... KArgs, typename... Args>
ssm_status launch_dependent(void (*kernel)(KArgs...), dim3 grid, int threads, int smem,
                            cudaStream_t st, const char *what, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(SSM_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  }
  return ok();
}

// Opt a kernel into > 48 KB of dynamic shared memory once per device.
template <auto Kernel>
ssm_status ensure_smem(int bytes, const char *what) {
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(SSM_ERR_CUDA, "%s: cudaGetDevice failed", what);
  if (!done[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
      return fail(SSM_ERR_CUDA, "%s: cudaFuncSetAttribute: %s", what, cudaGetErrorString(e));
    done[dev] = true;
  }
  return ok();
}

// ------------------------------------------------------------ scan launch
// Tile shape of the fast scan kernel: channels per CTA, steps per chunk,
// states per thread, and how many of a thread's state pairs take the
// FMA-pipe exp2 instead of the SFU.
#ifndef SSM_SCAN_DT
#define SSM_SCAN_DT 32
#endif
#ifndef SSM_SCAN_TC
#define SSM_SCAN_TC 32
#endif
#ifndef SSM_SCAN_NPT
#define SSM_SCAN_NPT 4
#endif
#ifndef SSM_SCAN_NPOLY
#define SSM_SCAN_NPOLY 0
#endif

// States per thread: the requested count, halved until a CTA (DT channels x
// N / NPT threads) is whole warps, and at least 2.
constexpr int fast_npt(int n, int want, int dt) {
  int npt = want < n ? want : n;
  while (npt > 2 && (dt * (n / npt)) % 32 != 0) npt /= 2;
  while (n / npt > 32) npt *= 2;
  return npt;
}

#ifndef SSM_SCAN_BCF
#define SSM_SCAN_BCF 0
#endif

template <auto Kernel>
ssm_status launch_fast_kernel(const ssm::ScanParams &p, dim3 grid, int threads, int smem,
                              cudaStream_t st, bool dependent = false) {
  if (ssm_status s = ensure_smem<Kernel>(smem, "ssm_scan_fwd")) return s;
  if (!dependent) {
    Kernel<<<grid, threads, smem, st>>>(p);
    return check_launch("ssm_scan_fwd");
  }
  return launch_dependent(Kernel, grid, threads, smem, st, "ssm_scan_fwd", p);
}

template <typename T, int N, bool HAS_Z, int WANT_NPT>
ssm_status launch_scan_fast_npt(const ssm::ScanParams &p, cudaStream_t st) {
  constexpr int NPT = fast_npt(N, WANT_NPT, SSM_SCAN_DT);
  constexpr int DT = SSM_SCAN_DT, TC = SSM_SCAN_TC;
  constexpr int NPOLY = SSM_SCAN_NPOLY < NPT / 2 ? SSM_SCAN_NPOLY : NPT / 2;
  constexpr bool BCF = SSM_SCAN_BCF != 0 && sizeof(T) == 2;  // widen bf16 B / C once per CTA
  using Cfg = ssm::FastScan<T, N, NPT, DT, TC, BCF>;
  const dim3 grid((unsigned)((p.d_in + DT - 1) / DT), (unsigned)p.b);
  if (p.chunk_h)  // the forward that also saves chunk-start states
    return launch_fast_kernel<ssm::scan_fast_kernel<T, N, NPT, DT, TC, HAS_Z, NPOLY, BCF, true>>(
        p, grid, Cfg::THREADS, Cfg::SMEM, st);
  return launch_fast_kernel<ssm::scan_fast_kernel<T, N, NPT, DT, TC, HAS_Z, NPOLY, BCF, false>>(
      p, grid, Cfg::THREADS, Cfg::SMEM, st);
}

// Fewer channels leave fewer warps per SM: split each channel's states over
// more threads (2 per thread instead of 4) when b * d_in is below the size
// where the measured crossover lies.
#ifndef SSM_SCAN_SPLIT_CHANNELS
#define SSM_SCAN_SPLIT_CHANNELS 12288
#endif
constexpr int64_t kScanSplitChannels = SSM_SCAN_SPLIT_CHANNELS;

template <typename T, int N, bool HAS_Z>
ssm_status launch_scan_fast(const ssm::ScanParams &p, cudaStream_t st) {
  if (p.b * p.d_in < kScanSplitChannels)
    return launch_scan_fast_npt<T, N, HAS_Z, SSM_SCAN_NPT / 2>(p, st);
  return launch_scan_fast_npt<T, N, HAS_Z, SSM_SCAN_NPT>(p, st);
}

// Warp-specialised scan (scan_ws.cuh): steps per chunk, helper warps, and
// chunks copied ahead of the pre-pass.
#ifndef SSM_WS_TC
#define SSM_WS_TC 32
#endif
#ifndef SSM_WS_HELPERS
#define SSM_WS_HELPERS 4
#endif
#ifndef SSM_WS_AHEAD
#define SSM_WS_AHEAD 1
#endif

// States per scan thread of the warp-specialised kernel: 4 up to d_state 16,
// 8 for 32 (four scan warps either way); 0 = not compiled for this d_state.
constexpr int ws_states(int n) { return n == 8 || n == 16 ? 4 : (n == 32 ? 8 : 0); }

// SMs of the current device (148 on B200; also the answer when no device is
// visible, so the workspace query works on a host without a GPU).
int device_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// Split of the sequence into blocks (scan_ws.cuh, split scan) for problems
// whose b * ceil(d_in / 32) CTAs would leave more than half of the SMs idle:
// at most four CTAs per SM (two whole waves of the two a scan-pass SM holds),
// each block a whole number of chunks and at least four chunks long.
// nblk = 1: one pass.  Depends on the sizes only, so
// ssm_scan_fwd_workspace_bytes and the launch agree.  Measured on B200
// (b = 1, L = 16384, N = 16, bf16): d_in = 256 575 -> 74 us, d_in = 1536
// 575 -> 313 us (329 us when the block count rounded up, a third wave);
// at d_in = 4096 (128 CTAs) one pass is faster (577 against 754 us), hence
// the half-the-SMs threshold.
struct SplitPlan {
  int64_t nblk = 1, Lb = 0;
};
SplitPlan split_plan(int64_t b, int64_t L, int64_t d_in, int64_t N) {
  SplitPlan sp;
  if (b <= 0 || L <= 0 || d_in <= 0 || d_in % 8 != 0 || !(N == 8 || N == 16 || N == 32)) return sp;
  const int64_t sms = device_sms();
  const int64_t ctas = b * ((d_in + 31) / 32);
  if (2 * ctas > sms) return sp;
  int64_t nblk = 4 * sms / ctas;  // two whole waves of two CTAs per SM
  const int64_t by_len = L / (4 * SSM_WS_TC);
  if (nblk > by_len) nblk = by_len;
  if (nblk > 4096) nblk = 4096;
  if (nblk < 2) return sp;
  const int64_t per = (L + nblk - 1) / nblk;
  sp.Lb = (per + SSM_WS_TC - 1) / SSM_WS_TC * SSM_WS_TC;
  sp.nblk = (L + sp.Lb - 1) / sp.Lb;
  if (sp.nblk < 2) sp = SplitPlan{};
  return sp;
}

template <typename T, int N, bool HAS_Z, bool SAVE, bool SUMMARY>
ssm_status launch_scan_ws_pass(const ssm::ScanParams &p, unsigned nz, cudaStream_t st,
                               bool dependent = false) {
  constexpr int NS = ws_states(N);
  using Cfg = ssm::WsScan<T, N, NS, SSM_WS_TC, SSM_WS_HELPERS, SSM_WS_AHEAD>;
  constexpr auto k = ssm::scan_ws_kernel<T, N, NS, SSM_WS_TC, SSM_WS_HELPERS, SSM_WS_AHEAD,
                                         HAS_Z, SAVE, SUMMARY>;
  const dim3 grid((unsigned)((p.d_in + Cfg::DT - 1) / Cfg::DT), (unsigned)p.b, nz);
  return launch_fast_kernel<k>(p, grid, Cfg::THREADS, Cfg::SMEM, st, dependent);
}

template <typename T, int N, bool HAS_Z, bool SAVE>
ssm_status launch_scan_ws(const ssm::ScanParams &p, cudaStream_t st) {
  if (p.Lb <= 0) return launch_scan_ws_pass<T, N, HAS_Z, SAVE, false>(p, 1, st);
  // split scan: block summaries, the carry pass, then every block at once
  const unsigned nblk = (unsigned)((p.L + p.Lb - 1) / p.Lb);
  if (ssm_status s = launch_scan_ws_pass<T, N, false, false, true>(p, nblk - 1, st)) return s;
  // the carry and scan passes start while the pass before each finishes
  const int64_t chains = p.d_in * N;  // per batch
  if (ssm_status s = launch_dependent(ssm::scan_carry_kernel,
                                      dim3((unsigned)((chains + 31) / 32), (unsigned)p.b),
                                      ssm::kCarryThreads, 0, st, "ssm_scan_fwd", p.h0, p.blk_decay,
                                      (const float *)p.blk_state, p.b, (int64_t)nblk, p.d_in,
                                      (int)N))
    return s;
  return launch_scan_ws_pass<T, N, HAS_Z, SAVE, false>(p, nblk, st, true);
}

template <typename T, int N>
ssm_status launch_scan(const ssm::ScanParams &p, bool fast, cudaStream_t st) {
  if constexpr (ws_states(N) > 0) {
    if (fast) {
      if (p.chunk_h)
        return p.z ? launch_scan_ws<T, N, true, true>(p, st) : launch_scan_ws<T, N, false, true>(p, st);
      return p.z ? launch_scan_ws<T, N, true, false>(p, st) : launch_scan_ws<T, N, false, false>(p, st);
    }
  } else if constexpr (N >= 8) {
    if (fast)
      return p.z ? launch_scan_fast<T, N, true>(p, st) : launch_scan_fast<T, N, false>(p, st);
  }
  const int64_t threads = p.b * p.d_in;
  const int block = 128;
  ssm::scan_generic_kernel<T, N><<<(unsigned)((threads + block - 1) / block), block, 0, st>>>(p);
  return check_launch("ssm_scan_fwd");
}

template <typename T>
ssm_status dispatch_scan_n(const ssm::ScanParams &p, int64_t N, bool fast, cudaStream_t st) {
  switch (N) {
    case 1: return launch_scan<T, 1>(p, fast, st);
    case 2: return launch_scan<T, 2>(p, fast, st);
    case 4: return launch_scan<T, 4>(p, fast, st);
    case 8: return launch_scan<T, 8>(p, fast, st);
    case 16: return launch_scan<T, 16>(p, fast, st);
    case 32: return launch_scan<T, 32>(p, fast, st);
    case 64: return launch_scan<T, 64>(p, fast, st);
  }
  return fail(SSM_ERR_UNSUPPORTED, "d_state %lld not compiled", (long long)N);
}

// L == 0: the last state is the start state (or zeros).
__global__ void copy_or_zero_kernel(const float *src, float *dst, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src ? src[i] : 0.0f;
}

// ------------------------------------------------------------ step launch
#ifndef SSM_STEP_CPT
#define SSM_STEP_CPT 1
#endif
#ifndef SSM_CONV_STEP_CPT
#define SSM_CONV_STEP_CPT 1
#endif

template <typename T, int N, bool CONV>
ssm_status launch_step(const ssm::StepParams &p, cudaStream_t st, const char *what) {
  const int block = 256;
  if constexpr (N == 4 || N == 8 || N == 16) {  // one thread per channel, 32-byte vectors
    constexpr size_t al = N == 4 ? 16 : 32;
    if (aligned(p.state, al) && aligned(p.A, al) && aligned(p.B, al) && aligned(p.C, al)) {
      const int64_t threads = p.b * p.d_in;
      ssm::state_update_lane_kernel<T, N, CONV>
          <<<(unsigned)((threads + block - 1) / block), block, 0, st>>>(p);
      return check_launch(what);
    }
  }
  if constexpr (N >= 4) {
    if (aligned(p.state, 16) && aligned(p.A, 16) && aligned(p.B, 16) && aligned(p.C, 16)) {
      constexpr int CPT = CONV ? SSM_CONV_STEP_CPT : SSM_STEP_CPT;
      const int64_t per = (p.b * p.d_in + CPT - 1) / CPT;
      const int64_t threads = per * (N / 4);
      ssm::state_update_vec_kernel<T, N, CPT, CONV>
          <<<(unsigned)((threads + block - 1) / block), block, 0, st>>>(p);
      return check_launch(what);
    }
    if (aligned(p.state, 16)) {
      const int64_t threads = p.b * p.d_in * (N / 4);
      ssm::state_update_kernel<T, N, 4, CONV>
          <<<(unsigned)((threads + block - 1) / block), block, 0, st>>>(p);
      return check_launch(what);
    }
  }
  const int64_t threads = p.b * p.d_in;
  ssm::state_update_kernel<T, N, N, CONV>
      <<<(unsigned)((threads + block - 1) / block), block, 0, st>>>(p);
  return check_launch(what);
}

template <typename T, bool CONV>
ssm_status dispatch_step_n(const ssm::StepParams &p, int64_t N, cudaStream_t st, const char *what) {
  switch (N) {
    case 1: return launch_step<T, 1, CONV>(p, st, what);
    case 2: return launch_step<T, 2, CONV>(p, st, what);
    case 4: return launch_step<T, 4, CONV>(p, st, what);
    case 8: return launch_step<T, 8, CONV>(p, st, what);
    case 16: return launch_step<T, 16, CONV>(p, st, what);
    case 32: return launch_step<T, 32, CONV>(p, st, what);
    case 64: return launch_step<T, 64, CONV>(p, st, what);
  }
  return fail(SSM_ERR_UNSUPPORTED, "%s: d_state %lld not compiled", what, (long long)N);
}

// Shared validation of ssm_state_update and ssm_conv_state_update.
ssm_status check_step_args(const char *what, float *ssm_state, const void *x, const void *dt,
                           const float *A, const void *B, const void *C, const float *D,
                           const void *z, const float *dt_bias, void *y, int64_t b, int64_t d_in,
                           int64_t d_state, ssm_dtype dtype, bool *empty) {
  *empty = false;
  if (b < 0 || d_in < 0) return fail(SSM_ERR_INVALID_ARG, "%s: negative size", what);
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "%s: unknown dtype %d", what, (int)dtype);
  if (!supported_state(d_state))
    return fail(SSM_ERR_UNSUPPORTED, "%s: d_state %lld not in {1,2,4,8,16,32,64}", what,
                (long long)d_state);
  int64_t t;
  if (!mul_ok(b, d_in, &t) || !mul_ok(t, d_state, &t) || t > INT64_MAX / 8)
    return fail(SSM_ERR_INVALID_ARG, "%s: sizes overflow int64", what);
  if (b == 0 || d_in == 0) {
    *empty = true;
    return ok();
  }
  if (!ssm_state || !x || !dt || !A || !B || !C || !y)
    return fail(SSM_ERR_INVALID_ARG, "%s: ssm_state, x, dt, A, B, C and y are required", what);
  const size_t es = esize(dtype);
  const void *act[] = {x, dt, B, C, z, y};
  for (const void *q : act)
    if (q && !aligned(q, es))
      return fail(SSM_ERR_INVALID_ARG, "%s: activation pointer not %zu-byte aligned", what, es);
  const void *f32[] = {ssm_state, A, D, dt_bias};
  for (const void *q : f32)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "%s: fp32 pointer not 4-byte aligned", what);
  const int64_t na = b * d_in * (int64_t)es, ns = b * d_in * d_state * 4;
  const int64_t nbc = b * d_state * (int64_t)es, np = d_in * 4;
  return check_disjoint(what, {{"ssm_state", ssm_state, ns}, {"y", y, na}},
                        {{"x", x, na}, {"dt", dt, na}, {"z", z, na}, {"B", B, nbc}, {"C", C, nbc},
                         {"A", A, np * d_state}, {"D", D, np}, {"dt_bias", dt_bias, np}});
}

unsigned grid_for(int64_t n) {
  const int64_t blocks = (n + 255) / 256;
  return (unsigned)(blocks < 148 * 32 ? (blocks > 0 ? blocks : 1) : 148 * 32);
}

// ------------------------------------------------------------ SS2D launch
// Segment length (odd), warps per CTA, and whether dA uses the FMA-pipe exp2.
#ifndef SSM_SS2D_TS
#define SSM_SS2D_TS 5
#endif
#ifndef SSM_SS2D_WARPS
#define SSM_SS2D_WARPS 8
#endif
#ifndef SSM_SS2D_APOLY
#define SSM_SS2D_APOLY 0
#endif
constexpr int kSs2dDT = 8;
// H RS (RS = W rounded up to odd) of the shared-memory fp32 accumulator, 32 B each
constexpr int64_t kSs2dSmemPixels = 6272;
int64_t ss2d_acc_pixels(int64_t H, int64_t W) { return H * (W | 1); }

// The direction split (ss2d_fwd.cuh, DSPLIT) runs one CTA per (tile,
// direction) when the caller's workspace holds the four fp32 direction
// slices (4, b, H W, d_in): for images whose accumulator would live in the
// workspace (the slices are only written, where that accumulator takes a
// read-modify-write per direction on the replay's path: 2.7-6.5x faster at
// 112 x 112), and for problems whose b * ceil(d_in / 8) CTAs would leave
// more than half of the SMs idle.
bool ss2d_dsplit_applies(int64_t b, int64_t H, int64_t W, int64_t d_in) {
  return b <= 65535 && (ss2d_acc_pixels(H, W) > kSs2dSmemPixels ||
                        2 * b * ((d_in + kSs2dDT - 1) / kSs2dDT) <= device_sms());
}

template <typename T, bool ACC_SMEM, bool ROW_ASYNC, bool BC_ASYNC, int ORDER, bool DSPLIT>
ssm_status launch_ss2d_cfg(const ssm::Ss2dParams &p, cudaStream_t st) {
  using Cfg = ssm::Ss2dCfg<T, SSM_SS2D_TS, SSM_SS2D_WARPS, ACC_SMEM>;
  constexpr auto k = ssm::ss2d_n1_kernel<T, SSM_SS2D_TS, SSM_SS2D_WARPS, ACC_SMEM,
                                         SSM_SS2D_APOLY != 0, ROW_ASYNC, BC_ASYNC, ORDER, DSPLIT>;
  const int smem =
      Cfg::AUX_BYTES + (ACC_SMEM ? (int)(ss2d_acc_pixels(p.H, p.W) * kSs2dDT * sizeof(float)) : 0);
  if (ssm_status s = ensure_smem<k>(Cfg::AUX_BYTES + (int)(kSs2dSmemPixels * kSs2dDT * 4),
                                    "ss2d_scan_fwd"))
    return s;
  const dim3 grid((unsigned)((p.d_in + kSs2dDT - 1) / kSs2dDT), (unsigned)p.b, DSPLIT ? 4u : 1u);
  k<<<grid, Cfg::THREADS, smem, st>>>(p);
  if (ssm_status s = check_launch("ss2d_scan_fwd")) return s;
  if constexpr (DSPLIT) {  // sum the four direction slices, round once
    const int64_t n = p.b * p.H * p.W * p.d_in;
    const bool vec4 = n % 4 == 0 && aligned(p.acc_global, 16) && aligned(p.y, 4 * sizeof(T));
    const unsigned blocks = grid_for(vec4 ? n / 4 : n);
    if (vec4)
      ssm::ss2d_merge4_kernel<T, true><<<blocks, 256, 0, st>>>(p.acc_global, static_cast<T *>(p.y), n);
    else
      ssm::ss2d_merge4_kernel<T, false><<<blocks, 256, 0, st>>>(p.acc_global, static_cast<T *>(p.y), n);
    return check_launch("ss2d_scan_fwd");
  }
  return ok();
}

template <typename T, bool ACC_SMEM, int ORDER, bool DSPLIT = false>
ssm_status launch_ss2d_acc(const ssm::Ss2dParams &p, bool row_async, bool bc_async,
                           cudaStream_t st) {
  if (row_async)
    return bc_async ? launch_ss2d_cfg<T, ACC_SMEM, true, true, ORDER, DSPLIT>(p, st)
                    : launch_ss2d_cfg<T, ACC_SMEM, true, false, ORDER, DSPLIT>(p, st);
  return bc_async ? launch_ss2d_cfg<T, ACC_SMEM, false, true, ORDER, DSPLIT>(p, st)
                  : launch_ss2d_cfg<T, ACC_SMEM, false, false, ORDER, DSPLIT>(p, st);
}

template <typename T, int ORDER>
ssm_status launch_ss2d_order(const ssm::Ss2dParams &p, bool dsplit, cudaStream_t st) {
  const int64_t L = p.H * p.W;
  const size_t es = sizeof(T);
  const bool row_async = (p.d_in % kSs2dDT) == 0 && aligned(p.u, 16) && aligned(p.delta, 16);
  const bool bc_async = (L * (int64_t)es) % 16 == 0 && aligned(p.B, 16) && aligned(p.C, 16);
  if (ss2d_acc_pixels(p.H, p.W) <= kSs2dSmemPixels)
    return dsplit ? launch_ss2d_acc<T, true, ORDER, true>(p, row_async, bc_async, st)
                  : launch_ss2d_acc<T, true, ORDER>(p, row_async, bc_async, st);
  return dsplit ? launch_ss2d_acc<T, false, ORDER, true>(p, row_async, bc_async, st)
                : launch_ss2d_acc<T, false, ORDER>(p, row_async, bc_async, st);
}

template <typename T>
ssm_status launch_ss2d(const ssm::Ss2dParams &p, ssm_ss2d_order order, bool dsplit,
                       cudaStream_t st) {
  return order == SSM_SS2D_SNAKE ? launch_ss2d_order<T, ssm::kOrderSnake>(p, dsplit, st)
                                 : launch_ss2d_order<T, ssm::kOrderCross>(p, dsplit, st);
}


// ------------------------------------------------------------ backward scan
// States per thread of the backward kernel for d_state >= 4.
#ifndef SSM_BWD_NPT
#define SSM_BWD_NPT 2
#endif

constexpr int64_t bwd_chunk(int64_t) { return ssm::BwdCfg<float, 16, 4>::TT; }

template <typename T, int N, int NPT, bool ASYNC>
ssm_status launch_bwd_cfg(const ssm::BwdParams &p, unsigned nz, cudaStream_t st) {
  using Cfg = ssm::BwdCfg<T, N, NPT>;
  static_assert(Cfg::TT == bwd_chunk(N), "bwd_chunk must match BwdCfg");
  constexpr auto k = ssm::scan_bwd_kernel<T, N, NPT, ASYNC>;
  if (ssm_status s = ensure_smem<k>((int)Cfg::SMEM, "ssm_scan_bwd")) return s;
  const dim3 grid((unsigned)((p.d_in + Cfg::DT - 1) / Cfg::DT), (unsigned)p.b, nz);
  k<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(p);
  return check_launch("ssm_scan_bwd");
}

// Split backward (ssm_scan_bwd with the fast workspace, d_state 8, 16, 32):
// when b * ceil(d_in / channels per CTA) backward CTAs would leave more than
// half of the SMs idle, the chunks are cut into blocks -- at most two waves
// of three CTAs per SM, each block at least four chunks.  The chunk-start
// states come from the forward's split (when it splits) and the adjoint each
// block starts from from scan_bwd_adjoint_kernel + scan_carry_kernel.
struct BwdSplitPlan {
  int64_t nblk = 1, Cb = 0;     // backward blocks of Cb chunks
  SplitPlan fwd;                // the forward's split for the chunk-start states
};
int64_t bwd_channels_per_cta(int64_t N) {
  return 128 / (N / (N < 4 ? N : SSM_BWD_NPT));
}
BwdSplitPlan bwd_split_plan(int64_t b, int64_t L, int64_t d_in, int64_t N) {
  BwdSplitPlan sp;
  if (b <= 0 || L <= 0 || d_in <= 0 || !(N == 8 || N == 16 || N == 32)) return sp;
  const int64_t sms = device_sms();
  const int64_t ctas = b * ((d_in + bwd_channels_per_cta(N) - 1) / bwd_channels_per_cta(N));
  if (2 * ctas > sms) return sp;
  const int64_t nC = (L + bwd_chunk(N) - 1) / bwd_chunk(N);
  int64_t nblk = 6 * sms / ctas;
  if (nblk > nC / 4) nblk = nC / 4;
  if (nblk > 4096) nblk = 4096;
  if (nblk < 2) return sp;
  sp.Cb = (nC + nblk - 1) / nblk;
  sp.nblk = (nC + sp.Cb - 1) / sp.Cb;
  if (sp.nblk < 2) return BwdSplitPlan{};
  sp.fwd = split_plan(b, L, d_in, N);
  return sp;
}
// Extra fp32 words of the split after the chunk states: the forward split's
// block decays and states, then the backward's adjoint maps.
int64_t bwd_split_words(const BwdSplitPlan &sp, int64_t b, int64_t d_in, int64_t N) {
  return 2 * b * (sp.fwd.nblk > 1 ? sp.fwd.nblk : 0) * d_in * N + 2 * b * sp.nblk * d_in * N;
}

template <typename T, int N, int NPT>
ssm_status launch_bwd_main(const ssm::BwdParams &p, bool async, unsigned nz, cudaStream_t st) {
  if constexpr (ssm::bwd_async_ok<T, N, NPT>()) {
    if (async) return launch_bwd_cfg<T, N, NPT, true>(p, nz, st);
  }
  return launch_bwd_cfg<T, N, NPT, false>(p, nz, st);
}

template <typename T, int N>
ssm_status launch_bwd_split(const ssm::BwdParams &p, bool async, const BwdSplitPlan &sp,
                            float *extra, cudaStream_t st) {
  constexpr int NPT = N < 4 ? N : SSM_BWD_NPT;
  if constexpr (ws_states(N) > 0) {
    // 1. chunk-start states (unless saved): the forward's states pass, split
    // like the forward
    ssm::ScanParams f{p.u, p.delta, p.A, p.B, p.C, nullptr, nullptr, p.dt_bias, p.h0,
                      nullptr, nullptr, p.b, p.L, p.d_in, p.softplus, p.chunk_h};
    float *adj = extra;
    if (p.states_saved) {
      // the states are there already; `extra` holds the adjoint's maps only
    } else if (sp.fwd.nblk > 1) {
      f.Lb = sp.fwd.Lb;
      f.blk_decay = extra;
      f.blk_state = extra + p.b * sp.fwd.nblk * p.d_in * N;
      adj = extra + 2 * p.b * sp.fwd.nblk * p.d_in * N;
      const unsigned nb = (unsigned)sp.fwd.nblk;
      if (ssm_status s = launch_scan_ws_pass<T, N, false, false, true>(f, nb - 1, st)) return s;
      if (ssm_status s = launch_dependent(
              ssm::scan_carry_kernel, dim3((unsigned)((p.d_in * N + 31) / 32), (unsigned)p.b),
              ssm::kCarryThreads, 0, st, "ssm_scan_bwd", p.h0, f.blk_decay,
              (const float *)f.blk_state, p.b, (int64_t)nb, p.d_in, (int)N))
        return s;
      if (ssm_status s = launch_scan_ws_pass<T, N, false, true, true>(f, nb, st, true)) return s;
    } else if (ssm_status s = launch_scan_ws_pass<T, N, false, true, true>(f, 1, st)) {
      return s;
    }
    // 2. each block's adjoint map, then the adjoint each block starts from
    ssm::BwdParams q = p;
    q.states_saved = 1;
    q.Cb = sp.Cb;
    float *adj_decay = adj, *adj_state = adj + p.b * sp.nblk * p.d_in * N;
    const dim3 agrid((unsigned)((p.d_in + ssm::kAdjChannels - 1) / ssm::kAdjChannels),
                     (unsigned)(sp.nblk - 1), (unsigned)p.b);
    if (async)
      ssm::scan_bwd_adjoint_kernel<T, N, true><<<agrid, 128, 0, st>>>(q, adj_decay, adj_state);
    else
      ssm::scan_bwd_adjoint_kernel<T, N, false><<<agrid, 128, 0, st>>>(q, adj_decay, adj_state);
    if (ssm_status s = check_launch("ssm_scan_bwd")) return s;
    if (ssm_status s = launch_dependent(
            ssm::scan_carry_kernel, dim3((unsigned)((p.d_in * N + 31) / 32), (unsigned)p.b),
            ssm::kCarryThreads, 0, st, "ssm_scan_bwd", p.dh_last, adj_decay,
            (const float *)adj_state, p.b, sp.nblk, p.d_in, (int)N))
      return s;
    // 3. every block's backward at once
    q.lam_in = adj_decay;
    return launch_bwd_main<T, N, NPT>(q, async, (unsigned)sp.nblk, st);
  } else {
    (void)p; (void)async; (void)sp; (void)extra; (void)st;
    return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_bwd: no split backward for d_state %d", N);
  }
}

template <typename T, int N>
ssm_status launch_bwd(const ssm::BwdParams &p, bool async, bool fwd_states, cudaStream_t st) {
  constexpr int NPT = N < 4 ? N : SSM_BWD_NPT;
  if constexpr (ws_states(N) > 0) {
    if (fwd_states && !p.states_saved) {
      // the chunk-start states come from the forward kernel's states pass
      // (no C, gate or output), written where the backward's own first
      // pass would write them; the backward then starts from them
      ssm::ScanParams f{p.u, p.delta, p.A, p.B, p.C, nullptr, nullptr, p.dt_bias, p.h0,
                        nullptr, nullptr, p.b, p.L, p.d_in, p.softplus, p.chunk_h};
      if (ssm_status s = launch_scan_ws_pass<T, N, false, true, true>(f, 1, st)) return s;
      ssm::BwdParams q = p;
      q.states_saved = 1;
      if constexpr (ssm::bwd_async_ok<T, N, NPT>()) {
        if (async) return launch_bwd_cfg<T, N, NPT, true>(q, 1, st);
      }
      return launch_bwd_cfg<T, N, NPT, false>(q, 1, st);
    }
  }
  if constexpr (ssm::bwd_async_ok<T, N, NPT>()) {
    if (async) return launch_bwd_cfg<T, N, NPT, true>(p, 1, st);
  }
  return launch_bwd_cfg<T, N, NPT, false>(p, 1, st);
}

template <typename T>
ssm_status dispatch_bwd_split_n(const ssm::BwdParams &p, int64_t N, bool async,
                                const BwdSplitPlan &sp, float *extra, cudaStream_t st) {
  switch (N) {
    case 8: return launch_bwd_split<T, 8>(p, async, sp, extra, st);
    case 16: return launch_bwd_split<T, 16>(p, async, sp, extra, st);
    case 32: return launch_bwd_split<T, 32>(p, async, sp, extra, st);
  }
  return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_bwd: no split backward for d_state %lld",
              (long long)N);
}

template <typename T>
ssm_status dispatch_bwd_n(const ssm::BwdParams &p, int64_t N, bool async, bool fwd_states,
                          cudaStream_t st) {
  switch (N) {
    case 1: return launch_bwd<T, 1>(p, async, fwd_states, st);
    case 2: return launch_bwd<T, 2>(p, async, fwd_states, st);
    case 4: return launch_bwd<T, 4>(p, async, fwd_states, st);
    case 8: return launch_bwd<T, 8>(p, async, fwd_states, st);
    case 16: return launch_bwd<T, 16>(p, async, fwd_states, st);
    case 32: return launch_bwd<T, 32>(p, async, fwd_states, st);
    case 64: return launch_bwd<T, 64>(p, async, fwd_states, st);
  }
  return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_bwd: d_state %lld not compiled", (long long)N);
}

}  // namespace

// ============================================================== C ABI
extern "C" {

const char *ssm_last_error(void) { return g_last_error.c_str(); }

const char *ssm_version(void) { return "0.1.0"; }

size_t ssm_scan_fwd_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state) {
  int64_t t;
  if (b < 0 || L < 0 || d_in < 0 || d_state < 1 || !mul_ok(b, L, &t) || !mul_ok(t, d_in, &t) ||
      !mul_ok(t, d_state, &t))
    return (size_t)-1;
  const SplitPlan sp = split_plan(b, L, d_in, d_state);
  if (sp.nblk <= 1) return 0;
  // block decays and block states, (b, nblk, d_in, d_state) fp32 each
  return (size_t)(2 * b * sp.nblk * d_in * d_state) * sizeof(float);
}

}  // extern "C"

namespace {

ssm_status scan_fwd_impl(const void *u, const void *delta, const float *A, const void *B,
                         const void *C, const float *D, const void *z, const float *dt_bias,
                         int delta_softplus, const float *h0, float *h_last, void *y, int64_t b,
                         int64_t L, int64_t d_in, int64_t d_state, ssm_dtype dtype,
                         void *workspace, size_t workspace_bytes, float *chunk_h,
                         ssm_stream_t stream) {
  g_last_error.clear();
  if (b < 0 || L < 0 || d_in < 0)
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: negative size (b=%lld L=%lld d_in=%lld)",
                (long long)b, (long long)L, (long long)d_in);
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_fwd: unknown dtype %d", (int)dtype);
  if (!supported_state(d_state))
    return fail(SSM_ERR_UNSUPPORTED, "ssm_scan_fwd: d_state %lld not in {1,2,4,8,16,32,64}",
                (long long)d_state);
  int64_t n_act, n_bc, n_state;
  if (!mul_ok(b, L, &n_act) || !mul_ok(n_act, d_in, &n_act) || !mul_ok(b, L, &n_bc) ||
      !mul_ok(n_bc, d_state, &n_bc) || !mul_ok(b, d_in, &n_state) ||
      !mul_ok(n_state, d_state, &n_state) || n_act > INT64_MAX / 4)
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: sizes overflow int64");
  // The split scan's workspace: the plain forward requires it; the forward
  // that saves chunk states takes the split only when given one (16-byte
  // aligned) and otherwise runs in one pass.
  const size_t split_bytes = ssm_scan_fwd_workspace_bytes(b, L, d_in, d_state);
  const size_t need = chunk_h ? 0 : split_bytes;
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(SSM_ERR_WORKSPACE, "ssm_scan_fwd: workspace %zu bytes < %zu needed",
                workspace_bytes, need);
  if (need > 0 && !aligned(workspace, 16))
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: workspace not 16-byte aligned");
  if (chunk_h && workspace && !aligned(workspace, 4))
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd_save: workspace not 4-byte aligned");
  const bool split = split_bytes > 0 && split_bytes != (size_t)-1 &&
                     (!chunk_h || (workspace && workspace_bytes >= split_bytes &&
                                   aligned(workspace, 16)));
  if (b == 0 || d_in == 0) return ok();
  if (!A) return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: A is NULL");
  if (L > 0 && (!u || !delta || !B || !C || !y))
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: u, delta, B, C and y are required");
  const size_t es = esize(dtype);
  const void *act[] = {u, delta, B, C, z, y};
  for (const void *q : act)
    if (q && !aligned(q, es))
      return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: activation pointer not %zu-byte aligned", es);
  const void *f32[] = {A, D, dt_bias, h0, h_last};
  for (const void *q : f32)
    if (q && !aligned(q, 4))
      return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd: fp32 pointer not 4-byte aligned");
  {
    const int64_t ba = n_act * (int64_t)es, bbc = n_bc * (int64_t)es, bs = n_state * 4;
    const int64_t nc = chunk_h ? (int64_t)ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state) : 0;
    if (ssm_status s = check_disjoint(
            "ssm_scan_fwd",
            {{"y", y, ba}, {"h_last", h_last, bs}, {"chunk_states", chunk_h, nc},
             {"workspace", split ? workspace : nullptr, split ? (int64_t)split_bytes : 0}},
            {{"u", u, ba}, {"delta", delta, ba}, {"z", z, ba}, {"B", B, bbc}, {"C", C, bbc},
             {"A", A, d_in * d_state * 4}, {"D", D, d_in * 4}, {"dt_bias", dt_bias, d_in * 4},
             {"h0", h0, bs}},
            h_last, h0))
      return s;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (L == 0) {  // no steps: the last state is the start state (or zeros)
    if (h_last && h_last != h0) {
      copy_or_zero_kernel<<<grid_for(n_state), 256, 0, st>>>(h0, h_last, n_state);
      return check_launch("ssm_scan_fwd");
    }
    return ok();
  }

  ssm::ScanParams p{u, delta, A, B, C, D, z, dt_bias, h0, h_last, y, b, L, d_in, delta_softplus,
                    chunk_h};
  if (split) {  // the split scan (its plan is the one split_bytes was sized for)
    const SplitPlan sp = split_plan(b, L, d_in, d_state);
    p.Lb = sp.Lb;
    p.blk_decay = static_cast<float *>(workspace);
    p.blk_state = p.blk_decay + b * sp.nblk * d_in * d_state;
  }
  const bool fast = d_state >= 8 && (d_in * (int64_t)es) % 16 == 0 && aligned(u, 16) &&
                    aligned(delta, 16) && aligned(B, 16) && aligned(C, 16) && aligned(y, 16) &&
                    (!z || aligned(z, 16)) && b <= 65535;
  if (dtype == SSM_BF16) return dispatch_scan_n<__nv_bfloat16>(p, d_state, fast, st);
  return dispatch_scan_n<float>(p, d_state, fast, st);
}

}  // namespace

extern "C" {

ssm_status ssm_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *dt_bias,
                        int delta_softplus, const float *h0, float *h_last, void *y, int64_t b,
                        int64_t L, int64_t d_in, int64_t d_state, ssm_dtype dtype,
                        void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, h_last, y, b, L,
                       d_in, d_state, dtype, workspace, workspace_bytes, nullptr, stream);
}

ssm_status ssm_scan_fwd_save_ex(const void *u, const void *delta, const float *A,
                                const void *B, const void *C, const float *D, const void *z,
                                const float *dt_bias, int delta_softplus, const float *h0,
                                float *h_last, void *y, float *chunk_states,
                                size_t chunk_states_bytes, int64_t b, int64_t L, int64_t d_in,
                                int64_t d_state, ssm_dtype dtype, void *workspace,
                                size_t workspace_bytes, ssm_stream_t stream) {
  g_last_error.clear();
  const size_t need = ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state);
  if (need == (size_t)-1)
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd_save: invalid sizes");
  if (chunk_states_bytes < need || (need > 0 && !chunk_states))
    return fail(SSM_ERR_WORKSPACE, "ssm_scan_fwd_save: chunk_states %zu bytes < %zu needed",
                chunk_states_bytes, need);
  if (chunk_states && !aligned(chunk_states, 16))
    return fail(SSM_ERR_INVALID_ARG, "ssm_scan_fwd_save: chunk_states not 16-byte aligned");
  if (need == 0)  // no chunk starts (b, L or d_in of 0): a plain forward
    return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, h_last, y, b, L,
                         d_in, d_state, dtype, nullptr, 0, nullptr, stream);
  return scan_fwd_impl(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, h_last, y, b, L,
                       d_in, d_state, dtype, workspace, workspace_bytes, chunk_states, stream);
}

ssm_status ssm_scan_fwd_save(const void *u, const void *delta, const float *A, const void *B,
                             const void *C, const float *D, const void *z, const float *dt_bias,
                             int delta_softplus, const float *h0, float *h_last, void *y,
                             float *chunk_states, size_t chunk_states_bytes, int64_t b,
                             int64_t L, int64_t d_in, int64_t d_state, ssm_dtype dtype,
                             ssm_stream_t stream) {
  return ssm_scan_fwd_save_ex(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, h_last, y,
                              chunk_states, chunk_states_bytes, b, L, d_in, d_state, dtype,
                              nullptr, 0, stream);
}

size_t ssm_scan_bwd_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state) {
  int64_t t;
  if (b < 0 || L < 0 || d_in < 0 || !supported_state(d_state)) return (size_t)-1;
  const int64_t n_chunks = (L + bwd_chunk(d_state) - 1) / bwd_chunk(d_state);
  if (!mul_ok(b, n_chunks, &t) || !mul_ok(t, d_in, &t) || !mul_ok(t, d_state, &t) ||
      t > INT64_MAX / 8)
    return (size_t)-1;
  return (size_t)t * sizeof(float);
}

size_t ssm_scan_bwd_fast_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state) {
  const size_t need = ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state);
  if (need == (size_t)-1) return need;
  const BwdSplitPlan sp = bwd_split_plan(b, L, d_in, d_state);
  if (sp.nblk < 2) return need;
  return need + (size_t)bwd_split_words(sp, b, d_in, d_state) * sizeof(float);
}

}  // extern "C"

namespace {

ssm_status scan_bwd_impl(const char *what, const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *D, const void *z,
                         const float *dt_bias, int delta_softplus, const float *h0,
                         const void *dout, const float *dh_last, void *du, void *ddelta,
                         float *dA, float *dB, float *dC, float *dD, void *dz, float *ddt_bias,
                         float *dh0, int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                         ssm_dtype dtype, void *workspace, size_t workspace_bytes,
                         int states_saved, ssm_stream_t stream, void *aux = nullptr,
                         size_t aux_bytes = 0) {
  g_last_error.clear();
  if (b < 0 || L < 0 || d_in < 0)
    return fail(SSM_ERR_INVALID_ARG, "%s: negative size (b=%lld L=%lld d_in=%lld)", what,
                (long long)b, (long long)L, (long long)d_in);
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "%s: unknown dtype %d", what, (int)dtype);
  if (!supported_state(d_state))
    return fail(SSM_ERR_UNSUPPORTED, "%s: d_state %lld not in {1,2,4,8,16,32,64}", what,
                (long long)d_state);
  int64_t n_act, n_bc, n_state;
  if (!mul_ok(b, L, &n_act) || !mul_ok(n_act, d_in, &n_act) || !mul_ok(b, L, &n_bc) ||
      !mul_ok(n_bc, d_state, &n_bc) || !mul_ok(b, d_in, &n_state) ||
      !mul_ok(n_state, d_state, &n_state) || n_act > INT64_MAX / 4 || n_bc > INT64_MAX / 4)
    return fail(SSM_ERR_INVALID_ARG, "%s: sizes overflow int64", what);
  const size_t need = ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state);
  if (need == (size_t)-1) return fail(SSM_ERR_INVALID_ARG, "%s: sizes overflow int64", what);
  if (b == 0 || d_in == 0) return ok();
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(SSM_ERR_WORKSPACE, "%s: workspace %zu bytes < %zu needed", what, workspace_bytes,
                need);
  if (b > 65535) return fail(SSM_ERR_UNSUPPORTED, "%s: b %lld > 65535", what, (long long)b);
  if (!A || !dA) return fail(SSM_ERR_INVALID_ARG, "%s: A and dA are required", what);
  if (L > 0 && (!u || !delta || !B || !C || !dout || !du || !ddelta || !dB || !dC))
    return fail(SSM_ERR_INVALID_ARG,
                "%s: u, delta, B, C, dout, du, ddelta, dB and dC are required", what);
  const size_t es = esize(dtype);
  const void *act[] = {u, delta, B, C, z, dout, du, ddelta, dz};
  for (const void *q : act)
    if (q && !aligned(q, es))
      return fail(SSM_ERR_INVALID_ARG, "%s: activation pointer not %zu-byte aligned", what, es);
  const void *f32[] = {A, D, dt_bias, h0, dh_last, dA, dB, dC, dD, ddt_bias, dh0, workspace};
  for (const void *q : f32)
    if (q && !aligned(q, 4))
      return fail(SSM_ERR_INVALID_ARG, "%s: fp32 pointer not 4-byte aligned", what);
  // the forward kernel's states pass needs its own 16-byte staging of u, delta, B
  const bool fwd_states = (d_in * (int64_t)es) % 16 == 0 && aligned(u, 16) &&
                          aligned(delta, 16) && aligned(B, 16) && b <= 65535;
  // The split backward.  Self-contained: when the workspace holds its block
  // buffers after the chunk states and the forward kernel can write those
  // states.  From saved states: when `aux` holds the adjoint's block maps.
  // `used` is the scratch the call writes (the workspace, or `aux`).
  bool split;
  size_t used;
  if (states_saved) {
    const size_t aux_need = ssm_scan_bwd_saved_workspace_bytes(b, L, d_in, d_state);
    split = aux_need > 0 && aux && aux_bytes >= aux_need && aligned(aux, 16);
    used = split ? aux_need : 0;
  } else {
    const size_t fast = ssm_scan_bwd_fast_workspace_bytes(b, L, d_in, d_state);
    split = fwd_states && fast > need && workspace && workspace_bytes >= fast &&
            aligned(workspace, 16);
    used = split ? fast : need;
  }
  if (aux && !aligned(aux, 4))
    return fail(SSM_ERR_INVALID_ARG, "%s: workspace not 4-byte aligned", what);
  {
    const int64_t ba = n_act * (int64_t)es, bbc = n_bc * (int64_t)es, bs = n_state * 4;
    const int64_t bp = d_in * 4, bA = d_in * d_state * 4;
    const Span ws{"workspace", states_saved ? aux : workspace, (int64_t)used};
    // from saved states the caller's `workspace` is the chunk states, read only
    const Span ws_in{"chunk_states", states_saved ? workspace : nullptr, (int64_t)need};
    if (ssm_status s = check_disjoint(
            what,
            {{"du", du, ba}, {"ddelta", ddelta, ba}, {"dz", z ? dz : nullptr, ba}, {"dA", dA, bA},
             {"dB", dB, n_bc * 4}, {"dC", dC, n_bc * 4}, {"dD", dD, bp},
             {"ddt_bias", ddt_bias, bp}, {"dh0", dh0, bs}, ws},
            {{"u", u, ba}, {"delta", delta, ba}, {"z", z, ba}, {"dout", dout, ba}, {"B", B, bbc},
             {"C", C, bbc}, {"A", A, bA}, {"D", D, bp}, {"dt_bias", dt_bias, bp}, {"h0", h0, bs},
             {"dh_last", dh_last, bs}, ws_in}))
      return s;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the sums over channels and over the batch accumulate into zeroed outputs
  cudaError_t e = cudaMemsetAsync(dA, 0, (size_t)(d_in * d_state) * sizeof(float), st);
  if (e == cudaSuccess && L > 0) e = cudaMemsetAsync(dB, 0, (size_t)n_bc * sizeof(float), st);
  if (e == cudaSuccess && L > 0) e = cudaMemsetAsync(dC, 0, (size_t)n_bc * sizeof(float), st);
  if (e == cudaSuccess && dD) e = cudaMemsetAsync(dD, 0, (size_t)d_in * sizeof(float), st);
  if (e == cudaSuccess && ddt_bias)
    e = cudaMemsetAsync(ddt_bias, 0, (size_t)d_in * sizeof(float), st);
  if (e != cudaSuccess)
    return fail(SSM_ERR_CUDA, "%s: cudaMemsetAsync: %s", what, cudaGetErrorString(e));
  if (L == 0) {  // no steps: the gradient reaching h0 is dh_last
    if (dh0) {
      copy_or_zero_kernel<<<grid_for(n_state), 256, 0, st>>>(dh_last, dh0, n_state);
      return check_launch(what);
    }
    return ok();
  }
  ssm::BwdParams p{u, delta, A, B, C, D, z, dt_bias, h0, dout, dh_last, du, ddelta, dz,
                   dA, dB, dC, dD, ddt_bias, dh0, static_cast<float *>(workspace),
                   b, L, d_in, delta_softplus, aligned(dB, 16) && aligned(dC, 16), states_saved};
  // the raw-tile prefetch copies 16-byte groups straight from the inputs
  const bool async = (d_in * (int64_t)es) % 16 == 0 && aligned(u, 16) && aligned(delta, 16) &&
                     aligned(dout, 16) && aligned(B, 16) && aligned(C, 16) && (!z || aligned(z, 16));
  if (split) {
    const BwdSplitPlan sp = bwd_split_plan(b, L, d_in, d_state);
    float *extra = states_saved ? static_cast<float *>(aux)
                                : static_cast<float *>(workspace) + need / sizeof(float);
    if (dtype == SSM_BF16) return dispatch_bwd_split_n<__nv_bfloat16>(p, d_state, async, sp, extra, st);
    return dispatch_bwd_split_n<float>(p, d_state, async, sp, extra, st);
  }
  if (dtype == SSM_BF16)
    return dispatch_bwd_n<__nv_bfloat16>(p, d_state, async, fwd_states, st);
  return dispatch_bwd_n<float>(p, d_state, async, fwd_states, st);
}

}  // namespace

extern "C" {

ssm_status ssm_scan_bwd(const void *u, const void *delta, const float *A, const void *B,
                        const void *C, const float *D, const void *z, const float *dt_bias,
                        int delta_softplus, const float *h0, const void *dout,
                        const float *dh_last, void *du, void *ddelta, float *dA, float *dB,
                        float *dC, float *dD, void *dz, float *ddt_bias, float *dh0, int64_t b,
                        int64_t L, int64_t d_in, int64_t d_state, ssm_dtype dtype,
                        void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  return scan_bwd_impl("ssm_scan_bwd", u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0,
                       dout, dh_last, du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, b, L, d_in,
                       d_state, dtype, workspace, workspace_bytes, 0, stream);
}

size_t ssm_scan_bwd_saved_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state) {
  if (ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state) == (size_t)-1) return (size_t)-1;
  const BwdSplitPlan sp = bwd_split_plan(b, L, d_in, d_state);
  if (sp.nblk < 2) return 0;
  return (size_t)(2 * b * sp.nblk * d_in * d_state) * sizeof(float);
}

ssm_status ssm_scan_bwd_saved_ex(const void *u, const void *delta, const float *A, const void *B,
                                 const void *C, const float *D, const void *z,
                                 const float *dt_bias, int delta_softplus, const void *dout,
                                 const float *dh_last, void *du, void *ddelta, float *dA,
                                 float *dB, float *dC, float *dD, void *dz, float *ddt_bias,
                                 float *dh0, int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                                 ssm_dtype dtype, const float *chunk_states,
                                 size_t chunk_states_bytes, void *workspace,
                                 size_t workspace_bytes, ssm_stream_t stream) {
  return scan_bwd_impl("ssm_scan_bwd_saved", u, delta, A, B, C, D, z, dt_bias, delta_softplus,
                       nullptr, dout, dh_last, du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, b, L,
                       d_in, d_state, dtype, const_cast<float *>(chunk_states),
                       chunk_states_bytes, 1, stream, workspace, workspace_bytes);
}

ssm_status ssm_scan_bwd_saved(const void *u, const void *delta, const float *A, const void *B,
                              const void *C, const float *D, const void *z, const float *dt_bias,
                              int delta_softplus, const void *dout, const float *dh_last,
                              void *du, void *ddelta, float *dA, float *dB, float *dC, float *dD,
                              void *dz, float *ddt_bias, float *dh0, int64_t b, int64_t L,
                              int64_t d_in, int64_t d_state, ssm_dtype dtype,
                              const float *chunk_states, size_t chunk_states_bytes,
                              ssm_stream_t stream) {
  // the kernel only reads the saved states in this mode
  return scan_bwd_impl("ssm_scan_bwd_saved", u, delta, A, B, C, D, z, dt_bias, delta_softplus,
                       nullptr, dout, dh_last, du, ddelta, dA, dB, dC, dD, dz, ddt_bias, dh0, b, L,
                       d_in, d_state, dtype, const_cast<float *>(chunk_states),
                       chunk_states_bytes, 1, stream);
}

size_t ss2d_scan_fwd_workspace_bytes(int64_t b, int64_t H, int64_t W, int64_t d_in,
                                     int64_t d_state) {
  int64_t L, t;
  if (b < 0 || H < 0 || W < 0 || d_in < 0 || d_state < 1 || !mul_ok(H, W, &L) ||
      !mul_ok(b, L, &t) || !mul_ok(t, d_in, &t) || !mul_ok(t, 4 * d_state, &t) ||
      t > INT64_MAX / 8)
    return (size_t)-1;
  if (ss2d_acc_pixels(H, W) <= kSs2dSmemPixels) return 0;
  return (size_t)(b * L * d_in) * sizeof(float);
}

size_t ss2d_scan_fwd_fast_workspace_bytes(int64_t b, int64_t H, int64_t W, int64_t d_in,
                                          int64_t d_state) {
  const size_t need = ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, d_state);
  if (need == (size_t)-1 || d_state != 1 || !ss2d_dsplit_applies(b, H, W, d_in)) return need;
  return (size_t)(4 * b * H * W * d_in) * sizeof(float);  // overflow excluded by the check above
}

ssm_status ss2d_scan_fwd(const void *u, const void *delta, const float *A, const void *B,
                         const void *C, const float *D, const float *dt_bias, int delta_softplus,
                         void *y, int64_t b, int64_t H, int64_t W, int64_t d_in, int64_t d_state,
                         ssm_dtype dtype, void *workspace, size_t workspace_bytes,
                         ssm_stream_t stream) {
  return ss2d_scan_fwd_ex(u, delta, A, B, C, D, dt_bias, delta_softplus, y, b, H, W, d_in,
                          d_state, SSM_SS2D_CROSS, dtype, workspace, workspace_bytes, stream);
}

ssm_status ss2d_scan_fwd_ex(const void *u, const void *delta, const float *A, const void *B,
                            const void *C, const float *D, const float *dt_bias,
                            int delta_softplus, void *y, int64_t b, int64_t H, int64_t W,
                            int64_t d_in, int64_t d_state, ssm_ss2d_order order, ssm_dtype dtype,
                            void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  g_last_error.clear();
  if (order != SSM_SS2D_CROSS && order != SSM_SS2D_SNAKE)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_scan_fwd: unknown scan order %d", (int)order);
  if (b < 0 || H < 0 || W < 0 || d_in < 0)
    return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd: negative size");
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_scan_fwd: unknown dtype %d", (int)dtype);
  if (d_state != 1)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_scan_fwd: d_state %lld (only 1 is compiled)",
                (long long)d_state);
  const size_t need = ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, d_state);
  if (need == (size_t)-1) return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd: sizes overflow int64");
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(SSM_ERR_WORKSPACE, "ss2d_scan_fwd: workspace %zu bytes < %zu needed",
                workspace_bytes, need);
  const int64_t L = H * W;
  if (b == 0 || d_in == 0 || L == 0) return ok();
  if (L >= (int64_t(1) << 22) || L * d_in >= (int64_t(1) << 31))
    return fail(SSM_ERR_UNSUPPORTED,
                "ss2d_scan_fwd: H * W = %lld must be < 2^22 and H * W * d_in < 2^31", (long long)L);
  if (!u || !delta || !A || !B || !C || !y)
    return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd: u, delta, A, B, C and y are required");
  if (b > 65535) return fail(SSM_ERR_UNSUPPORTED, "ss2d_scan_fwd: b > 65535");
  const size_t es = esize(dtype);
  const void *act[] = {u, delta, B, C, y};
  for (const void *q : act)
    if (!aligned(q, es))
      return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd: activation pointer not %zu-byte aligned", es);
  const void *f32[] = {A, D, dt_bias, workspace};
  for (const void *q : f32)
    if (q && !aligned(q, 4))
      return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd: fp32 pointer not 4-byte aligned");
  // the direction split when the workspace holds its four fp32 slices
  const size_t fast = ss2d_scan_fwd_fast_workspace_bytes(b, H, W, d_in, d_state);
  const bool dsplit = fast > need && workspace && workspace_bytes >= fast;
  const size_t used = dsplit ? fast : need;
  {
    const int64_t by = b * L * d_in * (int64_t)es, bk = 4 * by, bbc = b * 4 * L * d_state * (int64_t)es;
    if (ssm_status s = check_disjoint(
            "ss2d_scan_fwd", {{"y", y, by}, {"workspace", workspace, (int64_t)used}},
            {{"u", u, by}, {"delta", delta, bk}, {"B", B, bbc}, {"C", C, bbc},
             {"A", A, 4 * d_in * d_state * 4}, {"D", D, 4 * d_in * 4},
             {"dt_bias", dt_bias, 4 * d_in * 4}}))
      return s;
  }

  ssm::Ss2dParams p{u, delta, A, B, C, D, dt_bias, y, static_cast<float *>(workspace),
                    b, H, W, d_in, delta_softplus};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSM_BF16) return launch_ss2d<__nv_bfloat16>(p, order, dsplit, st);
  return launch_ss2d<float>(p, order, dsplit, st);
}

ssm_status ssm_state_update(float *ssm_state, const void *x, const void *dt, const float *A,
                            const void *B, const void *C, const float *D, const void *z,
                            const float *dt_bias, int dt_softplus, void *y, int64_t b,
                            int64_t d_in, int64_t d_state, ssm_dtype dtype,
                            ssm_stream_t stream) {
  g_last_error.clear();
  bool empty = false;
  if (ssm_status s = check_step_args("ssm_state_update", ssm_state, x, dt, A, B, C, D, z, dt_bias,
                                     y, b, d_in, d_state, dtype, &empty))
    return s;
  if (empty) return ok();
  ssm::StepParams p{ssm_state, x, dt, A, B, C, D, z, dt_bias, y, b, d_in, dt_softplus,
                    nullptr, nullptr, nullptr, 0};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSM_BF16) return dispatch_step_n<__nv_bfloat16, false>(p, d_state, st, "ssm_state_update");
  return dispatch_step_n<float, false>(p, d_state, st, "ssm_state_update");
}

ssm_status ssm_conv_state_update(void *conv_state, const float *conv_weight, const float *conv_bias,
                                 int64_t d_conv, float *ssm_state, const void *x, const void *dt,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const float *dt_bias, int dt_softplus, void *y,
                                 int64_t b, int64_t d_in, int64_t d_state, ssm_dtype dtype,
                                 ssm_stream_t stream) {
  g_last_error.clear();
  const char *what = "ssm_conv_state_update";
  bool empty = false;
  if (ssm_status s = check_step_args(what, ssm_state, x, dt, A, B, C, D, z, dt_bias, y, b, d_in,
                                     d_state, dtype, &empty))
    return s;
  if (d_conv < 1 || d_conv > ssm::kMaxConv)
    return fail(SSM_ERR_UNSUPPORTED, "%s: d_conv %lld not in [1, %d]", what, (long long)d_conv,
                ssm::kMaxConv);
  if (empty) return ok();
  if (!conv_state || !conv_weight)
    return fail(SSM_ERR_INVALID_ARG, "%s: conv_state and conv_weight are required", what);
  if (!aligned(conv_state, esize(dtype)) || !aligned(conv_weight, 4) ||
      (conv_bias && !aligned(conv_bias, 4)))
    return fail(SSM_ERR_INVALID_ARG, "%s: misaligned conv pointer", what);
  {
    const int64_t es = (int64_t)esize(dtype), bw = b * d_in * d_conv * es;
    if (ssm_status s = check_disjoint(
            what, {{"conv_state", conv_state, bw}},
            {{"ssm_state", ssm_state, b * d_in * d_state * 4}, {"y", y, b * d_in * es},
             {"x", x, b * d_in * es}, {"dt", dt, b * d_in * es}, {"z", z, b * d_in * es},
             {"B", B, b * d_state * es}, {"C", C, b * d_state * es},
             {"A", A, d_in * d_state * 4}, {"D", D, d_in * 4}, {"dt_bias", dt_bias, d_in * 4},
             {"conv_weight", conv_weight, d_in * d_conv * 4},
             {"conv_bias", conv_bias, d_in * 4}}))
      return s;
  }
  ssm::StepParams p{ssm_state, x, dt, A, B, C, D, z, dt_bias, y, b, d_in, dt_softplus,
                    conv_state, conv_weight, conv_bias, (int)d_conv};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == SSM_BF16) return dispatch_step_n<__nv_bfloat16, true>(p, d_state, st, what);
  return dispatch_step_n<float, true>(p, d_state, st, what);
}

ssm_status ss2d_cross_scan(const void *u, void *xs, int64_t b, int64_t H, int64_t W,
                           int64_t d_in, ssm_dtype dtype, ssm_stream_t stream) {
  return ss2d_cross_scan_ex(u, xs, b, H, W, d_in, SSM_SS2D_CROSS, dtype, stream);
}

ssm_status ss2d_cross_scan_ex(const void *u, void *xs, int64_t b, int64_t H, int64_t W,
                              int64_t d_in, ssm_ss2d_order order, ssm_dtype dtype,
                              ssm_stream_t stream) {
  g_last_error.clear();
  int64_t L, n;
  if (b < 0 || H < 0 || W < 0 || d_in < 0 || !mul_ok(H, W, &L) || !mul_ok(b, 4 * L, &n) ||
      !mul_ok(n, d_in, &n))
    return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_scan: bad sizes");
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_cross_scan: unknown dtype %d", (int)dtype);
  if (order != SSM_SS2D_CROSS && order != SSM_SS2D_SNAKE)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_cross_scan: unknown scan order %d", (int)order);
  if (n == 0) return ok();
  if (!u || !xs) return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_scan: NULL pointer");
  if (!aligned(u, esize(dtype)) || !aligned(xs, esize(dtype)))
    return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_scan: misaligned pointer");
  if (ssm_status s = check_disjoint("ss2d_cross_scan", {{"xs", xs, n * (int64_t)esize(dtype)}},
                                    {{"u", u, n / 4 * (int64_t)esize(dtype)}}))
    return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto run = [&](auto tag, auto ord) {
    using T = decltype(tag);
    constexpr int O = decltype(ord)::value;
    ssm::cross_scan_kernel<T, O><<<grid_for(n), 256, 0, st>>>(
        static_cast<const T *>(u), static_cast<T *>(xs), b, H, W, d_in);
  };
  using Cross = std::integral_constant<int, ssm::kOrderCross>;
  using Snake = std::integral_constant<int, ssm::kOrderSnake>;
  if (dtype == SSM_BF16)
    order == SSM_SS2D_SNAKE ? run(__nv_bfloat16(), Snake()) : run(__nv_bfloat16(), Cross());
  else
    order == SSM_SS2D_SNAKE ? run(float(), Snake()) : run(float(), Cross());
  return check_launch("ss2d_cross_scan");
}

ssm_status ss2d_cross_merge(const void *ys, void *y, int64_t b, int64_t H, int64_t W,
                            int64_t d_in, ssm_dtype dtype, ssm_stream_t stream) {
  return ss2d_cross_merge_ex(ys, y, b, H, W, d_in, SSM_SS2D_CROSS, dtype, stream);
}

ssm_status ss2d_cross_merge_ex(const void *ys, void *y, int64_t b, int64_t H, int64_t W,
                               int64_t d_in, ssm_ss2d_order order, ssm_dtype dtype,
                               ssm_stream_t stream) {
  g_last_error.clear();
  int64_t L, n;
  if (b < 0 || H < 0 || W < 0 || d_in < 0 || !mul_ok(H, W, &L) || !mul_ok(b, 4 * L, &n) ||
      !mul_ok(n, d_in, &n))
    return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_merge: bad sizes");
  if (dtype != SSM_F32 && dtype != SSM_BF16)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_cross_merge: unknown dtype %d", (int)dtype);
  if (order != SSM_SS2D_CROSS && order != SSM_SS2D_SNAKE)
    return fail(SSM_ERR_UNSUPPORTED, "ss2d_cross_merge: unknown scan order %d", (int)order);
  if (n == 0) return ok();
  if (!ys || !y) return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_merge: NULL pointer");
  if (!aligned(ys, esize(dtype)) || !aligned(y, esize(dtype)))
    return fail(SSM_ERR_INVALID_ARG, "ss2d_cross_merge: misaligned pointer");
  if (ssm_status s = check_disjoint("ss2d_cross_merge", {{"y", y, n / 4 * (int64_t)esize(dtype)}},
                                    {{"ys", ys, n * (int64_t)esize(dtype)}}))
    return s;
  const int64_t m = b * L * d_in;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto run = [&](auto tag, auto ord) {
    using T = decltype(tag);
    constexpr int O = decltype(ord)::value;
    ssm::cross_merge_kernel<T, O><<<grid_for(m), 256, 0, st>>>(
        static_cast<const T *>(ys), static_cast<T *>(y), b, H, W, d_in);
  };
  using Cross = std::integral_constant<int, ssm::kOrderCross>;
  using Snake = std::integral_constant<int, ssm::kOrderSnake>;
  if (dtype == SSM_BF16)
    order == SSM_SS2D_SNAKE ? run(__nv_bfloat16(), Snake()) : run(__nv_bfloat16(), Cross());
  else
    order == SSM_SS2D_SNAKE ? run(float(), Snake()) : run(float(), Cross());
  return check_launch("ss2d_cross_merge");
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc SS2D
// Scratch of ss2d_scan_fwd_noalloc: the fp32 per-pixel accumulator of the
// large-image SS2D path, in a file-scope device array instead of caller
// memory.  Every GPU that loads this library holds it (16 MiB) until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) float g_ss2d_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress (that device current) and cached per device.
// While `st` is not being captured the lookup is made on every call (cheap
// next to the launch; a device reset, which reloads the module, cannot leave
// a stale address behind); while it is, no lookup is made and the cached
// address is used.
ssm_status noalloc_scratch(cudaStream_t st, float **out) {
  static std::mutex mu;
  static float *ptr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64)
    return fail(SSM_ERR_CUDA, "ss2d_scan_fwd_noalloc: cudaGetDevice failed");
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess)
    return fail(SSM_ERR_CUDA, "ss2d_scan_fwd_noalloc: cudaStreamIsCapturing: %s",
                cudaGetErrorString(e));
  std::lock_guard<std::mutex> lock(mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void *addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_ss2d_noalloc_scratch);
    if (e != cudaSuccess || !addr)
      return fail(SSM_ERR_CUDA, "ss2d_scan_fwd_noalloc: cudaGetSymbolAddress: %s",
                  cudaGetErrorString(e));
    ptr[dev] = static_cast<float *>(addr);
  } else if (!ptr[dev]) {
    return fail(SSM_ERR_CUDA,
                "ss2d_scan_fwd_noalloc: no device address cached for this device while "
                "the stream is being captured");
  }
  *out = ptr[dev];
  return ok();
}

}  // namespace

extern "C" {

ssm_status ss2d_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                                 const void *B, const void *C, const float *D,
                                 const float *dt_bias, int delta_softplus, void *y, int64_t b,
                                 int64_t H, int64_t W, int64_t d_in, int64_t d_state,
                                 ssm_dtype dtype, ssm_stream_t stream) {
  g_last_error.clear();
  const size_t need = ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, d_state);
  if (need == (size_t)-1)
    return fail(SSM_ERR_INVALID_ARG, "ss2d_scan_fwd_noalloc: invalid or overflowing sizes");
  if (need > kNoAllocScratchBytes)
    return fail(SSM_ERR_WORKSPACE,
                "ss2d_scan_fwd_noalloc: needs %zu bytes of scratch, the static array holds %zu "
                "(b * H * W * d_in * 4 must not exceed it); use ss2d_scan_fwd with a workspace",
                need, kNoAllocScratchBytes);
  float *scratch = nullptr;
  if (need > 0) {
    if (ssm_status s = noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch)) return s;
  }
  // The accumulator needs no clearing: the first direction stores every
  // pixel before the others add to it.
  return ss2d_scan_fwd(u, delta, A, B, C, D, dt_bias, delta_softplus, y, b, H, W, d_in, d_state,
                       dtype, scratch, need, stream);
}

ssm_status ssm_check_device_errors(ssm_stream_t stream) {
  g_last_error.clear();
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(SSM_ERR_CUDA, "ssm_check_device_errors: %s", cudaGetErrorString(e));
#ifdef SSM_DEBUG_BOUNDS
  unsigned int w = 0;
  e = cudaMemcpyFromSymbol(&w, g_ssm_bounds_word, sizeof w);
  if (e != cudaSuccess)
    return fail(SSM_ERR_CUDA, "ssm_check_device_errors: %s", cudaGetErrorString(e));
  if (w) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_ssm_bounds_word, &zero, sizeof zero);
    if (e != cudaSuccess)
      return fail(SSM_ERR_CUDA, "ssm_check_device_errors: %s", cudaGetErrorString(e));
    return fail(SSM_ERR_DEVICE_BOUNDS,
                "a kernel computed an index outside its buffer (kinds 0x%08x: 1 activations, "
                "2 B / C, 4 parameters, 8 states, 16 chunk states / block maps, 32 workspace, "
                "0x80000000 self-test); the access was skipped",
                w);
  }
#endif
  return ok();
}

int ssm_debug_bounds_enabled(void) {
#ifdef SSM_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"

#ifdef SSM_DEBUG_BOUNDS
namespace {
// One check whose index is one past its one-element range: recorded and
// skipped in the debug-bounds build (nothing is read or written).
__global__ void bounds_self_test_kernel(float *never_written) {
  if (ssm::in_bounds(1, 1, ssm::kBndSelfTest)) never_written[0] = 0.0f;
}
}  // namespace
#endif

extern "C" {

ssm_status ssm_debug_bounds_self_test(ssm_stream_t stream) {
  g_last_error.clear();
#ifdef SSM_DEBUG_BOUNDS
  bounds_self_test_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(nullptr);
  return check_launch("ssm_debug_bounds_self_test");
#else
  (void)stream;
  return fail(SSM_ERR_UNSUPPORTED, "ssm_debug_bounds_self_test: not a debug-bounds build");
#endif
}

}  // extern "C"
