/*
 * ssmscan.h -- C ABI of the B200 (sm_100a) selective-scan library
 * (libssmscan.so).
 *
 * Operations (each defined by the passage cited beside it):
 *   ssm_scan_fwd      Mamba's selective scan:
 *                     "PyTorch新手也能懂：手把手拆解Mamba-minimal中的selective_scan实现"
 *                     §2 (signature selective_scan(u, delta, A, B, C, D) and the
 *                     shape table), §3 (deltaA = exp(delta A) by ZOH, deltaB_u =
 *                     delta B u by Euler), §4 (sequential loop: update the state,
 *                     then y = C.state), §5 (y + u D); plus the gate y * silu(z)
 *                     and delta = softplus(dt + dt_bias) of "代码连连看——mamba"
 *                     (Mamba.step()).
 *   ss2d_scan_fwd     VMamba's SS2D: CrossScan into four scan orders, a
 *                     selective scan per order, CrossMerge back ("关于代码SS2D中
 *                     的d_state设置", VMamba issue 206: the scan orders only
 *                     arrange the sequence; d_state = 1 for throughput).
 *   ssm_state_update  one decode step of Mamba.step() ("代码连连看——mamba",
 *                     the SSM step: softplus(dt + bias), dA = exp(dt A),
 *                     dB = dt B, state = state dA + x dB (in place),
 *                     y = state.C + D x, y * act(z)).
 *   ssm_scan_bwd      the gradients of ssm_scan_fwd by the reverse-time
 *                     adjoint of its recurrence (same passages);
 *                     ssm_scan_fwd_save / ssm_scan_bwd_saved split it as a
 *                     training step does (the forward keeps chunk states;
 *                     ssm_scan_fwd_save_ex and ssm_scan_bwd_saved_ex add
 *                     scratch for few channels).
 *   ssm_conv_state_update  the same step with the depthwise causal-conv1d
 *                     step of Mamba.step() in front of it (roll conv_state
 *                     left, append x, sum conv_state * weight + bias, SiLU).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" point to device memory of the current CUDA
 *     device, row-major and contiguous in the layout given.  The caller owns
 *     every buffer; the library never allocates or frees memory.
 *   - Every call enqueues its kernels on `stream` (NULL = the legacy default
 *     stream) and returns without synchronising.  Argument errors are
 *     reported synchronously, before anything is enqueued; launch errors are
 *     reported by the call that launched.  A fault while a kernel runs is a
 *     CUDA error of the stream, reported by the next call that synchronises
 *     it (ssm_check_device_errors() does).
 *   - Calls allocate nothing and never synchronise.  Those that take their
 *     scratch from the caller can be captured in a CUDA graph; make the
 *     first call of each kind and d_state outside any capture (it sets the
 *     kernel's shared-memory attribute once per device).
 *   - A non-OK status leaves a message in ssm_last_error() (per thread).
 *   - Outputs must not alias inputs unless stated.
 *   - dtype: SSM_F32 or SSM_BF16 applies to every activation-sized tensor of
 *     the call (u, delta, z, B, C, y / x, dt); A, D, dt_bias and every
 *     recurrent state are always fp32, and so are the backward's sums over
 *     channels or batch (dA, dB, dC, dD, ddt_bias, dh0).  Arithmetic is fp32
 *     throughout; each output is rounded once to its type.
 *   - d_state (N) must be one of 1, 2, 4, 8, 16, 32, 64; other values return
 *     SSM_ERR_UNSUPPORTED.  Any b, L, d_in >= 0 is accepted; b, L or d_in of
 *     0 is a valid empty problem.  Sizes whose element counts overflow int64
 *     return SSM_ERR_INVALID_ARG.
 */
#ifndef SSMSCAN_H
#define SSMSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA header. */
typedef struct CUstream_st *ssm_stream_t;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1,    /* NULL required pointer, negative size, misaligned pointer, overflow */
    SSM_ERR_UNSUPPORTED = 2,    /* valid but not compiled: d_state not in {1,2,4,...,64}, unknown dtype */
    SSM_ERR_WORKSPACE = 3,      /* workspace smaller than ssm_scan_fwd_workspace_bytes() */
    SSM_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed (message has the CUDA error) */
    SSM_ERR_DEVICE_TIMEOUT = 5, /* reserved for a kernel's bounded wait running out; no kernel of
                                   this build waits on another thread block or device, so no call
                                   returns it */
    SSM_ERR_DEVICE_BOUNDS = 6   /* debug-bounds build only: a kernel computed a global index outside
                                   its buffer and skipped that access (ssm_check_device_errors) */
} ssm_status;

typedef enum {
    SSM_F32 = 0,
    SSM_BF16 = 1
} ssm_dtype;

/* SS2D scan orders (see ss2d_scan_fwd_ex). */
typedef enum {
    SSM_SS2D_CROSS = 0,  /* row-major, column-major and both reversed (VMamba CrossScan) */
    SSM_SS2D_SNAKE = 1   /* as CROSS with odd rows / odd columns walked backwards */
} ssm_ss2d_order;

/*
 * Bytes of device workspace ssm_scan_fwd needs for this problem.  It is 0
 * unless the problem has too few (batch, channel) pairs to fill the device,
 * i.e. b * ceil(d_in / 32) CTAs fewer than half the SMs (d_state 8, 16 or 32,
 * d_in a multiple of 8, L long enough to cut).  Such a scan is split along L
 * into blocks scanned in parallel: every block's map h -> P h + Q is stored
 * in the workspace, a carry pass turns the maps into each block's start
 * state, and a replay writes y.  The workspace then holds two fp32 arrays
 * (b, nblk, d_in, d_state): the block decays P (which the carry pass
 * overwrites with the state each next block starts from), then the block
 * states Q; nblk depends on the device's SM count, so query it on the device
 * that runs the scan.  ssm_scan_fwd_save_ex takes the same workspace (there
 * it is optional).  Returns (size_t)-1 for invalid sizes.
 */
size_t ssm_scan_fwd_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state);

/*
 * Selective scan forward.  For every batch i, channel d and state n, with the
 * state h starting at h0[i,d,n] (or 0) and for t = 0 .. L-1:
 *     delta = delta_softplus ? softplus(dt + dt_bias[d]) : dt + dt_bias[d]
 *             (dt = delta[i,t,d]; softplus(x) = x for x > 20)
 *     h[n]  = exp(delta * A[d,n]) * h[n] + delta * B[i,t,n] * u[i,t,d]
 *     y     = sum_n C[i,t,n] * h[n] + D[d] * u[i,t,d]
 *     y[i,t,d] = z ? y * silu(z[i,t,d]) : y
 * and h_last[i,d,n] = h[n] after the last step.
 *
 *   u, delta, z   device, (b, L, d_in), dtype; z nullable (no gate)
 *   A             device fp32 (d_in, d_state); A = -exp(A_log) as the caller forms it
 *   B, C          device, (b, L, d_state), dtype; shared by all channels
 *   D, dt_bias    device fp32 (d_in), nullable (0 when NULL)
 *   h0            device fp32 (b, d_in, d_state), nullable (zero start)
 *   h_last        device fp32 (b, d_in, d_state), nullable; may equal h0
 *   y             device, (b, L, d_in), dtype; must not alias an input
 *   workspace     device, >= ssm_scan_fwd_workspace_bytes(...) bytes, 16-byte
 *                 aligned, not overlapping any other argument; may be NULL when
 *                 that is 0.  Scratch: its contents on entry are not read and
 *                 on return are unspecified.  Too small (or NULL when needed):
 *                 SSM_ERR_WORKSPACE and nothing is launched.
 */
ssm_status ssm_scan_fwd(const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *D,
                        const void *z, const float *dt_bias, int delta_softplus,
                        const float *h0, float *h_last, void *y,
                        int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                        ssm_dtype dtype, void *workspace, size_t workspace_bytes,
                        ssm_stream_t stream);

/*
 * ssm_scan_fwd that also saves the state at the start of every 16-step
 * chunk (h before step 16 c, c = 0 .. ceil(L / 16) - 1) into chunk_states:
 * device fp32 (b, ceil(L / 16), d_in, d_state), chunk_states_bytes >=
 * ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state), 16-byte aligned, not
 * aliasing another argument.  This is the backward's workspace layout: a
 * following ssm_scan_bwd_saved with the same inputs starts from these
 * states instead of walking the sequence forwards again (the saved chunk
 * states the backward of a training step keeps from its forward).  Every
 * other argument as for ssm_scan_fwd.  It runs in one pass (no workspace).
 */
ssm_status ssm_scan_fwd_save(const void *u, const void *delta, const float *A,
                             const void *B, const void *C, const float *D,
                             const void *z, const float *dt_bias, int delta_softplus,
                             const float *h0, float *h_last, void *y,
                             float *chunk_states, size_t chunk_states_bytes,
                             int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                             ssm_dtype dtype, ssm_stream_t stream);

/*
 * ssm_scan_fwd_save with a workspace for the split scan (few channels):
 * given ssm_scan_fwd_workspace_bytes(...) bytes or more (when that is not
 * 0), 16-byte aligned, the sequence is cut into blocks as in ssm_scan_fwd
 * (summary, carry and scan passes; the scan pass writes y, h_last and the
 * chunk states); with less, or NULL, it is ssm_scan_fwd_save.  The two
 * agree within rounding (the block start states are composed maps).
 *
 *   workspace     device, nullable; contents on entry are ignored.  Must be
 *                 4-byte aligned and share no byte with any argument.
 */
ssm_status ssm_scan_fwd_save_ex(const void *u, const void *delta, const float *A,
                                const void *B, const void *C, const float *D,
                                const void *z, const float *dt_bias, int delta_softplus,
                                const float *h0, float *h_last, void *y,
                                float *chunk_states, size_t chunk_states_bytes,
                                int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                                ssm_dtype dtype, void *workspace, size_t workspace_bytes,
                                ssm_stream_t stream);

/*
 * Workspace of ssm_scan_bwd: the state at the start of every 16-step chunk
 * of the sequence, fp32: b * ceil(L / 16) * d_in * d_state * 4 bytes.
 * Returns (size_t)-1 for invalid sizes.
 */
size_t ssm_scan_bwd_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state);

/*
 * Workspace with which ssm_scan_bwd takes its fastest path: for d_state 8,
 * 16 or 32 when b * ceil(d_in / channels per CTA) backward blocks would leave
 * more than half of the SMs idle, the chunk states followed by the split
 * backward's block buffers (the forward split's block decays and states, the
 * adjoint's block maps); otherwise ssm_scan_bwd_workspace_bytes.  With that
 * much (16-byte aligned), when d_in times the element size is a multiple of
 * 16 bytes and u, delta, B are 16-byte aligned (the forward kernel's
 * staging), ssm_scan_bwd cuts the sequence into blocks: the
 * chunk-start states from the forward's split scan, each block's adjoint map
 * composed from dh_last by the carry scan, every block's backward at once.
 * Otherwise it runs unsplit; the gradients agree within rounding (sums are
 * taken in a different order).  ssm_scan_bwd_saved runs unsplit;
 * ssm_scan_bwd_saved_ex splits from the saved states.
 */
size_t ssm_scan_bwd_fast_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state);

/*
 * Selective scan backward: the gradients of
 *     loss = sum dout[i,t,d] out[i,t,d] + sum dh_last[i,d,n] h_last[i,d,n]
 * for the forward of ssm_scan_fwd with the same inputs, by the chain rule
 * through its recurrence ("手把手拆解Mamba-minimal中的selective_scan实现"
 * §3-§5 and the gate of "代码连连看——mamba", Mamba.step()), walked backwards
 * in time.  With delta_t = softplus(dt_t + dt_bias), a_t = exp(delta_t A),
 * g_t = dout_t silu(z_t), lam = d loss / d h_t:
 *     lam += g_t C_t;  dC_t += g_t h_t;  dD += g_t u_t
 *     ddelta_t = softplus'(dt_t + dt_bias) sum_n lam (A a_t h_{t-1} + B_t u_t)
 *     dA += lam delta_t a_t h_{t-1};  dB_t += lam delta_t u_t
 *     du_t = g_t D + delta_t sum_n lam B_t;  lam *= a_t
 *     dz_t = dout_t (C_t.h_t + D u_t) silu'(z_t);  dh0 = lam after step 0
 * softplus' is the logistic sigmoid, and 1 above the threshold 20.
 * The forward states are recomputed from h0 inside the call (nothing from
 * ssm_scan_fwd is kept).
 *
 *   inputs        exactly those of ssm_scan_fwd (u, delta, A, B, C, D, z,
 *                 dt_bias, delta_softplus, h0), plus
 *   dout          device, (b, L, d_in), dtype: gradient of the output y
 *   dh_last       device fp32 (b, d_in, d_state), nullable (zero)
 *   du, ddelta    device, (b, L, d_in), dtype (ddelta is the gradient of
 *                 the raw delta input, before bias and softplus)
 *   dz            device, (b, L, d_in), dtype, nullable; written only when
 *                 z is given
 *   dA            device fp32 (d_in, d_state), required (summed over b, L)
 *   dB, dC        device fp32 (b, L, d_state) (summed over d_in)
 *   dD, ddt_bias  device fp32 (d_in), nullable (summed over b, L); dD is
 *                 the gradient at the given D (0 when D is NULL)
 *   dh0           device fp32 (b, d_in, d_state), nullable
 *   workspace     device, >= ssm_scan_bwd_workspace_bytes(...) bytes;
 *                 contents on entry are ignored
 * Every output is overwritten (the summed ones are zeroed on the stream
 * first); outputs must not alias inputs or each other.  b <= 65535.
 * Arithmetic is fp32; the sums over channels and batch are taken with fp32
 * atomics, so their rounding order varies from run to run.
 */
ssm_status ssm_scan_bwd(const void *u, const void *delta, const float *A,
                        const void *B, const void *C, const float *D,
                        const void *z, const float *dt_bias, int delta_softplus,
                        const float *h0, const void *dout, const float *dh_last,
                        void *du, void *ddelta, float *dA, float *dB, float *dC,
                        float *dD, void *dz, float *ddt_bias, float *dh0,
                        int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                        ssm_dtype dtype, void *workspace, size_t workspace_bytes,
                        ssm_stream_t stream);

/*
 * ssm_scan_bwd from the chunk-start states ssm_scan_fwd_save wrote for the
 * same inputs (chunk_states, read only; h0 is not needed, it is chunk 0's
 * state).  Same outputs and rules as ssm_scan_bwd.
 */
ssm_status ssm_scan_bwd_saved(const void *u, const void *delta, const float *A,
                              const void *B, const void *C, const float *D,
                              const void *z, const float *dt_bias, int delta_softplus,
                              const void *dout, const float *dh_last,
                              void *du, void *ddelta, float *dA, float *dB, float *dC,
                              float *dD, void *dz, float *ddt_bias, float *dh0,
                              int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                              ssm_dtype dtype, const float *chunk_states,
                              size_t chunk_states_bytes, ssm_stream_t stream);

/*
 * ssm_scan_bwd_saved with a workspace for the split backward (few channels):
 * given ssm_scan_bwd_saved_workspace_bytes(...) bytes or more (when that is
 * not 0), 16-byte aligned, the chunks are cut into blocks as in
 * ssm_scan_bwd, from the saved states (no states pass); with less, or NULL,
 * it is ssm_scan_bwd_saved.  The two agree within rounding.
 *
 *   workspace     device, nullable; contents on entry are ignored.  Must be
 *                 4-byte aligned and share no byte with any argument.
 * Other arguments, layouts and errors as ssm_scan_bwd_saved.
 */
ssm_status ssm_scan_bwd_saved_ex(const void *u, const void *delta, const float *A,
                                 const void *B, const void *C, const float *D,
                                 const void *z, const float *dt_bias, int delta_softplus,
                                 const void *dout, const float *dh_last,
                                 void *du, void *ddelta, float *dA, float *dB, float *dC,
                                 float *dD, void *dz, float *ddt_bias, float *dh0,
                                 int64_t b, int64_t L, int64_t d_in, int64_t d_state,
                                 ssm_dtype dtype, const float *chunk_states,
                                 size_t chunk_states_bytes, void *workspace,
                                 size_t workspace_bytes, ssm_stream_t stream);

/*
 * Workspace of ssm_scan_bwd_saved_ex's split: the adjoint's block maps,
 * 2 * b * blocks * d_in * d_state fp32, when the split applies (d_state 8,
 * 16, 32 and too few channels to fill the GPU); 0 otherwise.  (size_t)-1 for
 * invalid sizes.
 */
size_t ssm_scan_bwd_saved_workspace_bytes(int64_t b, int64_t L, int64_t d_in, int64_t d_state);

/*
 * SS2D forward on an H x W grid (pixels row-major, p = h W + w, L = H W).
 * Direction k visits pixel p_k(l) at step l: k = 0 row-major (p = l),
 * k = 1 column-major (l = w H + h), k = 2 the reverse of k = 0, k = 3 the
 * reverse of k = 1.  Each direction runs the selective scan above on
 * u[i, p_k(l), :] with its own delta/B/C (given in its scan order) and the
 * rows k*d_in .. k*d_in + d_in - 1 of A, D, dt_bias, with no gate and a zero
 * start; the output is y[i,p,d] = sum_k y_k at pixel p (fp32 sum, one
 * rounding).  The four orders are index arithmetic: no permuted copy of u is
 * stored, and per-direction outputs only by the direction split (below), in
 * the workspace.
 *
 *   u, y          device, (b, H W, d_in), dtype
 *   delta         device, (b, 4, H W, d_in), dtype
 *   A             device fp32 (4 d_in, d_state)
 *   B, C          device, (b, 4, H W, d_state), dtype
 *   D, dt_bias    device fp32 (4 d_in), nullable
 *   workspace     device, >= ss2d_scan_fwd_workspace_bytes(...) bytes; may be
 *                 NULL when that is 0.  Contents on entry are ignored.  With
 *                 ss2d_scan_fwd_fast_workspace_bytes(...) bytes or more the
 *                 call may take the direction split (below); with less it
 *                 runs the single-kernel path.  Same results either way.
 * Images whose accumulator would live in the workspace, and batches too
 * small to fill the GPU (b * ceil(d_in / 8) tiles at most half the SMs),
 * take the direction split when the workspace allows: one CTA per
 * (tile, direction), each storing its
 * direction's fp32 outputs in the workspace, then a second kernel that sums
 * them k0 + k1 + k2 + k3 and rounds once -- the single kernel's arithmetic in
 * its order, so the results are bit-identical.
 * d_state must be 1 (the SS2D setting of VMamba), H * W below 2^22 pixels,
 * H * W * d_in below 2^31 and b at most 65535; other values return
 * SSM_ERR_UNSUPPORTED.
 */
ssm_status ss2d_scan_fwd(const void *u, const void *delta, const float *A,
                         const void *B, const void *C, const float *D,
                         const float *dt_bias, int delta_softplus, void *y,
                         int64_t b, int64_t H, int64_t W, int64_t d_in,
                         int64_t d_state, ssm_dtype dtype, void *workspace,
                         size_t workspace_bytes, ssm_stream_t stream);

/*
 * ss2d_scan_fwd with a choice of scan order ("关于代码SS2D中的d_state设置",
 * VMamba issue 206, mentions a snake scan and snake merge besides
 * CrossScan).  SSM_SS2D_CROSS is ss2d_scan_fwd.  SSM_SS2D_SNAKE keeps the
 * four directions but walks them boustrophedon: direction 0 visits row h
 * left to right when h is even and right to left when h is odd; direction 1
 * visits column w top to bottom when w is even and bottom to top when w is
 * odd; directions 2 and 3 are the reverses of 0 and 1.  delta / B / C are
 * given in the chosen order's step order; everything else is as in
 * ss2d_scan_fwd.  An unknown order returns SSM_ERR_UNSUPPORTED.
 */
ssm_status ss2d_scan_fwd_ex(const void *u, const void *delta, const float *A,
                            const void *B, const void *C, const float *D,
                            const float *dt_bias, int delta_softplus, void *y,
                            int64_t b, int64_t H, int64_t W, int64_t d_in,
                            int64_t d_state, ssm_ss2d_order order, ssm_dtype dtype,
                            void *workspace, size_t workspace_bytes,
                            ssm_stream_t stream);

/*
 * Bytes of device workspace ss2d_scan_fwd needs (0 for d_state = 1 when
 * the fp32 accumulator of one (batch, 8-channel) tile, 32 * H * W' bytes with
 * W' = W rounded up to odd, fits in shared memory, i.e. H * W' <= 6272).
 * Larger images keep that accumulator in the workspace: b * H * W * d_in
 * fp32.  Returns (size_t)-1 for invalid sizes.
 */
size_t ss2d_scan_fwd_workspace_bytes(int64_t b, int64_t H, int64_t W, int64_t d_in,
                                     int64_t d_state);

/*
 * Bytes of device workspace with which ss2d_scan_fwd takes its fastest path
 * for this problem: 4 * b * H * W * d_in fp32 (the direction split's four
 * slices) when the direction split applies (large images, small batches),
 * else the same value as ss2d_scan_fwd_workspace_bytes.  Never less than
 * that minimum; (size_t)-1 for invalid sizes.
 */
size_t ss2d_scan_fwd_fast_workspace_bytes(int64_t b, int64_t H, int64_t W, int64_t d_in,
                                          int64_t d_state);

/*
 * ss2d_scan_fwd without a workspace, for callers that cannot allocate device
 * memory: code running inside a host framework that owns every device buffer
 * and hands out none for scratch, and real-time loops that must not call
 * cudaMalloc (it can synchronise the device and can fail on a fragmented
 * heap in the middle of a run).  The pages have no counterpart; this is a
 * packaging variant of ss2d_scan_fwd with the same arguments, layouts and
 * results, minus workspace / workspace_bytes.
 *
 * Large images keep their fp32 per-pixel accumulator in a 16 MiB array that
 * the library reserves statically on every GPU that loads it, held until
 * the process exits.  Limit: b * H * W * d_in * 4 bytes (the value
 * ss2d_scan_fwd_workspace_bytes returns) must not exceed 16 MiB, else
 * SSM_ERR_WORKSPACE; images whose accumulator fits in shared memory need
 * none of it.  The array's device address is looked up with
 * cudaGetSymbolAddress (the device current) and cached per device; a lookup
 * made after a device reset replaces the cached address.  All calls
 * on a device share the one array, which keeps the last call's contents
 * (nothing needs clearing: every call overwrites the part it reads); calls
 * whose kernels overlap on the GPU race on it.
 */
ssm_status ss2d_scan_fwd_noalloc(const void *u, const void *delta, const float *A,
                                 const void *B, const void *C, const float *D,
                                 const float *dt_bias, int delta_softplus, void *y,
                                 int64_t b, int64_t H, int64_t W, int64_t d_in,
                                 int64_t d_state, ssm_dtype dtype, ssm_stream_t stream);

/*
 * One-token state update (decode), in place on ssm_state:
 *     delta = dt_softplus ? softplus(dt[i,d] + dt_bias[d]) : dt[i,d] + dt_bias[d]
 *     s[i,d,n] = s[i,d,n] * exp(delta * A[d,n]) + x[i,d] * delta * B[i,n]
 *     y[i,d]   = (sum_n s[i,d,n] * C[i,n] + D[d] * x[i,d]) * (z ? silu(z[i,d]) : 1)
 *
 *   ssm_state     device fp32 (b, d_in, d_state), read and written in place
 *   x, dt, z      device, (b, d_in), dtype; z nullable
 *   A             device fp32 (d_in, d_state)
 *   B, C          device, (b, d_state), dtype
 *   D, dt_bias    device fp32 (d_in), nullable
 *   y             device, (b, d_in), dtype; must not alias an input
 */
ssm_status ssm_state_update(float *ssm_state, const void *x, const void *dt,
                            const float *A, const void *B, const void *C,
                            const float *D, const void *z, const float *dt_bias,
                            int dt_softplus, void *y, int64_t b, int64_t d_in,
                            int64_t d_state, ssm_dtype dtype, ssm_stream_t stream);

/*
 * One-token decode step with the depthwise causal conv1d of Mamba.step()
 * ("代码连连看——mamba", the conv step: the window is rolled one place left,
 * x goes into its last slot, x_conv = sum_j window[j] * weight[d, j] + bias,
 * then SiLU) fused in front of the state update above:
 *     w'[i,d,j] = w[i,d,j+1] (j < d_conv-1),  w'[i,d,d_conv-1] = x[i,d]
 *     xc[i,d]   = silu(sum_j w'[i,d,j] * conv_weight[d,j] + conv_bias[d])
 *     then ssm_state_update with x replaced by xc (D multiplies xc too).
 * xc stays in fp32 between the two steps (it is not rounded to dtype).
 *
 *   conv_state    device, (b, d_in, d_conv), dtype, read and written in place
 *                 (the new window w'); must not alias another argument
 *   conv_weight   device fp32 (d_in, d_conv): the depthwise kernel, tap j
 *                 multiplying the j-th oldest entry of the window
 *   conv_bias     device fp32 (d_in), nullable
 *   d_conv        1 .. 8, else SSM_ERR_UNSUPPORTED
 *   x             device, (b, d_in), dtype: the raw (pre-conv) input
 *   every other argument as for ssm_state_update
 */
ssm_status ssm_conv_state_update(void *conv_state, const float *conv_weight,
                                 const float *conv_bias, int64_t d_conv,
                                 float *ssm_state, const void *x, const void *dt,
                                 const float *A, const void *B, const void *C,
                                 const float *D, const void *z, const float *dt_bias,
                                 int dt_softplus, void *y, int64_t b, int64_t d_in,
                                 int64_t d_state, ssm_dtype dtype, ssm_stream_t stream);

/*
 * CrossScan as a stored permutation, for checking the index arithmetic of
 * ss2d_scan_fwd bit-exactly: xs[i,k,l,d] = u[i, p_k(l), d].
 *   u   device (b, H W, d_in), dtype;   xs  device (b, 4, H W, d_in), dtype
 */
ssm_status ss2d_cross_scan(const void *u, void *xs, int64_t b, int64_t H,
                           int64_t W, int64_t d_in, ssm_dtype dtype,
                           ssm_stream_t stream);

/* ss2d_cross_scan / ss2d_cross_merge in the given scan order. */
ssm_status ss2d_cross_scan_ex(const void *u, void *xs, int64_t b, int64_t H,
                              int64_t W, int64_t d_in, ssm_ss2d_order order,
                              ssm_dtype dtype, ssm_stream_t stream);
ssm_status ss2d_cross_merge_ex(const void *ys, void *y, int64_t b, int64_t H,
                               int64_t W, int64_t d_in, ssm_ss2d_order order,
                               ssm_dtype dtype, ssm_stream_t stream);

/*
 * CrossMerge: y[i,p,d] = sum_k ys[i, k, l_k(p), d] with l_k the inverse of
 * p_k, summed in fp32 in the order k = 0, 1, 2, 3 and rounded once.
 *   ys  device (b, 4, H W, d_in), dtype;  y  device (b, H W, d_in), dtype
 */
ssm_status ss2d_cross_merge(const void *ys, void *y, int64_t b, int64_t H,
                            int64_t W, int64_t d_in, ssm_dtype dtype,
                            ssm_stream_t stream);

/*
 * Synchronises `stream` and returns SSM_OK, or SSM_ERR_CUDA with the CUDA
 * error of the stream (a kernel fault) in ssm_last_error().  In the
 * debug-bounds build (libssmscan_debug.so, compiled with SSM_DEBUG_BOUNDS)
 * it then reads and clears the device's bounds word: SSM_ERR_DEVICE_BOUNDS
 * when a kernel computed a global index outside its buffer since the last
 * check (the access was skipped; the message names the buffer kinds).
 */
ssm_status ssm_check_device_errors(ssm_stream_t stream);

/*
 * Debug-bounds build: every kernel checks the global index of each load,
 * store and atomic against the size of its buffer, records a miss in a
 * device word and skips the access (no fault).  ssm_debug_bounds_enabled()
 * returns 1 in libssmscan_debug.so and 0 in libssmscan.so.
 * ssm_debug_bounds_self_test() enqueues one kernel whose single check is
 * given an index one past its one-element range: the check records it and
 * the access is skipped, so the next ssm_check_device_errors() on `stream`
 * returns SSM_ERR_DEVICE_BOUNDS.  It returns SSM_ERR_UNSUPPORTED in the
 * release library.  The pages have no counterpart; this is test
 * infrastructure for the kernels' index arithmetic.
 */
int ssm_debug_bounds_enabled(void);
ssm_status ssm_debug_bounds_self_test(ssm_stream_t stream);

/* Message of the last non-OK status returned on this thread ("" if none). */
const char *ssm_last_error(void);

/* Library version, "major.minor.patch". */
const char *ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSMSCAN_H */
