/*
 * ttt.h -- C ABI of the B200 large-chunk test-time-training (TTT) layer.
 *
 * The layer keeps, per head, SwiGLU fast weights
 *     f_W(x) = W2 (SiLU(W1 x) o (W3 x)),   W1, W3 in R^{m x d},  W2 in R^{d x m}
 * (ZipMap: Linear-Time Stateful 3D Reconstruction via Test-Time Training,
 * key design 1), takes one or more Muon steps of the per-token-weighted
 * dot-product loss
 *     L = sum_i eta_i * ( - f_W(k_i)^T v_i )
 * over every token of a chunk (Scal3R: Scalable Test-Time Training for
 * Large-Scale 3D Reconstruction, scheme 1, eq. (9)), with the gradient
 * orthogonalised by Newton-Schulz and a norm-preserving step
 *     Delta <- NewtonSchulz(g),  W^ <- ||W|| (W - lr Delta) / ||W - lr Delta||
 * (ZipMap key design 3), and then applies o_i = f_W^(q_i) (Scal3R eq. (4)).
 * Options: L2-normalised Q/K and a depthwise ShortConv2D on V (VGG-T3:
 * Offline Feed-Forward 3D Reconstruction at Scale, key designs 1 and 2), two
 * inner steps (VGG-T3 key design 3), causal chunk-to-chunk carry of W (ZipMap
 * key design 4; LoGeR: Long-Context Geometric Reconstruction with Hybrid
 * Memory, method overview).
 *
 * Conventions for every entry point:
 *  - All pointers are DEVICE pointers unless stated otherwise; the caller
 *    owns every buffer, including the workspace, and the library never
 *    allocates device memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream).  Argument, alignment and workspace
 *    errors are detected on the host and returned before anything is queued.
 *    A failed kernel launch returns TTT_ERR_CUDA.  A device-side wait that
 *    exceeds its time limit does not hang: the kernel records
 *    TTT_ERR_TIMEOUT in the workspace status word (read it with
 *    ttt_poll_status) and returns.
 *  - Token matrices Q, K, V, O are row-major [T][ld] with head h in columns
 *    [h*d, (h+1)*d); ld is the row stride in elements (0 means H*d, else
 *    ld >= H*d).  In TTT_BF16 mode they are bfloat16 and must be 16-byte
 *    aligned with ld a multiple of 8; in TTT_FP32 mode they are float.
 *  - eta is float [T][H] (per-token, per-head learning rate), contiguous.
 *  - Fast weights are float: W1, W3 [H][m][d], W2 [H][d][m], contiguous.
 *    In TTT_BF16 mode the GEMMs read a bfloat16 copy of W that the library
 *    writes into the workspace at the start of each call; W itself stays fp32.
 *  - TTT_BF16 mode runs the tensor-core path and needs d in {128, 192} and
 *    m a multiple of 64 (fused kernels), or d and m multiples of 256 (the
 *    wide-head path for heads such as ZipMap's single head of d = 1024,
 *    m = 2048: the same arithmetic as separate 2-SM tensor-core products with
 *    fp16 intermediates in the workspace); TTT_FP32 mode runs fp32 CUDA-core
 *    kernels for any d <= 256 and m a multiple of 32.  Other shapes return
 *    TTT_ERR_UNSUPPORTED.
 *  - Operand range of the TTT_BF16 update (ttt_grad, ttt_grad_prepared,
 *    ttt_update, ttt_update_conv, ttt_chunked, ttt_layer_host).  The gradient
 *    GEMMs run on fp16 operands with fp32
 *    accumulation: k^ (k / ||k|| with qk_l2norm = 1, else k itself),
 *    V' = -s eta v with a power of two s chosen per call so that
 *    s * max|eta| lies in [16, 32) (for ttt_layer_host with chunk = 0: one s
 *    for all T tokens), the fp16 copy of W, and dL/dh, u scaled by s.  So
 *    the scale of eta does not matter; what must hold is that each of these
 *    stays below fp16's 65504: without the key norm every key element |k|;
 *    every |V'_t| = s |eta_t| |v_t| < 32 |v_t| |eta_t| / max|eta| (so
 *    |v| < 2047 always suffices); and u = SiLU(W1 k^) o (W3 k^) and s dL/dh,
 *    which for normalised keys and weights of the initial scale stay far
 *    below it (without the key norm, u grows like |k|^2).  Without the key
 *    norm, key elements below 2^-14 in magnitude lose precision (fp16
 *    subnormals).  Beyond the range the gradient comes out non-finite: the
 *    call still returns TTT_OK (it is asynchronous), ttt_poll_status then
 *    reports TTT_ERR_RANGE, and the Muon step leaves W unchanged (ttt_grad
 *    returns the non-finite G as is).
 *  - No entry point falls back to the CPU.
 */
#ifndef TTT_H
#define TTT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID = -1,      /* bad argument: null pointer, non-positive size, ld < H*d, ... */
  TTT_ERR_UNSUPPORTED = -2,  /* valid but not implemented: shape or dtype outside the table above */
  TTT_ERR_WORKSPACE = -3,    /* workspace missing or smaller than ttt_workspace_bytes() */
  TTT_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed */
  TTT_ERR_TIMEOUT = -5,      /* a device-side wait gave up (reported through ttt_poll_status) */
  TTT_ERR_ALIGN = -6,        /* pointer or row stride violates the 16-byte alignment rule */
  TTT_ERR_SCRATCH = -7,      /* problem too large for the fixed scratch of ttt_apply_noalloc */
  TTT_ERR_RANGE = -8         /* the gradient came out non-finite: an fp16 operand of the tensor-core
                                update was out of range (reported through ttt_poll_status) */
} ttt_status;

typedef enum { TTT_FP32 = 0, TTT_BF16 = 1 } ttt_dtype;

/* Per-head fast-weight dimensions: H heads, head dim d, SwiGLU hidden width m. */
typedef struct { int heads, d, m; } ttt_dims;

/* fp32 device pointers: W1, W3 [H][m][d]; W2 [H][d][m]. */
typedef struct { float *W1, *W3, *W2; } ttt_weights;

/* Muon step (ZipMap key design 3).  For each per-head matrix G (g1, g3, g2):
 *   X = G / (||G||_F + eps), on the wide orientation (rows <= cols);
 *   iters times: A = X X^T, X <- a X + (b A + c A A) X;  Delta = X (original orientation).
 *   iters = 0: Delta = G (plain gradient step).
 *   renorm = 1: W <- ||W||_F (W - lr Delta) / ||W - lr Delta||_F;  renorm = 0: W <- W - lr Delta. */
typedef struct { int iters; float a, b, c, eps, lr; int renorm; } ttt_ns_cfg;

/* Row strides and the Q/K L2-normalisation switch (VGG-T3 key design 1):
 * qk_l2norm = 1 makes update/grad use k^ = k / max(||k||, 1e-12) and apply use
 * q^ likewise, per token and head, without modifying Q or K. */
typedef struct { int qk_l2norm; int64_t ld_q, ld_k, ld_v, ld_o; } ttt_io_cfg;

/* Workspace size in bytes for any call of this library with these dims, with
 * at most T tokens per call (for ttt_chunked: at most `chunk` tokens per chunk).
 * The workspace must be 256-byte aligned.  Returns 0 for invalid dims. */
size_t ttt_workspace_bytes(ttt_dims dims, int64_t T, ttt_dtype dtype);

/* Clear the status word of a workspace (asynchronously on `stream`). */
int ttt_reset_status(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream` and return the workspace status word: TTT_OK or the
 * first device-side error recorded since the last reset (TTT_ERR_TIMEOUT, or
 * TTT_ERR_RANGE for a non-finite gradient).  While an error is recorded, the
 * Muon step of every call on this workspace leaves W unchanged. */
int ttt_poll_status(const void* ws, void* stream);

/* In-place L2 normalisation of X [T][ld]: every (token, head) row of d values
 * becomes x / max(||x||_2, 1e-12) (VGG-T3 key design 1). */
int ttt_l2norm(void* X, int64_t T, ttt_dims dims, int64_t ld, ttt_dtype dtype, void* stream);

/* ShortConv2D (VGG-T3 key design 2): V [N*h*w][ld_v] is viewed as the patch
 * grid (N, h, w, C) with token t = (n*h + y)*w + x; each channel c is
 * cross-correlated with taps[c] (float [C][3][3], device) with zero padding
 * inside each frame, no bias; act = 1 applies SiLU.  Writes Vout [N*h*w][ld_out]
 * (C columns; may not alias V).  C must be a multiple of 8. */
int ttt_shortconv2d(const void* V, int64_t ld_v, void* Vout, int64_t ld_out, const float* taps,
                    int N, int h, int w, int C, int act, ttt_dtype dtype, void* stream);

/* Gradient of L w.r.t. (W1, W3, W2) summed over all T tokens, fp32, written to
 * G = [g1 (H*m*d) | g3 (H*m*d) | g2 (H*d*m)] (same layouts as W).  Uses K and V as
 * given (apply ttt_shortconv2d to V first if wanted); deterministic.
 * This and ttt_step split ttt_update so that a caller can sum G across devices
 * (Scal3R scheme 2, Global Context Synchronization) between the two. */
int ttt_grad(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T,
             ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype, float* G,
             void* ws, size_t ws_bytes, void* stream);

/* ttt_grad without the operand preparation: the workspace must hold what the last
 * ttt_grad (or ttt_grad_prepared) on it prepared, for the same K, V, eta, T and io
 * (bf16 mode: the fp16 K^ and V' and the |eta| maxima; fp32 mode: the per-token key
 * norms), while W may have changed since (e.g. by ttt_step).  This is the second
 * inner step of a multi-device update (ttt_grad, sum of G across devices, ttt_step,
 * then this): it saves the preparation pass, a read of K and V and a write of their
 * fp16 copies.  The fp16 weight copy is refreshed from W as in ttt_grad. */
int ttt_grad_prepared(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T,
                      ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype, float* G,
                      void* ws, size_t ws_bytes, void* stream);

/* Muon step from a given gradient G (layout as in ttt_grad); updates W in place.
 * Newton-Schulz precision: TTT_FP32 multiplies in fp32 on the CUDA cores;
 * TTT_BF16 multiplies on the tensor cores from split operands (each fp32
 * value as bf16 hi + bf16 lo, products hi*hi + hi*lo + lo*hi accumulated in
 * fp32), about 2^-16 relative per product. */
int ttt_step(ttt_weights W, const float* G, const ttt_ns_cfg* ns, ttt_dims dims, ttt_dtype dtype,
             void* ws, size_t ws_bytes, void* stream);

/* TTTUpdate: `steps` times { G = gradient over all T tokens at the current W; Muon step }.
 * steps = 2 is VGG-T3's test-time scaling.  T = 0 leaves W unchanged. */
int ttt_update(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, int steps,
               const ttt_ns_cfg* ns, ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype,
               void* ws, size_t ws_bytes, void* stream);

/* TTTUpdate with ShortConv2D on V (VGG-T3 key design 2) folded into the update's
 * operand preparation: the same result as ttt_shortconv2d(V -> V', taps, T /
 * (grid_h * grid_w) frames of grid_h x grid_w, act) followed by ttt_update(K, V'),
 * except that the convolved values are rounded once, to the update's fp16 value
 * operand, instead of first to bf16 -- V' itself is never written.  taps: device
 * float [H*d][3][3].  TTT_BF16 only; T must be whole frames; the head dim d must be
 * a multiple of 64 and a frame row must fit a shared-memory band (true for grids up
 * to several hundred tokens wide), else TTT_ERR_UNSUPPORTED.  The operand range of
 * the update (above) applies to the convolved values in place of V. */
int ttt_update_conv(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, int steps,
                    const ttt_ns_cfg* ns, const float* taps, int grid_h, int grid_w, int act, ttt_dims dims,
                    const ttt_io_cfg* io, ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/* Apply: O[i] = f_W(q_i) for T query rows (Q and O may not alias). */
int ttt_apply(ttt_weights W, const void* Q, void* O, int64_t T, ttt_dims dims,
              const ttt_io_cfg* io, ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/* Apply without a workspace and without any allocation (no counterpart in the
 * pages: this is a deployment convenience).  Computes exactly what ttt_apply
 * computes, for callers that cannot hand the library device memory for scratch:
 * hosts whose memory is fully reserved up front (a pool or arena that the
 * library cannot draw from), plugin environments that forbid cudaMalloc and
 * cudaFree, and latency-critical query loops that must not call into the
 * allocator at all.  Its scratch (the bf16 copies of W, the per-token Q norms
 * and a status word) lives in one fixed array of TTT_NOALLOC_SCRATCH_BYTES
 * (8 MiB) that the library declares statically in device memory, so every GPU
 * that loads the library holds those 8 MiB until the process exits.
 *  - Limit: 8 * H * m * d bytes of weight copies plus at least 128 tokens of
 *    norms (4 * H bytes each) must fit; larger dims return TTT_ERR_SCRATCH.
 *    T itself is unbounded: the call walks the queries in token chunks sized
 *    to the space left.  For 4 heads, d = 192, m = 768 that is 4.7 MiB of
 *    weights and chunks of up to ~200k tokens.
 *  - The first call on each device looks up that device's address of the
 *    array (a host-side lookup, no allocation); make the first call on a device
 *    before capturing a stream on it.
 *  - Every call reuses the same array and leaves its contents behind; the call
 *    clears the status word itself.  Calls whose work overlaps on the GPU (on
 *    different streams, or from different host threads) race on the array:
 *    order them on one stream.
 *  - A device-side wait that times out cannot be polled here (there is no
 *    workspace); O is then undefined.
 *  - The wide-head shapes (d and m multiples of 256) return TTT_ERR_UNSUPPORTED:
 *    their apply keeps a per-token intermediate in the workspace.
 *  - The looked-up address is kept for the life of the process: after
 *    cudaDeviceReset on a device, this entry point (like ttt_layer_host, whose
 *    copy streams and events are kept per device) must not be called again on
 *    that device.
 * Arguments and layouts as for ttt_apply, minus the workspace. */
#define TTT_NOALLOC_SCRATCH_BYTES (8u << 20)
int ttt_apply_noalloc(ttt_weights W, const void* Q, void* O, int64_t T, ttt_dims dims,
                      const ttt_io_cfg* io, ttt_dtype dtype, void* stream);

/* Gated output (ZipMap key design 3, the gated unit after the TTT read-out):
 *     o_t = RMSNorm(o'_t) * SiLU(W_g o'_t),  RMSNorm(x) = x / sqrt(mean(x^2) + 1e-6)
 * per token over the whole row of D values (all heads), without a learnable
 * scale and without a bias.
 *  - Oprime: [T][ld_in] bf16 (D columns used), e.g. the output of ttt_apply;
 *    O: [T][ld_out] bf16, may not alias Oprime.  ld 0 means D.
 *  - Wg: float [D][D] row-major, device (row j gives gate j: (W_g o')_j = Wg[j] . o').
 *  - ws: ttt_gate_workspace_bytes(T, D) bytes, 256-byte aligned: a bf16 copy of
 *    W_g and the per-token RMS factors.
 *  - TTT_BF16 only, D a multiple of 256 (the product runs on 2-SM tensor-core
 *    pairs in 256 x 256 tiles); other cases return TTT_ERR_UNSUPPORTED. */
size_t ttt_gate_workspace_bytes(int64_t T, int D);
int ttt_output_gate(const void* Oprime, int64_t ld_in, const float* Wg, void* O, int64_t ld_out, int64_t T, int D,
                    ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/* Causal chunk carry over T tokens in chunks of `chunk` (the last may be shorter).
 * order 0: O_c = f_{W_(c-1)}(Q_c), then W_c = TTTUpdate(W_(c-1); chunk c);
 * order 1: update first, then apply with W_c.  W is carried in place, so calling
 * again with the returned W resumes the stream. */
int ttt_chunked(ttt_weights W, const void* Q, const void* K, const void* V, const float* eta, void* O,
                int64_t T, int64_t chunk, int order, int steps, const ttt_ns_cfg* ns, ttt_dims dims,
                const ttt_io_cfg* io, ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/* The whole layer over HOST-resident tokens, with the host<->device copies
 * overlapped with the computation (no counterpart in the pages: this is how a
 * caller whose tokens live in host memory runs the layer without paying for
 * the copies and the computation one after the other).
 *  - hQ, hK, hV, hO: HOST pointers to dense [T][H*d] token matrices (dtype as
 *    given), hEta: HOST float [T][H].  They should be page-locked (pinned)
 *    memory; pageable memory works, but its copies do not overlap.
 *  - dbuf: DEVICE staging area of ttt_host_buffer_bytes(dims, T, dtype, conv)
 *    bytes, 256-byte aligned, owned by the caller; it receives the device
 *    copies of Q, K, V, eta and O (and V after ShortConv2D when conv = 1).
 *  - ws: the usual workspace, for T tokens (chunk = 0) or `chunk` tokens.
 *  - chunk = 0: `steps` Muon steps over all T tokens (as ttt_update), then the
 *    apply to all T queries.  K, V, eta arrive in token blocks; the first
 *    step's gradient is computed block by block while later blocks are still
 *    being copied (block gradients are summed, so the result equals ttt_update
 *    up to the order of that sum), and each block of O is copied back as soon
 *    as it has been computed, while later queries are still arriving.
 *  - chunk > 0: the causal carry of ttt_chunked with the given order (0: apply
 *    with the carried weights, then update; 1: update, then apply); chunk c+1
 *    is copied in while chunk c is computed and O of chunk c is copied back
 *    meanwhile.  order must be 0 or 1 (it is not read when chunk = 0).
 *  - taps (device float [H*d][3][3]) non-null applies ShortConv2D to V over
 *    frames of grid_h x grid_w tokens first (T must be whole frames); the
 *    token blocks of chunk = 0 are then whole frames, and chunk must be too.
 *  - io: only qk_l2norm is read (host rows are dense).
 * On return the work is queued on `stream`: when `stream` has completed, hO
 * holds the outputs and W the updated weights.  The library creates two copy
 * streams and a pool of events per device on first use and keeps them. */
size_t ttt_host_buffer_bytes(ttt_dims dims, int64_t T, ttt_dtype dtype, int conv);
int ttt_layer_host(ttt_weights W, const void* hQ, const void* hK, const void* hV, const float* hEta, void* hO,
                   int64_t T, int64_t chunk, int order, int steps, const ttt_ns_cfg* ns, const float* taps, int grid_h,
                   int grid_w, ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype, void* dbuf, size_t dbuf_bytes,
                   void* ws, size_t ws_bytes, void* stream);

/* Diagnostic for the timeout path: launches one single-warp kernel that waits on
 * a barrier nothing ever signals, with a wait limit of `timeout_us`
 * microseconds.  The wait gives up, records TTT_ERR_TIMEOUT in the workspace
 * status word and the kernel returns, so the CUDA context stays usable; a
 * following ttt_poll_status reports TTT_ERR_TIMEOUT until ttt_reset_status.
 * timeout_us must be in [1, 10^7]. */
int ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned timeout_us, void* stream);

/* Target the library's kernels were compiled for, from the compiler's
 * architecture list (1000 for sm_100a); needs no GPU. */
int ttt_compiled_arch(void);

/* Binary version the CUDA runtime reports for the library's kernels on the
 * current device (major * 10 + minor: 100 for sm_100a) into *version.
 * Returns TTT_ERR_CUDA without a usable device. */
int ttt_kernel_binary_version(int* version);

/* Human-readable name of a status code (static string). */
const char* ttt_status_string(int status);

/* Number of kernel launches the library queued since load (for launch accounting). */
uint64_t ttt_launch_count(void);

/* Per-kernel device timing.  While profiling is on, the library records a pair
 * of CUDA events on the launch stream around each of its kernels (or kernel
 * groups) and files the pair under one of the kinds below.  ttt_profile_query
 * waits for the recorded events, adds their durations to the kind's totals and
 * returns them; ttt_profile_reset clears the totals.  Host-thread safe; the
 * events cost a few microseconds per launch, so leave profiling off when not
 * measuring. */
typedef enum {
  TTT_PROF_GRAD = 0,    /* gradient kernel (tensor-core in bf16 mode) */
  TTT_PROF_APPLY = 1,   /* apply kernel */
  TTT_PROF_NS = 2,      /* Newton-Schulz iterations and the weight step */
  TTT_PROF_NORM = 3,    /* row norms (fp32 mode, ttt_l2norm) and the max |eta| of the bf16 update */
  TTT_PROF_CONV = 4,    /* ShortConv2D */
  TTT_PROF_REDUCE = 5,  /* split-K reduction of the gradient partials */
  TTT_PROF_SHADOW = 6,  /* bf16 copies of the fast weights */
  TTT_PROF_KINDS = 7
} ttt_prof_kind;

int ttt_profile_enable(int on);
int ttt_profile_reset(void);
int ttt_profile_query(int kind, double* total_ms, uint64_t* count);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H */
