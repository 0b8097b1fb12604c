// C ABI of the large-chunk TTT layer (see include/ttt.h for the contract).
//
// Host side: argument validation, workspace carving, TMA tensor-map encoding
// and the launch sequences of update / apply / chunked.  All device work runs
// in the kernels of kernels_tc.cuh (bf16 tensor-core path) and
// kernels_simt.cuh (memory-bound and fp32 paths); nothing here computes on
// the CPU.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels_nsmma.cuh"
#include "kernels_simt.cuh"
#include "kernels_tc.cuh"
#include "kernels_wide.cuh"
#include "ttt.h"

using namespace ttt;

namespace {

std::atomic<uint64_t> g_launches{0};

// ---- per-kernel event timing (ttt_profile_*)
struct ProfPair {
  cudaEvent_t a, b;
  int kind;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfPair> g_prof_pending;
std::vector<cudaEvent_t> g_prof_pool;
double g_prof_ms[TTT_PROF_KINDS] = {0};
uint64_t g_prof_n[TTT_PROF_KINDS] = {0};

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Records an event pair around the launches issued during its lifetime.
struct ProfScope {
  cudaEvent_t a = nullptr, b = nullptr;
  cudaStream_t s;
  int kind;
  ProfScope(int k, cudaStream_t st) : s(st), kind(k) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    a = prof_event();
    b = prof_event();
    if (a && b) cudaEventRecord(a, s);
  }
  ~ProfScope() {
    if (!a || !b) return;
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_pending.push_back({a, b, kind});
  }
};
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per device-side wait
constexpr int kMaxSplits = 64;
constexpr int kAssumedMaxSms = 160;

struct Ws {
  unsigned int* status;
  __nv_bfloat16* wsh;  // [3][H*m][d]: W1, W3, W2^T
  __nv_bfloat16* w2b;  // [H][d][m]
  float* G;            // [3][H*m*d]
  float* partial;      // [S_max][3][H*m*d]
  float* X;            // [3H][m*d] Newton-Schulz iterate, wide orientation (r x c)
  float* X2;           // [3H][m*d]
  float* XT;           // [3H][m*d] its transpose (c x r)
  float* XT2;          // [3H][m*d]
  float* A;            // [3H][r*r]
  float* B;            // [3H][r*r]
  float* gram;         // [max(NS_GRAM_SPLIT, NSM_GRAM_SPLIT_MAX)][3H][r*r] split-K partials of the Gram matrices
  float* norms;        // [3H][NORM_PARTS] partial sums of squares of G
  float* stepn;        // [3H][NORM_PARTS][2] partials of ||W||^2, ||W - lr D||^2
  float* rk;           // [T][H]
  float* rq;           // [T][H]
  __half* wsh16;       // [3][H*m][d] fp16: W1, W3, W2^T (gradient kernel)
  float* etapart;      // [ETA_PARTS] block maxima of |eta| (value scale s of V')
  __half* kh16;        // [T][H*d] fp16 K^ (gradient operand)
  __half* vh16;        // [T][H*d] fp16 V' = -s eta v
  // wide-head path only (d, m multiples of 256): fp16 intermediates [T][H*m]
  __half* z16;         // Z = V' W2 (scaled dL/du)
  __half* dh1;         // dL/dh1 (the apply's P, bf16, reuses this buffer)
  __half* dh3;         // dL/dh3
  __half* u16;         // u
  // wide-head Newton-Schulz: bf16 hi/lo parts of X (ping-pong), A and B = c A A + b A
  __nv_bfloat16 *xh, *xl, *x2h, *x2l, *ah, *al, *bh, *bl;
  size_t total;
  int s_max;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

int split_cap(const ttt_dims& d, ttt_dtype dt) {
  const int slices = dt == TTT_BF16 ? d.heads * d.m / TC_MS : d.heads * d.m / F32_MS;
  const int want = dt == TTT_BF16 ? kAssumedMaxSms / std::max(1, slices) : 2 * kAssumedMaxSms / std::max(1, slices);
  return std::max(1, std::min(kMaxSplits, want));
}

bool dims_ok(const ttt_dims& d) { return d.heads >= 1 && d.d >= 1 && d.m >= 1 && d.heads <= 4096; }

// bf16 heads of width d, m multiples of 256 (e.g. d = 1024, m = 2048) run the
// wide-head path of kernels_wide.cuh; d in {128, 192} the fused kernels.
bool wide_dims(const ttt_dims& d) { return d.d >= 256 && d.d % 256 == 0 && d.m % 256 == 0 && d.d <= 8192 && d.m <= 16384; }

int dims_supported(const ttt_dims& d, ttt_dtype dt) {
  if (dt == TTT_BF16)
    return ((d.d == 128 || d.d == 192) && d.m % TC_MS == 0) || wide_dims(d) ? TTT_OK : TTT_ERR_UNSUPPORTED;
  if (dt == TTT_FP32) return (d.d <= 256 && d.d % 4 == 0 && d.m % F32_MS == 0) ? TTT_OK : TTT_ERR_UNSUPPORTED;
  return TTT_ERR_INVALID;
}

Ws carve(void* base, const ttt_dims& dm, int64_t T, ttt_dtype dt) {
  Ws w{};
  const size_t H = dm.heads, d = dm.d, m = dm.m;
  const size_t n = H * m * d;
  const size_t r = std::min(d, m);
  w.s_max = split_cap(dm, dt);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = up256(off + bytes);
    return o;
  };
  const size_t o_status = take(256);
  const size_t o_wsh = take(3 * n * 2);
  const size_t o_w2b = take(n * 2);
  const size_t o_G = take(3 * n * 4);
  const size_t o_p = take((size_t)w.s_max * 3 * n * 4);
  const size_t o_X = take(3 * n * 4);
  const size_t o_X2 = take(3 * n * 4);
  const size_t o_XT = take(3 * n * 4);
  const size_t o_XT2 = take(3 * n * 4);
  const size_t o_A = take(3 * H * r * r * 4);
  const size_t o_B = take(3 * H * r * r * 4);
  const size_t o_gram = take((size_t)std::max(NS_GRAM_SPLIT, NSM_GRAM_SPLIT_MAX) * 3 * H * r * r * 4);
  const size_t o_norms = take(3 * H * NORM_PARTS * 4);
  const size_t o_stepn = take(3 * H * NORM_PARTS * 2 * 4);
  // every buffer whose size does not depend on T comes first, so its offset is the same
  // for any T (ttt_step carves with T = 0 beside ttt_grad's T-token layout)
  const bool tc = dt == TTT_BF16;
  const bool wide = tc && wide_dims(dm);
  const size_t o_wsh16 = tc ? take(3 * n * 2) : 0;
  const size_t o_etap = tc ? take(ETA_PARTS * 4) : 0;
  const size_t nsx = wide ? 3 * n * 2 : 0, nsa = wide ? 3 * H * r * r * 2 : 0;
  const size_t o_xh = wide ? take(nsx) : 0, o_xl = wide ? take(nsx) : 0;
  const size_t o_x2h = wide ? take(nsx) : 0, o_x2l = wide ? take(nsx) : 0;
  const size_t o_ah = wide ? take(nsa) : 0, o_al = wide ? take(nsa) : 0;
  const size_t o_bh = wide ? take(nsa) : 0, o_bl = wide ? take(nsa) : 0;
  // per-token buffers
  const size_t o_rk = take((size_t)std::max<int64_t>(T, 1) * H * 4);
  const size_t o_rq = take((size_t)std::max<int64_t>(T, 1) * H * 4);
  const size_t tokd = (size_t)std::max<int64_t>(T, 1) * H * d * 2, tokm = (size_t)std::max<int64_t>(T, 1) * H * m * 2;
  const size_t o_kh = tc ? take(tokd) : 0;
  const size_t o_vh = tc ? take(tokd) : 0;
  const size_t o_z = wide ? take(tokm) : 0;
  const size_t o_dh1 = wide ? take(tokm) : 0;
  const size_t o_dh3 = wide ? take(tokm) : 0;
  const size_t o_u = wide ? take(tokm) : 0;
  w.total = off;
  uint8_t* b = static_cast<uint8_t*>(base);
  if (b) {
    w.status = reinterpret_cast<unsigned int*>(b + o_status);
    w.wsh = reinterpret_cast<__nv_bfloat16*>(b + o_wsh);
    w.w2b = reinterpret_cast<__nv_bfloat16*>(b + o_w2b);
    w.G = reinterpret_cast<float*>(b + o_G);
    w.partial = reinterpret_cast<float*>(b + o_p);
    w.X = reinterpret_cast<float*>(b + o_X);
    w.X2 = reinterpret_cast<float*>(b + o_X2);
    w.XT = reinterpret_cast<float*>(b + o_XT);
    w.XT2 = reinterpret_cast<float*>(b + o_XT2);
    w.A = reinterpret_cast<float*>(b + o_A);
    w.B = reinterpret_cast<float*>(b + o_B);
    w.gram = reinterpret_cast<float*>(b + o_gram);
    w.norms = reinterpret_cast<float*>(b + o_norms);
    w.stepn = reinterpret_cast<float*>(b + o_stepn);
    w.rk = reinterpret_cast<float*>(b + o_rk);
    w.rq = reinterpret_cast<float*>(b + o_rq);
    if (tc) {
      w.wsh16 = reinterpret_cast<__half*>(b + o_wsh16);
      w.etapart = reinterpret_cast<float*>(b + o_etap);
      w.kh16 = reinterpret_cast<__half*>(b + o_kh);
      w.vh16 = reinterpret_cast<__half*>(b + o_vh);
      if (wide) {
        w.z16 = reinterpret_cast<__half*>(b + o_z);
        w.dh1 = reinterpret_cast<__half*>(b + o_dh1);
        w.dh3 = reinterpret_cast<__half*>(b + o_dh3);
        w.u16 = reinterpret_cast<__half*>(b + o_u);
        auto bf = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(b + o); };
        w.xh = bf(o_xh);
        w.xl = bf(o_xl);
        w.x2h = bf(o_x2h);
        w.x2l = bf(o_x2l);
        w.ah = bf(o_ah);
        w.al = bf(o_al);
        w.bh = bf(o_bh);
        w.bl = bf(o_bl);
      }
    }
  }
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

unsigned long long wait_timeout_ns() {
  static unsigned long long v = [] {
    const char* e = std::getenv("TTT_WAIT_TIMEOUT_MS");
    if (e && *e) {
      long long ms = std::atoll(e);
      if (ms > 0) return (unsigned long long)ms * 1000000ull;
    }
    return kDefaultTimeoutNs;
  }();
  return v;
}

// ---- TMA tensor maps (driver entry point fetched once through the runtime)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [outer][inner] with row stride `row_bytes`, 128-byte swizzled boxes.
bool tmap_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_inner, uint32_t box_outer,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

#define TTT_LAUNCHED()                                         \
  do {                                                         \
    g_launches.fetch_add(1, std::memory_order_relaxed);        \
    if (cudaPeekAtLastError() != cudaSuccess) {                \
      (void)cudaGetLastError();                                \
      return TTT_ERR_CUDA;                                     \
    }                                                          \
  } while (0)

#define TTT_CHECK(expr)                        \
  do {                                         \
    if ((expr) != cudaSuccess) {               \
      (void)cudaGetLastError();                \
      return TTT_ERR_CUDA;                     \
    }                                          \
  } while (0)

#define TTT_TRY(expr)           \
  do {                          \
    int rc_ = (expr);           \
    if (rc_ != TTT_OK) return rc_; \
  } while (0)

int grid1d(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)std::max<int64_t>(1, std::min<int64_t>(b, (int64_t)sm_count() * 32));
}

size_t esize(ttt_dtype dt) { return dt == TTT_BF16 ? 2 : 4; }

int64_t eff_ld(int64_t ld, const ttt_dims& d) { return ld == 0 ? (int64_t)d.heads * d.d : ld; }

int check_tokens(const void* p, int64_t ld, const ttt_dims& d, ttt_dtype dt, int64_t T) {
  if (T == 0) return TTT_OK;
  if (!p) return TTT_ERR_INVALID;
  if (ld < (int64_t)d.heads * d.d) return TTT_ERR_INVALID;
  if (!aligned16(p)) return TTT_ERR_ALIGN;
  if ((ld * (int64_t)esize(dt)) % 16 != 0) return TTT_ERR_ALIGN;
  return TTT_OK;
}

int check_common(const ttt_dims& dims, ttt_dtype dt, int64_t T, void* ws, size_t ws_bytes) {
  if (dt != TTT_FP32 && dt != TTT_BF16) return TTT_ERR_INVALID;
  if (!dims_ok(dims) || T < 0) return TTT_ERR_INVALID;
  TTT_TRY(dims_supported(dims, dt));
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTT_ERR_WORKSPACE;
  if (ws_bytes < carve(nullptr, dims, T, dt).total) return TTT_ERR_WORKSPACE;
  return TTT_OK;
}

int check_weights(const ttt_weights& W) {
  if (!W.W1 || !W.W3 || !W.W2) return TTT_ERR_INVALID;
  if (!aligned16(W.W1) || !aligned16(W.W3) || !aligned16(W.W2)) return TTT_ERR_ALIGN;
  return TTT_OK;
}

// ---- launch helpers

template <typename T>
int launch_rownorm(T* X, int64_t ld, int64_t rows, const ttt_dims& d, float* r_out, int mode, cudaStream_t s) {
  if (rows == 0) return TTT_OK;
  const int threads = 256;
  const int64_t warps = rows;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((warps * 32 + threads - 1) / threads,
                                                                   (int64_t)sm_count() * 8));
  ProfScope ps(TTT_PROF_NORM, s);
  k_rownorm<T><<<blocks, threads, 0, s>>>(X, ld, rows, d.heads, d.d, r_out, mode);
  TTT_LAUNCHED();
  return TTT_OK;
}

int launch_rownorm_any(const void* X, int64_t ld, int64_t rows, const ttt_dims& d, ttt_dtype dt, float* r_out,
                       cudaStream_t s) {
  if (dt == TTT_BF16)
    return launch_rownorm<__nv_bfloat16>((__nv_bfloat16*)X, ld, rows, d, r_out, 0, s);
  return launch_rownorm<float>((float*)X, ld, rows, d, r_out, 0, s);
}

// Rows per band of the two-output bf16 ShortConv2D kernel: the largest band that keeps two
// CTAs per SM (or one, for very wide frames); 0 when not even a band of one row fits.
int conv2_band_rows(int gh, int gw) {
  const size_t fixed = 9 * CONV_GROUP * sizeof(float);
  const size_t row2 = (size_t)conv2_row_slots(gw) * CONV_GROUP * 2;
  for (size_t budget : {(size_t)110 * 1024, (size_t)220 * 1024}) {
    const int64_t br = (int64_t)((budget - fixed) / (2 * row2)) - 2;
    if (br >= 1) return (int)std::min<int64_t>(br, gh);
  }
  return 0;
}

// ShortConv2D launch: the banded shared-memory kernel with the largest band
// that keeps two CTAs per SM (or one, for very wide frames); the direct kernel
// for frames too wide for one band of three rows.
int launch_conv_any(const void* V, int64_t ldv, void* Vout, int64_t ldo, const float* taps, int64_t N, int gh, int gw,
                    int C, int act, ttt_dtype dt, cudaStream_t s) {
  if (N == 0) return TTT_OK;
  const int esz = dt == TTT_BF16 ? 2 : 4;
  const size_t row = (size_t)gw * CONV_GROUP * esz, fixed = 9 * CONV_GROUP * sizeof(float);
  int BR = 0;
  for (size_t budget : {(size_t)110 * 1024, (size_t)220 * 1024}) {
    const int64_t br = (int64_t)((budget - fixed) / (2 * row)) - 2;
    if (br >= 1) {
      BR = (int)std::min<int64_t>(br, gh);
      break;
    }
  }
  const dim3 grid((C + CONV_GROUP - 1) / CONV_GROUP, (unsigned)std::min<int64_t>(N, 65535));
  ProfScope ps(TTT_PROF_CONV, s);
  if (dt == TTT_BF16) {
    // the two-outputs-per-thread bf16 kernel, same band choice with its padded rows
    const int BR2 = conv2_band_rows(gh, gw);
    if (BR2 >= 1) {
      const size_t smem = conv2_band_smem(BR2, gw);
      TTT_CHECK(cudaFuncSetAttribute(k_shortconv_band2<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      k_shortconv_band2<false><<<grid, 256, smem, s>>>((const __nv_bfloat16*)V, ldv, Vout, ldo, taps, (int)N, gh, gw, C,
                                                       act, BR2, nullptr, nullptr, 1, 1);
      TTT_LAUNCHED();
      return TTT_OK;
    }
  }
  if (BR >= 1) {
    const size_t smem = conv_band_smem(BR, gw, esz);
    if (dt == TTT_BF16) {
      TTT_CHECK(cudaFuncSetAttribute(k_shortconv_band<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
      k_shortconv_band<__nv_bfloat16><<<grid, 256, smem, s>>>((const __nv_bfloat16*)V, ldv, (__nv_bfloat16*)Vout, ldo,
                                                              taps, (int)N, gh, gw, C, act, BR);
    } else {
      TTT_CHECK(cudaFuncSetAttribute(k_shortconv_band<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      k_shortconv_band<float><<<grid, 256, smem, s>>>((const float*)V, ldv, (float*)Vout, ldo, taps, (int)N, gh, gw, C,
                                                      act, BR);
    }
  } else {
    const int vn = dt == TTT_BF16 ? 8 : 4;
    const int gv = CONV_GROUP / vn;
    const dim3 block(gv, 256 / gv);
    const dim3 grid2((unsigned)N, (C + CONV_GROUP - 1) / CONV_GROUP);
    if (N > 2147483647) return TTT_ERR_UNSUPPORTED;
    if (dt == TTT_BF16)
      k_shortconv<__nv_bfloat16><<<grid2, block, 0, s>>>((const __nv_bfloat16*)V, ldv, (__nv_bfloat16*)Vout, ldo, taps,
                                                         (int)N, gh, gw, C, act);
    else
      k_shortconv<float><<<grid2, block, 0, s>>>((const float*)V, ldv, (float*)Vout, ldo, taps, (int)N, gh, gw, C,
                                                 act);
  }
  TTT_LAUNCHED();
  return TTT_OK;
}

// Launch with programmatic stream serialisation: the kernel may begin while the
// previous kernel on the stream finishes, and must call pdl_wait() before it
// touches memory that kernel writes.  Used for the short dependent kernels of
// the Muon step, whose launch latency is otherwise a large share of their time.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  TTT_CHECK(cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...));
  return TTT_OK;
}

int launch_shadow(const ttt_weights& W, const Ws& w, const ttt_dims& d, cudaStream_t s, bool pdl = false) {
  const int64_t n = (int64_t)d.heads * d.m * d.d;
  if (n % SHADOW_EW_BLOCK || d.d % 32 || d.m % 32) return TTT_ERR_UNSUPPORTED;
  const int blocks = (int)(n / SHADOW_EW_BLOCK) + d.heads * (d.d / 32) * (d.m / 32);
  ProfScope ps(TTT_PROF_SHADOW, s);
  if (pdl)
    return launch_pdl(k_shadow, dim3(blocks), dim3(256), 0, s, W.W1, W.W3, W.W2, w.wsh, w.w2b, w.wsh16, d.heads, d.d,
                      d.m);
  k_shadow<<<blocks, 256, 0, s>>>(W.W1, W.W3, W.W2, w.wsh, w.w2b, w.wsh16, d.heads, d.d, d.m);
  TTT_LAUNCHED();
  return TTT_OK;
}

// block maxima of |eta| over T x H values -> w.etapart (they fix the value scale s)
int launch_eta_absmax(const float* eta, int64_t T, const ttt_dims& d, const Ws& w, cudaStream_t s) {
  const int64_t n = T * d.heads;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ETA_PARTS, (n + 2047) / 2048));
  ProfScope ps(TTT_PROF_NORM, s);
  k_eta_absmax<<<blocks, 512, 0, s>>>(eta, n, w.etapart, ETA_PARTS);
  TTT_LAUNCHED();
  return TTT_OK;
}

// fp16 gradient operands of T tokens (dense [T][H*d], written at kh, vh) from the
// caller's bf16 K, V: K^ and V' = -s eta v with the value scale s of w.etapart.
// self_max: the kernel reduces max|eta| itself and writes w.etapart (calls of at
// most kSelfMaxEta values, where one launch fewer matters more than each block
// reading all of eta); otherwise k_eta_absmax has written w.etapart.
constexpr int64_t kSelfMaxEta = 8192;
int launch_prep_kv(const void* K, int64_t ldk, const void* V, int64_t ldv, const float* eta, int64_t T,
                   const ttt_dims& d, int l2norm, const Ws& w, __half* kh, __half* vh, cudaStream_t s,
                   bool self_max = false) {
  if (T == 0) return TTT_OK;
  ProfScope ps(TTT_PROF_NORM, s);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((T * 32 + 255) / 256, (int64_t)sm_count() * 16));
  const int nvt = d.heads * d.d / 8;  // 16-byte vectors per row
  const float* part_in = self_max ? nullptr : w.etapart;
  float* part_out = self_max ? w.etapart : nullptr;
  if (nvt <= 96)
    k_prep_kv<3><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)K, ldk, (const __nv_bfloat16*)V, ldv, eta, part_in,
                                        kh, vh, T, d.heads, d.d, l2norm, part_out);
  else
    k_prep_kv<4><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)K, ldk, (const __nv_bfloat16*)V, ldv, eta, part_in,
                                        kh, vh, T, d.heads, d.d, l2norm, part_out);
  TTT_LAUNCHED();
  return TTT_OK;
}

struct UpdOperands {
  const void* K;
  int64_t ldk;
  const void* V;
  int64_t ldv;
  const float* rk;
};

// The fp16 gradient operands of N frames with ShortConv2D on V fused into the value
// operand: K^ from the preparation kernel (K only), V' = -s eta conv(V) straight from the
// conv kernel (bf16 mode; the |eta| maxima must be in w.etapart).  Returns
// TTT_ERR_UNSUPPORTED when the frames are too wide for a row band.
int launch_conv_prep(const void* K, int64_t ldk, const void* V, int64_t ldv, const float* taps, int64_t N, int gh,
                     int gw, int act, const float* eta, int l2norm, const ttt_dims& d, const Ws& w, cudaStream_t s) {
  const int C = d.heads * d.d;
  const int BR2 = conv2_band_rows(gh, gw);
  if (BR2 < 1 || d.d % CONV_GROUP) return TTT_ERR_UNSUPPORTED;
  const int64_t T = N * gh * gw;
  TTT_TRY(launch_prep_kv(K, ldk, nullptr, 0, eta, T, d, l2norm, w, w.kh16, nullptr, s));
  const size_t smem = conv2_band_smem(BR2, gw);
  const dim3 grid((C + CONV_GROUP - 1) / CONV_GROUP, (unsigned)std::min<int64_t>(N, 65535));
  ProfScope ps(TTT_PROF_CONV, s);
  TTT_CHECK(cudaFuncSetAttribute(k_shortconv_band2<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  k_shortconv_band2<true><<<grid, 256, smem, s>>>((const __nv_bfloat16*)V, ldv, w.vh16, C, taps, (int)N, gh, gw, C, act,
                                                  BR2, eta, w.etapart, d.heads, d.d);
  TTT_LAUNCHED();
  return TTT_OK;
}

// Operands of the gradient kernels for T tokens: fp16 K^/V' copies in bf16 mode
// (V' carries the per-token weights eta and the value scale s; w.etapart the
// |eta| maxima that fix s), the caller's K/V plus per-token inverse norms in
// fp32 mode.
int prepare_update_operands(const void* K, int64_t ldk, const void* V, int64_t ldv, const float* eta, int64_t T,
                            const ttt_dims& d, ttt_dtype dt, int l2norm, const Ws& w, cudaStream_t s,
                            UpdOperands* op) {
  if (dt == TTT_BF16) {
    const bool self_max = T * d.heads <= kSelfMaxEta;
    if (T > 0 && !self_max) TTT_TRY(launch_eta_absmax(eta, T, d, w, s));
    TTT_TRY(launch_prep_kv(K, ldk, V, ldv, eta, T, d, l2norm, w, w.kh16, w.vh16, s, self_max));
    const int64_t hd = (int64_t)d.heads * d.d;
    *op = {w.kh16, hd, w.vh16, hd, nullptr};
    return TTT_OK;
  }
  *op = {K, ldk, V, ldv, nullptr};
  if (l2norm && T > 0) {
    TTT_TRY(launch_rownorm_any(K, ldk, T, d, dt, w.rk, s));
    op->rk = w.rk;
  }
  return TTT_OK;
}

// ---- wide-head path (kernels_wide.cuh)

// One persistent launch of k_wgemm on 2-SM pairs: n_items output tiles, one pair per
// two SMs (or fewer pairs when there are fewer tiles).
template <int EPI, bool AMN, bool BMN>
int launch_wgemm(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& a2, const CUtensorMap& b0,
                 const CUtensorMap& b1, const WgArgs& args, int n_items, const Ws& w, cudaStream_t s) {
  if (n_items <= 0) return TTT_OK;
  auto k = k_wgemm<EPI, AMN, BMN>;
  TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, wg_smem_bytes<EPI>()));
  const int npairs = std::max(1, std::min(n_items, sm_count() / 2));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * npairs);
  cfg.blockDim = dim3(WG_THREADS);
  cfg.dynamicSmemBytes = wg_smem_bytes<EPI>();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TTT_CHECK(cudaLaunchKernelEx(&cfg, k, a0, a1, a2, b0, b1, args, n_items, w.status, wait_timeout_ns()));
  TTT_LAUNCHED();
  return TTT_OK;
}

WgArgs wg_args() {
  WgArgs a{};
  a.mt = a.nt = a.nt2 = a.nmat = a.heads = a.S = 1;
  return a;
}

// K-major operand map: rows of `cols` elements (2 bytes each), 64 x 128 boxes.
bool tmap_k(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows, uint64_t ld, bool f16) {
  return tmap_bf16(tm, base, cols, rows, ld * 2, 64, 128,
                   f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}
// MN-major operand map over token rows: 64 x 64 boxes (64 columns of 64 tokens).
bool tmap_mn(CUtensorMap* tm, const void* base, uint64_t cols, uint64_t rows, bool f16 = true) {
  return tmap_bf16(tm, base, cols, rows, cols * 2, 64, 64,
                   f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

// Newton-Schulz iterations of the wide-head path on the 2-SM GEMM kernel: nb matrices
// X (r x c, fp32, stacked) -> X after `iters` steps.  Every product takes split bf16
// operands (hi + lo) as three K segments, hi.hi + hi.lo + lo.hi, and its epilogue
// writes the fp32 result with its own hi/lo parts for the next product.
int run_ns_iters_wide(const ttt_ns_cfg& ns, int r, int c, int nb, const Ws& w, float*& X, float*& X2,
                      cudaStream_t s) {
  const int64_t nx = (int64_t)nb * r * c;
  __nv_bfloat16 *xh = w.xh, *xl = w.xl, *x2h = w.x2h, *x2l = w.x2l;
  k_split_bf16<<<grid1d(nx / 4, 256), 256, 0, s>>>(X, xh, xl, nx);
  TTT_LAUNCHED();
  CUtensorMap tAh, tAl, tBh, tBl;
  const uint64_t R = (uint64_t)nb * r;
  if (!tmap_k(&tAh, w.ah, (uint64_t)r, R, (uint64_t)r, false) || !tmap_k(&tAl, w.al, (uint64_t)r, R, (uint64_t)r, false) ||
      !tmap_k(&tBh, w.bh, (uint64_t)r, R, (uint64_t)r, false) || !tmap_k(&tBl, w.bl, (uint64_t)r, R, (uint64_t)r, false))
    return TTT_ERR_CUDA;
  for (int it = 0; it < ns.iters; ++it) {
    CUtensorMap tXh, tXl, tXmh, tXml;
    if (!tmap_k(&tXh, xh, (uint64_t)c, R, (uint64_t)c, false) || !tmap_k(&tXl, xl, (uint64_t)c, R, (uint64_t)c, false) ||
        !tmap_mn(&tXmh, xh, (uint64_t)c, R, false) || !tmap_mn(&tXml, xl, (uint64_t)c, R, false))
      return TTT_ERR_CUDA;
    WgArgs g = wg_args();
    g.M = r;
    g.heads = nb;
    g.a_row_head = r;
    g.idesc = idesc_bf16(256, 256, false, false);
    // A = X X^T (B rows = X rows)
    WgArgs a1 = g;
    a1.mt = a1.nt = r / 256;
    a1.kblocks = 3 * (c / 64);
    a1.b_head = r;
    a1.out = w.A;
    a1.out2 = w.ah;
    a1.out3 = w.al;
    a1.ldo = r;
    a1.alpha = 1.f;
    a1.beta = 0.f;
    TTT_TRY((launch_wgemm<WG_NSOUT, false, false>(tXh, tXl, tXl, tXh, tXl, a1, a1.mt * a1.nt * nb, w, s)));
    // B = c A A + b A (A symmetric: its rows serve as the B operand's rows)
    WgArgs a2 = g;
    a2.mt = a2.nt = r / 256;
    a2.kblocks = 3 * (r / 64);
    a2.b_head = r;
    a2.out = w.B;
    a2.out2 = w.bh;
    a2.out3 = w.bl;
    a2.ldo = r;
    a2.aux = w.A;
    a2.alpha = ns.c;
    a2.beta = ns.b;
    TTT_TRY((launch_wgemm<WG_NSOUT, false, false>(tAh, tAl, tAl, tAh, tAl, a2, a2.mt * a2.nt * nb, w, s)));
    // X' = B X + a X (X rows are the K rows of the MN-major B operand)
    WgArgs a3 = g;
    a3.mt = r / 256;
    a3.nt = c / 256;
    a3.kblocks = 3 * (r / 64);
    a3.b_y_head = r;
    a3.out = X2;
    a3.out2 = x2h;
    a3.out3 = x2l;
    a3.ldo = c;
    a3.aux = X;
    a3.alpha = 1.f;
    a3.beta = ns.a;
    a3.idesc = idesc_bf16(256, 256, false, true);
    TTT_TRY((launch_wgemm<WG_NSOUT, false, true>(tBh, tBl, tBl, tXmh, tXml, a3, a3.mt * a3.nt * nb, w, s)));
    std::swap(X, X2);
    std::swap(xh, x2h);
    std::swap(xl, x2l);
  }
  return TTT_OK;
}

// Gradient of the wide path from the prepared fp16 operands K^, V' ([T][H*d]):
// Z, dH1/dH3/u, then split-K weight gradients (partials scaled by 1/s) and the
// fixed-order reduction into G.
int run_grad_wide(const void* K, const void* V, int64_t T, const ttt_dims& d, const Ws& w, float* G,
                  cudaStream_t s, bool accumulate) {
  const int H = d.heads, dd = d.d, mm = d.m;
  const int64_t n = (int64_t)H * mm * dd;
  const uint64_t hd = (uint64_t)H * dd, hm = (uint64_t)H * mm;
  CUtensorMap tKh, tVh, tW, tKm, tVm, tD1, tD3, tU;
  if (!tmap_k(&tKh, K, hd, (uint64_t)T, hd, true) || !tmap_k(&tVh, V, hd, (uint64_t)T, hd, true) ||
      !tmap_k(&tW, w.wsh16, (uint64_t)dd, 3ull * H * mm, (uint64_t)dd, true) ||
      !tmap_mn(&tKm, K, hd, (uint64_t)T) || !tmap_mn(&tVm, V, hd, (uint64_t)T) ||
      !tmap_mn(&tD1, w.dh1, hm, (uint64_t)T) || !tmap_mn(&tD3, w.dh3, hm, (uint64_t)T) ||
      !tmap_mn(&tU, w.u16, hm, (uint64_t)T))
    return TTT_ERR_CUDA;
  const int mt = (int)((T + 255) / 256);
  ProfScope ps(TTT_PROF_GRAD, s);
  {  // Z = V' W2 (B rows: the W2^T block of the fp16 weight copy)
    WgArgs a = wg_args();
    a.M = (int)T;
    a.mt = mt;
    a.nt = mm / 256;
    a.heads = H;
    a.kblocks = dd / 64;
    a.a_head = dd;
    a.b_row0 = 2 * H * mm;
    a.b_head = mm;
    a.out_head = mm;
    a.out = w.z16;
    a.ldo = (int64_t)hm;
    a.idesc = idesc_f16(256, 256, false, false);
    TTT_TRY((launch_wgemm<WG_STORE16, false, false>(tVh, tVh, tVh, tW, tW, a, mt * a.nt * H, w, s)));
  }
  {  // [H1 | H3] = K^ [W1; W3]^T, 128 m columns per tile -> dH1, dH3, u
    WgArgs a = wg_args();
    a.M = (int)T;
    a.mt = mt;
    a.nt = mm / 128;
    a.heads = H;
    a.kblocks = dd / 64;
    a.a_head = dd;
    a.b_row0 = 0;
    a.b_head = mm;
    a.b_row1 = H * mm;
    a.m = mm;
    a.d = dd;
    a.out = w.dh1;
    a.out2 = w.dh3;
    a.out3 = w.u16;
    a.aux = w.z16;
    a.ldo = a.ldaux = (int64_t)hm;
    a.idesc = idesc_f16(256, 256, false, false);
    TTT_TRY((launch_wgemm<WG_SWIGLU_BWD, false, false>(tKh, tKh, tKh, tW, tW, a, mt * a.nt * H, w, s)));
  }
  int S = 1;
  {  // g1 = dH1^T K^, g3 = dH3^T K^, g2 = V'^T u: token-split partials
    WgArgs a = wg_args();
    const int tiles = (mm / 256) * (dd / 256);
    const int kblocks = (int)((T + 63) / 64);
    S = std::max(1, std::min({w.s_max, kblocks, (sm_count() / 2 * 4 + 3 * H * tiles - 1) / (3 * H * tiles)}));
    a.M = std::max(mm, dd);
    a.mt = mm / 256;
    a.nt = dd / 256;
    a.nt2 = mm / 256;
    a.nmat = 3;
    a.heads = H;
    a.S = S;
    a.kblocks = kblocks;
    a.a_head = mm;
    a.b_head = dd;
    a.mat2_a_head = dd;
    a.mat2_b_head = mm;
    a.m = mm;
    a.d = dd;
    a.out = w.partial;
    a.eta_part = w.etapart;
    a.idesc = idesc_f16(256, 256, true, true);
    TTT_TRY((launch_wgemm<WG_PARTIAL, true, true>(tD1, tD3, tVm, tKm, tU, a, S * 3 * H * tiles, w, s)));
  }
  k_reduce_splits<<<grid1d(3 * n / 4, 256), 256, 0, s>>>(w.partial, S, 3 * n, G, accumulate ? 1 : 0, w.status);
  TTT_LAUNCHED();
  return TTT_OK;
}

// Apply of the wide path: P = SiLU(r Q W1^T) o (r Q W3^T) (bf16, in the dH1 buffer), O = P W2^T.
int run_apply_wide(const void* Q, int64_t ldq, void* O, int64_t ldo, int qnorm, float* rq_buf, int64_t T,
                   const ttt_dims& d, const Ws& w, cudaStream_t s) {
  const int H = d.heads, dd = d.d, mm = d.m;
  const uint64_t hd = (uint64_t)H * dd, hm = (uint64_t)H * mm;
  if (qnorm) TTT_TRY(launch_rownorm_any(Q, ldq, T, d, TTT_BF16, rq_buf, s));
  __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(w.dh1);
  CUtensorMap tQ, tW, tP, tW2;
  if (!tmap_k(&tQ, Q, hd, (uint64_t)T, (uint64_t)ldq, false) ||
      !tmap_k(&tW, w.wsh, (uint64_t)dd, 3ull * H * mm, (uint64_t)dd, false) ||
      !tmap_k(&tP, P, hm, (uint64_t)T, hm, false) || !tmap_k(&tW2, w.w2b, (uint64_t)mm, hd, (uint64_t)mm, false))
    return TTT_ERR_CUDA;
  const int mt = (int)((T + 255) / 256);
  ProfScope ps(TTT_PROF_APPLY, s);
  {
    WgArgs a = wg_args();
    a.M = (int)T;
    a.mt = mt;
    a.nt = mm / 128;
    a.heads = H;
    a.kblocks = dd / 64;
    a.a_head = dd;
    a.b_row0 = 0;
    a.b_head = mm;
    a.b_row1 = H * mm;
    a.m = mm;
    a.d = dd;
    a.out = P;
    a.ldo = (int64_t)hm;
    a.rvec = qnorm ? rq_buf : nullptr;
    a.idesc = idesc_bf16(256, 256, false, false);
    TTT_TRY((launch_wgemm<WG_SWIGLU_FWD, false, false>(tQ, tQ, tQ, tW, tW, a, mt * a.nt * H, w, s)));
  }
  {
    WgArgs a = wg_args();
    a.M = (int)T;
    a.mt = mt;
    a.nt = dd / 256;
    a.heads = H;
    a.kblocks = mm / 64;
    a.a_head = mm;
    a.b_row0 = 0;
    a.b_head = dd;
    a.out_head = dd;
    a.out = O;
    a.ldo = ldo;
    a.idesc = idesc_bf16(256, 256, false, false);
    TTT_TRY((launch_wgemm<WG_STORE_BF16, false, false>(tP, tP, tP, tW2, tW2, a, mt * a.nt * H, w, s)));
  }
  return TTT_OK;
}

// gradient over T tokens -> G (fp32, [3][H*m*d]); shadow of W must be current.
// bf16 mode: K, V are the fp16 operands K^, V' of prepare_update_operands (ld = H*d)
// and w.etapart holds the |eta| maxima of these T tokens; qk is not read there
// (K^ is already normalised).  accumulate = true adds the gradient to G instead
// of overwriting it.
int run_grad(const ttt_weights& W, const void* K, int64_t ldk, const void* V, int64_t ldv, const float* eta,
             const float* rk, int qk, int64_t T, const ttt_dims& d, ttt_dtype dt, const Ws& w, float* G,
             cudaStream_t s, bool accumulate = false) {
  const int64_t n = (int64_t)d.heads * d.m * d.d;
  if (T == 0) {
    if (!accumulate) TTT_CHECK(cudaMemsetAsync(G, 0, 3 * n * sizeof(float), s));
    return TTT_OK;
  }
  (void)qk;
  if (dt == TTT_BF16 && wide_dims(d)) return run_grad_wide(K, V, T, d, w, G, s, accumulate);
  int S = 1;
  if (dt == TTT_BF16) {
    const int tiles = (int)((T + TC_TILE - 1) / TC_TILE);
    const int slices = d.m / TC_MS;
    S = std::max(1, std::min({sm_count() / std::max(1, slices * d.heads), w.s_max, tiles}));
    CUtensorMap tK, tV, tKb, tVb, tW;
    const uint64_t hd = (uint64_t)d.heads * d.d;
    const CUtensorMapDataType F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!tmap_bf16(&tK, K, hd, (uint64_t)T, (uint64_t)ldk * 2, 64, TC_TILE, F16)) return TTT_ERR_CUDA;
    if (!tmap_bf16(&tV, V, hd, (uint64_t)T, (uint64_t)ldv * 2, 64, TC_TILE, F16)) return TTT_ERR_CUDA;
    if (!tmap_bf16(&tKb, K, hd, (uint64_t)T, (uint64_t)ldk * 2, 64, UpdLayout<192>::BCH, F16)) return TTT_ERR_CUDA;
    if (!tmap_bf16(&tVb, V, hd, (uint64_t)T, (uint64_t)ldv * 2, 64, UpdLayout<192>::BCH, F16)) return TTT_ERR_CUDA;
    if (!tmap_bf16(&tW, w.wsh16, (uint64_t)d.d, 3ull * d.heads * d.m, (uint64_t)d.d * 2, 64, 64, F16))
      return TTT_ERR_CUDA;
    dim3 grid(slices, d.heads, S);
    ProfScope ps(TTT_PROF_GRAD, s);
    if (d.d == 192) {
      auto k = k_update_grad_tc<192>;
      TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, UpdLayout<192>::ALLOC));
      k<<<grid, UPD_THREADS, UpdLayout<192>::ALLOC, s>>>(tK, tV, tKb, tVb, tW, w.etapart, w.partial, T, d.heads,
                                                          d.m, tiles, S, w.status, wait_timeout_ns());
    } else {
      auto k = k_update_grad_tc<128>;
      TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, UpdLayout<128>::ALLOC));
      k<<<grid, UPD_THREADS, UpdLayout<128>::ALLOC, s>>>(tK, tV, tKb, tVb, tW, w.etapart, w.partial, T, d.heads,
                                                          d.m, tiles, S, w.status, wait_timeout_ns());
    }
    TTT_LAUNCHED();
  } else {
    const int tiles = (int)((T + F32_TT - 1) / F32_TT);
    const int slices = d.m / F32_MS;
    S = std::max(1, std::min({2 * sm_count() / std::max(1, slices * d.heads), w.s_max, tiles}));
    const size_t smem =
        (size_t)(3 * F32_MS * d.d + 2 * F32_TT * d.d + 3 * F32_TT * F32_MS + 2 * F32_TT) * sizeof(float);
    TTT_CHECK(cudaFuncSetAttribute(k_grad_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    ProfScope ps(TTT_PROF_GRAD, s);
    k_grad_f32<<<dim3(slices, d.heads, S), 256, smem, s>>>((const float*)K, ldk, (const float*)V, ldv, eta, rk, W.W1,
                                                           W.W3, W.W2, w.partial, T, d.heads, d.d, d.m, S);
    TTT_LAUNCHED();
  }
  ProfScope ps(TTT_PROF_REDUCE, s);
  k_reduce_splits<<<grid1d(3 * n / 4, 256), 256, 0, s>>>(w.partial, S, 3 * n, G, accumulate ? 1 : 0, w.status);
  TTT_LAUNCHED();
  return TTT_OK;
}

// Newton-Schulz + weight step from G; refreshes the bf16 shadow in bf16 mode.
// W <- ||W|| (W - lr D) / ||W - lr D|| with D given in W's orientation (Dw for wide, Dt for tall matrices)
int run_step_update(const ttt_weights& W, const float* Dw, const float* Dt, const ttt_ns_cfg& ns, const ttt_dims& d,
                    const Ws& w, cudaStream_t s) {
  const int H = d.heads, mm = d.m, dd = d.d, nb = 3 * H;
  const int64_t n = (int64_t)mm * dd;
  TTT_TRY(launch_pdl(k_step_partials, dim3(nb, NORM_PARTS), dim3(256), 0, s, W.W1, W.W3, W.W2, Dw, Dt, H, dd, mm,
                     ns.lr, w.stepn));
  return launch_pdl(k_step_apply, dim3(grid1d(n / 4, 256) / nb + 1, nb), dim3(256), 0, s, W.W1, W.W3, W.W2, Dw, Dt, H,
                    dd, mm, ns.lr, ns.renorm, (const float*)w.stepn, (const unsigned int*)w.status);
}

// C = alpha A B + beta Cin on the tensor cores (split bf16 parts); see kernels_nsmma.cuh
template <int NT, bool BK>
int launch_mm3(int M, int N, int K, int ksplit, int nsplit, int batch, const float* A, int lda, int64_t sA,
               const float* B, int ldb, int64_t sB, float* C, int ldc, int64_t sC, int64_t sCsplit, const float* Cin,
               float alpha, float beta, const Ws& w, cudaStream_t s) {
  auto k = k_mm3<NT, BK>;
  TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, NsmLayout<NT>::ALLOC));
  const dim3 grid((N + NT - 1) / NT, (M + 127) / 128, batch * nsplit);
  return launch_pdl(k, grid, dim3(NSM_THREADS), NsmLayout<NT>::ALLOC, s, M, N, K, ksplit, nsplit, A, lda, sA, B, ldb,
                    sB, C, ldc, sC, sCsplit, Cin, alpha, beta, w.status, wait_timeout_ns());
}

// the r x r products (Gram split-K, A A): N tile = r rounded up to 64
template <bool BK>
int launch_mm3_r(int r, int K, int ksplit, int nsplit, int batch, const float* A, int lda, int64_t sA, const float* B,
                 int ldb, int64_t sB, float* C, int64_t sC, int64_t sCsplit, const float* Cin, float alpha, float beta,
                 const Ws& w, cudaStream_t s) {
  if (r <= 64)
    return launch_mm3<64, BK>(r, r, K, ksplit, nsplit, batch, A, lda, sA, B, ldb, sB, C, r, sC, sCsplit, Cin, alpha,
                              beta, w, s);
  if (r <= 128)
    return launch_mm3<128, BK>(r, r, K, ksplit, nsplit, batch, A, lda, sA, B, ldb, sB, C, r, sC, sCsplit, Cin, alpha,
                               beta, w, s);
  if (r <= 192)
    return launch_mm3<192, BK>(r, r, K, ksplit, nsplit, batch, A, lda, sA, B, ldb, sB, C, r, sC, sCsplit, Cin, alpha,
                               beta, w, s);
  // wide heads: 128 x 128 tiles over the r x r product
  return launch_mm3<128, BK>(r, r, K, ksplit, nsplit, batch, A, lda, sA, B, ldb, sB, C, r, sC, sCsplit, Cin, alpha,
                             beta, w, s);
}

// Newton-Schulz iterations of the bf16 path on the tensor cores: X (r x c) -> X
// after `iters` steps, then XT = X^T.  Products carry ~2^-16 relative error.
int run_ns_iters_tc(const ttt_ns_cfg& ns, int r, int c, int nb, const Ws& w, float*& X, float*& X2, cudaStream_t s) {
  const int64_t n = (int64_t)r * c, rr = (int64_t)r * r;
  // Gram split-K: slices of >= 128 columns, at most NSM_GRAM_SPLIT_MAX of them
  const int ksplit = std::max(128, ((c + NSM_GRAM_SPLIT_MAX - 1) / NSM_GRAM_SPLIT_MAX + 63) / 64 * 64);
  const int nsplit = (c + ksplit - 1) / ksplit;
  for (int it = 0; it < ns.iters; ++it) {
    // Gram partials P[s][b] = X_b[:, split s] X_b[:, split s]^T (B^T rows = X rows)
    TTT_TRY(launch_mm3_r<true>(r, c, ksplit, nsplit, nb, X, c, n, X, c, n, w.gram, rr, (int64_t)nb * rr, nullptr, 1.f,
                               0.f, w, s));
    TTT_TRY(launch_pdl(k_gram_reduce, dim3(grid1d((int64_t)nb * rr, 256)), dim3(256), 0, s, r, nb, nsplit,
                       (const float*)w.gram, w.A));
    // B = c A A + b A (A symmetric: its rows serve as B^T rows)
    TTT_TRY(launch_mm3_r<true>(r, r, r, 1, nb, w.A, r, rr, w.A, r, rr, w.B, rr, 0, w.A, ns.c, ns.b, w, s));
    // X' = B X + a X (B rows of X: MN-major), 128-column tiles
    TTT_TRY((launch_mm3<128, false>(r, c, r, r, 1, nb, w.B, r, rr, X, c, n, X2, c, n, 0, X, 1.f, ns.a, w, s)));
    std::swap(X, X2);
  }
  return TTT_OK;
}

// One launch for all Newton-Schulz iterations of the bf16 path: a cluster of
// c / 128 CTAs per matrix (k_ns_cluster), X updated in place.  Usable when
// r is 128 or 192, c is a multiple of 128 with at most 8 column blocks, and
// such a cluster fits on the device.
template <int R>
int ns_cluster_launch(int c, int nb, const ttt_ns_cfg& ns, const Ws& w, cudaStream_t s, bool probe_only,
                      bool* fits) {
  auto k = k_ns_cluster<R>;
  TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, NscLayout<R>::ALLOC));
  const int cs = c / NSC_COLS;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, nb);
  cfg.blockDim = dim3(NSC_THREADS);
  cfg.dynamicSmemBytes = NscLayout<R>::ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  if (probe_only) {
    int n = 0;
    cfg.numAttrs = 1;
    *fits = cudaOccupancyMaxActiveClusters(&n, k, &cfg) == cudaSuccess && n >= 1;
    (void)cudaGetLastError();
    return TTT_OK;
  }
  TTT_CHECK(cudaLaunchKernelEx(&cfg, k, w.X, w.A, c, ns.iters, ns.a, ns.b, ns.c, w.status, wait_timeout_ns()));
  return TTT_OK;
}

bool ns_cluster_usable(int r, int c) {
  if ((r != 128 && r != 192) || c % NSC_COLS || c / NSC_COLS < 1 || c / NSC_COLS > 8) return false;
  static std::atomic<int> cache[2][9] = {};  // 0 unknown, 1 fits, 2 does not
  std::atomic<int>& e = cache[r == 192][c / NSC_COLS];
  if (e.load() == 0) {
    bool fits = false;
    const Ws none{};
    const int rc = r == 192 ? ns_cluster_launch<192>(c, 1, ttt_ns_cfg{}, none, nullptr, true, &fits)
                            : ns_cluster_launch<128>(c, 1, ttt_ns_cfg{}, none, nullptr, true, &fits);
    e.store(rc == TTT_OK && fits ? 1 : 2);
  }
  return e.load() == 1;
}

int run_ns_step(const ttt_weights& W, const float* G, const ttt_ns_cfg& ns, const ttt_dims& d, ttt_dtype dt,
                const Ws& w, cudaStream_t s) {
  const int H = d.heads, mm = d.m, dd = d.d;
  const int64_t n = (int64_t)mm * dd;
  const int nb = 3 * H;
  const int r = std::min(mm, dd), c = std::max(mm, dd);
  const float* Dw = G;
  const float* Dt = G;
  ProfScope ps(TTT_PROF_NS, s);
  if (ns.iters > 0) {
    k_frob_partials<<<dim3(nb, NORM_PARTS), 256, 0, s>>>(G, n, w.norms);
    TTT_LAUNCHED();
    TTT_TRY(launch_pdl(k_ns_init, dim3((c + 31) / 32, (c + 31) / 32, nb), dim3(32, 8), 0, s, G, w.X,
                       dt == TTT_BF16 ? (float*)nullptr : w.XT, (const float*)w.norms, H, dd, mm, ns.eps));
    float *X = w.X, *X2 = w.X2, *XT = w.XT, *XT2 = w.XT2;
    if (dt == TTT_BF16) {
      if (ns_cluster_usable(r, c)) {
        bool unused = false;
        TTT_TRY(r == 192 ? ns_cluster_launch<192>(c, nb, ns, w, s, false, &unused)
                         : ns_cluster_launch<128>(c, nb, ns, w, s, false, &unused));
      } else if (wide_dims(d)) {
        TTT_TRY(run_ns_iters_wide(ns, r, c, nb, w, X, X2, s));
      } else {
        TTT_TRY(run_ns_iters_tc(ns, r, c, nb, w, X, X2, s));
      }
      TTT_TRY(launch_pdl(k_transpose_batch, dim3((c + 31) / 32, (r + 31) / 32, nb), dim3(32, 8), 0, s,
                         (const float*)X, XT, r, c, n));
      return run_step_update(W, X, XT, ns, d, w, s);
    }
    const int rt = (r + 63) / 64, ct = (c + 63) / 64;
    TTT_CHECK(cudaFuncSetAttribute(k_gram_partial, cudaFuncAttributeMaxDynamicSharedMemorySize, NSC_DYN_BYTES));
    TTT_CHECK(cudaFuncSetAttribute(k_gemm_sym, cudaFuncAttributeMaxDynamicSharedMemorySize, NSC_DYN_BYTES));
    const int64_t rr = (int64_t)r * r;
    for (int it = 0; it < ns.iters; ++it) {
      // A = X X^T (from X^T), B = b A + c A A, X' = a X + B X (and X'^T)
      k_gram_partial<<<dim3(rt * (rt + 1) / 2, NS_GRAM_SPLIT, nb), 256, NSC_DYN_BYTES, s>>>(r, c, XT, n, w.gram);
      TTT_LAUNCHED();
      k_gram_reduce<<<grid1d((int64_t)nb * rr, 256), 256, 0, s>>>(r, nb, NS_GRAM_SPLIT, w.gram, w.A);
      TTT_LAUNCHED();
      k_gemm_sym<<<dim3(rt, rt, nb), 256, NSC_DYN_BYTES, s>>>(r, r, w.A, rr, w.A, r, rr, w.B, r, rr, nullptr, w.A,
                                                               ns.c, ns.b);
      TTT_LAUNCHED();
      k_gemm_sym<<<dim3(ct, rt, nb), 256, NSC_DYN_BYTES, s>>>(r, c, w.B, rr, X, c, n, X2, c, n, XT2, X, 1.f, ns.a);
      TTT_LAUNCHED();
      std::swap(X, X2);
      std::swap(XT, XT2);
    }
    Dw = X;
    Dt = XT;
  }
  return run_step_update(W, Dw, Dt, ns, d, w, s);
}

int run_step(const ttt_weights& W, const float* G, const ttt_ns_cfg& ns, const ttt_dims& d, ttt_dtype dt, const Ws& w,
             cudaStream_t s) {
  TTT_TRY(run_ns_step(W, G, ns, d, dt, w, s));
  if (dt == TTT_BF16) TTT_TRY(launch_shadow(W, w, d, s, true));
  return TTT_OK;
}

// Apply to T tokens.  qnorm: L2-normalise the queries per head (the tensor-core
// kernel computes the norms from its query tile; the fp32 path writes them to
// rq_buf [T][H] first).
int run_apply(const ttt_weights& W, const void* Q, int64_t ldq, void* O, int64_t ldo, int qnorm, float* rq_buf,
              int64_t T, const ttt_dims& d, ttt_dtype dt, const Ws& w, cudaStream_t s) {
  if (T == 0) return TTT_OK;
  if (dt == TTT_BF16 && wide_dims(d)) return run_apply_wide(Q, ldq, O, ldo, qnorm, rq_buf, T, d, w, s);
  if (dt == TTT_BF16) {
    const int pair_tiles = (int)((T + 2 * TC_TILE - 1) / (2 * TC_TILE));
    const int n_items = pair_tiles * d.heads;
    CUtensorMap tQ, tW, tW2, tO;
    const uint64_t hd = (uint64_t)d.heads * d.d;
    if (!tmap_bf16(&tQ, Q, hd, (uint64_t)T, (uint64_t)ldq * 2, 64, TC_TILE)) return TTT_ERR_CUDA;
    // output: [32 tokens x 32 columns] store boxes from 64-byte-swizzled staging tiles
    if (!tmap_bf16(&tO, O, hd, (uint64_t)T, (uint64_t)ldo * 2, 32, 32, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   CU_TENSOR_MAP_SWIZZLE_64B))
      return TTT_ERR_CUDA;
    if (!tmap_bf16(&tW, w.wsh, (uint64_t)d.d, 3ull * d.heads * d.m, (uint64_t)d.d * 2, 64, 64)) return TTT_ERR_CUDA;
    if (!tmap_bf16(&tW2, w.w2b, (uint64_t)d.m, (uint64_t)d.heads * d.d, (uint64_t)d.m * 2, 64, (uint32_t)d.d / 2))
      return TTT_ERR_CUDA;
    const int npairs = std::max(1, std::min(n_items, sm_count() / 2));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * npairs);
    cfg.blockDim = dim3(AP_THREADS);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ProfScope ps(TTT_PROF_APPLY, s);
    const unsigned long long to = wait_timeout_ns();
    if (d.d == 192) {
      auto k = k_apply_tc<192>;
      TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, ApLayout<192>::ALLOC));
      cfg.dynamicSmemBytes = ApLayout<192>::ALLOC;
      TTT_CHECK(cudaLaunchKernelEx(&cfg, k, tQ, tW, tW2, tO, qnorm, T, d.heads, d.m, n_items, w.status, to));
    } else {
      auto k = k_apply_tc<128>;
      TTT_CHECK(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, ApLayout<128>::ALLOC));
      cfg.dynamicSmemBytes = ApLayout<128>::ALLOC;
      TTT_CHECK(cudaLaunchKernelEx(&cfg, k, tQ, tW, tW2, tO, qnorm, T, d.heads, d.m, n_items, w.status, to));
    }
    TTT_LAUNCHED();
  } else {
    const float* rq = nullptr;
    if (qnorm) {
      TTT_TRY(launch_rownorm_any(Q, ldq, T, d, dt, rq_buf, s));
      rq = rq_buf;
    }
    const size_t smem = (size_t)(F32_TT * d.d + 2 * F32_MS * d.d + d.d * F32_MS + F32_TT * F32_MS + F32_TT) * 4;
    TTT_CHECK(cudaFuncSetAttribute(k_apply_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    ProfScope ps(TTT_PROF_APPLY, s);
    k_apply_f32<<<dim3((unsigned)((T + F32_TT - 1) / F32_TT), d.heads), 256, smem, s>>>(
        (const float*)Q, ldq, rq, W.W1, W.W3, W.W2, (float*)O, ldo, T, d.heads, d.d, d.m);
    TTT_LAUNCHED();
  }
  return TTT_OK;
}

int check_ns(const ttt_ns_cfg* ns) {
  if (!ns || ns->iters < 0 || ns->iters > 64 || !(ns->eps >= 0.f)) return TTT_ERR_INVALID;
  return TTT_OK;
}

const ttt_io_cfg kDefaultIo = {1, 0, 0, 0, 0};

// ---- scratch of ttt_apply_noalloc: one fixed array in device memory, no allocation.
// Host code only ever holds its per-device address from cudaGetSymbolAddress;
// the symbol itself names a host-side shadow and is never passed to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[TTT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {nullptr};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
int noalloc_scratch(void** out) {
  int dev = 0;
  TTT_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return TTT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    TTT_CHECK(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (!p) return TTT_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return TTT_OK;
}

// ---- host-buffer layer (ttt_layer_host): two copy streams and a pool of
// events per device, created on first use and kept for the process lifetime
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> ev;
};
std::mutex g_pipe_mu;  // held while a call queues its work (the events are shared)
HostPipe g_pipes[64];
constexpr int kHostBlocks = 16;  // token blocks of the bidirectional host pipeline

int host_pipe(HostPipe** out, size_t n_events) {
  int dev = 0;
  TTT_CHECK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return TTT_ERR_CUDA;
  HostPipe& p = g_pipes[dev];
  if (!p.h2d) TTT_CHECK(cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking));
  if (!p.d2h) TTT_CHECK(cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking));
  while (p.ev.size() < n_events) {
    cudaEvent_t e;
    TTT_CHECK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    p.ev.push_back(e);
  }
  *out = &p;
  return TTT_OK;
}

// dbuf layout: Q, K, V, O [T][H*d], eta [T][H], then V after ShortConv2D (conv)
struct HostLayout {
  size_t q, k, v, o, eta, vc, total;
};
HostLayout host_layout(const ttt_dims& d, int64_t T, ttt_dtype dt, bool conv) {
  const size_t tm = up256((size_t)std::max<int64_t>(T, 1) * d.heads * d.d * esize(dt));
  HostLayout L{};
  L.q = 0;
  L.k = tm;
  L.v = 2 * tm;
  L.o = 3 * tm;
  L.eta = 4 * tm;
  L.vc = L.eta + up256((size_t)std::max<int64_t>(T, 1) * d.heads * 4);
  L.total = L.vc + (conv ? tm : 0);
  return L;
}

int launch_conv(const void* V, void* Vout, const float* taps, int64_t frames, int gh, int gw, int C, ttt_dtype dt,
                cudaStream_t s) {
  return launch_conv_any(V, C, Vout, C, taps, frames, gh, gw, C, 0, dt, s);
}

}  // namespace

extern "C" {

size_t ttt_workspace_bytes(ttt_dims dims, int64_t T, ttt_dtype dtype) {
  if (!dims_ok(dims) || T < 0 || (dtype != TTT_FP32 && dtype != TTT_BF16)) return 0;
  return carve(nullptr, dims, T, dtype).total;
}

int ttt_reset_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return TTT_ERR_WORKSPACE;
  TTT_CHECK(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
  return TTT_OK;
}

int ttt_poll_status(const void* ws, void* stream) {
  if (!ws) return TTT_ERR_WORKSPACE;
  TTT_CHECK(cudaStreamSynchronize((cudaStream_t)stream));
  unsigned int v = 0;
  TTT_CHECK(cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost));
  if (v == DEV_OK) return TTT_OK;
  return v == DEV_RANGE ? TTT_ERR_RANGE : TTT_ERR_TIMEOUT;
}

int ttt_l2norm(void* X, int64_t T, ttt_dims dims, int64_t ld, ttt_dtype dtype, void* stream) {
  if ((dtype != TTT_FP32 && dtype != TTT_BF16) || !dims_ok(dims) || T < 0) return TTT_ERR_INVALID;
  if (dims.d % (dtype == TTT_BF16 ? 8 : 4)) return TTT_ERR_UNSUPPORTED;
  ld = eff_ld(ld, dims);
  TTT_TRY(check_tokens(X, ld, dims, dtype, T));
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == TTT_BF16) return launch_rownorm<__nv_bfloat16>((__nv_bfloat16*)X, ld, T, dims, nullptr, 1, s);
  return launch_rownorm<float>((float*)X, ld, T, dims, nullptr, 1, s);
}

int ttt_shortconv2d(const void* V, int64_t ld_v, void* Vout, int64_t ld_out, const float* taps, int N, int h, int w,
                    int C, int act, ttt_dtype dtype, void* stream) {
  if (dtype != TTT_FP32 && dtype != TTT_BF16) return TTT_ERR_INVALID;
  if (N < 0 || h < 1 || w < 1 || C < 1 || (act != 0 && act != 1)) return TTT_ERR_INVALID;
  if (C % 8) return TTT_ERR_UNSUPPORTED;
  if (ld_v == 0) ld_v = C;
  if (ld_out == 0) ld_out = C;
  if (ld_v < C || ld_out < C) return TTT_ERR_INVALID;
  if (N == 0) return TTT_OK;
  if (!V || !Vout || !taps || V == Vout) return TTT_ERR_INVALID;
  if (!aligned16(V) || !aligned16(Vout) || (ld_v * (int64_t)esize(dtype)) % 16 || (ld_out * (int64_t)esize(dtype)) % 16)
    return TTT_ERR_ALIGN;
  return launch_conv_any(V, ld_v, Vout, ld_out, taps, N, h, w, C, act, dtype, (cudaStream_t)stream);
}

int ttt_grad(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, ttt_dims dims,
             const ttt_io_cfg* io, ttt_dtype dtype, float* G, void* ws, size_t ws_bytes, void* stream) {
  TTT_TRY(check_common(dims, dtype, T, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  if (!io) io = &kDefaultIo;
  const int64_t ldk = eff_ld(io->ld_k, dims), ldv = eff_ld(io->ld_v, dims);
  TTT_TRY(check_tokens(K, ldk, dims, dtype, T));
  TTT_TRY(check_tokens(V, ldv, dims, dtype, T));
  if (!G) return TTT_ERR_INVALID;
  if (!aligned16(G)) return TTT_ERR_ALIGN;
  if (T > 0 && !eta) return TTT_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, T, dtype);
  UpdOperands op;
  TTT_TRY(prepare_update_operands(K, ldk, V, ldv, eta, T, dims, dtype, io->qk_l2norm, w, s, &op));
  if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
  return run_grad(W, op.K, op.ldk, op.V, op.ldv, eta, op.rk, io->qk_l2norm, T, dims, dtype, w, G, s);
}

int ttt_grad_prepared(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, ttt_dims dims,
                      const ttt_io_cfg* io, ttt_dtype dtype, float* G, void* ws, size_t ws_bytes, void* stream) {
  TTT_TRY(check_common(dims, dtype, T, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  if (!io) io = &kDefaultIo;
  const int64_t ldk = eff_ld(io->ld_k, dims), ldv = eff_ld(io->ld_v, dims);
  TTT_TRY(check_tokens(K, ldk, dims, dtype, T));
  TTT_TRY(check_tokens(V, ldv, dims, dtype, T));
  if (!G) return TTT_ERR_INVALID;
  if (!aligned16(G)) return TTT_ERR_ALIGN;
  if (T > 0 && !eta) return TTT_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, T, dtype);
  UpdOperands op;
  if (dtype == TTT_BF16) {
    const int64_t hd = (int64_t)dims.heads * dims.d;
    op = {w.kh16, hd, w.vh16, hd, nullptr};
    TTT_TRY(launch_shadow(W, w, dims, s));
  } else {
    op = {K, ldk, V, ldv, io->qk_l2norm && T > 0 ? w.rk : nullptr};
  }
  return run_grad(W, op.K, op.ldk, op.V, op.ldv, eta, op.rk, io->qk_l2norm, T, dims, dtype, w, G, s);
}

int ttt_step(ttt_weights W, const float* G, const ttt_ns_cfg* ns, ttt_dims dims, ttt_dtype dtype, void* ws,
             size_t ws_bytes, void* stream) {
  TTT_TRY(check_common(dims, dtype, 0, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  TTT_TRY(check_ns(ns));
  if (!G) return TTT_ERR_INVALID;
  Ws w = carve(ws, dims, 0, dtype);
  return run_step(W, G, *ns, dims, dtype, w, (cudaStream_t)stream);
}

int ttt_update(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, int steps,
               const ttt_ns_cfg* ns, ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype, void* ws, size_t ws_bytes,
               void* stream) {
  TTT_TRY(check_common(dims, dtype, T, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  TTT_TRY(check_ns(ns));
  if (steps < 0) return TTT_ERR_INVALID;
  if (!io) io = &kDefaultIo;
  const int64_t ldk = eff_ld(io->ld_k, dims), ldv = eff_ld(io->ld_v, dims);
  TTT_TRY(check_tokens(K, ldk, dims, dtype, T));
  TTT_TRY(check_tokens(V, ldv, dims, dtype, T));
  if (T > 0 && !eta) return TTT_ERR_INVALID;
  if (T == 0 || steps == 0) return TTT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, T, dtype);
  UpdOperands op;
  TTT_TRY(prepare_update_operands(K, ldk, V, ldv, eta, T, dims, dtype, io->qk_l2norm, w, s, &op));
  if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
  for (int st = 0; st < steps; ++st) {
    TTT_TRY(run_grad(W, op.K, op.ldk, op.V, op.ldv, eta, op.rk, io->qk_l2norm, T, dims, dtype, w, w.G, s));
    TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
  }
  return TTT_OK;
}

int ttt_update_conv(ttt_weights W, const void* K, const void* V, const float* eta, int64_t T, int steps,
                    const ttt_ns_cfg* ns, const float* taps, int grid_h, int grid_w, int act, ttt_dims dims,
                    const ttt_io_cfg* io, ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  TTT_TRY(check_common(dims, dtype, T, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  TTT_TRY(check_ns(ns));
  if (steps < 0 || grid_h < 1 || grid_w < 1 || (act != 0 && act != 1)) return TTT_ERR_INVALID;
  if (T % ((int64_t)grid_h * grid_w)) return TTT_ERR_INVALID;
  if (dtype != TTT_BF16) return TTT_ERR_UNSUPPORTED;
  if (!io) io = &kDefaultIo;
  const int64_t ldk = eff_ld(io->ld_k, dims), ldv = eff_ld(io->ld_v, dims);
  TTT_TRY(check_tokens(K, ldk, dims, dtype, T));
  TTT_TRY(check_tokens(V, ldv, dims, dtype, T));
  if (T > 0 && (!eta || !taps)) return TTT_ERR_INVALID;
  if (T == 0 || steps == 0) return TTT_OK;
  if (conv2_band_rows(grid_h, grid_w) < 1 || dims.d % CONV_GROUP) return TTT_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, T, dtype);
  TTT_TRY(launch_eta_absmax(eta, T, dims, w, s));
  TTT_TRY(launch_conv_prep(K, ldk, V, ldv, taps, T / ((int64_t)grid_h * grid_w), grid_h, grid_w, act, eta,
                           io->qk_l2norm, dims, w, s));
  TTT_TRY(launch_shadow(W, w, dims, s));
  const int64_t hd = (int64_t)dims.heads * dims.d;
  for (int st = 0; st < steps; ++st) {
    TTT_TRY(run_grad(W, w.kh16, hd, w.vh16, hd, eta, nullptr, io->qk_l2norm, T, dims, dtype, w, w.G, s));
    TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
  }
  return TTT_OK;
}

int ttt_apply(ttt_weights W, const void* Q, void* O, int64_t T, ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype,
              void* ws, size_t ws_bytes, void* stream) {
  TTT_TRY(check_common(dims, dtype, T, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  if (!io) io = &kDefaultIo;
  const int64_t ldq = eff_ld(io->ld_q, dims), ldo = eff_ld(io->ld_o, dims);
  TTT_TRY(check_tokens(Q, ldq, dims, dtype, T));
  TTT_TRY(check_tokens(O, ldo, dims, dtype, T));
  if (T > 0 && Q == O) return TTT_ERR_INVALID;
  if (T == 0) return TTT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, T, dtype);
  if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
  return run_apply(W, Q, ldq, O, ldo, io->qk_l2norm, w.rq, T, dims, dtype, w, s);
}

int ttt_apply_noalloc(ttt_weights W, const void* Q, void* O, int64_t T, ttt_dims dims, const ttt_io_cfg* io,
                      ttt_dtype dtype, void* stream) {
  if (dtype != TTT_FP32 && dtype != TTT_BF16) return TTT_ERR_INVALID;
  if (!dims_ok(dims) || T < 0) return TTT_ERR_INVALID;
  TTT_TRY(dims_supported(dims, dtype));
  TTT_TRY(check_weights(W));
  if (!io) io = &kDefaultIo;
  const int64_t ldq = eff_ld(io->ld_q, dims), ldo = eff_ld(io->ld_o, dims);
  TTT_TRY(check_tokens(Q, ldq, dims, dtype, T));
  TTT_TRY(check_tokens(O, ldo, dims, dtype, T));
  if (T > 0 && Q == O) return TTT_ERR_INVALID;
  // the wide-head apply needs a per-token intermediate that this fixed scratch does not hold
  if (dtype == TTT_BF16 && wide_dims(dims)) return TTT_ERR_UNSUPPORTED;
  // scratch plan: [status 256 B | W1,W3,W2^T bf16 | W2 bf16 | per-token inverse norms of one token chunk]
  const size_t n = (size_t)dims.heads * dims.m * dims.d;
  const size_t fixed = 256 + up256(3 * n * 2) + up256(n * 2);
  if (fixed >= TTT_NOALLOC_SCRATCH_BYTES) return TTT_ERR_SCRATCH;
  const int64_t per_tok = (int64_t)dims.heads * 4;
  const int64_t chunk = ((int64_t)(TTT_NOALLOC_SCRATCH_BYTES - fixed) / per_tok) / TC_TILE * TC_TILE;
  if (chunk < TC_TILE) return TTT_ERR_SCRATCH;
  if (T == 0) return TTT_OK;
  void* base = nullptr;
  TTT_TRY(noalloc_scratch(&base));
  uint8_t* b = static_cast<uint8_t*>(base);
  Ws w{};
  w.status = reinterpret_cast<unsigned int*>(b);
  w.wsh = reinterpret_cast<__nv_bfloat16*>(b + 256);
  w.w2b = reinterpret_cast<__nv_bfloat16*>(b + 256 + up256(3 * n * 2));
  float* rq_buf = reinterpret_cast<float*>(b + fixed);
  cudaStream_t s = (cudaStream_t)stream;
  TTT_CHECK(cudaMemsetAsync(w.status, 0, 256, s));
  if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
  const size_t es = esize(dtype);
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const int64_t tc = std::min(chunk, T - c0);
    const uint8_t* q = static_cast<const uint8_t*>(Q) + c0 * ldq * es;
    uint8_t* o = static_cast<uint8_t*>(O) + c0 * ldo * es;
    TTT_TRY(run_apply(W, q, ldq, o, ldo, io->qk_l2norm, rq_buf, tc, dims, dtype, w, s));
  }
  return TTT_OK;
}

int ttt_chunked(ttt_weights W, const void* Q, const void* K, const void* V, const float* eta, void* O, int64_t T,
                int64_t chunk, int order, int steps, const ttt_ns_cfg* ns, ttt_dims dims, const ttt_io_cfg* io,
                ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  if (chunk <= 0 || (order != 0 && order != 1) || steps < 0) return TTT_ERR_INVALID;
  const int64_t cmax = std::min<int64_t>(chunk, std::max<int64_t>(T, 0));
  TTT_TRY(check_common(dims, dtype, cmax, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  TTT_TRY(check_ns(ns));
  if (!io) io = &kDefaultIo;
  const int64_t ldq = eff_ld(io->ld_q, dims), ldk = eff_ld(io->ld_k, dims);
  const int64_t ldv = eff_ld(io->ld_v, dims), ldo = eff_ld(io->ld_o, dims);
  TTT_TRY(check_tokens(Q, ldq, dims, dtype, T));
  TTT_TRY(check_tokens(K, ldk, dims, dtype, T));
  TTT_TRY(check_tokens(V, ldv, dims, dtype, T));
  TTT_TRY(check_tokens(O, ldo, dims, dtype, T));
  if (T > 0 && (!eta || Q == O)) return TTT_ERR_INVALID;
  if (T == 0) return TTT_OK;
  cudaStream_t s = (cudaStream_t)stream;
  Ws w = carve(ws, dims, cmax, dtype);
  const size_t es = esize(dtype);
  if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const int64_t tc = std::min(chunk, T - c0);
    const uint8_t* q = static_cast<const uint8_t*>(Q) + c0 * ldq * es;
    const uint8_t* k = static_cast<const uint8_t*>(K) + c0 * ldk * es;
    const uint8_t* v = static_cast<const uint8_t*>(V) + c0 * ldv * es;
    uint8_t* o = static_cast<uint8_t*>(O) + c0 * ldo * es;
    const float* e = eta + c0 * dims.heads;
    UpdOperands op;
    TTT_TRY(prepare_update_operands(k, ldk, v, ldv, e, tc, dims, dtype, io->qk_l2norm, w, s, &op));
    if (order == 0) TTT_TRY(run_apply(W, q, ldq, o, ldo, io->qk_l2norm, w.rq, tc, dims, dtype, w, s));
    for (int st = 0; st < steps; ++st) {
      TTT_TRY(run_grad(W, op.K, op.ldk, op.V, op.ldv, e, op.rk, io->qk_l2norm, tc, dims, dtype, w, w.G, s));
      TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
    }
    if (order == 1) TTT_TRY(run_apply(W, q, ldq, o, ldo, io->qk_l2norm, w.rq, tc, dims, dtype, w, s));
  }
  return TTT_OK;
}

size_t ttt_host_buffer_bytes(ttt_dims dims, int64_t T, ttt_dtype dtype, int conv) {
  if (!dims_ok(dims) || T < 0 || (dtype != TTT_FP32 && dtype != TTT_BF16)) return 0;
  return host_layout(dims, T, dtype, conv != 0).total;
}

int ttt_layer_host(ttt_weights W, const void* hQ, const void* hK, const void* hV, const float* hEta, void* hO,
                   int64_t T, int64_t chunk, int order, int steps, const ttt_ns_cfg* ns, const float* taps, int grid_h,
                   int grid_w, ttt_dims dims, const ttt_io_cfg* io, ttt_dtype dtype, void* dbuf, size_t dbuf_bytes,
                   void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || chunk < 0 || steps < 0 || (order != 0 && order != 1)) return TTT_ERR_INVALID;
  const int64_t wsT = chunk > 0 ? std::min<int64_t>(chunk, T) : T;
  TTT_TRY(check_common(dims, dtype, wsT, ws, ws_bytes));
  TTT_TRY(check_weights(W));
  if (steps > 0) TTT_TRY(check_ns(ns));
  if (!io) io = &kDefaultIo;
  if (T == 0) return TTT_OK;
  if (!hQ || !hK || !hV || !hEta || !hO || !dbuf) return TTT_ERR_INVALID;
  const bool conv = taps != nullptr;
  const int64_t hd = (int64_t)dims.heads * dims.d;
  const int64_t fr = conv ? (int64_t)grid_h * grid_w : 1;
  if (conv) {
    if (grid_h < 1 || grid_w < 1 || T % fr || (chunk > 0 && chunk % fr)) return TTT_ERR_INVALID;
    if (hd % 8) return TTT_ERR_UNSUPPORTED;
  }
  const HostLayout L = host_layout(dims, T, dtype, conv);
  if (dbuf_bytes < L.total) return TTT_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(dbuf) & 255u) return TTT_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t es = esize(dtype);
  const size_t row = (size_t)hd * es;
  uint8_t* base = static_cast<uint8_t*>(dbuf);
  uint8_t* dQ = base + L.q;
  uint8_t* dK = base + L.k;
  uint8_t* dV = base + L.v;
  uint8_t* dO = base + L.o;
  uint8_t* dVc = base + L.vc;
  float* dEta = reinterpret_cast<float*>(base + L.eta);
  const uint8_t* cQ = static_cast<const uint8_t*>(hQ);
  const uint8_t* cK = static_cast<const uint8_t*>(hK);
  const uint8_t* cV = static_cast<const uint8_t*>(hV);
  uint8_t* cO = static_cast<uint8_t*>(hO);
  // token blocks: the chunks (chunk > 0), else kHostBlocks blocks of whole tiles (or frames)
  int64_t bt = chunk;
  if (chunk == 0) {
    const int64_t unit = conv ? fr : TC_TILE;
    const int64_t units = (T + unit - 1) / unit;
    bt = ((units + kHostBlocks - 1) / kHostBlocks) * unit;
  }
  const int64_t nb = (T + bt - 1) / bt;
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe* P = nullptr;
  TTT_TRY(host_pipe(&P, (size_t)(3 * nb + 3)));
  cudaEvent_t* ev = P->ev.data();
  cudaEvent_t ev_start = ev[0], ev_h2d_end = ev[1], ev_d2h_end = ev[2];
  cudaEvent_t* ev_in = ev + 3;            // [nb] K, V, eta (and Q in chunk mode) of block b on the device
  cudaEvent_t* ev_q = ev + 3 + nb;        // [nb] Q of block b on the device (chunk = 0)
  cudaEvent_t* ev_o = ev + 3 + 2 * nb;    // [nb] O of block b computed
  // the copies must not overwrite dbuf while earlier work on `stream` still uses it
  TTT_CHECK(cudaEventRecord(ev_start, s));
  TTT_CHECK(cudaStreamWaitEvent(P->h2d, ev_start, 0));
  TTT_CHECK(cudaStreamWaitEvent(P->d2h, ev_start, 0));
  auto up = [&](uint8_t* dst, const uint8_t* src, size_t bytes) {
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, P->h2d);
  };
  auto body = [&]() -> int {
    // bidirectional: all of eta first (4 H bytes per token), so the value scale of
    // the whole update is known before the first block's operands are prepared
    if (chunk == 0)
      TTT_CHECK(up(reinterpret_cast<uint8_t*>(dEta), reinterpret_cast<const uint8_t*>(hEta),
                   (size_t)T * dims.heads * 4));
    for (int64_t b = 0; b < nb; ++b) {
      const int64_t t0 = b * bt, tb = std::min(bt, T - t0);
      TTT_CHECK(up(dK + t0 * row, cK + t0 * row, tb * row));
      TTT_CHECK(up(dV + t0 * row, cV + t0 * row, tb * row));
      if (chunk > 0) {
        TTT_CHECK(up(reinterpret_cast<uint8_t*>(dEta + t0 * dims.heads),
                     reinterpret_cast<const uint8_t*>(hEta + t0 * dims.heads), (size_t)tb * dims.heads * 4));
        TTT_CHECK(up(dQ + t0 * row, cQ + t0 * row, tb * row));
      }
      TTT_CHECK(cudaEventRecord(ev_in[b], P->h2d));
    }
    if (chunk == 0)
      for (int64_t b = 0; b < nb; ++b) {
        const int64_t t0 = b * bt, tb = std::min(bt, T - t0);
        TTT_CHECK(up(dQ + t0 * row, cQ + t0 * row, tb * row));
        TTT_CHECK(cudaEventRecord(ev_q[b], P->h2d));
      }
    Ws w = carve(ws, dims, wsT, dtype);
    if (dtype == TTT_BF16) TTT_TRY(launch_shadow(W, w, dims, s));
    // V of block b after the optional ShortConv2D
    auto vsrc = [&](int64_t t0, int64_t tb) -> const uint8_t* {
      if (!conv) return dV + t0 * row;
      if (launch_conv(dV + t0 * row, dVc + t0 * row, taps, tb / fr, grid_h, grid_w, (int)hd, dtype, s) != TTT_OK)
        return nullptr;
      return dVc + t0 * row;
    };
    auto apply_block = [&](int64_t b, float* rq_buf) -> int {
      const int64_t t0 = b * bt, tb = std::min(bt, T - t0);
      TTT_TRY(run_apply(W, dQ + t0 * row, hd, dO + t0 * row, hd, io->qk_l2norm, rq_buf, tb, dims, dtype, w, s));
      TTT_CHECK(cudaEventRecord(ev_o[b], s));
      TTT_CHECK(cudaStreamWaitEvent(P->d2h, ev_o[b], 0));
      TTT_CHECK(cudaMemcpyAsync(cO + t0 * row, dO + t0 * row, tb * row, cudaMemcpyDeviceToHost, P->d2h));
      return TTT_OK;
    };
    if (chunk > 0) {
      // causal carry: order 0 O_c = f_(W_(c-1))(Q_c), then the update on chunk c;
      // order 1 the update on chunk c first, then O_c = f_(W_c)(Q_c)
      for (int64_t b = 0; b < nb; ++b) {
        const int64_t t0 = b * bt, tb = std::min(bt, T - t0);
        TTT_CHECK(cudaStreamWaitEvent(s, ev_in[b], 0));
        if (order == 0) TTT_TRY(apply_block(b, w.rq));
        if (steps > 0) {
          const uint8_t* v = vsrc(t0, tb);
          if (!v) return TTT_ERR_CUDA;
          UpdOperands op;
          TTT_TRY(prepare_update_operands(dK + t0 * row, hd, v, hd, dEta + t0 * dims.heads, tb, dims, dtype,
                                          io->qk_l2norm, w, s, &op));
          for (int st = 0; st < steps; ++st) {
            TTT_TRY(
                run_grad(W, op.K, op.ldk, op.V, op.ldv, dEta + t0 * dims.heads, op.rk, io->qk_l2norm, tb, dims, dtype, w, w.G, s));
            TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
          }
        }
        if (order == 1) TTT_TRY(apply_block(b, w.rq));
      }
      return TTT_OK;
    }
    if (steps > 0) {
      // first step: preparation and gradient block by block as the blocks land; the
      // bf16 operands of all blocks share the value scale of the whole eta
      if (dtype == TTT_BF16) {
        TTT_CHECK(cudaStreamWaitEvent(s, ev_in[0], 0));  // eta (copied first) is on the device
        TTT_TRY(launch_eta_absmax(dEta, T, dims, w, s));
      }
      for (int64_t b = 0; b < nb; ++b) {
        const int64_t t0 = b * bt, tb = std::min(bt, T - t0);
        TTT_CHECK(cudaStreamWaitEvent(s, ev_in[b], 0));
        const uint8_t* v = vsrc(t0, tb);
        if (!v) return TTT_ERR_CUDA;
        UpdOperands op;
        if (dtype == TTT_BF16) {
          TTT_TRY(launch_prep_kv(dK + t0 * row, hd, v, hd, dEta + t0 * dims.heads, tb, dims, io->qk_l2norm, w,
                                 w.kh16 + t0 * hd, w.vh16 + t0 * hd, s));
          op = {w.kh16 + t0 * hd, hd, w.vh16 + t0 * hd, hd, nullptr};
        } else {
          Ws wb = w;  // the per-token inverse norms shifted to the block
          wb.rk = w.rk + t0 * dims.heads;
          TTT_TRY(prepare_update_operands(dK + t0 * row, hd, v, hd, dEta + t0 * dims.heads, tb, dims, dtype,
                                          io->qk_l2norm, wb, s, &op));
        }
        TTT_TRY(run_grad(W, op.K, op.ldk, op.V, op.ldv, dEta + t0 * dims.heads, op.rk, io->qk_l2norm, tb, dims,
                         dtype, w, w.G, s, b > 0));
      }
      TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
      // further steps re-read the prepared operands of all T tokens
      UpdOperands full;
      if (dtype == TTT_BF16)
        full = {w.kh16, hd, w.vh16, hd, nullptr};
      else
        full = {dK, hd, conv ? dVc : dV, hd, io->qk_l2norm ? w.rk : nullptr};
      for (int st = 1; st < steps; ++st) {
        TTT_TRY(run_grad(W, full.K, full.ldk, full.V, full.ldv, dEta, full.rk, io->qk_l2norm, T, dims, dtype, w, w.G, s));
        TTT_TRY(run_step(W, w.G, *ns, dims, dtype, w, s));
      }
    }
    for (int64_t b = 0; b < nb; ++b) {
      TTT_CHECK(cudaStreamWaitEvent(s, ev_q[b], 0));
      TTT_TRY(apply_block(b, w.rq + b * bt * dims.heads));
    }
    return TTT_OK;
  };
  const int rc = body();
  // `stream` completes only after both copy streams (also when queueing failed midway)
  const cudaError_t e1 = cudaEventRecord(ev_h2d_end, P->h2d);
  const cudaError_t e2 = cudaEventRecord(ev_d2h_end, P->d2h);
  const cudaError_t e3 = cudaStreamWaitEvent(s, ev_h2d_end, 0);
  const cudaError_t e4 = cudaStreamWaitEvent(s, ev_d2h_end, 0);
  if (rc != TTT_OK) return rc;
  if (e1 != cudaSuccess || e2 != cudaSuccess || e3 != cudaSuccess || e4 != cudaSuccess) return TTT_ERR_CUDA;
  return TTT_OK;
}

size_t ttt_gate_workspace_bytes(int64_t T, int D) {
  if (T < 0 || D < 256 || D % 256) return 0;
  return 256 + up256((size_t)D * D * 2) + up256((size_t)std::max<int64_t>(T, 1) * 4);
}

int ttt_output_gate(const void* Oprime, int64_t ld_in, const float* Wg, void* O, int64_t ld_out, int64_t T, int D,
                    ttt_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  if (dtype != TTT_FP32 && dtype != TTT_BF16) return TTT_ERR_INVALID;
  if (T < 0 || D < 1) return TTT_ERR_INVALID;
  if (dtype != TTT_BF16 || D % 256 || D < 256 || T > INT32_MAX) return TTT_ERR_UNSUPPORTED;
  if (ld_in == 0) ld_in = D;
  if (ld_out == 0) ld_out = D;
  if (ld_in < D || ld_out < D) return TTT_ERR_INVALID;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTT_ERR_WORKSPACE;
  if (ws_bytes < ttt_gate_workspace_bytes(T, D)) return TTT_ERR_WORKSPACE;
  if (T == 0) return TTT_OK;
  if (!Oprime || !Wg || !O || Oprime == O) return TTT_ERR_INVALID;
  if (!aligned16(Oprime) || !aligned16(O) || !aligned16(Wg) || (ld_in * 2) % 16 || (ld_out * 2) % 16)
    return TTT_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* b = static_cast<uint8_t*>(ws);
  Ws w{};
  w.status = reinterpret_cast<unsigned int*>(b);
  __nv_bfloat16* wg16 = reinterpret_cast<__nv_bfloat16*>(b + 256);
  float* rinv = reinterpret_cast<float*>(b + 256 + up256((size_t)D * D * 2));
  const int64_t nn = (int64_t)D * D;
  ProfScope ps(TTT_PROF_APPLY, s);
  k_cast_bf16<<<grid1d(nn / 4, 256), 256, 0, s>>>(Wg, wg16, nn);
  TTT_LAUNCHED();
  k_rms_rows<<<(int)std::max<int64_t>(1, std::min<int64_t>((T * 32 + 255) / 256, (int64_t)sm_count() * 16)), 256, 0,
               s>>>((const __nv_bfloat16*)Oprime, ld_in, T, D, 1e-6f, rinv);
  TTT_LAUNCHED();
  CUtensorMap tA, tB;
  if (!tmap_k(&tA, Oprime, (uint64_t)D, (uint64_t)T, (uint64_t)ld_in, false) ||
      !tmap_k(&tB, wg16, (uint64_t)D, (uint64_t)D, (uint64_t)D, false))
    return TTT_ERR_CUDA;
  WgArgs a = wg_args();
  a.M = (int)T;
  a.mt = (int)((T + 255) / 256);
  a.nt = D / 256;
  a.kblocks = D / 64;
  a.out = O;
  a.ldo = ld_out;
  a.aux = Oprime;
  a.ldaux = ld_in;
  a.rvec = rinv;
  a.idesc = idesc_bf16(256, 256, false, false);
  return launch_wgemm<WG_GATE, false, false>(tA, tA, tA, tB, tB, a, a.mt * a.nt, w, s);
}

int ttt_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned timeout_us, void* stream) {
  if (!ws || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u)) return TTT_ERR_WORKSPACE;
  if (timeout_us < 1 || timeout_us > 10000000u) return TTT_ERR_INVALID;
  k_selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<unsigned int*>(ws),
                                                       (unsigned long long)timeout_us * 1000ull);
  TTT_LAUNCHED();
  return TTT_OK;
}

int ttt_compiled_arch(void) {
#ifdef __CUDA_ARCH_LIST__
  return __CUDA_ARCH_LIST__;
#else
  return 0;
#endif
}

int ttt_kernel_binary_version(int* version) {
  if (!version) return TTT_ERR_INVALID;
  cudaFuncAttributes a{};
  TTT_CHECK(cudaFuncGetAttributes(&a, k_selftest_wait));
  *version = a.binaryVersion;
  return TTT_OK;
}

const char* ttt_status_string(int status) {
  switch (status) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID: return "invalid argument";
    case TTT_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case TTT_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TTT_ERR_CUDA: return "CUDA runtime error or failed launch";
    case TTT_ERR_TIMEOUT: return "device-side wait timed out";
    case TTT_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case TTT_ERR_SCRATCH: return "problem too large for the fixed 8 MiB scratch of ttt_apply_noalloc";
    case TTT_ERR_RANGE: return "gradient not finite: an fp16 operand of the tensor-core update was out of range";
    default: return "unknown status";
  }
}

uint64_t ttt_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ttt_profile_enable(int on) {
  g_prof_on.store(on != 0);
  return TTT_OK;
}

int ttt_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& p : g_prof_pending) {
    cudaEventSynchronize(p.b);
    g_prof_pool.push_back(p.a);
    g_prof_pool.push_back(p.b);
  }
  g_prof_pending.clear();
  for (int k = 0; k < TTT_PROF_KINDS; ++k) {
    g_prof_ms[k] = 0;
    g_prof_n[k] = 0;
  }
  return TTT_OK;
}

int ttt_profile_query(int kind, double* total_ms, uint64_t* count) {
  if (kind < 0 || kind >= TTT_PROF_KINDS) return TTT_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& p : g_prof_pending) {
    if (cudaEventSynchronize(p.b) != cudaSuccess) return TTT_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) return TTT_ERR_CUDA;
    g_prof_ms[p.kind] += ms;
    g_prof_n[p.kind] += 1;
    g_prof_pool.push_back(p.a);
    g_prof_pool.push_back(p.b);
  }
  g_prof_pending.clear();
  if (total_ms) *total_ms = g_prof_ms[kind];
  if (count) *count = g_prof_n[kind];
  return TTT_OK;
}

}  // extern "C"
