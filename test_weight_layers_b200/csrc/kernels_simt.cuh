// CUDA-core kernels: memory-bound preprocessing (row norms, L2 norm, ShortConv2D),
// weight shadows, the deterministic split-K reduction, Newton-Schulz and the
// Muon weight step, and the fp32-mode gradient/apply used when the layer runs
// in full fp32 precision.
#pragma once

#include "common.cuh"

namespace ttt {

template <typename T>
struct Vec16;  // 16-byte vector of T
template <>
struct Vec16<float> {
  static constexpr int N = 4;
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
};

__device__ __forceinline__ void load16(const float* p, float (&v)[4]) {
  float4 x = *reinterpret_cast<const float4*>(p);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 x = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store16(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 x;
  x.x = pack_bf16x2(v[0], v[1]);
  x.y = pack_bf16x2(v[2], v[3]);
  x.z = pack_bf16x2(v[4], v[5]);
  x.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = x;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// L2 norms of (token, head) rows (VGG-T3 key design 1): one warp per token.
// mode 0: write r[t*H + h] = 1 / max(||x||, 1e-12);  mode 1: scale X in place.
// The whole row (H*d <= 128 16-byte vectors) is loaded before any reduction so
// every lane has its loads in flight together; per-head sums are warp
// reductions of lane partials masked by head.

constexpr int RN_MAX_VEC = 4;  // 16-byte vectors per lane: H*d <= 128 * VN elements
constexpr int RN_TOKS = 4;     // tokens per warp iteration when only the norms are written
constexpr int RN_TOK_VEC = 3;  // vectors per lane in that path: H*d <= 96 * VN elements

template <typename T>
__global__ void __launch_bounds__(256, 4) k_rownorm(T* X, int64_t ld, int64_t rows, int H, int d, float* r_out, int mode) {
  constexpr int VN = Vec16<T>::N;
  const int lane = threadIdx.x & 31;
  const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int nvt = H * d / VN;  // vectors per row
  if (nvt > 32 * RN_MAX_VEC) {
    // wide rows: one head at a time
    const int nv = d / VN;
    for (int64_t t = warp_id; t < rows; t += nwarps) {
      T* row = X + t * ld;
      for (int h = 0; h < H; ++h) {
        float ss = 0.f;
        for (int v = lane; v < nv; v += 32) {
          float x[VN];
          load16(row + h * d + v * VN, x);
#pragma unroll
          for (int i = 0; i < VN; ++i) ss = fmaf(x[i], x[i], ss);
        }
        ss = warp_sum(ss);
        const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
        if (mode == 0) {
          if (lane == 0) r_out[t * H + h] = inv;
        } else {
          for (int v = lane; v < nv; v += 32) {
            float x[VN];
            load16(row + h * d + v * VN, x);
#pragma unroll
            for (int i = 0; i < VN; ++i) x[i] *= inv;
            store16(row + h * d + v * VN, x);
          }
        }
      }
    }
    return;
  }
  if (mode == 0 && nvt <= 32 * RN_TOK_VEC) {
    // norms only: four tokens per warp iteration, all their loads in flight together
    for (int64_t t0 = warp_id * RN_TOKS; t0 < rows; t0 += nwarps * RN_TOKS) {
      float ss[RN_TOKS][RN_TOK_VEC];
      int hv[RN_TOK_VEC];
#pragma unroll
      for (int k = 0; k < RN_TOK_VEC; ++k) {
        const int v = lane + 32 * k;
        hv[k] = v < nvt ? v * VN / d : -1;
      }
#pragma unroll
      for (int u = 0; u < RN_TOKS; ++u) {
        const int64_t t = t0 + u;
#pragma unroll
        for (int k = 0; k < RN_TOK_VEC; ++k) {
          ss[u][k] = 0.f;
          if (hv[k] >= 0 && t < rows) {
            float x[VN];
            load16(X + t * ld + (lane + 32 * k) * VN, x);
#pragma unroll
            for (int i = 0; i < VN; ++i) ss[u][k] = fmaf(x[i], x[i], ss[u][k]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < RN_TOKS; ++u) {
        const int64_t t = t0 + u;
        for (int h = 0; h < H; ++h) {
          float p = 0.f;
#pragma unroll
          for (int k = 0; k < RN_TOK_VEC; ++k) p += (hv[k] == h) ? ss[u][k] : 0.f;
          p = warp_sum(p);
          if (lane == 0 && t < rows) r_out[t * H + h] = 1.0f / fmaxf(sqrtf(p), 1e-12f);
        }
      }
    }
    return;
  }
  for (int64_t t = warp_id; t < rows; t += nwarps) {
    T* row = X + t * ld;
    float x[RN_MAX_VEC][VN];
    float ss[RN_MAX_VEC];
    int hv[RN_MAX_VEC];
#pragma unroll
    for (int k = 0; k < RN_MAX_VEC; ++k) {
      const int v = lane + 32 * k;
      hv[k] = -1;
      ss[k] = 0.f;
      if (v < nvt) {
        load16(row + v * VN, x[k]);
        hv[k] = v * VN / d;
      }
    }
#pragma unroll
    for (int k = 0; k < RN_MAX_VEC; ++k)
      if (hv[k] >= 0) {
#pragma unroll
        for (int i = 0; i < VN; ++i) ss[k] = fmaf(x[k][i], x[k][i], ss[k]);
      }
    float inv_mine[RN_MAX_VEC];
#pragma unroll
    for (int k = 0; k < RN_MAX_VEC; ++k) inv_mine[k] = 0.f;
    for (int h = 0; h < H; ++h) {
      float p = 0.f;
#pragma unroll
      for (int k = 0; k < RN_MAX_VEC; ++k) p += (hv[k] == h) ? ss[k] : 0.f;
      p = warp_sum(p);
      const float inv = 1.0f / fmaxf(sqrtf(p), 1e-12f);
      if (mode == 0 && lane == 0) r_out[t * H + h] = inv;
#pragma unroll
      for (int k = 0; k < RN_MAX_VEC; ++k)
        if (hv[k] == h) inv_mine[k] = inv;
    }
    if (mode == 1) {
#pragma unroll
      for (int k = 0; k < RN_MAX_VEC; ++k)
        if (hv[k] >= 0) {
#pragma unroll
          for (int i = 0; i < VN; ++i) x[k][i] *= inv_mine[k];
          store16(row + (lane + 32 * k) * VN, x[k]);
        }
    }
  }
}

// ---------------------------------------------------------------------------
// Update-operand preparation: one pass over K and V that writes the fp16
// operands of the tensor-core gradient kernel, K^ = k / max(||k||, 1e-12) per
// head (or k itself) and V' = -s eta_(t,h) v, densely [T][H*d], with the
// power-of-two value scale s of the call (value_scale: s max|eta| in [16, 32)).
// The loss is linear in v, so folding the per-token weight and s into V is
// exact algebra: the forward then yields s dL/du directly and the gradient of
// W2 needs no per-token scaling.  bf16 -> fp16 is exact for values in fp16's
// normal range; fp16 carries three more significand bits than bf16, which the
// chained Muon updates need.  One warp per token, the whole row loaded before
// any reduction.

__device__ __forceinline__ void store16_h(__half* p, const float (&v)[8]) {
  uint4 x;
  x.x = pack_f16x2(v[0], v[1]);
  x.y = pack_f16x2(v[2], v[3]);
  x.z = pack_f16x2(v[4], v[5]);
  x.w = pack_f16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = x;
}

// RN: 16-byte vectors per lane of a row (H*d <= 256 RN); more than 4 takes the
// per-head loop
template <int RN>
__global__ void __launch_bounds__(256, RN <= 3 ? 3 : 2) k_prep_kv(const __nv_bfloat16* __restrict__ K, int64_t ldk,
                                                    const __nv_bfloat16* __restrict__ V, int64_t ldv,
                                                    const float* __restrict__ eta,
                                                    const float* __restrict__ eta_part,
                                                    __half* __restrict__ Kh, __half* __restrict__ Vh, int64_t rows,
                                                    int H, int d, int l2norm, float* __restrict__ part_out) {
  constexpr int VN = 8;
  // max|eta| from the block maxima of k_eta_absmax, or (part_out != nullptr, small
  // calls) reduced here by every block over all rows * H values, block 0 then
  // writing the maxima array the gradient kernel reads (its maximum first, zeros)
  float emax;
  if (part_out) {
    __shared__ float red[8];
    const int64_t n = rows * H;
    float mx = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) mx = fmaxf(mx, fabsf(__ldg(eta + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    emax = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) emax = fmaxf(emax, red[w]);
    if (blockIdx.x == 0 && threadIdx.x < ETA_PARTS) part_out[threadIdx.x] = threadIdx.x == 0 ? emax : 0.f;
  } else {
    emax = eta_parts_max(eta_part);
  }
  float vscale, inv_unused;  // V' = -s eta v with the value scale s of this call
  value_scale(emax, vscale, inv_unused);
  vscale = -vscale;
  const int lane = threadIdx.x & 31;
  const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int HD = H * d;
  const int nvt = HD / VN;
  if (nvt <= 32 * RN) {
    // The row stays packed (bf16) in registers: small footprint, many tokens in
    // flight per SM.  The next token's row is loaded while this one is
    // converted, so a warp always has a row's loads outstanding.
    int hv[RN];  // head of this lane's k-th vector (-1: past the row)
#pragma unroll
    for (int k = 0; k < RN; ++k) {
      const int v = lane + 32 * k;
      hv[k] = v < nvt ? v * VN / d : -1;
    }
    // eta of a token: lane h < H holds head h's weight (one load per token,
    // issued with the row loads); the vectors fetch theirs by shuffle
    auto load_row = [&](int64_t t, uint4 (&xk)[RN], uint4 (&xv)[RN], float& eh) {
      const __nv_bfloat16* krow = K + t * ldk;
      const __nv_bfloat16* vrow = V + t * ldv;
      eh = (lane < H) ? __ldg(eta + t * H + lane) : 0.f;
#pragma unroll
      for (int k = 0; k < RN; ++k) {
        const int v = lane + 32 * k;
        if (hv[k] >= 0) {
          xk[k] = __ldg(reinterpret_cast<const uint4*>(krow + v * VN));
          xv[k] = Vh ? __ldg(reinterpret_cast<const uint4*>(vrow + v * VN)) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    uint4 xk[RN], xv[RN];
    float eh = 0.f;
    int64_t t = warp_id;
    if (t < rows) load_row(t, xk, xv, eh);
    for (; t < rows; t += nwarps) {
      uint4 nk[RN], nv[RN];
      float ne = 0.f;
      if (t + nwarps < rows) load_row(t + nwarps, nk, nv, ne);
      float inv[RN];
#pragma unroll
      for (int k = 0; k < RN; ++k) inv[k] = 1.f;
      if (l2norm) {
        float ss[RN];
#pragma unroll
        for (int k = 0; k < RN; ++k) {
          ss[k] = 0.f;
          if (hv[k] >= 0) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&xk[k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(h2[i]);
              ss[k] = fmaf(f.x, f.x, fmaf(f.y, f.y, ss[k]));
            }
          }
        }
        for (int h = 0; h < H; ++h) {
          float p = 0.f;
#pragma unroll
          for (int k = 0; k < RN; ++k) p += (hv[k] == h) ? ss[k] : 0.f;
          p = warp_sum(p);
          const float r = 1.0f / fmaxf(sqrtf(p), 1e-12f);
#pragma unroll
          for (int k = 0; k < RN; ++k)
            if (hv[k] == h) inv[k] = r;
        }
      }
#pragma unroll
      for (int k = 0; k < RN; ++k) {
        const float vek = vscale * __shfl_sync(0xffffffffu, eh, hv[k] >= 0 ? hv[k] : 0);
        if (hv[k] >= 0) {
          const __nv_bfloat162* hk = reinterpret_cast<const __nv_bfloat162*>(&xk[k]);
          const __nv_bfloat162* hvv = reinterpret_cast<const __nv_bfloat162*>(&xv[k]);
          uint4 ok, ov;
          uint32_t* pk = reinterpret_cast<uint32_t*>(&ok);
          uint32_t* pv = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 fk = __bfloat1622float2(hk[i]), fv = __bfloat1622float2(hvv[i]);
            pk[i] = pack_f16x2(fk.x * inv[k], fk.y * inv[k]);
            pv[i] = pack_f16x2(fv.x * vek, fv.y * vek);
          }
          *reinterpret_cast<uint4*>(Kh + t * HD + (lane + 32 * k) * VN) = ok;
          if (Vh) *reinterpret_cast<uint4*>(Vh + t * HD + (lane + 32 * k) * VN) = ov;
        }
      }
#pragma unroll
      for (int k = 0; k < RN; ++k) {
        xk[k] = nk[k];
        xv[k] = nv[k];
      }
      eh = ne;
    }
  } else {
    for (int64_t t = warp_id; t < rows; t += nwarps) {
      const __nv_bfloat16* krow = K + t * ldk;
      const __nv_bfloat16* vrow = V + t * ldv;
      for (int h = 0; h < H; ++h) {
        float ss = 0.f;
        for (int v = lane; v < d / VN; v += 32) {
          float x[VN];
          load16(krow + h * d + v * VN, x);
#pragma unroll
          for (int i = 0; i < VN; ++i) ss = fmaf(x[i], x[i], ss);
        }
        ss = warp_sum(ss);
        const float r = l2norm ? 1.0f / fmaxf(sqrtf(ss), 1e-12f) : 1.f;
        const float ve = vscale * eta[t * H + h];
        for (int v = lane; v < d / VN; v += 32) {
          float x[VN], y[VN];
          load16(krow + h * d + v * VN, x);
          if (Vh) load16(vrow + h * d + v * VN, y);
#pragma unroll
          for (int i = 0; i < VN; ++i) {
            x[i] *= r;
            y[i] = Vh ? y[i] * ve : 0.f;
          }
          store16_h(Kh + t * HD + h * d + v * VN, x);
          if (Vh) store16_h(Vh + t * HD + h * d + v * VN, y);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// ShortConv2D (VGG-T3 key design 2): depthwise 3x3 zero-padded cross-correlation
// per frame on the (N, h, w, C) patch grid.  CTA = (frame, 64-channel group),
// taps in shared memory; threadIdx.x = 16-byte channel vector, threadIdx.y walks
// the frame's tokens, so a token's neighbours are read from HBM once and
// re-served from L1 to the nine taps.

constexpr int CONV_GROUP = 64;    // channels per CTA

__device__ __forceinline__ void load16_nc(const float* p, float (&v)[4]) {
  float4 x = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load16_nc(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 x = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <typename T>
__global__ void __launch_bounds__(256, 4) k_shortconv(const T* __restrict__ V, int64_t ldv, T* __restrict__ out,
                                                      int64_t ldo, const float* __restrict__ taps, int N, int gh,
                                                      int gw, int C, int act) {
  constexpr int VN = Vec16<T>::N;
  __shared__ __align__(16) float wt[9][CONV_GROUP];  // this CTA's taps, [tap][channel]
  const int n = blockIdx.x, g0 = blockIdx.y * CONV_GROUP;
  const int nthr = blockDim.x * blockDim.y, tid = threadIdx.y * blockDim.x + threadIdx.x;
  for (int i = tid; i < 9 * CONV_GROUP; i += nthr) {
    const int k = i / CONV_GROUP, c = i % CONV_GROUP;
    wt[k][c] = (g0 + c < C) ? taps[(g0 + c) * 9 + k] : 0.f;
  }
  __syncthreads();
  const int c0 = g0 + threadIdx.x * VN;
  if (c0 >= C) return;
  const int64_t frame0 = (int64_t)n * gh * gw;
  const int ntok = gh * gw;
  for (int p = threadIdx.y; p < ntok; p += blockDim.y) {
    const int y = p / gw, x = p % gw;
    float acc[VN];
#pragma unroll
    for (int i = 0; i < VN; ++i) acc[i] = 0.f;
#pragma unroll
    for (int dy = -1; dy <= 1; ++dy) {
      const int yy = y + dy;
      if (yy < 0 || yy >= gh) continue;
#pragma unroll
      for (int dx = -1; dx <= 1; ++dx) {
        const int xx = x + dx;
        if (xx < 0 || xx >= gw) continue;
        float v[VN];
        load16_nc(V + (frame0 + (int64_t)yy * gw + xx) * ldv + c0, v);
        const float* wk = &wt[(dy + 1) * 3 + (dx + 1)][threadIdx.x * VN];
#pragma unroll
        for (int i = 0; i < VN; i += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wk + i);
          acc[i] = fmaf(w4.x, v[i], acc[i]);
          acc[i + 1] = fmaf(w4.y, v[i + 1], acc[i + 1]);
          acc[i + 2] = fmaf(w4.z, v[i + 2], acc[i + 2]);
          acc[i + 3] = fmaf(w4.w, v[i + 3], acc[i + 3]);
        }
      }
    }
    if (act == 1) {
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[i] = acc[i] / (1.0f + expf(-acc[i]));
    }
    store16(out + (frame0 + p) * ldo + c0, acc);
  }
}

// Banded ShortConv2D: CTA = (64-channel group, frame slot); the frame is walked
// in bands of BR output rows.  Each band's BR + 2 input rows (one halo row on
// each side, zero-filled outside the frame) are staged in shared memory with
// 16-byte asynchronous copies, double-buffered so the next band loads while
// this one is computed; the 3x3 sums then read shared memory only.  Frames past
// gridDim.y are taken in a grid-stride loop.  Dynamic shared memory:
// conv_band_smem(BR, gw, sizeof(T)).
__host__ __device__ constexpr size_t conv_band_bytes(int BR, int gw, int esz) {
  return (size_t)(BR + 2) * gw * CONV_GROUP * esz;
}
__host__ __device__ constexpr size_t conv_band_smem(int BR, int gw, int esz) {
  return 9 * CONV_GROUP * sizeof(float) + 2 * conv_band_bytes(BR, gw, esz);
}

__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

template <typename T>
__global__ void __launch_bounds__(256, 2) k_shortconv_band(const T* __restrict__ V, int64_t ldv, T* __restrict__ out,
                                                        int64_t ldo, const float* __restrict__ taps, int N, int gh,
                                                        int gw, int C, int act, int BR) {
  constexpr int VN = Vec16<T>::N;           // elements per 16-byte chunk
  constexpr int TPT = CONV_GROUP / VN;      // threads (chunks) per token
  constexpr int NL = 256 / TPT;             // tokens per pass
  extern __shared__ __align__(16) uint8_t cdyn[];
  float* wt = reinterpret_cast<float*>(cdyn);  // [9][CONV_GROUP]
  uint8_t* bufs = cdyn + 9 * CONV_GROUP * sizeof(float);
  const size_t bb = conv_band_bytes(BR, gw, (int)sizeof(T));
  const int g0 = blockIdx.x * CONV_GROUP;
  const int tid = threadIdx.x;
  for (int i = tid; i < 9 * CONV_GROUP; i += 256) {
    const int k = i / CONV_GROUP, c = i % CONV_GROUP;
    wt[k * CONV_GROUP + c] = (g0 + c < C) ? taps[(g0 + c) * 9 + k] : 0.f;
  }
  const int chunk = tid % TPT, tl = tid / TPT;
  const int c0 = g0 + chunk * VN;
  const int ntok = gh * gw, nbands = (gh + BR - 1) / BR;
  __syncthreads();
  float wr[9][VN];  // this thread's taps, kept in registers for all its outputs
#pragma unroll
  for (int k = 0; k < 9; ++k)
#pragma unroll
    for (int i = 0; i < VN; ++i) wr[k][i] = wt[k * CONV_GROUP + chunk * VN + i];
  const int rowchunks = gw * TPT;
  for (int n = blockIdx.y; n < N; n += gridDim.y) {
    const int64_t frame0 = (int64_t)n * ntok;
    auto issue = [&](int bi, uint8_t* buf) {
      const int y0 = bi * BR - 1;
      for (int idx = tid; idx < (BR + 2) * rowchunks; idx += 256) {
        const int r = idx / rowchunks, rem = idx % rowchunks, x = rem / TPT, k = rem % TPT;
        const int yy = y0 + r, ch = g0 + k * VN;
        const bool in = yy >= 0 && yy < gh && ch < C;
        const T* src = in ? V + (frame0 + (int64_t)yy * gw + x) * ldv + ch : V;
        cp_async16_cg(buf + (size_t)idx * 16, src, in ? 16u : 0u);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // taps written; the previous frame's buffers are no longer read
    issue(0, bufs);
    for (int bi = 0; bi < nbands; ++bi) {
      uint8_t* cur = bufs + (bi & 1) * bb;
      if (bi + 1 < nbands) {
        issue(bi + 1, bufs + ((bi + 1) & 1) * bb);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();
      const int y0 = bi * BR, rows = min(BR, gh - y0);
      if (c0 < C) {
        for (int p = tl; p < rows * gw; p += NL) {
          const int ry = p / gw, x = p % gw;  // output row y0 + ry; its input rows are ry .. ry + 2 in the band
          float acc[VN];
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[i] = 0.f;
#pragma unroll
          for (int dy = 0; dy < 3; ++dy) {
#pragma unroll
            for (int dx = -1; dx <= 1; ++dx) {
              const int xx = x + dx;
              if (xx < 0 || xx >= gw) continue;
              float v[VN];
              load16(reinterpret_cast<const T*>(cur + ((size_t)((ry + dy) * gw + xx) * TPT + chunk) * 16), v);
#pragma unroll
              for (int i = 0; i < VN; ++i) acc[i] = fmaf(wr[dy * 3 + dx + 1][i], v[i], acc[i]);
            }
          }
          if (act == 1) {
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[i] = acc[i] / (1.0f + expf(-acc[i]));
          }
          store16(out + (frame0 + (int64_t)(y0 + ry) * gw + x) * ldo + c0, acc);
        }
      }
      __syncthreads();  // `cur` may be refilled by the prefetch of band bi + 2
    }
  }
}

// bf16 variant.  Each thread computes two horizontally adjacent outputs of one
// 8-channel chunk, so a chunk loaded from shared memory serves up to three taps
// of both; band rows carry a zero slot on each side (and one past an odd width),
// so the tap loop has no bounds tests; bf16 -> fp32 by a shift or a mask, and
// packed fp32x2 FMAs.  The sums are the same as k_shortconv_band's, in the same
// order (a tap outside the frame adds w * 0).
constexpr int CONV2_SX = 2;  // outputs per thread along x
__host__ __device__ constexpr int conv2_row_slots(int gw) { return (gw + CONV2_SX - 1) / CONV2_SX * CONV2_SX + 2; }
__host__ __device__ constexpr size_t conv2_band_bytes(int BR, int gw) {
  return (size_t)(BR + 2) * conv2_row_slots(gw) * CONV_GROUP * 2;
}
__host__ __device__ constexpr size_t conv2_band_smem(int BR, int gw) {
  return 9 * CONV_GROUP * sizeof(float) + 2 * conv2_band_bytes(BR, gw);
}

// 8 bf16 (one 16-byte chunk) -> 4 fp32 pairs
__device__ __forceinline__ void bf16x8_f2(const uint4 q, float2 (&f)[4]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) f[e] = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
}

// FUSE = false: the ShortConv2D output V' in bf16 (ttt_shortconv2d).  FUSE = true: the
// update's fp16 value operand -s eta_(t,h) V' directly (dense [T][C], head h = c / d), so
// V' never makes a bf16 round trip through HBM; s is the value scale of eta_part.
template <bool FUSE>
__global__ void __launch_bounds__(256, 2) k_shortconv_band2(const __nv_bfloat16* __restrict__ V, int64_t ldv,
                                                         void* __restrict__ out, int64_t ldo,
                                                         const float* __restrict__ taps, int N, int gh, int gw, int C,
                                                         int act, int BR, const float* __restrict__ eta,
                                                         const float* __restrict__ eta_part, int H, int d) {
  constexpr int TPT = CONV_GROUP / 8;  // threads (8-channel chunks) per token
  constexpr int NL = 256 / TPT;        // output pairs per pass
  extern __shared__ __align__(16) uint8_t cdyn[];
  float* wt = reinterpret_cast<float*>(cdyn);  // [9][CONV_GROUP]
  uint8_t* bufs = cdyn + 9 * CONV_GROUP * sizeof(float);
  const int RS = conv2_row_slots(gw);
  const size_t bb = conv2_band_bytes(BR, gw);
  const int g0 = blockIdx.x * CONV_GROUP;
  const int tid = threadIdx.x;
  for (int i = tid; i < 9 * CONV_GROUP; i += 256) {
    const int k = i / CONV_GROUP, c = i % CONV_GROUP;
    wt[k * CONV_GROUP + c] = (g0 + c < C) ? taps[(g0 + c) * 9 + k] : 0.f;
  }
  const int chunk = tid % TPT, tl = tid / TPT;
  const int c0 = g0 + chunk * 8;
  const int ntok = gh * gw, nbands = (gh + BR - 1) / BR, nstrips = (gw + CONV2_SX - 1) / CONV2_SX;
  float vscale = 0.f;
  if (FUSE) {
    float inv_unused;
    value_scale(eta_parts_max(eta_part), vscale, inv_unused);
  }
  const int head = FUSE ? c0 / d : 0;
  __syncthreads();
  float2 wr[9][4];  // this thread's taps as channel pairs, in registers for all its outputs
#pragma unroll
  for (int k = 0; k < 9; ++k)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      wr[k][i] = make_float2(wt[k * CONV_GROUP + chunk * 8 + 2 * i], wt[k * CONV_GROUP + chunk * 8 + 2 * i + 1]);
  const int rowchunks = RS * TPT;
  for (int n = blockIdx.y; n < N; n += gridDim.y) {
    const int64_t frame0 = (int64_t)n * ntok;
    // band bi: input rows bi*BR - 1 .. bi*BR + BR, slots x = -1 .. RS - 2 (zero outside the frame)
    auto issue = [&](int bi, uint8_t* buf) {
      const int y0 = bi * BR - 1;
      for (int idx = tid; idx < (BR + 2) * rowchunks; idx += 256) {
        const int r = idx / rowchunks, rem = idx % rowchunks, x = rem / TPT - 1, k = rem % TPT;
        const int yy = y0 + r, ch = g0 + k * 8;
        const bool in = yy >= 0 && yy < gh && x >= 0 && x < gw && ch < C;
        const __nv_bfloat16* src = in ? V + (frame0 + (int64_t)yy * gw + x) * ldv + ch : V;
        cp_async16_cg(buf + (size_t)idx * 16, src, in ? 16u : 0u);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // taps written; the previous frame's buffers are no longer read
    issue(0, bufs);
    for (int bi = 0; bi < nbands; ++bi) {
      uint8_t* cur = bufs + (bi & 1) * bb;
      if (bi + 1 < nbands) {
        issue(bi + 1, bufs + ((bi + 1) & 1) * bb);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();
      const int y0 = bi * BR, rows = min(BR, gh - y0);
      if (c0 < C) {
        for (int p = tl; p < rows * nstrips; p += NL) {
          const int ry = p / nstrips, x0 = (p % nstrips) * CONV2_SX;  // outputs (y0 + ry, x0), (y0 + ry, x0 + 1)
          float2 a0[4], a1[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) a0[i] = a1[i] = make_float2(0.f, 0.f);
#pragma unroll
          for (int dy = 0; dy < 3; ++dy) {
            // slots x0 .. x0 + 3 hold inputs x0 - 1 .. x0 + 2 of band row ry + dy
            const uint4* rp = reinterpret_cast<const uint4*>(cur) + ((size_t)(ry + dy) * RS + x0) * TPT + chunk;
            float2 in[4];
            bf16x8_f2(rp[0], in);
#pragma unroll
            for (int i = 0; i < 4; ++i) a0[i] = __ffma2_rn(wr[dy * 3][i], in[i], a0[i]);
            bf16x8_f2(rp[TPT], in);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              a0[i] = __ffma2_rn(wr[dy * 3 + 1][i], in[i], a0[i]);
              a1[i] = __ffma2_rn(wr[dy * 3][i], in[i], a1[i]);
            }
            bf16x8_f2(rp[2 * TPT], in);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              a0[i] = __ffma2_rn(wr[dy * 3 + 2][i], in[i], a0[i]);
              a1[i] = __ffma2_rn(wr[dy * 3 + 1][i], in[i], a1[i]);
            }
            bf16x8_f2(rp[3 * TPT], in);
#pragma unroll
            for (int i = 0; i < 4; ++i) a1[i] = __ffma2_rn(wr[dy * 3 + 2][i], in[i], a1[i]);
          }
          if (act == 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              a0[i].x = a0[i].x / (1.0f + expf(-a0[i].x));
              a0[i].y = a0[i].y / (1.0f + expf(-a0[i].y));
              a1[i].x = a1[i].x / (1.0f + expf(-a1[i].x));
              a1[i].y = a1[i].y / (1.0f + expf(-a1[i].y));
            }
          }
          const int64_t t0 = frame0 + (int64_t)(y0 + ry) * gw + x0;
          if (FUSE) {
            const float s0 = -vscale * __ldg(eta + t0 * H + head);
            __half* o = static_cast<__half*>(out) + t0 * ldo + c0;
            *reinterpret_cast<uint4*>(o) =
                make_uint4(pack_f16x2(a0[0].x * s0, a0[0].y * s0), pack_f16x2(a0[1].x * s0, a0[1].y * s0),
                           pack_f16x2(a0[2].x * s0, a0[2].y * s0), pack_f16x2(a0[3].x * s0, a0[3].y * s0));
            if (x0 + 1 < gw) {
              const float s1 = -vscale * __ldg(eta + (t0 + 1) * H + head);
              *reinterpret_cast<uint4*>(o + ldo) =
                  make_uint4(pack_f16x2(a1[0].x * s1, a1[0].y * s1), pack_f16x2(a1[1].x * s1, a1[1].y * s1),
                             pack_f16x2(a1[2].x * s1, a1[2].y * s1), pack_f16x2(a1[3].x * s1, a1[3].y * s1));
            }
          } else {
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + t0 * ldo + c0;
            *reinterpret_cast<uint4*>(o) = make_uint4(pack_bf16x2(a0[0].x, a0[0].y), pack_bf16x2(a0[1].x, a0[1].y),
                                                      pack_bf16x2(a0[2].x, a0[2].y), pack_bf16x2(a0[3].x, a0[3].y));
            if (x0 + 1 < gw)
              *reinterpret_cast<uint4*>(o + ldo) =
                  make_uint4(pack_bf16x2(a1[0].x, a1[0].y), pack_bf16x2(a1[1].x, a1[1].y),
                             pack_bf16x2(a1[2].x, a1[2].y), pack_bf16x2(a1[3].x, a1[3].y));
          }
        }
      }
      __syncthreads();  // `cur` may be refilled by the prefetch of band bi + 2
    }
  }
}

// ---------------------------------------------------------------------------
// Low-precision copies of the fp32 fast weights, laid out for the tensor-core kernels:
//   Wsh (bf16, apply) and Wsh16 (fp16, gradient) rows [0, Hm): W1 [H][m][d];
//   [Hm, 2Hm): W3;  [2Hm, 3Hm): W2^T [H][m][d];   W2b [H][d][m] (bf16 W2, apply)

// Blocks [0, n/1024): the element-wise copies, four elements per thread (16-byte
// reads, 8-byte writes).  Blocks past that: W2^T in 32 x 32 tiles through
// shared memory, so both the W2 reads and the W2^T writes are row-contiguous.
// n = H*m*d is a multiple of 1024 (m a multiple of 64, d of 16).
constexpr int SHADOW_EW_BLOCK = 256 * 4;

__device__ __forceinline__ uint2 pack4_bf16(float4 v) {
  return make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}
__device__ __forceinline__ uint2 pack4_f16(float4 v) {
  return make_uint2(pack_f16x2(v.x, v.y), pack_f16x2(v.z, v.w));
}

__global__ void __launch_bounds__(256) k_shadow(const float* __restrict__ W1, const float* __restrict__ W3,
                                                const float* __restrict__ W2, __nv_bfloat16* __restrict__ Wsh,
                                                __nv_bfloat16* __restrict__ W2b, __half* __restrict__ Wsh16, int H,
                                                int d, int m) {
  pdl_trigger();
  pdl_wait();
  const int64_t n = (int64_t)H * m * d;
  const int ew_blocks = (int)(n / SHADOW_EW_BLOCK);
  if ((int)blockIdx.x < ew_blocks) {
    const int64_t i = ((int64_t)blockIdx.x * 256 + threadIdx.x) * 4;
    const float4 a = *reinterpret_cast<const float4*>(W1 + i);
    const float4 b = *reinterpret_cast<const float4*>(W3 + i);
    const float4 c = *reinterpret_cast<const float4*>(W2 + i);
    *reinterpret_cast<uint2*>(Wsh + i) = pack4_bf16(a);
    *reinterpret_cast<uint2*>(Wsh + n + i) = pack4_bf16(b);
    *reinterpret_cast<uint2*>(W2b + i) = pack4_bf16(c);
    if (Wsh16) {  // fp16 copy only when a gradient kernel will read it
      *reinterpret_cast<uint2*>(Wsh16 + i) = pack4_f16(a);
      *reinterpret_cast<uint2*>(Wsh16 + n + i) = pack4_f16(b);
    }
    return;
  }
  // W2^T [h][j][k] <- W2 [h][k][j]: tile (h, k0, j0) of 32 x 32
  __shared__ float tile[32][33];
  const int t = (int)blockIdx.x - ew_blocks;
  const int kt = d / 32, jt = m / 32;
  const int h = t / (kt * jt), rem = t % (kt * jt);
  const int k0 = (rem / jt) * 32, j0 = (rem % jt) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const float* src = W2 + (int64_t)h * d * m;
  for (int y = ty; y < 32; y += 8) tile[y][tx] = src[(int64_t)(k0 + y) * m + j0 + tx];
  __syncthreads();
  const int64_t base = 2 * n + (int64_t)h * m * d;
  for (int y = ty; y < 32; y += 8) {
    const float v = tile[tx][y];  // W2[k0 + tx][j0 + y]
    const int64_t o = base + (int64_t)(j0 + y) * d + k0 + tx;
    Wsh[o] = __float2bfloat16_rn(v);
    if (Wsh16) Wsh16[o] = __float2half_rn(v);
  }
}

// ---------------------------------------------------------------------------
// Deterministic split-K reduction: G[i] = sum_{s=0..S-1} P[s][i] in that order.

// G = sum over the S split partials (accumulate = 1: G += that sum), fixed order.
// A non-finite entry of G (an fp16 operand of the tensor-core gradient out of
// range, or non-finite inputs) records DEV_RANGE in the status word; the weight
// step then leaves W unchanged.
__global__ void k_reduce_splits(const float* __restrict__ P, int S, int64_t n, float* __restrict__ G, int accumulate,
                                unsigned int* status) {
  const int64_t n4 = n / 4;
  bool finite = true;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(P)[i];
    for (int s = 1; s < S; ++s) {
      float4 v = reinterpret_cast<const float4*>(P + (int64_t)s * n)[i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (accumulate) {
      const float4 g = reinterpret_cast<const float4*>(G)[i];
      acc.x += g.x; acc.y += g.y; acc.z += g.z; acc.w += g.w;
    }
    // |x| <= FLT_MAX is false for inf and NaN
    finite &= fabsf(acc.x) <= 3.402823466e38f && fabsf(acc.y) <= 3.402823466e38f &&
              fabsf(acc.z) <= 3.402823466e38f && fabsf(acc.w) <= 3.402823466e38f;
    reinterpret_cast<float4*>(G)[i] = acc;
  }
  if (!__all_sync(0xffffffffu, finite) && (threadIdx.x & 31) == 0) atomicCAS(status, DEV_OK, (unsigned int)DEV_RANGE);
}

// Block maxima of |eta| over n values (grid of ETA_PARTS blocks or fewer; the
// missing parts are written as 0), for the value scale of the gradient kernel.
__global__ void __launch_bounds__(512) k_eta_absmax(const float* __restrict__ eta, int64_t n, float* __restrict__ part,
                                                    int nparts) {
  __shared__ float red[16];
  float m = 0.f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const float a = __ldg(eta + i), b = __ldg(eta + i + stride), c = __ldg(eta + i + 2 * stride),
                d = __ldg(eta + i + 3 * stride);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d))));
  }
  for (; i < n; i += stride) m = fmaxf(m, fabsf(__ldg(eta + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) {
      part[blockIdx.x] = m;
      if (blockIdx.x == 0)
        for (int p = gridDim.x; p < nparts; ++p) part[p] = 0.f;
    }
  }
}

// Fixed-shape block reduction (256 threads) -> deterministic.
__device__ __forceinline__ float block_sum_256(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 8; ++i) s += red[i];
    red[8] = s;
  }
  __syncthreads();
  return red[8];
}

// ---------------------------------------------------------------------------
// Newton-Schulz (ZipMap key design 3) on the 3H per-head gradient matrices.
// Matrix b < 2H is g1/g3 of shape (m, d); b >= 2H is g2 of shape (d, m).
// X_b = orient(G_b) / (||G_b||_F + eps) has the wide shape (r, c), r = min(m, d).

__device__ __forceinline__ void mat_shape(int b, int H, int d, int m, int& R, int& C) {
  if (b < 2 * H) { R = m; C = d; } else { R = d; C = m; }
}

constexpr int NORM_PARTS = 16;  // slices per matrix for the norm reductions

// partial sums of squares: out[b * NORM_PARTS + p] over slice p of matrix b (n_per % 4 == 0)
__global__ void __launch_bounds__(256) k_frob_partials(const float* __restrict__ src, int64_t n_per,
                                                       float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[9];
  const int b = blockIdx.x, p = blockIdx.y;
  const int64_t n4 = n_per / 4, per = (n4 + NORM_PARTS - 1) / NORM_PARTS;
  const int64_t i0 = p * per, i1 = min(n4, i0 + per);
  const float4* x = reinterpret_cast<const float4*>(src + (int64_t)b * n_per);
  float s = 0.f;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += 256) {
    const float4 v = x[i];
    s = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, s))));
  }
  s = block_sum_256(s, red);
  if (threadIdx.x == 0) out[b * NORM_PARTS + p] = s;
}

__device__ __forceinline__ float sum_parts(const float* parts) {
  float s = 0.f;
#pragma unroll
  for (int p = 0; p < NORM_PARTS; ++p) s += parts[p];
  return s;
}

// X_b = orient(G_b) / (||G_b||_F + eps) in the wide orientation (r x c) and its
// transpose XT_b (c x r), both written coalesced through a 32x32 shared tile.
// grid (ceil(C/32), ceil(R/32), 3H) over G_b's own shape (R, C); block (32, 8).
__global__ void k_ns_init(const float* __restrict__ G, float* __restrict__ X, float* __restrict__ XT,
                          const float* __restrict__ parts, int H, int d, int m, float eps) {
  pdl_trigger();
  pdl_wait();
  __shared__ float tile[32][33];
  const int b = blockIdx.z;
  int R, C;
  mat_shape(b, H, d, m, R, C);
  const bool tall = R > C;
  const int64_t n = (int64_t)m * d;
  const float sc = 1.0f / (sqrtf(sum_parts(parts + b * NORM_PARTS)) + eps);
  const float* g = G + (int64_t)b * n;
  // the copy with G's layout: X (wide) or XT (tall); the transposed copy: the
  // other.  XT == nullptr: only X is written (the tensor-core iterations never
  // read XT).
  float* same = tall ? (XT ? XT + (int64_t)b * n : nullptr) : X + (int64_t)b * n;
  float* trans = tall ? X + (int64_t)b * n : (XT ? XT + (int64_t)b * n : nullptr);
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  if (r0 >= R || c0 >= C) return;
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int r = r0 + yy, c = c0 + threadIdx.x;
    float v = 0.f;
    if (r < R && c < C) {
      v = g[(int64_t)r * C + c] * sc;
      if (same) same[(int64_t)r * C + c] = v;
    }
    tile[yy][threadIdx.x] = v;
  }
  if (!trans) return;
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int c = c0 + yy, r = r0 + threadIdx.x;  // trans is (C x R)
    if (c < C && r < R) trans[(int64_t)c * R + r] = tile[threadIdx.x][yy];
  }
}

// ---- fp32 64x64 tile products of the Newton-Schulz iteration (CUDA cores)
//
// Every product is C = A B with both operands available as rows k: A^T rows
// (A^T [K][M]; for the Gram, X^T; for A A and B X, the symmetric left factor
// itself) and B rows ([K][N]).  A tile stages both [K][64] slabs (K <= NSC_KMAX
// at a time) in shared memory with 16-byte asynchronous copies, all in flight
// together, then each k step reads one float4 of A and one of B: 3 shared-memory
// wavefronts per warp per 16 FMAs, so the FMAs, not shared memory, set the pace.

constexpr int NSC_KMAX = 192;  // K extent staged in shared memory at once
// dynamic shared memory: A^T slab [NSC_KMAX][64] then B slab [NSC_KMAX][64]
constexpr int NSC_DYN_BYTES = 2 * NSC_KMAX * 64 * 4;

// 16-byte asynchronous global -> shared copy; src_bytes = 0 fills zeros
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

// rows k0 .. k0 + K - 1, columns c0 .. c0 + 63 of the row-major src (ld floats;
// columns >= Cv read as 0) into dst[k][64]
__device__ __forceinline__ void nsc_stage(const float* __restrict__ src, int ld, int c0, int Cv, int k0, int K,
                                          float* dst) {
  for (int idx = threadIdx.x; idx < K * 16; idx += 256) {
    const int k = idx >> 4, q = idx & 15;
    const bool in = c0 + 4 * q < Cv;
    cp_async16(dst + k * 64 + 4 * q, src + (int64_t)(k0 + k) * ld + (in ? c0 + 4 * q : 0), in ? 16u : 0u);
  }
}

// acc += sum over k < K of A(m0 + i, k0 + k) B(k0 + k, n0 + j) for the 64x64 tile, with
// at = A^T rows (lda; rows of length >= Mv) and b = B rows (ldb; length >= Nv).
// Thread (ty, tx) = (tid / 16, tid % 16) owns rows 4 ty .. 4 ty + 3 and columns
// 4 tx .. 4 tx + 3.  K <= NSC_KMAX; leading dimensions and column offsets are
// multiples of 4 floats.
__device__ __forceinline__ void nsc_tile(const float* __restrict__ at, int lda, int m0, int Mv,
                                         const float* __restrict__ b, int ldb, int n0, int Nv, int k0, int K,
                                         float (&acc)[4][4], float* smA, float* smB) {
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  __syncthreads();  // the previous tile's reads of smA / smB are done
  nsc_stage(at, lda, m0, Mv, k0, K, smA);
  nsc_stage(b, ldb, n0, Nv, k0, K, smB);
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();
#pragma unroll 8
  for (int k = 0; k < K; ++k) {
    const float4 av = *reinterpret_cast<const float4*>(smA + k * 64 + ty * 4);
    const float4 bv = *reinterpret_cast<const float4*>(smB + k * 64 + tx * 4);
    const float a4[4] = {av.x, av.y, av.z, av.w};
    const float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
  }
}

// Batched C = alpha S B + beta Cin with S symmetric (M x M, so the rows of S
// serve as rows of S^T), B [M][N] (ldb), one 64x64 output tile per CTA.  With
// CT != null the tile is also written transposed to CT [N][M] (through shared
// memory, so both stores are coalesced).  Dynamic shared memory: NSC_DYN_BYTES.
__global__ void __launch_bounds__(256) k_gemm_sym(int M, int N, const float* __restrict__ S, int64_t sS,
                                                  const float* __restrict__ B, int ldb, int64_t sB,
                                                  float* __restrict__ C, int ldc, int64_t sC, float* __restrict__ CT,
                                                  const float* __restrict__ Cin, float alpha, float beta) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) float gemm_dyn[];
  float* smA = gemm_dyn;
  float* smB = gemm_dyn + NSC_KMAX * 64;
  const int b = blockIdx.z;
  S += b * sS;
  B += b * sB;
  C += b * sC;
  if (CT) CT += b * sC;
  if (Cin) Cin += b * sC;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < M; k0 += NSC_KMAX)
    nsc_tile(S, M, m0, M, B, ldb, n0, N, k0, min(NSC_KMAX, M - k0), acc, smA, smB);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      float v = alpha * acc[i][j];
      if (Cin && gm < M && gn < N) v = fmaf(beta, Cin[(int64_t)gm * ldc + gn], v);
      acc[i][j] = v;
      if (gm < M && gn < N) C[(int64_t)gm * ldc + gn] = v;
    }
  if (CT) {
    float* tt = smA;  // [64][65]; the staging slabs are no longer read
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) tt[(tx * 4 + j) * 65 + ty * 4 + i] = acc[i][j];
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * 64; e += 256) {
      const int nn = e >> 6, mm = e & 63;  // CT row n0 + nn, column m0 + mm
      if (n0 + nn < N && m0 + mm < M) CT[(int64_t)(n0 + nn) * M + m0 + mm] = tt[nn * 65 + mm];
    }
  }
}

// Gram matrices A_b = X_b X_b^T from X^T (c x r, row-major): upper-triangular
// 64x64 tiles only (A is symmetric), split-K over NS_GRAM_SPLIT slices of the
// long dimension for parallelism.  grid (tiles, NS_GRAM_SPLIT, batch); partial
// P[s][b][i][j] for the tile's (i, j); k_gram_reduce sums the slices in fixed
// order and mirrors the lower triangle.  Dynamic shared memory: NSC_DYN_BYTES.
constexpr int NS_GRAM_SPLIT = 4;

__global__ void __launch_bounds__(256) k_gram_partial(int r, int c, const float* __restrict__ XT, int64_t sX,
                                                      float* __restrict__ P) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) float gram_dyn[];
  float* smA = gram_dyn;
  float* smB = gram_dyn + NSC_KMAX * 64;
  const int rt = (r + 63) / 64;
  // tile index -> (ti <= tj) in row-major upper-triangular order
  int t = blockIdx.x, ti = 0;
  while (t >= rt - ti) { t -= rt - ti; ++ti; }
  const int tj = ti + t;
  const int s = blockIdx.y, b = blockIdx.z;
  const int kper = ((c + NS_GRAM_SPLIT - 1) / NS_GRAM_SPLIT + 15) / 16 * 16;
  const int k_begin = s * kper, k_end = min(c, k_begin + kper);
  const float* xt = XT + (int64_t)b * sX;
  const int m0 = ti * 64, n0 = tj * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = k_begin; k0 < k_end; k0 += NSC_KMAX)
    nsc_tile(xt, r, m0, r, xt, r, n0, r, k0, min(NSC_KMAX, k_end - k0), acc, smA, smB);
  float* out = P + ((int64_t)s * gridDim.z + b) * (int64_t)r * r;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      if (gm < r && gn < r) out[(int64_t)gm * r + gn] = acc[i][j];
    }
}

// A[b][i][j] = sum_s P[s][b][min(i,j)][max(i,j)] over nsplit slices, in fixed order
__global__ void k_gram_reduce(int r, int nb, int nsplit, const float* __restrict__ P, float* __restrict__ A) {
  pdl_trigger();
  pdl_wait();
  const int64_t n = (int64_t)r * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * nb; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = e / n, ij = e % n;
    const int i = (int)(ij / r), j = (int)(ij % r);
    const int64_t src = b * n + (int64_t)min(i, j) * r + max(i, j);
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) acc += P[(int64_t)s * nb * n + src];
    A[e] = acc;
  }
}

// ---------------------------------------------------------------------------
// Muon weight step (ZipMap key design 3): W <- ||W|| (W - lr D) / ||W - lr D||,
// Delta in W's orientation: X_b (r x c) for a wide W_b, XT_b for a tall one
// (Dw = X, Dt = XT), or G itself when Newton-Schulz is off (Dw = Dt = G).

__device__ __forceinline__ float* mat_ptr(float* W1, float* W3, float* W2, int b, int H, int64_t n) {
  return b < H ? W1 + (int64_t)b * n : (b < 2 * H ? W3 + (int64_t)(b - H) * n : W2 + (int64_t)(b - 2 * H) * n);
}

// partials out[(b * NORM_PARTS + p) * 2 + {0,1}] of ||W_b||^2 and ||W_b - lr D_b||^2
__device__ __forceinline__ const float* delta_of(const float* Dw, const float* Dt, int b, int H, int d, int m) {
  int R, C;
  mat_shape(b, H, d, m, R, C);
  return (R > C ? Dt : Dw) + (int64_t)b * m * d;
}

__global__ void __launch_bounds__(256) k_step_partials(float* W1, float* W3, float* W2, const float* __restrict__ Dw,
                                                       const float* __restrict__ Dt, int H, int d, int m, float lr,
                                                       float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[9];
  const int b = blockIdx.x, p = blockIdx.y;
  const int64_t n = (int64_t)m * d, n4 = n / 4, per = (n4 + NORM_PARTS - 1) / NORM_PARTS;
  const int64_t i0 = p * per, i1 = min(n4, i0 + per);
  const float4* w = reinterpret_cast<const float4*>(mat_ptr(W1, W3, W2, b, H, n));
  const float4* dl = reinterpret_cast<const float4*>(delta_of(Dw, Dt, b, H, d, m));
  float s0 = 0.f, s1 = 0.f;
  for (int64_t i = i0 + threadIdx.x; i < i1; i += 256) {
    const float4 a = w[i], q = dl[i];
    const float u0 = a.x - lr * q.x, u1 = a.y - lr * q.y, u2 = a.z - lr * q.z, u3 = a.w - lr * q.w;
    s0 = fmaf(a.x, a.x, fmaf(a.y, a.y, fmaf(a.z, a.z, fmaf(a.w, a.w, s0))));
    s1 = fmaf(u0, u0, fmaf(u1, u1, fmaf(u2, u2, fmaf(u3, u3, s1))));
  }
  s0 = block_sum_256(s0, red);
  s1 = block_sum_256(s1, red);
  if (threadIdx.x == 0) {
    out[(b * NORM_PARTS + p) * 2] = s0;
    out[(b * NORM_PARTS + p) * 2 + 1] = s1;
  }
}

// W <- sc (W - lr D).  Skipped when the status word holds an error (a gradient
// out of range or a timed-out wait), so W is never overwritten with garbage.
__global__ void k_step_apply(float* W1, float* W3, float* W2, const float* __restrict__ Dw, const float* __restrict__ Dt,
                             int H, int d, int m, float lr, int renorm, const float* __restrict__ parts,
                             const unsigned int* status) {
  pdl_trigger();
  pdl_wait();
  if (*(volatile const unsigned int*)status != DEV_OK) return;
  const int b = blockIdx.y;
  const int64_t n = (int64_t)m * d, n4 = n / 4;
  float4* w = reinterpret_cast<float4*>(mat_ptr(W1, W3, W2, b, H, n));
  const float4* dl = reinterpret_cast<const float4*>(delta_of(Dw, Dt, b, H, d, m));
  float sc = 1.f;
  if (renorm) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int p = 0; p < NORM_PARTS; ++p) {
      s0 += parts[(b * NORM_PARTS + p) * 2];
      s1 += parts[(b * NORM_PARTS + p) * 2 + 1];
    }
    sc = s1 > 0.f ? sqrtf(s0) / sqrtf(s1) : 1.f;
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    float4 a = w[i];
    const float4 q = dl[i];
    a.x = sc * (a.x - lr * q.x);
    a.y = sc * (a.y - lr * q.y);
    a.z = sc * (a.z - lr * q.z);
    a.w = sc * (a.w - lr * q.w);
    w[i] = a;
  }
}

// ---------------------------------------------------------------------------
// fp32 mode: gradient of the dot-product loss on CUDA cores (exact fp32 math).
// grid (m/32 slices, H, S); each CTA owns 32 rows of m and accumulates
// g1, g3 (rows) and g2 (columns) for its token range in registers.

constexpr int F32_MS = 32, F32_TT = 32;

__global__ void __launch_bounds__(256) k_grad_f32(const float* __restrict__ K, int64_t ldk, const float* __restrict__ V,
                                                  int64_t ldv, const float* __restrict__ eta, const float* __restrict__ rk,
                                                  const float* __restrict__ W1, const float* __restrict__ W3,
                                                  const float* __restrict__ W2, float* __restrict__ partial, int64_t T,
                                                  int H, int d, int m, int S) {
  constexpr int MS = F32_MS, TT = F32_TT, NQ = MS * 256 / 256;  // d <= 256 -> MS*d/256 <= 32
  extern __shared__ float sm[];
  const int slice = blockIdx.x, h = blockIdx.y, split = blockIdx.z, tid = threadIdx.x;
  const int j0 = slice * MS;
  float* w1 = sm;
  float* w3 = w1 + MS * d;
  float* w2 = w3 + MS * d;  // [d][MS]
  float* kt = w2 + d * MS;  // [TT][d]
  float* vt = kt + TT * d;
  float* f1 = vt + TT * d;  // [TT][MS]
  float* f3 = f1 + TT * MS;
  float* fz = f3 + TT * MS;
  float* ee = fz + TT * MS;  // [TT]
  float* rr = ee + TT;       // [TT]
  for (int i = tid; i < MS * d; i += 256) {
    const int jj = i / d, kk = i % d;
    w1[i] = W1[((int64_t)h * m + j0 + jj) * d + kk];
    w3[i] = W3[((int64_t)h * m + j0 + jj) * d + kk];
  }
  for (int i = tid; i < d * MS; i += 256) {
    const int kk = i / MS, jj = i % MS;
    w2[i] = W2[((int64_t)h * d + kk) * m + j0 + jj];
  }
  float a1[NQ], a3[NQ], a2[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) a1[q] = a3[q] = a2[q] = 0.f;
  const int64_t tiles = (T + TT - 1) / TT;
  const int64_t tb = tiles * split / S, te = tiles * (split + 1) / S;
  const int nacc = MS * d;
  for (int64_t tile = tb; tile < te; ++tile) {
    const int64_t t0 = tile * TT;
    __syncthreads();
    for (int i = tid; i < TT * d; i += 256) {
      const int t = i / d, kk = i % d;
      const bool in = t0 + t < T;
      kt[i] = in ? K[(t0 + t) * ldk + (int64_t)h * d + kk] : 0.f;
      vt[i] = in ? V[(t0 + t) * ldv + (int64_t)h * d + kk] : 0.f;
    }
    if (tid < TT) {
      const bool in = t0 + tid < T;
      ee[tid] = in ? eta[(t0 + tid) * H + h] : 0.f;
      rr[tid] = in ? (rk ? rk[(t0 + tid) * H + h] : 1.f) : 0.f;
    }
    __syncthreads();
    for (int o = tid; o < 3 * TT * MS; o += 256) {
      const int mat = o / (TT * MS), rem = o % (TT * MS), t = rem / MS, j = rem % MS;
      float acc = 0.f;
      if (mat == 0) {
        for (int kk = 0; kk < d; ++kk) acc = fmaf(kt[t * d + kk], w1[j * d + kk], acc);
        f1[rem] = acc;
      } else if (mat == 1) {
        for (int kk = 0; kk < d; ++kk) acc = fmaf(kt[t * d + kk], w3[j * d + kk], acc);
        f3[rem] = acc;
      } else {
        for (int kk = 0; kk < d; ++kk) acc = fmaf(vt[t * d + kk], w2[kk * MS + j], acc);
        fz[rem] = acc;
      }
    }
    __syncthreads();
    for (int o = tid; o < TT * MS; o += 256) {
      const int t = o / MS;
      const float r = rr[t], e = ee[t];
      const float h1 = f1[o] * r, h3 = f3[o] * r, z = fz[o];
      const float s = 1.0f / (1.0f + expf(-h1));
      const float a = h1 * s, u = a * h3, du = -e * z;
      f1[o] = du * h3 * s * (1.0f + h1 * (1.0f - s)) * r;  // dL/dh1, chained to the raw key
      f3[o] = du * a * r;                                   // dL/dh3
      fz[o] = -e * u;                                       // -eta u, the g2 factor
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + 256 * q;
      if (e < nacc) {
        const int jj = e / d, kk = e % d;
        float s1 = a1[q], s3 = a3[q];
        for (int t = 0; t < TT; ++t) {
          const float kv = kt[t * d + kk];
          s1 = fmaf(f1[t * MS + jj], kv, s1);
          s3 = fmaf(f3[t * MS + jj], kv, s3);
        }
        a1[q] = s1;
        a3[q] = s3;
        const int kk2 = e / MS, jj2 = e % MS;
        float s2 = a2[q];
        for (int t = 0; t < TT; ++t) s2 = fmaf(vt[t * d + kk2], fz[t * MS + jj2], s2);
        a2[q] = s2;
      }
    }
  }
  const int64_t n = (int64_t)m * d;
  float* p1 = partial + ((int64_t)split * 3 + 0) * H * n + (int64_t)h * n;
  float* p3 = partial + ((int64_t)split * 3 + 1) * H * n + (int64_t)h * n;
  float* p2 = partial + ((int64_t)split * 3 + 2) * H * n + (int64_t)h * n;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = tid + 256 * q;
    if (e < nacc) {
      const int jj = e / d, kk = e % d;
      p1[(int64_t)(j0 + jj) * d + kk] = a1[q];
      p3[(int64_t)(j0 + jj) * d + kk] = a3[q];
      const int kk2 = e / MS, jj2 = e % MS;
      p2[(int64_t)kk2 * m + j0 + jj2] = a2[q];
    }
  }
}

// fp32 mode apply: grid (ceil(T/32), H); O[t] = W2 (SiLU(W1 q^) o (W3 q^)).
__global__ void __launch_bounds__(256) k_apply_f32(const float* __restrict__ Q, int64_t ldq, const float* __restrict__ rq,
                                                   const float* __restrict__ W1, const float* __restrict__ W3,
                                                   const float* __restrict__ W2, float* __restrict__ O, int64_t ldo,
                                                   int64_t T, int H, int d, int m) {
  constexpr int TT = F32_TT, MC = F32_MS, NQ = 32;  // TT*d/256 <= 32
  extern __shared__ float sm[];
  const int h = blockIdx.y, tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  float* qt = sm;             // [TT][d]
  float* w1 = qt + TT * d;    // [MC][d]
  float* w3 = w1 + MC * d;    // [MC][d]
  float* w2 = w3 + MC * d;    // [d][MC]
  float* p = w2 + d * MC;     // [TT][MC]
  float* rr = p + TT * MC;    // [TT]
  for (int i = tid; i < TT * d; i += 256) {
    const int t = i / d, kk = i % d;
    qt[i] = (t0 + t < T) ? Q[(t0 + t) * ldq + (int64_t)h * d + kk] : 0.f;
  }
  if (tid < TT) rr[tid] = (t0 + tid < T) ? (rq ? rq[(t0 + tid) * H + h] : 1.f) : 0.f;
  float acc[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) acc[q] = 0.f;
  const int nacc = TT * d;
  for (int mc = 0; mc < m; mc += MC) {
    __syncthreads();
    for (int i = tid; i < MC * d; i += 256) {
      const int jj = i / d, kk = i % d;
      w1[i] = W1[((int64_t)h * m + mc + jj) * d + kk];
      w3[i] = W3[((int64_t)h * m + mc + jj) * d + kk];
    }
    for (int i = tid; i < d * MC; i += 256) {
      const int kk = i / MC, jj = i % MC;
      w2[i] = W2[((int64_t)h * d + kk) * m + mc + jj];
    }
    __syncthreads();
    for (int o = tid; o < TT * MC; o += 256) {
      const int t = o / MC, j = o % MC;
      float h1 = 0.f, h3 = 0.f;
      for (int kk = 0; kk < d; ++kk) {
        h1 = fmaf(qt[t * d + kk], w1[j * d + kk], h1);
        h3 = fmaf(qt[t * d + kk], w3[j * d + kk], h3);
      }
      h1 *= rr[t];
      h3 *= rr[t];
      p[o] = h1 / (1.0f + expf(-h1)) * h3;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + 256 * q;
      if (e < nacc) {
        const int t = e / d, kk = e % d;
        float s = acc[q];
        for (int j = 0; j < MC; ++j) s = fmaf(p[t * MC + j], w2[kk * MC + j], s);
        acc[q] = s;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = tid + 256 * q;
    if (e < nacc) {
      const int t = e / d, kk = e % d;
      if (t0 + t < T) O[(t0 + t) * ldo + (int64_t)h * d + kk] = acc[q];
    }
  }
}

// ---------------------------------------------------------------------------
// Timeout-path diagnostic: wait on a barrier that is initialised for one arrival
// that never comes.  The bounded wait records DEV_TIMEOUT and the kernel returns.
__global__ void k_selftest_wait(unsigned int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const Guard g{status, timeout_ns};
  const bool ok = mbar_wait(&bar, 0, g);
  (void)__all_sync(0xffffffffu, ok);
}

}  // namespace ttt
