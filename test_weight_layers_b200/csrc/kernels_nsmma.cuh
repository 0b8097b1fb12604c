// Tensor-core products of the Newton-Schulz iteration (bf16 mode).
//
// The iteration needs near-fp32 products: an fp16 Newton-Schulz left 3.9%
// error after 16 chained chunks.  Each fp32 operand x is split into two bf16
// parts, hi = bf16(x) and lo = bf16(x - hi), and a product is accumulated in
// fp32 TMEM as hi*hi + hi*lo + lo*hi (the lo*lo term and the rounding of lo are
// ~2^-16 relative), three kind::f16 MMAs per k step.
//
// C = alpha A B + beta Cin for one 128 x NT output tile per CTA, A fp32 row-major
// [M][lda] (K-major), B either as B^T rows (BK: fp32 row-major [N][ldb], K-major)
// or as B rows (fp32 row-major [K][ldb], MN-major).  K is walked in chunks of 64
// staged by all threads (load, split, store into 128-byte-swizzled layouts),
// double-buffered so chunk c+1 is staged while chunk c's MMAs run.  Split-K:
// grid z = batch * nsplit, split s covers K [s ksplit, (s+1) ksplit) and writes
// C + s sCsplit.
#pragma once

#include "common.cuh"

namespace ttt {

constexpr int NSM_KC = 64;  // K elements per staged chunk
constexpr int NSM_THREADS = 256;
constexpr int NSM_GRAM_SPLIT_MAX = 8;  // split-K slices of the Gram products (K chunks of >= 128)

template <int NT>
struct NsmLayout {
  static constexpr int A_BYTES = 128 * NSM_KC * 2;  // one bf16 part of the A chunk
  static constexpr int B_BYTES = NT * NSM_KC * 2;   // one bf16 part of the B chunk
  static constexpr int STAGE = 2 * A_BYTES + 2 * B_BYTES;
  static constexpr int BAR_OFF = 2 * STAGE;
  static constexpr int ALLOC = BAR_OFF + 64 + 1024;
  static constexpr int TMEM_COLS = NT <= 64 ? 64 : (NT <= 128 ? 128 : 256);
  static constexpr int TILE_LD = NT + 4;  // fp32 epilogue tile [128][NT + 4] over the stages
  static_assert(128 * TILE_LD * 4 <= BAR_OFF, "epilogue tile fits the staging buffers");
  static_assert(NT % 64 == 0 && NT <= 256 && (NT * 8) % NSM_THREADS == 0, "N tile");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

// 8 consecutive fp32 values -> 16 bytes of bf16 hi and 16 bytes of bf16 lo parts
__device__ __forceinline__ void nsm_split8(const float4 u, const float4 v, uint4& hi, uint4& lo) {
  const float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const float2 hf = __bfloat1622float2(hh);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
    h[i] = *reinterpret_cast<const uint32_t*>(&hh);
    l[i] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void nsm_load8(const float* p, bool in, float4& u, float4& v) {
  if (in) {
    u = *reinterpret_cast<const float4*>(p);
    v = *reinterpret_cast<const float4*>(p + 4);
  } else {
    u = make_float4(0.f, 0.f, 0.f, 0.f);
    v = u;
  }
}

template <int NT, bool BK>
__global__ void __launch_bounds__(NSM_THREADS, 1)
    k_mm3(int M, int N, int K, int ksplit, int nsplit, const float* __restrict__ A, int lda, int64_t sA,
          const float* __restrict__ B, int ldb, int64_t sB, float* __restrict__ C, int ldc, int64_t sC,
          int64_t sCsplit, const float* __restrict__ Cin, float alpha, float beta, unsigned int* status,
          unsigned long long timeout_ns) {
  using L = NsmLayout<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);  // [2] MMAs of a stage complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z / nsplit, s = blockIdx.z % nsplit;
  const int m0 = blockIdx.y * 128, n0 = blockIdx.x * NT;
  const int k_begin = s * ksplit, k_end = min(K, k_begin + ksplit);
  const int nch = max(0, (k_end - k_begin + NSM_KC - 1) / NSM_KC);
  A += b * sA;
  B += b * sB;
  C += b * sC + s * sCsplit;
  if (Cin) Cin += b * sC;

  if (tid == 0) {
    mbar_init(done, 1);
    mbar_init(done + 1, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // operands come from the previous kernel on the stream
  const Guard g{status, timeout_ns};
  constexpr uint32_t ID = idesc_bf16(128, NT, false, !BK);
  bool ok = true;

  for (int ch = 0; ch < nch; ++ch) {
    const int st = ch & 1;
    // the stage is free once the MMAs of chunk ch - 2 are done
    if (ch >= 2) ok &= __syncthreads_and(mbar_wait(done + st, ((ch - 2) >> 1) & 1, g));
    uint8_t* sa = smem + st * L::STAGE;  // A hi, A lo, B hi, B lo
    uint8_t* sb = sa + 2 * L::A_BYTES;
    const int k0 = k_begin + ch * NSM_KC;
    // all loads of the chunk are issued before any split/store so their
    // latencies overlap: A 128 rows x 64 k, B NT x 64 (8 floats per item)
    constexpr int A_IT = 128 * 8 / NSM_THREADS, B_IT = NT * 8 / NSM_THREADS;
    float4 au[A_IT], av[A_IT], bu[B_IT], bv[B_IT];
#pragma unroll
    for (int i = 0; i < A_IT; ++i) {
      const int idx = tid + i * NSM_THREADS, r = idx >> 3, kk = k0 + (idx & 7) * 8;
      nsm_load8(A + (int64_t)(m0 + r) * lda + kk, m0 + r < M && kk < k_end, au[i], av[i]);
    }
#pragma unroll
    for (int i = 0; i < B_IT; ++i) {
      const int idx = tid + i * NSM_THREADS;
      if (BK) {
        // B^T rows: NT rows x 64 k
        const int r = idx >> 3, kk = k0 + (idx & 7) * 8;
        nsm_load8(B + (int64_t)(n0 + r) * ldb + kk, n0 + r < N && kk < k_end, bu[i], bv[i]);
      } else {
        // B rows: 64 k x NT n
        const int kr = idx / (NT / 8), nn = (idx % (NT / 8)) * 8;
        nsm_load8(B + (int64_t)(k0 + kr) * ldb + n0 + nn, k0 + kr < k_end && n0 + nn < N, bu[i], bv[i]);
      }
    }
    // A -> [128][64] K-major, 128-byte swizzle (hi part, then lo part)
#pragma unroll
    for (int i = 0; i < A_IT; ++i) {
      const int idx = tid + i * NSM_THREADS;
      uint4 hi, lo;
      nsm_split8(au[i], av[i], hi, lo);
      const uint32_t off = sw128_offset(idx >> 3, idx & 7);
      *reinterpret_cast<uint4*>(sa + off) = hi;
      *reinterpret_cast<uint4*>(sa + L::A_BYTES + off) = lo;
    }
    // B -> [NT][64] K-major (BK) or NT/64 MN-major blocks [64 k][64 n]
#pragma unroll
    for (int i = 0; i < B_IT; ++i) {
      const int idx = tid + i * NSM_THREADS;
      uint4 hi, lo;
      nsm_split8(bu[i], bv[i], hi, lo);
      uint32_t off;
      if (BK) {
        off = sw128_offset(idx >> 3, idx & 7);
      } else {
        const int kr = idx / (NT / 8), nn = (idx % (NT / 8)) * 8;
        off = (nn >> 6) * (NSM_KC * 128) + sw128_offset(kr, (nn & 63) >> 3);
      }
      *reinterpret_cast<uint4*>(sb + off) = hi;
      *reinterpret_cast<uint4*>(sb + L::B_BYTES + off) = lo;
    }
    fence_async_smem();
    __syncthreads();
    if (warp == 0 && elect_one()) {
      tc_fence_after();
      const uint64_t dah = sdesc_sw128(smem_u32(sa), 16, 1024);
      const uint64_t dal = sdesc_sw128(smem_u32(sa + L::A_BYTES), 16, 1024);
      const uint64_t dbh = BK ? sdesc_sw128(smem_u32(sb), 16, 1024) : sdesc_sw128(smem_u32(sb), NSM_KC * 128, 1024);
      const uint64_t dbl = BK ? sdesc_sw128(smem_u32(sb + L::B_BYTES), 16, 1024)
                              : sdesc_sw128(smem_u32(sb + L::B_BYTES), NSM_KC * 128, 1024);
#pragma unroll
      for (int j = 0; j < NSM_KC / 16; ++j) {
        // k step j: K-major operands advance 32 bytes, MN-major ones 16 rows (2048 bytes)
        const uint64_t ao = (uint64_t)(j * 32 / 16), bo = BK ? (uint64_t)(j * 32 / 16) : (uint64_t)(j * 2048 / 16);
        umma_bf16_ss(tmem, dah + ao, dbh + bo, ID, (ch > 0 || j > 0) ? 1u : 0u);
        umma_bf16_ss(tmem, dah + ao, dbl + bo, ID, 1u);
        umma_bf16_ss(tmem, dal + ao, dbh + bo, ID, 1u);
      }
      umma_commit(done + st);
    }
  }
  pdl_trigger();
  if (nch > 0) ok &= __syncthreads_and(mbar_wait(done + ((nch - 1) & 1), ((nch - 1) >> 1) & 1, g));
  tc_fence_after();
  // epilogue: warp w reads TMEM lanes 32 (w % 4) (rows) and half w / 4 of the
  // columns into an fp32 tile in the (now idle) staging buffers.  Row stride
  // NT + 4 floats: a row starts 16 bytes past a bank-group boundary, so the
  // 16-byte writes of 8 consecutive rows and the 16-byte reads along a row are
  // both conflict-free.  The tile then leaves row by row with coalesced 16-byte
  // loads of Cin and stores of C (N, ldc and n0 are multiples of 4).
  float* tile = reinterpret_cast<float*>(smem);
  if (ok) {
    const int q = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    float* trow = tile + (q * 32 + lane) * L::TILE_LD;
    for (int c0 = half * (NT / 2); c0 < (half + 1) * (NT / 2); c0 += 32) {
      uint32_t v[32];
      if (nch > 0) {
        tmem_ld32(tmem + lane_base + c0, v);
        tmem_ld_wait(v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(trow + c0 + j) = make_float4(
            __uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    }
  }
  __syncthreads();
  if (ok) {
    constexpr int V_ROW = NT / 4, V_IT = 128 * V_ROW / NSM_THREADS, BATCH = V_IT <= 16 ? V_IT : V_IT / 2;
    static_assert(V_IT % BATCH == 0, "epilogue batches");
    for (int i0 = 0; i0 < V_IT; i0 += BATCH) {
      float4 cin[BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int idx = tid + (i0 + i) * NSM_THREADS, r = idx / V_ROW, n = n0 + (idx % V_ROW) * 4;
        cin[i] = (Cin && m0 + r < M && n < N) ? *reinterpret_cast<const float4*>(Cin + (int64_t)(m0 + r) * ldc + n)
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int idx = tid + (i0 + i) * NSM_THREADS, r = idx / V_ROW, cv = idx % V_ROW, n = n0 + cv * 4;
        if (m0 + r < M && n < N) {
          const float4 t = *reinterpret_cast<const float4*>(tile + r * L::TILE_LD + cv * 4);
          float4 o;
          o.x = fmaf(beta, cin[i].x, alpha * t.x);
          o.y = fmaf(beta, cin[i].y, alpha * t.y);
          o.z = fmaf(beta, cin[i].z, alpha * t.z);
          o.w = fmaf(beta, cin[i].w, alpha * t.w);
          *reinterpret_cast<float4*>(C + (int64_t)(m0 + r) * ldc + n) = o;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// XT_b = X_b^T for the batch (X_b r x c row-major); grid (ceil(c/32), ceil(r/32), batch), block (32, 8)
__global__ void k_transpose_batch(const float* __restrict__ X, float* __restrict__ XT, int r, int c, int64_t sX) {
  __shared__ float tile[32][33];
  pdl_trigger();
  pdl_wait();
  const float* x = X + (int64_t)blockIdx.z * sX;
  float* xt = XT + (int64_t)blockIdx.z * sX;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int i = r0 + yy, j = c0 + threadIdx.x;
    tile[yy][threadIdx.x] = (i < r && j < c) ? x[(int64_t)i * c + j] : 0.f;
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int j = c0 + yy, i = r0 + threadIdx.x;
    if (j < c && i < r) xt[(int64_t)j * r + i] = tile[threadIdx.x][yy];
  }
}

}  // namespace ttt
