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

// ---------------------------------------------------------------------------
// The whole Newton-Schulz loop of one matrix in one launch (bf16 mode).
//
// The quintic's coefficients (a, b, c) are na, nb_, nc here (c is the column
// count).  A cluster of CS = c / 128 CTAs per matrix; CTA j owns columns
// [128 j, 128 j + 128) of the wide iterate X (R x c, R in {128, 192}), which is
// updated in place in global memory.  With A = X X^T kept in global memory
// (R x R), one iteration is, in every CTA:
//   1. B = nc A A^T + nb_ A, computed whole by each CTA (K = R, both operands
//      are A's rows, resident in shared memory; A is symmetric up to rounding);
//   2. X_j <- B X_j + na X_j for its own columns (K = R in 64-row chunks
//      through two staging buffers; the first two are staged while step 1's
//      MMAs run);
//   3. unless it is the last iteration: P_j = X_j X_j^T (K = 128) into an fp32
//      shared tile; cluster barrier; CTA j sums the rows i = j (mod CS) of
//      A = sum_q P_q over q = 0..CS-1 in that fixed order, reading the other
//      CTAs' tiles through distributed shared memory, and writes them; cluster
//      barrier.
// Step 3 also runs once on X_0 before the first iteration.  Products use split
// bf16 operands (hi*hi + hi*lo + lo*hi, fp32 accumulation in TMEM) as in k_mm3.
// M tiles of 128 rows: rows 0..127 and, for R = 192, rows 64..191 (of the second
// tile only rows 128..191 are kept).  All threads stage operands; one elected
// thread issues the MMAs; every CTA runs the same sequence of cluster barriers
// whatever happens, so a failed wait (recorded in the status word) never
// leaves a peer waiting at a barrier.

constexpr int NSC_THREADS = 256;
constexpr int NSC_COLS = 128;  // columns of X per CTA

template <int R>
struct NscLayout {
  static constexpr int KB = R / 64;                          // 64-wide K blocks of an R-wide operand
  static constexpr int ROWBLK = R * 128;                     // one [R rows][64 bf16] K block, 128-byte swizzle
  static constexpr int PART = KB * ROWBLK;                   // one bf16 part (hi or lo) of an R x R operand
  static constexpr int P_LD = R + 4;                         // fp32 P tile row stride (floats)
  static constexpr int OPS = 2 * PART > R * P_LD * 4 ? 2 * PART : R * P_LD * 4;
  static constexpr int OPA_BYTES = (OPS + 1023) / 1024 * 1024;
  static constexpr int XCH = 64 * NSC_COLS * 2;              // one part of an X chunk: 2 MN blocks [64 k][64 n]
  static constexpr int XSTAGE = 2 * XCH;                     // hi + lo
  static constexpr int XST_OFF = OPA_BYTES;
  static constexpr int BAR_OFF = XST_OFF + 2 * XSTAGE;
  static constexpr int ALLOC = BAR_OFF + 64 + 1024;
  static constexpr int NMT = R == 192 ? 2 : 1;               // M tiles
  static_assert(8 * 32 * 36 * 4 <= 2 * XSTAGE, "transpose buffers fit the X stages");
  static_assert(R == 128 || R == 192, "rows");
  static_assert(ALLOC <= 232448, "shared memory budget");
  static_assert(NMT * R <= 512, "TMEM budget");
};

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// 32 consecutive fp32 values (one row, from registers) -> bf16 hi/lo parts of a
// K-major operand: columns col0..col0+31 of row `row` (col0 a multiple of 32)
template <int ROWBLK, int PART>
__device__ __forceinline__ void nsc_put_row32(uint8_t* op, int row, int col0, const float* x) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int col = col0 + 8 * c;
    uint4 hi, lo;
    nsm_split8(make_float4(x[8 * c], x[8 * c + 1], x[8 * c + 2], x[8 * c + 3]),
               make_float4(x[8 * c + 4], x[8 * c + 5], x[8 * c + 6], x[8 * c + 7]), hi, lo);
    const uint32_t off = (col >> 6) * ROWBLK + sw128_offset(row, (col & 63) >> 3);
    *reinterpret_cast<uint4*>(op + off) = hi;
    *reinterpret_cast<uint4*>(op + PART + off) = lo;
  }
}

// 8 floats through L2 (data written by other CTAs of the cluster in this kernel)
__device__ __forceinline__ void nsc_load8_cg(const float* p, float4& u, float4& v) {
  u = __ldcg(reinterpret_cast<const float4*>(p));
  v = __ldcg(reinterpret_cast<const float4*>(p + 4));
}

// inverse of nsc_put_row32: hi + lo of columns col0..col0+31 of row `row`
template <int ROWBLK, int PART>
__device__ __forceinline__ void nsc_get_row32(const uint8_t* op, int row, int col0, float* x) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int col = col0 + 8 * c;
    const uint32_t off = (col >> 6) * ROWBLK + sw128_offset(row, (col & 63) >> 3);
    const uint4 hi = *reinterpret_cast<const uint4*>(op + off);
    const uint4 lo = *reinterpret_cast<const uint4*>(op + PART + off);
    const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w}, lw[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 h2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[e]));
      const float2 l2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[e]));
      x[8 * c + 2 * e] = h2.x + l2.x;
      x[8 * c + 2 * e + 1] = h2.y + l2.y;
    }
  }
}

template <int R>
__global__ void __launch_bounds__(NSC_THREADS, 1)
    k_ns_cluster(float* X, float* A, int c, int iters, float na, float nb_, float nc,
                 unsigned int* status, unsigned long long timeout_ns) {
  using L = NscLayout<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* opa = smem;                   // K-major operands (hi part, then lo part) / fp32 P tile
  uint8_t* xst = smem + L::XST_OFF;      // [2] X chunk stages (MN-major, hi then lo)
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);  // MMAs of a phase complete
  uint64_t* xbar = mbar + 1;                                        // [2] MMAs of an X stage complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 2);
  float* ptile = reinterpret_cast<float*>(opa);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CS = (int)gridDim.x;  // cluster = the CTAs of one matrix
  const int j = (int)cluster_ctarank();
  const int b = blockIdx.y;
  X += (int64_t)b * R * c;
  A += (int64_t)b * R * R;
  const int col_base = j * NSC_COLS;
  pdl_trigger();

  if (tid == 0) {
    mbar_init(mbar, 1);
    mbar_init(xbar, 1);
    mbar_init(xbar + 1, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // X comes from the previous kernel on the stream
  const Guard g{status, timeout_ns};
  bool ok = true;
  uint32_t mph = 0, xph0 = 0, xph1 = 0;
  const bool issuer = warp == 0;
  const uint64_t d_oh = sdesc_sw128(smem_u32(opa), 16, 1024);
  const uint64_t d_ol = sdesc_sw128(smem_u32(opa + L::PART), 16, 1024);
  constexpr uint32_t ID_RR = idesc_bf16(128, R, false, false);         // B = A A^T, P = X X^T
  constexpr uint32_t ID_BX = idesc_bf16(128, NSC_COLS, false, true);   // B X (X chunk MN-major)
  const int q = warp & 3, half = warp >> 2;
  const uint32_t lane_base = (uint32_t)(q * 32) << 16;

  // wait for the MMAs committed to `bar` (all threads; uniform result)
  auto wait_bar = [&](uint64_t* bar, uint32_t& ph) {
    const bool w = ok ? mbar_wait(bar, ph, g) : false;
    ph ^= 1u;
    ok = __syncthreads_and(w ? 1 : 0) != 0 && ok;
    tc_fence_after();
  };
  // three MMAs of one split product k step
  auto mma3 = [&](uint32_t d, uint64_t ah, uint64_t al, uint64_t bh, uint64_t bl, uint32_t id, uint32_t acc) {
    umma_bf16_ss(d, ah, bh, id, acc);
    umma_bf16_ss(d, ah, bl, id, 1u);
    umma_bf16_ss(d, al, bh, id, 1u);
  };
  // rows of M tile t held by TMEM lane quarter q: tile 0 all, tile 1 (R = 192) quarters 2, 3 (rows 128..191)
  auto tile_row = [&](int t) { return t == 0 ? q * 32 + lane : 64 + q * 32 + lane; };
  auto tile_has = [&](int t) { return t == 0 || q >= 2; };

  // Gram of the CTA's columns from the operand in `opa` (K-major [R][128]) into
  // the fp32 tile, then the cluster reduction of A's rows
  auto gram_and_reduce = [&]() {
    fence_async_smem();
    __syncthreads();
    if (ok && issuer) {
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int t = 0; t < L::NMT; ++t)
#pragma unroll
          for (int kb = 0; kb < NSC_COLS / 64; ++kb)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              const uint32_t ao = (uint32_t)(kb * L::ROWBLK + t * 64 * 128 + s * 32) >> 4;
              const uint32_t bo = (uint32_t)(kb * L::ROWBLK + s * 32) >> 4;
              mma3(tmem + t * R, d_oh + ao, d_ol + ao, d_oh + bo, d_ol + bo, ID_RR, (kb | s) ? 1u : 0u);
            }
        umma_commit(mbar);
      }
      __syncwarp();
    }
    wait_bar(mbar, mph);
    // TMEM -> fp32 tile [R][P_LD] (the operands are no longer needed)
#pragma unroll
    for (int t = 0; t < L::NMT; ++t) {
      if (!tile_has(t)) continue;
      const int row = tile_row(t);
      for (int c0 = half * (R / 2); c0 < (half + 1) * (R / 2); c0 += 32) {
        uint32_t v[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + t * R + c0, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        float* dst = ptile + row * L::P_LD + c0;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                            __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
      }
    }
    tc_fence_before();
    cluster_sync_all();  // every CTA's P tile is complete
    // rows i = j (mod CS): A[i][:] = sum_q P_q[i][:], q in order
    {
      // two items per thread at a time, the CS partial tiles of both in flight at once
      constexpr int V4 = R / 4;
      const int nrows = (R - j + CS - 1) / CS;
      const int items = nrows * V4;
      for (int idx0 = tid; idx0 < items; idx0 += 2 * NSC_THREADS) {
        float4 pv[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = idx0 + u * NSC_THREADS;
          const int i = j + (idx / V4) * CS, c4 = idx % V4;
          const float* src = ptile + (idx < items ? i * L::P_LD + c4 * 4 : 0);
#pragma unroll
          for (int qq = 0; qq < 8; ++qq)
            if (qq < CS) pv[u][qq] = ld_cluster_f4(cluster_addr(src, (uint32_t)qq));
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = idx0 + u * NSC_THREADS;
          if (idx >= items) continue;
          float4 acc = pv[u][0];
#pragma unroll
          for (int qq = 1; qq < 8; ++qq)
            if (qq < CS) {
              acc.x += pv[u][qq].x;
              acc.y += pv[u][qq].y;
              acc.z += pv[u][qq].z;
              acc.w += pv[u][qq].w;
            }
          const int i = j + (idx / V4) * CS, c4 = idx % V4;
          *reinterpret_cast<float4*>(A + (int64_t)i * R + c4 * 4) = acc;
        }
      }
    }
    cluster_sync_all();  // A complete (global writes released to the cluster), peers done with the tiles
    tc_fence_after();
  };

  // X rows [64 kc, 64 kc + 64) of the CTA's columns -> stage st (MN-major [64 k][128 n], hi then lo)
  auto stage_x = [&](int kc, int st) {
    uint8_t* xs = xst + st * L::XSTAGE;
    constexpr int ITEMS = 64 * (NSC_COLS / 8), IT = ITEMS / NSC_THREADS;
    float4 u[IT], v[IT];
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const int idx = tid + i * NSC_THREADS, kr = idx >> 4, c8 = idx & 15;
      nsm_load8(X + (int64_t)(kc * 64 + kr) * c + col_base + c8 * 8, true, u[i], v[i]);
    }
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const int idx = tid + i * NSC_THREADS, kr = idx >> 4, c8 = idx & 15;
      uint4 hi, lo;
      nsm_split8(u[i], v[i], hi, lo);
      const uint32_t off = (c8 >> 3) * (64 * 128) + sw128_offset(kr, c8 & 7);
      *reinterpret_cast<uint4*>(xs + off) = hi;
      *reinterpret_cast<uint4*>(xs + L::XCH + off) = lo;
    }
  };

  // ---- X_0: Gram operand from global (rows 0..R-1, the CTA's 128 columns)
  {
    constexpr int ITEMS = R * (NSC_COLS / 8), BATCH = (ITEMS / NSC_THREADS) % 6 == 0 ? 6 : 4;
    static_assert(ITEMS % (NSC_THREADS * BATCH) == 0, "staging batches");
    for (int i0 = 0; i0 < ITEMS / NSC_THREADS; i0 += BATCH) {
      float4 u[BATCH], v[BATCH];
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int idx = tid + (i0 + i) * NSC_THREADS, row = idx >> 4, c8 = idx & 15;
        nsm_load8(X + (int64_t)row * c + col_base + c8 * 8, true, u[i], v[i]);
      }
#pragma unroll
      for (int i = 0; i < BATCH; ++i) {
        const int idx = tid + (i0 + i) * NSC_THREADS, row = idx >> 4, c8 = idx & 15;
        uint4 hi, lo;
        nsm_split8(u[i], v[i], hi, lo);
        const uint32_t off = (c8 >> 3) * L::ROWBLK + sw128_offset(row, c8 & 7);
        *reinterpret_cast<uint4*>(opa + off) = hi;
        *reinterpret_cast<uint4*>(opa + L::PART + off) = lo;
      }
    }
  }
  gram_and_reduce();

  for (int it = 0; it < iters; ++it) {
    const bool last = it + 1 == iters;
    // ---- 1. B = nc A A^T + nb A
    {
      constexpr int ITEMS = R * (R / 8), BATCH = (ITEMS / NSC_THREADS) % 6 == 0 ? 6 : 4;
      static_assert(ITEMS % (NSC_THREADS * BATCH) == 0, "staging batches");
      for (int i0 = 0; i0 < ITEMS / NSC_THREADS; i0 += BATCH) {
        float4 u[BATCH], v[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int idx = tid + (i0 + i) * NSC_THREADS, row = idx / (R / 8), c8 = idx % (R / 8);
          nsc_load8_cg(A + (int64_t)row * R + c8 * 8, u[i], v[i]);
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const int idx = tid + (i0 + i) * NSC_THREADS, row = idx / (R / 8), c8 = idx % (R / 8);
          uint4 hi, lo;
          nsm_split8(u[i], v[i], hi, lo);
          const uint32_t off = (c8 >> 3) * L::ROWBLK + sw128_offset(row, c8 & 7);
          *reinterpret_cast<uint4*>(opa + off) = hi;
          *reinterpret_cast<uint4*>(opa + L::PART + off) = lo;
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (ok && issuer) {
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int t = 0; t < L::NMT; ++t)
#pragma unroll
          for (int kb = 0; kb < L::KB; ++kb)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              const uint32_t ao = (uint32_t)(kb * L::ROWBLK + t * 64 * 128 + s * 32) >> 4;
              const uint32_t bo = (uint32_t)(kb * L::ROWBLK + s * 32) >> 4;
              mma3(tmem + t * R, d_oh + ao, d_ol + ao, d_oh + bo, d_ol + bo, ID_RR, (kb | s) ? 1u : 0u);
            }
        umma_commit(mbar);
      }
      __syncwarp();
    }
    // the first two X chunks of step 2 do not depend on B: stage them while the MMAs run
    // (the stages' previous MMAs completed before the last iteration's epilogue)
    stage_x(0, 0);
    if (L::KB > 1) stage_x(1, 1);
    wait_bar(mbar, mph);
    // B rows -> K-major operand in place of A's.  The b A term takes A = hi + lo
    // (within 2^-17 relative) from the operand itself: each thread reads exactly
    // the entries it then overwrites.
#pragma unroll
    for (int t = 0; t < L::NMT; ++t) {
      if (!tile_has(t)) continue;
      const int row = tile_row(t);
      for (int c0 = half * (R / 2); c0 < (half + 1) * (R / 2); c0 += 32) {
        float x[32];
        nsc_get_row32<L::ROWBLK, L::PART>(opa, row, c0, x);
        uint32_t v[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + t * R + c0, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = fmaf(nb_, x[e], nc * __uint_as_float(v[e]));
        nsc_put_row32<L::ROWBLK, L::PART>(opa, row, c0, x);
      }
    }
    tc_fence_before();
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    // ---- 2. X_j <- B X_j + a X_j: X rows in 64-row chunks (MN-major [64 k][128 n]) through two stages
#pragma unroll 1
    for (int kc = 0; kc < L::KB; ++kc) {
      const int st = kc & 1;
      uint8_t* xs = xst + st * L::XSTAGE;
      if (kc >= 2) {
        wait_bar(xbar + st, st ? xph1 : xph0);  // chunk kc - 2's MMAs released the stage
        stage_x(kc, st);
        fence_async_smem();
        __syncthreads();
      }
      if (ok && issuer) {
        tc_fence_after();
        if (elect_one()) {
          const uint64_t d_xh = sdesc_sw128(smem_u32(xs), 64 * 128, 1024);
          const uint64_t d_xl = sdesc_sw128(smem_u32(xs + L::XCH), 64 * 128, 1024);
#pragma unroll
          for (int t = 0; t < L::NMT; ++t)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              const uint32_t ao = (uint32_t)(kc * L::ROWBLK + t * 64 * 128 + s * 32) >> 4;
              const uint32_t bo = (uint32_t)(s * 2048) >> 4;
              mma3(tmem + t * NSC_COLS, d_oh + ao, d_ol + ao, d_xh + bo, d_xl + bo, ID_BX, (kc | s) ? 1u : 0u);
            }
          umma_commit(xbar + st);
        }
        __syncwarp();
      }
    }
    // The a X term: X is read in 32 x 32 blocks with coalesced 16-byte loads
    // (lane -> row 4k + lane / 8, columns 4 (lane % 8)) and turned into rows
    // through the warp's transpose buffer; X' leaves the same way.  Buffer row
    // stride 36 floats: conflict-free in both directions.  The first block's
    // loads are issued while the MMAs finish.
    auto load_blk = [&](int t, int c0, float4 (&xl)[8]) {
      const int rbase = tile_row(t) - lane;  // first row of this warp's 32
#pragma unroll
      for (int k = 0; k < 8; ++k)
        xl[k] = *reinterpret_cast<const float4*>(X + (int64_t)(rbase + 4 * k + (lane >> 3)) * c + col_base + c0 +
                                                 (lane & 7) * 4);
    };
    float4 xl[8];
    load_blk(0, half * 64, xl);
    // the last chunk's commit covers every MMA of the product
    {
      const int st = (L::KB - 1) & 1;
      wait_bar(xbar + st, st ? xph1 : xph0);
      // the other stage's last commit is complete too; keep its phase in step
      if (L::KB >= 2) {
        if (st) xph0 ^= 1u;
        else xph1 ^= 1u;
      }
    }
    // X' = acc + a X -> global (in place) and, unless last, the Gram operand
    float* tbuf = reinterpret_cast<float*>(xst) + warp * (32 * 36);
#pragma unroll
    for (int t = 0; t < L::NMT; ++t) {
      if (!tile_has(t)) continue;
      const int row = tile_row(t);
      const int rbase = row - lane;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int c0 = half * 64 + h2 * 32;
        // block -> rows
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<float4*>(tbuf + (4 * k + (lane >> 3)) * 36 + (lane & 7) * 4) = xl[k];
        __syncwarp();
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(tbuf + lane * 36 + e);
          x[e] = a4.x;
          x[e + 1] = a4.y;
          x[e + 2] = a4.z;
          x[e + 3] = a4.w;
        }
        // next block's loads in flight while this one is computed
        if (h2 == 0) load_blk(t, c0 + 32, xl);
        else if (t + 1 < L::NMT && tile_has(t + 1)) load_blk(t + 1, half * 64, xl);
        uint32_t v[32];
        if (ok) {
          tmem_ld32(tmem + lane_base + t * NSC_COLS + c0, v);
          tmem_ld_wait(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = fmaf(na, x[e], __uint_as_float(v[e]));
        // rows -> block, whole 128-byte row segments per store
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(tbuf + lane * 36 + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3), cc = (lane & 7) * 4;
          *reinterpret_cast<float4*>(X + (int64_t)(rbase + rr) * c + col_base + c0 + cc) =
              *reinterpret_cast<const float4*>(tbuf + rr * 36 + cc);
        }
        if (!last) nsc_put_row32<L::ROWBLK, L::PART>(opa, row, c0, x);
      }
    }
    tc_fence_before();
    if (!last) gram_and_reduce();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ttt
