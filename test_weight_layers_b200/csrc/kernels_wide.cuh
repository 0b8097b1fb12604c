// Wide-head path (d and m multiples of 256, e.g. ZipMap's single head with
// d = 1024, m = 2048 and state 6 d^2, ZipMap training section) and the gated
// output o = RMSNorm(o') * SiLU(W_g o') (ZipMap key design 3).
//
// At these widths neither the fused gradient kernel's tiling (the whole
// gradient slice of a head resident in TMEM) nor the apply kernel's resident
// query tile fits, and the arithmetic per token is large enough (12 d m flop
// per token for the update, against ~50 kB of per-token intermediates) that
// the products can exchange fp16 intermediates through HBM and still be bound
// by the tensor cores.  Every product runs on one persistent GEMM kernel on
// 2-SM tensor-core pairs (cta_group::2, 256 x 256 output tiles, K streamed in
// 64-wide stages by TMA, the accumulator double-buffered in TMEM so a tile's
// epilogue overlaps the next tile's MMAs) with a fused epilogue:
//
//   update: K^, V' = -s eta v (fp16, the preparation kernel k_prep_kv)
//           Z = V' W2                  -> fp16 [T][m]          (WG_STORE16)
//           [H1 | H3] = K^ [W1; W3]^T  -> dH1, dH3, u (fp16)   (WG_SWIGLU_BWD, reads Z)
//           g1 = dH1^T K^, g3 = dH3^T K^, g2 = V'^T u          (WG_PARTIAL, split-K over tokens)
//   apply:  P = SiLU(r H1) o (r H3) with H = Q [W1; W3]^T     (WG_SWIGLU_FWD, bf16)
//           O = P W2^T                                        (WG_STORE_BF16)
//   gate:   O = o' * rms(o') * SiLU(o' W_g^T)                 (WG_GATE)
//
// Operands are K-major (row = token or weight row, 64 K values per 128-byte
// swizzled row) except in the weight-gradient products, whose reduction runs
// over tokens: there both operands are token rows read MN-major (64 M or N
// values per 128-byte row, one row per token).
#pragma once

#include "common.cuh"

namespace ttt {

constexpr int WG_THREADS = 320;   // warp 0: TMA producer, 1: MMA issuer (even CTA), 2..9: epilogue
constexpr int WG_STAGES = 6;
constexpr int WG_HALF = 128 * 128;  // one CTA's operand tile of a stage: 128 rows x 64 K, 16 KB

struct WgLayout {
  static constexpr int A_OFF = 0;
  static constexpr int B_OFF = WG_STAGES * WG_HALF;
  static constexpr int BAR_OFF = 2 * WG_STAGES * WG_HALF;
  static constexpr int TB_ROW = 80;                  // a staged row: 32 16-bit values + 16 bytes of padding
  static constexpr int TB_WARP = 32 * TB_ROW;        // one epilogue warp's 32 rows
  static constexpr int TB_OFF = BAR_OFF + 256;       // 8 epilogue warps' staging buffers
  static constexpr int BYTES = TB_OFF + 8 * TB_WARP;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int ALLOC_NO_TB = TB_OFF + 1024;  // epilogues that stage no rows
  static_assert(ALLOC <= 232448, "shared memory budget");
};

enum WgEpi : int {
  WG_STORE16 = 0,      // C (fp16) = acc
  WG_SWIGLU_BWD = 1,   // acc = [H1 | H3] of 128 m columns; with Z: dH1, dH3, u (fp16)
  WG_PARTIAL = 2,      // fp32 split-K partial = acc * scale
  WG_SWIGLU_FWD = 3,   // acc = [H1 | H3]: P = SiLU(r H1) o (r H3) (bf16)
  WG_STORE_BF16 = 4,   // C (bf16) = acc
  WG_GATE = 5,         // acc = o' W_g^T: out = o' rinv SiLU(acc) (bf16)
  WG_NSOUT = 6         // Newton-Schulz product: C = alpha acc + beta Cin (fp32) and its bf16 hi/lo parts
};

// dynamic shared memory of an instance: the row-staging buffers for every epilogue
// but the fp32 split-K partials (written once per tile after the long K loop)
template <int EPI>
constexpr int wg_smem_bytes() {
  return EPI != WG_PARTIAL ? WgLayout::ALLOC : WgLayout::ALLOC_NO_TB;
}

// Everything a launch needs besides the tensor maps.  Items are
// (split, mat, head, tm, tn) with tn fastest, so pairs running side by side
// share the A rows (forward products) or the token range (weight gradients).
struct WgArgs {
  int M;          // output rows (T for token-row products)
  int mt, nt;     // output tiles (rows x columns) of each product
  int nt2;        // weight gradients: column tiles of g2 (its row tiles: mt * nt / nt2)
  int nmat;       // independent products (weight gradients: g1, g3, g2)
  int heads;
  int S;          // split-K slices over kblocks
  int kblocks;    // 64-wide K blocks of the whole reduction
  // operand coordinates (elements): K-major operands take x = (per-head offset) + k,
  // y = row; MN-major ones x = (per-head offset) + row-in-output, y = k (token)
  int a_head;     // per-head x offset of A (K-major) or of A's MN columns
  int b_row0;     // first row of B (K-major): the weight block inside the fp16/bf16 weight copy
  int b_head;     // per-head row offset of B (K-major) or x offset (MN-major)
  int b_row1;     // SwiGLU products: row of the second half (W3) relative to the first (W1)
  int a_row_head; // per-matrix row offset of A (K-major; Newton-Schulz batches)
  int b_y_head;   // per-matrix K-row offset of B (MN-major; Newton-Schulz batches)
  float alpha, beta;  // WG_NSOUT
  int out_head;   // per-head column offset of a stored output
  int mat2_a_head, mat2_b_head;  // weight gradients: per-head offsets of g2's operands (V', u)
  int m, d;       // head dims (weight gradients, epilogue column offsets)
  // epilogue
  void* out;            // primary output
  void* out2;           // dH3 (SWIGLU_BWD)
  void* out3;           // u (SWIGLU_BWD)
  const void* aux;      // Z (SWIGLU_BWD), o' (GATE)
  const float* rvec;    // per-row scale: r [T][H] (SWIGLU_FWD), rinv [T] (GATE)
  const float* eta_part;  // |eta| block maxima (PARTIAL: scale = 1/s)
  int64_t ldo, ldaux;   // row strides (elements) of out and aux
  uint32_t idesc;       // tcgen05 instruction descriptor (M = 256, N = 256)
};

// The mbarriers of one CTA.
struct WgBars {
  uint64_t* full;      // [WG_STAGES] even CTA: both CTAs' TMA bytes of a stage
  uint64_t* empty;     // [WG_STAGES] both: the stage's MMAs are done
  uint64_t* accfull;   // [2] both: an accumulator buffer is complete
  uint64_t* accempty;  // [2] even CTA: 512 epilogue arrivals (both CTAs)
  uint32_t* tmem_slot;
};

__device__ __forceinline__ WgBars wg_bars(uint8_t* smem) {
  uint64_t* b = reinterpret_cast<uint64_t*>(smem + WgLayout::BAR_OFF);
  WgBars r;
  r.full = b;
  r.empty = b + WG_STAGES;
  r.accfull = b + 2 * WG_STAGES;
  r.accempty = b + 2 * WG_STAGES + 2;
  r.tmem_slot = reinterpret_cast<uint32_t*>(b + 2 * WG_STAGES + 4);
  return r;
}

struct WgItem {
  int s, mat, h, tm, tn;
};

__device__ __forceinline__ WgItem wg_item(const WgArgs& a, int item) {
  WgItem it;
  const int tiles = a.mt * a.nt;
  const int t = item % tiles;
  item /= tiles;
  it.h = item % a.heads;
  item /= a.heads;
  it.mat = item % a.nmat;
  it.s = item / a.nmat;
  const int nt = it.mat == 2 ? a.nt2 : a.nt;  // g2 is [d][m], g1 and g3 [m][d]
  it.tm = t / nt;
  it.tn = t % nt;
  return it;
}

__device__ __forceinline__ void wg_krange(const WgArgs& a, int s, int& k0, int& k1) {
  k0 = (int)((int64_t)a.kblocks * s / a.S);
  k1 = (int)((int64_t)a.kblocks * (s + 1) / a.S);
}

// SiLU backward of one column pair (the fused gradient kernel's arithmetic):
// h1, h3, z (= s dL/du, the per-token weight already in z) -> dL/dh1, dL/dh3, u.
__device__ __forceinline__ void swiglu_bwd2(float2 h1, float2 h3, float2 z, float2& d1, float2& d3, float2& u) {
  const float2 half2 = make_float2(0.5f, 0.5f), mhalf2 = make_float2(-0.5f, -0.5f);
  const float2 hh = __fmul2_rn(h1, half2);
  float2 th;
  asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(hh.x));
  asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(hh.y));
  const float2 sg = __ffma2_rn(th, half2, half2);   // sigmoid(h1)
  const float2 oms = __ffma2_rn(th, mhalf2, half2); // 1 - sigmoid(h1)
  const float2 a = __fmul2_rn(h1, sg);              // SiLU(h1)
  u = __fmul2_rn(a, h3);
  const float2 qd = __ffma2_rn(a, oms, sg);         // SiLU'(h1) = s + a (1 - s)
  d1 = __fmul2_rn(__fmul2_rn(z, h3), qd);
  d3 = __fmul2_rn(z, a);
}

__device__ __forceinline__ float silu_f(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
  return x * fmaf(t, 0.5f, 0.5f);
}

// A warp's 32 rows x 32 16-bit columns (lane = row, four 16-byte vectors each) to
// global memory with coalesced stores: the rows go through the warp's staging
// buffer and leave as 8 rows x 64 contiguous bytes per store instruction, instead
// of 32 rows x 16 bytes (32 cache lines per instruction).  g0: the first row's
// first column; ldb: row stride in bytes; rows at or past nrows are not written.
__device__ __forceinline__ void warp_rows_out(uint8_t* tb, const uint4 (&v)[4], uint8_t* g0, int64_t ldb,
                                              int nrows) {
  const int lane = threadIdx.x & 31;
  __syncwarp();  // the previous use of the buffer has been read
#pragma unroll
  for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(tb + lane * WgLayout::TB_ROW + c * 16) = v[c];
  __syncwarp();
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int r = s * 8 + (lane >> 2), c = lane & 3;
    const uint4 x = *reinterpret_cast<const uint4*>(tb + r * WgLayout::TB_ROW + c * 16);
    if (r < nrows) *reinterpret_cast<uint4*>(g0 + r * ldb + c * 16) = x;
  }
}

// 8 consecutive fp16 / bf16 values from global memory as floats
__device__ __forceinline__ void ld8_f16(const __half* p, float (&v)[8]) {
  const uint4 x = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack_f16x2(w[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void ld8_bf16(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 x = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Persistent 2-SM GEMM: each cluster of two CTAs walks items pair, pair + npairs, ...
// AMN / BMN: A / B read MN-major (token rows) instead of K-major.
template <int EPI, bool AMN, bool BMN>
__global__ void __launch_bounds__(WG_THREADS, 1)
    k_wgemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
            const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB0,
            const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ WgArgs a, int n_items,
            unsigned int* status, unsigned long long timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const WgBars bars = wg_bars(smem);

  if (threadIdx.x == 0) {
    for (int i = 0; i < WG_STAGES; ++i) {
      mbar_init(bars.full + i, 1);
      mbar_init(bars.empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.accfull + i, 1);
      mbar_init(bars.accempty + i, 512);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(bars.tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;
  const Guard g{status, timeout_ns};
  pdl_wait();  // operands may come from the previous kernel on the stream

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs): this CTA's 128 rows of A and of B per stage
      const CUtensorMap* tA[3] = {&tmA0, &tmA1, &tmA2};
      const CUtensorMap* tB[2] = {&tmB0, &tmB1};
      for (int i = 0; i < 3; ++i) tma_prefetch_desc(tA[i]);
      for (int i = 0; i < 2; ++i) tma_prefetch_desc(tB[i]);
      int gs = 0;
      bool ok = true;
      for (int item = pair; ok && item < n_items; item += npairs) {
        const WgItem it = wg_item(a, item);
        int k0, k1;
        wg_krange(a, it.s, k0, k1);
        const CUtensorMap* mA = tA[it.mat];
        const CUtensorMap* mB = tB[it.mat == 2 ? 1 : 0];
        // Newton-Schulz products run over three K segments of split operands,
        // hi.hi + hi.lo + lo.hi: A = (hi, hi, lo), B = (hi, lo, hi)
        const int kseg = EPI == WG_NSOUT ? a.kblocks / 3 : a.kblocks;
        for (int kb = k0; kb < k1; ++kb, ++gs) {
          const int st = gs % WG_STAGES, use = gs / WG_STAGES;
          if (use > 0 && !mbar_wait(bars.empty + st, (use - 1) & 1, g)) { ok = false; break; }
          const uint32_t full_l = cluster_addr(bars.full + st, 0);
          if (leader) mbar_expect_tx(bars.full + st, 4 * WG_HALF);
          uint8_t* sa = smem + WgLayout::A_OFF + st * WG_HALF;
          uint8_t* sb = smem + WgLayout::B_OFF + st * WG_HALF;
          int kk = kb * 64;
          if (EPI == WG_NSOUT) {
            const int seg = kb / kseg;
            kk = (kb - seg * kseg) * 64;
            mA = tA[seg == 2 ? 1 : 0];
            mB = tB[seg == 1 ? 1 : 0];
          }
          if constexpr (!AMN) {
            // A rows = output rows (tokens): this CTA's 128 of the tile's 256
            tma_load_2d_pair(sa, mA, full_l, it.h * a.a_head + kk,
                             it.h * a.a_row_head + it.tm * 256 + (int)rank * 128);
          } else {
            // A^T: token rows, 128 output rows as two 64-wide column boxes
            const int ah = it.mat == 2 ? a.mat2_a_head : a.a_head;
            const int x0 = it.h * ah + it.tm * 256 + (int)rank * 128;
            tma_load_2d_pair(sa, mA, full_l, x0, kk);
            tma_load_2d_pair(sa + 8192, mA, full_l, x0 + 64, kk);
          }
          if constexpr (!BMN) {
            int brow;
            if (EPI == WG_SWIGLU_BWD || EPI == WG_SWIGLU_FWD)
              brow = a.b_row0 + it.h * a.b_head + it.tn * 128 + (int)rank * a.b_row1;  // W1 rows | W3 rows
            else
              brow = a.b_row0 + it.h * a.b_head + it.tn * 256 + (int)rank * 128;
            tma_load_2d_pair(sb, mB, full_l, kk, brow);
          } else {
            const int bh = it.mat == 2 ? a.mat2_b_head : a.b_head;
            const int x0 = it.h * bh + it.tn * 256 + (int)rank * 128;
            tma_load_2d_pair(sb, mB, full_l, x0, it.h * a.b_y_head + kk);
            tma_load_2d_pair(sb + 8192, mB, full_l, x0 + 64, it.h * a.b_y_head + kk);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------- MMA issuer (even CTA): whole warp waits, elected lane issues
      const bool el = elect_one();
      // K-major: 64 K per 128-byte row, a 16-wide K step is 32 bytes along the row.
      // MN-major: one token per 128-byte row, two 64-wide MN chunks 8 KB apart,
      // a 16-wide K step is 16 rows (2048 bytes).
      const uint64_t dA = AMN ? sdesc_sw128(smem_u32(smem + WgLayout::A_OFF), 8192, 1024)
                              : sdesc_sw128(smem_u32(smem + WgLayout::A_OFF), 16, 1024);
      const uint64_t dB = BMN ? sdesc_sw128(smem_u32(smem + WgLayout::B_OFF), 8192, 1024)
                              : sdesc_sw128(smem_u32(smem + WgLayout::B_OFF), 16, 1024);
      constexpr uint32_t KSA = AMN ? 2048 / 16 : 32 / 16;
      constexpr uint32_t KSB = BMN ? 2048 / 16 : 32 / 16;
      int gs = 0, it_n = 0;
      bool ok = true;
      for (int item = pair; ok && item < n_items; item += npairs, ++it_n) {
        const WgItem it = wg_item(a, item);
        int k0, k1;
        wg_krange(a, it.s, k0, k1);
        const uint32_t ab = it_n & 1;
        if (it_n >= 2 && !__all_sync(0xffffffffu, mbar_wait_cluster(bars.accempty + ab, ((it_n >> 1) - 1) & 1, g))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = k0; kb < k1; ++kb, ++gs) {
          const int st = gs % WG_STAGES, use = gs / WG_STAGES;
          if (!__all_sync(0xffffffffu, mbar_wait(bars.full + st, use & 1, g))) { ok = false; break; }
          tc_fence_after();
          if (el) {
            const uint64_t a0 = dA + (uint64_t)(st * (WG_HALF >> 4));
            const uint64_t b0 = dB + (uint64_t)(st * (WG_HALF >> 4));
#pragma unroll
            for (int kw = 0; kw < 4; ++kw)
              umma_bf16_pair(tmem + ab * 256, a0 + kw * KSA, b0 + kw * KSB, a.idesc, (kb > k0 || kw > 0) ? 1u : 0u);
            umma_commit_pair(bars.empty + st);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (el) umma_commit_pair(bars.accfull + ab);
        __syncwarp();
      }
    }
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs): warp (q, half) owns TMEM lane
    // quarter q (32 output rows) and half of the tile's columns
    const int q = warp & 3, half = (warp - 2) >> 2;
    const int rloc = q * 32 + lane;  // row within this CTA's 128
    uint8_t* tbuf = smem + WgLayout::TB_OFF + (warp - 2) * WgLayout::TB_WARP;  // this warp's staging rows
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const uint32_t accempty_l0 = cluster_addr(bars.accempty, 0), accempty_l1 = cluster_addr(bars.accempty + 1, 0);
    float scale = 1.f;
    if (EPI == WG_PARTIAL) {
      // readout scale 1/s of the value operand V' = -s eta v
      float mx = 0.f;
      for (int i = 0; i < ETA_PARTS; ++i) mx = fmaxf(mx, a.eta_part[i]);
      float s_;
      value_scale(mx, s_, scale);
    }
    // SwiGLU backward: this thread's 64 values of Z for an item (Z does not depend on the
    // MMAs, and its row-strided loads take an L2/HBM round trip)
    auto z_load = [&](int item, uint4 (&zq)[8]) {
      if (EPI != WG_SWIGLU_BWD || item >= n_items) return;
      const WgItem it = wg_item(a, item);
      const int64_t row = (int64_t)it.tm * 256 + rank * 128 + rloc;
      if (row >= a.M) return;
      const __half* zr = static_cast<const __half*>(a.aux) + row * a.ldaux + (int64_t)it.h * a.m + it.tn * 128 +
                         half * 64;
#pragma unroll
      for (int c = 0; c < 8; ++c) zq[c] = *reinterpret_cast<const uint4*>(zr + c * 8);
    };
    int it_n = 0;
    for (int item = pair; item < n_items; item += npairs, ++it_n) {
      const WgItem it = wg_item(a, item);
      const uint32_t ab = it_n & 1;
      const int64_t row = (int64_t)it.tm * 256 + rank * 128 + rloc;
      // the epilogue's own global inputs do not depend on the MMAs: their loads are issued
      // before waiting for the accumulator so their latency overlaps the wait
      uint4 pre[16], pre_z[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) pre_z[c] = make_uint4(0u, 0u, 0u, 0u);
      if (EPI == WG_SWIGLU_BWD) {
#pragma unroll
        z_load(item, pre_z);
        for (int c = 0; c < 8; ++c) pre[c] = pre_z[c];
      }
      if (EPI == WG_GATE && row < a.M) {
        const __nv_bfloat16* xr = static_cast<const __nv_bfloat16*>(a.aux) + row * a.ldaux + it.tn * 256 + half * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) pre[c] = *reinterpret_cast<const uint4*>(xr + c * 8);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bars.accfull + ab, (it_n >> 1) & 1, g))) break;
      tc_fence_after();
      const uint32_t base = tmem + lane_base + ab * 256;
      const uint32_t accempty_l = ab ? accempty_l1 : accempty_l0;
      if constexpr (EPI == WG_STORE16 || EPI == WG_STORE_BF16 || EPI == WG_PARTIAL) {
        // this thread's 128 columns: all TMEM loads, release the buffer, then store
        uint32_t v[4][32];
#pragma unroll
        for (int p = 0; p < 4; ++p) tmem_ld32(base + half * 128 + p * 32, v[p]);
#pragma unroll
        for (int p = 0; p < 4; ++p) tmem_ld_wait(v[p]);
        tc_fence_before();
        warp_arrive_cluster(accempty_l);
        if constexpr (EPI == WG_PARTIAL) {
          if (row >= a.M) continue;
          // partial[s][mat][h][M][N] (g1, g3: [m][d]; g2: [d][m]), scaled by 1/s
          const int Nn = it.mat == 2 ? a.m : a.d;
          const int64_t n = (int64_t)a.m * a.d;
          float* dst = static_cast<float*>(a.out) + ((int64_t)it.s * 3 + it.mat) * a.heads * n + (int64_t)it.h * n +
                       row * Nn + it.tn * 256 + half * 128;
#pragma unroll
          for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + p * 32 + c) =
                  make_float4(__uint_as_float(v[p][c]) * scale, __uint_as_float(v[p][c + 1]) * scale,
                              __uint_as_float(v[p][c + 2]) * scale, __uint_as_float(v[p][c + 3]) * scale);
        } else {
          // 32-column groups leave through the warp's staging buffer (coalesced)
          const int64_t col = (int64_t)it.h * a.out_head + it.tn * 256 + half * 128;
          const int64_t row0 = row - lane;
          const int nrows = (int)max((int64_t)0, min((int64_t)32, a.M - row0));
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            uint4 o[4];
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint32_t w4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i)
                w4[i] = EPI == WG_STORE16
                            ? pack_f16x2(__uint_as_float(v[p][c + 2 * i]), __uint_as_float(v[p][c + 2 * i + 1]))
                            : pack_bf16x2(__uint_as_float(v[p][c + 2 * i]), __uint_as_float(v[p][c + 2 * i + 1]));
              o[c >> 3] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            warp_rows_out(tbuf, o, static_cast<uint8_t*>(a.out) + (row0 * a.ldo + col + p * 32) * 2, a.ldo * 2,
                          nrows);
          }
        }
      } else if constexpr (EPI == WG_SWIGLU_BWD || EPI == WG_SWIGLU_FWD) {
        // m columns [tn*128 + half*64, +64) of head h, in two 32-column phases: H1 from
        // accumulator columns half*64 + .., H3 from 128 + half*64 + ..; each phase's
        // 32 x 32 outputs per warp leave through the staging buffer (coalesced)
        const int64_t col = (int64_t)it.h * a.m + it.tn * 128 + half * 64;
        const float r = (EPI == WG_SWIGLU_FWD && a.rvec && row < a.M) ? a.rvec[row * a.heads + it.h] : 1.f;
        const int64_t row0 = row - lane;  // this warp's first row
        const int nrows = (int)max((int64_t)0, min((int64_t)32, a.M - row0));
#pragma unroll
        for (int ph = 0; ph < 2; ++ph) {
          uint32_t v1[32], v3[32];
          tmem_ld32(base + half * 64 + ph * 32, v1);
          tmem_ld32(base + 128 + half * 64 + ph * 32, v3);
          tmem_ld_wait(v1);
          tmem_ld_wait(v3);
          if (ph == 1) {
            tc_fence_before();
            warp_arrive_cluster(accempty_l);
          }
          if (nrows == 0) continue;  // warp-uniform
          uint4 o1[4], o3[4], ou[4];
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) {
            uint32_t p1[4], p3[4], pu[4];
            if constexpr (EPI == WG_SWIGLU_BWD) {
              const uint4 zq = pre[(ph * 32 + c8) >> 3];
              const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
              for (int j = 0; j < 8; j += 2) {
                const float2 h1 = make_float2(__uint_as_float(v1[c8 + j]), __uint_as_float(v1[c8 + j + 1]));
                const float2 h3 = make_float2(__uint_as_float(v3[c8 + j]), __uint_as_float(v3[c8 + j + 1]));
                float2 d1, d3, u;
                swiglu_bwd2(h1, h3, unpack_f16x2(zw[j >> 1]), d1, d3, u);
                p1[j >> 1] = pack_f16x2(d1.x, d1.y);
                p3[j >> 1] = pack_f16x2(d3.x, d3.y);
                pu[j >> 1] = pack_f16x2(u.x, u.y);
              }
              o3[c8 >> 3] = make_uint4(p3[0], p3[1], p3[2], p3[3]);
              ou[c8 >> 3] = make_uint4(pu[0], pu[1], pu[2], pu[3]);
            } else {
#pragma unroll
              for (int j = 0; j < 8; j += 2) {
                const float h1a = r * __uint_as_float(v1[c8 + j]), h1b = r * __uint_as_float(v1[c8 + j + 1]);
                const float h3a = r * __uint_as_float(v3[c8 + j]), h3b = r * __uint_as_float(v3[c8 + j + 1]);
                p1[j >> 1] = pack_bf16x2(silu_f(h1a) * h3a, silu_f(h1b) * h3b);
              }
              (void)p3;
              (void)pu;
            }
            o1[c8 >> 3] = make_uint4(p1[0], p1[1], p1[2], p1[3]);
          }
          const int64_t ob = (row0 * a.ldo + col + ph * 32) * 2;  // byte offset of the warp's first row
          warp_rows_out(tbuf, o1, static_cast<uint8_t*>(a.out) + ob, a.ldo * 2, nrows);
          if constexpr (EPI == WG_SWIGLU_BWD) {
            warp_rows_out(tbuf, o3, static_cast<uint8_t*>(a.out2) + ob, a.ldo * 2, nrows);
            warp_rows_out(tbuf, ou, static_cast<uint8_t*>(a.out3) + ob, a.ldo * 2, nrows);
          }
        }
      } else if constexpr (EPI == WG_GATE) {
        // columns [tn*256 + half*128, +128) in four 32-column phases
        const int64_t col = (int64_t)it.tn * 256 + half * 128;
        const float ri = row < a.M ? a.rvec[row] : 0.f;
        const int64_t row0 = row - lane;
        const int nrows = (int)max((int64_t)0, min((int64_t)32, a.M - row0));
#pragma unroll
        for (int ph = 0; ph < 4; ++ph) {
          uint32_t v[32];
          tmem_ld32(base + half * 128 + ph * 32, v);
          tmem_ld_wait(v);
          if (ph == 3) {
            tc_fence_before();
            warp_arrive_cluster(accempty_l);
          }
          if (nrows == 0) continue;  // warp-uniform
          uint4 o[4];
#pragma unroll
          for (int c8 = 0; c8 < 32; c8 += 8) {
            const uint4 q = pre[(ph * 32 + c8) >> 3];
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float xa = __uint_as_float(w4[i] << 16), xb = __uint_as_float(w4[i] & 0xffff0000u);
              const float ga = __uint_as_float(v[c8 + 2 * i]), gb = __uint_as_float(v[c8 + 2 * i + 1]);
              pk[i] = pack_bf16x2(xa * ri * silu_f(ga), xb * ri * silu_f(gb));
            }
            o[c8 >> 3] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          warp_rows_out(tbuf, o, static_cast<uint8_t*>(a.out) + (row0 * a.ldo + col + ph * 32) * 2, a.ldo * 2, nrows);
        }
      } else if constexpr (EPI == WG_NSOUT) {
        // C = alpha acc + beta Cin for matrix h (rows M, stride ldo), plus C's bf16 hi and lo
        // parts (the next product's split operands), four 32-column phases
        const int64_t mbase = (int64_t)it.h * a.M * a.ldo + row * a.ldo + it.tn * 256 + half * 128;
        const float* cin = static_cast<const float*>(a.aux);
        const int64_t row0 = row - lane;
        const int nrows = (int)max((int64_t)0, min((int64_t)32, a.M - row0));
        const int64_t wbase = mbase - (int64_t)lane * a.ldo;  // this warp's first row
#pragma unroll
        for (int ph = 0; ph < 4; ++ph) {
          float4 ci[8];
          if (cin) {
#pragma unroll
            for (int q = 0; q < 8; ++q) ci[q] = *reinterpret_cast<const float4*>(cin + mbase + ph * 32 + q * 4);
          }
          uint32_t v[32];
          tmem_ld32(base + half * 128 + ph * 32, v);
          tmem_ld_wait(v);
          if (ph == 3) {
            tc_fence_before();
            warp_arrive_cluster(accempty_l);
          }
          // fp32 C in two 16-column halves and its bf16 hi/lo parts, each through the
          // staging buffer (rows of 64 bytes)
          uint4 oc[2][4], oh[4], ol[4];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 c = cin ? ci[q] : make_float4(0.f, 0.f, 0.f, 0.f);
            float o[4];
            o[0] = fmaf(a.alpha, __uint_as_float(v[4 * q + 0]), a.beta * c.x);
            o[1] = fmaf(a.alpha, __uint_as_float(v[4 * q + 1]), a.beta * c.y);
            o[2] = fmaf(a.alpha, __uint_as_float(v[4 * q + 2]), a.beta * c.z);
            o[3] = fmaf(a.alpha, __uint_as_float(v[4 * q + 3]), a.beta * c.w);
            oc[q >> 2][q & 3] = make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                                           __float_as_uint(o[3]));
            uint32_t hi[2], lo[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              hi[e] = pack_bf16x2(o[2 * e], o[2 * e + 1]);
              const float h0 = __uint_as_float(hi[e] << 16), h1 = __uint_as_float(hi[e] & 0xffff0000u);
              lo[e] = pack_bf16x2(o[2 * e] - h0, o[2 * e + 1] - h1);
            }
            // 8 consecutive bf16 per uint4: q pairs (2k, 2k + 1) fill vector k
            if (q & 1) {
              oh[q >> 1].z = hi[0];
              oh[q >> 1].w = hi[1];
              ol[q >> 1].z = lo[0];
              ol[q >> 1].w = lo[1];
            } else {
              oh[q >> 1].x = hi[0];
              oh[q >> 1].y = hi[1];
              ol[q >> 1].x = lo[0];
              ol[q >> 1].y = lo[1];
            }
          }
          if (nrows == 0) continue;  // warp-uniform
          const int64_t off = wbase + ph * 32;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            warp_rows_out(tbuf, oc[hf], reinterpret_cast<uint8_t*>(static_cast<float*>(a.out) + off + hf * 16),
                          a.ldo * 4, nrows);
          warp_rows_out(tbuf, oh, reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out2) + off), a.ldo * 2,
                        nrows);
          warp_rows_out(tbuf, ol, reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(a.out3) + off), a.ldo * 2,
                        nrows);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// CUDA-core helpers of the wide path

// RMSNorm factors of o' rows: rinv[t] = 1 / sqrt(mean_j o'_(t,j)^2 + eps), one warp per row.
__global__ void __launch_bounds__(256) k_rms_rows(const __nv_bfloat16* __restrict__ X, int64_t ld, int64_t T, int D,
                                                  float eps, float* __restrict__ rinv) {
  const int lane = threadIdx.x & 31;
  for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T;
       t += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    float ss = 0.f;
    for (int i = lane; i < D / 8; i += 32) {
      float x[8];
      ld8_bf16(X + t * ld + i * 8, x);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) rinv[t] = 1.0f / sqrtf(ss / (float)D + eps);
  }
}

// bf16 hi and lo parts of an fp32 array: hi = bf16(x), lo = bf16(x - hi) (n a multiple of 4).
__global__ void k_split_bf16(const float* __restrict__ x, __nv_bfloat16* __restrict__ hi,
                             __nv_bfloat16* __restrict__ lo, int64_t n) {
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    const uint32_t h0 = pack_bf16x2(v.x, v.y), h1 = pack_bf16x2(v.z, v.w);
    const uint32_t l0 = pack_bf16x2(v.x - __uint_as_float(h0 << 16), v.y - __uint_as_float(h0 & 0xffff0000u));
    const uint32_t l1 = pack_bf16x2(v.z - __uint_as_float(h1 << 16), v.w - __uint_as_float(h1 & 0xffff0000u));
    *reinterpret_cast<uint2*>(hi + i) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(lo + i) = make_uint2(l0, l1);
  }
}

// bf16 copy of an fp32 matrix (n a multiple of 4).
__global__ void k_cast_bf16(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int64_t n) {
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(x + i);
    *reinterpret_cast<uint2*>(y + i) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

}  // namespace ttt
