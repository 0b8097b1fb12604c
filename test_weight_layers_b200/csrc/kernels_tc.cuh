// Tensor-core (tcgen05 + TMEM + TMA) kernels for the bf16 hot path on sm_100a.
//
// 1. k_update_grad_tc -- fused forward + SwiGLU backward + gradient accumulation
//    of the dot-product TTT loss over a token range (Scal3R scheme 1 eq. (9);
//    ZipMap key design 1).  CTA = (64-row slice of m, head, token split); the
//    slice's gradient stays in TMEM for the whole token range:
//       TMEM cols [  0, 64) H1 = K W1s^T      (lane = token of the 128-token tile)
//                 [ 64,128) H3 = K W3s^T
//                 [128,192) Z  = V W2s        (Z_i = W2s^T v_i)
//                 [192,192+D) [g1s; g3s] += [dH1 | dH3]^T K   (lane = stacked m row)
//                 [192+D, +64) g2[0:128, s]  += V[:,0:128]^T U~ (lane = d row)
//                 [256+D, +64) g2[64:192, s] += V[:,64:192]^T U~ (D = 192 only)
//    dH1, dH3, U~ are produced by the epilogue warps as bf16 in shared memory
//    (MN-major operands), so the per-token intermediates never reach HBM.
// 2. k_apply_tc -- fused SwiGLU apply o = W2 (SiLU(W1 q) o (W3 q)) (Scal3R eq. (4)):
//    CTA loops over (128-token tile, head) items; m is walked in 64-wide chunks,
//    H = [H1 | H3] chunks are double-buffered in TMEM, P = SiLU(H1) o H3 goes to
//    shared memory as bf16 and O accumulates in TMEM.
//
// Roles (both kernels): warp 0 issues TMA loads, warp 1 issues MMAs (one
// thread), warps 2..9 run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// If the L2 normalisation of Q/K is on, the per-token inverse norm r_t scales
// the epilogue: H1, H3 rows by r_t and dH1, dH3 rows by r_t (the GEMMs use the
// raw keys/queries, which is exact because the norm is a row scale).
#pragma once

#include "common.cuh"

namespace ttt {

constexpr int TC_THREADS = 320;
constexpr int TC_TILE = 128;        // tokens per tile (MMA M)
constexpr int TC_MS = 64;           // m rows per update CTA / m chunk of apply
constexpr int TC_BLK = 128 * 128;   // one [128 rows x 64 bf16] swizzled block

template <int D>
struct UpdLayout {
  static constexpr int KB = D / 64;               // 64-wide d blocks
  static constexpr int W_BLK = 3 * 64 * 128;      // per d block: W1s, W3s, W2s^T rows (64 each)
  static constexpr int W_OFF = 0;
  static constexpr int K_OFF = W_OFF + KB * W_BLK;
  static constexpr int V_OFF = K_OFF + KB * TC_BLK;
  static constexpr int DH_OFF = V_OFF + KB * TC_BLK;  // [dH1 block | dH3 block]
  static constexpr int U_OFF = DH_OFF + 2 * TC_BLK;
  static constexpr int BAR_OFF = U_OFF + TC_BLK;
  static constexpr int BYTES = BAR_OFF + 256;
  static constexpr int ALLOC = BYTES + 1024;      // slack for 1024-byte alignment
  static constexpr int G13_COL = 192;
  static constexpr int G2_COL = 192 + D;
  static constexpr int N_G2 = (D == 192) ? 2 : 1;
  static_assert(G2_COL + 64 * N_G2 <= 512, "TMEM budget");
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_update_grad_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmW, const float* __restrict__ eta,
                     const float* __restrict__ rk, float* __restrict__ partial, int64_t T, int H, int m,
                     int tiles_total, int S, unsigned int* status, unsigned long long timeout_ns) {
  using L = UpdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int slice = blockIdx.x, h = blockIdx.y, split = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)((int64_t)tiles_total * split / S);
  const int t_end = (int)((int64_t)tiles_total * (split + 1) / S);
  const int ntiles = t_end - t_begin;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* wfull = bars + 0;
  uint64_t* kfull = bars + 1;
  uint64_t* vfull = bars + 2;
  uint64_t* kfree = bars + 3;
  uint64_t* vfree = bars + 4;
  uint64_t* fdone = bars + 5;
  uint64_t* edone = bars + 6;
  uint64_t* gdone = bars + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);

  if (threadIdx.x == 0) {
    mbar_init(wfull, 1);
    mbar_init(kfull, 1);
    mbar_init(vfull, 1);
    mbar_init(kfree, 1);
    mbar_init(vfree, 1);
    mbar_init(fdone, 1);
    mbar_init(edone, 256);
    mbar_init(gdone, 1);
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
  const Guard g{status, timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmW);
      mbar_expect_tx(wfull, L::KB * L::W_BLK);
      for (int kb = 0; kb < L::KB; ++kb) {
        uint8_t* dst = smem + L::W_OFF + kb * L::W_BLK;
        tma_load_2d(dst, &tmW, wfull, kb * 64, h * m + slice * TC_MS);
        tma_load_2d(dst + 8192, &tmW, wfull, kb * 64, H * m + h * m + slice * TC_MS);
        tma_load_2d(dst + 16384, &tmW, wfull, kb * 64, 2 * H * m + h * m + slice * TC_MS);
      }
      for (int i = 0; i < ntiles; ++i) {
        const int t0 = (t_begin + i) * TC_TILE;
        if (i > 0 && !mbar_wait(kfree, (i - 1) & 1, g)) break;
        mbar_expect_tx(kfull, L::KB * TC_BLK);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_2d(smem + L::K_OFF + kb * TC_BLK, &tmK, kfull, h * D + kb * 64, t0);
        if (i > 0 && !mbar_wait(vfree, (i - 1) & 1, g)) break;
        mbar_expect_tx(vfull, L::KB * TC_BLK);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_2d(smem + L::V_OFF + kb * TC_BLK, &tmV, vfull, h * D + kb * 64, t0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t sW = smem_u32(smem + L::W_OFF), sK = smem_u32(smem + L::K_OFF);
      const uint32_t sV = smem_u32(smem + L::V_OFF), sDH = smem_u32(smem + L::DH_OFF);
      const uint32_t sU = smem_u32(smem + L::U_OFF);
      constexpr uint32_t ID_F13 = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_Z = idesc_bf16(128, 64, false, false);
      constexpr uint32_t ID_G13 = idesc_bf16(128, D, true, true);
      constexpr uint32_t ID_G2 = idesc_bf16(128, 64, true, true);
      bool ok = mbar_wait(wfull, 0, g);
      for (int i = 0; ok && i < ntiles; ++i) {
        const uint32_t ph = i & 1;
        if (!mbar_wait(kfull, ph, g)) break;
        tc_fence_after();
        // [H1 | H3] = K [W1s; W3s]^T : M=128 tokens, N=128, K=D (A, B K-major)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int kb = ks >> 2, kw = ks & 3;
          umma_bf16_ss(tmem + 0, sdesc_sw128(sK + kb * TC_BLK + kw * 32, 16, 1024),
                       sdesc_sw128(sW + kb * L::W_BLK + kw * 32, 16, 1024), ID_F13, ks > 0);
        }
        if (!mbar_wait(vfull, ph, g)) break;
        tc_fence_after();
        // Z = V W2s : B = W2s^T rows (K-major)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int kb = ks >> 2, kw = ks & 3;
          umma_bf16_ss(tmem + 128, sdesc_sw128(sV + kb * TC_BLK + kw * 32, 16, 1024),
                       sdesc_sw128(sW + kb * L::W_BLK + 16384 + kw * 32, 16, 1024), ID_Z, ks > 0);
        }
        umma_commit(fdone);
        if (!mbar_wait(edone, ph, g)) break;
        tc_fence_after();
        // [g1s; g3s] += [dH1 | dH3]^T K : M=128 (stacked m rows), N=D, K=128 tokens (A, B MN-major)
#pragma unroll
        for (int ks = 0; ks < TC_TILE / 16; ++ks) {
          umma_bf16_ss(tmem + L::G13_COL, sdesc_sw128(sDH + ks * 2048, TC_BLK, 1024),
                       sdesc_sw128(sK + ks * 2048, TC_BLK, 1024), ID_G13, (i > 0 || ks > 0));
        }
        umma_commit(kfree);
        // g2[rows, s] += V[:, rows]^T U~ : M=128 d rows, N=64, K=128 tokens (A, B MN-major)
#pragma unroll
        for (int rb = 0; rb < L::N_G2; ++rb) {
#pragma unroll
          for (int ks = 0; ks < TC_TILE / 16; ++ks) {
            umma_bf16_ss(tmem + L::G2_COL + rb * 64, sdesc_sw128(sV + rb * TC_BLK + ks * 2048, TC_BLK, 1024),
                         sdesc_sw128(sU + ks * 2048, TC_BLK, 1024), ID_G2, (i > 0 || ks > 0));
          }
        }
        umma_commit(vfree);
      }
      umma_commit(gdone);
    }
  } else {
    // ---------------- epilogue warps 2..9
    const int q = warp & 3;            // TMEM lane quarter accessible to this warp
    const int ch = (warp - 2) >> 2;    // which 32-column half of the slice
    const int row = q * 32 + lane;     // token row within the tile / TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int64_t t = (int64_t)(t_begin + i) * TC_TILE + row;
      float e = 0.f, r = 0.f;
      if (t < T) {
        e = eta[t * H + h];
        r = rk ? rk[t * H + h] : 1.f;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(fdone, i & 1, g))) { ok = false; break; }
      tc_fence_after();
      uint32_t a1[32], a3[32], az[32];
      tmem_ld32(tmem + lane_base + 0 + ch * 32, a1);
      tmem_ld32(tmem + lane_base + 64 + ch * 32, a3);
      tmem_ld32(tmem + lane_base + 128 + ch * 32, az);
      tmem_ld_wait(a1);
      tmem_ld_wait(a3);
      tmem_ld_wait(az);
      uint32_t p1[16], p3[16], pu[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float o1[2], o3[2], ou[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float h1 = __uint_as_float(a1[j + k]) * r;
          const float h3 = __uint_as_float(a3[j + k]) * r;
          const float z = __uint_as_float(az[j + k]);
          const float s = 1.0f / (1.0f + __expf(-h1));
          const float a = h1 * s;
          const float du = -e * z;
          o1[k] = du * h3 * s * (1.0f + h1 * (1.0f - s)) * r;  // dL/dh1 chained to the raw key
          o3[k] = du * a * r;                                   // dL/dh3 chained to the raw key
          ou[k] = -e * a * h3;                                  // -eta u
        }
        p1[j >> 1] = pack_bf16x2(o1[0], o1[1]);
        p3[j >> 1] = pack_bf16x2(o3[0], o3[1]);
        pu[j >> 1] = pack_bf16x2(ou[0], ou[1]);
      }
      uint8_t* sdh = smem + L::DH_OFF;
      uint8_t* su = smem + L::U_OFF;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = sw128_offset(row, ch * 4 + c);
        *reinterpret_cast<uint4*>(sdh + off) = make_uint4(p1[4 * c], p1[4 * c + 1], p1[4 * c + 2], p1[4 * c + 3]);
        *reinterpret_cast<uint4*>(sdh + TC_BLK + off) =
            make_uint4(p3[4 * c], p3[4 * c + 1], p3[4 * c + 2], p3[4 * c + 3]);
        *reinterpret_cast<uint4*>(su + off) = make_uint4(pu[4 * c], pu[4 * c + 1], pu[4 * c + 2], pu[4 * c + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(edone);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(gdone, 0, g));
    if (ok && ntiles == 0) {
      // empty token range: the gradient partial is zero
      const int64_t n = (int64_t)m * D;
      for (int mat = 0; mat < 3; ++mat) {
        float* dst = partial + ((int64_t)split * 3 + mat) * H * n + (int64_t)h * n;
        for (int64_t i = (int64_t)(threadIdx.x - 64); i < (int64_t)TC_MS * D; i += 256) {
          const int64_t a = i / D, b = i % D;
          if (mat < 2) dst[(slice * TC_MS + a) * D + b] = 0.f;
          else dst[b * m + slice * TC_MS + a] = 0.f;
        }
      }
    } else if (ok) {
      tc_fence_after();
      const int64_t n = (int64_t)m * D;
      // [g1; g3] slice: lane < 64 -> g1 row, else g3 row; this warp writes D/2 columns
      {
        const int mat = row < 64 ? 0 : 1;
        const int mrow = slice * TC_MS + (row & 63);
        float* dst = partial + ((int64_t)split * 3 + mat) * H * n + (int64_t)h * n + (int64_t)mrow * D;
#pragma unroll
        for (int c0 = ch * (D / 2); c0 < (ch + 1) * (D / 2); c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + L::G13_COL + c0, v);
          tmem_ld_wait(v);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + c0 + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                            __uint_as_float(v[j + 3]));
        }
      }
      // g2 columns of this slice: block rb holds d rows 64*rb .. 64*rb+127
      float* g2 = partial + ((int64_t)split * 3 + 2) * H * n + (int64_t)h * n;
#pragma unroll
      for (int rb = 0; rb < L::N_G2; ++rb) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + L::G2_COL + rb * 64 + ch * 32, v);
        tmem_ld_wait(v);
        const int drow = rb * 64 + row;
        if (rb == 0 || row >= 64) {
          float* dst = g2 + (int64_t)drow * m + slice * TC_MS + ch * 32;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                              __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------

template <int D>
struct ApLayout {
  static constexpr int KB = D / 64;
  static constexpr int Q_OFF = 0;
  static constexpr int W13_BYTES = KB * TC_BLK;          // [W1c; W3c]: 128 rows per d block
  static constexpr int W2_BYTES = D * 128;               // W2c: D rows x 64 m
  static constexpr int STAGE = W13_BYTES + W2_BYTES;
  static constexpr int W_OFF = Q_OFF + KB * TC_BLK;
  static constexpr int P_OFF = W_OFF + 2 * STAGE;
  static constexpr int BAR_OFF = P_OFF + 2 * TC_BLK;
  static constexpr int BYTES = BAR_OFF + 256;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int H_COL = 256;  // two [128 x 128] H buffers at 256 and 384
};

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    k_apply_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmW,
               const __grid_constant__ CUtensorMap tmW2, const float* __restrict__ rq, __nv_bfloat16* __restrict__ O,
               int64_t ldo, int64_t T, int H, int m, int n_items, unsigned int* status,
               unsigned long long timeout_ns) {
  using L = ApLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = m / TC_MS;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* qfull = bars + 0;
  uint64_t* qfree = bars + 1;
  uint64_t* wfull = bars + 2;   // [2]
  uint64_t* wfree = bars + 4;   // [2]
  uint64_t* hfull = bars + 6;   // [2]
  uint64_t* hfree = bars + 8;   // [2]
  uint64_t* pfull = bars + 10;  // [2]
  uint64_t* pfree = bars + 12;  // [2]
  uint64_t* odone = bars + 14;
  uint64_t* ofree = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    mbar_init(qfree, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(wfull + i, 1);
      mbar_init(wfree + i, 1);
      mbar_init(hfull + i, 1);
      mbar_init(hfree + i, 256);
      mbar_init(pfull + i, 256);
      mbar_init(pfree + i, 1);
    }
    mbar_init(odone, 1);
    mbar_init(ofree, 256);
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
  const Guard g{status, timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmW);
      tma_prefetch_desc(&tmW2);
      int gc = 0, it = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
        const int tile = item / H, h = item % H;
        if (it > 0 && !mbar_wait(qfree, (it - 1) & 1, g)) break;
        mbar_expect_tx(qfull, L::KB * TC_BLK);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_2d(smem + L::Q_OFF + kb * TC_BLK, &tmQ, qfull, h * D + kb * 64, tile * TC_TILE);
        for (int c = 0; c < nc; ++c, ++gc) {
          const int st = gc & 1;
          if (gc >= 2 && !mbar_wait(wfree + st, ((gc >> 1) - 1) & 1, g)) { ok = false; break; }
          uint8_t* sw = smem + L::W_OFF + st * L::STAGE;
          mbar_expect_tx(wfull + st, L::STAGE);
          for (int kb = 0; kb < L::KB; ++kb) {
            tma_load_2d(sw + kb * TC_BLK, &tmW, wfull + st, kb * 64, h * m + c * TC_MS);
            tma_load_2d(sw + kb * TC_BLK + 8192, &tmW, wfull + st, kb * 64, H * m + h * m + c * TC_MS);
          }
          tma_load_2d(sw + L::W13_BYTES, &tmW2, wfull + st, c * TC_MS, h * D);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t sQ = smem_u32(smem + L::Q_OFF), sW = smem_u32(smem + L::W_OFF);
      const uint32_t sP = smem_u32(smem + L::P_OFF);
      constexpr uint32_t ID_H = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_O = idesc_bf16(128, D, false, false);
      int gc = 0, it = 0;
      bool ok = true;
      // O += P[g] W2c[g]^T for global chunk g (the chunk's W stage and P buffer are g & 1)
      auto do_o = [&](int gchunk, bool first_of_item) -> bool {
        const int pb = gchunk & 1;
        if (!mbar_wait(pfull + pb, (gchunk >> 1) & 1, g)) return false;
        if (first_of_item && it > 0 && !mbar_wait(ofree, (it - 1) & 1, g)) return false;
        tc_fence_after();
        const uint32_t sw2 = sW + pb * L::STAGE + L::W13_BYTES;
#pragma unroll
        for (int kw = 0; kw < 4; ++kw)
          umma_bf16_ss(tmem + 0, sdesc_sw128(sP + pb * TC_BLK + kw * 32, 16, 1024),
                       sdesc_sw128(sw2 + kw * 32, 16, 1024), ID_O, (!first_of_item || kw > 0));
        umma_commit(wfree + pb);
        umma_commit(pfree + pb);
        return true;
      };
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
        if (!mbar_wait(qfull, it & 1, g)) break;
        for (int c = 0; c < nc; ++c, ++gc) {
          const int st = gc & 1;
          if (!mbar_wait(wfull + st, (gc >> 1) & 1, g)) { ok = false; break; }
          if (gc >= 2 && !mbar_wait(hfree + st, ((gc >> 1) - 1) & 1, g)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sw = sW + st * L::STAGE;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int kb = ks >> 2, kw = ks & 3;
            umma_bf16_ss(tmem + L::H_COL + st * 128, sdesc_sw128(sQ + kb * TC_BLK + kw * 32, 16, 1024),
                         sdesc_sw128(sw + kb * TC_BLK + kw * 32, 16, 1024), ID_H, ks > 0);
          }
          umma_commit(hfull + st);
          if (c == nc - 1) umma_commit(qfree);
          if (c > 0 && !do_o(gc - 1, c - 1 == 0)) { ok = false; break; }
        }
        if (!ok) break;
        if (!do_o(gc - 1, nc == 1)) break;
        umma_commit(odone);
      }
    }
  } else {
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int gc = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++it) {
      const int tile = item / H, h = item % H;
      const int64_t t = (int64_t)tile * TC_TILE + row;
      const float r = (t < T) ? (rq ? rq[t * H + h] : 1.f) : 0.f;
      for (int c = 0; c < nc; ++c, ++gc) {
        const int hb = gc & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(hfull + hb, (gc >> 1) & 1, g))) { ok = false; break; }
        tc_fence_after();
        uint32_t a1[32], a3[32];
        tmem_ld32(tmem + lane_base + L::H_COL + hb * 128 + ch * 32, a1);
        tmem_ld32(tmem + lane_base + L::H_COL + hb * 128 + 64 + ch * 32, a3);
        tmem_ld_wait(a1);
        tmem_ld_wait(a3);
        tc_fence_before();
        mbar_arrive(hfree + hb);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float o[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float h1 = __uint_as_float(a1[j + k]) * r;
            const float h3 = __uint_as_float(a3[j + k]) * r;
            o[k] = h1 / (1.0f + __expf(-h1)) * h3;
          }
          pk[j >> 1] = pack_bf16x2(o[0], o[1]);
        }
        if (gc >= 2 && !__all_sync(0xffffffffu, mbar_wait(pfree + hb, ((gc >> 1) - 1) & 1, g))) { ok = false; break; }
        uint8_t* sp = smem + L::P_OFF + hb * TC_BLK;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          *reinterpret_cast<uint4*>(sp + sw128_offset(row, ch * 4 + cc)) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        fence_async_smem();
        mbar_arrive(pfull + hb);
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(odone, it & 1, g))) break;
      tc_fence_after();
      __nv_bfloat16* orow = O + t * ldo + (int64_t)h * D;
#pragma unroll
      for (int c0 = ch * (D / 2); c0 < (ch + 1) * (D / 2); c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + c0, v);
        tmem_ld_wait(v);
        if (t < T) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 x;
            x.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            x.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            x.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
            x.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
            *reinterpret_cast<uint4*>(orow + c0 + j) = x;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(ofree);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ttt
