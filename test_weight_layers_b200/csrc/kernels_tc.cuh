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
  static constexpr int NFB = 2 * KB;              // forward blocks per tile: K blocks, then V blocks
  static constexpr int NF = 3;                    // forward ring stages ([128 tok x 64 d] each)
  static constexpr int BCH = 32;                  // tokens per backward stage
  static constexpr int NBC = TC_TILE / BCH;       // backward stages per tile
  static constexpr int NB = 2;                    // backward ring stages
  static constexpr int W_BLK = 3 * 64 * 128;      // per d block: W1s, W3s, W2s^T rows (64 each)
  static constexpr int BCHUNK = BCH * 128;        // [32 tok x 64 d] swizzled
  static constexpr int BSTAGE = 2 * KB * BCHUNK;  // K chunks (KB) then V chunks (KB)
  static constexpr int W_OFF = 0;
  static constexpr int F_OFF = W_OFF + KB * W_BLK;
  static constexpr int B_OFF = F_OFF + NF * TC_BLK;
  static constexpr int DH_OFF = B_OFF + NB * BSTAGE;  // [dH1 block | dH3 block]
  static constexpr int U_OFF = DH_OFF + 2 * TC_BLK;
  static constexpr int BAR_OFF = U_OFF + TC_BLK;
  static constexpr int BYTES = BAR_OFF + 256;
  static constexpr int ALLOC = BYTES + 1024;      // slack for 1024-byte alignment
  static constexpr int G13_COL = 192;
  static constexpr int G2_COL = 192 + D;
  static constexpr int N_G2 = (D == 192) ? 2 : 1;
  static_assert(G2_COL + 64 * N_G2 <= 512, "TMEM budget");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

constexpr int UPD_THREADS = 352;  // warp 0: forward TMA, 1: MMA, 2..9: epilogue, 10: backward TMA

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Streaming gradient kernel.  Per 128-token tile i the tensor pipe runs the
// forward F_i (H1|H3 and Z from K, V d-blocks streamed through the forward ring)
// and the backward G_i (gradient GEMMs from K, V token chunks streamed a second
// time through the backward ring, with dH/U~ from shared memory).  The epilogue
// drains F_i from TMEM into registers first and releases it, so F_(i+1) runs
// while the epilogue computes; G_i is interleaved with F_(i+1) once the
// epilogue has written dH_i.  K and V are read twice from L2 (once per ring),
// which buys the latency hiding that a single resident tile cannot.
template <int D>
__global__ void __launch_bounds__(UPD_THREADS, 1)
    k_update_grad_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
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
  uint64_t* ffull = bars + 1;             // [NF]
  uint64_t* fempty = ffull + L::NF;       // [NF]
  uint64_t* bfull = fempty + L::NF;       // [NB]
  uint64_t* bempty = bfull + L::NB;       // [NB]
  uint64_t* fdone = bempty + L::NB;       // forward of a tile complete (TMEM F valid)
  uint64_t* ffree = fdone + 1;            // epilogue drained F (256 arrivals)
  uint64_t* edone = ffree + 1;            // epilogue wrote dH, U~ (256 arrivals)
  uint64_t* gdone = edone + 1;            // backward of a tile complete (dH buffer reusable)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gdone + 1);

  if (threadIdx.x == 0) {
    mbar_init(wfull, 1);
    for (int i = 0; i < L::NF; ++i) {
      mbar_init(ffull + i, 1);
      mbar_init(fempty + i, 1);
    }
    for (int i = 0; i < L::NB; ++i) {
      mbar_init(bfull + i, 1);
      mbar_init(bempty + i, 1);
    }
    mbar_init(fdone, 1);
    mbar_init(ffree, 256);
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
      // ---------------- forward ring producer: W once, then per tile K blocks then V blocks
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
      int fc = 0;
      bool ok = true;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int t0 = (t_begin + i) * TC_TILE;
        for (int b = 0; b < L::NFB; ++b, ++fc) {
          const int st = fc % L::NF, use = fc / L::NF;
          if (use > 0 && !mbar_wait(fempty + st, (use - 1) & 1, g)) { ok = false; break; }
          mbar_expect_tx(ffull + st, TC_BLK);
          const bool isk = b < L::KB;
          tma_load_2d(smem + L::F_OFF + st * TC_BLK, isk ? &tmK : &tmV, ffull + st, h * D + (isk ? b : b - L::KB) * 64,
                      t0);
        }
      }
    }
  } else if (warp == 10) {
    if (lane == 0) {
      // ---------------- backward ring producer: per tile, 32-token chunks of K and V (all d)
      tma_prefetch_desc(&tmKb);
      tma_prefetch_desc(&tmVb);
      int bc = 0;
      bool ok = true;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int t0 = (t_begin + i) * TC_TILE;
        for (int c = 0; c < L::NBC; ++c, ++bc) {
          const int st = bc % L::NB, use = bc / L::NB;
          if (use > 0 && !mbar_wait(bempty + st, (use - 1) & 1, g)) { ok = false; break; }
          mbar_expect_tx(bfull + st, L::BSTAGE);
          uint8_t* dst = smem + L::B_OFF + st * L::BSTAGE;
          for (int kb = 0; kb < L::KB; ++kb) {
            tma_load_2d(dst + kb * L::BCHUNK, &tmKb, bfull + st, h * D + kb * 64, t0 + c * L::BCH);
            tma_load_2d(dst + (L::KB + kb) * L::BCHUNK, &tmVb, bfull + st, h * D + kb * 64, t0 + c * L::BCH);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t sW = smem_u32(smem + L::W_OFF), sF = smem_u32(smem + L::F_OFF);
      const uint32_t sB = smem_u32(smem + L::B_OFF), sDH = smem_u32(smem + L::DH_OFF);
      const uint32_t sU = smem_u32(smem + L::U_OFF);
      constexpr uint32_t ID_F13 = idesc_bf16(128, 128, false, false);
      constexpr uint32_t ID_Z = idesc_bf16(128, 64, false, false);
      constexpr uint32_t ID_G13 = idesc_bf16(128, D, true, true);
      constexpr uint32_t ID_G2 = idesc_bf16(128, 64, true, true);
      int fc = 0, bc = 0;
      // one forward block b of the current forward tile
      auto f_block = [&](int b) -> bool {
        const int st = fc % L::NF, use = fc / L::NF;
        if (!mbar_wait(ffull + st, use & 1, g)) return false;
        tc_fence_after();
        const uint32_t a0 = sF + st * TC_BLK;
        if (b < L::KB) {
#pragma unroll
          for (int kw = 0; kw < 4; ++kw)
            umma_bf16_ss(tmem + 0, sdesc_sw128(a0 + kw * 32, 16, 1024),
                         sdesc_sw128(sW + b * L::W_BLK + kw * 32, 16, 1024), ID_F13, (b > 0 || kw > 0));
        } else {
          const int vb = b - L::KB;
#pragma unroll
          for (int kw = 0; kw < 4; ++kw)
            umma_bf16_ss(tmem + 128, sdesc_sw128(a0 + kw * 32, 16, 1024),
                         sdesc_sw128(sW + vb * L::W_BLK + 16384 + kw * 32, 16, 1024), ID_Z, (vb > 0 || kw > 0));
        }
        umma_commit(fempty + st);
        ++fc;
        return true;
      };
      // one backward chunk c of tile i (dH/U~ of tile i must be in shared memory)
      auto g_chunk = [&](int i, int c) -> bool {
        const int st = bc % L::NB, use = bc / L::NB;
        if (!mbar_wait(bfull + st, use & 1, g)) return false;
        tc_fence_after();
        const uint32_t b0 = sB + st * L::BSTAGE;
#pragma unroll
        for (int j = 0; j < L::BCH / 16; ++j) {
          const int ks = c * (L::BCH / 16) + j;
          const uint32_t acc = (i > 0 || ks > 0);
          umma_bf16_ss(tmem + L::G13_COL, sdesc_sw128(sDH + ks * 2048, TC_BLK, 1024),
                       sdesc_sw128(b0 + j * 2048, L::BCHUNK, 1024), ID_G13, acc);
#pragma unroll
          for (int rb = 0; rb < L::N_G2; ++rb)
            umma_bf16_ss(tmem + L::G2_COL + rb * 64,
                         sdesc_sw128(b0 + (L::KB + rb) * L::BCHUNK + j * 2048, L::BCHUNK, 1024),
                         sdesc_sw128(sU + ks * 2048, TC_BLK, 1024), ID_G2, acc);
        }
        umma_commit(bempty + st);
        ++bc;
        return true;
      };
      bool ok = mbar_wait(wfull, 0, g);
      if (ok && ntiles > 0) {
        for (int b = 0; ok && b < L::NFB; ++b) ok = f_block(b);
        if (ok) umma_commit(fdone);
      }
      for (int i = 0; ok && i < ntiles; ++i) {
        const bool has_next = i + 1 < ntiles;
        // F_(i+1) may overwrite TMEM F once the epilogue has drained F_i
        if (has_next && !mbar_wait(ffree, i & 1, g)) break;
        // the first forward blocks cover the epilogue's compute, then F and G alternate
        int fb = 0, gcn = 0;
        const int lead = has_next ? (L::NFB < 3 ? L::NFB : 3) : 0;
        for (; ok && fb < lead; ++fb) ok = f_block(fb);
        if (!ok) break;
        if (has_next && fb == L::NFB) umma_commit(fdone);
        if (!mbar_wait(edone, i & 1, g)) break;
        tc_fence_after();
        while (ok && (gcn < L::NBC || (has_next && fb < L::NFB))) {
          if (gcn < L::NBC) ok = g_chunk(i, gcn++);
          if (ok && has_next && fb < L::NFB) {
            ok = f_block(fb++);
            if (ok && fb == L::NFB) umma_commit(fdone);
          }
        }
        if (!ok) break;
        umma_commit(gdone);
      }
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
      tc_fence_before();
      mbar_arrive(ffree);  // F may now be overwritten by the next tile's forward
      const float2 r2 = make_float2(r, r);
      const float2 er2 = make_float2(-e * r, -e * r);   // -eta * r
      const float2 ne2 = make_float2(-e, -e);
      const float2 half2 = make_float2(0.5f, 0.5f);
      const float2 one2 = make_float2(1.f, 1.f);
      uint32_t p1[16], p3[16], pu[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 h1 = __fmul2_rn(make_float2(__uint_as_float(a1[j]), __uint_as_float(a1[j + 1])), r2);
        const float2 h3 = __fmul2_rn(make_float2(__uint_as_float(a3[j]), __uint_as_float(a3[j + 1])), r2);
        const float2 z = make_float2(__uint_as_float(az[j]), __uint_as_float(az[j + 1]));
        const float2 hh = __fmul2_rn(h1, half2);
        const float2 th = make_float2(tanh_approx(hh.x), tanh_approx(hh.y));
        const float2 s = __ffma2_rn(th, half2, half2);           // sigmoid(h1)
        const float2 a = __fmul2_rn(h1, s);                      // SiLU(h1)
        const float2 u = __fmul2_rn(a, h3);
        const float2 dz = __fmul2_rn(er2, z);                    // dL/du chained to the raw key
        const float2 oms = __fadd2_rn(one2, make_float2(-s.x, -s.y));
        const float2 qd = __ffma2_rn(a, oms, s);                 // SiLU'(h1) = s + a (1 - s)
        const float2 d1 = __fmul2_rn(__fmul2_rn(dz, h3), qd);    // dL/dh1 (raw key)
        const float2 d3 = __fmul2_rn(dz, a);                     // dL/dh3 (raw key)
        const float2 ut = __fmul2_rn(ne2, u);                    // -eta u
        p1[j >> 1] = pack_bf16x2(d1.x, d1.y);
        p3[j >> 1] = pack_bf16x2(d3.x, d3.y);
        pu[j >> 1] = pack_bf16x2(ut.x, ut.y);
      }
      // dH / U~ buffer is free once the previous tile's backward has completed
      if (i > 0 && !__all_sync(0xffffffffu, mbar_wait(gdone, (i - 1) & 1, g))) { ok = false; break; }
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
      mbar_arrive(edone);
    }
    if (ok && ntiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(gdone, (ntiles - 1) & 1, g));
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
