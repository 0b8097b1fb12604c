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
// The gradient kernel reads K^ already normalised (fp16 copy written by the
// preparation kernel).  In the apply kernel, if the L2 normalisation of Q is on,
// the per-token inverse norm r_t scales the H1, H3 rows in the epilogue (the
// GEMM uses the raw queries, which is exact because the norm is a row scale).
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
// which buys the latency hiding that a single resident tile cannot.  The MMA
// issue loop is straight-line code (compile-time block indices) run by a whole
// converged warp with one elected lane issuing.
template <int D>
__global__ void __launch_bounds__(UPD_THREADS, 1)
    k_update_grad_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                     const __grid_constant__ CUtensorMap tmW, const float* __restrict__ eta_part,
                     float* __restrict__ partial, int64_t T, int H, int m, int tiles_total, int S,
                     unsigned int* status, unsigned long long timeout_ns) {
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
    {  // ---------------- MMA issuer: the whole warp runs the loop and waits,
       // the elected lane issues the MMAs and commits
      const bool leader = elect_one();
      // Base descriptors; an operand at byte offset o from a base is the base
      // descriptor + o/16 (the address field holds addr/16 and every operand
      // lies below 256 KB, so the add never carries out of the field).
      const uint64_t dW = sdesc_sw128(smem_u32(smem + L::W_OFF), 16, 1024);
      const uint64_t dF = sdesc_sw128(smem_u32(smem + L::F_OFF), 16, 1024);
      const uint64_t dB = sdesc_sw128(smem_u32(smem + L::B_OFF), L::BCHUNK, 1024);
      const uint64_t dDH = sdesc_sw128(smem_u32(smem + L::DH_OFF), TC_BLK, 1024);
      const uint64_t dU = sdesc_sw128(smem_u32(smem + L::U_OFF), TC_BLK, 1024);
      constexpr uint32_t ID_F13 = idesc_f16(128, 128, false, false);
      constexpr uint32_t ID_Z = idesc_f16(128, 64, false, false);
      constexpr uint32_t ID_G13 = idesc_f16(128, D, true, true);
      constexpr uint32_t ID_G2 = idesc_f16(128, 64, true, true);
      uint32_t fst = 0, fph = 0, bst = 0, bph = 0;  // ring stage and phase parity
      bool ok = true;
      // forward block b (compile-time) of the current forward tile
      auto F = [&](auto bc) {
        constexpr int b = decltype(bc)::value;
        ok &= __all_sync(0xffffffffu, mbar_wait(ffull + fst, fph, g));
        tc_fence_after();
        const uint64_t a0 = dF + (uint64_t)(fst * (TC_BLK >> 4));
        if (leader) {
          if constexpr (b < L::KB) {
#pragma unroll
            for (int kw = 0; kw < 4; ++kw)
              umma_bf16_ss(tmem + 0, a0 + kw * 2, dW + (b * L::W_BLK + kw * 32) / 16, ID_F13,
                           (b > 0 || kw > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kw = 0; kw < 4; ++kw)
              umma_bf16_ss(tmem + 128, a0 + kw * 2, dW + ((b - L::KB) * L::W_BLK + 16384 + kw * 32) / 16, ID_Z,
                           (b > L::KB || kw > 0) ? 1u : 0u);
          }
          umma_commit(fempty + fst);
        }
        __syncwarp();
        fph ^= (fst == L::NF - 1) ? 1u : 0u;
        fst = (fst == L::NF - 1) ? 0u : fst + 1;
      };
      // backward chunk c (compile-time) of the current backward tile; acc0 = 0
      // only for the very first gradient MMA of the token range
      auto G = [&](auto cc, uint32_t acc0) {
        constexpr int c = decltype(cc)::value;
        ok &= __all_sync(0xffffffffu, mbar_wait(bfull + bst, bph, g));
        tc_fence_after();
        const uint64_t b0 = dB + (uint64_t)(bst * (L::BSTAGE >> 4));
        if (leader) {
#pragma unroll
          for (int j = 0; j < L::BCH / 16; ++j) {
            const int ks = c * (L::BCH / 16) + j;
            const uint32_t acc = (c == 0 && j == 0) ? acc0 : 1u;
            umma_bf16_ss(tmem + L::G13_COL, dDH + ks * 128, b0 + j * 128, ID_G13, acc);
#pragma unroll
            for (int rb = 0; rb < L::N_G2; ++rb)
              umma_bf16_ss(tmem + L::G2_COL + rb * 64, b0 + ((L::KB + rb) * L::BCHUNK + j * 2048) / 16,
                           dU + ks * 128, ID_G2, acc);
          }
          umma_commit(bempty + bst);
        }
        __syncwarp();
        bph ^= (bst == L::NB - 1) ? 1u : 0u;
        bst = (bst == L::NB - 1) ? 0u : bst + 1;
      };
      ok = __all_sync(0xffffffffu, mbar_wait(wfull, 0, g));
      if (ok && ntiles > 0) {
        static_for<0, L::NFB>(F);
        if (leader) umma_commit(fdone);
        __syncwarp();
      }
      // forward blocks issued before the backward: they cover the epilogue's
      // compute; then G_i and the rest of F_(i+1) alternate so both TMA rings
      // stay busy (issuing F_(i+1) whole drains the forward ring: slower)
      constexpr int LEAD = L::NFB < 3 ? L::NFB : 3;
      constexpr int NSTEP = (L::NBC > L::NFB - LEAD) ? L::NBC : L::NFB - LEAD;
      for (int i = 0; ok && i < ntiles; ++i) {
        const uint32_t acc0 = i > 0 ? 1u : 0u;
        if (i + 1 < ntiles) {
          // F_(i+1) may overwrite TMEM F once the epilogue has drained F_i
          ok &= __all_sync(0xffffffffu, mbar_wait(ffree, i & 1, g));
          static_for<0, LEAD>(F);
          if constexpr (LEAD == L::NFB) {
            if (leader) umma_commit(fdone);
            __syncwarp();
          }
          ok &= __all_sync(0xffffffffu, mbar_wait(edone, i & 1, g));
          tc_fence_after();
          static_for<0, NSTEP>([&](auto kc) {
            constexpr int k = decltype(kc)::value;
            if constexpr (k < L::NBC) G(kc, acc0);
            if constexpr (LEAD + k < L::NFB) {
              F(std::integral_constant<int, LEAD + k>{});
              if constexpr (LEAD + k + 1 == L::NFB) {
                if (leader) umma_commit(fdone);
                __syncwarp();
              }
            }
          });
        } else {
          ok &= __all_sync(0xffffffffu, mbar_wait(edone, i & 1, g));
          tc_fence_after();
          static_for<0, L::NBC>([&](auto kc) { G(kc, acc0); });
        }
        if (leader) umma_commit(gdone);
        __syncwarp();
      }
    }
  } else {
    // ---------------- epilogue warps 2..9
    const int q = warp & 3;            // TMEM lane quarter accessible to this warp
    const int ch = (warp - 2) >> 2;    // which 32-column half of the slice
    float vscale_unused, inv_vscale;   // the readout undoes the value scale s of V'
    value_scale(eta_parts_max(eta_part), vscale_unused, inv_vscale);
    const int row = q * 32 + lane;     // token row within the tile / TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive_n(ffree, 32);  // F may now be overwritten by the next tile's forward
      // V arrives as V' = -s eta v (the preparation kernel folds the per-token
      // weight into it), so Z = s dL/du (clear of fp16 subnormals) and dH is
      // scaled the same way; U~ = u, and g2 = V'^T U~ carries the s.  The
      // gradient readout multiplies by 1/s, which is exact.
      const float2 half2 = make_float2(0.5f, 0.5f);
      const float2 mhalf2 = make_float2(-0.5f, -0.5f);
      uint32_t p1[16], p3[16], pu[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 h1 = make_float2(__uint_as_float(a1[j]), __uint_as_float(a1[j + 1]));
        const float2 h3 = make_float2(__uint_as_float(a3[j]), __uint_as_float(a3[j + 1]));
        const float2 z = make_float2(__uint_as_float(az[j]), __uint_as_float(az[j + 1]));
        const float2 hh = __fmul2_rn(h1, half2);
        const float2 th = make_float2(tanh_approx(hh.x), tanh_approx(hh.y));
        const float2 s = __ffma2_rn(th, half2, half2);           // sigmoid(h1)
        const float2 oms = __ffma2_rn(th, mhalf2, half2);        // 1 - sigmoid(h1)
        const float2 a = __fmul2_rn(h1, s);                      // SiLU(h1)
        const float2 u = __fmul2_rn(a, h3);
        const float2 dz = z;                                     // dL/du = -eta z (scaled)
        const float2 qd = __ffma2_rn(a, oms, s);                 // SiLU'(h1) = s + a (1 - s)
        const float2 d1 = __fmul2_rn(__fmul2_rn(dz, h3), qd);    // dL/dh1
        const float2 d3 = __fmul2_rn(dz, a);                     // dL/dh3
        const float2 ut = u;
        p1[j >> 1] = pack_f16x2(d1.x, d1.y);
        p3[j >> 1] = pack_f16x2(d3.x, d3.y);
        pu[j >> 1] = pack_f16x2(ut.x, ut.y);
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
      __syncwarp();
      if (lane == 0) mbar_arrive_n(edone, 32);
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
                make_float4(__uint_as_float(v[j]) * inv_vscale, __uint_as_float(v[j + 1]) * inv_vscale,
                            __uint_as_float(v[j + 2]) * inv_vscale, __uint_as_float(v[j + 3]) * inv_vscale);
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
            *reinterpret_cast<float4*>(dst + j) =
                make_float4(__uint_as_float(v[j]) * inv_vscale, __uint_as_float(v[j + 1]) * inv_vscale,
                            __uint_as_float(v[j + 2]) * inv_vscale, __uint_as_float(v[j + 3]) * inv_vscale);
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
  static constexpr int Q_OFF = 0;                        // this CTA's 128 query tokens, all d
  static constexpr int W13_HALF = KB * 64 * 128;         // this CTA's 64 rows of [W1c; W3c] (W1c or W3c)
  static constexpr int W2_HALF = (D / 2) * 128;          // this CTA's D/2 rows of W2c (64 m each)
  static constexpr int NS13 = 3;                         // W1|W3 ring stages (freed after the H MMAs)
  static constexpr int NS2 = 4;                          // W2 ring stages (freed after the O MMAs)
  static constexpr int W13_OFF = Q_OFF + KB * TC_BLK;
  static constexpr int W2_OFF = W13_OFF + NS13 * W13_HALF;
  static constexpr int P_OFF = W2_OFF + NS2 * W2_HALF;
  static constexpr int OST = 32 * 64;                    // per epilogue warp: [32 rows x 32 cols] bf16 staging
  static constexpr int OST_OFF = P_OFF + 2 * TC_BLK;     // 8 warps' staging tiles (64-byte swizzle)
  static constexpr int BAR_OFF = OST_OFF + 8 * OST;
  static constexpr int BYTES = BAR_OFF + 256;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int H_COL = 256;  // two [128 x 128] H buffers at 256 and 384
  static_assert(ALLOC <= 232448, "shared memory budget");
  static_assert(2 * 2 + 2 * NS13 + 2 * NS2 + 4 * 2 + 2 <= 31, "barrier budget");
};

constexpr int AP_THREADS = 352;  // warp 0: Q + W1|W3 TMA, 1: MMA, 2..9: epilogue, 10: W2 TMA
// O of chunk c is issued after H of chunk c + AP_OLAG: the epilogue has that many
// H products' time to turn H_c into P_c before the tensor pipe needs it (H is
// double-buffered in TMEM and the epilogue drains H_c first, so H_(c+2) may
// already overwrite it)
constexpr int AP_OLAG = 2;

// Fused SwiGLU apply on 2-SM tensor-core pairs (cta_group::2).  A cluster of two
// CTAs owns a 256-token tile (128 per CTA) of one head; every MMA is M = 256:
// A (queries, P) comes from each CTA's own rows, B (weights) is split in halves
// between the two CTAs -- CTA 0 holds the W1 rows and CTA 1 the W3 rows of a
// 64-wide m chunk for [H1 | H3], and each holds D/2 rows of W2 for O -- so each
// CTA streams half the weight bytes per token.  W1|W3 and W2 stream through
// separate rings with their own producers: a W1|W3 stage is free as soon as its
// H MMAs complete, while W2 of chunk c is consumed only after H of chunk c+1
// (one ring would hold every stage across two chunks and leave the chunk
// period bound by the L2 round trip).  The even CTA issues the MMAs; both CTAs
// run TMA producers and epilogues, and the epilogues of both CTAs report to the
// even CTA's barriers.
template <int D>
__global__ void __launch_bounds__(AP_THREADS, 1)
    k_apply_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmW,
               const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmO,
               int qnorm, int64_t T, int H, int m, int n_items, unsigned int* status,
               unsigned long long timeout_ns) {
  using L = ApLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nc = m / TC_MS;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* qfull = bars + 0;              // leader: TMA bytes of both CTAs
  uint64_t* qfree = bars + 1;              // both: MMA done reading Q (1) + this CTA's epilogue read its norms
  uint64_t* w13full = bars + 2;            // [NS13] leader
  uint64_t* w13free = w13full + L::NS13;   // [NS13] both
  uint64_t* w2full = w13free + L::NS13;    // [NS2] leader
  uint64_t* w2free = w2full + L::NS2;      // [NS2] both
  uint64_t* hfull = w2free + L::NS2;       // [2] both
  uint64_t* hfree = hfull + 2;             // [2] leader: 256 arrivals (a chunk's epilogue group, both CTAs)
  uint64_t* pfull = hfree + 2;             // [2] leader: 256 arrivals
  uint64_t* pfree = pfull + 2;             // [2] both
  uint64_t* odone = pfree + 2;             // both
  uint64_t* ofree = odone + 1;             // leader: 512 arrivals
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ofree + 1);

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    // the MMAs' commit, and every epilogue warp that handles a chunk of the item (one
    // group of four when the item has a single chunk, else both)
    mbar_init(qfree, 1 + (nc >= 2 ? 256 : 128));
    for (int i = 0; i < L::NS13; ++i) {
      mbar_init(w13full + i, 1);
      mbar_init(w13free + i, 1);
    }
    for (int i = 0; i < L::NS2; ++i) {
      mbar_init(w2full + i, 1);
      mbar_init(w2free + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(hfull + i, 1);
      mbar_init(hfree + i, 256);  // one epilogue group (4 warps) of each CTA per chunk
      mbar_init(pfull + i, 256);
      mbar_init(pfree + i, 1);
    }
    mbar_init(odone, 1);
    mbar_init(ofree, 512);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{status, timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- Q + W1|W3 producer (both CTAs): own Q rows, own half of each [W1c; W3c]
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmW);
      const uint32_t qfull_l = cluster_addr(qfull, 0);
      int gc = 0, it = 0;
      bool ok = true;
      for (int item = pair; ok && item < n_items; item += npairs, ++it) {
        const int tile = item / H, h = item % H;
        if (it > 0 && !mbar_wait(qfree, (it - 1) & 1, g)) break;
        if (leader) mbar_expect_tx(qfull, 2 * L::KB * TC_BLK);
        for (int kb = 0; kb < L::KB; ++kb)
          tma_load_2d_pair(smem + L::Q_OFF + kb * TC_BLK, &tmQ, qfull_l, h * D + kb * 64,
                           tile * 2 * TC_TILE + (int)rank * TC_TILE);
        for (int c = 0; c < nc; ++c, ++gc) {
          const int st = gc % L::NS13, use = gc / L::NS13;
          if (use > 0 && !mbar_wait(w13free + st, (use - 1) & 1, g)) { ok = false; break; }
          uint8_t* sw = smem + L::W13_OFF + st * L::W13_HALF;
          const uint32_t full_l = cluster_addr(w13full + st, 0);
          if (leader) mbar_expect_tx(w13full + st, 2 * L::W13_HALF);
          const int wrow = (rank == 0 ? 0 : H * m) + h * m + c * TC_MS;  // W1 rows (CTA 0) or W3 rows (CTA 1)
          for (int kb = 0; kb < L::KB; ++kb) tma_load_2d_pair(sw + kb * 8192, &tmW, full_l, kb * 64, wrow);
        }
      }
    }
  } else if (warp == 10) {
    if (lane == 0) {
      // ---------------- W2 producer (both CTAs): own D/2 rows of each W2 chunk
      tma_prefetch_desc(&tmW2);
      int gc = 0;
      bool ok = true;
      for (int item = pair; ok && item < n_items; item += npairs) {
        const int h = item % H;
        for (int c = 0; c < nc; ++c, ++gc) {
          const int st = gc % L::NS2, use = gc / L::NS2;
          if (use > 0 && !mbar_wait(w2free + st, (use - 1) & 1, g)) { ok = false; break; }
          const uint32_t full_l = cluster_addr(w2full + st, 0);
          if (leader) mbar_expect_tx(w2full + st, 2 * L::W2_HALF);
          tma_load_2d_pair(smem + L::W2_OFF + st * L::W2_HALF, &tmW2, full_l, c * TC_MS,
                           h * D + (int)rank * (D / 2));
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------- MMA issuer (even CTA only): the whole warp runs the loop
      // and waits, the elected lane issues
      const bool el = elect_one();
      const uint64_t dQ = sdesc_sw128(smem_u32(smem + L::Q_OFF), 16, 1024);
      const uint64_t dW13 = sdesc_sw128(smem_u32(smem + L::W13_OFF), 16, 1024);
      const uint64_t dW2 = sdesc_sw128(smem_u32(smem + L::W2_OFF), 16, 1024);
      const uint64_t dP = sdesc_sw128(smem_u32(smem + L::P_OFF), 16, 1024);
      constexpr uint32_t ID_H = idesc_bf16(256, 128, false, false);
      constexpr uint32_t ID_O = idesc_bf16(256, D, false, false);
      uint32_t s13 = 0, p13 = 0;  // W1|W3 ring stage and parity
      uint32_t s2 = 0, p2 = 0;    // W2 ring stage and parity (of the next O chunk)
      // O += P_c W2_c for the previous chunk (global chunk index gcp)
      auto do_o = [&](uint32_t gcp, bool first_of_item, int it) -> bool {
        const uint32_t pb = gcp & 1;
        bool w = mbar_wait(w2full + s2, p2, g) && mbar_wait_cluster(pfull + pb, (gcp >> 1) & 1, g);
        if (first_of_item && it > 0) w = w && mbar_wait_cluster(ofree, (it - 1) & 1, g);
        if (!__all_sync(0xffffffffu, w)) return false;
        tc_fence_after();
        if (el) {
          const uint64_t a0 = dP + pb * (TC_BLK >> 4);
          const uint64_t b0 = dW2 + s2 * (L::W2_HALF >> 4);
#pragma unroll
          for (int kw = 0; kw < 4; ++kw)
            umma_bf16_pair(tmem + 0, a0 + kw * 2, b0 + kw * 2, ID_O, (!first_of_item || kw > 0) ? 1u : 0u);
          umma_commit_pair(w2free + s2);
          umma_commit_pair(pfree + pb);
        }
        __syncwarp();
        p2 ^= (s2 == L::NS2 - 1) ? 1u : 0u;
        s2 = (s2 == L::NS2 - 1) ? 0u : s2 + 1;
        return true;
      };
      uint32_t gc = 0;  // global chunk counter (H buffer gc & 1)
      int it = 0;
      bool ok = true;
      for (int item = pair; ok && item < n_items; item += npairs, ++it) {
        if (!__all_sync(0xffffffffu, mbar_wait(qfull, it & 1, g))) break;
        for (int c = 0; c < nc; ++c, ++gc) {
          const uint32_t hb = gc & 1;
          bool w = mbar_wait(w13full + s13, p13, g);
          if (gc >= 2) w = w && mbar_wait_cluster(hfree + hb, ((gc >> 1) - 1) & 1, g);
          if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
          tc_fence_after();
          if (el) {
            const uint64_t b0 = dW13 + s13 * (L::W13_HALF >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const int kb = ks >> 2, kw = ks & 3;
              umma_bf16_pair(tmem + L::H_COL + hb * 128, dQ + (kb * TC_BLK + kw * 32) / 16,
                             b0 + (kb * 8192 + kw * 32) / 16, ID_H, ks > 0 ? 1u : 0u);
            }
            umma_commit_pair(w13free + s13);
            umma_commit_pair(hfull + hb);
            if (c == nc - 1) umma_commit_pair(qfree);
          }
          __syncwarp();
          p13 ^= (s13 == L::NS13 - 1) ? 1u : 0u;
          s13 = (s13 == L::NS13 - 1) ? 0u : s13 + 1;
          if (c >= AP_OLAG && !do_o(gc - AP_OLAG, c == AP_OLAG, it)) { ok = false; break; }
        }
        if (!ok) break;
        // the item's last O products
        for (int j = nc > AP_OLAG ? nc - AP_OLAG : 0; ok && j < nc; ++j) ok = do_o(gc - nc + j, j == 0, it);
        if (!ok) break;
        if (el) umma_commit_pair(odone);
        __syncwarp();
      }
    }
  } else {
    // ---------------- epilogue warps 2..9 (both CTAs): two groups of four warps
    // take alternate chunks (group = chunk parity = H buffer), so one group turns
    // H_c into P_c while the other drains H_(c+1); each warp covers its 32 TMEM
    // lanes (token rows) and all 64 columns of the chunk, 32 at a time
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;  // this warp's group; also its half of O's columns
    const int row = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const uint32_t hfree_l0 = cluster_addr(hfree, 0), hfree_l1 = cluster_addr(hfree + 1, 0);
    const uint32_t pfull_l0 = cluster_addr(pfull, 0), pfull_l1 = cluster_addr(pfull + 1, 0);
    const uint32_t ofree_l = cluster_addr(ofree, 0);
    int gc = 0, it = 0;
    bool ok = true;
    for (int item = pair; ok && item < n_items; item += npairs, ++it) {
      const int tile = item / H, h = item % H;
      float r = 1.f;
      bool first = true;  // this group's first chunk of the item
      for (int c = 0; c < nc; ++c, ++gc) {
        const int hb = gc & 1;
        if (hb != ch) continue;  // the other group's chunk
        if (!__all_sync(0xffffffffu, mbar_wait(hfull + hb, (gc >> 1) & 1, g))) { ok = false; break; }
        tc_fence_after();
        if (first) {
          first = false;
          // The item's first H has read the query tile, so it is in shared
          // memory; it stays there until both groups' epilogues release it (qfree).
          // q^ = q / max(||q||, 1e-12): the GEMM used the raw query, so the
          // inverse norm scales H1 and H3 rows here (rows past T were zero-filled).
          if (qnorm) {
            float ss = 0.f;
#pragma unroll
            for (int kb = 0; kb < L::KB; ++kb) {
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                const uint4 v = *reinterpret_cast<const uint4*>(smem + L::Q_OFF + kb * TC_BLK + sw128_offset(row, cc));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k2 = 0; k2 < 4; ++k2) {
                  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[k2]));
                  ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                }
              }
            }
            r = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_n(qfree, 32);
        }
        uint32_t pk[2][16];
        const float2 r2 = make_float2(r, r);
        const float2 half2 = make_float2(0.5f, 0.5f);
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t a1[32], a3[32];
          tmem_ld32(tmem + lane_base + L::H_COL + hb * 128 + hc * 32, a1);
          tmem_ld32(tmem + lane_base + L::H_COL + hb * 128 + 64 + hc * 32, a3);
          tmem_ld_wait(a1);
          tmem_ld_wait(a3);
          if (hc == 1) {
            tc_fence_before();
            warp_arrive_cluster(hb ? hfree_l1 : hfree_l0);
          }
          // sigmoid(h1) = 1/2 + tanh(h1/2)/2, tanh.approx.f32 (one MUFU operation per
          // element; the half-precision pair form saves MUFU work but its three
          // conversions per pair cost more: 2.93 vs 2.86 ms in a same-process A/B)
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 h1 = __fmul2_rn(make_float2(__uint_as_float(a1[j]), __uint_as_float(a1[j + 1])), r2);
            const float2 h3 = __fmul2_rn(make_float2(__uint_as_float(a3[j]), __uint_as_float(a3[j + 1])), r2);
            const float2 hh = __fmul2_rn(h1, half2);
            const float2 th = make_float2(tanh_approx(hh.x), tanh_approx(hh.y));
            const float2 sg = __ffma2_rn(th, half2, half2);
            const float2 pv = __fmul2_rn(__fmul2_rn(h1, sg), h3);  // SiLU(h1) * h3
            pk[hc][j >> 1] = pack_bf16x2(pv.x, pv.y);
          }
        }
        if (gc >= 2 && !__all_sync(0xffffffffu, mbar_wait(pfree + hb, ((gc >> 1) - 1) & 1, g))) {
          ok = false;
          break;
        }
        uint8_t* sp = smem + L::P_OFF + hb * TC_BLK;
#pragma unroll
        for (int hc = 0; hc < 2; ++hc)
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            *reinterpret_cast<uint4*>(sp + sw128_offset(row, hc * 4 + cc)) =
                make_uint4(pk[hc][4 * cc], pk[hc][4 * cc + 1], pk[hc][4 * cc + 2], pk[hc][4 * cc + 3]);
        fence_async_smem();
        warp_arrive_cluster(hb ? pfull_l1 : pfull_l0);
      }
      if (!ok) break;
      if (!__all_sync(0xffffffffu, mbar_wait(odone, it & 1, g))) break;
      tc_fence_after();
      // O readout: this warp's 32 token rows x D/2 columns; all TMEM loads first,
      // then O is released to the next item's MMAs while the stores proceed
      constexpr int NP = D / 64;  // 32-column pieces per warp
      uint32_t ov[NP][32];
#pragma unroll
      for (int p = 0; p < NP; ++p) tmem_ld32(tmem + lane_base + ch * (D / 2) + p * 32, ov[p]);
#pragma unroll
      for (int p = 0; p < NP; ++p) tmem_ld_wait(ov[p]);
      tc_fence_before();
      warp_arrive_cluster(ofree_l);
      // each piece goes through this warp's swizzled staging tile and a TMA store
      // (rows past T are clipped by the tensor map)
      uint8_t* stg = smem + L::OST_OFF + (warp - 2) * L::OST;
      const int orow0 = tile * 2 * TC_TILE + (int)rank * TC_TILE + q * 32;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        if (p > 0 || it > 0) {
          if (lane == 0) bulk_wait_read0();  // the previous store has read the staging tile
          __syncwarp();
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 x;
          x.x = pack_bf16x2(__uint_as_float(ov[p][8 * k + 0]), __uint_as_float(ov[p][8 * k + 1]));
          x.y = pack_bf16x2(__uint_as_float(ov[p][8 * k + 2]), __uint_as_float(ov[p][8 * k + 3]));
          x.z = pack_bf16x2(__uint_as_float(ov[p][8 * k + 4]), __uint_as_float(ov[p][8 * k + 5]));
          x.w = pack_bf16x2(__uint_as_float(ov[p][8 * k + 6]), __uint_as_float(ov[p][8 * k + 7]));
          *reinterpret_cast<uint4*>(stg + sw64_offset(lane, k)) = x;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && orow0 < T) {
          tma_store_2d(&tmO, stg, h * D + ch * (D / 2) + p * 32, orow0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace ttt
