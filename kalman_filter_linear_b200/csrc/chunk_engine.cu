// Chunkwise tensor-core engine of the KDN layer forward (tcgen05 + TMA + TMEM).
//
// The Kalman-gain-driven delta rule ("Kalman Delta Networks: Uncertainty-
// aware Associative Memory", abstract; "Kalman Delta Networks:
// 不确定性感知的联想记忆", 方法 — 关键模块 steps 1-3: predict, gain-weighted
// residual write, scan-compatible variance) is evaluated 64 tokens at a time.
// Inside a chunk that starts from the state S0, with gamma_t the in-chunk
// cumulative decay and g_t the write vector (iso: beta_t k_t; diag:
// p-_t * k_t / s_t):
//     A_tj = (gamma_t/gamma_j) k_t.g_j  (j < t),   T = (I + A)^-1
//     Z    = V - diag(gamma) K S0'        U = T Z
//     O    = diag(gamma) Q S0' + ((Q G') o D) U,   D_tj = gamma_t/gamma_j (j <= t)
//     S    = gamma_C S0 + U' diag(gamma_C/gamma) G
// (derived from the token recursion S_t = a_t S_{t-1} + (v_t - a_t S_{t-1}
// k_t) g_t'; the pages only say a hardware-efficient chunkwise form exists).
// The variance recursion (a Mobius map per token) runs inside the chunk as a
// warp scan of 2x2 maps (iso) or a per-dimension recursion (diag), with the
// carried value passed from chunk to chunk.
//
// One CTA owns one (batch, head, block of NV value columns) for the whole
// sequence; 256 threads.  Per chunk:
//   MMA1  D1 = [K;Q] G~'          (iso: G~ = K; diag: G~ = p- * k, hi/lo)
//   MMA2  D2 = [K;Q] S'           (S as bf16 hi + lo)
//   SIMT  A, T = (I+A)^-1 (blocked 16x16 forward substitution), Z
//   MMA3  D3 = [T_hi;T_lo] [Z_hi Z_lo]  -> U = top + bottom
//   MMA4  D4 = [P_hi;P_lo] [U_hi U_lo]  -> O = D4 top + bottom + gamma Q S'
//   MMA5  D5 = G~' [B_hi B_lo]          (B = diag(coef) U) -> S update
// Every fp32 operand of a contraction that feeds the state or the output is
// carried as a bf16 (hi, lo) pair (16 significant bits); products of bf16
// inputs are exact in the fp32 accumulator.
//
// Shared-memory operand layouts use the 128-byte swizzle.  Every 128-row A
// operand is interleaved by 8-row groups: group 2h holds rows 8h..8h+7 of the
// first half (K, T_hi or P_hi) and group 2h+1 those of the second half (Q,
// T_lo or P_lo).  A token's two rows then land in TMEM lanes L and L+8 of the
// same warp, so the two halves combine with one shuffle.  K's rows are the
// even groups, so the same tile is K (B operand of MMA1, stride 2048 B) and K'
// (MN-major A operand of MMA5).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kC = 64;     // tokens per chunk
constexpr int kDK = 128;   // key dimension of the engine
constexpr int kThreads = 256;
constexpr int kScrLd = 68; // fp32 row stride of the 64x64 solve buffers

template <bool DIAG, int NV>
struct Plan {
  static constexpr int NVB = NV / 64;
  static constexpr uint32_t KQ_BYTES = 2u * 128u * 128u;       // [kb 2][128 rows][64] bf16
  static constexpr uint32_t V_BYTES = (uint32_t)NV * 64u * 2u; // [vb][64 t][64] bf16
  static constexpr uint32_t SREG_BYTES = (uint32_t)NV * 512u;  // S hi+lo [vb][128 k][64]
  static constexpr uint32_t ZU_BYTES = (uint32_t)NV * 128u;    // one of Z/U/B (hi or lo)
  static constexpr uint32_t OFF_KQ = 0;
  static constexpr uint32_t OFF_V = OFF_KQ + 2 * KQ_BYTES;
  static constexpr uint32_t OFF_S = OFF_V + 2 * V_BYTES;
  static constexpr uint32_t OFF_TP = OFF_S + SREG_BYTES;       // [128][64] bf16 (T or P)
  static constexpr uint32_t OFF_G = OFF_TP + 16384;            // diag: G~ hi, lo [kb][64][64]
  static constexpr uint32_t OFF_SA = OFF_G + (DIAG ? 32768u : 0u);  // fp32 A [64][68]
  static constexpr uint32_t OFF_ST = OFF_SA + 64u * kScrLd * 4u;    // fp32 T [64][68]
  static constexpr uint32_t OFF_X = OFF_ST + 64u * kScrLd * 4u;     // fp32 [3][16][17]
  static constexpr uint32_t OFF_SC = OFF_X + 3u * 16u * 17u * 4u + 64u;
  static constexpr uint32_t OFF_BAR = OFF_SC + 8u * 64u * 4u;
  static constexpr uint32_t TOTAL = OFF_BAR + 64u;
  static constexpr uint32_t ALLOC = TOTAL + 1024u;
  // TMEM columns
  static constexpr uint32_t COL_D1 = 0, COL_D2 = 64, COL_D3 = 64 + NV, COL_D4 = 64 + 2 * NV;
  static constexpr uint32_t COL_D5 = COL_D3;
  static constexpr uint32_t TMEM_COLS = (64 + 3 * NV) <= 256 ? 256u : 512u;
  static_assert(TOTAL <= 227u * 1024u, "shared memory plan too large");
};

// Token of 128-row interleaved operand row m, and whether it is the second half.
__device__ __forceinline__ int il_token(int m) { return 8 * (m >> 4) + (m & 7); }
__device__ __forceinline__ int il_second(int m) { return (m >> 3) & 1; }
__device__ __forceinline__ int il_row(int t, int second) { return 16 * (t >> 3) + (t & 7) + 8 * second; }

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

// Write 8 consecutive columns [col8*8, col8*8+8) of swizzled row `row` as hi
// and lo bf16 halves of x[0..7].
__device__ __forceinline__ void st_split8(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t row,
                                          uint32_t col8, const float* x) {
  __nv_bfloat16 h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) split_bf16(x[i], h[i], l[i]);
  const uint32_t off = sw128_offset(row, col8 * 8);
  *reinterpret_cast<uint4*>(hi_tile + off) =
      make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
  *reinterpret_cast<uint4*>(lo_tile + off) =
      make_uint4(pack2(l[0], l[1]), pack2(l[2], l[3]), pack2(l[4], l[5]), pack2(l[6], l[7]));
}

__device__ __forceinline__ float ld_bf16(const uint8_t* tile, uint32_t row, uint32_t col) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + sw128_offset(row, col)));
}

struct Mat2 { float a, b, c, d; };
__device__ __forceinline__ Mat2 mmul(const Mat2& x, const Mat2& y) {
  return {fmaf(x.a, y.a, x.b * y.c), fmaf(x.a, y.b, x.b * y.d), fmaf(x.c, y.a, x.d * y.c),
          fmaf(x.c, y.b, x.d * y.d)};
}
__device__ __forceinline__ Mat2 mnorm(const Mat2& x) {
  const float m = fmaxf(fmaxf(x.a, x.b), fmaxf(x.c, x.d));
  const int e = (int)((__float_as_uint(m) >> 23) & 0xffu) - 127;
  if (e > -100 && e < 100 && e != 0) {
    const float s = __uint_as_float((uint32_t)(127 - e) << 23);
    return {x.a * s, x.b * s, x.c * s, x.d * s};
  }
  return x;
}

// Issue K-steps of one MMA group: `steps` consecutive K=16 slices.
// a0/b0: descriptors of the first slice; a_step/b_step: byte advance per slice
// (applied to the 14-bit start-address field, >> 4).
__device__ __forceinline__ void mma_steps(uint32_t tmem_d, uint64_t a0, uint64_t b0,
                                          uint32_t a_step, uint32_t b_step, int steps,
                                          uint32_t idesc, bool accumulate_first) {
  for (int s = 0; s < steps; ++s) {
    const uint64_t a = a0 + (uint64_t)((s * a_step) >> 4);
    const uint64_t b = b0 + (uint64_t)((s * b_step) >> 4);
    umma_bf16(tmem_d, a, b, idesc, (accumulate_first || s > 0) ? 1u : 0u);
  }
}

// K-major SW128 operand whose K extent spans two 64-column blocks `kb_stride`
// apart: K-step s covers columns [16s, 16s+16).
__device__ __forceinline__ void mma_kmajor_2blocks(uint32_t tmem_d, uint32_t a_base,
                                                   uint32_t a_kb_stride, uint32_t a_sbo,
                                                   uint32_t b_base, uint32_t b_kb_stride,
                                                   uint32_t b_sbo, uint32_t b_lbo, uint32_t idesc,
                                                   bool accumulate_first, bool b_mn,
                                                   uint32_t b_mn_kstep) {
  for (int kb = 0; kb < 2; ++kb) {
    const uint64_t a0 = umma_desc_sw128(a_base + kb * a_kb_stride, 16, a_sbo);
    uint64_t b0;
    if (b_mn) {
      b0 = umma_desc_sw128(b_base + kb * 4 * b_mn_kstep, b_lbo, b_sbo);
    } else {
      b0 = umma_desc_sw128(b_base + kb * b_kb_stride, 16, b_sbo);
    }
    mma_steps(tmem_d, a0, b0, 32, b_mn ? b_mn_kstep : 32, 4, idesc, accumulate_first || kb > 0);
  }
}

struct Maps {
  CUtensorMap q, k, v;
};

template <bool DIAG, int NV>
__global__ void __launch_bounds__(kThreads, 1)
chunk_engine_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ Ag,
                    const float* __restrict__ Wg, const float* __restrict__ Rg, const float* S0,
                    const float* __restrict__ P0, float* __restrict__ O, float* S_out,
                    float* __restrict__ P_out, int T, int H, int dv, float kappa,
                    uint32_t* __restrict__ err) {
  using P = Plan<DIAG, NV>;
  constexpr int NVB = P::NVB;
  constexpr int HC = NV / 2;  // value columns per warp in the epilogues
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023u));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nvblk = dv / NV;
  const int bh = blockIdx.x / nvblk, vblk = blockIdx.x % nvblk;
  const int b = bh / H, h = bh % H;
  const int v0 = vblk * NV;
  const int nchunks = (T + kC - 1) / kC;
  const int sub = warp & 3;      // TMEM lane quarter of this warp
  const int colhalf = warp >> 2; // which half of the columns this warp handles

  float* sA = reinterpret_cast<float*>(smem + P::OFF_SA);
  float* sT = reinterpret_cast<float*>(smem + P::OFF_ST);
  float* sX = reinterpret_cast<float*>(smem + P::OFF_X);
  float* s_a = reinterpret_cast<float*>(smem + P::OFF_SC);
  float* s_w = s_a + 64;
  float* s_r = s_a + 128;
  float* s_n = s_a + 192;
  float* s_beta = s_a + 256;  // iso: beta_t; diag: 1 / s_t
  float* s_lg = s_a + 320;
  float* s_coef = s_a + 384;
  float* s_misc = s_a + 448;  // [0]: p carry (iso), [1]: abort flag
  uint64_t* bar_full = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* bar_mma = bar_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_full + 3);
  const uint32_t sbase = smem_u32(smem);
  uint8_t* sS = smem + P::OFF_S;
  uint8_t* sTP = smem + P::OFF_TP;
  uint8_t* sG = smem + P::OFF_G;

  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    s_misc[1] = 0.f;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, P::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = (uint32_t)(32 * sub) << 16;

  // ---- initial state: this thread holds S'[k][v] for k = 32*sub + lane and
  //      v in [colhalf*HC, colhalf*HC + HC) of the CTA's value block.
  const int my_k = 32 * sub + lane;
  float Sreg[HC];
  const size_t s_head = (size_t)bh * dv * kDK;
#pragma unroll
  for (int c = 0; c < HC; ++c) {
    const int v = v0 + colhalf * HC + c;
    Sreg[c] = S0 ? S0[s_head + (size_t)v * kDK + my_k] : 0.f;
  }
  // variance carry: iso in s_misc[0] (thread 0 of warp 0 owns it), diag in a
  // register of threads 0..127 (dimension i = tid)
  float p_dim = 1.f;
  if (DIAG) {
    if (tid < kDK) p_dim = P0 ? P0[(size_t)bh * kDK + tid] : 1.f;
  } else if (tid == 0) {
    s_misc[0] = P0 ? P0[bh] : 1.f;
  }

  auto write_state_operand = [&]() {
    // S' (K = k, N = v) as an MN-major operand: [vb][k 128][64 v], hi then lo
    uint8_t* hi = sS;
    uint8_t* lo = sS + P::SREG_BYTES / 2;
#pragma unroll
    for (int c8 = 0; c8 < HC / 8; ++c8) {
      const int v = colhalf * HC + c8 * 8;
      const int vb = v >> 6;
      st_split8(hi + vb * 16384, lo + vb * 16384, my_k, (v & 63) >> 3, &Sreg[c8 * 8]);
    }
  };
  write_state_operand();
  fence_async_smem();

  auto issue_loads = [&](int c, int s) {
    uint8_t* kq = smem + P::OFF_KQ + s * P::KQ_BYTES;
    uint8_t* vv = smem + P::OFF_V + s * P::V_BYTES;
    mbar_expect_tx(&bar_full[s], P::KQ_BYTES + P::V_BYTES);
    const int t0 = c * kC;
#pragma unroll 1
    for (int kb = 0; kb < 2; ++kb) {
#pragma unroll 1
      for (int g = 0; g < 8; ++g) {
        tma_load_4d(kq + kb * 16384 + (2 * g) * 1024, &tm_k, &bar_full[s], kb * 64, h,
                    t0 + 8 * g, b);
        tma_load_4d(kq + kb * 16384 + (2 * g + 1) * 1024, &tm_q, &bar_full[s], kb * 64, h,
                    t0 + 8 * g, b);
      }
    }
#pragma unroll 1
    for (int vb = 0; vb < NVB; ++vb)
      tma_load_4d(vv + vb * 8192, &tm_v, &bar_full[s], v0 + vb * 64, h, t0, b);
  };

  // MMA issue helpers (thread 0 only)
  constexpr uint32_t ID_D1 = umma_idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_D2 = umma_idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t ID_D34 = umma_idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t ID_D5 = umma_idesc_bf16(128, NV, 1, 1);

  // parity of a TMA stage load / MMA commit not yet seen complete (-1: none);
  // only thread 0 issues, so only its copies matter for the drain
  int pend_load[2] = {-1, -1};
  int pend_mma = -1;
  uint32_t mma_phase = 0;
  if (tid == 0) {
    issue_loads(0, 0);
    pend_load[0] = 0;
    if (nchunks > 1) {
      issue_loads(1, 1);
      pend_load[1] = 0;
    }
  }
  __syncthreads();

  // Bounded wait by every thread; on a timeout, record it and raise the abort
  // flag that all threads check after the next barrier.
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity)) {
      atomicOr(err, DEV_TIMEOUT);
      s_misc[1] = 1.f;
      return false;
    }
    return true;
  };


  for (int c = 0; c < nchunks; ++c) {
    const int s = c & 1;
    const int t0 = c * kC;
    const int valid = min(kC, T - t0);
    uint8_t* kq = smem + P::OFF_KQ + s * P::KQ_BYTES;
    uint8_t* vv = smem + P::OFF_V + s * P::V_BYTES;
    const uint32_t kq_a = sbase + P::OFF_KQ + s * P::KQ_BYTES;

    if (tid < kC) {
      const bool in = tid < valid;
      const size_t tok = ((size_t)b * T + t0 + tid) * H + h;
      s_a[tid] = in ? Ag[tok] : 1.f;
      s_r[tid] = in ? Rg[tok] : 1.f;
      if (!DIAG) s_w[tid] = in ? Wg[tok] : 0.f;
    }
    if (wait_bar(&bar_full[s], (uint32_t)((c >> 1) & 1)) && tid == 0) pend_load[s] = -1;
    tc_fence_before();
    __syncthreads();
    if (s_misc[1] != 0.f) break;

    // ---- MMA2 (both variants) and MMA1 (iso) need only the tiles and S
    if (tid == 0) {
      tc_fence_after();
      // D2 = [K;Q] S' (hi, then lo)
      mma_kmajor_2blocks(tmem + P::COL_D2, kq_a, 16384, 1024, sbase + P::OFF_S, 0, 1024, 16384,
                         ID_D2, false, true, 2048);
      mma_kmajor_2blocks(tmem + P::COL_D2, kq_a, 16384, 1024,
                         sbase + P::OFF_S + P::SREG_BYTES / 2, 0, 1024, 16384, ID_D2, true, true,
                         2048);
      if (!DIAG) {
        // D1 = [K;Q] K'  (B = the K rows: even 8-row groups, stride 2048 B)
        mma_kmajor_2blocks(tmem + P::COL_D1, kq_a, 16384, 1024, kq_a, 16384, 2048, 16, ID_D1,
                           false, false, 0);
      }
      if (!DIAG) {
        umma_commit(bar_mma);
        pend_mma = (int)mma_phase;
      }
    }

    // ---- per-token quantities
    if (!DIAG) {
      // n_t = ||k_t||^2 from the K tile (4 threads per token)
      {
        const int t = tid >> 2, q4 = tid & 3;
        const int row = il_row(t, 0);
        const uint8_t* tile = kq + (q4 >> 1) * 16384;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t chunk = (uint32_t)((q4 & 1) * 4 + i);
          const uint4 u = *reinterpret_cast<const uint4*>(
              tile + row * 128 + ((chunk ^ (uint32_t)(row & 7)) << 4));
          const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(wds[j] << 16);
            const float hi = __uint_as_float(wds[j] & 0xffff0000u);
            acc = fmaf(lo, lo, acc);
            acc = fmaf(hi, hi, acc);
          }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (q4 == 0) s_n[t] = acc;
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns tokens 2l, 2l+1: log-decay prefix and the Mobius scan
        const int t0l = 2 * lane, t1l = 2 * lane + 1;
        const float a0 = s_a[t0l], a1 = s_a[t1l];
        const float l0 = __logf(a0), l1 = __logf(a1);
        float incl = l0 + l1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float o = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += o;
        }
        const float lg0 = incl - l1, lg1 = incl;
        s_lg[t0l] = lg0;
        s_lg[t1l] = lg1;
        const float lg_last = __shfl_sync(0xffffffffu, lg1, 31);
        const float n0 = s_n[t0l], n1 = s_n[t1l];
        const float w0 = s_w[t0l], w1 = s_w[t1l], r0 = s_r[t0l], r1 = s_r[t1l];
        const float c0 = kappa * n0, c1 = kappa * n1;
        const Mat2 M0 = {r0 * a0 * a0, r0 * w0, c0 * a0 * a0, fmaf(c0, w0, r0)};
        const Mat2 M1 = {r1 * a1 * a1, r1 * w1, c1 * a1 * a1, fmaf(c1, w1, r1)};
        Mat2 Pm = mnorm(mmul(M1, M0));
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          Mat2 o;
          o.a = __shfl_up_sync(0xffffffffu, Pm.a, d);
          o.b = __shfl_up_sync(0xffffffffu, Pm.b, d);
          o.c = __shfl_up_sync(0xffffffffu, Pm.c, d);
          o.d = __shfl_up_sync(0xffffffffu, Pm.d, d);
          if (lane >= d) Pm = mnorm(mmul(Pm, o));
        }
        Mat2 ex;
        ex.a = __shfl_up_sync(0xffffffffu, Pm.a, 1);
        ex.b = __shfl_up_sync(0xffffffffu, Pm.b, 1);
        ex.c = __shfl_up_sync(0xffffffffu, Pm.c, 1);
        ex.d = __shfl_up_sync(0xffffffffu, Pm.d, 1);
        const float carry = s_misc[0];
        float p = lane == 0 ? carry : __fdividef(fmaf(ex.a, carry, ex.b), fmaf(ex.c, carry, ex.d));
        const float pp0 = fmaf(a0 * a0, p, w0);
        p = __fdividef(r0 * pp0, fmaf(c0, pp0, r0));
        const float pp1 = fmaf(a1 * a1, p, w1);
        p = __fdividef(r1 * pp1, fmaf(c1, pp1, r1));
        const float b0 = __fdividef(pp0, fmaf(pp0, n0, r0));
        const float b1 = __fdividef(pp1, fmaf(pp1, n1, r1));
        s_beta[t0l] = b0;
        s_beta[t1l] = b1;
        s_coef[t0l] = b0 * __expf(lg_last - lg0);
        s_coef[t1l] = b1 * __expf(lg_last - lg1);
        const float pnext = __shfl_sync(0xffffffffu, p, 31);
        __syncwarp();
        if (lane == 0) s_misc[0] = pnext;
      }
    } else {
      // diag: dimension i = tid (< 128) runs the recursion over the chunk and
      // writes the unnormalised gain G~ = p- * k (hi/lo, [kb][t][64]);
      // warp 4 forms the log-decay prefix.
      if (tid < kDK) {
        const int i = tid;
        const int kb = i >> 6, col = i & 63;
        const uint8_t* ktile = kq + kb * 16384;
        uint8_t* ghi = sG + kb * 8192;
        uint8_t* glo = sG + 16384 + kb * 8192;
        const size_t tok0 = ((size_t)b * T + t0) * H + h;
        float wv[kC];
#pragma unroll
        for (int t = 0; t < kC; ++t)
          wv[t] = (t < valid) ? Wg[(tok0 + (size_t)t * H) * kDK + i] : 0.f;
        float p = p_dim;
#pragma unroll
        for (int t = 0; t < kC; ++t) {
          const float a = s_a[t], r = s_r[t];
          const float k = ld_bf16(ktile, il_row(t, 0), col);
          const float pp = fmaf(a * a, p, wv[t]);
          p = __fdividef(r * pp, fmaf(k * k, pp, r));
          const float g = pp * k;
          __nv_bfloat16 gh, gl;
          split_bf16(g, gh, gl);
          *reinterpret_cast<__nv_bfloat16*>(ghi + sw128_offset(t, col)) = gh;
          *reinterpret_cast<__nv_bfloat16*>(glo + sw128_offset(t, col)) = gl;
        }
        p_dim = p;
      } else if (warp == 4) {
        const int t0l = 2 * lane, t1l = 2 * lane + 1;
        const float l0 = __logf(s_a[t0l]), l1 = __logf(s_a[t1l]);
        float incl = l0 + l1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float o = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += o;
        }
        s_lg[t0l] = incl - l1;
        s_lg[t1l] = incl;
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        // D1 = [K;Q] G~' (hi, then lo)
        mma_kmajor_2blocks(tmem + P::COL_D1, kq_a, 16384, 1024, sbase + P::OFF_G, 8192, 1024, 16,
                           ID_D1, false, false, 0);
        mma_kmajor_2blocks(tmem + P::COL_D1, kq_a, 16384, 1024, sbase + P::OFF_G + 16384, 8192,
                           1024, 16, ID_D1, true, false, 0);
        umma_commit(bar_mma);
        pend_mma = (int)mma_phase;
      }
    }
    __syncthreads();

    // ---- wait for MMA1 + MMA2
    if (wait_bar(bar_mma, mma_phase)) pend_mma = -1;
    mma_phase ^= 1u;
    tc_fence_after();

    // lane roles in the interleaved 128-row results
    const int m = 32 * sub + lane;
    const int tk = il_token(m);        // token of this lane's row
    const bool second = il_second(m);  // Q row (D1, D2) / lo row (D3, D4)

    // ---- D1 epilogue: A (first-half rows) and P (second-half rows)
    float d1[32];
    {
      float tmp[16];
      tmem_ld16(tmem + tm_lane + P::COL_D1 + colhalf * 32, tmp);
#pragma unroll
      for (int i = 0; i < 16; ++i) d1[i] = tmp[i];
      tmem_ld16(tmem + tm_lane + P::COL_D1 + colhalf * 32 + 16, tmp);
#pragma unroll
      for (int i = 0; i < 16; ++i) d1[16 + i] = tmp[i];
      tmem_wait_ld();
    }
    if (DIAG) {
      // innovation variance s_t = (K G~')_tt + r_t; 1/s_t into s_beta
      if (!second && (tk >> 5) == colhalf) s_beta[tk] = 1.f / (d1[tk & 31] + s_r[tk]);
      __syncthreads();
      if (tid < kC) {
        s_coef[tid] = s_beta[tid] * __expf(s_lg[kC - 1] - s_lg[tid]);
      }
    }
    const float lg_t = s_lg[tk];
    float preg[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int j = colhalf * 32 + i;
      const float wj = s_beta[j];  // iso: beta_j; diag: 1/s_j
      const float dec = __expf(lg_t - s_lg[j]);
      const float val = dec * wj * d1[i];
      if (!second) {
        sA[tk * kScrLd + j] = (j < tk) ? val : 0.f;
      } else {
        preg[i] = (j <= tk) ? val : 0.f;
      }
    }

    // ---- D2 epilogue: Z = V - gamma K S' (first-half lanes take the first
    //      half of this warp's columns, second-half lanes the rest)
    {
      const float gam = __expf(lg_t);
      float d2[HC];
#pragma unroll
      for (int c16 = 0; c16 < HC / 16; ++c16) {
        float tmp[16];
        tmem_ld16(tmem + tm_lane + P::COL_D2 + colhalf * HC + 16 * c16, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) d2[16 * c16 + i] = tmp[i];
      }
      tmem_wait_ld();
      constexpr int QC = HC / 2;
      float z[QC];
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, d2[QC + i], 8);
        const float ks = second ? other : d2[i];
        const int v = colhalf * HC + (second ? QC : 0) + i;  // column within the CTA block
        const float vv_ = ld_bf16(vv + (v >> 6) * 8192, tk, v & 63);
        z[i] = vv_ - gam * ks;
      }
      // Z hi -> sS[0 : ZU), Z lo -> sS[ZU : 2 ZU); layout [vb][t][64]
#pragma unroll
      for (int c8 = 0; c8 < QC / 8; ++c8) {
        const int v = colhalf * HC + (second ? QC : 0) + c8 * 8;
        st_split8(sS + (v >> 6) * 8192, sS + P::ZU_BYTES + (v >> 6) * 8192, tk, (v & 63) >> 3,
                  &z[c8 * 8]);
      }
    }
    __syncthreads();

    // ---- T = (I + A)^-1, blocked 16x16 forward substitution
    if (tid < 64) {
      const int blk = tid >> 4, cc = tid & 15;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < i; ++l) acc = fmaf(sA[(16 * blk + i) * kScrLd + 16 * blk + l], x[l], acc);
        x[i] = (i == cc) ? 1.f : (i < cc ? 0.f : -acc);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) sT[(16 * blk + i) * kScrLd + 16 * blk + cc] = x[i];
    }
    // upper blocks of T are zero
    for (int e = tid; e < 64 * 64; e += kThreads) {
      const int r = e >> 6, cl = e & 63;
      if ((cl >> 4) > (r >> 4)) sT[r * kScrLd + cl] = 0.f;
    }
    __syncthreads();
    // levels d = 1, 2, 3 of the block recursion T_ib = -T_ii sum_l A_il T_lb
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      const int npairs = 4 - d;
      const int r = tid >> 4, cc = tid & 15;
      for (int pr = 0; pr < npairs; ++pr) {
        const int bb = pr, ii = pr + d;
        float acc = 0.f;
        for (int l = bb; l < ii; ++l) {
#pragma unroll
          for (int mm = 0; mm < 16; ++mm)
            acc = fmaf(sA[(16 * ii + r) * kScrLd + 16 * l + mm], sT[(16 * l + mm) * kScrLd + 16 * bb + cc], acc);
        }
        sX[pr * 272 + r * 17 + cc] = acc;
      }
      __syncthreads();
      for (int pr = 0; pr < npairs; ++pr) {
        const int bb = pr, ii = pr + d;
        float acc = 0.f;
#pragma unroll
        for (int mm = 0; mm < 16; ++mm)
          acc = fmaf(sT[(16 * ii + r) * kScrLd + 16 * ii + mm], sX[pr * 272 + mm * 17 + cc], acc);
        sT[(16 * ii + r) * kScrLd + 16 * bb + cc] = -acc;
      }
      __syncthreads();
    }
    // T hi/lo into the interleaved A operand [128][64] (row il_row(t, 0|1))
    {
      const int t = tid >> 2, q = tid & 3;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = sT[t * kScrLd + 16 * q + i];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        __nv_bfloat16 hv[8], lv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) split_bf16(x[8 * half + i], hv[i], lv[i]);
        const uint32_t col8 = (uint32_t)(2 * q + half);
        *reinterpret_cast<uint4*>(sTP + sw128_offset(il_row(t, 0), col8 * 8)) =
            make_uint4(pack2(hv[0], hv[1]), pack2(hv[2], hv[3]), pack2(hv[4], hv[5]), pack2(hv[6], hv[7]));
        *reinterpret_cast<uint4*>(sTP + sw128_offset(il_row(t, 1), col8 * 8)) =
            make_uint4(pack2(lv[0], lv[1]), pack2(lv[2], lv[3]), pack2(lv[4], lv[5]), pack2(lv[6], lv[7]));
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- MMA3: D3 = [T_hi;T_lo] Z  (Z hi then lo; B MN-major [vb][t][64])
    if (tid == 0) {
      tc_fence_after();
      const uint64_t a0 = umma_desc_sw128(sbase + P::OFF_TP, 16, 1024);
      const uint64_t bz_hi = umma_desc_sw128(sbase + P::OFF_S, 8192, 1024);
      const uint64_t bz_lo = umma_desc_sw128(sbase + P::OFF_S + P::ZU_BYTES, 8192, 1024);
      mma_steps(tmem + P::COL_D3, a0, bz_hi, 32, 2048, 4, ID_D34, false);
      mma_steps(tmem + P::COL_D3, a0, bz_lo, 32, 2048, 4, ID_D34, true);
      umma_commit(bar_mma);
      pend_mma = (int)mma_phase;
    }
    if (wait_bar(bar_mma, mma_phase)) pend_mma = -1;
    mma_phase ^= 1u;
    tc_fence_after();

    // ---- D3 epilogue: U = top + bottom; U hi/lo and B = coef U hi/lo
    {
      constexpr int QC = HC / 2;
      float d3[HC];
#pragma unroll
      for (int c16 = 0; c16 < HC / 16; ++c16) {
        float tmp[16];
        tmem_ld16(tmem + tm_lane + P::COL_D3 + colhalf * HC + 16 * c16, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) d3[16 * c16 + i] = tmp[i];
      }
      tmem_wait_ld();
      float u[QC];
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, second ? d3[i] : d3[QC + i], 8);
        u[i] = (second ? d3[QC + i] : d3[i]) + other;
      }
      const float coef = s_coef[tk];
      float bu[QC];
#pragma unroll
      for (int i = 0; i < QC; ++i) bu[i] = coef * u[i];
      // U -> sS[0 : 2ZU) (hi, lo); B -> sS[2ZU : 4ZU)
#pragma unroll
      for (int c8 = 0; c8 < QC / 8; ++c8) {
        const int v = colhalf * HC + (second ? QC : 0) + c8 * 8;
        const uint32_t vo = (uint32_t)(v >> 6) * 8192;
        st_split8(sS + vo, sS + P::ZU_BYTES + vo, tk, (v & 63) >> 3, &u[c8 * 8]);
        st_split8(sS + 2 * P::ZU_BYTES + vo, sS + 3 * P::ZU_BYTES + vo, tk, (v & 63) >> 3,
                  &bu[c8 * 8]);
      }
      // P hi/lo (held by the second-half lanes) into the interleaved A operand
      if (second) {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          __nv_bfloat16 hv[8], lv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) split_bf16(preg[8 * c8 + i], hv[i], lv[i]);
          const uint32_t col = (uint32_t)(colhalf * 32 + 8 * c8);
          *reinterpret_cast<uint4*>(sTP + sw128_offset(il_row(tk, 0), col)) =
              make_uint4(pack2(hv[0], hv[1]), pack2(hv[2], hv[3]), pack2(hv[4], hv[5]), pack2(hv[6], hv[7]));
          *reinterpret_cast<uint4*>(sTP + sw128_offset(il_row(tk, 1), col)) =
              make_uint4(pack2(lv[0], lv[1]), pack2(lv[2], lv[3]), pack2(lv[4], lv[5]), pack2(lv[6], lv[7]));
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (s_misc[1] != 0.f) break;

    // ---- MMA4 (output) and MMA5 (state)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t a0 = umma_desc_sw128(sbase + P::OFF_TP, 16, 1024);
      const uint64_t bu_hi = umma_desc_sw128(sbase + P::OFF_S, 8192, 1024);
      const uint64_t bu_lo = umma_desc_sw128(sbase + P::OFF_S + P::ZU_BYTES, 8192, 1024);
      mma_steps(tmem + P::COL_D4, a0, bu_hi, 32, 2048, 4, ID_D34, false);
      mma_steps(tmem + P::COL_D4, a0, bu_lo, 32, 2048, 4, ID_D34, true);
      const uint64_t bb_hi = umma_desc_sw128(sbase + P::OFF_S + 2 * P::ZU_BYTES, 8192, 1024);
      const uint64_t bb_lo = umma_desc_sw128(sbase + P::OFF_S + 3 * P::ZU_BYTES, 8192, 1024);
      if (!DIAG) {
        // A = K' (MN-major view of the K rows: d-blocks 16 KB apart, token
        // groups 2048 B apart)
        const uint64_t ak = umma_desc_sw128(kq_a, 16384, 2048);
        mma_steps(tmem + P::COL_D5, ak, bb_hi, 4096, 2048, 4, ID_D5, false);
        mma_steps(tmem + P::COL_D5, ak, bb_lo, 4096, 2048, 4, ID_D5, true);
      } else {
        const uint64_t ag_hi = umma_desc_sw128(sbase + P::OFF_G, 8192, 1024);
        const uint64_t ag_lo = umma_desc_sw128(sbase + P::OFF_G + 16384, 8192, 1024);
        mma_steps(tmem + P::COL_D5, ag_hi, bb_hi, 2048, 2048, 4, ID_D5, false);
        mma_steps(tmem + P::COL_D5, ag_hi, bb_lo, 2048, 2048, 4, ID_D5, true);
        mma_steps(tmem + P::COL_D5, ag_lo, bb_hi, 2048, 2048, 4, ID_D5, true);
      }
      umma_commit(bar_mma);
      pend_mma = (int)mma_phase;
    }
    if (wait_bar(bar_mma, mma_phase)) pend_mma = -1;
    mma_phase ^= 1u;
    tc_fence_after();
    __syncthreads();
    if (s_misc[1] != 0.f) break;
    if (tid == 0 && c + 2 < nchunks) {
      issue_loads(c + 2, s);
      pend_load[s] = ((c + 2) >> 1) & 1;
    }

    // ---- output: o_t = D4 top + D4 bottom + gamma_t (Q S')_t
    {
      constexpr int QC = HC / 2;
      const float gam = __expf(lg_t);
      float d4[HC], q2[HC];
#pragma unroll
      for (int c16 = 0; c16 < HC / 16; ++c16) {
        float tmp[16], tmp2[16];
        tmem_ld16(tmem + tm_lane + P::COL_D4 + colhalf * HC + 16 * c16, tmp);
        tmem_ld16(tmem + tm_lane + P::COL_D2 + colhalf * HC + 16 * c16, tmp2);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          d4[16 * c16 + i] = tmp[i];
          q2[16 * c16 + i] = tmp2[i];
        }
      }
      tmem_wait_ld();
      float ov[QC];
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float send = second ? fmaf(gam, q2[i], d4[i]) : d4[QC + i];
        const float other = __shfl_xor_sync(0xffffffffu, send, 8);
        ov[i] = second ? (fmaf(gam, q2[QC + i], d4[QC + i]) + other) : (d4[i] + other);
      }
      if (tk < valid) {
        const int vcol = v0 + colhalf * HC + (second ? QC : 0);
        float* dst = O + (((size_t)b * T + t0 + tk) * H + h) * dv + vcol;
#pragma unroll
        for (int i = 0; i < QC; i += 4)
          *reinterpret_cast<float4*>(dst + i) = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
      }
    }

    // ---- state: S' = gamma_C S' + D5
    {
      const float gC = __expf(s_lg[kC - 1]);
#pragma unroll
      for (int c16 = 0; c16 < HC / 16; ++c16) {
        float tmp[16];
        tmem_ld16(tmem + tm_lane + P::COL_D5 + colhalf * HC + 16 * c16, tmp);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) Sreg[16 * c16 + i] = fmaf(gC, Sreg[16 * c16 + i], tmp[i]);
      }
    }
    __syncthreads();  // all reads of U/B in sS are long done (MMA waited); S overwrites them
    write_state_operand();
    fence_async_smem();
    tc_fence_before();
  }

  // ---- drain (only the abort path has anything left): bounded waits for
  //      the copies and MMAs still in flight before TMEM is released
  if (tid == 0) {
    for (int st = 0; st < 2; ++st)
      if (pend_load[st] >= 0) (void)mbar_wait(&bar_full[st], (uint32_t)pend_load[st]);
    if (pend_mma >= 0) (void)mbar_wait(bar_mma, (uint32_t)pend_mma);
  }
  __syncthreads();
  const bool aborted = s_misc[1] != 0.f;

  // ---- final state and variance
  if (!aborted) {
#pragma unroll
    for (int c = 0; c < HC; ++c) {
      const int v = v0 + colhalf * HC + c;
      S_out[s_head + (size_t)v * kDK + my_k] = Sreg[c];
    }
    if (vblk == 0) {
      if (DIAG) {
        if (tid < kDK) P_out[(size_t)bh * kDK + tid] = p_dim;
      } else if (tid == 0) {
        P_out[bh] = s_misc[0];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, P::TMEM_COLS);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B, T, H, d] bf16 tensor, boxes of (64 columns, 1 head, box_t tokens, 1 batch)
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int d, int box_t) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_t, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool DIAG, int NV>
kdn_status launch(const void* q, const void* k, const void* v, const float* a, const float* w,
                  const float* r, const float* S0, const float* p0, float* o, float* S_out,
                  float* p_out, int B, int T, int H, int dv, float kappa, void* ws,
                  cudaStream_t s) {
  using P = Plan<DIAG, NV>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, B, T, H, kDK, 8) || !make_map(&mk, k, B, T, H, kDK, 8) ||
      !make_map(&mv, v, B, T, H, dv, 64))
    return KDN_ERR_CUDA;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(chunk_engine_kernel<DIAG, NV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, P::ALLOC) != cudaSuccess)
      return KDN_ERR_CUDA;
    attr_set = true;
  }
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return KDN_ERR_CUDA;
  // Several CTAs of one head read p0 while one of them writes p_out, which
  // may alias p0: they read a snapshot taken on the stream first.
  if (p0) {
    float* snap = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
    const size_t n = (size_t)B * H * (DIAG ? kDK : 1);
    if (cudaMemcpyAsync(snap, p0, n * sizeof(float), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return KDN_ERR_CUDA;
    p0 = snap;
  }
  const unsigned grid = (unsigned)(B * H * (dv / NV));
  chunk_engine_kernel<DIAG, NV><<<grid, kThreads, P::ALLOC, s>>>(
      mq, mk, mv, a, w, r, S0, p0, o, S_out, p_out, T, H, dv, kappa,
      static_cast<uint32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

}  // namespace

bool chunk_engine_supported(kdn_dtype dt, int dk, int dv) {
  return dt == KDN_BF16 && dk == kDK && (dv == 64 || dv == 128);
}

size_t chunk_engine_workspace_size(bool diag, int B, int H) {
  const size_t snap = (size_t)B * H * (diag ? kDK : 1) * sizeof(float);
  return 256 + (snap + 255) / 256 * 256;
}

kdn_status chunk_engine_launch(bool diag, const void* q, const void* k, const void* v,
                               const float* a, const float* w, const float* r, const float* S0,
                               const float* p0, float* o, float* S_out, float* p_out, int B,
                               int T, int H, int dv, float kappa, void* ws, cudaStream_t s) {
  if (diag) return launch<true, 64>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, ws, s);
  if (dv == 128) return launch<false, 128>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, ws, s);
  return launch<false, 64>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, ws, s);
}

}  // namespace kdn
