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
// k_t) g_t'; the pages only say that a hardware-efficient chunkwise form
// exists).  The variance recursion (a Mobius map per token and lane) crosses
// chunks through one carried value per lane.
//
// Two engines.  The warp-specialised one further down serves d_v = 128 (both
// variants).  The lock-step one here serves d_v = 64: one CTA owns one
// (batch, head, block of NV = 64 value columns) for the whole sequence, 16
// warps.  The K/Q tiles are double-buffered and the V tile is
// single-buffered; the copies of chunk c+1 (and its per-token scalars) are
// issued during chunk c's diagonal-block solve, when 14 of the 16 warps are
// idle and both buffers are free.  Per chunk:
//   MMA1  D1 = [K;Q] G~'          (iso: G~ = K; diag: G~ = p- * k, hi/lo)
//   MMA2  D2 = [K;Q] S'           (S as bf16 hi + lo)
//   SIMT  A, T = (I+A)^-1 (16x16 blocks, in place), Z = V - gamma K S'
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
//
// Every wait is bounded.  A wait that gives up records DEV_TIMEOUT in the
// workspace error word and raises an abort flag; the CTA then waits (bounded)
// for its MMAs and copies in flight, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kC = 64;                   // tokens per chunk
constexpr int kDK = 128;                 // key dimension of the engine
constexpr int kCompute = 512;            // 16 warps
constexpr int kThreads = kCompute;
constexpr int kIssueWarp = 15;           // its lane 0 issues the TMA copies
constexpr int kScalarWarp = 14;          // fetches the per-token scalars
constexpr int kMma2Warp = 13;            // its lane 0 issues MMA2
constexpr int kLd = 68;                  // fp32 row stride of the 64x64 solve buffer

template <bool DIAG, int NV>
struct Plan {
  static constexpr int HC = NV / 4;  // result columns per warp
  static constexpr int QC = HC / 2;  // result columns per lane (interleaved results)
  static constexpr uint32_t KQ_BYTES = 2u * 128u * 128u;  // [kb 2][128 rows][64] bf16
  static constexpr uint32_t V_BYTES = NV * 128u;          // [vb][64 t][64] bf16
  static constexpr uint32_t S_BYTES = NV * 512u;          // S' hi+lo [vb][128 k][64]
  static constexpr uint32_t ZU_BYTES = NV * 128u;         // one of Z/U/B (hi or lo)
  static constexpr uint32_t OFF_KQ = 0;
  static constexpr uint32_t OFF_V = OFF_KQ + 2 * KQ_BYTES;
  static constexpr uint32_t OFF_S = OFF_V + V_BYTES;
  static constexpr uint32_t OFF_TP = OFF_S + S_BYTES;     // [128][64] bf16 (T, then P)
  static constexpr uint32_t OFF_G = OFF_TP + 16384u;      // diag: G~ hi, lo [kb][64][64]
  static constexpr uint32_t OFF_AT = OFF_G + (DIAG ? 32768u : 0u);  // fp32 [64][68]
  static constexpr uint32_t OFF_X = OFF_AT + 64u * kLd * 4u;          // fp32 [4][16][18]
  static constexpr uint32_t OFF_SC = OFF_X + 4608u;                   // 1152 floats
  static constexpr uint32_t OFF_BAR = OFF_SC + 4608u;
  static constexpr uint32_t TOTAL = OFF_BAR + 128u;
  static constexpr uint32_t ALLOC = TOTAL + 1024u;
  static constexpr uint32_t COL_D1 = 0, COL_D2 = 64, COL_D3 = 64 + NV, COL_D4 = 64 + 2 * NV;
  static constexpr uint32_t COL_D5 = COL_D3;
  static constexpr uint32_t TMEM_COLS = (64 + 3 * NV) <= 256 ? 256u : 512u;
  static_assert(TOTAL <= 227u * 1024u, "shared memory plan too large");
  static_assert(NV == 64 || NV == 128, "value block");
};

__device__ __forceinline__ int il_token(int m) { return 8 * (m >> 4) + (m & 7); }
__device__ __forceinline__ int il_second(int m) { return (m >> 3) & 1; }
__device__ __forceinline__ int il_row(int t, int second) {
  return 16 * (t >> 3) + (t & 7) + 8 * second;
}

// Byte offset of 16-byte chunk col8 of swizzled 128-byte row `row`.
__device__ __forceinline__ uint32_t chunk_off(uint32_t row, uint32_t col8) {
  return row * 128u + (((col8 ^ row) & 7u) << 4);
}

// (hi, lo) bf16 splits of 8 floats, packed as two uint4.
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    const uint32_t hu = *reinterpret_cast<const uint32_t*>(&hb);
    const float h0 = __uint_as_float(hu << 16);
    const float h1 = __uint_as_float(hu & 0xffff0000u);
    const __nv_bfloat162 lb = __floats2bfloat162_rn(x[2 * i] - h0, x[2 * i + 1] - h1);
    hw[i] = hu;
    lw[i] = *reinterpret_cast<const uint32_t*>(&lb);
  }
  hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// hi half of x[0..7] into (hi_tile, hi_row), lo half into (lo_tile, lo_row),
// both at 16-byte chunk col8.
__device__ __forceinline__ void st_split8(uint8_t* hi_tile, uint32_t hi_row, uint8_t* lo_tile,
                                          uint32_t lo_row, uint32_t col8, const float* x) {
  uint4 hv, lv;
  split8(x, hv, lv);
  *reinterpret_cast<uint4*>(hi_tile + chunk_off(hi_row, col8)) = hv;
  *reinterpret_cast<uint4*>(lo_tile + chunk_off(lo_row, col8)) = lv;
}

// 8 bf16 of chunk col8 of swizzled row `row`, as floats.
__device__ __forceinline__ void ld_bf16x8(const uint8_t* tile, uint32_t row, uint32_t col8,
                                          float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(tile + chunk_off(row, col8));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float ld_bf16(const uint8_t* tile, uint32_t row, uint32_t col) {
  return __bfloat162float(
      *reinterpret_cast<const __nv_bfloat16*>(tile + sw128_offset(row, col)));
}

struct Mat2 { float a, b, c, d; };
__device__ __forceinline__ Mat2 mmul(const Mat2& x, const Mat2& y) {
  return {fmaf(x.a, y.a, x.b * y.c), fmaf(x.a, y.b, x.b * y.d), fmaf(x.c, y.a, x.d * y.c),
          fmaf(x.c, y.b, x.d * y.d)};
}
// Exact power-of-two renormalisation by the largest entry's binade.
__device__ __forceinline__ Mat2 mnorm(const Mat2& x) {
  const float m = fmaxf(fmaxf(x.a, x.b), fmaxf(x.c, x.d));
  const int e = (int)((__float_as_uint(m) >> 23) & 0xffu) - 127;
  if (e > -100 && e < 100 && e != 0) {
    const float s = __uint_as_float((uint32_t)(127 - e) << 23);
    return {x.a * s, x.b * s, x.c * s, x.d * s};
  }
  return x;
}

// Named barriers are the aligned form, which needs the whole warp to arrive
// together: single-lane issue blocks and bounded waits diverge warps, so each
// barrier first reconverges its warp.
__device__ __forceinline__ void bar_compute() {
  __syncwarp();
  asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory");
}

// `steps` consecutive K=16 MMAs; descriptor start addresses advance by
// a_step / b_step bytes per step.
__device__ __forceinline__ void mma_steps(uint32_t tmem_d, uint64_t a0, uint64_t b0,
                                          uint32_t a_step, uint32_t b_step, int steps,
                                          uint32_t idesc, bool accumulate_first) {
  for (int s = 0; s < steps; ++s)
    umma_bf16(tmem_d, a0 + (uint64_t)((s * a_step) >> 4), b0 + (uint64_t)((s * b_step) >> 4),
              idesc, (accumulate_first || s > 0) ? 1u : 0u);
}

// The off-diagonal 16x16 blocks of T = (I + A)^-1 at level D (block row i =
// block column b + D): T_ib = -T_ii sum_{l=b}^{i-1} A_il T_lb, stored
// transposed in the upper triangle, T_ib[r][c] at AT[16 b + c][16 i + r].
// Each term A_il T_lb is a task of 64 threads (2x2 outputs each); every loop
// bound is a compile-time constant.
template <int BAR, int NT>
__device__ __forceinline__ void named_bar() {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Every level uses at most 256 threads (tid < 256); BAR / NT name the barrier
// of the threads that run the solve.
template <int D, int BAR = 1, int NT = kCompute>
__device__ __forceinline__ void t_level(float* AT, float* X, int tid) {
  constexpr int NP = 4 - D;
  const int task = tid >> 6, e = tid & 63;
  const int r0 = 2 * (e >> 3), c0 = 2 * (e & 7);
  if (task < NP * D) {
    const int pr = task / D, bb = pr, ii = pr + D, l = bb + task % D;
    float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
    const float* a_r0 = AT + (16 * ii + r0) * kLd + 16 * l;
    if (l == bb) {
      const float* tb = AT + (16 * bb) * kLd + 16 * bb + c0;
#pragma unroll
      for (int mm = 0; mm < 16; ++mm) {
        const float2 tt = *reinterpret_cast<const float2*>(tb + mm * kLd);
        const float a0v = a_r0[mm], a1v = a_r0[kLd + mm];
        x00 = fmaf(a0v, tt.x, x00);
        x01 = fmaf(a0v, tt.y, x01);
        x10 = fmaf(a1v, tt.x, x10);
        x11 = fmaf(a1v, tt.y, x11);
      }
    } else {
      const float* tb = AT + (16 * bb + c0) * kLd + 16 * l;
#pragma unroll
      for (int mm = 0; mm < 16; ++mm) {
        const float t0v = tb[mm], t1v = tb[kLd + mm];
        const float a0v = a_r0[mm], a1v = a_r0[kLd + mm];
        x00 = fmaf(a0v, t0v, x00);
        x01 = fmaf(a0v, t1v, x01);
        x10 = fmaf(a1v, t0v, x10);
        x11 = fmaf(a1v, t1v, x11);
      }
    }
    float* xs = X + task * 288;  // [16][18]
    *reinterpret_cast<float2*>(xs + r0 * 18 + c0) = make_float2(x00, x01);
    *reinterpret_cast<float2*>(xs + (r0 + 1) * 18 + c0) = make_float2(x10, x11);
  }
  named_bar<BAR, NT>();
  if (task < NP) {
    const int pr = task, bb = pr, ii = pr + D;
    const float* t_r0 = AT + (16 * ii + r0) * kLd + 16 * ii;
    const float* xs = X + pr * D * 288 + c0;
    float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
    for (int mm = 0; mm < 16; ++mm) {
      float2 xv = *reinterpret_cast<const float2*>(xs + mm * 18);
#pragma unroll
      for (int q = 1; q < D; ++q) {
        const float2 v = *reinterpret_cast<const float2*>(xs + q * 288 + mm * 18);
        xv.x += v.x;
        xv.y += v.y;
      }
      const float ta = t_r0[mm], tb = t_r0[kLd + mm];
      y00 = fmaf(ta, xv.x, y00);
      y01 = fmaf(ta, xv.y, y01);
      y10 = fmaf(tb, xv.x, y10);
      y11 = fmaf(tb, xv.y, y11);
    }
    float* out = AT + (16 * bb + c0) * kLd + 16 * ii + r0;
    out[0] = -y00;
    out[1] = -y10;
    out[kLd] = -y01;
    out[kLd + 1] = -y11;
  }
  named_bar<BAR, NT>();
}

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
  constexpr int HC = P::HC, QC = P::QC, NVB = NV / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nvblk = dv / NV;
  const int bh = blockIdx.x / nvblk, vblk = blockIdx.x % nvblk;
  const int b = bh / H, h = bh % H;
  const int v0 = vblk * NV;
  const int nchunks = (T + kC - 1) / kC;
  const uint32_t sbase = smem_u32(smem);

  // scalar area (floats); [2][64] arrays are indexed by chunk parity
  float* scf = reinterpret_cast<float*>(smem + P::OFF_SC);
  float* sc_a = scf;           // decay a_t
  float* sc_w = scf + 128;     // iso process noise w_t
  float* sc_r = scf + 256;     // observation noise r_t
  float* sc_n = scf + 384;     // iso ||k_t||^2
  float* sc_beta = scf + 512;  // iso beta_t; diag 1 / s_t
  float* sc_lg = scf + 640;    // log2 of the in-chunk cumulative decay
  float* sc_coef = scf + 768;  // state-update coefficient
  float* sc_pcar = scf + 896;  // [128] carried variance (iso: [0])
  float* sc_misc = scf + 1024; // [0] abort flag
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* full_kq = bars;       // [2] K/Q tiles of a stage landed
  uint64_t* full_v = bars + 2;    // V tile landed
  uint64_t* mma1_bar = bars + 3;  // MMA1 (D1) finished
  uint64_t* mma2_bar = bars + 4;  // MMA2 (D2) finished
  uint64_t* mma_bar = bars + 5;   // MMA3, then MMA4 + MMA5, finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  float* AT = reinterpret_cast<float*>(smem + P::OFF_AT);
  float* X = reinterpret_cast<float*>(smem + P::OFF_X);
  uint8_t* sS = smem + P::OFF_S;
  uint8_t* sTP = smem + P::OFF_TP;
  uint8_t* sG = smem + P::OFF_G;
  uint8_t* sV = smem + P::OFF_V;

  if (tid == 0) {
    mbar_init(&full_kq[0], 1);
    mbar_init(&full_kq[1], 1);
    mbar_init(full_v, 1);
    mbar_init(mma1_bar, 1);
    mbar_init(mma2_bar, 1);
    mbar_init(mma_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    sc_misc[0] = 0.f;
  }
  if (DIAG) {
    if (tid < kDK) sc_pcar[tid] = P0 ? P0[(size_t)bh * kDK + tid] : 1.f;
  } else if (tid == 0) {
    sc_pcar[0] = P0 ? P0[bh] : 1.f;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, P::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ------------------------------------------------------- copy issue helpers
  // per-token scalars of chunk c (warp kScalarWarp): loaded early into
  // registers, stored into the chunk-parity slot later
  float ps_a[2], ps_r[2], ps_w[2];
  auto fetch_scalars = [&](int c) {
    const int t0 = c * kC, valid = min(kC, T - t0);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = lane + 32 * i;
      const bool in = t < valid;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      ps_a[i] = in ? __ldg(Ag + tok) : 1.f;
      ps_r[i] = in ? __ldg(Rg + tok) : 1.f;
      ps_w[i] = (!DIAG && in) ? __ldg(Wg + tok) : 0.f;
    }
  };
  auto store_scalars = [&](int c) {
    const int st = c & 1;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = lane + 32 * i;
      sc_a[64 * st + t] = ps_a[i];
      sc_r[64 * st + t] = ps_r[i];
      sc_w[64 * st + t] = ps_w[i];
    }
  };
  // TMA copies (one thread): chunk c's K/Q tiles into stage c & 1, its V tile
  int pend_kq[2] = {-1, -1}, pend_v = -1;  // parities of copies not yet seen landed
  auto issue_kq = [&](int c) {
    const int st = c & 1, t0 = c * kC;
    uint8_t* kqd = smem + P::OFF_KQ + st * P::KQ_BYTES;
    mbar_expect_tx(&full_kq[st], P::KQ_BYTES);
    for (int kb = 0; kb < 2; ++kb)
      for (int g = 0; g < 8; ++g) {
        tma_load_4d(kqd + kb * 16384 + (2 * g) * 1024, &tm_k, &full_kq[st], kb * 64, h,
                    t0 + 8 * g, b);
        tma_load_4d(kqd + kb * 16384 + (2 * g + 1) * 1024, &tm_q, &full_kq[st], kb * 64, h,
                    t0 + 8 * g, b);
      }
    pend_kq[st] = (c >> 1) & 1;
  };
  auto issue_v = [&](int c) {
    mbar_expect_tx(full_v, P::V_BYTES);
    for (int vb = 0; vb < NVB; ++vb)
      tma_load_4d(sV + vb * 8192, &tm_v, full_v, v0 + 64 * vb, h, c * kC, b);
    pend_v = c & 1;
  };
  const bool issuer = (warp == kIssueWarp && lane == 0);
  const bool mma2_issuer = (warp == kMma2Warp && lane == 0);
  if (issuer) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    issue_kq(0);
    issue_v(0);
  }
  if (warp == kScalarWarp) {
    fetch_scalars(0);
    store_scalars(0);
  }

  // ----------------------------------------------------------- per-thread roles
  const uint32_t tmem = *tmem_slot;
  const int sub = warp & 3;  // TMEM lane quarter
  const int cq = warp >> 2;  // column quarter
  const uint32_t tm_lane = (uint32_t)(32 * sub) << 16;
  const int m = 32 * sub + lane;     // row of a 128-row result held by this lane
  const int tk = il_token(m);        // its token (interleaved results)
  const int second = il_second(m);   // Q / lo row
  const int my_k = m;                // state row k of this thread

  // state S'[k][v], k = my_k, v in [HC cq, HC cq + HC) of this CTA's block
  float Sreg[HC];
  const size_t s_head = (size_t)bh * dv * kDK;
#pragma unroll
  for (int c = 0; c < HC; ++c)
    Sreg[c] = S0 ? S0[s_head + (size_t)(v0 + HC * cq + c) * kDK + my_k] : 0.f;

  auto write_state_operand = [&]() {
    // S' as the MN-major B operand of MMA2: [vb][k 128][64 v]; hi, then lo
    const int vcol = HC * cq;
    uint8_t* base_hi = sS + (vcol >> 6) * 16384;
    uint8_t* base_lo = base_hi + P::S_BYTES / 2;
#pragma unroll
    for (int i = 0; i < HC / 8; ++i)
      st_split8(base_hi, (uint32_t)my_k, base_lo, (uint32_t)my_k,
                (uint32_t)(((vcol & 63) >> 3) + i), &Sreg[8 * i]);
  };
  write_state_operand();
  fence_async_smem();
  bar_compute();  // chunk 0's scalars are in place

  constexpr uint32_t ID_D1 = umma_idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_D2 = umma_idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t ID_D34 = umma_idesc_bf16(128, NV, 0, 1);
  constexpr uint32_t ID_D5 = umma_idesc_bf16(128, NV, 1, 1);

  auto wait_or_abort = [&](uint64_t* bar_, uint32_t parity) -> bool {
    if (!mbar_wait(bar_, parity)) {
      atomicOr(err, DEV_TIMEOUT);
      sc_misc[0] = 1.f;
      return false;
    }
    return true;
  };

  // iso: ||k_t||^2 (all threads), then warp 0's log2-decay prefix and Mobius
  // scan of chunk c; the K tile and scalars of chunk c must be in place.
  // Ends with a barrier.
  auto iso_variance = [&](int c) {
    const int cb = c & 1;
    const uint8_t* kq = smem + P::OFF_KQ + cb * P::KQ_BYTES;
    {
      const int t = tid >> 3, part = tid & 7;  // 8 threads per token
      float x[16];
      const uint8_t* kt = kq + (part >> 2) * 16384;
      ld_bf16x8(kt, (uint32_t)il_row(t, 0), (uint32_t)((part & 3) * 2), x);
      ld_bf16x8(kt, (uint32_t)il_row(t, 0), (uint32_t)((part & 3) * 2 + 1), x + 8);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) acc = fmaf(x[i], x[i], acc);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (part == 0) sc_n[64 * cb + t] = acc;
    }
    bar_compute();
    if (warp == 0) {
      const float* a_s = sc_a + 64 * cb;
      const float* w_s = sc_w + 64 * cb;
      const float* r_s = sc_r + 64 * cb;
      const int ta = 2 * lane, tb = ta + 1;
      const float a0 = a_s[ta], a1 = a_s[tb];
      const float l0 = __log2f(a0), l1 = __log2f(a1);
      float incl = l0 + l1;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
      }
      const float lg0 = incl - l1, lg1 = incl;
      sc_lg[64 * cb + ta] = lg0;
      sc_lg[64 * cb + tb] = lg1;
      const float lg_last = __shfl_sync(0xffffffffu, lg1, 31);
      const float n0 = sc_n[64 * cb + ta], n1 = sc_n[64 * cb + tb];
      const float w0 = w_s[ta], w1 = w_s[tb], r0 = r_s[ta], r1 = r_s[tb];
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
      const float carry = sc_pcar[0];
      float p = lane == 0 ? carry
                          : __fdividef(fmaf(ex.a, carry, ex.b), fmaf(ex.c, carry, ex.d));
      const float pp0 = fmaf(a0 * a0, p, w0);
      p = __fdividef(r0 * pp0, fmaf(c0, pp0, r0));
      const float pp1 = fmaf(a1 * a1, p, w1);
      p = __fdividef(r1 * pp1, fmaf(c1, pp1, r1));
      const float b0 = __fdividef(pp0, fmaf(pp0, n0, r0));
      const float b1 = __fdividef(pp1, fmaf(pp1, n1, r1));
      sc_beta[64 * cb + ta] = b0;
      sc_beta[64 * cb + tb] = b1;
      sc_coef[64 * cb + ta] = b0 * exp2f(lg_last - lg0);
      sc_coef[64 * cb + tb] = b1 * exp2f(lg_last - lg1);
      const float pnext = __shfl_sync(0xffffffffu, p, 31);
      __syncwarp();
      if (lane == 0) sc_pcar[0] = pnext;
    }
    bar_compute();
  };

  // diag: thread (di, dq) runs dimension di over tokens [16 dq, 16 dq + 16);
  // its w values for the next chunk are prefetched into registers.
  const int di = tid & 127, dq = tid >> 7;
  float wpre[DIAG ? 16 : 1];
  auto prefetch_w = [&](int c) {
    if constexpr (DIAG) {
      const int t0 = c * kC;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = t0 + 16 * dq + i;
        wpre[i] = (c < nchunks && t < T)
                      ? __ldg(Wg + (((size_t)b * T + t) * H + h) * kDK + di)
                      : 0.f;
      }
    }
  };
  prefetch_w(0);

  uint32_t mma_phase = 0;  // phase of mma_bar (two commits per chunk)
  // parities of MMA commits not yet seen complete (thread 0), for the drain
  int pend_mma = -1, pend_mma1 = -1, pend_mma2 = -1;
  // output of the previous chunk, finished while the next chunk's MMAs run:
  // gamma_t (Q S')_t for this lane's columns and the chunk's token range
  float qpart[QC];
  int prev_t0 = 0, prev_valid = 0;

  auto finish_output = [&]() {
    // o_t = D4 top + D4 bottom + gamma_t (Q S')_t (D4 holds the previous chunk)
    float d4[HC];
#pragma unroll
    for (int i = 0; i < HC / 16; ++i) tmem_ld16(tmem + tm_lane + P::COL_D4 + HC * cq + 16 * i,
                                                *reinterpret_cast<float(*)[16]>(d4 + 16 * i));
    tmem_wait_ld();
    float ov[QC];
#pragma unroll
    for (int i = 0; i < QC; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, second ? d4[i] : d4[QC + i], 8);
      ov[i] = (second ? d4[QC + i] : d4[i]) + other + qpart[i];
    }
    if (tk < prev_valid) {
      float* dst = O + (((size_t)b * T + prev_t0 + tk) * H + h) * dv + v0 + HC * cq + QC * second;
#pragma unroll
      for (int i = 0; i < QC; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
    }
  };

  if (!DIAG) {
    if (wait_or_abort(&full_kq[0], 0u) && issuer) pend_kq[0] = -1;
    iso_variance(0);
  }

  bool aborted = false;
  for (int c = 0; c < nchunks; ++c) {
    const int s = c & 1;
    const int t0 = c * kC;
    const int valid = min(kC, T - t0);
    const bool more = c + 1 < nchunks;
    const uint32_t kq_a = sbase + P::OFF_KQ + s * P::KQ_BYTES;
    const uint8_t* kq = smem + P::OFF_KQ + s * P::KQ_BYTES;
    const float* a_s = sc_a + 64 * s;
    const float* r_s = sc_r + 64 * s;
    float* lg_c = sc_lg + 64 * s;
    float* beta_c = sc_beta + 64 * s;
    float* coef_c = sc_coef + 64 * s;
    if (warp == kScalarWarp && more) fetch_scalars(c + 1);  // lands during this chunk

    if (wait_or_abort(&full_kq[s], (uint32_t)((c >> 1) & 1)) && issuer) pend_kq[s] = -1;
    tc_fence_before();
    bar_compute();
    if (sc_misc[0] != 0.f) { aborted = true; break; }

    if (!DIAG && tid == 0) {
      tc_fence_after();
      // D1 = [K;Q] K' (B = the K rows: even 8-row groups, 2048 B apart)
      for (int kb = 0; kb < 2; ++kb)
        mma_steps(tmem + P::COL_D1, umma_desc_sw128(kq_a + kb * 16384, 16, 1024),
                  umma_desc_sw128(kq_a + kb * 16384, 16, 2048), 32, 32, 4, ID_D1, kb > 0);
      umma_commit(mma1_bar);
      pend_mma1 = c & 1;
    }
    // the next chunk's scalars (their last readers are done)
    if (warp == kScalarWarp && more) store_scalars(c + 1);
    // the previous chunk's output (D4 is not overwritten before MMA4 below)
    if (c > 0) finish_output();

    if constexpr (DIAG) {
      // per-dimension variance: quarter products, exchanged through AT (free now)
      float* mob = AT;  // [4 quarters][128 dims][4]
      const int kb = di >> 6, col = di & 63;
      const uint8_t* ktile = kq + kb * 16384;
      float av[16], rv[16], kv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * dq + i;
        av[i] = a_s[t];
        rv[i] = r_s[t];
        kv[i] = ld_bf16(ktile, (uint32_t)il_row(t, 0), (uint32_t)col);
      }
      Mat2 Pq = {1.f, 0.f, 0.f, 1.f};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float kk = kv[i] * kv[i], a2 = av[i] * av[i];
        const Mat2 M = {rv[i] * a2, rv[i] * wpre[i], kk * a2, fmaf(kk, wpre[i], rv[i])};
        Pq = mmul(M, Pq);
        if ((i & 3) == 3) Pq = mnorm(Pq);
      }
      *reinterpret_cast<float4*>(mob + (dq * 128 + di) * 4) = make_float4(Pq.a, Pq.b, Pq.c, Pq.d);
      if (warp == 15) {
        // log2 decay prefix
        const int ta = 2 * lane, tb = ta + 1;
        const float l0 = __log2f(a_s[ta]), l1 = __log2f(a_s[tb]);
        float incl = l0 + l1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float o = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += o;
        }
        lg_c[ta] = incl - l1;
        lg_c[tb] = incl;
      }
      bar_compute();
      float p = sc_pcar[di];
      for (int q2 = 0; q2 < dq; ++q2) {
        const float4 e = *reinterpret_cast<const float4*>(mob + (q2 * 128 + di) * 4);
        p = __fdividef(fmaf(e.x, p, e.y), fmaf(e.z, p, e.w));
      }
      uint8_t* ghi = sG + kb * 8192;
      uint8_t* glo = sG + 16384 + kb * 8192;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 16 * dq + i;
        const float pp = fmaf(av[i] * av[i], p, wpre[i]);
        p = __fdividef(rv[i] * pp, fmaf(kv[i] * kv[i], pp, rv[i]));
        const float g = pp * kv[i];
        const __nv_bfloat16 gh = __float2bfloat16_rn(g);
        const __nv_bfloat16 gl = __float2bfloat16_rn(g - __bfloat162float(gh));
        const uint32_t off = sw128_offset((uint32_t)t, (uint32_t)col);
        *reinterpret_cast<__nv_bfloat16*>(ghi + off) = gh;
        *reinterpret_cast<__nv_bfloat16*>(glo + off) = gl;
      }
      bar_compute();  // every quarter has read the old carry
      if (dq == 3) sc_pcar[di] = p;
      prefetch_w(c + 1);
      fence_async_smem();
      bar_compute();
      if (tid == 0) {
        tc_fence_after();
        // D1 = [K;Q] G~' (hi, then lo)
        for (int hl = 0; hl < 2; ++hl)
          for (int kb2 = 0; kb2 < 2; ++kb2)
            mma_steps(tmem + P::COL_D1, umma_desc_sw128(kq_a + kb2 * 16384, 16, 1024),
                      umma_desc_sw128(sbase + P::OFF_G + hl * 16384 + kb2 * 8192, 16, 1024),
                      32, 32, 4, ID_D1, hl > 0 || kb2 > 0);
        umma_commit(mma1_bar);
        pend_mma1 = c & 1;
      }
    }

    // ---------------- D1 epilogue: A (first-half rows), P (second-half rows)
    if (wait_or_abort(mma1_bar, (uint32_t)(c & 1)) && tid == 0) pend_mma1 = -1;
    tc_fence_after();
    const float lg_t = lg_c[tk];
    float preg[16];
    {
      float d1[16];
      tmem_ld16(tmem + tm_lane + P::COL_D1 + 16 * cq, d1);
      tmem_wait_ld();
      if (DIAG) {
        if (!second && (tk >> 4) == cq) beta_c[tk] = 1.f / (d1[tk & 15] + r_s[tk]);
        bar_compute();
        if (tid < kC) coef_c[tid] = beta_c[tid] * exp2f(lg_c[kC - 1] - lg_c[tid]);
      }
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const float4 lgj = *reinterpret_cast<const float4*>(lg_c + 16 * cq + 4 * i4);
        const float4 wj = *reinterpret_cast<const float4*>(beta_c + 16 * cq + 4 * i4);
        const float lj[4] = {lgj.x, lgj.y, lgj.z, lgj.w};
        const float bj[4] = {wj.x, wj.y, wj.z, wj.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 16 * cq + 4 * i4 + e;
          const float v = exp2f(lg_t - lj[e]) * bj[e] * d1[4 * i4 + e];
          preg[4 * i4 + e] = (j < tk + second) ? v : 0.f;  // A: j < t; P: j <= t
        }
      }
      if (!second) {
        float* row = AT + tk * kLd + 16 * cq;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4)
          *reinterpret_cast<float4*>(row + 4 * i4) =
              make_float4(preg[4 * i4], preg[4 * i4 + 1], preg[4 * i4 + 2], preg[4 * i4 + 3]);
      }
    }
    bar_compute();

    // ---------------- T = (I + A)^-1 in place (overlaps MMA2)
    // diagonal 16x16 blocks: column cc of block blk per thread (right-looking)
    if (tid < 64) {
      const int blk = tid >> 4, cc = tid & 15;
      const float* Ab = AT + 16 * blk * kLd + 16 * blk;
      float x[16], acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) {
        x[l] = (l == cc) ? 1.f : (l < cc ? 0.f : -acc[l]);
#pragma unroll
        for (int i = l + 1; i < 16; ++i) acc[i] = fmaf(Ab[i * kLd + l], x[l], acc[i]);
      }
      named_bar<2, 64>();  // all A columns read
#pragma unroll
      for (int i = 0; i < 16; ++i) AT[(16 * blk + i) * kLd + 16 * blk + cc] = x[i];
    } else if (mma2_issuer) {
      // D2 = [K;Q] S' (A K-major, d blocks 16 KB apart; B MN-major S', hi then lo).
      // Issued here, while only two warps work, because issuing blocks.
      tc_fence_after();
      for (int hl = 0; hl < 2; ++hl)
        for (int kb = 0; kb < 2; ++kb)
          mma_steps(tmem + P::COL_D2, umma_desc_sw128(kq_a + kb * 16384, 16, 1024),
                    umma_desc_sw128(sbase + P::OFF_S + hl * (P::S_BYTES / 2) + kb * 8192,
                                    16384, 1024),
                    32, 2048, 4, ID_D2, hl > 0 || kb > 0);
      umma_commit(mma2_bar);
      pend_mma2 = c & 1;
    } else if (issuer && more) {
      issue_kq(c + 1);  // stage (c+1) & 1 was released when chunk c-1's MMA5 finished
    }
    bar_compute();
    t_level<1>(AT, X, tid);
    t_level<2>(AT, X, tid);
    t_level<3>(AT, X, tid);
    // T hi/lo into the interleaved A operand of MMA3: rows il_row(t, 0 | 1)
    {
      const int t = tid & 63, part = tid >> 6;  // columns [8 part, 8 part + 8)
      const int bt = t >> 4, bj = part >> 1;
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = 8 * part + i;
        x[i] = (bj == bt) ? AT[t * kLd + j] : (bj < bt ? AT[j * kLd + t] : 0.f);
      }
      st_split8(sTP, (uint32_t)il_row(t, 0), sTP, (uint32_t)il_row(t, 1), (uint32_t)part, x);
    }
    fence_async_smem();

    // ---------------- D2 epilogue: Z = V - gamma K S'
    if (wait_or_abort(mma2_bar, (uint32_t)(c & 1)) && mma2_issuer) pend_mma2 = -1;
    tc_fence_after();
    {
      float d2[HC];
#pragma unroll
      for (int i = 0; i < HC / 16; ++i) tmem_ld16(tmem + tm_lane + P::COL_D2 + HC * cq + 16 * i,
                                                  *reinterpret_cast<float(*)[16]>(d2 + 16 * i));
      tmem_wait_ld();
      if (wait_or_abort(full_v, (uint32_t)(c & 1)) && issuer) pend_v = -1;
      const float gam = exp2f(lg_t);
      const int vc = HC * cq + QC * second;  // this lane's first column
      float z[QC];
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, d2[QC + i], 8);
        z[i] = second ? other : d2[i];
      }
      const uint8_t* vt = sV + (vc >> 6) * 8192;
      uint8_t* zhi = sS + (vc >> 6) * 8192;
      uint8_t* zlo = zhi + P::ZU_BYTES;
#pragma unroll
      for (int i8 = 0; i8 < QC / 8; ++i8) {
        float vv[8];
        ld_bf16x8(vt, (uint32_t)tk, (uint32_t)(((vc & 63) >> 3) + i8), vv);
#pragma unroll
        for (int i = 0; i < 8; ++i) z[8 * i8 + i] = fmaf(-gam, z[8 * i8 + i], vv[i]);
        st_split8(zhi, (uint32_t)tk, zlo, (uint32_t)tk, (uint32_t)(((vc & 63) >> 3) + i8),
                  z + 8 * i8);
      }
      // gamma_t (Q S')_t of this lane's output columns, kept for the output
      // (D2 is overwritten by the next chunk's MMA2 before the output runs)
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, d2[i], 8);
        qpart[i] = gam * (second ? d2[QC + i] : other);
      }
    }
    fence_async_smem();
    tc_fence_before();
    bar_compute();

    // ---------------- MMA3: D3 = [T_hi;T_lo] Z (Z hi then lo; B MN-major [vb][t][64])
    if (tid == 0) {
      tc_fence_after();
      const uint64_t a0 = umma_desc_sw128(sbase + P::OFF_TP, 16, 1024);
      mma_steps(tmem + P::COL_D3, a0, umma_desc_sw128(sbase + P::OFF_S, 8192, 1024), 32, 2048,
                4, ID_D34, false);
      mma_steps(tmem + P::COL_D3, a0,
                umma_desc_sw128(sbase + P::OFF_S + P::ZU_BYTES, 8192, 1024), 32, 2048, 4,
                ID_D34, true);
      umma_commit(mma_bar);
      pend_mma = (int)mma_phase;
    }
    if (issuer && more) issue_v(c + 1);  // the V tile is consumed
    if (wait_or_abort(mma_bar, mma_phase) && tid == 0) pend_mma = -1;
    mma_phase ^= 1u;
    tc_fence_after();

    // ---------------- D3 epilogue: U = top + bottom; U hi/lo and B = coef U hi/lo
    {
      float d3[HC];
#pragma unroll
      for (int i = 0; i < HC / 16; ++i) tmem_ld16(tmem + tm_lane + P::COL_D3 + HC * cq + 16 * i,
                                                  *reinterpret_cast<float(*)[16]>(d3 + 16 * i));
      tmem_wait_ld();
      const int vc = HC * cq + QC * second;
      float u[QC], bu[QC];
      const float coef = coef_c[tk];
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, second ? d3[i] : d3[QC + i], 8);
        u[i] = (second ? d3[QC + i] : d3[i]) + other;
        bu[i] = coef * u[i];
      }
      uint8_t* uhi = sS + (vc >> 6) * 8192;
#pragma unroll
      for (int i8 = 0; i8 < QC / 8; ++i8) {
        const uint32_t col8 = (uint32_t)(((vc & 63) >> 3) + i8);
        st_split8(uhi, (uint32_t)tk, uhi + P::ZU_BYTES, (uint32_t)tk, col8, u + 8 * i8);
        st_split8(uhi + 2 * P::ZU_BYTES, (uint32_t)tk, uhi + 3 * P::ZU_BYTES, (uint32_t)tk, col8,
                  bu + 8 * i8);
      }
      if (second) {
        // P hi/lo into the interleaved A operand of MMA4 (T is consumed)
        st_split8(sTP, (uint32_t)il_row(tk, 0), sTP, (uint32_t)il_row(tk, 1),
                  (uint32_t)(2 * cq), preg);
        st_split8(sTP, (uint32_t)il_row(tk, 0), sTP, (uint32_t)il_row(tk, 1),
                  (uint32_t)(2 * cq + 1), preg + 8);
      }
    }
    fence_async_smem();
    tc_fence_before();
    bar_compute();
    if (sc_misc[0] != 0.f) { aborted = true; break; }

    // ---------------- MMA4 (output) and MMA5 (state)
    if (tid == 0) {
      tc_fence_after();
      const uint64_t a0 = umma_desc_sw128(sbase + P::OFF_TP, 16, 1024);
      mma_steps(tmem + P::COL_D4, a0, umma_desc_sw128(sbase + P::OFF_S, 8192, 1024), 32, 2048,
                4, ID_D34, false);
      mma_steps(tmem + P::COL_D4, a0,
                umma_desc_sw128(sbase + P::OFF_S + P::ZU_BYTES, 8192, 1024), 32, 2048, 4,
                ID_D34, true);
      const uint64_t b_hi = umma_desc_sw128(sbase + P::OFF_S + 2 * P::ZU_BYTES, 8192, 1024);
      const uint64_t b_lo = umma_desc_sw128(sbase + P::OFF_S + 3 * P::ZU_BYTES, 8192, 1024);
      if (!DIAG) {
        // A = K' (MN-major view of the K rows: d blocks 16 KB apart, token groups 2048 B)
        const uint64_t ak = umma_desc_sw128(kq_a, 16384, 2048);
        mma_steps(tmem + P::COL_D5, ak, b_hi, 4096, 2048, 4, ID_D5, false);
        mma_steps(tmem + P::COL_D5, ak, b_lo, 4096, 2048, 4, ID_D5, true);
      } else {
        const uint64_t ag_hi = umma_desc_sw128(sbase + P::OFF_G, 8192, 1024);
        const uint64_t ag_lo = umma_desc_sw128(sbase + P::OFF_G + 16384, 8192, 1024);
        mma_steps(tmem + P::COL_D5, ag_hi, b_hi, 2048, 2048, 4, ID_D5, false);
        mma_steps(tmem + P::COL_D5, ag_hi, b_lo, 2048, 2048, 4, ID_D5, true);
        mma_steps(tmem + P::COL_D5, ag_lo, b_hi, 2048, 2048, 4, ID_D5, true);
      }
      umma_commit(mma_bar);
      pend_mma = (int)mma_phase;
    }
    // iso: the next chunk's ||k||^2 and variances, in the shadow of MMA4 + MMA5
    if (!DIAG && more) {
      if (wait_or_abort(&full_kq[(c + 1) & 1], (uint32_t)(((c + 1) >> 1) & 1)) && issuer)
        pend_kq[(c + 1) & 1] = -1;
      iso_variance(c + 1);
    }
    if (wait_or_abort(mma_bar, mma_phase) && tid == 0) pend_mma = -1;
    mma_phase ^= 1u;
    tc_fence_after();

    // ---------------- state: S' = gamma_C S' + D5, then its hi/lo operand
    {
      const float gC = exp2f(lg_c[kC - 1]);
      float d5[HC];
#pragma unroll
      for (int i = 0; i < HC / 16; ++i) tmem_ld16(tmem + tm_lane + P::COL_D5 + HC * cq + 16 * i,
                                                  *reinterpret_cast<float(*)[16]>(d5 + 16 * i));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < HC; ++e) Sreg[e] = fmaf(gC, Sreg[e], d5[e]);
    }
    write_state_operand();
    prev_t0 = t0;
    prev_valid = valid;
    fence_async_smem();
    tc_fence_before();
  }
  if (!aborted && sc_misc[0] == 0.f && nchunks > 0) {
    tc_fence_after();
    finish_output();
  }

  // ---- abort path: bounded waits for MMAs and copies still in flight
  if (tid == 0) {
    if (pend_mma1 >= 0) (void)mbar_wait(mma1_bar, (uint32_t)pend_mma1);
    if (pend_mma >= 0) (void)mbar_wait(mma_bar, (uint32_t)pend_mma);
  }
  if (mma2_issuer && pend_mma2 >= 0) (void)mbar_wait(mma2_bar, (uint32_t)pend_mma2);
  if (issuer) {
    for (int st = 0; st < 2; ++st)
      if (pend_kq[st] >= 0) (void)mbar_wait(&full_kq[st], (uint32_t)pend_kq[st]);
    if (pend_v >= 0) (void)mbar_wait(full_v, (uint32_t)pend_v);
  }
  bar_compute();
  if (!aborted && sc_misc[0] == 0.f) {
#pragma unroll
    for (int c = 0; c < HC; ++c)
      S_out[s_head + (size_t)(v0 + HC * cq + c) * kDK + my_k] = Sreg[c];
    if (vblk == 0) {
      if (DIAG) {
        if (tid < kDK) P_out[(size_t)bh * kDK + tid] = sc_pcar[tid];
      } else if (tid == 0) {
        P_out[bh] = sc_pcar[0];
      }
    }
  }
  tc_fence_before();
  bar_compute();
  if (warp == 0) tmem_dealloc(tmem, P::TMEM_COLS);
}

// ===========================================================================
// Warp-specialised engine (one CTA per head, d_v = 128), both variants.
//
// Every product runs transposed, with the value index v on the 128 TMEM lanes,
// so that the fp32 state S'^T [v][k] stays in TMEM, every operand a lane
// produces is its own TMEM row (an A operand read from TMEM), and the keys and
// queries are B operands straight from the copies' tiles:
//   D2 = S'^T [K ; Q]^T                       (S' as bf16 hi/lo, exact K and Q)
//   Z = V - gamma K S',  gamma (Q S')          Z as bf16 hi/lo
//   D3 = Z^T T^T                              U^T (bf16 hi/lo Z and T, three terms)
//   D2 (query half) += U^T P^T                o^T (tf32: U as the tensor cores
//                                             truncate it, P rounded)
//   S'^T = gamma_C S'^T + B^T G,  B = coef U  (bf16 hi/lo B; G = K exact, or
//                                             the diagonal variant's G~ as bf16
//                                             hi/lo, three terms)
//
// Warps 0-7 (the chain) run the part that depends on the state.  Per chunk:
// MMA2; Z (with gamma_t (Q S')_t and the state decay); MMA3; B = coef U; MMA5
// and MMA4; the state's bf16 hi/lo operand for the next chunk and the output
// (isotropic: a staged tile and one tensor store; diagonal: direct stores).
// Warps 8-15 (prep) run the part that depends only on the chunk's inputs, one
// chunk ahead: the D1 epilogue (A, and P once MMA4 of the previous chunk has
// released its buffer) on all eight warps, then T = (I + A)^-1 on warps 8-11
// while warps 12-15 prepare the next chunk (isotropic: the solve's last two
// steps, the 32x32 block below the diagonal, on all eight warps, as the next
// chunk's scalars take warps 12-15 only part of the solve):
//   isotropic  ||k||^2, decay prefix and the variance scan; MMA1 of the next
//              chunk is issued as soon as D1 is read.
//   diagonal   decay prefix and the per-dimension variance (one thread per
//              dimension; each warp copies w of its 32 dimensions in 16-token
//              quarters, two ahead), whose G~ = p^- k (as bf16 hi/lo) is
//              parked in the free D1 columns until MMA5 of chunk c - 1 has
//              released the G~ buffer it goes to (two buffers); then MMA1 of
//              the next chunk, D1 = [K;Q] G~^T.  beta_t = 1 / (k_t.G~_t + r_t)
//              comes from the diagonal of D1 in the next D1 epilogue.
// The groups hand over through mbarriers:
//   t_ready / p_ready   prep -> chain: T / P written, with the chunk's scalars
//                       and the next chunk's decay
//   mma3 / mma4 / mma5  the chain's commits; they also hand T, P and G~ back
// Per-token scalars live in four slots (chunk index mod 4).
// TMEM columns: D1 [0,64) (prep); S'^T [64,192); D2 [192,320) (key half, then
// query half); D3 [320,384); W [384,512) holds in turn S'^T hi [384,448) and lo
// [448,512) (k pairs), Z^T hi [384,416) and lo [416,448), B^T hi and lo (same).
// ===========================================================================
template <bool DIAG>
struct WsPlan {
  static constexpr uint32_t KQ_BYTES = 32768;           // bf16 [kb 2][K|Q][64 t][64]
  static constexpr int kStages = DIAG ? 2 : 3;
  static constexpr uint32_t OFF_KQ = 0;                 // kStages stages
  static constexpr uint32_t OFF_V = kStages * KQ_BYTES; // bf16 [vb 2][64 t][64 v]
  static constexpr uint32_t OFF_T = OFF_V + 16384;      // bf16 hi, lo [64 t][64 j]
  static constexpr uint32_t OFF_P = OFF_T + 16384;      // fp32 [jb 2][64 t][32 j]
  static constexpr uint32_t OFF_AT = OFF_P + 16384;     // fp32 [64][68]
  static constexpr uint32_t OFF_X = OFF_AT + 64u * kLd * 4u;
  static constexpr uint32_t OFF_SC = OFF_X + 5120u;     // X: fp32 [4][16][20]
  // isotropic: fp32 [64 t][128 v] output tile; diagonal: two G~ buffers, each
  // bf16 hi then lo [kb 2][64 t][64 k]
  static constexpr uint32_t OFF_OUT = OFF_SC + 9216u;
  static constexpr uint32_t OFF_G = OFF_OUT;
  // diagonal: w of 16 tokens, per warp of the variance team two buffers of
  // fp32 [16 t][32 k] (its 32 dimensions)
  static constexpr uint32_t OFF_W = OFF_G + 65536u;
  static constexpr uint32_t OFF_BAR = DIAG ? OFF_W + 16384u : OFF_OUT + 32768u;
  static constexpr uint32_t TOTAL = OFF_BAR + 256u;
  static constexpr uint32_t ALLOC = TOTAL + 1024u;
  static constexpr uint32_t COL_D1 = 0, COL_ST = 64, COL_D2 = 192, COL_D3 = 320, COL_W = 384;
  static_assert(TOTAL <= 227u * 1024u, "shared memory plan too large");
  static_assert(OFF_V % 1024 == 0 && OFF_T % 1024 == 0 && OFF_P % 1024 == 0 &&
                    OFF_OUT % 1024 == 0,
                "operand alignment");
};

// 2^x from the hardware approximation (relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// (hi, lo) bf16 splits of two consecutive K elements, packed low-first as a
// 32-bit TMEM column of a bf16 A operand.
__device__ __forceinline__ void split_pack2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
  hi = *reinterpret_cast<const uint32_t*>(&hb);
  // x - hi for both halves in one packed FP32 add (rounds as two scalar ones)
  const float2 d = __fadd2_rn(make_float2(x0, x1), make_float2(-__uint_as_float(hi << 16),
                                                               -__uint_as_float(hi & 0xffff0000u)));
  const __nv_bfloat162 lb = __floats2bfloat162_rn(d.x, d.y);
  lo = *reinterpret_cast<const uint32_t*>(&lb);
}

// --------------------------------------------- 16x16 products on warp MMAs
// The off-diagonal blocks of T come from 16x16x16 products done by single
// warps with mma.sync (m16n8k8, tf32).  Each operand is split x = hi + lo in
// tf32 and the product keeps hi*hi + hi*lo + lo*hi in three accumulators, which
// leaves about fp32 accuracy.  Fragment layout of m16n8k8 (g = lane / 4,
// q = lane % 4): A (16x8) rows g, g+8 x cols q, q+4; B (8x8) rows q, q+4 x col
// g; C (16x8) rows g, g+8 x cols 2q, 2q+1.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = rna_tf32(x);
  lo = rna_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// acc[term][n tile] += A (16x16, element A(r, k)) * B (16x16, element B(k, n))
template <class FA, class FB>
__device__ __forceinline__ void warp_mm16(float (&acc)[3][2][4], FA A, FB B, int lane) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t ah[4], al[4];
    split_tf32(A(g, 8 * ks + q), ah[0], al[0]);
    split_tf32(A(g + 8, 8 * ks + q), ah[1], al[1]);
    split_tf32(A(g, 8 * ks + q + 4), ah[2], al[2]);
    split_tf32(A(g + 8, 8 * ks + q + 4), ah[3], al[3]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t bh[2], bl[2];
      split_tf32(B(8 * ks + q, 8 * nt + g), bh[0], bl[0]);
      split_tf32(B(8 * ks + q + 4, 8 * nt + g), bh[1], bl[1]);
      mma_tf32_16x8x8(acc[0][nt], ah, bh);
      mma_tf32_16x8x8(acc[1][nt], ah, bl);
      mma_tf32_16x8x8(acc[2][nt], al, bh);
    }
  }
}
// Hand the summed 16x16 result, scaled by s, to C(r, c, v_c, v_c+1) in pairs.
template <class FC>
__device__ __forceinline__ void warp_put16(const float (&acc)[3][2][4], float s, FC C, int lane) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = s * (acc[2][nt][e] + acc[1][nt][e] + acc[0][nt][e]);
    C(g, 8 * nt + 2 * q, v[0], v[1]);
    C(g + 8, 8 * nt + 2 * q, v[2], v[3]);
  }
}

// The same product for n-tile nt alone (B's columns [8 nt, 8 nt + 8)), with
// the same fragments, accumulation order and final sum, so that two warps
// taking one n-tile each give what one warp taking both gives.
template <class FA, class FB>
__device__ __forceinline__ void warp_mm16n(float (&acc)[3][4], FA A, FB B, int nt, int lane) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t ah[4], al[4];
    split_tf32(A(g, 8 * ks + q), ah[0], al[0]);
    split_tf32(A(g + 8, 8 * ks + q), ah[1], al[1]);
    split_tf32(A(g, 8 * ks + q + 4), ah[2], al[2]);
    split_tf32(A(g + 8, 8 * ks + q + 4), ah[3], al[3]);
    uint32_t bh[2], bl[2];
    split_tf32(B(8 * ks + q, 8 * nt + g), bh[0], bl[0]);
    split_tf32(B(8 * ks + q + 4, 8 * nt + g), bh[1], bl[1]);
    mma_tf32_16x8x8(acc[0], ah, bh);
    mma_tf32_16x8x8(acc[1], ah, bl);
    mma_tf32_16x8x8(acc[2], al, bh);
  }
}
template <class FC>
__device__ __forceinline__ void warp_put16n(const float (&acc)[3][4], float s, FC C, int nt,
                                            int lane) {
  const int g = lane >> 2, q = lane & 3;
  float v[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] = s * (acc[2][e] + acc[1][e] + acc[0][e]);
  C(g, 8 * nt + 2 * q, v[0], v[1]);
  C(g + 8, 8 * nt + 2 * q, v[2], v[3]);
}

constexpr int kChainBar = 3, kPrepBar = 4, kPhase1Bar = 5, kGroup = 256;

__device__ __forceinline__ void bar_group(int id) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGroup) : "memory");
}

// Barrier of one 256-thread group that also ORs a flag over the group, so an
// abort decision taken after it is the same in every thread of the group.
__device__ __forceinline__ bool bar_group_or(int id, bool flag) {
  uint32_t r;
  __syncwarp();
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "r"(id), "n"(kGroup)
      : "memory");
  return r != 0;
}

constexpr int kTeamA = 6, kTeamB = 7;

// Longest-first order of packed sequences.  The engine holds one CTA per SM,
// so when there are more (sequence, head) problems than SMs the hardware
// starts them in waves; a long sequence that starts in a late wave sets the
// end of the launch.  Starting them longest first (list scheduling by longest
// processing time, Graham 1969) bounds the launch by 4/3 of the best schedule.
// One CTA counting-sorts the sequences by their number of chunks, descending;
// equal counts land in any order, which changes no result (a sequence's
// arithmetic does not depend on the CTA that runs it).  order[] receives a
// permutation of [0, N) whatever cu_seqlens holds: lengths are clamped as
// the engine clamps them, and the engine reports bad offsets itself.
constexpr int kOrderBuckets = 4096, kOrderThreads = 1024;

__device__ __forceinline__ int order_bucket(const int* __restrict__ cu, int s, int T) {
  const int s0 = min(max(cu[s], 0), T);
  const int n = min(max(cu[s + 1], s0), T) - s0;
  return kOrderBuckets - 1 - min((n + kC - 1) / kC, kOrderBuckets - 1);  // 0: longest
}

__global__ void __launch_bounds__(kOrderThreads)
varlen_order_kernel(const int* __restrict__ cu, int N, int T, int* __restrict__ order) {
  constexpr int kPer = kOrderBuckets / kOrderThreads;
  __shared__ int start[kOrderBuckets];
  __shared__ int wsum[kOrderThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int i = tid; i < kOrderBuckets; i += kOrderThreads) start[i] = 0;
  __syncthreads();
  for (int s = tid; s < N; s += kOrderThreads) atomicAdd(&start[order_bucket(cu, s, T)], 1);
  __syncthreads();
  // exclusive prefix sum of the bucket counts: kPer buckets per thread, then
  // a warp scan and a scan of the warp totals
  int c[kPer], run = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    c[j] = start[tid * kPer + j];
    run += c[j];
  }
  int x = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int y = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    wsum[lane] = y;
  }
  __syncthreads();
  int base = x - run + (wid ? wsum[wid - 1] : 0);
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    start[tid * kPer + j] = base;
    base += c[j];
  }
  __syncthreads();
  for (int s = tid; s < N; s += kOrderThreads)
    order[atomicAdd(&start[order_bucket(cu, s, T)], 1)] = s;
}

// PACKED: the B "batch entries" are packed sequences given by cu_seqlens (the
// instantiation for ordinary [B, T, H, d] tensors carries none of its code).
template <bool DIAG, bool PACKED>
__global__ void __launch_bounds__(kThreads, 1)
chunk_engine_ws_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ Ag,
                       const float* __restrict__ Wg, const float* __restrict__ Rg,
                       const float* S0, const float* __restrict__ P0, float* __restrict__ O,
                       float* S_out, float* __restrict__ P_out, int T, int H, float kappa,
                       uint32_t* __restrict__ err, int debug_skip_v,
                       const int* __restrict__ cu_seqlens, const int* __restrict__ order) {
  using P = WsPlan<DIAG>;
  constexpr int DV = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // packed sequences may be taken longest first: CTA i runs sequence order[i / H]
  const int bh = PACKED && order ? order[blockIdx.x / H] * H + (int)(blockIdx.x % H)
                                 : (int)blockIdx.x;
  const int h = bh % H;
  // This CTA's sequence: batch entry b of [B, T, H, d] tensors, or (packed
  // sequences, cu_seqlens given) tokens [tbeg, tbeg + Tn) of [1, T, H, d] ones.
  int b = bh / H, tbeg = 0, Tn = T;
  if constexpr (PACKED) {
    const int s0 = cu_seqlens[bh / H], s1 = cu_seqlens[bh / H + 1];
    b = 0;
    tbeg = min(max(s0, 0), T);
    Tn = min(max(s1, tbeg), T) - tbeg;
    if (threadIdx.x == 0 && (s0 < 0 || s1 < s0 || s1 > T)) atomicOr(err, DEV_BAD_ARG);
  }
  const int nchunks = (Tn + kC - 1) / kC;
  const uint32_t sbase = smem_u32(smem);
  if (PACKED && Tn == 0) {
    // an empty sequence hands its initial state and variance through
    const size_t n = (size_t)DV * kDK;
    for (size_t i = threadIdx.x; i < n; i += kThreads)
      S_out[(size_t)bh * n + i] = S0 ? S0[(size_t)bh * n + i] : 0.f;
    const int np = DIAG ? kDK : 1;
    for (int i = threadIdx.x; i < np; i += kThreads)
      P_out[(size_t)bh * np + i] = P0 ? P0[(size_t)bh * np + i] : 1.f;
    return;
  }

  // scalar area (floats); [4][64] arrays are indexed by chunk & 3
  float* scf = reinterpret_cast<float*>(smem + P::OFF_SC);
  float* sc_a = scf;             // decay a_t
  float* sc_w = scf + 256;       // process noise w_t
  float* sc_r = scf + 512;       // observation noise r_t
  float* sc_beta = scf + 768;    // beta_t
  float* sc_lg = scf + 1024;     // log2 of the in-chunk cumulative decay
  float* sc_gam = scf + 1280;    // gamma_t
  float* sc_coef = scf + 1536;   // state-update coefficient
  float* sc_n = scf + 1792;      // [2 halves][64] partial ||k_t||^2 of one chunk
  float* sc_gC = scf + 1920;     // [4] gamma of the whole chunk
  volatile float* sc_abort = scf + 1924;
  float* sc_pcar = scf + 1928;   // carried variance (diagonal: [128])
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* full_kq = bars;        // [kStages] K/Q tiles of a stage landed
  uint64_t* full_v = bars + 3;     // V tile landed
  uint64_t* mma1_bar = bars + 4;   // MMA1 finished (D1)
  uint64_t* mma2_bar = bars + 5;   // MMA2 finished
  uint64_t* mma3_bar = bars + 6;   // MMA3 finished: T free
  uint64_t* mma4_bar = bars + 7;   // MMA4 finished: P free, output ready
  uint64_t* mma5_bar = bars + 8;   // MMA5 finished: state updated, stage free
  uint64_t* t_ready = bars + 9;    // T written
  uint64_t* p_ready = bars + 10;   // P and the next chunk's scalars written
  uint64_t* w_full = bars + 11;    // [4 warps][2] (diagonal) a w buffer landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  float* sOut = reinterpret_cast<float*>(smem + P::OFF_OUT);
  float* AT = reinterpret_cast<float*>(smem + P::OFF_AT);
  float* X = reinterpret_cast<float*>(smem + P::OFF_X);
  uint8_t* sT = smem + P::OFF_T;
  uint8_t* sP = smem + P::OFF_P;
  uint8_t* sV = smem + P::OFF_V;
  float* sW = reinterpret_cast<float*>(smem + P::OFF_W);

  if (tid == 0) {
    for (int i = 0; i < 19; ++i) mbar_init(&bars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *sc_abort = 0.f;
    if (!DIAG) sc_pcar[0] = P0 ? P0[bh] : 1.f;
  }
  if (DIAG && tid < kDK) sc_pcar[tid] = P0 ? P0[(size_t)bh * kDK + tid] : 1.f;
  // T operand (hi, lo): blocks above the diagonal are never written again
  for (int i = tid; i < 1024; i += kThreads)
    *reinterpret_cast<uint4*>(sT + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  fence_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Bounded wait; once any thread has recorded a timeout every later wait
  // fails at once, so an aborting CTA ends within a few wait limits.
  auto fail = [&](uint64_t* bar_, uint32_t parity) -> bool {
    if (*sc_abort != 0.f) return true;
    if (!mbar_wait(bar_, parity)) {
      atomicOr(err, DEV_TIMEOUT);
      *sc_abort = 1.f;
      return true;
    }
    return false;
  };

  const int m = 32 * (warp & 3) + lane;  // TMEM lane of this thread
  const uint32_t tm_lane = (uint32_t)(32 * (warp & 3)) << 16;

  // ---- the prep group's per-chunk scalars
  // a, w, r of chunk c (one warp): loaded a chunk ahead into registers
  float ps_a[2], ps_r[2], ps_w[2];
  auto fetch_scalars = [&](int c) {
    const int t0 = c * kC, valid = min(kC, Tn - t0);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = lane + 32 * i;
      const bool in = t < valid;
      const size_t tok = ((size_t)b * T + tbeg + t0 + t) * H + h;
      ps_a[i] = in ? __ldg(Ag + tok) : 1.f;
      ps_r[i] = in ? __ldg(Rg + tok) : 1.f;
      ps_w[i] = (!DIAG && in) ? __ldg(Wg + tok) : 0.f;
    }
  };
  auto store_scalars = [&](int c) {
    const int sl = c & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = lane + 32 * i;
      sc_a[64 * sl + t] = ps_a[i];
      sc_r[64 * sl + t] = ps_r[i];
      sc_w[64 * sl + t] = ps_w[i];
    }
  };
  // partial ||k_t||^2 of chunk c over d in [64 half, 64 half + 64), 128 threads
  auto key_norms = [&](int c, int pt) {
    const int t = pt & 63, half = pt >> 6;
    const uint8_t* kt = smem + P::OFF_KQ + (c % P::kStages) * P::KQ_BYTES + half * 16384;
    // (packed sequences: the tile runs on into the next one)
    const bool in = !PACKED || t < Tn - c * kC;
    float acc = 0.f;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      float x[8];
      ld_bf16x8(kt, (uint32_t)t, (uint32_t)cc, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(x[e], x[e], acc);
    }
    sc_n[64 * half + t] = in ? acc : 0.f;
  };
  // decay prefix and Mobius scan of the variance of chunk c (one warp, two
  // tokens per lane): lg, gamma, gamma_C, beta, the update coefficients, carry
  auto decay_and_variance = [&](int c) {
    const int sl = c & 3;
    const float* a_s = sc_a + 64 * sl;
    const float* w_s = sc_w + 64 * sl;
    const float* r_s = sc_r + 64 * sl;
    const int ta = 2 * lane, tb = ta + 1;
    const float a0 = a_s[ta], a1 = a_s[tb];
    const float l0 = __log2f(a0), l1 = __log2f(a1);
    float incl = l0 + l1;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const float o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    const float lg0 = incl - l1, lg1 = incl;
    const float lg_last = __shfl_sync(0xffffffffu, lg1, 31);
    sc_lg[64 * sl + ta] = lg0;
    sc_lg[64 * sl + tb] = lg1;
    sc_gam[64 * sl + ta] = exp2f(lg0);
    sc_gam[64 * sl + tb] = exp2f(lg1);
    if (lane == 31) sc_gC[sl] = exp2f(lg1);
    if constexpr (DIAG) return;  // beta and the coefficients come from D1
    const float n0 = sc_n[ta] + sc_n[64 + ta], n1 = sc_n[tb] + sc_n[64 + tb];
    const float w0 = w_s[ta], w1 = w_s[tb], r0 = r_s[ta], r1 = r_s[tb];
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
    const float carry = sc_pcar[0];
    float p = lane == 0 ? carry : __fdividef(fmaf(ex.a, carry, ex.b), fmaf(ex.c, carry, ex.d));
    const float pp0 = fmaf(a0 * a0, p, w0);
    p = __fdividef(r0 * pp0, fmaf(c0, pp0, r0));
    const float pp1 = fmaf(a1 * a1, p, w1);
    p = __fdividef(r1 * pp1, fmaf(c1, pp1, r1));
    // (tokens past the sequence end write nothing: beta = 0)
    float b0 = __fdividef(pp0, fmaf(pp0, n0, r0));
    float b1 = __fdividef(pp1, fmaf(pp1, n1, r1));
    if constexpr (PACKED) {
      const int vld = Tn - c * kC;
      b0 = ta < vld ? b0 : 0.f;
      b1 = tb < vld ? b1 : 0.f;
    }
    sc_beta[64 * sl + ta] = b0;
    sc_beta[64 * sl + tb] = b1;
    sc_coef[64 * sl + ta] = b0 * exp2f(lg_last - lg0);
    sc_coef[64 * sl + tb] = b1 * exp2f(lg_last - lg1);
    const float pnext = __shfl_sync(0xffffffffu, p, 31);
    __syncwarp();
    if (lane == 0) sc_pcar[0] = pnext;
  };
  const bool issuer = (warp == 0 && lane == 0);       // chain: MMAs and copies
  const bool mma1_issuer = (warp == 15 && lane == 0);  // prep: MMA1
  constexpr uint32_t ID_1 = umma_idesc(128, 64, 1, 0, 0);
  // (issuers) copies and MMAs not yet seen done: pend_kq holds per stage a
  // pending bit (2 st) and the parity to wait for (2 st + 1)
  uint32_t pend_kq = 0u;
  int pend_v = -1, pend_mma1 = -1;
  auto kq_parity = [](int c) { return (uint32_t)((c / P::kStages) & 1); };
  auto issue_kq = [&](int c) {
    const int st = c % P::kStages, t0 = c * kC;
    uint8_t* kqd = smem + P::OFF_KQ + st * P::KQ_BYTES;
    mbar_expect_tx(&full_kq[st], P::KQ_BYTES);
    for (int kb = 0; kb < 2; ++kb) {
      tma_load_4d(kqd + kb * 16384, &tm_k, &full_kq[st], kb * 64, h, tbeg + t0, b);
      tma_load_4d(kqd + kb * 16384 + 8192, &tm_q, &full_kq[st], kb * 64, h, tbeg + t0, b);
    }
    pend_kq = (pend_kq & ~(3u << (2 * st))) | ((1u | (kq_parity(c) << 1)) << (2 * st));
  };
  auto issue_v = [&](int c) {
    mbar_expect_tx(full_v, 16384);
    tma_load_4d(sV, &tm_v, full_v, 0, h, tbeg + c * kC, b);
    tma_load_4d(sV + 8192, &tm_v, full_v, 64, h, tbeg + c * kC, b);
    pend_v = c & 1;
  };
  // (diagonal) w quarter n: tokens [16 n, 16 n + 16) of the sequence, for the
  // 32 dimensions of variance warp wv (its lane 0 issues them)
  uint32_t pend_w = 0u;  // per buffer: pending bit (2 i) and parity (2 i + 1)
  auto issue_w = [&](int n, int wv) {
    const int bf = n & 1;
    uint64_t* bar_ = &w_full[2 * wv + bf];
    mbar_expect_tx(bar_, 2048);
    tma_load_4d(smem + P::OFF_W + (2 * wv + bf) * 2048, &tm_w, bar_, 32 * wv, h, tbeg + 16 * n, b);
    pend_w = (pend_w & ~(3u << (2 * bf))) | ((1u | ((uint32_t)((n >> 1) & 1) << 1)) << (2 * bf));
  };
  // D1 = [K;Q] K^T of chunk c (A: the stage's key rows then query rows per d
  // block); diagonal: D1 = [K;Q] G~^T (G~ hi, then lo)
  auto issue_mma1 = [&](int c) {
    const uint32_t kq_a = sbase + P::OFF_KQ + (c % P::kStages) * P::KQ_BYTES;
    tc_fence_after();
    const uint64_t d0 = umma_desc_sw128(kq_a, 16, 1024);
    if constexpr (DIAG) {
      const uint64_t g0 = umma_desc_sw128(sbase + P::OFF_G + (c & 1) * 32768u, 16, 1024);
#pragma unroll
      for (int hl = 0; hl < 2; ++hl)
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_bf16(tmem + P::COL_D1, d0 + (uint64_t)((kb * 16384 + ks * 32) >> 4),
                      g0 + (uint64_t)((hl * 16384 + kb * 8192 + ks * 32) >> 4), ID_1,
                      (hl > 0 || kb > 0 || ks > 0) ? 1u : 0u);
    } else {
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t d = d0 + (uint64_t)((kb * 16384 + ks * 32) >> 4);
          umma_bf16(tmem + P::COL_D1, d, d, ID_1, (kb > 0 || ks > 0) ? 1u : 0u);
        }
    }
    umma_commit(mma1_bar);
    pend_mma1 = c & 1;
  };

  bool bad = false;
  // diagonal: the variance of dimension d over chunk c (one thread per d,
  // tokens in order), p^- = a^2 p + w, p = r p^- / (k^2 p^- + r), with the
  // gain direction G~ = p^- k of each token (as a bf16 hi/lo pair) kept in the
  // free D1 columns (TMEM lane d) until its smem buffer is released
  // (write_gain).  w arrives in quarters of 16 tokens: quarter n = 4 c + q of
  // this warp's 32 dimensions in its buffer n & 1, copied two quarters ahead
  // by the warp's lane 0.
  auto diag_variance = [&](int c, int d) {
    const int sl = c & 3;
    const float* a_s = sc_a + 64 * sl;
    const float* r_s = sc_r + 64 * sl;
    uint8_t* kt = smem + P::OFF_KQ + (c % P::kStages) * P::KQ_BYTES + (d >> 6) * 16384;
    const uint32_t col = (uint32_t)(d & 63);
    // tokens past the end of a packed sequence (its tiles run on into the
    // next one) become identity steps: their k and w are zeroed in place
    // (in this thread's own column) before use
    const int vld = Tn - c * kC;
    // p = x / y, carried projectively so that no division sits on the
    // token-to-token chain: with u = a^2 x + w y (= p^- y), one token maps
    // (x, y) to (r u, k^2 u + r y), the Mobius map's matrix applied to the
    // pair; p^- k = u k / y is a division off the chain.  (x, y) is rescaled
    // by the binade of y (exact) every four tokens.
    float x = sc_pcar[d], y = 1.f;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
      const int n = 4 * c + q;
      if (fail(&w_full[2 * (d >> 5) + (n & 1)], (uint32_t)((n >> 1) & 1))) bad = true;
      if (!bad) {
        float* wq = sW + (2 * (d >> 5) + (n & 1)) * 512 + (d & 31);
        if (PACKED && vld < 16 * q + 16) {
          for (int e = max(vld - 16 * q, 0); e < 16; ++e) {
            wq[e * 32] = 0.f;
            *reinterpret_cast<__nv_bfloat16*>(kt + sw128_offset((uint32_t)(16 * q + e), col)) =
                __float2bfloat16_rn(0.f);
          }
        }
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const float4 a4 = *reinterpret_cast<const float4*>(a_s + 16 * q + 4 * i4);
          const float4 r4 = *reinterpret_cast<const float4*>(r_s + 16 * q + 4 * i4);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w}, rv[4] = {r4.x, r4.y, r4.z, r4.w};
          uint32_t g[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float k = ld_bf16(kt, (uint32_t)(16 * q + 4 * i4 + e), col);
            const float u = fmaf(av[e] * av[e], x, wq[(4 * i4 + e) * 32] * y);
            // G~ = p^- k as bf16 hi (low half) and lo (high half)
            const float gf = __fdividef(u * k, y);
            const __nv_bfloat16 g_hi = __float2bfloat16_rn(gf);
            const __nv_bfloat16 g_lo = __float2bfloat16_rn(gf - __bfloat162float(g_hi));
            g[e] = (uint32_t)__bfloat16_as_ushort(g_hi) |
                   ((uint32_t)__bfloat16_as_ushort(g_lo) << 16);
            x = rv[e] * u;
            y = fmaf(k * k, u, rv[e] * y);
          }
          tmem_st4u(tmem + tm_lane + P::COL_D1 + 16 * q + 4 * i4, g);
          const int ex = (int)((__float_as_uint(y) >> 23) & 0xffu) - 127;
          if (ex > -100 && ex < 100) {
            const float sc = __uint_as_float((uint32_t)(127 - ex) << 23);
            x *= sc;
            y *= sc;
          }
        }
      }
      __syncwarp();  // this warp's buffer n & 1 has been read
      if (lane == 0 && !bad && n + 2 < 4 * nchunks) issue_w(n + 2, d >> 5);
    }
    sc_pcar[d] = x / y;
    tmem_wait_st();
  };
  // G~ of chunk c (bf16 hi/lo pairs) from TMEM into its buffer c & 1 as
  // [hi|lo][kb][t][k]
  auto write_gain = [&](int c, int d) {
    uint8_t* gh = smem + P::OFF_G + (c & 1) * 32768 + (d >> 6) * 8192;
    const uint32_t col = (uint32_t)(d & 63);
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      float g[16];
      tmem_ld16(tmem + tm_lane + P::COL_D1 + 16 * blk, g);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t hl = __float_as_uint(g[i]);
        const uint32_t off = sw128_offset((uint32_t)(16 * blk + i), col);
        *reinterpret_cast<uint16_t*>(gh + off) = (uint16_t)(hl & 0xffffu);
        *reinterpret_cast<uint16_t*>(gh + 16384 + off) = (uint16_t)(hl >> 16);
      }
    }
  };

  // ---- prologue: copies, chunk 0's scalars and MMA1
  if (issuer) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
    issue_kq(0);
    issue_v(0);
    for (int c = 1; c < P::kStages && c < nchunks; ++c) issue_kq(c);
  }
  if (warp >= 8) {
    if (DIAG && warp >= 12 && lane == 0) {
      issue_w(0, warp - 12);
      issue_w(1, warp - 12);
    }
    if (warp == 13) {
      fetch_scalars(0);
      store_scalars(0);
      if (nchunks > 1) fetch_scalars(1);
    }
    if (fail(&full_kq[0], kq_parity(0))) bad = true;
    if constexpr (DIAG) {
      if (warp >= 12) {
        named_bar<kTeamB, 128>();  // chunk 0's scalars
        diag_variance(0, tid - 384);
        if (!bad) write_gain(0, tid - 384);
        if (warp == 12) decay_and_variance(0);
        fence_async_smem();
        tc_fence_before();
        named_bar<kTeamB, 128>();
        if (mma1_issuer && !bad) issue_mma1(0);
      }
    } else {
      if (mma1_issuer && !bad) issue_mma1(0);
      if (warp >= 12) {
        key_norms(0, tid - 384);
        named_bar<kTeamB, 128>();
        if (warp == 12) decay_and_variance(0);
      }
    }
  }
  __syncthreads();  // chunk 0's scalars are in place

  if (warp < 8) {
    // ================================================================ chain
    const int ch = warp >> 2;  // tokens [32 ch, 32 ch + 32), state columns [64 ch, 64 ch + 64)
    const int v = m;           // value index of this lane
    constexpr uint32_t ID_2 = umma_idesc(128, 128, 1, 0, 0);   // bf16
    constexpr uint32_t ID_3 = umma_idesc(128, 64, 1, 0, 0);    // bf16
    constexpr uint32_t ID_4 = umma_idesc(128, 64, 2, 0, 0);    // tf32
    constexpr uint32_t ID_5 = umma_idesc(128, 128, 1, 0, 1);   // bf16, B MN-major

    // S'^T [v][k], k in [64 ch, 64 ch + 64), as the bf16 hi/lo A operand of
    // MMA2 in W: k pairs per column, hi then lo
    auto split_state = [&]() {
#pragma unroll
      for (int h32 = 0; h32 < 2; ++h32) {
        float x[32];
        uint32_t hi[16], lo[16];
        tmem_ld32(tmem + tm_lane + P::COL_ST + 64 * ch + 32 * h32, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) split_pack2(x[2 * i], x[2 * i + 1], hi[i], lo[i]);
        tmem_st16u(tmem + tm_lane + P::COL_W + 32 * ch + 16 * h32, hi);
        tmem_st16u(tmem + tm_lane + P::COL_W + 64 + 32 * ch + 16 * h32, lo);
      }
    };

    // S'^T [v][k] into TMEM, k in [64 ch, 64 ch + 64)
    const size_t s_row = ((size_t)bh * DV + v) * kDK + 64 * ch;
#pragma unroll
    for (int h32 = 0; h32 < 2; ++h32) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 x = S0 ? *reinterpret_cast<const float4*>(S0 + s_row + 32 * h32 + i)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        r[i] = __float_as_uint(x.x);
        r[i + 1] = __float_as_uint(x.y);
        r[i + 2] = __float_as_uint(x.z);
        r[i + 3] = __float_as_uint(x.w);
      }
      tmem_st32(tmem + tm_lane + P::COL_ST + 64 * ch + 32 * h32, r);
    }
    tmem_wait_st();
    split_state();
    tmem_wait_st();
    tc_fence_before();
    bar_group(kChainBar);

    int pend_mma2 = -1, pend_mma3 = -1, pend_mma4 = -1, pend_mma5 = -1;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % P::kStages, sl = c & 3;
      const int t0 = c * kC;
      const uint32_t kq_a = sbase + P::OFF_KQ + s * P::KQ_BYTES;
      // ---- MMA2: D2 = S'^T [K; Q]^T (S' hi, then lo; B: the stage's key rows
      // then query rows per d block, K-major)
      if (issuer) {
        if (fail(&full_kq[s], kq_parity(c))) bad = true;
        else pend_kq &= ~(3u << (2 * s));
      }
      if (issuer && !bad) {
        tc_fence_after();
        // descriptor start addresses advance by (byte offset >> 4)
        const uint64_t dkq = umma_desc_sw128(kq_a, 16, 1024);
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_bf16_ts(tmem + P::COL_D2, tmem + P::COL_W + 64 * hl + 32 * kb + 8 * ks,
                           dkq + (uint64_t)((kb * 16384 + ks * 32) >> 4), ID_2,
                           (hl > 0 || kb > 0 || ks > 0) ? 1u : 0u);
        umma_commit(mma2_bar);
        pend_mma2 = c & 1;
      }
      if (fail(full_v, (uint32_t)(c & 1))) bad = true;
      else if (issuer) pend_v = -1;
      if (fail(mma2_bar, (uint32_t)(c & 1))) bad = true;
      else if (issuer) pend_mma2 = -1;
      tc_fence_after();

      // ---- Z^T = V^T - gamma (K S')^T as bf16 hi/lo token pairs (in W, which
      // MMA2 has read)
      {
        float z[32];
        uint32_t hi[16], lo[16];
        tmem_ld32(tmem + tm_lane + P::COL_D2 + 32 * ch, z);
        tmem_wait_ld();
        // V[t][v] of the swizzled tile: rows t = 32 ch + i, whose byte offset
        // within the row depends on t mod 8 = i mod 8 only
        const uint8_t* vrow = sV + (v >> 6) * 8192 + 4096 * ch;
        uint32_t voff[8];
#pragma unroll
        for (int r8 = 0; r8 < 8; ++r8)
          voff[r8] = (((((uint32_t)v & 63u) >> 3) ^ (uint32_t)r8) << 4) | (((uint32_t)v & 7u) << 1);
        const float4* gm4 = reinterpret_cast<const float4*>(sc_gam + 64 * sl + 32 * ch);
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 g4 = gm4[i4];
          const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int i = 4 * i4 + e;
            const uint16_t vb0 = *reinterpret_cast<const uint16_t*>(vrow + i * 128 + voff[i & 7]);
            const uint16_t vb1 =
                *reinterpret_cast<const uint16_t*>(vrow + (i + 1) * 128 + voff[(i + 1) & 7]);
            const float2 zz = __ffma2_rn(make_float2(-gv[e], -gv[e + 1]), make_float2(z[i], z[i + 1]),
                                         make_float2(__uint_as_float((uint32_t)vb0 << 16),
                                                     __uint_as_float((uint32_t)vb1 << 16)));
            z[i] = zz.x;
            z[i + 1] = zz.y;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) split_pack2(z[2 * i], z[2 * i + 1], hi[i], lo[i]);
        tmem_st16u(tmem + tm_lane + P::COL_W + 16 * ch, hi);
        tmem_st16u(tmem + tm_lane + P::COL_W + 32 + 16 * ch, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      bar_group(kChainBar);
      // (debug_skip_v: a test hook that leaves one chunk's V copy out, so the
      // bounded wait for it gives up and the CTA takes its abort path)
      if (issuer && !bad && c + 1 < nchunks && c + 1 != debug_skip_v)
        issue_v(c + 1);  // the V tile is consumed

      // ---- MMA3: D3 = Zhi Thi + Zlo Thi + Zhi Tlo (T from the prep warps)
      if (fail(t_ready, (uint32_t)(c & 1))) bad = true;
      // diagonal: stage s is free once MMA1 and the variance of chunk c (both
      // before t_ready) and MMA2 have read it; MMA5 reads G~ instead of K
      if (DIAG && issuer && !bad && c + P::kStages < nchunks) issue_kq(c + P::kStages);
      if (issuer && !bad) {
        tc_fence_after();
        const uint64_t dt = umma_desc_sw128(sbase + P::OFF_T, 16, 1024);
#pragma unroll
        for (int term = 0; term < 3; ++term)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_bf16_ts(tmem + P::COL_D3, tmem + P::COL_W + (term == 1 ? 32 : 0) + 8 * ks,
                         dt + (uint64_t)(((term == 2 ? 8192 : 0) + ks * 32) >> 4), ID_3,
                         (term > 0 || ks > 0) ? 1u : 0u);
        umma_commit(mma3_bar);
        pend_mma3 = c & 1;
      }
      // ---- while MMA3 runs: the state decay by gamma_C (before MMA5 adds to
      // it).  (Q S')^T stays in the query half of D2; MMA4 writes U^T P^T to
      // the key half, which Z has read, and the output pass combines them.
      {
        const float gC = sc_gC[sl];
#pragma unroll
        for (int h32 = 0; h32 < 2; ++h32) {
          float x[32];
          uint32_t r[32];
          tmem_ld32(tmem + tm_lane + P::COL_ST + 64 * ch + 32 * h32, x);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 d = __fmul2_rn(make_float2(gC, gC), make_float2(x[i], x[i + 1]));
            r[i] = __float_as_uint(d.x);
            r[i + 1] = __float_as_uint(d.y);
          }
          tmem_st32(tmem + tm_lane + P::COL_ST + 64 * ch + 32 * h32, r);
        }
      }
      if (fail(mma3_bar, (uint32_t)(c & 1))) bad = true;
      else if (issuer) pend_mma3 = -1;
      tc_fence_after();

      // ---- B^T = coef U^T as bf16 hi/lo token pairs
      {
        float u[32];
        tmem_ld32(tmem + tm_lane + P::COL_D3 + 32 * ch, u);
        tmem_wait_ld();
        const float4* cf4 = reinterpret_cast<const float4*>(sc_coef + 64 * sl + 32 * ch);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 c4 = cf4[i4];
          const float2 b0 = __fmul2_rn(make_float2(c4.x, c4.y), make_float2(u[4 * i4], u[4 * i4 + 1]));
          const float2 b1 =
              __fmul2_rn(make_float2(c4.z, c4.w), make_float2(u[4 * i4 + 2], u[4 * i4 + 3]));
          split_pack2(b0.x, b0.y, hi[2 * i4], lo[2 * i4]);
          split_pack2(b1.x, b1.y, hi[2 * i4 + 1], lo[2 * i4 + 1]);
        }
        tmem_st16u(tmem + tm_lane + P::COL_W + 16 * ch, hi);  // Z has been read
        tmem_st16u(tmem + tm_lane + P::COL_W + 32 + 16 * ch, lo);
      }
      if (!DIAG && issuer) bulk_wait_read_all();  // the previous output tile has been read
      tmem_wait_st();
      tc_fence_before();
      bar_group(kChainBar);

      // ---- MMA5: state += B^T K; MMA4: output += U^T P^T
      if (fail(p_ready, (uint32_t)(c & 1))) bad = true;
      if (issuer && !bad) {
        tc_fence_after();
        if constexpr (DIAG) {
          // state += B^T G~: Bhi G~hi + Blo G~hi + Bhi G~lo (G~ [t][k] MN-major:
          // k blocks 8 KB apart, token groups 1024 B)
          const uint64_t dg = umma_desc_sw128(sbase + P::OFF_G + (c & 1) * 32768u, 8192, 1024);
#pragma unroll
          for (int term = 0; term < 3; ++term)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_bf16_ts(tmem + P::COL_ST, tmem + P::COL_W + (term == 1 ? 32 : 0) + 8 * ks,
                           dg + (uint64_t)(((term == 2 ? 16384 : 0) + ks * 2048) >> 4), ID_5, 1u);
        } else {
          // B = K [t][k] MN-major: k blocks 16 KB apart, token groups 1024 B
          const uint64_t dk = umma_desc_sw128(kq_a, 16384, 1024);
#pragma unroll
          for (int hl = 0; hl < 2; ++hl)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              umma_bf16_ts(tmem + P::COL_ST, tmem + P::COL_W + 32 * hl + 8 * ks,
                           dk + (uint64_t)((ks * 2048) >> 4), ID_5, 1u);
        }
        umma_commit(mma5_bar);
        pend_mma5 = c & 1;
        const uint64_t dp = umma_desc_sw128(sbase + P::OFF_P, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          umma_tf32_ts(tmem + P::COL_D2, tmem + P::COL_D3 + 8 * ks,
                       dp + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4), ID_4,
                       ks > 0 ? 1u : 0u);
        umma_commit(mma4_bar);
        pend_mma4 = c & 1;
      }
      // ---- the state's operand for the next chunk (MMA5 has read B)
      if (fail(mma5_bar, (uint32_t)(c & 1))) bad = true;
      else if (issuer) pend_mma5 = -1;
      tc_fence_after();
      if (c + 1 < nchunks) split_state();
      // ---- o^T of this chunk's tokens [32 ch, 32 ch + 32)
      if (fail(mma4_bar, (uint32_t)(c & 1))) bad = true;
      else if (issuer) pend_mma4 = -1;
      tc_fence_after();
      // (isotropic: into the staging tile [t][v]; one bulk tensor store per
      // chunk writes it, rows past T excluded. diagonal: straight to memory,
      // each warp writing 128 contiguous bytes per token)
      // (also the isotropic variant for the last, partial chunk of a packed
      // sequence: a tile store there would run into the next sequence)
      const bool direct = DIAG || (PACKED && Tn - t0 < kC);
      // o^T [v][t] of this warp's tokens = gamma_t (Q S')^T (query half of D2)
      // + (U^T P^T) (key half)
      auto out_cols = [&](float (&x)[32]) {
        tmem_ld32(tmem + tm_lane + P::COL_D2 + 64 + 32 * ch, x);
        const float4* gm4 = reinterpret_cast<const float4*>(sc_gam + 64 * sl + 32 * ch);
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          float y[16];
          tmem_ld16(tmem + tm_lane + P::COL_D2 + 32 * ch + 16 * h16, y);
          tmem_wait_ld();
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const float4 g4 = gm4[4 * h16 + i4];
            const int i = 16 * h16 + 4 * i4;
            const float2 o0 = __ffma2_rn(make_float2(g4.x, g4.y), make_float2(x[i], x[i + 1]),
                                         make_float2(y[4 * i4], y[4 * i4 + 1]));
            const float2 o1 = __ffma2_rn(make_float2(g4.z, g4.w),
                                         make_float2(x[i + 2], x[i + 3]),
                                         make_float2(y[4 * i4 + 2], y[4 * i4 + 3]));
            x[i] = o0.x;
            x[i + 1] = o0.y;
            x[i + 2] = o1.x;
            x[i + 3] = o1.y;
          }
        }
      };
      if (direct) {
        float x[32];
        out_cols(x);
        const int valid = min(kC, Tn - t0);
        float* dst = O + (((size_t)b * T + tbeg + t0 + 32 * ch) * H + h) * DV + v;
        const size_t ostride = (size_t)H * DV;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (32 * ch + i < valid) dst[i * ostride] = x[i];
      } else {
        float x[32];
        out_cols(x);
        float* dst = sOut + (32 * ch) * DV + v;
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[i * DV] = x[i];
        fence_async_smem();
        // stage s is free (a chunk with the direct store above is the last)
        if (issuer && !bad && c + P::kStages < nchunks) issue_kq(c + P::kStages);
      }
      tmem_wait_st();
      tc_fence_before();
      if (bar_group_or(kChainBar, bad || *sc_abort != 0.f)) {
        bad = true;
        break;
      }
      if (!direct && issuer) {
        tma_store_4d(&tm_o, sOut, 0, h, tbeg + t0, b);
        bulk_commit();
      }
    }
    // abort path: bounded waits for this group's MMAs and copies in flight
    if (issuer) {
      if (pend_mma2 >= 0) (void)mbar_wait(mma2_bar, (uint32_t)pend_mma2);
      if (pend_mma3 >= 0) (void)mbar_wait(mma3_bar, (uint32_t)pend_mma3);
      if (pend_mma4 >= 0) (void)mbar_wait(mma4_bar, (uint32_t)pend_mma4);
      if (pend_mma5 >= 0) (void)mbar_wait(mma5_bar, (uint32_t)pend_mma5);
      for (int st = 0; st < P::kStages; ++st)
        if ((pend_kq >> (2 * st)) & 1u) (void)mbar_wait(&full_kq[st], (pend_kq >> (2 * st + 1)) & 1u);
      if (pend_v >= 0) (void)mbar_wait(full_v, (uint32_t)pend_v);
      if (!DIAG) bulk_wait_all();  // output stores complete
    }
    if (!bad) {
      tc_fence_after();
#pragma unroll
      for (int h32 = 0; h32 < 2; ++h32) {
        float x[32];
        tmem_ld32(tmem + tm_lane + P::COL_ST + 64 * ch + 32 * h32, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(S_out + s_row + 32 * h32 + i) =
              make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
      }
    }
  } else {
    // ================================================================= prep
    const int ptid = tid - kGroup;
    const int pw = warp - 8;
    const int pch = pw >> 2;          // D1 columns [32 pch, 32 pch + 32)
    const bool qrow = m >= 64;        // D1 row: query (P) or key (A) of token tk
    const int tk = m & 63;
    for (int c = 0; c < nchunks; ++c) {
      const int sl = c & 3;
      // ---- D1 epilogue: A (key rows) into AT; P (query rows) kept
      if (fail(mma1_bar, (uint32_t)(c & 1))) bad = true;
      else if (mma1_issuer) pend_mma1 = -1;
      tc_fence_after();
      const float* lg_c = sc_lg + 64 * sl;
      const float* beta_c = sc_beta + 64 * sl;
      float preg[32];
      {
        float d1[32];
        tmem_ld32(tmem + tm_lane + P::COL_D1 + 32 * pch, d1);
        tmem_wait_ld();
        if constexpr (DIAG) {
          // beta_t = 1 / (k_t . G~_t + r_t) from the diagonal of D1, then the
          // state-update coefficients
          if (!qrow && (tk >> 5) == pch) {
            float dd = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) dd = (i == (tk & 31)) ? d1[i] : dd;
            sc_beta[64 * sl + tk] = 1.f / (dd + sc_r[64 * sl + tk]);
          }
          bar_group(kPrepBar);
          if (ptid < 64)
            sc_coef[64 * sl + ptid] = beta_c[ptid] * exp2f(lg_c[kC - 1] - lg_c[ptid]);
        }
        const float lg_t = lg_c[tk];
        const int lim = tk + (qrow ? 1 : 0);  // A: j < t; P: j <= t
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const int j0 = 32 * pch + 4 * i4;
          const float4 lgj = *reinterpret_cast<const float4*>(lg_c + j0);
          const float4 bj = *reinterpret_cast<const float4*>(beta_c + j0);
          const float lj[4] = {lgj.x, lgj.y, lgj.z, lgj.w};
          const float bv[4] = {bj.x, bj.y, bj.z, bj.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            // (gamma_t / gamma_j) beta_j D1, a pair per packed FP32 operation
            const float2 dl = __fadd2_rn(make_float2(lg_t, lg_t), make_float2(-lj[e], -lj[e + 1]));
            const float2 val = __fmul2_rn(
                __fmul2_rn(make_float2(ex2_approx(dl.x), ex2_approx(dl.y)),
                           make_float2(bv[e], bv[e + 1])),
                make_float2(d1[4 * i4 + e], d1[4 * i4 + e + 1]));
            preg[4 * i4 + e] = (j0 + e < lim) ? val.x : 0.f;
            preg[4 * i4 + e + 1] = (j0 + e + 1 < lim) ? val.y : 0.f;
          }
        }
      }
      tc_fence_before();
      if (!qrow) {
        float* row = AT + tk * kLd + 32 * pch;
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4)
          *reinterpret_cast<float4*>(row + 4 * i4) =
              make_float4(preg[4 * i4], preg[4 * i4 + 1], preg[4 * i4 + 2], preg[4 * i4 + 3]);
      } else {
        // P as the tf32 B operand [t][j], once MMA4 of the previous chunk
        // released the buffer
        if (c > 0 && fail(mma4_bar, (uint32_t)((c - 1) & 1))) bad = true;
        uint8_t* dst = sP + pch * 8192;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(dst + chunk_off((uint32_t)tk, (uint32_t)q)) =
              make_uint4(rna_tf32(preg[4 * q]), rna_tf32(preg[4 * q + 1]),
                         rna_tf32(preg[4 * q + 2]), rna_tf32(preg[4 * q + 3]));
      }
      bar_group(kPrepBar);
      // MMA1 of the next chunk: D1 has been read (diagonal: once G~ is written)
      if (!DIAG && mma1_issuer && !bad && c + 1 < nchunks) {
        if (fail(&full_kq[(c + 1) % P::kStages], kq_parity(c + 1))) bad = true;
        else issue_mma1(c + 1);
      }

      // AT and T accessors: A's blocks below the diagonal, T's diagonal blocks,
      // T's blocks below the diagonal (stored transposed above it)
      auto Ael = [&](int i, int l, int r, int k) { return AT[(16 * i + r) * kLd + 16 * l + k]; };
      auto Tdg = [&](int i, int r, int k) { return AT[(16 * i + r) * kLd + 16 * i + k]; };
      auto Tlo = [&](int i, int bb, int r, int k) { return AT[(16 * bb + k) * kLd + 16 * i + r]; };
      auto Tset = [&](int i, int bb, int r, int k, float v0, float v1) {
        AT[(16 * bb + k) * kLd + 16 * i + r] = v0;
        AT[(16 * bb + k + 1) * kLd + 16 * i + r] = v1;
      };
      auto Top = [&](int i, int bb, int r, int k, float v0, float v1) {
        // T[16 i + r][16 bb + k, +1] as bf16 hi/lo pairs
        uint32_t hi, lo;
        split_pack2(v0, v1, hi, lo);
        const uint32_t row = (uint32_t)(16 * i + r), col = (uint32_t)(16 * bb + k);
        const uint32_t off = chunk_off(row, col >> 3) + ((col & 7u) << 1);
        *reinterpret_cast<uint32_t*>(sT + off) = hi;
        *reinterpret_cast<uint32_t*>(sT + 8192 + off) = lo;
      };
      if (pw < 4) {
        // ---- T = (I + A)^-1 (warps 8-11) into AT and as the bf16 hi/lo B
        // operand [t][j] of MMA3, once MMA3 of the previous chunk released it.
        // AT keeps A below the diagonal blocks; T's blocks below the diagonal
        // go to the transposed places above it (T_ib[r][c] at AT[16 b + c][16 i + r]).
        if (c > 0 && fail(mma3_bar, (uint32_t)((c - 1) & 1))) bad = true;
        if (ptid < 64) {
          const int blk = ptid >> 4, cc = ptid & 15;
          const float* Ab = AT + 16 * blk * kLd + 16 * blk;
          float x[16], acc[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
          for (int l = 0; l < 16; ++l) {
            x[l] = (l == cc) ? 1.f : (l < cc ? 0.f : -acc[l]);
#pragma unroll
            for (int i = l + 1; i < 16; ++i) acc[i] = fmaf(Ab[i * kLd + l], x[l], acc[i]);
          }
          named_bar<kPhase1Bar, 64>();  // all A columns read
#pragma unroll
          for (int i = 0; i < 16; ++i) AT[(16 * blk + i) * kLd + 16 * blk + cc] = x[i];
        }
        named_bar<kTeamA, 128>();
        // T_{b+1,b} = -T_{b+1,b+1} A_{b+1,b} T_bb inside each 32-block
        // (b = 0, 2) on the 128 threads: 64 per product, 2x2 outputs each
        {
          const int pr = ptid >> 6, e = ptid & 63;
          const int bb = 2 * pr, i = bb + 1;
          const int r0 = 2 * (e >> 3), c0 = 2 * (e & 7);
          float x00 = 0.f, x01 = 0.f, x10 = 0.f, x11 = 0.f;
          const float* a_r0 = AT + (16 * i + r0) * kLd + 16 * bb;
          const float* tb = AT + (16 * bb) * kLd + 16 * bb + c0;
#pragma unroll
          for (int mm = 0; mm < 16; ++mm) {
            const float2 tt = *reinterpret_cast<const float2*>(tb + mm * kLd);
            const float a0v = a_r0[mm], a1v = a_r0[kLd + mm];
            x00 = fmaf(a0v, tt.x, x00);
            x01 = fmaf(a0v, tt.y, x01);
            x10 = fmaf(a1v, tt.x, x10);
            x11 = fmaf(a1v, tt.y, x11);
          }
          float* xs = X + pr * 320;
          *reinterpret_cast<float2*>(xs + r0 * 20 + c0) = make_float2(x00, x01);
          *reinterpret_cast<float2*>(xs + (r0 + 1) * 20 + c0) = make_float2(x10, x11);
          named_bar<kTeamA, 128>();
          const float* t_r0 = AT + (16 * i + r0) * kLd + 16 * i;
          float y00 = 0.f, y01 = 0.f, y10 = 0.f, y11 = 0.f;
#pragma unroll
          for (int mm = 0; mm < 16; ++mm) {
            const float2 xv = *reinterpret_cast<const float2*>(xs + mm * 20 + c0);
            const float ta = t_r0[mm], tbv = t_r0[kLd + mm];
            y00 = fmaf(ta, xv.x, y00);
            y01 = fmaf(ta, xv.y, y01);
            y10 = fmaf(tbv, xv.x, y10);
            y11 = fmaf(tbv, xv.y, y11);
          }
          // T_ib rows r0, r0 + 1, columns c0, c0 + 1: AT (transposed) and operand
          Tset(i, bb, r0, c0, -y00, -y01);
          Tset(i, bb, r0 + 1, c0, -y10, -y11);
          Top(i, bb, r0, c0, -y00, -y01);
          Top(i, bb, r0 + 1, c0, -y10, -y11);
        }
        // the diagonal blocks into the operand: item -> row 16 i + r, 8 columns
        {
          const int i = ptid >> 5, r = (ptid >> 1) & 15, half = ptid & 1;
          const float* src = AT + (16 * i + r) * kLd + 16 * i + 8 * half;
          const float4 x0 = *reinterpret_cast<const float4*>(src);
          const float4 x1 = *reinterpret_cast<const float4*>(src + 4);
          const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          st_split8(sT, (uint32_t)(16 * i + r), sT + 8192, (uint32_t)(16 * i + r),
                    (uint32_t)(2 * i + half), x);
        }
        named_bar<kTeamA, 128>();
        // the 32x32 block below the diagonal: T^(10) = -T^(1) (A^(10) T^(0)),
        // first X2 = A^(10) T^(0), one 16x16 block per warp (isotropic: on
        // all eight prep warps, below)
        if constexpr (DIAG) {
          const int i2 = 2 + (pw >> 1), b2 = pw & 1;
          {
            float acc[3][2][4] = {};
            if (b2 == 0) {
              warp_mm16(acc, [&](int r, int k) { return Ael(i2, 0, r, k); },
                        [&](int k, int n) { return Tdg(0, k, n); }, lane);
              warp_mm16(acc, [&](int r, int k) { return Ael(i2, 1, r, k); },
                        [&](int k, int n) { return Tlo(1, 0, k, n); }, lane);
            } else {
              warp_mm16(acc, [&](int r, int k) { return Ael(i2, 1, r, k); },
                        [&](int k, int n) { return Tdg(1, k, n); }, lane);
            }
            float* xs = X + pw * 320;
            warp_put16(acc, 1.f, [&](int r, int k, float v0, float v1) {
              *reinterpret_cast<float2*>(xs + r * 20 + k) = make_float2(v0, v1); }, lane);
          }
          named_bar<kTeamA, 128>();
          {
            // X2 block (mm, b2) sits in X slot 2 (mm - 2) + b2
            float acc[3][2][4] = {};
            if (i2 == 2) {
              warp_mm16(acc, [&](int r, int k) { return Tdg(2, r, k); },
                        [&](int k, int n) { return X[b2 * 320 + k * 20 + n]; }, lane);
            } else {
              warp_mm16(acc, [&](int r, int k) { return Tlo(3, 2, r, k); },
                        [&](int k, int n) { return X[b2 * 320 + k * 20 + n]; }, lane);
              warp_mm16(acc, [&](int r, int k) { return Tdg(3, r, k); },
                        [&](int k, int n) { return X[(2 + b2) * 320 + k * 20 + n]; }, lane);
            }
            warp_put16(acc, -1.f, [&](int r, int k, float v0, float v1) {
              Top(i2, b2, r, k, v0, v1); }, lane);
          }
          fence_async_smem();
          named_bar<kTeamA, 128>();
          if (ptid == 0) mbar_arrive(t_ready);
        }
      } else if (c + 1 < nchunks) {
        // ---- the next chunk's scalars (warps 12-15)
        if (warp == 13) {
          store_scalars(c + 1);
          if (c + 2 < nchunks) fetch_scalars(c + 2);
        }
        if (fail(&full_kq[(c + 1) % P::kStages], kq_parity(c + 1))) bad = true;
        if constexpr (DIAG) {
          named_bar<kTeamB, 128>();  // the scalars of chunk c + 1
          tc_fence_after();          // (D1 has been read)
          diag_variance(c + 1, ptid - 128);
          if (warp == 12) decay_and_variance(c + 1);
          // G~ buffer (c + 1) & 1 is free once MMA5 of chunk c - 1 has read it
          if (c > 0 && fail(mma5_bar, (uint32_t)((c - 1) & 1))) bad = true;
          if (!bad) write_gain(c + 1, ptid - 128);
          fence_async_smem();
          tc_fence_before();
          named_bar<kTeamB, 128>();
          if (mma1_issuer && !bad) issue_mma1(c + 1);
        } else {
          key_norms(c + 1, ptid - 128);
          named_bar<kTeamB, 128>();
          if (warp == 12) decay_and_variance(c + 1);
        }
      }
      if constexpr (!DIAG) {
        // ---- isotropic: X2 = A^(10) T^(0), then T^(10) = -T^(1) X2, on all
        // eight prep warps (the next chunk's scalars take warps 12-15 only a
        // part of the T solve): warp pw takes n-tile pw >> 2 of the 16x16
        // block pw & 3; X2 block (mm, b2) sits in X slot 2 (mm - 2) + b2
        const int blk = pw & 3, nt = pw >> 2;
        const int i2 = 2 + (blk >> 1), b2 = blk & 1;
        bar_group(kPrepBar);  // T's diagonal and level-1 blocks are in AT
        {
          float acc[3][4] = {};
          if (b2 == 0) {
            warp_mm16n(acc, [&](int r, int k) { return Ael(i2, 0, r, k); },
                       [&](int k, int n) { return Tdg(0, k, n); }, nt, lane);
            warp_mm16n(acc, [&](int r, int k) { return Ael(i2, 1, r, k); },
                       [&](int k, int n) { return Tlo(1, 0, k, n); }, nt, lane);
          } else {
            warp_mm16n(acc, [&](int r, int k) { return Ael(i2, 1, r, k); },
                       [&](int k, int n) { return Tdg(1, k, n); }, nt, lane);
          }
          float* xs = X + blk * 320;
          warp_put16n(acc, 1.f, [&](int r, int k, float v0, float v1) {
            *reinterpret_cast<float2*>(xs + r * 20 + k) = make_float2(v0, v1); }, nt, lane);
        }
        bar_group(kPrepBar);
        {
          float acc[3][4] = {};
          if (i2 == 2) {
            warp_mm16n(acc, [&](int r, int k) { return Tdg(2, r, k); },
                       [&](int k, int n) { return X[b2 * 320 + k * 20 + n]; }, nt, lane);
          } else {
            warp_mm16n(acc, [&](int r, int k) { return Tlo(3, 2, r, k); },
                       [&](int k, int n) { return X[b2 * 320 + k * 20 + n]; }, nt, lane);
            warp_mm16n(acc, [&](int r, int k) { return Tdg(3, r, k); },
                       [&](int k, int n) { return X[(2 + b2) * 320 + k * 20 + n]; }, nt, lane);
          }
          warp_put16n(acc, -1.f, [&](int r, int k, float v0, float v1) {
            Top(i2, b2, r, k, v0, v1); }, nt, lane);
        }
      }

      fence_async_smem();
      if (bar_group_or(kPrepBar, bad || *sc_abort != 0.f)) {
        bad = true;
        break;
      }
      if (!DIAG && ptid == 0) mbar_arrive(t_ready);
      if (ptid == 0) mbar_arrive(p_ready);
    }
    if (mma1_issuer && pend_mma1 >= 0) (void)mbar_wait(mma1_bar, (uint32_t)pend_mma1);
    if (DIAG && warp >= 12 && lane == 0)
      for (int bf = 0; bf < 2; ++bf)
        if ((pend_w >> (2 * bf)) & 1u)
          (void)mbar_wait(&w_full[2 * (warp - 12) + bf], (pend_w >> (2 * bf + 1)) & 1u);
    if constexpr (DIAG) {
      if (ptid >= 128 && !bad) P_out[(size_t)bh * kDK + ptid - 128] = sc_pcar[ptid - 128];
    } else {
      if (ptid == 0 && !bad) P_out[bh] = sc_pcar[0];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
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

// [B, T, H, d] fp32 tensor, boxes of (box_d columns (default d), 1 head, box_t
// tokens, 1 batch)
bool make_out_map(CUtensorMap* m, const void* base, int B, int T, int H, int d, int box_t,
                  int box_d = 0) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)T * H * d * 4};
  cuuint32_t box[4] = {(cuuint32_t)(box_d > 0 ? box_d : d), 1, (cuuint32_t)box_t, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

// (cu_seqlens: B packed sequences in [1, T, H, d] tensors, T = total tokens)
// (v_zero_rows > 0: v is a zeroed [1, v_zero_rows, H, 128] buffer, so every V
// copy reads zeros, inside it or past its bounds, where TMA fills zeros)
template <bool DIAG>
kdn_status launch_ws(const void* q, const void* k, const void* v, const float* a,
                     const float* w, const float* r, const float* S0, const float* p0, float* o,
                     float* S_out, float* p_out, int B, int T, int H, float kappa, void* ws,
                     cudaStream_t s, int debug_skip_v, const int* cu_seqlens,
                     int v_zero_rows = 0) {
  const int Bm = cu_seqlens ? 1 : B;  // batch extent of the tensor maps
  using P = WsPlan<DIAG>;
  CUtensorMap mq, mk, mv, mo, mw;
  if (!make_map(&mq, q, Bm, T, H, kDK, 64) || !make_map(&mk, k, Bm, T, H, kDK, 64) ||
      !(v_zero_rows > 0 ? make_map(&mv, v, 1, v_zero_rows, H, 128, 64)
                        : make_map(&mv, v, Bm, T, H, 128, 64)))
    return KDN_ERR_CUDA;
  // isotropic: the output tile map; diagonal: the output is written without a
  // map, and w [B, T, H, 128] is read in boxes of 16 tokens
  if (DIAG) {
    mo = mq;
    if (!make_out_map(&mw, w, Bm, T, H, kDK, 16, 32)) return KDN_ERR_CUDA;
  } else {
    if (!make_out_map(&mo, o, Bm, T, H, 128, 64)) return KDN_ERR_CUDA;
    mw = mq;
  }
  static bool attr_set[2] = {false, false};
  auto kern = cu_seqlens ? chunk_engine_ws_kernel<DIAG, true> : chunk_engine_ws_kernel<DIAG, false>;
  if (!attr_set[cu_seqlens ? 1 : 0]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P::ALLOC) !=
        cudaSuccess)
      return KDN_ERR_CUDA;
    attr_set[cu_seqlens ? 1 : 0] = true;
  }
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return KDN_ERR_CUDA;
  // packed sequences: longest first once the problems outnumber the SMs (the
  // order goes after the error word; the workspace holds B * H floats there)
  int* order = nullptr;
  if (cu_seqlens) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return KDN_ERR_CUDA;
    if (B * H > sms) {
      order = reinterpret_cast<int*>(static_cast<char*>(ws) + 256);
      varlen_order_kernel<<<1, kOrderThreads, 0, s>>>(cu_seqlens, B, T, order);
    }
  }
  kern<<<(unsigned)(B * H), kThreads, P::ALLOC, s>>>(
      mq, mk, mv, mo, mw, a, w, r, S0, p0, o, S_out, p_out, T, H, kappa,
      static_cast<uint32_t*>(ws), debug_skip_v, cu_seqlens, order);
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
                               int T, int H, int dv, float kappa, void* ws, cudaStream_t s,
                               int debug_skip_v, const int* cu_seqlens) {
  if (dv == 128) {
    // one CTA per head reads p0 and writes p_out: no snapshot needed
    return diag ? launch_ws<true>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, kappa, ws,
                                  s, debug_skip_v, cu_seqlens)
                : launch_ws<false>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, kappa, ws,
                                   s, debug_skip_v, cu_seqlens);
  }
  // the hook and packed sequences exist at d_v = 128 only
  if (debug_skip_v >= 0 || cu_seqlens) return KDN_ERR_UNSUPPORTED;
  return diag ? launch<true, 64>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, ws, s)
              : launch<false, 64>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, ws, s);
}

// The d_v = 128 engine with V taken as zero: v_zero is a zeroed [1, 64, H,
// 128] bf16 buffer (16-byte aligned).  Used for the state-transition runs of
// the segmented long-sequence forward.
kdn_status chunk_engine_launch_zero_v(bool diag, const void* q, const void* k, const void* v_zero,
                                      const float* a, const float* w, const float* r,
                                      const float* S0, const float* p0, float* o, float* S_out,
                                      float* p_out, int B, int T, int H, float kappa, void* ws,
                                      cudaStream_t s) {
  return diag ? launch_ws<true>(q, k, v_zero, a, w, r, S0, p0, o, S_out, p_out, B, T, H, kappa, ws,
                                s, -1, nullptr, 64)
              : launch_ws<false>(q, k, v_zero, a, w, r, S0, p0, o, S_out, p_out, B, T, H, kappa,
                                 ws, s, -1, nullptr, 64);
}

}  // namespace kdn
