// Chunked tensor-core engine of the information-form diagonal filter (KLA),
// d_k = d_v = 128, bf16 q, k, v.
//
// "Kalman Linear Attention: Parallel Bayesian Filtering ..." (方法论 §2):
// given the precision path, the information mean is an affine recursion, so
// it can run in parallel over a stretch of tokens.  On the KDN memory model,
// per token and key dimension i (all value rows share it):
//   p-  = a^2 p + w,   p = p- r / (r + p- k^2)       (p = 1 / lambda)
//   f_i = a r / (r + p- k^2)    forget gate (a lambda- / lambda)
//   u_i = k p- / (r + p- k^2)   write gate ((k / r) / lambda)
//   S   = S diag(f) + v u^T,    o = S q
// Over a piece [o, o + L) of tokens, with G_t = prod_{r = o..t} f_r per key
// dimension (inclusive, so G_o = f_o), the state after token t is
//   S_t = (S_start + sum_{s in [o, t]} v_s (u_s / G_s)^T) diag(G_t),
// hence, with Q~ = Q . G and U~ = U / G (elementwise, rows = tokens):
//   o_t   = S_start Q~_t + sum_{s <= t} A_ts v_s,   A = (Q~ U~^T) masked to s <= t
//   S_end = (S_start + V^T U~) diag(G_L).
// Every product is a dense contraction, so each 64-token chunk runs on the
// tensor cores (tcgen05, operands in shared memory or TMEM, fp32 accumulation
// in TMEM), transposed so that the value index v lies on the 128 TMEM lanes:
//   MMA-A:  D_A[r][s] = sum_i Qs[r][i] U~[s][i]    Qs = [Q~ hi; Q~ lo] (128 rows),
//           U~ as hi then lo; the two halves of D_A sum to A
//   MMA-O:  D_o[v][t] = sum_i S[v][i] Q~[t][i]      S as bf16 hi/lo in TMEM
//   MMA-dS: S[v][i]  += sum_s V[s][v] U~[s][i]
//   MMA-I:  D_o[v][t] += sum_s V[s][v] A[t][s]       A as hi/lo (top half) + hi (bottom)
// and a TMEM pass per piece scales S by G_L and splits it into bf16 hi/lo for
// the next piece.  Every fp32 operand is split into bf16 hi + lo (16
// significant bits), v, q and k are exact bf16.
//
// Range.  U~ = U / G grows as the forget gates multiply down.  A piece keeps
// every G_t >= 2^-100, so U~ <= 2^100 |u| and Q~ >= 2^-100 |q| stay normal
// numbers and S + V^T U~ stays far below the fp32 limit.  A chunk is one
// piece when its gates allow it (checked once per chunk: G only falls); else it
// is cut where G would cross the bound, down to single tokens.  A single
// token with f below the bound is scaled by the bound instead: its own term
// A_tt = q.u does not depend on the scale, and the inter-piece terms then
// differ from the exact ones by at most 2^-100 of S_start.
//
// Roles (14 warps, one CTA per (b, h)):
//  - warps 0-3, prep: thread i runs key dimension i's variance recursion in
//    projective form (p = x / y; no division on the token-to-token chain),
//    forms Q~ and U~ rows (bf16 hi/lo, 128-byte swizzled K-major tiles) into
//    one of two operand sets, and closes pieces.  Their barrier and range vote
//    go through an mbarrier with a bounded wait, so no thread can wait for
//    one that has left on a timeout.
//  - warps 4-7, state: one TMEM lane quarter each; after MMA-dS they scale S
//    by G_L and write its bf16 hi/lo split (or, after the last piece, S_T).
//  - warps 8-11, A and output: after MMA-A they sum the two halves of D_A
//    through the MMA-I operand (top half as hi/lo, bottom half as hi: the
//    bottom is Q~ lo U~, below 2^-8 of A), mask it causal and write it as
//    bf16 tiles; after a chunk's last MMA-I they drain D_o to o.  Warp 8
//    lane 0 copies each chunk's V tile once the previous chunk is done with it.
//  - warp 12, lane 0: issues every MMA and commit.
//  - warp 13, loader: copies q, k and w of each 16-token quarter into one of
//    three stages (bulk tensor copies, with an L2 prefetch further ahead) and
//    writes the quarter's a^2, a r and r beside them.
// Hand-over is by mbarriers with bounded waits; a wait that gives up records
// DEV_TIMEOUT in the workspace's error word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kKC = 64;                 // tokens per chunk
constexpr int kKQ = 16;                 // tokens per staged quarter
constexpr int kKStages = 3;             // quarter stages
constexpr int kKWarps = 14;
constexpr int kKThreads = kKWarps * 32;
constexpr float kRangeFloor = 7.8886090522101181e-31f;  // 2^-100

struct KP {
  // operand set: Qs [2 K halves][128 rows][128 B] | U~ hi [2][64][128 B] | U~ lo
  static constexpr uint32_t QS = 0, UH = 32768, UL = 49152, SET = 65536;
  static constexpr uint32_t OFF_SET = 0;                       // two sets
  static constexpr uint32_t OFF_V = 2 * SET;                   // [2 v halves][64 s][128 B]
  static constexpr uint32_t OFF_A = OFF_V + 16384;             // A top hi | top lo | bottom hi
  static constexpr uint32_t A_TILE = 8192;
  static constexpr uint32_t OFF_STG = OFF_A + 3 * A_TILE;      // quarter stages
  // stage: q [16][128] bf16 | k | w [16][128] fp32 | a^2, a r, r [16] each
  static constexpr uint32_t STG_Q = 0, STG_K = 4096, STG_W = 8192, STG_AR = 16384;
  static constexpr uint32_t STG_TX = 16384, STG = 16640;
  static constexpr uint32_t OFF_META = OFF_STG + kKStages * STG;  // [4 slots] G_L[128] + info
  static constexpr uint32_t META = 528;
  static constexpr uint32_t OFF_BAR = OFF_META + 4 * META;
  static constexpr uint32_t NBAR = 26;
  // tmem base, abort flag, three rotating vote words of the prep barrier
  static constexpr uint32_t OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr uint32_t TOTAL = OFF_MISC + 32;
  static constexpr uint32_t SMEM = TOTAL + 1024;               // 1024-byte alignment slack
};
static_assert(KP::OFF_STG % 1024 == 0 && KP::OFF_A % 1024 == 0, "tile alignment");
static_assert(KP::SMEM <= 232448, "shared memory plan");

// TMEM columns: S fp32 [0,128), S hi/lo [128,256), D_o x2 [256,384), D_A [384,448)
constexpr uint32_t kColS = 0, kColSP = 128, kColO = 256, kColA = 384, kTmemCols = 512;

// mbarrier indices
enum : int {
  B_OP_FULL = 0,    // [2] prep -> issuer: operand set written (count 1)
  B_OP_EMPTY = 2,   // [2] issuer commit: the set's MMAs are done
  B_META = 4,       // [4] prep -> state, A warps: piece info (count 1)
  B_A_FULL = 8,     // MMA-A done
  B_A_READY = 9,    // A tiles written (count 4)
  B_A_FREE = 10,    // MMA-I done (A tiles reusable)
  B_DS_DONE = 11,   // MMA-dS done
  B_S_READY = 12,   // S scaled and split (count 4)
  B_O_FULL = 13,    // [2] a chunk's D_o complete
  B_O_EMPTY = 15,   // [2] D_o drained (count 4)
  B_V_FULL = 17,    // V tile landed (tx)
  B_STG = 18,       // [3] quarter stage landed (tx, and the loader's a/r stores)
  B_STG_EMPTY = 21, // [3] the prep is done with a stage (count 4)
  B_FINAL = 24,     // the issuer's last commit
  B_PREP = 25,      // the prep warps' barrier (count 128)
};
static_assert(B_FINAL < (int)KP::NBAR, "barrier count");

// piece info flags
enum : uint32_t { PF_FIRST = 1u, PF_LAST_OF_CHUNK = 2u, PF_LAST = 4u };

__device__ __forceinline__ void tma_load_4d_prefetch(const void* tmap, int c0, int c1, int c2,
                                                     int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   tmap),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// (hi, lo) bf16 pairs of two consecutive fp32 values, the lower index in the
// low half of each word.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  // both remainders in one packed FMA (each rounded as the scalar subtraction)
  const float2 r = __ffma2_rn(hf, make_float2(-1.f, -1.f), make_float2(x0, x1));
  const __nv_bfloat162 l = __floats2bfloat162_rn(r.x, r.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// 1 / x to within an ulp or two (one MUFU operation); x is a normal number
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One token of key dimension i's filter in projective form, p = x / y:
// (x, y) -> (r um, um k^2 + r y) with um = a^2 x + w y (= p- y).  Returns the
// forget gate f = a r y / den and the write gate u = k um / den.  a2 = a^2
// and ar = a r are the token's scalars.
__device__ __forceinline__ void kla_step(float a2, float ar, float r, float kk, float w, float& x,
                                         float& y, float& f, float& u) {
  const float um = __fmaf_rn(a2, x, w * y);
  const float den = __fmaf_rn(um * kk, kk, r * y);
  const float inv = rcp_fast(den);
  f = (ar * y) * inv;
  u = (kk * um) * inv;
  x = r * um;
  y = den;
}

// Exact power-of-two rescale of (x, y) that brings y into [1, 2).
__device__ __forceinline__ void kla_rescale(float& x, float& y) {
  const float s = __uint_as_float((254u - ((__float_as_uint(y) >> 23) & 0xffu)) << 23);
  x *= s;
  y *= s;
}

// Operand-tile stores of the prep.  They carry no memory clobber, so the
// compiler may move the stage loads of later tokens above them: the stages
// and the operand sets never overlap.  Every path from these stores to an MMA
// passes a fence and a barrier (asm volatile, which keeps their order).
__device__ __forceinline__ void st_bf16(uint8_t* p, __nv_bfloat16 x) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_u32(p)), "h"(__bfloat16_as_ushort(x)));
}
// One token row of a set from packed pairs: hi = (Q~ hi, U~ hi), lo = (Q~ lo,
// U~ lo), each with Q~ in the low half.
__device__ __forceinline__ void st_row4p(uint32_t qa, uint32_t ua, uint32_t hi, uint32_t lo) {
  asm volatile(
      "{\n\t.reg .b16 qh, uh, ql, ul;\n\t"
      "mov.b32 {qh, uh}, %2;\n\t"
      "mov.b32 {ql, ul}, %3;\n\t"
      "st.shared.b16 [%0], qh;\n\t"
      "st.shared.b16 [%0+8192], ql;\n\t"
      "st.shared.b16 [%1], uh;\n\t"
      "st.shared.b16 [%1+16384], ul;\n\t}" ::"r"(qa),
      "r"(ua), "r"(hi), "r"(lo));
}

__global__ void __launch_bounds__(kKThreads, 1)
kla_engine_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const __grid_constant__ CUtensorMap mw, const __grid_constant__ CUtensorMap mv,
                  const float* __restrict__ A_in, const float* __restrict__ R_in,
                  const __nv_bfloat16* __restrict__ Qg, const __nv_bfloat16* __restrict__ Kg,
                  const float* __restrict__ Wg,
                  const float* S0, const float* L0, float* __restrict__ O, float* S_out,
                  float* L_out, int T, int H, uint32_t* err, int debug_skip_v) {
  extern __shared__ uint8_t ksm_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that every
  // access through `sm` stays a shared-memory access
  uint8_t* sm = ksm_raw + ((1024u - (smem_u32(ksm_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int nchunks = (T + kKC - 1) / kKC;
  const int nquarters = (T + kKQ - 1) / kKQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + KP::OFF_BAR);
  uint32_t* misc = reinterpret_cast<uint32_t*>(sm + KP::OFF_MISC);
  volatile uint32_t* abort_flag = misc + 1;

  auto fail = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return true;
    if (mbar_wait(bar, parity)) return false;
    *abort_flag = 1u;
    atomicOr(err, DEV_TIMEOUT);
    return true;
  };
  auto tok_index = [&](int t) -> size_t { return ((size_t)b * T + t) * H + h; };

  // ------------------------------------------------------------- set-up
  if (tid == 0) {
    mbar_init(&bars[B_OP_FULL], 1);
    mbar_init(&bars[B_OP_FULL + 1], 1);
    mbar_init(&bars[B_OP_EMPTY], 1);
    mbar_init(&bars[B_OP_EMPTY + 1], 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars[B_META + i], 1);
    mbar_init(&bars[B_A_FULL], 1);
    mbar_init(&bars[B_A_READY], 4);
    mbar_init(&bars[B_A_FREE], 1);
    mbar_init(&bars[B_DS_DONE], 1);
    mbar_init(&bars[B_S_READY], 4);
    mbar_init(&bars[B_O_FULL], 1);
    mbar_init(&bars[B_O_FULL + 1], 1);
    mbar_init(&bars[B_O_EMPTY], 4);
    mbar_init(&bars[B_O_EMPTY + 1], 4);
    mbar_init(&bars[B_V_FULL], 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars[B_STG + i], 2);
      mbar_init(&bars[B_STG_EMPTY + i], 4);
    }
    mbar_init(&bars[B_FINAL], 1);
    mbar_init(&bars[B_PREP], 128);
    misc[1] = 0u;
    misc[2] = misc[3] = misc[4] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mw);
    tma_prefetch_desc(&mv);
  }
  if (warp == 12) {
    tmem_alloc(misc, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  // first copy: the V tile of chunk 0
  if (warp == 8 && lane == 0) {
    mbar_expect_tx(&bars[B_V_FULL], 16384);
    tma_load_4d(sm + KP::OFF_V, &mv, &bars[B_V_FULL], 0, h, 0, b);
    tma_load_4d(sm + KP::OFF_V + 8192, &mv, &bars[B_V_FULL], 64, h, 0, b);
    if (nchunks > 1) {
      tma_load_4d_prefetch(&mv, 0, h, kKC, b);
      tma_load_4d_prefetch(&mv, 64, h, kKC, b);
    }
  }
  if (warp >= 4 && warp < 8) {
    // S0 row v into TMEM (fp32) and its bf16 hi/lo split
    const int v = 32 * (warp & 3) + lane;
    const uint32_t tl = (uint32_t)(32 * (warp & 3)) << 16;
#pragma unroll 1
    for (int g = 0; g < 4; ++g) {
      float x[32];
      const float* src = S0 ? S0 + ((size_t)bh * 128 + v) * 128 + 32 * g : nullptr;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 y = src ? *reinterpret_cast<const float4*>(src + j)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        x[j] = y.x; x[j + 1] = y.y; x[j + 2] = y.z; x[j + 3] = y.w;
      }
      uint32_t xs[32], hi[16], lo[16];
#pragma unroll
      for (int j = 0; j < 32; ++j) xs[j] = __float_as_uint(x[j]);
#pragma unroll
      for (int j = 0; j < 16; ++j) split2(x[2 * j], x[2 * j + 1], hi[j], lo[j]);
      tmem_st32(tmem + tl + kColS + 32 * g, xs);
      tmem_st16u(tmem + tl + kColSP + 16 * g, hi);
      tmem_st16u(tmem + tl + kColSP + 64 + 16 * g, lo);
    }
    tmem_wait_st();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();

  if (warp < 4) {
    // ============================================================== prep
    const int i = tid;                      // key dimension
    const uint32_t col_half = (uint32_t)(i >> 6), col = (uint32_t)(i & 63);
    float x = L0 ? 1.f / L0[(size_t)bh * 128 + i] : 1.f, y = 1.f;  // p = x / y
    int p = 0;                              // pieces closed so far
    bool bad = false;
    auto set_ptr = [&](int pc) { return sm + KP::OFF_SET + (uint32_t)(pc & 1) * KP::SET; };
    auto acquire_set = [&](int pc) {
      if (pc >= 2 && fail(&bars[B_OP_EMPTY + (pc & 1)], (uint32_t)(((pc >> 1) - 1) & 1)))
        bad = true;
    };
    // this column's byte offset within a swizzled row r, by r % 8
    uint32_t swz[8];
#pragma unroll
    for (int k8 = 0; k8 < 8; ++k8) swz[k8] = (((col >> 3) ^ (uint32_t)k8) << 4) + (col & 7u) * 2u;
    // row t of a set: Q~ hi (row t), Q~ lo (row 64 + t), U~ hi, U~ lo; `off`
    // is the row's offset t * 128 + swizzled column
    const uint32_t qcol = KP::QS + col_half * 16384u, ucol = KP::UH + col_half * 8192u;
    auto write_row_at = [&](uint8_t* st, uint32_t off, float qt, float ut) {
      uint32_t hi, lo;
      split2(qt, ut, hi, lo);
      st_row4p(smem_u32(st) + qcol + off, smem_u32(st) + ucol + off, hi, lo);
    };
    auto write_row = [&](uint8_t* st, int t, float qt, float ut) {
      write_row_at(st, sw128_offset((uint32_t)t, col), qt, ut);
    };
    auto zero_rows = [&](uint8_t* st, int r0, int r1) {
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
      for (int t = r0; t < r1; ++t) {
        uint8_t* qs = st + KP::QS + col_half * 16384;
        st_bf16(qs + sw128_offset((uint32_t)t, col), z);
        st_bf16(qs + sw128_offset((uint32_t)(64 + t), col), z);
        st_bf16(st + KP::UH + col_half * 8192 + sw128_offset((uint32_t)t, col), z);
        st_bf16(st + KP::UL + col_half * 8192 + sw128_offset((uint32_t)t, col), z);
      }
    };
    // Barrier of the 128 prep threads with a vote: true when `ok` held on all
    // of them.  Use k arrives on the mbarrier's phase k and ORs this warp's
    // failures into vote word k % 3; word k + 2 is cleared after the wait (no
    // thread can still read it: use k completes only after every thread has
    // finished use k - 1).  A wait that gives up sets `bad`.
    volatile uint32_t* vote = misc + 2;
    int puse = 0;
    auto prep_vote = [&](bool ok) -> bool {
      const int k = puse++;
      if (!__all_sync(0xffffffffu, ok) && (i & 31) == 0) atomicOr((uint32_t*)&vote[k % 3], 1u);
      __syncwarp();
      mbar_arrive(&bars[B_PREP]);
      if (fail(&bars[B_PREP], (uint32_t)(k & 1))) {
        bad = true;
        return false;
      }
      const bool all = vote[k % 3] == 0u;
      if (i == 0) vote[(k + 2) % 3] = 0u;
      return all;
    };
    // publish piece p: its G_L and flags, then hand the set to the issuer
    auto close_piece = [&](int c, float GL, uint32_t flags) {
      uint8_t* meta = sm + KP::OFF_META + (uint32_t)(p & 3) * KP::META;
      reinterpret_cast<float*>(meta)[i] = GL;
      if (i == 0) {
        reinterpret_cast<uint32_t*>(meta + 512)[0] = (uint32_t)c;
        reinterpret_cast<uint32_t*>(meta + 512)[1] = flags;
      }
      fence_async_smem();
      prep_vote(true);
      if (bad) return;
      if (i == 0) {
        mbar_arrive(&bars[B_OP_FULL + (p & 1)]);
        mbar_arrive(&bars[B_META + (p & 3)]);
      }
      ++p;
    };

    int qi = 0;
    for (int c = 0; c < nchunks && !bad; ++c) {
      const int n = min(kKC, T - kKC * c);
      acquire_set(p);
      if (bad) break;
      uint8_t* st = set_ptr(p);
      bool first = true;       // the open piece is the chunk's first
      float G = 1.f;           // prod of f over the open piece
      const float xc = x, yc = y;  // for the slow path
      for (int j = 0; kKQ * j < n; ++j, ++qi) {
        const int nq = min(kKQ, n - kKQ * j);
        const int stage = qi % kKStages;
        if (fail(&bars[B_STG + stage], (uint32_t)((qi / kKStages) & 1))) { bad = true; break; }
        const uint8_t* sg = sm + KP::OFF_STG + stage * KP::STG;
        const float* ar = reinterpret_cast<const float*>(sg + KP::STG_AR);

        const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(sg + KP::STG_Q) + i;
        const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(sg + KP::STG_K) + i;
        const float* sw = reinterpret_cast<const float*>(sg + KP::STG_W) + i;
        const uint32_t row0 = (uint32_t)(kKQ * j) * 128u;
        if (nq == kKQ) {
          // a whole quarter: eight tokens' inputs into registers, then their
          // rows
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float kv[8], wv[8], qv[8], a2v[8], arv[8], rv[8];
#pragma unroll
            for (int e = 0; e < 8; e += 4) {
              const float4 x2 = *reinterpret_cast<const float4*>(ar + 8 * hh + e);
              const float4 xa = *reinterpret_cast<const float4*>(ar + 16 + 8 * hh + e);
              const float4 xr = *reinterpret_cast<const float4*>(ar + 32 + 8 * hh + e);
              a2v[e] = x2.x; a2v[e + 1] = x2.y; a2v[e + 2] = x2.z; a2v[e + 3] = x2.w;
              arv[e] = xa.x; arv[e + 1] = xa.y; arv[e + 2] = xa.z; arv[e + 3] = xa.w;
              rv[e] = xr.x; rv[e + 1] = xr.y; rv[e + 2] = xr.z; rv[e + 3] = xr.w;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int tt = 8 * hh + e;
              kv[e] = __bfloat162float(sk[tt * 128]);
              wv[e] = sw[tt * 128];
              qv[e] = __bfloat162float(sq[tt * 128]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int tt = 8 * hh + e;
              float f, u;
              kla_step(a2v[e], arv[e], rv[e], kv[e], wv[e], x, y, f, u);
              if ((tt & 3) == 3) kla_rescale(x, y);
              G *= f;
              write_row_at(st, row0 + (uint32_t)tt * 128u + swz[tt & 7], qv[e] * G,
                           u * rcp_fast(G));
            }
          }
        } else {
          for (int tt = 0; tt < nq; ++tt) {
            float f, u;
            kla_step(ar[tt], ar[16 + tt], ar[32 + tt], __bfloat162float(sk[tt * 128]),
                     sw[tt * 128], x, y, f, u);
            if ((tt & 3) == 3) kla_rescale(x, y);
            G *= f;
            write_row(st, kKQ * j + tt, __bfloat162float(sq[tt * 128]) * G, u * rcp_fast(G));
          }
        }
        // this warp's reads of the stage are done: hand it back to the loader
        __syncwarp();
        if ((i & 31) == 0) mbar_arrive(&bars[B_STG_EMPTY + stage]);
      }
      if (bad) break;
      // G only falls, so its value at the chunk's end bounds every token's
      const bool in_range = prep_vote(G >= kRangeFloor);
      if (bad) break;
      if (!in_range) {
        // cut the chunk into pieces that keep G >= 2^-100: run it again from
        // its start, one vote per token, with its inputs read from global
        // memory (the stages have gone back to the loader)
        x = xc;
        y = yc;
        G = 1.f;
        int start = 0;  // first row of the open piece
        for (int t = 0; t < n; ++t) {
          const size_t tok = tok_index(kKC * c + t);
          const float a = A_in[tok], r = R_in[tok];
          float f, u;
          kla_step(a * a, a * r, r, __bfloat162float(Kg[tok * 128 + i]), Wg[tok * 128 + i], x,
                   y, f, u);
          if ((t & 3) == 3) kla_rescale(x, y);
          float Gt = G * f;
          const bool t_in_range = prep_vote(Gt >= kRangeFloor);
          if (bad) break;
          if (!t_in_range) {
            if (t > start) {
              zero_rows(st, t, kKC);
              close_piece(c, G, first ? PF_FIRST : 0u);
              if (bad) break;
              first = false;
              acquire_set(p);
              if (bad) break;
              st = set_ptr(p);
              zero_rows(st, 0, t);
            }
            start = t;
            Gt = fmaxf(f, kRangeFloor);
          }
          G = Gt;
          write_row(st, t, __bfloat162float(Qg[tok * 128 + i]) * G, u * rcp_fast(G));
        }
        if (bad) break;
      }
      if (n < kKC) zero_rows(st, n, kKC);
      close_piece(c, G, (first ? PF_FIRST : 0u) | PF_LAST_OF_CHUNK |
                            (c == nchunks - 1 ? PF_LAST : 0u));
    }
    if (!bad) L_out[(size_t)bh * 128 + i] = y / x;
  } else if (warp < 8) {
    // ============================================================= state
    const int v = 32 * (warp & 3) + lane;
    const uint32_t tl = (uint32_t)(32 * (warp & 3)) << 16;
    for (int p = 0;; ++p) {
      if (fail(&bars[B_META + (p & 3)], (uint32_t)((p >> 2) & 1))) break;
      const uint8_t* meta = sm + KP::OFF_META + (uint32_t)(p & 3) * KP::META;
      const uint32_t flags = reinterpret_cast<const uint32_t*>(meta + 512)[1];
      const float* GL = reinterpret_cast<const float*>(meta);
      if (fail(&bars[B_DS_DONE], (uint32_t)(p & 1))) break;
      tc_fence_after();
      // 32 columns at a time, two loads in flight per wait
      auto scale_split = [&](float (&x)[32], int g) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 gl = *reinterpret_cast<const float4*>(GL + 32 * g + j);
          const float2 p0 = __fmul2_rn(make_float2(x[j], x[j + 1]), make_float2(gl.x, gl.y));
          const float2 p1 = __fmul2_rn(make_float2(x[j + 2], x[j + 3]), make_float2(gl.z, gl.w));
          x[j] = p0.x; x[j + 1] = p0.y; x[j + 2] = p1.x; x[j + 3] = p1.y;
        }
        if (flags & PF_LAST) {
          float* dst = S_out + ((size_t)bh * 128 + v) * 128 + 32 * g;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
        } else {
          uint32_t xs[32], hi[16], lo[16];
#pragma unroll
          for (int j = 0; j < 32; ++j) xs[j] = __float_as_uint(x[j]);
#pragma unroll
          for (int j = 0; j < 16; ++j) split2(x[2 * j], x[2 * j + 1], hi[j], lo[j]);
          tmem_st32(tmem + tl + kColS + 32 * g, xs);
          tmem_st16u(tmem + tl + kColSP + 16 * g, hi);
          tmem_st16u(tmem + tl + kColSP + 64 + 16 * g, lo);
        }
      };
#pragma unroll 1
      for (int g = 0; g < 4; g += 2) {
        float x0[32], x1[32];
        tmem_ld32(tmem + tl + kColS + 32 * g, x0);
        tmem_ld32(tmem + tl + kColS + 32 * (g + 1), x1);
        tmem_wait_ld();
        scale_split(x0, g);
        scale_split(x1, g + 1);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_S_READY]);
      if (flags & PF_LAST) break;
    }
  } else if (warp < 12) {
    // ======================================================= A and output
    const int L = 32 * (warp & 3) + lane;  // TMEM lane: D_A row, D_o value index
    const uint32_t tl = (uint32_t)(32 * (warp & 3)) << 16;
    const bool top = L < 64;
    const int t = L & 63;
    uint8_t* a_hi = sm + KP::OFF_A + (top ? 0u : 2u * KP::A_TILE);
    uint8_t* a_lo = sm + KP::OFF_A + KP::A_TILE;
    int v_last = 0;  // chunk of the last V copy issued
    for (int p = 0;; ++p) {
      if (fail(&bars[B_META + (p & 3)], (uint32_t)((p >> 2) & 1))) break;
      const uint8_t* meta = sm + KP::OFF_META + (uint32_t)(p & 3) * KP::META;
      const int c = (int)reinterpret_cast<const uint32_t*>(meta + 512)[0];
      const uint32_t flags = reinterpret_cast<const uint32_t*>(meta + 512)[1];
      if (fail(&bars[B_A_FULL], (uint32_t)(p & 1))) break;
      if (p >= 1 && fail(&bars[B_A_FREE], (uint32_t)((p - 1) & 1))) break;
      tc_fence_after();
      // row t of A (this lane's half): s > t masked, bf16 tiles [t][s]
      {
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
          float xg[32];
          tmem_ld32(tmem + tl + kColA + 32 * g, xg);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (32 * g + j > t) xg[j] = 0.f;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t hv[4], lv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              split2(xg[8 * q8 + 2 * e], xg[8 * q8 + 2 * e + 1], hv[e], lv[e]);
            const uint32_t off = sw128_offset((uint32_t)t, (uint32_t)(32 * g + 8 * q8));
            *reinterpret_cast<uint4*>(a_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            if (top) *reinterpret_cast<uint4*>(a_lo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_A_READY]);

      if (flags & PF_LAST_OF_CHUNK) {
        if (fail(&bars[B_O_FULL + (c & 1)], (uint32_t)((c >> 1) & 1))) break;
        tc_fence_after();
        // every reader of this chunk's V tile is done: copy the next one
        if (warp == 8 && lane == 0 && c + 1 < nchunks && c + 1 != debug_skip_v) {
          mbar_expect_tx(&bars[B_V_FULL], 16384);
          tma_load_4d(sm + KP::OFF_V, &mv, &bars[B_V_FULL], 0, h, kKC * (c + 1), b);
          tma_load_4d(sm + KP::OFF_V + 8192, &mv, &bars[B_V_FULL], 64, h, kKC * (c + 1), b);
          v_last = c + 1;
          if (c + 2 < nchunks) {
            tma_load_4d_prefetch(&mv, 0, h, kKC * (c + 2), b);
            tma_load_4d_prefetch(&mv, 64, h, kKC * (c + 2), b);
          }
        }
        const int n = min(kKC, T - kKC * c);
        const uint32_t ocol = kColO + 64u * (uint32_t)(c & 1);
        const size_t ostride = (size_t)H * 128;  // floats from one token to the next
        float* dst = O + tok_index(kKC * c) * 128 + L;
        float xo[2][32];
        tmem_ld32(tmem + tl + ocol, xo[0]);
        tmem_ld32(tmem + tl + ocol + 32, xo[1]);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          float* d = dst + (size_t)(32 * g) * ostride;
          if (n == kKC) {
#pragma unroll
            for (int j = 0; j < 32; ++j) __stcs(d + (size_t)j * ostride, xo[g][j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (32 * g + j < n) __stcs(d + (size_t)j * ostride, xo[g][j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_O_EMPTY + (c & 1)]);
      }
      if (flags & PF_LAST) break;
    }
    // after a timeout, no V copy may land once the CTA has ended
    if (warp == 8 && lane == 0 && *abort_flag) mbar_wait(&bars[B_V_FULL], (uint32_t)(v_last & 1));
  } else if (warp == 13) {
    // ============================================================ loader
    int issued = 0;
    for (int qi = 0; qi < nquarters; ++qi) {
      const int s2 = qi % kKStages;
      if (qi >= kKStages &&
          fail(&bars[B_STG_EMPTY + s2], (uint32_t)(((qi / kKStages) - 1) & 1)))
        break;
      uint8_t* st2 = sm + KP::OFF_STG + s2 * KP::STG;
      if (lane == 0) {
        mbar_expect_tx(&bars[B_STG + s2], KP::STG_TX);
        tma_load_4d(st2 + KP::STG_Q, &mq, &bars[B_STG + s2], 0, h, kKQ * qi, b);
        tma_load_4d(st2 + KP::STG_K, &mk, &bars[B_STG + s2], 0, h, kKQ * qi, b);
        tma_load_4d(st2 + KP::STG_W, &mw, &bars[B_STG + s2], 0, h, kKQ * qi, b);
        if (qi + 4 < nquarters) {
          tma_load_4d_prefetch(&mq, 0, h, kKQ * (qi + 4), b);
          tma_load_4d_prefetch(&mk, 0, h, kKQ * (qi + 4), b);
          tma_load_4d_prefetch(&mw, 0, h, kKQ * (qi + 4), b);
        }
      }
      ++issued;
      // a^2, a r and r of the quarter's tokens (lanes 0-15 load a, 16-31 r)
      const int t = kKQ * qi + (lane & 15);
      const float val = t < T ? (lane < 16 ? A_in : R_in)[tok_index(t)] : 0.f;
      const float a = __shfl_sync(0xffffffffu, val, lane & 15);
      const float r = __shfl_sync(0xffffffffu, val, 16 + (lane & 15));
      float* arq = reinterpret_cast<float*>(st2 + KP::STG_AR);
      if (lane < 16) {
        arq[lane] = a * a;
        arq[16 + lane] = a * r;
      } else {
        arq[16 + lane] = r;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_STG + s2]);
    }
    // no stage copy may land after the CTA ends (after a timeout the prep may
    // not have consumed the last ones)
    if (lane == 0 && *abort_flag) {
      for (int q2 = max(0, issued - kKStages); q2 < issued; ++q2)
        mbar_wait(&bars[B_STG + q2 % kKStages], (uint32_t)((q2 / kKStages) & 1));
    }
  } else if (lane == 0) {
    // ============================================================ issuer
    constexpr uint32_t ID_A = umma_idesc(128, 64, 1, 0, 0);   // Qs x U~^T
    constexpr uint32_t ID_O = umma_idesc(128, 64, 1, 0, 0);   // S (TMEM) x Q~^T
    constexpr uint32_t ID_DS = umma_idesc(128, 128, 1, 1, 1); // V^T x U~, both MN-major
    constexpr uint32_t ID_I = umma_idesc(128, 64, 1, 1, 0);   // V^T x A^T, A MN-major
    bool issued = false;
    for (int p = 0;; ++p) {
      const int set = p & 1;
      if (fail(&bars[B_OP_FULL + set], (uint32_t)((p >> 1) & 1))) break;
      const uint8_t* meta = sm + KP::OFF_META + (uint32_t)(p & 3) * KP::META;
      const int c = (int)reinterpret_cast<const uint32_t*>(meta + 512)[0];
      const uint32_t flags = reinterpret_cast<const uint32_t*>(meta + 512)[1];
      if (flags & PF_FIRST) {
        if (c >= 2 && fail(&bars[B_O_EMPTY + (c & 1)], (uint32_t)(((c >> 1) - 1) & 1))) break;
        if (fail(&bars[B_V_FULL], (uint32_t)(c & 1))) break;
      }
      tc_fence_after();
      const uint32_t qs = sbase + KP::OFF_SET + (uint32_t)set * KP::SET + KP::QS;
      const uint32_t uh = sbase + KP::OFF_SET + (uint32_t)set * KP::SET + KP::UH;
      const uint32_t ul = sbase + KP::OFF_SET + (uint32_t)set * KP::SET + KP::UL;
      const uint32_t vt = sbase + KP::OFF_V;
      // MMA-A: D_A = Qs U~hi^T + Qs U~lo^T (K = i: 8 steps of 16, halves 16 KB / 8 KB apart)
#pragma unroll
      for (int term = 0; term < 2; ++term)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ko = (uint32_t)(ks & 3) * 32u;
          umma_bf16(tmem + kColA,
                    umma_desc_sw128(qs + (uint32_t)(ks >> 2) * 16384u + ko, 16, 1024),
                    umma_desc_sw128((term ? ul : uh) + (uint32_t)(ks >> 2) * 8192u + ko, 16, 1024),
                    ID_A, (term > 0 || ks > 0) ? 1u : 0u);
        }
      umma_commit(&bars[B_A_FULL]);
      issued = true;
      if (p >= 1 && fail(&bars[B_S_READY], (uint32_t)((p - 1) & 1))) break;
      tc_fence_after();
      // MMA-O: D_o (+)= S hi Q~hi^T + S lo Q~hi^T + S hi Q~lo^T
      const uint32_t ocol = kColO + 64u * (uint32_t)(c & 1);
#pragma unroll
      for (int term = 0; term < 3; ++term)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t bq = qs + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u +
                              (term == 2 ? 8192u : 0u);
          umma_bf16_ts(tmem + ocol, tmem + kColSP + (term == 1 ? 64u : 0u) + 8u * ks,
                       umma_desc_sw128(bq, 16, 1024), ID_O,
                       ((flags & PF_FIRST) && term == 0 && ks == 0) ? 0u : 1u);
        }
      // MMA-dS: S += V^T U~hi + V^T U~lo (K = s: 4 steps of 16 rows, 2048 B)
#pragma unroll
      for (int term = 0; term < 2; ++term)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_bf16(tmem + kColS, umma_desc_sw128(vt + 2048u * ks, 8192, 1024),
                    umma_desc_sw128((term ? ul : uh) + 2048u * ks, 8192, 1024), ID_DS, 1u);
      umma_commit(&bars[B_DS_DONE]);
      umma_commit(&bars[B_OP_EMPTY + set]);
      if (fail(&bars[B_A_READY], (uint32_t)(p & 1))) break;
      tc_fence_after();
      // MMA-I: D_o += V^T (A top hi + A top lo + A bottom hi)^T (K = s: 4 steps of 32 B)
#pragma unroll
      for (int term = 0; term < 3; ++term)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_bf16(tmem + ocol, umma_desc_sw128(vt + 2048u * ks, 8192, 1024),
                    umma_desc_sw128(sbase + KP::OFF_A + (uint32_t)term * KP::A_TILE + 32u * ks,
                                    16, 1024),
                    ID_I, 1u);
      umma_commit(&bars[B_A_FREE]);
      if (flags & PF_LAST_OF_CHUNK) umma_commit(&bars[B_O_FULL + (c & 1)]);
      if (flags & PF_LAST) break;
    }
    // nothing of this CTA's may be in flight on the tensor pipe when TMEM is freed
    if (issued) {
      umma_commit(&bars[B_FINAL]);
      mbar_wait(&bars[B_FINAL], 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 kla_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// [B, T, H, 128] tensor of 2- or 4-byte elements, boxes of (box_d, 1 head,
// box_t tokens, 1 batch); tokens past T read as zeros.
bool kla_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int B, int T,
             int H, int box_d, int box_t, bool swizzle) {
  auto enc = kla_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {128u, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {128u * (cuuint64_t)esize, (cuuint64_t)H * 128u * esize,
                           (cuuint64_t)T * H * 128u * esize};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1u, (cuuint32_t)box_t, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool kla_engine_supported(kdn_dtype dt, int dk, int dv, int T) {
  return dt == KDN_BF16 && dk == 128 && dv == 128 && T >= 1;
}

kdn_status kla_engine_launch(const void* q, const void* k, const void* v, const float* a,
                             const float* w, const float* r, const float* S0, const float* L0,
                             float* o, float* S_out, float* L_out, int B, int T, int H, void* ws,
                             cudaStream_t s, int debug_skip_v) {
  CUtensorMap mq, mk, mw, mv;
  if (!kla_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, T, H, 128, kKQ, false) ||
      !kla_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, T, H, 128, kKQ, false) ||
      !kla_map(&mw, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, H, 128, kKQ, false) ||
      !kla_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, T, H, 64, kKC, true))
    return KDN_ERR_CUDA;
  static bool smem_set = false;
  if (!smem_set) {
    if (cudaFuncSetAttribute(kla_engine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)KP::SMEM) != cudaSuccess)
      return KDN_ERR_CUDA;
    smem_set = true;
  }
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return KDN_ERR_CUDA;
  kla_engine_kernel<<<(unsigned)(B * H), kKThreads, KP::SMEM, s>>>(
      mq, mk, mw, mv, a, r, static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k), w, S0, L0, o, S_out, L_out, T, H,
      static_cast<uint32_t*>(ws), debug_skip_v);
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

}  // namespace kdn
