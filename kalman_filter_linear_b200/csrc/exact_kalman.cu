// Dense (full-covariance) Kalman filter of the KDN memory model, token by token.
//
// The KDN layer carries a projected covariance: one variance per head
// (isotropic) or per key dimension (diagonal).  The exact filter of the same
// linear-Gaussian model keeps the full d_k x d_k covariance P instead and runs
// the Riccati recursion, which the paper's projection exists to avoid ("Kalman
// Delta Networks: Uncertainty-aware Associative Memory", abstract: exact
// tracking needs the dense, state-dependent recursion; "Kalman Delta Networks:
// 不确定性感知的联想记忆", 局限: the projection's approximation error).
// Per token, with S (d_v x d_k) the memory and rows of S sharing P:
//   P- = a^2 P + W            W = w I (isotropic) or diag(w) (diagonal)
//   u  = P- k,  s = k.u + r,  g = u / s
//   e  = v - a S k,  S <- a S + e g^T,  o = S q = a S q + e (g.q)
//   P  = P- - u u^T / s
// It is the reference for the projection's approximation error at small d_k.
//
// One CTA of 8 warps per (b, h).  Warp w holds rows w, w + 8, ... of S and of
// P in registers; lane l holds columns [l CPL, (l + 1) CPL), CPL = d_k / 32.
//  - u = P- k is formed as column sums (P- is symmetric): each warp sums its
//    own rows and the 8 partial vectors meet in shared memory, the one block
//    barrier per token.
//  - P stays exactly symmetric: P-_ij and P-_ji are computed from the same
//    operands, and so are u_i u_j and u_j u_i; s is the same in every warp.
//  - The row sums S k and S q of a warp's rows are reduced across the lanes
//    by recursive halving (each exchange step halves the values a lane keeps),
//    2 RPW values in about 2 RPW shuffles rather than 5 per value.
//  - Inputs come into shared memory by cp.async in chunks of 16 tokens, one
//    chunk ahead of the compute; outputs leave per chunk in coalesced rows.
#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kXWarps = 8, kXThreads = kXWarps * 32, kTC = 16;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_newest_pending() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// One recursive-halving step at lane offset O over n values: a lane with bit
// O set keeps the upper half, its partner the lower half; each adds what the
// partner sends.
template <int N, int O>
__device__ __forceinline__ void halve(float* x, int lane) {
  const bool up = (lane & O) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? x[i] : x[i + N / 2];
    const float keep = up ? x[i + N / 2] : x[i];
    x[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}

// Sums item i of x[N] over the 32 lanes; afterwards every lane l holds the
// total of item l / (32 / N).  N in {8, 16, 32}.
template <int N>
__device__ __forceinline__ float transpose_sum(float (&x)[N], int lane) {
  static_assert(N == 8 || N == 16 || N == 32, "items per lane");
  halve<N, 16>(x, lane);
  halve<N / 2, 8>(x, lane);
  halve<N / 4, 4>(x, lane);
  if constexpr (N >= 16) halve<N / 8, 2>(x, lane);
  if constexpr (N >= 32) halve<N / 16, 1>(x, lane);
  float y = x[0];
  if constexpr (N <= 16) y += __shfl_xor_sync(0xffffffffu, y, 1);
  if constexpr (N <= 8) y += __shfl_xor_sync(0xffffffffu, y, 2);
  return y;
}

// Shared-memory plan of one CTA (bytes): two input stages, the partial sums
// of u (two buffers, by token parity) and the output rows of one chunk.
template <int DK, int RPW, bool DIAG, typename InT>
struct XPlan {
  static constexpr int DVP = RPW * kXWarps;                 // d_v rounded up
  static constexpr int KQ = kTC * 2 * DK * (int)sizeof(InT);  // [t][k | q]
  static constexpr int VB = kTC * DVP * (int)sizeof(InT);     // [t][v]
  static constexpr int WN = DIAG ? DK : 1;
  static constexpr int F32 = kTC * (2 + WN) * 4;              // a[t], r[t], w[t][WN]
  static constexpr int STAGE = (KQ + VB + F32 + 15) / 16 * 16;
  static constexpr int OFF_RED = 2 * STAGE;
  static constexpr int OFF_OUT = OFF_RED + 2 * kXWarps * DK * 4;
  static constexpr int TOTAL = OFF_OUT + kTC * DVP * 4;
};

template <int DK, int RPW, bool DIAG, typename InT>
__global__ void __launch_bounds__(kXThreads)
exact_kalman_kernel(const InT* __restrict__ Q, const InT* __restrict__ K,
                    const InT* __restrict__ V, const float* __restrict__ A,
                    const float* __restrict__ Wn, const float* __restrict__ R, const float* S0,
                    const float* P0, float* __restrict__ O, float* S_out, float* P_out, int T,
                    int H, int dv) {
  using X = XPlan<DK, RPW, DIAG, InT>;
  constexpr int CPL = DK / 32;   // columns per lane
  static_assert(CPL == 1 || CPL == 2, "d_k 32 or 64");
  constexpr int PR = DK / kXWarps;  // rows of P per warp
  constexpr int N = 2 * RPW;     // row sums per warp and token: S k, then S q
  constexpr int G = 32 / N;      // lanes that share one row sum
  extern __shared__ __align__(16) uint8_t xsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  float* red = reinterpret_cast<float*>(xsm + X::OFF_RED);  // [2][8][DK]
  float* obuf = reinterpret_cast<float*>(xsm + X::OFF_OUT);  // [kTC][DVP]

  // stage the inputs of tokens [16 c, 16 c + 16) into buffer c & 1
  auto issue = [&](int c) {
    uint8_t* st = xsm + (c & 1) * X::STAGE;
    InT* skq = reinterpret_cast<InT*>(st);
    InT* sv = reinterpret_cast<InT*>(st + X::KQ);
    float* sf = reinterpret_cast<float*>(st + X::KQ + X::VB);
    const int t0 = c * kTC, nt = min(kTC, T - t0);
    constexpr int PK = DK * (int)sizeof(InT) / 16;  // 16-byte pieces of one k row
    for (int i = tid; i < nt * 2 * PK; i += kXThreads) {
      const int t = i / (2 * PK), p = i % (2 * PK), half = p / PK, pp = p % PK;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      const InT* src = (half ? Q : K) + tok * DK;
      cp_async16(skq + (t * 2 + half) * DK + pp * (16 / (int)sizeof(InT)),
                 reinterpret_cast<const uint8_t*>(src) + pp * 16);
    }
    const int pv = dv * (int)sizeof(InT) / 16;
    for (int i = tid; i < nt * pv; i += kXThreads) {
      const int t = i / pv, pp = i % pv;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      cp_async16(sv + t * X::DVP + pp * (16 / (int)sizeof(InT)),
                 reinterpret_cast<const uint8_t*>(V + tok * dv) + pp * 16);
    }
    if constexpr (DIAG) {
      constexpr int PW = DK * 4 / 16;
      for (int i = tid; i < nt * PW; i += kXThreads) {
        const int t = i / PW, pp = i % PW;
        const size_t tok = ((size_t)b * T + t0 + t) * H + h;
        cp_async16(sf + 2 * kTC + t * DK + pp * 4, Wn + tok * DK + pp * 4);
      }
    }
    if (tid < 3 * nt) {
      const int which = tid / nt, t = tid % nt;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      if (which == 0) cp_async4(sf + t, A + tok);
      else if (which == 1) cp_async4(sf + kTC + t, R + tok);
      else if (!DIAG) cp_async4(sf + 2 * kTC + t, Wn + tok);
    }
  };

  // ---- state into registers.  S_out may alias S0 and P_out P0: every read
  // of the initial state comes before the barrier that precedes the stores.
  float S[RPW][CPL], P[PR][CPL];
  const size_t s_base = (size_t)bh * dv * DK, p_base = (size_t)bh * DK * DK;
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int j = warp + kXWarps * i;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      S[i][c] = (S0 && j < dv) ? S0[s_base + (size_t)j * DK + lane * CPL + c] : 0.f;
  }
#pragma unroll
  for (int m = 0; m < PR; ++m) {
    const int i = warp + kXWarps * m;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int j = lane * CPL + c;
      // the symmetric part of P0: the same value at (i, j) and (j, i)
      P[m][c] = P0 ? 0.5f * (P0[p_base + (size_t)i * DK + j] + P0[p_base + (size_t)j * DK + i])
                   : (i == j ? 1.f : 0.f);
    }
  }

  const int nchunks = (T + kTC - 1) / kTC;
  if (nchunks > 0) issue(0);
  cp_async_commit();
  for (int ch = 0; ch < nchunks; ++ch) {
    if (ch + 1 < nchunks) issue(ch + 1);  // its buffer was released by the barrier below
    cp_async_commit();
    cp_async_wait_newest_pending();       // chunk ch has landed (this thread's copies)
    __syncthreads();                      // ... and everyone's
    const uint8_t* st = xsm + (ch & 1) * X::STAGE;
    const InT* skq = reinterpret_cast<const InT*>(st);
    const InT* sv = reinterpret_cast<const InT*>(st + X::KQ);
    const float* sf = reinterpret_cast<const float*>(st + X::KQ + X::VB);
    const int t0 = ch * kTC, nt = min(kTC, T - t0);
    for (int t = 0; t < nt; ++t) {
      const InT* kq = skq + t * 2 * DK;
      float k[CPL], q[CPL], krow[PR];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        k[c] = to_f32(kq[lane * CPL + c]);
        q[c] = to_f32(kq[DK + lane * CPL + c]);
      }
#pragma unroll
      for (int m = 0; m < PR; ++m) krow[m] = to_f32(kq[warp + kXWarps * m]);
      const float a = sf[t], r = sf[kTC + t], aa = a * a;

      // P- = a^2 P + W, and this warp's share of u = P- k (column sums)
      float Pm[PR][CPL], part[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) part[c] = 0.f;
#pragma unroll
      for (int m = 0; m < PR; ++m) {
        const int i = warp + kXWarps * m;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const int j = lane * CPL + c;
          const float wij = i == j ? (DIAG ? sf[2 * kTC + t * DK + i] : sf[2 * kTC + t]) : 0.f;
          Pm[m][c] = __fmaf_rn(aa, P[m][c], wij);
          part[c] = __fmaf_rn(Pm[m][c], krow[m], part[c]);
        }
      }
      float* rd = red + (t & 1) * kXWarps * DK;
#pragma unroll
      for (int c = 0; c < CPL; ++c) rd[warp * DK + lane * CPL + c] = part[c];
      __syncthreads();
      float u[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < kXWarps; ++w) x += rd[w * DK + lane * CPL + c];
        u[c] = x;
      }
      float ku = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) ku = __fmaf_rn(k[c], u[c], ku);
      const float s = warp_sum(ku) + r;
      const float inv_s = 1.f / s;
      float g[CPL], gq = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        g[c] = u[c] * inv_s;
        gq = __fmaf_rn(g[c], q[c], gq);
      }
      gq = warp_sum(gq);

      // P = P- - u u^T / s; u_i of this warp's rows comes from the lane that owns column i
#pragma unroll
      for (int m = 0; m < PR; ++m) {
        const int i = warp + kXWarps * m;
        const float own = CPL == 1 ? u[0] : ((i & 1) ? u[CPL - 1] : u[0]);  // CPL <= 2
        const float ui = __shfl_sync(0xffffffffu, own, i / CPL);
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          P[m][c] = __fmaf_rn(-__fmul_rn(ui, u[c]), inv_s, Pm[m][c]);
      }

      // e = v - a S k and o = a S q + e (g.q) for this warp's rows
      float x[N];
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          sk = __fmaf_rn(S[i][c], k[c], sk);
          sq = __fmaf_rn(S[i][c], q[c], sq);
        }
        x[i] = sk;
        x[RPW + i] = sq;
      }
      const float tot = transpose_sum<N>(x, lane);
      const int item = lane / G;
      float e = 0.f;
      if (item < RPW) {
        const int j = warp + kXWarps * item;
        e = (j < dv ? to_f32(sv[t * X::DVP + j]) : 0.f) - a * tot;
      }
      // lanes of item RPW + i take e_i from the first lane of item i
      const float ei = __shfl_sync(0xffffffffu, e, (item - RPW) * G & 31);
      if (item >= RPW && lane % G == 0) {
        const int j = warp + kXWarps * (item - RPW);
        obuf[t * X::DVP + j] = __fmaf_rn(ei, gq, a * tot);
      }
#pragma unroll
      for (int i = 0; i < RPW; ++i) {
        const float e_i = __shfl_sync(0xffffffffu, e, i * G);
#pragma unroll
        for (int c = 0; c < CPL; ++c) S[i][c] = __fmaf_rn(e_i, g[c], a * S[i][c]);
      }
    }
    __syncthreads();  // obuf complete; stage ch & 1 free for chunk ch + 2
    for (int i = tid; i < nt * dv; i += kXThreads) {
      const int t = i / dv, j = i % dv;
      O[(((size_t)b * T + t0 + t) * H + h) * dv + j] = obuf[t * X::DVP + j];
    }
  }
  __syncthreads();  // every read of S0 / P0 is done before the stores

  // ---- state out
#pragma unroll
  for (int i = 0; i < RPW; ++i) {
    const int j = warp + kXWarps * i;
    if (j < dv) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) S_out[s_base + (size_t)j * DK + lane * CPL + c] = S[i][c];
    }
  }
#pragma unroll
  for (int m = 0; m < PR; ++m) {
    const int i = warp + kXWarps * m;
#pragma unroll
    for (int c = 0; c < CPL; ++c) P_out[p_base + (size_t)i * DK + lane * CPL + c] = P[m][c];
  }
}

template <int DK, int RPW, bool DIAG, typename InT>
kdn_status launch_x(const void* q, const void* k, const void* v, const float* a, const float* w,
                    const float* r, const float* S0, const float* P0, float* o, float* S_out,
                    float* P_out, int B, int T, int H, int dv, cudaStream_t s) {
  using X = XPlan<DK, RPW, DIAG, InT>;
  auto kern = exact_kalman_kernel<DK, RPW, DIAG, InT>;
  if (X::TOTAL > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, X::TOTAL) !=
          cudaSuccess)
    return KDN_ERR_CUDA;
  kern<<<(unsigned)(B * H), kXThreads, X::TOTAL, s>>>(
      static_cast<const InT*>(q), static_cast<const InT*>(k), static_cast<const InT*>(v), a, w, r,
      S0, P0, o, S_out, P_out, T, H, dv);
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

template <int DK, bool DIAG, typename InT>
kdn_status launch_dv(const void* q, const void* k, const void* v, const float* a, const float* w,
                     const float* r, const float* S0, const float* P0, float* o, float* S_out,
                     float* P_out, int B, int T, int H, int dv, cudaStream_t s) {
  if (dv <= 32)
    return launch_x<DK, 4, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  if (dv <= 64)
    return launch_x<DK, 8, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  return launch_x<DK, 16, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
}

template <bool DIAG, typename InT>
kdn_status launch_dk(const void* q, const void* k, const void* v, const float* a, const float* w,
                     const float* r, const float* S0, const float* P0, float* o, float* S_out,
                     float* P_out, int B, int T, int H, int dk, int dv, cudaStream_t s) {
  if (dk == 32)
    return launch_dv<32, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  return launch_dv<64, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
}

}  // namespace

bool exact_kalman_supported(int dk, int dv) {
  return (dk == 32 || dk == 64) && dv >= 8 && dv <= 128 && dv % 8 == 0;
}

kdn_status exact_kalman_launch(bool diag, kdn_dtype dt, const void* q, const void* k,
                               const void* v, const float* a, const float* w, const float* r,
                               const float* S0, const float* P0, float* o, float* S_out,
                               float* P_out, int B, int T, int H, int dk, int dv,
                               cudaStream_t s) {
  if (diag)
    return dt == KDN_BF16
               ? launch_dk<true, __nv_bfloat16>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dk, dv, s)
               : launch_dk<true, float>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dk, dv, s);
  return dt == KDN_BF16
             ? launch_dk<false, __nv_bfloat16>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dk, dv, s)
             : launch_dk<false, float>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dk, dv, s);
}

}  // namespace kdn
