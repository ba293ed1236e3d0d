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
// One CTA per (b, h).  Every matrix row is held by SPLIT = d_k / 32 adjacent
// lanes, 32 columns each, so the per-row products run inside the lanes and
// one xor shuffle joins the halves.  The covariance recursion does not read
// S, so it runs on its own warps, one 16-token chunk ahead of the state:
//  - Covariance warps (d_k SPLIT / 32 of them): half h of row i holds
//    Pr[c'] = P[i][(i + SPLIT c' + h) mod d_k], the row rotated by i, so the
//    diagonal that W touches is always register 0 of half 0.
//    u_i = sum_c P-[i][i + c] k[i + c] reads k rotated from shared memory,
//    where k is stored twice in a row so that the reads of a lane are fixed
//    offsets from one address (distinct lanes, distinct banks).  k.u and q.u
//    are reduced across the lanes and warps, g = u / s and g.q = q.u / s go
//    to shared memory for the state warps, and P is updated with u read
//    rotated the same way.  P stays exactly symmetric: entry (i, j) and
//    (j, i) are formed from the same operands in the same order.
//  - State warps: half h of row j holds S[j][32 h + c'].  S k and S q are
//    in-lane dot products with k and q read as broadcasts; the update
//    S_j <- a S_j + e_j g likewise.
//  - Both roles run their per-element arithmetic on column pairs with the
//    packed FP32 instructions (two FMAs per instruction).
//  - Inputs come into shared memory by cp.async in chunks of 16 tokens, three
//    stages deep; outputs leave per chunk in coalesced rows.
#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kTC = 16;  // tokens per chunk

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

// barrier of the covariance warps only (named barrier 1)
template <int NT>
__device__ __forceinline__ void pbar() {
  if constexpr (NT == 32) {
    __syncwarp();
  } else {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
  }
}

// Shared-memory plan of one CTA (bytes).
template <int DK, int SW, bool DIAG, typename InT>
struct XPlan {
  static constexpr int SPLIT = DK / 32;                       // lanes per row
  static constexpr int PW = DK * SPLIT / 32;                  // covariance warps
  static constexpr int DVP = SW * 32 / SPLIT;                 // d_v rounded up
  static constexpr int KQ = kTC * 2 * DK * (int)sizeof(InT);  // [t][k | q] as read
  static constexpr int VB = kTC * DVP * (int)sizeof(InT);     // [t][v]
  static constexpr int WN = DIAG ? DK : 1;
  static constexpr int F32 = kTC * (2 + WN) * 4;              // a[t], r[t], w[t][WN]
  static constexpr int STAGE = (KQ + VB + F32 + 15) / 16 * 16;
  static constexpr int OFF_KQF = 3 * STAGE;                   // [2][kTC][k | q] fp32
  static constexpr int OFF_G = OFF_KQF + 2 * kTC * 2 * DK * 4;  // [2][kTC][DK] gains
  static constexpr int OFF_KD = OFF_G + 2 * kTC * DK * 4;       // [kTC][2 DK] k, k again
  static constexpr int OFF_U = OFF_KD + kTC * 2 * DK * 4;       // [2][2 DK] u, u again, by parity
  static constexpr int OFF_GQ = OFF_U + 2 * 2 * DK * 4;         // [2][kTC] g.q
  static constexpr int OFF_RED = OFF_GQ + 2 * kTC * 4;          // [2][PW][2] k.u, q.u
  static constexpr int OFF_OUT = (OFF_RED + 2 * PW * 2 * 4 + 15) / 16 * 16;  // [2][kTC][DVP]
  static constexpr int TOTAL = OFF_OUT + 2 * kTC * DVP * 4;
};

template <int DK, int SW, bool DIAG, typename InT>
__global__ void __launch_bounds__((DK * DK / 1024 + SW) * 32)
exact_kalman_kernel(const InT* __restrict__ Q, const InT* __restrict__ K,
                    const InT* __restrict__ V, const float* __restrict__ A,
                    const float* __restrict__ Wn, const float* __restrict__ R, const float* S0,
                    const float* P0, float* __restrict__ O, float* S_out, float* P_out, int T,
                    int H, int dv) {
  using X = XPlan<DK, SW, DIAG, InT>;
  constexpr int PW = X::PW, SPLIT = X::SPLIT, NTH = (PW + SW) * 32, M = DK - 1;
  extern __shared__ __align__(16) uint8_t xsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool pwarp = warp < PW;
  const int rt = pwarp ? tid : tid - PW * 32;
  const int row = rt / SPLIT, hf = rt % SPLIT;  // row of P or S, and which half of it
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  float* kqf = reinterpret_cast<float*>(xsm + X::OFF_KQF);
  float* gring = reinterpret_cast<float*>(xsm + X::OFF_G);
  float* ubuf = reinterpret_cast<float*>(xsm + X::OFF_U);
  float* kdup = reinterpret_cast<float*>(xsm + X::OFF_KD);
  float* gqring = reinterpret_cast<float*>(xsm + X::OFF_GQ);
  float* red = reinterpret_cast<float*>(xsm + X::OFF_RED);
  float* obuf = reinterpret_cast<float*>(xsm + X::OFF_OUT);

  struct Stage {
    const InT* kq;
    const InT* v;
    const float* f;
  };
  auto stage = [&](int c) {
    const uint8_t* st = xsm + (c % 3) * X::STAGE;
    return Stage{reinterpret_cast<const InT*>(st), reinterpret_cast<const InT*>(st + X::KQ),
                 reinterpret_cast<const float*>(st + X::KQ + X::VB)};
  };
  // stage the inputs of tokens [16 c, 16 c + 16) into buffer c % 3
  auto issue = [&](int c) {
    uint8_t* st = xsm + (c % 3) * X::STAGE;
    InT* skq = reinterpret_cast<InT*>(st);
    InT* sv = reinterpret_cast<InT*>(st + X::KQ);
    float* sf = reinterpret_cast<float*>(st + X::KQ + X::VB);
    const int t0 = c * kTC, nt = min(kTC, T - t0);
    constexpr int PK = DK * (int)sizeof(InT) / 16;  // 16-byte pieces of one k row
    for (int i = tid; i < nt * 2 * PK; i += NTH) {
      const int t = i / (2 * PK), p = i % (2 * PK), half = p / PK, pp = p % PK;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      const InT* src = (half ? Q : K) + tok * DK;
      cp_async16(skq + (t * 2 + half) * DK + pp * (16 / (int)sizeof(InT)),
                 reinterpret_cast<const uint8_t*>(src) + pp * 16);
    }
    const int pv = dv * (int)sizeof(InT) / 16;
    for (int i = tid; i < nt * pv; i += NTH) {
      const int t = i / pv, pp = i % pv;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      cp_async16(sv + t * X::DVP + pp * (16 / (int)sizeof(InT)),
                 reinterpret_cast<const uint8_t*>(V + tok * dv) + pp * 16);
    }
    if constexpr (DIAG) {
      constexpr int PWN = DK * 4 / 16;
      for (int i = tid; i < nt * PWN; i += NTH) {
        const int t = i / PWN, pp = i % PWN;
        const size_t tok = ((size_t)b * T + t0 + t) * H + h;
        cp_async16(sf + 2 * kTC + t * DK + pp * 4, Wn + tok * DK + pp * 4);
      }
    }
    for (int i = tid; i < 3 * nt; i += NTH) {
      const int which = i / nt, t = i % nt;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      if (which == 0) cp_async4(sf + t, A + tok);
      else if (which == 1) cp_async4(sf + kTC + t, R + tok);
      else if (!DIAG) cp_async4(sf + 2 * kTC + t, Wn + tok);
    }
  };

  // ---- state into registers.  S_out may alias S0 and P_out P0: every read
  // of the initial state comes before the barrier that precedes the stores.
  // covariance warps: Pr[c'] = P[row][(row + SPLIT c' + hf) mod DK];
  // state warps: S[row][32 hf + c']
  float X_[32];
  const size_t s_base = (size_t)bh * dv * DK, p_base = (size_t)bh * DK * DK;
  if (pwarp) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int j = (row + SPLIT * c + hf) & M;
      // the symmetric part of P0: the same value at (i, j) and (j, i)
      X_[c] = P0 ? 0.5f * (P0[p_base + (size_t)row * DK + j] + P0[p_base + (size_t)j * DK + row])
                 : (c == 0 && hf == 0 ? 1.f : 0.f);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (S0 && row < dv)
        x = *reinterpret_cast<const float4*>(S0 + s_base + (size_t)row * DK + 32 * hf + c);
      X_[c] = x.x;
      X_[c + 1] = x.y;
      X_[c + 2] = x.z;
      X_[c + 3] = x.w;
    }
  }

  // The covariance warps turn chunk cc's inputs into its gains and g.q, and
  // leave k and q of the chunk in fp32 for the state warps.
  auto gains = [&](int cc) {
    const Stage st = stage(cc);
    const int nt = min(kTC, T - cc * kTC);
    float* kf = kqf + (cc & 1) * kTC * 2 * DK;
    float* gout = gring + (cc & 1) * kTC * DK;
    // k and q of the chunk in fp32 for the state warps, and k written twice
    // in a row for the rotated reads here (no index wraps around)
    for (int i = rt; i < nt * 2 * DK; i += PW * 32) {
      const float x = to_f32(st.kq[i]);
      kf[i] = x;
      if ((i & (2 * DK - 1)) < DK) {
        const int t = i / (2 * DK), j = i & M;
        kdup[t * 2 * DK + j] = x;
        kdup[t * 2 * DK + DK + j] = x;
      }
    }
    pbar<PW * 32>();
    for (int t = 0; t < nt; ++t) {
      const float* kt = kf + t * 2 * DK;  // k, then q
      const float ki = kt[row], qi = kt[DK + row];
      const float* krot = kdup + t * 2 * DK + row + hf;  // krot[SPLIT c] = k[(row + SPLIT c + hf) mod DK]
      const float aa = st.f[t] * st.f[t], r = st.f[kTC + t];
      const float wd = hf == 0 ? (DIAG ? st.f[2 * kTC + t * DK + row] : st.f[2 * kTC + t]) : 0.f;
      float* ub = ubuf + (t & 1) * 2 * DK;
      const float* urot = ub + row + hf;  // urot[SPLIT c] = u[(row + SPLIT c + hf) mod DK]
      // P- = a^2 P + W (W on the diagonal: register 0 of half 0) and
      // u_i = (P- k)_i; P- is formed again, identically, in the update
      // (column pairs on the packed FP32 pipe; each element rounds as a scalar
      // operation would, so (i, j) and (j, i) still agree bit for bit)
      const float2 aa2 = make_float2(aa, aa);
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float2 pm = __ffma2_rn(aa2, make_float2(X_[c], X_[c + 1]),
                                     make_float2(c == 0 ? wd : 0.f, 0.f));
        acc[(c >> 1) & 1] = __ffma2_rn(pm, make_float2(krot[SPLIT * c], krot[SPLIT * (c + 1)]),
                                       acc[(c >> 1) & 1]);
      }
      float u = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
      if constexpr (SPLIT == 2) u += __shfl_xor_sync(0xffffffffu, u, 1);
      if (hf == 0) {
        ub[row] = u;
        ub[DK + row] = u;
      }
      // k.u and q.u, each row counted once (half 0)
      const float ku = warp_sum(hf == 0 ? ki * u : 0.f), qu = warp_sum(hf == 0 ? qi * u : 0.f);
      float* rd = red + (t & 1) * PW * 2;
      if (lane == 0) {
        rd[2 * warp] = ku;
        rd[2 * warp + 1] = qu;
      }
      pbar<PW * 32>();  // u and the partial sums visible
      float kus = 0.f, qus = 0.f;
#pragma unroll
      for (int w = 0; w < PW; ++w) {
        kus += rd[2 * w];
        qus += rd[2 * w + 1];
      }
      const float inv_s = __frcp_rn(kus + r);
      if (hf == 0) gout[t * DK + row] = u * inv_s;
      if (tid == 0) gqring[(cc & 1) * kTC + t] = qus * inv_s;
      // P = P- - u u^T / s
      const float2 nu = make_float2(-u, -u), is2 = make_float2(inv_s, inv_s);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float2 pm = __ffma2_rn(aa2, make_float2(X_[c], X_[c + 1]),
                                     make_float2(c == 0 ? wd : 0.f, 0.f));
        const float2 uu = __fmul2_rn(nu, make_float2(urot[SPLIT * c], urot[SPLIT * (c + 1)]));
        const float2 x = __ffma2_rn(uu, is2, pm);
        X_[c] = x.x;
        X_[c + 1] = x.y;
      }
      // (u and the partial sums are double-buffered by token parity: the
      // barrier of the next token orders this token's reads before their reuse)
    }
  };

  // The state warps run chunk cc's tokens through S with its gains.
  auto states = [&](int cc) {
    const Stage st = stage(cc);
    const int nt = min(kTC, T - cc * kTC);
    const float* kf = kqf + (cc & 1) * kTC * 2 * DK;
    const float* gin = gring + (cc & 1) * kTC * DK;
    float* ob = obuf + (cc & 1) * kTC * X::DVP;
    for (int t = 0; t < nt; ++t) {
      const float4* k4 = reinterpret_cast<const float4*>(kf + t * 2 * DK + 32 * hf);
      const float4* q4 = reinterpret_cast<const float4*>(kf + t * 2 * DK + DK + 32 * hf);
      float2 sk[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float2 sq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 kk = k4[c4], qq = q4[c4];
        const float2 x0 = make_float2(X_[4 * c4], X_[4 * c4 + 1]);
        const float2 x1 = make_float2(X_[4 * c4 + 2], X_[4 * c4 + 3]);
        sk[0] = __ffma2_rn(x0, make_float2(kk.x, kk.y), sk[0]);
        sk[1] = __ffma2_rn(x1, make_float2(kk.z, kk.w), sk[1]);
        sq[0] = __ffma2_rn(x0, make_float2(qq.x, qq.y), sq[0]);
        sq[1] = __ffma2_rn(x1, make_float2(qq.z, qq.w), sq[1]);
      }
      float skt = (sk[0].x + sk[1].x) + (sk[0].y + sk[1].y);
      float sqt = (sq[0].x + sq[1].x) + (sq[0].y + sq[1].y);
      if constexpr (SPLIT == 2) {
        skt += __shfl_xor_sync(0xffffffffu, skt, 1);
        sqt += __shfl_xor_sync(0xffffffffu, sqt, 1);
      }
      const float a = st.f[t], gq = gqring[(cc & 1) * kTC + t];
      const float vj = row < dv ? to_f32(st.v[t * X::DVP + row]) : 0.f;
      const float e = vj - a * skt;
      if (hf == 0) ob[t * X::DVP + row] = __fmaf_rn(e, gq, a * sqt);
      const float4* g4 = reinterpret_cast<const float4*>(gin + t * DK + 32 * hf);
      const float2 e2 = make_float2(e, e), a2 = make_float2(a, a);
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 gg = g4[c4];
        const float2 x0 = __ffma2_rn(e2, make_float2(gg.x, gg.y),
                                     __fmul2_rn(a2, make_float2(X_[4 * c4], X_[4 * c4 + 1])));
        const float2 x1 = __ffma2_rn(e2, make_float2(gg.z, gg.w),
                                     __fmul2_rn(a2, make_float2(X_[4 * c4 + 2], X_[4 * c4 + 3])));
        X_[4 * c4] = x0.x;
        X_[4 * c4 + 1] = x0.y;
        X_[4 * c4 + 2] = x1.x;
        X_[4 * c4 + 3] = x1.y;
      }
    }
  };

  // output rows of chunk cc, staged in obuf, go out coalesced
  auto flush = [&](int cc) {
    const int t0 = cc * kTC, nt = min(kTC, T - t0);
    const float* ob = obuf + (cc & 1) * kTC * X::DVP;
    for (int i = tid; i < nt * dv; i += NTH) {
      const int t = i / dv, j = i % dv;
      O[(((size_t)b * T + t0 + t) * H + h) * dv + j] = ob[t * X::DVP + j];
    }
  };

  // Phase c: the covariance warps compute the gains of chunk c + 1 while the
  // state warps run chunk c.  Inputs are three stages deep: chunk c + 2 is
  // copied during phase c into the stage chunk c - 1 used.
  const int nchunks = (T + kTC - 1) / kTC;
  issue(0);
  cp_async_commit();
  if (nchunks > 1) issue(1);
  cp_async_commit();
  cp_async_wait_newest_pending();  // chunk 0 landed (this thread's copies)
  __syncthreads();                 // ... and everyone's
  if (pwarp) gains(0);
  for (int c = 0; c < nchunks; ++c) {
    __syncthreads();  // phase c - 1 done: gains of chunk c written, chunk c - 1 read
    if (c > 0) flush(c - 1);
    if (c + 2 < nchunks) issue(c + 2);
    cp_async_commit();
    cp_async_wait_newest_pending();  // chunk c + 1 landed (this thread's copies)
    __syncthreads();                 // ... and everyone's
    if (pwarp) {
      if (c + 1 < nchunks) gains(c + 1);
    } else {
      states(c);
    }
  }
  __syncthreads();  // the last chunk's outputs; every read of S0 / P0 is done
  if (nchunks > 0) flush(nchunks - 1);

  // ---- state out
  if (pwarp) {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      P_out[p_base + (size_t)row * DK + ((row + SPLIT * c + hf) & M)] = X_[c];
  } else if (row < dv) {
#pragma unroll
    for (int c = 0; c < 32; c += 4)
      *reinterpret_cast<float4*>(S_out + s_base + (size_t)row * DK + 32 * hf + c) =
          make_float4(X_[c], X_[c + 1], X_[c + 2], X_[c + 3]);
  }
}

template <int DK, int SW, bool DIAG, typename InT>
kdn_status launch_x(const void* q, const void* k, const void* v, const float* a, const float* w,
                    const float* r, const float* S0, const float* P0, float* o, float* S_out,
                    float* P_out, int B, int T, int H, int dv, cudaStream_t s) {
  using X = XPlan<DK, SW, DIAG, InT>;
  auto kern = exact_kalman_kernel<DK, SW, DIAG, InT>;
  // the shared-memory opt-in is a property of the function: set it once per
  // instantiation (a race between first calls sets the same value twice)
  static bool smem_set = false;
  if (X::TOTAL > 48 * 1024 && !smem_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, X::TOTAL) !=
        cudaSuccess)
      return KDN_ERR_CUDA;
    smem_set = true;
  }
  kern<<<(unsigned)(B * H), (X::PW + SW) * 32, X::TOTAL, s>>>(
      static_cast<const InT*>(q), static_cast<const InT*>(k), static_cast<const InT*>(v), a, w, r,
      S0, P0, o, S_out, P_out, T, H, dv);
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

template <int DK, bool DIAG, typename InT>
kdn_status launch_dv(const void* q, const void* k, const void* v, const float* a, const float* w,
                     const float* r, const float* S0, const float* P0, float* o, float* S_out,
                     float* P_out, int B, int T, int H, int dv, cudaStream_t s) {
  // state warps: d_v rows of DK / 32 lanes each, rounded up to 1, 2, 4 or 8 warps
  const int need = (dv * (DK / 32) + 31) / 32;
  if (need <= 1)
    return launch_x<DK, 1, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  if (need <= 2)
    return launch_x<DK, 2, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  if constexpr (DK == 32) {
    return launch_x<DK, 4, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  } else {
    if (need <= 4)
      return launch_x<DK, 4, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
    return launch_x<DK, 8, DIAG, InT>(q, k, v, a, w, r, S0, P0, o, S_out, P_out, B, T, H, dv, s);
  }
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
