// Backward pass of the KDN layer (token-recurrent): gradients of a loss with
// respect to q, k, v, a, w, r, S0 and p0, given its gradients with respect to
// the outputs o and the final state (S_T, p_T).
//
// The layer is trained end to end ("Kalman Delta Networks: 不确定性感知的
// 联想记忆", 实验: pretrained language models), so its forward recurrence has
// an adjoint that runs from the last token to the first, carrying dS (the
// gradient with respect to the state after the token) and dp.  Per token,
// with S the state before it (saved by the forward pass), S' after it:
//   dS += do q^T;  dq = S'^T do
//   de = dS g;  dg = dS^T e;  da += <dS, S> - <de, S k>;  dv = de
//   dk = -a S^T de + (gain terms);  dS <- a (dS - de k^T)
// then the terms of the gain g and of the variance recursion p, which give
// dk, da, dw, dr and carry dp to the token before (dp <- a^2 dp-).
//
// Layout as the recurrent forward kernel: one CTA per (b, h) of NW warps
// (8, or 16 at d_k = 128 so that S and dS of a warp's rows fit in its
// registers); warp w holds rows w, w + NW, ... of S and dS, lane l holds
// columns [l CPL, (l + 1) CPL).  Row sums (S k, dS g) are butterfly
// reductions inside a warp; the column sums over all rows (S'^T do, dS^T e,
// S^T de) and the scalar <dS, S> meet in shared memory, one block barrier per
// token.  The gain and variance terms are per column and are computed by
// every warp identically, so no further exchange is needed.
//
// States: the forward keeps S only before every 16th token (a checkpoint)
// and p before every token.  The backward walks blocks of 16 tokens from
// the last to the first; for each it rebuilds the block's states from its
// checkpoint with the forward's own arithmetic into a per-CTA scratch of 16
// states (small enough to stay in L2 for all CTAs of a launch), then runs
// the adjoint over them.  Each thread reads back only what it wrote itself.
#include "kdn_common.cuh"
#include "bwd_checkpoint.h"

namespace kdn {
namespace {

template <int CPL>
struct BwdShape {
  static constexpr int NW = CPL == 4 ? 16 : 8;  // warps
  static constexpr int NR = 128 / NW;            // rows of S per warp (d_v <= 128)
  static constexpr int DK = CPL * 32;
  static constexpr int RED = 3 * DK + 1;
  static constexpr size_t SMEM = 2u * NW * RED * sizeof(float);
};

template <bool DIAG, int CPL, typename InT>
__global__ void __launch_bounds__(BwdShape<CPL>::NW * 32)
kdn_bwd_kernel(const InT* __restrict__ Q, const InT* __restrict__ K,
               const InT* __restrict__ V, const float* __restrict__ A,
               const float* __restrict__ Wn, const float* __restrict__ R,
               const float* __restrict__ dO, const float* __restrict__ dS_T,
               const float* __restrict__ dp_T, const float* __restrict__ Sck,
               const float* __restrict__ Psave, float* __restrict__ scratch,
               float* __restrict__ dQ, float* __restrict__ dK, float* __restrict__ dV,
               float* __restrict__ dA, float* __restrict__ dW, float* __restrict__ dR,
               float* __restrict__ dS0, float* __restrict__ dP0, int T, int H, int dv,
               float kappa) {
  using X = BwdShape<CPL>;
  constexpr int NW = X::NW, NR = X::NR, DK = X::DK, RED = X::RED, NP = DIAG ? CPL : 1;
  extern __shared__ float red_dyn[];  // [2][NW][RED]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;

  float dS[NR][CPL], dp[NP];
  const size_t s_base = (size_t)bh * dv * DK;
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int j = warp + NW * i;
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      dS[i][c] = (dS_T && j < dv) ? dS_T[s_base + (size_t)j * DK + lane * CPL + c] : 0.f;
  }
#pragma unroll
  for (int c = 0; c < NP; ++c)
    dp[c] = dp_T ? dp_T[DIAG ? (size_t)bh * DK + lane * CPL + c : (size_t)bh] : 0.f;

  const int nck = (T + kBwdCheckpoint - 1) / kBwdCheckpoint;
  float* scr = scratch + (size_t)bh * kBwdCheckpoint * dv * DK;
  for (int blk = nck - 1; blk >= 0; --blk) {
    const int t0 = blk * kBwdCheckpoint, t1 = min(T, t0 + kBwdCheckpoint);
    // ---- the block's states, rebuilt from its checkpoint (the forward's
    // arithmetic, token by token) into the scratch
    {
      float S[NR][CPL];
      const float* ck = Sck + ((size_t)bh * nck + blk) * dv * DK;
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const int j = warp + NW * i;
#pragma unroll
        for (int c = 0; c < CPL; ++c) S[i][c] = j < dv ? ck[(size_t)j * DK + lane * CPL + c] : 0.f;
      }
      for (int t = t0; t < t1; ++t) {
        float* dst = scr + (size_t)(t - t0) * dv * DK;
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int j = warp + NW * i;
          if (j < dv) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) dst[(size_t)j * DK + lane * CPL + c] = S[i][c];
          }
        }
        if (t + 1 == t1) break;
        const size_t tok = ((size_t)b * T + t) * H + h;
        const size_t sv = ((size_t)bh * T + t);
        float k[CPL], g[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) k[c] = to_f32(K[tok * DK + lane * CPL + c]);
        const float a = A[tok], r = R[tok];
        if constexpr (DIAG) {
          float pp[CPL], part = 0.f;
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            pp[c] = fmaf(a * a, Psave[sv * DK + lane * CPL + c], Wn[tok * DK + lane * CPL + c]);
            part = fmaf(pp[c] * k[c], k[c], part);
          }
          const float inv_s = 1.f / (warp_sum(part) + r);
#pragma unroll
          for (int c = 0; c < CPL; ++c) g[c] = pp[c] * k[c] * inv_s;
        } else {
          float part = 0.f;
#pragma unroll
          for (int c = 0; c < CPL; ++c) part = fmaf(k[c], k[c], part);
          const float n = warp_sum(part);
          const float pp = fmaf(a * a, Psave[sv], Wn[tok]);
          const float beta = pp / fmaf(pp, n, r);
#pragma unroll
          for (int c = 0; c < CPL; ++c) g[c] = beta * k[c];
        }
        float sk[NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          float x = 0.f;
#pragma unroll
          for (int c = 0; c < CPL; ++c) x = fmaf(S[i][c], k[c], x);
          sk[i] = x;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < NR; ++i) sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int j = warp + NW * i;
          const float e = (j < dv ? to_f32(V[tok * dv + j]) : 0.f) - a * sk[i];
#pragma unroll
          for (int c = 0; c < CPL; ++c) S[i][c] = fmaf(e, g[c], a * S[i][c]);
        }
      }
    }

    // ---- the adjoint over the block, last token first
    for (int t = t1 - 1; t >= t0; --t) {
    const size_t tok = ((size_t)b * T + t) * H + h;
    const size_t sv = ((size_t)bh * T + t);
    const float* Ssrc = scr + (size_t)(t - t0) * dv * DK;
    float k[CPL], q[CPL], S[NR][CPL], p[NP], wv[NP];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      k[c] = to_f32(K[tok * DK + lane * CPL + c]);
      q[c] = to_f32(Q[tok * DK + lane * CPL + c]);
    }
    const float a = A[tok], r = R[tok];
#pragma unroll
    for (int c = 0; c < NP; ++c) {
      p[c] = Psave[DIAG ? sv * DK + lane * CPL + c : sv];
      wv[c] = Wn[DIAG ? tok * DK + lane * CPL + c : tok];
    }
    float vi[NR], doi[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int j = warp + NW * i;
      vi[i] = j < dv ? to_f32(V[tok * dv + j]) : 0.f;
      doi[i] = j < dv ? dO[tok * dv + j] : 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c)
        S[i][c] = j < dv ? Ssrc[(size_t)j * DK + lane * CPL + c] : 0.f;
    }
    // the token's gain, recomputed from the saved variance
    float g[CPL], pm[NP], pn[NP], n = 0.f, den = 0.f, beta = 0.f, s = 0.f;
    if constexpr (DIAG) {
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        pm[c] = a * a * p[c] + wv[c];
        part = fmaf(pm[c] * k[c], k[c], part);
        pn[c] = 1.f / (1.f / pm[c] + k[c] * k[c] / r);
      }
      s = warp_sum(part) + r;
#pragma unroll
      for (int c = 0; c < CPL; ++c) g[c] = pm[c] * k[c] / s;
    } else {
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) part = fmaf(k[c], k[c], part);
      n = warp_sum(part);
      pm[0] = a * a * p[0] + wv[0];
      den = pm[0] * n + r;
      beta = pm[0] / den;
      pn[0] = 1.f / (1.f / pm[0] + kappa * n / r);
#pragma unroll
      for (int c = 0; c < CPL; ++c) g[c] = beta * k[c];
    }

    // S k per row (all lanes end with the sums), e = v - a S k
    float sk[NR], e[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      float x = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) x = fmaf(S[i][c], k[c], x);
      sk[i] = x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < NR; ++i) sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
#pragma unroll
    for (int i = 0; i < NR; ++i) e[i] = vi[i] - a * sk[i];

    // dS += do q^T, then de = dS g per row
    float de[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      float x = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dS[i][c] = fmaf(doi[i], q[c], dS[i][c]);
        x = fmaf(dS[i][c], g[c], x);
      }
      de[i] = x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < NR; ++i) de[i] += __shfl_xor_sync(0xffffffffu, de[i], o);

    // column sums over this warp's rows: S'^T do, dS^T e, S^T de; and <dS, S>
    float cq[CPL], cg[CPL], cs[CPL], dss = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      cq[c] = 0.f;
      cg[c] = 0.f;
      cs[c] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < NR; ++i) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const float snew = fmaf(e[i], g[c], a * S[i][c]);
        cq[c] = fmaf(snew, doi[i], cq[c]);
        cg[c] = fmaf(dS[i][c], e[i], cg[c]);
        cs[c] = fmaf(S[i][c], de[i], cs[c]);
        dss = fmaf(dS[i][c], S[i][c], dss);
      }
    }
    dss = warp_sum(dss);
    float dek = 0.f;  // <de, S k> over this warp's rows (the same in every lane)
#pragma unroll
    for (int i = 0; i < NR; ++i) dek = fmaf(de[i], sk[i], dek);
    float* rd = red_dyn + ((size_t)(t & 1) * NW + warp) * RED;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      rd[lane * CPL + c] = cq[c];
      rd[DK + lane * CPL + c] = cg[c];
      rd[2 * DK + lane * CPL + c] = cs[c];
    }
    if (lane == 0) rd[3 * DK] = dss - dek;
    __syncthreads();
    float dq[CPL], dg[CPL], sde[CPL], da = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      dq[c] = 0.f;
      dg[c] = 0.f;
      sde[c] = 0.f;
    }
#pragma unroll
    for (int w = 0; w < NW; ++w) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dq[c] += red_dyn[((size_t)(t & 1) * NW + w) * RED + lane * CPL + c];
        dg[c] += red_dyn[((size_t)(t & 1) * NW + w) * RED + DK + lane * CPL + c];
        sde[c] += red_dyn[((size_t)(t & 1) * NW + w) * RED + 2 * DK + lane * CPL + c];
      }
      da += red_dyn[((size_t)(t & 1) * NW + w) * RED + 3 * DK];
    }

    // the gain and variance terms
    float dk[CPL], dw[NP], dr = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dk[c] = -a * sde[c];
    if constexpr (DIAG) {
      float dpm[CPL], pg = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dpm[c] = dg[c] * k[c] / s;
        dk[c] += dg[c] * pm[c] / s;
        pg = fmaf(dg[c], g[c], pg);
      }
      const float ds = -warp_sum(pg) / s;
      float dDk = 0.f, pdpm = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dpm[c] += ds * k[c] * k[c];
        dk[c] += 2.f * ds * pm[c] * k[c];
        const float dD = -dp[c] * pn[c] * pn[c];
        dpm[c] -= dD / (pm[c] * pm[c]);
        dk[c] += 2.f * dD * k[c] / r;
        dDk = fmaf(dD, k[c] * k[c], dDk);
        pdpm = fmaf(p[c], dpm[c], pdpm);
        dw[c] = dpm[c];
        dp[c] = a * a * dpm[c];
      }
      dr = ds - warp_sum(dDk) / (r * r);
      da += 2.f * a * warp_sum(pdpm);
    } else {
      float kg = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dk[c] += beta * dg[c];
        kg = fmaf(dg[c], k[c], kg);
      }
      const float dbeta = warp_sum(kg);
      float dpm = dbeta * r / (den * den);
      float dn = -dbeta * pm[0] * pm[0] / (den * den);
      dr = -dbeta * pm[0] / (den * den);
      const float dD = -dp[0] * pn[0] * pn[0];
      dpm -= dD / (pm[0] * pm[0]);
      dn += dD * kappa / r;
      dr -= dD * kappa * n / (r * r);
#pragma unroll
      for (int c = 0; c < CPL; ++c) dk[c] += 2.f * dn * k[c];
      da += 2.f * a * p[0] * dpm;
      dw[0] = dpm;
      dp[0] = a * a * dpm;
    }

    // outputs of token t: the column vectors and scalars from warp 0, the
    // rows of dv from the warp that holds them
    if (warp == 0) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        dQ[tok * DK + lane * CPL + c] = dq[c];
        dK[tok * DK + lane * CPL + c] = dk[c];
        if constexpr (DIAG) dW[tok * DK + lane * CPL + c] = dw[c];
      }
      if (lane == 0) {
        dA[tok] = da;
        dR[tok] = dr;
        if constexpr (!DIAG) dW[tok] = dw[0];
      }
    }
    if (lane < NR) {
      // lane i writes row warp + 8 i (every lane holds every de after the butterfly)
      float mine = 0.f;
#pragma unroll
      for (int i = 0; i < NR; ++i) mine = lane == i ? de[i] : mine;
      const int j = warp + NW * lane;
      if (j < dv) dV[tok * dv + j] = mine;
    }
    // dS before the token: a (dS - de k^T)
#pragma unroll
    for (int i = 0; i < NR; ++i)
#pragma unroll
      for (int c = 0; c < CPL; ++c) dS[i][c] = a * fmaf(-de[i], k[c], dS[i][c]);
    }
  }

#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int j = warp + NW * i;
    if (j < dv) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) dS0[s_base + (size_t)j * DK + lane * CPL + c] = dS[i][c];
    }
  }
  if (warp == 0) {
    if constexpr (DIAG) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) dP0[(size_t)bh * DK + lane * CPL + c] = dp[c];
    } else {
      if (lane == 0) dP0[bh] = dp[0];
    }
  }
}

template <bool DIAG, int CPL, typename InT>
kdn_status launch_b(const void* q, const void* k, const void* v, const float* a, const float* w,
                    const float* r, const float* dO, const float* dS_T, const float* dp_T,
                    const float* Sck, const float* Psave, float* scratch, float* dq, float* dk,
                    float* dv_, float* da, float* dw, float* dr, float* dS0, float* dp0, int B,
                    int T, int H, int dv, float kappa, cudaStream_t s) {
  using X = BwdShape<CPL>;
  auto kern = kdn_bwd_kernel<DIAG, CPL, InT>;
  if (X::SMEM > 48u * 1024u &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)X::SMEM) !=
          cudaSuccess)
    return KDN_ERR_CUDA;
  kern<<<B * H, X::NW * 32, X::SMEM, s>>>(
      static_cast<const InT*>(q), static_cast<const InT*>(k), static_cast<const InT*>(v), a, w, r,
      dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk, dv_, da, dw, dr, dS0, dp0, T, H, dv, kappa);
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

template <bool DIAG, typename InT>
kdn_status launch_bdk(const void* q, const void* k, const void* v, const float* a,
                      const float* w, const float* r, const float* dO, const float* dS_T,
                      const float* dp_T, const float* Sck, const float* Psave, float* scratch,
                      float* dq, float* dk, float* dv_, float* da, float* dw, float* dr,
                      float* dS0, float* dp0, int B, int T, int H, int dkk, int dv, float kappa,
                      cudaStream_t s) {
  switch (dkk) {
    case 32:
      return launch_b<DIAG, 1, InT>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk,
                                    dv_, da, dw, dr, dS0, dp0, B, T, H, dv, kappa, s);
    case 64:
      return launch_b<DIAG, 2, InT>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk,
                                    dv_, da, dw, dr, dS0, dp0, B, T, H, dv, kappa, s);
    default:
      return launch_b<DIAG, 4, InT>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk,
                                    dv_, da, dw, dr, dS0, dp0, B, T, H, dv, kappa, s);
  }
}

}  // namespace

bool backward_supported(int dk, int dv) {
  return (dk == 32 || dk == 64 || dk == 128) && dv >= 1 && dv <= 128;
}

kdn_status backward_launch(bool diag, kdn_dtype dt, const void* q, const void* k, const void* v,
                           const float* a, const float* w, const float* r, const float* dO,
                           const float* dS_T, const float* dp_T, const float* Sck,
                           const float* Psave, float* scratch, float* dq, float* dk, float* dv_,
                           float* da, float* dw, float* dr, float* dS0, float* dp0, int B, int T,
                           int H, int dkk, int dv, float kappa, cudaStream_t s) {
  if (diag)
    return dt == KDN_BF16
               ? launch_bdk<true, __nv_bfloat16>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk, dv_, da, dw, dr, dS0, dp0, B, T, H, dkk, dv, kappa, s)
               : launch_bdk<true, float>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk, dv_, da, dw, dr, dS0, dp0, B, T, H, dkk, dv, kappa, s);
  return dt == KDN_BF16
             ? launch_bdk<false, __nv_bfloat16>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk, dv_, da, dw, dr, dS0, dp0, B, T, H, dkk, dv, kappa, s)
             : launch_bdk<false, float>(q, k, v, a, w, r, dO, dS_T, dp_T, Sck, Psave, scratch, dq, dk, dv_, da, dw, dr, dS0, dp0, B, T, H, dkk, dv, kappa, s);
}

}  // namespace kdn
