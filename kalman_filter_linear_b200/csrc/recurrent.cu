// Token-by-token KDN kernel: the decode step, and the recurrent forward path.
//
// One CTA owns one (b, h) state S (dv x dk fp32) for the whole sequence.
// Warp w holds rows j = w, w+8, w+16, ... of S in registers; lane l holds
// columns [l*CPL, (l+1)*CPL) of each (CPL = dk/32).  Per token every warp
// recomputes the (cheap) variance and gain for itself, so warps never wait
// on each other:
//   iso:  n = ||k||^2, p- = a^2 p + w, beta = p-/(p- n + r),
//         p = 1/(1/p- + kappa n / r), g = beta k
//   diag: p-_i = a^2 p_i + w_i, s = sum_i p-_i k_i^2 + r, g = p- * k / s,
//         p_i = 1/(1/p-_i + k_i^2 / r)
// and for each row j (predict, then gain-weighted residual write, then read):
//   sk = S_j.k, sq = S_j.q, e_j = v_j - a sk,
//   S_j <- a S_j + e_j g,   o_j = a sq + e_j (g.q)
// ("Kalman Delta Networks: 不确定性感知的联想记忆", 方法 — 关键模块 steps
// 1-3 and 输出与差异点; "Kalman Delta Networks: Uncertainty-aware
// Associative Memory", abstract).  o_j needs no second pass over S because
// S_new q = a S q + e (g.q).
//
// With T = 1 and the state updated in place this is the constant-memory
// decode step; the grid then spans all B*H heads and the kernel streams S
// once in and once out (HBM-bound).
#include "kdn_common.cuh"
#include "bwd_checkpoint.h"

namespace kdn {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxRowsPerWarp = 16;  // dv <= 128

template <int CPL, typename InT>
__device__ __forceinline__ void load_vec(const InT* __restrict__ p, int lane, float (&x)[CPL]) {
#pragma unroll
  for (int c = 0; c < CPL; ++c) x[c] = to_f32(p[lane * CPL + c]);
}

template <int CPL>
__device__ __forceinline__ void load_vec(const float* __restrict__ p, int lane, float (&x)[CPL]) {
  if constexpr (CPL == 4) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(p) + lane);
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else if constexpr (CPL == 2) {
    const float2 f = __ldg(reinterpret_cast<const float2*>(p) + lane);
    x[0] = f.x; x[1] = f.y;
  } else {
#pragma unroll
    for (int c = 0; c < CPL; ++c) x[c] = __ldg(p + lane * CPL + c);
  }
}

// State loads use plain (coherent) loads: S0 / P0 may alias S_out / P_out.
template <int CPL>
__device__ __forceinline__ void load_state(const float* p, int lane, float (&x)[CPL]) {
  if constexpr (CPL == 4) {
    const float4 f = reinterpret_cast<const float4*>(p)[lane];
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else {
#pragma unroll
    for (int c = 0; c < CPL; ++c) x[c] = p[lane * CPL + c];
  }
}

// Layout of the per-token tensors: q/k/v at ((b*T + t)*H + h)*d; a/w/r at
// (b*T + t)*H + h (diag w: ((b*T + t)*H + h)*dk).  The decode step is T = 1.
// SAVE: for the backward pass, the variance p before every token goes to
// Psave ([B H][T][1 or dk]) and the state S before every kBwdCheckpoint-th
// token (t = 0, 16, 32, ...) to Ssave ([B H][ceil(T / 16)][dv][dk]).
template <bool DIAG, int CPL, typename InT, bool SAVE>
__global__ void __launch_bounds__(kWarps * 32)
recurrent_kernel(const InT* __restrict__ Q, const InT* __restrict__ K, const InT* __restrict__ V,
                 const float* __restrict__ A, const float* __restrict__ Wn,
                 const float* __restrict__ R, const float* S0, const float* P0,
                 float* __restrict__ O, float* S_out, float* P_out, int T, int H, int dv,
                 float kappa, const int* __restrict__ cu_seqlens, uint32_t* err,
                 float* __restrict__ Ssave, float* __restrict__ Psave) {
  constexpr int DK = CPL * 32;
  const int bh = blockIdx.x;
  const int h = bh % H;
  // this CTA's tokens: rows [row0, row0 + Tn) of the [rows, H, ...] tensors
  // (batch entry bh / H, or packed sequence bh / H when cu_seqlens is given)
  size_t row0 = (size_t)(bh / H) * T;
  int Tn = T;
  if (cu_seqlens) {
    const int s0 = cu_seqlens[bh / H], s1 = cu_seqlens[bh / H + 1];
    const int tbeg = min(max(s0, 0), T);
    Tn = min(max(s1, tbeg), T) - tbeg;
    row0 = (size_t)tbeg;
    if (err && threadIdx.x == 0 && (s0 < 0 || s1 < s0 || s1 > T)) atomicOr(err, DEV_BAD_ARG);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // ---- state into registers
  float S[kMaxRowsPerWarp][CPL];
  const size_t s_base = (size_t)bh * dv * DK;
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) {
    const int j = warp + kWarps * i;
    if (j < dv && S0) {
      load_state<CPL>(S0 + s_base + (size_t)j * DK, lane, S[i]);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[i][c] = 0.f;
    }
  }
  float p[DIAG ? CPL : 1];
  if constexpr (DIAG) {
    if (P0) {
      load_state<CPL>(P0 + (size_t)bh * DK, lane, p);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) p[c] = 1.f;
    }
  } else {
    p[0] = P0 ? P0[bh] : 1.f;
  }

  for (int t = 0; t < Tn; ++t) {
    const size_t tok = (row0 + t) * H + h;
    if constexpr (SAVE) {
      if (t % kBwdCheckpoint == 0) {
        const int nck = (T + kBwdCheckpoint - 1) / kBwdCheckpoint;
        const size_t sb = ((size_t)bh * nck + t / kBwdCheckpoint) * dv * DK;
#pragma unroll
        for (int i = 0; i < kMaxRowsPerWarp; ++i) {
          const int j = warp + kWarps * i;
          if (j < dv) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) Ssave[sb + (size_t)j * DK + lane * CPL + c] = S[i][c];
          }
        }
      }
      if constexpr (DIAG) {
        if (warp == 0) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) Psave[((size_t)bh * T + t) * DK + lane * CPL + c] = p[c];
        }
      } else {
        if (threadIdx.x == 0) Psave[(size_t)bh * T + t] = p[0];
      }
    }
    float k[CPL], q[CPL];
    load_vec<CPL>(K + tok * DK, lane, k);
    load_vec<CPL>(Q + tok * DK, lane, q);
    // v for this warp's rows: lane i < rows fetches row (warp + 8 i)
    float vmine = 0.f;
    {
      const int j = warp + kWarps * lane;
      if (lane < kMaxRowsPerWarp && j < dv) vmine = to_f32(V[tok * dv + j]);
    }
    const float a = __ldg(A + tok), r = __ldg(R + tok);

    float g[CPL];
    if constexpr (DIAG) {
      float w[CPL];
      load_vec<CPL>(Wn + tok * DK, lane, w);
      float pp[CPL], s_part = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        pp[c] = fmaf(a * a, p[c], w[c]);
        s_part = fmaf(pp[c] * k[c], k[c], s_part);
      }
      const float s = warp_sum(s_part) + r;
      const float inv_s = 1.f / s;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        g[c] = pp[c] * k[c] * inv_s;
        p[c] = 1.f / (1.f / pp[c] + k[c] * k[c] / r);
      }
    } else {
      float n_part = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) n_part = fmaf(k[c], k[c], n_part);
      const float n = warp_sum(n_part);
      const float pp = fmaf(a * a, p[0], __ldg(Wn + tok));
      const float beta = pp / fmaf(pp, n, r);
      p[0] = 1.f / (1.f / pp + kappa * n / r);
#pragma unroll
      for (int c = 0; c < CPL; ++c) g[c] = beta * k[c];
    }
    float gq_part = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) gq_part = fmaf(g[c], q[c], gq_part);
    const float gq = warp_sum(gq_part);

    float sk[kMaxRowsPerWarp], sq[kMaxRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kMaxRowsPerWarp; ++i) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        x = fmaf(S[i][c], k[c], x);
        y = fmaf(S[i][c], q[c], y);
      }
      sk[i] = x;
      sq[i] = y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < kMaxRowsPerWarp; ++i) {
        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], o);
        sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], o);
      }
    }
    float omine = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxRowsPerWarp; ++i) {
      const float vj = __shfl_sync(0xffffffffu, vmine, i);
      const float e = vj - a * sk[i];
#pragma unroll
      for (int c = 0; c < CPL; ++c) S[i][c] = fmaf(e, g[c], a * S[i][c]);
      const float oj = fmaf(e, gq, a * sq[i]);
      if (lane == i) omine = oj;
    }
    {
      const int j = warp + kWarps * lane;
      if (lane < kMaxRowsPerWarp && j < dv) O[tok * dv + j] = omine;
    }
  }

  // ---- state out
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) {
    const int j = warp + kWarps * i;
    if (j < dv) {
      float* dst = S_out + s_base + (size_t)j * DK;
      if constexpr (CPL == 4) {
        reinterpret_cast<float4*>(dst)[lane] = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[lane * CPL + c] = S[i][c];
      }
    }
  }
  if constexpr (DIAG) {
    if (warp == 0) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) P_out[(size_t)bh * DK + lane * CPL + c] = p[c];
    }
  } else {
    if (threadIdx.x == 0) P_out[bh] = p[0];
  }
}

template <bool DIAG, int CPL, typename InT>
kdn_status launch_t(const void* q, const void* k, const void* v, const float* a, const float* w,
                    const float* r, const float* S0, const float* p0, float* o, float* S_out,
                    float* p_out, int B, int T, int H, int dv, float kappa, cudaStream_t s,
                    const int* cu, uint32_t* err, float* Ssave, float* Psave) {
  if (Ssave) {
    recurrent_kernel<DIAG, CPL, InT, true><<<B * H, kWarps * 32, 0, s>>>(
        static_cast<const InT*>(q), static_cast<const InT*>(k), static_cast<const InT*>(v), a, w,
        r, S0, p0, o, S_out, p_out, T, H, dv, kappa, cu, err, Ssave, Psave);
  } else {
    recurrent_kernel<DIAG, CPL, InT, false><<<B * H, kWarps * 32, 0, s>>>(
        static_cast<const InT*>(q), static_cast<const InT*>(k), static_cast<const InT*>(v), a, w,
        r, S0, p0, o, S_out, p_out, T, H, dv, kappa, cu, err, nullptr, nullptr);
  }
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

template <bool DIAG, typename InT>
kdn_status launch_dk(const void* q, const void* k, const void* v, const float* a, const float* w,
                     const float* r, const float* S0, const float* p0, float* o, float* S_out,
                     float* p_out, int B, int T, int H, int dk, int dv, float kappa,
                     cudaStream_t s, const int* cu, uint32_t* err, float* Ssave, float* Psave) {
  switch (dk) {
    case 32: return launch_t<DIAG, 1, InT>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, s, cu, err, Ssave, Psave);
    case 64: return launch_t<DIAG, 2, InT>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, s, cu, err, Ssave, Psave);
    case 128: return launch_t<DIAG, 4, InT>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv, kappa, s, cu, err, Ssave, Psave);
    default: return KDN_ERR_UNSUPPORTED;
  }
}

}  // namespace

// S_out may alias S0 and P_out may alias P0: each CTA reads its state fully
// before it writes it.
kdn_status recurrent_launch(bool diag, kdn_dtype dt, const void* q, const void* k, const void* v,
                            const float* a, const float* w, const float* r, const float* S0,
                            const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                            int H, int dk, int dv, float kappa, cudaStream_t s,
                            const int* cu_seqlens, uint32_t* err, float* Ssave, float* Psave) {
  if (diag) {
    return dt == KDN_BF16
               ? launch_dk<true, __nv_bfloat16>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk, dv, kappa, s, cu_seqlens, err, Ssave, Psave)
               : launch_dk<true, float>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk, dv, kappa, s, cu_seqlens, err, Ssave, Psave);
  }
  return dt == KDN_BF16
             ? launch_dk<false, __nv_bfloat16>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk, dv, kappa, s, cu_seqlens, err, Ssave, Psave)
             : launch_dk<false, float>(q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk, dv, kappa, s, cu_seqlens, err, Ssave, Psave);
}

}  // namespace kdn
