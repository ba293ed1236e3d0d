// Information-form diagonal Kalman filter (KLA), token by token.
//
// "Kalman Linear Attention: Parallel Bayesian Filtering ..." (方法论 §1-§3)
// carries a diagonal linear-Gaussian filter in information form: a precision
// per state dimension, updated by a Mobius map of the previous precision, and
// an information mean that, given the precision path, is an affine
// recursion; its forget and write gates are ratios of precisions.  On the
// KDN memory model (state S, d_v x d_k; decay a_t; process noise w_t per key
// dimension; value precision 1 / r_t), with every element of S filtered on
// its own, that is, per token and key dimension i (all rows share it):
//   p-  = a^2 p + w                 (p = 1 / lambda, the variance)
//   p   = p- r / (r + p- k^2)       (lambda = lambda- + k^2 / r)
//   f_i = a lambda- / lambda = a r / (r + p- k^2)      forget gate
//   u_i = (k / r) / lambda   = k p- / (r + p- k^2)     write gate
//   S   = S diag(f) + v u^T,   o = S q
// The variance form needs one reciprocal per token and dimension.
//
// One CTA per (b, h), in two roles, the precision one 16-token chunk ahead:
//  - Precision warps (d_k / 32 of them): thread i runs dimension i's
//    recursion over the chunk, with no barrier, and leaves f, u and q (fp32)
//    in shared memory.
//  - State warps: warp w holds rows [8 w, 8 w + 8) of S; lane l holds
//    columns [l CPL, (l + 1) CPL), CPL = d_k / 32.  A lane therefore reads
//    only its own columns' f, u and q per token (one load each, consecutive
//    across the warp) and its rows' v in one 16-byte word (bf16), and
//    o_j = S_j . q, 8 row sums per warp, is joined
//    across the lanes by recursive halving (each exchange step halves the
//    values a lane keeps).
//    The update and the row sums run on column pairs with the packed FP32
//    instructions (two FMAs per instruction).
//  - Inputs come in by cp.async in 16-token chunks, three stages deep;
//    outputs leave per chunk in coalesced rows.
#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kLC = 16;  // tokens per chunk

__device__ __forceinline__ void la_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void la_cp4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void la_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void la_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Sums item i of x[8] over the 32 lanes by recursive halving: at lane offsets
// 16, 8 and 4 a lane keeps half of its values and adds its partner's copy of
// that half; two xor steps then finish.  Lane l ends with the total of item
// l / 4.
template <int N, int O>
__device__ __forceinline__ void la_halve(float* x, int lane) {
  const bool up = (lane & O) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? x[i] : x[i + N / 2];
    const float keep = up ? x[i + N / 2] : x[i];
    x[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
  }
}
__device__ __forceinline__ float la_transpose_sum8(float (&x)[8], int lane) {
  la_halve<8, 16>(x, lane);
  la_halve<4, 8>(x, lane);
  la_halve<2, 4>(x, lane);
  float y = x[0];
  y += __shfl_xor_sync(0xffffffffu, y, 2);
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  return y;
}

template <int DK, int SW, typename InT>
struct LPlan {
  static constexpr int PW = DK / 32;                          // precision warps
  static constexpr int DVP = SW * 8;                          // d_v rounded up: 8 rows a warp
  static constexpr int KQ = kLC * 2 * DK * (int)sizeof(InT);  // [t][k | q]
  static constexpr int VB = kLC * DVP * (int)sizeof(InT);     // [t][v]
  static constexpr int F32 = kLC * (2 + DK) * 4;              // a[t], r[t], w[t][DK]
  static constexpr int STAGE = (KQ + VB + F32 + 15) / 16 * 16;
  static constexpr int OFF_G = 3 * STAGE;                     // [2][kLC][3][DK]: f, u, q
  static constexpr int OFF_OUT = OFF_G + 2 * kLC * 3 * DK * 4;  // [2][kLC][DVP]
  static constexpr int TOTAL = OFF_OUT + 2 * kLC * DVP * 4;
};

template <int DK, int SW, typename InT>
__global__ void __launch_bounds__((DK / 32 + SW) * 32)
kla_kernel(const InT* __restrict__ Q, const InT* __restrict__ K, const InT* __restrict__ V,
           const float* __restrict__ A, const float* __restrict__ Wn,
           const float* __restrict__ R, const float* S0, const float* L0,
           float* __restrict__ O, float* S_out, float* L_out, int T, int H, int dv) {
  using X = LPlan<DK, SW, InT>;
  constexpr int PW = X::PW, CPL = DK / 32, NTH = (PW + SW) * 32;
  extern __shared__ __align__(16) uint8_t lsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool pwarp = warp < PW;
  const int sw = warp - PW;  // state warp: rows 8 sw + i
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  float* gates = reinterpret_cast<float*>(lsm + X::OFF_G);
  float* obuf = reinterpret_cast<float*>(lsm + X::OFF_OUT);

  struct Stage {
    const InT* kq;
    const InT* v;
    const float* f;
  };
  auto stage = [&](int c) {
    const uint8_t* st = lsm + (c % 3) * X::STAGE;
    return Stage{reinterpret_cast<const InT*>(st), reinterpret_cast<const InT*>(st + X::KQ),
                 reinterpret_cast<const float*>(st + X::KQ + X::VB)};
  };
  auto issue = [&](int c) {
    uint8_t* st = lsm + (c % 3) * X::STAGE;
    InT* skq = reinterpret_cast<InT*>(st);
    InT* sv = reinterpret_cast<InT*>(st + X::KQ);
    float* sf = reinterpret_cast<float*>(st + X::KQ + X::VB);
    const int t0 = c * kLC, nt = min(kLC, T - t0);
    constexpr int PK = DK * (int)sizeof(InT) / 16;
    for (int i = tid; i < nt * 2 * PK; i += NTH) {
      const int t = i / (2 * PK), p = i % (2 * PK), half = p / PK, pp = p % PK;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      la_cp16(skq + (t * 2 + half) * DK + pp * (16 / (int)sizeof(InT)),
              reinterpret_cast<const uint8_t*>((half ? Q : K) + tok * DK) + pp * 16);
    }
    const int pv = dv * (int)sizeof(InT) / 16;
    for (int i = tid; i < nt * pv; i += NTH) {
      const int t = i / pv, pp = i % pv;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      la_cp16(sv + t * X::DVP + pp * (16 / (int)sizeof(InT)),
              reinterpret_cast<const uint8_t*>(V + tok * dv) + pp * 16);
    }
    constexpr int PWN = DK * 4 / 16;
    for (int i = tid; i < nt * PWN; i += NTH) {
      const int t = i / PWN, pp = i % PWN;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      la_cp16(sf + 2 * kLC + t * DK + pp * 4, Wn + tok * DK + pp * 4);
    }
    for (int i = tid; i < 2 * nt; i += NTH) {
      const int which = i / nt, t = i % nt;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      la_cp4(sf + which * kLC + t, (which ? R : A) + tok);
    }
  };

  // ---- state: the precision lanes carry the variance p_i = 1 / lambda_i;
  // the state lanes hold their CPL columns of 8 rows.  S_out / L_out may alias
  // S0 / L0: every read comes before the barrier that precedes the stores.
  float p = 1.f;
  float Sr[8][CPL];
  const size_t s_base = (size_t)bh * dv * DK;
  if (pwarp) {
    p = L0 ? 1.f / L0[(size_t)bh * DK + tid] : 1.f;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * sw + i;
#pragma unroll
      for (int c = 0; c < CPL; ++c)
        Sr[i][c] = (S0 && j < dv) ? S0[s_base + (size_t)j * DK + lane * CPL + c] : 0.f;
    }
  }

  // precision lanes: gates of chunk cc
  auto gates_of = [&](int cc) {
    const Stage st = stage(cc);
    const int nt = min(kLC, T - cc * kLC);
    float* g = gates + (cc & 1) * kLC * 3 * DK;
    for (int t = 0; t < nt; ++t) {
      const float a = st.f[t], r = st.f[kLC + t], w = st.f[2 * kLC + t * DK + tid];
      const float k = to_f32(st.kq[t * 2 * DK + tid]);
      const float pm = __fmaf_rn(a * a, p, w);
      const float inv = __frcp_rn(__fmaf_rn(pm * k, k, r));
      g[(t * 3 + 0) * DK + tid] = a * r * inv;   // forget gate
      g[(t * 3 + 1) * DK + tid] = k * pm * inv;  // write gate
      g[(t * 3 + 2) * DK + tid] = to_f32(st.kq[t * 2 * DK + DK + tid]);
      p = pm * r * inv;
    }
  };

  // state lanes: chunk cc through S
  auto states = [&](int cc) {
    const Stage st = stage(cc);
    const int nt = min(kLC, T - cc * kLC);
    const float* g = gates + (cc & 1) * kLC * 3 * DK;
    float* ob = obuf + (cc & 1) * kLC * X::DVP;
    for (int t = 0; t < nt; ++t) {
      float f[CPL], u[CPL], q[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        f[c] = g[(t * 3 + 0) * DK + lane * CPL + c];
        u[c] = g[(t * 3 + 1) * DK + lane * CPL + c];
        q[c] = g[(t * 3 + 2) * DK + lane * CPL + c];
      }
      // v of this warp's 8 rows (rows at or past d_v were never staged: zero)
      float vr[8];
      const InT* vp = st.v + t * X::DVP + 8 * sw;
      if constexpr (sizeof(InT) == 2) {
        const uint4 raw = *reinterpret_cast<const uint4*>(vp);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          vr[2 * e] = __uint_as_float(wd[e] << 16);
          vr[2 * e + 1] = __uint_as_float(wd[e] & 0xffff0000u);
        }
      } else {
        const float4 v0 = *reinterpret_cast<const float4*>(vp);
        const float4 v1 = *reinterpret_cast<const float4*>(vp + 4);
        vr[0] = v0.x; vr[1] = v0.y; vr[2] = v0.z; vr[3] = v0.w;
        vr[4] = v1.x; vr[5] = v1.y; vr[6] = v1.z; vr[7] = v1.w;
      }
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float vj = 8 * sw + i < dv ? vr[i] : 0.f;
        if constexpr (CPL == 1) {
          Sr[i][0] = __fmaf_rn(vj, u[0], Sr[i][0] * f[0]);
          x[i] = Sr[i][0] * q[0];
        } else {
          // column pairs on the packed FP32 pipe: S <- (S f) + v u, acc += S q
          float2 acc = make_float2(0.f, 0.f);
          const float2 v2 = make_float2(vj, vj);
#pragma unroll
          for (int c = 0; c < CPL; c += 2) {
            float2 sp = make_float2(Sr[i][c], Sr[i][c + 1]);
            sp = __ffma2_rn(v2, make_float2(u[c], u[c + 1]),
                            __fmul2_rn(sp, make_float2(f[c], f[c + 1])));
            acc = __ffma2_rn(sp, make_float2(q[c], q[c + 1]), acc);
            Sr[i][c] = sp.x;
            Sr[i][c + 1] = sp.y;
          }
          x[i] = acc.x + acc.y;
        }
      }
      // lane l ends with the row sum of row 8 sw + l / 4
      const float o = la_transpose_sum8(x, lane);
      if ((lane & 3) == 0) ob[t * X::DVP + 8 * sw + (lane >> 2)] = o;
    }
  };

  auto flush = [&](int cc) {
    const int t0 = cc * kLC, nt = min(kLC, T - t0);
    const float* ob = obuf + (cc & 1) * kLC * X::DVP;
    for (int i = tid; i < nt * dv; i += NTH) {
      const int t = i / dv, j = i % dv;
      O[(((size_t)b * T + t0 + t) * H + h) * dv + j] = ob[t * X::DVP + j];
    }
  };

  // Phase c: gates of chunk c + 1 while the state lanes run chunk c; chunk
  // c + 2 is copied into the stage chunk c - 1 used.
  const int nchunks = (T + kLC - 1) / kLC;
  issue(0);
  la_commit();
  if (nchunks > 1) issue(1);
  la_commit();
  la_wait1();
  __syncthreads();
  if (pwarp) gates_of(0);
  for (int c = 0; c < nchunks; ++c) {
    __syncthreads();  // phase c - 1 done
    if (c > 0) flush(c - 1);
    if (c + 2 < nchunks) issue(c + 2);
    la_commit();
    la_wait1();       // chunk c + 1 landed (this thread's copies)
    __syncthreads();  // ... and everyone's
    if (pwarp) {
      if (c + 1 < nchunks) gates_of(c + 1);
    } else {
      states(c);
    }
  }
  __syncthreads();
  if (nchunks > 0) flush(nchunks - 1);

  if (pwarp) {
    L_out[(size_t)bh * DK + tid] = 1.f / p;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * sw + i;
      if (j < dv) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) S_out[s_base + (size_t)j * DK + lane * CPL + c] = Sr[i][c];
      }
    }
  }
}

template <int DK, int SW, typename InT>
kdn_status launch_l(const void* q, const void* k, const void* v, const float* a, const float* w,
                    const float* r, const float* S0, const float* L0, float* o, float* S_out,
                    float* L_out, int B, int T, int H, int dv, cudaStream_t s) {
  using X = LPlan<DK, SW, InT>;
  auto kern = kla_kernel<DK, SW, InT>;
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
      S0, L0, o, S_out, L_out, T, H, dv);
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

// state warps: 8 rows of S each, d_v / 8 rounded up to 1, 2, 4, 8 or 16 warps
template <int DK, typename InT>
kdn_status launch_ldv(const void* q, const void* k, const void* v, const float* a, const float* w,
                      const float* r, const float* S0, const float* L0, float* o, float* S_out,
                      float* L_out, int B, int T, int H, int dv, cudaStream_t s) {
  const int need = (dv + 7) / 8;
  if (need <= 1) return launch_l<DK, 1, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
  if (need <= 2) return launch_l<DK, 2, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
  if (need <= 4) return launch_l<DK, 4, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
  if (need <= 8) return launch_l<DK, 8, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
  return launch_l<DK, 16, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
}

template <typename InT>
kdn_status launch_ldk(const void* q, const void* k, const void* v, const float* a, const float* w,
                      const float* r, const float* S0, const float* L0, float* o, float* S_out,
                      float* L_out, int B, int T, int H, int dk, int dv, cudaStream_t s) {
  switch (dk) {
    case 32: return launch_ldv<32, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
    case 64: return launch_ldv<64, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
    default: return launch_ldv<128, InT>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dv, s);
  }
}

}  // namespace

bool kla_supported(int dk, int dv) {
  return (dk == 32 || dk == 64 || dk == 128) && dv >= 8 && dv <= 128 && dv % 8 == 0;
}

kdn_status kla_launch(kdn_dtype dt, const void* q, const void* k, const void* v, const float* a,
                      const float* w, const float* r, const float* S0, const float* L0, float* o,
                      float* S_out, float* L_out, int B, int T, int H, int dk, int dv,
                      cudaStream_t s) {
  return dt == KDN_BF16
             ? launch_ldk<__nv_bfloat16>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dk, dv, s)
             : launch_ldk<float>(q, k, v, a, w, r, S0, L0, o, S_out, L_out, B, T, H, dk, dv, s);
}

}  // namespace kdn
