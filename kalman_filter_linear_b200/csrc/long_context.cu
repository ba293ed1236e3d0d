// Segmented forward for long sequences over few heads.
//
// The chunked engine runs one CTA per (batch entry, head) and walks that
// head's chunks in order, so a call with few heads and a long sequence (for
// example B1 T65536 H16: 16 CTAs, 1024 chunks each) leaves most SMs idle.
// The memory recursion is affine in the state ("Kalman Delta Networks:
// Uncertainty-aware Associative Memory", abstract: a gain-weighted delta-rule
// write per token): over a stretch of tokens whose variances are known,
//     S_end = S_start F + E,
// with F (d_k x d_k) the state transition of the stretch and E (d_v x d_k)
// the state the stretch reaches from S_start = 0.  The variance recursion is
// a Mobius map per token and composes by matrix products ("Kalman Linear
// Attention ...", 方法论 §2; the same abstract), so the variance at the start
// of each stretch follows from the composed maps of the stretches before it.
//
// The sequence is cut into S segments of L = T / S tokens, viewed as S extra
// batch entries of the same [B, T, H, d] tensors ([B S, L, H, d] is the same
// memory).  Then:
//   1. every lane composes the Mobius maps of blocks of 512 tokens in
//      parallel, and one pass per lane applies the block products in order,
//      recording the variance at each segment start;
//   2. the engine runs all segments from S_start = 0 (giving E) and, with V
//      read as zero, from S_start = I (giving F: with d_v = d_k the final
//      state is I F);
//   3. a pass per (batch entry, head, block of 16 state rows) chains the
//      segments: S_start(s + 1) = S_start(s) F(s) + E(s);
//   4. the engine runs all segments from their true S_start, writing o and
//      each segment's final state, of which the last segment's is S_T.
// Steps 2 and 4 have S times the heads of the call, at 1/S of its length.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "kdn_common.cuh"

namespace kdn {

kdn_status chunk_engine_launch(bool diag, const void* q, const void* k, const void* v,
                               const float* a, const float* w, const float* r, const float* S0,
                               const float* p0, float* o, float* S_out, float* p_out, int B,
                               int T, int H, int dv, float kappa, void* ws, cudaStream_t s,
                               int debug_skip_v, const int* cu_seqlens);
kdn_status chunk_engine_launch_zero_v(bool diag, const void* q, const void* k, const void* v_zero,
                                      const float* a, const float* w, const float* r,
                                      const float* S0, const float* p0, float* o, float* S_out,
                                      float* p_out, int B, int T, int H, float kappa, void* ws,
                                      cudaStream_t s);

namespace {

constexpr int kD = 128;          // d_k = d_v of the engine
constexpr int kBlock = 512;      // tokens per composed Mobius block
constexpr int kMinSegments = 4;  // three engine passes over 1/S of the tokens each

struct M2 {
  float a, b, c, d;  // [[a, b], [c, d]]
};
// x * y (x the later map)
__device__ __forceinline__ M2 mul(const M2& x, const M2& y) {
  return {fmaf(x.a, y.a, x.b * y.c), fmaf(x.a, y.b, x.b * y.d), fmaf(x.c, y.a, x.d * y.c),
          fmaf(x.c, y.b, x.d * y.d)};
}
// scale by a power of two that brings the largest entry to [1, 2): exact
__device__ __forceinline__ M2 renorm(const M2& x) {
  const float m = fmaxf(fmaxf(x.a, x.b), fmaxf(x.c, x.d));
  const int e = (int)((__float_as_uint(m) >> 23) & 0xffu) - 127;
  if (e > -120 && e < 120) {
    const float sc = __uint_as_float((uint32_t)(127 - e) << 23);
    return {x.a * sc, x.b * sc, x.c * sc, x.d * sc};
  }
  return x;
}
// the variance step p -> r (a^2 p + w) / (c (a^2 p + w) + r) as a matrix
__device__ __forceinline__ M2 step_map(float a, float w, float r, float c) {
  const float a2 = a * a;
  return {r * a2, r * w, c * a2, fmaf(c, w, r)};
}

// Diagonal variant: lanes (b, h, i) for i in a group of 4 dimensions, block
// j of kBlock tokens, composed by kSub threads (consecutive lanes) of
// kBlock / kSub tokens each and joined by an ordered product over those lanes.
// A warp takes 8 consecutive groups (32 dimensions of one head) times kSub
// sub-blocks, so each token's w (16 bytes) and k (8 bytes) reads are 128- and
// 64-byte runs; the four chains of a thread are independent.
constexpr int kSub = 4;
__global__ void __launch_bounds__(256)
block_maps_diag_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ A,
                       const float* __restrict__ W, const float* __restrict__ R, int B, int T,
                       int H, int nblk, float4* __restrict__ prod) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t groups = (int64_t)B * H * (kD / 4);
  // (the thread count is a multiple of 128, so whole warps leave together)
  if (gid >= groups * nblk * kSub) return;
  const int sub = (int)(gid % kSub);
  const int64_t rest = gid / kSub;
  const int j = (int)(rest / groups);
  const int64_t grp = rest % groups;
  const int i0 = (int)(grp % (kD / 4)) * 4;
  const int h = (int)((grp / (kD / 4)) % H);
  const int b = (int)(grp / ((int64_t)(kD / 4) * H));
  const int t0 = min(T, j * kBlock + sub * (kBlock / kSub));
  const int t1 = min(T, t0 + kBlock / kSub);
  M2 P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) P[e] = {1.f, 0.f, 0.f, 1.f};
#pragma unroll 8
  for (int t = t0; t < t1; ++t) {
    const size_t tok = ((size_t)b * T + t) * H + h;
    const float4 w4 = __ldg(reinterpret_cast<const float4*>(W + tok * kD + i0));
    const uint2 k2 = __ldg(reinterpret_cast<const uint2*>(K + tok * kD + i0));
    const float a = __ldg(A + tok), r = __ldg(R + tok);
    const float kv[4] = {__uint_as_float(k2.x << 16), __uint_as_float(k2.x & 0xffff0000u),
                         __uint_as_float(k2.y << 16), __uint_as_float(k2.y & 0xffff0000u)};
    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      P[e] = mul(step_map(a, wv[e], r, kv[e] * kv[e]), P[e]);
      if ((t & 3) == 3) P[e] = renorm(P[e]);
    }
  }
  // ordered product over the kSub lanes: lane sub's tokens follow lane sub - 1's
  const int l = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    M2 Q = renorm(P[e]);
#pragma unroll
    for (int d = 1; d < kSub; d <<= 1) {
      M2 o;
      o.a = __shfl_down_sync(0xffffffffu, Q.a, d);
      o.b = __shfl_down_sync(0xffffffffu, Q.b, d);
      o.c = __shfl_down_sync(0xffffffffu, Q.c, d);
      o.d = __shfl_down_sync(0xffffffffu, Q.d, d);
      if ((l & (2 * d - 1)) == 0) Q = renorm(mul(o, Q));
    }
    P[e] = Q;
  }
  if (sub == 0) {
    const int64_t lane0 = ((int64_t)b * H + h) * kD + i0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      prod[(lane0 + e) * nblk + j] = make_float4(P[e].a, P[e].b, P[e].c, P[e].d);
  }
}

// Isotropic variant: lane (b, h), block j; one warp per (lane, block), lane
// l composing the l-th 1/32 of the block's tokens (c = kappa ||k||^2), then
// the 32 partial products combined in token order.
__global__ void __launch_bounds__(256)
block_maps_iso_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ A,
                      const float* __restrict__ W, const float* __restrict__ R, int B, int T,
                      int H, int nblk, float kappa, float4* __restrict__ prod) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int l = threadIdx.x & 31;
  const int64_t lanes = (int64_t)B * H;
  if (wid >= lanes * nblk) return;  // (whole warps leave together)
  const int j = (int)(wid / lanes);
  const int64_t lane = wid % lanes;
  const int h = (int)(lane % H), b = (int)(lane / H);
  const int t0 = j * kBlock + (kBlock / 32) * l, t1 = min(T, t0 + kBlock / 32);
  M2 P = {1.f, 0.f, 0.f, 1.f};
  for (int t = t0; t < t1; ++t) {
    const size_t tok = ((size_t)b * T + t) * H + h;
    const uint4* kr = reinterpret_cast<const uint4*>(K + tok * kD);
    float n = 0.f;
#pragma unroll
    for (int c = 0; c < kD / 8; ++c) {
      const uint4 u = __ldg(kr + c);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(wv[e] << 16), x1 = __uint_as_float(wv[e] & 0xffff0000u);
        n = fmaf(x0, x0, fmaf(x1, x1, n));
      }
    }
    P = mul(step_map(__ldg(A + tok), __ldg(W + tok), __ldg(R + tok), kappa * n), P);
    if ((t & 3) == 3) P = renorm(P);
  }
  P = renorm(P);
  // ordered product over the warp: lane l's tokens come after lane l - 1's
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    M2 o;
    o.a = __shfl_down_sync(0xffffffffu, P.a, d);
    o.b = __shfl_down_sync(0xffffffffu, P.b, d);
    o.c = __shfl_down_sync(0xffffffffu, P.c, d);
    o.d = __shfl_down_sync(0xffffffffu, P.d, d);
    // lane l holds the product of lanes [l, l + d); combine with [l + d, l + 2 d)
    if ((l & (2 * d - 1)) == 0) P = renorm(mul(o, P));
  }
  if (l == 0) prod[lane * nblk + j] = make_float4(P.a, P.b, P.c, P.d);
}

// Per lane: apply the block products in order from p0, recording the variance
// at the start of every segment (segments are bps blocks long) in the layout
// of the segment view's p0: [(b S + s), H, dim].
__global__ void __launch_bounds__(256)
segment_starts_kernel(const float4* __restrict__ prod, const float* __restrict__ p0, int B,
                      int H, int dim, int nseg, int bps, float* __restrict__ p_start) {
  const int64_t lane = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t lanes = (int64_t)B * H * dim;
  if (lane >= lanes) return;
  const int64_t b = lane / ((int64_t)H * dim), hd = lane % ((int64_t)H * dim);
  float p = p0 ? p0[lane] : 1.f;
  const int nblk = nseg * bps;
  for (int j = 0; j < nblk; ++j) {
    if (j % bps == 0) p_start[((b * nseg) + j / bps) * H * dim + hd] = p;
    const float4 m = prod[lane * nblk + j];
    p = __fdividef(fmaf(m.x, p, m.y), fmaf(m.z, p, m.w));
  }
}

// Identity states for the transition runs: [n][kD][kD].
__global__ void identity_kernel(float* __restrict__ S, int64_t n) {
  const int64_t total = n * kD * kD;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i % (kD * kD);
    S[i] = (e / kD == e % kD) ? 1.f : 0.f;
  }
}

// Segment starts: S_start(0) = S0 (or 0), S_start(s + 1) = S_start(s) F(s) +
// E(s), and after the last segment the call's final state S_T into S_out
// ([B, H, kD, kD]).  One CTA per (batch entry, head, block of 16 rows of S); rows of S
// do not mix, so the blocks are independent.  Each F(s) is staged in shared
// memory (64 KB) with coalesced loads before the products.  State layouts:
// [(b S + s), H, kD, kD] for F, E and S_start; S0 [B, H, kD, kD].
constexpr int kRows = 16;
constexpr size_t kChainSmem = (size_t)(kD * kD + kRows * kD) * sizeof(float);
__global__ void __launch_bounds__(256)
chain_segments_kernel(const float* __restrict__ S0, const float* __restrict__ F,
                      const float* __restrict__ E, int B, int H, int nseg,
                      float* __restrict__ S_start, float* __restrict__ S_out) {
  extern __shared__ float4 chain_smem[];
  float* Fsm = reinterpret_cast<float*>(chain_smem);  // [kD][kD]
  float* cur = Fsm + kD * kD;                         // [kRows][kD]
  const int rb = blockIdx.x % (kD / kRows);
  const int h = (blockIdx.x / (kD / kRows)) % H;
  const int b = blockIdx.x / ((kD / kRows) * H);
  const int tid = threadIdx.x;
  const int r = tid >> 4, c0 = (tid & 15) * 8;  // row r, columns c0 .. c0 + 7
  const int row = rb * kRows + r;
  const auto at = [&](int s) { return ((((size_t)b * nseg + s) * H + h) * kD) * kD; };
  {
    float* dst = S_start + at(0) + (size_t)row * kD + c0;
    const float* src = S0 ? S0 + ((((size_t)b * H + h) * kD) + row) * kD + c0 : nullptr;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = src ? src[e] : 0.f;
      cur[r * kD + c0 + e] = x;
      dst[e] = x;
    }
  }
  for (int s = 0; s < nseg; ++s) {
    const float4* Fs4 = reinterpret_cast<const float4*>(F + at(s));
    for (int i = tid; i < kD * kD / 4; i += 256) chain_smem[i] = __ldg(Fs4 + i);
    __syncthreads();  // F(s) staged; cur written
    const float* Es = E + at(s) + (size_t)row * kD + c0;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = Es[e];
#pragma unroll 4
    for (int j = 0; j < kD; ++j) {
      const float x = cur[r * kD + j];
      const float4 f0 = *reinterpret_cast<const float4*>(Fsm + j * kD + c0);
      const float4 f1 = *reinterpret_cast<const float4*>(Fsm + j * kD + c0 + 4);
      acc[0] = fmaf(x, f0.x, acc[0]);
      acc[1] = fmaf(x, f0.y, acc[1]);
      acc[2] = fmaf(x, f0.z, acc[2]);
      acc[3] = fmaf(x, f0.w, acc[3]);
      acc[4] = fmaf(x, f1.x, acc[4]);
      acc[5] = fmaf(x, f1.y, acc[5]);
      acc[6] = fmaf(x, f1.z, acc[6]);
      acc[7] = fmaf(x, f1.w, acc[7]);
    }
    __syncthreads();  // every thread has read cur and F(s)
    // (after the last segment: the final state of the call)
    float* dst = s + 1 < nseg ? S_start + at(s + 1) + (size_t)row * kD + c0
                              : S_out + ((((size_t)b * H + h) * kD) + row) * kD + c0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cur[r * kD + c0 + e] = acc[e];
      dst[e] = acc[e];
    }
  }
}

__global__ void or_error_words(uint32_t* dst, const uint32_t* a, const uint32_t* b,
                               const uint32_t* c) {
  atomicOr(dst, *a | *b | *c);
}

// ----------------------------------------------------- output correction
// o(t) = o_E(t) + S_start o_F(t) for every token of a segment: the pass from
// S_start = I with V = 0 reads out o_F(t) = F_(0..t) q_t, so the state at
// token t, S_start F_(0..t) + E_t, gives the output through one matrix
// product per token.  Per (segment, head) it is a [128 v x 128 k] x [128 k x
// tokens] product, D[v][t] = sum_k S_start[v][k] o_F[t][k], on the tensor
// cores in tf32 (both operands fp32 in shared memory, K-major, 128-byte
// swizzle; the correction's relative error is about 2^-10 of its size, well
// inside the output bound), with the fp32 accumulator in TMEM.  One CTA of
// eight warps per (segment, head, 8 or 4 tiles of 128 tokens): S_start comes
// in once, each token tile by TMA, 16 MMAs of K = 8, then each thread (one
// value row v, half of the tile's tokens; two warps per TMEM lane quarter)
// adds its TMEM row to o in place, 32 tokens at a time, coalesced over v.
constexpr int kCorrTiles = 8;  // token tiles of 128 per CTA (4 when 8 does not divide a segment)
constexpr uint32_t kOperandBytes = 128u * 128u * 4u;  // 64 KB, [4 kb][128 rows][32 k]
constexpr uint32_t kCorrSmem = 2 * kOperandBytes + 1024 + 64;

__device__ __forceinline__ void umma_tf32_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__global__ void __launch_bounds__(256, 1)
correct_outputs_kernel(const __grid_constant__ CUtensorMap tm_s,
                       const __grid_constant__ CUtensorMap tm_of, float* __restrict__ O, int H,
                       int L, int ntile, uint32_t* __restrict__ err) {
  extern __shared__ uint8_t corr_raw[];
  uint8_t* smem = corr_raw + ((1024u - (smem_u32(corr_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;                    // S_start [4 kb][128 v][32 k]
  uint8_t* sB = smem + kOperandBytes;    // o_F tile [4 kb][128 t][32 k]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kOperandBytes);
  uint64_t* full_a = bars;
  uint64_t* full_b = bars + 1;
  uint64_t* mma_done = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  __shared__ int s_bad;

  const int groups = (L / 128) / ntile;
  const int g = blockIdx.x % groups;
  const int h = (blockIdx.x / groups) % H;
  const int bs = blockIdx.x / (groups * H);  // segment (b, s) of the [B S, L, H, d] view
  const int tid = threadIdx.x, warp = tid >> 5;

  if (tid == 0) {
    mbar_init(full_a, 1);
    mbar_init(full_b, 1);
    mbar_init(mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_bad = 0;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto load_b = [&](int tile) {
    mbar_expect_tx(full_b, kOperandBytes);
    for (int kb = 0; kb < 4; ++kb)
      tma_load_4d(sB + kb * 16384, &tm_of, full_b, 32 * kb, h, 128 * tile, bs);
  };
  const int tile0 = g * ntile;
  if (tid == 0) {
    mbar_expect_tx(full_a, kOperandBytes);
    for (int kb = 0; kb < 4; ++kb)
      tma_load_4d(sA + kb * 16384, &tm_s, full_a, 32 * kb, 0, h, bs);
    load_b(tile0);
  }
  constexpr uint32_t IDESC = umma_idesc(128, 128, 2, 0, 0);  // tf32, both K-major
  bool bad = !mbar_wait(full_a, 0);
  for (int i = 0; i < ntile; ++i) {
    if (!bad && !mbar_wait(full_b, (uint32_t)(i & 1))) bad = true;
    if (tid == 0 && !bad) {
      tc_fence_after();
      const uint64_t da = umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t db = umma_desc_sw128(smem_u32(sB), 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const uint64_t off = (uint64_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        umma_tf32_ss(tmem, da + off, db + off, IDESC, ks > 0 ? 1u : 0u);
      }
      umma_commit(mma_done);
    }
    if (!bad && !mbar_wait(mma_done, (uint32_t)(i & 1))) bad = true;
    if (__syncthreads_or(bad)) {
      if (tid == 0) {
        atomicOr(err, DEV_TIMEOUT);
        s_bad = 1;
      }
      break;
    }
    tc_fence_after();
    // the tile's operand has been read: copy the next one during the epilogue
    if (tid == 0 && i + 1 < ntile) load_b(tile0 + i + 1);
    const int t0 = 128 * (tile0 + i);
    // warp w reads TMEM lanes [32 (w % 4), + 32) (v) and column blocks 2 (w / 4), + 1
    const int v = 32 * (warp & 3) + (tid & 31);
    float* orow = O + (((size_t)bs * L + t0) * H + h) * 128 + v;
    const size_t tstride = (size_t)H * 128;
#pragma unroll 1
    for (int c = 2 * (warp >> 2); c < 2 * (warp >> 2) + 2; ++c) {
      // the 32 o_E values first (all loads in flight at once), then the
      // TMEM columns, then the sums
      float e[32], d[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) e[j] = __ldcs(orow + (size_t)(32 * c + j) * tstride);
      tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 32 * c, d);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) __stcs(orow + (size_t)(32 * c + j) * tstride, e[j] + d[j]);
    }
    tc_fence_before();
    __syncthreads();  // every thread has read D before the next MMA writes it
  }
  if (tid == 0 && s_bad) {
    // bounded waits for what may still be in flight
    (void)mbar_wait(mma_done, 0);
    (void)mbar_wait(full_b, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// fp32 4-D map, 128-byte swizzle, box (32, box1, box2, 1)
bool make_f32_map(CUtensorMap* m, const void* base, const cuuint64_t (&dims)[4], int box1,
                  int box2) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t strides[3] = {dims[0] * 4, dims[0] * dims[1] * 4, dims[0] * dims[1] * dims[2] * 4};
  cuuint32_t box[4] = {32, (cuuint32_t)box1, (cuuint32_t)box2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct SegLayout {
  size_t err_e, err_f, err_g, prod, p_start, p_scratch, p_scratch2, ident, E, F, S_start, zero_v,
      o_f, total;
};

// Workspace: the call's error word (bytes 0-3, first 256-byte block), one
// error word per engine pass, then the segment data.
SegLayout seg_layout(bool diag, int B, int T, int H, int nseg) {
  SegLayout L{};
  size_t off = 256;
  auto take = [&](size_t n) {
    const size_t at = off;
    off = up256(off + n);
    return at;
  };
  const int dim = diag ? kD : 1;
  const size_t states = (size_t)B * nseg * H * kD * kD * 4;
  const size_t vars = (size_t)B * nseg * H * dim * 4;
  L.err_e = take(256);
  L.err_f = take(256);
  L.err_g = take(256);
  L.prod = take((size_t)B * H * dim * (T / kBlock) * 16);
  L.p_start = take(vars);
  L.p_scratch = take(vars);
  L.p_scratch2 = take(vars);
  L.ident = take(states);
  L.E = take(states);
  L.F = take(states);
  L.S_start = take(states);
  L.zero_v = take((size_t)64 * H * kD * 2);
  L.o_f = take((size_t)B * T * H * kD * 4);  // output of the S_start = I pass
  L.total = off;
  return L;
}

}  // namespace

// Number of segments for a call of the d_v = 128 engine on the current
// device: the largest power of two S >= 4 with B H S CTAs fitting on the SMs
// at once and T a multiple of 512 S (whole composed blocks per segment), or
// 1 (no segmentation).
int segment_count(int B, int T, int H) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 1;
  const int64_t heads = (int64_t)B * H;
  int S = 1;
  while ((int64_t)heads * S * 2 <= sms && T % (kBlock * S * 2) == 0) S *= 2;
  return S >= kMinSegments ? S : 1;
}

size_t segmented_workspace_size(bool diag, int B, int T, int H, int nseg) {
  return seg_layout(diag, B, T, H, nseg).total;
}

kdn_status segmented_forward(bool diag, const void* q, const void* k, const void* v,
                             const float* a, const float* w, const float* r, const float* S0,
                             const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                             int H, float kappa, int nseg, void* ws, cudaStream_t st) {
  const SegLayout L = seg_layout(diag, B, T, H, nseg);
  char* base = static_cast<char*>(ws);
  const int dim = diag ? kD : 1;
  const int Bs = B * nseg, Ls = T / nseg;
  const int nblk = T / kBlock, bps = nblk / nseg;
  float4* prod = reinterpret_cast<float4*>(base + L.prod);
  float* p_start = reinterpret_cast<float*>(base + L.p_start);
  float* p_scratch = reinterpret_cast<float*>(base + L.p_scratch);
  float* ident = reinterpret_cast<float*>(base + L.ident);
  float* E = reinterpret_cast<float*>(base + L.E);
  float* F = reinterpret_cast<float*>(base + L.F);
  float* S_start = reinterpret_cast<float*>(base + L.S_start);
  if (cudaMemsetAsync(ws, 0, 4, st) != cudaSuccess) return KDN_ERR_CUDA;
  if (cudaMemsetAsync(base + L.zero_v, 0, (size_t)64 * H * kD * 2, st) != cudaSuccess)
    return KDN_ERR_CUDA;

  // 1. variances at the segment starts
  const int64_t lanes = (int64_t)B * H * dim;
  if (diag) {
    const int64_t n = lanes / 4 * nblk * kSub;
    block_maps_diag_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), a, w, r, B, T, H, nblk, prod);
  } else {
    const int64_t nthr = lanes * nblk * 32;
    block_maps_iso_kernel<<<(unsigned)((nthr + 255) / 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), a, w, r, B, T, H, nblk, kappa, prod);
  }
  segment_starts_kernel<<<(unsigned)((lanes + 255) / 256), 256, 0, st>>>(prod, p0, B, H, dim,
                                                                         nseg, bps, p_start);
  identity_kernel<<<592, 256, 0, st>>>(ident, (int64_t)Bs * H);
  if (cudaGetLastError() != cudaSuccess) return KDN_ERR_CUDA;

  // 2. every segment from S_start = 0 (E; o_E into o), and with V read as
  // zero from S_start = I (F; o_F(t) = F_(0..t) q_t into the workspace)
  float* o_f = reinterpret_cast<float*>(base + L.o_f);
  float* p_scratch2 = reinterpret_cast<float*>(base + L.p_scratch2);
  kdn_status stt = chunk_engine_launch(diag, q, k, v, a, w, r, nullptr, p_start, o, E, p_scratch,
                                       Bs, Ls, H, kD, kappa, base + L.err_e, st, -1, nullptr);
  if (stt != KDN_OK) return stt;
  stt = chunk_engine_launch_zero_v(diag, q, k, base + L.zero_v, a, w, r, ident, p_start, o_f, F,
                                   p_scratch2, Bs, Ls, H, kappa, base + L.err_f, st);
  if (stt != KDN_OK) return stt;

  // 3. the true state at every segment start, and the final state
  if (cudaFuncSetAttribute(chain_segments_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kChainSmem) != cudaSuccess)
    return KDN_ERR_CUDA;
  chain_segments_kernel<<<(unsigned)(B * H * (kD / kRows)), 256, kChainSmem, st>>>(
      S0, F, E, B, H, nseg, S_start, S_out);
  if (cudaGetLastError() != cudaSuccess) return KDN_ERR_CUDA;

  // 4. o += S_start o_F on every segment (segment 0 of each batch entry too,
  // unless it starts from zero)
  CUtensorMap tm_s, tm_of;
  const cuuint64_t sdims[4] = {(cuuint64_t)kD, (cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)Bs};
  const cuuint64_t odims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)Ls, (cuuint64_t)Bs};
  if (!make_f32_map(&tm_s, S_start, sdims, kD, 1) || !make_f32_map(&tm_of, o_f, odims, 1, 128))
    return KDN_ERR_CUDA;
  if (cudaFuncSetAttribute(correct_outputs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kCorrSmem) != cudaSuccess)
    return KDN_ERR_CUDA;
  if (cudaMemsetAsync(base + L.err_g, 0, 4, st) != cudaSuccess) return KDN_ERR_CUDA;
  // (every segment: the first of each batch entry adds S0 o_F, zero without S0)
  const int ntile = (Ls / 128) % kCorrTiles == 0 ? kCorrTiles : 4;
  const int groups = (Ls / 128) / ntile;
  correct_outputs_kernel<<<(unsigned)(Bs * H * groups), 256, kCorrSmem, st>>>(
      tm_s, tm_of, o, H, Ls, ntile, reinterpret_cast<uint32_t*>(base + L.err_g));
  if (cudaGetLastError() != cudaSuccess) return KDN_ERR_CUDA;

  // the call's final variance: the end variance of the last segment
  const size_t pbytes = (size_t)H * dim * 4;
  if (cudaMemcpy2DAsync(p_out, pbytes, p_scratch + (size_t)(nseg - 1) * H * dim, pbytes * nseg,
                        pbytes, B, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return KDN_ERR_CUDA;
  or_error_words<<<1, 1, 0, st>>>(static_cast<uint32_t*>(ws),
                                  reinterpret_cast<const uint32_t*>(base + L.err_e),
                                  reinterpret_cast<const uint32_t*>(base + L.err_f),
                                  reinterpret_cast<const uint32_t*>(base + L.err_g));
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

}  // namespace kdn
