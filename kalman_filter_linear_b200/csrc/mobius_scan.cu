// kdn_mobius_scan: the KDN uncertainty recursion over N independent lanes.
//
// Each step of a lane is the Mobius map of the variance,
//   p_t = (r a^2 p + r w) / (c a^2 p + r + c w),   c = info_scale * n,
// i.e. the 2x2 matrix M_t = [[r a^2, r w], [c a^2, r + c w]] acting
// projectively ("Kalman Delta Networks: Uncertainty-aware Associative
// Memory", abstract: the recursion is a Mobius map and composes by an
// associative scan; "Kalman Linear Attention ...", 方法论 §2: O(T) work,
// O(log T) depth).  Prefix compositions P_t = M_t ... M_1 (later maps on the
// left) give p_t = P_t(p_0).
//
// Kernel layout (one CTA per 2048-token tile of one lane):
//   1. 256 threads load 8 consecutive steps each (two 16-byte loads per
//      array), build their maps and compose them serially in registers;
//   2. warp-shuffle inclusive scan of the thread products, then a block scan
//      of the 8 warp totals (through shared memory, one barrier; every warp
//      scans them itself);
//   3. decoupled look-back across the tiles of the lane: a tile publishes its
//      inclusive prefix at once when its predecessor's was published as the
//      tile started (the usual case), else its aggregate first, then the
//      inclusive prefix once it has combined the predecessors' published
//      values (thread 0, while the other threads wait at a second barrier).
//      Tiles are handed out by an atomic counter in tile-index-major order
//      (all lanes' tile 0 first), so a predecessor has almost always
//      finished already.  Every wait is
//      bounded in wall-clock time; a wait that gives up records
//      DEV_TIMEOUT in the workspace error word and the tile goes on with
//      what it has.
//   4. each thread applies its exclusive prefix to p_0 and runs the scalar
//      recursion over its 8 steps, writing p (and optionally p^- and the
//      isotropic write strength).
// All products have non-negative entries (no cancellation).  They are
// renormalised by powers of two, which is exact, so renormalisation adds no
// rounding.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "kdn_common.cuh"

namespace kdn {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kTile = kThreads * kPerThread;  // 2048 steps
static_assert(kPerThread % 4 == 0 && kThreads % 32 == 0, "tile shape");

struct Mat2 {
  float a, b, c, d;  // [[a, b], [c, d]]
};

__device__ __forceinline__ Mat2 identity() { return {1.f, 0.f, 0.f, 1.f}; }

// x * y (x is the later map).
__device__ __forceinline__ Mat2 mul(const Mat2& x, const Mat2& y) {
  Mat2 z;
  z.a = fmaf(x.a, y.a, x.b * y.c);
  z.b = fmaf(x.a, y.b, x.b * y.d);
  z.c = fmaf(x.c, y.a, x.d * y.c);
  z.d = fmaf(x.c, y.b, x.d * y.d);
  return z;
}

// Scale by 2^-e where 2^e is the binade of the largest entry.  Exact.
__device__ __forceinline__ Mat2 renorm(const Mat2& x) {
  const float m = fmaxf(fmaxf(x.a, x.b), fmaxf(x.c, x.d));
  const int e = (int)((__float_as_uint(m) >> 23) & 0xffu) - 127;
  if (e > -100 && e < 100 && e != 0) {
    const float s = __uint_as_float((uint32_t)(127 - e) << 23);
    return {x.a * s, x.b * s, x.c * s, x.d * s};
  }
  return x;
}

__device__ __forceinline__ float apply(const Mat2& m, float lam) {
  return __fdividef(fmaf(m.a, lam, m.b), fmaf(m.c, lam, m.d));
}

__device__ __forceinline__ Mat2 shfl_up(const Mat2& x, int delta) {
  return {__shfl_up_sync(0xffffffffu, x.a, delta), __shfl_up_sync(0xffffffffu, x.b, delta),
          __shfl_up_sync(0xffffffffu, x.c, delta), __shfl_up_sync(0xffffffffu, x.d, delta)};
}

// (lane, tile index within the lane) of a tile.  Tiles number below 2^31
// (checked on the host), so 32-bit division does.
__device__ __forceinline__ void split_tile(int64_t tile, int64_t N, int64_t& j, int64_t& seq) {
  const uint32_t t = (uint32_t)tile, n = (uint32_t)N;
  const uint32_t q = t / n;
  j = q;
  seq = t - q * n;
}

struct ScanWs {
  uint32_t* error;    // device error word
  uint32_t* counter;  // next tile to hand out
  uint32_t* flag;     // per tile: 0 none, 1 aggregate, 2 inclusive prefix
  float4* agg;        // per tile aggregate
  float4* incl;       // per tile inclusive prefix
};

__device__ __forceinline__ float4 as_f4(const Mat2& m) { return make_float4(m.a, m.b, m.c, m.d); }
__device__ __forceinline__ Mat2 as_mat(const float4& f) { return {f.x, f.y, f.z, f.w}; }

struct TileShared {
  Mat2 warp_incl[kThreads / 32];
  Mat2 tile_prefix;
  Mat2 pred_incl;    // the predecessor's inclusive prefix, when published
  uint32_t pred_ok;  // 1: it was published when this tile started
};

// The decoupled look-back of tile `tile` (index j in lane seq) whose
// predecessor had not published its inclusive prefix when the tile started
// (its flag then: f_pre): publish the aggregate, combine the predecessors'
// aggregates back to the first inclusive prefix, publish this tile's.
// Returns the tile's exclusive prefix.
__device__ __forceinline__ Mat2 look_back(const ScanWs& ws, int64_t tile, int64_t j, int64_t seq,
                                       int64_t N, uint32_t f_pre, Mat2 agg, bool skip_publish) {
  Mat2 excl = identity();
  if (!skip_publish) {
    ws.agg[tile] = as_f4(agg);
    st_release_u32(ws.flag + tile, 1u);
  }
  const uint64_t start = globaltimer_ns();
  bool timed_out = false;
  uint32_t f0 = f_pre;
  for (int64_t p = j - 1; p >= 0 && !timed_out;) {
    const int64_t pt = p * N + seq;
    uint32_t f = (p == j - 1) ? f0 : ld_acquire_u32(ws.flag + pt);
    while (f == 0u) {
      if (globaltimer_ns() - start > kWaitLimitNs) {
        timed_out = true;
        break;
      }
      __nanosleep(64);
      f = ld_acquire_u32(ws.flag + pt);
    }
    if (timed_out) break;
    if (f == 2u) {
      excl = renorm(mul(excl, as_mat(__ldcg(ws.incl + pt))));
      break;
    }
    excl = renorm(mul(excl, as_mat(__ldcg(ws.agg + pt))));
    f0 = 0u;
    --p;
  }
  if (timed_out) atomicOr(ws.error, DEV_TIMEOUT);
  if (!skip_publish) {
    ws.incl[tile] = as_f4(renorm(mul(agg, excl)));
    st_release_u32(ws.flag + tile, 2u);
  }
  return excl;
}

// Steps 1-4 for one tile, given this thread's 8 inputs (a, w, r, n).
__device__ __forceinline__ void scan_tile(const float (&a)[kPerThread], const float (&w)[kPerThread],
                                          const float (&r)[kPerThread], const float (&n)[kPerThread],
                                          int64_t tile, const float* __restrict__ lambda0,
                                          float info_scale, float* __restrict__ lam_out,
                                          float* __restrict__ prior_out,
                                          float* __restrict__ gain_out, int64_t N, int64_t T,
                                          const ScanWs& ws, int vec_ok, int64_t debug_skip_tile,
                                          TileShared& sh) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  int64_t j, seq;  // tile index within the lane, lane
  split_tile(tile, N, j, seq);
  const int64_t t0 = j * kTile + (int64_t)tid * kPerThread;
  const int64_t base = seq * T;
  Mat2* s_warp = sh.warp_incl;
  // The predecessor's inclusive prefix is usually published already: ask for
  // it now, so that the read overlaps this tile's local scan.
  const int64_t pt0 = (j - 1) * N + seq;
  uint32_t f_pre = 0u;
  float4 incl_pre = make_float4(1.f, 0.f, 0.f, 1.f);
  if (tid == 0 && j > 0) {
    f_pre = ld_acquire_u32(ws.flag + pt0);
    incl_pre = __ldcg(ws.incl + pt0);
  }

  // (steps past the end of the lane come in as identity steps: a = r = 1,
  // w = n = 0)
  Mat2 P = identity();
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const float c = info_scale * n[i];
    const float a2 = a[i] * a[i];
    const Mat2 M = {r[i] * a2, r[i] * w[i], c * a2, fmaf(c, w[i], r[i])};
    P = mul(M, P);
    if (i & 1) P = renorm(P);
  }

  // ---- 2. warp inclusive scan, then block scan of warp totals
  Mat2 incl = P;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const Mat2 prev = shfl_up(incl, d);
    if (lane >= d) incl = renorm(mul(incl, prev));
  }
  if (lane == 31) s_warp[warp] = incl;
  if (tid == 0) {
    sh.pred_ok = (j == 0 || f_pre == 2u) ? 1u : 0u;
    sh.pred_incl = j == 0 ? identity() : as_mat(incl_pre);
  }
  __syncthreads();
  // ---- block scan of the warp totals, in every warp.  Warp 0 takes the
  // tile's aggregate from it (its thread 0 publishes), every other warp the
  // product over the warps before it.
  Mat2 x = lane < kThreads / 32 ? s_warp[lane] : identity();
#pragma unroll
  for (int d = 1; d < kThreads / 32; d <<= 1) {
    const Mat2 prev = shfl_up(x, d);
    if (lane >= d) x = renorm(mul(x, prev));
  }
  const int src = warp > 0 ? warp - 1 : kThreads / 32 - 1;
  const Mat2 blk = {__shfl_sync(0xffffffffu, x.a, src), __shfl_sync(0xffffffffu, x.b, src),
                    __shfl_sync(0xffffffffu, x.c, src), __shfl_sync(0xffffffffu, x.d, src)};
  const Mat2& agg = blk;  // (warp 0)
  // this thread's prefix within the tile (warps 1-7: blk is the product over
  // the warps before)
  Mat2 thread_excl = shfl_up(incl, 1);
  if (lane == 0) thread_excl = identity();
  if (warp > 0) thread_excl = mul(thread_excl, blk);
  thread_excl = renorm(thread_excl);
  // ---- 3. the tile's prefix.  Usually the predecessor had published its
  // inclusive prefix when this tile started (thread 0 read it then): every
  // thread takes it from shared memory and no second barrier is needed.
  // Otherwise thread 0 publishes the aggregate and looks back tile by tile
  // while the others wait at a barrier (the choice is the same in every
  // thread: all read one shared flag).  The release store of a flag orders
  // this thread's earlier stores of the prefix data before it.
  const bool skip_publish = (tile == debug_skip_tile);  // fault-injection hook
  Mat2 tile_prefix;
  if (sh.pred_ok) {
    tile_prefix = sh.pred_incl;
    if (tid == 0 && !skip_publish) {
      ws.incl[tile] = as_f4(j == 0 ? agg : renorm(mul(agg, tile_prefix)));
      st_release_u32(ws.flag + tile, 2u);
    }
  } else {
    if (tid == 0) sh.tile_prefix = look_back(ws, tile, j, seq, N, f_pre, agg, skip_publish);
    __syncthreads();
    tile_prefix = sh.tile_prefix;
  }

  // ---- 4. apply the exclusive prefix and run the recursion
  thread_excl = renorm(mul(thread_excl, tile_prefix));
  const float lam0 = lambda0 ? __ldg(lambda0 + seq) : 1.f;
  float lam = apply(thread_excl, lam0);

  float out_l[kPerThread], out_p[kPerThread], out_g[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const float prior = fmaf(a[i] * a[i], lam, w[i]);
    const float c = info_scale * n[i];
    lam = __fdividef(r[i] * prior, fmaf(c, prior, r[i]));
    out_l[i] = lam;
    out_p[i] = prior;
    out_g[i] = __fdividef(prior, fmaf(prior, n[i], r[i]));
  }
  if (vec_ok && t0 + kPerThread <= T) {
    float4* l4 = reinterpret_cast<float4*>(lam_out + base + t0);
#pragma unroll
    for (int h = 0; h < kPerThread / 4; ++h)
      l4[h] = make_float4(out_l[4 * h], out_l[4 * h + 1], out_l[4 * h + 2], out_l[4 * h + 3]);
    if (prior_out) {
      float4* p4 = reinterpret_cast<float4*>(prior_out + base + t0);
#pragma unroll
      for (int h = 0; h < kPerThread / 4; ++h)
        p4[h] = make_float4(out_p[4 * h], out_p[4 * h + 1], out_p[4 * h + 2], out_p[4 * h + 3]);
    }
    if (gain_out) {
      float4* g4 = reinterpret_cast<float4*>(gain_out + base + t0);
#pragma unroll
      for (int h = 0; h < kPerThread / 4; ++h)
        g4[h] = make_float4(out_g[4 * h], out_g[4 * h + 1], out_g[4 * h + 2], out_g[4 * h + 3]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      if (t0 + i < T) {
        lam_out[base + t0 + i] = out_l[i];
        if (prior_out) prior_out[base + t0 + i] = out_p[i];
        if (gain_out) gain_out[base + t0 + i] = out_g[i];
      }
    }
  }
}

// One tile per CTA, inputs straight from global memory (any T).
__global__ void __launch_bounds__(kThreads)
mobius_scan_kernel(const float* __restrict__ A, const float* __restrict__ W,
                   const float* __restrict__ R, const float* __restrict__ Nsq,
                   const float* __restrict__ lambda0, float info_scale,
                   float* __restrict__ lam_out, float* __restrict__ prior_out,
                   float* __restrict__ gain_out, int64_t N, int64_t T, ScanWs ws, int vec_ok,
                   int64_t debug_skip_tile) {
  __shared__ TileShared sh;
  __shared__ uint32_t s_tile;
  const int tid = threadIdx.x;
  if (tid == 0) s_tile = atomicAdd(ws.counter, 1u);
  __syncthreads();
  const int64_t tile = s_tile;
  int64_t j, seq;
  split_tile(tile, N, j, seq);
  const int64_t t0 = j * kTile + (int64_t)tid * kPerThread;
  const int64_t base = seq * T;
  float a[kPerThread], w[kPerThread], r[kPerThread], n[kPerThread];
  if (vec_ok && t0 + kPerThread <= T) {
    const float4* a4 = reinterpret_cast<const float4*>(A + base + t0);
    const float4* w4 = reinterpret_cast<const float4*>(W + base + t0);
    const float4* r4 = reinterpret_cast<const float4*>(R + base + t0);
    const float4* n4 = reinterpret_cast<const float4*>(Nsq + base + t0);
#pragma unroll
    for (int h = 0; h < kPerThread / 4; ++h) {
      float4 x = __ldg(a4 + h), y = __ldg(w4 + h), z = __ldg(r4 + h), u = __ldg(n4 + h);
      a[4 * h] = x.x; a[4 * h + 1] = x.y; a[4 * h + 2] = x.z; a[4 * h + 3] = x.w;
      w[4 * h] = y.x; w[4 * h + 1] = y.y; w[4 * h + 2] = y.z; w[4 * h + 3] = y.w;
      r[4 * h] = z.x; r[4 * h + 1] = z.y; r[4 * h + 2] = z.z; r[4 * h + 3] = z.w;
      n[4 * h] = u.x; n[4 * h + 1] = u.y; n[4 * h + 2] = u.z; n[4 * h + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const bool in = t0 + i < T;
      a[i] = in ? __ldg(A + base + t0 + i) : 1.f;
      w[i] = in ? __ldg(W + base + t0 + i) : 0.f;
      r[i] = in ? __ldg(R + base + t0 + i) : 1.f;
      n[i] = in ? __ldg(Nsq + base + t0 + i) : 0.f;
    }
  }
  scan_tile(a, w, r, n, tile, lambda0, info_scale, lam_out, prior_out, gain_out, N, T, ws, vec_ok,
            debug_skip_tile, sh);
}

// Persistent form for T a multiple of 4: each CTA takes tiles in counter
// order.  Once its threads have moved a tile's inputs into registers, it
// copies the next tile's inputs into the shared-memory buffer (bulk async
// copies) while it scans the current tile, so input traffic is in flight
// during the look-back and the recursion.  A CTA takes the next tile before
// it finishes the current one; every tile it waits on has a smaller index and
// was taken earlier, so some CTA is working on it.
constexpr uint32_t kTileBytes = kTile * 4;  // one input array of a tile
constexpr uint32_t kBufBytes = 4 * kTileBytes;
constexpr int kPersistentCtasPerSm = 4;

__global__ void __launch_bounds__(kThreads, kPersistentCtasPerSm)
mobius_scan_persistent(const float* __restrict__ A, const float* __restrict__ W,
                       const float* __restrict__ R, const float* __restrict__ Nsq,
                       const float* __restrict__ lambda0, float info_scale,
                       float* __restrict__ lam_out, float* __restrict__ prior_out,
                       float* __restrict__ gain_out, int64_t N, int64_t T, int64_t ntiles,
                       ScanWs ws, int64_t debug_skip_tile) {
  extern __shared__ __align__(128) uint8_t s_in[];  // [a, w, r, n][kTile] fp32
  __shared__ TileShared sh;
  __shared__ int64_t s_tile[2];
  __shared__ uint64_t s_full;
  const int tid = threadIdx.x;
  // copies the inputs of `tile` into the buffer (thread 0)
  auto fetch = [&](int64_t tile) {
    const float* src[4] = {A, W, R, Nsq};
    int64_t j, seq;
    split_tile(tile, N, j, seq);
    const int64_t first = j * kTile;
    const uint32_t bytes = (uint32_t)(min((int64_t)kTile, T - first) * 4);
    mbar_expect_tx(&s_full, 4u * bytes);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(smem_u32(s_in + k * kTileBytes)), "l"(src[k] + seq * T + first), "r"(bytes),
          "r"(smem_u32(&s_full))
          : "memory");
    }
  };
  if (tid == 0) {
    mbar_init(&s_full, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const int64_t first = atomicAdd(ws.counter, 1u);
    s_tile[0] = first;
    if (first < ntiles) fetch(first);
  }
  __syncthreads();
  for (int it = 0;; ++it) {
    const int64_t tile = s_tile[it & 1];
    if (tile >= ntiles) break;
    // this tile's inputs; if any thread's wait gives up, the CTA records the
    // timeout and stops
    const bool late = !mbar_wait(&s_full, (uint32_t)(it & 1));
    if (__syncthreads_or(late)) {
      if (tid == 0) {
        atomicOr(ws.error, DEV_TIMEOUT);
        // the copy may still land in this CTA's buffer: give it one more
        // bounded wait before the CTA exits and its shared memory is reused
        (void)mbar_wait(&s_full, (uint32_t)(it & 1));
      }
      break;
    }
    int64_t j, seq;
    split_tile(tile, N, j, seq);
    const int64_t t0 = j * kTile + (int64_t)tid * kPerThread;
    const float* buf = reinterpret_cast<const float*>(s_in);
    float a[kPerThread], w[kPerThread], r[kPerThread], n[kPerThread];
#pragma unroll
    for (int h = 0; h < kPerThread / 4; ++h) {
      const float4 x = *reinterpret_cast<const float4*>(buf + 0 * kTile + tid * kPerThread + 4 * h);
      const float4 y = *reinterpret_cast<const float4*>(buf + 1 * kTile + tid * kPerThread + 4 * h);
      const float4 z = *reinterpret_cast<const float4*>(buf + 2 * kTile + tid * kPerThread + 4 * h);
      const float4 u = *reinterpret_cast<const float4*>(buf + 3 * kTile + tid * kPerThread + 4 * h);
      a[4 * h] = x.x; a[4 * h + 1] = x.y; a[4 * h + 2] = x.z; a[4 * h + 3] = x.w;
      w[4 * h] = y.x; w[4 * h + 1] = y.y; w[4 * h + 2] = y.z; w[4 * h + 3] = y.w;
      r[4 * h] = z.x; r[4 * h + 1] = z.y; r[4 * h + 2] = z.z; r[4 * h + 3] = z.w;
      n[4 * h] = u.x; n[4 * h + 1] = u.y; n[4 * h + 2] = u.z; n[4 * h + 3] = u.w;
    }
    __syncthreads();  // the buffer is free: start the next tile's copies
    if (tid == 0) {
      const int64_t next = atomicAdd(ws.counter, 1u);
      s_tile[(it + 1) & 1] = next;
      if (next < ntiles) fetch(next);
    }
    if (t0 + kPerThread > T) {
      const int nvalid = (int)max((int64_t)0, T - t0);
#pragma unroll
      for (int i = 0; i < kPerThread; ++i)
        if (i >= nvalid) {  // past the end of the lane: identity steps
          a[i] = 1.f;
          w[i] = 0.f;
          r[i] = 1.f;
          n[i] = 0.f;
        }
    }
    scan_tile(a, w, r, n, tile, lambda0, info_scale, lam_out, prior_out, gain_out, N, T, ws, 1,
              debug_skip_tile, sh);
    // (the next iteration's first barrier keeps the shared tile state until
    // every thread is done with it)
  }
  // A copy is started only for a tile below ntiles, and the next iteration
  // waits for it, so on the normal path nothing is in flight at exit.  After
  // a timeout the CTA waits for the late copy once more (bounded); if that
  // wait gives up too, the copy can still be in flight when the CTA exits.
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct ScanLayout {
  int64_t tiles_per_lane, ntiles;
  size_t off_flag, off_agg, off_incl, total, clear_bytes;
};

inline ScanLayout scan_layout(int64_t N, int64_t T) {
  ScanLayout L;
  L.tiles_per_lane = (T + kTile - 1) / kTile;
  L.ntiles = L.tiles_per_lane * N;
  L.off_flag = 256;
  L.off_agg = align_up(L.off_flag + (size_t)L.ntiles * 4, 256);
  L.off_incl = align_up(L.off_agg + (size_t)L.ntiles * 16, 256);
  L.total = align_up(L.off_incl + (size_t)L.ntiles * 16, 256);
  L.clear_bytes = L.off_flag + (size_t)L.ntiles * 4;
  return L;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// CTAs of the persistent kernel that fit on the current device at once (its
// SM count times the CTAs per SM), found once per device with that device
// current; 0 on a CUDA error.  Devices may differ, so the value is kept per
// device ordinal, and the first calls from several host threads agree
// through the lock.
constexpr int kCapDevices = 64;
std::atomic<int> g_grid_cap[kCapDevices];
std::mutex g_grid_cap_mu;

int persistent_grid_cap() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < kCapDevices) {
    const int cap = g_grid_cap[dev].load(std::memory_order_acquire);
    if (cap > 0) return cap;
  }
  std::lock_guard<std::mutex> lock(g_grid_cap_mu);
  if (dev < kCapDevices) {
    const int cap = g_grid_cap[dev].load(std::memory_order_acquire);
    if (cap > 0) return cap;
  }
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaFuncSetAttribute(mobius_scan_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kBufBytes) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mobius_scan_persistent, kThreads,
                                                    kBufBytes) != cudaSuccess ||
      per_sm < 1 || sms < 1)
    return 0;
  if (dev < kCapDevices) g_grid_cap[dev].store(sms * per_sm, std::memory_order_release);
  return sms * per_sm;
}

}  // namespace

size_t mobius_scan_workspace_size(int64_t N, int64_t T) {
  if (N <= 0 || T <= 0) return 0;
  return scan_layout(N, T).total;
}

kdn_status mobius_scan_launch(const float* a, const float* w, const float* r, const float* n,
                              const float* lambda0, float info_scale, float* lambda_out,
                              float* prior_out, float* gain_out, int64_t N, int64_t T,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream,
                              int64_t debug_skip_tile) {
  if (!a || !w || !r || !n || !lambda_out) return KDN_ERR_INVALID_ARG;
  if (N <= 0 || T <= 0 || N * T >= (int64_t(1) << 40)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale >= 0.f) || !(info_scale < 3.0e38f)) return KDN_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(r) || !aligned16(n) ||
      !aligned16(lambda_out) || (prior_out && !aligned16(prior_out)) ||
      (gain_out && !aligned16(gain_out)))
    return KDN_ERR_INVALID_ARG;
  const ScanLayout L = scan_layout(N, T);
  if (!workspace || workspace_bytes < L.total) return KDN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDN_ERR_INVALID_ARG;
  if (L.ntiles > (int64_t)0x7fffffff) return KDN_ERR_UNSUPPORTED;

  char* base = static_cast<char*>(workspace);
  ScanWs ws;
  ws.error = reinterpret_cast<uint32_t*>(base);
  ws.counter = reinterpret_cast<uint32_t*>(base + 4);
  ws.flag = reinterpret_cast<uint32_t*>(base + L.off_flag);
  ws.agg = reinterpret_cast<float4*>(base + L.off_agg);
  ws.incl = reinterpret_cast<float4*>(base + L.off_incl);

  if (cudaMemsetAsync(workspace, 0, L.clear_bytes, stream) != cudaSuccess) return KDN_ERR_CUDA;
  const int vec_ok = (T % 4 == 0) ? 1 : 0;
  if (vec_ok) {
    const int grid_cap = persistent_grid_cap();
    if (grid_cap < 1) return KDN_ERR_CUDA;
    const int64_t grid = std::min<int64_t>(L.ntiles, grid_cap);
    mobius_scan_persistent<<<(unsigned)grid, kThreads, kBufBytes, stream>>>(
        a, w, r, n, lambda0, info_scale, lambda_out, prior_out, gain_out, N, T, L.ntiles, ws,
        debug_skip_tile);
  } else {
    mobius_scan_kernel<<<(unsigned)L.ntiles, kThreads, 0, stream>>>(
        a, w, r, n, lambda0, info_scale, lambda_out, prior_out, gain_out, N, T, ws, vec_ok,
        debug_skip_tile);
  }
  return cudaGetLastError() == cudaSuccess ? KDN_OK : KDN_ERR_CUDA;
}

}  // namespace kdn

// ----------------------------------------------------------------------------
// Allocation-free variant (kdn_mobius_scan_noalloc).
//
// Some callers cannot allocate device memory where they call the scan, for
// example a host program that hands all device memory to its own pool at
// start-up and allows no cudaMalloc afterwards, or a plug-in that such a host
// gives only its input and output buffers.  For them the look-back scratch
// (tile flags, aggregates, prefixes, tile counter, error word) lives in the
// fixed-size array below, which every GPU that loads this library holds until
// the process exits.
// ----------------------------------------------------------------------------
namespace kdn {
namespace {

constexpr int64_t kNoAllocMaxTiles = KDN_SCAN_NOALLOC_MAX_TILES;
constexpr size_t align_up_c(size_t x, size_t a) { return (x + a - 1) / a * a; }
// Same layout as a caller workspace for kNoAllocMaxTiles tiles.
constexpr size_t kNoAllocBytes =
    align_up_c(align_up_c(align_up_c(256 + (size_t)kNoAllocMaxTiles * 4, 256) +
                              (size_t)kNoAllocMaxTiles * 16, 256) +
                   (size_t)kNoAllocMaxTiles * 16, 256);

static __device__ __align__(256) uint8_t g_noalloc_scan_scratch[kNoAllocBytes];

// Device address of the scratch array in the caller's current context.  In
// host code the array's name is a host-side stand-in, not a device address,
// so it is never passed to a kernel.  The address is looked up on every call
// with the caller's device and context current: the lookup allocates
// nothing, and it stays right when the caller switches contexts on a device
// or resets the device between calls (a cached address would then point into
// a context that no longer exists).  The first lookup in a context loads the
// library's device code there, which is why that first call belongs before
// any stream capture.
void* noalloc_scratch_in_current_context() {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scan_scratch) != cudaSuccess) return nullptr;
  return addr;
}

}  // namespace
}  // namespace kdn

extern "C" kdn_status kdn_mobius_scan_noalloc(const float* a, const float* w, const float* r,
                                              const float* n, const float* lambda0,
                                              float info_scale, float* lambda_out,
                                              float* prior_out, float* gain_out, int64_t N,
                                              int64_t T, void* stream) {
  if (N <= 0 || T <= 0 || N * T >= (int64_t(1) << 40)) return KDN_ERR_INVALID_ARG;
  const int64_t tiles = N * ((T + kdn::kTile - 1) / kdn::kTile);
  if (tiles > kdn::kNoAllocMaxTiles) return KDN_ERR_WORKSPACE;
  void* scratch = kdn::noalloc_scratch_in_current_context();
  if (!scratch) return KDN_ERR_CUDA;
  return kdn::mobius_scan_launch(a, w, r, n, lambda0, info_scale, lambda_out, prior_out, gain_out,
                                 N, T, scratch, kdn::kNoAllocBytes,
                                 static_cast<cudaStream_t>(stream), -1);
}
