// extern "C" entry points of libkdn: argument checks, then kernel dispatch.
// Every check runs before anything is enqueued; a call that returns an error
// has enqueued nothing (kdn_forward_host: except for KDN_ERR_CUDA from a
// runtime call part-way, after which the caller's stream still waits for
// whatever was enqueued).
#include <cstring>

#include <algorithm>
#include <mutex>

#include "kdn_common.cuh"
#include "../../include/kdn_testing.h"
#include "bwd_checkpoint.h"

namespace kdn {
size_t mobius_scan_workspace_size(int64_t N, int64_t T);
kdn_status mobius_scan_launch(const float* a, const float* w, const float* r, const float* n,
                              const float* lambda0, float info_scale, float* lambda_out,
                              float* prior_out, float* gain_out, int64_t N, int64_t T,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream,
                              int64_t debug_skip_tile);
kdn_status recurrent_launch(bool diag, kdn_dtype dt, const void* q, const void* k, const void* v,
                            const float* a, const float* w, const float* r, const float* S0,
                            const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                            int H, int dk, int dv, float kappa, cudaStream_t s,
                            const int* cu_seqlens = nullptr, uint32_t* err = nullptr,
                            float* Ssave = nullptr, float* Psave = nullptr);
bool chunk_engine_supported(kdn_dtype dt, int dk, int dv);
size_t chunk_engine_workspace_size(bool diag, int B, int H);
int segment_count(int B, int T, int H);
size_t segmented_workspace_size(bool diag, int B, int T, int H, int nseg);
kdn_status segmented_forward(bool diag, const void* q, const void* k, const void* v,
                             const float* a, const float* w, const float* r, const float* S0,
                             const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                             int H, float kappa, int nseg, void* ws, cudaStream_t st);
kdn_status chunk_engine_launch(bool diag, const void* q, const void* k, const void* v,
                               const float* a, const float* w, const float* r, const float* S0,
                               const float* p0, float* o, float* S_out, float* p_out, int B,
                               int T, int H, int dv, float kappa, void* workspace,
                               cudaStream_t s, int debug_skip_v = -1,
                               const int* cu_seqlens = nullptr);
bool exact_kalman_supported(int dk, int dv);
kdn_status exact_kalman_launch(bool diag, kdn_dtype dt, const void* q, const void* k,
                               const void* v, const float* a, const float* w, const float* r,
                               const float* S0, const float* P0, float* o, float* S_out,
                               float* P_out, int B, int T, int H, int dk, int dv, cudaStream_t s);
bool backward_supported(int dk, int dv);
kdn_status backward_launch(bool diag, kdn_dtype dt, const void* q, const void* k, const void* v,
                           const float* a, const float* w, const float* r, const float* dO,
                           const float* dS_T, const float* dp_T, const float* Sck,
                           const float* Psave, float* scratch, float* dq, float* dk, float* dv_,
                           float* da, float* dw, float* dr, float* dS0, float* dp0, int B, int T,
                           int H, int dkk, int dv, float kappa, cudaStream_t s);
bool kla_supported(int dk, int dv);
bool kla_engine_supported(kdn_dtype dt, int dk, int dv, int T);
kdn_status kla_engine_launch(const void* q, const void* k, const void* v, const float* a,
                             const float* w, const float* r, const float* S0, const float* L0,
                             float* o, float* S_out, float* L_out, int B, int T, int H, void* ws,
                             cudaStream_t s, int debug_skip_v);
kdn_status kla_launch(kdn_dtype dt, const void* q, const void* k, const void* v, const float* a,
                      const float* w, const float* r, const float* S0, const float* L0, float* o,
                      float* S_out, float* L_out, int B, int T, int H, int dk, int dv,
                      cudaStream_t s);
}  // namespace kdn

namespace {

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool al16_or_null(const void* p) { return !p || al16(p); }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool shape_ok(int B, int T, int H, int dk, int dv) {
  if (B < 1 || T < 1 || H < 1) return false;
  if ((int64_t)B * H > 0x7fffffffLL) return false;
  if ((int64_t)B * T * H > (int64_t(1) << 40)) return false;
  if (dv < 1) return false;
  (void)dk;
  return true;
}
inline bool dims_supported(int dk, int dv) {
  return (dk == 32 || dk == 64 || dk == 128) && dv >= 1 && dv <= 128;
}

// Which forward path a call takes: 0 recurrent, 1 chunked, -1 unsupported.
int select_path(int chunk, kdn_dtype dt, int dk, int dv) {
  const bool chunked_ok = kdn::chunk_engine_supported(dt, dk, dv);
  switch (chunk) {
    case KDN_CHUNK_AUTO: return chunked_ok ? 1 : 0;
    case KDN_CHUNK_RECURRENT: return 0;
    case KDN_CHUNK_64: return chunked_ok ? 1 : -1;
    default: return -2;
  }
}

kdn_status forward_common(bool diag, const void* q, const void* k, const void* v,
                          kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                          const float* S0, const float* p0, float* o, float* S_out, float* p_out,
                          int B, int T, int H, int dk, int dv, float info_scale, int chunk,
                          void* workspace, size_t workspace_bytes, void* stream,
                          int debug_skip_v = -1, const int* cu_seqlens = nullptr) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !p_out) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  // (packed sequences: B sequences of T tokens in all, T >= 0)
  if (!shape_ok(B, cu_seqlens ? std::max(T, 1) : T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale == info_scale) || info_scale > 3.0e38f) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(o) ||
      !al16(S_out) || !al16(p_out) || !al16_or_null(S0) || !al16_or_null(p0))
    return KDN_ERR_INVALID_ARG;
  if (!dims_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  int path = select_path(chunk, in_dtype, dk, dv);
  if (path == -2) return KDN_ERR_INVALID_ARG;
  if (path == -1) return KDN_ERR_UNSUPPORTED;
  if (cu_seqlens) {
    // packed sequences: the chunked engine at d_v = 128, otherwise the
    // token-recurrent kernel; a workspace always carries the error word
    if (path == 1 && (dv != 128 || T == 0)) {
      if (chunk == KDN_CHUNK_64 && dv != 128) return KDN_ERR_UNSUPPORTED;
      path = 0;
    }
    if (!workspace || workspace_bytes < 256) return KDN_ERR_WORKSPACE;
  }
  const float kappa = info_scale > 0.f ? info_scale : 1.f / (float)dk;
  if (path == 0) {
    uint32_t* err = nullptr;
    if (cu_seqlens) {
      if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDN_ERR_INVALID_ARG;
      err = static_cast<uint32_t*>(workspace);
      if (cudaMemsetAsync(err, 0, 4, as_stream(stream)) != cudaSuccess) return KDN_ERR_CUDA;
    }
    return kdn::recurrent_launch(diag, in_dtype, q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T,
                                 H, dk, dv, kappa, as_stream(stream), cu_seqlens, err);
  }
  // few heads over a long sequence: the segmented forward (whole segments as
  // extra heads of the same engine)
  const int nseg = (dv == 128 && !cu_seqlens && debug_skip_v < 0) ? kdn::segment_count(B, T, H) : 1;
  const size_t need = nseg > 1 ? kdn::segmented_workspace_size(diag, B, T, H, nseg)
                               : kdn::chunk_engine_workspace_size(diag, B, H);
  if (need && (!workspace || workspace_bytes < need)) return KDN_ERR_WORKSPACE;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDN_ERR_INVALID_ARG;
  if (nseg > 1)
    return kdn::segmented_forward(diag, q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, kappa,
                                  nseg, workspace, as_stream(stream));
  return kdn::chunk_engine_launch(diag, q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv,
                                  kappa, workspace, as_stream(stream), debug_skip_v, cu_seqlens);
}

// ------------------------------------------------------------ host buffers
// kdn_forward_host runs the forward on batch slices whose inputs and outputs
// live in pinned host memory.  Slice i uses device slot i & 1 and internal
// stream i & 1, so the copies of one slice (in and out, PCIe is full duplex)
// overlap those of the next and the kernels; a slot is reused only after the
// earlier work on its own stream.

__global__ void or_error_word(uint32_t* dst, const uint32_t* src) { atomicOr(dst, *src); }

inline size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Offsets of one slice's device buffers (of nb batch entries) in a slot.
struct HostSlot {
  size_t q, k, v, a, w, r, s0, p0, o, s, p, fws, fws_bytes, bytes;
};

HostSlot host_slot(bool diag, int nb, int T, int H, int dk, int dv, size_t es, int chunk) {
  HostSlot L{};
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t at = off;
    off = up256(off + n);
    return at;
  };
  const size_t tok = (size_t)nb * T * H;
  const size_t pdim = diag ? (size_t)dk : 1;
  L.q = take(tok * dk * es);
  L.k = take(tok * dk * es);
  L.v = take(tok * dv * es);
  L.a = take(tok * 4);
  L.w = take(tok * pdim * 4);
  L.r = take(tok * 4);
  L.s0 = take((size_t)nb * H * dv * dk * 4);
  L.p0 = take((size_t)nb * H * pdim * 4);
  L.o = take(tok * dv * 4);
  L.s = take((size_t)nb * H * dv * dk * 4);
  L.p = take((size_t)nb * H * pdim * 4);
  L.fws_bytes = std::max<size_t>(256, kdn_forward_workspace_size(diag ? KDN_DIAG : KDN_ISO, nb, T,
                                                                  H, dk, dv, chunk));
  L.fws = take(L.fws_bytes);
  L.bytes = off;
  return L;
}

// Two streams and three events per device, created once.
struct HostStreams {
  cudaStream_t st[2];
  cudaEvent_t start, done[2];
};
constexpr int kMaxHostDevices = 64;
HostStreams g_host_streams[kMaxHostDevices];
bool g_host_ready[kMaxHostDevices];
std::mutex g_host_mu;  // also serialises the enqueue of concurrent calls

}  // namespace

extern "C" {

const char* kdn_status_string(kdn_status status) {
  switch (status) {
    case KDN_OK: return "KDN_OK";
    case KDN_ERR_INVALID_ARG: return "KDN_ERR_INVALID_ARG: invalid argument";
    case KDN_ERR_UNSUPPORTED: return "KDN_ERR_UNSUPPORTED: unsupported shape, dtype or path";
    case KDN_ERR_WORKSPACE: return "KDN_ERR_WORKSPACE: workspace missing or too small";
    case KDN_ERR_TIMEOUT: return "KDN_ERR_TIMEOUT: a bounded device wait gave up";
    case KDN_ERR_CUDA: return "KDN_ERR_CUDA: CUDA runtime error";
  }
  return "unknown kdn_status";
}

int kdn_version(void) { return 200; }

size_t kdn_mobius_scan_workspace_size(int64_t N, int64_t T) {
  return kdn::mobius_scan_workspace_size(N, T);
}

kdn_status kdn_mobius_scan(const float* a, const float* w, const float* r, const float* n,
                           const float* lambda0, float info_scale, float* lambda_out,
                           float* prior_out, float* gain_out, int64_t N, int64_t T,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return kdn::mobius_scan_launch(a, w, r, n, lambda0, info_scale, lambda_out, prior_out, gain_out,
                                 N, T, workspace, workspace_bytes, as_stream(stream), -1);
}

size_t kdn_forward_workspace_size(kdn_variant variant, int B, int T, int H, int dk, int dv,
                                  int chunk) {
  if (!dims_supported(dk, dv) || B < 1 || H < 1 || T < 0) return 0;
  if (select_path(chunk, KDN_BF16, dk, dv) != 1) return 0;
  const bool diag = variant == KDN_DIAG;
  const int nseg = dv == 128 && T > 0 ? kdn::segment_count(B, T, H) : 1;
  return nseg > 1 ? kdn::segmented_workspace_size(diag, B, T, H, nseg)
                  : kdn::chunk_engine_workspace_size(diag, B, H);
}

kdn_status kdn_iso_forward(const void* q, const void* k, const void* v, kdn_dtype in_dtype,
                           const float* a, const float* w, const float* r, const float* S0,
                           const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                           int H, int dk, int dv, float info_scale, int chunk, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return forward_common(false, q, k, v, in_dtype, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk,
                        dv, info_scale, chunk, workspace, workspace_bytes, stream);
}

kdn_status kdn_diag_forward(const void* q, const void* k, const void* v, kdn_dtype in_dtype,
                            const float* a, const float* w, const float* r, const float* S0,
                            const float* p0, float* o, float* S_out, float* p_out, int B, int T,
                            int H, int dk, int dv, int chunk, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return forward_common(true, q, k, v, in_dtype, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dk,
                        dv, 1.0f, chunk, workspace, workspace_bytes, stream);
}

size_t kdn_forward_varlen_workspace_size(kdn_variant variant, int N, int H, int dk, int dv,
                                         int chunk) {
  if (N < 1 || H < 1 || !dims_supported(dk, dv)) return 0;
  const size_t need = kdn_forward_workspace_size(variant, N, 1, H, dk, dv, chunk);
  return need > 256 ? need : 256;
}

kdn_status kdn_forward_varlen(kdn_variant variant, const void* q, const void* k, const void* v,
                              kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                              const int32_t* cu_seqlens, const float* S0, const float* p0,
                              float* o, float* S_out, float* p_out, int N, int total, int H,
                              int dk, int dv, float info_scale, int chunk, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (!cu_seqlens || total < 0) return KDN_ERR_INVALID_ARG;
  return forward_common(variant == KDN_DIAG, q, k, v, in_dtype, a, w, r, S0, p0, o, S_out, p_out,
                        N, total, H, dk, dv, variant == KDN_DIAG ? 1.f : info_scale, chunk,
                        workspace, workspace_bytes, stream, -1, cu_seqlens);
}

kdn_status kdn_decode_step(kdn_variant variant, const void* q, const void* k, const void* v,
                           kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                           float* S, float* p, float* o, int B, int H, int dk, int dv,
                           float info_scale, void* stream) {
  if (!q || !k || !v || !a || !w || !r || !S || !p || !o) return KDN_ERR_INVALID_ARG;
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, 1, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale == info_scale) || info_scale > 3.0e38f) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(S) ||
      !al16(p) || !al16(o))
    return KDN_ERR_INVALID_ARG;
  if (!dims_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  const float kappa = info_scale > 0.f ? info_scale : 1.f / (float)dk;
  return kdn::recurrent_launch(variant == KDN_DIAG, in_dtype, q, k, v, a, w, r, S, p, o, S, p, B,
                               1, H, dk, dv, kappa, as_stream(stream));
}

kdn_status kdn_exact_forward(kdn_variant variant, const void* q, const void* k, const void* v,
                             kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                             const float* S0, const float* P0, float* o, float* S_out,
                             float* P_out, int B, int T, int H, int dk, int dv, void* stream) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !P_out) return KDN_ERR_INVALID_ARG;
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(o) ||
      !al16(S_out) || !al16(P_out) || !al16_or_null(S0) || !al16_or_null(P0))
    return KDN_ERR_INVALID_ARG;
  if (!kdn::exact_kalman_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  return kdn::exact_kalman_launch(variant == KDN_DIAG, in_dtype, q, k, v, a, w, r, S0, P0, o,
                                  S_out, P_out, B, T, H, dk, dv, as_stream(stream));
}

namespace {
// backward workspace: the state checkpoints (every 16th token), the
// variance before every token, the per-CTA scratch of 16 rebuilt states,
// then the forward's outputs (o, S_T, p_T), each region 256-byte aligned
struct BwdLayout {
  size_t states, vars, scratch, o, s, p, bytes;
};
inline size_t al256(size_t x) { return (x + 255) / 256 * 256; }
BwdLayout bwd_layout(bool diag, int B, int T, int H, int dk, int dv) {
  BwdLayout L{};
  const size_t bh = (size_t)B * H, np = diag ? (size_t)dk : 1;
  const size_t nck = ((size_t)T + kdn::kBwdCheckpoint - 1) / kdn::kBwdCheckpoint;
  L.states = 0;
  L.vars = al256(bh * nck * dv * dk * 4);
  L.scratch = L.vars + al256(bh * T * np * 4);
  L.o = L.scratch + al256(bh * kdn::kBwdCheckpoint * dv * dk * 4);
  L.s = L.o + al256((size_t)B * T * H * dv * 4);
  L.p = L.s + al256(bh * dv * dk * 4);
  L.bytes = L.p + al256(bh * np * 4);
  return L;
}
}  // namespace

size_t kdn_backward_workspace_size(kdn_variant variant, int B, int T, int H, int dk, int dv) {
  if ((variant != KDN_ISO && variant != KDN_DIAG) || !shape_ok(B, T, H, dk, dv) ||
      !kdn::backward_supported(dk, dv))
    return 0;
  return bwd_layout(variant == KDN_DIAG, B, T, H, dk, dv).bytes;
}

kdn_status kdn_backward(kdn_variant variant, const void* q, const void* k, const void* v,
                        kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                        const float* S0, const float* p0, const float* dO, const float* dS_T,
                        const float* dp_T, float* dq, float* dk_, float* dv_, float* da,
                        float* dw, float* dr, float* dS0, float* dp0, int B, int T, int H, int dk,
                        int dv, float info_scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (!q || !k || !v || !a || !w || !r || !dO || !dq || !dk_ || !dv_ || !da || !dw || !dr ||
      !dS0 || !dp0)
    return KDN_ERR_INVALID_ARG;
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale == info_scale) || info_scale > 3.0e38f) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(dO) ||
      !al16(dq) || !al16(dk_) || !al16(dv_) || !al16(da) || !al16(dw) || !al16(dr) ||
      !al16(dS0) || !al16(dp0) || !al16_or_null(S0) || !al16_or_null(p0) ||
      !al16_or_null(dS_T) || !al16_or_null(dp_T))
    return KDN_ERR_INVALID_ARG;
  if (!kdn::backward_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  const bool diag = variant == KDN_DIAG;
  const BwdLayout L = bwd_layout(diag, B, T, H, dk, dv);
  if (!workspace || workspace_bytes < L.bytes) return KDN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDN_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  float* Ssave = reinterpret_cast<float*>(ws + L.states);  // checkpoints
  float* Psave = reinterpret_cast<float*>(ws + L.vars);
  const float kappa = diag ? 1.f : (info_scale > 0.f ? info_scale : 1.f / (float)dk);
  // the forward again, saving the variance before every token and the state
  // before every 16th
  kdn_status st = kdn::recurrent_launch(
      diag, in_dtype, q, k, v, a, w, r, S0, p0, reinterpret_cast<float*>(ws + L.o),
      reinterpret_cast<float*>(ws + L.s), reinterpret_cast<float*>(ws + L.p), B, T, H, dk, dv,
      kappa, as_stream(stream), nullptr, nullptr, Ssave, Psave);
  if (st != KDN_OK) return st;
  return kdn::backward_launch(diag, in_dtype, q, k, v, a, w, r, dO, dS_T, dp_T, Ssave, Psave,
                              reinterpret_cast<float*>(ws + L.scratch), dq, dk_, dv_, da, dw, dr,
                              dS0, dp0, B, T, H, dk, dv, kappa, as_stream(stream));
}

kdn_status kdn_kla_forward(const void* q, const void* k, const void* v, kdn_dtype in_dtype,
                           const float* a, const float* w, const float* r, const float* S0,
                           const float* lam0, float* o, float* S_out, float* lam_out, int B,
                           int T, int H, int dk, int dv, void* stream) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !lam_out) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(o) ||
      !al16(S_out) || !al16(lam_out) || !al16_or_null(S0) || !al16_or_null(lam0))
    return KDN_ERR_INVALID_ARG;
  if (!kdn::kla_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  return kdn::kla_launch(in_dtype, q, k, v, a, w, r, S0, lam0, o, S_out, lam_out, B, T, H, dk,
                         dv, as_stream(stream));
}

size_t kdn_kla_workspace_size(int B, int T, int H, int dk, int dv) {
  if (!shape_ok(B, T, H, dk, dv) || !kdn::kla_supported(dk, dv)) return 0;
  return 256;
}

kdn_status kdn_kla_forward_ws(const void* q, const void* k, const void* v, kdn_dtype in_dtype,
                              const float* a, const float* w, const float* r, const float* S0,
                              const float* lam0, float* o, float* S_out, float* lam_out, int B,
                              int T, int H, int dk, int dv, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !lam_out) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(o) ||
      !al16(S_out) || !al16(lam_out) || !al16_or_null(S0) || !al16_or_null(lam0))
    return KDN_ERR_INVALID_ARG;
  if (!kdn::kla_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  if (!workspace || !al16(workspace) || workspace_bytes < kdn_kla_workspace_size(B, T, H, dk, dv))
    return KDN_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  if (!kdn::kla_engine_supported(in_dtype, dk, dv, T)) {
    if (cudaMemsetAsync(workspace, 0, 4, s) != cudaSuccess) return KDN_ERR_CUDA;
    return kdn::kla_launch(in_dtype, q, k, v, a, w, r, S0, lam0, o, S_out, lam_out, B, T, H, dk,
                           dv, s);
  }
  return kdn::kla_engine_launch(q, k, v, a, w, r, S0, lam0, o, S_out, lam_out, B, T, H, workspace,
                                s, -1);
}

kdn_status kdn_testing_kla_skip_v_copy(const void* q, const void* k, const void* v,
                                       const float* a, const float* w, const float* r, float* o,
                                       float* S_out, float* lam_out, int B, int T, int H,
                                       int skip_chunk, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !lam_out) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, 128, 128)) return KDN_ERR_INVALID_ARG;
  if (skip_chunk < 1 || skip_chunk >= (T + 63) / 64) return KDN_ERR_INVALID_ARG;
  if (!workspace || !al16(workspace) ||
      workspace_bytes < kdn_kla_workspace_size(B, T, H, 128, 128))
    return KDN_ERR_WORKSPACE;
  return kdn::kla_engine_launch(q, k, v, a, w, r, nullptr, nullptr, o, S_out, lam_out, B, T, H,
                                workspace, as_stream(stream), skip_chunk);
}

size_t kdn_forward_host_workspace_size(kdn_variant variant, int B, int T, int H, int dk, int dv,
                                       kdn_dtype in_dtype, int chunk, int slice_b) {
  if (B < 1 || T < 1 || H < 1 || !dims_supported(dk, dv)) return 0;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return 0;
  const int nb = std::min(B, slice_b > 0 ? slice_b : 1);
  const size_t es = in_dtype == KDN_BF16 ? 2 : 4;
  return 256 + 2 * host_slot(variant == KDN_DIAG, nb, T, H, dk, dv, es, chunk).bytes;
}

kdn_status kdn_forward_host(kdn_variant variant, const void* q, const void* k, const void* v,
                            kdn_dtype in_dtype, const float* a, const float* w, const float* r,
                            const float* S0, const float* p0, float* o, float* S_out,
                            float* p_out, int B, int T, int H, int dk, int dv, float info_scale,
                            int chunk, int slice_b, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !p_out) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale == info_scale) || info_scale > 3.0e38f) return KDN_ERR_INVALID_ARG;
  if (!dims_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  const int path = select_path(chunk, in_dtype, dk, dv);
  if (path == -2) return KDN_ERR_INVALID_ARG;
  if (path == -1) return KDN_ERR_UNSUPPORTED;
  const bool diag = variant == KDN_DIAG;
  const int nb = std::min(B, slice_b > 0 ? slice_b : 1);
  const size_t es = in_dtype == KDN_BF16 ? 2 : 4;
  const HostSlot L = host_slot(diag, nb, T, H, dk, dv, es, chunk);
  if (!workspace || workspace_bytes < 256 + 2 * L.bytes) return KDN_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return KDN_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxHostDevices)
    return KDN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostStreams& hs = g_host_streams[dev];
  if (!g_host_ready[dev]) {
    if (cudaStreamCreateWithFlags(&hs.st[0], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hs.st[1], cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hs.start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hs.done[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hs.done[1], cudaEventDisableTiming) != cudaSuccess)
      return KDN_ERR_CUDA;
    g_host_ready[dev] = true;
  }
  cudaStream_t s0 = as_stream(stream);
  char* base = static_cast<char*>(workspace);
  uint32_t* err = reinterpret_cast<uint32_t*>(base);
  // the header error word and both slots' forward error words start clear
  bool ok = cudaMemsetAsync(err, 0, 4, s0) == cudaSuccess;
  for (int i = 0; i < 2 && ok; ++i)
    ok = cudaMemsetAsync(base + 256 + i * L.bytes + L.fws, 0, 4, s0) == cudaSuccess;
  ok = ok && cudaEventRecord(hs.start, s0) == cudaSuccess &&
       cudaStreamWaitEvent(hs.st[0], hs.start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(hs.st[1], hs.start, 0) == cudaSuccess;
  kdn_status status = ok ? KDN_OK : KDN_ERR_CUDA;
  const size_t pdim = diag ? (size_t)dk : 1;
  const auto H2D = cudaMemcpyHostToDevice;
  const auto D2H = cudaMemcpyDeviceToHost;
  for (int b0 = 0, i = 0; b0 < B && status == KDN_OK; b0 += nb, ++i) {
    const int n = std::min(nb, B - b0);
    cudaStream_t st = hs.st[i & 1];
    char* sb = base + 256 + (size_t)(i & 1) * L.bytes;
    const size_t tok0 = (size_t)b0 * T * H, tok = (size_t)n * T * H;
    const size_t hd0 = (size_t)b0 * H, hd = (size_t)n * H;
    auto cp = [&](size_t dst_off, const void* src, size_t off_bytes, size_t bytes,
                  cudaMemcpyKind kind, bool to_dev) {
      if (status != KDN_OK) return;
      cudaError_t e = to_dev ? cudaMemcpyAsync(sb + dst_off, static_cast<const char*>(src) + off_bytes,
                                               bytes, kind, st)
                             : cudaMemcpyAsync(static_cast<char*>(const_cast<void*>(src)) + off_bytes,
                                               sb + dst_off, bytes, kind, st);
      if (e != cudaSuccess) status = KDN_ERR_CUDA;
    };
    cp(L.q, q, tok0 * dk * es, tok * dk * es, H2D, true);
    cp(L.k, k, tok0 * dk * es, tok * dk * es, H2D, true);
    cp(L.v, v, tok0 * dv * es, tok * dv * es, H2D, true);
    cp(L.a, a, tok0 * 4, tok * 4, H2D, true);
    cp(L.w, w, tok0 * pdim * 4, tok * pdim * 4, H2D, true);
    cp(L.r, r, tok0 * 4, tok * 4, H2D, true);
    if (S0) cp(L.s0, S0, hd0 * dv * dk * 4, hd * dv * dk * 4, H2D, true);
    if (p0) cp(L.p0, p0, hd0 * pdim * 4, hd * pdim * 4, H2D, true);
    if (status != KDN_OK) break;
    const kdn_status fs = forward_common(
        diag, sb + L.q, sb + L.k, sb + L.v, in_dtype, reinterpret_cast<float*>(sb + L.a),
        reinterpret_cast<float*>(sb + L.w), reinterpret_cast<float*>(sb + L.r),
        S0 ? reinterpret_cast<float*>(sb + L.s0) : nullptr,
        p0 ? reinterpret_cast<float*>(sb + L.p0) : nullptr, reinterpret_cast<float*>(sb + L.o),
        reinterpret_cast<float*>(sb + L.s), reinterpret_cast<float*>(sb + L.p), n, T, H, dk, dv,
        diag ? 1.f : info_scale, chunk, sb + L.fws, L.fws_bytes, st);
    if (fs != KDN_OK) {
      status = fs;
      break;
    }
    or_error_word<<<1, 1, 0, st>>>(err, reinterpret_cast<const uint32_t*>(sb + L.fws));
    if (cudaGetLastError() != cudaSuccess) status = KDN_ERR_CUDA;
    cp(L.o, o, tok0 * dv * 4, tok * dv * 4, D2H, false);
    cp(L.s, S_out, hd0 * dv * dk * 4, hd * dv * dk * 4, D2H, false);
    cp(L.p, p_out, hd0 * pdim * 4, hd * pdim * 4, D2H, false);
  }
  // the caller's stream waits for both internal streams, also after an error,
  // so that no copy outlives the call's stream order
  for (int j = 0; j < 2; ++j)
    if (cudaEventRecord(hs.done[j], hs.st[j]) != cudaSuccess ||
        cudaStreamWaitEvent(s0, hs.done[j], 0) != cudaSuccess)
      status = KDN_ERR_CUDA;
  return status;
}

kdn_status kdn_read_workspace_status(const void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!workspace || workspace_bytes < 4) return KDN_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return KDN_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KDN_ERR_CUDA;
  if (word & kdn::DEV_TIMEOUT) return KDN_ERR_TIMEOUT;
  return word == kdn::DEV_OK ? KDN_OK : KDN_ERR_INVALID_ARG;
}

kdn_status kdn_testing_forward_skip_v_copy(kdn_variant variant, const void* q, const void* k,
                                           const void* v, const float* a, const float* w,
                                           const float* r, float* o, float* S_out, float* p_out,
                                           int B, int T, int H, int skip_chunk, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (variant != KDN_ISO && variant != KDN_DIAG) return KDN_ERR_INVALID_ARG;
  if (skip_chunk < 1 || skip_chunk >= (T + 63) / 64) return KDN_ERR_INVALID_ARG;
  return forward_common(variant == KDN_DIAG, q, k, v, KDN_BF16, a, w, r, nullptr, nullptr, o,
                        S_out, p_out, B, T, H, 128, 128, 0.f, KDN_CHUNK_64, workspace,
                        workspace_bytes, stream, skip_chunk);
}

kdn_status kdn_testing_mobius_scan_unpublished_tile(
    const float* a, const float* w, const float* r, const float* n, const float* lambda0,
    float info_scale, float* lambda_out, int64_t N, int64_t T, void* workspace,
    size_t workspace_bytes, int64_t silent_tile, void* stream) {
  if (silent_tile < 0) return KDN_ERR_INVALID_ARG;
  return kdn::mobius_scan_launch(a, w, r, n, lambda0, info_scale, lambda_out, nullptr, nullptr, N,
                                 T, workspace, workspace_bytes, as_stream(stream), silent_tile);
}

}  // extern "C"
