// extern "C" entry points of libkdn: argument checks, then kernel dispatch.
// Every check runs before anything is enqueued; a call that returns an error
// has enqueued nothing.
#include <cstring>

#include "kdn_common.cuh"
#include "../../include/kdn_testing.h"

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
                            int H, int dk, int dv, float kappa, cudaStream_t s);
bool chunk_engine_supported(kdn_dtype dt, int dk, int dv);
size_t chunk_engine_workspace_size(bool diag, int B, int H);
kdn_status chunk_engine_launch(bool diag, const void* q, const void* k, const void* v,
                               const float* a, const float* w, const float* r, const float* S0,
                               const float* p0, float* o, float* S_out, float* p_out, int B,
                               int T, int H, int dv, float kappa, void* workspace,
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
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !a || !w || !r || !o || !S_out || !p_out) return KDN_ERR_INVALID_ARG;
  if (in_dtype != KDN_F32 && in_dtype != KDN_BF16) return KDN_ERR_INVALID_ARG;
  if (!shape_ok(B, T, H, dk, dv)) return KDN_ERR_INVALID_ARG;
  if (!(info_scale == info_scale) || info_scale > 3.0e38f) return KDN_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(a) || !al16(w) || !al16(r) || !al16(o) ||
      !al16(S_out) || !al16(p_out) || !al16_or_null(S0) || !al16_or_null(p0))
    return KDN_ERR_INVALID_ARG;
  if (!dims_supported(dk, dv)) return KDN_ERR_UNSUPPORTED;
  const int path = select_path(chunk, in_dtype, dk, dv);
  if (path == -2) return KDN_ERR_INVALID_ARG;
  if (path == -1) return KDN_ERR_UNSUPPORTED;
  const float kappa = info_scale > 0.f ? info_scale : 1.f / (float)dk;
  if (path == 0) {
    return kdn::recurrent_launch(diag, in_dtype, q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T,
                                 H, dk, dv, kappa, as_stream(stream));
  }
  const size_t need = kdn::chunk_engine_workspace_size(diag, B, H);
  if (need && (!workspace || workspace_bytes < need)) return KDN_ERR_WORKSPACE;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return KDN_ERR_INVALID_ARG;
  return kdn::chunk_engine_launch(diag, q, k, v, a, w, r, S0, p0, o, S_out, p_out, B, T, H, dv,
                                  kappa, workspace, as_stream(stream));
}

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

int kdn_version(void) { return 100; }

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
  (void)T;
  if (!dims_supported(dk, dv) || B < 1 || H < 1) return 0;
  return select_path(chunk, KDN_BF16, dk, dv) == 1
             ? kdn::chunk_engine_workspace_size(variant == KDN_DIAG, B, H)
             : 0;
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

kdn_status kdn_read_workspace_status(const void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!workspace || workspace_bytes < 4) return KDN_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return KDN_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KDN_ERR_CUDA;
  return word == kdn::DEV_OK ? KDN_OK : KDN_ERR_TIMEOUT;
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
