/*
 * kdn_testing.h -- test-only entry points of libkdn.  They exist so the
 * failure paths of the library can be exercised without faulting a GPU.
 * They have no counterpart on the pages and are not part of the layer API.
 */
#ifndef KDN_TESTING_H_
#define KDN_TESTING_H_

#include <stddef.h>
#include <stdint.h>

#include "kdn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* kdn_mobius_scan (lambda only), except that the tile with hand-out index
 * `silent_tile` never publishes its aggregate or prefix.  Tiles are handed
 * out tile-index-major: tile id = j * N + lane, where j is the 2048-step tile
 * within the lane.  The successor tile's bounded look-back therefore runs
 * out (after about one second), records KDN_ERR_TIMEOUT in the workspace
 * error word and finishes.  The call returns normally;
 * kdn_read_workspace_status() then reports KDN_ERR_TIMEOUT.  Outputs after
 * the silent tile are not meaningful.  Arguments as kdn_mobius_scan;
 * silent_tile >= 0. */
kdn_status kdn_testing_mobius_scan_unpublished_tile(
    const float* a, const float* w, const float* r, const float* n,
    const float* lambda0, float info_scale, float* lambda_out, int64_t N,
    int64_t T, void* workspace, size_t workspace_bytes, int64_t silent_tile,
    void* stream);

/* kdn_iso_forward / kdn_diag_forward (variant) on the chunked engine at
 * dk = dv = 128, bf16 q/k/v, S0 = 0, p0 = 1, except that the copy of chunk
 * `skip_chunk`'s V tile is never issued.  The bounded wait for it gives up
 * (after about one second), records KDN_ERR_TIMEOUT in the workspace error
 * word, and every CTA takes its abort path: it waits (bounded) for its
 * copies and MMAs in flight, frees its TMEM and returns.  The call returns
 * normally; kdn_read_workspace_status() then reports KDN_ERR_TIMEOUT.
 * Outputs are not meaningful.  1 <= skip_chunk < ceil(T / 64). */
kdn_status kdn_testing_forward_skip_v_copy(kdn_variant variant, const void* q,
                                           const void* k, const void* v,
                                           const float* a, const float* w,
                                           const float* r, float* o,
                                           float* S_out, float* p_out, int B,
                                           int T, int H, int skip_chunk,
                                           void* workspace,
                                           size_t workspace_bytes,
                                           void* stream);

/* kdn_kla_forward_ws on the chunked KLA engine (dk = dv = 128, bf16 q/k/v,
 * S0 = 0, lam0 = 1), except that the copy of chunk `skip_chunk`'s V tile is
 * never issued.  The issuer's bounded wait for it gives up (after about one
 * second) and records KDN_ERR_TIMEOUT in the workspace error word; every
 * role of every CTA then leaves through its bounded waits, waits (bounded)
 * for its copies and MMAs in flight, frees its TMEM and returns.  The call
 * returns normally; kdn_read_workspace_status() then reports
 * KDN_ERR_TIMEOUT.  Outputs are not meaningful.
 * 1 <= skip_chunk < ceil(T / 64). */
kdn_status kdn_testing_kla_skip_v_copy(const void* q, const void* k,
                                       const void* v, const float* a,
                                       const float* w, const float* r,
                                       float* o, float* S_out, float* lam_out,
                                       int B, int T, int H, int skip_chunk,
                                       void* workspace, size_t workspace_bytes,
                                       void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDN_TESTING_H_ */
