// mao_soap_step / mao_foam_step: argument validation and workspace planning.
#include <cmath>

#include "host_common.h"

using namespace mao;

namespace {

mao_status check_refresh(const mao_refresh& r) {
  if (r.kind < MAO_REFRESH_EVERY_K || r.kind > MAO_REFRESH_NEVER) return MAO_ERR_INVALID_ARG;
  if (r.kind == MAO_REFRESH_EVERY_K && r.k < 1) return MAO_ERR_INVALID_ARG;
  if (r.kind == MAO_REFRESH_ADAPTIVE && (r.pf < 1 || !std::isfinite(r.tol))) return MAO_ERR_INVALID_ARG;
  if (r.sort != 0 && r.sort != 1) return MAO_ERR_INVALID_ARG;
  return MAO_OK;
}

mao_status check_hyper(float b1, float b2, float eps, float lr, float wd, int64_t t) {
  if (!std::isfinite(b1) || !std::isfinite(b2) || !std::isfinite(eps) || !std::isfinite(lr) || !std::isfinite(wd))
    return MAO_ERR_INVALID_ARG;
  if (b1 < 0.f || b1 >= 1.f || b2 < 0.f || b2 >= 1.f || eps < 0.f || t < 1) return MAO_ERR_INVALID_ARG;
  return MAO_OK;
}

mao_status check_mat(int m, int n, const void* G, int g_dtype) {
  if (m < 1 || n < 1) return MAO_ERR_SHAPE;
  if ((long long)m * n > (1ll << 31) - 1) return MAO_ERR_SHAPE;
  if (g_dtype != MAO_F32 && g_dtype != MAO_BF16) return MAO_ERR_DTYPE;
  if (m % 4 || n % 4) return MAO_ERR_SHAPE;
  if (g_dtype == MAO_BF16 && n % 8) return MAO_ERR_SHAPE;
  (void)G;
  return MAO_OK;
}

}  // namespace

extern "C" mao_status mao_soap_workspace_size(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p,
                                              size_t* bytes) {
  if (bytes == nullptr || p == nullptr || count < 0 || (count > 0 && mats == nullptr)) return MAO_ERR_INVALID_ARG;
  MAO_TRY(check_refresh(p->refresh));
  MAO_TRY(check_hyper(p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t));
  for (int i = 0; i < count; ++i) MAO_TRY(check_mat(mats[i].m, mats[i].n, mats[i].G, mats[i].g_dtype));
  *bytes = kStatusBytes;
  return MAO_OK;
}

extern "C" mao_status mao_soap_step(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p,
                                   void* workspace, size_t ws_bytes, mao_stats* stats, mao_stream_t stream) {
  size_t need = 0;
  MAO_TRY(mao_soap_workspace_size(mats, count, p, &need));
  (void)workspace;
  (void)ws_bytes;
  (void)stats;
  (void)stream;
  return MAO_ERR_UNSUPPORTED;
}

extern "C" mao_status mao_foam_workspace_size(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p,
                                              size_t* bytes) {
  if (bytes == nullptr || p == nullptr || count < 0 || (count > 0 && mats == nullptr)) return MAO_ERR_INVALID_ARG;
  MAO_TRY(check_refresh(p->refresh));
  MAO_TRY(check_hyper(p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t));
  if (p->tau_raw_trace != 0 && p->tau_raw_trace != 1) return MAO_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) MAO_TRY(check_mat(mats[i].m, mats[i].n, mats[i].G, mats[i].g_dtype));
  *bytes = kStatusBytes;
  return MAO_OK;
}

extern "C" mao_status mao_foam_step(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p,
                                   void* workspace, size_t ws_bytes, mao_stats* stats, mao_stream_t stream) {
  size_t need = 0;
  MAO_TRY(mao_foam_workspace_size(mats, count, p, &need));
  (void)workspace;
  (void)ws_bytes;
  (void)stats;
  (void)stream;
  return MAO_ERR_UNSUPPORTED;
}
