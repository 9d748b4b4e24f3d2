// Small C-ABI entry points: status strings, state accounting, device checks,
// the workspace status word, and the GEMM verification entry point.
#include "host_common.h"
#include "mao_testing.h"

using namespace mao;

extern "C" const char* mao_status_string(int32_t s) {
  switch (s) {
    case MAO_OK: return "ok";
    case MAO_ERR_INVALID_ARG: return "invalid argument";
    case MAO_ERR_SHAPE: return "invalid shape";
    case MAO_ERR_DTYPE: return "invalid dtype";
    case MAO_ERR_ALIGN: return "misaligned pointer";
    case MAO_ERR_WORKSPACE: return "workspace missing or too small";
    case MAO_ERR_CUDA: return "CUDA error";
    case MAO_ERR_NONFINITE: return "non-finite values";
    case MAO_ERR_TIMEOUT: return "device wait timed out";
    case MAO_ERR_UNSUPPORTED: return "unsupported";
    case MAO_ERR_NOT_INITIALIZED: return "not initialized";
    default: return "unknown status";
  }
}

extern "C" uint64_t mao_muon_state_elems(int32_t m, int32_t n) {
  if (m < 1 || n < 1) return 0;
  return (uint64_t)m * (uint64_t)n;
}
extern "C" uint64_t mao_soap_state_elems(int32_t m, int32_t n) {
  if (m < 1 || n < 1) return 0;
  const uint64_t M = (uint64_t)m, N = (uint64_t)n;
  return 2 * M * N + 2 * M * M + 2 * N * N;
}
extern "C" uint64_t mao_foam_state_elems(int32_t m, int32_t n) {
  if (m < 1 || n < 1) return 0;
  const uint64_t M = (uint64_t)m, N = (uint64_t)n;
  return M * N + 2 * N * N + M + N;
}

extern "C" int32_t mao_version(void) { return MAO_VERSION; }

extern "C" mao_status mao_device_check(void) {
  DeviceInfo* d = nullptr;
  return device_info(&d);
}

extern "C" mao_status mao_workspace_status(const void* workspace, mao_stream_t stream, int32_t* where) {
  if (workspace == nullptr) return MAO_ERR_INVALID_ARG;
  DevStatus st;
  MAO_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  MAO_CUDA_TRY(cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost));
  if (where) *where = st.where;
  return static_cast<mao_status>(st.code);
}

// ------------------------------------------------------------------ GEMM check
namespace {
mao_status gemm_ws(int32_t kind, int32_t batch, int32_t M, int32_t N, int32_t K, Carver& cv, size_t* a_hi,
                   size_t* a_lo, size_t* b_hi, size_t* b_lo) {
  if (batch < 1 || M < 1 || N < 1 || K < 1) return MAO_ERR_SHAPE;
  if (kind != MAO_GEMM_BF16 && kind != MAO_GEMM_TF32X3) return MAO_ERR_INVALID_ARG;
  cv.take(kStatusBytes);
  if (kind == MAO_GEMM_TF32X3) {
    const size_t an = (size_t)batch * M * K, bn = (size_t)batch * N * K;
    *a_hi = cv.take(4 * an);
    *a_lo = cv.take(4 * an);
    *b_hi = cv.take(4 * bn);
    *b_lo = cv.take(4 * bn);
  }
  return MAO_OK;
}
}  // namespace

extern "C" mao_status mao_test_gemm_workspace_size(int32_t kind, int32_t batch, int32_t M, int32_t N, int32_t K,
                                                   size_t* bytes) {
  if (bytes == nullptr) return MAO_ERR_INVALID_ARG;
  Carver cv;
  size_t a, b, c, d;
  MAO_TRY(gemm_ws(kind, batch, M, N, K, cv, &a, &b, &c, &d));
  *bytes = cv.total();
  return MAO_OK;
}

extern "C" mao_status mao_test_gemm(int32_t kind, int32_t a_mn_major, int32_t b_mn_major, const void* A,
                                    const void* B, float* D, int32_t batch, int32_t M, int32_t N, int32_t K,
                                    void* workspace, size_t ws_bytes, mao_stream_t stream_) {
  if (A == nullptr || B == nullptr || D == nullptr || workspace == nullptr) return MAO_ERR_INVALID_ARG;
  if ((a_mn_major != 0 && a_mn_major != 1) || (b_mn_major != 0 && b_mn_major != 1)) return MAO_ERR_INVALID_ARG;
  Carver cv;
  size_t oah = 0, oal = 0, obh = 0, obl = 0;
  MAO_TRY(gemm_ws(kind, batch, M, N, K, cv, &oah, &oal, &obh, &obl));
  if (ws_bytes < cv.total()) return MAO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MAO_ERR_ALIGN;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return MAO_ERR_ALIGN;
  const int vec = (kind == MAO_GEMM_BF16) ? 8 : 4;
  const int a_inner = a_mn_major ? M : K, b_inner = b_mn_major ? N : K;
  if (a_inner % vec || b_inner % vec || N % 4) return MAO_ERR_SHAPE;
  DeviceInfo* dev = nullptr;
  MAO_TRY(device_info(&dev));
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  MAO_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(DevStatus), stream));

  const int okind = (kind == MAO_GEMM_BF16) ? OP_BF16 : OP_TF32X3;
  const void* a_src = A;
  const void* b_src = B;
  const size_t an = (size_t)batch * M * K, bn = (size_t)batch * N * K;
  GemmLoMaps lo;
  std::memset(&lo, 0, sizeof(lo));
  if (okind == OP_TF32X3) {
    MAO_TRY(launch_tf32_split(static_cast<const float*>(A), reinterpret_cast<float*>(ws + oah),
                              reinterpret_cast<float*>(ws + oal), an, stream));
    MAO_TRY(launch_tf32_split(static_cast<const float*>(B), reinterpret_cast<float*>(ws + obh),
                              reinterpret_cast<float*>(ws + obl), bn, stream));
    a_src = ws + oah;
    b_src = ws + obh;
  }
  auto view = [&](const void* base, int mn, int mn_major) {
    OperandView v;
    v.base = base;
    v.batch = (uint64_t)batch;
    if (mn_major) {
      v.inner = (uint64_t)mn;
      v.rows = (uint64_t)K;
    } else {
      v.inner = (uint64_t)K;
      v.rows = (uint64_t)mn;
    }
    v.ld = v.inner;
    v.bstride = (uint64_t)mn * K;
    return v;
  };
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.nclasses = 1;
  p.alpha = 1.0f;
  p.status = reinterpret_cast<DevStatus*>(ws);
  MAO_TRY(encode_operand(&p.mapA[0], okind, a_mn_major, 128, view(a_src, M, a_mn_major)));
  MAO_TRY(encode_operand(&p.mapB[0], okind, b_mn_major, 256, view(b_src, N, b_mn_major)));
  if (okind == OP_TF32X3) {
    MAO_TRY(encode_operand(&lo.mapAlo[0], okind, a_mn_major, 128, view(ws + oal, M, a_mn_major)));
    MAO_TRY(encode_operand(&lo.mapBlo[0], okind, b_mn_major, 256, view(ws + obl, N, b_mn_major)));
  }
  p.cls[0] = GemmClass{M, N, K, batch, 0, 0, 0, D, (long long)M * N, N, nullptr, 0, 0, nullptr, 0, 0, nullptr};
  finalize_classes(p);
  (void)dev;
  return launch_gemm(okind, a_mn_major, b_mn_major, EPI_STORE_F32, p, okind == OP_TF32X3 ? &lo : nullptr, stream,
                     MAO_K_GEMM_TEST);
}

namespace mao {
Profiler& profiler() {
  static Profiler p;
  return p;
}
}  // namespace mao

extern "C" mao_status mao_profile_start(void** events, mao_launch_info* info, int32_t capacity) {
  if (capacity < 0 || (capacity > 0 && (events == nullptr || info == nullptr))) return MAO_ERR_INVALID_ARG;
  Profiler& P = profiler();
  P.events = events;
  P.info = info;
  P.capacity = capacity;
  P.count = 0;
  P.active = true;
  return MAO_OK;
}

extern "C" int32_t mao_profile_stop(void) {
  Profiler& P = profiler();
  P.active = false;
  return P.count;
}
