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

struct TestLayout {
  size_t planes[2] = {0, 0};  // SPLIT3: planes of A and B
  size_t arena = 0, arena_bytes = 0;
  size_t total = 0;
};

// planes of A and B for a table-mode kind (0 for the class-mode bf16 kind)
void kind_planes(int32_t kind, int* pa, int* pb) {
  switch (kind) {
    case MAO_GEMM_SPLIT3: *pa = 3; *pb = 3; return;
    case MAO_GEMM_BF16_FOLD: *pa = 1; *pb = 1; return;
    case MAO_GEMM_SPLIT3_BF16: *pa = 3; *pb = 1; return;
    case MAO_GEMM_BF16_SPLIT3: *pa = 1; *pb = 3; return;
    case MAO_GEMM_SPLIT2: *pa = 2; *pb = 2; return;
    default: *pa = 0; *pb = 0; return;
  }
}

mao_status gemm_layout(int32_t kind_flags, int32_t batch, int32_t M, int32_t N, int32_t K, TestLayout& T) {
  if (batch < 1 || M < 1 || N < 1 || K < 1) return MAO_ERR_SHAPE;
  const int32_t kind = kind_flags & 15;
  if ((kind_flags & ~(15 | MAO_GEMM_FORCE_ONE_CTA | MAO_GEMM_FORCE_CTA_PAIR)) != 0) return MAO_ERR_INVALID_ARG;
  if (kind < MAO_GEMM_BF16 || kind > MAO_GEMM_SPLIT2) return MAO_ERR_INVALID_ARG;
  Carver cv;
  cv.take(kStatusBytes);
  if (kind != MAO_GEMM_BF16) {
    T.planes[0] = cv.take(3 * 2 * (size_t)batch * M * K);
    T.planes[1] = cv.take(3 * 2 * (size_t)batch * N * K);
    // per batch element: one problem and six descriptors
    T.arena_bytes = align_up((sizeof(GemmProblem) + 2 * sizeof(int)) * batch, 64) + sizeof(CUtensorMap) * 6 * batch + 256;
    T.arena = cv.take(T.arena_bytes);
  }
  T.total = cv.total();
  return MAO_OK;
}

}  // namespace

extern "C" mao_status mao_test_set_table_kernel(int32_t policy) { return set_table_kernel_policy(policy); }

namespace {

// One thread waits on an mbarrier that nothing arrives at, through the same bounded
// wait every kernel of the library uses: after kWaitLimitNs it records
// MAO_ERR_TIMEOUT (site kTestWaitSite) and returns.  The other threads leave at once.
constexpr int kTestWaitSite = 40;

__global__ void test_wait_timeout_kernel(DevStatus* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  abort_sh = 0;
  volatile int* abort_flag = &abort_sh;
  (void)mbar_wait(&bar, 0, status, kTestWaitSite, abort_flag);  // nothing completes the phase
}

}  // namespace

extern "C" mao_status mao_test_wait_timeout(void* workspace, size_t ws_bytes, mao_stream_t stream_) {
  if (workspace == nullptr || ws_bytes < sizeof(DevStatus)) return MAO_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MAO_ERR_ALIGN;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  DevStatus* status = reinterpret_cast<DevStatus*>(workspace);
  MAO_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream));
  test_wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

extern "C" mao_status mao_test_gemm_workspace_size(int32_t kind, int32_t batch, int32_t M, int32_t N, int32_t K,
                                                   size_t* bytes) {
  if (bytes == nullptr) return MAO_ERR_INVALID_ARG;
  TestLayout T;
  MAO_TRY(gemm_layout(kind, batch, M, N, K, T));
  *bytes = T.total;
  return MAO_OK;
}

extern "C" mao_status mao_test_gemm(int32_t kind_flags, int32_t a_mn_major, int32_t b_mn_major, const void* A,
                                    const void* B, float* D, int32_t batch, int32_t M, int32_t N, int32_t K,
                                    void* workspace, size_t ws_bytes, mao_stream_t stream_) {
  if (A == nullptr || B == nullptr || D == nullptr || workspace == nullptr) return MAO_ERR_INVALID_ARG;
  if ((a_mn_major != 0 && a_mn_major != 1) || (b_mn_major != 0 && b_mn_major != 1)) return MAO_ERR_INVALID_ARG;
  TestLayout T;
  MAO_TRY(gemm_layout(kind_flags, batch, M, N, K, T));
  const int32_t kind = kind_flags & 15;
  if (ws_bytes < T.total) return MAO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MAO_ERR_ALIGN;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return MAO_ERR_ALIGN;
  const int a_inner = a_mn_major ? M : K, b_inner = b_mn_major ? N : K;
  if (a_inner % 8 || b_inner % 8 || N % 4) return MAO_ERR_SHAPE;
  DeviceInfo* dev = nullptr;
  MAO_TRY(device_info(&dev));
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  MAO_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(DevStatus), stream));
  const int a_rows = a_mn_major ? K : M, b_rows = b_mn_major ? K : N;

  if (kind == MAO_GEMM_BF16) {
    auto view = [&](const void* base, int rows, int inner) {
      OperandView v;
      v.base = base;
      v.batch = (uint64_t)batch;
      v.inner = (uint64_t)inner;
      v.rows = (uint64_t)rows;
      v.ld = v.inner;
      v.bstride = (uint64_t)rows * inner;
      return v;
    };
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.nclasses = 1;
    p.alpha = 1.0f;
    p.status = status;
    MAO_TRY(encode_operand(&p.mapA[0], OP_BF16, a_mn_major, 128, view(A, a_rows, a_inner)));
    MAO_TRY(encode_operand(&p.mapB[0], OP_BF16, b_mn_major, 128, view(B, b_rows, b_inner)));
    p.cls[0] = GemmClass{M, N, K, batch, 0, 0, 0, D, (long long)M * N, N, nullptr, 0, 0, nullptr, 0, 0, nullptr};
    finalize_classes(p);
    const int force = (kind_flags & MAO_GEMM_FORCE_CTA_PAIR) ? 2 : (kind_flags & MAO_GEMM_FORCE_ONE_CTA) ? 1 : 0;
    return launch_gemm(OP_BF16, a_mn_major, b_mn_major, EPI_STORE_F32, p, stream, MAO_K_GEMM_TEST, force);
  }

  // table mode: the fp32 operands split into bf16 planes (a bf16 operand is its
  // own single plane), then one problem per batch element
  int pa = 0, pb = 0;
  kind_planes(kind, &pa, &pb);
  const size_t an = (size_t)batch * M * K, bn = (size_t)batch * N * K;
  __nv_bfloat16* ap = reinterpret_cast<__nv_bfloat16*>(ws + T.planes[0]);
  __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(ws + T.planes[1]);
  if (pa > 1) MAO_TRY(launch_split3(static_cast<const float*>(A), ap, ap + an, ap + 2 * an, an, stream));
  if (pb > 1) MAO_TRY(launch_split3(static_cast<const float*>(B), bp, bp + bn, bp + 2 * bn, bn, stream));
  const __nv_bfloat16* a0 = pa > 1 ? ap : static_cast<const __nv_bfloat16*>(A);
  const __nv_bfloat16* b0 = pb > 1 ? bp : static_cast<const __nv_bfloat16*>(B);
  Arena arena;
  arena.dev = ws + T.arena;
  MapSet maps;
  TableLaunch L;
  L.a_mn = a_mn_major;
  L.b_mn = b_mn_major;
  L.pa = pa;
  L.pb = pb;
  L.force_kernel = (kind_flags & MAO_GEMM_FORCE_CTA_PAIR) ? 2 : (kind_flags & MAO_GEMM_FORCE_ONE_CTA) ? 1 : 0;
  L.kernel_id = MAO_K_GEMM_TEST;
  for (int b = 0; b < batch; ++b) {
    const size_t ao = (size_t)b * M * K, bo = (size_t)b * N * K;
    Split3 As{{a0 + ao, nullptr, nullptr}, a_rows, a_inner, a_inner};
    Split3 Bs{{b0 + bo, nullptr, nullptr}, b_rows, b_inner, b_inner};
    for (int q = 1; q < pa; ++q) As.p[q] = ap + q * an + ao;
    for (int q = 1; q < pb; ++q) Bs.p[q] = bp + q * bn + bo;
    MAO_TRY(table_add(L, maps, As, Bs, M, N, K, 0, 0, D + (size_t)b * M * N, nullptr, N, nullptr, 0, 1.f, 0.f,
                      nullptr));
  }
  MAO_TRY(maps.encode_all());
  const size_t maps_off = arena.take(sizeof(CUtensorMap) * maps.maps.size(), 64);
  std::memcpy(arena.host.data() + maps_off, maps.maps.data(), sizeof(CUtensorMap) * maps.maps.size());
  const StagedLaunch S = table_stage(arena, L, maps_off);
  if (arena.host.size() > T.arena_bytes) return MAO_ERR_WORKSPACE;
  MAO_CUDA_TRY(cudaMemcpyAsync(arena.dev, arena.host.data(), arena.host.size(), cudaMemcpyHostToDevice, stream));
  (void)dev;
  return table_launch(arena, S, status, stream);
}

namespace mao {
Profiler& profiler() {
  static Profiler p;
  return p;
}
}  // namespace mao

extern "C" mao_status mao_profile_start(void** events, mao_launch_info* info, int32_t capacity) {
  if (capacity < 0 || (capacity > 0 && info == nullptr)) return MAO_ERR_INVALID_ARG;
  Profiler& P = profiler();
  if (info != nullptr && capacity > 0) {
    // executed-work counters: kept for the process, grown on demand, cleared here
    if (P.work_cap < capacity) {
      if (P.work) cudaFree(P.work);
      P.work = nullptr;
      P.work_cap = 0;
      MAO_CUDA_TRY(cudaMalloc(reinterpret_cast<void**>(&P.work), 2 * sizeof(unsigned long long) * capacity));
      P.work_cap = capacity;
    }
    MAO_CUDA_TRY(cudaMemset(P.work, 0, 2 * sizeof(unsigned long long) * capacity));
    P.counted.assign(capacity, 0);
  } else {
    P.counted.assign(std::max(capacity, 0), 0);
  }
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
  if (P.info == nullptr) return P.count;
  const int n = std::min(P.count, P.capacity);
  std::vector<unsigned long long> h;
  bool have = false;
  bool any = false;
  for (int i = 0; i < n; ++i) any = any || P.counted[i];
  if (any && P.work != nullptr) {
    h.resize(2 * (size_t)n);
    have = cudaDeviceSynchronize() == cudaSuccess &&
           cudaMemcpy(h.data(), P.work, sizeof(unsigned long long) * h.size(), cudaMemcpyDeviceToHost) == cudaSuccess;
  }
  for (int i = 0; i < n; ++i) {
    if (have && P.counted[i]) {
      P.info[i].exec_flops = (double)h[2 * i];
      P.info[i].exec_tc_flops = (double)h[2 * i + 1];
    } else {
      P.info[i].exec_flops = P.info[i].flops;
      P.info[i].exec_tc_flops = P.info[i].tc_flops;
    }
  }
  return P.count;
}
