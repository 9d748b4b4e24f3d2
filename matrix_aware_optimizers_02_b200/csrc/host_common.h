// Host-side helpers shared by the C-ABI entry points: status plumbing, device
// facts, TMA descriptor encoding, workspace carving, GEMM launch helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "gemm_tc.cuh"
#include "mao.h"

namespace mao {

#define MAO_CUDA_TRY(expr)                     \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return MAO_ERR_CUDA; \
  } while (0)

#define MAO_TRY(expr)                 \
  do {                                \
    mao_status _s = (expr);           \
    if (_s != MAO_OK) return _s;      \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int round_up_int(int x, int a) { return (x + a - 1) / a * a; }

// Sequential carving of a workspace into 256-byte aligned regions.
struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    off = align_up(off, 256);
    size_t at = off;
    off += bytes;
    return at;
  }
  size_t total() const { return align_up(off, 256); }
};

constexpr size_t kStatusBytes = 256;  // DevStatus at workspace offset 0

struct DeviceInfo {
  int sm_count = 0;
  int major = 0, minor = 0;
  bool gemm_attr_set[64] = {};
};

mao_status device_info(DeviceInfo** out);
mao_status encode_3d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                     uint64_t rows, uint64_t batch, uint64_t ld_elems, uint64_t batch_stride_elems,
                     uint32_t box_inner, uint32_t box_rows, bool atom32 = false);

// Operand descriptor for one class of a grouped GEMM: tensor [batch][rows][ld]
// (rows x inner valid), plus the box shape the kernel expects for its major.
struct OperandView {
  const void* base;
  uint64_t inner, rows, batch, ld, bstride;
};

// Encode the TMA descriptor of an operand: K-major operands are [batch][MN][K]
// and use boxes {128 B of K, R rows}; MN-major ones are [batch][K][MN] and use
// boxes {128 B of MN, BK K-rows}.
mao_status encode_operand(CUtensorMap* map, int kind, int mn_major, int R, const OperandView& v);

// Launch one grouped GEMM of the given instantiation.  `lo` may be null for bf16.
// kernel_id tags the launch for the profiler.
mao_status launch_gemm(int kind, int a_mn, int b_mn, int epi, const GemmParams& p, const GemmLoMaps* lo,
                       cudaStream_t stream, int kernel_id);

// Fill tile bookkeeping of the classes in p (M, N, K, count must be set).
void finalize_classes(GemmParams& p);

mao_status launch_tf32_split(const float* src, float* hi, float* lo, size_t n, cudaStream_t stream);

}  // namespace mao

namespace mao {

// Launch profiler state (see mao_profile_start in mao.h).
struct Profiler {
  bool active = false;
  void** events = nullptr;
  mao_launch_info* info = nullptr;
  int capacity = 0;
  int count = 0;
};
Profiler& profiler();

// RAII bracket around one kernel launch: while the profiler is active, records
// an event before the launch (constructor) and one after it (destructor) on the
// launching stream, with the launch's algorithmic work.
struct LaunchScope {
  cudaStream_t s;
  int slot = -1;
  LaunchScope(cudaStream_t stream, int kernel, double flops, double bytes) : s(stream) {
    Profiler& P = profiler();
    if (!P.active) return;
    const int i = P.count++;
    if (i < P.capacity) {
      slot = i;
      P.info[i].kernel = kernel;
      P.info[i].pad = 0;
      P.info[i].flops = flops;
      P.info[i].bytes = bytes;
      cudaEventRecord(static_cast<cudaEvent_t>(P.events[2 * i]), s);
    }
  }
  ~LaunchScope() {
    if (slot >= 0) cudaEventRecord(static_cast<cudaEvent_t>(profiler().events[2 * slot + 1]), s);
  }
};

}  // namespace mao
