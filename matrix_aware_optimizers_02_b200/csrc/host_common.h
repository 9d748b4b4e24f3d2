// Host-side helpers shared by the C-ABI entry points: status plumbing, device
// facts, TMA descriptor encoding, workspace carving, GEMM launch helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
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
  bool gemm_pair_attr_set[64] = {};
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

// Launch one class-mode (bf16) grouped GEMM of the given instantiation;
// kernel_id tags the launch for the profiler.  force: 0 = the library's choice
// between the one-CTA kernel (128 x 256 tiles) and the CTA-pair kernel (256 x 256),
// 1 = one CTA, 2 = CTA pairs.
mao_status launch_gemm(int kind, int a_mn, int b_mn, int epi, const GemmParams& p, cudaStream_t stream,
                       int kernel_id, int force = 0);

// Fill tile bookkeeping of the classes in p (M, N, K, count must be set).
void finalize_classes(GemmParams& p);

// fp32 -> three bf16 planes (x = p0 + p1 + p2).
mao_status launch_split3(const float* src, __nv_bfloat16* p0, __nv_bfloat16* p1, __nv_bfloat16* p2, size_t n,
                         cudaStream_t stream);

}  // namespace mao

namespace mao {

// Launch profiler state (see mao_profile_start in mao.h).
struct Profiler {
  bool active = false;
  void** events = nullptr;
  mao_launch_info* info = nullptr;
  int capacity = 0;
  int count = 0;
  // device counters of executed work, two per recorded launch (table-mode products
  // only: `counted` marks the slots whose launch writes them)
  unsigned long long* work = nullptr;
  int work_cap = 0;
  std::vector<char> counted;
};
Profiler& profiler();

// RAII bracket around one kernel launch: while the profiler is active, records
// an event before the launch (constructor) and one after it (destructor) on the
// launching stream, with the launch's algorithmic work.
struct LaunchScope {
  cudaStream_t s;
  int slot = -1;
  LaunchScope(cudaStream_t stream, int kernel, double flops, double bytes, double tc_flops = -1.0) : s(stream) {
    Profiler& P = profiler();
    if (!P.active) return;
    const int i = P.count++;
    if (i < P.capacity) {
      slot = i;
      P.info[i].kernel = kernel;
      P.info[i].pad = 0;
      P.info[i].flops = flops;
      P.info[i].bytes = bytes;
      P.info[i].tc_flops = tc_flops >= 0.0 ? tc_flops : flops;
      if (P.events) cudaEventRecord(static_cast<cudaEvent_t>(P.events[2 * i]), s);
    }
  }
  ~LaunchScope() {
    if (slot >= 0 && profiler().events) cudaEventRecord(static_cast<cudaEvent_t>(profiler().events[2 * slot + 1]), s);
  }
};

}  // namespace mao

namespace mao {

// ---------------------------------------------------------------- staging arena
// Host image of a device region: everything a step needs in device memory that
// the host prepares (problem tables, tensor maps, per-matrix descriptors) is
// laid out here and copied with one cudaMemcpyAsync.
struct Arena {
  uint8_t* dev = nullptr;   // device base (inside the workspace), or nullptr while sizing
  size_t cap = 0;
  std::vector<uint8_t> host;
  size_t take(size_t bytes, size_t align = 64) {
    size_t at = align_up(host.size(), align);
    host.resize(at + bytes);
    return at;
  }
  template <class T>
  T* hptr(size_t off) { return reinterpret_cast<T*>(host.data() + off); }
  template <class T>
  T* dptr(size_t off) const { return dev ? reinterpret_cast<T*>(dev + off) : nullptr; }
};

// An fp32 row-major matrix held as three bf16 planes x = p0 + p1 + p2 (operand
// of an fp32-faithful SPLIT3 product); ld in elements, a multiple of 8.  A bf16
// matrix is its own single plane (p[1] = p[2] = nullptr).
struct Split3 {
  const __nv_bfloat16* p[3];
  int rows, cols, ld;
};

// Collects the problems of one table-mode SPLIT3 launch (fixed operand majors):
//   out (M x N) = alpha * op(A) op(B) + beta * aux
// with op(A) = A (a_mn = 0, A stored M x K) or A^T (a_mn = 1, A stored K x M), and
// op(B) = B^T (b_mn = 0, B stored N x K) or B (b_mn = 1, B stored K x N).
//
// pa / pb: planes used per operand (1: a bf16 operand, exact in one plane; 3: an
// fp32 operand; 2: a 16-bit-significand approximation).  Every problem of a
// launch uses the same counts.
struct TableLaunch {
  int a_mn = 0, b_mn = 0;
  int pa = 3, pb = 3;
  int force_kernel = 0;  // 0: choose, 1: one-CTA kernel, 2: CTA-pair kernel (verification)
  int kernel_id = 0;
  const int* any = nullptr;  // launch-level gate (GemmTableParams::any), or nullptr
  std::vector<GemmProblem> probs;
  std::vector<int> map_idx;  // 6 per problem: A planes 0..2, B planes 0..2 (indices into the step's map list)
};

struct MapKey {
  const void* p;
  int inner, rows, ld, box_rows, mn;
  bool operator==(const MapKey& o) const {
    return p == o.p && inner == o.inner && rows == o.rows && ld == o.ld && box_rows == o.box_rows && mn == o.mn;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<const void*>()(k.p);
    h ^= (size_t)k.inner * 0x9E3779B97F4A7C15ull + (size_t)k.rows * 0xC2B2AE3D27D4EB4Full +
         (size_t)k.ld * 0x165667B19E3779F9ull + (size_t)k.box_rows * 31 + (size_t)k.mn;
    return h;
  }
};

// The tensor maps one step needs, de-duplicated.
struct MapSet {
  std::vector<MapKey> keys;
  std::vector<CUtensorMap> maps;
  std::unordered_map<MapKey, int, MapKeyHash> index;
  int get(const void* p, int inner, int rows, int ld, int box_rows, int mn);  // index (encodes lazily)
  mao_status encode_all();
};

// Add a problem; A/B describe the stored matrices (see TableLaunch).  m_off / n_off
// shift the operand coordinates (sub-block products); they must be multiples of 8
// when the operand is MN-major (TMA inner coordinate alignment).  k_off starts the
// product at K index k_off of both operands (a K slice); a multiple of 8 when
// either operand is K-major.  `outp`, when
// given, receives the three-plane split of the result.
mao_status table_add(TableLaunch& L, MapSet& maps, const Split3& A, const Split3& B, int M, int N, int K,
                     int m_off, int n_off, float* out, const Split3* outp, int ld_out, const float* aux,
                     int ld_aux, float alpha, float beta, const int* flag, int k_off = 0);

// Give the last problem added to L an alternate destination, used when *sel == 0
// on the device (sel is read by every tile's epilogue).
mao_status table_set_alt(TableLaunch& L, const int* sel, float* out2, const Split3* out2p, int ld_out2);

// Ask the last problem added to L for update statistics (see GemmProblem::upd):
// `upd` holds ceil(M / 32) * ceil(N / 64) float2 slots.  Needs an aux operand.
mao_status table_set_stats(TableLaunch& L, float2* upd);

// Process-wide kernel choice for table-mode launches (0 auto, 1 one CTA, 2 CTA pair).
int table_kernel_policy();
mao_status set_table_kernel_policy(int policy);

// Stage a launch's problem table into the arena (maps live at maps_off) and launch it.
struct StagedLaunch {
  size_t probs_off = 0;
  int nprob = 0;
  int total_tiles = 0;
  int a_mn = 0, b_mn = 0, kernel_id = 0;
  int pa = 3, pb = 3;
  int total_tiles2 = 0;  // 256-row tiles (CTA-pair kernel)
  bool pair = false;     // launch the CTA-pair kernel
  double flops = 0.0;
  const int* any = nullptr;
};
StagedLaunch table_stage(Arena& A, const TableLaunch& L, size_t maps_off);
mao_status table_launch(const Arena& A, const StagedLaunch& S, DevStatus* status, cudaStream_t stream);

// One table-mode launch for a plane pair (instantiated in gemm_table_p*.cu).
template <int PA, int PB>
mao_status launch_table_planes(const GemmTableParams& p, int a_mn, int b_mn, cudaStream_t stream, int kernel_id,
                               double flops, bool pair);

}  // namespace mao
