// Host side of the grouped tcgen05 GEMM: device facts, TMA descriptor
// encoding, tile bookkeeping and the launch dispatchers; plus the fp32 ->
// three bf16 planes split used by the fp32-faithful (SPLIT3) products.
#include <cudaTypedefs.h>

#include <atomic>

#include "host_common.h"

namespace mao {

namespace {

std::mutex g_mu;
DeviceInfo g_dev[64];
bool g_dev_ok[64] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

mao_status get_encode(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || f == nullptr)
      return MAO_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  *fn = g_encode;
  return MAO_OK;
}

}  // namespace

mao_status device_info(DeviceInfo** out) {
  int dev = 0;
  MAO_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MAO_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_dev_ok[dev]) {
    DeviceInfo& d = g_dev[dev];
    MAO_CUDA_TRY(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
    MAO_CUDA_TRY(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
    MAO_CUDA_TRY(cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev));
    g_dev_ok[dev] = true;
  }
  if (g_dev[dev].major != 10) return MAO_ERR_UNSUPPORTED;
  *out = &g_dev[dev];
  return MAO_OK;
}

mao_status encode_3d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                     uint64_t rows, uint64_t batch, uint64_t ld_elems, uint64_t batch_stride_elems,
                     uint32_t box_inner, uint32_t box_rows, bool atom32) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  MAO_TRY(get_encode(&enc));
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {ld_elems * (uint64_t)esize, batch_stride_elems * (uint64_t)esize};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MAO_OK : MAO_ERR_CUDA;
}

mao_status encode_operand(CUtensorMap* map, int kind, int mn_major, int R, const OperandView& v) {
  (void)kind;  // every operand plane is bf16
  const uint32_t row_elems = 64;  // bf16 elements in one 128-byte swizzle row
  return encode_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v.base, v.inner, v.rows, v.batch, v.ld, v.bstride,
                   row_elems, mn_major ? row_elems : (uint32_t)R, false);
}

void finalize_classes(GemmParams& p) {
  int t = 0, t2 = 0;
  for (int c = 0; c < p.nclasses; ++c) {
    GemmClass& C = p.cls[c];
    C.tiles_n = (C.N + 255) / 256;
    C.tiles_per_mat = ((C.M + 127) / 128) * C.tiles_n;
    C.tiles_per_mat2 = ((C.M + 255) / 256) * C.tiles_n;
    C.tile_begin = t;
    C.tile_begin2 = t2;
    t += C.tiles_per_mat * C.count;
    t2 += C.tiles_per_mat2 * C.count;
  }
  p.total_tiles = p.total_tiles1 = t;
  p.total_tiles2 = t2;
}

namespace {

template <int KIND, int A_MN, int B_MN, int EPI>
mao_status launch_one(const GemmParams& p, cudaStream_t stream, int kernel_id) {
  using Cfg = GemmCfg<KIND, A_MN, B_MN>;
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  auto kern = gemm_tc_kernel<KIND, A_MN, B_MN, EPI>;
  const int slot = ((KIND * 2 + A_MN) * 2 + B_MN) * 4 + EPI;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d->gemm_attr_set[slot]) {
      MAO_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
      d->gemm_attr_set[slot] = true;
    }
  }
  if (p.total_tiles <= 0) return MAO_OK;
  const int grid = p.total_tiles < d->sm_count ? p.total_tiles : d->sm_count;
  double flops = 0.0, bytes = 0.0;
  const double es = Cfg::ESIZE, ob = (EPI == EPI_STORE_F32) ? 4.0 : 2.0;
  for (int c = 0; c < p.nclasses; ++c) {
    const GemmClass& C = p.cls[c];
    flops += 2.0 * C.count * (double)C.M * C.N * C.K;
    bytes += C.count * (es * ((double)C.M * C.K + (double)C.N * C.K) + ob * (double)C.M * C.N *
                                                                                         (EPI == EPI_AXPY_T ? 2 : 1) +
                        ((EPI == EPI_POLY || EPI == EPI_AXPY_T) ? 2.0 * C.M * C.N : 0.0));
  }
  LaunchScope ls(stream, kernel_id, flops, bytes);
  kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

// The same products on CTA pairs: 256 x 256 tiles (each CTA loads its 128 rows of A
// and 128 of B's 256 columns), one cta_group::2 MMA per k-step.
template <int A_MN, int B_MN, int EPI>
mao_status launch_one_pair(const GemmParams& p, cudaStream_t stream, int kernel_id) {
  using Cfg = GemmPairCfg<A_MN, B_MN, 1, 1, OP_BF16>;
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  auto kern = gemm_tc_pair_class_kernel<A_MN, B_MN, EPI>;
  const int slot = (A_MN * 2 + B_MN) * 4 + EPI;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d->gemm_pair_attr_set[slot]) {
      MAO_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
      d->gemm_pair_attr_set[slot] = true;
    }
  }
  GemmParams q = p;
  q.total_tiles = p.total_tiles2;
  if (q.total_tiles <= 0) return MAO_OK;
  const int max_pairs = d->sm_count / 2;
  const int pairs = q.total_tiles < max_pairs ? q.total_tiles : max_pairs;
  double flops = 0.0, bytes = 0.0;
  const double ob = (EPI == EPI_STORE_F32) ? 4.0 : 2.0;
  for (int c = 0; c < p.nclasses; ++c) {
    const GemmClass& C = p.cls[c];
    flops += 2.0 * C.count * (double)C.M * C.N * C.K;
    bytes += C.count * (2.0 * ((double)C.M * C.K + (double)C.N * C.K) + ob * (double)C.M * C.N *
                                                                              (EPI == EPI_AXPY_T ? 2 : 1) +
                        ((EPI == EPI_POLY || EPI == EPI_AXPY_T) ? 2.0 * C.M * C.N : 0.0));
  }
  LaunchScope ls(stream, kernel_id, flops, bytes);
  kern<<<2 * pairs, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(q);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

template <int KIND, int A_MN, int B_MN>
mao_status launch_epi(int epi, const GemmParams& p, cudaStream_t s, int k, bool pair) {
  if (pair) {
    switch (epi) {
      case EPI_STORE_F32: return launch_one_pair<A_MN, B_MN, EPI_STORE_F32>(p, s, k);
      case EPI_GRAM: return launch_one_pair<A_MN, B_MN, EPI_GRAM>(p, s, k);
      case EPI_POLY: return launch_one_pair<A_MN, B_MN, EPI_POLY>(p, s, k);
      case EPI_AXPY_T: return launch_one_pair<A_MN, B_MN, EPI_AXPY_T>(p, s, k);
      default: return MAO_ERR_INVALID_ARG;
    }
  }
  switch (epi) {
    case EPI_STORE_F32: return launch_one<KIND, A_MN, B_MN, EPI_STORE_F32>(p, s, k);
    case EPI_GRAM: return launch_one<KIND, A_MN, B_MN, EPI_GRAM>(p, s, k);
    case EPI_POLY: return launch_one<KIND, A_MN, B_MN, EPI_POLY>(p, s, k);
    case EPI_AXPY_T: return launch_one<KIND, A_MN, B_MN, EPI_AXPY_T>(p, s, k);
    default: return MAO_ERR_INVALID_ARG;
  }
}

}  // namespace

mao_status launch_gemm(int kind, int a_mn, int b_mn, int epi, const GemmParams& p, cudaStream_t stream, int k,
                       int force) {
  if (kind != OP_BF16) return MAO_ERR_UNSUPPORTED;
  // CTA pairs when their 256-row tiles fill the GPU's pairs and waste at most a fifth
  // of the rows (as for the table-mode products)
  const int f = force ? force : table_kernel_policy();
  const bool pair = f == 2 || (f == 0 && p.total_tiles2 >= 74 && 2.0 * p.total_tiles2 <= 1.2 * p.total_tiles1);
  if (!a_mn && !b_mn) return launch_epi<OP_BF16, 0, 0>(epi, p, stream, k, pair);
  if (!a_mn && b_mn) return launch_epi<OP_BF16, 0, 1>(epi, p, stream, k, pair);
  if (epi != EPI_STORE_F32) return MAO_ERR_UNSUPPORTED;
  if (a_mn && !b_mn)
    return pair ? launch_one_pair<1, 0, EPI_STORE_F32>(p, stream, k) : launch_one<OP_BF16, 1, 0, EPI_STORE_F32>(p, stream, k);
  return pair ? launch_one_pair<1, 1, EPI_STORE_F32>(p, stream, k) : launch_one<OP_BF16, 1, 1, EPI_STORE_F32>(p, stream, k);
}

// ------------------------------------------------------------------ three-plane split
namespace {

// x = p0 + p1 + p2 with each plane the bf16 rounding of what the previous planes
// left over; the three planes keep 24 significant bits of x.
__global__ void split3_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ p0,
                              __nv_bfloat16* __restrict__ p1, __nv_bfloat16* __restrict__ p2, size_t n) {
  size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (; i < n; i += stride) {
    float r = src[i];
    const __nv_bfloat16 a = __float2bfloat16_rn(r);
    r -= __bfloat162float(a);
    const __nv_bfloat16 b = __float2bfloat16_rn(r);
    r -= __bfloat162float(b);
    p0[i] = a;
    p1[i] = b;
    p2[i] = __float2bfloat16_rn(r);
  }
}

}  // namespace

mao_status launch_split3(const float* src, __nv_bfloat16* p0, __nv_bfloat16* p1, __nv_bfloat16* p2, size_t n,
                         cudaStream_t stream) {
  if (n == 0) return MAO_OK;
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  size_t blocks = (n + 255) / 256;
  const size_t cap = (size_t)d->sm_count * 8;
  if (blocks > cap) blocks = cap;
  LaunchScope ls(stream, MAO_K_SPLIT3, 0.0, 10.0 * (double)n);
  split3_kernel<<<(unsigned)blocks, 256, 0, stream>>>(src, p0, p1, p2, n);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

}  // namespace mao

// ------------------------------------------------------------------ table mode
namespace mao {

int MapSet::get(const void* p, int inner, int rows, int ld, int box_rows, int mn) {
  MapKey k{p, inner, rows, ld, box_rows, mn};
  auto it = index.find(k);
  if (it != index.end()) return it->second;
  keys.push_back(k);
  const int i = (int)keys.size() - 1;
  index.emplace(k, i);
  return i;
}

mao_status MapSet::encode_all() {
  maps.resize(keys.size());
  for (size_t i = 0; i < keys.size(); ++i) {
    const MapKey& k = keys[i];
    MAO_TRY(encode_3d(&maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k.p, (uint64_t)k.inner, (uint64_t)k.rows, 1,
                      (uint64_t)k.ld, (uint64_t)k.ld * k.rows, 64, (uint32_t)k.box_rows, false));
  }
  return MAO_OK;
}

mao_status table_add(TableLaunch& L, MapSet& maps, const Split3& A, const Split3& B, int M, int N, int K,
                     int m_off, int n_off, float* out, const Split3* outp, int ld_out, const float* aux,
                     int ld_aux, float alpha, float beta, const int* flag, int k_off) {
  if (M <= 0 || N <= 0 || K <= 0) return MAO_OK;
  if ((L.a_mn && (m_off & 7)) || (L.b_mn && (n_off & 7))) return MAO_ERR_INVALID_ARG;
  if (k_off < 0 || ((!L.a_mn || !L.b_mn) && (k_off & 7))) return MAO_ERR_INVALID_ARG;
  if ((A.ld & 7) || (B.ld & 7)) return MAO_ERR_SHAPE;
  for (int q = 0; q < L.pa; ++q)
    if (A.p[q] == nullptr) return MAO_ERR_INVALID_ARG;
  for (int q = 0; q < L.pb; ++q)
    if (B.p[q] == nullptr) return MAO_ERR_INVALID_ARG;
  // operand views: inner extent = the stored matrix's columns, rows = its rows
  // B boxes are 64 rows in both majors: a CTA pair loads half of a 128-column B tile each
  const int abox = L.a_mn ? 64 : 128, bbox = 64;
  int idx[6];
  for (int q = 0; q < 3; ++q) {
    idx[q] = q < L.pa ? maps.get(A.p[q], A.cols, A.rows, A.ld, abox, L.a_mn) : -1;
    idx[3 + q] = q < L.pb ? maps.get(B.p[q], B.cols, B.rows, B.ld, bbox, L.b_mn) : -1;
  }
  GemmProblem P;
  std::memset(&P, 0, sizeof(P));
  P.out = out;
  if (outp) {
    if (outp->ld & 7) return MAO_ERR_SHAPE;
    for (int q = 0; q < 3; ++q) P.out_p[q] = const_cast<__nv_bfloat16*>(outp->p[q]);
    P.ld_outp = outp->ld;
  }
  P.aux = aux;
  P.flag = flag;
  P.M = M;
  P.N = N;
  P.K = K;
  P.m_off = m_off;
  P.n_off = n_off;
  P.k_off = k_off;
  P.ld_out = ld_out;
  P.ld_aux = ld_aux;
  P.tiles_n = (N + 127) / 128;
  P.alpha = alpha;
  P.beta = beta;
  L.probs.push_back(P);
  L.map_idx.insert(L.map_idx.end(), idx, idx + 6);
  return MAO_OK;
}

namespace {
std::atomic<int> g_table_policy{0};
}
int table_kernel_policy() { return g_table_policy.load(std::memory_order_relaxed); }
mao_status set_table_kernel_policy(int policy) {
  if (policy < 0 || policy > 2) return MAO_ERR_INVALID_ARG;
  g_table_policy.store(policy, std::memory_order_relaxed);
  return MAO_OK;
}

mao_status table_set_stats(TableLaunch& L, float2* upd) {
  if (L.probs.empty() || upd == nullptr || L.probs.back().aux == nullptr) return MAO_ERR_INVALID_ARG;
  L.probs.back().upd = upd;
  return MAO_OK;
}

mao_status table_set_alt(TableLaunch& L, const int* sel, float* out2, const Split3* out2p, int ld_out2) {
  if (L.probs.empty() || sel == nullptr) return MAO_ERR_INVALID_ARG;
  GemmProblem& P = L.probs.back();
  P.sel = sel;
  P.out2 = out2;
  P.ld_out2 = ld_out2;
  if (out2p) {
    if (out2p->ld & 7) return MAO_ERR_SHAPE;
    for (int q = 0; q < 3; ++q) P.out2_p[q] = const_cast<__nv_bfloat16*>(out2p->p[q]);
    P.ld_out2p = out2p->ld;
  }
  return MAO_OK;
}

StagedLaunch table_stage(Arena& A, const TableLaunch& L, size_t maps_off) {
  StagedLaunch S;
  S.nprob = (int)L.probs.size();
  S.a_mn = L.a_mn;
  S.b_mn = L.b_mn;
  S.pa = L.pa;
  S.pb = L.pb;
  S.kernel_id = L.kernel_id;
  if (S.nprob == 0) return S;
  // the problem records, then their first tiles in both numberings (searched by the kernels)
  S.probs_off = A.take(sizeof(GemmProblem) * S.nprob + 2 * sizeof(int) * S.nprob, 64);
  GemmProblem* hp = A.hptr<GemmProblem>(S.probs_off);
  int* starts = reinterpret_cast<int*>(hp + S.nprob);
  const CUtensorMap* mbase = A.dptr<const CUtensorMap>(maps_off);
  int t = 0, t2 = 0;
  for (int i = 0; i < S.nprob; ++i) {
    GemmProblem P = L.probs[i];
    for (int q = 0; q < 3; ++q) {
      const int ia = L.map_idx[6 * i + q], ib = L.map_idx[6 * i + 3 + q];
      P.mapA[q] = (mbase && ia >= 0) ? mbase + ia : nullptr;
      P.mapB[q] = (mbase && ib >= 0) ? mbase + ib : nullptr;
    }
    // column tiles: the one-CTA kernel's are 256 wide for one-plane operands (GemmCfg)
    const int bn1 = (L.pa == 1 && L.pb == 1) ? 256 : 128;
    P.tiles_n = (P.N + bn1 - 1) / bn1;
    P.tiles_n2 = (P.N + 127) / 128;
    P.tile_begin = t;
    t += ((P.M + 127) / 128) * P.tiles_n;
    P.tile_begin2 = t2;
    t2 += ((P.M + 255) / 256) * P.tiles_n2;
    // work recorded for the profiler: only problems that always run (a problem gated
    // by a device flag may be skipped, so it counts nothing: a lower bound)
    if (P.flag == nullptr) S.flops += 2.0 * P.M * (double)P.N * P.K;
    hp[i] = P;
    starts[i] = P.tile_begin;
    starts[S.nprob + i] = P.tile_begin2;
  }
  S.total_tiles = t;
  S.total_tiles2 = t2;
  // the CTA-pair kernel when its 256-row tiles fill the GPU's pairs and waste at most
  // a fifth of the rows (a 128-row remainder of M costs a half tile).  The library
  // chooses it for products with a three-plane operand, where it relieves the
  // shared-memory operand stream; bf16 x bf16 products are bound by their epilogue
  // and stay on one CTA unless a caller forces the pair kernel.
  const bool pair_auto = L.pa == 3 || L.pb == 3;
  const int force = L.force_kernel ? L.force_kernel : table_kernel_policy();
  S.pair = force == 2 || (force == 0 && pair_auto && t2 >= 74 && 2.0 * t2 <= 1.2 * t);
  S.any = L.any;
  return S;
}

mao_status table_launch(const Arena& A, const StagedLaunch& S, DevStatus* status, cudaStream_t stream) {
  if (S.nprob == 0) return MAO_OK;
  GemmTableParams p;
  p.probs = A.dptr<const GemmProblem>(S.probs_off);
  p.nprob = S.nprob;
  p.total_tiles = S.pair ? S.total_tiles2 : S.total_tiles;
  p.status = status;
  p.any = S.any;
  p.work = nullptr;
  Profiler& prof = profiler();
  const int total = S.pair ? S.total_tiles2 : S.total_tiles;
  if (prof.active && prof.work != nullptr && total > 0 && prof.count < prof.capacity) {
    // the launch below takes the profiler's next slot
    p.work = prof.work + 2 * (size_t)prof.count;
    prof.counted[prof.count] = 1;
  }
  const int key = S.pa * 10 + S.pb;
  switch (key) {
    case 33: return launch_table_planes<3, 3>(p, S.a_mn, S.b_mn, stream, S.kernel_id, S.flops, S.pair);
    case 31: return launch_table_planes<3, 1>(p, S.a_mn, S.b_mn, stream, S.kernel_id, S.flops, S.pair);
    case 13: return launch_table_planes<1, 3>(p, S.a_mn, S.b_mn, stream, S.kernel_id, S.flops, S.pair);
    case 11: return launch_table_planes<1, 1>(p, S.a_mn, S.b_mn, stream, S.kernel_id, S.flops, S.pair);
    case 22: return launch_table_planes<2, 2>(p, S.a_mn, S.b_mn, stream, S.kernel_id, S.flops, S.pair);
    default: return MAO_ERR_INVALID_ARG;
  }
}

}  // namespace mao
