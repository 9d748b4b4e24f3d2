// Host side of the grouped tcgen05 GEMM: device facts, TMA descriptor
// encoding, tile bookkeeping and the launch dispatcher; plus the fp32 -> hi/lo
// tf32 split used by the fp32-faithful (3xTF32) products.
#include <cudaTypedefs.h>

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
  const int esize = (kind == OP_BF16) ? 2 : 4;
  const CUtensorMapDataType dt =
      (kind == OP_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint32_t row_elems = 128 / esize;  // elements in one 128-byte swizzle row
  if (!mn_major)
    return encode_3d(map, dt, esize, v.base, v.inner, v.rows, v.batch, v.ld, v.bstride, row_elems, R, false);
  // MN-major 32-bit operands need the 32-byte-atom variant of the 128-byte swizzle
  return encode_3d(map, dt, esize, v.base, v.inner, v.rows, v.batch, v.ld, v.bstride, row_elems, row_elems,
                   esize == 4);
}

void finalize_classes(GemmParams& p) {
  int t = 0;
  for (int c = 0; c < p.nclasses; ++c) {
    GemmClass& C = p.cls[c];
    const int tm = (C.M + 127) / 128;
    C.tiles_n = (C.N + 255) / 256;
    C.tiles_per_mat = tm * C.tiles_n;
    C.tile_begin = t;
    t += C.tiles_per_mat * C.count;
  }
  p.total_tiles = t;
}

namespace {

template <int KIND, int A_MN, int B_MN, int EPI>
mao_status launch_one(const GemmParams& p, const GemmLoMaps* lo, cudaStream_t stream, int kernel_id) {
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
  static const GemmLoMaps kEmptyLo = {};
  const int grid = p.total_tiles < d->sm_count ? p.total_tiles : d->sm_count;
  double flops = 0.0, bytes = 0.0;
  const double es = Cfg::ESIZE, ob = (EPI == EPI_STORE_F32) ? 4.0 : 2.0;
  for (int c = 0; c < p.nclasses; ++c) {
    const GemmClass& C = p.cls[c];
    flops += 2.0 * C.count * (double)C.M * C.N * C.K;
    bytes += C.count * (es * ((double)C.M * C.K + (double)C.N * C.K) * Cfg::PLANES + ob * (double)C.M * C.N *
                                                                                         (EPI == EPI_AXPY_T ? 2 : 1) +
                        ((EPI == EPI_POLY || EPI == EPI_AXPY_T) ? 2.0 * C.M * C.N : 0.0));
  }
  LaunchScope ls(stream, kernel_id, flops, bytes);
  kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(p, lo ? *lo : kEmptyLo);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

template <int KIND, int A_MN, int B_MN>
mao_status launch_epi(int epi, const GemmParams& p, const GemmLoMaps* lo, cudaStream_t s, int k) {
  switch (epi) {
    case EPI_STORE_F32: return launch_one<KIND, A_MN, B_MN, EPI_STORE_F32>(p, lo, s, k);
    case EPI_GRAM: return launch_one<KIND, A_MN, B_MN, EPI_GRAM>(p, lo, s, k);
    case EPI_POLY: return launch_one<KIND, A_MN, B_MN, EPI_POLY>(p, lo, s, k);
    case EPI_AXPY_T: return launch_one<KIND, A_MN, B_MN, EPI_AXPY_T>(p, lo, s, k);
    default: return MAO_ERR_INVALID_ARG;
  }
}

}  // namespace

mao_status launch_gemm(int kind, int a_mn, int b_mn, int epi, const GemmParams& p, const GemmLoMaps* lo,
                       cudaStream_t stream, int k) {
  if (kind == OP_BF16) {
    if (!a_mn && !b_mn) return launch_epi<OP_BF16, 0, 0>(epi, p, lo, stream, k);
    if (!a_mn && b_mn) return launch_epi<OP_BF16, 0, 1>(epi, p, lo, stream, k);
    if (epi != EPI_STORE_F32) return MAO_ERR_UNSUPPORTED;
    if (a_mn && !b_mn) return launch_one<OP_BF16, 1, 0, EPI_STORE_F32>(p, lo, stream, k);
    return launch_one<OP_BF16, 1, 1, EPI_STORE_F32>(p, lo, stream, k);
  }
  if (kind == OP_TF32X3) {
    if (epi != EPI_STORE_F32 || lo == nullptr) return MAO_ERR_UNSUPPORTED;
    if (!a_mn && !b_mn) return launch_one<OP_TF32X3, 0, 0, EPI_STORE_F32>(p, lo, stream, k);
    if (!a_mn && b_mn) return launch_one<OP_TF32X3, 0, 1, EPI_STORE_F32>(p, lo, stream, k);
    if (a_mn && !b_mn) return launch_one<OP_TF32X3, 1, 0, EPI_STORE_F32>(p, lo, stream, k);
    return launch_one<OP_TF32X3, 1, 1, EPI_STORE_F32>(p, lo, stream, k);
  }
  return MAO_ERR_INVALID_ARG;
}

// ------------------------------------------------------------------ tf32 split
namespace {

// x = hi + lo with hi = tf32(x) and lo = tf32(x - hi): both exactly representable
// in tf32, so the tensor core sees them without further rounding.
__global__ void tf32_split_kernel(const float* __restrict__ src, float* __restrict__ hi, float* __restrict__ lo,
                                  size_t n) {
  size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  const size_t stride = (size_t)gridDim.x * blockDim.x * 4;
  for (; i < n; i += stride) {
    if (i + 4 <= n) {
      float4 x = *reinterpret_cast<const float4*>(src + i);
      float4 h = make_float4(tf32_rna(x.x), tf32_rna(x.y), tf32_rna(x.z), tf32_rna(x.w));
      float4 l = make_float4(tf32_rna(x.x - h.x), tf32_rna(x.y - h.y), tf32_rna(x.z - h.z), tf32_rna(x.w - h.w));
      *reinterpret_cast<float4*>(hi + i) = h;
      *reinterpret_cast<float4*>(lo + i) = l;
    } else {
      for (size_t j = i; j < n; ++j) {
        float h = tf32_rna(src[j]);
        hi[j] = h;
        lo[j] = tf32_rna(src[j] - h);
      }
    }
  }
}

}  // namespace

mao_status launch_tf32_split(const float* src, float* hi, float* lo, size_t n, cudaStream_t stream) {
  if (n == 0) return MAO_OK;
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  size_t blocks = (n / 4 + 255) / 256 + 1;
  const size_t cap = (size_t)d->sm_count * 8;
  if (blocks > cap) blocks = cap;
  LaunchScope ls(stream, MAO_K_TF32_SPLIT, 0.0, 12.0 * (double)n);
  tf32_split_kernel<<<(unsigned)blocks, 256, 0, stream>>>(src, hi, lo, n);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

}  // namespace mao
