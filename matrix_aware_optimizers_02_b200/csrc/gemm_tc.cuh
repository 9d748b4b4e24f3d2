// Grouped, persistent tcgen05 GEMM for sm_100a.
//
// D[b] = A[b] * B[b]^T over many problems at once.  Problems are grouped into
// "classes" of identical (M, N, K); a class's operands are 3-D tensors
// [count][rows][cols] reached through one TMA descriptor each, so a batch of
// hundreds of same-shape matrices costs two descriptors.  One CTA per SM walks
// the linear tile space (class, matrix, tile_m, tile_n) with a static stride.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one elected lane): fills a STAGES-deep ring of
//               A/B tiles in shared memory, 128-byte swizzled.
//   warp 1      TMEM owner + MMA issuer (one elected lane): tcgen05.mma into one
//               of two TMEM accumulators (BN fp32 columns each), commits free
//               the smem slots and hand finished accumulators to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), fused arithmetic, stores.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
//
// Operand kinds:
//   BF16   kind::f16, bf16 operands, fp32 accumulate, BK = 64 (128 B rows).
//   TF32X3 kind::tf32 with each fp32 operand pre-split into hi + lo tf32
//          planes; D = Ahi*Bhi + Ahi*Blo + Alo*Bhi (fp32-faithful), BK = 32.
// Operand majors: K-major (rows of the operand run along K) or MN-major
// (rows run along M/N, i.e. the row-major matrix is K x MN).
#pragma once

#include "common.cuh"

namespace mao {

constexpr int kMaxClasses = 8;

enum OperandKind : int { OP_BF16 = 0, OP_TF32X3 = 1 };

enum EpiKind : int {
  EPI_STORE_F32 = 0,  // out0 (f32) = alpha * acc
  EPI_GRAM = 1,       // out0 (bf16) = acc * s_b^2                    (A = X X^T)
  EPI_POLY = 2,       // out0 (bf16) = beta * aux + gamma * acc       (B = b A + c A A)
  EPI_AXPY_T = 3,     // v = s_b * (alpha * aux + acc); out0 (bf16) = v, out1 = v^T if given  (X = a X + B X)
};

struct GemmClass {
  int M, N, K, count;
  int tiles_n, tiles_per_mat;
  int tile_begin;
  // Output 0 / output 1 / aux input: element pointers to matrix 0 of the class,
  // batch stride and leading dimension in elements.
  void* out0;
  long long out0_bs;
  int out0_ld;
  void* out1;
  long long out1_bs;
  int out1_ld;
  const void* aux;
  long long aux_bs;
  int aux_ld;
  const float* scale;  // per matrix of the class, or nullptr (= 1)
};

struct GemmParams {
  // Per class: A and B descriptors; for TF32X3 also the lo planes.
  CUtensorMap mapA[kMaxClasses];
  CUtensorMap mapB[kMaxClasses];
  GemmClass cls[kMaxClasses];
  int nclasses;
  int total_tiles;
  float alpha, beta, gamma;
  DevStatus* status;
};

// TF32X3 needs the lo planes too; they live in a second parameter block so the
// bf16 kernels keep a small parameter footprint.
struct GemmLoMaps {
  CUtensorMap mapAlo[kMaxClasses];
  CUtensorMap mapBlo[kMaxClasses];
};

template <int KIND, int A_MN, int B_MN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 256;
  static constexpr int ESIZE = (KIND == OP_BF16) ? 2 : 4;
  static constexpr int BK = 128 / ESIZE;              // elements per 128-byte row
  static constexpr int UMMA_K = (KIND == OP_BF16) ? 16 : 8;  // 32 bytes of K per MMA
  static constexpr int PLANES = (KIND == OP_BF16) ? 1 : 2;
  static constexpr int A_TILE = BM * 128;              // bytes per plane
  static constexpr int B_TILE = BN * 128;
  static constexpr int STAGE_BYTES = PLANES * (A_TILE + B_TILE);
  static constexpr int STAGES = (KIND == OP_BF16) ? 4 : 2;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr uint32_t IDESC = make_idesc(KIND == OP_BF16 ? 1u : 2u, A_MN, B_MN, BM, BN);
  static constexpr int THREADS = 192;
};

// Descriptor of one operand tile (rows = MN extent R, K extent = BK) at smem
// address `base`, advanced to MMA k-step `k`.
template <int MN_MAJOR, int R, int ESIZE>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int k) {
  constexpr int UMMA_K_BYTES = 32;
  if constexpr (!MN_MAJOR) {
    // K-major: rows of 128 B; the k-th 32-byte slice of every row.
    return smem_desc_sw128(base + k * UMMA_K_BYTES, 16, 1024);
  } else {
    // MN-major: the tile is R/(128/ESIZE) chunks of [BK rows x 128 B], each chunk
    // BK*128 bytes; a k-step covers UMMA_K K-rows = (32/ESIZE) rows of 128 B.
    constexpr int BK = 128 / ESIZE;
    constexpr int ROWS_PER_STEP = UMMA_K_BYTES / ESIZE;
    if constexpr (ESIZE == 4)  // tf32: 128-byte swizzle of 32-byte atoms, 4-row (512 B) groups
      return smem_desc_sw128(base + k * ROWS_PER_STEP * 128, BK * 128, 512, 1);
    return smem_desc_sw128(base + k * ROWS_PER_STEP * 128, BK * 128, 1024);
  }
}

// Issue the TMA loads of one operand tile (one plane).
template <int MN_MAJOR, int R, int ESIZE>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int k0,
                                             int mn0, int b) {
  if constexpr (!MN_MAJOR) {
    tma_load_3d(dst, map, bar, k0, mn0, b);
  } else {
    constexpr int CHUNK = 128 / ESIZE;  // MN elements per 128-byte row
    constexpr int BK = 128 / ESIZE;
#pragma unroll
    for (int c = 0; c < R / CHUNK; ++c) tma_load_3d(dst + c * BK * 128, map, bar, mn0 + c * CHUNK, k0, b);
  }
}

__device__ __forceinline__ int find_class(const GemmParams& p, int tile) {
  int c = 0;
#pragma unroll 1
  while (c + 1 < p.nclasses && tile >= p.cls[c + 1].tile_begin) ++c;
  return c;
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4 pk[4];
  uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    w[j] = *reinterpret_cast<uint32_t*>(&h);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d[j] = pk[j];
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 q = s[j];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      v[8 * j + 2 * e] = f.x;
      v[8 * j + 2 * e + 1] = f.y;
    }
  }
}

// Epilogue for 32 consecutive columns [col0, col0+32) of one tile row.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmParams& p, const GemmClass& C, int b, int row,
                                               int col0, float* v) {
  if (row >= C.M) return;
  const bool full = (col0 + 32 <= C.N);
  if constexpr (EPI == EPI_STORE_F32) {
    float* out = reinterpret_cast<float*>(C.out0) + (long long)b * C.out0_bs + (long long)row * C.out0_ld + col0;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(out + j) =
            make_float4(p.alpha * v[j], p.alpha * v[j + 1], p.alpha * v[j + 2], p.alpha * v[j + 3]);
    } else {
      for (int j = 0; j < 32 && col0 + j < C.N; ++j) out[j] = p.alpha * v[j];
    }
  } else {
    const float s = C.scale ? C.scale[b] : 1.0f;
    if constexpr (EPI == EPI_GRAM) {
      const float s2 = s * s;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= s2;
    } else {
      float a[32];
      const __nv_bfloat16* aux = reinterpret_cast<const __nv_bfloat16*>(C.aux) + (long long)b * C.aux_bs +
                                 (long long)row * C.aux_ld + col0;
      if (full) {
        load_bf16x32(aux, a);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) a[j] = (col0 + j < C.N) ? __bfloat162float(aux[j]) : 0.0f;
      }
      if constexpr (EPI == EPI_POLY) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = p.beta * a[j] + p.gamma * v[j];
      } else {  // EPI_AXPY_T
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = s * (p.alpha * a[j] + v[j]);
      }
    }
    __nv_bfloat16* out =
        reinterpret_cast<__nv_bfloat16*>(C.out0) + (long long)b * C.out0_bs + (long long)row * C.out0_ld + col0;
    if (full) {
      store_bf16x32(out, v);
    } else {
      for (int j = 0; j < 32 && col0 + j < C.N; ++j) out[j] = __float2bfloat16_rn(v[j]);
    }
    if constexpr (EPI == EPI_AXPY_T) {
      if (C.out1 != nullptr) {
        // optional transposed copy: for each column j, the 32 lanes (consecutive
        // rows) write 32 consecutive elements of row (col0 + j) of out1.
        __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(C.out1) + (long long)b * C.out1_bs + row;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < C.N) t[(long long)(col0 + j) * C.out1_ld] = __float2bfloat16_rn(v[j]);
      }
    }
  }
}

template <int KIND, int A_MN, int B_MN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ GemmLoMaps lo) {
  using Cfg = GemmCfg<KIND, A_MN, B_MN>;
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int prod_it_sh, mma_it_sh;

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    prod_it_sh = 0;
    mma_it_sh = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.nclasses; ++c) {
      tma_prefetch_desc(&p.mapA[c]);
      tma_prefetch_desc(&p.mapB[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x) {
        const int c = find_class(p, tile);
        const GemmClass& C = p.cls[c];
        const int local = tile - C.tile_begin;
        const int b = local / C.tiles_per_mat;
        const int r = local - b * C.tiles_per_mat;
        const int m0 = (r / C.tiles_n) * BM;
        const int n0 = (r % C.tiles_n) * BN;
        const int nk = (C.K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty_bar[s], ph ^ 1, p.status, 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Cfg::STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], Cfg::STAGE_BYTES);
          load_operand<A_MN, BM, Cfg::ESIZE>(st, &p.mapA[c], &full_bar[s], kb * BK, m0, b);
          load_operand<B_MN, BN, Cfg::ESIZE>(st + Cfg::A_TILE, &p.mapB[c], &full_bar[s], kb * BK, n0, b);
          if constexpr (KIND == OP_TF32X3) {
            load_operand<A_MN, BM, Cfg::ESIZE>(st + Cfg::A_TILE + Cfg::B_TILE, &lo.mapAlo[c], &full_bar[s],
                                               kb * BK, m0, b);
            load_operand<B_MN, BN, Cfg::ESIZE>(st + 2 * Cfg::A_TILE + Cfg::B_TILE, &lo.mapBlo[c],
                                               &full_bar[s], kb * BK, n0, b);
          }
        }
        if (!ok) break;
      }
      prod_it_sh = it;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int it = 0, tl = 0;
      for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tl) {
        const int c = find_class(p, tile);
        const GemmClass& C = p.cls[c];
        const int nk = (C.K + BK - 1) / BK;
        const int acc = tl & 1;
        const uint32_t aph = (tl >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], aph ^ 1, p.status, 2, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full_bar[s], ph, p.status, 3, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t b_base = a_base + Cfg::A_TILE;
#pragma unroll
          for (int k = 0; k < BK / Cfg::UMMA_K; ++k) {
            const uint64_t ad = operand_desc<A_MN, BM, Cfg::ESIZE>(a_base, k);
            const uint64_t bd = operand_desc<B_MN, BN, Cfg::ESIZE>(b_base, k);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            if constexpr (KIND == OP_BF16) {
              umma_f16(d_tmem, ad, bd, Cfg::IDESC, accum);
            } else {
              const uint32_t alo_base = b_base + Cfg::B_TILE;
              const uint32_t blo_base = alo_base + Cfg::A_TILE;
              const uint64_t adl = operand_desc<A_MN, BM, Cfg::ESIZE>(alo_base, k);
              const uint64_t bdl = operand_desc<B_MN, BN, Cfg::ESIZE>(blo_base, k);
              // small cross terms first, the dominant hi*hi product last
              umma_tf32(d_tmem, adl, bd, Cfg::IDESC, accum);
              umma_tf32(d_tmem, ad, bdl, Cfg::IDESC, 1u);
              umma_tf32(d_tmem, ad, bd, Cfg::IDESC, 1u);
            }
          }
          umma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_it_sh = it;
      umma_commit(&drain_bar);
      mbar_wait(&drain_bar, 0, p.status, 5, abort_flag, false);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int tl = 0;
    for (int tile = blockIdx.x; tile < p.total_tiles; tile += gridDim.x, ++tl) {
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      const bool ok = mbar_wait(&tfull_bar[acc], aph, p.status, 4, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int c = find_class(p, tile);
      const GemmClass& C = p.cls[c];
      const int local = tile - C.tile_begin;
      const int b = local / C.tiles_per_mat;
      const int r = local - b * C.tiles_per_mat;
      const int m0 = (r / C.tiles_n) * BM;
      const int n0 = (r % C.tiles_n) * BN;
      const int row = m0 + row_in_tile;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t rr[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + ch * 32, rr);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rr[j]);
        if (n0 + ch * 32 < C.N) epilogue_chunk<EPI>(p, C, b, row, n0 + ch * 32, v);
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
    }
  }

  __syncthreads();
  if (warp == 0 && lane == 0) {
    // after an early exit, let TMA loads still in flight land before the CTA ends
    for (int j = mma_it_sh; j < prod_it_sh; ++j)
      mbar_wait(&full_bar[j % STAGES], (j / STAGES) & 1, p.status, 6, abort_flag, false);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace mao
