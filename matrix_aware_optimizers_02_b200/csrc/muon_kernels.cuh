// Muon / Muon+ elementwise and reduction kernels (HBM-bound passes).
//
// Every pass walks the matrix in 64 x 64 tiles (256 threads, 16 elements per
// thread: rows ty + 16 i, columns 4 tx .. 4 tx + 3).  The Newton-Schulz operand
// X is kept in one layout only, s x l with s = min(m, n): for a tall matrix
// (m > n) X holds M^T, and the passes that read O in W's orientation transpose
// through shared memory so that both the X reads and the W accesses stay
// coalesced.
//
//   muon_prep_kernel       M <- mu M + (1-mu) G; per-tile sum of M^2 (fixed order);
//                          bf16(M) written as X (transposed for tall matrices).
//   muon_scale_kernel      per matrix: s = 1 / (sqrt(sum M^2) + eps), summing the
//                          tile partials in a fixed order (deterministic).
//   muon_norm_tile_kernel  Muon+ partial sums of squares per tile: column sums
//                          over the tile's rows and/or row sums over its columns,
//                          optionally after applying the other direction's scale.
//   muon_norm_final_kernel row or column scale 1 / (sqrt(sum) + 1e-7).
//   muon_update_kernel     W <- W (1 - lr wd) - lr sqrt(m/n) rs_i cs_j O_ij, with
//                          per-tile partial sums for the optional stats.
//   muon_stats_kernel      update_rms and the non-finite count per matrix.
#pragma once

#include "common.cuh"

namespace mao {

constexpr float kMuonNormEps = 1e-7f;
constexpr int kTile = 64;  // 64 x 64 elements per block, 256 threads

// One entry per matrix of a Muon call (device copy of the host plan).
struct MuonMatDev {
  float* W;
  const void* G;
  float* M;
  __nv_bfloat16* X0;       // iteration-0 operand, s x l (ld = ldx)
  const __nv_bfloat16* O;  // final orthogonalised X, s x l (ld = ldx)
  float* rowscale;         // m entries (Muon+), or nullptr
  float* colscale;         // n entries (Muon+), or nullptr
  float* rowpart;          // tiles_c x m partial row sums (Muon+ row pass), or nullptr
  float* colpart;          // tiles_r x n partial column sums (Muon+ column pass), or nullptr
  const float* oscale;     // multiplier of O (the pre-normalisation scale when no NS step ran), or nullptr
  int scale_slot;          // index of this matrix in the per-class-ordered scale array
  int m, n;
  int ld;                  // leading dimension of W, G and M (n, or the stored width of a split matrix)
  int g_bf16;
  int trans;               // 1 if m > n: X = M^T
  int ldx;                 // leading dimension of X (elements, multiple of 8)
  int tiles_r, tiles_c;    // 64 x 64 tiles of the m x n matrix
  int tile_begin;          // first tile (global block index) of this matrix
  float out_scale;         // lr * sqrt(m/n)
  // exact polar factor (MOP): fp32 X0 = M / (||M||_F + eps) (s x l, ld = ldx) and its
  // three bf16 planes (plane stride xep_stride), and the final fp32 O; nullptr otherwise
  float* Xe;
  __nv_bfloat16* Xep;
  long long xep_stride;
  const float* Of;
};

// The device table of `count` records is followed by the records' first tiles
// (a compact int array): the block's matrix by a search that stays in L1.
__device__ __forceinline__ int find_mat(const MuonMatDev* T, int count, int blk) {
  return find_start(reinterpret_cast<const int*>(T + count), count, blk);
}

// Start moving a line toward L2 without holding registers for it (the load that
// follows finds it there, so the row loads of a thread overlap instead of queuing).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void bf16x4_to_float(uint2 raw, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

// Tile of O in W's orientation: thread (ty, tx) receives rows r0 + ty + 16 i,
// columns c0 + 4 tx + e; entries outside the matrix are 0.  `sm` is a 64 x 65
// bf16 staging tile used for the transposed case (one __syncthreads inside).
// The staging tile of load_o_tile for O stored as OT.  Rows of 65 elements: the
// transposed reads walk down a column with a stride of 4 rows across the lanes, which a
// 65-element row spreads over distinct banks (a 72-element row put half the lanes on
// one bank); every access to the tile is scalar, so no alignment is needed.
template <typename OT>
struct OTile {
  static constexpr int kPad = 1;
  typedef OT Row[kTile + kPad];
};

__device__ __forceinline__ void o_to_float4(const float* p, float* v) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void o_to_float4(const __nv_bfloat16* p, float* v) {
  bf16x4_to_float(*reinterpret_cast<const uint2*>(p), v);
}
__device__ __forceinline__ float o_to_float(float x) { return x; }
__device__ __forceinline__ float o_to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename OT>
__device__ __forceinline__ OT o_zero() { return OT(0.0f); }

template <typename OT>
__device__ __forceinline__ void load_o_tile(const MuonMatDev& D, const OT* X, int r0, int c0, float (&v)[4][4],
                                            typename OTile<OT>::Row* sm) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  if (!D.trans) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = r0 + ty + 16 * i, col = c0 + 4 * tx;
      if (row < D.m && col < D.n) {
        o_to_float4(X + (long long)row * D.ldx + col, v[i]);
      } else {
        v[i][0] = v[i][1] = v[i][2] = v[i][3] = 0.f;
      }
    }
  } else {
    // X is n x m: O[r][c] = X[c][r].  Stage X rows c0.. (O columns), X columns r0.. (O rows).
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int xr = c0 + ty + 16 * i, xc = r0 + 4 * tx;
      const OT* src = X + (long long)xr * D.ldx + xc;
      if (xr < D.n && xc + 4 <= D.m) {
        OT h[4];
        if constexpr (sizeof(OT) == 2) {
          *reinterpret_cast<uint2*>(h) = *reinterpret_cast<const uint2*>(src);
        } else {
          *reinterpret_cast<float4*>(h) = *reinterpret_cast<const float4*>(src);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) sm[ty + 16 * i][4 * tx + e] = h[e];
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sm[ty + 16 * i][4 * tx + e] = (xr < D.n && xc + e < D.m) ? src[e] : o_zero<OT>();
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) v[i][e] = o_to_float(sm[4 * tx + e][ty + 16 * i]);
  }
}

template <typename OT>
__device__ __forceinline__ const OT* o_of(const MuonMatDev& D);
template <>
__device__ __forceinline__ const __nv_bfloat16* o_of<__nv_bfloat16>(const MuonMatDev& D) { return D.O; }
template <>
__device__ __forceinline__ const float* o_of<float>(const MuonMatDev& D) { return D.Of; }

// ------------------------------------------------------------------ prep
__global__ void __launch_bounds__(256) muon_prep_kernel(const MuonMatDev* __restrict__ T, int count, float mu,
                                                        float* __restrict__ partial) {
  __shared__ __nv_bfloat16 tileT[kTile][kTile + 1];  // 65-element rows: conflict-free column writes
  __shared__ float wsum[8];
  const int blk = blockIdx.x;
  const MuonMatDev& D = T[find_mat(T, count, blk)];
  const int local = blk - D.tile_begin;
  const int r0 = (local / D.tiles_c) * kTile;
  const int c0 = (local % D.tiles_c) * kTile;
  const int tx = threadIdx.x & 15;
  const int ty = threadIdx.x >> 4;
  const int col = c0 + tx * 4;
  const float om = 1.0f - mu;
  float acc = 0.0f;
  if (col < D.n) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = r0 + ty + 16 * i;
      if (row < D.m) {
        const long long off = (long long)row * D.ld + col;
        prefetch_l2(D.M + off);
        prefetch_l2(static_cast<const char*>(D.G) + off * (D.g_bf16 ? 2 : 4));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = ty + 16 * i;
    const int row = r0 + rl;
    float mv[4] = {0.f, 0.f, 0.f, 0.f};
    if (row < D.m && col < D.n) {  // n % 4 == 0: the 4 columns are all in or all out
      const long long off = (long long)row * D.ld + col;
      float4 m4 = *reinterpret_cast<const float4*>(D.M + off);
      float g[4];
      if (D.g_bf16) {
        bf16x4_to_float(*reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(D.G) + off), g);
      } else {
        float4 g4 = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(D.G) + off);
        g[0] = g4.x; g[1] = g4.y; g[2] = g4.z; g[3] = g4.w;
      }
      mv[0] = mu * m4.x + om * g[0];
      mv[1] = mu * m4.y + om * g[1];
      mv[2] = mu * m4.z + om * g[2];
      mv[3] = mu * m4.w + om * g[3];
      *reinterpret_cast<float4*>(D.M + off) = make_float4(mv[0], mv[1], mv[2], mv[3]);
      acc += mv[0] * mv[0] + mv[1] * mv[1] + mv[2] * mv[2] + mv[3] * mv[3];
      if (!D.trans) {
        __nv_bfloat162 h0 = __floats2bfloat162_rn(mv[0], mv[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(mv[2], mv[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&h0);
        pk.y = *reinterpret_cast<uint32_t*>(&h1);
        *reinterpret_cast<uint2*>(D.X0 + (long long)row * D.ldx + col) = pk;
      }
    }
    if (D.trans) {
#pragma unroll
      for (int e = 0; e < 4; ++e) tileT[tx * 4 + e][rl] = __float2bfloat16_rn(mv[e]);
    }
  }
  if (D.trans) {
    __syncthreads();
    // X row = column of M, 4 consecutive source rows per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int cl = ty + 16 * i;
      const int xrow = c0 + cl;
      const int xcol = r0 + tx * 4;
      if (xrow < D.n) {
        __nv_bfloat16* dst = D.X0 + (long long)xrow * D.ldx + xcol;
        if (xcol + 4 <= D.m) {
          uint2 pk;
          __nv_bfloat162 h0, h1;
          h0.x = tileT[cl][tx * 4 + 0]; h0.y = tileT[cl][tx * 4 + 1];
          h1.x = tileT[cl][tx * 4 + 2]; h1.y = tileT[cl][tx * 4 + 3];
          pk.x = *reinterpret_cast<uint32_t*>(&h0);
          pk.y = *reinterpret_cast<uint32_t*>(&h1);
          *reinterpret_cast<uint2*>(dst) = pk;
        } else {
          for (int e = 0; e < 4 && xcol + e < D.m; ++e) dst[e] = tileT[cl][tx * 4 + e];
        }
      }
    }
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += wsum[w];
    partial[blk] = s;
  }
}

// ------------------------------------------------------------------ exact polar factor
// X0 = s M (s = 1 / (||M||_F + eps) from muon_scale_kernel) in fp32, transposed for a
// tall matrix, and its three bf16 planes: the operand of the fp32-faithful iteration.
// One 64 x 64 tile of the m x n matrix per block, as muon_prep_kernel.
__global__ void __launch_bounds__(256) mop_init_kernel(const MuonMatDev* __restrict__ T, int count,
                                                       const float* __restrict__ scale) {
  __shared__ float tileT[kTile][kTile + 1];
  const MuonMatDev& D = T[find_mat(T, count, blockIdx.x)];
  const int local = blockIdx.x - D.tile_begin;
  const int r0 = (local / D.tiles_c) * kTile, c0 = (local % D.tiles_c) * kTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int col = c0 + 4 * tx;
  const float sc = scale[D.scale_slot];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = ty + 16 * i, row = r0 + rl;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < D.m && col < D.n) {
      x = *reinterpret_cast<const float4*>(D.M + (long long)row * D.ld + col);
      x = make_float4(sc * x.x, sc * x.y, sc * x.z, sc * x.w);
      if (!D.trans) {
        const long long o = (long long)row * D.ldx + col;
        *reinterpret_cast<float4*>(D.Xe + o) = x;
        store_split3x4(x, D.Xep, o, D.xep_stride);
      }
    }
    if (D.trans) {
      tileT[4 * tx + 0][rl] = x.x;
      tileT[4 * tx + 1][rl] = x.y;
      tileT[4 * tx + 2][rl] = x.z;
      tileT[4 * tx + 3][rl] = x.w;
    }
  }
  if (!D.trans) return;
  __syncthreads();
  // X row = column of M: rows c0 + cl, columns r0 + 4 tx .. (m need not be a multiple of 4)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int cl = ty + 16 * i, xrow = c0 + cl, xcol = r0 + 4 * tx;
    if (xrow >= D.n) continue;
    const long long o = (long long)xrow * D.ldx + xcol;
    if (xcol + 4 <= D.m) {
      const float4 x = make_float4(tileT[cl][4 * tx], tileT[cl][4 * tx + 1], tileT[cl][4 * tx + 2],
                                   tileT[cl][4 * tx + 3]);
      *reinterpret_cast<float4*>(D.Xe + o) = x;
      store_split3x4(x, D.Xep, o, D.xep_stride);
    } else {
      for (int e = 0; e < 4 && xcol + e < D.m; ++e) {
        D.Xe[o + e] = tileT[cl][4 * tx + e];
        store_split3(tileT[cl][4 * tx + e], D.Xep, o + e, D.xep_stride);
      }
    }
  }
}

// One warp per matrix.
__global__ void muon_scale_kernel(const MuonMatDev* __restrict__ T, int count, const float* __restrict__ partial,
                                  float eps, float* __restrict__ scale) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= count) return;
  const MuonMatDev& D = T[p];
  const int nt = D.tiles_r * D.tiles_c;
  double s = 0.0;
  for (int i = lane; i < nt; i += 32) s += (double)partial[D.tile_begin + i];
  s = warp_sum_d(s);
  if (lane == 0) scale[D.scale_slot] = (float)(1.0 / (sqrt(s) + (double)eps));
}

// ------------------------------------------------------------------ Muon+
// want_cols: write column partials (sum over the tile's rows of (O rs)^2)
// want_rows: write row partials (sum over the tile's columns of (O cs)^2)
// use_rows / use_cols: apply rowscale / colscale before squaring.
// OT: element type of O (bf16 after Newton-Schulz, fp32 for the exact polar factor).
// The tile is read in storage order (X = O^T for a tall matrix), so no transpose is
// needed: a storage row of a tall matrix is a column of O.  Thread (tx, ty) holds
// storage rows ty + 16 i and storage columns 4 tx + e; "along" sums (over e and the
// 16 threads of a half-warp) give per-storage-row partials, "across" sums (over i and
// the 16 thread rows, in shared memory) per-storage-column partials.
template <typename OT>
__global__ void __launch_bounds__(256) muon_norm_tile_kernel(const MuonMatDev* __restrict__ T, int count,
                                                             int want_cols, int want_rows, int use_rows,
                                                             int use_cols) {
  __shared__ float csum[16][kTile];
  const MuonMatDev& D = T[find_mat(T, count, blockIdx.x)];
  const int local = blockIdx.x - D.tile_begin;
  const int tr = local / D.tiles_c, tc = local % D.tiles_c;
  const int r0 = tr * kTile, c0 = tc * kTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const bool t = D.trans != 0;
  // storage extents and origin: rows s0.., columns q0.. of X (ld ldx)
  const int srows = t ? D.n : D.m, scols = t ? D.m : D.n;
  const int s0 = t ? c0 : r0, q0 = t ? r0 : c0;
  const OT* X = o_of<OT>(D);
  const float om = D.oscale ? *D.oscale : 1.0f;
  // the scale applied before squaring: rowscale (O rows) for column partials,
  // colscale (O columns) for row partials; in storage order it is indexed by the
  // storage column (O row) or storage row (O column)
  const bool scale_on = want_cols ? (use_rows != 0) : (use_cols != 0);
  const float* sc = want_cols ? D.rowscale : D.colscale;
  const bool sc_by_col = want_cols ? t : !t;  // false: indexed by the storage row
  float v[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int sr = s0 + ty + 16 * i, q = q0 + 4 * tx;
    if (sr < srows && q + 4 <= scols) {
      o_to_float4(X + (long long)sr * D.ldx + q, v[i]);
    } else {  // the storage rows of a tall matrix are m long, which may not be a multiple of 4
#pragma unroll
      for (int e = 0; e < 4; ++e)
        v[i][e] = (sr < srows && q + e < scols) ? o_to_float(X[(long long)sr * D.ldx + q + e]) : 0.f;
    }
    float f[4] = {om, om, om, om};
    if (scale_on) {
      if (sc_by_col) {
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] *= (q + e < scols) ? sc[q + e] : 1.0f;
      } else {
        const float r = (sr < srows) ? sc[sr] : 1.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] *= r;
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x = v[i][e] * f[e];
      v[i][e] = x * x;
    }
  }
  // per storage row: O rows of a wide matrix (row partials), O columns of a tall one
  const bool along = t ? want_cols : want_rows;
  if (along) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = (v[i][0] + v[i][1]) + (v[i][2] + v[i][3]);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const int sr = s0 + ty + 16 * i;
      if (tx == 0 && sr < srows) {
        if (t) D.colpart[(long long)tr * D.n + sr] = s;  // O column sr, over O rows r0..
        else D.rowpart[(long long)tc * D.m + sr] = s;    // O row sr, over O columns c0..
      }
    }
  } else {
    // per storage column: O columns of a wide matrix (column partials), O rows of a tall one
#pragma unroll
    for (int e = 0; e < 4; ++e) csum[ty][4 * tx + e] = (v[0][e] + v[1][e]) + (v[2][e] + v[3][e]);
    __syncthreads();
    if (threadIdx.x < kTile) {
      const int q = q0 + threadIdx.x;
      float s = 0.f;
      for (int g = 0; g < 16; ++g) s += csum[g][threadIdx.x];
      if (q < scols) {
        if (t) D.rowpart[(long long)tc * D.m + q] = s;  // O row q, over O columns c0..
        else D.colpart[(long long)tr * D.n + q] = s;    // O column q, over O rows r0..
      }
    }
  }
}

// which = 0: rows (rowscale from rowpart over tiles_c), 1: columns.  grid.y = matrix.
__global__ void muon_norm_final_kernel(const MuonMatDev* __restrict__ T, int count, int which) {
  const int p = blockIdx.y;
  if (p >= count) return;
  const MuonMatDev& D = T[p];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int len = which == 0 ? D.m : D.n;
  if (i >= len) return;
  const int parts = which == 0 ? D.tiles_c : D.tiles_r;
  const float* src = which == 0 ? D.rowpart : D.colpart;
  double s = 0.0;
  for (int c = 0; c < parts; ++c) s += (double)src[(long long)c * len + i];
  const float r = (float)(1.0 / (sqrt(s) + (double)kMuonNormEps));
  if (which == 0) D.rowscale[i] = r; else D.colscale[i] = r;
}

// ------------------------------------------------------------------ update
template <typename OT>
__global__ void __launch_bounds__(256) muon_update_kernel(const MuonMatDev* __restrict__ T, int count,
                                                          float decay, int use_rows, int use_cols,
                                                          float* __restrict__ upd_partial,
                                                          int* __restrict__ upd_nonfinite) {
  __shared__ __align__(16) typename OTile<OT>::Row sm[kTile];
  __shared__ float wsum[8];
  __shared__ int wbad[8];
  const MuonMatDev& D = T[find_mat(T, count, blockIdx.x)];
  const int local = blockIdx.x - D.tile_begin;
  const int r0 = (local / D.tiles_c) * kTile, c0 = (local % D.tiles_c) * kTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int col = c0 + 4 * tx;
  if (col < D.n) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = r0 + ty + 16 * i;
      if (row < D.m) prefetch_l2(D.W + (long long)row * D.ld + col);
    }
  }
  float v[4][4];
  load_o_tile<OT>(D, o_of<OT>(D), r0, c0, v, sm);
  const float om = D.oscale ? *D.oscale : 1.0f;
  float cs[4] = {1.f, 1.f, 1.f, 1.f};
  if (use_cols && col < D.n) {
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[e] = D.colscale[col + e];
  }
  float acc = 0.f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = r0 + ty + 16 * i;
    if (row >= D.m || col >= D.n) continue;
    const float rs = om * (use_rows ? D.rowscale[row] : 1.0f);
    float* wp = D.W + (long long)row * D.ld + col;
    float4 w = *reinterpret_cast<float4*>(wp);
    float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float nw = wv[e] * decay - D.out_scale * (v[i][e] * rs * cs[e]);
      const float d = nw - wv[e];
      acc += d * d;
      bad += isfinite(nw) ? 0 : 1;
      wv[e] = nw;
    }
    *reinterpret_cast<float4*>(wp) = make_float4(wv[0], wv[1], wv[2], wv[3]);
  }
  if (upd_partial == nullptr) return;
  acc = warp_sum(acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0) {
    wsum[threadIdx.x >> 5] = acc;
    wbad[threadIdx.x >> 5] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    int b = 0;
    for (int w = 0; w < 8; ++w) {
      s += wsum[w];
      b += wbad[w];
    }
    upd_partial[blockIdx.x] = s;
    upd_nonfinite[blockIdx.x] = b;
  }
}

// Tiles of one caller matrix (the blocks of a split matrix are consecutive).
struct MuonStatsRange {
  int tile_begin, tiles;
  int m, n;
};

// One warp per caller matrix.  A non-finite weight is also recorded in the workspace
// status word as MAO_ERR_NONFINITE (site 30), unless an error came first.
__global__ void muon_stats_kernel(const MuonStatsRange* __restrict__ R, int count, const float* __restrict__ upd_partial,
                                  const int* __restrict__ upd_nonfinite, mao_stats* __restrict__ stats,
                                  DevStatus* status) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= count) return;
  const MuonStatsRange& D = R[p];
  double s = 0.0;
  int b = 0;
  for (int i = lane; i < D.tiles; i += 32) {
    s += (double)upd_partial[D.tile_begin + i];
    b += upd_nonfinite[D.tile_begin + i];
  }
  s = warp_sum_d(s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
  if (lane == 0) {
    stats[p].update_rms = (float)sqrt(s / ((double)D.m * (double)D.n));
    stats[p].offdiag_ratio = -1.0f;
    stats[p].refreshed = 0;
    stats[p].nonfinite = b;
    if (b > 0) report(status, MAO_ERR_NONFINITE, 30, p, b);
  }
}

}  // namespace mao
