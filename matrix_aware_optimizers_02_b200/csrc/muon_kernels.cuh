// Muon / Muon+ elementwise and reduction kernels (HBM-bound passes).
//
//   muon_prep_kernel      M <- mu M + (1-mu) G; per-tile sum of M^2 (fixed order);
//                         bf16(M) written in W's layout and transposed (the two
//                         Newton-Schulz operand layouts X and X^T).
//   muon_scale_kernel     per matrix: s = 1 / (sqrt(sum M^2) + eps), summing the tile
//                         partials in a fixed order (deterministic).
//   muon_colsq_kernel     Muon+ column sums of squares, partial over row chunks.
//   muon_colscale_kernel  column scale 1 / (sqrt(sum) + 1e-7).
//   muon_rowscale_kernel  Muon+ row scale, one warp per row.
//   muon_update_kernel    W <- W (1 - lr wd) - lr sqrt(m/n) rs_i cs_j O_ij, with
//                         per-tile partial sums for the optional stats.
//   muon_stats_kernel     update_rms and the non-finite count per matrix.
#pragma once

#include "common.cuh"

namespace mao {

constexpr float kMuonNormEps = 1e-7f;

// One entry per matrix of a Muon call (device copy of the host plan).
struct MuonMatDev {
  float* W;
  const void* G;
  float* M;
  __nv_bfloat16* Xw;  // iteration-0 operand in W's layout (m x n, ld = ldw)
  __nv_bfloat16* Xt;  // iteration-0 operand transposed (n x m, ld = ldt)
  const __nv_bfloat16* O;  // final orthogonalised matrix in W's layout (m x n, ld = ldw)
  float* rowscale;    // m entries (Muon+), or nullptr
  float* colscale;    // n entries (Muon+), or nullptr
  float* colpart;     // col_chunks x n partial column sums (Muon+), or nullptr
  const float* oscale;  // multiplier of O (the pre-normalisation scale when no NS step ran), or nullptr
  int scale_slot;     // index of this matrix in the per-class-ordered scale array
  int m, n;
  int g_bf16;
  int ldw, ldt;
  int prep_tiles_c;   // tiles along columns in the prep pass
  int prep_begin;     // first prep tile (global) of this matrix
  int prep_count;
  int col_chunks;     // row chunks of the column-sum pass
  int colsq_begin;    // first colsq block of this matrix
  int upd_begin;      // first update block of this matrix
  int upd_count;
  float out_scale;    // lr * sqrt(m/n)
};

__device__ __forceinline__ int find_mat(const MuonMatDev* T, int count, int blk, int MuonMatDev::*begin) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (T[mid].*begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

constexpr int kPrepTile = 64;  // 64 x 64 elements per block, 256 threads

__global__ void __launch_bounds__(256) muon_prep_kernel(const MuonMatDev* __restrict__ T, int count, float mu,
                                                        float* __restrict__ partial) {
  __shared__ __nv_bfloat16 tileT[kPrepTile][kPrepTile + 8];
  __shared__ float wsum[8];
  const int blk = blockIdx.x;
  const int p = find_mat(T, count, blk, &MuonMatDev::prep_begin);
  const MuonMatDev& D = T[p];
  const int local = blk - D.prep_begin;
  const int r0 = (local / D.prep_tiles_c) * kPrepTile;
  const int c0 = (local % D.prep_tiles_c) * kPrepTile;
  const int tx = threadIdx.x & 15;  // 4-column group
  const int ty = threadIdx.x >> 4;  // 0..15
  const int col = c0 + tx * 4;
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rl = ty + 16 * i;
    const int row = r0 + rl;
    float mv[4] = {0.f, 0.f, 0.f, 0.f};
    if (row < D.m && col < D.n) {  // n % 4 == 0, so the 4 columns are all in or all out
      const long long off = (long long)row * D.n + col;
      float4 m4 = *reinterpret_cast<const float4*>(D.M + off);
      float g[4];
      if (D.g_bf16) {
        uint2 raw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(D.G) + off);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
      } else {
        float4 g4 = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(D.G) + off);
        g[0] = g4.x; g[1] = g4.y; g[2] = g4.z; g[3] = g4.w;
      }
      const float om = 1.0f - mu;
      mv[0] = mu * m4.x + om * g[0];
      mv[1] = mu * m4.y + om * g[1];
      mv[2] = mu * m4.z + om * g[2];
      mv[3] = mu * m4.w + om * g[3];
      *reinterpret_cast<float4*>(D.M + off) = make_float4(mv[0], mv[1], mv[2], mv[3]);
      acc += mv[0] * mv[0] + mv[1] * mv[1] + mv[2] * mv[2] + mv[3] * mv[3];
      __nv_bfloat162 h0 = __floats2bfloat162_rn(mv[0], mv[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(mv[2], mv[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&h0);
      pk.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(D.Xw + (long long)row * D.ldw + col) = pk;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) tileT[tx * 4 + e][rl] = __float2bfloat16_rn(mv[e]);
  }
  __syncthreads();
  // transposed write: Xt row = column of M, 4 consecutive source rows per thread
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int cl = ty + 16 * i;  // column within tile -> row of Xt
    const int trow = c0 + cl;
    const int tcol = r0 + tx * 4;
    if (trow < D.n) {
      __nv_bfloat16* dst = D.Xt + (long long)trow * D.ldt + tcol;
      if (tcol + 4 <= D.m) {
        uint2 pk;
        __nv_bfloat162 h0, h1;
        h0.x = tileT[cl][tx * 4 + 0]; h0.y = tileT[cl][tx * 4 + 1];
        h1.x = tileT[cl][tx * 4 + 2]; h1.y = tileT[cl][tx * 4 + 3];
        pk.x = *reinterpret_cast<uint32_t*>(&h0);
        pk.y = *reinterpret_cast<uint32_t*>(&h1);
        *reinterpret_cast<uint2*>(dst) = pk;
      } else {
        for (int e = 0; e < 4 && tcol + e < D.m; ++e) dst[e] = tileT[cl][tx * 4 + e];
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

// One warp per matrix.
__global__ void muon_scale_kernel(const MuonMatDev* __restrict__ T, int count, const float* __restrict__ partial,
                                  float eps, float* __restrict__ scale) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= count) return;
  const MuonMatDev& D = T[p];
  double s = 0.0;
  for (int i = lane; i < D.prep_count; i += 32) s += (double)partial[D.prep_begin + i];
  s = warp_sum_d(s);
  if (lane == 0) scale[D.scale_slot] = (float)(1.0 / (sqrt(s) + (double)eps));
}

// ------------------------------------------------------------------ Muon+
constexpr int kColChunkRows = 64;

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* src, float* v) {
  uint4 q = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}

// Block = 256 threads over (64-row chunk) x (256 columns): thread owns one column,
// sums (O_ij * rs_i)^2 over the chunk's rows in order.  use_rows: apply rowscale.
__global__ void __launch_bounds__(256) muon_colsq_kernel(const MuonMatDev* __restrict__ T, int count,
                                                         int use_rows) {
  const int p = find_mat(T, count, blockIdx.x, &MuonMatDev::colsq_begin);
  const MuonMatDev& D = T[p];
  const int local = blockIdx.x - D.colsq_begin;
  const int ncb = (D.n + 255) / 256;
  const int chunk = local / ncb;
  const int col = (local % ncb) * 256 + threadIdx.x;
  if (col >= D.n) return;
  const int r0 = chunk * kColChunkRows;
  const int r1 = min(D.m, r0 + kColChunkRows);
  const float om = D.oscale ? *D.oscale : 1.0f;
  float s = 0.f;
  for (int r = r0; r < r1; ++r) {
    float v = om * __bfloat162float(D.O[(long long)r * D.ldw + col]);
    if (use_rows) v *= D.rowscale[r];
    s += v * v;
  }
  D.colpart[(long long)chunk * D.n + col] = s;
}

__global__ void muon_colscale_kernel(const MuonMatDev* __restrict__ T, int count) {
  const int p = blockIdx.y;
  if (p >= count) return;
  const MuonMatDev& D = T[p];
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  if (col >= D.n) return;
  double s = 0.0;
  for (int c = 0; c < D.col_chunks; ++c) s += (double)D.colpart[(long long)c * D.n + col];
  D.colscale[col] = (float)(1.0 / (sqrt(s) + (double)kMuonNormEps));
}

// One warp per row; use_cols: apply colscale before squaring.
__global__ void muon_rowscale_kernel(const MuonMatDev* __restrict__ T, int count, const int* __restrict__ row_begin,
                                     int total_rows, int use_cols) {
  const int g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (g >= total_rows) return;
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (row_begin[mid] <= g) lo = mid; else hi = mid - 1;
  }
  const MuonMatDev& D = T[lo];
  const int r = g - row_begin[lo];
  const __nv_bfloat16* row = D.O + (long long)r * D.ldw;
  const float om = D.oscale ? *D.oscale : 1.0f;
  float s = 0.f;
  for (int c = lane * 8; c < D.n; c += 256) {
    float v[8];
    if (c + 8 <= D.n) {
      load_bf16x8(row + c, v);
    } else {
      for (int e = 0; e < 8; ++e) v[e] = (c + e < D.n) ? __bfloat162float(row[c + e]) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = om * v[e];
      if (use_cols && c + e < D.n) x *= D.colscale[c + e];
      s += x * x;
    }
  }
  s = warp_sum(s);
  if (lane == 0) D.rowscale[r] = 1.0f / (sqrtf(s) + kMuonNormEps);
}

// ------------------------------------------------------------------ update
constexpr int kUpdElems = 4096;  // elements per update block (256 threads x 16)

__global__ void __launch_bounds__(256) muon_update_kernel(const MuonMatDev* __restrict__ T, int count,
                                                          float decay, int use_rows, int use_cols,
                                                          float* __restrict__ upd_partial,
                                                          int* __restrict__ upd_nonfinite) {
  __shared__ float wsum[8];
  __shared__ int wbad[8];
  const int p = find_mat(T, count, blockIdx.x, &MuonMatDev::upd_begin);
  const MuonMatDev& D = T[p];
  const int local = blockIdx.x - D.upd_begin;
  // the block covers flat elements [local*4096, +4096) of the m x n matrix, 8 per step
  const long long total = (long long)D.m * D.n;
  const long long base = (long long)local * kUpdElems;
  float acc = 0.f;
  int bad = 0;
  const float om = D.oscale ? *D.oscale : 1.0f;
  for (int k = 0; k < 2; ++k) {
    const long long e0 = base + (long long)(k * 256 + threadIdx.x) * 8;
    if (e0 >= total) continue;
    // n % 4 == 0: a group of 8 may straddle a row end only in 4-element halves
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const long long e = e0 + 4 * h;
      if (e >= total) break;
      const int rr = (int)(e / D.n);
      const int cc = (int)(e - (long long)rr * D.n);
      float o[4];
      {
        uint2 raw = *reinterpret_cast<const uint2*>(D.O + (long long)rr * D.ldw + cc);
        const __nv_bfloat162* hh = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float2 a = __bfloat1622float2(hh[0]), b = __bfloat1622float2(hh[1]);
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
      }
      const float rs = om * (use_rows ? D.rowscale[rr] : 1.0f);
      float4 w = *reinterpret_cast<float4*>(D.W + e);
      float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float cs = use_cols ? D.colscale[cc + q] : 1.0f;
        const float nw = wv[q] * decay - D.out_scale * (o[q] * rs * cs);
        const float d = nw - wv[q];
        acc += d * d;
        bad += isfinite(nw) ? 0 : 1;
        wv[q] = nw;
      }
      *reinterpret_cast<float4*>(D.W + e) = make_float4(wv[0], wv[1], wv[2], wv[3]);
    }
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

// One warp per matrix.
__global__ void muon_stats_kernel(const MuonMatDev* __restrict__ T, int count, const float* __restrict__ upd_partial,
                                  const int* __restrict__ upd_nonfinite, mao_stats* __restrict__ stats) {
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= count) return;
  const MuonMatDev& D = T[p];
  double s = 0.0;
  int b = 0;
  for (int i = lane; i < D.upd_count; i += 32) {
    s += (double)upd_partial[D.upd_begin + i];
    b += upd_nonfinite[D.upd_begin + i];
  }
  s = warp_sum_d(s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
  if (lane == 0) {
    stats[p].update_rms = (float)sqrt(s / ((double)D.m * (double)D.n));
    stats[p].offdiag_ratio = -1.0f;
    stats[p].refreshed = 0;
    stats[p].nonfinite = b;
  }
}

}  // namespace mao
