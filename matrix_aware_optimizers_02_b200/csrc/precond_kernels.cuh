// Kernels of the SOAP and FOAM steps other than the tensor-core products:
// HBM-bound elementwise passes, deterministic reductions, the eigenbasis sort,
// and the panel pieces of the QR orthogonalisation.
//
// Every per-matrix work list is a device array of small job records; a block
// finds its record by binary search on the job's first block index.  Every
// kernel that belongs to a basis refresh can be gated by a per-matrix flag
// (skipped when the flag is 0), so adaptive refreshes need no host round trip.
#pragma once

#include "common.cuh"

namespace mao {

constexpr int kElemsPerBlock = 4096;  // 256 threads x 16 elements

// A matrix pass over rows x cols elements (row-major).  Plane sets hold an fp32
// matrix as three bf16 planes x = p0 + p1 + p2 (plane q at base + q*pstride,
// leading dimension ldp).
struct EwJob {
  const void* a;        // primary input (fp32, or bf16 when a_bf16)
  const float* b;       // secondary fp32 input
  float* f0;            // fp32 output (in place where noted)
  const float* f1;      // extra fp32 input
  const float* vr;      // per-row vector
  const float* vc;      // per-column vector
  __nv_bfloat16* pa;    // plane sets
  __nv_bfloat16* pb;
  long long pstride;
  const int* flag;      // nullptr, or skip when *flag == 0
  int rows, cols;
  int lda, ldb, ldf, ldp;
  int a_bf16;
  int blk_begin;
};

__device__ __forceinline__ int find_job(const EwJob* J, int n, int blk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Three-plane split of 4 consecutive values, stored as 8-byte groups per plane.
__device__ __forceinline__ void store_split3x4(float4 x, __nv_bfloat16* base, long long off, long long pstride) {
  float r[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    __nv_bfloat16 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h[e] = __float2bfloat16_rn(r[e]);
      r[e] -= __bfloat162float(h[e]);
    }
    *reinterpret_cast<uint2*>(base + q * pstride + off) = *reinterpret_cast<const uint2*>(h);
  }
}

__device__ __forceinline__ void store_split3(float x, __nv_bfloat16* base, long long off, long long pstride) {
#pragma unroll
  for (int q = 0; q < 3; ++q) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    base[q * pstride + off] = h;
    x -= __bfloat162float(h);
  }
}

__device__ __forceinline__ float4 load4(const void* base, long long off, int is_bf16) {
  if (is_bf16) {
    uint2 raw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
}

// Iterate the 4-element groups of the job handled by this block.  cols % 4 == 0.
#define MAO_EW_LOOP(J, local, ...)                                                         \
  {                                                                                        \
    const long long _groups = (long long)(J).rows * ((J).cols / 4);                        \
    const long long _g0 = (long long)(local) * (kElemsPerBlock / 4);                       \
    for (int _k = 0; _k < kElemsPerBlock / 4 / 256; ++_k) {                                \
      const long long _g = _g0 + _k * 256 + threadIdx.x;                                   \
      if (_g >= _groups) break;                                                            \
      const int r = (int)(_g / ((J).cols / 4));                                            \
      const int c = (int)(_g - (long long)r * ((J).cols / 4)) * 4;                         \
      __VA_ARGS__                                                                          \
    }                                                                                      \
  }

// M <- b1 M + (1-b1) G.  a = G (lda), f0 = M (in place, ldf); planes of G -> pa,
// planes of the new M -> pb (ldp).
__global__ void __launch_bounds__(256) pc_momentum_kernel(const EwJob* __restrict__ J, int n, float b1) {
  const EwJob& j = J[find_job(J, n, blockIdx.x)];
  const int local = blockIdx.x - j.blk_begin;
  MAO_EW_LOOP(j, local, {
    const float4 g = load4(j.a, (long long)r * j.lda + c, j.a_bf16);
    float* mp = j.f0 + (long long)r * j.ldf + c;
    const float4 m = *reinterpret_cast<const float4*>(mp);
    const float4 mn = make_float4(b1 * m.x + (1.f - b1) * g.x, b1 * m.y + (1.f - b1) * g.y,
                                  b1 * m.z + (1.f - b1) * g.z, b1 * m.w + (1.f - b1) * g.w);
    *reinterpret_cast<float4*>(mp) = mn;
    const long long o = (long long)r * j.ldp + c;
    store_split3x4(g, j.pa, o, j.pstride);
    store_split3x4(mn, j.pb, o, j.pstride);
  })
}

// Three-plane split of an fp32 matrix: a (lda) -> pa planes (ldp).  Gated by flag.
__global__ void __launch_bounds__(256) pc_split_kernel(const EwJob* __restrict__ J, int n) {
  const EwJob& j = J[find_job(J, n, blockIdx.x)];
  if (j.flag && *j.flag == 0) return;
  const int local = blockIdx.x - j.blk_begin;
  MAO_EW_LOOP(j, local, {
    const float4 x = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(j.a) + (long long)r * j.lda + c);
    store_split3x4(x, j.pa, (long long)r * j.ldp + c, j.pstride);
  })
}

// SOAP Adam in the eigenbasis.  a = Ghat (lda), b = Mhat (ldb), f0 = V (caller, ldf),
// f1 = permuted previous V (ldf) or nullptr (read V itself); N planes -> pa.
// V <- b2 Vprev + (1-b2) Ghat^2 ; N = (Mhat/bc1) / (sqrt(V/bc2) + eps)
__global__ void __launch_bounds__(256) soap_adam_kernel(const EwJob* __restrict__ J, int n, float b2, float inv_bc1,
                                                        float inv_bc2, float eps) {
  const EwJob& j = J[find_job(J, n, blockIdx.x)];
  const int local = blockIdx.x - j.blk_begin;
  MAO_EW_LOOP(j, local, {
    const float4 g = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(j.a) + (long long)r * j.lda + c);
    const float4 m = *reinterpret_cast<const float4*>(j.b + (long long)r * j.ldb + c);
    const long long of = (long long)r * j.ldf + c;
    const float4 vp = *reinterpret_cast<const float4*>((j.f1 ? j.f1 : j.f0) + of);
    float gv[4] = {g.x, g.y, g.z, g.w}, mv[4] = {m.x, m.y, m.z, m.w}, v[4] = {vp.x, vp.y, vp.z, vp.w}, nv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[e] = b2 * v[e] + (1.f - b2) * gv[e] * gv[e];
      nv[e] = (mv[e] * inv_bc1) / (sqrtf(v[e] * inv_bc2) + eps);
    }
    *reinterpret_cast<float4*>(j.f0 + of) = make_float4(v[0], v[1], v[2], v[3]);
    store_split3x4(make_float4(nv[0], nv[1], nv[2], nv[3]), j.pa, (long long)r * j.ldp + c, j.pstride);
  })
}

// ------------------------------------------------------------------ sort keys / permutation
// Per matrix (k x k row-major P and Q, ld k): key_i = sum_r Q[r][i] * P[r][i] in fp64.
struct SortJob {
  const float* Q;
  const float* P;
  double* key;
  int* perm;          // workspace permutation (always written when the refresh runs)
  int* perm_out;      // caller's copy, or nullptr
  const int* flag;
  int k;
  int col_blk_begin;  // blocks of 256 columns (keys) / 256 ranks (argsort)
};

__device__ __forceinline__ int find_sort(const SortJob* J, int n, int blk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].col_blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) pc_keys_kernel(const SortJob* __restrict__ J, int n) {
  const SortJob& j = J[find_sort(J, n, blockIdx.x)];
  if (j.flag && *j.flag == 0) return;
  const int i = (blockIdx.x - j.col_blk_begin) * 256 + threadIdx.x;
  if (i >= j.k) return;
  double s = 0.0;
  for (int r = 0; r < j.k; ++r) s += (double)j.Q[(long long)r * j.k + i] * (double)j.P[(long long)r * j.k + i];
  if (!(s == s)) s = -INFINITY;  // a NaN key sorts last, so the permutation stays a bijection
  j.key[i] = s;
}

// Sorting disabled: strictly decreasing keys, so the argsort yields the identity.
__global__ void __launch_bounds__(256) pc_identity_keys_kernel(const SortJob* __restrict__ J, int n) {
  const SortJob& j = J[find_sort(J, n, blockIdx.x)];
  if (j.flag && *j.flag == 0) return;
  const int i = (blockIdx.x - j.col_blk_begin) * 256 + threadIdx.x;
  if (i < j.k) j.key[i] = -(double)i;
}

// Stable descending argsort by rank counting: rank_i = #{key_j > key_i} + #{j < i: key_j == key_i};
// perm[rank_i] = i.  Exact and deterministic.
// A refresh that does not run (flag 0) reports the identity permutation.
__global__ void __launch_bounds__(256) pc_argsort_kernel(const SortJob* __restrict__ J, int n) {
  __shared__ double sk[2048];
  const SortJob& j = J[find_sort(J, n, blockIdx.x)];
  const int i = (blockIdx.x - j.col_blk_begin) * 256 + threadIdx.x;
  if (j.flag && *j.flag == 0) {
    if (j.perm_out && i < j.k) j.perm_out[i] = i;
    return;
  }
  const double ki = (i < j.k) ? j.key[i] : 0.0;
  int rank = 0;
  for (int base = 0; base < j.k; base += 2048) {
    const int len = min(2048, j.k - base);
    __syncthreads();
    for (int t = threadIdx.x; t < len; t += 256) sk[t] = j.key[base + t];
    __syncthreads();
    if (i < j.k) {
      for (int t = 0; t < len; ++t) {
        const double kt = sk[t];
        rank += (kt > ki) || (kt == ki && base + t < i);
      }
    }
  }
  if (i < j.k) {
    j.perm[rank] = i;
    if (j.perm_out) j.perm_out[rank] = i;
  }
}

// Column gather of a k x k matrix: dst[r][i] = src[r][perm[i]], plus its planes.
struct GatherJob {
  const float* src;
  float* dst;
  __nv_bfloat16* dstp;  // plane set (ldp, pstride)
  long long pstride;
  const int* perm;
  const int* flag;
  int rows, cols, ld, ldp;
  int blk_begin;
};

__global__ void __launch_bounds__(256) pc_gather_cols_kernel(const GatherJob* __restrict__ J, int n) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].blk_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const GatherJob& j = J[lo];
  if (j.flag && *j.flag == 0) return;
  const long long total = (long long)j.rows * j.cols;
  const long long e0 = (long long)(blockIdx.x - j.blk_begin) * kElemsPerBlock;
  for (int k = 0; k < kElemsPerBlock / 256; ++k) {
    const long long e = e0 + k * 256 + threadIdx.x;
    if (e >= total) break;
    const int r = (int)(e / j.cols), c = (int)(e - (long long)r * j.cols);
    const float x = j.src[(long long)r * j.ld + j.perm[c]];
    if (j.dst) j.dst[(long long)r * j.ld + c] = x;
    if (j.dstp) store_split3(x, j.dstp, (long long)r * j.ldp + c, j.pstride);
  }
}

// SOAP V permutation into a scratch copy: dst[i][j] = V[pl[i]][pr[j]] (pl, pr
// nullable = identity).  Uses the flags of the two sides through the perms:
// a side that did not refresh passes nullptr.
struct VPermJob {
  const float* V;
  float* dst;
  const int* pl;
  const int* pr;
  const int* fl;  // left refresh flag (nullable = refreshed when pl != nullptr)
  const int* fr;
  int m, n;
  int blk_begin;
};

__global__ void __launch_bounds__(256) soap_vperm_kernel(const VPermJob* __restrict__ J, int cnt) {
  int lo = 0, hi = cnt - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].blk_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const VPermJob& j = J[lo];
  const bool ul = j.pl && (!j.fl || *j.fl != 0);
  const bool ur = j.pr && (!j.fr || *j.fr != 0);
  const long long total = (long long)j.m * j.n;
  const long long e0 = (long long)(blockIdx.x - j.blk_begin) * kElemsPerBlock;
  for (int k = 0; k < kElemsPerBlock / 256; ++k) {
    const long long e = e0 + k * 256 + threadIdx.x;
    if (e >= total) break;
    const int r = (int)(e / j.n), c = (int)(e - (long long)r * j.n);
    const int sr = ul ? j.pl[r] : r, sc = ur ? j.pr[c] : c;
    j.dst[e] = j.V[(long long)sr * j.n + sc];
  }
}

// ------------------------------------------------------------------ QR panel pieces
// A panel W (rows x w, w <= 64, leading dimension ld) of one matrix.
constexpr int kPanel = 64;
constexpr int kGramRows = 512;  // rows per Gram partial block

struct PanelJob {
  float* W;          // panel base (column 0 of the panel), fp32
  __nv_bfloat16* Wp; // optional plane set written by the apply pass (ld kPanel, stride wps)
  long long wps;
  float* Q;          // optional final destination (column 0 of the panel in Q), or nullptr
  __nv_bfloat16* Qp; // planes of Q (column 0 of the panel; ld ldqp, stride qps)
  long long qps;
  int ldqp;
  double* gram;      // chunks x 64 x 64 partial Grams
  double* rinv;      // 64 x 64 inverse of the Cholesky factor
  int* bad;          // counts non-positive pivots
  const int* flag;
  int rows, w, ld, ldq;
  int chunks;        // ceil(rows / kGramRows)
  int blk_begin;     // gram: chunk blocks; apply: row blocks of 64
};

__device__ __forceinline__ int find_panel(const PanelJob* J, int n, int blk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].blk_begin <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Partial Gram over kGramRows rows: thread (ty, tx) owns G[4ty..4ty+3][4tx..4tx+3].
__global__ void __launch_bounds__(256) qr_gram_kernel(const PanelJob* __restrict__ J, int n) {
  __shared__ float sw[32][kPanel + 1];
  const PanelJob& j = J[find_panel(J, n, blockIdx.x)];
  if (j.flag && *j.flag == 0) return;
  const int chunk = blockIdx.x - j.blk_begin;
  const int r0 = chunk * kGramRows, r1 = min(j.rows, r0 + kGramRows);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[4][4] = {};
  for (int rb = r0; rb < r1; rb += 32) {
    __syncthreads();
    for (int t = threadIdx.x; t < 32 * kPanel; t += 256) {
      const int rr = t / kPanel, cc = t % kPanel;
      const int r = rb + rr;
      sw[rr][cc] = (r < r1 && cc < j.w) ? j.W[(long long)r * j.ld + cc] : 0.f;
    }
    __syncthreads();
    const int nr = min(32, r1 - rb);
    for (int rr = 0; rr < nr; ++rr) {
      double a[4], b[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a[e] = (double)sw[rr][4 * ty + e];
        b[e] = (double)sw[rr][4 * tx + e];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] += a[p] * b[q];
    }
  }
  double* g = j.gram + (long long)chunk * kPanel * kPanel;
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) g[(4 * ty + p) * kPanel + 4 * tx + q] = acc[p][q];
}

// One block per matrix: G = sum of the partial Grams (fixed order), Cholesky
// G = R^T R (R upper, positive diagonal), then R^{-1} (upper triangular).
// R lives in the strict upper triangle of G with its diagonal in Rd; R^{-1} is
// built transposed in the lower triangle (diagonal included).
__global__ void __launch_bounds__(256) qr_chol_kernel(const PanelJob* __restrict__ J, int n) {
  __shared__ double G[kPanel][kPanel + 1];
  __shared__ double Rd[kPanel];
  const PanelJob& j = J[blockIdx.x];
  if (j.flag && *j.flag == 0) return;
  const int w = j.w;
  for (int t = threadIdx.x; t < kPanel * kPanel; t += 256) {
    const int a = t / kPanel, b = t % kPanel;
    double s = 0.0;
    for (int c = 0; c < j.chunks; ++c) s += j.gram[(long long)c * kPanel * kPanel + t];
    G[a][b] = (a < w && b < w) ? s : (a == b ? 1.0 : 0.0);
  }
  __syncthreads();
  // right-looking Cholesky on the upper triangle: row k of R
  for (int k = 0; k < kPanel; ++k) {
    if (threadIdx.x == 0) {
      double d = G[k][k];
      if (!(d > 0.0)) {
        atomicAdd(j.bad, 1);
        d = 1e-300;
      }
      G[k][k] = sqrt(d);
      Rd[k] = G[k][k];
    }
    __syncthreads();
    const double rkk = G[k][k];
    for (int c = k + 1 + threadIdx.x; c < kPanel; c += 256) G[k][c] /= rkk;
    __syncthreads();
    // trailing update G[a][b] -= R[k][a] R[k][b] for k < a <= b
    for (int t = threadIdx.x; t < kPanel * kPanel; t += 256) {
      const int a = t / kPanel, b = t % kPanel;
      if (a > k && b >= a) G[a][b] -= G[k][a] * G[k][b];
    }
    __syncthreads();
  }
  // R^{-1}: thread c solves R x = e_c by back substitution; x_r is kept at G[c][r]
  if (threadIdx.x < kPanel) {
    const int c = threadIdx.x;
    for (int r = c; r >= 0; --r) {
      double s = (r == c) ? 1.0 : 0.0;
      for (int k = r + 1; k <= c; ++k) s -= G[r][k] * G[c][k];
      G[c][r] = s / Rd[r];
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < kPanel * kPanel; t += 256) {
    const int r = t / kPanel, c = t % kPanel;
    j.rinv[t] = (r <= c) ? G[c][r] : 0.0;
  }
}

// W <- W R^{-1} for kApplyRows rows per block (fp64 accumulation); optionally
// also writes the result and its three-plane split to Q and to W's plane set.
constexpr int kApplyRows = 32;

__global__ void __launch_bounds__(256) qr_apply_kernel(const PanelJob* __restrict__ J, int n) {
  __shared__ double Ri[kPanel][kPanel + 1];
  __shared__ float sw[kApplyRows][kPanel + 1];
  const PanelJob& j = J[find_panel(J, n, blockIdx.x)];
  if (j.flag && *j.flag == 0) return;
  const int r0 = (blockIdx.x - j.blk_begin) * kApplyRows;
  for (int t = threadIdx.x; t < kPanel * kPanel; t += 256) Ri[t / kPanel][t % kPanel] = j.rinv[t];
  for (int t = threadIdx.x; t < kApplyRows * kPanel; t += 256) {
    const int rr = t / kPanel, cc = t % kPanel;
    const int r = r0 + rr;
    sw[rr][cc] = (r < j.rows && cc < j.w) ? j.W[(long long)r * j.ld + cc] : 0.f;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < kApplyRows * kPanel; t += 256) {
    const int rr = t / kPanel, c = t % kPanel;
    const int r = r0 + rr;
    if (r >= j.rows || c >= j.w) continue;
    double s = 0.0;
    for (int a = 0; a <= c; ++a) s += (double)sw[rr][a] * Ri[a][c];
    const float x = (float)s;
    j.W[(long long)r * j.ld + c] = x;
    if (j.Wp) store_split3(x, j.Wp, (long long)r * kPanel + c, j.wps);
    if (j.Q) {
      j.Q[(long long)r * j.ldq + c] = x;
      store_split3(x, j.Qp, (long long)r * j.ldqp + c, j.qps);
    }
  }
}

// ------------------------------------------------------------------ FOAM pieces
// Row/column partial sums of Gr^2 over 64 x 64 tiles (Gr m x n fp32, ld n).
struct RcJob {
  const float* Gr;
  float* rowpart;  // tiles_c x m
  float* colpart;  // tiles_r x n
  int m, n, tiles_c, tiles_r;
  int blk_begin;
};

__global__ void __launch_bounds__(256) foam_rc_partial_kernel(const RcJob* __restrict__ J, int cnt) {
  __shared__ float csum[16][64];
  int lo = 0, hi = cnt - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (J[mid].blk_begin <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  const RcJob& j = J[lo];
  const int local = blockIdx.x - j.blk_begin;
  const int tr = local / j.tiles_c, tc = local % j.tiles_c;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int c = tc * 64 + 4 * tx;
  float cs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr * 64 + ty + 16 * i;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < j.m && c < j.n) {
      const float4 q = *reinterpret_cast<const float4*>(j.Gr + (long long)r * j.n + c);
      v[0] = q.x * q.x; v[1] = q.y * q.y; v[2] = q.z * q.z; v[3] = q.w * q.w;
    }
    float s = v[0] + v[1] + v[2] + v[3];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (tx == 0 && r < j.m) j.rowpart[(long long)tc * j.m + r] = s;
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[e] += v[e];
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) csum[ty][4 * tx + e] = cs[e];
  __syncthreads();
  if (threadIdx.x < 64) {
    const int col = tc * 64 + threadIdx.x;
    float s = 0.f;
    for (int g = 0; g < 16; ++g) s += csum[g][threadIdx.x];
    if (col < j.n) j.colpart[(long long)tr * j.n + col] = s;
  }
}

// Per matrix: r, c EMAs (c follows the refresh permutation), trace of R, and
// tau = tr(R^) / (|r^|_1 |c^|_1), one block per matrix, fixed-order sums.
struct TauJob {
  float* r;
  float* c;
  const float* rowpart;
  const float* colpart;
  const float* R;
  const int* perm;   // refresh permutation of c (valid when flag != 0), or nullptr
  const int* flag;
  float* c_tmp;      // n scratch
  float* tau;        // 1 value
  int m, n, tiles_c, tiles_r;
};

__global__ void __launch_bounds__(256) foam_tau_kernel(const TauJob* __restrict__ J, float b2, float inv_bc2,
                                                       int raw_trace) {
  __shared__ double red[3][256];
  const TauJob& j = J[blockIdx.x];
  const bool permute = j.perm && (!j.flag || *j.flag != 0);
  // c permuted into scratch first (the EMA below reads old values at permuted positions)
  if (permute) {
    for (int i = threadIdx.x; i < j.n; i += 256) j.c_tmp[i] = j.c[j.perm[i]];
    __syncthreads();
  }
  double sr = 0.0, sc = 0.0, st = 0.0;
  for (int i = threadIdx.x; i < j.m; i += 256) {
    double s = 0.0;
    for (int t = 0; t < j.tiles_c; ++t) s += (double)j.rowpart[(long long)t * j.m + i];
    const float v = b2 * j.r[i] + (1.f - b2) * (float)(s / j.n);
    j.r[i] = v;
    sr += fabs((double)v);
  }
  for (int i = threadIdx.x; i < j.n; i += 256) {
    double s = 0.0;
    for (int t = 0; t < j.tiles_r; ++t) s += (double)j.colpart[(long long)t * j.n + i];
    const float old = permute ? j.c_tmp[i] : j.c[i];
    const float v = b2 * old + (1.f - b2) * (float)(s / j.m);
    j.c[i] = v;
    sc += fabs((double)v);
    st += (double)j.R[(long long)i * j.n + i];
  }
  red[0][threadIdx.x] = sr;
  red[1][threadIdx.x] = sc;
  red[2][threadIdx.x] = st;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o)
      for (int q = 0; q < 3; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double rn = red[0][0] * inv_bc2, cn = red[1][0] * inv_bc2;
    const double tr = raw_trace ? red[2][0] : red[2][0] * inv_bc2;
    *j.tau = (float)(tr / (rn * cn));
  }
}

// FOAM update direction in the rotated space:
// N_ij = (Mr_ij / bc1) / (sqrt(tau r^_i c^_j) + eps), written as three planes.
// a = Mr (fp32, lda), b = tau, vr = r, vc = c, N planes -> pa (ldp).
__global__ void __launch_bounds__(256) foam_n_kernel(const EwJob* __restrict__ J, int n, float inv_bc1,
                                                     float inv_bc2, float eps) {
  const EwJob& j = J[find_job(J, n, blockIdx.x)];
  const int local = blockIdx.x - j.blk_begin;
  const float tau = *j.b;
  MAO_EW_LOOP(j, local, {
    const float4 mr = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(j.a) + (long long)r * j.lda + c);
    const float ri = j.vr[r] * inv_bc2;
    const float mv[4] = {mr.x, mr.y, mr.z, mr.w};
    float nv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float v = tau * ri * (j.vc[c + e] * inv_bc2);
      nv[e] = (mv[e] * inv_bc1) / (sqrtf(v) + eps);
    }
    store_split3x4(make_float4(nv[0], nv[1], nv[2], nv[3]), j.pa, (long long)r * j.ldp + c, j.pstride);
  })
}

// Adaptive check: rho = ||offdiag D||_F / ||D||_F, flag = rho > tol (one block per matrix).
struct CheckJob {
  const float* D;
  int* flag;
  float* rho;
  int k;
};

__global__ void __launch_bounds__(256) pc_check_kernel(const CheckJob* __restrict__ J, float tol) {
  __shared__ double red[2][256];
  const CheckJob& j = J[blockIdx.x];
  double off = 0.0, tot = 0.0;
  const long long total = (long long)j.k * j.k;
  for (long long e = threadIdx.x; e < total; e += 256) {
    const double x = j.D[e];
    const int r = (int)(e / j.k), c = (int)(e - (long long)r * j.k);
    tot += x * x;
    if (r != c) off += x * x;
  }
  red[0][threadIdx.x] = off;
  red[1][threadIdx.x] = tot;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      red[0][threadIdx.x] += red[0][threadIdx.x + o];
      red[1][threadIdx.x] += red[1][threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double rho = red[1][0] > 0.0 ? sqrt(red[0][0]) / sqrt(red[1][0]) : 0.0;
    *j.rho = (float)rho;
    *j.flag = (rho > (double)tol) ? 1 : 0;
  }
}

// Per-matrix diagnostics of a SOAP / FOAM step: refresh bits and the check ratio.
// fixed_bits >= 0: the refresh was decided on the host (bits given); otherwise
// read the device flags (bit 0 right side, bit 1 left side).
struct StatsJob {
  const int* flag_r;
  const int* flag_l;
  const float* rho;
  int fixed_bits;
  int index;  // position in the caller's stats array
};

__global__ void pc_stats_kernel(const StatsJob* __restrict__ J, int n, mao_stats* __restrict__ stats) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const StatsJob& j = J[i];
  int bits = j.fixed_bits;
  if (bits < 0) bits = ((j.flag_r && *j.flag_r) ? 1 : 0) | ((j.flag_l && *j.flag_l) ? 2 : 0);
  mao_stats& st = stats[j.index];
  st.update_rms = -1.0f;
  st.offdiag_ratio = j.rho ? *j.rho : -1.0f;
  st.refreshed = bits;
  st.nonfinite = 0;
}

}  // namespace mao
