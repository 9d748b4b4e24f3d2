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

// Every job array of n records is followed by the compact first-block indices of
// its records (two arrays for SortJob: the key pass's, then the argsort's).
template <class J>
__device__ __forceinline__ const int* job_starts(const J* jobs, int n, int which = 0) {
  return reinterpret_cast<const int*>(jobs + n) + which * n;
}

__device__ __forceinline__ int find_job(const EwJob* J, int n, int blk) {
  return find_start(job_starts(J, n), n, blk);
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

// M <- b1 M + (1-b1) G.  a = G (lda), f0 = M (in place, ldf); planes of G -> pa
// (unless nullptr), planes of the new M -> pb (ldp).
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
    if (j.pa) store_split3x4(g, j.pa, o, j.pstride);
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
  float* pn;          // squared column norms of P (original order)
  float* pn_sorted;   // ... in the sorted order (argsort), or nullptr
  double* dg;         // diag(Q^T F Q) = the dot products (adaptive check), or nullptr
  const int* kflag;   // gate of the key pass (nullptr: always runs)
  int* perm;          // workspace permutation (always written when the refresh runs)
  int* perm_out;      // caller's copy, or nullptr
  const int* flag;
  int k;
  int col_blk_begin;  // blocks of 256 ranks (argsort, identity keys)
  int key_blk_begin;  // blocks of 32 columns (keys)
};

template <bool KEYS>
__device__ __forceinline__ int find_sort(const SortJob* J, int n, int blk) {
  return find_start(job_starts(J, n, KEYS ? 0 : 1), n, blk);
}

// key_i = sum_r Q[r][i] P[r][i] in fp64 (or -i when sorting is off, which makes
// the argsort the identity), and the squared column norms of P in the same pass:
// one block per 32 columns, warp w sums the rows w, w + 8, ... (each warp reads 128
// contiguous bytes per row of Q and P), then the eight warp sums are added in warp order.
__global__ void __launch_bounds__(256) pc_keys_kernel(const SortJob* __restrict__ J, int n, int sort) {
  __shared__ double part[8][32];
  __shared__ float partn[8][32];
  const SortJob& j = J[find_sort<true>(J, n, blockIdx.x)];
  if (j.kflag && *j.kflag == 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = (blockIdx.x - j.key_blk_begin) * 32 + lane;
  const bool dots = sort || j.dg;
  // four rows per iteration (independent accumulators keep eight loads in flight)
  double s[4] = {0.0, 0.0, 0.0, 0.0};
  float nrm[4] = {0.f, 0.f, 0.f, 0.f};
  if (i < j.k) {
    const float* P = j.P + i;
    const float* Q = j.Q + i;
    int r = warp;
    for (; r + 24 < j.k; r += 32) {
      float p[4], q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) p[u] = P[(long long)(r + 8 * u) * j.k];
      if (dots) {
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = Q[(long long)(r + 8 * u) * j.k];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        nrm[u] += p[u] * p[u];
        if (dots) s[u] += (double)q[u] * (double)p[u];
      }
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {  // at most three rows remain
      const int rr = r + 8 * u;
      if (rr < j.k) {
        const float p0 = P[(long long)rr * j.k];
        nrm[u] += p0 * p0;
        if (dots) s[u] += (double)Q[(long long)rr * j.k] * (double)p0;
      }
    }
  }
  part[warp][lane] = (s[0] + s[1]) + (s[2] + s[3]);
  partn[warp][lane] = (nrm[0] + nrm[1]) + (nrm[2] + nrm[3]);
  __syncthreads();
  if (warp == 0 && i < j.k) {
    double s = 0.0;
    float nn = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      s += part[w][lane];
      nn += partn[w][lane];
    }
    if (j.dg) j.dg[i] = s;
    if (!sort) s = -(double)i;
    if (!(s == s)) s = -INFINITY;  // a NaN key sorts last, so the permutation stays a bijection
    j.key[i] = s;
    j.pn[i] = nn;
  }
}

// Stable descending argsort by rank counting: rank_i = #{key_j > key_i} + #{j < i: key_j == key_i};
// perm[rank_i] = i.  Exact and deterministic.
// A refresh that does not run (flag 0) reports the identity permutation.
__global__ void __launch_bounds__(256) pc_argsort_kernel(const SortJob* __restrict__ J, int n) {
  __shared__ double sk[2048];
  const SortJob& j = J[find_sort<false>(J, n, blockIdx.x)];
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
    if (j.pn_sorted) j.pn_sorted[rank] = j.pn[i];
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

// Four consecutive destination columns per thread (cols is a multiple of 4): one
// 16-byte store of the fp32 copy and 8-byte stores of the planes.
__global__ void __launch_bounds__(256) pc_gather_cols_kernel(const GatherJob* __restrict__ J, int n) {
  const int lo = find_start(job_starts(J, n), n, (int)blockIdx.x);
  const GatherJob& j = J[lo];
  if (j.flag && *j.flag == 0) return;
  const int q4 = j.cols / 4;
  const long long groups = (long long)j.rows * q4;
  const long long g0 = (long long)(blockIdx.x - j.blk_begin) * (kElemsPerBlock / 4);
  for (int k = 0; k < kElemsPerBlock / 4 / 256; ++k) {
    const long long g = g0 + k * 256 + threadIdx.x;
    if (g >= groups) break;
    const int r = (int)(g / q4), c = 4 * (int)(g - (long long)r * q4);
    const int4 pc = *reinterpret_cast<const int4*>(j.perm + c);
    const float* srow = j.src + (long long)r * j.ld;
    const float4 x = make_float4(srow[pc.x], srow[pc.y], srow[pc.z], srow[pc.w]);
    if (j.dst) *reinterpret_cast<float4*>(j.dst + (long long)r * j.ld + c) = x;
    if (j.dstp) store_split3x4(x, j.dstp, (long long)r * j.ldp + c, j.pstride);
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
  const int lo = find_start(job_starts(J, cnt), cnt, (int)blockIdx.x);
  const VPermJob& j = J[lo];
  const bool ul = j.pl && (!j.fl || *j.fl != 0);
  const bool ur = j.pr && (!j.fr || *j.fr != 0);
  // four consecutive columns per thread (n is a multiple of 4)
  const int q4 = j.n / 4;
  const long long groups = (long long)j.m * q4;
  const long long g0 = (long long)(blockIdx.x - j.blk_begin) * (kElemsPerBlock / 4);
  for (int k = 0; k < kElemsPerBlock / 4 / 256; ++k) {
    const long long g = g0 + k * 256 + threadIdx.x;
    if (g >= groups) break;
    const int r = (int)(g / q4), c = 4 * (int)(g - (long long)r * q4);
    const float* srow = j.V + (long long)(ul ? j.pl[r] : r) * j.n;
    float4 x;
    if (ur) {
      const int4 pc = *reinterpret_cast<const int4*>(j.pr + c);
      x = make_float4(srow[pc.x], srow[pc.y], srow[pc.z], srow[pc.w]);
    } else {
      x = *reinterpret_cast<const float4*>(srow + c);
    }
    *reinterpret_cast<float4*>(j.dst + (long long)r * j.n + c) = x;
  }
}

// ------------------------------------------------------------------ QR panel pieces
// Cholesky-QR of one panel W (rows x w, w <= kPanel) per matrix:
//   Gram G = W^T W as fp32-faithful tensor-core products over K slices (fp32
//   partials)
//   -> reduction (many blocks per panel): the slices summed in fp64 in slice order,
//      column scaling Gs = D^-1/2 G D^-1/2 (D = diag G), the packed upper triangle of
//      Gs, ||Gs - I||_F partials, and the first-order inverse factor (below)
//   -> Cholesky Gs = Rs^T Rs and blocked inverse Rs^-1 in fp64, one block per
//      panel, only when Gs is not already close to the identity
//   -> R^{-1} = D^-1/2 Rs^{-1}, three bf16 planes, for the product W R^{-1}.
// Nearly orthonormal panel (the usual case after a first Cholesky-QR): with
// Gs = I + E and ||E||_F <= kFastTol, Rs = I + U + O(E^2) where U is the strict
// upper triangle of E plus half its diagonal, so Rs^{-1} = I - U to O(E^2) <= 1e-8,
// below the fp32 unit roundoff.
// A first pass of a panel that needs the full factorisation shifts Gs by
// kCholShift (by kCholShiftRetry after a breakdown) so it stays defined for nearly
// dependent columns, and asks for a second pass, which restores orthogonality; the
// triangular structure makes the final Q the positive-diagonal QR factor either way.
constexpr int kPanel = 128;
constexpr int kSuper = 2 * kPanel;  // columns projected together against the finished ones
constexpr int kPanelSq = kPanel * kPanel;
constexpr int kPackedUpper = kPanel * (kPanel + 1) / 2;  // packed upper triangle, row-major
constexpr int kMaxParts = 16;                             // K slices of a panel Gram
constexpr int kRedRows = 8;                               // Gram rows per reduction block
constexpr int kRedBlocks = kPanel / kRedRows;
constexpr int kGsDoubles = kPackedUpper + kPanel + kRedBlocks;  // Gs | D^-1/2 | ||E||^2 partials
constexpr int kCholSmem = (kPanel * (kPanel + 1) + (kPanel - 32) * 32 + 2 * kPanel) * 8;
constexpr double kCholShift = 1e-4;  // relative to the unit diagonal of Gs, after a non-positive pivot
constexpr double kAgainMeanInv = 16.0;  // mean of 1/eig(Gs) (= ||Rs^-1||_F^2 / w) above which a first
                                        // pass is followed by a second one
constexpr double kFastTol = 1e-4;

struct PanelJob {
  const float* part;     // nparts x kPanel x kPanel fp32 partial Grams (ld kPanel)
  double* gs;            // kGsDoubles
  __nv_bfloat16* rinv;   // three planes (kPanel x kPanel each) of R^{-1}: upper triangle, zero elsewhere
  int* bad;              // counts panels whose shifted factorisation still broke down
  int* again;            // first pass: set to 1 when a second Cholesky-QR pass is needed, else 0
  const float* pnorm2;   // first pass after a projection: squared norms of the panel's columns
                         // before the projection (else nullptr)
  int* reorth;           // ... and the flag set to 1 when a second projection is needed, else 0
  int* fin;              // first pass: set to 1 when the panel needs a final Cholesky-QR pass
                         // (a second pass or a second projection ran), else 0
  const int* flag;
  // first pass: launch-level gates set to 1 when this panel takes the second pass,
  // the second projection or the final pass (nullptr: not tracked)
  int* any_again;
  int* any_reorth;
  int* any_fin;
  int w, nparts;
  int first;
};

// Indices of a group's launch-level gates (ints): any second Cholesky-QR pass, any
// second projection, any final pass.
constexpr int kAnyAgain = 0, kAnyReorth = 1, kAnyFin = 2;

// Selective reorthogonalisation (the classical criterion of Daniel, Gragg, Kaufman
// and Stewart, per column): a second projection pass is needed when the first pass
// removed more than half of some column's squared norm.
constexpr double kReorthRatio = 0.5;

// (r, c), r <= c, of the packed upper triangle
__device__ __forceinline__ int pk(int r, int c) { return ((r * (2 * kPanel + 1 - r)) >> 1) + (c - r); }

// kRedBlocks blocks per panel, block rb owns Gram rows [rb*kRedRows, +kRedRows).
__global__ void __launch_bounds__(256) qr_gram_reduce_kernel(const PanelJob* __restrict__ J,
                                                              const int* __restrict__ any) {
  __shared__ double dsh[kPanel];
  __shared__ double red[8];
  if (any && *any == 0) return;  // no panel of the launch takes this pass
  const PanelJob& j = J[blockIdx.x / kRedBlocks];
  const int rb = blockIdx.x % kRedBlocks;
  if (j.flag && *j.flag == 0) return;
  const int w = j.w, tid = threadIdx.x;
  int cancel = 0;
  if (tid < kPanel) {
    double d = 1.0;
    if (tid < w) {
      float v[kMaxParts];
#pragma unroll
      for (int p = 0; p < kMaxParts; ++p)
        v[p] = p < j.nparts ? j.part[(long long)p * kPanelSq + tid * (kPanel + 1)] : 0.0f;
      d = 0.0;
#pragma unroll
      for (int p = 0; p < kMaxParts; ++p) d += (double)v[p];
      if (j.pnorm2 && rb == 0) cancel = d < kReorthRatio * (double)j.pnorm2[tid];
    }
    const double s = (d > 0.0) ? rsqrt(d) : 1.0;
    dsh[tid] = s;
    if (rb == 0) j.gs[kPackedUpper + tid] = s;
  }
  cancel = __syncthreads_or(cancel);
  if (j.pnorm2 && rb == 0 && tid == 0) {
    *j.reorth = cancel ? 1 : 0;
    if (cancel && j.any_reorth) *j.any_reorth = 1;
  }
  // one 4-column group of one row per thread
  const int a = rb * kRedRows + (tid >> 5), b0 = (tid & 31) * 4;
  double g[4] = {0.0, 0.0, 0.0, 0.0};
  if (a < w && b0 < w) {
    float4 v[kMaxParts];
#pragma unroll
    for (int p = 0; p < kMaxParts; ++p)
      if (p < j.nparts) v[p] = *reinterpret_cast<const float4*>(j.part + (long long)p * kPanelSq + a * kPanel + b0);
#pragma unroll
    for (int p = 0; p < kMaxParts; ++p)
      if (p < j.nparts) {
        g[0] += (double)v[p].x;
        g[1] += (double)v[p].y;
        g[2] += (double)v[p].z;
        g[3] += (double)v[p].w;
      }
  }
  double e2 = 0.0;
  float rv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = b0 + e;
    const double id = (a == b) ? 1.0 : 0.0;
    const double x = (a < w && b < w) ? g[e] * dsh[a] * dsh[b] : id;
    rv[e] = 0.0f;
    if (b >= a) {
      j.gs[pk(a, b)] = x;
      const double ee = x - id;
      e2 += (a == b ? 1.0 : 2.0) * ee * ee;
      if (b < w) rv[e] = (float)(dsh[a] * (id - (a == b ? 0.5 * ee : ee)));
    }
  }
  store_split3x4(make_float4(rv[0], rv[1], rv[2], rv[3]), j.rinv, (long long)a * kPanel + b0, kPanelSq);
  e2 = warp_sum_d(e2);
  if ((tid & 31) == 0) red[tid >> 5] = e2;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) t += red[i];
    j.gs[kPackedUpper + kPanel + rb] = t;
  }
}

// Cholesky of Gs and the inverse of its factor, fp64 in shared memory (row-major,
// leading dimension kLdA; only the upper triangle is meaningful).  Work is laid
// out so that a warp's shared-memory accesses are a row segment across lanes or a
// broadcast, and inner products keep several independent accumulators.
constexpr int kLdA = kPanel + 1;

__global__ void __launch_bounds__(256, 1) qr_chol_kernel(const PanelJob* __restrict__ J, const int* __restrict__ any) {
  extern __shared__ double chol_smem[];
  double* A = chol_smem;                  // [kPanel][kLdA]: Gs, then Rs, then Rs^{-1}
  double* T = A + kPanel * kLdA;          // [kPanel - 32][32] block-column workspace of the inverse
  double* ds = T + (kPanel - 32) * 32;    // D^-1/2
  double* rdi = ds + kPanel;              // 1 / Rs[k][k]
  __shared__ int nbad_sh;
  __shared__ double red_sh[8];
  if (any && *any == 0) return;  // no panel of the launch takes this pass
  const PanelJob& j = J[blockIdx.x];
  if (j.flag && *j.flag == 0) return;
  const int w = j.w;
  const int nb = (w + 31) / 32, wp = nb * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr unsigned FULL = 0xffffffffu;

  double tot = 0.0;
#pragma unroll
  for (int i = 0; i < kRedBlocks; ++i) tot += j.gs[kPackedUpper + kPanel + i];
  if (tot <= kFastTol * kFastTol) {  // the first-order inverse is already in place
    if (j.first && tid == 0) {
      *j.again = 0;
      const int fin = j.reorth ? *j.reorth : 0;
      *j.fin = fin;
      if (fin && j.any_fin) *j.any_fin = 1;
    }
    return;
  }
  if (tid < kPanel) ds[tid] = j.gs[kPackedUpper + tid];

  int shifted = 0;
  for (int attempt = 0; attempt < 2; ++attempt) {
    // unpack the upper triangle, row r by warp r % 8
    for (int r = warp; r < wp; r += 8) {
      const double* src = j.gs + pk(r, r) - r;  // so that src[c] = Gs[r][c] for c >= r
      for (int c = r + lane; c < wp; c += 32) A[r * kLdA + c] = src[c];
    }
    if (tid == 0) nbad_sh = 0;
    __syncthreads();
    if (attempt && tid < wp) A[tid * kLdA + tid] += kCholShift;
    __syncthreads();
    // ---- blocked Cholesky, upper: Gs = Rs^T Rs
    for (int bk = 0; bk < nb; ++bk) {
      const int o = bk * 32;
      if (warp == 0) {
        // lane c holds column o + c of the diagonal block (rows <= c)
        double v[32];
        int nbad = 0;
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = (r <= lane) ? A[(o + r) * kLdA + o + lane] : 0.0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          double d = __shfl_sync(FULL, v[k], k);
          nbad += (d > 0.0) ? 0 : 1;
          d = (d > 0.0) ? d : 1e-300;
          const double ri = rsqrt(d);  // 1 / Rs[k][k]
          const double rk = (lane == k) ? d * ri : (lane > k ? v[k] * ri : 0.0);  // Rs[k][c]
          if (lane == k) rdi[o + k] = ri;
          v[k] = rk;
#pragma unroll
          for (int i = 1; i < 32; ++i) {
            if (i > k) {  // constant trip count keeps v[] in registers
              const double rki = __shfl_sync(FULL, rk, i);
              if (i <= lane) v[i] -= rki * rk;
            }
          }
        }
#pragma unroll
        for (int r = 0; r < 32; ++r)
          if (r <= lane) A[(o + r) * kLdA + o + lane] = v[r];
        if (lane == 0 && nbad) nbad_sh += nbad;
      }
      __syncthreads();
      if (attempt == 0 && nbad_sh) break;  // broke down: start over, shifted
      const int nt = wp - o - 32;  // trailing columns
      if (nt == 0) break;
      // block row: Rs_bc = Rs_bb^{-T} G_bc, one column per thread (right-looking in registers)
      if (tid < nt) {
        const int c = o + 32 + tid;
        double x[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) x[r] = A[(o + r) * kLdA + c];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          x[r] *= rdi[o + r];
          const double* rrow = A + (o + r) * kLdA + o;
#pragma unroll
          for (int i = r + 1; i < 32; ++i) x[i] -= rrow[i] * x[r];
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) A[(o + r) * kLdA + c] = x[r];
      }
      __syncthreads();
      // trailing update G_cd -= sum_i Rs[o+i][c] Rs[o+i][d] over the whole trailing
      // square (the lower half is never read): a warp owns two rows c, lanes own
      // columns d, d + 32, d + 64
      {
        const int t0 = o + 32;
        for (int cp = warp * 2; cp < nt; cp += 16) {
          const int c0 = t0 + cp, c1 = c0 + 1;
          double acc[2][3] = {};
#pragma unroll 4
          for (int i = 0; i < 32; ++i) {
            const double* row = A + (o + i) * kLdA;
            const double a0 = row[c0], a1 = row[c1];
#pragma unroll
            for (int q = 0; q < 3; ++q) {
              const int d = t0 + lane + 32 * q;
              const double b = (d < wp) ? row[d] : 0.0;
              acc[0][q] = fma(a0, b, acc[0][q]);
              acc[1][q] = fma(a1, b, acc[1][q]);
            }
          }
#pragma unroll
          for (int q = 0; q < 3; ++q) {
            const int d = t0 + lane + 32 * q;
            if (d < wp) {
              A[c0 * kLdA + d] -= acc[0][q];
              A[c1 * kLdA + d] -= acc[1][q];
            }
          }
        }
      }
      __syncthreads();
    }
    __syncthreads();
    shifted = attempt;
    if (nbad_sh == 0 || attempt == 1) break;  // retry once, shifted
    __syncthreads();
  }
  if (tid == 0 && nbad_sh) atomicAdd(j.bad, 1);

  // ---- inverse in place.  Diagonal blocks first, one warp each: column c = lane of
  // Rs_bb^{-1}, from the last row up, written over Rs_bb as it goes (row k of the
  // block is not read again once step k is done).
  if (warp < nb) {
    const int o = warp * 32;
    double acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.0;
#pragma unroll
    for (int k = 31; k >= 0; --k) {
      const double ri = rdi[o + k];
      const double xk = (k == lane) ? ri : (k < lane ? -acc[k] * ri : 0.0);
#pragma unroll
      for (int i = 0; i < 31; ++i)
        if (i < k) acc[i] += A[(o + i) * kLdA + o + k] * xk;
      __syncwarp();
      if (k <= lane) A[(o + k) * kLdA + o + lane] = xk;
      __syncwarp();
    }
  }
  __syncthreads();
  // off-diagonal blocks by block columns: X_ij = -(sum_{k=i..j-1} X_ik Rs_kj) X_jj, i < j.
  // A warp owns four rows r of T, lanes the 32 columns.
  for (int bj = 1; bj < nb; ++bj) {
    const int oj = bj * 32;
    for (int r0 = warp * 4; r0 < oj; r0 += 32) {
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
      for (int k = r0; k < oj; ++k) {
        const double rkc = A[k * kLdA + oj + lane];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (r0 + q <= k) acc[q] = fma(A[(r0 + q) * kLdA + k], rkc, acc[q]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) T[(r0 + q) * 32 + lane] = acc[q];
    }
    __syncthreads();
    for (int r0 = warp * 4; r0 < oj; r0 += 32) {
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
      for (int m = 0; m < 32; ++m) {
        const double xm = (m <= lane) ? A[(oj + m) * kLdA + oj + lane] : 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = fma(T[(r0 + q) * 32 + m], xm, acc[q]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) A[(r0 + q) * kLdA + oj + lane] = -acc[q];
    }
    __syncthreads();
  }
  // R^{-1} = D^-1/2 Rs^{-1}: three bf16 planes over the full kPanel x kPanel square
  double x2 = 0.0;
  for (int q = tid; q < kPanelSq / 4; q += 256) {
    const int r = q >> 5, c0 = (q & 31) * 4;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c0 + e;
      v[e] = 0.0f;
      if (r <= c && c < w) {
        const double xs = A[r * kLdA + c];
        x2 += xs * xs;
        v[e] = (float)(ds[r] * xs);
      }
    }
    store_split3x4(make_float4(v[0], v[1], v[2], v[3]), j.rinv, 4LL * q, kPanelSq);
  }
  if (j.first) {
    // the first pass is final unless it had to be shifted or Gs is poorly conditioned
    // (Cholesky-QR loses orthogonality in proportion to cond(Gs))
    x2 = warp_sum_d(x2);
    if (lane == 0) red_sh[warp] = x2;
    __syncthreads();
    if (tid == 0) {
      double tot2 = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) tot2 += red_sh[i];
      const int again = (shifted || tot2 > kAgainMeanInv * w) ? 1 : 0;
      const int fin = again | (j.reorth ? *j.reorth : 0);
      *j.again = again;
      *j.fin = fin;
      if (again && j.any_again) *j.any_again = 1;
      if (fin && j.any_fin) *j.any_fin = 1;
    }
  }
}

// Sum of the K-slice partials of a panel's projection coefficients C (rows x
// kPanel fp32 each, in slice order), written as three bf16 planes (ld kPanel).
// 1024 elements per block.
struct CoefJob {
  const float* part;      // nparts partials, part_stride elements apart (rows x ld each)
  __nv_bfloat16* cp;      // planes (plane stride pstride, ld ld)
  long long part_stride, pstride;
  const int* flag;
  int rows, ld, nparts;
  int blk_begin;
};

__global__ void __launch_bounds__(256) pc_coef_reduce_kernel(const CoefJob* __restrict__ J, int n,
                                                              const int* __restrict__ any) {
  if (any && *any == 0) return;  // no factor of the launch takes this projection
  const int lo = find_start(job_starts(J, n), n, (int)blockIdx.x);
  const CoefJob& j = J[lo];
  if (j.flag && *j.flag == 0) return;
  const long long e = ((long long)(blockIdx.x - j.blk_begin) * 256 + threadIdx.x) * 4;
  if (e >= (long long)j.rows * j.ld) return;
  float4 v[8];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = 0; p0 < j.nparts; p0 += 8) {
#pragma unroll
    for (int p = 0; p < 8; ++p)
      if (p0 + p < j.nparts) v[p] = *reinterpret_cast<const float4*>(j.part + (long long)(p0 + p) * j.part_stride + e);
#pragma unroll
    for (int p = 0; p < 8; ++p)
      if (p0 + p < j.nparts) {
        acc.x += v[p].x;
        acc.y += v[p].y;
        acc.z += v[p].z;
        acc.w += v[p].w;
      }
  }
  store_split3x4(acc, j.cp, e, j.pstride);
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
  const int lo = find_start(job_starts(J, cnt), cnt, (int)blockIdx.x);
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
// Adaptive refresh check.  With D = Q^T F Q and an orthogonal Q, ||D||_F = ||F||_F =
// ||F Q||_F and diag(D)_i = q_i^T F q_i, so
//   rho^2 = ||D - diag(D)||_F^2 / ||D||_F^2 = 1 - sum_i diag(D)_i^2 / ||P||_F^2,  P = F Q,
// from the power product the refresh needs anyway (same value as forming D, up to
// rounding).  One block per factor; sums in a fixed order.
struct CheckJob {
  const double* dg;   // diag(D) (k)
  const float* pn;    // squared column norms of P (k)
  int* flag;
  float* rho;
  int k;
};

__global__ void __launch_bounds__(256) pc_check_kernel(const CheckJob* __restrict__ J, float tol) {
  __shared__ double red[2][256];
  const CheckJob& j = J[blockIdx.x];
  double d2 = 0.0, p2 = 0.0;
  for (int i = threadIdx.x; i < j.k; i += 256) {
    const double d = j.dg[i];
    d2 += d * d;
    p2 += (double)j.pn[i];
  }
  red[0][threadIdx.x] = d2;
  red[1][threadIdx.x] = p2;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      red[0][threadIdx.x] += red[0][threadIdx.x + o];
      red[1][threadIdx.x] += red[1][threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double r2 = red[1][0] > 0.0 ? 1.0 - red[0][0] / red[1][0] : 0.0;
    const double rho = r2 > 0.0 ? sqrt(r2) : 0.0;  // NaN input: no refresh
    *j.rho = (float)rho;
    *j.flag = (rho > (double)tol) ? 1 : 0;
  }
}

// Per-matrix diagnostics of a SOAP / FOAM step: refresh bits, the check ratio and
// the update statistics.  fixed_bits >= 0: the refresh was decided on the host
// (bits given); otherwise read the device flags (bit 0 right side, bit 1 left side).
// upd holds the update product's per-block partials (sum of squared weight
// changes, non-finite count), nslots of them; they are summed in a fixed order.
struct StatsJob {
  const int* flag_r;
  const int* flag_l;
  const float* rho;
  const float2* upd;
  int nslots;
  int fixed_bits;
  int index;  // position in the caller's stats array
  int m, n;
};

// One block of 256 threads per matrix.  A non-finite weight is also recorded in the
// workspace status word as MAO_ERR_NONFINITE (site 31), unless an error came first.
__global__ void __launch_bounds__(256) pc_stats_kernel(const StatsJob* __restrict__ J, mao_stats* __restrict__ stats,
                                                       DevStatus* status) {
  __shared__ double red[2][256];
  const StatsJob& j = J[blockIdx.x];
  double ss = 0.0, nf = 0.0;
  for (int i = threadIdx.x; i < j.nslots; i += 256) {
    const float2 v = j.upd[i];
    ss += (double)v.x;
    nf += (double)v.y;
  }
  red[0][threadIdx.x] = ss;
  red[1][threadIdx.x] = nf;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      red[0][threadIdx.x] += red[0][threadIdx.x + o];
      red[1][threadIdx.x] += red[1][threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x != 0) return;
  int bits = j.fixed_bits;
  if (bits < 0) bits = ((j.flag_r && *j.flag_r) ? 1 : 0) | ((j.flag_l && *j.flag_l) ? 2 : 0);
  const int bad = (int)red[1][0];
  mao_stats& st = stats[j.index];
  st.update_rms = (float)sqrt(red[0][0] / ((double)j.m * (double)j.n));
  st.offdiag_ratio = j.rho ? *j.rho : -1.0f;
  st.refreshed = bits;
  st.nonfinite = bad;
  if (bad > 0) report(status, MAO_ERR_NONFINITE, 31, j.index, bad);
}

}  // namespace mao
