// mao_muon_step: one Muon / Muon+ step over a batch of matrices.
//
// Launch sequence on the caller's stream (no host synchronisation):
//   1. muon_prep_kernel      momentum EMA, sum-of-squares partials, bf16 X (s x l)
//   2. muon_scale_kernel     per-matrix 1/(||M||_F + eps)
//   3. ns_steps x 3 grouped tcgen05 GEMMs over every shape class at once:
//        A = s^2 X X^T            (EPI_GRAM; both operands X, K-major)
//        B = b A + c A A          (EPI_POLY; A is symmetric, so A A = A A^T, K-major)
//        X' = s (a X + B X)       (EPI_AXPY_T; B K-major, X read MN-major)
//      Iteration 0 works on the unnormalised bf16(M) and applies the per-matrix
//      scale s in the epilogues, which equals normalising first:
//        s^2 X X^T = (sX)(sX)^T and s (a X + B X) = a (sX) + B (sX).
//   4. Muon+ row/column scales (optional), 64 x 64 tile passes
//   5. muon_update_kernel    W <- W (1 - lr wd) - lr sqrt(m/n) Norm(O)
//   6. muon_stats_kernel     (optional)
#include <algorithm>
#include <cmath>
#include <map>

#include "host_common.h"
#include "muon_kernels.cuh"

namespace mao {

namespace {

constexpr float kDefaultCoef[3] = {3.4445f, -4.7750f, 2.0315f};
constexpr int kMaxNsSteps = 16;

// The exact polar factor (MOP): a fixed Newton-Schulz schedule run in fp32-faithful
// arithmetic that converges to U V^T.  kMopGrow quintic steps with the default
// coefficients lift every singular value of X0 = M / (||M||_F + eps) that is at least
// ~2e-7 into [0.23, 1.21] (each multiplies a small singular value by 3.4445); kMopConv
// steps of x -> (15 x - 10 x^3 + 3 x^5) / 8, whose fixed point 1 has zero first and
// second derivatives (cubic convergence), then take all of them to 1 to fp32 rounding.
constexpr int kMopGrow = 11, kMopConv = 5, kMopSteps = kMopGrow + kMopConv;
constexpr float kMopConvCoef[3] = {15.0f / 8.0f, -10.0f / 8.0f, 3.0f / 8.0f};

struct MuonClass {
  int s = 0, l = 0;           // X is s x l
  std::vector<int> mats;      // global matrix indices, in batch order
  int ld_l = 0, ld_s = 0;     // padded leading dimensions (multiples of 8)
  size_t off_X[2] = {}, off_A = 0, off_B = 0;
  int scale_begin = 0;        // first slot in the scale array
};

// Per logical matrix buffers of the exact polar factor.
struct ExactBuf {
  size_t Xf[2], Xp[2];  // fp32 X (s x ld_l) and its three bf16 planes, ping-pong
  size_t Af, Ap, Bp;    // fp32 A = X X^T (s x ld_s) and its planes; planes of B
};

struct MuonPlan {
  std::vector<MuonClass> cls;
  bool exact = false;
  std::vector<ExactBuf> ex;
  size_t off_arena = 0, arena_cap = 0;  // staged problem tables and tensor maps (exact)
  std::vector<int> mat_class, mat_slot;  // class of matrix p, its index in the class
  size_t off_table = 0, off_scale = 0, off_partial = 0, off_rowscale = 0, off_colscale = 0, off_rowpart = 0,
         off_colpart = 0, off_updpart = 0, off_updbad = 0, off_ranges = 0;
  int tiles = 0;
  size_t total = 0;
  bool use_rows = false, use_cols = false;
  std::vector<MuonMatDev> table;  // filled without device pointers by plan()
};

bool norm_uses_rows(int mode) { return mode == MAO_NORM_ROW || mode == MAO_NORM_COL_ROW || mode == MAO_NORM_ROW_COL; }
bool norm_uses_cols(int mode) { return mode == MAO_NORM_COL || mode == MAO_NORM_COL_ROW || mode == MAO_NORM_ROW_COL; }

mao_status validate(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p, bool check_ptrs) {
  if (p == nullptr || count < 0 || (count > 0 && mats == nullptr)) return MAO_ERR_INVALID_ARG;
  if (p->ns_steps < 0 || p->ns_steps > kMaxNsSteps) return MAO_ERR_INVALID_ARG;
  if (p->norm < MAO_NORM_NONE || p->norm > MAO_NORM_ROW_COL) return MAO_ERR_INVALID_ARG;
  if (!std::isfinite(p->mu) || !std::isfinite(p->lr) || !std::isfinite(p->wd) || !std::isfinite(p->eps) ||
      p->eps < 0.0f)
    return MAO_ERR_INVALID_ARG;
  if (p->ns_coef != nullptr)
    for (int i = 0; i < 3 * p->ns_steps; ++i)
      if (!std::isfinite(p->ns_coef[i])) return MAO_ERR_INVALID_ARG;
  if (p->polar != MAO_POLAR_NS && p->polar != MAO_POLAR_EXACT) return MAO_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const mao_muon_mat& a = mats[i];
    if (a.m < 1 || a.n < 1) return MAO_ERR_SHAPE;
    if ((long long)a.m * a.n > (1ll << 31) - 1) return MAO_ERR_SHAPE;
    if (a.g_dtype != MAO_F32 && a.g_dtype != MAO_BF16) return MAO_ERR_DTYPE;
    if (a.split_rows < 0 || a.split_cols < 0) return MAO_ERR_INVALID_ARG;
    const int sr = std::max(a.split_rows, 1), sc = std::max(a.split_cols, 1);
    if (a.m % sr != 0 || a.n % sc != 0) return MAO_ERR_SHAPE;
    const int nb = a.n / sc;
    if (nb % 4 != 0) return MAO_ERR_SHAPE;
    if (a.g_dtype == MAO_BF16 && nb % 8 != 0) return MAO_ERR_SHAPE;
    if (check_ptrs) {
      if (a.W == nullptr || a.G == nullptr || a.M == nullptr) return MAO_ERR_INVALID_ARG;
      if (!aligned16(a.W) || !aligned16(a.G) || !aligned16(a.M)) return MAO_ERR_ALIGN;
    }
  }
  return MAO_OK;
}

// The logical matrices of a call: each caller matrix, or each block of a split one
// (row-major block order, consecutive), with its leading dimension and owner.
struct Logical {
  std::vector<mao_muon_mat> mats;
  std::vector<int> ld, owner;
};

void expand(const mao_muon_mat* mats, int count, Logical& L) {
  L = Logical();
  for (int i = 0; i < count; ++i) {
    const mao_muon_mat& a = mats[i];
    const int sr = std::max(a.split_rows, 1), sc = std::max(a.split_cols, 1);
    const int mb = a.m / sr, nb = a.n / sc;
    const size_t ge = a.g_dtype == MAO_BF16 ? 2 : 4;
    for (int r = 0; r < sr; ++r)
      for (int c = 0; c < sc; ++c) {
        const size_t off = (size_t)r * mb * a.n + (size_t)c * nb;
        mao_muon_mat b = a;
        b.m = mb;
        b.n = nb;
        b.split_rows = b.split_cols = 1;
        b.W = a.W ? a.W + off : nullptr;
        b.M = a.M ? a.M + off : nullptr;
        b.G = a.G ? static_cast<const void*>(static_cast<const uint8_t*>(a.G) + off * ge) : nullptr;
        L.mats.push_back(b);
        L.ld.push_back(a.n);
        L.owner.push_back(i);
      }
  }
}

void plan(const mao_muon_mat* mats, int count, const int* ld, int callers, const mao_muon_params* p, MuonPlan& P) {
  P = MuonPlan();
  P.use_rows = norm_uses_rows(p->norm);
  P.use_cols = norm_uses_cols(p->norm);
  std::map<std::pair<int, int>, int> idx;
  P.mat_class.resize(count);
  P.mat_slot.resize(count);
  for (int i = 0; i < count; ++i) {
    const int s = std::min(mats[i].m, mats[i].n), l = std::max(mats[i].m, mats[i].n);
    auto key = std::make_pair(s, l);
    auto it = idx.find(key);
    if (it == idx.end()) {
      it = idx.emplace(key, (int)P.cls.size()).first;
      MuonClass c;
      c.s = s;
      c.l = l;
      c.ld_l = round_up_int(l, 8);
      c.ld_s = round_up_int(s, 8);
      P.cls.push_back(c);
    }
    P.mat_class[i] = it->second;
    P.mat_slot[i] = (int)P.cls[it->second].mats.size();
    P.cls[it->second].mats.push_back(i);
  }
  Carver cv;
  cv.take(kStatusBytes);
  // the table, then the compact first-tile array that find_mat searches
  P.off_table = cv.take((sizeof(MuonMatDev) + sizeof(int)) * (size_t)std::max(count, 1));
  P.off_scale = cv.take(sizeof(float) * (size_t)std::max(count, 1));
  int sb = 0;
  for (auto& c : P.cls) {
    c.scale_begin = sb;
    sb += (int)c.mats.size();
  }
  P.table.assign(count, MuonMatDev());
  int tiles = 0;
  size_t rs_elems = 0, cs_elems = 0, rp_elems = 0, cp_elems = 0;
  for (int i = 0; i < count; ++i) {
    MuonMatDev& D = P.table[i];
    D.m = mats[i].m;
    D.n = mats[i].n;
    D.ld = ld[i];
    D.g_bf16 = mats[i].g_dtype == MAO_BF16;
    D.trans = D.m > D.n ? 1 : 0;
    D.ldx = round_up_int(std::max(D.m, D.n), 8);
    D.tiles_r = (D.m + kTile - 1) / kTile;
    D.tiles_c = (D.n + kTile - 1) / kTile;
    D.tile_begin = tiles;
    tiles += D.tiles_r * D.tiles_c;
    D.out_scale = p->lr * std::sqrt((float)D.m / (float)D.n);
    rs_elems += D.m;
    cs_elems += D.n;
    rp_elems += (size_t)D.tiles_c * D.m;
    cp_elems += (size_t)D.tiles_r * D.n;
  }
  P.tiles = tiles;
  P.off_partial = cv.take(sizeof(float) * (size_t)std::max(tiles, 1));
  if (P.use_rows) {
    P.off_rowscale = cv.take(sizeof(float) * rs_elems);
    P.off_rowpart = cv.take(sizeof(float) * rp_elems);
  }
  if (P.use_cols) {
    P.off_colscale = cv.take(sizeof(float) * cs_elems);
    P.off_colpart = cv.take(sizeof(float) * cp_elems);
  }
  P.off_updpart = cv.take(sizeof(float) * (size_t)std::max(tiles, 1));
  P.off_updbad = cv.take(sizeof(int) * (size_t)std::max(tiles, 1));
  P.off_ranges = cv.take(sizeof(MuonStatsRange) * (size_t)std::max(callers, 1));
  for (auto& c : P.cls) {
    const size_t cnt = c.mats.size();
    for (int k = 0; k < 2; ++k) c.off_X[k] = cv.take(2 * cnt * (size_t)c.s * c.ld_l);
    c.off_A = cv.take(2 * cnt * (size_t)c.s * c.ld_s);
    c.off_B = cv.take(2 * cnt * (size_t)c.s * c.ld_s);
  }
  P.exact = p->polar == MAO_POLAR_EXACT;
  if (P.exact) {
    P.ex.assign(count, ExactBuf());
    for (int i = 0; i < count; ++i) {
      const MuonClass& C = P.cls[P.mat_class[i]];
      ExactBuf& e = P.ex[i];
      for (int k = 0; k < 2; ++k) {
        e.Xf[k] = cv.take(4 * (size_t)C.s * C.ld_l);
        e.Xp[k] = cv.take(2 * 3 * (size_t)C.s * C.ld_l);
      }
      e.Af = cv.take(4 * (size_t)C.s * C.ld_s);
      e.Ap = cv.take(2 * 3 * (size_t)C.s * C.ld_s);
      e.Bp = cv.take(2 * 3 * (size_t)C.s * C.ld_s);
    }
    // at most 27 tensor maps per matrix (3 planes of X[2] in three views, of A in two,
    // of B in one) and one problem per matrix in each of 3 launches per iteration
    P.arena_cap =
        (size_t)count * (27 * sizeof(CUtensorMap) + 3 * kMopSteps * (sizeof(GemmProblem) + 2 * sizeof(int))) +
        (3 * kMopSteps + 1) * 64 + 4096;
    P.off_arena = cv.take(P.arena_cap);
  }
  P.total = cv.total();
}

// The fp32-faithful Newton-Schulz iteration of the exact polar factor, for every
// logical matrix: per iteration A = X X^T, B = b A + c A A^T, X' = a X + B X as
// table-mode products (the same arithmetic as the SOAP / FOAM contractions), with
// the problem tables and tensor maps staged in the workspace's arena.
mao_status run_exact_iterations(const MuonPlan& P, uint8_t* ws, DevStatus* status, cudaStream_t stream) {
  const int count = (int)P.ex.size();
  MapSet maps;
  std::vector<TableLaunch> launches;
  launches.reserve(3 * kMopSteps);
  auto planes = [&](size_t off, int rows, int cols, int ld) {
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(ws + off);
    const size_t st = (size_t)rows * ld;
    return Split3{{b, b + st, b + 2 * st}, rows, cols, ld};
  };
  for (int it = 0; it < kMopSteps; ++it) {
    const float* cf = it < kMopGrow ? kDefaultCoef : kMopConvCoef;
    const int cur = it % 2, nxt = 1 - cur;
    launches.emplace_back();
    TableLaunch& g = launches.back();
    g.kernel_id = MAO_K_NS_GRAM;
    launches.emplace_back();
    TableLaunch& q = launches.back();
    q.kernel_id = MAO_K_NS_POLY;
    launches.emplace_back();
    TableLaunch& x = launches.back();
    x.kernel_id = MAO_K_NS_AXPY;
    x.b_mn = 1;
    for (int i = 0; i < count; ++i) {
      const MuonClass& C = P.cls[P.mat_class[i]];
      const ExactBuf& e = P.ex[i];
      const Split3 Xc = planes(e.Xp[cur], C.s, C.l, C.ld_l), Xn = planes(e.Xp[nxt], C.s, C.l, C.ld_l);
      const Split3 Ap = planes(e.Ap, C.s, C.s, C.ld_s), Bp = planes(e.Bp, C.s, C.s, C.ld_s);
      float* Af = reinterpret_cast<float*>(ws + e.Af);
      float* Xfc = reinterpret_cast<float*>(ws + e.Xf[cur]);
      float* Xfn = reinterpret_cast<float*>(ws + e.Xf[nxt]);
      // A = X X^T (s x s)
      MAO_TRY(table_add(g, maps, Xc, Xc, C.s, C.s, C.l, 0, 0, Af, &Ap, C.ld_s, nullptr, 0, 1.f, 0.f, nullptr));
      // B = c A A^T + b A (A is symmetric)
      MAO_TRY(table_add(q, maps, Ap, Ap, C.s, C.s, C.s, 0, 0, nullptr, &Bp, C.ld_s, Af, C.ld_s, cf[2], cf[1],
                        nullptr));
      // X' = B X + a X (X read as K x N, MN-major)
      MAO_TRY(table_add(x, maps, Bp, Xc, C.s, C.l, C.s, 0, 0, Xfn, &Xn, C.ld_l, Xfc, C.ld_l, 1.f, cf[0],
                        nullptr));
    }
  }
  MAO_TRY(maps.encode_all());
  Arena arena;
  arena.dev = ws + P.off_arena;
  const size_t maps_off = arena.take(sizeof(CUtensorMap) * maps.maps.size(), 64);
  std::memcpy(arena.host.data() + maps_off, maps.maps.data(), sizeof(CUtensorMap) * maps.maps.size());
  std::vector<StagedLaunch> staged;
  for (const TableLaunch& L : launches) staged.push_back(table_stage(arena, L, maps_off));
  if (arena.host.size() > P.arena_cap) return MAO_ERR_WORKSPACE;  // the bound above is wrong: a defect
  MAO_CUDA_TRY(cudaMemcpyAsync(arena.dev, arena.host.data(), arena.host.size(), cudaMemcpyHostToDevice, stream));
  for (const StagedLaunch& S : staged) MAO_TRY(table_launch(arena, S, status, stream));
  return MAO_OK;
}

}  // namespace

}  // namespace mao

using namespace mao;

extern "C" mao_status mao_muon_workspace_size(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p,
                                              size_t* bytes) {
  if (bytes == nullptr) return MAO_ERR_INVALID_ARG;
  MAO_TRY(validate(mats, count, p, false));
  Logical L;
  expand(mats, count, L);
  MuonPlan P;
  plan(L.mats.data(), (int)L.mats.size(), L.ld.data(), count, p, P);
  *bytes = P.total;
  return MAO_OK;
}

extern "C" mao_status mao_muon_step(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p,
                                   void* workspace, size_t ws_bytes, mao_stats* stats, mao_stream_t stream_) {
  const mao_muon_mat* const mats_in = mats;
  MAO_TRY(validate(mats, count, p, true));
  if (count == 0) return MAO_OK;
  // from here on, work on the logical matrices (the blocks of split matrices)
  Logical L;
  expand(mats, count, L);
  const int callers = count;
  mats = L.mats.data();
  count = (int)L.mats.size();
  MuonPlan P;
  plan(mats, count, L.ld.data(), callers, p, P);
  if (workspace == nullptr || ws_bytes < P.total) return MAO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MAO_ERR_ALIGN;
  if (stats != nullptr && !aligned16(stats)) return MAO_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  MAO_TRY(device_info(&dev));
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  float* scale = reinterpret_cast<float*>(ws + P.off_scale);
  float* partial = reinterpret_cast<float*>(ws + P.off_partial);
  float* rowscale = P.use_rows ? reinterpret_cast<float*>(ws + P.off_rowscale) : nullptr;
  float* rowpart = P.use_rows ? reinterpret_cast<float*>(ws + P.off_rowpart) : nullptr;
  float* colscale = P.use_cols ? reinterpret_cast<float*>(ws + P.off_colscale) : nullptr;
  float* colpart = P.use_cols ? reinterpret_cast<float*>(ws + P.off_colpart) : nullptr;
  float* updpart = reinterpret_cast<float*>(ws + P.off_updpart);
  int* updbad = reinterpret_cast<int*>(ws + P.off_updbad);
  const int fin = p->ns_steps % 2;

  // device table
  size_t rs_off = 0, cs_off = 0, rp_off = 0, cp_off = 0;
  for (int i = 0; i < count; ++i) {
    MuonMatDev& D = P.table[i];
    const MuonClass& C = P.cls[P.mat_class[i]];
    const int b = P.mat_slot[i];
    D.W = mats[i].W;
    D.G = mats[i].G;
    D.M = mats[i].M;
    D.X0 = reinterpret_cast<__nv_bfloat16*>(ws + C.off_X[0]) + (size_t)b * C.s * C.ld_l;
    D.O = reinterpret_cast<__nv_bfloat16*>(ws + C.off_X[fin]) + (size_t)b * C.s * C.ld_l;
    D.rowscale = rowscale ? rowscale + rs_off : nullptr;
    D.rowpart = rowpart ? rowpart + rp_off : nullptr;
    D.colscale = colscale ? colscale + cs_off : nullptr;
    D.colpart = colpart ? colpart + cp_off : nullptr;
    D.oscale = (p->ns_steps == 0 && !P.exact) ? scale + C.scale_begin + b : nullptr;
    D.scale_slot = C.scale_begin + b;
    if (P.exact) {
      const ExactBuf& e = P.ex[i];
      D.Xe = reinterpret_cast<float*>(ws + e.Xf[0]);
      D.Xep = reinterpret_cast<__nv_bfloat16*>(ws + e.Xp[0]);
      D.xep_stride = (long long)C.s * C.ld_l;
      D.Of = reinterpret_cast<const float*>(ws + e.Xf[kMopSteps % 2]);
    }
    rs_off += D.m;
    cs_off += D.n;
    rp_off += (size_t)D.tiles_c * D.m;
    cp_off += (size_t)D.tiles_r * D.n;
  }
  MAO_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream));
  std::vector<uint8_t> image((sizeof(MuonMatDev) + sizeof(int)) * count);
  std::memcpy(image.data(), P.table.data(), sizeof(MuonMatDev) * count);
  int* starts = reinterpret_cast<int*>(image.data() + sizeof(MuonMatDev) * count);
  for (int i = 0; i < count; ++i) starts[i] = P.table[i].tile_begin;
  MAO_CUDA_TRY(cudaMemcpyAsync(ws + P.off_table, image.data(), image.size(), cudaMemcpyHostToDevice, stream));
  const MuonMatDev* T = reinterpret_cast<const MuonMatDev*>(ws + P.off_table);

  // algorithmic bytes of the elementwise passes
  double elems = 0.0, g_bytes = 0.0;
  int maxdim = 0;
  for (int i = 0; i < count; ++i) {
    const double e = (double)mats[i].m * mats[i].n;
    elems += e;
    g_bytes += e * (mats[i].g_dtype == MAO_BF16 ? 2.0 : 4.0);
    maxdim = std::max(maxdim, std::max(mats[i].m, mats[i].n));
  }

  // 1-2: momentum, partial norms, bf16 operand, per-matrix scale
  {
    LaunchScope ls(stream, MAO_K_MUON_PREP, 0.0, g_bytes + elems * (4.0 + 4.0 + 2.0));
    muon_prep_kernel<<<P.tiles, 256, 0, stream>>>(T, count, p->mu, partial);
  }
  MAO_CUDA_TRY(cudaGetLastError());
  {
    LaunchScope ls(stream, MAO_K_MUON_SCALE, 0.0, 4.0 * P.tiles);
    muon_scale_kernel<<<(count + 7) / 8, 256, 0, stream>>>(T, count, partial, p->eps, scale);
  }
  MAO_CUDA_TRY(cudaGetLastError());

  // 3 (exact polar factor): fp32 X0 and its planes, then the fp32-faithful iteration
  if (P.exact) {
    {
      LaunchScope ls(stream, MAO_K_MOP_INIT, 0.0, elems * (4.0 + 4.0 + 6.0));
      mop_init_kernel<<<P.tiles, 256, 0, stream>>>(T, count, scale);
    }
    MAO_CUDA_TRY(cudaGetLastError());
    MAO_TRY(run_exact_iterations(P, ws, status, stream));
  }
  // 3: Newton-Schulz over every class, at most kMaxClasses per launch
  if (p->ns_steps > 0 && !P.exact) {
    const int ncls = (int)P.cls.size();
    struct ClassMaps {
      CUtensorMap XA[2], XB[2], XMN[2], AA, AB, BA;
    };
    std::vector<ClassMaps> maps(ncls);
    for (int c = 0; c < ncls; ++c) {
      const MuonClass& C = P.cls[c];
      const uint64_t cnt = C.mats.size();
      for (int k = 0; k < 2; ++k) {
        OperandView xv{ws + C.off_X[k], (uint64_t)C.l, (uint64_t)C.s, cnt, (uint64_t)C.ld_l,
                       (uint64_t)C.s * C.ld_l};
        MAO_TRY(encode_operand(&maps[c].XA[k], OP_BF16, 0, 128, xv));
        MAO_TRY(encode_operand(&maps[c].XB[k], OP_BF16, 0, 128, xv));  // B boxes: 128 rows (a pair CTA's half)
        MAO_TRY(encode_operand(&maps[c].XMN[k], OP_BF16, 1, 256, xv));  // X as K x N (K = s rows)
      }
      OperandView av{ws + C.off_A, (uint64_t)C.s, (uint64_t)C.s, cnt, (uint64_t)C.ld_s, (uint64_t)C.s * C.ld_s};
      MAO_TRY(encode_operand(&maps[c].AA, OP_BF16, 0, 128, av));
      MAO_TRY(encode_operand(&maps[c].AB, OP_BF16, 0, 128, av));
      OperandView bv{ws + C.off_B, (uint64_t)C.s, (uint64_t)C.s, cnt, (uint64_t)C.ld_s, (uint64_t)C.s * C.ld_s};
      MAO_TRY(encode_operand(&maps[c].BA, OP_BF16, 0, 128, bv));
    }
    for (int it = 0; it < p->ns_steps; ++it) {
      const float* cf = p->ns_coef ? p->ns_coef + 3 * it : kDefaultCoef;
      const int cur = it % 2, nxt = (it + 1) % 2;
      for (int g0 = 0; g0 < ncls; g0 += kMaxClasses) {
        const int g1 = std::min(ncls, g0 + kMaxClasses);
        GemmParams g1p, g2p, g3p;
        std::memset(&g1p, 0, sizeof(g1p));
        std::memset(&g2p, 0, sizeof(g2p));
        std::memset(&g3p, 0, sizeof(g3p));
        g1p.nclasses = g2p.nclasses = g3p.nclasses = g1 - g0;
        g1p.status = g2p.status = g3p.status = status;
        g2p.beta = cf[1];
        g2p.gamma = cf[2];
        g3p.alpha = cf[0];
        for (int c = g0; c < g1; ++c) {
          const MuonClass& C = P.cls[c];
          const int k = c - g0;
          const int cnt = (int)C.mats.size();
          const long long xs = (long long)C.s * C.ld_l, as = (long long)C.s * C.ld_s;
          const float* sc = (it == 0) ? scale + C.scale_begin : nullptr;
          // A = s^2 X X^T
          g1p.mapA[k] = maps[c].XA[cur];
          g1p.mapB[k] = maps[c].XB[cur];
          g1p.cls[k] = GemmClass{C.s, C.s, C.l, cnt, 0, 0, 0, ws + C.off_A, as, C.ld_s, nullptr, 0, 0,
                                 nullptr, 0, 0, sc};
          // B = b A + c A A^T
          g2p.mapA[k] = maps[c].AA;
          g2p.mapB[k] = maps[c].AB;
          g2p.cls[k] = GemmClass{C.s, C.s, C.s, cnt, 0, 0, 0, ws + C.off_B, as, C.ld_s, nullptr, 0, 0,
                                 ws + C.off_A, as, C.ld_s, nullptr};
          // X' = s (a X + B X)
          g3p.mapA[k] = maps[c].BA;
          g3p.mapB[k] = maps[c].XMN[cur];
          g3p.cls[k] = GemmClass{C.s, C.l, C.s, cnt, 0, 0, 0, ws + C.off_X[nxt], xs, C.ld_l, nullptr, 0, 0,
                                 ws + C.off_X[cur], xs, C.ld_l, sc};
        }
        finalize_classes(g1p);
        finalize_classes(g2p);
        finalize_classes(g3p);
        MAO_TRY(launch_gemm(OP_BF16, 0, 0, EPI_GRAM, g1p, stream, MAO_K_NS_GRAM));
        MAO_TRY(launch_gemm(OP_BF16, 0, 0, EPI_POLY, g2p, stream, MAO_K_NS_POLY));
        MAO_TRY(launch_gemm(OP_BF16, 0, 1, EPI_AXPY_T, g3p, stream, MAO_K_NS_AXPY));
      }
    }
  }

  // 4: Muon+ scales (each direction: tile partials, then a fixed-order final sum)
  auto norm_pass = [&](int rows_dir, int use_other) -> mao_status {
    {
      LaunchScope ls(stream, rows_dir ? MAO_K_MUON_ROWSCALE : MAO_K_MUON_COLSQ, 0.0, 2.0 * elems);
      const int wc = rows_dir ? 0 : 1, wr = rows_dir ? 1 : 0;
      const int ur = (!rows_dir && use_other) ? 1 : 0, uc = (rows_dir && use_other) ? 1 : 0;
      if (P.exact)
        muon_norm_tile_kernel<float><<<P.tiles, 256, 0, stream>>>(T, count, wc, wr, ur, uc);
      else
        muon_norm_tile_kernel<__nv_bfloat16><<<P.tiles, 256, 0, stream>>>(T, count, wc, wr, ur, uc);
    }
    MAO_CUDA_TRY(cudaGetLastError());
    dim3 g((maxdim + 255) / 256, count);
    {
      LaunchScope ls(stream, MAO_K_MUON_COLSCALE, 0.0, 0.0);
      muon_norm_final_kernel<<<g, 256, 0, stream>>>(T, count, rows_dir ? 0 : 1);
    }
    MAO_CUDA_TRY(cudaGetLastError());
    return MAO_OK;
  };
  const int mode = p->norm;
  if (mode == MAO_NORM_COL) {
    MAO_TRY(norm_pass(0, 0));
  } else if (mode == MAO_NORM_ROW) {
    MAO_TRY(norm_pass(1, 0));
  } else if (mode == MAO_NORM_COL_ROW) {
    MAO_TRY(norm_pass(0, 0));
    MAO_TRY(norm_pass(1, 1));
  } else if (mode == MAO_NORM_ROW_COL) {
    MAO_TRY(norm_pass(1, 0));
    MAO_TRY(norm_pass(0, 1));
  }

  // 5-6: update and stats
  const float decay = 1.0f - p->lr * p->wd;
  {
    LaunchScope ls(stream, MAO_K_MUON_UPDATE, 0.0, elems * (2.0 + 4.0 + 4.0));
    float* up = stats ? updpart : nullptr;
    int* ub = stats ? updbad : nullptr;
    if (P.exact)
      muon_update_kernel<float><<<P.tiles, 256, 0, stream>>>(T, count, decay, P.use_rows ? 1 : 0,
                                                            P.use_cols ? 1 : 0, up, ub);
    else
      muon_update_kernel<__nv_bfloat16><<<P.tiles, 256, 0, stream>>>(T, count, decay, P.use_rows ? 1 : 0,
                                                                    P.use_cols ? 1 : 0, up, ub);
  }
  MAO_CUDA_TRY(cudaGetLastError());
  if (stats) {
    std::vector<MuonStatsRange> ranges(callers);
    for (int c = 0; c < callers; ++c) ranges[c] = MuonStatsRange{0, 0, mats_in[c].m, mats_in[c].n};
    for (int i = count - 1; i >= 0; --i) {  // blocks of one caller are consecutive
      MuonStatsRange& r = ranges[L.owner[i]];
      r.tile_begin = P.table[i].tile_begin;
      r.tiles += P.table[i].tiles_r * P.table[i].tiles_c;
    }
    MAO_CUDA_TRY(cudaMemcpyAsync(ws + P.off_ranges, ranges.data(), sizeof(MuonStatsRange) * callers,
                                 cudaMemcpyHostToDevice, stream));
    {
      LaunchScope ls(stream, MAO_K_MUON_STATS, 0.0, 8.0 * P.tiles);
      muon_stats_kernel<<<(callers + 7) / 8, 256, 0, stream>>>(
          reinterpret_cast<const MuonStatsRange*>(ws + P.off_ranges), callers, updpart, updbad, stats, status);
    }
    MAO_CUDA_TRY(cudaGetLastError());
  }
  (void)dev;
  return MAO_OK;
}
