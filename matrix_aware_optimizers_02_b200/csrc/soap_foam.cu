// mao_soap_step / mao_foam_step: one SOAP or FOAM step over a batch of matrices.
//
// Matrices are processed in groups whose scratch fits a fixed budget; each group
// runs the whole step with every phase batched over the group's matrices:
//
//   momentum      M <- b1 M + (1-b1) G; three-plane bf16 splits of G and M
//   factor EMAs   L <- b2 L + (1-b2) G G^T (SOAP), R <- b2 R + (1-b2) G^T G
//                 (fp32-faithful SPLIT3 tensor-core GEMMs with the EMA in the epilogue)
//   refresh       per side, when the policy says so: [adaptive check D = Q^T F Q,
//                 rho, flag] -> P = F Q -> keys diag(Q^T F Q) in fp64 -> stable
//                 descending argsort -> gathered P -> QR (block Gram-Schmidt by
//                 256-column super-panels, 128-column panels orthonormalised by
//                 Cholesky-QR with an fp64 factorisation; second passes and
//                 re-orthogonalisation decided on the device) -> Q.  Every refresh
//                 kernel reads a per-matrix device flag, so adaptive refreshes need
//                 no host sync.
//   SOAP          Gh, Mh = Q_L^T {G, M} Q_R ; Adam in the eigenbasis (V follows the
//                 permutations) ; U = Q_L N Q_R^T fused with W <- W(1 - lr wd) - lr U
//   FOAM          Gr, Mr = {G, M} Q_R ; r, c EMAs of row/column means of Gr^2 ; tau ;
//                 N = (Mr/bc1)/(sqrt(tau r c^T)+eps) ; U = N Q_R^T fused with the W update
#include <algorithm>
#include <cmath>
#include <list>
#include <memory>
#include <string>

#include "host_common.h"
#include "precond_kernels.cuh"

using namespace mao;

namespace {

constexpr size_t kGroupBudget = (size_t)48 << 30;  // scratch bytes per group of matrices
constexpr int kCoefSplitMinK = 4096;  // factors at least this large may split their projection products over K
constexpr int kMaxCoefParts = 8;

mao_status check_refresh(const mao_refresh& r) {
  if (r.kind < MAO_REFRESH_EVERY_K || r.kind > MAO_REFRESH_NEVER) return MAO_ERR_INVALID_ARG;
  if (r.kind == MAO_REFRESH_EVERY_K && r.k < 1) return MAO_ERR_INVALID_ARG;
  if (r.kind == MAO_REFRESH_ADAPTIVE && (r.pf < 1 || !std::isfinite(r.tol))) return MAO_ERR_INVALID_ARG;
  if (r.sort != 0 && r.sort != 1) return MAO_ERR_INVALID_ARG;
  if (r.lag != 0 && r.lag != 1) return MAO_ERR_INVALID_ARG;
  return MAO_OK;
}

mao_status check_hyper(float b1, float b2, float eps, float lr, float wd, int64_t t) {
  if (!std::isfinite(b1) || !std::isfinite(b2) || !std::isfinite(eps) || !std::isfinite(lr) || !std::isfinite(wd))
    return MAO_ERR_INVALID_ARG;
  if (b1 < 0.f || b1 >= 1.f || b2 < 0.f || b2 >= 1.f || eps < 0.f || t < 1) return MAO_ERR_INVALID_ARG;
  return MAO_OK;
}

mao_status check_mat(int m, int n, int g_dtype) {
  if (m < 1 || n < 1) return MAO_ERR_SHAPE;
  if ((long long)m * n > (1ll << 31) - 1 || (long long)m * m > (1ll << 31) - 1 || (long long)n * n > (1ll << 31) - 1)
    return MAO_ERR_SHAPE;
  if (g_dtype != MAO_F32 && g_dtype != MAO_BF16) return MAO_ERR_DTYPE;
  if (m % 4 || n % 4) return MAO_ERR_SHAPE;
  if (g_dtype == MAO_BF16 && n % 8) return MAO_ERR_SHAPE;
  return MAO_OK;
}

// Unified per-matrix view.
struct PcMat {
  int m, n;
  float* W;
  const void* G;
  int g_bf16;
  float* M;
  float* V;             // SOAP
  float *L, *R, *QL, *QR;
  int *perm_L, *perm_R;
  float *r, *c;         // FOAM
};

// Refresh decision known on the host: 0 = no refresh, 1 = refresh, 2 = adaptive check on device.
int host_refresh_mode(const mao_refresh& rf, int64_t t) {
  if (rf.kind == MAO_REFRESH_NEVER) return 0;
  if (rf.kind == MAO_REFRESH_EVERY_K) return ((t - 1) % rf.k) == 0 ? 1 : 0;
  return ((t - 1) % rf.pf) == 0 ? 2 : 0;
}

inline int ldp_of(int cols) { return round_up_int(cols, 8); }

// K slice of the panel Gram products of a launch with `nact` panels: enough
// slices to give about two tiles per SM, at most kMaxParts, at least 256 rows each,
// a multiple of 64 (whole K blocks, so slices never overlap).
inline int gram_slice(int k, int nact) {
  const int want = std::max(1, std::min(kMaxParts, (2 * 148 + nact - 1) / std::max(nact, 1)));
  const int sl = round_up_int(std::max(256, (k + want - 1) / want), 64);
  return std::max(sl, round_up_int((k + kMaxParts - 1) / kMaxParts, 64));
}

// Bytes of a three-plane bf16 set of a rows x cols matrix.
inline size_t planes_bytes(int rows, int cols) { return 3 * 2 * (size_t)rows * ldp_of(cols); }

// Scratch of one side (k x k factor F with basis Q) of one matrix.
struct SideBuf {
  size_t Fp, Qp, P, Ps, Psp;
  size_t W, Wp, Cp;  // super-panel buffer (k x kSuper, fp32 and planes) and the coefficients
  size_t Cpart;      // K-slice partials of the coefficients (large factors only)
  size_t pn, pnorm2, reorth, fin;  // squared column norms of P (original, sorted order); panel decisions
  size_t part, gs, rinv, keys, perm, flag, rho, bad, again;
  size_t dg;     // adaptive check: diag(Q^T F Q)
};

struct MatBuf {
  size_t Gp, Mp, T1G, T1M, Vtmp, Gh, Mh;  // SOAP (N reuses T1G, T2 reuses Mp)
  size_t Gr, Mr;                          // FOAM (N reuses Gp)
  size_t rowpart, colpart, ctmp, tau;
  size_t upd;                             // update-statistics slots of the weight-update product
  SideBuf L, R;
};

// Update-statistics slots of an m x n weight (32-row by 64-column blocks).
inline int upd_slots(int m, int n) { return ((m + 31) / 32) * ((n + 63) / 64); }

void side_layout(int k, bool check, Carver& cv, SideBuf& s, size_t flag_block) {
  const size_t kk = (size_t)k * k;
  const int parts = (k + gram_slice(k, 1) - 1) / gram_slice(k, 1);  // the most slices any launch uses
  s.Fp = cv.take(planes_bytes(k, k));
  s.Qp = cv.take(planes_bytes(k, k));
  s.P = cv.take(4 * kk);
  s.Ps = cv.take(4 * kk);
  s.Psp = cv.take(planes_bytes(k, k));
  s.W = cv.take(4 * (size_t)k * kSuper);
  s.Wp = cv.take(planes_bytes(k, kSuper));
  s.Cp = cv.take(planes_bytes(k, kSuper));
  s.Cpart = k >= kCoefSplitMinK ? cv.take(4 * (size_t)kMaxCoefParts * k * kSuper) : 0;
  s.part = cv.take(4 * (size_t)parts * kPanelSq);
  s.gs = cv.take(8 * (size_t)kGsDoubles);
  s.rinv = cv.take(2 * 3 * (size_t)kPanelSq);
  s.keys = cv.take(8 * (size_t)k);
  s.perm = cv.take(4 * (size_t)k);
  s.flag = flag_block;  // flag, rho, the failure counter and the second-pass flag share one 64-byte block
  s.rho = s.flag + 16;
  s.bad = s.flag + 32;
  s.again = s.flag + 48;
  s.reorth = s.flag + 56;
  s.fin = s.flag + 60;
  s.pn = cv.take(4 * (size_t)k);
  s.pnorm2 = cv.take(4 * (size_t)k);
  if (check) s.dg = cv.take(8 * (size_t)k);
}

struct Ctx {
  bool foam;
  const PcMat* mats;
  int count;
  float b1, b2, eps, lr, wd;
  int64_t t;
  mao_refresh rf;
  int raw_trace;
  int mode;  // host refresh mode
};

struct GroupPlan {
  int g0 = 0, g1 = 0;   // matrices [g0, g1)
  size_t scratch = 0;   // bytes of per-matrix scratch
  size_t flags = 0, flags_bytes = 0;  // all 64-byte flag blocks of the group, contiguous
  // launch-level gates of the QR's device-decided passes (ints: any second pass, any
  // second projection, any final pass among the group's factors), cleared before each
  // sub-panel's first pass
  size_t any = 0;
  std::vector<MatBuf> mb;
};

void plan_group_scratch(const Ctx& X, GroupPlan& G, size_t base) {
  Carver cv;
  cv.off = base;
  G.mb.assign(G.g1 - G.g0, MatBuf());
  const bool check = X.mode == 2;
  G.flags_bytes = (size_t)64 * 2 * (G.g1 - G.g0);
  G.flags = cv.take(G.flags_bytes);
  G.any = cv.take(16);
  bool g_one = true;  // every gradient of the group bf16: G is read directly (SOAP needs no plane copy)
  for (int i = G.g0; i < G.g1; ++i) g_one = g_one && X.mats[i].g_bf16;
  for (int i = G.g0; i < G.g1; ++i) {
    const PcMat& a = X.mats[i];
    MatBuf& b = G.mb[i - G.g0];
    const size_t mn = (size_t)a.m * a.n;
    b.Gp = (X.foam || !g_one) ? cv.take(planes_bytes(a.m, a.n)) : 0;
    b.Mp = cv.take(planes_bytes(a.m, a.n));
    if (!X.foam) {
      b.T1G = cv.take(planes_bytes(a.m, a.n));
      b.T1M = cv.take(planes_bytes(a.m, a.n));
      b.Vtmp = cv.take(4 * mn);
      b.Gh = cv.take(4 * mn);
      b.Mh = cv.take(4 * mn);
      side_layout(a.m, check, cv, b.L, G.flags + (size_t)128 * (i - G.g0));
    } else {
      b.Gr = cv.take(4 * mn);
      b.Mr = cv.take(4 * mn);
      const int tr = (a.m + 63) / 64, tc = (a.n + 63) / 64;
      b.rowpart = cv.take(4 * (size_t)tc * a.m);
      b.colpart = cv.take(4 * (size_t)tr * a.n);
      b.ctmp = cv.take(4 * (size_t)a.n);
      b.tau = cv.take(16);
    }
    side_layout(a.n, check, cv, b.R, G.flags + (size_t)128 * (i - G.g0) + 64);
    b.upd = cv.take(8 * (size_t)upd_slots(a.m, a.n));
  }
  G.scratch = cv.off - base;
}

size_t mat_scratch_estimate(const Ctx& X, int i) {
  GroupPlan g;
  g.g0 = i;
  g.g1 = i + 1;
  plan_group_scratch(X, g, 0);
  return g.scratch;
}

void make_groups(const Ctx& X, std::vector<GroupPlan>& groups) {
  groups.clear();
  int i = 0;
  while (i < X.count) {
    GroupPlan g;
    g.g0 = i;
    size_t acc = 0;
    int j = i;
    while (j < X.count) {
      const size_t s = mat_scratch_estimate(X, j);
      if (j > i && acc + s > kGroupBudget) break;
      acc += s;
      ++j;
    }
    g.g1 = j;
    groups.push_back(g);
    i = j;
  }
}

// ------------------------------------------------------------------ the builder
// Records every launch of one group into `ops`, with all device data staged in
// the arena; in sizing mode (ws == nullptr) only the sizes matter.
struct Op {
  enum Kind { GEMM, EW, SPLIT, ADAM, KEYS, ARGSORT, GATHER, VPERM, REDUCE, CHOL, COEFRED, RC, TAU, FOAMN, CHECK, ZERO }
      kind;
  size_t jobs = 0;
  int njobs = 0;
  int blocks = 0;
  double bytes = 0.0;
  const int* any = nullptr;  // launch-level gate (REDUCE, CHOL, COEFRED), or nullptr
  void* zero = nullptr;      // ZERO: device bytes cleared
  size_t zero_bytes = 0;
};

struct Builder {
  const Ctx& X;
  uint8_t* ws;      // workspace base or nullptr
  Arena arena;
  MapSet maps;
  std::vector<TableLaunch> gemms;  // staged after all maps are known
  std::vector<Op> ops;
  std::vector<int> gemm_of_op;     // op index -> gemm index (or -1)
  size_t zero_flag_off = 0;        // an int 0 in the arena

  Builder(const Ctx& x, uint8_t* w) : X(x), ws(w) {}

  // In sizing mode, pointers are fake but non-null and 16-byte aligned (never dereferenced).
  template <class T>
  T* wp(size_t off) const { return ws ? reinterpret_cast<T*>(ws + off) : reinterpret_cast<T*>(off + 16); }

  // Plane set at workspace offset `off` of a rows x cols matrix.
  Split3 planes(size_t off, int rows, int cols) const {
    const int ldp = ldp_of(cols);
    __nv_bfloat16* b = wp<__nv_bfloat16>(off);
    const size_t st = (size_t)rows * ldp;
    return Split3{{b, b + st, b + 2 * st}, rows, cols, ldp};
  }
  long long pstride(int rows, int cols) const { return (long long)rows * ldp_of(cols); }

  TableLaunch& new_gemm(int a_mn, int b_mn, int kernel_id) {
    gemms.emplace_back();
    gemms.back().a_mn = a_mn;
    gemms.back().b_mn = b_mn;
    gemms.back().kernel_id = kernel_id;
    Op o;
    o.kind = Op::GEMM;
    ops.push_back(o);
    gemm_of_op.push_back((int)gemms.size() - 1);
    return gemms.back();
  }

  // A job array of n records, followed by room for two compact arrays of the
  // records' first-block indices (filled by fill_starts once the records are final).
  template <class J>
  J* new_jobs(Op::Kind kind, int n, size_t& off) {
    const size_t bytes = sizeof(J) * std::max(n, 1) + 2 * sizeof(int) * std::max(n, 1);
    off = arena.take(bytes, 64);
    Op o;
    o.kind = kind;
    o.jobs = off;
    o.njobs = n;
    ops.push_back(o);
    gemm_of_op.push_back(-1);
    J* p = arena.hptr<J>(off);
    std::memset(static_cast<void*>(p), 0, bytes);
    return p;
  }
};

// The compact first-block index arrays after every job array (job_starts() on the device).
template <class J, class F>
void fill_starts_of(Builder& B, const Op& op, F first_block, int which = 0) {
  const int n = op.njobs;
  const J* jobs = B.arena.hptr<J>(op.jobs);
  int* st = reinterpret_cast<int*>(B.arena.host.data() + op.jobs + sizeof(J) * n) + which * n;
  for (int i = 0; i < n; ++i) st[i] = first_block(jobs[i]);
}

void fill_starts(Builder& B) {
  for (const Op& op : B.ops) {
    if (op.kind == Op::GEMM || op.njobs <= 0) continue;
    switch (op.kind) {
      case Op::EW: case Op::SPLIT: case Op::ADAM: case Op::FOAMN:
        fill_starts_of<EwJob>(B, op, [](const EwJob& j) { return j.blk_begin; });
        break;
      case Op::KEYS: case Op::ARGSORT:
        fill_starts_of<SortJob>(B, op, [](const SortJob& j) { return j.key_blk_begin; }, 0);
        fill_starts_of<SortJob>(B, op, [](const SortJob& j) { return j.col_blk_begin; }, 1);
        break;
      case Op::GATHER:
        fill_starts_of<GatherJob>(B, op, [](const GatherJob& j) { return j.blk_begin; });
        break;
      case Op::VPERM:
        fill_starts_of<VPermJob>(B, op, [](const VPermJob& j) { return j.blk_begin; });
        break;
      case Op::COEFRED:
        fill_starts_of<CoefJob>(B, op, [](const CoefJob& j) { return j.blk_begin; });
        break;
      case Op::RC:
        fill_starts_of<RcJob>(B, op, [](const RcJob& j) { return j.blk_begin; });
        break;
      default:
        break;  // one block per record (REDUCE, CHOL, TAU, CHECK): no search
    }
  }
}

int ew_blocks(int rows, int cols) {
  const long long e = (long long)rows * cols;
  return (int)((e + kElemsPerBlock - 1) / kElemsPerBlock);
}

// Adds the jobs of the basis refresh of every factor of the group: both sides of
// every SOAP matrix and the input side of every FOAM matrix, swept together so
// that each launch covers all of them (and the QR advances every factor by one
// panel per step).
mao_status build_refresh(Builder& B, GroupPlan& G) {
  const Ctx& X = B.X;
  const bool check = X.mode == 2;
  const int nm = G.g1 - G.g0;
  struct Unit {
    int i;
    bool left;
  };
  std::vector<Unit> units;
  for (int i = 0; i < nm; ++i) {
    if (!X.foam) units.push_back({i, true});
    units.push_back({i, false});
  }
  const int nu = (int)units.size();
  auto side = [&](int u) -> SideBuf& { return units[u].left ? G.mb[units[u].i].L : G.mb[units[u].i].R; };
  auto mat = [&](int u) -> const PcMat& { return X.mats[G.g0 + units[u].i]; };
  auto kof = [&](int u) { return units[u].left ? mat(u).m : mat(u).n; };
  auto Qp = [&](int u) { return units[u].left ? mat(u).QL : mat(u).QR; };
  auto permo = [&](int u) { return units[u].left ? mat(u).perm_L : mat(u).perm_R; };
  auto flagp = [&](int u) -> const int* { return check ? B.wp<int>(side(u).flag) : nullptr; };
  auto anyp = [&](int which) -> int* { return B.wp<int>(G.any) + which; };

  // three-plane split of Q (F's planes come from the factor products)
  {
    size_t off;
    EwJob* J = B.new_jobs<EwJob>(Op::SPLIT, nu, off);
    int blk = 0;
    for (int i = 0; i < nu; ++i) {
      const int k = kof(i);
      EwJob& j = J[i];
      j.a = Qp(i);
      j.pa = B.wp<__nv_bfloat16>(side(i).Qp);
      j.pstride = B.pstride(k, k);
      j.rows = k;
      j.cols = k;
      j.lda = k;
      j.ldp = ldp_of(k);
      j.blk_begin = blk;
      blk += ew_blocks(k, k);
    }
    B.ops.back().blocks = blk;
    {  // algorithmic bytes: the fp32 source read, three bf16 planes written
      double bytes = 0;
      for (int q = 0; q < B.ops.back().njobs; ++q) bytes += (double)J[q].rows * J[q].cols * (4 + 6);
      B.ops.back().bytes = bytes;
    }
  }
  // power step P = F Q (A = F K-major, B = Q stored K x N)
  {
    TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_POWER);
    for (int i = 0; i < nu; ++i) {
      const int k = kof(i);
      // an adaptive check needs P itself, so the product is not gated
      MAO_TRY(table_add(g, B.maps, B.planes(side(i).Fp, k, k), B.planes(side(i).Qp, k, k), k, k, k, 0, 0,
                        B.wp<float>(side(i).P), nullptr, k, nullptr, 0, 1.f, 0.f, nullptr));
    }
  }
  // keys and argsort
  {
    size_t off;
    SortJob* J = B.new_jobs<SortJob>(Op::KEYS, nu, off);
    int blk = 0, kblk = 0;
    for (int i = 0; i < nu; ++i) {
      const int k = kof(i);
      SortJob& j = J[i];
      j.Q = Qp(i);
      j.P = B.wp<float>(side(i).P);
      j.key = B.wp<double>(side(i).keys);
      j.pn = B.wp<float>(side(i).pn);
      j.pn_sorted = B.wp<float>(side(i).pnorm2);
      j.dg = check ? B.wp<double>(side(i).dg) : nullptr;
      j.kflag = nullptr;
      j.perm = B.wp<int>(side(i).perm);
      j.perm_out = permo(i);
      j.flag = flagp(i);
      j.k = k;
      j.col_blk_begin = blk;
      blk += (k + 255) / 256;
      j.key_blk_begin = kblk;
      kblk += (k + 31) / 32;
    }
    B.ops.back().blocks = kblk;
    Op o = B.ops.back();  // the argsort reuses the job array
    if (check) {
      size_t coff;
      CheckJob* C = B.new_jobs<CheckJob>(Op::CHECK, nu, coff);
      for (int i = 0; i < nu; ++i) {
        C[i].dg = B.wp<double>(side(i).dg);
        C[i].pn = B.wp<float>(side(i).pn);
        C[i].flag = B.wp<int>(side(i).flag);
        C[i].rho = B.wp<float>(side(i).rho);
        C[i].k = kof(i);
      }
      B.ops.back().blocks = nu;
    }
    o.kind = Op::ARGSORT;
    o.blocks = blk;
    B.ops.push_back(o);
    B.gemm_of_op.push_back(-1);
  }
  // gathered P and its planes
  {
    size_t off;
    GatherJob* J = B.new_jobs<GatherJob>(Op::GATHER, nu, off);
    int blk = 0;
    for (int i = 0; i < nu; ++i) {
      const int k = kof(i);
      GatherJob& j = J[i];
      j.src = B.wp<float>(side(i).P);
      j.dst = B.wp<float>(side(i).Ps);
      j.dstp = B.wp<__nv_bfloat16>(side(i).Psp);
      j.pstride = B.pstride(k, k);
      j.perm = B.wp<int>(side(i).perm);
      j.flag = flagp(i);
      j.rows = k;
      j.cols = k;
      j.ld = k;
      j.ldp = ldp_of(k);
      j.blk_begin = blk;
      blk += ew_blocks(k, k);
    }
    B.ops.back().blocks = blk;
  }
  // QR by super-panels of kSuper columns (block Gram-Schmidt).  For each super-panel
  // [c0, c0 + kSuper): one projection of all its columns against the finished columns
  // [0, c0) (each pass over Q's planes serves kSuper columns), then its kPanel-column
  // sub-panels in turn: each after the first is projected against the super-panel's
  // finished sub-panels, and each is orthonormalised by Cholesky-QR (up to three
  // passes, and a second projection against every finished column, all decided on
  // the device).
  int maxk = 0;
  for (int i = 0; i < nu; ++i) maxk = std::max(maxk, kof(i));
  const int nsuper = (maxk + kSuper - 1) / kSuper;
  enum { PS = 0, WA = 1, QF = 2 };
  for (int sp = 0; sp < nsuper; ++sp) {
    const int c0 = sp * kSuper;
    for (int sub = 0; sub < kSuper / kPanel; ++sub) {
      const int cs = c0 + sub * kPanel;  // first column of the sub-panel
      std::vector<int> act;
      for (int i = 0; i < nu; ++i)
        if (kof(i) > cs) act.push_back(i);
      if (act.empty()) break;
      auto wdt = [&](int i) { return std::min(kPanel, kof(i) - cs); };
      // a sub-panel's fp32 storage and plane view: columns cs .. cs + w of Ps / Q, or
      // the sub-panel's columns of the super-panel buffer W
      auto fp = [&](int i, int where, int* ld) -> float* {
        const int k = kof(i);
        switch (where) {
          case PS: *ld = k; return B.wp<float>(side(i).Ps) + cs;
          case WA: *ld = kSuper; return B.wp<float>(side(i).W) + sub * kPanel;
          default: *ld = k; return Qp(i) + cs;
        }
      };
      auto pv = [&](int i, int where) -> Split3 {
        const int k = kof(i), w = wdt(i);
        Split3 v;
        switch (where) {
          case PS: v = B.planes(side(i).Psp, k, k); break;
          case WA: v = B.planes(side(i).Wp, k, kSuper); break;
          default: v = B.planes(side(i).Qp, k, k); break;
        }
        const int off = where == WA ? sub * kPanel : cs;
        for (int q = 0; q < 3; ++q) v.p[q] += off;
        v.cols = w;
        return v;
      };
      // one Cholesky-QR of every active sub-panel: dst = src R^{-1} (dst may be src).
      // pass 0: the first pass; it decides on the device whether the second pass
      //         (flag again), the second projection (reorth) and the final pass (fin)
      //         run, and writes straight into Q's columns when none does;
      // pass 1: the second pass (gated by again); pass 2: the final pass (gated by fin)
      auto cholqr = [&](int src, int dst, int pass) -> mao_status {
        auto gate = [&](int u) -> const int* {
          return pass == 1 ? B.wp<int>(side(u).again) : pass == 2 ? B.wp<int>(side(u).fin) : flagp(u);
        };
        // the launch-level gate of a gated pass: set by the first pass when any factor
        // takes it, so that a pass no factor takes costs no more than its launches
        const int* lgate = pass == 1 ? anyp(kAnyAgain) : pass == 2 ? anyp(kAnyFin) : nullptr;
        if (pass == 0) {
          Op z;
          z.kind = Op::ZERO;
          z.zero = B.wp<int>(G.any);
          z.zero_bytes = 16;
          B.ops.push_back(z);
          B.gemm_of_op.push_back(-1);
        }
        // Gram partials over K slices (fp32-faithful), one 128 x 128 tile each
        TableLaunch& gg = B.new_gemm(1, 1, MAO_K_PC_PANEL);
        gg.any = lgate;
        const int nact = (int)act.size();
        for (int i : act) {
          const int k = kof(i), w = wdt(i);
          const int sl = gram_slice(k, nact);
          float* part = B.wp<float>(side(i).part);
          const Split3 Wv = pv(i, src);
          for (int s0 = 0, p = 0; s0 < k; s0 += sl, ++p)
            MAO_TRY(table_add(gg, B.maps, Wv, Wv, w, w, std::min(sl, k - s0), 0, 0, part + (size_t)p * kPanelSq,
                              nullptr, kPanel, nullptr, 0, 1.f, 0.f, gate(i), s0));
        }
        size_t off;
        PanelJob* J = B.new_jobs<PanelJob>(Op::REDUCE, (int)act.size(), off);
        for (size_t a = 0; a < act.size(); ++a) {
          const int i = act[a];
          const int k = kof(i);
          PanelJob& j = J[a];
          j.part = B.wp<float>(side(i).part);
          j.gs = B.wp<double>(side(i).gs);
          j.rinv = B.wp<__nv_bfloat16>(side(i).rinv);
          j.bad = B.wp<int>(side(i).bad);
          j.again = B.wp<int>(side(i).again);
          j.flag = gate(i);
          j.w = wdt(i);
          j.nparts = (k + gram_slice(k, nact) - 1) / gram_slice(k, nact);
          j.first = pass == 0 ? 1 : 0;
          if (pass == 0) {
            j.fin = B.wp<int>(side(i).fin);
            j.any_again = anyp(kAnyAgain);
            j.any_fin = anyp(kAnyFin);
          }
          if (pass == 0 && cs > 0) {
            j.pnorm2 = B.wp<float>(side(i).pnorm2) + cs;
            j.reorth = B.wp<int>(side(i).reorth);
            j.any_reorth = anyp(kAnyReorth);
          }
        }
        B.ops.back().blocks = (int)act.size() * kRedBlocks;
        B.ops.back().any = lgate;
        Op ch = B.ops.back();  // the factorisation reuses the job array
        ch.kind = Op::CHOL;
        ch.blocks = (int)act.size();
        B.ops.push_back(ch);
        B.gemm_of_op.push_back(-1);
        TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_QR_APPLY);
        g.any = lgate;
        for (int i : act) {
          const int k = kof(i), w = wdt(i);
          __nv_bfloat16* r = B.wp<__nv_bfloat16>(side(i).rinv);
          const Split3 Ri{{r, r + kPanelSq, r + 2 * kPanelSq}, w, w, kPanel};
          const Split3 out_p = pv(i, dst);
          int ld = 0;
          float* out = fp(i, dst, &ld);
          MAO_TRY(table_add(g, B.maps, pv(i, src), Ri, k, w, w, 0, 0, out, &out_p, ld, nullptr, 0, 1.f, 0.f,
                            gate(i)));
          if (pass == 0) {  // final already: Q's columns
            const Split3 q_p = pv(i, QF);
            int ldq = 0;
            float* q = fp(i, QF, &ldq);
            MAO_TRY(table_set_alt(g, B.wp<int>(side(i).fin), q, &q_p, ldq));
          }
        }
        return MAO_OK;
      };
      // remove the columns [a0, a1) of Q from `width` columns of the source:
      //   C = Q[:, a0:a1]^T Y (rows a0 .. a1 of the coefficient buffer);
      //   W = Y - Q[:, a0:a1] C (fp32 and planes, into the super-panel buffer at column
      //   `wcol`)
      // `width` > kPanel projects the whole super-panel (its sources are Ps's columns).
      // When the coefficient product has too few tiles to fill the GPU, the large
      // factors split it over K into fp32 partials, summed (in slice order) into C's planes.
      auto project = [&](const std::vector<int>& units, int from, int col, int a0, int a1, int wcol, int width,
                         bool reorth) -> mao_status {
        auto pflag = [&](int u) -> const int* { return reorth ? B.wp<int>(side(u).reorth) : flagp(u); };
        auto wof = [&](int i) { return std::min(width, kof(i) - col); };
        // a source view of `width` columns starting at column `col` (Ps) or `wcol` (W)
        auto src_p = [&](int i) -> Split3 {
          const int k = kof(i);
          Split3 v = from == PS ? B.planes(side(i).Psp, k, k) : B.planes(side(i).Wp, k, kSuper);
          const int off = from == PS ? col : wcol;
          for (int q = 0; q < 3; ++q) v.p[q] += off;
          v.cols = wof(i);
          return v;
        };
        auto src_f = [&](int i, int* ld) -> const float* {
          if (from == PS) {
            *ld = kof(i);
            return B.wp<float>(side(i).Ps) + col;
          }
          *ld = kSuper;
          return B.wp<float>(side(i).W) + wcol;
        };
        const int rows = a1 - a0;
        int tiles = 0;
        for (size_t u = 0; u < units.size(); ++u) tiles += ((rows + 127) / 128) * ((width + 127) / 128);
        const int want = std::min(kMaxCoefParts, std::max(1, (2 * 148 + tiles - 1) / std::max(tiles, 1)));
        const int* lgate = reorth ? anyp(kAnyReorth) : nullptr;
        TableLaunch& gc = B.new_gemm(1, 1, MAO_K_PC_QR);
        gc.any = lgate;
        std::vector<CoefJob> red;
        int rblk = 0;
        for (int i : units) {
          const int k = kof(i), w = wof(i);
          Split3 C = B.planes(side(i).Cp, k, kSuper);
          for (int q = 0; q < 3; ++q) C.p[q] += (size_t)a0 * kSuper;
          C.rows = rows;
          C.cols = w;
          const int S = k >= kCoefSplitMinK ? want : 1;
          if (S == 1) {
            MAO_TRY(table_add(gc, B.maps, B.planes(side(i).Qp, k, k), src_p(i), rows, w, k, a0, 0, nullptr, &C,
                              kSuper, nullptr, 0, 1.f, 0.f, pflag(i)));
            continue;
          }
          const int sl = round_up_int((k + S - 1) / S, 64);
          float* part = B.wp<float>(side(i).Cpart);
          const long long pst = (long long)k * kSuper;
          int p = 0;
          for (int s0 = 0; s0 < k; s0 += sl, ++p)
            MAO_TRY(table_add(gc, B.maps, B.planes(side(i).Qp, k, k), src_p(i), rows, w, std::min(sl, k - s0), a0,
                              0, part + p * pst + (size_t)a0 * kSuper, nullptr, kSuper, nullptr, 0, 1.f, 0.f,
                              pflag(i), s0));
          CoefJob cj;
          std::memset(&cj, 0, sizeof(cj));
          cj.part = part + (size_t)a0 * kSuper;
          cj.cp = B.wp<__nv_bfloat16>(side(i).Cp) + (size_t)a0 * kSuper;
          cj.part_stride = pst;
          cj.pstride = B.pstride(k, kSuper);
          cj.flag = pflag(i);
          cj.rows = rows;
          cj.ld = kSuper;
          cj.nparts = p;
          cj.blk_begin = rblk;
          rblk += (rows * kSuper + 1023) / 1024;
          red.push_back(cj);
        }
        if (!red.empty()) {
          size_t off;
          CoefJob* J = B.new_jobs<CoefJob>(Op::COEFRED, (int)red.size(), off);
          for (size_t a = 0; a < red.size(); ++a) J[a] = red[a];
          B.ops.back().blocks = rblk;
          B.ops.back().any = lgate;
        }
        TableLaunch& gw = B.new_gemm(0, 1, MAO_K_PC_QR);
        gw.any = lgate;
        for (int i : units) {
          const int k = kof(i), w = wof(i);
          Split3 C = B.planes(side(i).Cp, k, kSuper);
          C.rows = a1;  // the product reads rows a0 .. a1 (K slice from a0)
          C.cols = w;
          Split3 Wp = B.planes(side(i).Wp, k, kSuper);
          for (int q = 0; q < 3; ++q) Wp.p[q] += wcol;
          Wp.cols = w;
          int lda = 0;
          const float* aux = src_f(i, &lda);
          float* W = B.wp<float>(side(i).W) + wcol;
          MAO_TRY(table_add(gw, B.maps, B.planes(side(i).Qp, k, k), C, k, w, rows, 0, 0, W, &Wp, kSuper, aux, lda,
                            -1.f, 1.f, pflag(i), a0));
        }
        return MAO_OK;
      };
      // The products W R^{-1} run in place (each output row block reads only its own
      // rows of W, all of K in one tile).
      if (sub == 0) {
        if (c0 == 0) {
          MAO_TRY(cholqr(PS, WA, 0));
          MAO_TRY(cholqr(WA, WA, 1));
          MAO_TRY(cholqr(WA, QF, 2));
        } else {
          MAO_TRY(project(act, PS, c0, 0, c0, 0, kSuper, false));  // the whole super-panel
          MAO_TRY(cholqr(WA, WA, 0));
          MAO_TRY(cholqr(WA, WA, 1));
          MAO_TRY(project(act, WA, cs, 0, cs, 0, kPanel, true));
          MAO_TRY(cholqr(WA, QF, 2));
        }
      } else {
        // against the super-panel's finished sub-panels (from Ps when the super-panel is
        // the first)
        MAO_TRY(project(act, c0 == 0 ? PS : WA, cs, c0, cs, sub * kPanel, kPanel, false));
        MAO_TRY(cholqr(WA, WA, 0));
        MAO_TRY(cholqr(WA, WA, 1));
        MAO_TRY(project(act, WA, cs, 0, cs, sub * kPanel, kPanel, true));
        MAO_TRY(cholqr(WA, QF, 2));
      }
    }
  }
  return MAO_OK;
}

mao_status build_group(Builder& B, GroupPlan& G) {
  const Ctx& X = B.X;
  const int nm = G.g1 - G.g0;
  const bool foam = X.foam;
  auto A = [&](int i) -> const PcMat& { return X.mats[G.g0 + i]; };
  B.zero_flag_off = B.arena.take(16, 16);
  std::memset(B.arena.hptr<int>(B.zero_flag_off), 0, 16);

  // A group whose gradients are all bf16 reads each G directly as a one-plane
  // operand (exact); otherwise the momentum pass writes three planes of G.
  bool g_one = true;
  for (int i = 0; i < nm; ++i) g_one = g_one && A(i).g_bf16;
  const int gpl = g_one ? 1 : 3;
  auto Gop = [&](int i) -> Split3 {
    const PcMat& a = A(i);
    if (!g_one) return B.planes(G.mb[i].Gp, a.m, a.n);
    // sizing mode: a distinct stand-in address per matrix, never dereferenced
    const __nv_bfloat16* g = B.ws ? static_cast<const __nv_bfloat16*>(a.G)
                                  : reinterpret_cast<const __nv_bfloat16*>((1ull << 60) + 256ull * (G.g0 + i));
    return Split3{{g, nullptr, nullptr}, a.m, a.n, a.n};
  };

  // momentum + planes of M (and of G unless it is read directly)
  {
    size_t off;
    EwJob* J = B.new_jobs<EwJob>(Op::EW, nm, off);
    int blk = 0;
    double bytes = 0;
    for (int i = 0; i < nm; ++i) {
      const PcMat& a = A(i);
      EwJob& j = J[i];
      j.a = a.G;
      j.a_bf16 = a.g_bf16;
      j.f0 = a.M;
      j.pa = g_one ? nullptr : B.wp<__nv_bfloat16>(G.mb[i].Gp);
      j.pb = B.wp<__nv_bfloat16>(G.mb[i].Mp);
      j.pstride = B.pstride(a.m, a.n);
      j.rows = a.m;
      j.cols = a.n;
      j.lda = a.n;
      j.ldf = a.n;
      j.ldp = ldp_of(a.n);
      j.blk_begin = blk;
      blk += ew_blocks(a.m, a.n);
      bytes += (double)a.m * a.n * ((a.g_bf16 ? 2 : 4) + 8 + 6 + (g_one ? 0 : 6));
    }
    B.ops.back().blocks = blk;
    B.ops.back().bytes = bytes;
  }
  // factor EMAs; with `planes` their epilogue also writes F's planes for the refresh
  auto factor_products = [&](bool planes) -> mao_status {
    if (!foam) {
      TableLaunch& g = B.new_gemm(0, 0, MAO_K_PC_FACTOR);
      g.pa = g.pb = gpl;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        const Split3 Fp = B.planes(G.mb[i].L.Fp, a.m, a.m);
        MAO_TRY(table_add(g, B.maps, Gop(i), Gop(i), a.m, a.m, a.n, 0, 0, a.L, planes ? &Fp : nullptr, a.m, a.L,
                          a.m, 1.f - X.b2, X.b2, nullptr));
      }
    }
    TableLaunch& g = B.new_gemm(1, 1, MAO_K_PC_FACTOR);
    g.pa = g.pb = gpl;
    for (int i = 0; i < nm; ++i) {
      const PcMat& a = A(i);
      const Split3 Fp = B.planes(G.mb[i].R.Fp, a.n, a.n);
      MAO_TRY(table_add(g, B.maps, Gop(i), Gop(i), a.n, a.n, a.m, 0, 0, a.R, planes ? &Fp : nullptr, a.n, a.R,
                        a.n, 1.f - X.b2, X.b2, nullptr));
    }
    return MAO_OK;
  };
  const bool lag = X.rf.lag != 0 && X.mode != 0;
  if (lag) {
    // The refresh sees the factors before this step's gradient: planes of the old
    // F, the refresh, then the factor EMAs.
    size_t off;
    const int per = foam ? 1 : 2;
    EwJob* J = B.new_jobs<EwJob>(Op::SPLIT, per * nm, off);
    int blk = 0;
    for (int i = 0; i < nm; ++i) {
      const PcMat& a = A(i);
      for (int s = 0; s < per; ++s) {
        const bool right = foam || s == 1;
        const int k = right ? a.n : a.m;
        EwJob& j = J[per * i + s];
        j.a = right ? a.R : a.L;
        j.pa = B.wp<__nv_bfloat16>(right ? G.mb[i].R.Fp : G.mb[i].L.Fp);
        j.pstride = B.pstride(k, k);
        j.rows = k;
        j.cols = k;
        j.lda = k;
        j.ldp = ldp_of(k);
        j.blk_begin = blk;
        blk += ew_blocks(k, k);
      }
    }
    B.ops.back().blocks = blk;
    {  // algorithmic bytes: the fp32 source read, three bf16 planes written
      double bytes = 0;
      for (int q = 0; q < B.ops.back().njobs; ++q) bytes += (double)J[q].rows * J[q].cols * (4 + 6);
      B.ops.back().bytes = bytes;
    }
    MAO_TRY(build_refresh(B, G));
    MAO_TRY(factor_products(false));
  } else {
    MAO_TRY(factor_products(X.mode != 0));
  }
  // refresh, or plain planes of the bases
  if (lag) {
    // done above
  } else if (X.mode != 0) {
    MAO_TRY(build_refresh(B, G));
  } else {
    size_t off;
    const int per = foam ? 1 : 2;
    EwJob* J = B.new_jobs<EwJob>(Op::SPLIT, per * nm, off);
    int blk = 0;
    for (int i = 0; i < nm; ++i) {
      const PcMat& a = A(i);
      for (int s = 0; s < per; ++s) {
        const bool right = foam || s == 1;
        const int k = right ? a.n : a.m;
        EwJob& j = J[per * i + s];
        j.a = right ? a.QR : a.QL;
        j.pa = B.wp<__nv_bfloat16>(right ? G.mb[i].R.Qp : G.mb[i].L.Qp);
        j.pstride = B.pstride(k, k);
        j.rows = k;
        j.cols = k;
        j.lda = k;
        j.ldp = ldp_of(k);
        j.blk_begin = blk;
        blk += ew_blocks(k, k);
      }
    }
    B.ops.back().blocks = blk;
    {  // algorithmic bytes: the fp32 source read, three bf16 planes written
      double bytes = 0;
      for (int q = 0; q < B.ops.back().njobs; ++q) bytes += (double)J[q].rows * J[q].cols * (4 + 6);
      B.ops.back().bytes = bytes;
    }
    // identity permutations for the callers that asked for them
    bool any = false;
    for (int i = 0; i < nm; ++i) any = any || A(i).perm_R || (!foam && A(i).perm_L);
    if (any) {
      size_t off2;
      SortJob* S = B.new_jobs<SortJob>(Op::ARGSORT, per * nm, off2);
      int blk2 = 0;
      int* zero = B.arena.dev ? B.arena.dptr<int>(B.zero_flag_off) : reinterpret_cast<int*>(16);
      for (int i = 0; i < nm; ++i)
        for (int s = 0; s < per; ++s) {
          const bool right = foam || s == 1;
          SortJob& j = S[per * i + s];
          j.perm_out = right ? A(i).perm_R : A(i).perm_L;
          j.flag = zero;
          j.k = right ? A(i).n : A(i).m;
          j.col_blk_begin = blk2;
          blk2 += (j.k + 255) / 256;
        }
      B.ops.back().blocks = blk2;
    }
  }

  if (!foam) {
    // V follows the refresh permutations
    if (X.mode != 0) {
      size_t off;
      VPermJob* J = B.new_jobs<VPermJob>(Op::VPERM, nm, off);
      int blk = 0;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        VPermJob& j = J[i];
        j.V = a.V;
        j.dst = B.wp<float>(G.mb[i].Vtmp);
        j.pl = B.wp<int>(G.mb[i].L.perm);
        j.pr = B.wp<int>(G.mb[i].R.perm);
        j.fl = X.mode == 2 ? B.wp<int>(G.mb[i].L.flag) : nullptr;
        j.fr = X.mode == 2 ? B.wp<int>(G.mb[i].R.flag) : nullptr;
        j.m = a.m;
        j.n = a.n;
        j.blk_begin = blk;
        blk += ew_blocks(a.m, a.n);
      }
      B.ops.back().blocks = blk;
    }
    // Gh = Q_L^T G Q_R and Mh = Q_L^T M Q_R.  A bf16 G makes its first product a
    // three-product one (one exact plane) and the second a six-product one (both
    // operands three-plane), so G's pair is ordered to put the cheap product on the
    // larger side: Q_L^T G first for m >= n, G Q_R first for m < n.  M's two products
    // cost the same in either order: Q_L^T M first.
    auto tall = [&](int i) { return gpl == 3 || A(i).m >= A(i).n; };
    bool any_tall = false, any_wide = false;
    for (int i = 0; i < nm; ++i) (tall(i) ? any_tall : any_wide) = true;
    // T1G = Q_L^T G (tall G)   (A = Q_L stored K x M, B = G stored K x N)
    if (any_tall) {
      TableLaunch& g = B.new_gemm(1, 1, MAO_K_PC_ROTATE);
      g.pb = gpl;
      for (int i = 0; i < nm; ++i) {
        if (!tall(i)) continue;
        const PcMat& a = A(i);
        const Split3 T1G = B.planes(G.mb[i].T1G, a.m, a.n);
        MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].L.Qp, a.m, a.m), Gop(i), a.m, a.n, a.m, 0, 0, nullptr, &T1G,
                          a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // T1G = G Q_R (wide G)   (A = G K-major, B = Q_R stored K x N)
    if (any_wide) {
      TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_ROTATE);
      g.pa = gpl;
      for (int i = 0; i < nm; ++i) {
        if (tall(i)) continue;
        const PcMat& a = A(i);
        const Split3 T1G = B.planes(G.mb[i].T1G, a.m, a.n);
        MAO_TRY(table_add(g, B.maps, Gop(i), B.planes(G.mb[i].R.Qp, a.n, a.n), a.m, a.n, a.n, 0, 0, nullptr, &T1G,
                          a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // T1M = Q_L^T M, and Gh = Q_L^T T1G for the wide G
    {
      TableLaunch& g2 = B.new_gemm(1, 1, MAO_K_PC_ROTATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        const Split3 T1M = B.planes(G.mb[i].T1M, a.m, a.n);
        MAO_TRY(table_add(g2, B.maps, B.planes(G.mb[i].L.Qp, a.m, a.m), B.planes(G.mb[i].Mp, a.m, a.n), a.m, a.n,
                          a.m, 0, 0, nullptr, &T1M, a.n, nullptr, 0, 1.f, 0.f, nullptr));
        if (!tall(i))
          MAO_TRY(table_add(g2, B.maps, B.planes(G.mb[i].L.Qp, a.m, a.m), B.planes(G.mb[i].T1G, a.m, a.n), a.m,
                            a.n, a.m, 0, 0, B.wp<float>(G.mb[i].Gh), nullptr, a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // Gh = T1G Q_R (tall G), Mh = T1M Q_R (fp32)
    {
      TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_ROTATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        const Split3 Qr = B.planes(G.mb[i].R.Qp, a.n, a.n);
        if (tall(i))
          MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].T1G, a.m, a.n), Qr, a.m, a.n, a.n, 0, 0,
                            B.wp<float>(G.mb[i].Gh), nullptr, a.n, nullptr, 0, 1.f, 0.f, nullptr));
        MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].T1M, a.m, a.n), Qr, a.m, a.n, a.n, 0, 0,
                          B.wp<float>(G.mb[i].Mh), nullptr, a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // Adam: V and the planes of N (into T1G's planes)
    {
      size_t off;
      EwJob* J = B.new_jobs<EwJob>(Op::ADAM, nm, off);
      int blk = 0;
      double bytes = 0;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        EwJob& j = J[i];
        j.a = B.wp<float>(G.mb[i].Gh);
        j.b = B.wp<float>(G.mb[i].Mh);
        j.f0 = a.V;
        j.f1 = X.mode != 0 ? B.wp<float>(G.mb[i].Vtmp) : nullptr;
        j.pa = B.wp<__nv_bfloat16>(G.mb[i].T1G);
        j.pstride = B.pstride(a.m, a.n);
        j.rows = a.m;
        j.cols = a.n;
        j.lda = a.n;
        j.ldb = a.n;
        j.ldf = a.n;
        j.ldp = ldp_of(a.n);
        j.blk_begin = blk;
        blk += ew_blocks(a.m, a.n);
        bytes += (double)a.m * a.n * (4 + 4 + 8 + 6);
      }
      B.ops.back().blocks = blk;
      B.ops.back().bytes = bytes;
    }
    // T2 = Q_L N -> the (free) M planes
    {
      TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_ROTATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        const Split3 T2 = B.planes(G.mb[i].Mp, a.m, a.n);
        MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].L.Qp, a.m, a.m), B.planes(G.mb[i].T1G, a.m, a.n), a.m, a.n,
                          a.m, 0, 0, nullptr, &T2, a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // U = T2 Q_R^T ; W <- W (1 - lr wd) - lr U
    {
      TableLaunch& g = B.new_gemm(0, 0, MAO_K_PC_UPDATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].Mp, a.m, a.n), B.planes(G.mb[i].R.Qp, a.n, a.n), a.m, a.n,
                          a.n, 0, 0, a.W, nullptr, a.n, a.W, a.n, -X.lr, 1.f - X.lr * X.wd, nullptr));
        MAO_TRY(table_set_stats(g, B.wp<float2>(G.mb[i].upd)));
      }
    }
  } else {
    // Gr, Mr = {G, M} Q_R  (A K-major, B = Q_R stored K x N)
    {
      TableLaunch& g = B.new_gemm(0, 1, MAO_K_PC_ROTATE);
      g.pa = gpl;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        MAO_TRY(table_add(g, B.maps, Gop(i), B.planes(G.mb[i].R.Qp, a.n, a.n), a.m, a.n, a.n, 0, 0,
                          B.wp<float>(G.mb[i].Gr), nullptr, a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
      TableLaunch& g2 = B.new_gemm(0, 1, MAO_K_PC_ROTATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        MAO_TRY(table_add(g2, B.maps, B.planes(G.mb[i].Mp, a.m, a.n), B.planes(G.mb[i].R.Qp, a.n, a.n), a.m, a.n,
                          a.n, 0, 0, B.wp<float>(G.mb[i].Mr), nullptr, a.n, nullptr, 0, 1.f, 0.f, nullptr));
      }
    }
    // row/col partials of Gr^2, r/c EMAs and tau, N
    {
      size_t off;
      RcJob* J = B.new_jobs<RcJob>(Op::RC, nm, off);
      int blk = 0;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        RcJob& j = J[i];
        j.Gr = B.wp<float>(G.mb[i].Gr);
        j.rowpart = B.wp<float>(G.mb[i].rowpart);
        j.colpart = B.wp<float>(G.mb[i].colpart);
        j.m = a.m;
        j.n = a.n;
        j.tiles_c = (a.n + 63) / 64;
        j.tiles_r = (a.m + 63) / 64;
        j.blk_begin = blk;
        blk += j.tiles_c * j.tiles_r;
      }
      B.ops.back().blocks = blk;
      double bytes = 0;
      for (int q = 0; q < nm; ++q) bytes += (double)J[q].m * J[q].n * 4;  // Gr read once
      B.ops.back().bytes = bytes;
    }
    {
      size_t off;
      TauJob* J = B.new_jobs<TauJob>(Op::TAU, nm, off);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        TauJob& j = J[i];
        j.r = a.r;
        j.c = a.c;
        j.rowpart = B.wp<float>(G.mb[i].rowpart);
        j.colpart = B.wp<float>(G.mb[i].colpart);
        j.R = a.R;
        j.perm = X.mode != 0 ? B.wp<int>(G.mb[i].R.perm) : nullptr;
        j.flag = X.mode == 2 ? B.wp<int>(G.mb[i].R.flag) : nullptr;
        j.c_tmp = B.wp<float>(G.mb[i].ctmp);
        j.tau = B.wp<float>(G.mb[i].tau);
        j.m = a.m;
        j.n = a.n;
        j.tiles_c = (a.n + 63) / 64;
        j.tiles_r = (a.m + 63) / 64;
      }
      B.ops.back().blocks = nm;
    }
    {
      size_t off;
      EwJob* J = B.new_jobs<EwJob>(Op::FOAMN, nm, off);
      int blk = 0;
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        EwJob& j = J[i];
        j.a = B.wp<float>(G.mb[i].Mr);
        j.b = B.wp<float>(G.mb[i].tau);
        j.vr = a.r;
        j.vc = a.c;
        j.pa = B.wp<__nv_bfloat16>(G.mb[i].Gp);
        j.pstride = B.pstride(a.m, a.n);
        j.rows = a.m;
        j.cols = a.n;
        j.lda = a.n;
        j.ldp = ldp_of(a.n);
        j.blk_begin = blk;
        blk += ew_blocks(a.m, a.n);
      }
      B.ops.back().blocks = blk;
      double bytes = 0;
      for (int q = 0; q < nm; ++q) bytes += (double)J[q].rows * J[q].cols * (4 + 6);  // Mr read, N planes
      B.ops.back().bytes = bytes;
    }
    // U = N Q_R^T ; W update
    {
      TableLaunch& g = B.new_gemm(0, 0, MAO_K_PC_UPDATE);
      for (int i = 0; i < nm; ++i) {
        const PcMat& a = A(i);
        MAO_TRY(table_add(g, B.maps, B.planes(G.mb[i].Gp, a.m, a.n), B.planes(G.mb[i].R.Qp, a.n, a.n), a.m, a.n,
                          a.n, 0, 0, a.W, nullptr, a.n, a.W, a.n, -X.lr, 1.f - X.lr * X.wd, nullptr));
        MAO_TRY(table_set_stats(g, B.wp<float2>(G.mb[i].upd)));
      }
    }
  }
  return MAO_OK;
}

// Everything one group needs at launch time, independent of the caller's
// descriptor array: the staged host image of the arena and the launch list.
struct BuiltGroup {
  size_t maps_off = 0;
  std::vector<StagedLaunch> staged;
  std::vector<Op> ops;
  std::vector<int> gemm_of_op;
  std::vector<uint8_t> arena;
  size_t stats_jobs = 0;  // StatsJob array in the arena
};

mao_status finish_build(Builder& B, BuiltGroup& out) {
  fill_starts(B);
  // maps after all problems are known
  out.maps_off = B.arena.take(sizeof(CUtensorMap) * std::max<size_t>(B.maps.keys.size(), 1), 64);
  if (B.ws) {
    MAO_TRY(B.maps.encode_all());
    std::memcpy(B.arena.host.data() + out.maps_off, B.maps.maps.data(), sizeof(CUtensorMap) * B.maps.maps.size());
  }
  out.staged.clear();
  for (const TableLaunch& L : B.gemms) out.staged.push_back(table_stage(B.arena, L, out.maps_off));
  return MAO_OK;
}

// Per-matrix diagnostics records of a group (one launch).
void add_stats_jobs(Builder& B, GroupPlan& G, BuiltGroup& bg) {
  const int nm = G.g1 - G.g0;
  bg.stats_jobs = B.arena.take(sizeof(StatsJob) * std::max(nm, 1), 64);
  StatsJob* S = B.arena.hptr<StatsJob>(bg.stats_jobs);
  std::memset(static_cast<void*>(S), 0, sizeof(StatsJob) * std::max(nm, 1));
  for (int i = 0; i < nm; ++i) {
    StatsJob& j = S[i];
    const PcMat& a = B.X.mats[G.g0 + i];
    j.index = G.g0 + i;
    j.upd = B.wp<float2>(G.mb[i].upd);
    j.nslots = upd_slots(a.m, a.n);
    j.m = a.m;
    j.n = a.n;
    if (B.X.mode == 2) {
      j.flag_r = B.wp<int>(G.mb[i].R.flag);
      j.flag_l = B.X.foam ? nullptr : B.wp<int>(G.mb[i].L.flag);
      j.rho = B.wp<float>(G.mb[i].R.rho);
      j.fixed_bits = -1;
    } else {
      j.fixed_bits = B.X.mode == 1 ? (B.X.foam ? 1 : 3) : 0;
    }
  }
}

// The Cholesky kernel's shared memory exceeds the default 48 KB: opt in once per device.
mao_status chol_attr() {
  static std::mutex mu;
  static bool set[64] = {};
  int dev = 0;
  MAO_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MAO_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (!set[dev]) {
    MAO_CUDA_TRY(cudaFuncSetAttribute(qr_chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCholSmem));
    set[dev] = true;
  }
  return MAO_OK;
}

mao_status run_ops(const Ctx& X, uint8_t* arena_dev, const BuiltGroup& bg, DevStatus* status, cudaStream_t s) {
  Arena A;  // device view of the staged arena
  A.dev = arena_dev;
  const float bc1 = (float)(1.0 - std::pow((double)X.b1, (double)X.t));
  const float bc2 = (float)(1.0 - std::pow((double)X.b2, (double)X.t));
  for (size_t o = 0; o < bg.ops.size(); ++o) {
    const Op& op = bg.ops[o];
    if (op.kind == Op::GEMM) {
      MAO_TRY(table_launch(A, bg.staged[bg.gemm_of_op[o]], status, s));
      continue;
    }
    if (op.kind == Op::ZERO) {
      MAO_CUDA_TRY(cudaMemsetAsync(op.zero, 0, op.zero_bytes, s));
      continue;
    }
    if (op.blocks <= 0) continue;
    const int n = op.njobs;
    switch (op.kind) {
      case Op::EW: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, op.bytes);
        pc_momentum_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<EwJob>(op.jobs), n, X.b1);
        break;
      }
      case Op::SPLIT: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, op.bytes);
        pc_split_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<EwJob>(op.jobs), n);
        break;
      }
      case Op::ADAM: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, op.bytes);
        soap_adam_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<EwJob>(op.jobs), n, X.b2, 1.f / bc1, 1.f / bc2, X.eps);
        break;
      }
      case Op::KEYS: {
        LaunchScope ls(s, MAO_K_PC_SORT, 0.0, 0.0);
        pc_keys_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<SortJob>(op.jobs), n, X.rf.sort ? 1 : 0);
        break;
      }
      case Op::ARGSORT: {
        LaunchScope ls(s, MAO_K_PC_SORT, 0.0, 0.0);
        pc_argsort_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<SortJob>(op.jobs), n);
        break;
      }
      case Op::GATHER: {
        LaunchScope ls(s, MAO_K_PC_SORT, 0.0, 0.0);
        pc_gather_cols_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<GatherJob>(op.jobs), n);
        break;
      }
      case Op::VPERM: {
        LaunchScope ls(s, MAO_K_PC_SORT, 0.0, 0.0);
        soap_vperm_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<VPermJob>(op.jobs), n);
        break;
      }
      case Op::REDUCE: {
        LaunchScope ls(s, MAO_K_PC_PANEL, 0.0, 0.0);
        qr_gram_reduce_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<PanelJob>(op.jobs), op.any);
        break;
      }
      case Op::COEFRED: {
        LaunchScope ls(s, MAO_K_PC_QR_REDUCE, 0.0, 0.0);
        pc_coef_reduce_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<CoefJob>(op.jobs), n, op.any);
        break;
      }
      case Op::CHOL: {
        MAO_TRY(chol_attr());
        LaunchScope ls(s, MAO_K_PC_CHOL, 0.0, 0.0);
        qr_chol_kernel<<<op.blocks, 256, kCholSmem, s>>>(A.dptr<PanelJob>(op.jobs), op.any);
        break;
      }
      case Op::RC: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, op.bytes);
        foam_rc_partial_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<RcJob>(op.jobs), n);
        break;
      }
      case Op::TAU: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, 0.0);
        foam_tau_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<TauJob>(op.jobs), X.b2, 1.f / bc2, X.raw_trace);
        break;
      }
      case Op::FOAMN: {
        LaunchScope ls(s, MAO_K_PC_ELEMENTWISE, 0.0, op.bytes);
        foam_n_kernel<<<op.blocks, 256, 0, s>>>(A.dptr<EwJob>(op.jobs), n, 1.f / bc1, 1.f / bc2, X.eps);
        break;
      }
      case Op::CHECK: {
        LaunchScope ls(s, MAO_K_PC_CHECK, 0.0, 0.0);
        pc_check_kernel<<<n, 256, 0, s>>>(A.dptr<CheckJob>(op.jobs), X.rf.tol);
        break;
      }
      default:
        return MAO_ERR_INVALID_ARG;
    }
    MAO_CUDA_TRY(cudaGetLastError());
  }
  return MAO_OK;
}

// Workspace = status | scratch (max over groups) | arena (max over groups)
struct Layout {
  size_t scratch_off = 0, scratch = 0, arena_off = 0, arena = 0, total = 0;
};

// A whole step's launch plan for one (descriptor array, parameters, workspace).
struct StepPlan {
  Layout L;
  std::vector<GroupPlan> groups;
  std::vector<BuiltGroup> built;
};

// ws == nullptr: sizing only (layout), nothing encoded.
mao_status make_plan(const Ctx& X, uint8_t* ws, StepPlan& P) {
  make_groups(X, P.groups);
  Layout& L = P.L;
  L.scratch_off = align_up(kStatusBytes, 256);
  for (GroupPlan& g : P.groups) {
    plan_group_scratch(X, g, L.scratch_off);
    L.scratch = std::max(L.scratch, g.scratch);
  }
  L.arena_off = align_up(L.scratch_off + L.scratch, 256);
  P.built.assign(P.groups.size(), BuiltGroup());
  for (size_t gi = 0; gi < P.groups.size(); ++gi) {
    GroupPlan& g = P.groups[gi];
    Builder B(X, ws);
    if (ws) B.arena.dev = ws + L.arena_off;
    MAO_TRY(build_group(B, g));
    BuiltGroup& bg = P.built[gi];
    add_stats_jobs(B, g, bg);
    MAO_TRY(finish_build(B, bg));
    L.arena = std::max(L.arena, B.arena.host.size());
    if (ws) {
      bg.ops = std::move(B.ops);
      bg.gemm_of_op = std::move(B.gemm_of_op);
      bg.arena = std::move(B.arena.host);
    }
  }
  L.total = align_up(L.arena_off + L.arena + 64, 256);
  return MAO_OK;
}

// Recently used plans, keyed by the exact bytes of everything they depend on
// (descriptor array, hyper-parameters, refresh mode, workspace).  A training loop
// that calls the step with the same buffers every iteration builds its plan
// (tables, tensor maps) once per refresh mode.
struct PlanCache {
  std::mutex mu;
  std::list<std::pair<std::string, std::shared_ptr<StepPlan>>> lru;
  static constexpr size_t kMax = 16;
};
PlanCache& plan_cache() {
  static PlanCache c;
  return c;
}

std::string plan_key(const Ctx& X, const void* mats, size_t mats_bytes, const void* ws, size_t ws_bytes) {
  struct Head {
    int foam, count, mode, raw_trace;
    float b1, b2, eps, lr, wd;
    mao_refresh rf;
    const void* ws;
    size_t ws_bytes;
  } h;
  std::memset(&h, 0, sizeof(h));
  h.foam = X.foam;
  h.count = X.count;
  h.mode = X.mode;
  h.raw_trace = X.raw_trace;
  h.b1 = X.b1;
  h.b2 = X.b2;
  h.eps = X.eps;
  h.lr = X.lr;
  h.wd = X.wd;
  h.rf = X.rf;
  h.ws = ws;
  h.ws_bytes = ws_bytes;
  std::string k(reinterpret_cast<const char*>(&h), sizeof(h));
  k.append(reinterpret_cast<const char*>(mats), mats_bytes);
  return k;
}

mao_status run_step(const Ctx& X, const void* mats, size_t mats_bytes, void* workspace, size_t ws_bytes,
                    mao_stats* stats, cudaStream_t s) {
  if (workspace == nullptr) return MAO_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MAO_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const std::string key = plan_key(X, mats, mats_bytes, workspace, ws_bytes);
  std::shared_ptr<StepPlan> P;
  {
    PlanCache& C = plan_cache();
    std::lock_guard<std::mutex> lk(C.mu);
    for (auto it = C.lru.begin(); it != C.lru.end(); ++it)
      if (it->first == key) {
        P = it->second;
        C.lru.splice(C.lru.begin(), C.lru, it);
        break;
      }
  }
  if (!P) {
    StepPlan sizing;
    MAO_TRY(make_plan(X, nullptr, sizing));
    if (ws_bytes < sizing.L.total) return MAO_ERR_WORKSPACE;
    P = std::make_shared<StepPlan>();
    MAO_TRY(make_plan(X, ws, *P));
    if (P->L.total > sizing.L.total) return MAO_ERR_WORKSPACE;
    PlanCache& C = plan_cache();
    std::lock_guard<std::mutex> lk(C.mu);
    C.lru.emplace_front(key, P);
    if (C.lru.size() > PlanCache::kMax) C.lru.pop_back();
  }
  DeviceInfo* dev = nullptr;
  MAO_TRY(device_info(&dev));
  DevStatus* status = reinterpret_cast<DevStatus*>(ws);
  MAO_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(DevStatus), s));
  uint8_t* arena_dev = ws + P->L.arena_off;
  for (size_t gi = 0; gi < P->groups.size(); ++gi) {
    const GroupPlan& g = P->groups[gi];
    const BuiltGroup& bg = P->built[gi];
    // refresh flags, check ratios and failure counters start at zero
    MAO_CUDA_TRY(cudaMemsetAsync(ws + g.flags, 0, g.flags_bytes, s));
    MAO_CUDA_TRY(cudaMemcpyAsync(arena_dev, bg.arena.data(), bg.arena.size(), cudaMemcpyHostToDevice, s));
    MAO_TRY(run_ops(X, arena_dev, bg, status, s));
    if (stats) {
      const int nm = g.g1 - g.g0;
      LaunchScope ls(s, MAO_K_PC_STATS, 0.0, 0.0);
      pc_stats_kernel<<<nm, 256, 0, s>>>(reinterpret_cast<const StatsJob*>(arena_dev + bg.stats_jobs), stats,
                                         status);
      MAO_CUDA_TRY(cudaGetLastError());
    }
  }
  return MAO_OK;
}

// Bytes that serve every step of this descriptor set, whatever t: the maximum
// over the refresh modes the policy can take (plain steps, and refresh or check
// steps).
mao_status workspace_size(const Ctx& X, size_t* bytes) {
  int modes[2] = {0, 0};
  int nmodes = 1;
  if (X.rf.kind == MAO_REFRESH_EVERY_K) modes[nmodes++] = 1;
  if (X.rf.kind == MAO_REFRESH_ADAPTIVE) modes[nmodes++] = 2;
  size_t best = 0;
  for (int i = 0; i < nmodes; ++i) {
    Ctx Y = X;
    Y.mode = modes[i];
    StepPlan sizing;
    MAO_TRY(make_plan(Y, nullptr, sizing));
    best = std::max(best, sizing.L.total);
  }
  *bytes = best;
  return MAO_OK;
}

// ------------------------------------------------------------------ ABI helpers
mao_status soap_ctx(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p, std::vector<PcMat>& v,
                    Ctx& X, bool ptrs) {
  if (p == nullptr || count < 0 || (count > 0 && mats == nullptr)) return MAO_ERR_INVALID_ARG;
  MAO_TRY(check_refresh(p->refresh));
  MAO_TRY(check_hyper(p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t));
  v.resize(count);
  for (int i = 0; i < count; ++i) {
    const mao_soap_mat& a = mats[i];
    MAO_TRY(check_mat(a.m, a.n, a.g_dtype));
    if (ptrs) {
      const void* req[] = {a.W, a.G, a.M, a.V, a.L, a.R, a.QL, a.QR};
      for (const void* q : req) {
        if (q == nullptr) return MAO_ERR_INVALID_ARG;
        if (!aligned16(q)) return MAO_ERR_ALIGN;
      }
      if ((a.perm_L && !aligned16(a.perm_L)) || (a.perm_R && !aligned16(a.perm_R))) return MAO_ERR_ALIGN;
    }
    v[i] = PcMat{a.m, a.n, a.W, a.G, a.g_dtype == MAO_BF16, a.M, a.V, a.L, a.R, a.QL, a.QR, a.perm_L, a.perm_R,
                 nullptr, nullptr};
  }
  X = Ctx{false, v.data(), count, p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t, p->refresh, 0,
          host_refresh_mode(p->refresh, p->t)};
  return MAO_OK;
}

mao_status foam_ctx(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p, std::vector<PcMat>& v,
                    Ctx& X, bool ptrs) {
  if (p == nullptr || count < 0 || (count > 0 && mats == nullptr)) return MAO_ERR_INVALID_ARG;
  MAO_TRY(check_refresh(p->refresh));
  MAO_TRY(check_hyper(p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t));
  if (p->tau_raw_trace != 0 && p->tau_raw_trace != 1) return MAO_ERR_INVALID_ARG;
  v.resize(count);
  for (int i = 0; i < count; ++i) {
    const mao_foam_mat& a = mats[i];
    MAO_TRY(check_mat(a.m, a.n, a.g_dtype));
    if (ptrs) {
      const void* req[] = {a.W, a.G, a.M, a.r, a.c, a.R, a.QR};
      for (const void* q : req) {
        if (q == nullptr) return MAO_ERR_INVALID_ARG;
        if (!aligned16(q)) return MAO_ERR_ALIGN;
      }
      if (a.perm_R && !aligned16(a.perm_R)) return MAO_ERR_ALIGN;
    }
    v[i] = PcMat{a.m, a.n, a.W, a.G, a.g_dtype == MAO_BF16, a.M, nullptr, nullptr, a.R, nullptr, a.QR, nullptr,
                 a.perm_R, a.r, a.c};
  }
  X = Ctx{true, v.data(), count, p->beta1, p->beta2, p->eps, p->lr, p->wd, p->t, p->refresh, p->tau_raw_trace,
          host_refresh_mode(p->refresh, p->t)};
  return MAO_OK;
}

}  // namespace

extern "C" mao_status mao_soap_workspace_size(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p,
                                              size_t* bytes) {
  if (bytes == nullptr) return MAO_ERR_INVALID_ARG;
  std::vector<PcMat> v;
  Ctx X;
  MAO_TRY(soap_ctx(mats, count, p, v, X, false));
  return workspace_size(X, bytes);
}

extern "C" mao_status mao_soap_step(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p,
                                   void* workspace, size_t ws_bytes, mao_stats* stats, mao_stream_t stream) {
  std::vector<PcMat> v;
  Ctx X;
  MAO_TRY(soap_ctx(mats, count, p, v, X, true));
  if (count == 0) return MAO_OK;
  if (stats != nullptr && !aligned16(stats)) return MAO_ERR_ALIGN;
  return run_step(X, mats, sizeof(mao_soap_mat) * (size_t)count, workspace, ws_bytes, stats,
                  reinterpret_cast<cudaStream_t>(stream));
}

extern "C" mao_status mao_foam_workspace_size(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p,
                                              size_t* bytes) {
  if (bytes == nullptr) return MAO_ERR_INVALID_ARG;
  std::vector<PcMat> v;
  Ctx X;
  MAO_TRY(foam_ctx(mats, count, p, v, X, false));
  return workspace_size(X, bytes);
}

extern "C" mao_status mao_foam_step(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p,
                                   void* workspace, size_t ws_bytes, mao_stats* stats, mao_stream_t stream) {
  std::vector<PcMat> v;
  Ctx X;
  MAO_TRY(foam_ctx(mats, count, p, v, X, true));
  if (count == 0) return MAO_OK;
  if (stats != nullptr && !aligned16(stats)) return MAO_ERR_ALIGN;
  return run_step(X, mats, sizeof(mao_foam_mat) * (size_t)count, workspace, ws_bytes, stats,
                  reinterpret_cast<cudaStream_t>(stream));
}
