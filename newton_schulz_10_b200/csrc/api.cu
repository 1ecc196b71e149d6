// C ABI of libmuon.so (declared in include/muon.h): argument validation,
// workspace layout and the order of kernel launches for each entry point.
#include <atomic>
#include <cmath>
#include <cstring>
#include <vector>

#include "internal.h"
#include "rowops.cuh"

namespace muon {

Counters& counters() {
  static thread_local Counters c;
  return c;
}

namespace {

std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};

// Optional per-phase CUDA events of a profiled step.
struct PhaseEvents {
  cudaEvent_t ev[5] = {};
  bool on = false;
  void mark(int i, cudaStream_t s) {
    if (on) cudaEventRecord(ev[i], s);
  }
};

uint64_t timeout_ns() { return g_timeout_ns.load(); }

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool op_of(muon_dtype d, Op* t) {
  switch (d) {
    case MUON_BF16: *t = Op::BF16; return true;
    case MUON_F16: *t = Op::F16; return true;
    case MUON_F32: *t = Op::F32; return true;
  }
  return false;
}

muon_status check_ns(const muon_ns_params* p) {
  if (!p) return MUON_ERR_INVALID_ARG;
  if (p->T < 1 || p->T > MUON_MAX_T) return MUON_ERR_INVALID_ARG;
  if (!(p->norm_eps >= 0.f) || !std::isfinite(p->norm_eps)) return MUON_ERR_INVALID_ARG;
  if (p->restart_at < 0 || (p->gram != 0 && p->gram != 1)) return MUON_ERR_INVALID_ARG;
  for (int t = 0; t < p->T; ++t)
    for (int j = 0; j < 3; ++j)
      if (!std::isfinite(p->coeffs[t][j])) return MUON_ERR_INVALID_ARG;
  Op t;
  if (!op_of(p->compute, &t)) return MUON_ERR_DTYPE;
  return MUON_OK;
}

// Storage scale of the operand copy of X_0: stored = kappa * X_0. fp16 keeps
// rows of unit average norm so entries stay in its normal range.
float kappa_for(Op t, int64_t n) { return t == Op::F16 ? std::sqrt((float)n) : 1.f; }
float rho_for(Op t, int64_t n) { return t == Op::F16 ? (float)n : 1.f; }

// Workspace layout of one shape group's NS buffers, starting at `off`.
struct GroupBufs {
  size_t X[2];
  size_t nb[4];
  size_t part, part_bytes;
};

size_t layout_group(int64_t rows, int64_t cols, int count, Op t, const muon_ns_params* p, size_t off,
                    GroupBufs* b) {
  const int64_t n = rows < cols ? rows : cols;
  const size_t es = op_size(t);
  const size_t xbytes = up((size_t)count * rows * pad_ld(cols) * es);
  const size_t nbytes = up((size_t)count * n * pad_ld(n) * es);
  for (int i = 0; i < 2; ++i) {
    if (b) b->X[i] = off;
    off += xbytes;
  }
  const int nw = ns_work_buffers(p);
  for (int i = 0; i < nw; ++i) {
    if (b) b->nb[i] = off;
    off += nbytes;
  }
  const size_t pb = t == Op::F32 ? 0 : tc_split_scratch(n, rows < cols ? cols : rows, count);
  if (b) {
    b->part = off;
    b->part_bytes = pb;
  }
  return off + up(pb);
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

#define TRY(x)                        \
  do {                                \
    muon_status _r = (x);             \
    if (_r != MUON_OK) return _r;     \
  } while (0)

// Launch a row kernel over any number of matrices, kMaxRowMats at a time.
template <typename F>
muon_status row_batches(const std::vector<RowMat>& mats, const RowLaunch& proto, F launch) {
  for (size_t b0 = 0; b0 < mats.size(); b0 += kMaxRowMats) {
    RowLaunch L = proto;
    L.count = 0;
    for (size_t i = b0; i < mats.size() && L.count < kMaxRowMats; ++i) L.m[L.count++] = mats[i];
    TRY(launch(L));
  }
  return MUON_OK;
}

// ---------------------------------------------------------------------------
// ns_polar / gram_ns_polar
// ---------------------------------------------------------------------------

struct PolarPlan {
  size_t s, xscale, rsum, ctr;
  GroupBufs g;
  size_t total;
};

PolarPlan plan_polar(int64_t rows, int64_t cols, Op t, const muon_ns_params* p) {
  PolarPlan q;
  size_t off = kAlign;  // status word
  q.s = off; off += kAlign;
  q.xscale = off; off += kAlign;
  q.rsum = off; off += up((size_t)rows * sizeof(double));
  q.ctr = off; off += up(ns_counter_words(p, 1) * sizeof(unsigned));
  q.total = layout_group(rows, cols, 1, t, p, off, &q.g);
  return q;
}

muon_status polar_impl(const void* X, muon_dtype x_dtype, void* O, muon_dtype o_dtype, int64_t rows, int64_t cols,
                       const muon_ns_params* p, int gram, void* ws, size_t ws_bytes, void* stream) {
  TRY(check_ns(p));
  if (rows < 0 || cols < 0 || rows > INT32_MAX || cols > INT32_MAX) return MUON_ERR_SHAPE;
  if (x_dtype != MUON_F32 && x_dtype != MUON_BF16) return MUON_ERR_DTYPE;
  if (o_dtype != MUON_F32 && o_dtype != MUON_BF16) return MUON_ERR_DTYPE;
  if (rows == 0 || cols == 0) return MUON_OK;
  if (!X || !O || !ws) return X && O ? MUON_ERR_WORKSPACE : MUON_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(O) || !aligned16(ws)) return MUON_ERR_ALIGN;
  muon_ns_params pp = *p;
  pp.gram = gram;
  Op t;
  op_of(pp.compute, &t);
  const PolarPlan q = plan_polar(rows, cols, t, &pp);
  if (ws_bytes < q.total) return MUON_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(ws, 0);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;

  const int64_t n = rows < cols ? rows : cols;
  const float kappa = kappa_for(t, n);
  const Op xt = x_dtype == MUON_F32 ? Op::F32 : Op::BF16;
  RowMat m{};
  m.src = X;
  m.rsum = at<double>(ws, q.rsum);
  m.rows = rows;
  m.cols = cols;
  m.ntask = (int32_t)rows;
  RowLaunch L{};
  L.status = status;
  L.count = 1;
  L.m[0] = m;
  TRY(launch_row_stats(L, xt, s));
  NormOut no{m.rsum, rows, at<float>(ws, q.s), at<float>(ws, q.xscale), 1.f / kappa};
  TRY(launch_norm_finalize(&no, 1, pp.norm_eps, status, s));
  m.X = at<void>(ws, q.g.X[0]);
  m.ldx = pad_ld(cols);
  m.mult = at<float>(ws, q.s);
  m.kappa = kappa;
  L.m[0] = m;
  TRY(launch_cast_rows(L, xt, t, s));

  NsGroup g{};
  g.rows = rows;
  g.cols = cols;
  g.count = 1;
  g.X[0] = at<void>(ws, q.g.X[0]);
  g.X[1] = at<void>(ws, q.g.X[1]);
  g.cur = 0;
  g.xscale = at<float>(ws, q.xscale);
  for (int i = 0; i < ns_work_buffers(&pp); ++i) g.nb[i] = at<void>(ws, q.g.nb[i]);
  g.rho = rho_for(t, n);
  g.part = q.g.part_bytes ? at<float>(ws, q.g.part) : nullptr;
  g.part_bytes = q.g.part_bytes;
  TRY(ns_run(t, &g, 1, &pp, status, timeout_ns(), s, at<unsigned>(ws, q.ctr)));
  return launch_copy_out(g.X[g.cur], t, pad_ld(cols), O, o_dtype == MUON_F32 ? Op::F32 : Op::BF16, rows, cols,
                         status, s);
}

// ---------------------------------------------------------------------------
// muon_step
// ---------------------------------------------------------------------------

struct StepPlan {
  struct Mat {
    int group, gidx;
    int64_t rows_eff;  // rows orthogonalised (k for Dion3)
    size_t row_base;   // into rsum / rkey (stored rows)
    size_t task_base;  // into rscale / idx (rows_eff)
  };
  struct Grp {
    int64_t rows, cols;
    int count;
    int slot0;  // first per-matrix scalar slot of the group (slots are group-major)
    GroupBufs b;
  };
  std::vector<Mat> mats;
  std::vector<Grp> groups;
  size_t s, xscale, rsum, rkey, rscale, idx, ctr, total;
};

// Which fields of each muon_matrix an entry point reads (NEED_NONE: shapes
// only, for the size queries).
enum : int { NEED_NONE = 0, NEED_W = 1, NEED_M = 2, NEED_G = 4, NEED_V = 8, NEED_ALL = 15 };

muon_status check_step(const muon_matrix* mats, int32_t count, const muon_params* p, int need = NEED_ALL) {
  if (!p || count < 0 || (count > 0 && !mats)) return MUON_ERR_INVALID_ARG;
  TRY(check_ns(&p->ns));
  if (!std::isfinite(p->mu) || !std::isfinite(p->lr)) return MUON_ERR_INVALID_ARG;
  if (p->normuon != 0 && p->normuon != 1) return MUON_ERR_INVALID_ARG;
  if (p->normuon && (!std::isfinite(p->beta2) || !(p->normuon_eps >= 0.f) || !std::isfinite(p->normuon_eps)))
    return MUON_ERR_INVALID_ARG;
  if (p->dion3 != 0 && p->dion3 != 1) return MUON_ERR_INVALID_ARG;
  if (p->dion3 && (p->frac_num <= 0 || p->frac_den <= 0 || p->frac_num > p->frac_den)) return MUON_ERR_INVALID_ARG;
  if (p->select_norm != MUON_NORM_L1 && p->select_norm != MUON_NORM_L2) return MUON_ERR_INVALID_ARG;
  if (p->dev_status && (reinterpret_cast<uintptr_t>(p->dev_status) & 3u)) return MUON_ERR_ALIGN;
  for (int i = 0; i < count; ++i) {
    const muon_matrix& m = mats[i];
    if (m.rows < 0 || m.cols < 0 || m.rows > INT32_MAX || m.cols > INT32_MAX) return MUON_ERR_SHAPE;
    if (m.rows == 0 || m.cols == 0) continue;
    if (((need & NEED_W) && !m.W) || ((need & NEED_M) && !m.M) || ((need & NEED_G) && !m.G) ||
        ((need & NEED_V) && p->normuon && !m.v))
      return MUON_ERR_INVALID_ARG;
    if (((need & NEED_W) && !aligned16(m.W)) || ((need & NEED_M) && !aligned16(m.M)) ||
        ((need & NEED_G) && !aligned16(m.G)) || (m.v && (reinterpret_cast<uintptr_t>(m.v) & 3u)))
      return MUON_ERR_ALIGN;
  }
  return MUON_OK;
}

StepPlan plan_step(const muon_matrix* mats, int32_t count, const muon_params* p) {
  StepPlan q;
  Op t;
  op_of(p->ns.compute, &t);
  size_t rows_total = 0, tasks_total = 0;
  for (int i = 0; i < count; ++i) {
    const muon_matrix& m = mats[i];
    StepPlan::Mat e{};
    e.group = -1;
    if (m.rows == 0 || m.cols == 0) {
      q.mats.push_back(e);
      continue;
    }
    e.rows_eff = p->dion3 ? muon_rows_for_fraction(m.rows, p->frac_num, p->frac_den) : m.rows;
    e.row_base = rows_total;
    e.task_base = tasks_total;
    rows_total += m.rows;
    tasks_total += e.rows_eff;
    for (size_t gi = 0; gi < q.groups.size(); ++gi)
      if (q.groups[gi].rows == e.rows_eff && q.groups[gi].cols == m.cols) e.group = (int)gi;
    if (e.group < 0) {
      q.groups.push_back(StepPlan::Grp{e.rows_eff, m.cols, 0, 0, {}});
      e.group = (int)q.groups.size() - 1;
    }
    e.gidx = q.groups[e.group].count++;
    q.mats.push_back(e);
  }
  int slot = 0;
  for (auto& g : q.groups) {
    g.slot0 = slot;
    slot += g.count;
  }
  size_t off = kAlign;  // status word
  q.s = off; off += up(count * sizeof(float) + 4);
  q.xscale = off; off += up(count * sizeof(float) + 4);
  q.rsum = off; off += up(rows_total * sizeof(double) + 8);
  q.rkey = off; off += up(rows_total * sizeof(double) + 8);
  q.rscale = off; off += up(tasks_total * sizeof(float) + 4);
  q.idx = off; off += up(tasks_total * sizeof(int32_t) + 4);
  // fused-chain completion counters: each batch of up to kMaxGemmGroups
  // shape groups runs its own chain, so the largest batch's matrices bound it
  int64_t chain_mats = 0;
  for (size_t g0 = 0; g0 < q.groups.size(); g0 += kMaxGemmGroups) {
    int64_t m = 0;
    for (size_t gi = g0; gi < q.groups.size() && gi < g0 + kMaxGemmGroups; ++gi) m += q.groups[gi].count;
    chain_mats = m > chain_mats ? m : chain_mats;
  }
  q.ctr = off; off += up(ns_counter_words(&p->ns, chain_mats) * sizeof(unsigned) + 4);
  for (auto& g : q.groups) off = layout_group(g.rows, g.cols, g.count, t, &p->ns, off, &g.b);
  q.total = off;
  return q;
}

// True when a (valid) step has no matrix with work: step_impl then queues nothing.
bool plan_step_empty(const muon_matrix* mats, int32_t count) {
  for (int i = 0; i < count; ++i)
    if (mats[i].rows > 0 && mats[i].cols > 0) return false;
  return true;
}

muon_status step_impl(const muon_matrix* mats, int32_t count, const muon_params* p, void* ws, size_t ws_bytes,
                      cudaStream_t s, PhaseEvents& E, muon_step_profile* prof) {
  TRY(check_step(mats, count, p));
  const StepPlan q = plan_step(mats, count, p);
  if (q.groups.empty()) return MUON_OK;
  if (!ws) return MUON_ERR_WORKSPACE;
  if (!aligned16(ws)) return MUON_ERR_ALIGN;
  if (ws_bytes < q.total) return MUON_ERR_WORKSPACE;
  Op t;
  op_of(p->ns.compute, &t);
  const size_t es = op_size(t);
  int* status = p->dev_status ? p->dev_status : at<int>(ws, 0);
  E.mark(0, s);
  if (!p->dev_status && cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;
  if (prof) {
    // compulsory HBM bytes of the memory-bound phases
    double pro = 0, upd = 0;
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const double el = (double)mats[i].rows * mats[i].cols, sel = (double)e.rows_eff * mats[i].cols;
      const bool one = !p->dion3 && t == Op::BF16;
      pro += 12.0 * el + (one ? es * el : (4.0 + es) * sel);
      upd += (8.0 + es) * sel + (p->dion3 ? 8.0 * sel : 0.0) + (p->normuon ? es * sel : 0.0);
    }
    prof->bytes_prologue = pro;
    prof->bytes_update = upd;
  }

  // Where the operand copy of matrix i lives: slot gidx of its group's X[0].
  auto xslot = [&](int i) -> void* {
    const StepPlan::Mat& e = q.mats[i];
    const StepPlan::Grp& g = q.groups[e.group];
    return at<char>(ws, g.b.X[0]) + (size_t)e.gidx * g.rows * pad_ld(g.cols) * es;
  };
  // Single pass (cast inside the momentum kernel, Frobenius scale folded into
  // the first GEMM epilogues) for plain Muon in bf16; otherwise the scaled
  // cast is a second pass once the norm is known.
  const bool one_pass = !p->dion3 && t == Op::BF16;

  // 1. momentum, fused row statistics (+ cast)
  std::vector<RowMat> rm;
  for (int i = 0; i < count; ++i) {
    const StepPlan::Mat& e = q.mats[i];
    if (e.group < 0) continue;
    RowMat r{};
    r.M = mats[i].M;
    r.G = mats[i].G;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.rsum = at<double>(ws, q.rsum) + e.row_base;
    r.rkey = p->dion3 ? at<double>(ws, q.rkey) + e.row_base : nullptr;
    r.X = one_pass ? xslot(i) : nullptr;
    r.ldx = pad_ld(mats[i].cols);
    r.ntask = (int32_t)mats[i].rows;
    rm.push_back(r);
  }
  RowLaunch proto{};
  proto.mu = p->mu;
  proto.lr = p->lr;
  proto.mode = p->dion3 ? MOM_DION3 : MOM_MUON;
  proto.key_l2 = p->select_norm == MUON_NORM_L2;
  proto.status = status;
  TRY(row_batches(rm, proto, [&](RowLaunch& L) { return launch_momentum_rows(L, t, s); }));

  // 2. Frobenius scale (+ selection, + cast)
  float* sc = at<float>(ws, q.s);
  float* xs = at<float>(ws, q.xscale);
  int32_t* idx = at<int32_t>(ws, q.idx);
  std::vector<RowMat> cm;
  if (!p->dion3) {
    std::vector<NormOut> no;
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const int64_t n = mats[i].rows < mats[i].cols ? mats[i].rows : mats[i].cols;
      const int sl = q.groups[e.group].slot0 + e.gidx;
      no.push_back(NormOut{at<double>(ws, q.rsum) + e.row_base, mats[i].rows, sc + sl, xs + sl,
                           one_pass ? -1.f : 1.f / kappa_for(t, n)});
    }
    TRY(launch_norm_finalize(no.data(), (int)no.size(), p->ns.norm_eps, status, s));
  } else {
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const int64_t n = e.rows_eff < mats[i].cols ? e.rows_eff : mats[i].cols;
      const int sl = q.groups[e.group].slot0 + e.gidx;
      TRY(launch_select(at<double>(ws, q.rkey) + e.row_base, at<double>(ws, q.rsum) + e.row_base, mats[i].rows,
                        e.rows_eff, idx + e.task_base, sc + sl, xs + sl, p->ns.norm_eps, 1.f / kappa_for(t, n),
                        status, s));
    }
  }
  if (!one_pass) {
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const int64_t n = e.rows_eff < mats[i].cols ? e.rows_eff : mats[i].cols;
      RowMat r{};
      r.src = mats[i].M;
      r.X = xslot(i);
      r.idx = p->dion3 ? idx + e.task_base : nullptr;
      r.mult = sc + q.groups[e.group].slot0 + e.gidx;
      r.kappa = kappa_for(t, n);
      r.rows = mats[i].rows;
      r.cols = mats[i].cols;
      r.ldx = pad_ld(mats[i].cols);
      r.ntask = (int32_t)e.rows_eff;
      cm.push_back(r);
    }
    TRY(row_batches(cm, proto, [&](RowLaunch& L) { return launch_cast_rows(L, Op::F32, t, s); }));
  }

  // 3. Newton-Schulz, up to kMaxGemmGroups shape groups per launch
  std::vector<NsGroup> ns(q.groups.size());
  for (size_t gi = 0; gi < q.groups.size(); ++gi) {
    const StepPlan::Grp& g = q.groups[gi];
    NsGroup& n = ns[gi];
    n.rows = g.rows;
    n.cols = g.cols;
    n.count = g.count;
    n.X[0] = at<void>(ws, g.b.X[0]);
    n.X[1] = at<void>(ws, g.b.X[1]);
    n.cur = 0;
    for (int k = 0; k < ns_work_buffers(&p->ns); ++k) n.nb[k] = at<void>(ws, g.b.nb[k]);
    n.rho = rho_for(t, g.rows < g.cols ? g.rows : g.cols);
    n.part = g.b.part_bytes ? at<float>(ws, g.b.part) : nullptr;
    n.part_bytes = g.b.part_bytes;
  }
  for (size_t gi = 0; gi < q.groups.size(); ++gi) ns[gi].xscale = xs + q.groups[gi].slot0;
  E.mark(1, s);
  for (size_t g0 = 0; g0 < ns.size(); g0 += kMaxGemmGroups) {
    const int ng = (int)(ns.size() - g0 < (size_t)kMaxGemmGroups ? ns.size() - g0 : kMaxGemmGroups);
    TRY(ns_run(t, ns.data() + g0, ng, &p->ns, status, timeout_ns(), s, at<unsigned>(ws, q.ctr)));
  }
  E.mark(2, s);

  // 4. NorMuon row scales, 5. update
  auto oslot = [&](int i) -> void* {
    const StepPlan::Mat& e = q.mats[i];
    const StepPlan::Grp& g = q.groups[e.group];
    return static_cast<char*>(ns[e.group].X[ns[e.group].cur]) + (size_t)e.gidx * g.rows * pad_ld(g.cols) * es;
  };
  float* rscale = at<float>(ws, q.rscale);
  std::vector<RowMat> um;
  for (int i = 0; i < count; ++i) {
    const StepPlan::Mat& e = q.mats[i];
    if (e.group < 0) continue;
    RowMat r{};
    r.W = mats[i].W;
    r.M = mats[i].M;
    r.v = mats[i].v;
    r.X = oslot(i);
    r.ldx = pad_ld(mats[i].cols);
    r.idx = p->dion3 ? idx + e.task_base : nullptr;
    r.rscale = p->normuon ? rscale + e.task_base : nullptr;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.ntask = (int32_t)e.rows_eff;
    um.push_back(r);
  }
  if (p->normuon) {
    TRY(row_batches(um, proto, [&](RowLaunch& L) { return launch_normuon_rows(L, t, s); }));
    std::vector<NormuonMat> nm;
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      nm.push_back(NormuonMat{rscale + e.task_base, e.rows_eff, mats[i].cols, mats[i].v,
                              p->dion3 ? idx + e.task_base : nullptr});
    }
    TRY(launch_normuon_finalize_batched(nm.data(), (int)nm.size(), p->beta2, p->normuon_eps, status, s));
  }
  E.mark(3, s);
  RowLaunch up_proto = proto;
  up_proto.mode = p->dion3 ? 1 : 0;
  TRY(row_batches(um, up_proto, [&](RowLaunch& L) { return launch_update_rows(L, t, s); }));
  E.mark(4, s);
  return MUON_OK;
}

// The middle of a step, on momentum already updated (muon_orthogonalize):
// norms / selection, the operand cast, the Newton-Schulz chain and NorMuon,
// exactly as step_impl computes them, with the orthogonalised rows, their
// update scales and the selection written to caller buffers.
muon_status ortho_impl(const muon_matrix* mats, int32_t count, const muon_params* p, void* const* O,
                       float* const* row_scale, int32_t* const* selected, void* ws, size_t ws_bytes, cudaStream_t s) {
  TRY(check_step(mats, count, p, NEED_M | NEED_V));
  if (count > 0 && (!O || !row_scale || (p->dion3 && !selected))) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (mats[i].rows == 0 || mats[i].cols == 0) continue;
    if (!O[i] || !row_scale[i] || (p->dion3 && !selected[i])) return MUON_ERR_INVALID_ARG;
    if (!aligned16(O[i]) || (reinterpret_cast<uintptr_t>(row_scale[i]) & 3u) ||
        (p->dion3 && (reinterpret_cast<uintptr_t>(selected[i]) & 3u)))
      return MUON_ERR_ALIGN;
  }
  const StepPlan q = plan_step(mats, count, p);
  if (q.groups.empty()) return MUON_OK;
  if (!ws) return MUON_ERR_WORKSPACE;
  if (!aligned16(ws)) return MUON_ERR_ALIGN;
  if (ws_bytes < q.total) return MUON_ERR_WORKSPACE;
  Op t;
  op_of(p->ns.compute, &t);
  const size_t es = op_size(t);
  int* status = p->dev_status ? p->dev_status : at<int>(ws, 0);
  if (!p->dev_status && cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;
  auto xslot = [&](int i) -> void* {
    const StepPlan::Mat& e = q.mats[i];
    const StepPlan::Grp& g = q.groups[e.group];
    return at<char>(ws, g.b.X[0]) + (size_t)e.gidx * g.rows * pad_ld(g.cols) * es;
  };
  // muon_step casts plain-Muon bf16 operands unscaled (the Frobenius scale
  // enters the first GEMM epilogues); the same here, so the operands agree
  const bool unscaled = !p->dion3 && t == Op::BF16;
  RowLaunch proto{};
  proto.mu = p->mu;
  proto.lr = p->lr;
  proto.key_l2 = p->select_norm == MUON_NORM_L2;
  proto.status = status;

  // 1. row sums of squares and selection keys of the momentum
  std::vector<RowMat> rm;
  for (int i = 0; i < count; ++i) {
    const StepPlan::Mat& e = q.mats[i];
    if (e.group < 0) continue;
    RowMat r{};
    r.src = mats[i].M;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.rsum = at<double>(ws, q.rsum) + e.row_base;
    r.rkey = p->dion3 ? at<double>(ws, q.rkey) + e.row_base : nullptr;
    r.ntask = (int32_t)mats[i].rows;
    rm.push_back(r);
  }
  TRY(row_batches(rm, proto, [&](RowLaunch& L) { return launch_row_stats(L, Op::F32, s); }));

  // 2. Frobenius scale (+ selection), then the operand cast
  float* sc = at<float>(ws, q.s);
  float* xs = at<float>(ws, q.xscale);
  int32_t* idx = at<int32_t>(ws, q.idx);
  if (!p->dion3) {
    std::vector<NormOut> no;
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const int64_t n = mats[i].rows < mats[i].cols ? mats[i].rows : mats[i].cols;
      const int sl = q.groups[e.group].slot0 + e.gidx;
      no.push_back(NormOut{at<double>(ws, q.rsum) + e.row_base, mats[i].rows, sc + sl, xs + sl,
                           unscaled ? -1.f : 1.f / kappa_for(t, n)});
    }
    TRY(launch_norm_finalize(no.data(), (int)no.size(), p->ns.norm_eps, status, s));
  } else {
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      const int64_t n = e.rows_eff < mats[i].cols ? e.rows_eff : mats[i].cols;
      const int sl = q.groups[e.group].slot0 + e.gidx;
      TRY(launch_select(at<double>(ws, q.rkey) + e.row_base, at<double>(ws, q.rsum) + e.row_base, mats[i].rows,
                        e.rows_eff, idx + e.task_base, sc + sl, xs + sl, p->ns.norm_eps, 1.f / kappa_for(t, n),
                        status, s));
    }
  }
  std::vector<RowMat> cm;
  for (int i = 0; i < count; ++i) {
    const StepPlan::Mat& e = q.mats[i];
    if (e.group < 0) continue;
    const int64_t n = e.rows_eff < mats[i].cols ? e.rows_eff : mats[i].cols;
    RowMat r{};
    r.src = mats[i].M;
    r.X = xslot(i);
    r.idx = p->dion3 ? idx + e.task_base : nullptr;
    r.mult = unscaled ? nullptr : sc + q.groups[e.group].slot0 + e.gidx;
    r.kappa = unscaled ? 1.f : kappa_for(t, n);
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.ldx = pad_ld(mats[i].cols);
    r.ntask = (int32_t)e.rows_eff;
    cm.push_back(r);
  }
  TRY(row_batches(cm, proto, [&](RowLaunch& L) { return launch_cast_rows(L, Op::F32, t, s); }));

  // 3. Newton-Schulz
  std::vector<NsGroup> ns(q.groups.size());
  for (size_t gi = 0; gi < q.groups.size(); ++gi) {
    const StepPlan::Grp& g = q.groups[gi];
    NsGroup& n = ns[gi];
    n.rows = g.rows;
    n.cols = g.cols;
    n.count = g.count;
    n.X[0] = at<void>(ws, g.b.X[0]);
    n.X[1] = at<void>(ws, g.b.X[1]);
    n.cur = 0;
    for (int k = 0; k < ns_work_buffers(&p->ns); ++k) n.nb[k] = at<void>(ws, g.b.nb[k]);
    n.rho = rho_for(t, g.rows < g.cols ? g.rows : g.cols);
    n.part = g.b.part_bytes ? at<float>(ws, g.b.part) : nullptr;
    n.part_bytes = g.b.part_bytes;
    n.xscale = xs + g.slot0;
  }
  for (size_t g0 = 0; g0 < ns.size(); g0 += kMaxGemmGroups) {
    const int ng = (int)(ns.size() - g0 < (size_t)kMaxGemmGroups ? ns.size() - g0 : kMaxGemmGroups);
    TRY(ns_run(t, ns.data() + g0, ng, &p->ns, status, timeout_ns(), s, at<unsigned>(ws, q.ctr)));
  }

  // 4. NorMuon row scales, 5. the rows, scales and selection to the caller
  float* rscale = at<float>(ws, q.rscale);
  std::vector<RowMat> um;
  for (int i = 0; i < count; ++i) {
    const StepPlan::Mat& e = q.mats[i];
    if (e.group < 0) continue;
    const StepPlan::Grp& g = q.groups[e.group];
    RowMat r{};
    r.v = mats[i].v;
    r.X = static_cast<char*>(ns[e.group].X[ns[e.group].cur]) + (size_t)e.gidx * g.rows * pad_ld(g.cols) * es;
    r.ldx = pad_ld(mats[i].cols);
    r.idx = p->dion3 ? idx + e.task_base : nullptr;
    r.rscale = p->normuon ? rscale + e.task_base : nullptr;
    r.out = O[i];
    r.out_scale = row_scale[i];
    r.out_flag = p->dion3 ? selected[i] : nullptr;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.ntask = (int32_t)e.rows_eff;
    um.push_back(r);
  }
  if (p->normuon) {
    TRY(row_batches(um, proto, [&](RowLaunch& L) { return launch_normuon_rows(L, t, s); }));
    std::vector<NormuonMat> nm;
    for (int i = 0; i < count; ++i) {
      const StepPlan::Mat& e = q.mats[i];
      if (e.group < 0) continue;
      nm.push_back(NormuonMat{rscale + e.task_base, e.rows_eff, mats[i].cols, mats[i].v,
                              p->dion3 ? idx + e.task_base : nullptr});
    }
    TRY(launch_normuon_finalize_batched(nm.data(), (int)nm.size(), p->beta2, p->normuon_eps, status, s));
  }
  if (p->dion3) {
    // rows that are not selected: zero update, scale 0, flag 0
    for (int i = 0; i < count; ++i) {
      if (q.mats[i].group < 0) continue;
      const size_t rows = (size_t)mats[i].rows;
      if (cudaMemsetAsync(O[i], 0, rows * mats[i].cols * es, s) != cudaSuccess ||
          cudaMemsetAsync(row_scale[i], 0, rows * sizeof(float), s) != cudaSuccess ||
          cudaMemsetAsync(selected[i], 0, rows * sizeof(int32_t), s) != cudaSuccess)
        return MUON_ERR_CUDA;
    }
  }
  return row_batches(um, proto, [&](RowLaunch& L) { return launch_scatter_rows(L, t, s); });
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" {

void muon_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs); }

void muon_set_gemm_cta_pair(int32_t enable) { set_gemm_pair_mode(enable ? 2 : 1); }

void muon_set_gemm_chain(int32_t enable) { set_gemm_chain(enable); }

const char* muon_status_str(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_SHAPE: return "MUON_ERR_SHAPE";
    case MUON_ERR_DTYPE: return "MUON_ERR_DTYPE";
    case MUON_ERR_ALIGN: return "MUON_ERR_ALIGN";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_NONFINITE: return "MUON_ERR_NONFINITE";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
  }
  return "MUON_ERR_UNKNOWN";
}

int64_t muon_rows_for_fraction(int64_t n, int32_t f_num, int32_t f_den) {
  if (n < 0 || f_num <= 0 || f_den <= 0 || f_num > f_den) return -1;
  return (n * (int64_t)f_num + f_den - 1) / f_den;
}

void muon_ns_params_default(muon_ns_params* p) {
  if (!p) return;
  memset(p, 0, sizeof(*p));
  p->T = 5;
  for (int t = 0; t < MUON_MAX_T; ++t) {
    p->coeffs[t][0] = 3.4445f;
    p->coeffs[t][1] = -4.7750f;
    p->coeffs[t][2] = 2.0315f;
  }
  p->norm_eps = 1e-7f;
  p->gram = 0;
  p->restart_at = 3;
  p->compute = MUON_BF16;
}

size_t muon_ns_workspace_size(int64_t rows, int64_t cols, const muon_ns_params* p) {
  if (check_ns(p) != MUON_OK || rows < 0 || cols < 0) return 0;
  Op t;
  op_of(p->compute, &t);
  muon_ns_params pp = *p;
  pp.gram = 1;  // room for either chain
  return plan_polar(rows, cols, t, &pp).total;
}

muon_status ns_polar(const void* X, muon_dtype x_dtype, void* O, muon_dtype o_dtype, int64_t rows, int64_t cols,
                     const muon_ns_params* p, void* ws, size_t ws_bytes, void* stream) {
  if (!p) return MUON_ERR_INVALID_ARG;
  return polar_impl(X, x_dtype, O, o_dtype, rows, cols, p, p->gram, ws, ws_bytes, stream);
}

muon_status gram_ns_polar(const void* X, muon_dtype x_dtype, void* O, muon_dtype o_dtype, int64_t rows,
                          int64_t cols, const muon_ns_params* p, void* ws, size_t ws_bytes, void* stream) {
  return polar_impl(X, x_dtype, O, o_dtype, rows, cols, p, 1, ws, ws_bytes, stream);
}

muon_status normuon_scale(const void* O, muon_dtype o_dtype, int64_t k, int64_t m, float* v, const int32_t* rows,
                          float beta2, float eps, float* row_scale_out, int32_t* dev_status, void* stream) {
  if (k < 0 || m < 0 || k > INT32_MAX || m > INT32_MAX) return MUON_ERR_SHAPE;
  if (o_dtype != MUON_F32 && o_dtype != MUON_BF16) return MUON_ERR_DTYPE;
  if (!std::isfinite(beta2) || !(eps >= 0.f) || !std::isfinite(eps)) return MUON_ERR_INVALID_ARG;
  if (k == 0) return MUON_OK;
  if (m == 0) return MUON_ERR_SHAPE;
  if (!O || !v || !row_scale_out) return MUON_ERR_INVALID_ARG;
  if (!aligned16(O)) return MUON_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Op ot = o_dtype == MUON_F32 ? Op::F32 : Op::BF16;
  RowLaunch L{};
  L.count = 1;
  L.status = dev_status;
  RowMat& r = L.m[0];
  r.X = const_cast<void*>(O);
  r.ldx = m;
  r.cols = m;
  r.rows = k;
  r.ntask = (int32_t)k;
  r.rscale = row_scale_out;
  TRY(launch_normuon_rows(L, ot, s));
  return launch_normuon_finalize(row_scale_out, k, m, v, rows, beta2, eps, dev_status, s);
}

size_t muon_select_workspace_size(int64_t n) {
  if (n < 0) return 0;
  return kAlign * 3 + 2 * up((size_t)n * sizeof(double) + 8);
}

muon_status select_rows(const float* M, int64_t n, int64_t m, int64_t k, muon_norm norm, int32_t* idx_out, void* ws,
                        size_t ws_bytes, void* stream) {
  if (n < 0 || m < 0 || n > INT32_MAX || m > INT32_MAX) return MUON_ERR_SHAPE;
  if (k < 1 || k > n) return MUON_ERR_SHAPE;
  if (norm != MUON_NORM_L1 && norm != MUON_NORM_L2) return MUON_ERR_INVALID_ARG;
  if (!M || !idx_out) return MUON_ERR_INVALID_ARG;
  if (!ws) return MUON_ERR_WORKSPACE;
  if (!aligned16(M) || !aligned16(ws)) return MUON_ERR_ALIGN;
  if (ws_bytes < muon_select_workspace_size(n)) return MUON_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int>(ws, 0);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MUON_ERR_CUDA;
  const size_t o_s = kAlign, o_x = 2 * kAlign, o_sum = 3 * kAlign;
  const size_t o_key = o_sum + up((size_t)n * sizeof(double) + 8);
  RowLaunch L{};
  L.count = 1;
  L.status = status;
  L.key_l2 = norm == MUON_NORM_L2;
  RowMat& r = L.m[0];
  r.src = M;
  r.rows = n;
  r.cols = m;
  r.ntask = (int32_t)n;
  r.rsum = at<double>(ws, o_sum);
  r.rkey = at<double>(ws, o_key);
  TRY(launch_row_stats(L, Op::F32, s));
  return launch_select(at<double>(ws, o_key), at<double>(ws, o_sum), n, k, idx_out, at<float>(ws, o_s),
                       at<float>(ws, o_x), 0.f, -1.f, status, s);
}

size_t muon_workspace_size(const muon_matrix* mats, int32_t count, const muon_params* p) {
  if (check_step(mats, count, p, NEED_NONE) != MUON_OK) return 0;
  return plan_step(mats, count, p).total;
}

muon_status muon_step(const muon_matrix* mats, int32_t count, const muon_params* p, void* ws, size_t ws_bytes,
                      void* stream) {
  PhaseEvents E;
  return step_impl(mats, count, p, ws, ws_bytes, static_cast<cudaStream_t>(stream), E, nullptr);
}

muon_status muon_step_profiled(const muon_matrix* mats, int32_t count, const muon_params* p, void* ws,
                               size_t ws_bytes, void* stream, muon_step_profile* prof) {
  if (!prof) return MUON_ERR_INVALID_ARG;
  memset(prof, 0, sizeof(*prof));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PhaseEvents E;
  for (int i = 0; i < 5; ++i)
    if (cudaEventCreate(&E.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(E.ev[j]);
      return MUON_ERR_CUDA;
    }
  E.on = true;
  const Counters before = counters();
  muon_status r = step_impl(mats, count, p, ws, ws_bytes, s, E, prof);
  const Counters& after = counters();
  prof->kernel_launches = after.launches - before.launches;
  prof->gemm_launches = after.gemm_launches - before.gemm_launches;
  prof->ns_flops = after.flops_sym - before.flops_sym;
  prof->ns_flops_dense = after.flops_dense - before.flops_dense;
  prof->ns_flops_executed = after.flops_exec - before.flops_exec;
  if (r == MUON_OK && prof->kernel_launches > 0) {
    if (cudaEventSynchronize(E.ev[4]) != cudaSuccess) r = MUON_ERR_CUDA;
    float t[4] = {0, 0, 0, 0};
    for (int i = 0; i < 4 && r == MUON_OK; ++i)
      if (cudaEventElapsedTime(&t[i], E.ev[i], E.ev[i + 1]) != cudaSuccess) r = MUON_ERR_CUDA;
    prof->ms_prologue = t[0];
    prof->ms_ns = t[1];
    prof->ms_normuon = t[2];
    prof->ms_update = t[3];
    prof->ms_total = t[0] + t[1] + t[2] + t[3];
  }
  for (int i = 0; i < 5; ++i) cudaEventDestroy(E.ev[i]);
  return r;
}

muon_status muon_step_events(const muon_matrix* mats, int32_t count, const muon_params* p, void* ws,
                             size_t ws_bytes, void* stream, void* const* events) {
  if (!events) return MUON_ERR_INVALID_ARG;
  PhaseEvents E;
  for (int i = 0; i < 5; ++i) {
    if (!events[i]) return MUON_ERR_INVALID_ARG;
    E.ev[i] = static_cast<cudaEvent_t>(events[i]);
  }
  E.on = true;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  muon_status r = step_impl(mats, count, p, ws, ws_bytes, s, E, nullptr);
  if (r != MUON_OK) return r;
  // a step with no work still records every event, so the caller's timing
  // loop never reads an event that was not recorded
  if (plan_step_empty(mats, count))
    for (int i = 0; i < 5; ++i)
      if (cudaEventRecord(E.ev[i], s) != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status muon_momentum(const muon_matrix* mats, int32_t count, const muon_params* p, void* stream) {
  TRY(check_step(mats, count, p, NEED_M | NEED_G));
  std::vector<RowMat> rm;
  for (int i = 0; i < count; ++i) {
    if (mats[i].rows == 0 || mats[i].cols == 0) continue;
    RowMat r{};
    r.M = mats[i].M;
    r.G = mats[i].G;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.ntask = (int32_t)mats[i].rows;
    rm.push_back(r);
  }
  RowLaunch proto{};
  proto.mu = p->mu;
  proto.mode = p->dion3 ? MOM_DION3 : MOM_MUON;
  proto.status = p->dev_status;
  Op t;
  op_of(p->ns.compute, &t);
  return row_batches(rm, proto, [&](RowLaunch& L) {
    return launch_momentum_rows(L, t, static_cast<cudaStream_t>(stream));
  });
}

muon_status muon_orthogonalize(const muon_matrix* mats, int32_t count, const muon_params* p, void* const* O,
                               float* const* row_scale, int32_t* const* selected, void* ws, size_t ws_bytes,
                               void* stream) {
  return ortho_impl(mats, count, p, O, row_scale, selected, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

muon_status muon_apply_update(const muon_matrix* mats, int32_t count, const muon_params* p, const void* const* O,
                              const float* const* row_scale, const int32_t* const* selected, void* stream) {
  TRY(check_step(mats, count, p, NEED_W | (p && p->dion3 ? NEED_M : 0)));
  if (count > 0 && (!O || !row_scale || (p->dion3 && !selected))) return MUON_ERR_INVALID_ARG;
  Op t;
  op_of(p->ns.compute, &t);
  std::vector<RowMat> um;
  for (int i = 0; i < count; ++i) {
    if (mats[i].rows == 0 || mats[i].cols == 0) continue;
    if (!O[i] || !row_scale[i] || (p->dion3 && !selected[i])) return MUON_ERR_INVALID_ARG;
    if (!aligned16(O[i])) return MUON_ERR_ALIGN;
    RowMat r{};
    r.W = mats[i].W;
    r.M = mats[i].M;
    r.X = const_cast<void*>(O[i]);
    r.ldx = mats[i].cols;
    r.rscale = const_cast<float*>(row_scale[i]);
    r.flag = p->dion3 ? selected[i] : nullptr;
    r.rows = mats[i].rows;
    r.cols = mats[i].cols;
    r.ntask = (int32_t)mats[i].rows;
    um.push_back(r);
  }
  RowLaunch proto{};
  proto.mu = p->mu;
  proto.lr = p->lr;
  proto.mode = p->dion3 ? 1 : 0;
  proto.status = p->dev_status;
  return row_batches(um, proto, [&](RowLaunch& L) {
    return launch_update_rows(L, t, static_cast<cudaStream_t>(stream));
  });
}

int64_t muon_kernel_launch_count(void) { return counters().launches; }

}  // extern "C"
