// The Newton-Schulz chains ("Standard Newton-Schulz" and "1. Gram
// Newton-Schulz" of the Dion3 page) as sequences of grouped GEMM launches.
//
// Standard, per step t with (a, b, c):
//   A = X X^T                  symmetric, K = m
//   B = c A A + b A            symmetric, K = n   (epilogue adds b*A)
//   X <- B X + a X             K = n              (epilogue adds a*X)
// Gram (Theorem 2, naive structure, restart of Algorithm 3), R kept as
// rho * X X^T:
//   R = rho X X^T
//   per step: Z = a I + (b/rho) R + (c/rho^2) R R      symmetric
//             Q = Z (first step after a start/restart) or Q Z
//             R <- (Z R) Z                             (not after the last
//                                                       step, nor before a restart)
//   restart before step r: X <- Q X, R = rho X X^T, Q = I
//   output Q X
// The Frobenius scale of X_0 (xscale) enters the first products' epilogues.
#include <vector>

#include "internal.h"

namespace muon {

namespace {

struct Shape {
  int64_t n, m, ldx, ldn;
  bool tall;
};

Shape shape_of(const NsGroup& g) {
  Shape s;
  s.tall = g.rows > g.cols;
  s.n = s.tall ? g.cols : g.rows;
  s.m = s.tall ? g.rows : g.cols;
  s.ldx = pad_ld(g.cols);
  s.ldn = pad_ld(s.n);
  return s;
}

GemmDesc base(const NsGroup& g) {
  GemmDesc d{};
  d.batch = g.count;
  d.alpha = 1.f;
  return d;
}

// D = alpha * s^apow * X X^T (n x n, symmetric) of the wide view of X.
GemmDesc gram_of(const NsGroup& g, const void* X, void* D, float alpha, const float* scale, int apow) {
  const Shape sh = shape_of(g);
  GemmDesc d = base(g);
  d.A = X; d.lda = sh.ldx; d.strideA = g.rows * sh.ldx;
  d.B = X; d.ldb = sh.ldx; d.strideB = g.rows * sh.ldx;
  d.a_mn = d.b_mn = sh.tall ? 1 : 0;  // tall storage holds X^T: the wide rows are its columns
  d.D = D; d.ldd = sh.ldn; d.strideD = sh.n * sh.ldn;
  d.M = d.N = (int)sh.n;
  d.K = (int)sh.m;
  d.sym = 1;
  d.alpha = alpha;
  d.scale = scale;
  d.alpha_pow = apow;
  d.part = g.part;
  d.part_bytes = g.part_bytes;
  return d;
}

// D = alpha * P Q + beta * C + gamma * I for symmetric n x n P, Q whose
// product is symmetric (all operands K-major thanks to the symmetry of Q).
GemmDesc sym_of(const NsGroup& g, const void* P, const void* Q, void* D, const void* C, float alpha, float beta,
                float gamma) {
  const Shape sh = shape_of(g);
  GemmDesc d = base(g);
  d.A = P; d.lda = sh.ldn; d.strideA = sh.n * sh.ldn;
  d.B = Q; d.ldb = sh.ldn; d.strideB = sh.n * sh.ldn;
  d.D = D; d.ldd = sh.ldn; d.strideD = sh.n * sh.ldn;
  d.C = C; d.ldc = sh.ldn; d.strideC = sh.n * sh.ldn;
  d.M = d.N = d.K = (int)sh.n;
  d.sym = 1;
  d.alpha = alpha;
  d.beta = beta;
  d.gamma = gamma;
  d.part = g.part;
  d.part_bytes = g.part_bytes;
  return d;
}

// Stored-layout D = alpha*s^apow * (P X) + beta*s^bpow * X for symmetric
// n x n P: wide D = P X (B operand X read MN-major); tall D = X^T P = X P.
GemmDesc apply_of(const NsGroup& g, const void* P, const void* X, void* D, float alpha, float beta,
                  const float* scale, int apow, int bpow) {
  const Shape sh = shape_of(g);
  GemmDesc d = base(g);
  if (!sh.tall) {
    d.A = P; d.lda = sh.ldn; d.strideA = sh.n * sh.ldn; d.a_mn = 0;
    d.B = X; d.ldb = sh.ldx; d.strideB = g.rows * sh.ldx; d.b_mn = 1;
    d.M = (int)sh.n; d.N = (int)sh.m;
  } else {
    d.A = X; d.lda = sh.ldx; d.strideA = g.rows * sh.ldx; d.a_mn = 0;
    d.B = P; d.ldb = sh.ldn; d.strideB = sh.n * sh.ldn; d.b_mn = 0;
    d.M = (int)sh.m; d.N = (int)sh.n;
  }
  d.K = (int)sh.n;
  d.D = D; d.ldd = sh.ldx; d.strideD = g.rows * sh.ldx;
  d.C = beta != 0.f ? X : nullptr; d.ldc = sh.ldx; d.strideC = g.rows * sh.ldx;
  d.alpha = alpha;
  d.beta = beta;
  d.scale = scale;
  d.alpha_pow = apow;
  d.beta_pow = bpow;
  return d;
}

struct Launcher {
  Op t;
  int* status;
  uint64_t timeout;
  cudaStream_t s;
  std::vector<GemmDesc>* chain;  // fused chain: products are recorded, then run by tc_chain
  muon_status operator()(const GemmDesc* d, int n) const {
    if (chain) {
      chain->insert(chain->end(), d, d + n);
      return MUON_OK;
    }
    if (t == Op::F32) {
      for (int i = 0; i < n; ++i) {
        muon_status r = simt_gemm(d[i], s);
        if (r != MUON_OK) return r;
      }
      return MUON_OK;
    }
    return tc_gemm(t, d, n, status, timeout, s);
  }
};

#define TRY(x)                          \
  do {                                  \
    muon_status _r = (x);               \
    if (_r != MUON_OK) return _r;       \
  } while (0)

muon_status run_standard(const Launcher& L, NsGroup* gs, int ng, const muon_ns_params* p) {
  GemmDesc d[kMaxGemmGroups];
  for (int t = 0; t < p->T; ++t) {
    const float a = p->coeffs[t][0], b = p->coeffs[t][1], c = p->coeffs[t][2];
    const bool first = t == 0;
    for (int i = 0; i < ng; ++i)
      d[i] = gram_of(gs[i], gs[i].X[gs[i].cur], gs[i].nb[0], 1.f, first ? gs[i].xscale : nullptr, 2);
    TRY(L(d, ng));
    for (int i = 0; i < ng; ++i) d[i] = sym_of(gs[i], gs[i].nb[0], gs[i].nb[0], gs[i].nb[1], gs[i].nb[0], c, b, 0.f);
    TRY(L(d, ng));
    for (int i = 0; i < ng; ++i) {
      NsGroup& g = gs[i];
      d[i] = apply_of(g, g.nb[1], g.X[g.cur], g.X[g.cur ^ 1], 1.f, a, first ? g.xscale : nullptr, 1, 1);
    }
    TRY(L(d, ng));
    for (int i = 0; i < ng; ++i) gs[i].cur ^= 1;
  }
  return MUON_OK;
}

muon_status run_gram(const Launcher& L, NsGroup* gs, int ng, const muon_ns_params* p) {
  GemmDesc d[kMaxGemmGroups];
  // buffer roles (indices into nb), identical for every group
  int R = 0, Q = -1;
  auto free_buf = [&](int x, int y, int z) {
    for (int i = 0; i < 4; ++i)
      if (i != x && i != y && i != z) return i;
    return -1;
  };
  for (int i = 0; i < ng; ++i) {
    NsGroup& g = gs[i];
    d[i] = gram_of(g, g.X[g.cur], g.nb[R], g.rho, g.xscale, 2);
  }
  TRY(L(d, ng));
  const int T = p->T, rs = p->restart_at;
  for (int t = 1; t <= T; ++t) {
    const float a = p->coeffs[t - 1][0], b = p->coeffs[t - 1][1], c = p->coeffs[t - 1][2];
    if (rs > 0 && t == rs && Q >= 0) {
      // restart: X <- Q X (same storage scale), R = rho X X^T, Q = I
      for (int i = 0; i < ng; ++i) {
        NsGroup& g = gs[i];
        d[i] = apply_of(g, g.nb[Q], g.X[g.cur], g.X[g.cur ^ 1], 1.f, 0.f, nullptr, 0, 0);
      }
      TRY(L(d, ng));
      for (int i = 0; i < ng; ++i) {
        NsGroup& g = gs[i];
        g.cur ^= 1;
        d[i] = gram_of(g, g.X[g.cur], g.nb[R], g.rho, g.xscale, 2);
      }
      TRY(L(d, ng));
      Q = -1;
    }
    const int Z = free_buf(R, Q, -1);
    for (int i = 0; i < ng; ++i) {
      NsGroup& g = gs[i];
      const float rho = g.rho;
      d[i] = sym_of(g, g.nb[R], g.nb[R], g.nb[Z], g.nb[R], c / (rho * rho), b / rho, a);
    }
    TRY(L(d, ng));
    if (Q < 0) {
      Q = Z;  // Q_t = Z_t when Q_{t-1} = I (no product)
    } else {
      const int Qn = free_buf(R, Q, Z);
      for (int i = 0; i < ng; ++i) d[i] = sym_of(gs[i], gs[i].nb[Q], gs[i].nb[Z], gs[i].nb[Qn], nullptr, 1.f, 0.f, 0.f);
      TRY(L(d, ng));
      Q = Qn;
    }
    const bool update_R = t < T && !(rs > 0 && t + 1 == rs);
    if (update_R) {
      const int T1 = free_buf(R, Q, Z);
      for (int i = 0; i < ng; ++i)
        d[i] = sym_of(gs[i], gs[i].nb[Z], gs[i].nb[R], gs[i].nb[T1], nullptr, 1.f, 0.f, 0.f);
      TRY(L(d, ng));
      for (int i = 0; i < ng; ++i)
        d[i] = sym_of(gs[i], gs[i].nb[T1], gs[i].nb[Z], gs[i].nb[R], nullptr, 1.f, 0.f, 0.f);
      TRY(L(d, ng));
    }
  }
  // O = xscale * Q X
  for (int i = 0; i < ng; ++i) {
    NsGroup& g = gs[i];
    d[i] = apply_of(g, g.nb[Q], g.X[g.cur], g.X[g.cur ^ 1], 1.f, 0.f, g.xscale, 1, 0);
  }
  TRY(L(d, ng));
  for (int i = 0; i < ng; ++i) gs[i].cur ^= 1;
  return MUON_OK;
}

}  // namespace

int ns_max_phases(const muon_ns_params* p) { return p->gram ? 4 * p->T + 4 : 3 * p->T; }

muon_status ns_run(Op t, NsGroup* gs, int ng, const muon_ns_params* p, int* status, uint64_t timeout_ns,
                   cudaStream_t s, unsigned* counters) {
  if (ng < 1 || ng > kMaxGemmGroups) return MUON_ERR_INVALID_ARG;
  if (t == Op::F32 || !counters || !gemm_chain()) {
    const Launcher L{t, status, timeout_ns, s, nullptr};
    return p->gram ? run_gram(L, gs, ng, p) : run_standard(L, gs, ng, p);
  }
  // fused chain: record every product, then run them as one chain
  std::vector<GemmDesc> chain;
  const Launcher L{t, status, timeout_ns, s, &chain};
  const muon_status r = p->gram ? run_gram(L, gs, ng, p) : run_standard(L, gs, ng, p);
  if (r != MUON_OK || chain.empty()) return r;
  const int nphase = (int)(chain.size() / ng);
  if (nphase > ns_max_phases(p)) return MUON_ERR_INVALID_ARG;  // the counters are sized for ns_max_phases
  return tc_chain(t, chain.data(), nphase, ng, counters, status, timeout_ns, s);
}

}  // namespace muon
