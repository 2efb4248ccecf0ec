// C-ABI entry points of libshampoo (declared in include/shampoo.h): argument
// checks, the block planner, workspace carving and the method drivers that
// sequence the GEMM engine and the streaming kernels on the caller's stream.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/shampoo.h"
#include <nvtx3/nvToolsExt.h>
#include "internal.h"
#include "step.h"

using namespace shp;

struct shp_plan {
  std::vector<int32_t> rows, cols;  // per layer
  int32_t block_size = 0;
  std::vector<int32_t> blocks;      // n_blocks x kBlockFields
  std::vector<int32_t> gb;          // n_gbuckets x 3 (rows, cols, count)
  std::vector<int32_t> fb;          // n_fbuckets x 2 (n, count)
  std::vector<int32_t> gside, fside;  // per bucket: 0 two-sided, 1 one-sided (left factors only)
  // device table image: blocks | per gbucket (l_idx, r_idx) | layer_first | gstack_off
  std::vector<int32_t> image;
  std::vector<size_t> off_lidx, off_ridx;
  size_t off_layer_first = 0, off_gstack = 0;
  const int32_t* dev = nullptr;  // bound device copy of `image`
  int n_blocks() const { return (int)(blocks.size() / kBlockFields); }
  int n_g() const { return (int)(gb.size() / 3); }
  int n_f() const { return (int)(fb.size() / 2); }
  int n_layers() const { return (int)rows.size(); }
};

namespace {

thread_local std::string g_last_error;

shp_status fail(shp_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                             \
  do {                                                                                             \
    cudaError_t e_ = (expr);                                                                       \
    if (e_ != cudaSuccess) return fail(SHP_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_));    \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// An NVTX range around each entry point, so timelines from Nsight tools show
// the library's calls by name (a cheap no-op when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Bump allocator over the caller's workspace; with base == nullptr it only
// measures, so the *_workspace_bytes queries run the same code.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

bool valid_dtype(int d) { return d >= SHP_DTYPE_FP32 && d <= SHP_DTYPE_BF16; }

// Planes for `count` matrices rows x cols in precision `prec`.
Planes make_planes(Carver& c, int count, int rows, int cols, Prec prec, bool need_f32 = true) {
  Planes P;
  P.rows = rows;
  P.cols = cols;
  P.ld = round_up(cols, 32);
  P.bs = (long long)rows * P.ld;
  P.count = count;
  const size_t n = (size_t)count * (size_t)P.bs;
  if (prec == P_FP32) {
    if (need_f32) P.f32 = static_cast<float*>(c.take(n * 4));
    P.h16 = c.take(n * 2);
    P.h16lo = c.take(n * 2);
    P.exp = static_cast<int*>(c.take(sizeof(int) * count));
    P.amax = static_cast<float*>(c.take(sizeof(float) * count));
  } else if (prec == P_TF32) {
    P.f32 = static_cast<float*>(c.take(n * 4));
  } else {
    if (need_f32) P.f32 = static_cast<float*>(c.take(n * 4));
    P.h16 = c.take(n * 2);
    P.h16_bf = prec == P_BF16;
  }
  return P;
}

EpiC as_c(const Planes& P) {
  EpiC c;
  c.f32 = P.f32;
  c.amax = P.amax;
  c.ld = P.ld;
  c.bs = P.bs;
  return c;
}
// Output into planes; with full = false the fp32 copy of the FP32 / FP16 /
// BF16 planes is not written (the value is only read by tensor-core passes).
EpiOut as_out(const Planes& P, bool full = true) {
  EpiOut o;
  o.f32 = (full || !(P.h16)) ? P.f32 : nullptr;
  o.h16 = P.h16;
  o.h16lo = P.h16lo;
  o.exp = P.exp;
  o.amax = P.amax;
  o.amax_n = P.amax ? P.count : 0;
  o.h16_bf = P.h16_bf;
  o.ld = P.ld;
  o.bs = P.bs;
  return o;
}
EpiOut plain_out(float* p, int ld, long long bs) {
  EpiOut o;
  o.f32 = p;
  o.ld = ld;
  o.bs = bs;
  return o;
}

// sym = 1: the product is symmetric in exact arithmetic (both operands are
// polynomials in one symmetric matrix, or G G^T / G^T G, and C is
// symmetric), so only the tiles on and above the diagonal are computed.
// Used for the statistics and the Chebyshev recurrence only: mirroring the
// products of the coupled iterations (Newton-DB: Y T, T Z, Z Y; coupled
// Newton: X T, T^2, T^p M) breaks the error coupling that keeps them
// stable -- Newton-DB-20 on 1024^2 factors with kappa ~ 5e6 overflowed on
// the GPU and in a float32 model, coupled Newton lost a factor 6.
GemmGroup group(int M, int N, int K, const Planes* A, int a_mn, const Planes* B, int b_mn, int sym = 0) {
  GemmGroup g;
  g.sym = sym;
  g.M = M;
  g.N = N;
  g.K = K;
  g.A = A;
  g.a_mn = a_mn;
  g.B = B;
  g.b_mn = b_mn;
  return g;
}

// ---- planner -------------------------------------------------------------

void split_dim(int d, int B, std::vector<int>& out) {
  out.clear();
  if (B <= 0 || d <= B) {
    out.push_back(d);
    return;
  }
  for (int i = 0; i < d / B; ++i) out.push_back(B);
  if (d % B) out.push_back(d % B);
}

// ---- workspace layouts -----------------------------------------------------

struct RootBufs {
  Planes Y[2], Z[2], T, T2, T4;
  double* sums = nullptr;
  float* lmax = nullptr;  // max |L| per matrix, bounds the FP32 plane exponents
  float* fscale = nullptr;
  Planes A16, Vt, W;
};

RootBufs carve_roots(Carver& c, int count, int n, int method, Prec pr, int scaling, int pi_vectors) {
  RootBufs r;
  r.sums = static_cast<double*>(c.take(sizeof(double) * count));
  r.lmax = static_cast<float*>(c.take(sizeof(float) * count));
  if (method == SHP_METHOD_NDB) {
    for (int i = 0; i < 2; ++i) {
      r.Y[i] = make_planes(c, count, n, n, pr);
      r.Z[i] = make_planes(c, count, n, n, pr);
    }
    r.T = make_planes(c, count, n, n, pr);
  } else if (method == SHP_METHOD_CN) {
    for (int i = 0; i < 2; ++i) {
      r.Y[i] = make_planes(c, count, n, n, pr);  // X iterates
      r.Z[i] = make_planes(c, count, n, n, pr);  // M iterates
    }
    r.T = make_planes(c, count, n, n, pr);   // T
    r.T2 = make_planes(c, count, n, n, pr);  // T^2
    r.T4 = make_planes(c, count, n, n, pr);  // T^4
  } else {
    r.Y[0] = make_planes(c, count, n, n, pr);  // S
    r.Z[0] = make_planes(c, count, n, n, pr);  // B_{k+1}
    r.Z[1] = make_planes(c, count, n, n, pr);  // B_{k+2}
    r.T = make_planes(c, count, n, n, pr);     // B_k
  }
  if (scaling == SHP_SCALE_POWER) {
    r.fscale = static_cast<float*>(c.take(sizeof(float) * count));
    r.A16 = make_planes(c, count, n, n, P_FP16, false);
    r.Vt = make_planes(c, count, pi_vectors, n, P_FP16, false);
    r.W = make_planes(c, count, n, pi_vectors, P_TF32);
  }
  return r;
}

// Chebyshev coefficients of x^(-1/p) on [eps, 1 + eps] in T_k(t), t in
// [-1, 1], by interpolation at the degree+1 first-kind nodes ("DASH", A.1).
std::vector<double> cheb_coeffs(int degree, double eps, int p) {
  const int N = degree + 1;
  std::vector<double> f(N), th(N), c(N);
  for (int j = 0; j < N; ++j) {
    th[j] = M_PI * (j + 0.5) / N;
    const double x = eps + (std::cos(th[j]) + 1.0) * 0.5;
    f[j] = std::pow(x, -1.0 / p);
  }
  for (int k = 0; k < N; ++k) {
    double s = 0.0;
    for (int j = 0; j < N; ++j) s += f[j] * std::cos(k * th[j]);
    c[k] = 2.0 * s / N;
  }
  c[0] *= 0.5;
  return c;
}

shp_status check_gemm(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SHP_OK;
}
#define GEMM_TRY(expr)                          \
  do {                                          \
    shp_status s_ = check_gemm((expr), #expr);  \
    if (s_ != SHP_OK) return s_;                \
  } while (0)

// Scale s_b of L_b (+ eps I): Frobenius norm or multi-power-iteration.
shp_status compute_scale(const float* A, int count, int n, float eps_s, int scaling, int pi_vectors, int pi_iters,
                         const float* pi_starts, RootBufs& r, float* scale_out, cudaStream_t st) {
  GEMM_TRY(launch_frob_sumsq(A, n, n, (long long)n * n, count, eps_s, r.sums, st, r.lmax));
  if (scaling == SHP_SCALE_FROBENIUS) {
    GEMM_TRY(launch_sqrt_scale(r.sums, nullptr, scale_out, count, st));
    return SHP_OK;
  }
  // power iteration on (A / ||A||_F) in fp16
  GEMM_TRY(launch_sqrt_scale(r.sums, nullptr, r.fscale, count, st));
  GEMM_TRY(launch_to_planes(A, n, (long long)n * n, nullptr, count, n, n, 1.f, eps_s, 0.f, r.fscale, r.A16, P_FP16,
                            st));
  GEMM_TRY(launch_pi_start_batched(pi_starts, pi_vectors, n, r.Vt.h16, r.Vt.ld, r.Vt.bs, count, st));
  GemmGroup g = group(n, pi_vectors, n, &r.A16, 0, &r.Vt, 0);
  g.epi.O = plain_out(r.W.f32, r.W.ld, r.W.bs);
  for (int it = 0; it <= pi_iters; ++it) {
    GEMM_TRY(launch_gemm(&g, 1, count, P_FP16, st));
    if (it < pi_iters)
      GEMM_TRY(launch_pi_normalize(r.W.f32, n, pi_vectors, r.W.ld, r.W.bs, count, r.Vt.h16, r.Vt.ld, r.Vt.bs, st));
  }
  GEMM_TRY(launch_pi_rayleigh(r.W.f32, r.Vt.h16, n, pi_vectors, r.W.ld, r.W.bs, r.Vt.ld, r.Vt.bs, count, r.sums,
                              scale_out, st));
  return SHP_OK;
}

EpiOut final_out(float* X, int n) { return plain_out(X, n, (long long)n * n); }

// Newton-DB inverse fourth root: two chained coupled inverse-square-root
// calls ("DASH", §3 Newton-DB).
shp_status run_ndb(const float* A, int count, int n, float eps, int iters, int p, Prec pr, RootBufs& r,
                   const float* scale, float* X, int* status, cudaStream_t st) {
  // p = 2^calls: each call halves the power, the next one starting from
  // the previous Y with Z = I
  const int calls = p == 2 ? 1 : (p == 4 ? 2 : 3);
  GEMM_TRY(launch_to_planes(A, n, (long long)n * n, nullptr, count, n, n, 1.f, eps, 0.f, scale, r.Y[0], pr, st,
                            r.lmax));
  int cur = 0;
  for (int call = 0; call < calls; ++call) {
    const bool final_call = call == calls - 1;
    // iteration 1 (Z_0 = I): Y_1 = Y_0 (3I - Y_0)/2 = 1.5 Y_0 - 0.5 Y_0^2, Z_1 = 1.5 I - 0.5 Y_0
    // Y keeps its fp32 copy only where it will be the next call's C
    GemmGroup g = group(n, n, n, &r.Y[cur], 0, &r.Y[cur], 1);
    g.epi.alpha = -0.5f;
    g.epi.beta = 1.5f;
    g.epi.C = as_c(r.Y[cur]);
    g.epi.O = as_out(r.Y[1 - cur], !final_call && iters == 1);
    g.epi.X = as_out(r.Z[1 - cur], false);
    g.epi.beta2 = -0.5f;
    g.epi.gamma2 = 1.5f;
    if (final_call && iters == 1) {
      g.epi.X = final_out(X, n);
      g.epi.bscale = scale;
      g.epi.root_p = p;
      g.epi.status = status;
    }
    GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
    cur = 1 - cur;
    for (int it = 2; it <= iters; ++it) {
      const bool last = it == iters;
      // T = (3I - Z Y)/2
      GemmGroup gt = group(n, n, n, &r.Z[cur], 0, &r.Y[cur], 1);
      gt.epi.alpha = -0.5f;
      gt.epi.gamma = 1.5f;
      gt.epi.O = as_out(r.T, false);
      GEMM_TRY(launch_gemm(&gt, 1, count, pr, st));
      // Y' = Y T and Z' = T Z in one grouped launch (drop what is not needed:
      // the final call's last Y, a non-final call's last Z)
      GemmGroup gs[2];
      int ng = 0;
      if (!(final_call && last)) {
        gs[ng] = group(n, n, n, &r.Y[cur], 0, &r.T, 1);
        gs[ng].epi.O = as_out(r.Y[1 - cur], !final_call && last);
        ++ng;
      }
      if (!(!final_call && last)) {
        gs[ng] = group(n, n, n, &r.T, 0, &r.Z[cur], 1);
        if (final_call && last) {
          gs[ng].epi.O = final_out(X, n);
          gs[ng].epi.bscale = scale;
          gs[ng].epi.root_p = p;
          gs[ng].epi.status = status;
        } else {
          gs[ng].epi.O = as_out(r.Z[1 - cur], false);
        }
        ++ng;
      }
      GEMM_TRY(launch_gemm(gs, ng, count, pr, st));
      cur = 1 - cur;
    }
  }
  return SHP_OK;
}

// Coupled Newton for A^(-1/p) ("Shampoo" notes, coupled Newton of Guo and
// Higham): X <- X T, M <- T^p M, T = ((p+1)I - M)/p, T^p by squarings.
shp_status run_cn(const float* A, int count, int n, float eps, int iters, int p, Prec pr, RootBufs& r,
                  const float* scale, float* X, int* status, cudaStream_t st) {
  // Buffers: X iterates r.Y[0..1], M iterates r.Z[0..1], T in r.T, T^2 in
  // r.T2, T^4 in r.T4, T^8 back in r.T2.  Products in the order X T, T T,
  // (T^2 T^2, T^4 T^4), T^p M; the epilogue of T^p M also writes the next T.
  Planes* Xp = r.Y;
  Planes* Mp = r.Z;
  const long long bs = (long long)n * n;
  const float ip = 1.f / (float)p, pp = (float)(p + 1) / (float)p;
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, 1.f, eps, 0.f, scale, Mp[0], pr, st, r.lmax));
  // T_0 = ((p+1) I - M_0)/p = (-1/(p s)) L + ((p+1)/p - eps/(p s)) I ; X_1 = X_0 T_0 = T_0
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, -ip, -ip * eps, pp, scale, r.T, pr, st, r.lmax));
  if (iters == 1) {
    GEMM_TRY(launch_scaled_copy(r.T, n, count, scale, p, X, status, st));
    return SHP_OK;
  }
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, -ip, -ip * eps, pp, scale, Xp[0], pr, st, r.lmax));
  int cx = 0, cm = 0;
  for (int it = 1; it <= iters; ++it) {
    const bool last = it == iters;
    if (it > 1) {
      GemmGroup gs[2];
      gs[0] = group(n, n, n, &Xp[cx], 0, &r.T, 1);  // X' = X T
      if (last) {
        gs[0].epi.O = final_out(X, n);
        gs[0].epi.bscale = scale;
        gs[0].epi.root_p = p;
        gs[0].epi.status = status;
        GEMM_TRY(launch_gemm(gs, 1, count, pr, st));
        break;
      }
      gs[0].epi.O = as_out(Xp[1 - cx], false);
      gs[1] = group(n, n, n, &r.T, 0, &r.T, 1);  // T^2 = T T
      gs[1].epi.O = as_out(r.T2, false);
      GEMM_TRY(launch_gemm(gs, 2, count, pr, st));
      cx = 1 - cx;
    } else {
      GemmGroup g2 = group(n, n, n, &r.T, 0, &r.T, 1);  // T_0^2
      g2.epi.O = as_out(r.T2, false);
      GEMM_TRY(launch_gemm(&g2, 1, count, pr, st));
    }
    Planes* Tp = &r.T2;
    if (p >= 4) {
      GemmGroup g4 = group(n, n, n, &r.T2, 0, &r.T2, 1);  // T^4 = T^2 T^2
      g4.epi.O = as_out(r.T4, false);
      GEMM_TRY(launch_gemm(&g4, 1, count, pr, st));
      Tp = &r.T4;
    }
    if (p == 8) {
      GemmGroup g8 = group(n, n, n, &r.T4, 0, &r.T4, 1);  // T^8 = T^4 T^4
      g8.epi.O = as_out(r.T2, false);
      GEMM_TRY(launch_gemm(&g8, 1, count, pr, st));
      Tp = &r.T2;
    }
    GemmGroup gm = group(n, n, n, Tp, 0, &Mp[cm], 1);  // M' = T^p M, next T = ((p+1) I - M')/p
    gm.epi.O = as_out(Mp[1 - cm], false);
    gm.epi.X = as_out(r.T, false);
    gm.epi.alpha2 = -ip;
    gm.epi.gamma2 = pp;
    GEMM_TRY(launch_gemm(&gm, 1, count, pr, st));
    cm = 1 - cm;
  }
  return SHP_OK;
}

// Coupled Newton warm-started from a previous root X0 (the iteration the
// "Shampoo" notes describe under "Roots on idle CPUs"): X_0 = X0 and
// M_0 = X0^p (L + eps I), the invariant M = X^p A of the cold start, with no
// scaling and no final multiplier.  Then the update of run_cn, where the
// first X product is a real GEMM.  Products: X0^2 (X0^4, X0^8 by squaring),
// X0^p A, then X T, T T, (T^2 T^2, T^4 T^4), T^p M per iteration and X T
// alone in the last one: 4 k for p = 4.
shp_status run_cn_warm(const float* A, const float* X0, int count, int n, float eps, int iters, int p, Prec pr,
                       RootBufs& r, float* X, int* status, cudaStream_t st) {
  Planes* Xp = r.Y;
  Planes* Mp = r.Z;
  const long long bs = (long long)n * n;
  const float ip = 1.f / (float)p, pp = (float)(p + 1) / (float)p;
  GEMM_TRY(launch_to_planes(X0, n, bs, nullptr, count, n, n, 1.f, 0.f, 0.f, nullptr, Xp[0], pr, st));
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, 1.f, eps, 0.f, nullptr, Mp[1], pr, st));
  GemmGroup g = group(n, n, n, &Xp[0], 0, &Xp[0], 1);  // X0^2
  g.epi.O = as_out(r.T2, false);
  GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
  Planes* Xpow = &r.T2;
  if (p >= 4) {
    g = group(n, n, n, &r.T2, 0, &r.T2, 1);  // X0^4
    g.epi.O = as_out(r.T4, false);
    GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
    Xpow = &r.T4;
  }
  if (p == 8) {
    g = group(n, n, n, &r.T4, 0, &r.T4, 1);  // X0^8
    g.epi.O = as_out(r.T2, false);
    GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
    Xpow = &r.T2;
  }
  g = group(n, n, n, Xpow, 0, &Mp[1], 1);  // M_0 = X0^p A, T_0 = ((p+1) I - M_0)/p
  g.epi.O = as_out(Mp[0], false);
  g.epi.X = as_out(r.T, false);
  g.epi.alpha2 = -ip;
  g.epi.gamma2 = pp;
  GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
  int cx = 0, cm = 0;
  for (int it = 1; it <= iters; ++it) {
    GemmGroup gs[2];
    gs[0] = group(n, n, n, &Xp[cx], 0, &r.T, 1);  // X' = X T
    if (it == iters) {
      gs[0].epi.O = final_out(X, n);
      gs[0].epi.root_p = p;
      gs[0].epi.status = status;
      GEMM_TRY(launch_gemm(gs, 1, count, pr, st));
      break;
    }
    gs[0].epi.O = as_out(Xp[1 - cx], false);
    gs[1] = group(n, n, n, &r.T, 0, &r.T, 1);  // T^2
    gs[1].epi.O = as_out(r.T2, false);
    GEMM_TRY(launch_gemm(gs, 2, count, pr, st));
    cx = 1 - cx;
    Planes* Tp = &r.T2;
    if (p >= 4) {
      GemmGroup g4 = group(n, n, n, &r.T2, 0, &r.T2, 1);
      g4.epi.O = as_out(r.T4, false);
      GEMM_TRY(launch_gemm(&g4, 1, count, pr, st));
      Tp = &r.T4;
    }
    if (p == 8) {
      GemmGroup g8 = group(n, n, n, &r.T4, 0, &r.T4, 1);
      g8.epi.O = as_out(r.T2, false);
      GEMM_TRY(launch_gemm(&g8, 1, count, pr, st));
      Tp = &r.T2;
    }
    GemmGroup gm = group(n, n, n, Tp, 0, &Mp[cm], 1);  // M' = T^p M, next T
    gm.epi.O = as_out(Mp[1 - cm], false);
    gm.epi.X = as_out(r.T, false);
    gm.epi.alpha2 = -ip;
    gm.epi.gamma2 = pp;
    GEMM_TRY(launch_gemm(&gm, 1, count, pr, st));
    cm = 1 - cm;
  }
  return SHP_OK;
}

// Chebyshev approximation with the optimised matrix Clenshaw recurrence
// ("DASH", A.2): d - 1 matmuls for degree d.
shp_status run_cheb(const float* A, int count, int n, float eps, int degree, int p, Prec pr, RootBufs& r,
                    const float* scale, float* X, int* status, cudaStream_t st) {
  const std::vector<double> c = cheb_coeffs(degree, eps, p);
  const long long bs = (long long)n * n;
  Planes& S = r.Y[0];
  Planes* Bk1 = &r.Z[0];
  Planes* Bk2 = &r.Z[1];
  Planes* Bk = &r.T;
  if (degree == 0) {
    GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, 0.f, 0.f, (float)c[0], nullptr, *Bk2, pr, st,
                              r.lmax));
    GEMM_TRY(launch_scaled_copy(*Bk2, n, count, scale, p, X, status, st));
    return SHP_OK;
  }
  if (degree == 1) {  // c0 I + c1 S = (2 c1/s) L + (c0 - c1) I
    GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, (float)(2 * c[1]), 0.f, (float)(c[0] - c[1]), scale,
                              *Bk2, pr, st, r.lmax));
    GEMM_TRY(launch_scaled_copy(*Bk2, n, count, scale, p, X, status, st));
    return SHP_OK;
  }
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, 2.f, 0.f, -1.f, scale, S, pr, st, r.lmax));
  // B_d = c_d I ; B_{d-1} = c_{d-1} I + 2 c_d S = (4 c_d / s) L + (c_{d-1} - 2 c_d) I
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, 0.f, 0.f, (float)c[degree], nullptr, *Bk2, pr, st,
                            r.lmax));
  GEMM_TRY(launch_to_planes(A, n, bs, nullptr, count, n, n, (float)(4 * c[degree]), 0.f,
                            (float)(c[degree - 1] - 2 * c[degree]), scale, *Bk1, pr, st, r.lmax));
  for (int k = degree - 2; k >= 1; --k) {
    // B_k = c_k I + 2 S B_{k+1} - B_{k+2}; three buffers, so that no launch
    // writes a matrix it reads
    GemmGroup g = group(n, n, n, &S, 0, Bk1, 1, 1);
    g.epi.alpha = 2.f;
    g.epi.beta = -1.f;
    g.epi.gamma = (float)c[k];
    g.epi.C = as_c(*Bk2);
    g.epi.O = as_out(*Bk);
    GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
    Planes* t = Bk2;
    Bk2 = Bk1;
    Bk1 = Bk;
    Bk = t;
  }
  // result = c_0 I + S B_1 - B_2, times s^(-1/4)
  GemmGroup g = group(n, n, n, &S, 0, Bk1, 1, 1);
  g.epi.alpha = 1.f;
  g.epi.beta = -1.f;
  g.epi.gamma = (float)c[0];
  g.epi.C = as_c(*Bk2);
  g.epi.O = final_out(X, n);
  g.epi.bscale = scale;
  g.epi.root_p = p;
  g.epi.status = status;
  GEMM_TRY(launch_gemm(&g, 1, count, pr, st));
  return SHP_OK;
}

shp_status check_plan(const shp_plan* plan, bool need_bound) {
  if (!plan) return fail(SHP_ERR_INVALID_ARG, "plan is NULL");
  if (need_bound && !plan->dev) return fail(SHP_ERR_INVALID_ARG, "plan has no device tables (call shampoo_plan_bind)");
  return SHP_OK;
}

// Layer pointer tables for layers [l0, l1) of one launch.
LayerArgs layer_args(const shp_plan* plan, int l0, int l1, float* const* W, const float* const* G, float* const* m,
                     float* const* v) {
  LayerArgs la;
  memset(&la, 0, sizeof(la));
  la.layer0 = l0;
  for (int l = l0; l < l1; ++l) {
    la.W[l - l0] = W ? W[l] : nullptr;
    la.G[l - l0] = G ? G[l] : nullptr;
    la.m[l - l0] = m ? m[l] : nullptr;
    la.v[l - l0] = v ? v[l] : nullptr;
    la.cols[l - l0] = plan->cols[l];
  }
  return la;
}

}  // namespace

void shp::set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

// ============================================================================
extern "C" {

const char* shampoo_last_error(void) { return g_last_error.c_str(); }

int32_t shampoo_version(void) { return 100; }

uint64_t shampoo_launch_count(void) { return launch_total(); }

shp_status shampoo_device_error(int32_t* out) {
  if (!out) return fail(SHP_ERR_INVALID_ARG, "out is NULL");
  int h = 0;
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(read_and_clear_dev_error(&h));
  *out = h;
  return SHP_OK;
}

shp_status shampoo_plan_create(const int32_t* rows, const int32_t* cols, int32_t n_layers, int32_t block_size,
                               shp_plan** plan_out) {
  return shampoo_plan_create_ex(rows, cols, nullptr, n_layers, block_size, 0, plan_out);
}

shp_status shampoo_plan_create_ex(const int32_t* rows, const int32_t* cols, const int32_t* left_only,
                                  int32_t n_layers, int32_t block_size, int32_t flags, shp_plan** plan_out) {
  if (!plan_out) return fail(SHP_ERR_INVALID_ARG, "plan_out is NULL");
  if (flags & ~SHP_PLAN_LAYERWISE) return fail(SHP_ERR_INVALID_ARG, "unknown plan flags 0x%x", flags);
  const bool layerwise = (flags & SHP_PLAN_LAYERWISE) != 0;
  *plan_out = nullptr;
  if (n_layers < 1 || !rows || !cols) return fail(SHP_ERR_INVALID_ARG, "need n_layers >= 1 and rows/cols arrays");
  if (block_size < 0) return fail(SHP_ERR_INVALID_ARG, "block_size must be >= 0");
  for (int l = 0; l < n_layers; ++l)
    if (rows[l] < 1 || cols[l] < 1 || rows[l] >= (1 << 30) || cols[l] >= (1 << 30))
      return fail(SHP_ERR_SHAPE, "layer %d has invalid shape %d x %d", l, rows[l], cols[l]);
  shp_plan* p = new shp_plan();
  p->rows.assign(rows, rows + n_layers);
  p->cols.assign(cols, cols + n_layers);
  p->block_size = block_size;
  std::vector<int> rs, cs;
  std::vector<int> fkey, flayer;  // factor bucket n values (and layers, when layerwise) in order
  std::vector<int> glayer;        // gradient bucket layers, when layerwise
  int cur_layer = 0, cur_side = 0;
  auto fslot = [&](int n, int32_t* bucket, int32_t* index) {
    int b = -1;
    for (size_t i = 0; i < fkey.size(); ++i)
      if (fkey[i] == n && p->fside[i] == cur_side && (!layerwise || flayer[i] == cur_layer)) b = (int)i;
    if (b < 0) {
      b = (int)fkey.size();
      fkey.push_back(n);
      flayer.push_back(cur_layer);
      p->fside.push_back(cur_side);
      p->fb.push_back(n);
      p->fb.push_back(0);
    }
    *bucket = b;
    *index = p->fb[2 * b + 1]++;
  };
  for (int l = 0; l < n_layers; ++l) {
    cur_layer = l;
    cur_side = left_only && left_only[l] ? 1 : 0;
    split_dim(rows[l], block_size, rs);
    split_dim(cols[l], block_size, cs);
    const size_t first = p->blocks.size();
    int r0 = 0;
    for (size_t br = 0; br < rs.size(); ++br) {
      int c0 = 0;
      for (size_t bc = 0; bc < cs.size(); ++bc) {
        const int r = rs[br], c = cs[bc];
        if (r > SHP_MAX_N || c > SHP_MAX_N) {
          delete p;
          return fail(SHP_ERR_SHAPE, "block %d x %d exceeds SHP_MAX_N (use a block_size)", r, c);
        }
        int g = -1;
        for (int i = 0; i < (int)p->gb.size() / 3; ++i)
          if (p->gb[3 * i] == r && p->gb[3 * i + 1] == c && p->gside[i] == cur_side && (!layerwise || glayer[i] == l))
            g = i;
        if (g < 0) {
          g = (int)p->gb.size() / 3;
          glayer.push_back(l);
          p->gside.push_back(cur_side);
          p->gb.push_back(r);
          p->gb.push_back(c);
          p->gb.push_back(0);
        }
        const int gi = p->gb[3 * g + 2]++;
        const int32_t rec[kBlockFields] = {l, (int)br, (int)bc, r0, c0, r, c, g, gi, -1, -1, -1, -1};
        p->blocks.insert(p->blocks.end(), rec, rec + kBlockFields);
        c0 += c;
      }
      r0 += rs[br];
    }
    const size_t nb = (p->blocks.size() - first) / kBlockFields;
    for (size_t i = 0; i < nb; ++i) {  // left factors of the layer, row-major
      int32_t* rec = &p->blocks[first + i * kBlockFields];
      fslot(rec[5], &rec[9], &rec[10]);
    }
    for (size_t i = 0; i < nb && !cur_side; ++i) {  // then its right factors (two-sided layers)
      int32_t* rec = &p->blocks[first + i * kBlockFields];
      fslot(rec[6], &rec[11], &rec[12]);
    }
  }
  // device image
  const int nb = p->n_blocks(), ng = p->n_g();
  p->image = p->blocks;
  p->off_lidx.resize(ng);
  p->off_ridx.resize(ng);
  for (int g = 0; g < ng; ++g) {
    const int cnt = p->gb[3 * g + 2];
    std::vector<int32_t> li(cnt), ri(cnt);
    for (int b = 0; b < nb; ++b) {
      const int32_t* rec = &p->blocks[b * kBlockFields];
      if (rec[7] == g) {
        li[rec[8]] = rec[10];
        ri[rec[8]] = rec[12];
      }
    }
    p->off_lidx[g] = p->image.size();
    p->image.insert(p->image.end(), li.begin(), li.end());
    p->off_ridx[g] = p->image.size();
    p->image.insert(p->image.end(), ri.begin(), ri.end());
  }
  p->off_layer_first = p->image.size();
  {
    std::vector<int32_t> lf(n_layers + 1, nb);
    for (int b = nb - 1; b >= 0; --b) lf[p->blocks[b * kBlockFields]] = b;
    for (int l = n_layers - 1; l >= 0; --l)
      if (lf[l] > lf[l + 1]) lf[l] = lf[l + 1];
    p->image.insert(p->image.end(), lf.begin(), lf.end());
  }
  p->off_gstack = p->image.size();
  {
    int acc = 0;
    for (int g = 0; g < ng; ++g) {
      p->image.push_back(acc);
      acc += p->gb[3 * g + 2];
    }
    p->image.push_back(acc);
  }
  *plan_out = p;
  return SHP_OK;
}

void shampoo_plan_destroy(shp_plan* plan) { delete plan; }

shp_status shampoo_plan_sizes(const shp_plan* plan, int32_t* n_blocks, int32_t* n_gbuckets, int32_t* n_fbuckets,
                              size_t* device_bytes) {
  if (!plan) return fail(SHP_ERR_INVALID_ARG, "plan is NULL");
  if (n_blocks) *n_blocks = plan->n_blocks();
  if (n_gbuckets) *n_gbuckets = plan->n_g();
  if (n_fbuckets) *n_fbuckets = plan->n_f();
  if (device_bytes) *device_bytes = plan->image.size() * sizeof(int32_t);
  return SHP_OK;
}

shp_status shampoo_plan_tables(const shp_plan* plan, int32_t* blocks, int32_t* gbuckets, int32_t* fbuckets) {
  if (!plan) return fail(SHP_ERR_INVALID_ARG, "plan is NULL");
  if (blocks) memcpy(blocks, plan->blocks.data(), plan->blocks.size() * sizeof(int32_t));
  if (gbuckets) memcpy(gbuckets, plan->gb.data(), plan->gb.size() * sizeof(int32_t));
  if (fbuckets) memcpy(fbuckets, plan->fb.data(), plan->fb.size() * sizeof(int32_t));
  return SHP_OK;
}

shp_status shampoo_plan_factor_sides(const shp_plan* plan, int32_t* sides) {
  if (!plan || !sides) return fail(SHP_ERR_INVALID_ARG, "plan and sides must be non-NULL");
  memcpy(sides, plan->fside.data(), plan->fside.size() * sizeof(int32_t));
  return SHP_OK;
}

shp_status shampoo_plan_bind(shp_plan* plan, void* device_tables, size_t bytes, void* stream) {
  if (!plan || !device_tables) return fail(SHP_ERR_INVALID_ARG, "plan and device_tables must be non-NULL");
  const size_t need = plan->image.size() * sizeof(int32_t);
  if (bytes < need) return fail(SHP_ERR_WORKSPACE, "device table buffer has %zu bytes, needs %zu", bytes, need);
  CUDA_TRY(cudaMemcpyAsync(device_tables, plan->image.data(), need, cudaMemcpyHostToDevice, as_stream(stream)));
  plan->dev = static_cast<const int32_t*>(device_tables);
  return SHP_OK;
}

shp_status shampoo_stack_blocks(const shp_plan* plan, const float* const* grads, float* const* g_stacks,
                                void* stream) {
  const NvtxRange nvtx_range("shampoo_stack_blocks");
  shp_status s = check_plan(plan, true);
  if (s) return s;
  if (!grads || !g_stacks) return fail(SHP_ERR_INVALID_ARG, "grads and g_stacks must be non-NULL");
  if (plan->n_g() > kMaxBuckets) return fail(SHP_ERR_UNSUPPORTED, "more than %d gradient buckets", kMaxBuckets);
  for (int l = 0; l < plan->n_layers(); ++l)
    if (!grads[l]) return fail(SHP_ERR_INVALID_ARG, "grads[%d] is NULL", l);
  BucketArgs ba;
  for (int g = 0; g < plan->n_g(); ++g) {
    if (!g_stacks[g]) return fail(SHP_ERR_INVALID_ARG, "g_stacks[%d] is NULL", g);
    ba.ptr[g] = g_stacks[g];
  }
  const int32_t* lf = plan->image.data() + plan->off_layer_first;
  for (int l0 = 0; l0 < plan->n_layers(); l0 += kMaxLayersPerLaunch) {
    const int l1 = std::min(plan->n_layers(), l0 + kMaxLayersPerLaunch);
    LayerArgs la = layer_args(plan, l0, l1, nullptr, grads, nullptr, nullptr);
    long long mx = 0;
    for (int b = lf[l0]; b < lf[l1]; ++b) {
      const int32_t* rec = &plan->blocks[b * kBlockFields];
      mx = std::max(mx, (long long)rec[5] * rec[6]);
    }
    CUDA_TRY(launch_gather(plan->dev, lf[l0], lf[l1] - lf[l0], mx, la, ba, as_stream(stream)));
  }
  return SHP_OK;
}

// ---- statistics ------------------------------------------------------------

static size_t stats_ws(const shp_plan* plan, int dtype, void* base, Planes* out_g) {
  size_t mx = 0;
  for (int g = 0; g < plan->n_g(); ++g) {
    Carver c(base);
    Planes P = make_planes(c, plan->gb[3 * g + 2], plan->gb[3 * g], plan->gb[3 * g + 1], (Prec)dtype, false);
    if (out_g) out_g[g] = P;
    mx = std::max(mx, c.off);
  }
  return mx;
}

size_t shampoo_update_stats_workspace_bytes(const shp_plan* plan, int32_t dtype) {
  if (!plan || !valid_dtype(dtype)) return 0;
  return stats_ws(plan, dtype, nullptr, nullptr);
}

shp_status shampoo_update_stats(const shp_plan* plan, const float* const* g_stacks, float* const* f_stacks,
                                float beta2, float alpha, int32_t dtype, void* workspace, size_t ws_bytes,
                                void* stream) {
  const NvtxRange nvtx_range("shampoo_update_stats");
  shp_status s = check_plan(plan, true);
  if (s) return s;
  if (!g_stacks || !f_stacks) return fail(SHP_ERR_INVALID_ARG, "g_stacks and f_stacks must be non-NULL");
  if (!valid_dtype(dtype)) return fail(SHP_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (!std::isfinite(beta2) || !std::isfinite(alpha)) return fail(SHP_ERR_INVALID_ARG, "beta2/alpha not finite");
  const size_t need = stats_ws(plan, dtype, nullptr, nullptr);
  if (need && (!workspace || ws_bytes < need))
    return fail(SHP_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  for (int g = 0; g < plan->n_g(); ++g)
    if (!g_stacks[g]) return fail(SHP_ERR_INVALID_ARG, "g_stacks[%d] is NULL", g);
  for (int f = 0; f < plan->n_f(); ++f)
    if (!f_stacks[f]) return fail(SHP_ERR_INVALID_ARG, "f_stacks[%d] is NULL", f);
  for (int g = 0; g < plan->n_g(); ++g)
    if (plan->gb[3 * g + 2] > 32767 || plan->gb[3 * g] % 4 || plan->gb[3 * g + 1] % 4)
      return fail(SHP_ERR_UNSUPPORTED, "gradient bucket %d: count <= 32767 and sides % 4 == 0 required", g);
  cudaStream_t st = as_stream(stream);
  const Prec pr = (Prec)dtype;
  for (int g = 0; g < plan->n_g(); ++g) {
    const int m = plan->gb[3 * g], n = plan->gb[3 * g + 1], cnt = plan->gb[3 * g + 2];
    Carver c(workspace);
    Planes P = make_planes(c, cnt, m, n, pr, false);
    CUDA_TRY(launch_to_planes(g_stacks[g], n, (long long)m * n, nullptr, cnt, m, n, 1.f, 0.f, 0.f, nullptr, P, pr,
                              st));
    // the factor bucket of this gradient bucket's left / right factors
    int lb = -1, rb = -1;
    for (int b = 0; b < plan->n_blocks(); ++b) {
      const int32_t* rec = &plan->blocks[b * kBlockFields];
      if (rec[7] == g) {
        lb = rec[9];
        rb = rec[11];
        break;
      }
    }
    GemmGroup gs[2];
    gs[0] = group(m, m, n, &P, 0, &P, 0, 1);  // G G^T
    gs[0].a_idx = nullptr;
    gs[0].epi.o_idx = plan->dev + plan->off_lidx[g];
    gs[0].epi.alpha = alpha;
    gs[0].epi.beta = beta2;
    gs[0].epi.C.f32 = f_stacks[lb];
    gs[0].epi.C.ld = m;
    gs[0].epi.C.bs = (long long)m * m;
    gs[0].epi.O = plain_out(f_stacks[lb], m, (long long)m * m);
    gs[1] = group(n, n, m, &P, 1, &P, 1, 1);  // G^T G
    gs[1].epi.o_idx = plan->dev + plan->off_ridx[g];
    gs[1].epi.alpha = alpha;
    gs[1].epi.beta = beta2;
    if (rb < 0) rb = lb;  // one-sided bucket: the second problem is not launched
    gs[1].epi.C.f32 = f_stacks[rb];
    gs[1].epi.C.ld = n;
    gs[1].epi.C.bs = (long long)n * n;
    gs[1].epi.O = plain_out(f_stacks[rb], n, (long long)n * n);
    if (beta2 == 0.f) {  // do not read (possibly uninitialised) old statistics
      gs[0].epi.C = EpiC();
      gs[1].epi.C = EpiC();
    }
    const int nprob = plan->gside[g] ? 1 : 2;  // one-sided: no right factor
    cudaError_t e = launch_gemm(gs, nprob, cnt, pr, st);
    if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "statistics GEMM: %s", cudaGetErrorString(e));
  }
  return SHP_OK;
}

// ---- inverse roots ---------------------------------------------------------

static shp_status check_root_args(int32_t count, int32_t n, int32_t p, int32_t method, int32_t iters, int32_t dtype,
                                  int32_t scaling, int32_t pi_vectors) {
  if (method < SHP_METHOD_NDB || method > SHP_METHOD_CHEB) return fail(SHP_ERR_INVALID_ARG, "bad method %d", method);
  if (!valid_dtype(dtype)) return fail(SHP_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (scaling != SHP_SCALE_FROBENIUS && scaling != SHP_SCALE_POWER)
    return fail(SHP_ERR_INVALID_ARG, "bad scaling %d", scaling);
  if (count < 1 || count > 32767) return fail(SHP_ERR_SHAPE, "count %d outside [1, 32767]", count);
  if (n < 4 || n > SHP_MAX_N || n % 4) return fail(SHP_ERR_SHAPE, "n %d: need 4 <= n <= %d, n %% 4 == 0", n, SHP_MAX_N);
  if (p != 2 && p != 4 && p != 8) return fail(SHP_ERR_UNSUPPORTED, "root power p must be 2, 4 or 8");
  if (method == SHP_METHOD_CHEB ? (iters < 0 || iters > 1000) : (iters < 1 || iters > 1000))
    return fail(SHP_ERR_INVALID_ARG, "iters %d out of range", iters);
  if (scaling == SHP_SCALE_POWER && (pi_vectors < 1 || pi_vectors > 256 || pi_vectors % 8))
    return fail(SHP_ERR_INVALID_ARG, "pi_vectors %d: need a multiple of 8 in [8, 256]", pi_vectors);
  return SHP_OK;
}

size_t shampoo_inv_root_workspace_bytes(int32_t count, int32_t n, int32_t method, int32_t dtype, int32_t scaling,
                                        int32_t pi_vectors) {
  if (check_root_args(count, n, 4, method, method == SHP_METHOD_CHEB ? 0 : 1, dtype, scaling, pi_vectors)) return 0;
  Carver c(nullptr);
  carve_roots(c, count, n, method, (Prec)dtype, scaling, pi_vectors);
  return c.off;
}

shp_status shampoo_inv_root(const float* A, int32_t count, int32_t n, float eps, int32_t p, int32_t method,
                            int32_t iters, int32_t dtype, int32_t scaling, int32_t pi_vectors, int32_t pi_iters,
                            const float* pi_starts, float* X_out, float* scale_out, int32_t* status_out,
                            void* workspace, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("shampoo_inv_root");
  shp_status s = check_root_args(count, n, p, method, iters, dtype, scaling, pi_vectors);
  if (s) return s;
  if (!A || !X_out || !scale_out || !status_out || !workspace)
    return fail(SHP_ERR_INVALID_ARG, "A, X_out, scale_out, status_out and workspace must be non-NULL");
  if (!std::isfinite(eps) || eps < 0.f) return fail(SHP_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (scaling == SHP_SCALE_POWER && (!pi_starts || pi_iters < 0 || pi_iters > 1000))
    return fail(SHP_ERR_INVALID_ARG, "power scaling needs pi_starts and 0 <= pi_iters <= 1000");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(A) & 15) ||
      (reinterpret_cast<uintptr_t>(X_out) & 15))
    return fail(SHP_ERR_INVALID_ARG, "workspace must be 256-byte aligned, A and X_out 16-byte aligned");
  Carver c(workspace);
  RootBufs r = carve_roots(c, count, n, method, (Prec)dtype, scaling, pi_vectors);
  if (c.off > ws_bytes) return fail(SHP_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, c.off);
  cudaStream_t st = as_stream(stream);
  CUDA_TRY(launch_zero_i32(status_out, count, st));
  const float eps_s = method == SHP_METHOD_CHEB ? 0.f : eps;
  s = compute_scale(A, count, n, eps_s, scaling, pi_vectors, pi_iters, pi_starts, r, scale_out, st);
  if (s) return s;
  const Prec pr = (Prec)dtype;
  if (method == SHP_METHOD_NDB) return run_ndb(A, count, n, eps, iters, p, pr, r, scale_out, X_out, status_out, st);
  if (method == SHP_METHOD_CN) return run_cn(A, count, n, eps, iters, p, pr, r, scale_out, X_out, status_out, st);
  return run_cheb(A, count, n, eps, iters, p, pr, r, scale_out, X_out, status_out, st);
}

size_t shampoo_inv_root_warm_workspace_bytes(int32_t count, int32_t n, int32_t dtype) {
  if (check_root_args(count, n, 4, SHP_METHOD_CN, 1, dtype, SHP_SCALE_FROBENIUS, 16)) return 0;
  Carver c(nullptr);
  carve_roots(c, count, n, SHP_METHOD_CN, (Prec)dtype, SHP_SCALE_FROBENIUS, 16);
  return c.off;
}

shp_status shampoo_inv_root_warm(const float* A, const float* X0, int32_t count, int32_t n, float eps, int32_t p,
                                 int32_t iters, int32_t dtype, float* X_out, int32_t* status_out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("shampoo_inv_root_warm");
  shp_status s = check_root_args(count, n, p, SHP_METHOD_CN, iters, dtype, SHP_SCALE_FROBENIUS, 16);
  if (s) return s;
  if (!A || !X0 || !X_out || !status_out || !workspace)
    return fail(SHP_ERR_INVALID_ARG, "A, X0, X_out, status_out and workspace must be non-NULL");
  if (!std::isfinite(eps) || eps < 0.f) return fail(SHP_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) || (reinterpret_cast<uintptr_t>(A) & 15) ||
      (reinterpret_cast<uintptr_t>(X0) & 15) || (reinterpret_cast<uintptr_t>(X_out) & 15))
    return fail(SHP_ERR_INVALID_ARG, "workspace must be 256-byte aligned, A, X0 and X_out 16-byte aligned");
  Carver c(workspace);
  RootBufs r = carve_roots(c, count, n, SHP_METHOD_CN, (Prec)dtype, SHP_SCALE_FROBENIUS, 16);
  if (c.off > ws_bytes) return fail(SHP_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, c.off);
  cudaStream_t st = as_stream(stream);
  CUDA_TRY(launch_zero_i32(status_out, count, st));
  return run_cn_warm(A, X0, count, n, eps, iters, p, (Prec)dtype, r, X_out, status_out, st);
}

shp_status shampoo_inv_root_evd(const float* A, int32_t count, int32_t n, float eps, int32_t p, int32_t heuristic,
                                float* X_out, float* eig_out, int32_t* status_out, void* stream) {
  const NvtxRange nvtx_range("shampoo_inv_root_evd");
  if (n < 1 || n > SHP_EVD_MAX_N) return fail(SHP_ERR_SHAPE, "n %d: need 1 <= n <= %d", n, SHP_EVD_MAX_N);
  if (count < 1) return fail(SHP_ERR_SHAPE, "count %d must be >= 1", count);
  if (p != 2 && p != 4 && p != 8) return fail(SHP_ERR_UNSUPPORTED, "root power p must be 2, 4 or 8");
  if (heuristic < SHP_EVD_CORRECTED || heuristic > SHP_EVD_SHMP)
    return fail(SHP_ERR_INVALID_ARG, "bad heuristic %d", heuristic);
  if (!A || !X_out || !status_out) return fail(SHP_ERR_INVALID_ARG, "A, X_out and status_out must be non-NULL");
  if (!std::isfinite(eps) || eps < 0.f) return fail(SHP_ERR_INVALID_ARG, "eps must be finite and >= 0");
  cudaError_t e = launch_evd_root(A, count, n, eps, p, heuristic, X_out, eig_out, status_out, as_stream(stream));
  if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "EVD launch: %s", cudaGetErrorString(e));
  return SHP_OK;
}

// ---- precondition ----------------------------------------------------------

struct PrecBufs {
  Planes G, XL, XR, P;
};

static PrecBufs carve_prec(Carver& c, int cnt, int m, int n, Prec pr) {
  PrecBufs b;
  b.G = make_planes(c, cnt, m, n, pr, false);
  b.XL = make_planes(c, cnt, m, m, pr, false);
  b.XR = make_planes(c, cnt, n, n, pr, false);
  b.P = make_planes(c, cnt, m, n, pr, false);
  return b;
}

size_t shampoo_precondition_workspace_bytes(const shp_plan* plan, int32_t dtype) {
  if (!plan || !valid_dtype(dtype)) return 0;
  size_t mx = 0;
  for (int g = 0; g < plan->n_g(); ++g) {
    Carver c(nullptr);
    carve_prec(c, plan->gb[3 * g + 2], plan->gb[3 * g], plan->gb[3 * g + 1], (Prec)dtype);
    mx = std::max(mx, c.off);
  }
  return mx;
}

shp_status shampoo_precondition(const shp_plan* plan, const float* const* roots, const float* const* g_stacks,
                                float* const* d_stacks, float* block_dnorm2, int32_t dtype, void* workspace,
                                size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("shampoo_precondition");
  shp_status s = check_plan(plan, true);
  if (s) return s;
  if (!roots || !g_stacks || !d_stacks || !block_dnorm2)
    return fail(SHP_ERR_INVALID_ARG, "roots, g_stacks, d_stacks and block_dnorm2 must be non-NULL");
  if (!valid_dtype(dtype)) return fail(SHP_ERR_INVALID_ARG, "bad dtype %d", dtype);
  const size_t need = shampoo_precondition_workspace_bytes(plan, dtype);
  if (!workspace || ws_bytes < need) return fail(SHP_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  for (int g = 0; g < plan->n_g(); ++g)
    if (plan->gb[3 * g + 2] > 65535 || plan->gb[3 * g] % 4 || plan->gb[3 * g + 1] % 4)
      return fail(SHP_ERR_UNSUPPORTED, "gradient bucket %d: count <= 65535 and sides % 4 == 0 required", g);
  cudaStream_t st = as_stream(stream);
  const Prec pr = (Prec)dtype;
  CUDA_TRY(cudaMemsetAsync(block_dnorm2, 0, sizeof(float) * plan->n_blocks(), st));
  const int32_t* gstack = plan->image.data() + plan->off_gstack;
  for (int g = 0; g < plan->n_g(); ++g) {
    const int m = plan->gb[3 * g], n = plan->gb[3 * g + 1], cnt = plan->gb[3 * g + 2];
    int lb = -1, rb = -1;
    for (int b = 0; b < plan->n_blocks(); ++b) {
      const int32_t* rec = &plan->blocks[b * kBlockFields];
      if (rec[7] == g) {
        lb = rec[9];
        rb = rec[11];
        break;
      }
    }
    const bool one_sided = plan->gside[g] != 0;
    if (!roots[lb] || (!one_sided && !roots[rb]) || !g_stacks[g] || !d_stacks[g])
      return fail(SHP_ERR_INVALID_ARG, "NULL stack pointer for gradient bucket %d", g);
    Carver c(workspace);
    PrecBufs b = carve_prec(c, cnt, m, n, pr);
    CUDA_TRY(launch_to_planes(g_stacks[g], n, (long long)m * n, nullptr, cnt, m, n, 1.f, 0.f, 0.f, nullptr, b.G, pr,
                              st));
    CUDA_TRY(launch_to_planes(roots[lb], m, (long long)m * m, plan->dev + plan->off_lidx[g], cnt, m, m, 1.f, 0.f, 0.f,
                              nullptr, b.XL, pr, st));
    if (one_sided) {  // D = X_L G
      GemmGroup g1 = group(m, n, m, &b.XL, 0, &b.G, 1);
      g1.epi.O = plain_out(d_stacks[g], n, (long long)m * n);
      g1.epi.sumsq = block_dnorm2 + gstack[g];
      cudaError_t e = launch_gemm(&g1, 1, cnt, pr, st);
      if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "precondition GEMM: %s", cudaGetErrorString(e));
      continue;
    }
    CUDA_TRY(launch_to_planes(roots[rb], n, (long long)n * n, plan->dev + plan->off_ridx[g], cnt, n, n, 1.f, 0.f, 0.f,
                              nullptr, b.XR, pr, st));
    GemmGroup g1 = group(m, n, n, &b.G, 0, &b.XR, 1);  // P = G X_R
    g1.epi.O = as_out(b.P, false);
    cudaError_t e = launch_gemm(&g1, 1, cnt, pr, st);
    if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "precondition GEMM 1: %s", cudaGetErrorString(e));
    GemmGroup g2 = group(m, n, m, &b.XL, 0, &b.P, 1);  // D = X_L P
    g2.epi.O = plain_out(d_stacks[g], n, (long long)m * n);
    g2.epi.sumsq = block_dnorm2 + gstack[g];
    e = launch_gemm(&g2, 1, cnt, pr, st);
    if (e != cudaSuccess) return fail(SHP_ERR_CUDA, "precondition GEMM 2: %s", cudaGetErrorString(e));
  }
  return SHP_OK;
}

// ---- graft + update --------------------------------------------------------

size_t shampoo_graft_step_workspace_bytes(const shp_plan* plan) {
  if (!plan) return 0;
  return sizeof(double) * (size_t)plan->n_blocks();
}

shp_status shampoo_graft_step(const shp_plan* plan, float* const* W, const float* const* G,
                              const float* const* d_stacks, const float* block_dnorm2, float* const* m,
                              float* const* v, int32_t graft, float lr, float beta1, float beta2, float eps,
                              float weight_decay, int32_t step, int32_t graft_per_block, void* workspace,
                              size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range("shampoo_graft_step");
  shp_status s = check_plan(plan, true);
  if (s) return s;
  if (graft < SHP_GRAFT_NONE || graft > SHP_GRAFT_ADAM) return fail(SHP_ERR_INVALID_ARG, "bad graft %d", graft);
  if (!W || !d_stacks || !block_dnorm2) return fail(SHP_ERR_INVALID_ARG, "W, d_stacks, block_dnorm2 must be non-NULL");
  if (graft != SHP_GRAFT_NONE && !G) return fail(SHP_ERR_INVALID_ARG, "G is required for grafting");
  if (step < 1) return fail(SHP_ERR_INVALID_ARG, "step must be >= 1");
  if (!std::isfinite(lr) || !std::isfinite(weight_decay) || !std::isfinite(eps))
    return fail(SHP_ERR_INVALID_ARG, "non-finite scalar");
  const size_t need = shampoo_graft_step_workspace_bytes(plan);
  if (!workspace || ws_bytes < need) return fail(SHP_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  if (plan->n_g() > kMaxBuckets) return fail(SHP_ERR_UNSUPPORTED, "more than %d gradient buckets", kMaxBuckets);
  for (int l = 0; l < plan->n_layers(); ++l) {
    if (!W[l] || (graft != SHP_GRAFT_NONE && !G[l])) return fail(SHP_ERR_INVALID_ARG, "NULL pointer for layer %d", l);
    if (graft == SHP_GRAFT_ADAM && (!m || !v || !m[l] || !v[l]))
      return fail(SHP_ERR_INVALID_ARG, "Adam grafting needs m and v for layer %d", l);
    if (graft == SHP_GRAFT_ADAGRAD && (!v || !v[l])) return fail(SHP_ERR_INVALID_ARG, "AdaGrad needs v for layer %d", l);
  }
  BucketArgs dp;
  for (int g = 0; g < plan->n_g(); ++g) dp.ptr[g] = const_cast<float*>(d_stacks[g]);
  GraftScalars sc;
  sc.kind = graft;
  sc.per_block = graft_per_block ? 1 : 0;
  sc.beta1 = beta1;
  sc.beta2 = beta2;
  sc.eps = eps;
  sc.bc1 = (float)(1.0 - std::pow((double)beta1, (double)step));
  sc.bc2 = (float)(1.0 - std::pow((double)beta2, (double)step));
  sc.lr = lr;
  sc.wd = weight_decay;
  if (graft == SHP_GRAFT_ADAM && (sc.bc1 <= 0.f || sc.bc2 <= 0.f))
    return fail(SHP_ERR_INVALID_ARG, "Adam needs beta1, beta2 < 1");
  cudaStream_t st = as_stream(stream);
  double* gsum = static_cast<double*>(workspace);
  CUDA_TRY(cudaMemsetAsync(gsum, 0, need, st));
  const int32_t* lf = plan->image.data() + plan->off_layer_first;
  const int32_t* dlf = plan->dev + plan->off_layer_first;
  const int32_t* dgs = plan->dev + plan->off_gstack;
  // pass 1 over all layers first: layerwise rho needs every block's sum
  if (graft != SHP_GRAFT_NONE) {
    for (int l0 = 0; l0 < plan->n_layers(); l0 += kMaxLayersPerLaunch) {
      const int l1 = std::min(plan->n_layers(), l0 + kMaxLayersPerLaunch);
      LayerArgs la = layer_args(plan, l0, l1, W, G, m, v);
      long long mx = 0;
      for (int b = lf[l0]; b < lf[l1]; ++b)
        mx = std::max(mx, (long long)plan->blocks[b * kBlockFields + 5] * plan->blocks[b * kBlockFields + 6]);
      CUDA_TRY(launch_graft_pass1(plan->dev, lf[l0], lf[l1] - lf[l0], mx, la, sc, gsum, st));
    }
  }
  for (int l0 = 0; l0 < plan->n_layers(); l0 += kMaxLayersPerLaunch) {
    const int l1 = std::min(plan->n_layers(), l0 + kMaxLayersPerLaunch);
    LayerArgs la = layer_args(plan, l0, l1, W, G, m, v);
    long long mx = 0;
    for (int b = lf[l0]; b < lf[l1]; ++b)
      mx = std::max(mx, (long long)plan->blocks[b * kBlockFields + 5] * plan->blocks[b * kBlockFields + 6]);
    CUDA_TRY(launch_graft_pass2(plan->dev, dlf, dgs, lf[l0], lf[l1] - lf[l0], mx, la, dp, sc, gsum, block_dnorm2, st));
  }
  return SHP_OK;
}

}  // extern "C"
