// Inverse roots by eigendecomposition with the dampening heuristics of
// "DASH: Faster Shampoo via Batched Block Preconditioning and Efficient
// Inverse-Root Solvers", B.1 (regularisation for EVD) and B.2 (corrected
// spectrum, shifted ReLU, ABS), the fourth method that paper compares with
// Newton-DB, coupled Newton and Chebyshev (§3, §5).
//
// One CTA per matrix.  The damped matrix L + eps I (float64) and the
// accumulated rotations V (float32) live in shared memory with row stride
// n + 1, so row and column sweeps are both free of bank conflicts; that
// bounds n at 128 (128 x 129 x (8 + 4) B = 198 KB).  The eigensolver is
// two-sided cyclic Jacobi in the round-robin pair order: each round rotates
// n/2 disjoint (p, q) planes at once, one warp per plane: the warp works
// out its plane's rotation and rotates the two rows, and after a barrier the
// same warps rotate the two columns of A and of V (two barriers a round).
// A plane is
// rotated only while its off-diagonal entry is above 2^-21 sqrt(|a_pp
// a_qq|); a sweep without rotations ends the solve.  Then X = V diag(f(mu))
// V^T with f the chosen heuristic, written row-major in float32.
//
// Precision: every entry of A is rotated twice per round and a solve takes
// 10-15 sweeps, so in float32 the rounding of A grows to ~10 u |A| and the
// roots of ill-conditioned matrices lose two digits against a float32
// LAPACK solve; A is therefore kept and rotated in float64 (half the FP32
// rate on this part, and the kernel is bound by its barriers, not by ALU).
// V stays float32 and is updated in Rutishauser's form x - s (y + tau x),
// tau = s / (1 + c), whose rounding keeps the rotation orthogonal to O(s^4)
// instead of letting tiny late rotations grow the columns.
#include "../../include/shampoo.h"
#include "internal.h"
#include "ptx.cuh"

namespace shp {
namespace {

constexpr int kEvdThreads = 512;
constexpr int kEvdWarps = kEvdThreads / 32;
constexpr int kEvdMaxSweeps = 40;
constexpr float kRelTol = 4.76837158e-7f;  // 2^-21

__device__ __forceinline__ float heuristic_factor(double mu, double mu_min, double eps, int p, int heuristic) {
  const double lam = mu - eps;  // corrected spectrum: the eigenvalue of L
  double d;
  if (heuristic == SHP_EVD_SHIFTED_RELU) {
    const double r = lam - eps;
    return r > 0.0 ? inv_root_mult((float)r, p) : 0.f;
  } else if (heuristic == SHP_EVD_ABS_ADD) {
    d = fabs(lam) + eps;
  } else if (heuristic == SHP_EVD_SHMP) {
    d = mu - fmin(mu_min, 0.0) + eps;
  } else {
    d = fmax(lam, 0.0) + eps;
  }
  return inv_root_mult((float)d, p);
}

__global__ void __launch_bounds__(kEvdThreads, 1)
    evd_root_kernel(const float* __restrict__ A, int n, float eps, int p, int heuristic, float* __restrict__ X,
                    float* __restrict__ eig, int* __restrict__ status) {
  extern __shared__ double smem[];
  __shared__ int pr_p[64], pr_q[64];
  __shared__ double pr_s[64], pr_tau[64], pr_t[64], pr_app[64], pr_aqq[64], pr_apq[64];
  __shared__ float fval[128];
  __shared__ int rotated, flags;
  __shared__ double mu_min_s;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int ld = n + 1;
  double* a = smem;
  float* v = reinterpret_cast<float*>(smem + n * ld);
  const long long nn = (long long)n * n;
  const float* Ab = A + (long long)blockIdx.x * nn;

  for (int i = tid; i < n * n; i += blockDim.x) {
    const int r = i / n, c = i - r * n;
    a[r * ld + c] = (double)Ab[i];
    v[r * ld + c] = r == c ? 1.f : 0.f;
  }
  if (tid == 0) {
    rotated = 0;
    flags = 0;
  }
  __syncthreads();
  for (int i = tid; i < n * n; i += blockDim.x) {  // symmetrise, damp
    const int r = i / n, c = i - r * n;
    if (r < c) {
      const double s = 0.5 * (a[r * ld + c] + a[c * ld + r]);
      a[r * ld + c] = s;
      a[c * ld + r] = s;
    } else if (r == c) {
      a[r * ld + c] += (double)eps;
    }
  }
  __syncthreads();

  const int m = n + (n & 1);  // an odd n plays a dummy index n
  const int half = m / 2;
  bool converged = n == 1;
  int sweeps = 0;
  for (; sweeps < kEvdMaxSweeps && !converged; ++sweeps) {
    for (int round = 0; round < m - 1; ++round) {
      // Rotation angles and rows: warp w owns pairs w, w + 16, ...; its
      // lanes read the pivot entries (broadcast), agree on the rotation,
      // then rotate rows p and q, 32 columns at a time.  No other warp
      // touches those two rows in this phase.
      for (int k = warp; k < half; k += kEvdWarps) {
        int P = k == 0 ? 0 : 1 + (k - 1 + round) % (m - 1);
        int Q = 1 + (m - 2 - k + round) % (m - 1);
        if (P > Q) {
          const int t = P;
          P = Q;
          Q = t;
        }
        double s = 0.0, tau2 = 0.0, t = 0.0, app = 0.0, aqq = 0.0, apq = 0.0;
        if (Q < n) {
          app = a[P * ld + P];
          aqq = a[Q * ld + Q];
          apq = a[P * ld + Q];
          if (apq != 0.0 && fabs(apq) > kRelTol * sqrt(fabs(app) * fabs(aqq))) {
            // tan of the angle that zeroes a_pq, the smaller root (|t| <= 1)
            const double th = (aqq - app) / (2.0 * apq);
            const double ath = fabs(th);
            t = ath > 1e150 ? 0.5 / th : copysign(1.0, th) / (ath + sqrt(1.0 + th * th));
            const double c = 1.0 / sqrt(1.0 + t * t);
            s = t * c;
            tau2 = s / (1.0 + c);
          }
        }
        if (lane == 0) {
          pr_p[k] = P;
          pr_q[k] = Q;
          pr_s[k] = s;
          pr_tau[k] = tau2;
          pr_t[k] = t;
          pr_app[k] = app;
          pr_aqq[k] = aqq;
          pr_apq[k] = apq;
          if (s != 0.0) rotated = 1;
        }
        __syncwarp();  // every lane has read the pivot entries
        if (s == 0.0) continue;
        double* rp = a + P * ld;
        double* rq = a + Q * ld;
        for (int j = lane; j < n; j += 32) {
          const double x = rp[j], y = rq[j];
          rp[j] = x - s * (y + tau2 * x);
          rq[j] = y + s * (x - tau2 * y);
        }
      }
      __syncthreads();
      // columns p, q of A and V <- . J; the 2 x 2 pivot block set exactly
      for (int k = warp; k < half; k += kEvdWarps) {
        const double s = pr_s[k];
        if (s == 0.0) continue;
        const double tau2 = pr_tau[k];
        const int P = pr_p[k], Q = pr_q[k];
        const float sf = (float)s, tf = (float)tau2;
        for (int r = lane; r < n; r += 32) {
          double* ar = a + r * ld;
          const double x = ar[P], y = ar[Q];
          double nx = x - s * (y + tau2 * x), ny = y + s * (x - tau2 * y);
          if (r == P) {
            nx = pr_app[k] - pr_t[k] * pr_apq[k];
            ny = 0.0;
          } else if (r == Q) {
            nx = 0.0;
            ny = pr_aqq[k] + pr_t[k] * pr_apq[k];
          }
          ar[P] = nx;
          ar[Q] = ny;
          float* vr = v + r * ld;
          const float vx = vr[P], vy = vr[Q];
          vr[P] = vx - sf * (vy + tf * vx);
          vr[Q] = vy + sf * (vx - tf * vy);
        }
      }
      __syncthreads();
    }
    const int any = rotated;
    __syncthreads();
    if (tid == 0) rotated = 0;
    __syncthreads();
    converged = any == 0;
  }

  // eigenvalues mu_i = a_ii of L + eps I; the SHMP shift needs min mu
  if (tid < 32) {
    double mn = INFINITY;
    for (int i = tid; i < n; i += 32) mn = fmin(mn, a[i * ld + i]);
    for (int o = 16; o; o >>= 1) mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    if (tid == 0) mu_min_s = mn;
  }
  __syncthreads();
  const double mu_min = mu_min_s;
  for (int i = tid; i < n; i += blockDim.x) fval[i] = heuristic_factor(a[i * ld + i], mu_min, eps, p, heuristic);
  if (eig) {  // corrected spectrum, ascending (ties by index)
    for (int i = tid; i < n; i += blockDim.x) {
      const double mi = a[i * ld + i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const double mj = a[j * ld + j];
        rank += (mj < mi) || (mj == mi && j < i);
      }
      eig[(long long)blockIdx.x * n + rank] = (float)(mi - (double)eps);
    }
  }
  __syncthreads();

  float* Xb = X + (long long)blockIdx.x * nn;
  bool bad = false;
  for (int idx = tid; idx < n * n; idx += blockDim.x) {
    const int i = idx / n, j = idx - i * n;
    const float* vi = v + i * ld;
    const float* vj = v + j * ld;
    float acc = 0.f;
    for (int k = 0; k < n; ++k) acc = fmaf(vi[k] * fval[k], vj[k], acc);
    Xb[idx] = acc;
    bad |= !isfinite(acc);
  }
  if (bad) atomicOr(&flags, SHP_ROOT_NONFINITE);
  __syncthreads();
  if (tid == 0) status[blockIdx.x] = flags | (converged ? 0 : SHP_ROOT_UNCONVERGED) | (sweeps << 8);
}

}  // namespace

size_t evd_smem_bytes(int n) { return (sizeof(double) + sizeof(float)) * (size_t)n * (n + 1); }

cudaError_t launch_evd_root(const float* A, int count, int n, float eps, int p, int heuristic, float* X, float* eig,
                            int* status, cudaStream_t stream) {
  const size_t smem = evd_smem_bytes(n);
  cudaError_t e = cudaFuncSetAttribute(evd_root_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  evd_root_kernel<<<count, kEvdThreads, smem, stream>>>(A, n, eps, p, heuristic, X, eig, status);
  count_launch();
  return cudaGetLastError();
}

}  // namespace shp
