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
// n/2 disjoint (p, q) planes at once.  The rotations are worked out first;
// after a barrier, A <- J^T A J is applied one 2 x 2 block (two rows of one
// plane, two columns of another) at a time in registers, V <- V J alongside,
// so every entry of A and V is read and written once a round (two barriers
// a round).  A plane is
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
  __shared__ int pr_x[64], pr_y[64];
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

  bool bad_in = false;  // a NaN / Inf in A: the rotation test skips such entries, so flag it here
  for (int i = tid; i < n * n; i += blockDim.x) {
    const int r = i / n, c = i - r * n;
    const float x = Ab[i];
    bad_in |= !isfinite(x);
    a[r * ld + c] = (double)x;
    v[r * ld + c] = r == c ? 1.f : 0.f;
  }
  if (tid == 0) {
    rotated = 0;
    flags = 0;
  }
  __syncthreads();
  if (bad_in) atomicOr(&flags, SHP_ROOT_NONFINITE);
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
      // Rotations of this round's planes (X, Y) = (players at positions k
      // and m-1-k; the formulas need no ordering).
      for (int k = tid; k < half; k += blockDim.x) {
        const int X = k == 0 ? 0 : 1 + (k - 1 + round) % (m - 1);
        const int Y = 1 + (m - 2 - k + round) % (m - 1);
        double s = 0.0, tau2 = 0.0, t = 0.0, axx = 0.0, ayy = 0.0, axy = 0.0;
        if (X < n && Y < n) {
          axx = a[X * ld + X];
          ayy = a[Y * ld + Y];
          axy = a[X * ld + Y];
          if (axy != 0.0 && fabs(axy) > kRelTol * sqrt(fabs(axx) * fabs(ayy))) {
            // tan of the angle that zeroes a_xy, the smaller root (|t| <= 1)
            const double th = (ayy - axx) / (2.0 * axy);
            const double ath = fabs(th);
            t = ath > 1e150 ? 0.5 / th : copysign(1.0, th) / (ath + sqrt(1.0 + th * th));
            const double c = 1.0 / sqrt(1.0 + t * t);
            s = t * c;
            tau2 = s / (1.0 + c);
            rotated = 1;
          }
        }
        pr_x[k] = X;
        pr_y[k] = Y;
        pr_s[k] = s;
        pr_tau[k] = tau2;
        pr_t[k] = t;
        pr_app[k] = axx;
        pr_aqq[k] = ayy;
        pr_apq[k] = axy;
      }
      __syncthreads();
      // A <- J^T A J and V <- V J one 2 x 2 block at a time: block (k, kc)
      // holds rows X_k, Y_k and columns X_kc, Y_kc; it is rotated by plane
      // k on the left and plane kc on the right, in registers.  Warp w takes
      // row planes w, w + 16, ...; its lanes take consecutive column planes,
      // whose columns are consecutive players (conflict-free).
      for (int k = warp; k < half; k += kEvdWarps) {
        const int X = pr_x[k], Y = pr_y[k];
        const bool xv = X < n, yv = Y < n;
        const double s = pr_s[k], tau2 = pr_tau[k];
        for (int kc = lane; kc < half; kc += 32) {
          const double sc = pr_s[kc];
          if (s == 0.0 && sc == 0.0) continue;
          const double tc = pr_tau[kc];
          const int Xc = pr_x[kc], Yc = pr_y[kc];
          const bool xcv = Xc < n, ycv = Yc < n;
          double* ax = a + X * ld;
          double* ay = a + Y * ld;
          double b00 = (xv && xcv) ? ax[Xc] : 0.0, b01 = (xv && ycv) ? ax[Yc] : 0.0;
          double b10 = (yv && xcv) ? ay[Xc] : 0.0, b11 = (yv && ycv) ? ay[Yc] : 0.0;
          if (s != 0.0) {  // rows X, Y <- J_k^T
            double u = b00, w = b10;
            b00 = u - s * (w + tau2 * u);
            b10 = w + s * (u - tau2 * w);
            u = b01;
            w = b11;
            b01 = u - s * (w + tau2 * u);
            b11 = w + s * (u - tau2 * w);
          }
          if (sc != 0.0) {  // columns X_kc, Y_kc <- . J_kc
            double u = b00, w = b01;
            b00 = u - sc * (w + tc * u);
            b01 = w + sc * (u - tc * w);
            u = b10;
            w = b11;
            b10 = u - sc * (w + tc * u);
            b11 = w + sc * (u - tc * w);
          }
          if (kc == k && s != 0.0) {  // the pivot block, exactly
            b00 = pr_app[k] - pr_t[k] * pr_apq[k];
            b11 = pr_aqq[k] + pr_t[k] * pr_apq[k];
            b01 = 0.0;
            b10 = 0.0;
          }
          if (xv && xcv) ax[Xc] = b00;
          if (xv && ycv) ax[Yc] = b01;
          if (yv && xcv) ay[Xc] = b10;
          if (yv && ycv) ay[Yc] = b11;
          if (sc != 0.0) {  // V rows X, Y, columns X_kc, Y_kc <- . J_kc
            const float sf = (float)sc, tf = (float)tc;
            if (xv) {
              float* vx = v + X * ld;
              const float u = vx[Xc], w = vx[Yc];
              vx[Xc] = u - sf * (w + tf * u);
              vx[Yc] = w + sf * (u - tf * w);
            }
            if (yv) {
              float* vy = v + Y * ld;
              const float u = vy[Xc], w = vy[Yc];
              vy[Xc] = u - sf * (w + tf * u);
              vy[Yc] = w + sf * (u - tf * w);
            }
          }
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
