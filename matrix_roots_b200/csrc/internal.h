// Host/device structures shared by the kernels and the C-ABI layer.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace shp {

enum Prec : int { P_FP32 = 0, P_TF32 = 1, P_FP16 = 2, P_BF16 = 3 };

// A stack of `count` matrices (rows x cols, leading dimension ld, batch
// stride bs elements) stored in the planes a tensor-core pass reads:
//   FP32 : per matrix b a power-of-two scale 2^exp[b]; with y = x * 2^e,
//          h16 = fp16(y) and h16lo = fp16((y - h16) * 2^11), so that
//          y = h16 + h16lo * 2^-11 to about 22 bits; f32 = x (may be null);
//          amax[b] = max |x| of the matrix
//   TF32 : f32 = full value
//   FP16 / BF16 : f32 = full value (may be null), h16 = half copy
struct Planes {
  float* f32 = nullptr;
  void* h16 = nullptr;
  void* h16lo = nullptr;
  int* exp = nullptr;
  float* amax = nullptr;
  int h16_bf = 0;  // 1 when h16 holds bfloat16
  int rows = 0, cols = 0, ld = 0;
  long long bs = 0;
  int count = 0;
};

// Epilogue input C (its full fp32 value) and outputs.
struct EpiC {
  const float* f32 = nullptr;
  const float* amax = nullptr;  // per-matrix max |C| (FP32 planes), for the output scale bound
  int ld = 0;
  long long bs = 0;
};
struct EpiOut {
  float* f32 = nullptr;  // full value (may be null)
  void* h16 = nullptr;   // half copy, or the scaled fp16 high part when h16lo != null
  void* h16lo = nullptr;
  int* exp = nullptr;
  float* amax = nullptr;
  int amax_n = 0;  // entries of amax, cleared before the launch
  int h16_bf = 0;
  int ld = 0;
  long long bs = 0;
};

// One problem of a (grouped) batched GEMM  D[b] = A[b] (M x K) * B[b] (K x N)
// followed by the fused epilogue
//   r = mult_b * (alpha * D + beta * C + gamma * I)        -> O
//   x = mult_b * (alpha2 * r0 + beta2 * C + gamma2 * I)     -> X (optional)
// with r0 = alpha * D + beta * C + gamma * I (r before the multiplier)
//   sumsq[ob] += sum r^2 ; status[ob] |= 1 if r not finite
// where mult_b = bscale[b]^(-1/root_p) when bscale != null, else 1.
struct GroupDev {
  int M = 0, N = 0, K = 0;
  int a_mn = 0, b_mn = 0;  // 1: operand stored MN-major (K rows x M/N cols)
  const int* a_idx = nullptr;
  const int* b_idx = nullptr;
  // FP32 planes of the operands: scale exponents and max |x|
  const int* a_exp = nullptr;
  const int* b_exp = nullptr;
  const float* a_amax = nullptr;
  const float* b_amax = nullptr;
  const int* o_idx = nullptr;
  float alpha = 1.f, beta = 0.f, gamma = 0.f;
  const float* bscale = nullptr;
  EpiC C;
  EpiOut O;
  EpiOut X;
  float alpha2 = 0.f, beta2 = 0.f, gamma2 = 0.f;
  float* sumsq = nullptr;
  int* status = nullptr;
  int root_p = 4;  // the multiplier is bscale^(-1/root_p)
  int vec4 = 0;  // set by the launcher: N, leading dimensions and bases allow 16-byte row segments
  // set by the launcher from GemmGroup::sym: only the tiles on and above the
  // diagonal are computed, each off-diagonal one also written transposed
  int sym = 0;
};

struct alignas(64) GemmParams {
  CUtensorMap tmA[2][2];  // [group][plane]
  CUtensorMap tmB[2][2];
  GroupDev g[2];
  int ngroups;
  int batch;
  // persistent schedule: tiles of group 0 (batch x mt x nt, matrix-major)
  // come first, then group 1
  int mt[2], nt[2];
  int tiles0, total_tiles;
  // 1: the MN-major operand's map is a 4-D view (inner BK-element chunk,
  // K rows, chunk index, matrix) that brings a whole tile in one load
  int a4d[2], b4d[2];
};

// Host description of one group before tensor maps are built.
struct GemmGroup {
  int M = 0, N = 0, K = 0;
  const Planes* A = nullptr;
  int a_mn = 0;
  const int* a_idx = nullptr;
  const Planes* B = nullptr;
  int b_mn = 0;
  const int* b_idx = nullptr;
  // 1: the product is symmetric in exact arithmetic (both operands are
  // polynomials in one symmetric matrix, or G G^T / G^T G) and C, when read,
  // is symmetric: the launcher computes the upper tiles only and mirrors
  // them (ignored unless M == N, the tile is square and rows are 16-byte)
  int sym = 0;
  GroupDev epi;  // epilogue part (M/N/K/majors/idx filled by the launcher)
};

// prec: the arithmetic of the tensor-core passes (FP32 = three fp16 passes on
// the scaled hi / lo split).
cudaError_t launch_gemm(const GemmGroup* groups, int ngroups, int batch, Prec prec, cudaStream_t stream);

// ---- elementwise / reduction kernels (kernels.cu) ------------------------

// dst = (alpha/s_b) * src + (eps/s_b + delta) * I, written in the planes of
// `dst` for precision `prec`.  src: count matrices rows x cols (ld, bs),
// optional batch index map; s_b = scale[b] or 1.  For FP32 planes the scale
// exponent comes from max |dst| per matrix: found by a first pass, or bounded
// by |alpha/s_b| src_amax[src b] + |eps/s_b + delta| when src_amax is given.
cudaError_t launch_to_planes(const float* src, int src_ld, long long src_bs, const int* src_idx, int count,
                             int rows, int cols, float alpha, float eps, float delta, const float* scale,
                             const Planes& dst, Prec prec, cudaStream_t stream, const float* src_amax = nullptr);

// sums[b] = sum_ij (L_ij + eps*delta_ij)^2 for each matrix (double atomics)
// and, when amax is given, amax[b] = max_ij |L_ij|.  n, ld, bs multiples of 4.
cudaError_t launch_frob_sumsq(const float* L, int n, int ld, long long bs, int count, float eps, double* sums,
                              cudaStream_t stream, float* amax = nullptr);
// scale[b] = sqrt(sums[b]) * factor[b] (factor may be null)
cudaError_t launch_sqrt_scale(const double* sums, const float* factor, float* scale, int count,
                              cudaStream_t stream);

// Multi-power-iteration helpers (fp16 matvec operands, fp32 accumulation).
cudaError_t launch_pi_start_batched(const float* starts, int v, int n, void* vt_h16, int ld, long long bs, int count,
                                    cudaStream_t stream);
cudaError_t launch_pi_normalize(const float* W, int n, int v, int w_ld, long long w_bs, int count, void* vt_h16,
                                int vt_ld, long long vt_bs, cudaStream_t stream);
cudaError_t launch_pi_rayleigh(const float* W, const void* vt_h16, int n, int v, int w_ld, long long w_bs,
                               int vt_ld, long long vt_bs, int count, const double* frob_sums, float* scale,
                               cudaStream_t stream);

cudaError_t launch_zero_i32(int* p, size_t n, cudaStream_t stream);

// Inverse roots by Jacobi eigendecomposition, one CTA per matrix (evd.cu).
size_t evd_smem_bytes(int n);
cudaError_t launch_evd_root(const float* A, int count, int n, float eps, int p, int heuristic, float* X, float* eig,
                            int* status, cudaStream_t stream);

// Host-side count of kernel launches issued by the library.
void count_launch();
unsigned long long launch_total();

// Reads and clears the device error word (synchronous).
cudaError_t read_and_clear_dev_error(int* out);

// Sets the calling thread's shampoo_last_error() message.
void set_last_error(const char* msg);

}  // namespace shp
