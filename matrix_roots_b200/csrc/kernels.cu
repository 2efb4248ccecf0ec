// Streaming kernels around the GEMM engine: operand-plane conversion with the
// damping / scaling prologues of the root iterations, the Frobenius-norm
// reduction and the multi-power-iteration helpers ("DASH: Faster Shampoo via
// Batched Block Preconditioning and Efficient Inverse-Root Solvers", §3
// Matrix scaling and Power-Iteration).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace shp {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void put(const Planes& d, long long off, float v, int prec, float sc) {
  if (d.f32) d.f32[off] = v;
  if (prec == P_FP32) {
    __half hi, lo;
    split16(v * sc, hi, lo);
    reinterpret_cast<__half*>(d.h16)[off] = hi;
    reinterpret_cast<__half*>(d.h16lo)[off] = lo;
  } else if (prec == P_FP16 || prec == P_BF16) {
    if (d.h16_bf)
      reinterpret_cast<__nv_bfloat16*>(d.h16)[off] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<__half*>(d.h16)[off] = __float2half_rn(v);
  }
}

// amax[b] = max |(alpha/s_b) src_b + (eps/s_b + delta) I| (amax cleared before).
__global__ void amax_affine_kernel(const float* __restrict__ src, int src_ld, long long src_bs,
                                   const int* __restrict__ src_idx, int rows, int cols, float alpha, float eps,
                                   float delta, const float* __restrict__ scale, float* __restrict__ amax) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const long long sb = src_idx ? src_idx[b] : b;
  const float inv_s = scale ? 1.f / scale[b] : 1.f;
  const float a = alpha * inv_s;
  const float d = eps * inv_s + delta;
  const float* s = src + sb * src_bs;
  const long long total = (long long)rows * cols;
  float m = 0.f;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / cols);
    const int c = (int)(e - (long long)r * cols);
    const float x = (a != 0.f) ? a * s[(long long)r * src_ld + c] : 0.f;
    m = fmaxf(m, fabsf(x + (r == c ? d : 0.f)));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = m;
  __syncthreads();
  if (w == 0) {
    m = l < (int)(blockDim.x >> 5) ? red[l] : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // non-negative floats order like their bit patterns
    if (l == 0) atomicMax(reinterpret_cast<unsigned int*>(amax) + b, __float_as_uint(m));
  }
}

__global__ void to_planes_kernel(const float* __restrict__ src, int src_ld, long long src_bs,
                                 const int* __restrict__ src_idx, int rows, int cols, float alpha, float eps,
                                 float delta, const float* __restrict__ scale, Planes dst, int prec) {
  const int b = blockIdx.y;
  const long long sb = src_idx ? src_idx[b] : b;
  const float inv_s = scale ? 1.f / scale[b] : 1.f;
  const float a = alpha * inv_s;
  const float d = eps * inv_s + delta;
  const float* s = src + sb * src_bs;
  const long long dbase = (long long)b * dst.bs;
  float sc = 1.f;
  if (prec == P_FP32) {
    const int ex = split_exp(dst.amax[b]);
    sc = pow2f(ex);
    if (blockIdx.x == 0 && threadIdx.x == 0) dst.exp[b] = ex;
  }
  const int per_row = cols;
  const long long total = (long long)rows * per_row;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / per_row);
    const int c = (int)(e - (long long)r * per_row);
    const float x = (a != 0.f) ? a * s[(long long)r * src_ld + c] : 0.f;  // a == 0: identity only
    const float v = x + (r == c ? d : 0.f);
    put(dst, dbase + (long long)r * dst.ld + c, v, prec, sc);
  }
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < (blockDim.x >> 5)) t = red[threadIdx.x];
  if (w == 0) {
#pragma unroll
    for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;  // valid in thread 0
}

__global__ void frob_kernel(const float* __restrict__ L, int n, int ld, long long bs, float eps,
                            double* __restrict__ sums) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const float* A = L + (long long)b * bs;
  const long long total = (long long)n * n;
  float acc = 0.f;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / n);
    const int c = (int)(e - (long long)r * n);
    const float v = A[(long long)r * ld + c] + (r == c ? eps : 0.f);
    acc = fmaf(v, v, acc);
  }
  const float t = block_sum(acc, red);
  if (threadIdx.x == 0) atomicAdd(sums + b, (double)t);
}

__global__ void sqrt_scale_kernel(const double* sums, const float* factor, float* scale, int count) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < count) scale[b] = (float)sqrt(sums[b]) * (factor ? factor[b] : 1.f);
}

// V^T rows = normalised start vectors, replicated for every matrix.
__global__ void pi_start_kernel(const float* __restrict__ starts, int v, int n, __half* vt, int ld, long long bs) {
  __shared__ float red[32];
  const int j = blockIdx.x;  // vector
  const int b = blockIdx.y;  // matrix
  float acc = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float x = starts[(long long)j * n + i];
    acc = fmaf(x, x, acc);
  }
  __shared__ float inv;
  const float t = block_sum(acc, red);
  if (threadIdx.x == 0) inv = t > 0.f ? rsqrtf(t) : 0.f;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    vt[(long long)b * bs + (long long)j * ld + i] = __float2half_rn(starts[(long long)j * n + i] * inv);
}

// W (n x v, per matrix) -> V^T rows normalised to unit length (fp16).
__global__ void pi_normalize_kernel(const float* __restrict__ W, int n, int v, int w_ld, long long w_bs,
                                    __half* vt, int vt_ld, long long vt_bs) {
  __shared__ float red[32];
  __shared__ float inv;
  const int j = blockIdx.x;
  const int b = blockIdx.y;
  const float* w = W + (long long)b * w_bs;
  float acc = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float x = w[(long long)i * w_ld + j];
    acc = fmaf(x, x, acc);
  }
  const float t = block_sum(acc, red);
  if (threadIdx.x == 0) inv = t > 0.f ? rsqrtf(t) : 0.f;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    vt[(long long)b * vt_bs + (long long)j * vt_ld + i] = __float2half_rn(w[(long long)i * w_ld + j] * inv);
}

// scale[b] = f_b * max_j v_j^T (A/f) v_j with W = (A/f) V already formed.
__global__ void pi_rayleigh_kernel(const float* __restrict__ W, const __half* __restrict__ vt, int n, int v,
                                   int w_ld, long long w_bs, int vt_ld, long long vt_bs,
                                   const double* __restrict__ frob_sums, float* scale) {
  __shared__ float red[32];
  __shared__ float best;
  const int b = blockIdx.x;
  const float* w = W + (long long)b * w_bs;
  const __half* q = vt + (long long)b * vt_bs;
  if (threadIdx.x == 0) best = -INFINITY;
  __syncthreads();
  for (int j = 0; j < v; ++j) {
    float acc = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      acc = fmaf(__half2float(q[(long long)j * vt_ld + i]), w[(long long)i * w_ld + j], acc);
    const float t = block_sum(acc, red);
    if (threadIdx.x == 0) best = fmaxf(best, t);
    __syncthreads();
  }
  if (threadIdx.x == 0) scale[b] = best * (float)sqrt(frob_sums[b]);
}

int grid_for(long long work, int per_block_items) {
  long long g = (work + per_block_items - 1) / per_block_items;
  if (g < 1) g = 1;
  if (g > 1184) g = 1184;  // 8 x 148 SMs
  return (int)g;
}

}  // namespace

cudaError_t launch_to_planes(const float* src, int src_ld, long long src_bs, const int* src_idx, int count,
                             int rows, int cols, float alpha, float eps, float delta, const float* scale,
                             const Planes& dst, Prec prec, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  const long long per = (long long)rows * cols;
  int gx = grid_for(per, kThreads * 8);
  dim3 grid(gx, count);
  if (prec == P_FP32) {
    cudaError_t e = cudaMemsetAsync(dst.amax, 0, sizeof(float) * count, stream);
    if (e != cudaSuccess) return e;
    amax_affine_kernel<<<grid, kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps, delta,
                                                      scale, dst.amax);
    count_launch();
  }
  to_planes_kernel<<<grid, kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps, delta,
                                                  scale, dst, (int)prec);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_frob_sumsq(const float* L, int n, int ld, long long bs, int count, float eps, double* sums,
                              cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(sums, 0, sizeof(double) * count, stream);
  if (e != cudaSuccess) return e;
  int gx = grid_for((long long)n * n, kThreads * 16);
  frob_kernel<<<dim3(gx, count), kThreads, 0, stream>>>(L, n, ld, bs, eps, sums);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_sqrt_scale(const double* sums, const float* factor, float* scale, int count,
                              cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  sqrt_scale_kernel<<<(count + 255) / 256, 256, 0, stream>>>(sums, factor, scale, count);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pi_start_batched(const float* starts, int v, int n, void* vt_h16, int ld, long long bs,
                                    int count, cudaStream_t stream) {
  pi_start_kernel<<<dim3(v, count), kThreads, 0, stream>>>(starts, v, n, reinterpret_cast<__half*>(vt_h16), ld,
                                                           bs);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pi_normalize(const float* W, int n, int v, int w_ld, long long w_bs, int count, void* vt_h16,
                                int vt_ld, long long vt_bs, cudaStream_t stream) {
  pi_normalize_kernel<<<dim3(v, count), kThreads, 0, stream>>>(W, n, v, w_ld, w_bs,
                                                               reinterpret_cast<__half*>(vt_h16), vt_ld, vt_bs);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_pi_rayleigh(const float* W, const void* vt_h16, int n, int v, int w_ld, long long w_bs,
                               int vt_ld, long long vt_bs, int count, const double* frob_sums, float* scale,
                               cudaStream_t stream) {
  pi_rayleigh_kernel<<<count, kThreads, 0, stream>>>(W, reinterpret_cast<const __half*>(vt_h16), n, v, w_ld, w_bs,
                                                     vt_ld, vt_bs, frob_sums, scale);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_zero_i32(int* p, size_t n, cudaStream_t stream) {
  return n ? cudaMemsetAsync(p, 0, n * sizeof(int), stream) : cudaSuccess;
}

}  // namespace shp
