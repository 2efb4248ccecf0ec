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

// Affine map of one source matrix: dst = a * src + d * I.
struct Affine {
  const float* s;  // source matrix b
  float a, d;
};

__device__ __forceinline__ Affine affine_of(const float* src, long long src_bs, const int* src_idx, int b,
                                            float alpha, float eps, float delta, const float* scale) {
  Affine f;
  const long long sb = src_idx ? src_idx[b] : b;
  const float inv_s = scale ? 1.f / scale[b] : 1.f;
  f.a = alpha * inv_s;
  f.d = eps * inv_s + delta;
  f.s = src + sb * src_bs;
  return f;
}

// 4 consecutive values of row r starting at column c (c % 4 == 0).
__device__ __forceinline__ float4 affine4(const Affine& f, int src_ld, int r, int c) {
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  if (f.a != 0.f) {  // a == 0: identity only
    x = *reinterpret_cast<const float4*>(f.s + (long long)r * src_ld + c);
    x.x *= f.a;
    x.y *= f.a;
    x.z *= f.a;
    x.w *= f.a;
  }
  const int k = r - c;
  if (k == 0) x.x += f.d;
  if (k == 1) x.y += f.d;
  if (k == 2) x.z += f.d;
  if (k == 3) x.w += f.d;
  return x;
}

__device__ __forceinline__ float block_max_to(float m, float* red, float* out) {
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
    if (l == 0) atomicMax(reinterpret_cast<unsigned int*>(out), __float_as_uint(m));
  }
  return m;
}

// amax[b] = max |(alpha/s_b) src_b + (eps/s_b + delta) I| (amax cleared
// before).  VEC: rows go as float4 quads (cols, ld and bases multiples of 4).
template <bool VEC>
__global__ void amax_affine_kernel(const float* __restrict__ src, int src_ld, long long src_bs,
                                   const int* __restrict__ src_idx, int rows, int cols, float alpha, float eps,
                                   float delta, const float* __restrict__ scale, float* __restrict__ amax) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const Affine f = affine_of(src, src_bs, src_idx, b, alpha, eps, delta, scale);
  float m = 0.f;
  if (VEC) {
    // four independent quads in flight per thread
    const int q = cols >> 2;
    const int total = rows * q;
    const int stride = gridDim.x * blockDim.x;
    for (int e0 = blockIdx.x * blockDim.x + threadIdx.x; e0 < total; e0 += 4 * stride) {
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = e0 + u * stride;
        x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < total) {
          const int r = e / q, c = (e - r * q) * 4;
          x[u] = affine4(f, src_ld, r, c);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(x[u].x), fabsf(x[u].y)), fmaxf(fabsf(x[u].z), fabsf(x[u].w))));
    }
  } else {
    const long long total = (long long)rows * cols;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / cols);
      const int c = (int)(e - (long long)r * cols);
      const float x = (f.a != 0.f) ? f.a * f.s[(long long)r * src_ld + c] : 0.f;
      m = fmaxf(m, fabsf(x + (r == c ? f.d : 0.f)));
    }
  }
  block_max_to(m, red, amax + b);
}

__device__ __forceinline__ uint2 half4(__half a, __half b, __half c, __half d) {
  __half2 p = __halves2half2(a, b), q = __halves2half2(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&p);
  u.y = *reinterpret_cast<uint32_t*>(&q);
  return u;
}

__device__ __forceinline__ void put4(const Planes& d, long long off, float4 v, int prec, float sc) {
  if (d.f32) *reinterpret_cast<float4*>(d.f32 + off) = v;
  if (prec == P_FP32) {
    __half2 h01, h23, l01, l23;
    split16x2(v.x * sc, v.y * sc, h01, l01);
    split16x2(v.z * sc, v.w * sc, h23, l23);
    *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(d.h16) + off) = make_uint2(h2bits(h01), h2bits(h23));
    *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(d.h16lo) + off) = make_uint2(h2bits(l01), h2bits(l23));
  } else if (prec == P_FP16 || prec == P_BF16) {
    if (d.h16_bf) {
      __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), c = __floats2bfloat162_rn(v.z, v.w);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&a);
      u.y = *reinterpret_cast<uint32_t*>(&c);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(d.h16) + off) = u;
    } else {
      *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(d.h16) + off) =
          half4(__float2half_rn(v.x), __float2half_rn(v.y), __float2half_rn(v.z), __float2half_rn(v.w));
    }
  }
}

// dst = (alpha/s_b) src_b + (eps/s_b + delta) I in the planes of `dst`.  For
// FP32 planes the exponent comes from dst.amax[b] (filled by the amax pass),
// or, when src_amax is given, from the bound |a| max|src| + |d|, which is
// then stored as dst.amax[b].
template <bool VEC>
__global__ void to_planes_kernel(const float* __restrict__ src, int src_ld, long long src_bs,
                                 const int* __restrict__ src_idx, int rows, int cols, float alpha, float eps,
                                 float delta, const float* __restrict__ scale, const float* __restrict__ src_amax,
                                 Planes dst, int prec) {
  const int b = blockIdx.y;
  const Affine f = affine_of(src, src_bs, src_idx, b, alpha, eps, delta, scale);
  const long long dbase = (long long)b * dst.bs;
  float sc = 1.f;
  if (prec == P_FP32) {
    float bound;
    if (src_amax) {
      bound = fabsf(f.a) * src_amax[src_idx ? src_idx[b] : b] + fabsf(f.d);
      if (blockIdx.x == 0 && threadIdx.x == 0) dst.amax[b] = bound;
    } else {
      bound = dst.amax[b];
    }
    const int ex = split_exp(bound);
    sc = pow2f(ex);
    if (blockIdx.x == 0 && threadIdx.x == 0) dst.exp[b] = ex;
  }
  if (VEC) {
    const int q = cols >> 2;
    const int total = rows * q;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
      const int r = e / q, c = (e - r * q) * 4;
      put4(dst, dbase + (long long)r * dst.ld + c, affine4(f, src_ld, r, c), prec, sc);
    }
  } else {
    const long long total = (long long)rows * cols;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / cols);
      const int c = (int)(e - (long long)r * cols);
      const float x = (f.a != 0.f) ? f.a * f.s[(long long)r * src_ld + c] : 0.f;  // a == 0: identity only
      put(dst, dbase + (long long)r * dst.ld + c, x + (r == c ? f.d : 0.f), prec, sc);
    }
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

// sums[b] += sum (L + eps I)^2 and, when amax is given, amax[b] = max |L|
// (both cleared before).  n, ld and bs are multiples of 4: rows go as float4.
__global__ void frob_kernel(const float* __restrict__ L, int n, int ld, long long bs, float eps,
                            double* __restrict__ sums, float* __restrict__ amax) {
  __shared__ float red[32];
  __shared__ float red2[32];
  const int b = blockIdx.y;
  const float* A = L + (long long)b * bs;
  const int q = n >> 2;
  const int total = n * q;
  float acc = 0.f, m = 0.f;
  const int stride = gridDim.x * blockDim.x;
  // four independent quads in flight per thread
  for (int e0 = blockIdx.x * blockDim.x + threadIdx.x; e0 < total; e0 += 4 * stride) {
    float4 xs[4];
    int ks[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * stride;
      xs[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      ks[u] = -1;
      if (e < total) {
        const int r = e / q, c = (e - r * q) * 4;
        xs[u] = *reinterpret_cast<const float4*>(A + (long long)r * ld + c);
        ks[u] = r - c;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float4 x = xs[u];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
      const int k = ks[u];
      if (k == 0) x.x += eps;
      if (k == 1) x.y += eps;
      if (k == 2) x.z += eps;
      if (k == 3) x.w += eps;
      acc = fmaf(x.x, x.x, acc);
      acc = fmaf(x.y, x.y, acc);
      acc = fmaf(x.z, x.z, acc);
      acc = fmaf(x.w, x.w, acc);
    }
  }
  const float t = block_sum(acc, red);
  if (threadIdx.x == 0) atomicAdd(sums + b, (double)t);
  if (amax) block_max_to(m, red2, amax + b);
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
                             const Planes& dst, Prec prec, cudaStream_t stream, const float* src_amax) {
  if (count <= 0) return cudaSuccess;
  auto al16 = [](const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const bool vec = cols % 4 == 0 && src_ld % 4 == 0 && src_bs % 4 == 0 && dst.ld % 4 == 0 && dst.bs % 4 == 0 &&
                   al16(src) && al16(dst.f32) && (long long)rows * cols < (1ll << 31);
  const long long per = (long long)rows * cols;
  const int gx = grid_for(vec ? per / 4 : per, kThreads * 2);
  const dim3 grid(gx, count);
  if (prec == P_FP32 && !src_amax) {
    cudaError_t e = cudaMemsetAsync(dst.amax, 0, sizeof(float) * count, stream);
    if (e != cudaSuccess) return e;
    if (vec)
      amax_affine_kernel<true><<<dim3(grid_for(per / 4, kThreads * 4), count), kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps,
                                                               delta, scale, dst.amax);
    else
      amax_affine_kernel<false><<<grid, kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps,
                                                                delta, scale, dst.amax);
    count_launch();
  }
  if (vec)
    to_planes_kernel<true><<<grid, kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps,
                                                           delta, scale, src_amax, dst, (int)prec);
  else
    to_planes_kernel<false><<<grid, kThreads, 0, stream>>>(src, src_ld, src_bs, src_idx, rows, cols, alpha, eps,
                                                            delta, scale, src_amax, dst, (int)prec);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_frob_sumsq(const float* L, int n, int ld, long long bs, int count, float eps, double* sums,
                              cudaStream_t stream, float* amax) {
  if (count <= 0) return cudaSuccess;
  if (n % 4 || ld % 4 || bs % 4 || (reinterpret_cast<uintptr_t>(L) & 15u)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(sums, 0, sizeof(double) * count, stream);
  if (e != cudaSuccess) return e;
  if (amax) {
    e = cudaMemsetAsync(amax, 0, sizeof(float) * count, stream);
    if (e != cudaSuccess) return e;
  }
  const int gx = grid_for((long long)n * n / 4, kThreads * 4);
  frob_kernel<<<dim3(gx, count), kThreads, 0, stream>>>(L, n, ld, bs, eps, sums, amax);
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
