// Streaming kernels of the step outside the contractions: gathering gradient
// blocks into their stacks ("DASH: Faster Shampoo via Batched Block
// Preconditioning and Efficient Inverse-Root Solvers", §4 Blocking Strategy),
// the grafted parameter update (§2; "3D-Shampoo optimizer" README,
// graft_type / weight_decay) and the scaled copy that finishes a root when
// the iteration count leaves no GEMM to fuse it into.
#include "internal.h"
#include "ptx.cuh"
#include "step.h"

namespace shp {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ const int* blk(const int* table, int b) { return table + b * kBlockFields; }

// One CTA row (blockIdx.y) per block, grid-stride over its elements.
__global__ void gather_kernel(const int* __restrict__ blocks, int block0, LayerArgs la, BucketArgs ba) {
  const int bid = block0 + blockIdx.y;
  const int* t = blk(blocks, bid);
  const int li = t[0] - la.layer0, r0 = t[3], c0 = t[4], rows = t[5], cols = t[6], gb = t[7], gi = t[8];
  const float* src = la.G[li];
  const int lc = la.cols[li];
  float* dst = ba.ptr[gb] + (long long)gi * rows * cols;
  const long long total = (long long)rows * cols;
  const bool vec = ((cols & 3) == 0) && ((c0 & 3) == 0) && ((lc & 3) == 0);
  if (vec) {
    const int c4 = cols >> 2;
    const long long tot4 = (long long)rows * c4;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < tot4;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / c4), c = (int)(e - (long long)r * c4) * 4;
      const float4 x = *reinterpret_cast<const float4*>(src + (long long)(r0 + r) * lc + c0 + c);
      *reinterpret_cast<float4*>(dst + (long long)r * cols + c) = x;
    }
  } else {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / cols), c = (int)(e - (long long)r * cols);
      dst[(long long)r * cols + c] = src[(long long)(r0 + r) * lc + c0 + c];
    }
  }
}

__device__ __forceinline__ float graft_value(int kind, float g, float* m, float* v, const GraftScalars& s) {
  if (kind == GRAFT_SGD) return g;
  if (kind == GRAFT_ADAGRAD) {
    const float vv = *v + g * g;
    *v = vv;
    return g / (sqrtf(vv) + s.eps);
  }
  // Adam
  const float mm = s.beta1 * *m + (1.f - s.beta1) * g;
  const float vv = s.beta2 * *v + (1.f - s.beta2) * g * g;
  *m = mm;
  *v = vv;
  return (mm / s.bc1) / (sqrtf(vv / s.bc2) + s.eps);
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
  return t;
}

// Pass 1: moments update and sum of squares of the graft direction per block.
__global__ void graft_pass1_kernel(const int* __restrict__ blocks, int block0, LayerArgs la, GraftScalars s,
                                   double* __restrict__ gsum) {
  __shared__ float red[32];
  const int bid = block0 + blockIdx.y;
  const int* t = blk(blocks, bid);
  const int li = t[0] - la.layer0, r0 = t[3], c0 = t[4], rows = t[5], cols = t[6];
  const int lc = la.cols[li];
  const float* G = la.G[li];
  float* M = la.m[li];
  float* V = la.v[li];
  const long long total = (long long)rows * cols;
  float acc = 0.f;
  if (((cols | c0 | lc) & 3) == 0) {
    // float4 quads of a row; 32-bit indices (a block holds < 2^31 elements)
    const int q = cols >> 2, tq = rows * q;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < tq; e += gridDim.x * blockDim.x) {
      const int r = e / q, c = (e - r * q) * 4;
      const long long off = (long long)(r0 + r) * lc + c0 + c;
      const float4 g4 = *reinterpret_cast<const float4*>(G + off);
      float4 m4 = M ? *reinterpret_cast<const float4*>(M + off) : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 v4 = V ? *reinterpret_cast<const float4*>(V + off) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float a = graft_value(s.kind, g4.x, &m4.x, &v4.x, s);
      const float b = graft_value(s.kind, g4.y, &m4.y, &v4.y, s);
      const float c2 = graft_value(s.kind, g4.z, &m4.z, &v4.z, s);
      const float d = graft_value(s.kind, g4.w, &m4.w, &v4.w, s);
      if (M && s.kind == GRAFT_ADAM) *reinterpret_cast<float4*>(M + off) = m4;
      if (V && s.kind != GRAFT_SGD) *reinterpret_cast<float4*>(V + off) = v4;
      acc = fmaf(a, a, acc);
      acc = fmaf(b, b, acc);
      acc = fmaf(c2, c2, acc);
      acc = fmaf(d, d, acc);
    }
  } else {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / cols), c = (int)(e - (long long)r * cols);
      const long long off = (long long)(r0 + r) * lc + c0 + c;
      float dm = 0.f, dv = 0.f;
      float* pm = M ? M + off : &dm;
      float* pv = V ? V + off : &dv;
      const float g = graft_value(s.kind, G[off], pm, pv, s);
      acc = fmaf(g, g, acc);
    }
  }
  const float tot = block_sum(acc, red);
  if (threadIdx.x == 0) atomicAdd(gsum + bid, (double)tot);
}

// Pass 2: rho per layer / block, then W <- W - lr rho D - lr wd W.
__global__ void graft_pass2_kernel(const int* __restrict__ blocks, const int* __restrict__ layer_first,
                                   const int* __restrict__ gstack_off, int block0, LayerArgs la, BucketArgs dptr,
                                   GraftScalars s, const double* __restrict__ gsum,
                                   const float* __restrict__ dnorm2) {
  __shared__ float rho_s;
  const int bid = block0 + blockIdx.y;
  const int* t = blk(blocks, bid);
  const int layer = t[0];
  const int li = layer - la.layer0, r0 = t[3], c0 = t[4], rows = t[5], cols = t[6], gb = t[7], gi = t[8];
  if (threadIdx.x == 0) {
    float rho = 1.f;
    if (s.kind != GRAFT_NONE) {
      double gn = 0.0, dn = 0.0;
      int lo = bid, hi = bid + 1;
      if (!s.per_block) {
        lo = layer_first[layer];
        hi = layer_first[layer + 1];
      }
      for (int q = lo; q < hi; ++q) {
        const int* u = blk(blocks, q);
        gn += gsum[q];
        dn += (double)dnorm2[gstack_off[u[7]] + u[8]];
      }
      rho = dn > 0.0 ? (float)sqrt(gn / dn) : 0.f;
    }
    rho_s = rho;
  }
  __syncthreads();
  const float step = s.lr * rho_s;
  const float keep = 1.f - s.lr * s.wd;
  const int lc = la.cols[li];
  float* W = la.W[li];
  const float* D = dptr.ptr[gb] + (long long)gi * rows * cols;
  const long long total = (long long)rows * cols;
  if (((cols | c0 | lc) & 3) == 0) {
    const int q = cols >> 2, tq = rows * q;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < tq; e += gridDim.x * blockDim.x) {
      const int r = e / q, c = (e - r * q) * 4;
      const long long off = (long long)(r0 + r) * lc + c0 + c;
      float4 w = *reinterpret_cast<const float4*>(W + off);
      const float4 d = *reinterpret_cast<const float4*>(D + (long long)r * cols + c);
      w.x = keep * w.x - step * d.x;
      w.y = keep * w.y - step * d.y;
      w.z = keep * w.z - step * d.z;
      w.w = keep * w.w - step * d.w;
      *reinterpret_cast<float4*>(W + off) = w;
    }
  } else {
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
      const int r = (int)(e / cols), c = (int)(e - (long long)r * cols);
      const long long off = (long long)(r0 + r) * lc + c0 + c;
      W[off] = keep * W[off] - step * D[(long long)r * cols + c];
    }
  }
}

__global__ void scaled_copy_kernel(Planes P, int n, const float* __restrict__ scale, int p, float* __restrict__ out,
                                   int* __restrict__ status) {
  const int b = blockIdx.y;
  const float mult = inv_root_mult(scale[b], p);
  const long long total = (long long)n * n;
  int bad = 0;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / n), c = (int)(e - (long long)r * n);
    const long long off = (long long)b * P.bs + (long long)r * P.ld + c;
    const float x = P.f32[off] * mult;
    out[(long long)b * n * n + e] = x;
    bad |= !isfinite(x);
  }
  if (bad && status) atomicOr(status + b, 1);
}

int grid_x(long long work) {
  long long g = (work + kThreads * 8 - 1) / (kThreads * 8);
  if (g < 1) g = 1;
  if (g > 512) g = 512;
  return (int)g;
}

}  // namespace

cudaError_t launch_gather(const int* blocks, int block0, int nblk, long long max_elems, const LayerArgs& la,
                          const BucketArgs& ba, cudaStream_t stream) {
  if (nblk <= 0) return cudaSuccess;
  gather_kernel<<<dim3(grid_x(max_elems), nblk), kThreads, 0, stream>>>(blocks, block0, la, ba);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_graft_pass1(const int* blocks, int block0, int nblk, long long max_elems, const LayerArgs& la,
                               const GraftScalars& s, double* gsum, cudaStream_t stream) {
  if (nblk <= 0) return cudaSuccess;
  graft_pass1_kernel<<<dim3(grid_x(max_elems), nblk), kThreads, 0, stream>>>(blocks, block0, la, s, gsum);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_graft_pass2(const int* blocks, const int* layer_first, const int* gstack_off, int block0, int nblk,
                               long long max_elems, const LayerArgs& la, const BucketArgs& d, const GraftScalars& s,
                               const double* gsum, const float* dnorm2, cudaStream_t stream) {
  if (nblk <= 0) return cudaSuccess;
  graft_pass2_kernel<<<dim3(grid_x(max_elems), nblk), kThreads, 0, stream>>>(blocks, layer_first, gstack_off, block0,
                                                                             la, d, s, gsum, dnorm2);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_scaled_copy(const Planes& P, int n, int count, const float* scale, int p, float* out, int* status,
                               cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  scaled_copy_kernel<<<dim3(grid_x((long long)n * n), count), kThreads, 0, stream>>>(P, n, scale, p, out, status);
  count_launch();
  return cudaGetLastError();
}

}  // namespace shp
