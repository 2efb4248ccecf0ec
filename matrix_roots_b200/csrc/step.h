// Launch interfaces of the streaming step kernels (step_kernels.cu).
#pragma once
#include "internal.h"

namespace shp {

constexpr int kBlockFields = 13;
constexpr int kMaxLayersPerLaunch = 192;
constexpr int kMaxBuckets = 64;

enum GraftKind : int { GRAFT_NONE = 0, GRAFT_SGD = 1, GRAFT_ADAGRAD = 2, GRAFT_ADAM = 3 };

// Per-layer pointers of one launch, covering layers [layer0, layer0 + n).
struct LayerArgs {
  float* W[kMaxLayersPerLaunch];
  const float* G[kMaxLayersPerLaunch];
  float* m[kMaxLayersPerLaunch];
  float* v[kMaxLayersPerLaunch];
  int cols[kMaxLayersPerLaunch];
  int layer0;
};

struct BucketArgs {
  float* ptr[kMaxBuckets];
};

struct GraftScalars {
  int kind;
  int per_block;
  float beta1, beta2, eps, bc1, bc2, lr, wd;
};

cudaError_t launch_gather(const int* blocks, int block0, int nblk, long long max_elems, const LayerArgs& la,
                          const BucketArgs& ba, cudaStream_t stream);
cudaError_t launch_graft_pass1(const int* blocks, int block0, int nblk, long long max_elems, const LayerArgs& la,
                               const GraftScalars& s, double* gsum, cudaStream_t stream);
cudaError_t launch_graft_pass2(const int* blocks, const int* layer_first, const int* gstack_off, int block0, int nblk,
                               long long max_elems, const LayerArgs& la, const BucketArgs& d, const GraftScalars& s,
                               const double* gsum, const float* dnorm2, cudaStream_t stream);
// out = P * scale^(-1/p) (the root multiplier), status |= 1 where not finite.
cudaError_t launch_scaled_copy(const Planes& P, int n, int count, const float* scale, int p, float* out, int* status,
                               cudaStream_t stream);

}  // namespace shp
