// Batched tcgen05 GEMM with fused epilogues, the contraction engine behind
// the statistics update, every inverse-root iteration and the two-sided
// preconditioning ("DASH: Faster Shampoo via Batched Block Preconditioning
// and Efficient Inverse-Root Solvers", §4: same-shape blocks stacked into 3D
// tensors and processed by batched matmuls).
//
// One persistent CTA per SM walks the 128 x BN output tiles of every matrix
// of the stack (and of up to two problems per launch):
//   warp 9       TMA producer: 128B-swizzled operand tiles into a STAGES-deep
//                shared-memory ring (mbarrier complete_tx)
//   warp 8       TMEM allocator + single-thread tcgen05.mma issuer; one
//                tcgen05.commit per K-block onto a ring of completion barriers
//                that the producer and the draining warps both wait on
//   warps 0-7    draining warps (warp w reads TMEM lanes 32*(w%4).., group
//                h = w/4 owns columns [h*BN/2, (h+1)*BN/2) of the tile)
//   warps 10-13  epilogue warps (one per TMEM lane quadrant)
// The tensor core's FP32 accumulation error grows with the number of
// products chained into one accumulator, so partial products go into a ring
// of three TMEM slots that the draining warps add into fp32 registers (round
// to nearest) and release; at the end of a tile they store the sums into a
// fourth block of TMEM, the handoff, and move on while the epilogue warps
// read it.  FP32 mode runs three fp16 passes on a scaled hi / lo split of
// each operand (x * 2^e = hi + lo * 2^-11, e per matrix): per 32 K it issues
// the correction products lo*hi and hi*lo into a fresh slot, then hi*hi with
// the input-D scale 2^-11 on the first, so the corrections enter at their
// true weight.  Every output plane set in that mode gets its exponent from a
// bound on its values and records its max |value| for the next product.  The
// epilogue transposes 32x32 blocks through shared memory so that reads of C
// and writes of the output planes are 128-byte (or 16-byte-per-lane)
// coalesced.
#include <atomic>
#include <cstdio>
#include <mutex>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace shp {
__device__ int shp_dev_error = 0;
}  // namespace shp

#define SHP_DEV_ERROR_DEFINED
#include "ptx.cuh"

namespace shp {

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
unsigned long long launch_total() { return g_launches.load(std::memory_order_relaxed); }

cudaError_t read_and_clear_dev_error(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, shp_dev_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(shp_dev_error, &zero, sizeof(int));
}

namespace {

// MMA kind: 0 = tf32, 1 = f16, 2 = bf16 (all with FP32 accumulation).
template <int KIND>
struct KindTraits;
template <>
struct KindTraits<0> {
  static constexpr int ESZ = 4;
  static constexpr uint32_t FMT = 2;
  static constexpr int KINST = 8;
  // MN-major tf32 tiles: 128B swizzle with 32-byte atoms (UMMA layout 1,
  // 4-row atoms of 512 B), the only MN-major layout the tensor core accepts
  // for 32-bit operands
  static constexpr uint32_t MN_LAYOUT = 1, MN_SBO = 512;
};
template <>
struct KindTraits<1> {
  static constexpr int ESZ = 2;
  static constexpr uint32_t FMT = 0;
  static constexpr int KINST = 16;
  static constexpr uint32_t MN_LAYOUT = 2, MN_SBO = 1024;
};
template <>
struct KindTraits<2> {
  static constexpr int ESZ = 2;
  static constexpr uint32_t FMT = 1;
  static constexpr int KINST = 16;
  static constexpr uint32_t MN_LAYOUT = 2, MN_SBO = 1024;
};

template <int KIND, int NPASS, int BN>
struct Cfg {
  static constexpr int ESZ = KindTraits<KIND>::ESZ;
  static constexpr int BKE = 128 / ESZ;  // K elements per K-block (one 128-byte swizzle row)
  static constexpr int NPL = (NPASS == 3) ? 2 : 1;
  static constexpr int A_TILE = 128 * 128;
  static constexpr int B_TILE = BN * 128;
  static constexpr int STAGE_BYTES = NPL * (A_TILE + B_TILE);
  static constexpr int NBUF = 3;  // accumulation slots; a fourth block of BN columns is the epilogue handoff
  // K-blocks accumulated in one TMEM slot before it is drained in the
  // one-pass modes, whose operand rounding (2^-11) dwarfs the accumulation
  // error; FP32 mode instead drains every half K-block (32 K), for accuracy
  static constexpr int DRAIN = (NPASS == 3) ? 1 : 4;
  static constexpr int TCOLS = 4 * BN;
  static constexpr int THREADS = 448;
  static constexpr int STAGE_OUT = 4 * 32 * 32 * 4;  // 32x32 transpose buffer per epilogue warp
  static constexpr int RESERVED = 1024 + 512 + STAGE_OUT;
  static constexpr int STAGES_RAW = (227 * 1024 - RESERVED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + RESERVED;
  static_assert(STAGES >= 2 && TCOLS <= 512 && BN <= 128, "tile does not fit");
};

struct Tile {
  int grp, b, m0, n0, nk;
};

__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int t, int BN, int BKE) {
  Tile x;
  x.grp = t >= p.tiles0 ? 1 : 0;
  int r = x.grp ? t - p.tiles0 : t;
  x.nk = (p.g[x.grp].K + BKE - 1) / BKE;
  if (p.g[x.grp].sym) {  // upper triangle of square tiles, row by row
    const int mt = p.mt[x.grp];
    const int per = mt * (mt + 1) / 2;
    x.b = r / per;
    r -= x.b * per;
    int mi = 0;
    while (r >= mt - mi) {
      r -= mt - mi;
      ++mi;
    }
    x.m0 = mi * 128;
    x.n0 = (mi + r) * 128;
    return x;
  }
  const int per = p.mt[x.grp] * p.nt[x.grp];
  x.b = r / per;
  r -= x.b * per;
  const int mi = r / p.nt[x.grp];
  x.m0 = mi * 128;
  x.n0 = (r - mi * p.nt[x.grp]) * BN;
  return x;
}

// One output plane set with its pointers already offset to (row0, col).
struct OutPtrs {
  float* f32;
  void* h16;
  __half* h16lo;  // non-null: h16 / h16lo hold the scaled fp16 hi / lo split
  int bf;
  int ld;
  float sc;  // 2^exp of the split
};

__device__ __forceinline__ OutPtrs out_ptrs(const EpiOut& o, int ob, int row0, int col, float sc) {
  OutPtrs r;
  const long long off = (long long)ob * o.bs + (long long)row0 * o.ld + col;
  r.f32 = o.f32 ? o.f32 + off : nullptr;
  r.h16 = o.h16 ? (o.h16_bf ? (void*)(reinterpret_cast<__nv_bfloat16*>(o.h16) + off)
                            : (void*)(reinterpret_cast<__half*>(o.h16) + off))
                : nullptr;
  r.h16lo = o.h16lo ? reinterpret_cast<__half*>(o.h16lo) + off : nullptr;
  r.bf = o.h16_bf;
  r.ld = o.ld;
  r.sc = sc;
  return r;
}

// Per-tile epilogue constants of one problem and matrix.
struct EpiCtx {
  int ob;
  float mult, alpha, beta, gamma, alpha2, beta2, gamma2;
  bool has_x, need_c;
  float scO, scX;
};

// r0 = alpha*AB + beta*C + gamma*I with the operand scales undone; the
// scale exponent of a split output comes from the bound
//   |r0| <= |alpha| K max|A| max|B| + |beta| max|C| + |gamma|
// (and the same for the aux output), and is stored for the next GEMM.
__device__ __forceinline__ EpiCtx make_ctx(const GroupDev& g, int b, bool write_exp) {
  EpiCtx c;
  c.ob = g.o_idx ? g.o_idx[b] : b;
  c.mult = g.bscale ? inv_root_mult(g.bscale[b], g.root_p) : 1.f;
  c.has_x = (g.X.f32 != nullptr) || (g.X.h16 != nullptr);
  c.need_c = (g.beta != 0.f) || (c.has_x && g.beta2 != 0.f);
  c.alpha = g.alpha;
  c.beta = g.beta;
  c.gamma = g.gamma;
  c.alpha2 = g.alpha2;
  c.beta2 = g.beta2;
  c.gamma2 = g.gamma2;
  c.scO = 1.f;
  c.scX = 1.f;
  if (g.a_exp) {
    const int ai = g.a_idx ? g.a_idx[b] : b;
    const int bi = g.b_idx ? g.b_idx[b] : b;
    c.alpha = g.alpha * pow2f(-g.a_exp[ai]) * pow2f(-g.b_exp[bi]);
    const float cmax = (c.need_c && g.C.amax) ? g.C.amax[c.ob] : 0.f;
    const float r0 = fabsf(g.alpha) * (float)g.K * g.a_amax[ai] * g.b_amax[bi] + fabsf(g.beta) * cmax + fabsf(g.gamma);
    if (g.O.h16lo) {
      const int e = split_exp(fabsf(c.mult) * r0);
      c.scO = pow2f(e);
      if (write_exp) g.O.exp[c.ob] = e;
    }
    if (c.has_x && g.X.h16lo) {
      const int e = split_exp(fabsf(c.mult) * (fabsf(g.alpha2) * r0 + fabsf(g.beta2) * cmax + fabsf(g.gamma2)));
      c.scX = pow2f(e);
      if (write_exp) g.X.exp[c.ob] = e;
    }
  }
  return c;
}

// Stores rows [r0, r0 + 8) of values v (rows >= rmax skipped) into one
// output plane set; the format tests are uniform and sit outside the rows.
__device__ __forceinline__ void put_rows(const OutPtrs& o, int r0, int rmax, const float (&v)[8]) {
  const long long ld = o.ld;
  if (o.f32) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (r0 + i < rmax) o.f32[(r0 + i) * ld] = v[i];
  }
  if (o.h16lo) {
    __half* h = reinterpret_cast<__half*>(o.h16);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (r0 + i < rmax) {
        __half hi, lo;
        split16(v[i] * o.sc, hi, lo);
        h[(r0 + i) * ld] = hi;
        o.h16lo[(r0 + i) * ld] = lo;
      }
  } else if (o.h16) {
    if (o.bf) {
      __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(o.h16);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (r0 + i < rmax) h[(r0 + i) * ld] = __float2bfloat16_rn(v[i]);
    } else {
      __half* h = reinterpret_cast<__half*>(o.h16);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (r0 + i < rmax) h[(r0 + i) * ld] = __float2half_rn(v[i]);
    }
  }
}

// Epilogue of a 32-row x 32-column block whose accumulators sit transposed
// in `stage` (element (r, c) at r*32 + (c ^ r)): lane = column, so every
// load of C and every store of an output plane is one 128-byte segment.
// Rows go in groups of 8: values first, then the stores of the group.
__device__ __forceinline__ void epilogue_block(const GroupDev& g, const EpiCtx& x, int row0, int col,
                                               const float* stage, int lane, float& ss, int& bad, float& mo,
                                               float& mx) {
  if (col >= g.N) return;
  const OutPtrs O = out_ptrs(g.O, x.ob, row0, col, x.scO);
  const OutPtrs X = x.has_x ? out_ptrs(g.X, x.ob, row0, col, x.scX) : O;
  const float* cf = x.need_c ? g.C.f32 + (long long)x.ob * g.C.bs + (long long)row0 * g.C.ld + col : nullptr;
  const long long cld = g.C.ld;
  const int rmax = g.M - row0 < 32 ? g.M - row0 : 32;
  const int dr = col - row0;  // the diagonal sits in row dr of this block
#pragma unroll 1
  for (int r0 = 0; r0 < rmax; r0 += 8) {
    float cv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) cv[i] = 0.f;
    if (x.need_c) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (r0 + i < rmax) cv[i] = cf[(r0 + i) * cld];
    }
    float v[8], xv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = r0 + i;
      const float diag = (r == dr) ? 1.f : 0.f;
      const float q0 = x.alpha * stage[r * 32 + (lane ^ r)] + x.beta * cv[i] + x.gamma * diag;
      v[i] = q0 * x.mult;
      xv[i] = x.mult * (x.alpha2 * q0 + x.beta2 * cv[i] + x.gamma2 * diag);
      if (r < rmax) {
        ss += v[i] * v[i];
        bad |= !isfinite(v[i]);
        mo = fmaxf(mo, fabsf(v[i]));
        mx = fmaxf(mx, fabsf(xv[i]));
      }
    }
    put_rows(O, r0, rmax, v);
    if (x.has_x) put_rows(X, r0, rmax, xv);
  }
}

// 16-byte version of the epilogue for one 32x32 block: the block sits in
// `stage` as rows of eight float4 slots, slot j of row r at r*8 + (j ^ (r&7));
// each lane handles four consecutive columns of one row, a warp four rows
// per step, so each store is a 128-byte row segment per eight lanes.
__device__ __forceinline__ uint2 pack_half4(__half a, __half b, __half c, __half d) {
  __half2 p = __halves2half2(a, b), q = __halves2half2(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&p);
  u.y = *reinterpret_cast<uint32_t*>(&q);
  return u;
}

__device__ __forceinline__ void put4(const OutPtrs& o, long long off, float4 v) {
  if (o.f32) *reinterpret_cast<float4*>(o.f32 + off) = v;
  if (o.h16lo) {
    __half2 h01, h23, l01, l23;
    split16x2(v.x * o.sc, v.y * o.sc, h01, l01);
    split16x2(v.z * o.sc, v.w * o.sc, h23, l23);
    *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(o.h16) + off) = make_uint2(h2bits(h01), h2bits(h23));
    *reinterpret_cast<uint2*>(o.h16lo + off) = make_uint2(h2bits(l01), h2bits(l23));
  } else if (o.h16) {
    if (o.bf) {
      __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&a);
      u.y = *reinterpret_cast<uint32_t*>(&b);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(o.h16) + off) = u;
    } else {
      *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(o.h16) + off) =
          pack_half4(__float2half_rn(v.x), __float2half_rn(v.y), __float2half_rn(v.z), __float2half_rn(v.w));
    }
  }
}

__device__ __forceinline__ float max4(float4 v) { return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))); }

// TRANS: write the transpose of the staged block at (row0, col0), the
// mirror image of an off-diagonal tile of a symmetric product; output
// element (r, c) is then staged element (c, r).
template <bool NEED_C, bool HAS_X, bool TRANS = false>
__device__ __forceinline__ void epilogue_block4(const GroupDev& g, const EpiCtx& x, int row0, int col0,
                                                const float4* stage, int lane, float& ss, int& bad, float& mo,
                                                float& mx) {
  const int cq = lane & 7;
  const int col = col0 + 4 * cq;
  if (col >= g.N) return;
  const OutPtrs O = out_ptrs(g.O, x.ob, row0, col, x.scO);
  const OutPtrs X = HAS_X ? out_ptrs(g.X, x.ob, row0, col, x.scX) : O;
  const float* cf = NEED_C ? g.C.f32 + (long long)x.ob * g.C.bs + (long long)row0 * g.C.ld + col : nullptr;
  const long long cld = g.C.ld;
  const int rmax = g.M - row0 < 32 ? g.M - row0 : 32;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = it * 4 + (lane >> 3);
    if (r >= rmax) continue;
    float4 a;
    if (TRANS) {
      const float* sf = reinterpret_cast<const float*>(stage);
      float t4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int sr = 4 * cq + i;  // staged row = output column
        t4[i] = sf[(sr * 8 + ((r >> 2) ^ (sr & 7))) * 4 + (r & 3)];
      }
      a = make_float4(t4[0], t4[1], t4[2], t4[3]);
    } else {
      a = stage[r * 8 + (cq ^ (r & 7))];
    }
    float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
    if (NEED_C) c = *reinterpret_cast<const float4*>(cf + r * cld);
    const int e = row0 + r - col;  // component on the diagonal, if 0..3
    const float d0 = e == 0 ? 1.f : 0.f, d1 = e == 1 ? 1.f : 0.f, d2 = e == 2 ? 1.f : 0.f, d3 = e == 3 ? 1.f : 0.f;
    float4 q;
    q.x = x.alpha * a.x + x.gamma * d0;
    q.y = x.alpha * a.y + x.gamma * d1;
    q.z = x.alpha * a.z + x.gamma * d2;
    q.w = x.alpha * a.w + x.gamma * d3;
    if (NEED_C) {
      q.x += x.beta * c.x;
      q.y += x.beta * c.y;
      q.z += x.beta * c.z;
      q.w += x.beta * c.w;
    }
    const float4 v = make_float4(q.x * x.mult, q.y * x.mult, q.z * x.mult, q.w * x.mult);
    put4(O, (long long)r * O.ld, v);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
    mo = fmaxf(mo, max4(v));
    if (HAS_X) {
      float4 xv = make_float4(x.alpha2 * q.x + x.gamma2 * d0, x.alpha2 * q.y + x.gamma2 * d1,
                              x.alpha2 * q.z + x.gamma2 * d2, x.alpha2 * q.w + x.gamma2 * d3);
      if (NEED_C) {
        xv.x += x.beta2 * c.x;
        xv.y += x.beta2 * c.y;
        xv.z += x.beta2 * c.z;
        xv.w += x.beta2 * c.w;
      }
      xv = make_float4(xv.x * x.mult, xv.y * x.mult, xv.z * x.mult, xv.w * x.mult);
      put4(X, (long long)r * X.ld, xv);
      mx = fmaxf(mx, max4(xv));
    }
  }
}

template <int KIND>
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (KIND == 0)
    mma_tf32(d, a, b, idesc, acc);
  else
    mma_f16(d, a, b, idesc, acc);
}

// Ring position: index and the parity of its current round.
struct Ring {
  uint32_t i = 0, ph = 0;
  template <int N>
  __device__ __forceinline__ void next() {
    if (++i == N) {
      i = 0;
      ph ^= 1;
    }
  }
};

template <int KIND, int NPASS, int BN>
__global__ void __launch_bounds__(448, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<KIND, NPASS, BN>;
  using KT = KindTraits<KIND>;
  constexpr int S = C::STAGES;
  constexpr int BKE = C::BKE;
  constexpr int KS = BKE / KT::KINST;  // MMA slices per K-block (4)
  // TMEM: NS accumulation slots of BN columns in a ring, then the handoff
  // block read by the epilogue warps.  FP32 mode fills two slots per K-block
  // (two 32-deep halves), the one-pass modes one slot per DRAIN K-blocks.
  constexpr int NS = C::NBUF;
  constexpr int SPK = (NPASS == 3) ? 2 : 1;  // slots per drained group
  constexpr int KPG = (NPASS == 3) ? 1 : C::DRAIN;
  constexpr uint32_t HANDOFF = NS * BN;
  // one tcgen05.commit per K-block, onto kdone[k % Q]: the producer waits on
  // it to reuse the K-block's stage, the draining warps to read its slots;
  // neither lags the issuer by Q K-blocks or more
  constexpr int Q = 32;
  static_assert(S < Q && NS * KPG < Q, "completion ring too short");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S + Q + NS + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars);        // [S] stage loaded (TMA complete_tx)
  const uint32_t kdone0 = full0 + 8 * S;        // [Q] MMAs of a K-block complete
  const uint32_t tempty0 = kdone0 + 8 * Q;      // [NS] slot drained by all 8 draining warps
  const uint32_t hfull = tempty0 + 8 * NS;      // handoff written by the 8 draining warps
  const uint32_t hempty = hfull + 8;            // handoff read by the 4 epilogue warps
  const uint32_t done_bar = hempty + 8;         // last MMAs of this CTA complete

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) mbar_init(full0 + 8 * s, 1);
    for (int j = 0; j < Q; ++j) mbar_init(kdone0 + 8 * j, 1);
    for (int j = 0; j < NS; ++j) mbar_init(tempty0 + 8 * j, 8);  // one arrival per draining warp
    mbar_init(hfull, 8);
    mbar_init(hempty, 4);
    mbar_init(done_bar, 1);
    // skip all tiles once any CTA has given up on a barrier
    *abort_flag = (*reinterpret_cast<volatile int*>(&shp_dev_error) != 0) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), C::TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = p.total_tiles;

  if (warp == 9) {
    // ---- TMA producer ----
    if (lane == 0) {
      Ring st;
      uint32_t gk = 0;  // K-blocks loaded so far
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
        const Tile x = decode_tile(p, t, BN, BKE);
        const GroupDev& g = p.g[x.grp];
        const int ab = g.a_idx ? g.a_idx[x.b] : x.b;
        const int bb = g.b_idx ? g.b_idx[x.b] : x.b;
        const CUtensorMap* ma = &p.tmA[x.grp][0];
        const CUtensorMap* mb = &p.tmB[x.grp][0];
        const int a_mn = g.a_mn, b_mn = g.b_mn;
        const int a4 = p.a4d[x.grp], b4 = p.b4d[x.grp];
        bool ok = true;
        for (int kb = 0, k0 = 0; kb < x.nk; ++kb, k0 += BKE, ++gk) {
          // the stage was last read by K-block gk - S
          if (gk >= (uint32_t)S) {
            const uint32_t o = gk - S;
            if (!mbar_wait(kdone0 + 8 * (o % Q), (o / Q) & 1)) {
              ok = false;
              break;
            }
          }
          const uint32_t fb = full0 + 8 * st.i;
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + st.i * C::STAGE_BYTES);
          const uint32_t sb = sa + C::NPL * C::A_TILE;
#pragma unroll
          for (int pl = 0; pl < C::NPL; ++pl) {
            if (!a_mn) {
              tma_load_3d(sa + pl * C::A_TILE, ma + pl, fb, k0, x.m0, ab);
            } else if (a4) {
              tma_load_4d(sa + pl * C::A_TILE, ma + pl, fb, 0, k0, x.m0 / BKE, ab);
            } else {  // boxes of BKE (M) x BKE (K rows)
#pragma unroll
              for (int j = 0; j < 128 / BKE; ++j)
                tma_load_3d(sa + pl * C::A_TILE + j * BKE * 128, ma + pl, fb, x.m0 + j * BKE, k0, ab);
            }
            if (!b_mn) {
              tma_load_3d(sb + pl * C::B_TILE, mb + pl, fb, k0, x.n0, bb);
            } else if (b4) {
              tma_load_4d(sb + pl * C::B_TILE, mb + pl, fb, 0, k0, x.n0 / BKE, bb);
            } else {
#pragma unroll
              for (int j = 0; j < BN / BKE; ++j)
                tma_load_3d(sb + pl * C::B_TILE + j * BKE * 128, mb + pl, fb, x.n0 + j * BKE, k0, bb);
            }
          }
          st.template next<S>();
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
      // after an abort, loads may still be landing in stages nobody waited
      // for: let the latest load of every stage finish before the shared
      // memory is given up (immediate when all were consumed)
      for (long long n = (long long)gk - 1; n >= 0 && n >= (long long)gk - S; --n)
        mbar_wait(full0 + 8 * (n % S), (n / S) & 1);
    }
  } else if (warp == 8) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t KSTEP_K = KT::KINST * C::ESZ;  // 32 bytes along a K-major row
      constexpr uint32_t KSTEP_MN = KT::KINST * 128;    // KINST rows of 128 bytes
      constexpr uint32_t LBO_MN = BKE * 128;            // one TMA box along M/N
      const uint32_t smem0 = smem_u32(smem);
      Ring st, sl;
      uint32_t gk = 0;  // K-blocks issued so far
      int in_group = 0;  // K-blocks already accumulated in the current slot (one-pass modes)
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
        const Tile x = decode_tile(p, t, BN, BKE);
        const GroupDev& g = p.g[x.grp];
        const uint32_t idesc = idesc_f32acc(KT::FMT, KT::FMT, g.a_mn, g.b_mn, 128, BN);
        // descriptors of stage 0; the start-address field (address >> 4)
        // never carries out of its 14 bits inside shared memory, so the
        // stage and slice offsets are added to the 64-bit descriptor
        const uint64_t a0 = g.a_mn ? sdesc_sw128(smem0, LBO_MN, KT::MN_SBO, KT::MN_LAYOUT)
                                   : sdesc_sw128(smem0, 16u, 1024u, 2u);
        const uint64_t b0 = g.b_mn ? sdesc_sw128(smem0 + C::NPL * C::A_TILE, LBO_MN, KT::MN_SBO, KT::MN_LAYOUT)
                                   : sdesc_sw128(smem0 + C::NPL * C::A_TILE, 16u, 1024u, 2u);
        const uint64_t a_step = (g.a_mn ? KSTEP_MN : KSTEP_K) >> 4;
        const uint64_t b_step = (g.b_mn ? KSTEP_MN : KSTEP_K) >> 4;
        bool ok = true;
        for (int kb = 0; kb < x.nk && ok; ++kb, ++gk) {
          if (!mbar_wait(full0 + 8 * st.i, st.ph)) {
            ok = false;
            break;
          }
          const uint64_t so = (uint64_t)(st.i * (C::STAGE_BYTES >> 4));
          const uint64_t ad = a0 + so, bd = b0 + so;
          if constexpr (NPASS == 3) {
            // two slots, 32 K each: in each, the correction products lo*hi
            // and hi*lo first (in units of 2^-11), then hi*hi, the first of
            // which scales the slot by 2^-11
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
              if (!mbar_wait(tempty0 + 8 * sl.i, sl.ph ^ 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d = tmem + sl.i * BN;
#pragma unroll
              for (int ks = 2 * hs; ks < 2 * hs + 2; ++ks) {
                mma<KIND>(d, ad + (C::A_TILE >> 4) + ks * a_step, bd + ks * b_step, idesc, ks > 2 * hs ? 1u : 0u);
                mma<KIND>(d, ad + ks * a_step, bd + (C::B_TILE >> 4) + ks * b_step, idesc, 1u);
              }
              mma_f16_scale11(d, ad + 2 * hs * a_step, bd + 2 * hs * b_step, idesc);
              mma<KIND>(d, ad + (2 * hs + 1) * a_step, bd + (2 * hs + 1) * b_step, idesc, 1u);
              sl.template next<NS>();
            }
            if (!ok) break;
          } else {
            if (in_group == 0 && !mbar_wait(tempty0 + 8 * sl.i, sl.ph ^ 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + sl.i * BN;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks)
              mma<KIND>(d, ad + ks * a_step, bd + ks * b_step, idesc, (in_group | ks) ? 1u : 0u);
            if (++in_group == KPG || kb == x.nk - 1) {
              sl.template next<NS>();
              in_group = 0;
            }
          }
          tc_commit(kdone0 + 8 * (gk % Q));
          st.template next<S>();
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
      // every MMA of this CTA has finished before TMEM is given up
      tc_commit(done_bar);
      mbar_wait(done_bar, 0);
    }
  } else if (warp < 8) {
    // ---- draining warps: TMEM slots -> fp32 registers -> handoff ----
    constexpr int HC = BN / 2;
    const int h = warp >> 2;
    const int q = warp & 3;
    const uint32_t lanes = (uint32_t)(q * 32) << 16;
    Ring sl, ho;
    uint32_t gkb = 0;  // K-blocks of the tiles before this one
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (*abort_flag) break;
      const Tile x = decode_tile(p, t, BN, BKE);
      float acc[HC];
#pragma unroll
      for (int i = 0; i < HC; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int k0 = 0; k0 < x.nk; k0 += KPG) {
        // the group is complete once its last K-block's MMAs are
        const uint32_t last = gkb + (uint32_t)((k0 + KPG < x.nk ? k0 + KPG : x.nk) - 1);
        ok = __all_sync(0xffffffffu, mbar_wait(kdone0 + 8 * (last % Q), (last / Q) & 1));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int sj = 0; sj < SPK; ++sj) {
          const uint32_t base = tmem + lanes + (uint32_t)(sl.i * BN + h * HC);
#pragma unroll
          for (int c = 0; c < HC; c += 32) {
            uint32_t r[32];
            tmem_ld32_nowait(base + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c + i] += __uint_as_float(r[i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty0 + 8 * sl.i);
          sl.template next<NS>();
        }
      }
      gkb += (uint32_t)x.nk;
      // hand the tile's sums to the epilogue warps through TMEM
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(hempty, ho.ph ^ 1));
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HC; c += 32) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(acc[c + i]);
        tmem_st32(tmem + lanes + HANDOFF + (uint32_t)(h * HC + c), r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(hfull);
      ho.template next<1>();
    }
  } else {
    // ---- epilogue warps 10-13: handoff -> fused epilogue -> HBM ----
    const int q = warp & 3;  // the TMEM lane quadrant this warp may read
    const uint32_t lanes = (uint32_t)(q * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + S * C::STAGE_BYTES + 512) + (warp - 10) * 1024;
    Ring ho;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (*abort_flag) break;
      const Tile x = decode_tile(p, t, BN, BKE);
      const GroupDev& g = p.g[x.grp];
      const EpiCtx ec = make_ctx(g, x.b, lane == 0);
      if (!__all_sync(0xffffffffu, mbar_wait(hfull, ho.ph))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int bad = 0;
      float ss = 0.f, mo = 0.f, mx = 0.f;
      const int r0 = x.m0 + q * 32;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32_nowait(tmem + lanes + HANDOFF + (uint32_t)(ch * 32), r);
        tmem_wait_ld();
        if (ch == BN / 32 - 1) {  // the handoff is free once its last columns are read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(hempty);
        }
        const int c0 = x.n0 + ch * 32;
        if (g.vec4) {
          float4* stage4 = reinterpret_cast<float4*>(stage);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            stage4[lane * 8 + (j ^ (lane & 7))] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                              __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          __syncwarp();
          if (ec.need_c) {
            if (ec.has_x)
              epilogue_block4<true, true>(g, ec, r0, c0, stage4, lane, ss, bad, mo, mx);
            else
              epilogue_block4<true, false>(g, ec, r0, c0, stage4, lane, ss, bad, mo, mx);
          } else {
            if (ec.has_x)
              epilogue_block4<false, true>(g, ec, r0, c0, stage4, lane, ss, bad, mo, mx);
            else
              epilogue_block4<false, false>(g, ec, r0, c0, stage4, lane, ss, bad, mo, mx);
          }
          if (g.sym && x.m0 != x.n0) {  // the mirrored block of an off-diagonal tile
            if (ec.need_c) {
              if (ec.has_x)
                epilogue_block4<true, true, true>(g, ec, c0, r0, stage4, lane, ss, bad, mo, mx);
              else
                epilogue_block4<true, false, true>(g, ec, c0, r0, stage4, lane, ss, bad, mo, mx);
            } else {
              if (ec.has_x)
                epilogue_block4<false, true, true>(g, ec, c0, r0, stage4, lane, ss, bad, mo, mx);
              else
                epilogue_block4<false, false, true>(g, ec, c0, r0, stage4, lane, ss, bad, mo, mx);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) stage[lane * 32 + (c ^ lane)] = __uint_as_float(r[c]);
          __syncwarp();
          epilogue_block(g, ec, r0, c0 + lane, stage, lane, ss, bad, mo, mx);
        }
        __syncwarp();
      }
      if (g.sumsq) {
#pragma unroll
        for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) atomicAdd(g.sumsq + ec.ob, ss);
      }
      // max |value| of the split outputs, for the scale bound of the next GEMM
      // (non-negative floats order like their bit patterns)
      if (g.O.amax) {
#pragma unroll
        for (int o = 16; o; o >>= 1) mo = fmaxf(mo, __shfl_xor_sync(0xffffffffu, mo, o));
        if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(g.O.amax) + ec.ob, __float_as_uint(mo));
      }
      if (ec.has_x && g.X.amax) {
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(g.X.amax) + ec.ob, __float_as_uint(mx));
      }
      if (g.status && bad) atomicOr(g.status + ec.ob, 1);
      ho.template next<1>();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TCOLS);
  }
}

// ---- host side -------------------------------------------------------------

int num_sms() {
  static std::atomic<int> sms[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int v = sms[dev].load(std::memory_order_relaxed);
  if (!v) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 148;
    sms[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Tensor map over one plane of a stack; box = {bx elements, by rows, 1}.
// atom32: 128-byte swizzle with 32-byte atoms (MN-major tf32 operands).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esz, const Planes& P, int bx, int by,
              bool atom32) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !base) return false;
  cuuint64_t dims[3] = {(cuuint64_t)P.cols, (cuuint64_t)P.rows, (cuuint64_t)P.count};
  cuuint64_t strides[2] = {(cuuint64_t)P.ld * esz, (cuuint64_t)P.bs * esz};
  cuuint32_t box[3] = {(cuuint32_t)bx, (cuuint32_t)by, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D view of an MN-major plane: {bk inner elements, rows (K), column
// chunk, matrix}; one box = `chunks` chunks of bk x bk, stored chunk after
// chunk (the layout of the multi-box loads).  Needs ld % bk == 0 so that
// the last chunk of a row stays inside the padded row.
bool make_map_4d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esz, const Planes& P, int bk,
                 int chunks, bool atom32) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !base) return false;
  cuuint64_t dims[4] = {(cuuint64_t)bk, (cuuint64_t)P.rows, (cuuint64_t)((P.cols + bk - 1) / bk), (cuuint64_t)P.count};
  cuuint64_t strides[3] = {(cuuint64_t)P.ld * esz, (cuuint64_t)bk * esz, (cuuint64_t)P.bs * esz};
  cuuint32_t box[4] = {(cuuint32_t)bk, (cuuint32_t)bk, (cuuint32_t)chunks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int KIND, int NPASS, int BN>
cudaError_t run(GemmParams& prm, cudaStream_t stream) {
  using C = Cfg<KIND, NPASS, BN>;
  // the shared-memory opt-in is per device; set it once on each
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<KIND, NPASS, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev].store(true, std::memory_order_release);
  }
  const int grid = prm.total_tiles < num_sms() ? prm.total_tiles : num_sms();
  gemm_kernel<KIND, NPASS, BN><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmGroup* groups, int ngroups, int batch, Prec prec, cudaStream_t stream) {
  if (ngroups < 1 || ngroups > 2 || batch < 1) return cudaErrorInvalidValue;
  const int kind = (prec == P_FP16 || prec == P_FP32) ? 1 : (prec == P_BF16) ? 2 : 0;
  const int npass = (prec == P_FP32) ? 3 : 1;
  const int esz = kind ? 2 : 4;
  const int bke = 128 / esz;
  const CUtensorMapDataType dt = kind == 0   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : kind == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  int maxN = 0;
  for (int i = 0; i < ngroups; ++i) maxN = groups[i].N > maxN ? groups[i].N : maxN;
  const int BN = maxN <= 64 ? 64 : 128;

  GemmParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.ngroups = ngroups;
  prm.batch = batch;
  long long total = 0;
  for (int i = 0; i < ngroups; ++i) {
    const GemmGroup& G = groups[i];
    if (G.M < 1 || G.N < 1 || G.K < 1) return cudaErrorInvalidValue;
    GroupDev d = G.epi;
    d.M = G.M;
    d.N = G.N;
    d.K = G.K;
    d.a_mn = G.a_mn;
    d.b_mn = G.b_mn;
    d.a_idx = G.a_idx;
    d.b_idx = G.b_idx;
    if (npass == 3) {
      if (!G.A->exp || !G.B->exp || !G.A->amax || !G.B->amax || !G.A->h16lo || !G.B->h16lo)
        return cudaErrorInvalidValue;
      d.a_exp = G.A->exp;
      d.b_exp = G.B->exp;
      d.a_amax = G.A->amax;
      d.b_amax = G.B->amax;
    } else {
      d.a_exp = d.b_exp = nullptr;
      d.a_amax = d.b_amax = nullptr;
      // the split output format needs the operand scales
      if (d.O.h16lo || d.X.h16lo) return cudaErrorInvalidValue;
    }
    prm.g[i] = d;
    prm.a4d[i] = G.a_mn && G.A->ld % bke == 0;
    {
      auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
      auto al8 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 7u) == 0; };
      auto ok_out = [&](const EpiOut& o) {
        return (o.ld % 4 == 0) && (o.bs % 4 == 0) && al16(o.f32) && al8(o.h16) && al8(o.h16lo);
      };
      const bool has_x = d.X.f32 || d.X.h16;
      const bool need_c = d.beta != 0.f || (has_x && d.beta2 != 0.f);
      bool v = G.N % 4 == 0 && ok_out(d.O) && (!has_x || ok_out(d.X));
      if (need_c) v = v && d.C.ld % 4 == 0 && d.C.bs % 4 == 0 && al16(d.C.f32);
      prm.g[i].vec4 = v ? 1 : 0;
    }
    prm.b4d[i] = G.b_mn && G.B->ld % bke == 0;
    for (int pl = 0; pl < (npass == 3 ? 2 : 1); ++pl) {
      const void* abase = kind ? (pl ? G.A->h16lo : G.A->h16) : (const void*)G.A->f32;
      const void* bbase = kind ? (pl ? G.B->h16lo : G.B->h16) : (const void*)G.B->f32;
      if (prm.a4d[i]) {
        if (!make_map_4d(&prm.tmA[i][pl], abase, dt, esz, *G.A, bke, 128 / bke, kind == 0))
          return cudaErrorInvalidValue;
      } else if (!make_map(&prm.tmA[i][pl], abase, dt, esz, *G.A, bke, G.a_mn ? bke : 128, kind == 0 && G.a_mn)) {
        return cudaErrorInvalidValue;
      }
      if (prm.b4d[i]) {
        if (!make_map_4d(&prm.tmB[i][pl], bbase, dt, esz, *G.B, bke, BN / bke, kind == 0))
          return cudaErrorInvalidValue;
      } else if (!make_map(&prm.tmB[i][pl], bbase, dt, esz, *G.B, bke, G.b_mn ? bke : BN, kind == 0 && G.b_mn)) {
        return cudaErrorInvalidValue;
      }
    }
    prm.mt[i] = (G.M + 127) / 128;
    prm.nt[i] = (G.N + BN - 1) / BN;
    prm.g[i].sym = (G.sym && G.M == G.N && BN == 128 && prm.g[i].vec4) ? 1 : 0;
    const long long ti = prm.g[i].sym ? (long long)batch * prm.mt[i] * (prm.mt[i] + 1) / 2
                                      : (long long)batch * prm.mt[i] * prm.nt[i];
    if (i == 0) prm.tiles0 = (int)ti;
    total += ti;
  }
  if (total > (1ll << 30)) return cudaErrorInvalidValue;
  prm.total_tiles = (int)total;
  // the outputs' max |value| accumulate by atomic max from zero
  for (int i = 0; i < ngroups; ++i) {
    const EpiOut* outs[2] = {&groups[i].epi.O, &groups[i].epi.X};
    for (const EpiOut* o : outs)
      if (o->amax && o->amax_n > 0) {
        cudaError_t e = cudaMemsetAsync(o->amax, 0, sizeof(float) * o->amax_n, stream);
        if (e != cudaSuccess) return e;
      }
  }
  if (npass == 3) return BN == 64 ? run<1, 3, 64>(prm, stream) : run<1, 3, 128>(prm, stream);
  if (kind == 0) return BN == 64 ? run<0, 1, 64>(prm, stream) : run<0, 1, 128>(prm, stream);
  if (kind == 1) return BN == 64 ? run<1, 1, 64>(prm, stream) : run<1, 1, 128>(prm, stream);
  return BN == 64 ? run<2, 1, 64>(prm, stream) : run<2, 1, 128>(prm, stream);
}

}  // namespace shp
