// msda_device.cuh -- device-side building blocks shared by the forward and
// backward kernels of the MSDeformAttn core (sm_100a).
//
// Sampling rule ("Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch:
// grid = 2*loc - 1, grid_sample bilinear, zeros padding, align_corners=False):
// the pixel coordinate of a normalised location is x = loc * W - 0.5, the
// bilinear cell is [floor(x), floor(x) + 1) and a corner outside [0, W) reads 0.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "msda_launch.h"

namespace msda {

constexpr unsigned kFullMask = 0xffffffffu;

// ---------------------------------------------------------------------------
// Bounds checks of the debug build (libmsda_debug.so, compiled with
// MSDA_DEBUG_BOUNDS).  Every gather of a value or grad_output row and every
// reduction into grad_value (or the deterministic path's integer accumulators)
// first checks that its bytes lie inside a buffer of the current call, which the
// C ABI registers before it launches (bounds_ranges: two readable, two writable).
// An access outside them is skipped -- a read gives zeros -- and the first one
// is recorded in bounds_error as kind << 60 | address (kind 1: read, 2: write),
// for msda_debug_bounds_check to report.  In the release build in_bounds() is a
// constant true and the checks compile away.
// ---------------------------------------------------------------------------
struct BoundsRanges {
  unsigned long long lo[4];  // [0, 2): readable; [2, 4): writable
  unsigned long long hi[4];  // one past the end; lo == hi: no buffer
};

#ifdef MSDA_DEBUG_BOUNDS
extern __device__ BoundsRanges bounds_ranges;
extern __device__ unsigned long long bounds_error;
#endif

__device__ __forceinline__ bool in_bounds(const void* p, int bytes, bool write) {
#ifdef MSDA_DEBUG_BOUNDS
  const unsigned long long a = reinterpret_cast<unsigned long long>(p);
  const int first = write ? 2 : 0;
#pragma unroll
  for (int i = first; i < first + 2; ++i)
    if (a >= bounds_ranges.lo[i] && a + bytes <= bounds_ranges.hi[i]) return true;
  atomicCAS(&bounds_error, 0ull, ((write ? 2ull : 1ull) << 60) | (a & ((1ull << 60) - 1)));
  return false;
#else
  (void)p;
  (void)bytes;
  (void)write;
  return true;
#endif
}

// Per-level metadata staged in shared memory.  A level whose metadata would
// reach outside `value` is staged as 0 x 0, so none of its corners is valid and
// it is never read.
struct Levels {
  int H[kMaxLevels];
  int W[kMaxLevels];
  long long start[kMaxLevels];
};

__device__ __forceinline__ void stage_levels(Levels& lv, const int64_t* __restrict__ shapes,
                                             const int64_t* __restrict__ level_start, int L,
                                             int64_t S) {
  for (int l = threadIdx.x; l < L; l += blockDim.x) {
    const int64_t h = shapes[2 * l + 0];
    const int64_t w = shapes[2 * l + 1];
    const int64_t st = level_start[l];
    const bool ok = h >= 1 && w >= 1 && h < kMaxLevelExtent && w < kMaxLevelExtent &&
                    st >= 0 && st <= S && h * w <= S - st;
    lv.H[l] = ok ? static_cast<int>(h) : 0;
    lv.W[l] = ok ? static_cast<int>(w) : 0;
    lv.start[l] = ok ? st : 0;
  }
  __syncthreads();
}

// One axis of the pixel mapping, exact in the floor.
//   x = loc * n - 0.5 (real arithmetic);  c = floor(x);  f = x - c rounded once.
// fmaf gives x rounded once, which may land on the wrong side of an integer;
// the sign of fmaf(loc, n, -(c + 0.5)) = RN(x - c) is exact (round-to-nearest
// keeps signs, and x - c is a nonzero multiple of 2^-149 or exactly zero), so c is
// corrected by at most one step.  c + 0.5 and c + 1.5 are exact for |c| < 2^22.
// A coordinate outside (-2, n + 1) has no corner inside the map and is reported
// as c = -2 (with f = 0; no weight of it multiplies a value).  A non-finite
// location also gets c = -2 but f = NaN, so the point's weights -- and its
// sample, as in grid_sample -- are NaN.
__device__ __forceinline__ void pixel_coordinate(float loc, float n, float& c, float& f) {
  const float t = fmaf(loc, n, -0.5f);
  if (!(fabsf(loc) <= 3.402823466e38f)) {
    c = -2.0f;
    f = loc - loc;  // NaN for NaN and for +-Inf
  } else if (t > -2.0f && t < n + 1.0f) {
    c = floorf(t);
    f = fmaf(loc, n, -(c + 0.5f));
    if (f < 0.0f) {
      c -= 1.0f;
      f = fmaf(loc, n, -(c + 0.5f));
    } else if (fmaf(loc, n, -(c + 1.5f)) >= 0.0f) {
      c += 1.0f;
      f = fmaf(loc, n, -(c + 0.5f));
    }
  } else {
    c = -2.0f;
    f = 0.0f;
  }
}

// The sampling geometry of one point on its level.
// The level of point j of a group, floor(j / K), without an integer division
// per point: with m = ceil(2^32 / K) (K >= 2), floor(j m / 2^32) = floor(j / K)
// for 0 <= j < 2^16 and K <= 2^16.  j m / 2^32 exceeds j / K by less than
// j / 2^32 < 2^-16 <= 1 / K, while the fraction of j / K is at most 1 - 1 / K,
// so the sum stays below the next integer.  Here j < L K <= 1024.  m = 0
// stands for K = 1.
__device__ __forceinline__ unsigned level_magic(int K) {
  return K > 1 ? 0xFFFFFFFFu / static_cast<unsigned>(K) + 1u : 0u;
}
__device__ __forceinline__ int level_of(int j, unsigned magic) {
  return magic != 0u ? static_cast<int>(__umulhi(static_cast<unsigned>(j), magic)) : j;
}

struct Cell {
  int x0, y0;                 // top-left corner (may lie outside the map)
  float fx, fy;               // position inside the cell
  bool vx0, vx1, vy0, vy1;    // corner columns / rows inside the map
};

__device__ __forceinline__ Cell locate(float lx, float ly, int H, int W) {
  Cell c;
  float cx, cy;
  pixel_coordinate(lx, static_cast<float>(W), cx, c.fx);
  pixel_coordinate(ly, static_cast<float>(H), cy, c.fy);
  c.x0 = static_cast<int>(cx);
  c.y0 = static_cast<int>(cy);
  c.vx0 = static_cast<unsigned>(c.x0) < static_cast<unsigned>(W);
  c.vx1 = static_cast<unsigned>(c.x0 + 1) < static_cast<unsigned>(W);
  c.vy0 = static_cast<unsigned>(c.y0) < static_cast<unsigned>(H);
  c.vy1 = static_cast<unsigned>(c.y0 + 1) < static_cast<unsigned>(H);
  return c;
}

// Packed float32 pair FMA (sm_100): d = a * b + c on both halves, each rounded
// once as fmaf would.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}

// Packed float32 pair subtraction and product (sm_100): each half rounded once,
// as the scalar operation would.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

// Weight of a corner whose grad_value contribution was merged into another
// point's (a signalling NaN: float arithmetic never produces one).
constexpr unsigned kNoScatterBits = 0x7f800001u;

// Two points of one group and one level can share a corner pixel (same or
// neighbouring cells).  Their grad_value contributions there are w1 gO and
// w2 gO with the group's gO, so one reduction of (w1 + w2) gO does the work of
// two.  The level's K = 4 points sit in 4 aligned consecutive lanes, each with
// its cell (x0, y0), the mask vm of its corners that may merge (inside the map,
// bit i + 2j for corner (x0 + i, y0 + j)) and its corner weights `w`.  Partner cells at
// (dx, dy) with |dx|, |dy| <= 1 share corner c of this point with the
// partner's corner c - dx - 2 dy.  The lowest lane holding a pixel adds the
// others' weights to its own; the others mark theirs kNoScatterBits, which the
// scatter skips while the gathers still read the corner.  A NaN or Inf weight
// lands on the same pixel either way.  All 32 lanes of the warp must call this.
__device__ __forceinline__ void merge_shared_corners(int x0, int y0, unsigned vm, float4& w) {
  const int me = threadIdx.x & 3;
  // y0 and vm in one word (y0 of a point with a corner in the map is below 2^22).
  const unsigned ky = (static_cast<unsigned>(y0) << 4) | vm;
  const float w0[4] = {w.x, w.y, w.z, w.w};
  float sum[4] = {w.x, w.y, w.z, w.w};
  unsigned merged = 0;
#pragma unroll
  for (int o = 1; o < 4; ++o) {
    const int px = __shfl_xor_sync(kFullMask, x0, o, 4);
    const unsigned pky = __shfl_xor_sync(kFullMask, ky, o, 4);
    float pw[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) pw[c] = __shfl_xor_sync(kFullMask, w0[c], o, 4);
    // Unsigned differences: a point with no corner in the map (vm = 0) may
    // carry any cell, and it matches nothing below.
    const unsigned ux = static_cast<unsigned>(px) - static_cast<unsigned>(x0);
    const unsigned uy = static_cast<unsigned>(static_cast<int>(pky) >> 4) -
                        static_cast<unsigned>(y0);
    if (ux + 1u <= 2u && uy + 1u <= 2u) {
      const int dx = static_cast<int>(ux), dy = static_cast<int>(uy);
      const int sh = dx + 2 * dy;  // partner corner = this corner - sh
      const unsigned mx = dx == 0 ? 15u : (dx > 0 ? 0xau : 0x5u);  // corners with x0 + i in both cells
      const unsigned my = dy == 0 ? 15u : (dy > 0 ? 0xcu : 0x3u);
      const unsigned pvm = pky & 15u;
      const unsigned m = mx & my & vm & (sh >= 0 ? pvm << sh : pvm >> -sh) & 15u;
      if ((me ^ o) < me) {
        merged |= m;
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int i = c - sh;
          const float v = i == 0 ? pw[0] : i == 1 ? pw[1] : i == 2 ? pw[2] : pw[3];
          if ((m >> c) & 1u) sum[c] += v;
        }
      }
    }
  }
  const float skip = __uint_as_float(kNoScatterBits);
  w = make_float4((merged & 1u) ? skip : sum[0], (merged & 2u) ? skip : sum[1],
                  (merged & 4u) ? skip : sum[2], (merged & 8u) ? skip : sum[3]);
}

// Phase-1 step of the float backward kernels, after a point's corner offsets
// `off` (-1 outside the map) and weights `w` are formed (every lane of the warp,
// with off = -1 on lanes that hold no point): with K = 4 (`merge`, uniform over
// the warp) the corners shared by the level's points are merged; then every
// corner that scatters nothing is marked kNoScatterBits, so that the scatter
// tests the weight alone.  A zero weight is not merged: 0 * gO is NaN where gO
// is infinite, and (0 + w2) gO would not be.
__device__ __forceinline__ void prepare_scatter_weights(int x0, int y0, const int4& off,
                                                        bool merge, float4& w) {
  if (merge) {
    const unsigned vm = (off.x >= 0 ? 1u : 0u) | (off.y >= 0 ? 2u : 0u) |
                        (off.z >= 0 ? 4u : 0u) | (off.w >= 0 ? 8u : 0u);
    const unsigned nz = (w.x != 0.0f ? 1u : 0u) | (w.y != 0.0f ? 2u : 0u) |
                        (w.z != 0.0f ? 4u : 0u) | (w.w != 0.0f ? 8u : 0u);
    merge_shared_corners(x0, y0, vm & nz, w);
  }
  const float skip = __uint_as_float(kNoScatterBits);
  if (off.x < 0) w.x = skip;
  if (off.y < 0) w.y = skip;
  if (off.z < 0) w.z = skip;
  if (off.w < 0) w.w = skip;
}

// The four sums of one point over a lane's 4 channels: P = sum gO V00,
// Ex = sum gO (V10 - V00), Ey = sum gO (V01 - V00),
// Exy = sum gO ((V11 - V01) - (V10 - V00)), with q[i] the corners in the order
// V00, V10, V01, V11.  The corner differences are taken per channel, so a common
// offset of the value field cancels exactly, not between large dot products.
// Channel pairs go through the packed two-wide float32 unit.
__device__ __forceinline__ void corner_sums4(const float (&q)[4][4], const float (&go)[4],
                                             float (&dot)[4]) {
  float2 d2[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) d2[k] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float2 v00 = make_float2(q[0][2 * h], q[0][2 * h + 1]);
    const float2 v10 = make_float2(q[1][2 * h], q[1][2 * h + 1]);
    const float2 v01 = make_float2(q[2][2 * h], q[2][2 * h + 1]);
    const float2 v11 = make_float2(q[3][2 * h], q[3][2 * h + 1]);
    const float2 dx = sub2(v10, v00);
    const float2 dy = sub2(v01, v00);
    const float2 dxy = sub2(sub2(v11, v01), dx);
    const float2 g = make_float2(go[2 * h], go[2 * h + 1]);
    d2[0] = fma2(g, v00, d2[0]);
    d2[1] = fma2(g, dx, d2[1]);
    d2[2] = fma2(g, dy, d2[2]);
    d2[3] = fma2(g, dxy, d2[3]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) dot[k] = d2[k].x + d2[k].y;
}

// The lane reduction of the backward kernels, two points at a time.  Each lane
// of a sub-warp of LANES lanes holds three partial sums of points A and B (ta,
// tb) over its channels.  The first exchange sends the lower half of the
// sub-warp B's partials and the upper half A's, so after log2(LANES) rounds of
// three shuffles lanes [0, LANES/2) hold A's totals and lanes [LANES/2, LANES)
// B's (4.5 shuffles per point for LANES = 8, against 12 for a butterfly of four
// sums per point).
template <int LANES>
__device__ __forceinline__ void reduce_pair3(const float (&ta)[3], const float (&tb)[3], int lane,
                                             float (&v)[3]) {
  constexpr int HALF = LANES / 2;
  const bool upper = (lane & HALF) != 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const float send = upper ? ta[i] : tb[i];
    const float mine = upper ? tb[i] : ta[i];
    v[i] = mine + __shfl_xor_sync(kFullMask, send, HALF, LANES);
  }
#pragma unroll
  for (int sh = HALF / 2; sh > 0; sh >>= 1) {
#pragma unroll
    for (int i = 0; i < 3; ++i) v[i] += __shfl_xor_sync(kFullMask, v[i], sh, LANES);
  }
}

// The point of a batch of LANES points whose totals lane `lane` keeps after
// reduce_pair3 over the pairs (0, 1), (2, 3), ...: lane u keeps point 2u, lane
// LANES/2 + u point 2u + 1 (lane 0 keeps point 0 when LANES = 1).
template <int LANES>
__device__ __forceinline__ int pair_lane_point(int lane) {
  if constexpr (LANES == 1) {
    return 0;
  } else {
    constexpr int HALF = LANES / 2;
    return (lane & HALF) ? 2 * (lane - HALF) + 1 : 2 * lane;
  }
}

// A point's three sums over a lane's channels from its four corner sums
// (corner_sums4), with its fx, fy applied before the lane reduction (linear, so
// the order of the two does not matter in real arithmetic):
//   t0 = P + fx Ex + fy Ey + fx fy Exy   (grad_attn),
//   t1 = Ex + fy Exy,  t2 = Ey + fx Exy    (grad_loc / (A W, A H)).
__device__ __forceinline__ void point_sums3(const float (&dot)[4], float fx, float fy,
                                            float (&t)[3]) {
  t[1] = fmaf(fy, dot[3], dot[1]);
  t[2] = fmaf(fx, dot[3], dot[2]);
  t[0] = fmaf(fx, t[1], fmaf(fy, dot[2], dot[0]));
}

// grad_value[p .. p + 3] += w * g[0 .. 3], one 16-byte vector reduction.
__device__ __forceinline__ void scatter_row4(float* p, float w, const float (&g)[4]) {
  if (!in_bounds(p, 16, true)) return;
  const float2 ww = make_float2(w, w);
  const float2 lo = mul2(ww, make_float2(g[0], g[1]));
  const float2 hi = mul2(ww, make_float2(g[2], g[3]));
  atomicAdd(reinterpret_cast<float4*>(p), make_float4(lo.x, lo.y, hi.x, hi.y));
}

// ---------------------------------------------------------------------------
// 16-byte lane vectors: 4 x float32 or 8 x bfloat16, widened to float32.
// ---------------------------------------------------------------------------
template <typename T>
struct Vec;

template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float (&v)[N]) {
    const float4 r = in_bounds(p, 16, false) ? __ldg(reinterpret_cast<const float4*>(p))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
  __device__ __forceinline__ static void store(float* p, const float (&v)[N]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[N]) {
    const uint4 r = in_bounds(p, 16, false) ? __ldg(reinterpret_cast<const uint4*>(p))
                                            : make_uint4(0u, 0u, 0u, 0u);
    const unsigned w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i + 0] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float (&v)[N]) {
    unsigned w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i + 0], v[2 * i + 1]);
      w[i] = *reinterpret_cast<const unsigned*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

// 4 channels per lane, widened to float32: 16 bytes of float32 or 8 bytes of
// bfloat16 (the backward's lane width for both dtypes).
template <typename T>
struct Vec4;

template <>
struct Vec4<float> {
  __device__ __forceinline__ static void load(const float* p, float (&v)[4]) {
    const float4 r = in_bounds(p, 16, false) ? __ldg(reinterpret_cast<const float4*>(p))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
};

template <>
struct Vec4<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 r = in_bounds(p, 8, false) ? __ldg(reinterpret_cast<const uint2*>(p))
                                           : make_uint2(0u, 0u);
    v[0] = __uint_as_float(r.x << 16);
    v[1] = __uint_as_float(r.x & 0xffff0000u);
    v[2] = __uint_as_float(r.y << 16);
    v[3] = __uint_as_float(r.y & 0xffff0000u);
  }
};

// Decomposition of a flat work-group index g = ((b * Lq + q) * M + m) * chunks + c.
struct Group {
  long long bq;    // b * Lq + q
  long long bqm;   // (b * Lq + q) * M + m
  long long b;
  int m;
  int chunk;
};

__device__ __forceinline__ Group decompose(long long g, int chunks, int M, long long Lq) {
  Group r;
  if (g < (1ll << 31)) {
    // 32-bit divisions: a 64-bit one costs several times the instructions, and
    // this runs per thread per work unit.  g < 2^31 implies bq < 2^31.
    const unsigned u = static_cast<unsigned>(g);
    unsigned bqm = u;
    r.chunk = 0;
    if (chunks != 1) {
      bqm = u / static_cast<unsigned>(chunks);
      r.chunk = static_cast<int>(u - bqm * static_cast<unsigned>(chunks));
    }
    const unsigned bq = bqm / static_cast<unsigned>(M);
    r.m = static_cast<int>(bqm - bq * static_cast<unsigned>(M));
    r.bqm = bqm;
    r.bq = bq;
    // Lq > bq means b = 0 (this also covers Lq >= 2^31, which would not fit the
    // 32-bit division).
    r.b = Lq > static_cast<long long>(bq) ? 0 : bq / static_cast<unsigned>(Lq);
    return r;
  }
  r.chunk = static_cast<int>(g % chunks);
  r.bqm = g / chunks;
  r.m = static_cast<int>(r.bqm % M);
  r.bq = r.bqm / M;
  r.b = r.bq / Lq;
  return r;
}

}  // namespace msda
