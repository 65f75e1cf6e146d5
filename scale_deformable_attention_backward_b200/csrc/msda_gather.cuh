// msda_gather.cuh -- the per-point setup and the corner accumulation of the
// gather (forward) kernels, and the location formula of the fused op:
// msda_forward.cu and msda_fused.cu (sm_100a).
//
// Sampling rule of "Deformable DETR模型解读（附源码+论文）",
// ms_deform_attn_core_pytorch: a point's four bilinear corners, each weighted
// by A * (1 - fx or fx) * (1 - fy or fy) and read as zero outside the map.
#pragma once

#include "msda_device.cuh"

namespace msda {

// The setup of one point: element offsets of its four corners relative to the
// (b, m, channel) base pointer, -1 for a corner outside the map, in the order
// V(x0,y0), V(x0+1,y0), V(x0,y0+1), V(x0+1,y0+1); and the four weights
// A * bilinear in the same order.
struct PointSetup {
  int4 off;
  float4 w;
};

__device__ __forceinline__ PointSetup setup_point(float lx, float ly, float a, int H, int W,
                                                  long long start, int MD) {
  const Cell c = locate(lx, ly, H, W);
  const float hx = 1.0f - c.fx, hy = 1.0f - c.fy;
  PointSetup s;
  s.w = make_float4(a * hx * hy, a * c.fx * hy, a * hx * c.fy, a * c.fx * c.fy);
  const int base = static_cast<int>(start + static_cast<long long>(c.y0) * W + c.x0);
  // Offsets are formed only for corners inside the map, where 0 <= pixel < S and
  // pixel * M * D < 2^31 (checked by the C ABI).
  s.off.x = (c.vx0 && c.vy0) ? base * MD : -1;
  s.off.y = (c.vx1 && c.vy0) ? (base + 1) * MD : -1;
  s.off.z = (c.vx0 && c.vy1) ? (base + W) * MD : -1;
  s.off.w = (c.vx1 && c.vy1) ? (base + W + 1) * MD : -1;
  // A point with no corner in the map adds A * 0 to the output, which is NaN when
  // its weights are not finite (a non-finite location or weight).  Such a point
  // reads the level's first pixel with a NaN weight, so the NaN reaches the sum.
  if ((s.off.x & s.off.y & s.off.z & s.off.w) < 0 && W > 0 &&
      !isfinite(s.w.x + s.w.y + s.w.z + s.w.w)) {
    s.off.x = static_cast<int>(start) * MD;
    s.w.x = __int_as_float(0x7fffffff);
  }
  return s;
}

template <typename T>
struct Corner;

template <>
struct Corner<float> {
  static constexpr int N = 4;
  // acc += w * value[0..3] for one corner inside the map.
  __device__ __forceinline__ static void accumulate(const float* p, float w, float2 (&acc)[2]) {
    if (!in_bounds(p, 16, false)) return;
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    const float2 ww = make_float2(w, w);
    acc[0] = fma2(ww, make_float2(v.x, v.y), acc[0]);
    acc[1] = fma2(ww, make_float2(v.z, v.w), acc[1]);
  }
  // All four corners of one point: the loads are predicated (a corner outside the
  // map reads as zero without being loaded), then the accumulation runs in the
  // corners' order.  A corner outside the map still takes its FMA with the zero
  // it read: w * 0 leaves the sum unchanged (up to the sign of a zero sum), NaN
  // weights still make it NaN, and issuing the FMAs unconditionally measured
  // faster than branching around them.
  __device__ __forceinline__ static void accumulate4(const float* vbase, const int4& o,
                                                     const float4& w, float2 (&acc)[2]) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v0 = z, v1 = z, v2 = z, v3 = z;
    if (o.x >= 0 && in_bounds(vbase + o.x, 16, false))
      v0 = __ldg(reinterpret_cast<const float4*>(vbase + o.x));
    if (o.y >= 0 && in_bounds(vbase + o.y, 16, false))
      v1 = __ldg(reinterpret_cast<const float4*>(vbase + o.y));
    if (o.z >= 0 && in_bounds(vbase + o.z, 16, false))
      v2 = __ldg(reinterpret_cast<const float4*>(vbase + o.z));
    if (o.w >= 0 && in_bounds(vbase + o.w, 16, false))
      v3 = __ldg(reinterpret_cast<const float4*>(vbase + o.w));
    const float4 vs[4] = {v0, v1, v2, v3};
    const float ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 ww = make_float2(ws[c], ws[c]);
      acc[0] = fma2(ww, make_float2(vs[c].x, vs[c].y), acc[0]);
      acc[1] = fma2(ww, make_float2(vs[c].z, vs[c].w), acc[1]);
    }
  }
  __device__ __forceinline__ static void store(float* p, const float2 (&acc)[2]) {
    *reinterpret_cast<float4*>(p) = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
  }
};

template <>
struct Corner<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void accumulate(const __nv_bfloat16* p, float w,
                                                    float2 (&acc)[4]) {
    if (!in_bounds(p, 16, false)) return;
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const unsigned u[4] = {r.x, r.y, r.z, r.w};
    const float2 ww = make_float2(w, w);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc[i] = fma2(ww, make_float2(__uint_as_float(u[i] << 16),
                                    __uint_as_float(u[i] & 0xffff0000u)), acc[i]);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float2 (&acc)[4]) {
    unsigned u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(acc[i].x, acc[i].y);
      u[i] = *reinterpret_cast<const unsigned*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
  }
};

// The sampling location of one point, formed as the pages' float32 tensors do.
__device__ __forceinline__ float2 fused_location(const float* __restrict__ ref, float2 off, int R,
                                                 int W, int H, int K) {
  if (R == 2)
    return make_float2(__fadd_rn(__ldg(ref + 0), __fdiv_rn(off.x, static_cast<float>(W))),
                       __fadd_rn(__ldg(ref + 1), __fdiv_rn(off.y, static_cast<float>(H))));
  const float fk = static_cast<float>(K);
  const float tx = __fmul_rn(__fmul_rn(__fdiv_rn(off.x, fk), __ldg(ref + 2)), 0.5f);
  const float ty = __fmul_rn(__fmul_rn(__fdiv_rn(off.y, fk), __ldg(ref + 3)), 0.5f);
  return make_float2(__fadd_rn(__ldg(ref + 0), tx), __fadd_rn(__ldg(ref + 1), ty));
}

// A maximum that keeps NaN, so that a NaN logit makes the whole group's
// weights NaN (as the softmax does).
__device__ __forceinline__ float nan_max(float a, float b) { return (b > a || b != b) ? b : a; }

}  // namespace msda
