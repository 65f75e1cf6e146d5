// msda_forward.cu -- forward kernel of the MSDeformAttn core (sm_100a).
//
//   out[b, q, m*D + d] = sum_{l,k} A[b,q,m,l,k] * bilinear(value_l[b, :, m, d], loc[b,q,m,l,k])
//
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation; sampling rule and output layout of
// "Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch.
//
// Work decomposition: a sub-warp of LANES lanes owns one (b, q, m, channel
// chunk) group; each lane owns 16 contiguous bytes of the head's channels, so one
// corner of one point is a single fully used 128-byte line for D = 32 float32.
// The group's 2*L*K locations and L*K weights are read coalesced, LANES points at
// a time (lane j holds point j of the round), and broadcast with shuffles; every
// lane then maps the point to its cell and gathers its slice of the four corners
// with 16-byte read-only loads, accumulating in float32 registers.  Consecutive
// groups are consecutive heads of consecutive queries, so the blocks resident at
// any moment cover neighbouring queries, whose samples overlap in L1 and L2.
#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

template <typename T, int LANES>
__global__ void __launch_bounds__(256)
forward_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
               const int64_t* __restrict__ level_start_index,
               const float* __restrict__ sampling_locations,
               const float* __restrict__ attention_weights, T* __restrict__ output,
               long long S, int M, int D, long long Lq, int L, int K, int chunks,
               long long groups) {
  using V = Vec<T>;
  constexpr int E = V::N;
  __shared__ Levels lv;
  stage_levels(lv, spatial_shapes, level_start_index, L, S);

  const int lane = threadIdx.x % LANES;
  const int groups_per_block = blockDim.x / LANES;
  const int LK = L * K;
  const long long MD = static_cast<long long>(M) * D;

  for (long long g0 = static_cast<long long>(blockIdx.x) * groups_per_block; g0 < groups;
       g0 += static_cast<long long>(gridDim.x) * groups_per_block) {
    const long long g_raw = g0 + threadIdx.x / LANES;
    const bool active = g_raw < groups;
    // Inactive groups (the tail of the last block) still take part in the
    // shuffles, on a clamped group, and store nothing.
    const Group grp = decompose(active ? g_raw : groups - 1, chunks, M, Lq);
    const int ch = (grp.chunk * LANES + lane) * E;
    const bool lane_on = active && ch < D;  // clamped tail groups touch no memory
    const T* vbase = value + (grp.b * S * M + grp.m) * static_cast<long long>(D) + ch;
    const float* gloc = sampling_locations + grp.bqm * LK * 2;
    const float* gatt = attention_weights + grp.bqm * LK;

    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0f;

    int l = 0, k = 0;
    int H = lv.H[0], W = lv.W[0];
    long long start = lv.start[0];
    for (int p0 = 0; p0 < LK; p0 += LANES) {
      const int pj = p0 + lane;
      float2 xy = make_float2(0.0f, 0.0f);
      float aj = 0.0f;
      if (pj < LK) {
        xy = __ldg(reinterpret_cast<const float2*>(gloc) + pj);
        aj = __ldg(gatt + pj);
      }
      const int n = min(LANES, LK - p0);
      for (int j = 0; j < n; ++j) {
        const float lx = __shfl_sync(kFullMask, xy.x, j, LANES);
        const float ly = __shfl_sync(kFullMask, xy.y, j, LANES);
        const float a = __shfl_sync(kFullMask, aj, j, LANES);
        const Cell c = locate(lx, ly, H, W);
        if (lane_on) {
          // Corner weights, w<i><j> for V(x0 + i, y0 + j).
          const float hx = 1.0f - c.fx, hy = 1.0f - c.fy;
          const float w00 = a * hx * hy, w10 = a * c.fx * hy;
          const float w01 = a * hx * c.fy, w11 = a * c.fx * c.fy;
          const long long row = static_cast<long long>(W) * MD;
          const long long off = (start + static_cast<long long>(c.y0) * W + c.x0) * MD;
          float v[E];
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = 0.0f;
          if (c.vx0 && c.vy0) V::load(vbase + off, v);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w00, v[e], acc[e]);
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = 0.0f;
          if (c.vx1 && c.vy0) V::load(vbase + off + MD, v);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w10, v[e], acc[e]);
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = 0.0f;
          if (c.vx0 && c.vy1) V::load(vbase + off + row, v);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w01, v[e], acc[e]);
#pragma unroll
          for (int e = 0; e < E; ++e) v[e] = 0.0f;
          if (c.vx1 && c.vy1) V::load(vbase + off + row + MD, v);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(w11, v[e], acc[e]);
        }
        if (++k == K) {
          k = 0;
          if (++l < L) {
            H = lv.H[l];
            W = lv.W[l];
            start = lv.start[l];
          }
        }
      }
    }
    if (lane_on) V::store(output + grp.bq * MD + static_cast<long long>(grp.m) * D + ch, acc);
  }
}

template <typename T, int LANES>
static cudaError_t launch_forward_t(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int kThreads = 256;
  const long long per_block = kThreads / LANES;
  long long blocks = (a.groups + per_block - 1) / per_block;
  if (blocks > (1ll << 30)) blocks = 1ll << 30;
  forward_kernel<T, LANES><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.sampling_locations, a.attention_weights, static_cast<T*>(a.output), a.S, a.M, a.D,
      a.Lq, a.L, a.K, a.chunks, a.groups);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t dispatch_lanes(const ForwardArgs& a, cudaStream_t stream) {
  switch (a.lanes) {
    case 1: return launch_forward_t<T, 1>(a, stream);
    case 2: return launch_forward_t<T, 2>(a, stream);
    case 4: return launch_forward_t<T, 4>(a, stream);
    case 8: return launch_forward_t<T, 8>(a, stream);
    case 16: return launch_forward_t<T, 16>(a, stream);
    case 32: return launch_forward_t<T, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_forward(const ForwardArgs& a, cudaStream_t stream) {
  return a.bf16 ? dispatch_lanes<__nv_bfloat16>(a, stream) : dispatch_lanes<float>(a, stream);
}

}  // namespace msda
