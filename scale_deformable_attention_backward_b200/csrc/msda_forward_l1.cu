// msda_forward_l1.cu -- forward of the MSDeformAttn core for the encoder form,
// with 2-D query tiles whose value windows stay in L1 (sm_100a).
//
//   out[b, q, m*D + d] = sum_{l,k} A[b,q,m,l,k] * bilinear(value_l[b, :, m, d], loc[b,q,m,l,k])
//
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation; sampling rule and output layout of
// "Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch.
//
// The per-point gather of msda_forward.cu with a different assignment of work:
// one CTA of 1024 threads per SM owns a rectangle of up to TH x TW queries of
// one image and one head (msda_tile.cuh), a sub-warp per query, and walks the
// sampled levels one step at a time.  The points of a step then fall into one
// small window of one head's value plane, which stays in L1 while the step's
// corners are gathered with read-only 16-byte loads; each CTA takes a
// contiguous run of tiles in row-major order, so the next tile's windows
// overlap the current ones.  Each step is the gather kernel's two phases --
// set up the step's points into a swizzled shared table, then gather -- with
// the next step's locations and weights loaded during the gathers and its
// table built in the other buffer, one barrier per step.  The float32 sums run
// in the gather kernel's order (level, point, corner), so the outputs are the
// same bits.
#include <atomic>
#include <climits>

#include "msda_device.cuh"
#include "msda_gather.cuh"
#include "msda_launch.h"
#include "msda_tile.cuh"

namespace msda {

namespace {

constexpr int kL1Threads = 1024;
constexpr int kL1MaxK = 8;

}  // namespace

template <typename T, int LANES>
__global__ void __launch_bounds__(kL1Threads, 1)
forward_l1_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                  const int64_t* __restrict__ level_start_index,
                  const float* __restrict__ sampling_locations,
                  const float* __restrict__ attention_weights, T* __restrict__ output, int B,
                  long long S, int M, long long Lq, int L, int K, int TH, int TW) {
  using C = Corner<T>;
  constexpr int E = C::N;
  constexpr int D = LANES * E;
  constexpr int G = kL1Threads / LANES;                // queries (sub-warps) per tile
  constexpr int PER = (G * kL1MaxK + kL1Threads - 1) / kL1Threads;  // points set up per thread
  static_assert(G >= 8, "the shared-table swizzle needs at least 8 groups");
  extern __shared__ __align__(16) unsigned char smem[];
  const int P = G * K;  // points per step (table entries per buffer)
  int4* s_off = reinterpret_cast<int4*>(smem);          // [2][P]
  float4* s_w = reinterpret_cast<float4*>(smem + 2 * P * 16);  // [2][P]
  __shared__ Levels lv;
  __shared__ TileGrid tg;
  stage_levels(lv, spatial_shapes, level_start_index, L, S);
  const int Q = TH * TW;  // <= G
  build_tile_grid(tg, lv, L, S, Lq, TH, TW, Q);

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int LK = L * K;
  const int MD = M * D;

  // This CTA's run of items; item = (b * M + m) * tiles + tile.
  const long long items = static_cast<long long>(tg.tiles) * B * M;
  const long long first = items * blockIdx.x / gridDim.x;
  const long long last = items * (blockIdx.x + 1) / gridDim.x;
  if (first >= last) return;
  const long long steps = (last - first) * L;

  // Per step: which item and level.
  struct StepPos {
    int b, m, l;
    TileQueries tq;
  };
  auto position = [&](long long s) {
    StepPos p;
    const long long it = first + s / L;
    p.l = static_cast<int>(s % L);
    const int t = static_cast<int>(it % tg.tiles);
    const int bm = static_cast<int>(it / tg.tiles);
    p.b = bm / M;
    p.m = bm - p.b * M;
    p.tq = tile_queries(tg, lv, L, t, Q, Lq);
    return p;
  };

  float2 pxy[PER];
  float pa[PER];
  auto prefetch = [&](const StepPos& sp) {
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int p = threadIdx.x + r * kL1Threads;
      const int qi = p / K;
      if (p < P && qi < sp.tq.count) {
        const int k = p - qi * K;
        const long long idx =
            ((sp.b * Lq + sp.tq.query(qi)) * M + sp.m) * static_cast<long long>(LK) +
            sp.l * K + k;
        pxy[r] = __ldg(reinterpret_cast<const float2*>(sampling_locations) + idx);
        pa[r] = __ldg(attention_weights + idx);
      }
    }
  };
  auto setup = [&](const StepPos& sp, int buf) {
    const int H = lv.H[sp.l], W = lv.W[sp.l];
    const long long start = lv.start[sp.l];
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int p = threadIdx.x + r * kL1Threads;
      const int qi = p / K;
      if (p < P && qi < sp.tq.count) {
        const int k = p - qi * K;
        const PointSetup su = setup_point(pxy[r].x, pxy[r].y, pa[r], H, W, start, MD);
        const int slot = k * G + (qi ^ (k & 7));
        s_off[buf * P + slot] = su.off;
        s_w[buf * P + slot] = su.w;
      }
    }
  };

  StepPos cur = position(0);
  prefetch(cur);
  setup(cur, 0);
  __syncthreads();
  float2 acc[E / 2];
#pragma unroll
  for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
  int buf = 0;
  for (long long s = 0; s < steps; ++s) {
    const bool more = s + 1 < steps;
    StepPos nxt;
    if (more) {
      nxt = position(s + 1);
      prefetch(nxt);
    }
    if (gi < cur.tq.count) {
      const T* vbase = value + (static_cast<long long>(cur.b) * S * M + cur.m) * D + lane * E;
      if constexpr (E == 4) {
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
          const int slot = buf * P + k * G + (gi ^ (k & 7));
          C::accumulate4(vbase, s_off[slot], s_w[slot], acc);
        }
      } else {
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
          const int slot = buf * P + k * G + (gi ^ (k & 7));
          const int4 o = s_off[slot];
          const float4 w = s_w[slot];
          if (o.x >= 0) C::accumulate(vbase + o.x, w.x, acc);
          if (o.y >= 0) C::accumulate(vbase + o.y, w.y, acc);
          if (o.z >= 0) C::accumulate(vbase + o.z, w.z, acc);
          if (o.w >= 0) C::accumulate(vbase + o.w, w.w, acc);
        }
      }
      if (cur.l == L - 1) {
        C::store(output + (static_cast<long long>(cur.b) * Lq + cur.tq.query(gi)) * MD +
                     cur.m * D + lane * E,
                 acc);
      }
    }
    if (cur.l == L - 1) {
#pragma unroll
      for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
    }
    if (more) setup(nxt, buf ^ 1);
    __syncthreads();
    cur = nxt;
    buf ^= 1;
  }
}

namespace {

template <typename T, int LANES>
cudaError_t launch_l1_t(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int G = kL1Threads / LANES;
  const size_t smem = static_cast<size_t>(2) * G * a.K * 32;
  static std::atomic<int> sm_count[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sm_count[dev].load() == 0) {
    int n = 0;
    if ((err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return err;
    sm_count[dev].store(n > 0 ? n : 1);
  }
  if ((err = cudaFuncSetAttribute(forward_l1_kernel<T, LANES>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
    return err;
  // Tiles of G queries: 8 x 16 for 128, 16 x 16 for 256, 8 x 8 for 64.
  const int TH = G >= 256 ? 16 : 8;
  const int TW = G / TH;
  long long blocks = sm_count[dev].load();
  const long long upper = a.B * a.M * a.Lq;
  if (blocks > upper) blocks = upper;
  forward_l1_kernel<T, LANES><<<static_cast<unsigned>(blocks), kL1Threads, smem, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.sampling_locations, a.attention_weights, static_cast<T*>(a.output),
      static_cast<int>(a.B), a.S, a.M, a.Lq, a.L, a.K, TH, TW);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_l1(const ForwardArgs& a, cudaStream_t stream) {
  if (a.K > kL1MaxK) return cudaErrorNotSupported;
  const int row = a.bf16 ? a.D * 2 : a.D * 4;
  if (a.bf16) {
    switch (row) {
      case 64: return launch_l1_t<__nv_bfloat16, 4>(a, stream);
      case 128: return launch_l1_t<__nv_bfloat16, 8>(a, stream);
      case 256: return launch_l1_t<__nv_bfloat16, 16>(a, stream);
      default: return cudaErrorNotSupported;
    }
  }
  switch (row) {
    case 64: return launch_l1_t<float, 4>(a, stream);
    case 128: return launch_l1_t<float, 8>(a, stream);
    case 256: return launch_l1_t<float, 16>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace msda
