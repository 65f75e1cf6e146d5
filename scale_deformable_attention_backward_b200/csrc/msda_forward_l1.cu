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
// one image and one head (msda_tile.cuh) -- a sub-warp of LANES lanes per
// query, each lane 16 bytes of the head's channels -- and all its sub-warps
// walk their queries' points in the same order (level, point).  So at any
// moment the CTA samples one small window of one head's value plane, which
// stays in L1 while its corners are gathered with read-only 16-byte loads; each
// CTA takes a contiguous run of tiles in row-major order, so the next tile's
// windows overlap the current ones.
//
// Per item (tile, b, m) the gather kernel's two phases: every thread maps up to
// PER of the item's points (queries x L x K) -- exact floor, corner validity,
// 32-bit corner offsets, the four weights A * bilinear -- into a swizzled shared
// table; after a barrier each sub-warp gathers its query's points from it,
// with the gather kernel's arithmetic in the gather kernel's order (level,
// point, corner), so the outputs are the same bits.  The next item's
// locations and weights load during the gathers; a second barrier frees the
// table.
#include <atomic>
#include <climits>

#include "msda_device.cuh"
#include "msda_gather.cuh"
#include "msda_launch.h"
#include "msda_tile.cuh"

namespace msda {

namespace {

constexpr int kL1Threads = 1024;
constexpr int kL1Blocks = 1;  // CTAs per SM
constexpr int kL1TableEntries = 4096;  // points per item at most (128 KB of table)

}  // namespace

// PER: points each thread sets up per item (queries x L x K <= PER * 1024).
template <typename T, int LANES, int PER>
__global__ void __launch_bounds__(kL1Threads, kL1Blocks)
forward_l1_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                  const int64_t* __restrict__ level_start_index,
                  const float* __restrict__ sampling_locations,
                  const float* __restrict__ attention_weights, T* __restrict__ output, int B,
                  long long S, int M, long long Lq, int L, int K, int TH, int TW) {
  using C = Corner<T>;
  constexpr int E = C::N;
  constexpr int D = LANES * E;
  constexpr int G = kL1Threads / LANES;  // queries (sub-warps) per tile
  static_assert(G >= 8, "the shared-table swizzle needs at least 8 groups");
  extern __shared__ __align__(16) unsigned char smem[];
  const int LK = L * K;
  const int P = G * LK;  // table entries
  int4* s_off = reinterpret_cast<int4*>(smem);               // [P]
  float4* s_w = reinterpret_cast<float4*>(smem + P * 16);    // [P]
  __shared__ Levels lv;
  __shared__ TileGrid tg;
  stage_levels(lv, spatial_shapes, level_start_index, L, S);
  const int Q = TH * TW;  // <= G
  build_tile_grid(tg, lv, L, S, Lq, TH, TW, Q);

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int MD = M * D;

  // This CTA's run of items; item = (b * M + m) * tiles + tile (< 2^31).
  const long long items = static_cast<long long>(tg.tiles) * B * M;
  const int first = static_cast<int>(items * blockIdx.x / gridDim.x);
  const int last = static_cast<int>(items * (blockIdx.x + 1) / gridDim.x);
  if (first >= last) return;

  // This thread's points of an item: p = query qi * LK + point j (fixed).
  int qi_r[PER], j_r[PER], l_r[PER];
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const int p = threadIdx.x + r * kL1Threads;
    qi_r[r] = p < P ? p / LK : G;  // G: never a query of a tile
    j_r[r] = p - qi_r[r] * LK;
    l_r[r] = p < P ? j_r[r] / K : 0;
  }
  struct Item {
    int b, m;
    TileQueries tq;
  };
  auto decode = [&](int it) {
    Item r;
    const int t = it % tg.tiles;
    const int bm = it / tg.tiles;
    r.b = bm / M;
    r.m = bm - r.b * M;
    r.tq = tile_queries(tg, lv, L, t, Q, Lq);
    return r;
  };
  float2 pxy[PER];
  float pa[PER];
  auto prefetch = [&](const Item& it) {
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      if (qi_r[r] < it.tq.count) {
        const long long idx =
            ((it.b * Lq + it.tq.query(qi_r[r])) * M + it.m) * static_cast<long long>(LK) + j_r[r];
        pxy[r] = __ldg(reinterpret_cast<const float2*>(sampling_locations) + idx);
        pa[r] = __ldg(attention_weights + idx);
      }
    }
  };

  Item cur = decode(first);
  prefetch(cur);
  for (int it = first; it < last; ++it) {
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int qi = qi_r[r];
      if (qi < cur.tq.count) {
        const int l = l_r[r], j = j_r[r];
        const PointSetup su =
            setup_point(pxy[r].x, pxy[r].y, pa[r], lv.H[l], lv.W[l], lv.start[l], MD);
        const int slot = j * G + (qi ^ (j & 7));
        s_off[slot] = su.off;
        s_w[slot] = su.w;
      }
    }
    __syncthreads();  // the item's table is complete
    const Item nxt = it + 1 < last ? decode(it + 1) : cur;
    if (it + 1 < last) prefetch(nxt);
    if (gi < cur.tq.count) {
      const T* vbase = value + (static_cast<long long>(cur.b) * S * M + cur.m) * D + lane * E;
      float2 acc[E / 2];
#pragma unroll
      for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
      if constexpr (E == 4) {
#pragma unroll 8
        for (int j = 0; j < LK; ++j) {
          const int slot = j * G + (gi ^ (j & 7));
          C::accumulate4(vbase, s_off[slot], s_w[slot], acc);
        }
      } else {
#pragma unroll 4
        for (int j = 0; j < LK; ++j) {
          const int slot = j * G + (gi ^ (j & 7));
          const int4 o = s_off[slot];
          const float4 w = s_w[slot];
          if (o.x >= 0) C::accumulate(vbase + o.x, w.x, acc);
          if (o.y >= 0) C::accumulate(vbase + o.y, w.y, acc);
          if (o.z >= 0) C::accumulate(vbase + o.z, w.z, acc);
          if (o.w >= 0) C::accumulate(vbase + o.w, w.w, acc);
        }
      }
      C::store(output + (static_cast<long long>(cur.b) * Lq + cur.tq.query(gi)) * MD +
                   cur.m * D + lane * E,
               acc);
    }
    __syncthreads();  // the table is free for the next item
    cur = nxt;
  }
}

namespace {

template <typename T, int LANES, int PER>
cudaError_t launch_l1_t(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int G = kL1Threads / LANES;
  const size_t smem = static_cast<size_t>(G) * a.L * a.K * 32;
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
  if ((err = cudaFuncSetAttribute(forward_l1_kernel<T, LANES, PER>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
    return err;
  // Tiles of G queries: 8 x 16 for 128, 16 x 16 for 256, 8 x 8 for 64.
  const int TH = G >= 256 ? 16 : 8;
  const int TW = G / TH;
  long long blocks = static_cast<long long>(sm_count[dev].load()) * kL1Blocks;
  const long long upper = a.B * a.M * a.Lq;
  if (blocks > upper) blocks = upper;
  forward_l1_kernel<T, LANES, PER><<<static_cast<unsigned>(blocks), kL1Threads, smem, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.sampling_locations, a.attention_weights, static_cast<T*>(a.output),
      static_cast<int>(a.B), a.S, a.M, a.Lq, a.L, a.K, TH, TW);
  return cudaGetLastError();
}

}  // namespace

// An item's table holds tile queries x L x K points: at most 4096 (128 KB).
template <typename T, int LANES>
cudaError_t launch_l1_lanes(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int G = kL1Threads / LANES;
  const int points = G * a.L * a.K;
  if (points <= 2 * kL1Threads) return launch_l1_t<T, LANES, 2>(a, stream);
  if (points <= kL1TableEntries) return launch_l1_t<T, LANES, 4>(a, stream);
  return cudaErrorNotSupported;
}

cudaError_t launch_forward_l1(const ForwardArgs& a, cudaStream_t stream) {
  const int row = a.bf16 ? a.D * 2 : a.D * 4;
  if (a.bf16) {
    switch (row) {
      case 64: return launch_l1_lanes<__nv_bfloat16, 4>(a, stream);
      case 128: return launch_l1_lanes<__nv_bfloat16, 8>(a, stream);
      case 256: return launch_l1_lanes<__nv_bfloat16, 16>(a, stream);
      default: return cudaErrorNotSupported;
    }
  }
  switch (row) {
    case 64: return launch_l1_lanes<float, 4>(a, stream);
    case 128: return launch_l1_lanes<float, 8>(a, stream);
    case 256: return launch_l1_lanes<float, 16>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace msda
