// msda_backward_sorted.cu -- training backward of the MSDeformAttn core with
// the points grouped by bilinear cell (sm_100a).
//
// Same derivatives as msda_backward.cu (exact derivative of the forward of
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation, sampled as in "Deformable DETR模型
// 解读（附源码+论文）", ms_deform_attn_core_pytorch).  All three gradients of a
// point are linear in the four corner dot products
//     G_ij = sum_d gO[d] * V(x0 + i, y0 + j)[d]
// of its cell:
//     grad_attn  = hy (hx G00 + fx G10) + fy (hx G01 + fx G11)
//     grad_loc.x = A W (hy (G10 - G00) + fy (G11 - G01))
//     grad_loc.y = A H (hx (G01 - G00) + fx (G11 - G10))
// and its grad_value contribution to corner ij is A w_ij gO.  Points that
// share a cell (the same (b, m, level, x0, y0)) share the four corner rows of
// value and the four target rows of grad_value, so they are processed together:
//
//   1. bin     one thread per point: the cell of the point, a slot in it
//              (atomic increment of the cell's count); points with no corner in
//              the map get their (zero or NaN) gradients here and no slot;
//   2. scan    exclusive prefix sum of the counts (three small launches);
//   3. place   one thread per point: its (id, A, fx, fy) record at
//              offset[cell] + slot;
//   4. cells   a sub-warp per cell: the four corner rows loaded once, then for
//              every point of the cell one 16-byte load of grad_output per lane,
//              the four partial dot products and the four grad_value
//              accumulators in registers; dot products are reduced for a batch
//              of points at once (reduce-scatter across the lanes, so lane j
//              finishes point j), and each corner gets one vector atomic per
//              cell instead of one per point.
//
// Scratch (caller-provided workspace, see msda_backward_workspace_size): cell
// counts / offsets, scan block sums, one (cell, slot) pair and one 16-byte
// record per point.
#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kThreads = 256;
constexpr int kScanItems = 8;                        // per thread
constexpr int kScanTile = kThreads * kScanItems;     // elements per scan block

// Cells of level l occupy [base[l], base[l] + count[l]) inside the segment of
// one (b, m), count[l] = (H_l + 1)(W_l + 1); cell (x0, y0), x0 in [-1, W-1],
// y0 in [-1, H-1], is at (y0 + 1)(W + 1) + (x0 + 1).  With consistent metadata
// the levels fill at most 2 S + 2 L cells, the segment length; a level that would
// reach past the segment (possible only when levels overlap in `value`) gets
// count 0, so its points are never binned and no cell index leaves the array.
struct CellLevels {
  int base[kMaxLevels];
  int count[kMaxLevels];
};

__device__ __forceinline__ void stage_cells(CellLevels& cl, const Levels& lv, int L,
                                            long long cells_per_bm) {
  if (threadIdx.x == 0) {
    long long acc = 0;
    for (int l = 0; l < L; ++l) {
      const long long n = (lv.H[l] > 0) ? (lv.H[l] + 1ll) * (lv.W[l] + 1ll) : 0;
      const bool fits = acc + n <= cells_per_bm;
      cl.base[l] = static_cast<int>(acc);
      cl.count[l] = fits ? static_cast<int>(n) : 0;
      if (fits) acc += n;
    }
  }
  __syncthreads();
}

struct PointIndex {
  long long bq;
  int m, l;
};

__device__ __forceinline__ PointIndex split_point(long long p, int LK, int K, int M) {
  PointIndex r;
  const long long bqm = p / LK;
  r.l = static_cast<int>(p - bqm * LK) / K;
  r.m = static_cast<int>(bqm % M);
  r.bq = bqm / M;
  return r;
}

__global__ void __launch_bounds__(kThreads)
bin_kernel(const int64_t* __restrict__ spatial_shapes, const int64_t* __restrict__ level_start,
           const float* __restrict__ sampling_locations,
           const float* __restrict__ attention_weights, float* __restrict__ grad_loc,
           float* __restrict__ grad_attn, int* __restrict__ counts, int2* __restrict__ bin_slot,
           long long S, int M, long long Lq, int L, int K, long long cells_per_bm,
           long long points) {
  __shared__ Levels lv;
  __shared__ CellLevels cl;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  stage_cells(cl, lv, L, cells_per_bm);
  const int LK = L * K;
  for (long long p = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; p < points;
       p += static_cast<long long>(gridDim.x) * kThreads) {
    const PointIndex pi = split_point(p, LK, K, M);
    const int H = lv.H[pi.l], W = lv.W[pi.l];
    const float2 xy = __ldg(reinterpret_cast<const float2*>(sampling_locations) + p);
    const Cell c = locate(xy.x, xy.y, H, W);
    if ((c.vx0 || c.vx1) && (c.vy0 || c.vy1) && cl.count[pi.l] > 0) {
      const long long b = pi.bq / Lq;
      const long long bin = (b * M + pi.m) * cells_per_bm + cl.base[pi.l] +
                            static_cast<long long>(c.y0 + 1) * (W + 1) + (c.x0 + 1);
      const int slot = atomicAdd(counts + bin, 1);
      bin_slot[p] = make_int2(static_cast<int>(bin), slot);
    } else {
      // No corner in the map: every corner dot product is 0.  The products with
      // the weights keep the NaN of a non-finite location, as the oracle does.
      bin_slot[p] = make_int2(-1, 0);
      const float a = __ldg(attention_weights + p);
      grad_attn[p] = 0.0f * (c.fx + c.fy);
      reinterpret_cast<float2*>(grad_loc)[p] =
          make_float2(a * static_cast<float>(W) * (0.0f * c.fy),
                      a * static_cast<float>(H) * (0.0f * c.fx));
    }
  }
}

// Exclusive scan, pass 1: each block scans its tile in place and records the
// tile total.
__global__ void __launch_bounds__(kThreads)
scan_tiles_kernel(int* __restrict__ data, int* __restrict__ tile_sums, long long n) {
  __shared__ int warp_sums[kThreads / 32];
  const long long base = blockIdx.x * static_cast<long long>(kScanTile) +
                         threadIdx.x * static_cast<long long>(kScanItems);
  int v[kScanItems];
  int total = 0;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    v[i] = (base + i < n) ? data[base + i] : 0;
    total += v[i];
  }
  // Block-wide exclusive scan of the per-thread totals.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(kFullMask, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kThreads / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFullMask, w, o);
      if (lane >= o) w += t;
    }
    if (lane < kThreads / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  int run = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    if (base + i < n) data[base + i] = run;
    run += v[i];
  }
  if (threadIdx.x == kThreads - 1) tile_sums[blockIdx.x] = run;
}

// Pass 2: exclusive scan of the tile sums, one block looping over them.
__global__ void __launch_bounds__(1024) scan_sums_kernel(int* __restrict__ sums, int n) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int b0 = 0; b0 < n; b0 += 1024) {
    const int i = b0 + threadIdx.x;
    const int v = (i < n) ? sums[i] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFullMask, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFullMask, w, o);
        if (lane >= o) w += t;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int excl = carry + incl - v + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (i < n) sums[i] = excl;
    __syncthreads();
    if (threadIdx.x == 1023) carry = excl + v;
    __syncthreads();
  }
}

// Pass 3: add each tile's offset.
__global__ void __launch_bounds__(kThreads)
scan_add_kernel(int* __restrict__ data, const int* __restrict__ tile_sums, long long n) {
  const long long base = blockIdx.x * static_cast<long long>(kScanTile);
  const int add = tile_sums[blockIdx.x];
  for (int i = threadIdx.x; i < kScanTile; i += kThreads)
    if (base + i < n) data[base + i] += add;
}

__global__ void __launch_bounds__(kThreads)
place_kernel(const int64_t* __restrict__ spatial_shapes, const int64_t* __restrict__ level_start,
             const float* __restrict__ sampling_locations,
             const float* __restrict__ attention_weights, const int* __restrict__ offsets,
             const int2* __restrict__ bin_slot, float4* __restrict__ records, long long S,
             int M, int L, int K, long long points) {
  __shared__ Levels lv;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  const int LK = L * K;
  for (long long p = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; p < points;
       p += static_cast<long long>(gridDim.x) * kThreads) {
    const int2 bs = bin_slot[p];
    if (bs.x < 0) continue;
    const int l = static_cast<int>(p % LK) / K;
    const float2 xy = __ldg(reinterpret_cast<const float2*>(sampling_locations) + p);
    const Cell c = locate(xy.x, xy.y, lv.H[l], lv.W[l]);
    const float a = __ldg(attention_weights + p);
    records[offsets[bs.x] + bs.y] =
        make_float4(__int_as_float(static_cast<int>(p)), a, c.fx, c.fy);
  }
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

__device__ __forceinline__ void axpy4(float w, const float4& x, float4& y) {
  y.x = fmaf(w, x.x, y.x);
  y.y = fmaf(w, x.y, y.y);
  y.z = fmaf(w, x.z, y.z);
  y.w = fmaf(w, x.w, y.w);
}

// Cell pass.  LANES lanes per cell, 4 channels per lane (D <= 4 * LANES); NB =
// min(LANES, 8) points per batch.
template <int LANES>
__global__ void __launch_bounds__(kThreads)
cell_kernel(const float* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
            const int64_t* __restrict__ level_start, const float* __restrict__ grad_output,
            const int* __restrict__ offsets, const float4* __restrict__ records,
            float* __restrict__ grad_value, float* __restrict__ grad_loc,
            float* __restrict__ grad_attn, long long S, int M, int D, long long Lq, int L,
            int K, long long cells_per_bm, long long bins) {
  constexpr int NB = LANES < 8 ? LANES : 8;
  __shared__ Levels lv;
  __shared__ CellLevels cl;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  stage_cells(cl, lv, L, cells_per_bm);
  const int lane = threadIdx.x % LANES;
  const int per_block = kThreads / LANES;
  const int LK = L * K;
  const int MD = M * D;
  const int ch = lane * 4;
  // Sub-warps work on different cells with different point counts, so their
  // shuffles name only their own lanes.
  const unsigned sub_mask =
      LANES == 32 ? kFullMask
                  : ((1u << (LANES & 31)) - 1u) << ((threadIdx.x & 31) & ~(LANES - 1));

  for (long long bin0 = blockIdx.x * static_cast<long long>(per_block); bin0 < bins;
       bin0 += static_cast<long long>(gridDim.x) * per_block) {
    const long long bin = bin0 + threadIdx.x / LANES;
    // Every lane of a sub-warp sees the same bin, so the sub-warp stays converged.
    const int begin = bin < bins ? offsets[bin] : 0;
    const int end = bin < bins ? offsets[bin + 1] : 0;
    if (begin >= end) continue;
    const long long seg = bin / cells_per_bm;
    const int within = static_cast<int>(bin - seg * cells_per_bm);
    const int m = static_cast<int>(seg % M);
    const long long b = seg / M;
    // The level whose cell range holds this (non-empty) bin.
    int l = 0;
    while (l + 1 < L && !(within >= cl.base[l] && within < cl.base[l] + cl.count[l])) ++l;
    const int H = lv.H[l], W = lv.W[l];
    const int cell = within - cl.base[l];
    const int y0 = cell / (W + 1) - 1, x0 = cell % (W + 1) - 1;
    const bool vx0 = x0 >= 0, vx1 = x0 + 1 < W, vy0 = y0 >= 0, vy1 = y0 + 1 < H;
    const bool lane_on = ch < D;
    const long long vofs = (b * S * M + m) * static_cast<long long>(D) + ch;
    const long long pix = lv.start[l] + static_cast<long long>(y0) * W + x0;
    // Corner rows of this cell: c00 = V(x0, y0), c10 = V(x0+1, y0), c01 = V(x0, y0+1), ...
    const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float4 c00 = zero, c10 = zero, c01 = zero, c11 = zero;
    if (lane_on) {
      if (vx0 && vy0) c00 = __ldg(reinterpret_cast<const float4*>(value + vofs + pix * MD));
      if (vx1 && vy0) c10 = __ldg(reinterpret_cast<const float4*>(value + vofs + (pix + 1) * MD));
      if (vx0 && vy1) c01 = __ldg(reinterpret_cast<const float4*>(value + vofs + (pix + W) * MD));
      if (vx1 && vy1)
        c11 = __ldg(reinterpret_cast<const float4*>(value + vofs + (pix + W + 1) * MD));
    }
    float4 a00 = zero, a10 = zero, a01 = zero, a11 = zero;  // grad_value accumulators

    for (int i0 = begin; i0 < end; i0 += NB) {
      // Lane j < NB holds record i0 + j.
      float4 rec = make_float4(__int_as_float(-1), 0.0f, 0.0f, 0.0f);
      if (lane < NB && i0 + lane < end) rec = records[i0 + lane];
      float part[4][NB];
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const int p = __float_as_int(__shfl_sync(sub_mask, rec.x, j, LANES));
        const float a = __shfl_sync(sub_mask, rec.y, j, LANES);
        const float fx = __shfl_sync(sub_mask, rec.z, j, LANES);
        const float fy = __shfl_sync(sub_mask, rec.w, j, LANES);
        float4 go = zero;
        if (p >= 0 && lane_on) {
          const long long bq = static_cast<long long>(p) / (static_cast<long long>(M) * LK);
          go = __ldg(reinterpret_cast<const float4*>(grad_output + bq * MD +
                                                     static_cast<long long>(m) * D + ch));
        }
        part[0][j] = dot4(go, c00);
        part[1][j] = dot4(go, c10);
        part[2][j] = dot4(go, c01);
        part[3][j] = dot4(go, c11);
        const float hx = 1.0f - fx, hy = 1.0f - fy;
        axpy4(a * hx * hy, go, a00);
        axpy4(a * fx * hy, go, a10);
        axpy4(a * hx * fy, go, a01);
        axpy4(a * fx * fy, go, a11);
      }
      // Full butterfly over the lane bits above the batch, then a reduce-scatter
      // so that lane j (< NB) ends with the totals of point j.
#pragma unroll
      for (int o = LANES / 2; o >= NB; o >>= 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < NB; ++j) part[q][j] += __shfl_xor_sync(sub_mask, part[q][j], o, LANES);
      }
#pragma unroll
      for (int o = NB / 2; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < o; ++j) {
            // Keep indices with bit o equal to this lane's bit; send the others.
            const float send = upper ? part[q][j] : part[q][j + o];
            const float keep = upper ? part[q][j + o] : part[q][j];
            part[q][j] = keep + __shfl_xor_sync(sub_mask, send, o, LANES);
          }
      }
      // part[q][0] now holds the totals of point `lane` (for lane < NB).
      const int p = __float_as_int(rec.x);
      if (lane < NB && p >= 0) {
        const float a = rec.y, fx = rec.z, fy = rec.w;
        const float hx = 1.0f - fx, hy = 1.0f - fy;
        const float g00 = part[0][0], g10 = part[1][0], g01 = part[2][0], g11 = part[3][0];
        grad_attn[p] = fmaf(hy, fmaf(fx, g10, hx * g00), fy * fmaf(fx, g11, hx * g01));
        reinterpret_cast<float2*>(grad_loc)[p] = make_float2(
            a * static_cast<float>(W) * fmaf(hy, g10 - g00, fy * (g11 - g01)),
            a * static_cast<float>(H) * fmaf(hx, g01 - g00, fx * (g11 - g10)));
      }
    }
    if (lane_on) {
      float* gv = grad_value + vofs;
      if (vx0 && vy0) atomicAdd(reinterpret_cast<float4*>(gv + pix * MD), a00);
      if (vx1 && vy0) atomicAdd(reinterpret_cast<float4*>(gv + (pix + 1) * MD), a10);
      if (vx0 && vy1) atomicAdd(reinterpret_cast<float4*>(gv + (pix + W) * MD), a01);
      if (vx1 && vy1) atomicAdd(reinterpret_cast<float4*>(gv + (pix + W + 1) * MD), a11);
    }
  }
}

template <typename T>
T* carve(char*& cursor, long long count) {
  T* p = reinterpret_cast<T*>(cursor);
  cursor += (count * static_cast<long long>(sizeof(T)) + 255) / 256 * 256;
  return p;
}

unsigned grid_for(long long items, long long per_block) {
  long long blocks = (items + per_block - 1) / per_block;
  if (blocks > (1ll << 30)) blocks = 1ll << 30;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

template <int LANES>
cudaError_t launch_cells(const BackwardArgs& a, const SortedLayout& w, const int* offsets,
                         const float4* records, cudaStream_t stream) {
  cell_kernel<LANES><<<grid_for(w.bins, kThreads / LANES), kThreads, 0, stream>>>(
      a.value, a.spatial_shapes, a.level_start_index, a.grad_output, offsets, records,
      a.grad_value, a.grad_sampling_locations, a.grad_attention_weights, a.S, a.M, a.D, a.Lq,
      a.L, a.K, w.cells_per_bm, w.bins);
  return cudaGetLastError();
}

}  // namespace

SortedLayout sorted_layout(long long B, long long S, long long M, long long Lq, int L, int K) {
  SortedLayout w;
  // sum_l (H_l + 1)(W_l + 1) <= 2 S + 2 L, because H + W <= H W + 1 for H, W >= 1.
  w.cells_per_bm = 2 * S + 2 * L;
  w.bins = B * M * w.cells_per_bm;
  w.points = B * Lq * M * L * K;
  w.scan_tiles = (w.bins + 1 + kScanTile - 1) / kScanTile;
  auto up = [](long long bytes) { return (bytes + 255) / 256 * 256; };
  w.bytes = up(4 * (w.bins + 1)) + up(4 * w.scan_tiles) + up(8 * w.points) + up(16 * w.points);
  return w;
}

cudaError_t launch_backward_sorted(const BackwardArgs& a, void* workspace,
                                   cudaStream_t stream) {
  const SortedLayout w = sorted_layout(a.B, a.S, a.M, a.Lq, a.L, a.K);
  char* cursor = static_cast<char*>(workspace);
  int* counts = carve<int>(cursor, w.bins + 1);
  int* tile_sums = carve<int>(cursor, w.scan_tiles);
  int2* bin_slot = carve<int2>(cursor, w.points);
  float4* records = carve<float4>(cursor, w.points);

  cudaError_t err = launch_zero(a.grad_value, a.value_elements, stream);
  if (err != cudaSuccess) return err;
  err = launch_zero_words(counts, w.bins + 1, stream);
  if (err != cudaSuccess || w.points == 0) return err;

  bin_kernel<<<grid_for(w.points, kThreads), kThreads, 0, stream>>>(
      a.spatial_shapes, a.level_start_index, a.sampling_locations, a.attention_weights,
      a.grad_sampling_locations, a.grad_attention_weights, counts, bin_slot, a.S, a.M, a.Lq,
      a.L, a.K, w.cells_per_bm, w.points);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_tiles_kernel<<<static_cast<unsigned>(w.scan_tiles), kThreads, 0, stream>>>(
      counts, tile_sums, w.bins + 1);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_sums_kernel<<<1, 1024, 0, stream>>>(tile_sums, static_cast<int>(w.scan_tiles));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_add_kernel<<<static_cast<unsigned>(w.scan_tiles), kThreads, 0, stream>>>(
      counts, tile_sums, w.bins + 1);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  place_kernel<<<grid_for(w.points, kThreads), kThreads, 0, stream>>>(
      a.spatial_shapes, a.level_start_index, a.sampling_locations, a.attention_weights, counts,
      bin_slot, records, a.S, a.M, a.L, a.K, w.points);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  switch (a.lanes) {
    case 1: return launch_cells<1>(a, w, counts, records, stream);
    case 2: return launch_cells<2>(a, w, counts, records, stream);
    case 4: return launch_cells<4>(a, w, counts, records, stream);
    case 8: return launch_cells<8>(a, w, counts, records, stream);
    case 16: return launch_cells<16>(a, w, counts, records, stream);
    case 32: return launch_cells<32>(a, w, counts, records, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace msda
