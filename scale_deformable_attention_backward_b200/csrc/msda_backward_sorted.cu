// msda_backward_sorted.cu -- training backward of the MSDeformAttn core with
// the points grouped by bilinear cell (sm_100a).
//
// Same derivatives as msda_backward.cu (exact derivative of the forward of
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation, sampled as in "Deformable DETR模型
// 解读（附源码+论文）", ms_deform_attn_core_pytorch).  All three gradients of a
// point are linear in four sums over the channels of its cell's corners,
// with the corner differences taken per channel (corner_sums):
//     P = sum_d gO V00,  Ex = sum_d gO (V10 - V00),  Ey = sum_d gO (V01 - V00),
//     Exy = sum_d gO (V11 - V01 - V10 + V00)
//     grad_attn  = P + fx Ex + fy Ey + fx fy Exy
//     grad_loc.x = A W (Ex + fy Exy)
//     grad_loc.y = A H (Ey + fx Exy)
// and its grad_value contribution to corner ij is A w_ij gO.  Points that
// share a cell (the same (b, m, level, x0, y0)) add to the same four rows of
// grad_value, so they are summed in registers first.
//
// Why sort: measured on B200, L2 serves about 4.8e10 atomic requests per second
// (one request = one 128-byte line, whether it carries a 16-byte vector
// reduction from each of 8 lanes or a bulk TMA reduction), i.e. about 1.5e12
// float adds/s.  One atomic per point corner costs ~0.85 ms on the encoder
// training workload; one per cell corner a few tens of microseconds.  Global
// atomics are kept out of the sort as well (a per-point global counter costs as
// much as the scatter it replaces).
//
// A segment is one (b, m, level); it holds Lq * K points, cut into chunks of
// kChunkPoints.  The cells of a segment are indexed (y0 + 1)(W + 1) + (x0 + 1),
// x0 in [-1, W-1], y0 in [-1, H-1]; key = (b * M + m) * cells_per_bm + base_l +
// cell identifies a cell globally (base_l: cells of the levels before l).
//
//   1. hist    one block per (segment, chunk): the cell of each point and its slot
//              among the chunk's points of that cell (shared-memory atomic);
//              the chunk's per-cell counts go to counts[chunk][key] (coalesced
//              rows).  no_corner_kernel, launched after it, gives the points
//              with no corner in the map their (zero or NaN) gradients.
//   2. offsets per-key totals over the chunks, their exclusive prefix sum (three
//              launches), then counts[chunk][key] becomes the position of the
//              (key, chunk) run in the sorted record array.
//   3. place   one block per (segment, chunk): the chunk's run offsets of the
//              segment's cells are staged in shared memory; each point's record
//              (id, A, fx, fy) and key go to offset + slot.
//   4. cells   every sub-warp takes a fixed run of consecutive records, so the
//              work is balanced whatever the cell sizes.  For a batch of records
//              it issues all their corner and grad_output loads at once (in sorted
//              order the corners are mostly L1 hits), forms the four dot
//              products and adds A w_ij gO into four accumulators that belong to
//              the current cell; when the cell changes they are flushed with one
//              16-byte vector atomic per lane and corner (two when the next cell
//              is the right neighbour, whose left column they share).  Dot
//              products are reduced for a batch at once (reduce-scatter across
//              the lanes; lane j finishes record j).
//
// Scratch (caller-provided workspace, see msda_backward_workspace_size): counts
// per (chunk, cell), per-cell totals, scan tile sums, the slot of every point,
// and the sorted records (16 bytes) and keys (4 bytes).
#include <mutex>

#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;                    // points in flight per thread (hist / place)
constexpr int kChunkPoints = 16384;           // points of a segment per hist / place block
constexpr int kHistCells = 16 * 1024;         // shared counters per band (64 KB: 3 blocks / SM)
constexpr int kScanItems = 8;                 // per thread
constexpr int kScanTile = kThreads * kScanItems;
constexpr int kRunRecords = 64;               // records per sub-warp in the cell pass
constexpr int kCellChannels = 4;              // channels per lane in the cell pass

// Cells of level l occupy [base[l], base[l] + count[l]) of a (b, m) block of
// keys, count[l] = (H_l + 1)(W_l + 1).  With consistent metadata the levels fill
// at most 2 S + 2 L keys (the block length); a level that would reach past it
// (possible only when levels overlap in `value`) gets count 0, so its points
// are never binned and no key leaves the array.
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

// Exact floor(n / d) for 0 <= n < 2^31 and 1 <= d < 2^31 with one 64-bit
// multiply: magic = ceil(2^(32+s) / d), s = ceil(log2 d).  The rounding error of
// magic adds less than n / 2^(32+s) < 1 / (2d) to n / d, which never carries past
// the next integer.
struct FastDiv {
  unsigned long long magic;
  int shift;
};

FastDiv make_fastdiv(long long d) {
  FastDiv f;
  int s = 0;
  while ((1ll << s) < d) ++s;
  f.shift = 32 + s;
  f.magic = ((1ull << f.shift) + static_cast<unsigned long long>(d) - 1) /
            static_cast<unsigned long long>(d);
  return f;
}

__device__ __forceinline__ int fast_div(int n, const FastDiv& f) {
  return static_cast<int>((static_cast<unsigned long long>(n) * f.magic) >> f.shift);
}

// Segment seg = (b * M + m) * L + l; its point i = q * K + k is sampling point
// p = ((b * Lq + q) * M + m) * L * K + l * K + k.
struct Segment {
  long long b;
  int m, l;
  long long p_base;  // p of point 0
  long long p_q;     // p stride between queries: M * L * K
};

__device__ __forceinline__ Segment segment_of(long long seg, int M, int L, int K, long long Lq) {
  Segment s;
  s.l = static_cast<int>(seg % L);
  const long long bm = seg / L;
  s.m = static_cast<int>(bm % M);
  s.b = bm / M;
  s.p_q = static_cast<long long>(M) * L * K;
  s.p_base = (s.b * Lq * M + s.m) * static_cast<long long>(L) * K + static_cast<long long>(s.l) * K;
  return s;
}

// The cell of one point, or -1 when none of its corners is in the map.
__device__ __forceinline__ int point_cell(const Cell& c, int W) {
  return ((c.vx0 || c.vx1) && (c.vy0 || c.vy1)) ? (c.y0 + 1) * (W + 1) + (c.x0 + 1) : -1;
}

// The gradients of the points with no corner in the map, which take no part in
// the sort.  Every corner sum of such a point is sum_d gO[d] * 0: 0, or NaN when
// the group's grad_output holds an Inf or NaN.  The products with the weights
// keep the NaN of a non-finite location, as the oracle does.  Two streaming
// passes, each with its loads issued ahead of their use:
//   no_corner_kernel         the location-only gradients of every such point
//                            (reads all locations and weights);
//   nonfinite_output_kernel  reads grad_output once; a (rare) group whose row
//                            holds an Inf or NaN makes its no-corner points' gradients NaN.
// I: the point index type (32-bit when the points fit).
constexpr int kNoCornerUnroll = 4;

template <typename I>
__global__ void __launch_bounds__(kThreads)
no_corner_kernel(const int64_t* __restrict__ spatial_shapes, const int64_t* __restrict__ level_start,
                 const float* __restrict__ sampling_locations,
                 const float* __restrict__ attention_weights, float* __restrict__ grad_loc,
                 float* __restrict__ grad_attn, long long S, int L, int K, I points) {
  constexpr int U = kNoCornerUnroll;
  __shared__ Levels lv;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  const I step = static_cast<I>(gridDim.x) * kThreads * U;
  for (I p0 = static_cast<I>(blockIdx.x) * kThreads * U + threadIdx.x; p0 < points; p0 += step) {
    float2 xy[U];
    float a[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I p = p0 + static_cast<I>(u) * kThreads;
      if (p < points) {
        xy[u] = __ldcs(reinterpret_cast<const float2*>(sampling_locations) + p);
        a[u] = __ldcs(attention_weights + p);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I p = p0 + static_cast<I>(u) * kThreads;
      if (p >= points) continue;
      const int l = static_cast<int>((p / static_cast<I>(K)) % static_cast<I>(L));
      const int H = lv.H[l], W = lv.W[l];
      const Cell c = locate(xy[u].x, xy[u].y, H, W);
      if (point_cell(c, W) >= 0) continue;
      grad_attn[p] = 0.0f * (c.fx + c.fy);
      reinterpret_cast<float2*>(grad_loc)[p] =
          make_float2(a[u] * static_cast<float>(W) * (0.0f * c.fy),
                      a[u] * static_cast<float>(H) * (0.0f * c.fx));
    }
  }
}

template <typename I>
__global__ void __launch_bounds__(kThreads)
nonfinite_output_kernel(const int64_t* __restrict__ spatial_shapes,
                        const int64_t* __restrict__ level_start,
                        const float* __restrict__ sampling_locations,
                        const float* __restrict__ grad_output, float* __restrict__ grad_loc,
                        float* __restrict__ grad_attn, long long S, int D, int L, int K, I n4) {
  constexpr int U = kNoCornerUnroll;
  __shared__ Levels lv;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  // 16-byte loads: D % 4 == 0 and grad_output is 16-byte aligned.
  const float4* go = reinterpret_cast<const float4*>(grad_output);
  const I step = static_cast<I>(gridDim.x) * kThreads * U;
  for (I i0 = static_cast<I>(blockIdx.x) * kThreads * U + threadIdx.x; i0 < n4; i0 += step) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I i = i0 + static_cast<I>(u) * kThreads;
      if (i < n4) v[u] = __ldcs(go + i);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const I i = i0 + static_cast<I>(u) * kThreads;
      if (i >= n4) continue;
      const float t = (0.0f * v[u].x + 0.0f * v[u].y) + (0.0f * v[u].z + 0.0f * v[u].w);
      if (t == t) continue;
      // This group's grad_output holds an Inf or NaN: its points with no corner
      // in the map get NaN (other threads of the group may write the same NaNs).
      const I g = i / static_cast<I>(D / 4);
      const int LK = L * K;
      const float nan = __int_as_float(0x7fffffff);
      for (int j = 0; j < LK; ++j) {
        const I p = g * static_cast<I>(LK) + static_cast<I>(j);
        const int l = j / K;
        const float2 xy = __ldg(reinterpret_cast<const float2*>(sampling_locations) + p);
        const Cell c = locate(xy.x, xy.y, lv.H[l], lv.W[l]);
        if (point_cell(c, lv.W[l]) >= 0) continue;
        grad_attn[p] = nan;
        reinterpret_cast<float2*>(grad_loc)[p] = make_float2(nan, nan);
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads)
hist_kernel(const int64_t* __restrict__ spatial_shapes, const int64_t* __restrict__ level_start,
            const float* __restrict__ sampling_locations,
            int* __restrict__ counts, int* __restrict__ slots, long long S, int M, long long Lq,
            int L, int K, long long cells_per_bm, int chunks, long long keys) {
  extern __shared__ int hist[];
  __shared__ Levels lv;
  __shared__ CellLevels cl;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  stage_cells(cl, lv, L, cells_per_bm);
  const long long seg = blockIdx.x / chunks;
  const int chunk = static_cast<int>(blockIdx.x - seg * chunks);
  const Segment sg = segment_of(seg, M, L, K, Lq);
  const int H = lv.H[sg.l], W = lv.W[sg.l];
  const int ncells = cl.count[sg.l];
  const long long seg_len = Lq * K;
  const long long i_begin = static_cast<long long>(chunk) * kChunkPoints;
  const long long i_end = min(seg_len, i_begin + kChunkPoints);
  // counts index of (chunk, cell): chunk * keys + key.
  const long long key0 = (sg.b * M + sg.m) * cells_per_bm + cl.base[sg.l];

  int lo = 0;
  do {
    const int span = min(kHistCells, ncells - lo);
    for (int c = threadIdx.x; c < span; c += kThreads) hist[c] = 0;
    __syncthreads();
    for (long long i0 = i_begin + threadIdx.x; i0 < i_end; i0 += kThreads * kUnroll) {
      float2 xy[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const long long i = i0 + u * kThreads;
        if (i < i_end) {
          const long long q = i / K;
          xy[u] = __ldcs(reinterpret_cast<const float2*>(sampling_locations) + sg.p_base +
                         q * sg.p_q + (i - q * K));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const long long i = i0 + u * kThreads;
        if (i >= i_end) continue;
        const long long q = i / K;
        const long long p = sg.p_base + q * sg.p_q + (i - q * K);
        const Cell c = locate(xy[u].x, xy[u].y, H, W);
        const int cell = ncells > 0 ? point_cell(c, W) : -1;
        if (cell >= lo && cell < lo + span) {
          __stcs(slots + p, atomicAdd(hist + (cell - lo), 1));
        }
      }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < span; c += kThreads)
      counts[chunk * keys + key0 + lo + c] = hist[c];
    lo += kHistCells;
    __syncthreads();
  } while (lo < ncells);
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
             const int* __restrict__ slots, float4* __restrict__ records,
             int* __restrict__ record_keys, long long S, int M, long long Lq, int L, int K,
             long long cells_per_bm, int chunks, long long keys) {
  extern __shared__ int s_off[];  // this chunk's offsets of the band's cells
  __shared__ Levels lv;
  __shared__ CellLevels cl;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  stage_cells(cl, lv, L, cells_per_bm);
  const long long seg = blockIdx.x / chunks;
  const int chunk = static_cast<int>(blockIdx.x - seg * chunks);
  const Segment sg = segment_of(seg, M, L, K, Lq);
  const int H = lv.H[sg.l], W = lv.W[sg.l];
  const int ncells = cl.count[sg.l];
  if (ncells == 0) return;
  const long long seg_len = Lq * K;
  const long long i_begin = static_cast<long long>(chunk) * kChunkPoints;
  const long long i_end = min(seg_len, i_begin + kChunkPoints);
  const long long key0 = (sg.b * M + sg.m) * cells_per_bm + cl.base[sg.l];
  const int* chunk_offsets = offsets + chunk * keys + key0;
  for (int lo = 0; lo < ncells; lo += kHistCells) {
  const int span = min(kHistCells, ncells - lo);
  for (int c = threadIdx.x; c < span; c += kThreads) s_off[c] = chunk_offsets[lo + c];
  __syncthreads();
  for (long long i0 = i_begin + threadIdx.x; i0 < i_end; i0 += kThreads * kUnroll) {
    float2 xy[kUnroll];
    float a[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = i0 + u * kThreads;
      if (i < i_end) {
        const long long q = i / K;
        const long long p = sg.p_base + q * sg.p_q + (i - q * K);
        // One-touch streams are marked evict-first, so that the randomly read
        // offsets stay in L2.
        xy[u] = __ldcs(reinterpret_cast<const float2*>(sampling_locations) + p);
        a[u] = __ldcs(attention_weights + p);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = i0 + u * kThreads;
      if (i >= i_end) continue;
      const long long q = i / K;
      const long long p = sg.p_base + q * sg.p_q + (i - q * K);
      const Cell c = locate(xy[u].x, xy[u].y, H, W);
      const int cell = point_cell(c, W);
      if (cell < lo || cell >= lo + span) continue;
      const int pos = s_off[cell - lo] + __ldcs(slots + p);
      __stcs(records + pos, make_float4(__int_as_float(static_cast<int>(p)), a[u], c.fx, c.fy));
      __stcs(record_keys + pos, static_cast<int>(key0 + cell));
    }
  }
  __syncthreads();  // s_off is reloaded for the next band
  }
}

// Per-key totals over the chunks of the chunk-major counts[chunk][key].
__global__ void __launch_bounds__(kThreads)
column_totals_kernel(const int* __restrict__ counts, int* __restrict__ totals, long long keys,
                     int chunks) {
  for (long long k = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; k <= keys;
       k += static_cast<long long>(gridDim.x) * kThreads) {
    int s = 0;
    if (k < keys)
      for (int c = 0; c < chunks; ++c) s += counts[c * keys + k];
    totals[k] = s;  // totals[keys] = 0: after the exclusive scan, the record count
  }
}

// counts[chunk][key] -> position of the (key, chunk) run: the key's base (scanned
// totals) plus the counts of the key's earlier chunks.
__global__ void __launch_bounds__(kThreads)
finalize_offsets_kernel(int* __restrict__ counts, const int* __restrict__ bases, long long keys,
                        int chunks) {
  for (long long k = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; k < keys;
       k += static_cast<long long>(gridDim.x) * kThreads) {
    int run = bases[k];
    for (int c = 0; c < chunks; ++c) {
      const int v = counts[c * keys + k];
      counts[c * keys + k] = run;
      run += v;
    }
  }
}

// A lane's CPL consecutive channels of one row (CPL = 4 or 8), moved as float4s;
// `on[h]` tells whether float4 h of the lane lies inside the D channels.
template <int CPL>
struct Row {
  float v[CPL];
};

template <int CPL>
__device__ __forceinline__ Row<CPL> zero_row() {
  Row<CPL> r;
#pragma unroll
  for (int i = 0; i < CPL; ++i) r.v[i] = 0.0f;
  return r;
}

template <int CPL>
__device__ __forceinline__ Row<CPL> load_row(const float* p, const bool (&on)[CPL / 4]) {
  Row<CPL> r = zero_row<CPL>();
#pragma unroll
  for (int h = 0; h < CPL / 4; ++h)
    if (on[h] && in_bounds(p + 4 * h, 16, false)) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(p + 4 * h));
      r.v[4 * h + 0] = x.x;
      r.v[4 * h + 1] = x.y;
      r.v[4 * h + 2] = x.z;
      r.v[4 * h + 3] = x.w;
    }
  return r;
}

template <int CPL>
__device__ __forceinline__ void red_row(float* p, const Row<CPL>& r, const bool (&on)[CPL / 4]) {
#pragma unroll
  for (int h = 0; h < CPL / 4; ++h)
    if (on[h] && in_bounds(p + 4 * h, 16, true))
      atomicAdd(reinterpret_cast<float4*>(p + 4 * h),
                make_float4(r.v[4 * h], r.v[4 * h + 1], r.v[4 * h + 2], r.v[4 * h + 3]));
}

// The four corner sums of a record over this lane's channels, with the corner
// differences taken per channel before any sum (a common offset of the value
// field cancels exactly, and an infinite grad_output channel meets one
// difference, as in the pages' per-channel product):
//   P = sum gO V00, Ex = sum gO (V10 - V00), Ey = sum gO (V01 - V00),
//   Exy = sum gO ((V11 - V01) - (V10 - V00)).
template <int CPL>
__device__ __forceinline__ void corner_sums(const Row<CPL>& go, const Row<CPL>& c00,
                                            const Row<CPL>& c10, const Row<CPL>& c01,
                                            const Row<CPL>& c11, float (&s)[4]) {
  s[0] = s[1] = s[2] = s[3] = 0.0f;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    const float dx = c10.v[i] - c00.v[i];
    const float dy = c01.v[i] - c00.v[i];
    const float dxy = (c11.v[i] - c01.v[i]) - dx;
    s[0] = fmaf(go.v[i], c00.v[i], s[0]);
    s[1] = fmaf(go.v[i], dx, s[1]);
    s[2] = fmaf(go.v[i], dy, s[2]);
    s[3] = fmaf(go.v[i], dxy, s[3]);
  }
}

template <int CPL>
__device__ __forceinline__ void axpy_row(float w, const Row<CPL>& x, Row<CPL>& y) {
#pragma unroll
  for (int i = 0; i < CPL; ++i) y.v[i] = fmaf(w, x.v[i], y.v[i]);
}

// The geometry of the cell behind a key, with this lane's value / grad_value
// row offset of pixel (x0, y0) and the element strides to its neighbours.
struct CellGeom {
  int m, W, H, x0;
  bool vx0, vx1, vy0, vy1;
  long long ofs;  // ((b * S + start + y0 * W + x0) * M + m) * D + ch
  long long dy;   // W * M * D
};

// The divisions by cells_per_bm and M use precomputed magic numbers.
struct KeyDiv {
  FastDiv per_cells;  // key -> b * M + m
  FastDiv per_m;      // b * M + m -> b
  int cells_per_bm;
};

__device__ __forceinline__ int key_head(int key, const KeyDiv& kd, int M) {
  const int bm = fast_div(key, kd.per_cells);
  return bm - fast_div(bm, kd.per_m) * M;
}

__device__ __forceinline__ CellGeom decode_key(int key, const KeyDiv& kd, int M, int L,
                                               long long S, int D, int ch, const Levels& lv,
                                               const CellLevels& cl) {
  CellGeom g;
  const int bm = fast_div(key, kd.per_cells);
  const int within = key - bm * kd.cells_per_bm;
  const int b = fast_div(bm, kd.per_m);
  g.m = bm - b * M;
  int l = 0;
  while (l + 1 < L && !(within >= cl.base[l] && within < cl.base[l] + cl.count[l])) ++l;
  g.W = lv.W[l];
  g.H = lv.H[l];
  const int cell = within - cl.base[l];
  const int y0 = cell / (g.W + 1) - 1;
  g.x0 = cell - (y0 + 1) * (g.W + 1) - 1;
  g.vx0 = g.x0 >= 0;
  g.vx1 = g.x0 + 1 < g.W;
  g.vy0 = y0 >= 0;
  g.vy1 = y0 + 1 < g.H;
  const long long MD = static_cast<long long>(M) * D;
  const long long pix = lv.start[l] + static_cast<long long>(y0) * g.W + g.x0;
  g.ofs = (static_cast<long long>(b) * S + pix) * MD + static_cast<long long>(g.m) * D + ch;
  g.dy = g.W * MD;
  return g;
}

// Cell pass.  LANES lanes per sub-warp, CPL channels per lane (D <= CPL * LANES);
// records are reduced NB = min(LANES, 4) at a time.
template <int LANES, int CPL>
__global__ void __launch_bounds__(kThreads)
cell_kernel(const float* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
            const int64_t* __restrict__ level_start, const float* __restrict__ grad_output,
            const int* __restrict__ total_records, const float4* __restrict__ records,
            const int* __restrict__ record_keys, float* __restrict__ grad_value,
            float* __restrict__ grad_loc, float* __restrict__ grad_attn, long long S, int M,
            int D, int L, long long cells_per_bm, KeyDiv kd, FastDiv per_bq) {
  constexpr int NB = LANES < 4 ? LANES : 4;
  using R = Row<CPL>;
  __shared__ Levels lv;
  __shared__ CellLevels cl;
  stage_levels(lv, spatial_shapes, level_start, L, S);
  stage_cells(cl, lv, L, cells_per_bm);

  const int lane = threadIdx.x % LANES;
  // Sub-warps follow their own runs, so their shuffles name only their lanes.
  const unsigned mask =
      LANES == 32 ? kFullMask
                  : ((1u << (LANES & 31)) - 1u) << ((threadIdx.x & 31) & ~(LANES - 1));
  const long long run = (blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x) / LANES;
  const int total = *total_records;
  if (run * kRunRecords >= total) return;
  const int r0 = static_cast<int>(run * kRunRecords);
  const int r1 = min(r0 + kRunRecords, total);
  const int ch = lane * CPL;
  bool on[CPL / 4];
#pragma unroll
  for (int h = 0; h < CPL / 4; ++h) on[h] = ch + 4 * h < D;
  const long long MD = static_cast<long long>(M) * D;

  // The current cell (key cur): corner rows cIJ = V(x0 + I, y0 + J) of value and
  // the grad_value accumulators aIJ of the same corners.
  int cur = -1;
  CellGeom g{};
  R c00 = zero_row<CPL>(), c10 = zero_row<CPL>(), c01 = zero_row<CPL>(), c11 = zero_row<CPL>();
  R a00 = zero_row<CPL>(), a10 = zero_row<CPL>(), a01 = zero_row<CPL>(), a11 = zero_row<CPL>();
  auto flush = [&](bool keep_right) {
    float* gv = grad_value + g.ofs;
    if (g.vx0 && g.vy0) red_row(gv, a00, on);
    if (g.vx0 && g.vy1) red_row(gv + g.dy, a01, on);
    if (!keep_right) {
      if (g.vx1 && g.vy0) red_row(gv + MD, a10, on);
      if (g.vx1 && g.vy1) red_row(gv + g.dy + MD, a11, on);
    }
  };
  auto enter = [&](int key) {
    const CellGeom ng = decode_key(key, kd, M, L, S, D, ch, lv, cl);
    // Moving right along a row keeps the shared column: values and sums.
    const bool right = cur >= 0 && key == cur + 1 && ng.x0 >= 0;
    if (cur >= 0) flush(right);
    if (right) {
      c00 = c10;
      c01 = c11;
      a00 = a10;
      a01 = a11;
    } else {
      c00 = (ng.vx0 && ng.vy0) ? load_row<CPL>(value + ng.ofs, on) : zero_row<CPL>();
      c01 = (ng.vx0 && ng.vy1) ? load_row<CPL>(value + ng.ofs + ng.dy, on) : zero_row<CPL>();
      a00 = zero_row<CPL>();
      a01 = zero_row<CPL>();
    }
    c10 = (ng.vx1 && ng.vy0) ? load_row<CPL>(value + ng.ofs + MD, on) : zero_row<CPL>();
    c11 = (ng.vx1 && ng.vy1) ? load_row<CPL>(value + ng.ofs + ng.dy + MD, on) : zero_row<CPL>();
    a10 = zero_row<CPL>();
    a11 = zero_row<CPL>();
    // Records come in row order: the next cell is most often the right
    // neighbour, whose new column is prefetched into L1 now.
    if (ng.x0 + 2 < ng.W && on[0]) {
      const float* nx = value + ng.ofs + 2 * MD;
      if (ng.vy0) asm volatile("prefetch.global.L1 [%0];" ::"l"(nx));
      if (ng.vy1) asm volatile("prefetch.global.L1 [%0];" ::"l"(nx + ng.dy));
    }
    g = ng;
    cur = key;
  };

  // Software pipeline: the records of batch b + 1 sit in registers and their
  // grad_output slices are being copied (cp.async) into shared memory while
  // batch b is computed.  Each lane copies exactly the 16-byte slices it later
  // reads, so the copies need no barrier, only the lane's own wait.
  __shared__ float4 ring[2][NB][CPL / 4][kThreads];
  const int nb = (r1 - r0 + NB - 1) / NB;
  auto load_batch = [&](int bb, float4& rec, int& key) {
    rec = make_float4(__int_as_float(-1), 0.0f, 0.0f, 0.0f);
    key = -1;
    const int i = r0 + bb * NB + lane;
    if (lane < NB && bb < nb && i < r1) {
      key = __ldcs(record_keys + i);
      rec = __ldcs(records + i);
    }
  };
  auto issue_go = [&](const float4& rec, int key, int stage) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int kj = __shfl_sync(mask, key, j, LANES);
      const int pj = __float_as_int(__shfl_sync(mask, rec.x, j, LANES));
      if (kj >= 0) {
        const int bq = fast_div(pj, per_bq);
        const int m = key_head(kj, kd, M);
        const float* src = grad_output + static_cast<long long>(bq) * MD +
                           static_cast<long long>(m) * D + ch;
#pragma unroll
        for (int h = 0; h < CPL / 4; ++h)
          if (on[h]) {
            if (!in_bounds(src + 4 * h, 16, false)) {  // debug build only: a zero slice
              ring[stage][j][h][threadIdx.x] = make_float4(0.f, 0.f, 0.f, 0.f);
              continue;
            }
            const unsigned dst =
                static_cast<unsigned>(__cvta_generic_to_shared(&ring[stage][j][h][threadIdx.x]));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src + 4 * h)
                         : "memory");
          }
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float4 rec_cur, rec_nxt, rec_nn;
  int key_cur, key_nxt, key_nn;
  load_batch(0, rec_cur, key_cur);
  issue_go(rec_cur, key_cur, 0);
  load_batch(1, rec_nxt, key_nxt);
  for (int b = 0; b < nb; ++b) {
    const int stage = b & 1;
    issue_go(rec_nxt, key_nxt, stage ^ 1);  // batch b + 1
    load_batch(b + 2, rec_nn, key_nn);
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // batch b's slices are in

    float part[4][NB];
    float myW = 0.0f, myH = 0.0f;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int kj = __shfl_sync(mask, key_cur, j, LANES);
      const float a = __shfl_sync(mask, rec_cur.y, j, LANES);
      const float fx = __shfl_sync(mask, rec_cur.z, j, LANES);
      const float fy = __shfl_sync(mask, rec_cur.w, j, LANES);
      part[0][j] = part[1][j] = part[2][j] = part[3][j] = 0.0f;
      if (kj < 0) continue;  // past the end of the run (uniform in the sub-warp)
      if (kj != cur) enter(kj);
      if (lane == j) {
        myW = static_cast<float>(g.W);
        myH = static_cast<float>(g.H);
      }
      R go = zero_row<CPL>();
#pragma unroll
      for (int h = 0; h < CPL / 4; ++h)
        if (on[h]) {
          const float4 x = ring[stage][j][h][threadIdx.x];
          go.v[4 * h + 0] = x.x;
          go.v[4 * h + 1] = x.y;
          go.v[4 * h + 2] = x.z;
          go.v[4 * h + 3] = x.w;
        }
      float cs[4];
      corner_sums(go, c00, c10, c01, c11, cs);
      part[0][j] = cs[0];
      part[1][j] = cs[1];
      part[2][j] = cs[2];
      part[3][j] = cs[3];
      const float hx = 1.0f - fx, hy = 1.0f - fy;
      axpy_row(a * hx * hy, go, a00);
      axpy_row(a * fx * hy, go, a10);
      axpy_row(a * hx * fy, go, a01);
      axpy_row(a * fx * fy, go, a11);
    }
    // Butterfly over the lane bits above the batch, then a reduce-scatter so that
    // lane j (< NB) ends with the totals of record j.
#pragma unroll
    for (int o = LANES / 2; o >= NB; o >>= 1)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < NB; ++j) part[q][j] += __shfl_xor_sync(mask, part[q][j], o, LANES);
#pragma unroll
    for (int o = NB / 2; o >= 1; o >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < o; ++j) {
          // Keep the indices whose bit o matches this lane's; send the others.
          const float send = upper ? part[q][j] : part[q][j + o];
          const float keep = upper ? part[q][j + o] : part[q][j];
          part[q][j] = keep + __shfl_xor_sync(mask, send, o, LANES);
        }
    }
    if (lane < NB && key_cur >= 0) {
      const int p = __float_as_int(rec_cur.x);
      const float a = rec_cur.y, fx = rec_cur.z, fy = rec_cur.w;
      const float P = part[0][0], Ex = part[1][0], Ey = part[2][0], Exy = part[3][0];
      // The derivatives regrouped with hx + fx = hy + fy = 1.
      grad_attn[p] = fmaf(fx, fmaf(fy, Exy, Ex), fmaf(fy, Ey, P));
      reinterpret_cast<float2*>(grad_loc)[p] =
          make_float2(a * myW * fmaf(fy, Exy, Ex), a * myH * fmaf(fx, Exy, Ey));
    }
    rec_cur = rec_nxt;
    key_cur = key_nxt;
    rec_nxt = rec_nn;
    key_nxt = key_nn;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (cur >= 0) flush(false);
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

template <int LANES, int CPL>
cudaError_t launch_cells(const BackwardArgs& a, const SortedLayout& w, const int* total,
                         const float4* records, const int* record_keys, cudaStream_t stream) {
  const long long runs = (w.points + kRunRecords - 1) / kRunRecords;
  const FastDiv per_bq = make_fastdiv(static_cast<long long>(a.M) * a.L * a.K);
  KeyDiv kd;
  kd.per_cells = make_fastdiv(w.cells_per_bm);
  kd.per_m = make_fastdiv(a.M);
  kd.cells_per_bm = static_cast<int>(w.cells_per_bm);
  cell_kernel<LANES, CPL><<<grid_for(runs * LANES, kThreads), kThreads, 0, stream>>>(
      static_cast<const float*>(a.value), a.spatial_shapes, a.level_start_index,
      static_cast<const float*>(a.grad_output), total, records, record_keys,
      a.grad_value, a.grad_sampling_locations, a.grad_attention_weights, a.S, a.M, a.D, a.L,
      w.cells_per_bm, kd, per_bq);
  return cudaGetLastError();
}

}  // namespace

SortedLayout sorted_layout(long long B, long long S, long long M, long long Lq, int L, int K) {
  SortedLayout w;
  // sum_l (H_l + 1)(W_l + 1) <= 2 S + 2 L, because H + W <= H W + 1 for H, W >= 1.
  w.cells_per_bm = 2 * S + 2 * L;
  w.keys = B * M * w.cells_per_bm;
  w.segments = B * M * L;
  w.segment_len = Lq * K;
  w.chunks = (w.segment_len + kChunkPoints - 1) / kChunkPoints;
  if (w.chunks < 1) w.chunks = 1;
  w.points = w.segments * w.segment_len;
  w.counts = w.keys * w.chunks;
  w.scan_tiles = (w.keys + 1 + kScanTile - 1) / kScanTile;
  auto up = [](long long bytes) { return (bytes + 255) / 256 * 256; };
  w.bytes = up(4 * w.counts) + up(4 * (w.keys + 1)) + up(4 * w.scan_tiles) + up(4 * w.points) +
            up(16 * w.points) + up(4 * w.points);
  return w;
}

cudaError_t launch_backward_sorted(const BackwardArgs& a, void* workspace,
                                   cudaStream_t stream) {
  const SortedLayout w = sorted_layout(a.B, a.S, a.M, a.Lq, a.L, a.K);
  char* cursor = static_cast<char*>(workspace);
  int* counts = carve<int>(cursor, w.counts);      // counts[chunk][key], then run offsets
  int* totals = carve<int>(cursor, w.keys + 1);    // per-key totals, then key bases
  int* tile_sums = carve<int>(cursor, w.scan_tiles);
  int* slots = carve<int>(cursor, w.points);
  float4* records = carve<float4>(cursor, w.points);
  int* record_keys = carve<int>(cursor, w.points);

  cudaError_t err = launch_zero(a.grad_value, a.value_elements, stream);
  if (err != cudaSuccess || w.points == 0) return err;
  // Counts of keys that no block writes (keys past a segment's levels) stay 0;
  // the zero fill covers whole float4s, which the 256-byte carve leaves room for.
  if ((err = launch_zero(reinterpret_cast<float*>(counts), (w.counts + 3) / 4 * 4, stream)) !=
      cudaSuccess)
    return err;

  // The hist and place kernels' per-cell tables exceed the default 48 KB of
  // dynamic shared memory; the opt-in is set once per device.
  const size_t cell_smem = sizeof(int) * static_cast<size_t>(kHistCells);
  static std::mutex smem_mu;
  static bool smem_set[64] = {};
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  {
    std::lock_guard<std::mutex> lock(smem_mu);
    if (dev < 0 || dev >= 64 || !smem_set[dev]) {
      if ((err = cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(cell_smem))) != cudaSuccess ||
          (err = cudaFuncSetAttribute(place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(cell_smem))) != cudaSuccess)
        return err;
      if (dev >= 0 && dev < 64) smem_set[dev] = true;
    }
  }
  const unsigned blocks = static_cast<unsigned>(w.segments * w.chunks);
  const int chunks = static_cast<int>(w.chunks);
  hist_kernel<<<blocks, kThreads, cell_smem, stream>>>(
      a.spatial_shapes, a.level_start_index, a.sampling_locations, counts, slots, a.S, a.M,
      a.Lq, a.L, a.K, w.cells_per_bm, chunks, w.keys);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  {
    // The points with no corner in the map (see no_corner_kernel); the second
    // launch runs after the first, so its NaNs win.
    const long long points = a.groups * a.L * a.K;
    const long long n4 = a.groups * (a.D / 4);
    const long long per_block = static_cast<long long>(kThreads) * kNoCornerUnroll;
    long long b1 = (points + per_block - 1) / per_block, b2 = (n4 + per_block - 1) / per_block;
    if (b1 > 148 * 16) b1 = 148 * 16;
    if (b2 > 148 * 16) b2 = 148 * 16;
    const bool narrow = points < (1ll << 31) - per_block * 148 * 16 &&
                        n4 < (1ll << 31) - per_block * 148 * 16;
    const float* go = static_cast<const float*>(a.grad_output);
    if (narrow) {
      no_corner_kernel<unsigned><<<static_cast<unsigned>(b1), kThreads, 0, stream>>>(
          a.spatial_shapes, a.level_start_index, a.sampling_locations, a.attention_weights,
          a.grad_sampling_locations, a.grad_attention_weights, a.S, a.L, a.K,
          static_cast<unsigned>(points));
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
      nonfinite_output_kernel<unsigned><<<static_cast<unsigned>(b2), kThreads, 0, stream>>>(
          a.spatial_shapes, a.level_start_index, a.sampling_locations, go,
          a.grad_sampling_locations, a.grad_attention_weights, a.S, a.D, a.L, a.K,
          static_cast<unsigned>(n4));
    } else {
      no_corner_kernel<unsigned long long><<<static_cast<unsigned>(b1), kThreads, 0, stream>>>(
          a.spatial_shapes, a.level_start_index, a.sampling_locations, a.attention_weights,
          a.grad_sampling_locations, a.grad_attention_weights, a.S, a.L, a.K,
          static_cast<unsigned long long>(points));
      if ((err = cudaGetLastError()) != cudaSuccess) return err;
      nonfinite_output_kernel<unsigned long long><<<static_cast<unsigned>(b2), kThreads, 0,
                                                    stream>>>(
          a.spatial_shapes, a.level_start_index, a.sampling_locations, go,
          a.grad_sampling_locations, a.grad_attention_weights, a.S, a.D, a.L, a.K,
          static_cast<unsigned long long>(n4));
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  // Key-major positions from the chunk-major counts: per-key totals, their
  // exclusive scan, then each (key, chunk) run's offset.
  column_totals_kernel<<<grid_for(w.keys + 1, kThreads), kThreads, 0, stream>>>(
      counts, totals, w.keys, chunks);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_tiles_kernel<<<static_cast<unsigned>(w.scan_tiles), kThreads, 0, stream>>>(
      totals, tile_sums, w.keys + 1);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_sums_kernel<<<1, 1024, 0, stream>>>(tile_sums, static_cast<int>(w.scan_tiles));
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scan_add_kernel<<<static_cast<unsigned>(w.scan_tiles), kThreads, 0, stream>>>(
      totals, tile_sums, w.keys + 1);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  finalize_offsets_kernel<<<grid_for(w.keys, kThreads), kThreads, 0, stream>>>(
      counts, totals, w.keys, chunks);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  place_kernel<<<blocks, kThreads, cell_smem, stream>>>(
      a.spatial_shapes, a.level_start_index, a.sampling_locations, a.attention_weights, counts,
      slots, records, record_keys, a.S, a.M, a.Lq, a.L, a.K, w.cells_per_bm, chunks, w.keys);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  // totals[keys] now holds the number of records.
  const int* total = totals + w.keys;
  int lanes = 1;
  while (lanes * kCellChannels < a.D) lanes <<= 1;
  switch (lanes) {
    case 1: return launch_cells<1, kCellChannels>(a, w, total, records, record_keys, stream);
    case 2: return launch_cells<2, kCellChannels>(a, w, total, records, record_keys, stream);
    case 4: return launch_cells<4, kCellChannels>(a, w, total, records, record_keys, stream);
    case 8: return launch_cells<8, kCellChannels>(a, w, total, records, record_keys, stream);
    case 16: return launch_cells<16, kCellChannels>(a, w, total, records, record_keys, stream);
    case 32: return launch_cells<32, kCellChannels>(a, w, total, records, record_keys, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace msda
