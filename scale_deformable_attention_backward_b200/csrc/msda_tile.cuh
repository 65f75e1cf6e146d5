// msda_tile.cuh -- 2-D query tiles for the encoder form of the MSDeformAttn
// core, where the queries are the value's own pixels (sm_100a).
//
// In the encoder every token of every level is a query whose reference point
// is its own pixel centre ("Deformable DETR" blog notes on juhe.plus,
// 重点知识1, get_reference_points), and its samples lie a few pixels around
// that centre on every level ("Deformable DETR Deformable Transformers for
// End-to-End Object Detection", 核心洞察 2).  A rectangle of neighbouring queries
// therefore samples one compact window per level.  The tiled kernels give one
// CTA such a rectangle (of one image b and one head m) and stage its windows in
// shared memory.  Nothing here assumes the locality for correctness: the
// windows are the bounding boxes of the points actually sampled, and a step
// whose box does not fit reads value from global memory instead.
#pragma once

#include "msda_device.cuh"

namespace msda {

// The tiling of the queries of one (b, m), built once per CTA in shared memory.
//   two_d == 1  the queries are the value's pixels: Lq == S, every level is
//               valid and level_start_index is the exclusive prefix sum of H*W.
//               Level l's H x W queries are cut into nty x ntx rectangles of at
//               most TH x TW, rows and columns split as evenly as possible: with
//               H = qy * nty + ry, tile rows 0 .. ry-1 get qy + 1 rows and the
//               others qy (likewise for columns).
//   two_d == 0  anything else: tiles are runs of Q consecutive queries.
struct TileGrid {
  int two_d;
  int nty[kMaxLevels];
  int ntx[kMaxLevels];
  int qy[kMaxLevels], ry[kMaxLevels];  // H = qy * nty + ry
  int qx[kMaxLevels], rx[kMaxLevels];  // W = qx * ntx + rx
  int first[kMaxLevels + 1];  // tiles before level l (two_d)
  int tiles;                  // tiles per (b, m); Lq < 2^31 is required by the caller
};

// The queries of one tile: query(i) = base + (i / width) * pitch + i % width.
struct TileQueries {
  int base;
  int pitch;
  int width;
  int count;
  __device__ __forceinline__ int query(int i) const {
    const int r = i / width;
    return base + r * pitch + (i - r * width);
  }
};

__device__ __forceinline__ void build_tile_grid(TileGrid& tg, const Levels& lv, int L,
                                                long long S, long long Lq, int TH, int TW,
                                                int Q) {
  if (threadIdx.x == 0) {
    bool ok = Lq == S;
    long long total = 0;
    for (int l = 0; l < L; ++l) {
      ok = ok && lv.W[l] > 0 && lv.start[l] == total;
      total += static_cast<long long>(lv.H[l]) * lv.W[l];
    }
    ok = ok && total == Lq;
    int tiles = 0;
    if (ok) {
      for (int l = 0; l < L; ++l) {
        tg.first[l] = tiles;
        tg.nty[l] = (lv.H[l] + TH - 1) / TH;
        tg.ntx[l] = (lv.W[l] + TW - 1) / TW;
        tg.qy[l] = lv.H[l] / tg.nty[l];
        tg.ry[l] = lv.H[l] - tg.qy[l] * tg.nty[l];
        tg.qx[l] = lv.W[l] / tg.ntx[l];
        tg.rx[l] = lv.W[l] - tg.qx[l] * tg.ntx[l];
        tiles += tg.nty[l] * tg.ntx[l];
      }
      tg.first[L] = tiles;
    } else {
      tiles = static_cast<int>((Lq + Q - 1) / Q);
    }
    tg.two_d = ok ? 1 : 0;
    tg.tiles = tiles;
  }
  __syncthreads();
}

__device__ __forceinline__ TileQueries tile_queries(const TileGrid& tg, const Levels& lv, int L,
                                                    int t, int Q, long long Lq) {
  TileQueries r;
  if (tg.two_d) {
    int l = 0;
    while (l + 1 < L && t >= tg.first[l + 1]) ++l;
    const int u = t - tg.first[l];
    const int nx = tg.ntx[l];
    const int ty = u / nx, tx = u - ty * nx;
    const int W = lv.W[l];
    const int r0 = ty * tg.qy[l] + min(ty, tg.ry[l]);
    const int h = tg.qy[l] + (ty < tg.ry[l] ? 1 : 0);
    const int c0 = tx * tg.qx[l] + min(tx, tg.rx[l]);
    const int w = tg.qx[l] + (tx < tg.rx[l] ? 1 : 0);
    // start + r * W + c < start + H * W <= Lq < 2^31.
    r.base = static_cast<int>(lv.start[l]) + r0 * W + c0;
    r.pitch = W;
    r.width = w;
    r.count = h * w;
  } else {
    r.base = t * Q;
    r.pitch = Q;
    r.width = Q;
    r.count = static_cast<int>(min(static_cast<long long>(Q), Lq - static_cast<long long>(t) * Q));
  }
  return r;
}

// One step of a tiled kernel: sampled level l of tile t for image b, head m.
// Items (t, b, m) are dealt to the persistent CTAs round-robin, heads fastest
// (the heads of one query share its rows of locations, weights and output);
// each item is L consecutive steps.
struct TileStep {
  int live;
  int b, m, l;
  TileQueries tq;
};

__device__ __forceinline__ TileStep tile_step(const TileGrid& tg, const Levels& lv, int s, int B,
                                              int M, int L, int Q, long long Lq) {
  TileStep st;
  const int item_round = s / L;
  st.l = s - item_round * L;
  const long long item = blockIdx.x + static_cast<long long>(item_round) * gridDim.x;
  const long long items = static_cast<long long>(tg.tiles) * B * M;
  st.live = item < items;
  const int it = st.live ? static_cast<int>(item) : 0;
  st.m = it % M;
  const int rest = it / M;
  st.b = rest % B;
  st.tq = tile_queries(tg, lv, L, st.live ? rest / B : 0, Q, Lq);
  return st;
}

__device__ __forceinline__ unsigned smem_addr(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async_16(unsigned dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// The in-map corner box of one point's cell, for the window bounds; an empty
// box (lo > hi) when no corner is inside the map.
struct Box {
  int xlo, xhi, ylo, yhi;
};

__device__ __forceinline__ Box corner_box(const Cell& c) {
  Box b;
  const bool any = (c.vx0 || c.vx1) && (c.vy0 || c.vy1);
  b.xlo = any ? (c.vx0 ? c.x0 : c.x0 + 1) : INT_MAX;
  b.xhi = any ? (c.vx1 ? c.x0 + 1 : c.x0) : INT_MIN;
  b.ylo = any ? (c.vy0 ? c.y0 : c.y0 + 1) : INT_MAX;
  b.yhi = any ? (c.vy1 ? c.y0 + 1 : c.y0) : INT_MIN;
  return b;
}

// A step's value window: pixels [x0, x0 + w) x [y0, y0 + h) of its level, all
// inside the map, staged row-major (one row of `row_bytes` per pixel) when
// w * h fits the buffer.
struct Window {
  int x0, y0, w, h;
  bool staged;
};

// Reduces the CTA's corner boxes: each warp's lane 0 writes its warp's box to
// part[warp] (min of xlo, -xhi, ylo, -yhi); after a barrier window_of() merges
// the warps' boxes.
__device__ __forceinline__ void reduce_box_warp(Box b, int4* part) {
  const int a = __reduce_min_sync(kFullMask, b.xlo);
  const int c = __reduce_min_sync(kFullMask, b.xhi == INT_MIN ? INT_MAX : -b.xhi);
  const int d = __reduce_min_sync(kFullMask, b.ylo);
  const int e = __reduce_min_sync(kFullMask, b.yhi == INT_MIN ? INT_MAX : -b.yhi);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = make_int4(a, c, d, e);
}

__device__ __forceinline__ Window window_of(const int4* part, int warps, int capacity) {
  int4 m = part[0];
  for (int w = 1; w < warps; ++w) {
    const int4 p = part[w];
    m.x = min(m.x, p.x);
    m.y = min(m.y, p.y);
    m.z = min(m.z, p.z);
    m.w = min(m.w, p.w);
  }
  Window win;
  if (m.x == INT_MAX) {  // no corner of the step is inside the map
    win.x0 = win.y0 = win.w = win.h = 0;
    win.staged = true;
    return win;
  }
  win.x0 = m.x;
  win.y0 = m.z;
  win.w = -m.y - m.x + 1;
  win.h = -m.w - m.z + 1;
  win.staged = static_cast<long long>(win.w) * win.h <= capacity;
  return win;
}

}  // namespace msda
