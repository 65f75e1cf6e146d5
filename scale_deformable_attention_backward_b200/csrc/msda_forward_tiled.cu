// msda_forward_tiled.cu -- forward of the MSDeformAttn core for the encoder
// form, in which the queries are the value's own pixels (sm_100a).
//
//   out[b, q, m*D + d] = sum_{l,k} A[b,q,m,l,k] * bilinear(value_l[b, :, m, d], loc[b,q,m,l,k])
//
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation; sampling rule and output layout of
// "Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch.
//
// Why a second forward kernel.  The per-point gather (msda_forward.cu) fetches
// every corner of every point as its own 128-byte line; on the encoder most of
// those lines come from L2, and the kernel runs at the rate at which an SM can
// receive random L2 lines.  Encoder queries sample a few pixels around their own
// pixel centre on every level (msda_tile.cuh), so the points of a rectangle of
// neighbouring queries of one head fall into one small window per level.  Here
// a CTA stages that window in shared memory once and gathers the corners from
// there: each value line crosses from L2 about four times per tile (the
// window's margin) instead of once per corner that reads it.
//
// Work decomposition.  One persistent CTA per SM, warp-specialised: 4
// producer warps and 8 consumer warps around a ring of two shared-memory slots
// (records + value window), synchronised by mbarriers only.  Items are (tile
// of <= TH x TW queries on their own level, b, m); an item is L steps, one per
// sampled level l.
//   producers  per step, map the step's points (queries x K, up to 4 per
//              thread; locations and weights are loaded one step ahead):
//              exact floor, corner validity; reduce the bounding box of all
//              in-map corners -- the window; write one 16-byte record per point
//              (A, fx, fy, and the window pixel of its (x0, y0) corner with the
//              four corners' validity bits); copy the window's pixels (one row
//              of D channels each) into the slot with cp.async, 16 bytes per
//              lane, L2 only.  A window larger than the slot makes the step a
//              "global" step: its records hold value pixel indices and the
//              consumers read value directly.
//   consumers  a sub-warp of LANES lanes owns QPS queries of the tile and keeps
//              their accumulators in registers across the item's steps; each
//              lane holds 16 bytes of the head's channels.  Per point it forms
//              the four weights A * bilinear, reads the four corners from the
//              window and accumulates in float32 with packed two-wide FMAs, in
//              the order level, point, corner -- the per-point gather kernel's
//              order, so both kernels give the same bits.
// A slot's "full" barrier completes when every producer thread has written its
// records and its copies have landed (cp.async arrive-on); its "empty" barrier
// when all consumer warps have read it.  So the copies of step s+1 are in
// flight while step s is gathered, and setup never waits for a gather.
//
// A corner outside the map reads nothing: its load is predicated off and its
// weight multiplies zero, so a non-finite location (NaN weights) still makes
// the output NaN, as grid_sample does, and a finite one adds nothing.
#include <climits>
#include <cstdlib>
#include <cstring>
#include <atomic>

#include "msda_device.cuh"
#include "msda_launch.h"
#include "msda_sync.cuh"
#include "msda_tile.cuh"

namespace msda {

namespace {

constexpr int kProducerWarps = 4;
constexpr int kConsumerWarps = 8;
constexpr int kProducers = 32 * kProducerWarps;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = kProducers + kConsumers;
constexpr int kStages = 2;
constexpr int kMaxTileQueries = 128;
constexpr int kStepPoints = 512;                  // queries x K per step, at most
constexpr int kMaxK = 8;                          // samples per level per query, at most
// The consumers' records (int4 offsets + float4 weights) and per slot the raw points.
constexpr int kRecordBytes = kStepPoints * 32 + kStages * kStepPoints * 16;
constexpr int kMaxDynamicSmem = 227 * 1024 - 1024;  // opt-in limit minus static smem
constexpr int kProducerBarrier = 1;                 // named barrier of the producer warps

// 16 bytes of T, widened to float32.
template <typename T>
struct Lane16;

template <>
struct Lane16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void shared(const char* p, float (&v)[E]) {
    const float4 r = *reinterpret_cast<const float4*>(p);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
  __device__ __forceinline__ static void global(const float* p, float (&v)[E]) {
    const float4 r = in_bounds(p, 16, false) ? __ldg(reinterpret_cast<const float4*>(p))
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
};

template <>
struct Lane16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void widen(uint4 r, float (&v)[E]) {
    const unsigned w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i + 0] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static void shared(const char* p, float (&v)[E]) {
    widen(*reinterpret_cast<const uint4*>(p), v);
  }
  __device__ __forceinline__ static void global(const __nv_bfloat16* p, float (&v)[E]) {
    widen(in_bounds(p, 16, false) ? __ldg(reinterpret_cast<const uint4*>(p))
                                  : make_uint4(0u, 0u, 0u, 0u), v);
  }
};

template <int E>
__device__ __forceinline__ void fma_lane(float2 (&acc)[E / 2], float w, const float (&v)[E]) {
  const float2 ww = make_float2(w, w);
#pragma unroll
  for (int e = 0; e < E / 2; ++e) acc[e] = fma2(ww, make_float2(v[2 * e], v[2 * e + 1]), acc[e]);
}

// What the consumers need to know about the step in a slot.
struct SlotInfo {
  int live;                // 0: no more steps
  int b, m, l;
  int wx0, wy0, ww, wh;    // the window: pixels [wx0, wx0 + ww) x [wy0, wy0 + wh) of level l
  TileQueries tq;
};

// OR of `pred` over the producer warps, which also synchronises them.
__device__ __forceinline__ bool producers_any(bool pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.s32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1 : 0), "r"(kProducerBarrier), "r"(kProducers)
      : "memory");
  return r != 0;
}

}  // namespace

// T: value / output dtype.  LANES: lanes per consumer sub-warp (D * sizeof(T) / 16).
template <typename T, int LANES>
__global__ void __launch_bounds__(kThreads, 1)
forward_tiled_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                     const int64_t* __restrict__ level_start_index,
                     const float* __restrict__ sampling_locations,
                     const float* __restrict__ attention_weights, T* __restrict__ output,
                     int B, long long S, int M, long long Lq, int L, int K, int TH, int TW,
                     int capacity, int* __restrict__ failed) {
  using LV = Lane16<T>;
  constexpr int E = LV::E;
  constexpr int D = LANES * E;
  constexpr int ROW = D * static_cast<int>(sizeof(T));  // bytes of one pixel of one head
  constexpr int CPR = ROW / 16;                           // 16-byte chunks per pixel
  constexpr int NSW = kConsumers / LANES;                 // consumer sub-warps
  constexpr int QPS = kMaxTileQueries / NSW;              // queries per sub-warp
  constexpr int SETUP = (QPS * kMaxK + LANES - 1) / LANES;  // points a lane sets up, at most
  static_assert(CPR >= 1 && 32 % CPR == 0, "a warp copies whole pixels");
  static_assert(QPS >= 1 && QPS * NSW == kMaxTileQueries, "queries split evenly");
  static_assert(NSW % 8 == 0, "the record swizzle needs a multiple of 8 sub-warps");

  // Dynamic shared memory: the consumers' record table; per slot the step's raw
  // points (x, y, A) and a window of `capacity` pixel rows plus one row of zeros
  // (read by corners outside the map).
  extern __shared__ __align__(128) unsigned char smem[];
  int4* s_off = reinterpret_cast<int4*>(smem);                             // [kStepPoints]
  float4* s_w = reinterpret_cast<float4*>(smem + kStepPoints * 16);        // [kStepPoints]
  float4* s_raw = reinterpret_cast<float4*>(smem + 2 * kStepPoints * 16);  // [kStages][kStepPoints]
  unsigned char* s_win = smem + kRecordBytes;
  const int slot_bytes = (capacity + 1) * ROW;
  const int zero_row = capacity * ROW;
  __shared__ Levels lv;
  __shared__ TileGrid tg;
  __shared__ int4 s_box[2][kProducerWarps];
  __shared__ SlotInfo s_info[kStages];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ int stop_flag;
  volatile int* stop = &stop_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], 2 * kProducers);  // a store arrival + a copy arrival per producer
      mbar_init(&empty_bar[i], kConsumerWarps);
    }
    stop_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < kStages * CPR; i += kThreads)
    *reinterpret_cast<float4*>(s_win + (i / CPR) * slot_bytes + zero_row + (i % CPR) * 16) =
        make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  stage_levels(lv, spatial_shapes, level_start_index, L, S);
  const int Q = TH * TW;
  build_tile_grid(tg, lv, L, S, Lq, TH, TW, Q);  // ends with a CTA barrier
  const int LK = L * K;
  const int MD = M * D;

  if (threadIdx.x < kProducers) {
    // ------------------------------------------------------------------ producers
    // Producer thread qi handles query qi of the tile (Q <= 128 = kProducers).
    const int qi = threadIdx.x;
    const int pwarp = qi >> 5;
    const long long items = static_cast<long long>(tg.tiles) * B * M;
    long long item = blockIdx.x;
    int l = 0;
    auto decode = [&](long long it) {
      TileStep st;
      st.live = it < items;
      const int i = st.live ? static_cast<int>(it) : 0;
      st.m = i % M;
      const int rest = i / M;
      st.b = rest % B;
      st.l = 0;
      st.tq = tile_queries(tg, lv, L, rest / B, Q, Lq);
      return st;
    };
    long long qbase = 0;  // index of (b, query, m, level 0, point 0) in [B, Lq, M, L, K]
    auto item_base = [&](const TileStep& st) {
      if (qi < st.tq.count)
        qbase = ((st.b * Lq + st.tq.query(qi)) * M + st.m) * static_cast<long long>(LK);
    };
    float2 pxy[kMaxK];
    float pa[kMaxK];
    auto prefetch = [&](const TileStep& st, int lvl) {
      if (qi < st.tq.count) {
        const long long idx = qbase + lvl * K;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
          if (k < K) {
            pxy[k] = __ldg(reinterpret_cast<const float2*>(sampling_locations) + idx + k);
            pa[k] = __ldg(attention_weights + idx + k);
          }
        }
      }
    };
    TileStep cur = decode(item);
    if (cur.live) {
      item_base(cur);
      prefetch(cur, 0);
    }

    for (int s = 0;; ++s) {
      const int slot = s % kStages;
      const unsigned use = static_cast<unsigned>(s / kStages);
      if (!cur.live) {
        // End marker: the slot completes with live = 0 and no copies.
        const bool ok =
            s < kStages || wait_bounded(&empty_bar[slot], (use - 1) & 1u, stop, failed);
        if (producers_any(!ok)) break;
        if (qi == 0) s_info[slot].live = 0;
        mbar_arrive(&full_bar[slot]);
        mbar_arrive_cp_async(&full_bar[slot]);
        break;
      }
      // The window: the box of the cells of the points that may have a corner in
      // the map, from the pixel coordinates rounded once.  Consumers check each
      // point's exact cell against it, so it only has to be good, not exact.
      const int H = lv.H[l], W = lv.W[l];
      const long long start = lv.start[l];
      const float fw = static_cast<float>(W), fh = static_cast<float>(H);
      Box box{INT_MAX, INT_MIN, INT_MAX, INT_MIN};
      if (qi < cur.tq.count) {
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
          if (k < K) {
            const float x = fmaf(pxy[k].x, fw, -0.5f), y = fmaf(pxy[k].y, fh, -0.5f);
            if (x > -1.0f && x < fw && y > -1.0f && y < fh) {
              const int ix = static_cast<int>(floorf(x)), iy = static_cast<int>(floorf(y));
              box.xlo = min(box.xlo, ix);
              box.xhi = max(box.xhi, ix + 1);
              box.ylo = min(box.ylo, iy);
              box.yhi = max(box.yhi, iy + 1);
            }
          }
        }
        box.xlo = max(box.xlo, 0);
        box.ylo = max(box.ylo, 0);
        box.xhi = min(box.xhi, W - 1);
        box.yhi = min(box.yhi, H - 1);
      }
      reduce_box_warp(box, s_box[s & 1]);
      // The slot must have been read by the consumers (two steps ago).
      const bool ok = s < kStages || wait_bounded(&empty_bar[slot], (use - 1) & 1u, stop, failed);
      if (producers_any(!ok)) break;  // also the barrier that completes the box
      if (qi < cur.tq.count) {
        float4* raw = s_raw + slot * kStepPoints + qi * K;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k)
          if (k < K) raw[k] = make_float4(pxy[k].x, pxy[k].y, pa[k], 0.0f);
      }
      // The next step's inputs load while this one is copied and gathered.
      TileStep nxt = cur;
      int nl = l + 1;
      if (nl == L) {
        nl = 0;
        item += gridDim.x;
        nxt = decode(item);
        if (nxt.live) item_base(nxt);
      }
      if (nxt.live) prefetch(nxt, nl);
      Window win = window_of(s_box[s & 1], kProducerWarps, capacity);
      if (!win.staged) {
        // Too large: keep the middle rows that fit (points outside read value
        // directly), or nothing if one row is already too wide.
        if (win.w <= capacity) {
          const int h = capacity / win.w;
          win.y0 += (win.h - h) / 2;
          win.h = h;
          win.staged = true;
        } else {
          win.w = win.h = 0;
        }
      }
      if (win.w > 0 && win.h > 0) {
        const T* src = value + (static_cast<long long>(cur.b) * S * M + cur.m) * D +
                       (qi % CPR) * (16 / static_cast<int>(sizeof(T)));
        const unsigned dst0 = smem_addr(s_win + slot * slot_bytes) + (qi % CPR) * 16;
        const int px = (qi & 31) / CPR;
        for (int row = pwarp; row < win.h; row += kProducerWarps) {
          const long long prow = start + static_cast<long long>(win.y0 + row) * W + win.x0;
          const T* sp = src + (prow + px) * MD;
          unsigned dp = dst0 + (row * win.w + px) * ROW;
          for (int x = px; x < win.w; x += 32 / CPR) {
            if (in_bounds(sp, 16, false)) cp_async_16(dp, sp);  // debug build: skipped
            sp += (32 / CPR) * static_cast<long long>(MD);
            dp += (32 / CPR) * ROW;
          }
        }
      }
      if (qi == 0) {
        SlotInfo& si = s_info[slot];
        si.live = 1;
        si.b = cur.b;
        si.m = cur.m;
        si.l = l;
        si.wx0 = win.x0;
        si.wy0 = win.y0;
        si.ww = win.w;
        si.wh = win.h;
        si.tq = cur.tq;
      }
      mbar_arrive(&full_bar[slot]);
      mbar_arrive_cp_async(&full_bar[slot]);
      cur = nxt;
      l = nl;
    }
    cp_async_wait_all();
    return;
  }

  // -------------------------------------------------------------------- consumers
  const int ctid = threadIdx.x - kProducers;
  const int sw = ctid / LANES;
  const int lane = ctid % LANES;
  // The sub-warp's points of a step are t = j * K + k (query j * NSW + sw,
  // sample k); lane `lane` sets up t = lane, lane + LANES, ...
  int tj[SETUP], tk[SETUP];
#pragma unroll
  for (int i = 0; i < SETUP; ++i) {
    const int t = lane + i * LANES;
    tj[i] = t / K;
    tk[i] = t - tj[i] * K;
  }
  float2 acc[QPS][E / 2];
#pragma unroll
  for (int j = 0; j < QPS; ++j)
#pragma unroll
    for (int e = 0; e < E / 2; ++e) acc[j][e] = make_float2(0.0f, 0.0f);

  for (int s = 0;; ++s) {
    const int slot = s % kStages;
    const unsigned use = static_cast<unsigned>(s / kStages);
    const bool ok = wait_bounded(&full_bar[slot], use & 1u, stop, failed);
    if (!__all_sync(kFullMask, ok)) break;
    const SlotInfo info = s_info[slot];
    if (!info.live) break;
    const int count = info.tq.count;
    // Setup of the sub-warp's points: exact cell, weights, corner offsets.
    {
      const int H = lv.H[info.l], W = lv.W[info.l];
      const long long start = lv.start[info.l];
      const float4* raw = s_raw + slot * kStepPoints;
#pragma unroll
      for (int i = 0; i < SETUP; ++i) {
        const int qj = tj[i] * NSW + sw;
        if (tj[i] < QPS && qj < count) {
          const float4 p = raw[qj * K + tk[i]];
          const Cell c = locate(p.x, p.y, H, W);
          const float hx = 1.0f - c.fx, hy = 1.0f - c.fy;
          const bool v00 = c.vx0 && c.vy0, v10 = c.vx1 && c.vy0;
          const bool v01 = c.vx0 && c.vy1, v11 = c.vx1 && c.vy1;
          const int rx = c.x0 - info.wx0, ry = c.y0 - info.wy0;
          const bool ix0 = static_cast<unsigned>(rx) < static_cast<unsigned>(info.ww);
          const bool ix1 = static_cast<unsigned>(rx + 1) < static_cast<unsigned>(info.ww);
          const bool iy0 = static_cast<unsigned>(ry) < static_cast<unsigned>(info.wh);
          const bool iy1 = static_cast<unsigned>(ry + 1) < static_cast<unsigned>(info.wh);
          const bool inside = (!v00 || (ix0 && iy0)) && (!v10 || (ix1 && iy0)) &&
                              (!v01 || (ix0 && iy1)) && (!v11 || (ix1 && iy1));
          int4 o;
          if (inside) {
            // Byte offsets into the slot's window; the zero row for a corner
            // outside the map.
            const int rel = (ry * info.ww + rx) * ROW;
            o.x = v00 ? rel : zero_row;
            o.y = v10 ? rel + ROW : zero_row;
            o.z = v01 ? rel + info.ww * ROW : zero_row;
            o.w = v11 ? rel + (info.ww + 1) * ROW : zero_row;
          } else {
            // Read from value: ~(element offset) (negative; 0 <= pixel < S and
            // pixel * M * D < 2^31), INT_MIN for a corner outside the map.
            const int base = static_cast<int>(start + static_cast<long long>(c.y0) * W + c.x0);
            o.x = v00 ? ~(base * MD) : INT_MIN;
            o.y = v10 ? ~((base + 1) * MD) : INT_MIN;
            o.z = v01 ? ~((base + W) * MD) : INT_MIN;
            o.w = v11 ? ~((base + W + 1) * MD) : INT_MIN;
          }
          // Entry t * NSW + (sw ^ (t & 7)): the sub-warps of a warp read one t
          // at a time from different bank groups, and a sub-warp's lanes write
          // different t to different bank groups.
          const int t = tj[i] * K + tk[i];
          s_off[t * NSW + (sw ^ (t & 7))] = o;
          s_w[t * NSW + (sw ^ (t & 7))] =
              make_float4(p.z * hx * hy, p.z * c.fx * hy, p.z * hx * c.fy, p.z * c.fx * c.fy);
        }
      }
    }
    __syncwarp();
    const char* wb = reinterpret_cast<const char*>(s_win) + slot * slot_bytes + lane * 16;
    const T* vb = value + (static_cast<long long>(info.b) * S * M + info.m) * D + lane * E;
#pragma unroll
    for (int j = 0; j < QPS; ++j) {
      if (j * NSW + sw < count) {
#pragma unroll 4
        for (int k = 0; k < K; ++k) {
          const int t = j * K + k;
          const int idx = t * NSW + (sw ^ (t & 7));
          const int4 o = s_off[idx];
          const float4 w = s_w[idx];
          float v0[E], v1[E], v2[E], v3[E];
          if (o.x >= 0) {
            LV::shared(wb + o.x, v0);
            LV::shared(wb + o.y, v1);
            LV::shared(wb + o.z, v2);
            LV::shared(wb + o.w, v3);
          } else {
#pragma unroll
            for (int e = 0; e < E; ++e) v0[e] = v1[e] = v2[e] = v3[e] = 0.0f;
            if (o.x != INT_MIN) LV::global(vb + ~o.x, v0);
            if (o.y != INT_MIN) LV::global(vb + ~o.y, v1);
            if (o.z != INT_MIN) LV::global(vb + ~o.z, v2);
            if (o.w != INT_MIN) LV::global(vb + ~o.w, v3);
          }
          fma_lane<E>(acc[j], w.x, v0);
          fma_lane<E>(acc[j], w.y, v1);
          fma_lane<E>(acc[j], w.z, v2);
          fma_lane<E>(acc[j], w.w, v3);
        }
      }
    }
    if (info.l == L - 1) {
#pragma unroll
      for (int j = 0; j < QPS; ++j) {
        const int qj = j * NSW + sw;
        if (qj < count) {
          T* o = output + (static_cast<long long>(info.b) * Lq + info.tq.query(qj)) * MD +
                 info.m * D + lane * E;
          if constexpr (E == 4) {
            *reinterpret_cast<float4*>(o) =
                make_float4(acc[j][0].x, acc[j][0].y, acc[j][1].x, acc[j][1].y);
          } else {
            unsigned u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(acc[j][i].x, acc[j][i].y);
              u[i] = *reinterpret_cast<const unsigned*>(&h);
            }
            *reinterpret_cast<uint4*>(o) = make_uint4(u[0], u[1], u[2], u[3]);
          }
        }
#pragma unroll
        for (int e = 0; e < E / 2; ++e) acc[j][e] = make_float2(0.0f, 0.0f);
      }
    }
    __syncwarp();  // the records are read; the next step may overwrite them
    if ((ctid & 31) == 0) mbar_arrive(&empty_bar[slot]);
  }
}

// Set when a tiled kernel gave up a bounded wait.
__device__ int g_tiled_wait_failed;

cudaError_t tiled_wait_flag(int** flag) {
  // Looked up on every call (no allocation once the module is loaded), so the
  // address always belongs to the current context.
  return cudaGetSymbolAddress(reinterpret_cast<void**>(flag), g_tiled_wait_failed);
}

namespace {

template <typename T, int LANES>
constexpr int row_bytes() {
  return LANES * 16;
}

struct TiledConfig {
  int TH, TW;
};

TiledConfig tiled_config(int K) {
  if (K <= 4) return {8, 16};
  return {8, 8};
}

template <typename T, int LANES>
cudaError_t launch_tiled_t(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int ROW = row_bytes<T, LANES>();
  const int capacity = (kMaxDynamicSmem - kRecordBytes) / (kStages * ROW) - 1;
  const size_t smem = kRecordBytes + static_cast<size_t>(kStages) * (capacity + 1) * ROW;
  static std::atomic<int> attr_set[64];
  static std::atomic<int> sm_count[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (attr_set[dev].load() == 0) {
    err = cudaFuncSetAttribute(forward_tiled_kernel<T, LANES>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    attr_set[dev].store(1);
  }
  if (sm_count[dev].load() == 0) {
    int n = 0;
    err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    sm_count[dev].store(n > 0 ? n : 1);
  }
  int* failed = nullptr;
  if ((err = tiled_wait_flag(&failed)) != cudaSuccess) return err;
  const TiledConfig tc = tiled_config(a.K);
  // Items number at most B * M * Lq (every tile holds a query); one CTA per SM.
  long long blocks = sm_count[dev].load();
  const long long upper = a.B * a.M * a.Lq;
  if (blocks > upper) blocks = upper;
  forward_tiled_kernel<T, LANES><<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.sampling_locations, a.attention_weights, static_cast<T*>(a.output),
      static_cast<int>(a.B), a.S, a.M, a.Lq, a.L, a.K, tc.TH, tc.TW, capacity, failed);
  return cudaGetLastError();
}

}  // namespace

bool forward_tiles_apply(const ForwardArgs& a) {
  if (a.Lq != a.S || a.chunks != 1 || a.K > 8 || a.Lq <= 0 || a.M <= 0 || a.B <= 0)
    return false;
  // Query, tile and item indices are 32-bit: B * Lq * M < 2^31.
  if (a.B * a.Lq * a.M >= (1ll << 31)) return false;
  // A point's record packs a pixel index of value in 28 bits.
  if (a.S >= (1ll << 26)) return false;
  const int row = a.bf16 ? a.D * 2 : a.D * 4;
  return row == 64 || row == 128 || row == 256;
}

cudaError_t launch_forward_tiled(const ForwardArgs& a, cudaStream_t stream) {
  const int row = a.bf16 ? a.D * 2 : a.D * 4;
  if (a.bf16) {
    switch (row) {
      case 64: return launch_tiled_t<__nv_bfloat16, 4>(a, stream);
      case 128: return launch_tiled_t<__nv_bfloat16, 8>(a, stream);
      case 256: return launch_tiled_t<__nv_bfloat16, 16>(a, stream);
      default: return cudaErrorNotSupported;
    }
  }
  switch (row) {
    case 64: return launch_tiled_t<float, 4>(a, stream);
    case 128: return launch_tiled_t<float, 8>(a, stream);
    case 256: return launch_tiled_t<float, 16>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace msda
