// msda_fused.cu -- the MSDeformAttn core fused with the step before it: the
// sampling locations and attention weights are formed in registers from the
// raw reference points, sampling offsets and attention logits (sm_100a).
//
// The step before the core ("Deformable DETR模型解读（附源码+论文）",
// MultiScaleDeformableAttention.forward, and MSDeformAttn.forward on the
// phdsky.com notes of "Deformable DETR Deformable Transformers for End-to-End
// Object Detection"):
//   A[b,q,m,:]   = softmax over the L*K logits of (b, q, m)
//   R = 2:  loc  = ref[b,q,l] + off[b,q,m,l,k] / (W_l, H_l)
//   R = 4:  loc  = ref[b,q,l,0:2] + off[b,q,m,l,k] / K * ref[b,q,l,2:4] * 0.5
// The location is formed in float32 with every operation rounded once in that
// order (the pages' float32 tensors compute it so), which keeps the floor of
// the pixel coordinate identical to theirs; the core then runs as in
// msda_forward.cu / msda_backward.cu.
//
// Backward (the derivative of the real-number formula; the pages print none):
//   d off   = d loc / (W_l, H_l)                      (R = 2)
//           = d loc * ref[2:4] * 0.5 / K              (R = 4)
//   d ref   = sum over (m, k) of d loc, and for R = 4 also
//     d ref[2:4] = sum over (m, k) of d loc * off * 0.5 / K
//   d z_i   = A_i (dA_i - sum_j A_j dA_j)             over the (b, q, m) group
// where d loc and dA are the core's grad_sampling_locations and
// grad_attention_weights.
#include <atomic>
#include <cmath>

#include "msda_device.cuh"
#include "msda_gather.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kThreads = 256;
constexpr int kChunkPoints = 512;

// (max, 1 / sum exp(z - max)) over the LK logits of one group, computed by the
// LANES lanes of a sub-warp (every lane of the warp takes part).
template <int LANES>
__device__ __forceinline__ float2 softmax_norm(const float* __restrict__ z, int LK, int lane) {
  float m = -INFINITY;
  for (int i = lane; i < LK; i += LANES) m = nan_max(m, __ldg(z + i));
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) m = nan_max(m, __shfl_xor_sync(kFullMask, m, o, LANES));
  float s = 0.0f;
  for (int i = lane; i < LK; i += LANES) s += expf(__ldg(z + i) - m);
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) s += __shfl_xor_sync(kFullMask, s, o, LANES);
  return make_float2(m, 1.0f / s);
}

// Forward for any L*K: the two phases of msda_forward.cu (per-point setup into a
// swizzled shared table, then sub-warp gathers), preceded per tile by the
// softmax normaliser of each group.  When a group's L*K points fit one unit of
// the pipelined forward kernel, that kernel is used instead (FUSED variant in
// msda_forward.cu).
template <typename T, int LANES>
__global__ void __launch_bounds__(kThreads)
fused_forward_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                     const int64_t* __restrict__ level_start_index,
                     const float* __restrict__ reference_points,
                     const float* __restrict__ sampling_offsets,
                     const float* __restrict__ attention_logits, T* __restrict__ output,
                     long long S, int M, int D, long long Lq, int L, int K, int R, int chunks,
                     long long groups) {
  using C = Corner<T>;
  constexpr int E = C::N;
  constexpr int G = kThreads / LANES;
  constexpr int PC = kChunkPoints / G;
  constexpr int PER = kChunkPoints / kThreads;
  static_assert(G >= 8, "the shared-memory swizzle needs at least 8 groups per block");
  __shared__ Levels lv;
  __shared__ int4 s_off[kChunkPoints];
  __shared__ float4 s_w[kChunkPoints];
  __shared__ float2 s_norm[G];
  stage_levels(lv, spatial_shapes, level_start_index, L, S);

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int LK = L * K;
  const unsigned kmagic = level_magic(K);
  const int MD = M * D;
  const long long tiles = (groups + G - 1) / G;

  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const long long g_raw = tile * G + gi;
    const bool active = g_raw < groups;
    const Group grp = decompose(active ? g_raw : groups - 1, chunks, M, Lq);
    const float2 nz = softmax_norm<LANES>(attention_logits + grp.bqm * LK, LK, lane);
    if (lane == 0) s_norm[gi] = nz;
    __syncthreads();

    const int ch = (grp.chunk * LANES + lane) * E;
    const bool lane_on = active && ch < D;
    const T* vbase = value + (grp.b * S * M + grp.m) * static_cast<long long>(D) + ch;
    float2 acc[E / 2];
#pragma unroll
    for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);

    for (int p0 = 0; p0 < LK; p0 += PC) {
      const int pc = min(PC, LK - p0);
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        const int t = threadIdx.x + r * kThreads;
        const int tg = t / PC, tj = t % PC;
        const long long g = tile * G + tg;
        if (tj < pc && g < groups) {
          const long long bqm = chunks == 1 ? g : g / chunks;
          const long long bq = bqm / M;
          const int i = p0 + tj;
          const int l = level_of(i, kmagic);
          const long long p = bqm * LK + i;
          const float2 off = __ldg(reinterpret_cast<const float2*>(sampling_offsets) + p);
          const float2 loc = fused_location(reference_points + (bq * L + l) * R, off, R,
                                            lv.W[l], lv.H[l], K);
          const float2 n = s_norm[tg];
          const float a = expf(__ldg(attention_logits + p) - n.x) * n.y;
          const PointSetup su = setup_point(loc.x, loc.y, a, lv.H[l], lv.W[l], lv.start[l], MD);
          const int slot = tj * G + (tg ^ (tj & 7));
          s_off[slot] = su.off;
          s_w[slot] = su.w;
        }
      }
      __syncthreads();
      if (lane_on) {
#pragma unroll 4
        for (int j = 0; j < pc; ++j) {
          const int slot = j * G + (gi ^ (j & 7));
          const int4 o = s_off[slot];
          const float4 w = s_w[slot];
          if (o.x >= 0) C::accumulate(vbase + o.x, w.x, acc);
          if (o.y >= 0) C::accumulate(vbase + o.y, w.y, acc);
          if (o.z >= 0) C::accumulate(vbase + o.z, w.z, acc);
          if (o.w >= 0) C::accumulate(vbase + o.w, w.w, acc);
        }
      }
      __syncthreads();  // the table and s_norm are rewritten next
    }
    if (lane_on) C::store(output + grp.bq * MD + static_cast<long long>(grp.m) * D + ch, acc);
  }
}

// Backward: the two phases of msda_backward.cu's backward_kernel with the
// locations and weights formed from the raw inputs in phase 1, and the chain
// rule through them applied per point when its four dot products (P, Ex, Ey,
// Exy: the value and its corner differences against gO) are complete.  Per tile, each group's lanes first compute its softmax normaliser
// (max and 1 / sum) into shared memory, so that any thread can form any of the
// tile's weights.  grad_logits holds dA until the group's sum_j A_j dA_j is
// known, then d z.  Lane i of a group combines (and later revisits) the points
// p with p % LANES == pair_lane_point(i).
// T: dtype of value and grad_output (float32, or bfloat16 read 8 bytes per
// lane); arithmetic and every gradient are float32 for both.
//
// As in backward_kernel, the corners shared by two points of one level
// (K = 4) are merged before the scatter, and the block is held to 5 per SM.
template <typename T, int LANES>
__global__ void __launch_bounds__(kThreads, 5)
fused_backward_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                      const int64_t* __restrict__ level_start_index,
                      const float* __restrict__ reference_points,
                      const float* __restrict__ sampling_offsets,
                      const float* __restrict__ attention_logits,
                      const T* __restrict__ grad_output, float* __restrict__ grad_value,
                      float* __restrict__ grad_offsets, float* __restrict__ grad_logits,
                      float* __restrict__ grad_reference, long long S, int M, int D,
                      long long Lq, int L, int K, int R, long long groups) {
  using V = Vec4<T>;
  constexpr int E = 4;
  constexpr int G = kThreads / LANES;
  constexpr int PC = kChunkPoints / G;
  constexpr int PER = kChunkPoints / kThreads;
  static_assert(G >= 8, "the shared-memory swizzle needs at least 8 groups per block");
  static_assert(PC % LANES == 0, "a lane must own the same points in every unit");
  __shared__ Levels lv;
  __shared__ int4 s_off[kChunkPoints];
  __shared__ float4 s_w[kChunkPoints];
  __shared__ float4 s_g[kChunkPoints];  // fx, fy, A, 0
  __shared__ float2 s_norm[G];
  stage_levels(lv, spatial_shapes, level_start_index, L, S);

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int LK = L * K;
  const unsigned kmagic = level_magic(K);
  const int MD = M * D;  // < 2^31: one image's value block is (checked by the C ABI)
  const float half_over_k = 0.5f / static_cast<float>(K);
  const long long tiles = (groups + G - 1) / G;

  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const long long g_raw = tile * G + gi;
    const bool active = g_raw < groups;
    const Group grp = decompose(active ? g_raw : groups - 1, 1, M, Lq);
    const int ch = lane * E;
    const bool lane_on = active && ch < D;
    const long long vofs = (grp.b * S * M + grp.m) * static_cast<long long>(D) + ch;
    const T* vbase = value + vofs;
    float* gvbase = grad_value + vofs;
    const float* zg = attention_logits + grp.bqm * LK;
    const float2 nz = softmax_norm<LANES>(zg, LK, lane);
    if (lane == 0) s_norm[gi] = nz;

    float go[E];
#pragma unroll
    for (int e = 0; e < E; ++e) go[e] = 0.0f;
    if (lane_on)
      V::load(grad_output + grp.bq * static_cast<long long>(MD) + static_cast<long long>(grp.m) * D +
                  ch,
              go);
    float sum_adA = 0.0f;  // this lane's share of sum_j A_j dA_j
    __syncthreads();       // s_norm is complete

    for (int q0 = 0; q0 < LK; q0 += PC) {
      const int pc = min(PC, LK - q0);
      // Phase 1: locations, weights and cells of the unit's points.
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        const int t = threadIdx.x + r * kThreads;
        const int tg = t / PC, tj = t % PC;
        const long long g = tile * G + tg;
        const bool live = tj < pc && g < groups;
        int4 off = make_int4(-1, -1, -1, -1);
        float4 w = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        float4 fg = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        int cx0 = 0, cy0 = 0;
        if (live) {
          const long long pidx = g * LK + q0 + tj;
          const int l = level_of(q0 + tj, kmagic);
          const int H = lv.H[l], W = lv.W[l];
          const float2 offj = __ldg(reinterpret_cast<const float2*>(sampling_offsets) + pidx);
          const long long bq = g / M;
          const float2 xy = fused_location(reference_points + (bq * L + l) * R, offj, R, W, H, K);
          const float2 n = s_norm[tg];
          const float a = expf(__ldg(attention_logits + pidx) - n.x) * n.y;
          const Cell c = locate(xy.x, xy.y, H, W);
          const float hx = 1.0f - c.fx, hy = 1.0f - c.fy;
          // Offsets only for corners inside the map (0 <= pixel < S).
          const int base = static_cast<int>(lv.start[l] + static_cast<long long>(c.y0) * W + c.x0);
          off.x = (c.vx0 && c.vy0) ? base * MD : -1;
          off.y = (c.vx1 && c.vy0) ? (base + 1) * MD : -1;
          off.z = (c.vx0 && c.vy1) ? (base + W) * MD : -1;
          off.w = (c.vx1 && c.vy1) ? (base + W + 1) * MD : -1;
          w = make_float4(a * hx * hy, a * c.fx * hy, a * hx * c.fy, a * c.fx * c.fy);
          fg = make_float4(c.fx, c.fy, a, 0.0f);
          cx0 = c.x0;
          cy0 = c.y0;
        }
        // A level's K = 4 points are 4 aligned lanes (PC % 4 == 0).
        prepare_scatter_weights(cx0, cy0, off, K == 4 && PC % 4 == 0, w);
        if (live) {
          const int slot = tj * G + (tg ^ (tj & 7));
          s_off[slot] = off;
          s_w[slot] = w;
          s_g[slot] = fg;
        }
      }
      __syncthreads();

      // Phase 2: gathers, scatters, corner dot products, and the chain rule.
      for (int j0 = 0; j0 < pc; j0 += LANES) {
        const int nb = min(LANES, pc - j0);
        // Point j's three sums over this lane's channels (point_sums3); the
        // gathers and the grad_value scatters happen here.
        auto point_part = [&](int j, float (&t)[3]) {
          t[0] = t[1] = t[2] = 0.0f;
          const int slot = j * G + (gi ^ (j & 7));
          const int4 o = s_off[slot];
          if (lane_on) {
            const float4 w = s_w[slot];
            const float2 f = *reinterpret_cast<const float2*>(&s_g[slot]);  // fx, fy
            const int os[4] = {o.x, o.y, o.z, o.w};
            const float ws[4] = {w.x, w.y, w.z, w.w};
            float q[4][E];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int e = 0; e < E; ++e) q[i][e] = 0.0f;
              if (os[i] >= 0) V::load(vbase + os[i], q[i]);
            }
            float dot[4];
            corner_sums4(q, go, dot);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (__float_as_uint(ws[i]) != kNoScatterBits) scatter_row4(gvbase + os[i], ws[i], go);
            }
            point_sums3(dot, f.x, f.y, t);
          }
        };
        float keep[3] = {0.0f, 0.0f, 0.0f};
        if constexpr (LANES == 1) {
          if (nb > 0) point_part(j0, keep);
        } else {
          for (int jj = 0; jj < nb; jj += 2) {
            float ta[3], tb[3], v[3];
            point_part(j0 + jj, ta);
            if (jj + 1 < nb) {
              point_part(j0 + jj + 1, tb);
            } else {
              tb[0] = tb[1] = tb[2] = 0.0f;
            }
            reduce_pair3<LANES>(ta, tb, lane, v);
            if ((lane & (LANES / 2 - 1)) == (jj >> 1)) {
#pragma unroll
              for (int i = 0; i < 3; ++i) keep[i] = v[i];
            }
          }
        }
        const int jl = pair_lane_point<LANES>(lane);  // this lane's point of the batch
        if (active && jl < nb) {
          const int pj = q0 + j0 + jl;
          const long long p = grp.bqm * LK + pj;
          const int lj = level_of(pj, kmagic);
          const float a = s_g[(j0 + jl) * G + (gi ^ ((j0 + jl) & 7))].z;
          const float dA = keep[0], s_x = keep[1], s_y = keep[2];
          sum_adA = fmaf(a, dA, sum_adA);
          grad_logits[p] = dA;  // dA for now
          const float kx = a * s_x, ky = a * s_y;  // grad_loc / (W, H)
          const float gx = kx * static_cast<float>(lv.W[lj]);
          const float gy = ky * static_cast<float>(lv.H[lj]);
          const float* rp = reference_points + (grp.bq * L + lj) * R;
          float2 goff;
          if (R == 2)
            goff = make_float2(kx, ky);
          else
            goff = make_float2(gx * __ldg(rp + 2) * half_over_k, gy * __ldg(rp + 3) * half_over_k);
          reinterpret_cast<float2*>(grad_offsets)[p] = goff;
          if (grad_reference != nullptr) {
            float* gr = grad_reference + (grp.bq * L + lj) * R;
            atomicAdd(gr + 0, gx);
            atomicAdd(gr + 1, gy);
            if (R == 4) {
              const float2 offj = __ldg(reinterpret_cast<const float2*>(sampling_offsets) + p);
              atomicAdd(gr + 2, gx * offj.x * half_over_k);
              atomicAdd(gr + 3, gy * offj.y * half_over_k);
            }
          }
        }
      }
      __syncthreads();  // the table and s_norm are rewritten next
    }
    // Softmax Jacobian: d z_j = A_j (dA_j - sum_i A_i dA_i).  Each lane revisits
    // the points it wrote.
#pragma unroll
    for (int o = LANES / 2; o > 0; o >>= 1) sum_adA += __shfl_xor_sync(kFullMask, sum_adA, o, LANES);
    if (active) {
      for (int pj = pair_lane_point<LANES>(lane); pj < LK; pj += LANES) {
        const long long p = grp.bqm * LK + pj;
        const float aj = expf(__ldg(zg + pj) - nz.x) * nz.y;
        grad_logits[p] = aj * (grad_logits[p] - sum_adA);
      }
    }
  }
}

template <typename T, int LANES>
long long resident_forward_blocks() {
  static std::atomic<long long> cached[64];  // 0 until known; benign concurrent fills
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev].load() > 0) return cached[dev].load();
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_forward_kernel<T, LANES>,
                                                    kThreads, 0) != cudaSuccess ||
      sms <= 0 || per_sm <= 0)
    return 148;
  const long long n = static_cast<long long>(sms) * per_sm;
  if (dev >= 0 && dev < 64) cached[dev].store(n);
  return n;
}

template <typename T, int LANES>
cudaError_t launch_fused_forward_t(const FusedArgs& a, cudaStream_t stream) {
  constexpr int G = kThreads / LANES;
  const long long tiles = (a.groups + G - 1) / G;
  long long blocks = resident_forward_blocks<T, LANES>();
  if (blocks > tiles) blocks = tiles;
  fused_forward_kernel<T, LANES><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index, a.reference_points,
      a.sampling_offsets, a.attention_logits, static_cast<T*>(a.output), a.S, a.M, a.D, a.Lq,
      a.L, a.K, a.R, a.chunks, a.groups);
  return cudaGetLastError();
}

template <typename T>
cudaError_t fused_forward_lanes(const FusedArgs& a, cudaStream_t stream) {
  switch (a.lanes) {
    case 1: return launch_fused_forward_t<T, 1>(a, stream);
    case 2: return launch_fused_forward_t<T, 2>(a, stream);
    case 4: return launch_fused_forward_t<T, 4>(a, stream);
    case 8: return launch_fused_forward_t<T, 8>(a, stream);
    case 16: return launch_fused_forward_t<T, 16>(a, stream);
    case 32: return launch_fused_forward_t<T, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int LANES>
cudaError_t launch_fused_backward_t(const FusedArgs& a, cudaStream_t stream) {
  const long long per_block = kThreads / LANES;
  long long blocks = (a.groups + per_block - 1) / per_block;
  if (blocks > (1ll << 30)) blocks = 1ll << 30;
  fused_backward_kernel<T, LANES><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.reference_points, a.sampling_offsets, a.attention_logits,
      static_cast<const T*>(a.grad_output), a.grad_value,
      a.grad_sampling_offsets, a.grad_attention_logits, a.grad_reference_points, a.S, a.M, a.D,
      a.Lq, a.L, a.K, a.R, a.groups);
  return cudaGetLastError();
}

template <typename T>
cudaError_t fused_backward_lanes(const FusedArgs& a, cudaStream_t stream) {
  switch (a.lanes) {
    case 1: return launch_fused_backward_t<T, 1>(a, stream);
    case 2: return launch_fused_backward_t<T, 2>(a, stream);
    case 4: return launch_fused_backward_t<T, 4>(a, stream);
    case 8: return launch_fused_backward_t<T, 8>(a, stream);
    case 16: return launch_fused_backward_t<T, 16>(a, stream);
    case 32: return launch_fused_backward_t<T, 32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_fused_forward(const FusedArgs& a, cudaStream_t stream) {
  if (a.groups == 0) return cudaSuccess;
  // The pipelined kernel of msda_forward.cu when a group's points fit one unit.
  const cudaError_t err = launch_fused_forward_pipelined(a, stream);
  if (err != cudaErrorNotSupported) return err;
  return a.bf16 ? fused_forward_lanes<__nv_bfloat16>(a, stream)
                : fused_forward_lanes<float>(a, stream);
}

cudaError_t launch_fused_backward(const FusedArgs& a, cudaStream_t stream) {
  cudaError_t err = launch_zero(a.grad_value, a.value_elements, stream);
  if (err != cudaSuccess) return err;
  if (a.grad_reference_points != nullptr && a.reference_elements > 0) {
    err = cudaMemsetAsync(a.grad_reference_points, 0,
                          sizeof(float) * static_cast<size_t>(a.reference_elements), stream);
    if (err != cudaSuccess) return err;
  }
  if (a.groups == 0) return cudaSuccess;
  return a.bf16 ? fused_backward_lanes<__nv_bfloat16>(a, stream)
                : fused_backward_lanes<float>(a, stream);
}

}  // namespace msda
