// msda_backward.cu -- training backward of the MSDeformAttn core (sm_100a).
//
// The pages print no backward.  These are the exact derivatives of the forward
// ("Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation, sampled as in "Deformable DETR模型
// 解读（附源码+论文）", ms_deform_attn_core_pytorch), taken inside the cell
// [x0, x0+1) x [y0, y0+1), x0 = floor(x), y0 = floor(y).  With
// V_ij = V(x0 + i, y0 + j) (zero outside the map), hx = 1 - fx, hy = 1 - fy and
// gO = grad_output[b, q, m*D : m*D + D]:
//
//   grad_attn[p]    = sum_d gO * (hy (hx V00 + fx V10) + fy (hx V01 + fx V11))
//   grad_loc[p].x   = A * W_l * sum_d gO * (hy (V10 - V00) + fy (V11 - V01))
//   grad_loc[p].y   = A * H_l * sum_d gO * (hx (V01 - V00) + fx (V11 - V10))
//   grad_value[corner ij] += A * (i ? fx : hx) * (j ? fy : hy) * gO   (corners in the map)
//
// (dx/dloc_x = W_l because x = loc_x * W_l - 0.5.)
//
// The grad_value contributions are scattered with 16-byte vector atomics
// (red.global.add.v4.f32); the work decomposition is described at
// backward_kernel.
#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

// Header of the deterministic backward's workspace: the scale pass's per-block
// partials, then its result.
struct FixedHeader {
  float sum_abs_weights[kScaleBlocks];
  float max_abs_grad[kScaleBlocks];
  int fixed;         // 1: all inputs finite, integer accumulation; 0: float atomics
  float scale;       // 2^e
  float inv_scale;   // 2^-e
};
static_assert(sizeof(FixedHeader) <= kFixedHeaderBytes, "header must fit its slot");

constexpr int kBwdThreads = 256;

constexpr int kBwdPoints = 512;  // points set up per unit (two per thread)
// Channels of a head per kernel pass: one sub-warp of at most 32 lanes, 4 per lane.
constexpr int kPassChannels = 128;

// T: dtype of value and grad_output (float32, or bfloat16 read 8 bytes per lane);
// arithmetic and grad_value are float32 for both.
//
// Work decomposition.  A sub-warp of LANES lanes owns one (b, q, m) group and
// each lane 4 of the head's channels, so a point corner is one 128-byte line of
// grad_value for D = 32.  A block owns G = 256 / LANES consecutive groups and
// walks their points in units of PC = 512 / G points per group:
//   phase 1  each thread maps two of the unit's points once -- exact floor,
//            corner validity, 32-bit corner offsets, the four weights
//            A * bilinear and (fx, fy, A * W_l, A * H_l) -- into a swizzled
//            shared table;
//   phase 2  per point, each sub-warp reads the setup (broadcast), gathers its
//            slice of the four corners, scatters the grad_value contributions,
//            and forms over its channels the four dot products
//              P  = sum_d gO V00,          Ex = sum_d gO (V10 - V00),
//              Ey = sum_d gO (V01 - V00),  Exy = sum_d gO (V11 - V01 - V10 + V00)
//            (differences taken per channel, so a common offset of the value
//            field cancels exactly), applies the point's fx, fy to them
//            (point_sums3) and reduces the three results over the lanes, two
//            points per exchange (reduce_pair3).  After each batch of LANES
//            points every lane holds one point's totals
//              grad_attn = P + fx Ex + fy Ey + fx fy Exy
//              grad_x / (A W_l) = Ex + fy Exy
//              grad_y / (A H_l) = Ey + fx Exy
//            and writes its gradients.
// These are the derivatives above, regrouped with hx + fx = hy + fy = 1.
// In the float path with K = 4, phase 1 also merges the corners that two points
// of one level share (merge_shared_corners), so such a pixel takes one
// reduction of (w1 + w2) gO instead of two; on the encoder workloads that is
// about one corner in nine.  The block is held to 5 per SM (48 registers),
// which measured faster than the compiler's own choice.
//
// FIXED (the deterministic backward): each grad_value contribution A w_ij gO[d]
// (the same float32 product as the default path) is multiplied by 2^e, rounded
// to an integer and added with a 64-bit integer atomic.  Integer addition is
// associative, so the sums -- and after fixed_to_float_kernel, grad_value -- do
// not depend on the order in which the atomics land.  e is chosen so that no
// partial sum can reach 2^62 (see scale_final_kernel).  The accumulator row of a
// (b, pixel, m) keeps channel 4i + c of lane i at c * D/4 + i, so each 64-bit
// atomic instruction of a sub-warp covers one contiguous span.  If an input is
// not finite (header->fixed == 0) the kernel falls back to float atomics into
// grad_value: the NaN / Inf pattern does not depend on the order either.
template <typename T, int LANES, bool FIXED, int SPLIT>
__global__ void __launch_bounds__(kBwdThreads, 5)
backward_kernel(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
                const int64_t* __restrict__ level_start_index,
                const float* __restrict__ sampling_locations,
                const float* __restrict__ attention_weights,
                const T* __restrict__ grad_output, float* __restrict__ grad_value,
                float* __restrict__ grad_sampling_locations,
                float* __restrict__ grad_attention_weights, long long S, int M, int D,
                long long Lq, int L, int K, long long groups, int c0, int Dc,
                unsigned long long* __restrict__ fixed_acc,
                const FixedHeader* __restrict__ header) {
  using V = Vec4<T>;
  constexpr int E = 4;
  constexpr int G = kBwdThreads / LANES;
  constexpr int PC = kBwdPoints / G;
  constexpr int PER = kBwdPoints / kBwdThreads;
  static_assert(G >= 8, "the shared-memory swizzle needs at least 8 groups per block");
  __shared__ Levels lv;
  __shared__ int4 s_off[kBwdPoints];
  __shared__ float4 s_w[kBwdPoints];
  __shared__ float4 s_g[kBwdPoints];
  bool use_fixed = false;
  float scale = 1.0f;
  if constexpr (FIXED) {
    use_fixed = header->fixed != 0;
    scale = header->scale;
  }
  const int dq = D / 4;
  // Corners shared by two points of one level of one group are merged before the
  // scatter (merge_shared_corners).  The merge depends only on the inputs (the
  // weights are summed in lane order), so the deterministic path keeps its
  // bit-identical results with it.
  constexpr bool kMerge = SPLIT == 1 && PC % 4 == 0;

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int LK = L * K;
  const unsigned kmagic = level_magic(K);
  const int MD = M * D;  // < 2^31: one image's value block is (checked by the C ABI)
  // Point split (SPLIT > 1): SPLIT consecutive sub-warps share one group,
  // subset s taking its points s, s + SPLIT, ...  Every result of the backward is
  // per point (or an atomic), so the subsets need no reduction; work units run
  // over the virtual groups (groups * SPLIT) and their LKv points.
  const long long vgroups = groups * SPLIT;
  const int LKv = (LK + SPLIT - 1) / SPLIT;
  const long long tiles = (vgroups + G - 1) / G;
  // Virtual point (group v, point jv) -> real group g and point index jr.
  auto real_point = [&](long long v, int jv, long long& g, int& jr) {
    g = v / SPLIT;
    jr = jv * SPLIT + static_cast<int>(v - g * SPLIT);
  };

  // The first unit's locations and weights are pulled into L2 before the level
  // metadata is staged, so the two memory round trips overlap.
  if (blockIdx.x < tiles) {
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int t = threadIdx.x + r * kBwdThreads;
      const int tg = t / PC, tj = t % PC;
      long long g;
      int jr;
      real_point(blockIdx.x * G + tg, tj, g, jr);
      if (tj < min(PC, LKv) && g < groups && jr < LK) {
        asm volatile("prefetch.global.L2 [%0];" ::"l"(sampling_locations + 2 * (g * LK + jr)));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(attention_weights + g * LK + jr));
      }
    }
  }
  stage_levels(lv, spatial_shapes, level_start_index, L, S);

  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const long long v_raw = tile * G + gi;
    const bool active = v_raw < vgroups;
    long long g_raw;
    int subset_first;
    real_point(v_raw, 0, g_raw, subset_first);  // subset_first = this sub-warp's subset s
    const Group grp = decompose(active ? g_raw : groups - 1, 1, M, Lq);
    const int ch = lane * E;
    const bool lane_on = active && ch < Dc;  // clamped tail groups touch no memory
    const long long vofs = (grp.b * S * M + grp.m) * static_cast<long long>(D) + c0 + ch;
    const T* vbase = value + vofs;
    float* gvbase = grad_value + vofs;
    unsigned long long* abase =
        FIXED ? fixed_acc + (grp.b * S * M + grp.m) * static_cast<long long>(D) + lane : nullptr;
    // grad_value corner at element offset o (relative to the (b, m, lane) base) += w gO.
    auto scatter = [&](int o, float w, const float (&g)[E]) {
      if constexpr (FIXED) {
        if (use_fixed) {
#pragma unroll
          for (int c = 0; c < E; ++c)
            if (in_bounds(abase + o + c * dq, 8, true))
              atomicAdd(abase + o + c * dq, static_cast<unsigned long long>(
                                                __float2ll_rn(__fmul_rn(w * g[c], scale))));
          return;
        }
      }
      scatter_row4(gvbase + o, w, g);
    };

    float go[E];
#pragma unroll
    for (int e = 0; e < E; ++e) go[e] = 0.0f;
    if (lane_on)
      V::load(grad_output + grp.bq * static_cast<long long>(MD) + static_cast<long long>(grp.m) * D +
                  c0 + ch,
              go);

    for (int q0 = 0; q0 < LKv; q0 += PC) {
      const int pc = min(PC, LKv - q0);
      // Phase 1: the unit's points, two per thread.
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        const int t = threadIdx.x + r * kBwdThreads;
        const int tg = t / PC, tj = t % PC;
        long long g;
        int jr;
        real_point(tile * G + tg, q0 + tj, g, jr);
        // A subset's slot past its group's last point (SPLIT > 1) is written
        // with no corner and no output.
        const bool live = tj < pc && g < groups && jr < LK;
        int4 off = make_int4(-1, -1, -1, -1);
        float4 w = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        float4 fg = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        int cx0 = 0, cy0 = 0;
        if (live) {
          const long long pidx = g * LK + jr;
          const float2 xy = __ldg(reinterpret_cast<const float2*>(sampling_locations) + pidx);
          const float a = __ldg(attention_weights + pidx);
          const int l = level_of(jr, kmagic);
          const int H = lv.H[l], W = lv.W[l];
          const Cell c = locate(xy.x, xy.y, H, W);
          const float hx = 1.0f - c.fx, hy = 1.0f - c.fy;
          // Offsets only for corners inside the map (0 <= pixel < S).
          const int base = static_cast<int>(lv.start[l] + static_cast<long long>(c.y0) * W + c.x0);
          off.x = (c.vx0 && c.vy0) ? base * MD : -1;
          off.y = (c.vx1 && c.vy0) ? (base + 1) * MD : -1;
          off.z = (c.vx0 && c.vy1) ? (base + W) * MD : -1;
          off.w = (c.vx1 && c.vy1) ? (base + W + 1) * MD : -1;
          w = make_float4(a * hx * hy, a * c.fx * hy, a * hx * c.fy, a * c.fx * c.fy);
          cx0 = c.x0;
          cy0 = c.y0;
          fg = make_float4(c.fx, c.fy, a * static_cast<float>(W), a * static_cast<float>(H));
        }
        // K = 4 and PC % 4 == 0: a level's points are 4 aligned lanes.
        if constexpr (kMerge) prepare_scatter_weights(cx0, cy0, off, K == 4, w);
        if (live || (SPLIT > 1 && tj < pc && g < groups)) {
          const int slot = tj * G + (tg ^ (tj & 7));
          s_off[slot] = off;
          s_w[slot] = w;
          s_g[slot] = fg;
        }
      }
      __syncthreads();

      // Phase 2: gathers, scatters and the corner dot products.  The first
      // scatter waits for the kernel that zeroes grad_value, which may still be
      // running when this one starts (programmatic dependent launch; without it
      // the wait returns at once).
      if (!FIXED) asm volatile("griddepcontrol.wait;" ::: "memory");
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
              if (kMerge ? __float_as_uint(ws[i]) != kNoScatterBits : os[i] >= 0)
                scatter(os[i], ws[i], go);
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
        const int jr_out = (q0 + j0 + jl) * SPLIT + subset_first;
        if (active && jl < nb && jr_out < LK) {
          const int j = j0 + jl;
          const float4 gg = s_g[j * G + (gi ^ (j & 7))];
          const long long pidx = grp.bqm * LK + jr_out;
          float2* gl = reinterpret_cast<float2*>(grad_sampling_locations) + pidx;
          if (c0 == 0) {
            grad_attention_weights[pidx] = keep[0];
            *gl = make_float2(gg.z * keep[1], gg.w * keep[2]);
          } else {
            // A later channel pass adds its channels' share (this thread wrote the
            // earlier passes' value; the passes run in stream order).
            grad_attention_weights[pidx] += keep[0];
            const float2 prev = *gl;
            *gl = make_float2(prev.x + gg.z * keep[1], prev.y + gg.w * keep[2]);
          }
        }
      }
      // The next unit's setup overwrites the table.
      __syncthreads();
    }
  }
}

__global__ void zero_kernel(float4* __restrict__ p, long long n4) {
  // A kernel launched after this one with programmatic stream serialization may
  // start now; it waits (griddepcontrol.wait) before touching p.
  asm volatile("griddepcontrol.launch_dependents;");
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    p[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

cudaError_t launch_zero(float* p, long long n, cudaStream_t stream) {
  // n is a multiple of 4 (D % 4 == 0) and p is 16-byte aligned.
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  long long blocks = (n4 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  zero_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(reinterpret_cast<float4*>(p), n4);
  return cudaGetLastError();
}

// The deterministic backward's scale, pass 1: a fixed grid of kScaleBlocks
// blocks, each summing |A| and taking max |gO| over a fixed strided share in a
// fixed order (so the result is the same on every run and every device).
// A NaN anywhere makes the block's sum or max NaN; an Inf makes it Inf.
__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__global__ void __launch_bounds__(256)
scale_partials_kernel(const float* __restrict__ attention_weights, long long n_weights,
                      const T* __restrict__ grad_output, long long n_grad,
                      FixedHeader* __restrict__ header) {
  __shared__ float s_sum[8], s_max[8];
  const long long stride = static_cast<long long>(kScaleBlocks) * 256;
  float sum = 0.0f, mx = 0.0f;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n_weights; i += stride)
    sum += fabsf(attention_weights[i]);
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n_grad; i += stride) {
    const float g = fabsf(to_float(grad_output[i]));
    mx = (g > mx || g != g) ? g : mx;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(kFullMask, sum, o);
    const float y = __shfl_xor_sync(kFullMask, mx, o);
    mx = (y > mx || y != y) ? y : mx;
  }
  if ((threadIdx.x & 31) == 0) {
    s_sum[threadIdx.x >> 5] = sum;
    s_max[threadIdx.x >> 5] = mx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.0f, m = 0.0f;
    for (int w = 0; w < 8; ++w) {
      t += s_sum[w];
      m = (s_max[w] > m || s_max[w] != s_max[w]) ? s_max[w] : m;
    }
    header->sum_abs_weights[blockIdx.x] = t;
    header->max_abs_grad[blockIdx.x] = m;
  }
}

// Pass 2 (one warp): bound = sum |A| * max |gO| bounds every grad_value element
// (a point adds A w_ij gO to a corner, and the w_ij of a point sum to 1), so
// with e = 60 - ceil(log2(bound)) no sum of scaled contributions reaches 2^60.
__global__ void scale_final_kernel(FixedHeader* __restrict__ header) {
  const int lane = threadIdx.x;
  float sum = 0.0f, mx = 0.0f;
  for (int i = lane; i < kScaleBlocks; i += 32) {
    sum += header->sum_abs_weights[i];
    const float m = header->max_abs_grad[i];
    mx = (m > mx || m != m) ? m : mx;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sum += __shfl_xor_sync(kFullMask, sum, o);
    const float y = __shfl_xor_sync(kFullMask, mx, o);
    mx = (y > mx || y != y) ? y : mx;
  }
  if (lane == 0) {
    const float bound = sum * mx;
    const bool finite = isfinite(bound);
    int e = 60;
    if (finite && bound > 0.0f) {
      int ex = 0;
      frexpf(bound, &ex);  // bound < 2^ex
      e = 60 - ex;
    }
    e = max(-60, min(100, e));
    header->fixed = finite ? 1 : 0;
    header->scale = ldexpf(1.0f, e);
    header->inv_scale = ldexpf(1.0f, -e);
  }
}

// grad_value = accumulator * 2^-e (one rounding of the exact integer sum), with
// the accumulator row's channel order undone.  Nothing to do on the float
// fallback, whose atomics wrote grad_value directly.
__global__ void fixed_to_float_kernel(const unsigned long long* __restrict__ acc,
                                      const FixedHeader* __restrict__ header,
                                      float* __restrict__ grad_value, long long n, int D) {
  if (header->fixed == 0) return;
  const float inv = header->inv_scale;
  const int dq = D / 4;
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = j / D;
    const int d = static_cast<int>(j - row * D);
    const long long v = static_cast<long long>(acc[row * D + (d & 3) * dq + (d >> 2)]);
    grad_value[j] = __fmul_rn(__ll2float_rn(v), inv);
  }
}

template <typename T, int LANES, bool FIXED>
static cudaError_t launch_backward_t(const BackwardArgs& a, unsigned long long* acc,
                                     const FixedHeader* header, cudaStream_t stream) {
  const long long per_block = kBwdThreads / LANES;
  // Fewer blocks than about two waves of 148 SMs x 4 (a decoder's few hundred
  // queries): split each group's points over up to 4 sub-warps.
  int split = 1;
  while (split < 4 && (a.groups * split * 2 + per_block - 1) / per_block <= 148 * 4 * 2)
    split *= 2;
  long long blocks = (a.groups * split + per_block - 1) / per_block;
  if (blocks > (1ll << 30)) blocks = 1ll << 30;
  auto go = [&](auto kernel) {
    // Heads wider than kPassChannels run as channel passes in stream order: every
    // pass scatters its channels of grad_value, and the later passes add their
    // share of grad_attn and grad_loc to what the first wrote.  The first pass
    // overlaps its start (metadata, locations, corner loads) with the zeroing of
    // grad_value launched just before it; the deterministic path (one pass) reads
    // the scale pass's header first, so it is launched plainly.
    for (int c0 = 0; c0 < a.D; c0 += kPassChannels) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(blocks));
      cfg.blockDim = dim3(kBwdThreads);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = (FIXED || c0 > 0) ? 0 : 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const int dc = min(kPassChannels, a.D - c0);
      const cudaError_t err =
          cudaLaunchKernelEx(&cfg, kernel, static_cast<const T*>(a.value), a.spatial_shapes,
                             a.level_start_index, a.sampling_locations, a.attention_weights,
                             static_cast<const T*>(a.grad_output), a.grad_value,
                             a.grad_sampling_locations, a.grad_attention_weights, a.S, a.M,
                             a.D, a.Lq, a.L, a.K, a.groups, c0, dc, acc, header);
      if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
  };
  if (split == 4) return go(backward_kernel<T, LANES, FIXED, 4>);
  if (split == 2) return go(backward_kernel<T, LANES, FIXED, 2>);
  return go(backward_kernel<T, LANES, FIXED, 1>);
}

template <typename T, bool FIXED>
static cudaError_t backward_lanes(const BackwardArgs& a, unsigned long long* acc,
                                  const FixedHeader* header, cudaStream_t stream) {
  switch (a.lanes) {
    case 1: return launch_backward_t<T, 1, FIXED>(a, acc, header, stream);
    case 2: return launch_backward_t<T, 2, FIXED>(a, acc, header, stream);
    case 4: return launch_backward_t<T, 4, FIXED>(a, acc, header, stream);
    case 8: return launch_backward_t<T, 8, FIXED>(a, acc, header, stream);
    case 16: return launch_backward_t<T, 16, FIXED>(a, acc, header, stream);
    case 32: return launch_backward_t<T, 32, FIXED>(a, acc, header, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t stream) {
  cudaError_t err = launch_zero(a.grad_value, a.value_elements, stream);
  if (err != cudaSuccess || a.groups == 0) return err;
  return a.bf16 ? backward_lanes<__nv_bfloat16, false>(a, nullptr, nullptr, stream)
                : backward_lanes<float, false>(a, nullptr, nullptr, stream);
}

cudaError_t launch_backward_deterministic(const BackwardArgs& a, void* workspace,
                                          cudaStream_t stream) {
  auto* header = static_cast<FixedHeader*>(workspace);
  auto* acc = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) +
                                                    kFixedHeaderBytes);
  cudaError_t err = launch_zero(a.grad_value, a.value_elements, stream);
  if (err != cudaSuccess || a.groups == 0) return err;
  // The accumulators (8 bytes per element) are zeroed as twice as many floats.
  if ((err = launch_zero(reinterpret_cast<float*>(acc), 2 * a.value_elements, stream)) !=
      cudaSuccess)
    return err;
  const long long n_weights = a.groups * a.L * a.K;
  const long long n_grad = a.groups * a.D;
  if (a.bf16)
    scale_partials_kernel<__nv_bfloat16><<<kScaleBlocks, 256, 0, stream>>>(
        a.attention_weights, n_weights, static_cast<const __nv_bfloat16*>(a.grad_output),
        n_grad, header);
  else
    scale_partials_kernel<float><<<kScaleBlocks, 256, 0, stream>>>(
        a.attention_weights, n_weights, static_cast<const float*>(a.grad_output), n_grad,
        header);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  scale_final_kernel<<<1, 32, 0, stream>>>(header);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  err = a.bf16 ? backward_lanes<__nv_bfloat16, true>(a, acc, header, stream)
               : backward_lanes<float, true>(a, acc, header, stream);
  if (err != cudaSuccess) return err;
  long long blocks = (a.value_elements + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks > 0)
    fixed_to_float_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        acc, header, a.grad_value, a.value_elements, a.D);
  return cudaGetLastError();
}

}  // namespace msda
