// msda_forward.cu -- forward kernel of the MSDeformAttn core (sm_100a).
//
//   out[b, q, m*D + d] = sum_{l,k} A[b,q,m,l,k] * bilinear(value_l[b, :, m, d], loc[b,q,m,l,k])
//
// "Deformable DETR Deformable Transformers for End-to-End Object Detection",
// multi-scale deformable attention equation; sampling rule and output layout of
// "Deformable DETR模型解读（附源码+论文）", ms_deform_attn_core_pytorch.
//
// Work decomposition.  A sub-warp of LANES lanes owns one (b, q, m, channel
// chunk) group; each lane owns 16 contiguous bytes of the head's channels, so
// one corner of one point is a single fully used 128-byte line for D = 32
// float32.  A block of 256 threads owns G = 256 / LANES consecutive groups and
// walks their points in chunks of PC = 2 * LANES points per group (G * PC = 512
// points per chunk):
//   phase 1  every thread maps two of the chunk's points to their cell -- exact
//            floor, corner validity, the four corners' element offsets and the
//            four weights A * bilinear -- reading locations and weights
//            coalesced, and writes them to shared memory (swizzled so that both
//            the writes and the phase-2 broadcasts are free of bank conflicts);
//   phase 2  every sub-warp reads its points' setups (one broadcast per 16
//            bytes), gathers its slice of the four corners with 16-byte
//            read-only loads and accumulates in float32 with packed two-wide
//            FMAs.
// The per-point index arithmetic is thus done once per point instead of once
// per lane.  The grid holds as many blocks as are resident at once; block i
// takes tiles i, i + grid, i + 2 grid, ..., so at any moment the blocks work on
// one window of neighbouring queries (consecutive groups are consecutive heads
// of consecutive queries), whose samples overlap in L2.  The setup table is
// double-buffered: the locations and weights of a block's next unit (chunk of a
// tile) are loaded before the current unit's gathers and turned into setups
// after them, so their HBM latency hides behind the gathers and one barrier
// per unit suffices.  (Head-major tiles and contiguous per-block tile ranges,
// which favour L1 reuse, measured slower on the encoder workload.)
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "msda_device.cuh"
#include "msda_gather.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kThreads = 256;
constexpr int kChunkPoints = 512;

// Tuning per value dtype (measured on the encoder workloads): for float32 the
// gathers of up to 8 points are issued back to back (predicated corner loads,
// Corner::accumulate4) and the kernel is held to 5 blocks per SM (48
// registers); bfloat16 keeps one branch per corner, a 4-point unroll and 4
// blocks per SM (64 registers), which measured faster for it.  The two
// dtypes therefore get their own __global__ entry (forward_kernel below) around
// one body.

}  // namespace

// FUSED: the inputs are the step before the core (msda_fused.cu): the
// locations array holds sampling offsets and the weights array holds the
// attention logits (same shapes), and reference_points [B, Lq, L, R] is read;
// the setup forms each point's location and softmax weight in registers.  This
// needs a group's L*K points in one unit (L*K <= PC <= 32), so the softmax is a
// shuffle reduction over the PC consecutive threads that set the group up.
template <typename T, int LANES, bool FUSED, int SPLIT>
__device__ __forceinline__ void
forward_body(const T* __restrict__ value, const int64_t* __restrict__ spatial_shapes,
             const int64_t* __restrict__ level_start_index,
             const float* __restrict__ sampling_locations,
             const float* __restrict__ attention_weights, T* __restrict__ output,
             long long S, int M, int D, long long Lq, int L, int K, int chunks,
             long long groups, const float* __restrict__ reference_points, int R) {
  using C = Corner<T>;
  constexpr int E = C::N;
  constexpr int G = kThreads / LANES;
  constexpr int PC = kChunkPoints / G;
  constexpr int PER = kChunkPoints / kThreads;  // points set up per thread
  static_assert(G >= 8, "the shared-memory swizzle needs at least 8 groups per block");
  __shared__ Levels lv;
  __shared__ int4 s_off[2][kChunkPoints];
  __shared__ float4 s_w[2][kChunkPoints];

  const int lane = threadIdx.x % LANES;
  const int gi = threadIdx.x / LANES;
  const int LK = L * K;
  const int MD = M * D;
  const unsigned kmagic = level_magic(K);
  // Point split (SPLIT > 1, non-fused, chunks == 1): SPLIT consecutive
  // sub-warps share one group, subset s taking its points s, s + SPLIT, ...;
  // their partial sums are added with shuffles before the store.  Work units
  // then run over the virtual groups (groups * SPLIT) and their LKv points.
  static_assert(SPLIT == 1 || (!FUSED && LANES * SPLIT <= 32), "a split group fits one warp");
  const long long vgroups = groups * SPLIT;
  const int LKv = (LK + SPLIT - 1) / SPLIT;
  const long long tiles = (vgroups + G - 1) / G;
  long long tile = blockIdx.x;
  int p0 = 0;

  // Prefetched inputs of the next unit's points.
  float2 pxy[PER];
  float pa[PER];
  // Virtual point (group v, point q0 + tj) -> real group and point index jr.
  auto real_point = [&](long long v, int jv, long long& g, int& jr) {
    g = v / SPLIT;
    jr = jv * SPLIT + static_cast<int>(v - g * SPLIT);
  };
  auto prefetch = [&](long long t_, int q0) {
    const int pc = min(PC, LKv - q0);
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int t = threadIdx.x + r * kThreads;
      const int tg = t / PC, tj = t % PC;
      long long g;
      int jr;
      real_point(t_ * G + tg, q0 + tj, g, jr);
      if (tj < pc && g < groups && jr < LK) {
        const long long bqm = chunks == 1 ? g : g / chunks;
        pxy[r] = __ldg(reinterpret_cast<const float2*>(sampling_locations) + bqm * LK + jr);
        pa[r] = __ldg(attention_weights + bqm * LK + jr);
      }
    }
  };
  auto setup = [&](long long t_, int q0, int buf) {
    const int pc = min(PC, LKv - q0);
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int t = threadIdx.x + r * kThreads;
      const int tg = t / PC, tj = t % PC;
      long long g;
      int jr;
      real_point(t_ * G + tg, q0 + tj, g, jr);
      const bool live = tj < pc && g < groups && jr < LK;
      if (SPLIT > 1 && tj < pc && g < groups && jr >= LK) {
        // A subset's slot past its group's last point reads nothing and adds zero.
        const int slot = tj * G + (tg ^ (tj & 7));
        s_off[buf][slot] = make_int4(-1, -1, -1, -1);
        s_w[buf][slot] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
      if constexpr (FUSED) {
        // Softmax over the group's L*K = pc logits, held by PC consecutive lanes.
        float z = live ? pa[r] : -INFINITY;
        float mx = z;
#pragma unroll
        for (int o = PC / 2; o > 0; o >>= 1) {
          const float y = __shfl_xor_sync(kFullMask, mx, o, PC);
          mx = (y > mx || y != y) ? y : mx;
        }
        const float e = live ? expf(z - mx) : 0.0f;
        float sum = e;
#pragma unroll
        for (int o = PC / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(kFullMask, sum, o, PC);
        pa[r] = e * (1.0f / sum);
        if (live) {
          const int l = level_of(jr, kmagic);
          const long long bq = decompose(g, chunks, M, Lq).bq;
          pxy[r] = fused_location(reference_points + (bq * L + l) * R, pxy[r], R, lv.W[l],
                                  lv.H[l], K);
        }
      }
      if (live) {
        const int l = level_of(jr, kmagic);
        const PointSetup su = setup_point(pxy[r].x, pxy[r].y, pa[r], lv.H[l], lv.W[l], lv.start[l], MD);
        const int slot = tj * G + (tg ^ (tj & 7));
        s_off[buf][slot] = su.off;
        s_w[buf][slot] = su.w;
      }
    }
  };

  // The first unit's locations and weights are requested before the level
  // metadata is staged, so the two memory round trips overlap.
  if (tile < tiles) prefetch(tile, 0);
  stage_levels(lv, spatial_shapes, level_start_index, L, S);
  if (tile >= tiles) return;
  setup(tile, 0, 0);
  __syncthreads();
  int buf = 0;
  float2 acc[E / 2];
#pragma unroll
  for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
  while (true) {
    // The unit after this one: the next chunk of this tile, or the next tile.
    long long ntile = tile;
    int np0 = p0 + PC;
    if (np0 >= LKv) {
      ntile = tile + gridDim.x;
      np0 = 0;
    }
    const bool more = ntile < tiles;
    if (more) prefetch(ntile, np0);
    const long long v_raw = tile * G + gi;
    const bool active = v_raw < vgroups;
    const long long g_raw = v_raw / SPLIT;
    const Group grp = decompose(active ? g_raw : groups - 1, chunks, M, Lq);
    const int ch = (grp.chunk * LANES + lane) * E;
    const bool lane_on = active && ch < D;
    const T* vbase = value + (grp.b * S * M + grp.m) * static_cast<long long>(D) + ch;
    const int pc = min(PC, LKv - p0);
    if (lane_on) {
      if constexpr (std::is_same<T, float>::value) {
#pragma unroll 8
        for (int j = 0; j < pc; ++j) {
          const int slot = j * G + (gi ^ (j & 7));
          const int4 o = s_off[buf][slot];
          const float4 w = s_w[buf][slot];
          C::accumulate4(vbase, o, w, acc);
        }
      } else {
#pragma unroll 4
        for (int j = 0; j < pc; ++j) {
          const int slot = j * G + (gi ^ (j & 7));
          const int4 o = s_off[buf][slot];
          const float4 w = s_w[buf][slot];
          if (o.x >= 0) C::accumulate(vbase + o.x, w.x, acc);
          if (o.y >= 0) C::accumulate(vbase + o.y, w.y, acc);
          if (o.z >= 0) C::accumulate(vbase + o.z, w.z, acc);
          if (o.w >= 0) C::accumulate(vbase + o.w, w.w, acc);
        }
      }
    }
    if (p0 + PC >= LKv) {
      if constexpr (SPLIT > 1) {
        // The split sub-warps of a group are consecutive in the warp.
#pragma unroll
        for (int o = LANES; o < LANES * SPLIT; o <<= 1) {
#pragma unroll
          for (int e = 0; e < E / 2; ++e) {
            acc[e].x += __shfl_xor_sync(kFullMask, acc[e].x, o);
            acc[e].y += __shfl_xor_sync(kFullMask, acc[e].y, o);
          }
        }
      }
      if (lane_on && v_raw % SPLIT == 0)
        C::store(output + grp.bq * MD + static_cast<long long>(grp.m) * D + ch, acc);
#pragma unroll
      for (int e = 0; e < E / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
    }
    if (more) setup(ntile, np0, buf ^ 1);
    __syncthreads();
    if (!more) break;
    tile = ntile;
    p0 = np0;
    buf ^= 1;
  }
}

#define MSDA_FORWARD_PARAMS(T)                                                           \
  const T *__restrict__ value, const int64_t *__restrict__ spatial_shapes,               \
      const int64_t *__restrict__ level_start_index,                                     \
      const float *__restrict__ sampling_locations,                                      \
      const float *__restrict__ attention_weights, T *__restrict__ output, long long S,   \
      int M, int D, long long Lq, int L, int K, int chunks, long long groups,            \
      const float *__restrict__ reference_points, int R
#define MSDA_FORWARD_ARGS                                                                \
  value, spatial_shapes, level_start_index, sampling_locations, attention_weights, output, \
      S, M, D, Lq, L, K, chunks, groups, reference_points, R

template <int LANES, bool FUSED, int SPLIT>
__global__ void __launch_bounds__(kThreads, 5) forward_kernel_f32(MSDA_FORWARD_PARAMS(float)) {
  forward_body<float, LANES, FUSED, SPLIT>(MSDA_FORWARD_ARGS);
}

template <int LANES, bool FUSED, int SPLIT>
__global__ void __launch_bounds__(kThreads, 4)
    forward_kernel_bf16(MSDA_FORWARD_PARAMS(__nv_bfloat16)) {
  forward_body<__nv_bfloat16, LANES, FUSED, SPLIT>(MSDA_FORWARD_ARGS);
}

#undef MSDA_FORWARD_PARAMS
#undef MSDA_FORWARD_ARGS

// The entry of each value dtype.
template <typename T, int LANES, bool FUSED, int SPLIT = 1>
struct ForwardKernel;
template <int LANES, bool FUSED, int SPLIT>
struct ForwardKernel<float, LANES, FUSED, SPLIT> {
  static constexpr auto fn = forward_kernel_f32<LANES, FUSED, SPLIT>;
};
template <int LANES, bool FUSED, int SPLIT>
struct ForwardKernel<__nv_bfloat16, LANES, FUSED, SPLIT> {
  static constexpr auto fn = forward_kernel_bf16<LANES, FUSED, SPLIT>;
};

// Blocks of this kernel that are resident on the current device at once
// (SM count x blocks per SM), cached per device.
template <typename T, int LANES, bool FUSED>
static long long resident_blocks() {
  static std::atomic<long long> cached[64];  // 0 until known; benign concurrent fills
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev].load() > 0) return cached[dev].load();
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ForwardKernel<T, LANES, FUSED>::fn,
                                                    kThreads, 0) != cudaSuccess ||
      sms <= 0 || per_sm <= 0)
    return 148;
  const long long n = static_cast<long long>(sms) * per_sm;
  if (dev >= 0 && dev < 64) cached[dev].store(n);
  return n;
}

template <typename T, int LANES>
static cudaError_t launch_forward_t(const ForwardArgs& a, cudaStream_t stream) {
  constexpr int G = kThreads / LANES;
  const long long resident = resident_blocks<T, LANES, false>();
  // Too few tiles to fill the GPU (a decoder's few hundred queries): split each
  // group's points over up to 4 sub-warps of one warp.
  int split = 1;
  if (a.chunks == 1)
    while (split < 4 && LANES * split * 2 <= 32 && (a.groups * split + G - 1) / G * 2 <= resident)
      split *= 2;
  const long long tiles = (a.groups * split + G - 1) / G;
  long long blocks = resident;
  if (blocks > tiles) blocks = tiles;
  auto go = [&](auto kernel) {
    kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
        a.sampling_locations, a.attention_weights, static_cast<T*>(a.output), a.S, a.M, a.D,
        a.Lq, a.L, a.K, a.chunks, a.groups, nullptr, 0);
    return cudaGetLastError();
  };
  if constexpr (LANES <= 8) {
    if (split == 4) return go(ForwardKernel<T, LANES, false, 4>::fn);
  }
  if constexpr (LANES <= 16) {
    if (split == 2) return go(ForwardKernel<T, LANES, false, 2>::fn);
  }
  return go(ForwardKernel<T, LANES, false, 1>::fn);
}

template <typename T, int LANES>
static cudaError_t launch_fused_pipelined_t(const FusedArgs& a, cudaStream_t stream) {
  constexpr int G = kThreads / LANES;
  constexpr int PC = kChunkPoints / G;
  if (PC > 32 || a.L * a.K > PC) return cudaErrorNotSupported;
  const long long tiles = (a.groups + G - 1) / G;
  long long blocks = resident_blocks<T, LANES, true>();
  if (blocks > tiles) blocks = tiles;
  ForwardKernel<T, LANES, true>::fn<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const T*>(a.value), a.spatial_shapes, a.level_start_index,
      a.sampling_offsets, a.attention_logits, static_cast<T*>(a.output), a.S, a.M, a.D, a.Lq,
      a.L, a.K, a.chunks, a.groups, a.reference_points, a.R);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t fused_pipelined_lanes(const FusedArgs& a, cudaStream_t stream) {
  switch (a.lanes) {
    case 1: return launch_fused_pipelined_t<T, 1>(a, stream);
    case 2: return launch_fused_pipelined_t<T, 2>(a, stream);
    case 4: return launch_fused_pipelined_t<T, 4>(a, stream);
    case 8: return launch_fused_pipelined_t<T, 8>(a, stream);
    case 16: return launch_fused_pipelined_t<T, 16>(a, stream);
    default: return cudaErrorNotSupported;
  }
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
  if (forward_tiles_apply(a)) {
    // The encoder-form kernels (queries = value pixels): selected by
    // MSDA_FORWARD_KERNEL=staged (shared-memory windows) or =l1 (L1 windows);
    // the per-point gather below otherwise.
    const char* v = std::getenv("MSDA_FORWARD_KERNEL");
    if (v != nullptr && std::strcmp(v, "staged") == 0) return launch_forward_tiled(a, stream);
    if (v != nullptr && std::strcmp(v, "l1") == 0) return launch_forward_l1(a, stream);
  }
  return a.bf16 ? dispatch_lanes<__nv_bfloat16>(a, stream) : dispatch_lanes<float>(a, stream);
}

cudaError_t launch_fused_forward_pipelined(const FusedArgs& a, cudaStream_t stream) {
  return a.bf16 ? fused_pipelined_lanes<__nv_bfloat16>(a, stream)
                : fused_pipelined_lanes<float>(a, stream);
}

}  // namespace msda
