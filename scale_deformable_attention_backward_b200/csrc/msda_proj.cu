// msda_proj.cu -- the output projection after the MSDeformAttn core on the
// 5th-generation tensor cores (sm_100a: tcgen05.mma with the accumulator in
// tensor memory).
//
// "Deformable DETR模型解读（附源码+论文）", MultiScaleDeformableAttention.forward:
// the core's output [N, Lq, M*D] goes through output_proj, a Linear layer:
//     Y[r, n] = sum_k X[r, k] * Wt[n, k] + bias[n]      (Wt: [C_out, C_in])
// This is a dense contraction, so it runs on the tensor cores: kind::tf32
// (float32 operands read as TF32, float32 accumulation).
//
// One CTA of 128 threads owns 128 rows of X at a time (a persistent loop over
// row tiles).  Per K chunk of 32 it stages the X chunk [128 x 32] and the Wt
// chunk [C_out x 32] in shared memory as K-major core matrices without swizzle
// (a core matrix is 8 rows x 16 bytes; K-neighbouring core matrices are LBO
// bytes apart, 8-row groups SBO bytes apart), then thread 0 issues four
// M=128 x N=C_out x K=8 MMAs into a C_out-column float32 accumulator in tensor
// memory and commits them to an mbarrier.  After the last chunk every warp
// reads its 32 rows of the accumulator (tcgen05.ld 32x32b), adds the bias and
// writes them.  Every wait on the mbarrier is bounded: past the limit the CTA
// sets a device flag (read by msda_output_projection_check) and stops,
// releasing its tensor memory.
#include <cstdint>

#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kProjThreads = 128;
constexpr int kProjRows = 128;        // MMA M
constexpr int kProjChunk = 32;        // K per staged chunk (4 MMAs of K = 8)
constexpr int kProjMaxOut = 256;      // MMA N limit (one accumulator)
// Shared memory: X chunk 128 x 32 floats (16 KB) + Wt chunk up to 256 x 32
// floats (32 KB), plus padding that limits residency to 2 CTAs per SM, so two
// 256-column accumulators always fit the SM's 512 tensor-memory columns.
constexpr int kProjXBytes = kProjRows * kProjChunk * 4;
constexpr int kProjWBytes = kProjMaxOut * kProjChunk * 4;
constexpr int kProjSmemBytes = 80 * 1024;
constexpr long long kProjWaitLimit = 1ll << 26;  // polls of the mbarrier before giving up

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Offset in bytes of element (row, k) of a [rows x kProjChunk] K-major chunk of
// 4-byte elements laid out as core matrices: k groups of 4 are LBO = rows * 16
// bytes apart, 8-row groups SBO = 128 bytes apart.
__device__ __forceinline__ uint32_t core_offset(int row, int k, int rows) {
  return static_cast<uint32_t>((k >> 2) * rows * 16 + (row >> 3) * 128 + (row & 7) * 16 +
                               (k & 3) * 4);
}

// Shared-memory matrix descriptor: start, LBO, SBO (all >> 4), version 1,
// no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((start >> 4) & 0x3fff) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3fff) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::tf32: D float32, A and B TF32, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t tf32_idesc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kProjRows >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return done != 0;
}

__global__ void __launch_bounds__(kProjThreads)
proj_kernel(const float* __restrict__ x, const float* __restrict__ wt,
            const float* __restrict__ bias, float* __restrict__ y, long long rows, int c_in,
            int c_out, int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* xs = smem;
  unsigned char* ws = smem + kProjXBytes;
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int failed;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  // Accumulator columns: the next power of two >= max(32, c_out).
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(c_out)) cols <<= 1;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tmem_base)),
                 "r"(cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    mbar_init(&mma_done, 1);
    failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;
  const uint32_t idesc = tf32_idesc(c_out);
  const int n_pad = (c_out + 7) & ~7;  // rows of the Wt chunk (multiple of 8)
  uint32_t phase = 0;

  const long long tiles = (rows + kProjRows - 1) / kProjRows;
  for (long long tile = blockIdx.x; tile < tiles && !failed; tile += gridDim.x) {
    const long long r0 = tile * kProjRows;
    for (int k0 = 0; k0 < c_in; k0 += kProjChunk) {
      const int kc = min(kProjChunk, c_in - k0);  // a multiple of 8
      // Stage the chunks: X rows past the end and K past c_in read as zero.
      for (int i = tid; i < kProjRows * (kProjChunk / 4); i += kProjThreads) {
        const int row = i / (kProjChunk / 4), kq = (i % (kProjChunk / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r0 + row < rows && kq < kc)
          v = __ldg(reinterpret_cast<const float4*>(x + (r0 + row) * c_in + k0 + kq));
        *reinterpret_cast<float4*>(xs + core_offset(row, kq, kProjRows)) = v;
      }
      for (int i = tid; i < n_pad * (kProjChunk / 4); i += kProjThreads) {
        const int n = i / (kProjChunk / 4), kq = (i % (kProjChunk / 4)) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n < c_out && kq < kc)
          v = __ldg(reinterpret_cast<const float4*>(wt + static_cast<long long>(n) * c_in + k0 + kq));
        *reinterpret_cast<float4*>(ws + core_offset(n, kq, n_pad)) = v;
      }
      // The generic-proxy stores must be visible to the tensor core's reads.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (tid == 0) {
        const uint32_t xa = smem_u32(xs), wa = smem_u32(ws);
        for (int s = 0; s < kc / 8; ++s) {
          // K step s covers k groups 2s, 2s + 1.
          const uint64_t da = smem_desc(xa + 2 * s * kProjRows * 16, kProjRows * 16, 128);
          const uint64_t db = smem_desc(wa + 2 * s * n_pad * 16, n_pad * 16, 128);
          const uint32_t accumulate = (k0 > 0 || s > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
              :
              : "r"(tmem), "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u),
                "r"(0u), "r"(0u));
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&mma_done))
            : "memory");
      }
      // Bounded wait for the MMAs (they also release the staged chunks).
      long long polls = 0;
      while (!mbar_try_wait(&mma_done, phase)) {
        if (++polls > kProjWaitLimit) {
          failed = 1;
          break;
        }
      }
      phase ^= 1u;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      __syncthreads();
      if (failed) break;
    }
    if (failed) break;
    // Epilogue: warp w holds accumulator lanes (rows) 32w .. 32w + 31.
    const long long r = r0 + warp * 32 + lane;
    for (int c0 = 0; c0 < c_out; c0 += 16) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
          "%10, %11, %12, %13, %14, %15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0)));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (r < rows) {
        float* dst = y + r * c_out + c0;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          if (c0 + j < c_out) {
            float4 o = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                   __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            if (bias != nullptr) {
              o.x += __ldg(bias + c0 + j);
              o.y += __ldg(bias + c0 + j + 1);
              o.z += __ldg(bias + c0 + j + 2);
              o.w += __ldg(bias + c0 + j + 3);
            }
            *reinterpret_cast<float4*>(dst + j) = o;
          }
        }
      }
    }
    // The next tile's first MMA overwrites the accumulator.
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  if (failed && tid == 0) atomicExch(status, 1);
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(cols));
}

// Set by a CTA whose wait for its MMAs ran past the limit.
__device__ int g_projection_failed;

}  // namespace

cudaError_t projection_failed_flag(int** flag) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(flag), g_projection_failed);
}

cudaError_t launch_projection(const float* x, const float* weight, const float* bias, float* y,
                              long long rows, int c_in, int c_out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  int* status = nullptr;
  cudaError_t err0 = projection_failed_flag(&status);
  if (err0 != cudaSuccess) return err0;
  static_assert(kProjXBytes + kProjWBytes <= kProjSmemBytes, "staging must fit");
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  if ((err = cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kProjSmemBytes)) != cudaSuccess)
    return err;
  const long long tiles = (rows + kProjRows - 1) / kProjRows;
  long long grid = 2ll * sms;
  if (grid > tiles) grid = tiles;
  proj_kernel<<<static_cast<unsigned>(grid), kProjThreads, kProjSmemBytes, stream>>>(
      x, weight, bias, y, rows, c_in, c_out, status);
  return cudaGetLastError();
}

}  // namespace msda
