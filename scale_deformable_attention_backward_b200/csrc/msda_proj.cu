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
// One CTA of 256 threads owns 128 rows of X at a time (a persistent loop over
// row tiles).  Per K chunk of 32 it copies (cp.async, 16 bytes per copy) the X
// chunk [128 x 32] and the Wt chunk [C_out x 32] into shared memory as K-major
// core matrices without swizzle (a core matrix is 8 rows x 16 bytes;
// K-neighbouring core matrices are LBO bytes apart, 8-row groups SBO bytes
// apart); the chunks are double-buffered, so the copies of chunk c + 1 run
// while the tensor core works on chunk c.  Thread 0 issues four
// M=128 x N=C_out x K=8 MMAs per chunk into a C_out-column float32 accumulator
// in tensor memory and commits them to the buffer's mbarrier.  After the last
// chunk the 8 warps read the accumulator (tcgen05.ld 32x32b; warp w takes rows
// 32 (w % 4) .. + 31 and every other 16-column block), add the bias and write.  Every wait on the mbarrier is bounded: past the limit the CTA
// sets a device flag (read by msda_output_projection_check) and stops,
// releasing its tensor memory.
#include <cstdint>

#include "msda_device.cuh"
#include "msda_launch.h"

namespace msda {

namespace {

constexpr int kProjThreads = 256;
constexpr int kProjRows = 128;        // MMA M
constexpr int kProjChunk = 32;        // K per staged chunk (4 MMAs of K = 8)
constexpr int kProjMaxOut = 256;      // MMA N limit (one accumulator)
// Shared memory: two stages of an X chunk 128 x 32 floats (16 KB) and a Wt
// chunk up to 256 x 32 floats (32 KB).  96 KB per CTA keeps residency at 2 CTAs
// per SM, so two 256-column accumulators always fit the SM's 512 tensor-memory
// columns.
constexpr int kProjXBytes = kProjRows * kProjChunk * 4;
constexpr int kProjWBytes = kProjMaxOut * kProjChunk * 4;
constexpr int kProjStageBytes = kProjXBytes + kProjWBytes;
constexpr int kProjSmemBytes = 2 * kProjStageBytes;
constexpr long long kProjWaitLimit = 1ll << 26;  // polls of an mbarrier before giving up

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

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

__global__ void __launch_bounds__(kProjThreads)
proj_kernel(const float* __restrict__ x, const float* __restrict__ wt,
            const float* __restrict__ bias, float* __restrict__ y, long long rows, int c_in,
            int c_out, int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t mma_done[2];  // one per staging buffer
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
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    failed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;
  const uint32_t idesc = tf32_idesc(c_out);
  const int n_pad = (c_out + 7) & ~7;  // rows of the Wt chunk (multiple of 8)
  const int nch = (c_in + kProjChunk - 1) / kProjChunk;
  uint32_t phase0 = 0u, phase1 = 0u;  // parity of each buffer's next completion

  // Waits for the MMAs committed to buffer b's barrier (every thread), bounded.
  auto wait_mma = [&](int b) {
    const uint32_t ph = b ? phase1 : phase0;
    long long polls = 0;
    while (!mbar_try_wait(&mma_done[b], ph)) {
      if (++polls > kProjWaitLimit) {
        failed = 1;
        break;
      }
    }
    if (b)
      phase1 ^= 1u;
    else
      phase0 ^= 1u;
  };
  // Issues the copies of K chunk c of row tile r0 into buffer b.
  auto stage = [&](long long r0, int c, int b) {
    const int k0 = c * kProjChunk;
    const int kc = min(kProjChunk, c_in - k0);
    const uint32_t xs = smem_u32(smem + b * kProjStageBytes);
    const uint32_t ws = xs + kProjXBytes;
    for (int i = tid; i < kProjRows * (kProjChunk / 4); i += kProjThreads) {
      const int row = i / (kProjChunk / 4), kq = (i % (kProjChunk / 4)) * 4;
      const bool in = r0 + row < rows && kq < kc;
      const float* src = in ? x + (r0 + row) * c_in + k0 + kq : x;
      cp_async16(xs + core_offset(row, kq, kProjRows), src, in ? 16 : 0);
    }
    for (int i = tid; i < n_pad * (kProjChunk / 4); i += kProjThreads) {
      const int n = i / (kProjChunk / 4), kq = (i % (kProjChunk / 4)) * 4;
      const bool in = n < c_out && kq < kc;
      const float* src = in ? wt + static_cast<long long>(n) * c_in + k0 + kq : wt;
      cp_async16(ws + core_offset(n, kq, n_pad), src, in ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  const long long tiles = (rows + kProjRows - 1) / kProjRows;
  if (blockIdx.x < tiles) stage(static_cast<long long>(blockIdx.x) * kProjRows, 0, 0);
  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const long long r0 = tile * kProjRows;
    // Chunk 0 of this tile was issued before the previous tile's epilogue.
    for (int c = 0; c < nch; ++c) {
      if (c + 1 < nch) {
        // Buffer (c + 1) & 1 was read by chunk c - 1's MMAs.
        if (c >= 1) wait_mma((c - 1) & 1);
        stage(r0, c + 1, (c + 1) & 1);
        asm volatile("cp.async.wait_group 1;" ::: "memory");  // chunk c has landed
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      // The copies must be visible to the tensor core's (async proxy) reads.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (failed) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (tid == 0) {
        const int b = c & 1;
        const int kc = min(kProjChunk, c_in - c * kProjChunk);
        const uint32_t xa = smem_u32(smem + b * kProjStageBytes), wa = xa + kProjXBytes;
        for (int s = 0; s < kc / 8; ++s) {
          // K step s covers k groups 2s, 2s + 1.
          const uint64_t da = smem_desc(xa + 2 * s * kProjRows * 16, kProjRows * 16, 128);
          const uint64_t db = smem_desc(wa + 2 * s * n_pad * 16, n_pad * 16, 128);
          const uint32_t accumulate = (c > 0 || s > 0) ? 1u : 0u;
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
                smem_u32(&mma_done[b]))
            : "memory");
      }
    }
    // The commits not waited for inside the loop: chunks nch - 2 and nch - 1.
    if (!failed) {
      if (nch >= 2) wait_mma((nch - 2) & 1);
      wait_mma((nch - 1) & 1);
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    __syncthreads();
    if (failed) break;
    // Both buffers are free again: the next tile's first chunk loads during
    // this tile's epilogue.
    if (tile + gridDim.x < tiles) stage((tile + gridDim.x) * kProjRows, 0, 0);
    // Epilogue: warp w reads accumulator lanes (rows) 32 (w % 4) .. + 31 and
    // every other 16-column block, starting at 16 (w / 4).
    const int quarter = warp & 3;
    const long long r = r0 + quarter * 32 + lane;
    for (int c0 = (warp >> 2) * 16; c0 < c_out; c0 += 32) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, "
          "%10, %11, %12, %13, %14, %15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(c0)));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (r < rows) {
        float* dst = y + r * c_out + c0;
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
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
    // The next tile's first MMA overwrites the accumulator.
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
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
  static_assert(kProjSmemBytes <= 113 * 1024, "two CTAs per SM must fit");
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
